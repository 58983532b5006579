// Chunked forward that allocates nothing: its scratch lives in a fixed-size
// array of device memory that belongs to this file.
//
// Some callers cannot call cudaMalloc: an engine that owns every byte of
// device memory through its own pool and forbids side allocations, or a
// latency-bound serving loop where an allocation (and the synchronisation
// cudaMalloc/cudaFree can cause) is not allowed after start-up. For them this
// entry point runs the chunked forward with its workspace placed in
// GDR_NOALLOC_SCRATCH_BYTES of scratch reserved in a file-scope __device__
// array; sizes served by the fused single-kernel path need no workspace and
// leave the array untouched. The caller still passes every input and output.
//
// The array is allocated by the CUDA runtime when this file's device code is
// loaded on a GPU and stays reserved on every GPU that loaded it until the
// process exits. Its address is looked up once per device, with that device
// current, on the first call made on that device; make that first call before
// any stream capture. All calls share the one array and its contents carry
// over from the previous call: every region a call reads is written earlier
// in the same call, so nothing needs clearing, but calls that overlap in time
// on one GPU (other streams, other threads) race on it and must be serialised
// by the caller.
#include <stdio.h>

#include <mutex>

#include "../../include/gdr.h"
#include "kernels.h"

namespace gdr {
int set_failure(int status, const char *msg);
}

namespace {

static __device__ __align__(256) unsigned char g_scratch[GDR_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices];  // device address of g_scratch, per device

}  // namespace

extern "C" int gdr_fwd_chunked_noalloc(const void *q, const void *k, const void *v, const float *g,
                                       const float *beta, const float *h0, void *o, float *hT,
                                       int B, int T, int Hk, int Hv, int Dk, int Dv, int gate_mode,
                                       int dtype, void *stream)
{
    const size_t need = gdr_fwd_workspace_size(B, T, Hk, Hv, Dk, Dv, gate_mode, dtype);
    if (need > (size_t)GDR_NOALLOC_SCRATCH_BYTES) {
        char msg[256];
        snprintf(msg, sizeof(msg),
                 "these sizes need %zu bytes of scratch; gdr_fwd_chunked_noalloc holds %zu "
                 "(use gdr_fwd_chunked with a caller-allocated workspace)",
                 need, (size_t)GDR_NOALLOC_SCRATCH_BYTES);
        return gdr::set_failure(GDR_ERR_WORKSPACE, msg);
    }
    void *scratch = nullptr;
    if (need > 0) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return gdr::set_failure(GDR_ERR_CUDA, cudaGetErrorString(e));
        if (dev < 0 || dev >= kMaxDevices)
            return gdr::set_failure(GDR_ERR_UNSUPPORTED, "device ordinal beyond 63");
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_scratch_addr[dev]) {
            void *p = nullptr;
            e = cudaGetSymbolAddress(&p, g_scratch);
            if (e != cudaSuccess) return gdr::set_failure(GDR_ERR_CUDA, cudaGetErrorString(e));
            g_scratch_addr[dev] = p;
        }
        scratch = g_scratch_addr[dev];
    }
    return gdr_fwd_chunked(q, k, v, g, beta, h0, o, hT, B, T, Hk, Hv, Dk, Dv, gate_mode, dtype, scratch,
                           scratch ? (size_t)GDR_NOALLOC_SCRATCH_BYTES : 0, stream);
}
