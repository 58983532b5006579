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
// any stream capture. The address belongs to the context it was looked up in:
// after a device reset (cudaDeviceReset) the next context may place the array
// elsewhere, so the address is kept with the id of its context and looked up
// again, on the first call after the reset, when the calling thread's current
// context has another id. All calls share the one array and its contents carry
// over from the previous call: every region a call reads is written earlier
// in the same call, so nothing needs clearing, but calls that overlap in time
// on one GPU (other streams, other threads) race on it and must be serialised
// by the caller.
#include <cuda.h>
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
struct ScratchAddr {
    unsigned long long ctx_id;  // id of the context the address belongs to
    void *addr;                 // device address of g_scratch in that context
};
ScratchAddr g_scratch_addr[kMaxDevices];

// Id of the calling thread's current context (unique for the life of the process);
// false when no context is current or the driver lacks the calls. The two driver calls
// are resolved through the runtime, so the library links no driver library.
bool current_context_id(unsigned long long *id)
{
    using GetCurrent = CUresult (*)(CUcontext *);
    using GetId = CUresult (*)(CUcontext, unsigned long long *);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    if (!get_current || !get_id) {
        void *p1 = nullptr, *p2 = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p1, cudaEnableDefault, &q1) != cudaSuccess ||
            q1 != cudaDriverEntryPointSuccess ||
            cudaGetDriverEntryPoint("cuCtxGetId", &p2, cudaEnableDefault, &q2) != cudaSuccess ||
            q2 != cudaDriverEntryPointSuccess)
            return false;
        get_current = reinterpret_cast<GetCurrent>(p1);
        get_id = reinterpret_cast<GetId>(p2);
    }
    CUcontext ctx = nullptr;
    return get_current(&ctx) == CUDA_SUCCESS && ctx && get_id(ctx, id) == CUDA_SUCCESS;
}

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
        ScratchAddr &sa = g_scratch_addr[dev];
        unsigned long long id = 0;
        if (!sa.addr || !current_context_id(&id) || id != sa.ctx_id) {
            // First call on this device, or on a context other than the one the cached
            // address was looked up in. The lookup makes the device's primary context
            // current if none is.
            void *p = nullptr;
            e = cudaGetSymbolAddress(&p, g_scratch);
            if (e != cudaSuccess) return gdr::set_failure(GDR_ERR_CUDA, cudaGetErrorString(e));
            if (!current_context_id(&id))
                return gdr::set_failure(GDR_ERR_CUDA, "no current CUDA context after the scratch lookup");
            sa.ctx_id = id;
            sa.addr = p;
        }
        scratch = sa.addr;
    }
    return gdr_fwd_chunked(q, k, v, g, beta, h0, o, hT, B, T, Hk, Hv, Dk, Dv, gate_mode, dtype, scratch,
                           scratch ? (size_t)GDR_NOALLOC_SCRATCH_BYTES : 0, stream);
}
