// Internal launch interface between the C ABI (gdr_api.cu) and the kernels.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>

namespace gdr {

// dtype codes (include/gdr.h): 0 bf16 in/out, 1 fp32 in/out, 2 bf16 in / fp32 out.
inline bool in_bf16(int dtype) { return dtype != 1; }
inline bool out_f32(int dtype) { return dtype != 0; }

struct DecodeArgs {
    const void *q, *k, *v;
    const float *g, *beta;
    float *state;
    void *o;
    int B, Hk, Hv, Dk, Dv, gate_mode, dtype;
};

struct FwdArgs {
    const void *q, *k, *v;
    const float *g, *beta, *h0;
    void *o;
    float *hT;
    int B, T, Hk, Hv, Dk, Dv, gate_mode, dtype;
    // Packed variable-length input (fused kernel only): B sequences packed along one
    // token axis of length T; sequence n is tokens [cu_seqlens[n], cu_seqlens[n + 1]).
    const int *cu_seqlens = nullptr;
    // Fused kernel only. qk_l2norm: q and k rows are divided by sqrt(sum of squares + 1e-6)
    // as they are loaded. z: when set ([B, T, Hv, Dv] bf16, like o), o receives
    // o / sqrt(mean(o^2) + norm_eps) * norm_w * SiLU(z) per row of Dv (norm_w [Dv] fp32).
    int qk_l2norm = 0;
    const void *z = nullptr;
    const float *norm_w = nullptr;
    float norm_eps = 0.f;
    // tcgen05 kernel, fixed-length sequences with more (batch row, value head) units than
    // SMs: sched_len chunk-steps per CTA (0: one CTA per unit); the per-launch tag, flags and
    // states of the units cut between two CTAs live in the caller's workspace.
    int sched_len = 0;
    unsigned long long sched_tag = 0;
    unsigned long long *sched_flags = nullptr;
    float *sched_states = nullptr;
    // tcgen05 kernel, scalar gate: the chunked backward's forward pass. Per (unit, chunk), the
    // fp16 images of 128-byte swizzled tiles (64-column atoms): the entering state S^T
    // [Dv][Dk] and P [Dk][Dk] (32 KB), Qh^T [Dk][64] (16 KB), T [64][64] (8 KB; the lower
    // triangle, entries above the diagonal blocks are not written). No o is stored.
    void *save_s = nullptr, *save_p = nullptr, *save_qh = nullptr, *save_t = nullptr;
};

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t st);

// Fused chunked forward on the warp-level tensor cores (bf16 inputs, Dk = Dv = 128,
// either gate): one kernel, no workspace.
bool fused_supported(const FwdArgs &a);
cudaError_t launch_fwd_fused(const FwdArgs &a, cudaStream_t st);
// Device-side failure counts of the fused kernel since the library was loaded on this
// device: chunk loads that timed out, and per-channel gate factors outside the fp16 range.
unsigned int fused_error_counts(unsigned int *load_timeouts, unsigned int *range_errors);

// Chunked forward on the tcgen05 tensor cores (scalar gate, bf16 inputs, Dk = Dv = 128,
// fixed-length sequences, no layer options): one kernel, no workspace.
bool tc_supported(const FwdArgs &a);
cudaError_t launch_fwd_tc(const FwdArgs &a, cudaStream_t st);
// Workspace bytes that let the tcgen05 kernel balance units over the SMs (0 when it runs one
// CTA per unit anyway), and the schedule it then takes: fills a.sched_len, a.sched_tag and
// the workspace pointers.
size_t tc_sched_bytes(const FwdArgs &a);
void tc_set_sched(FwdArgs &a, void *workspace);
// Waits of the tcgen05 kernel that timed out since the library was loaded on this device,
// and its units in which a value rounded to an fp16 operand was inf or NaN.
unsigned int tc_error_count();
unsigned int tc_range_error_count();

// Backward of the recurrence (bwd.cu): gradients of L = sum(dout * o) + sum(dhT * hT), all
// fp32 [q, k: B,T,Hk,Dk; v: B,T,Hv,Dv; g: g's layout; beta: B,T,Hv; h0: B,Hv,Dk,Dv].
// dq, dk, dg and dbeta are accumulated with atomics and must be zero on entry.
struct BwdArgs {
    const void *q, *k, *v;
    const float *g, *beta, *h0;
    const void *dout;
    const float *dhT;
    float *dq, *dk, *dv, *dg, *dbeta, *dh0;
    int B, T, Hk, Hv, Dk, Dv, gate_mode, dtype;
};
bool bwd_supported(const BwdArgs &a);
size_t bwd_workspace_size(const BwdArgs &a);
cudaError_t launch_bwd(const BwdArgs &a, void *ws, cudaStream_t st);
// Chunked backward on tensor cores (bwd_chunk.cu): scalar gate, bf16 inputs, Dk = Dv = 128.
// With more value heads than key heads dq and dk are accumulated with atomics and must be
// zero on entry; otherwise they are written once, as are dv, dg, dbeta and dh0.
bool bwdc_supported(const BwdArgs &a);
size_t bwdc_workspace_size(const BwdArgs &a);
cudaError_t launch_bwdc(const BwdArgs &a, void *ws, cudaStream_t st);

// fp32 CUDA-core chunked forward (three kernels). Needs simt_workspace_size() bytes.
size_t simt_workspace_size(const FwdArgs &a);
cudaError_t launch_fwd_simt(const FwdArgs &a, void *ws, cudaStream_t st);

// Short causal convolution (4 taps) + SiLU over [rows, Ch] (prologue.cu). Sequence n
// is tokens [cu_seqlens[n], cu_seqlens[n + 1]) when cu_seqlens is given, else
// [n T, n T + T); states are [nseq, Ch, 3] in the dtype of x (oldest input first).
struct ConvArgs {
    const void *x;
    const float *w, *bias;
    const void *state_in;
    void *state_out, *y;
    const int *cu_seqlens;
    int nseq, T;
    long rows;
    int Ch;
    bool fp32;
};
int conv_launches(const ConvArgs &a);
cudaError_t launch_conv_silu(const ConvArgs &a, cudaStream_t st);

// y = o / sqrt(mean(o^2) + eps) * w * SiLU(z) per row of D (64 or 128) elements.
struct NormArgs {
    const void *o, *z;
    const float *w;
    void *y;
    long rows;
    int D;
    float eps;
    bool fp32;
};
cudaError_t launch_rmsnorm_gated(const NormArgs &a, cudaStream_t st);

}  // namespace gdr
