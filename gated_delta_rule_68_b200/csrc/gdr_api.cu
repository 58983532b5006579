// C ABI of libgdr: argument checks, workspace sizing and kernel dispatch.
// The contract of every entry point is documented in include/gdr.h.
#include <stdarg.h>
#include <atomic>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "../../include/gdr.h"
#include "kernels.h"

namespace {

thread_local char g_err[512] = "no error";
std::atomic<unsigned long long> g_launches{0};

int fail(int status, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return status;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

bool supported_dim(int d) { return d == 64 || d == 128; }

int check_common(int B, int T, int Hk, int Hv, int Dk, int Dv, int gate_mode, int dtype)
{
    if (B < 0 || T < 0 || Hk <= 0 || Hv <= 0 || Dk <= 0 || Dv <= 0)
        return fail(GDR_ERR_INVALID_ARG, "sizes must be positive (B=%d T=%d Hk=%d Hv=%d Dk=%d Dv=%d)",
                    B, T, Hk, Hv, Dk, Dv);
    if (Hv % Hk != 0)
        return fail(GDR_ERR_INVALID_ARG, "Hv (%d) must be a multiple of Hk (%d)", Hv, Hk);
    if (gate_mode != GDR_GATE_SCALAR && gate_mode != GDR_GATE_CHANNEL)
        return fail(GDR_ERR_INVALID_ARG, "gate_mode must be GDR_GATE_SCALAR or GDR_GATE_CHANNEL (got %d)", gate_mode);
    if (dtype != GDR_BF16 && dtype != GDR_FP32 && dtype != GDR_BF16_OUT_F32)
        return fail(GDR_ERR_INVALID_ARG, "dtype must be GDR_BF16, GDR_FP32 or GDR_BF16_OUT_F32 (got %d)",
                    dtype);
    if (!supported_dim(Dk) || !supported_dim(Dv))
        return fail(GDR_ERR_UNSUPPORTED, "Dk and Dv must each be 64 or 128 (got Dk=%d Dv=%d)", Dk, Dv);
    if ((long long)B * Hv > (1LL << 31) - 1)
        return fail(GDR_ERR_INVALID_ARG, "B*Hv too large");
    return GDR_OK;
}

gdr::FwdArgs make_fwd(const void *q, const void *k, const void *v, const float *g, const float *beta,
                      const float *h0, void *o, float *hT, int B, int T, int Hk, int Hv, int Dk, int Dv,
                      int gate_mode, int dtype)
{
    gdr::FwdArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.h0 = h0; a.o = o; a.hT = hT;
    a.B = B; a.T = T; a.Hk = Hk; a.Hv = Hv; a.Dk = Dk; a.Dv = Dv;
    a.gate_mode = gate_mode; a.dtype = dtype;
    return a;
}

}  // namespace

namespace gdr {
// Records a failure message for gdr_last_error() from another translation unit.
int set_failure(int status, const char *msg) { return fail(status, "%s", msg); }
}  // namespace gdr

namespace gdr {
// Device-side failure counts of the chunked backward (bwd_chunk.cu).
unsigned int bwdc_error_counts(unsigned int *timeouts, unsigned int *range_errors);
}  // namespace gdr

extern "C" {

int gdr_version(void) { return 300; }

const char *gdr_last_error(void) { return g_err; }

unsigned long long gdr_kernel_launches(void) { return g_launches.load(); }

unsigned int gdr_fused_error_counts(unsigned int *load_timeouts, unsigned int *range_errors)
{
    unsigned int t = 0, r = 0;
    gdr::fused_error_counts(&t, &r);
    t += gdr::tc_error_count();
    r += gdr::tc_range_error_count();
    unsigned int bt = 0, br = 0;
    gdr::bwdc_error_counts(&bt, &br);
    t += bt;
    r += br;
    if (load_timeouts) *load_timeouts = t;
    if (range_errors) *range_errors = r;
    return t + r;
}

size_t gdr_fwd_workspace_size(int B, int T, int Hk, int Hv, int Dk, int Dv, int gate_mode, int dtype)
{
    if (check_common(B, T, Hk, Hv, Dk, Dv, gate_mode, dtype) != GDR_OK) return 0;
    if (B == 0 || T == 0) return 0;
    const gdr::FwdArgs a = make_fwd(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                                    nullptr, B, T, Hk, Hv, Dk, Dv, gate_mode, dtype);
    if (gdr::tc_supported(a)) return gdr::tc_sched_bytes(a);
    return gdr::fused_supported(a) ? 0 : gdr::simt_workspace_size(a);
}

int gdr_fwd_chunked(const void *q, const void *k, const void *v, const float *g, const float *beta,
                    const float *h0, void *o, float *hT, int B, int T, int Hk, int Hv, int Dk, int Dv,
                    int gate_mode, int dtype, void *workspace, size_t workspace_bytes, void *stream)
{
    int st = check_common(B, T, Hk, Hv, Dk, Dv, gate_mode, dtype);
    if (st != GDR_OK) return st;
    const bool work = B > 0 && T > 0;
    if (work && (!q || !k || !v || !g || !beta || !o))
        return fail(GDR_ERR_INVALID_ARG, "q, k, v, g, beta and o must be non-NULL");
    const void *ptrs[] = {q, k, v, g, beta, h0, o, hT};
    const char *names[] = {"q", "k", "v", "g", "beta", "h0", "o", "hT"};
    for (int i = 0; i < 8; ++i)
        if (ptrs[i] && !aligned16(ptrs[i]))
            return fail(GDR_ERR_MISALIGNED, "%s is not 16-byte aligned", names[i]);
    if (workspace && ((uintptr_t)workspace & 255u))
        return fail(GDR_ERR_MISALIGNED, "workspace is not 256-byte aligned");
    if (o && (o == q || o == k || o == v))
        return fail(GDR_ERR_INVALID_ARG, "o must not alias q, k or v");
    cudaStream_t s = (cudaStream_t)stream;

    if (!work) {  // empty input: hT = h0 (or zeros)
        if (hT) {
            const size_t bytes = (size_t)B * Hv * Dk * Dv * sizeof(float);
            cudaError_t e = h0 ? (h0 == hT ? cudaSuccess
                                           : cudaMemcpyAsync(hT, h0, bytes, cudaMemcpyDeviceToDevice, s))
                               : cudaMemsetAsync(hT, 0, bytes, s);
            if (e != cudaSuccess) return fail(GDR_ERR_CUDA, "CUDA: %s", cudaGetErrorString(e));
        }
        return GDR_OK;
    }

    gdr::FwdArgs a = make_fwd(q, k, v, g, beta, h0, o, hT, B, T, Hk, Hv, Dk, Dv, gate_mode, dtype);
    if (gdr::tc_supported(a)) {
        // More units than SMs: a workspace of gdr_fwd_workspace_size() bytes lets the kernel
        // spread the units' chunks evenly over the SMs; without it, one CTA per unit.
        const size_t need = gdr::tc_sched_bytes(a);
        if (need > 0 && workspace && workspace_bytes >= need) gdr::tc_set_sched(a, workspace);
        cudaError_t e = gdr::launch_fwd_tc(a, s);
        if (e != cudaSuccess) return fail(GDR_ERR_CUDA, "CUDA launch failed: %s", cudaGetErrorString(e));
        g_launches += 1;
        return GDR_OK;
    }
    if (gdr::fused_supported(a)) {
        cudaError_t e = gdr::launch_fwd_fused(a, s);
        if (e != cudaSuccess) return fail(GDR_ERR_CUDA, "CUDA launch failed: %s", cudaGetErrorString(e));
        g_launches += 1;
        return GDR_OK;
    }
    if (B > 65535)   // its kernels put the batch row on the grid's z axis
        return fail(GDR_ERR_UNSUPPORTED, "the CUDA-core path (fp32 inputs, d = 64, rectangular states) takes at "
                                         "most 65535 batch rows; got %d", B);
    const size_t need = gdr::simt_workspace_size(a);
    if (need > 0 && (!workspace || workspace_bytes < need))
        return fail(GDR_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given%s", need, workspace_bytes,
                    workspace ? "" : " (NULL)");
    cudaError_t e = gdr::launch_fwd_simt(a, workspace, s);
    if (e != cudaSuccess) return fail(GDR_ERR_CUDA, "CUDA launch failed: %s", cudaGetErrorString(e));
    g_launches += 3;
    return GDR_OK;
}

int gdr_fwd_chunked_varlen(const void *q, const void *k, const void *v, const float *g, const float *beta,
                           const float *h0, void *o, float *hT, const int *cu_seqlens, int N, int T_total, int Hk,
                           int Hv, int Dk, int Dv, int gate_mode, int dtype, void *stream)
{
    int st = check_common(N, T_total, Hk, Hv, Dk, Dv, gate_mode, dtype);
    if (st != GDR_OK) return st;
    if (N > 0 && !cu_seqlens) return fail(GDR_ERR_INVALID_ARG, "cu_seqlens must be non-NULL");
    if (cu_seqlens && ((uintptr_t)cu_seqlens & 3u)) return fail(GDR_ERR_MISALIGNED, "cu_seqlens is not 4-byte aligned");
    const bool work = N > 0 && T_total > 0;
    if (work && (!q || !k || !v || !g || !beta || !o))
        return fail(GDR_ERR_INVALID_ARG, "q, k, v, g, beta and o must be non-NULL");
    const void *ptrs[] = {q, k, v, g, beta, h0, o, hT};
    const char *names[] = {"q", "k", "v", "g", "beta", "h0", "o", "hT"};
    for (int i = 0; i < 8; ++i)
        if (ptrs[i] && !aligned16(ptrs[i]))
            return fail(GDR_ERR_MISALIGNED, "%s is not 16-byte aligned", names[i]);
    if (o && (o == q || o == k || o == v))
        return fail(GDR_ERR_INVALID_ARG, "o must not alias q, k or v");
    gdr::FwdArgs a = make_fwd(q, k, v, g, beta, h0, o, hT, N, T_total, Hk, Hv, Dk, Dv, gate_mode, dtype);
    a.cu_seqlens = cu_seqlens;
    if (!gdr::fused_supported(a))
        return fail(GDR_ERR_UNSUPPORTED, "packed sequences need bf16 inputs and Dk = Dv = 128");
    cudaStream_t s = (cudaStream_t)stream;
    if (!work) {
        if (hT && N > 0) {
            const size_t bytes = (size_t)N * Hv * Dk * Dv * sizeof(float);
            cudaError_t e = h0 ? (h0 == hT ? cudaSuccess
                                           : cudaMemcpyAsync(hT, h0, bytes, cudaMemcpyDeviceToDevice, s))
                               : cudaMemsetAsync(hT, 0, bytes, s);
            if (e != cudaSuccess) return fail(GDR_ERR_CUDA, "CUDA: %s", cudaGetErrorString(e));
        }
        return GDR_OK;
    }
    cudaError_t e = gdr::tc_supported(a) ? gdr::launch_fwd_tc(a, s) : gdr::launch_fwd_fused(a, s);
    if (e != cudaSuccess) return fail(GDR_ERR_CUDA, "CUDA launch failed: %s", cudaGetErrorString(e));
    g_launches += 1;
    return GDR_OK;
}

int gdr_fwd_chunked_norm(const void *q, const void *k, const void *v, const float *g, const float *beta,
                         const float *h0, void *o, float *hT, const int *cu_seqlens, int B, int T, int Hk, int Hv,
                         int Dk, int Dv, int gate_mode, int dtype, int qk_l2norm, const void *z,
                         const float *norm_weight, float norm_eps, void *stream)
{
    int st = check_common(B, T, Hk, Hv, Dk, Dv, gate_mode, dtype);
    if (st != GDR_OK) return st;
    if (cu_seqlens && ((uintptr_t)cu_seqlens & 3u)) return fail(GDR_ERR_MISALIGNED, "cu_seqlens is not 4-byte aligned");
    const bool work = B > 0 && T > 0;
    if (work && (!q || !k || !v || !g || !beta || !o))
        return fail(GDR_ERR_INVALID_ARG, "q, k, v, g, beta and o must be non-NULL");
    if (z && !norm_weight) return fail(GDR_ERR_INVALID_ARG, "norm_weight must be non-NULL when z is given");
    if (!(norm_eps >= 0.f)) return fail(GDR_ERR_INVALID_ARG, "norm_eps must be non-negative");
    const void *ptrs[] = {q, k, v, g, beta, h0, o, hT, z};
    const char *names[] = {"q", "k", "v", "g", "beta", "h0", "o", "hT", "z"};
    for (int i = 0; i < 9; ++i)
        if (ptrs[i] && !aligned16(ptrs[i])) return fail(GDR_ERR_MISALIGNED, "%s is not 16-byte aligned", names[i]);
    if ((uintptr_t)norm_weight & 3u) return fail(GDR_ERR_MISALIGNED, "norm_weight is not 4-byte aligned");
    if (o && (o == q || o == k || o == v || o == z)) return fail(GDR_ERR_INVALID_ARG, "o must not alias q, k, v or z");
    gdr::FwdArgs a = make_fwd(q, k, v, g, beta, h0, o, hT, B, T, Hk, Hv, Dk, Dv, gate_mode, dtype);
    a.cu_seqlens = cu_seqlens;
    a.qk_l2norm = qk_l2norm != 0;
    a.z = z;
    a.norm_w = norm_weight;
    a.norm_eps = norm_eps;
    if (!gdr::fused_supported(a))
        return fail(GDR_ERR_UNSUPPORTED, "the fused options need bf16 inputs and Dk = Dv = 128");
    cudaStream_t s = (cudaStream_t)stream;
    if (!work) {
        if (hT && B > 0) {
            const size_t bytes = (size_t)B * Hv * Dk * Dv * sizeof(float);
            cudaError_t e = h0 ? (h0 == hT ? cudaSuccess
                                           : cudaMemcpyAsync(hT, h0, bytes, cudaMemcpyDeviceToDevice, s))
                               : cudaMemsetAsync(hT, 0, bytes, s);
            if (e != cudaSuccess) return fail(GDR_ERR_CUDA, "CUDA: %s", cudaGetErrorString(e));
        }
        return GDR_OK;
    }
    cudaError_t e = gdr::tc_supported(a) ? gdr::launch_fwd_tc(a, s) : gdr::launch_fwd_fused(a, s);
    if (e != cudaSuccess) return fail(GDR_ERR_CUDA, "CUDA launch failed: %s", cudaGetErrorString(e));
    g_launches += 1;
    return GDR_OK;
}

size_t gdr_bwd_workspace_size(int B, int T, int Hk, int Hv, int Dk, int Dv, int gate_mode, int dtype)
{
    if (check_common(B, T, Hk, Hv, Dk, Dv, gate_mode, dtype) != GDR_OK) return 0;
    gdr::BwdArgs a{};
    a.B = B; a.T = T; a.Hk = Hk; a.Hv = Hv; a.Dk = Dk; a.Dv = Dv; a.gate_mode = gate_mode; a.dtype = dtype;
    return (B == 0 || T == 0) ? 0 : gdr::bwd_workspace_size(a);
}

int gdr_bwd(const void *q, const void *k, const void *v, const float *g, const float *beta, const float *h0,
            const void *dout, const float *dhT, float *dq, float *dk, float *dv, float *dg, float *dbeta,
            float *dh0, int B, int T, int Hk, int Hv, int Dk, int Dv, int gate_mode, int dtype, void *workspace,
            size_t workspace_bytes, void *stream)
{
    int st = check_common(B, T, Hk, Hv, Dk, Dv, gate_mode, dtype);
    if (st != GDR_OK) return st;
    const bool work = B > 0 && T > 0;
    if (B > 0 && !dh0) return fail(GDR_ERR_INVALID_ARG, "dh0 must be non-NULL");
    if (work && (!q || !k || !v || !g || !beta || !dout || !dq || !dk || !dv || !dg || !dbeta))
        return fail(GDR_ERR_INVALID_ARG, "q, k, v, g, beta, dout and the gradient outputs must be non-NULL");
    const void *ptrs[] = {q, k, v, g, beta, h0, dout, dhT, dq, dk, dv, dg, dbeta, dh0, workspace};
    const char *names[] = {"q", "k", "v", "g", "beta", "h0", "dout", "dhT", "dq", "dk", "dv", "dg", "dbeta", "dh0",
                           "workspace"};
    for (int i = 0; i < 15; ++i)
        if (ptrs[i] && !aligned16(ptrs[i])) return fail(GDR_ERR_MISALIGNED, "%s is not 16-byte aligned", names[i]);
    cudaStream_t s = (cudaStream_t)stream;
    if (!work) {   // dh0 = dhT (or zeros); no token, no other gradient
        if (B > 0) {
            const size_t bytes = (size_t)B * Hv * Dk * Dv * sizeof(float);
            cudaError_t e = dhT ? cudaMemcpyAsync(dh0, dhT, bytes, cudaMemcpyDeviceToDevice, s)
                                : cudaMemsetAsync(dh0, 0, bytes, s);
            if (e != cudaSuccess) return fail(GDR_ERR_CUDA, "CUDA: %s", cudaGetErrorString(e));
        }
        return GDR_OK;
    }
    gdr::BwdArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.h0 = h0; a.dout = dout; a.dhT = dhT;
    a.dq = dq; a.dk = dk; a.dv = dv; a.dg = dg; a.dbeta = dbeta; a.dh0 = dh0;
    a.B = B; a.T = T; a.Hk = Hk; a.Hv = Hv; a.Dk = Dk; a.Dv = Dv; a.gate_mode = gate_mode; a.dtype = dtype;
    if (!gdr::bwd_supported(a)) return fail(GDR_ERR_UNSUPPORTED, "the backward needs Dk of 64 or 128");
    if ((long)B * Hv > 65535)   // (batch row, value head) is the grid's y axis
        return fail(GDR_ERR_UNSUPPORTED, "the backward takes at most 65535 (batch row, value head) pairs; got %ld",
                    (long)B * Hv);
    const size_t need = gdr::bwd_workspace_size(a);
    if (!workspace || workspace_bytes < need)
        return fail(GDR_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given%s", need, workspace_bytes,
                    workspace ? "" : " (NULL)");
    // dq, dk, dg and dbeta are sums over CTAs
    const size_t nqk = (size_t)B * T * Hk * Dk * sizeof(float), nb = (size_t)B * T * Hv * sizeof(float);
    const size_t ng = gate_mode == GDR_GATE_CHANNEL ? nb * Dk : nb;
    cudaError_t e = cudaMemsetAsync(dq, 0, nqk, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dk, 0, nqk, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dg, 0, ng, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dbeta, 0, nb, s);
    if (e == cudaSuccess) e = gdr::launch_bwd(a, workspace, s);
    if (e != cudaSuccess) return fail(GDR_ERR_CUDA, "CUDA launch failed: %s", cudaGetErrorString(e));
    g_launches += 2;
    return GDR_OK;
}

size_t gdr_bwd_chunked_workspace_size(int B, int T, int Hk, int Hv, int Dk, int Dv, int gate_mode, int dtype)
{
    if (check_common(B, T, Hk, Hv, Dk, Dv, gate_mode, dtype) != GDR_OK) return 0;
    gdr::BwdArgs a{};
    a.B = B; a.T = T; a.Hk = Hk; a.Hv = Hv; a.Dk = Dk; a.Dv = Dv; a.gate_mode = gate_mode; a.dtype = dtype;
    return (B == 0 || T == 0 || !gdr::bwdc_supported(a)) ? 0 : gdr::bwdc_workspace_size(a);
}

int gdr_bwd_chunked(const void *q, const void *k, const void *v, const float *g, const float *beta,
                    const float *h0, const void *dout, const float *dhT, float *dq, float *dk, float *dv, float *dg,
                    float *dbeta, float *dh0, int B, int T, int Hk, int Hv, int Dk, int Dv, int gate_mode, int dtype,
                    void *workspace, size_t workspace_bytes, void *stream)
{
    int st = check_common(B, T, Hk, Hv, Dk, Dv, gate_mode, dtype);
    if (st != GDR_OK) return st;
    gdr::BwdArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.h0 = h0; a.dout = dout; a.dhT = dhT;
    a.dq = dq; a.dk = dk; a.dv = dv; a.dg = dg; a.dbeta = dbeta; a.dh0 = dh0;
    a.B = B; a.T = T; a.Hk = Hk; a.Hv = Hv; a.Dk = Dk; a.Dv = Dv; a.gate_mode = gate_mode; a.dtype = dtype;
    if (!gdr::bwdc_supported(a))
        return fail(GDR_ERR_UNSUPPORTED, "the chunked backward needs the scalar gate, bf16 inputs and Dk = Dv = 128");
    const bool work = B > 0 && T > 0;
    if (B > 0 && !dh0) return fail(GDR_ERR_INVALID_ARG, "dh0 must be non-NULL");
    if (work && (!q || !k || !v || !g || !beta || !dout || !dq || !dk || !dv || !dg || !dbeta))
        return fail(GDR_ERR_INVALID_ARG, "q, k, v, g, beta, dout and the gradient outputs must be non-NULL");
    const void *ptrs[] = {q, k, v, g, beta, h0, dout, dhT, dq, dk, dv, dg, dbeta, dh0, workspace};
    const char *names[] = {"q", "k", "v", "g", "beta", "h0", "dout", "dhT", "dq", "dk", "dv", "dg", "dbeta", "dh0",
                           "workspace"};
    for (int i = 0; i < 15; ++i)
        if (ptrs[i] && !aligned16(ptrs[i])) return fail(GDR_ERR_MISALIGNED, "%s is not 16-byte aligned", names[i]);
    cudaStream_t s = (cudaStream_t)stream;
    if (!work) {   // dh0 = dhT (or zeros); no token, no other gradient
        if (B > 0) {
            const size_t bytes = (size_t)B * Hv * Dk * Dv * sizeof(float);
            cudaError_t e = dhT ? cudaMemcpyAsync(dh0, dhT, bytes, cudaMemcpyDeviceToDevice, s)
                                : cudaMemsetAsync(dh0, 0, bytes, s);
            if (e != cudaSuccess) return fail(GDR_ERR_CUDA, "CUDA: %s", cudaGetErrorString(e));
        }
        return GDR_OK;
    }
    const long cus = (long)B * Hv * ((T + 63) / 64);
    if (cus > 2147483647L)
        return fail(GDR_ERR_UNSUPPORTED, "the chunked backward takes at most 2^31 - 1 (unit, chunk) pairs");
    const size_t need = gdr::bwdc_workspace_size(a);
    if (!workspace || workspace_bytes < need)
        return fail(GDR_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given%s", need, workspace_bytes,
                    workspace ? "" : " (NULL)");
    // dq and dk are sums over the value heads of a key head; with one value head per key head
    // each element has one writer and no zeroing is needed
    const size_t nqk = (size_t)B * T * Hk * Dk * sizeof(float);
    cudaError_t e = cudaSuccess;
    if (Hv != Hk) {
        e = cudaMemsetAsync(dq, 0, nqk, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(dk, 0, nqk, s);
    }
    if (e == cudaSuccess) e = gdr::launch_bwdc(a, workspace, s);
    if (e != cudaSuccess) return fail(GDR_ERR_CUDA, "CUDA launch failed: %s", cudaGetErrorString(e));
    g_launches += 3;
    return GDR_OK;
}

int gdr_decode_step(const void *q, const void *k, const void *v, const float *g, const float *beta,
                    float *state, void *o, int B, int Hk, int Hv, int Dk, int Dv, int gate_mode, int dtype,
                    void *stream)
{
    int st = check_common(B, 1, Hk, Hv, Dk, Dv, gate_mode, dtype);
    if (st != GDR_OK) return st;
    if (B == 0) return GDR_OK;
    if (!q || !k || !v || !g || !beta || !state || !o)
        return fail(GDR_ERR_INVALID_ARG, "q, k, v, g, beta, state and o must be non-NULL");
    // The state is streamed with 128-bit accesses; every other operand is read or
    // written one element at a time and needs only its element's alignment.
    if (!aligned16(state)) return fail(GDR_ERR_MISALIGNED, "state is not 16-byte aligned");
    const uintptr_t in_es = dtype == GDR_FP32 ? 4 : 2, out_es = dtype == GDR_BF16 ? 2 : 4;
    const void *ptrs[] = {q, k, v, g, beta, o};
    const uintptr_t need[] = {in_es, in_es, in_es, 4, 4, out_es};
    const char *names[] = {"q", "k", "v", "g", "beta", "o"};
    for (int i = 0; i < 6; ++i)
        if ((uintptr_t)ptrs[i] % need[i])
            return fail(GDR_ERR_MISALIGNED, "%s is not aligned to its element size", names[i]);
    gdr::DecodeArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.state = state; a.o = o;
    a.B = B; a.Hk = Hk; a.Hv = Hv; a.Dk = Dk; a.Dv = Dv; a.gate_mode = gate_mode; a.dtype = dtype;
    cudaError_t e = gdr::launch_decode(a, (cudaStream_t)stream);
    if (e != cudaSuccess) return fail(GDR_ERR_CUDA, "CUDA launch failed: %s", cudaGetErrorString(e));
    g_launches += 1;
    return GDR_OK;
}

int gdr_causal_conv_silu(const void *x, const float *w, const float *bias, const void *state_in, void *state_out,
                         void *y, const int *cu_seqlens, int B, int T, int Ch, int width, int dtype, void *stream)
{
    if (B < 0 || T < 0 || Ch <= 0) return fail(GDR_ERR_INVALID_ARG, "sizes must be non-negative, Ch positive");
    if (dtype != GDR_BF16 && dtype != GDR_FP32)
        return fail(GDR_ERR_INVALID_ARG, "dtype must be GDR_BF16 or GDR_FP32 (got %d)", dtype);
    if (width != 4) return fail(GDR_ERR_UNSUPPORTED, "the convolution has 4 taps (got width %d)", width);
    if (Ch % 8) return fail(GDR_ERR_UNSUPPORTED, "Ch must be a multiple of 8 (got %d)", Ch);
    const long rows = cu_seqlens ? (long)T : (long)B * T;
    if (rows > 0 && (!x || !w || !y)) return fail(GDR_ERR_INVALID_ARG, "x, w and y must be non-NULL");
    if (rows > 0 && B == 0) return fail(GDR_ERR_INVALID_ARG, "packed tokens need at least one sequence");
    if (B > 0 && cu_seqlens && ((uintptr_t)cu_seqlens & 3u))
        return fail(GDR_ERR_MISALIGNED, "cu_seqlens is not 4-byte aligned");
    const void *ptrs[] = {x, w, y};
    const char *names[] = {"x", "w", "y"};
    for (int i = 0; i < 3; ++i)
        if (ptrs[i] && !aligned16(ptrs[i])) return fail(GDR_ERR_MISALIGNED, "%s is not 16-byte aligned", names[i]);
    const uintptr_t es = dtype == GDR_FP32 ? 4 : 2;
    if (((uintptr_t)state_in % es) || ((uintptr_t)state_out % es) || ((uintptr_t)bias & 3u))
        return fail(GDR_ERR_MISALIGNED, "a state or bias pointer is not aligned to its element size");
    if (x && x == y) return fail(GDR_ERR_INVALID_ARG, "y must not alias x");
    if (rows == 0 && (!state_out || B == 0)) return GDR_OK;   // nothing to compute or pass through
    gdr::ConvArgs a;
    a.x = x; a.w = w; a.bias = bias; a.state_in = state_in; a.state_out = state_out; a.y = y;
    a.cu_seqlens = cu_seqlens; a.nseq = B; a.T = T; a.rows = rows; a.Ch = Ch; a.fp32 = dtype == GDR_FP32;
    cudaError_t e = gdr::launch_conv_silu(a, (cudaStream_t)stream);
    if (e != cudaSuccess) return fail(GDR_ERR_CUDA, "CUDA launch failed: %s", cudaGetErrorString(e));
    g_launches += gdr::conv_launches(a);
    return GDR_OK;
}

int gdr_rmsnorm_gated(const void *o, const void *z, const float *weight, void *y, long rows, int D, float eps,
                      int dtype, void *stream)
{
    if (rows < 0) return fail(GDR_ERR_INVALID_ARG, "rows must be non-negative");
    if (dtype != GDR_BF16 && dtype != GDR_FP32)
        return fail(GDR_ERR_INVALID_ARG, "dtype must be GDR_BF16 or GDR_FP32 (got %d)", dtype);
    if (D != 64 && D != 128) return fail(GDR_ERR_UNSUPPORTED, "D must be 64 or 128 (got %d)", D);
    if (!(eps >= 0.f)) return fail(GDR_ERR_INVALID_ARG, "eps must be non-negative");
    if (rows == 0) return GDR_OK;
    if (!o || !z || !weight || !y) return fail(GDR_ERR_INVALID_ARG, "o, z, weight and y must be non-NULL");
    if (!aligned16(o) || !aligned16(z) || !aligned16(y) || ((uintptr_t)weight & 3u))
        return fail(GDR_ERR_MISALIGNED, "o, z and y must be 16-byte aligned, weight 4-byte aligned");
    gdr::NormArgs a;
    a.o = o; a.z = z; a.w = weight; a.y = y; a.rows = rows; a.D = D; a.eps = eps; a.fp32 = dtype == GDR_FP32;
    cudaError_t e = gdr::launch_rmsnorm_gated(a, (cudaStream_t)stream);
    if (e != cudaSuccess) return fail(GDR_ERR_CUDA, "CUDA launch failed: %s", cudaGetErrorString(e));
    g_launches += 1;
    return GDR_OK;
}

}  // extern "C"
