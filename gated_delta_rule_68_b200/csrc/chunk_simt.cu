// fp32 CUDA-core chunked forward of the gated delta rule (three kernels).
//
// This path serves fp32 inputs, where the 1e-4 accuracy asked of fp32 rules
// out bf16 or tf32 tensor-core operands, and any shape the tensor-core path
// does not take. It evaluates the recurrence chunk by chunk with no
// approximation (SinkProbe (Attention-Sink) README, description of its
// delta-rule layer), with chunks of C = 64 tokens. For one (b, h) and one chunk with
// cumulative log-gate G_r = sum_{j<=r} g_j and Gamma = exp(G):
//
//   prep  (chunk-parallel)  A = tril(diag(beta)(K*Gamma)(K/Gamma)^T, -1)
//                           T = (I + A)^-1 by blocked forward substitution
//                           W = T diag(beta)(K*Gamma),  U = T diag(beta) V
//                           M = tril((Q*Gamma)(K/Gamma)^T, 0)
//   scan  (sequential)      S_c = S;  U' = U - W S;
//                           S <- diag(Gamma_C) S + (K*Gamma_C/Gamma)^T U'
//   out   (chunk-parallel)  O = (Q*Gamma) S_c + M U'
//
// The (K*Gamma)(K/Gamma)^T products are formed element by element as
// k_r k_i exp(G_r - G_i), so no exp(-G) factor can overflow whatever the gate
// strength (NextTransformer "Source notes", "Backend and numerical limits":
// whole-chunk KDA algebra can overflow fp32 for strong gates).
//
// The kernels exchange W, U/U', M, G and S_c through the caller's workspace.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace gdr {
namespace {

constexpr int C = kChunk;
constexpr int NT = 256;

struct Work {
    float *W, *U, *M, *G, *Sc;
};

inline size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

Work carve(const FwdArgs &a, void *ws, size_t *total)
{
    const size_t NC = (size_t)(a.T + C - 1) / C;
    const size_t units = (size_t)a.B * a.Hv * NC;
    const size_t nW = a256(units * C * a.Dk * 4), nU = a256(units * C * a.Dv * 4);
    const size_t nM = a256(units * C * C * 4), nG = a256(units * C * (a.gate_mode ? a.Dk : 1) * 4);
    const size_t nS = a256(units * (size_t)a.Dk * a.Dv * 4);
    *total = nW + nU + nM + nG + nS;
    Work w{};
    if (ws) {
        char *p = (char *)ws;
        w.W = (float *)p; p += nW;
        w.U = (float *)p; p += nU;
        w.M = (float *)p; p += nM;
        w.G = (float *)p; p += nG;
        w.Sc = (float *)p;
    }
    return w;
}

template <int DK, int DV, int GATE>
struct PrepSmem {
    static constexpr int LDK = DK + 1, LDV = DV + 1, LDC = C + 1;
    static constexpr int LDX = (LDK > LDV ? LDK : LDV);
    static constexpr int floats = C * LDK + C * LDX + (GATE ? C * LDK : C) + 2 * C * LDC + 16 * 48 + C;
    static constexpr size_t bytes = (size_t)floats * 4;
};

// ---------------------------------------------------------------- prep kernel
template <typename TIn, int DK, int DV, int GATE>
__global__ void __launch_bounds__(NT) prep_kernel(FwdArgs a, Work w, int NC)
{
    using L = PrepSmem<DK, DV, GATE>;
    constexpr int LDK = L::LDK, LDV = L::LDV, LDC = L::LDC;
    extern __shared__ float sm[];
    float *Ks = sm;                         // [C][LDK]  K, later beta*K*Gamma
    float *Qs = Ks + C * LDK;               // [C][LDX]  Q, later beta*V
    float *Gs = Qs + C * L::LDX;            // [C][LDK] or [C]
    float *As = Gs + (GATE ? C * LDK : C);  // [C][LDC]
    float *Ts = As + C * LDC;               // [C][LDC]
    float *Xs = Ts + C * LDC;               // [16][48]
    float *bs = Xs + 16 * 48;               // [C]

    const int tid = threadIdx.x;
    const int ch = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int hk = h / (a.Hv / a.Hk);
    const int t0 = ch * C, n = min(C, a.T - t0);
    const long unit = ((long)b * a.Hv + h) * NC + ch;
    const TIn *qg = (const TIn *)a.q, *kg = (const TIn *)a.k, *vg = (const TIn *)a.v;

    for (int idx = tid; idx < C * DK; idx += NT) {
        const int r = idx / DK, c = idx % DK;
        float kv = 0.f, qv = 0.f;
        if (r < n) {
            const long off = (((long)b * a.T + t0 + r) * a.Hk + hk) * DK + c;
            kv = In<TIn>::load(kg + off);
            qv = In<TIn>::load(qg + off);
        }
        Ks[r * LDK + c] = kv;
        Qs[r * LDK + c] = qv;
    }
    if (tid < C) bs[tid] = tid < n ? a.beta[((long)b * a.T + t0 + tid) * a.Hv + h] : 0.f;
    if (GATE == 0) {
        if (tid < 32) {  // inclusive scan of 64 gates, two per lane
            const long base = ((long)b * a.T + t0) * a.Hv + h;
            const float x0 = (2 * tid < n) ? a.g[base + (long)(2 * tid) * a.Hv] : 0.f;
            const float x1 = (2 * tid + 1 < n) ? a.g[base + (long)(2 * tid + 1) * a.Hv] : 0.f;
            float s = x0 + x1;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, s, off);
                if (tid >= off) s += y;
            }
            const float excl = s - (x0 + x1);
            Gs[2 * tid] = excl + x0;
            Gs[2 * tid + 1] = excl + x0 + x1;
        }
    } else {
        for (int c = tid; c < DK; c += NT) {
            float s = 0.f;
#pragma unroll 8
            for (int r = 0; r < C; ++r) {
                if (r < n) s += a.g[(((long)b * a.T + t0 + r) * a.Hv + h) * DK + c];
                Gs[r * LDK + c] = s;
            }
        }
    }
    __syncthreads();

    float *Gw = w.G + unit * C * (GATE ? DK : 1);
    if (GATE == 0) {
        if (tid < C) Gw[tid] = Gs[tid];
    } else {
        for (int idx = tid; idx < C * DK; idx += NT) Gw[idx] = Gs[(idx / DK) * LDK + idx % DK];
    }

    // Gram: A (strictly lower, times beta_r) and M (lower with diagonal).
    float *Mw = w.M + unit * C * C;
    for (int p = tid; p < C * (C + 1) / 2; p += NT) {
        int r = (int)((sqrtf(8.f * p + 1.f) - 1.f) * 0.5f);
        while ((r + 1) * (r + 2) / 2 <= p) ++r;
        while (r * (r + 1) / 2 > p) --r;
        const int i = p - r * (r + 1) / 2;
        float acc_a = 0.f, acc_m = 0.f;
        if (GATE == 0) {
#pragma unroll 8
            for (int c = 0; c < DK; ++c) {
                const float ki = Ks[i * LDK + c];
                acc_a += Ks[r * LDK + c] * ki;
                acc_m += Qs[r * LDK + c] * ki;
            }
            const float e = expf(Gs[r] - Gs[i]);
            acc_a *= e;
            acc_m *= e;
        } else {
#pragma unroll 8
            for (int c = 0; c < DK; ++c) {
                const float e = expf(Gs[r * LDK + c] - Gs[i * LDK + c]);
                const float ki = Ks[i * LDK + c] * e;
                acc_a += Ks[r * LDK + c] * ki;
                acc_m += Qs[r * LDK + c] * ki;
            }
        }
        As[r * LDC + i] = (i < r) ? bs[r] * acc_a : 0.f;
        Mw[r * C + i] = acc_m;
    }
    for (int idx = tid; idx < C * LDC; idx += NT) Ts[idx] = 0.f;
    __syncthreads();

    // T = (I + A)^-1: invert the four 16x16 diagonal blocks by forward
    // substitution (one thread per block column), then fill block rows
    // bi = 1..3 with T_{bi,bj} = -T_{bi,bi} sum_{m=bj}^{bi-1} A_{bi,m} T_{m,bj}.
    if (tid < C) {
        const int base = (tid >> 4) * 16, col = tid & 15;
        float t[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float s = 0.f;
#pragma unroll
            for (int i = 0; i < r; ++i) s += As[(base + r) * LDC + base + i] * t[i];
            t[r] = (r < col) ? 0.f : (r == col ? 1.f : -s);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Ts[(base + r) * LDC + base + col] = t[r];
    }
    __syncthreads();
    for (int bi = 1; bi < 4; ++bi) {
        for (int e = tid; e < bi * 256; e += NT) {
            const int bj = e >> 8, r = (e >> 4) & 15, c = e & 15;
            float s = 0.f;
            for (int x = 16 * bj; x < 16 * bi; ++x)
                s += As[(16 * bi + r) * LDC + x] * Ts[x * LDC + 16 * bj + c];
            Xs[r * 48 + bj * 16 + c] = s;
        }
        __syncthreads();
        for (int e = tid; e < bi * 256; e += NT) {
            const int bj = e >> 8, r = (e >> 4) & 15, c = e & 15;
            float s = 0.f;
#pragma unroll
            for (int x = 0; x < 16; ++x) s += Ts[(16 * bi + r) * LDC + 16 * bi + x] * Xs[x * 48 + bj * 16 + c];
            Ts[(16 * bi + r) * LDC + 16 * bj + c] = -s;
        }
        __syncthreads();
    }

    // W = T diag(beta) (K*Gamma)
    for (int idx = tid; idx < C * DK; idx += NT) {
        const int r = idx / DK, c = idx % DK;
        const float gam = expf(GATE ? Gs[r * LDK + c] : Gs[r]);
        Ks[r * LDK + c] *= bs[r] * gam;
    }
    // beta * V into the Q buffer (Q is no longer needed)
    for (int idx = tid; idx < C * DV; idx += NT) {
        const int r = idx / DV, c = idx % DV;
        float x = 0.f;
        if (r < n) x = In<TIn>::load(vg + (((long)b * a.T + t0 + r) * a.Hv + h) * DV + c);
        Qs[r * LDV + c] = x * bs[r];
    }
    __syncthreads();
    float *Wg = w.W + unit * C * DK;
    for (int idx = tid; idx < C * DK; idx += NT) {
        const int r = idx / DK, c = idx % DK;
        float s = 0.f;
        for (int i = 0; i <= r; ++i) s += Ts[r * LDC + i] * Ks[i * LDK + c];
        Wg[idx] = s;
    }
    float *Ug = w.U + unit * C * DV;
    for (int idx = tid; idx < C * DV; idx += NT) {
        const int r = idx / DV, c = idx % DV;
        float s = 0.f;
        for (int i = 0; i <= r; ++i) s += Ts[r * LDC + i] * Qs[i * LDV + c];
        Ug[idx] = s;
    }
}

// ---------------------------------------------------------------- scan kernel
constexpr int DVS = 32;  // state columns per CTA

template <int DK>
struct ScanSmem {
    static constexpr int LDK = DK + 1, LDS = DVS + 1;
    static constexpr size_t bytes = (size_t)(DK * DVS + 2 * C * LDK + C * LDS + DK) * 4;
};

template <typename TIn, int DK, int DV, int GATE>
__global__ void __launch_bounds__(NT) scan_kernel(FwdArgs a, Work w, int NC)
{
    constexpr int LDK = DK + 1, LDS = DVS + 1;
    extern __shared__ float sm[];
    float *Ss = sm;               // [DK][DVS]
    float *Ws = Ss + DK * DVS;    // [C][LDK]
    float *Kt = Ws + C * LDK;     // [C][LDK]  K * Gamma_C / Gamma
    float *Us = Kt + C * LDK;     // [C][LDS]
    float *gl = Us + C * LDS;     // [DK]      Gamma_C

    const int tid = threadIdx.x;
    const int j0 = blockIdx.x * DVS, h = blockIdx.y, b = blockIdx.z;
    const int hk = h / (a.Hv / a.Hk);
    const long bh = (long)b * a.Hv + h;
    const TIn *kg = (const TIn *)a.k;

    for (int idx = tid; idx < DK * DVS; idx += NT) {
        const int c = idx / DVS, j = idx % DVS;
        Ss[idx] = a.h0 ? a.h0[(bh * DK + c) * DV + j0 + j] : 0.f;
    }
    for (int ch = 0; ch < NC; ++ch) {
        const long unit = bh * NC + ch;
        const int t0 = ch * C, n = min(C, a.T - t0);
        __syncthreads();
        float *Sc = w.Sc + unit * DK * DV;
        for (int idx = tid; idx < DK * DVS; idx += NT) {
            const int c = idx / DVS, j = idx % DVS;
            Sc[(long)c * DV + j0 + j] = Ss[idx];
        }
        const float *Wg = w.W + unit * C * DK;
        const float *Gw = w.G + unit * C * (GATE ? DK : 1);
        for (int idx = tid; idx < C * DK; idx += NT) {
            const int r = idx / DK, c = idx % DK;
            Ws[r * LDK + c] = Wg[idx];
            float kv = 0.f;
            if (r < n) kv = In<TIn>::load(kg + (((long)b * a.T + t0 + r) * a.Hk + hk) * DK + c);
            const float gr = GATE ? Gw[r * DK + c] : Gw[r];
            const float gL = GATE ? Gw[(C - 1) * DK + c] : Gw[C - 1];
            Kt[r * LDK + c] = kv * expf(gL - gr);
        }
        for (int c = tid; c < DK; c += NT) gl[c] = expf(GATE ? Gw[(C - 1) * DK + c] : Gw[C - 1]);
        float *Ug = w.U + unit * C * DV;
        for (int idx = tid; idx < C * DVS; idx += NT) {
            const int r = idx / DVS, j = idx % DVS;
            Us[r * LDS + j] = Ug[(long)r * DV + j0 + j];
        }
        __syncthreads();
        {   // U' = U - W S
            const int j = tid % DVS;
            for (int r = tid / DVS; r < C; r += NT / DVS) {
                float s = 0.f;
#pragma unroll 8
                for (int c = 0; c < DK; ++c) s += Ws[r * LDK + c] * Ss[c * DVS + j];
                const float up = Us[r * LDS + j] - s;
                Us[r * LDS + j] = up;
                Ug[(long)r * DV + j0 + j] = up;
            }
        }
        __syncthreads();
        {   // S <- diag(Gamma_C) S + Kt^T U'
            const int j = tid % DVS;
            for (int c = tid / DVS; c < DK; c += NT / DVS) {
                float s = gl[c] * Ss[c * DVS + j];
#pragma unroll 8
                for (int r = 0; r < C; ++r) s += Kt[r * LDK + c] * Us[r * LDS + j];
                Ss[c * DVS + j] = s;
            }
        }
    }
    __syncthreads();
    if (a.hT) {
        for (int idx = tid; idx < DK * DVS; idx += NT) {
            const int c = idx / DVS, j = idx % DVS;
            a.hT[(bh * DK + c) * DV + j0 + j] = Ss[idx];
        }
    }
}

// ---------------------------------------------------------------- output kernel
template <int DK, int DV>
struct OutSmem {
    static constexpr size_t bytes = (size_t)(C * (DK + 1) + DK * DV + C * (C + 1) + C * (DV + 1)) * 4;
};

template <typename TIn, typename TOut, int DK, int DV, int GATE>
__global__ void __launch_bounds__(NT) out_kernel(FwdArgs a, Work w, int NC)
{
    constexpr int LDK = DK + 1, LDV = DV + 1, LDC = C + 1;
    extern __shared__ float sm[];
    float *QG = sm;              // [C][LDK]  Q * Gamma
    float *Ss = QG + C * LDK;    // [DK][DV]  chunk entry state
    float *Ms = Ss + DK * DV;    // [C][LDC]
    float *Up = Ms + C * LDC;    // [C][LDV]

    const int tid = threadIdx.x;
    const int ch = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int hk = h / (a.Hv / a.Hk);
    const int t0 = ch * C, n = min(C, a.T - t0);
    const long unit = ((long)b * a.Hv + h) * NC + ch;
    const TIn *qg = (const TIn *)a.q;
    const float *Gw = w.G + unit * C * (GATE ? DK : 1);

    for (int idx = tid; idx < C * DK; idx += NT) {
        const int r = idx / DK, c = idx % DK;
        float x = 0.f;
        if (r < n) {
            x = In<TIn>::load(qg + (((long)b * a.T + t0 + r) * a.Hk + hk) * DK + c);
            x *= expf(GATE ? Gw[r * DK + c] : Gw[r]);
        }
        QG[r * LDK + c] = x;
    }
    const float *Sc = w.Sc + unit * DK * DV;
    for (int idx = tid; idx < DK * DV; idx += NT) Ss[idx] = Sc[idx];
    const float *Mw = w.M + unit * C * C;
    for (int idx = tid; idx < C * C; idx += NT) {
        const int r = idx / C, i = idx % C;
        Ms[r * LDC + i] = (i <= r) ? Mw[idx] : 0.f;
    }
    const float *Ug = w.U + unit * C * DV;
    for (int idx = tid; idx < C * DV; idx += NT) Up[(idx / DV) * LDV + idx % DV] = Ug[idx];
    __syncthreads();

    TOut *og = (TOut *)a.o;
    for (int idx = tid; idx < C * DV; idx += NT) {
        const int r = idx / DV, j = idx % DV;
        if (r >= n) continue;
        float s = 0.f;
#pragma unroll 8
        for (int c = 0; c < DK; ++c) s += QG[r * LDK + c] * Ss[c * DV + j];
        for (int i = 0; i <= r; ++i) s += Ms[r * LDC + i] * Up[i * LDV + j];
        In<TOut>::store(og + (((long)b * a.T + t0 + r) * a.Hv + h) * DV + j, s);
    }
}

template <typename TIn, typename TOut, int DK, int DV, int GATE>
cudaError_t launch_t(const FwdArgs &a, const Work &w, cudaStream_t st)
{
    const int NC = (a.T + C - 1) / C;
    const size_t s1 = PrepSmem<DK, DV, GATE>::bytes, s2 = ScanSmem<DK>::bytes, s3 = OutSmem<DK, DV>::bytes;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(prep_kernel<TIn, DK, DV, GATE>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1))) return e;
    if ((e = cudaFuncSetAttribute(scan_kernel<TIn, DK, DV, GATE>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2))) return e;
    if ((e = cudaFuncSetAttribute(out_kernel<TIn, TOut, DK, DV, GATE>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s3))) return e;
    prep_kernel<TIn, DK, DV, GATE><<<dim3(NC, a.Hv, a.B), NT, s1, st>>>(a, w, NC);
    scan_kernel<TIn, DK, DV, GATE><<<dim3(DV / DVS, a.Hv, a.B), NT, s2, st>>>(a, w, NC);
    out_kernel<TIn, TOut, DK, DV, GATE><<<dim3(NC, a.Hv, a.B), NT, s3, st>>>(a, w, NC);
    return cudaGetLastError();
}

template <typename TIn, typename TOut, int DK, int DV>
cudaError_t launch_g(const FwdArgs &a, const Work &w, cudaStream_t st)
{
    return a.gate_mode == 0 ? launch_t<TIn, TOut, DK, DV, 0>(a, w, st)
                            : launch_t<TIn, TOut, DK, DV, 1>(a, w, st);
}

template <typename TIn, typename TOut>
cudaError_t launch_d(const FwdArgs &a, const Work &w, cudaStream_t st)
{
    if (a.Dk == 128 && a.Dv == 128) return launch_g<TIn, TOut, 128, 128>(a, w, st);
    if (a.Dk == 128 && a.Dv == 64) return launch_g<TIn, TOut, 128, 64>(a, w, st);
    if (a.Dk == 64 && a.Dv == 128) return launch_g<TIn, TOut, 64, 128>(a, w, st);
    return launch_g<TIn, TOut, 64, 64>(a, w, st);
}

}  // namespace

size_t simt_workspace_size(const FwdArgs &a)
{
    size_t total = 0;
    carve(a, nullptr, &total);
    return total;
}

cudaError_t launch_fwd_simt(const FwdArgs &a, void *ws, cudaStream_t st)
{
    size_t total = 0;
    const Work w = carve(a, ws, &total);
    if (!in_bf16(a.dtype)) return launch_d<float, float>(a, w, st);
    return out_f32(a.dtype) ? launch_d<__nv_bfloat16, float>(a, w, st)
                            : launch_d<__nv_bfloat16, __nv_bfloat16>(a, w, st);
}

}  // namespace gdr
