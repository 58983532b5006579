// Backward of the gated delta rule: gradients of L = sum(do * o) + sum(dhT * hT)
// with respect to q, k, v, g, beta and h0, in fp32 on the CUDA cores.
//
// Per token t (NextTransformer, "Source notes", "Linear attention", rows gdn and
// kda: decay before the delta update, readout after it):
//   forward   Sb = diag(a_t) S,  a_t = exp(g_t);  p = Sb^T k;  e = v - p;  u = beta e;
//             S' = Sb + k u^T;  o = S'^T q
//   backward  dS += q do^T;  dq = S' do;  du = dS^T k;  dk = dS u + Sb dp;
//             dbeta = du . e;  dv = beta du;  dp = -beta du;  dSb = dS + k dp^T;
//             dg = row sums of dSb * Sb (summed over rows for a scalar gate);
//             dS <- diag(a_t) dSb;  and dh0 = dS after the first token.
//
// The columns of S (value channels) evolve independently, so one CTA takes a
// (batch row, value head, 32-column slice) and each of its Dk threads a row of
// that slice. Two kernels:
//   1. a forward pass that stores the state before every 8th token (workspace);
//   2. a reverse pass that, per block of 8 tokens, recomputes the decayed states
//      Sb from the block's checkpoint into shared memory, then runs the 8 reverse
//      steps. dv and dh0 belong to one slice and are stored; dq and dk (summed
//      over slices and over the value heads that share a key head), dbeta and dg
//      are accumulated with atomics into zeroed outputs.
// Column sums over the Dk rows (p and du) use a shuffle transpose-reduce per warp
// and shared memory across warps.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace gdr {
namespace {

constexpr int BW = 32;      // value columns per CTA
constexpr int BLK = 8;      // tokens between checkpoints
constexpr int SBLD = 36;    // fp32 row stride of a recomputed state slice (conflict-free 16-byte stores)

// Sum over the block's rows of x[j] for the 32 columns: a transpose-reduce inside each
// warp (lane j ends with the warp's sum of column j), then across warps through shared
// memory. Every thread returns with all 32 totals in tot (shared, read after the call).
template <int NWARP>
__device__ __forceinline__ void column_sums(float x[BW], float *red, float *tot)
{
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) {
        const bool upper = (lane & s) != 0;
#pragma unroll
        for (int i = 0; i < s; ++i) {
            const float send = upper ? x[i] : x[i + s];
            const float keep = upper ? x[i + s] : x[i];
            x[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
        }
    }
    red[w * BW + lane] = x[0];
    __syncthreads();
    if (threadIdx.x < BW) {
        float s = 0.f;
#pragma unroll
        for (int k = 0; k < NWARP; ++k) s += red[k * BW + threadIdx.x];
        tot[threadIdx.x] = s;
    }
    __syncthreads();
}

template <typename TIn>
__device__ __forceinline__ float ld(const TIn *p) { return In<TIn>::load(p); }

template <typename TIn, int GATE, int DK>
__global__ void __launch_bounds__(DK)
bwd_ckpt_kernel(BwdArgs a, float *ck)
{
    constexpr int NWARP = DK / 32;
    __shared__ float red[NWARP * BW], tot[BW], vrows[2 * BW];   // v rows of even and odd tokens
    const int i = threadIdx.x, j0 = blockIdx.x * BW, unit = blockIdx.y;
    const int b = unit / a.Hv, h = unit % a.Hv, hk = h / (a.Hv / a.Hk);
    const int T = a.T, M = (T + BLK - 1) / BLK, Dv = a.Dv;
    float S[BW];
    const float *h0 = a.h0 ? a.h0 + ((size_t)unit * DK + i) * Dv + j0 : nullptr;
#pragma unroll
    for (int j = 0; j < BW; ++j) S[j] = h0 ? h0[j] : 0.f;
    float *cku = ck + (size_t)unit * M * DK * Dv;
    auto store = [&](int m) {
        float4 *dst = reinterpret_cast<float4 *>(cku + ((size_t)m * DK + i) * Dv + j0);
#pragma unroll
        for (int j = 0; j < BW / 4; ++j) dst[j] = make_float4(S[4 * j], S[4 * j + 1], S[4 * j + 2], S[4 * j + 3]);
    };
    store(0);
    for (int t = 0; t < T; ++t) {
        const size_t tv = (size_t)b * T + t;
        const float ai = __expf(GATE ? a.g[(tv * a.Hv + h) * DK + i] : a.g[tv * a.Hv + h]);
        const float ki = ld(reinterpret_cast<const TIn *>(a.k) + (tv * a.Hk + hk) * DK + i);
        const float bt = a.beta[tv * a.Hv + h];
        float *vrow = vrows + (t & 1) * BW;
        if (i < BW) vrow[i] = ld(reinterpret_cast<const TIn *>(a.v) + (tv * a.Hv + h) * Dv + j0 + i);
        float x[BW];
#pragma unroll
        for (int j = 0; j < BW; ++j) S[j] *= ai, x[j] = S[j] * ki;
        column_sums<NWARP>(x, red, tot);
#pragma unroll
        for (int j = 0; j < BW; ++j) S[j] = fmaf(ki, bt * (vrow[j] - tot[j]), S[j]);
        if ((t + 1) % BLK == 0 && t + 1 < T) store((t + 1) / BLK);
    }
}

template <typename TIn, int GATE, int DK>
__global__ void __launch_bounds__(DK)
bwd_kernel(BwdArgs a, const float *ck)
{
    constexpr int NWARP = DK / 32;
    extern __shared__ __align__(16) float smf[];
    float *Sbs = smf;                                   // [BLK][DK][SBLD] recomputed Sb of the block's tokens
    float *es = Sbs + BLK * DK * SBLD;                  // [BLK][32] e of the block's tokens
    float *red = es + BLK * BW, *tot = red + NWARP * BW, *vrows = tot + BW, *drow = vrows + 2 * BW;
    const int i = threadIdx.x, lane = i & 31, j0 = blockIdx.x * BW, unit = blockIdx.y;
    const int b = unit / a.Hv, h = unit % a.Hv, hk = h / (a.Hv / a.Hk);
    const int T = a.T, M = (T + BLK - 1) / BLK, Dv = a.Dv;
    const TIn *q = reinterpret_cast<const TIn *>(a.q), *k = reinterpret_cast<const TIn *>(a.k);
    const TIn *v = reinterpret_cast<const TIn *>(a.v), *dout = reinterpret_cast<const TIn *>(a.dout);
    float dS[BW];
    const float *dhT = a.dhT ? a.dhT + ((size_t)unit * DK + i) * Dv + j0 : nullptr;
#pragma unroll
    for (int j = 0; j < BW; ++j) dS[j] = dhT ? dhT[j] : 0.f;
    const float *cku = ck + (size_t)unit * M * DK * Dv;
    for (int m = M - 1; m >= 0; --m) {
        const int t0 = m * BLK, n = min(BLK, T - t0);
        // recompute the block's decayed states Sb and e from its checkpoint
        float S[BW];
        {
            const float4 *src = reinterpret_cast<const float4 *>(cku + ((size_t)m * DK + i) * Dv + j0);
#pragma unroll
            for (int j = 0; j < BW / 4; ++j) {
                const float4 x = src[j];
                S[4 * j] = x.x, S[4 * j + 1] = x.y, S[4 * j + 2] = x.z, S[4 * j + 3] = x.w;
            }
        }
        for (int tt = 0; tt < n; ++tt) {
            const size_t tv = (size_t)b * T + t0 + tt;
            const float ai = __expf(GATE ? a.g[(tv * a.Hv + h) * DK + i] : a.g[tv * a.Hv + h]);
            const float ki = ld(k + (tv * a.Hk + hk) * DK + i);
            const float bt = a.beta[tv * a.Hv + h];
            float *vrow = vrows + (tt & 1) * BW;   // even and odd tokens alternate
            if (i < BW) vrow[i] = ld(v + (tv * a.Hv + h) * Dv + j0 + i);
            float x[BW];
            float4 *sb = reinterpret_cast<float4 *>(Sbs + ((size_t)tt * DK + i) * SBLD);
#pragma unroll
            for (int j = 0; j < BW; ++j) S[j] *= ai, x[j] = S[j] * ki;
#pragma unroll
            for (int j = 0; j < BW / 4; ++j) sb[j] = make_float4(S[4 * j], S[4 * j + 1], S[4 * j + 2], S[4 * j + 3]);
            column_sums<NWARP>(x, red, tot);
            if (i < BW) es[tt * BW + i] = vrow[i] - tot[i];
#pragma unroll
            for (int j = 0; j < BW; ++j) S[j] = fmaf(ki, bt * (vrow[j] - tot[j]), S[j]);
        }
        __syncthreads();
        // reverse the block's steps
        for (int tt = n - 1; tt >= 0; --tt) {
            const size_t tv = (size_t)b * T + t0 + tt;
            const float ai = __expf(GATE ? a.g[(tv * a.Hv + h) * DK + i] : a.g[tv * a.Hv + h]);
            const size_t kq = (tv * a.Hk + hk) * DK + i;
            const float ki = ld(k + kq), qi = ld(q + kq);
            const float bt = a.beta[tv * a.Hv + h];
            if (i < BW) drow[i] = ld(dout + (tv * a.Hv + h) * Dv + j0 + i);
            __syncthreads();
            float Sb[BW], e[BW], dd[BW];
            {
                const float4 *sb = reinterpret_cast<const float4 *>(Sbs + ((size_t)tt * DK + i) * SBLD);
#pragma unroll
                for (int j = 0; j < BW / 4; ++j) {
                    const float4 x = sb[j];
                    Sb[4 * j] = x.x, Sb[4 * j + 1] = x.y, Sb[4 * j + 2] = x.z, Sb[4 * j + 3] = x.w;
                }
            }
#pragma unroll
            for (int j = 0; j < BW; ++j) e[j] = es[tt * BW + j], dd[j] = drow[j];
            // o = S'^T q
            float dq = 0.f;
#pragma unroll
            for (int j = 0; j < BW; ++j) {
                dS[j] = fmaf(qi, dd[j], dS[j]);
                dq = fmaf(fmaf(ki, bt * e[j], Sb[j]), dd[j], dq);
            }
            atomicAdd(a.dq + kq, dq);
            // S' = Sb + k u^T
            float x[BW];
#pragma unroll
            for (int j = 0; j < BW; ++j) x[j] = dS[j] * ki;
            column_sums<NWARP>(x, red, tot);
            float dk = 0.f, db = 0.f, rg = 0.f;
#pragma unroll
            for (int j = 0; j < BW; ++j) {
                const float du = tot[j], dp = -bt * du;
                dk = fmaf(dS[j], bt * e[j], dk);       // dS u
                db = fmaf(du, e[j], db);
                dk = fmaf(Sb[j], dp, dk);              // Sb dp
                const float dSb = fmaf(ki, dp, dS[j]);
                rg = fmaf(dSb, Sb[j], rg);
                dS[j] = ai * dSb;
            }
            atomicAdd(a.dk + kq, dk);
            if (i == 0) atomicAdd(a.dbeta + tv * a.Hv + h, db);
            if (i < BW) a.dv[(tv * a.Hv + h) * Dv + j0 + i] = bt * tot[i];
            if (GATE) {
                atomicAdd(a.dg + (tv * a.Hv + h) * DK + i, rg);
            } else {
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) rg += __shfl_xor_sync(0xffffffffu, rg, off);
                if (lane == 0) atomicAdd(a.dg + tv * a.Hv + h, rg);
            }
        }
    }
    float *dh0 = a.dh0 + ((size_t)unit * DK + i) * Dv + j0;
#pragma unroll
    for (int j = 0; j < BW / 4; ++j)
        reinterpret_cast<float4 *>(dh0)[j] = make_float4(dS[4 * j], dS[4 * j + 1], dS[4 * j + 2], dS[4 * j + 3]);
}

template <int DK>
constexpr size_t bwd_smem() { return ((size_t)BLK * DK * SBLD + BLK * BW + (DK / 32) * BW + 4 * BW) * sizeof(float); }

template <typename TIn, int GATE, int DK>
cudaError_t launch_t(const BwdArgs &a, void *ws, cudaStream_t st)
{
    const dim3 grid(a.Dv / BW, a.B * a.Hv);
    float *ck = reinterpret_cast<float *>(ws);
    bwd_ckpt_kernel<TIn, GATE, DK><<<grid, DK, 0, st>>>(a, ck);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bwd_kernel<TIn, GATE, DK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)bwd_smem<DK>());
    if (e != cudaSuccess) return e;
    bwd_kernel<TIn, GATE, DK><<<grid, DK, bwd_smem<DK>(), st>>>(a, ck);
    return cudaGetLastError();
}

template <typename TIn, int GATE>
cudaError_t launch_g(const BwdArgs &a, void *ws, cudaStream_t st)
{
    return a.Dk == 64 ? launch_t<TIn, GATE, 64>(a, ws, st) : launch_t<TIn, GATE, 128>(a, ws, st);
}

}  // namespace

bool bwd_supported(const BwdArgs &a)
{
    return (a.Dk == 64 || a.Dk == 128) && a.Dv % BW == 0 && a.Dv > 0;
}

size_t bwd_workspace_size(const BwdArgs &a)
{
    const size_t M = (size_t)(a.T + BLK - 1) / BLK;
    return (size_t)a.B * a.Hv * M * a.Dk * a.Dv * sizeof(float);
}

cudaError_t launch_bwd(const BwdArgs &a, void *ws, cudaStream_t st)
{
    if (in_bf16(a.dtype))
        return a.gate_mode ? launch_g<__nv_bfloat16, 1>(a, ws, st) : launch_g<__nv_bfloat16, 0>(a, ws, st);
    return a.gate_mode ? launch_g<float, 1>(a, ws, st) : launch_g<float, 0>(a, ws, st);
}

}  // namespace gdr
