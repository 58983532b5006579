// Backward of the gated delta rule: gradients of L = sum(do * o) + sum(dhT * hT) with respect
// to q, k, v, g, beta and h0, in fp32 on the CUDA cores.
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
// (batch row, value head, 16-column slice) and each of its Dk threads a row of
// that slice. Two kernels:
//   1. a forward pass that stores the state before every 8th token (workspace);
//   2. a reverse pass that, per block of 8 tokens, recomputes the decayed states
//      Sb from the block's checkpoint into shared memory, then runs the 8 reverse
//      steps. dv and dh0 belong to one slice and are stored; dq and dk (summed
//      over slices and over the value heads that share a key head), dbeta and dg
//      are accumulated with atomics into zeroed outputs.
// Both kernels stage a block's inputs (k, q, the slice's v and do columns, g, beta)
// in shared memory with asynchronous copies one block ahead, so no token waits on a
// global load. Column sums over the Dk rows (p and du) use a shuffle transpose-reduce
// per warp and shared memory across warps. The reverse kernel's shared memory (about
// 92 KB for bf16 inputs and the scalar gate, 110 KB at most) lets two CTAs share an SM.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace gdr {
namespace {

constexpr int BW = 16;      // value columns per CTA
constexpr int BLK = 8;      // tokens between checkpoints
constexpr int SBLD = 20;    // fp32 row stride of a recomputed state slice (conflict-free 16-byte stores)

__device__ __forceinline__ uint32_t saddr(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void cp16(void *dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp4(void *dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(saddr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// One block's inputs in shared memory: k and q rows of the key head, the slice's
// columns of v and do, the gate (one value, or Dk for the per-channel gate) and beta.
template <typename TIn, int GATE, int DK>
struct alignas(16) Stage {
    TIn k[BLK][DK];
    TIn q[BLK][DK];
    TIn v[BLK][BW];
    TIn d[BLK][BW];
    float g[BLK][GATE ? DK : 4];
    float beta[BLK];
};

// Issue the asynchronous copies of tokens t0 .. t0 + n - 1 (q and do only for the reverse
// pass) as one commit group. Every source row starts on a 16-byte boundary: the API checks
// the base pointers, and row strides and slice offsets are multiples of 16 bytes.
template <typename TIn, int GATE, int DK, bool REV>
__device__ __forceinline__ void stage_issue(Stage<TIn, GATE, DK> &s, const BwdArgs &a, int b, int h, int hk,
                                            int j0, int t0, int n)
{
    constexpr int E = 16 / sizeof(TIn);            // elements per 16-byte copy
    constexpr int CR = DK / E, CV = BW / E;        // copies per k row and per v slice row
    const int tid = threadIdx.x;
    const TIn *k = reinterpret_cast<const TIn *>(a.k), *q = reinterpret_cast<const TIn *>(a.q);
    const TIn *v = reinterpret_cast<const TIn *>(a.v), *d = reinterpret_cast<const TIn *>(a.dout);
    for (int c = tid; c < n * CR; c += DK) {
        const int tt = c / CR, x = (c % CR) * E;
        const size_t off = (((size_t)b * a.T + t0 + tt) * a.Hk + hk) * DK + x;
        cp16(&s.k[tt][x], k + off);
        if (REV) cp16(&s.q[tt][x], q + off);
    }
    for (int c = tid; c < n * CV; c += DK) {
        const int tt = c / CV, x = (c % CV) * E;
        const size_t off = (((size_t)b * a.T + t0 + tt) * a.Hv + h) * a.Dv + j0 + x;
        cp16(&s.v[tt][x], v + off);
        if (REV) cp16(&s.d[tt][x], d + off);
    }
    if (GATE) {
        for (int c = tid; c < n * (DK / 4); c += DK) {
            const int tt = c / (DK / 4), x = (c % (DK / 4)) * 4;
            cp16(&s.g[tt][x], a.g + (((size_t)b * a.T + t0 + tt) * a.Hv + h) * DK + x);
        }
    } else if (tid < n) {
        cp4(&s.g[tid][0], a.g + ((size_t)b * a.T + t0 + tid) * a.Hv + h);
    }
    if (tid >= 32 && tid < 32 + n)
        cp4(&s.beta[tid - 32], a.beta + ((size_t)b * a.T + t0 + tid - 32) * a.Hv + h);
    cp_commit();
}

template <typename TIn>
__device__ __forceinline__ float ld(const TIn *p) { return In<TIn>::load(p); }

// The BW values of a staged slice row (broadcast reads).
__device__ __forceinline__ void load_row(const float *p, float x[BW])
{
#pragma unroll
    for (int j = 0; j < BW / 4; ++j) {
        const float4 f = reinterpret_cast<const float4 *>(p)[j];
        x[4 * j] = f.x, x[4 * j + 1] = f.y, x[4 * j + 2] = f.z, x[4 * j + 3] = f.w;
    }
}
__device__ __forceinline__ void load_row(const __nv_bfloat16 *p, float x[BW])
{
#pragma unroll
    for (int j = 0; j < BW / 8; ++j) {
        const uint4 u = reinterpret_cast<const uint4 *>(p)[j];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int m = 0; m < 4; ++m) {   // a bf16 is the high half of its fp32 value
            x[8 * j + 2 * m] = __uint_as_float(w[m] << 16);
            x[8 * j + 2 * m + 1] = __uint_as_float(w[m] & 0xffff0000u);
        }
    }
}

// Sum over the block's rows of x[j] for the BW columns: a transpose-reduce inside each
// warp (lanes j and j + 16 end with the warp's sum of column j), then across warps
// through shared memory. Every thread returns with all BW totals in tot (shared).
template <int NWARP>
__device__ __forceinline__ void column_sums(float x[BW], float *red, float *tot)
{
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int s = BW / 2; s >= 1; s >>= 1) {
        const bool upper = (lane & s) != 0;
#pragma unroll
        for (int i = 0; i < s; ++i) {
            const float send = upper ? x[i] : x[i + s];
            const float keep = upper ? x[i + s] : x[i];
            x[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
        }
    }
    x[0] += __shfl_xor_sync(0xffffffffu, x[0], 16);
    if (lane < BW) red[w * BW + lane] = x[0];
    __syncthreads();
    if (threadIdx.x < BW) {
        float s = 0.f;
#pragma unroll
        for (int k = 0; k < NWARP; ++k) s += red[k * BW + threadIdx.x];
        tot[threadIdx.x] = s;
    }
    __syncthreads();
}

template <typename TIn, int GATE, int DK>
__global__ void __launch_bounds__(DK)
bwd_ckpt_kernel(BwdArgs a, float *ck)
{
    constexpr int NWARP = DK / 32;
    __shared__ Stage<TIn, GATE, DK> st[2];
    __shared__ __align__(16) float red[NWARP * BW], tot[BW];
    const int i = threadIdx.x, j0 = blockIdx.x * BW, unit = blockIdx.y;
    const int b = unit / a.Hv, h = unit % a.Hv, hk = h / (a.Hv / a.Hk);
    const int T = a.T, M = (T + BLK - 1) / BLK, Dv = a.Dv;
    if (M > 0) stage_issue<TIn, GATE, DK, false>(st[0], a, b, h, hk, j0, 0, min(BLK, T));
    float S[BW];
    const float *h0 = a.h0 ? a.h0 + ((size_t)unit * DK + i) * Dv + j0 : nullptr;
#pragma unroll
    for (int j = 0; j < BW; ++j) S[j] = h0 ? h0[j] : 0.f;
    float *cku = ck + (size_t)unit * M * DK * Dv;
    for (int m = 0; m < M; ++m) {
        const int t0 = m * BLK, n = min(BLK, T - t0);
        float4 *dst = reinterpret_cast<float4 *>(cku + ((size_t)m * DK + i) * Dv + j0);
#pragma unroll
        for (int j = 0; j < BW / 4; ++j) dst[j] = make_float4(S[4 * j], S[4 * j + 1], S[4 * j + 2], S[4 * j + 3]);
        cp_wait_all();
        __syncthreads();   // block m staged; every thread is done with block m - 1's buffer
        if (m + 1 < M)
            stage_issue<TIn, GATE, DK, false>(st[(m + 1) & 1], a, b, h, hk, j0, t0 + BLK, min(BLK, T - t0 - BLK));
        const Stage<TIn, GATE, DK> &s = st[m & 1];
        for (int tt = 0; tt < n; ++tt) {
            const float ai = __expf(s.g[tt][GATE ? i : 0]);
            const float ki = ld(&s.k[tt][i]);
            const float bt = s.beta[tt];
            float x[BW], vr[BW];
#pragma unroll
            for (int j = 0; j < BW; ++j) S[j] *= ai, x[j] = S[j] * ki;
            column_sums<NWARP>(x, red, tot);
            load_row(&s.v[tt][0], vr);
#pragma unroll
            for (int j = 0; j < BW; ++j) S[j] = fmaf(ki, bt * (vr[j] - tot[j]), S[j]);
        }
    }
}

template <typename TIn, int GATE, int DK>
__global__ void __launch_bounds__(DK)
bwd_kernel(BwdArgs a, const float *ck)
{
    constexpr int NWARP = DK / 32;
    extern __shared__ __align__(16) unsigned char smraw[];
    Stage<TIn, GATE, DK> *st = reinterpret_cast<Stage<TIn, GATE, DK> *>(smraw);
    float *Sbs = reinterpret_cast<float *>(smraw + 2 * sizeof(Stage<TIn, GATE, DK>));  // [BLK][DK][SBLD]
    float *es = Sbs + BLK * DK * SBLD;                  // [BLK][BW] e of the block's tokens
    float *red = es + BLK * BW, *tot = red + NWARP * BW;
    const int i = threadIdx.x, lane = i & 31, j0 = blockIdx.x * BW, unit = blockIdx.y;
    const int b = unit / a.Hv, h = unit % a.Hv, hk = h / (a.Hv / a.Hk);
    const int T = a.T, M = (T + BLK - 1) / BLK, Dv = a.Dv;
    if (M > 0) stage_issue<TIn, GATE, DK, true>(st[(M - 1) & 1], a, b, h, hk, j0, (M - 1) * BLK, T - (M - 1) * BLK);
    float dS[BW];
    const float *dhT = a.dhT ? a.dhT + ((size_t)unit * DK + i) * Dv + j0 : nullptr;
#pragma unroll
    for (int j = 0; j < BW; ++j) dS[j] = dhT ? dhT[j] : 0.f;
    const float *cku = ck + (size_t)unit * M * DK * Dv;
    for (int m = M - 1; m >= 0; --m) {
        const int t0 = m * BLK, n = min(BLK, T - t0);
        float S[BW];
        {
            const float4 *src = reinterpret_cast<const float4 *>(cku + ((size_t)m * DK + i) * Dv + j0);
#pragma unroll
            for (int j = 0; j < BW / 4; ++j) {
                const float4 x = src[j];
                S[4 * j] = x.x, S[4 * j + 1] = x.y, S[4 * j + 2] = x.z, S[4 * j + 3] = x.w;
            }
        }
        cp_wait_all();
        __syncthreads();   // block m staged; every thread is done with block m + 1 (its buffer, Sbs, es)
        if (m > 0) stage_issue<TIn, GATE, DK, true>(st[(m - 1) & 1], a, b, h, hk, j0, t0 - BLK, BLK);
        const Stage<TIn, GATE, DK> &s = st[m & 1];
        // recompute the block's decayed states Sb and e from its checkpoint
        for (int tt = 0; tt < n; ++tt) {
            const float ai = __expf(s.g[tt][GATE ? i : 0]);
            const float ki = ld(&s.k[tt][i]);
            const float bt = s.beta[tt];
            float x[BW], vr[BW];
            float4 *sb = reinterpret_cast<float4 *>(Sbs + ((size_t)tt * DK + i) * SBLD);
#pragma unroll
            for (int j = 0; j < BW; ++j) S[j] *= ai, x[j] = S[j] * ki;
#pragma unroll
            for (int j = 0; j < BW / 4; ++j) sb[j] = make_float4(S[4 * j], S[4 * j + 1], S[4 * j + 2], S[4 * j + 3]);
            column_sums<NWARP>(x, red, tot);
            load_row(&s.v[tt][0], vr);
            if (i < BW) es[tt * BW + i] = ld(&s.v[tt][i]) - tot[i];
#pragma unroll
            for (int j = 0; j < BW; ++j) S[j] = fmaf(ki, bt * (vr[j] - tot[j]), S[j]);
        }
        __syncthreads();   // es of the block visible to every thread
        // reverse the block's steps
        for (int tt = n - 1; tt >= 0; --tt) {
            const size_t tv = (size_t)b * T + t0 + tt;
            const float ai = __expf(s.g[tt][GATE ? i : 0]);
            const float ki = ld(&s.k[tt][i]), qi = ld(&s.q[tt][i]);
            const float bt = s.beta[tt];
            const size_t kq = (tv * a.Hk + hk) * DK + i;
            float Sb[BW], e[BW], dd[BW];
            {
                const float4 *sb = reinterpret_cast<const float4 *>(Sbs + ((size_t)tt * DK + i) * SBLD);
#pragma unroll
                for (int j = 0; j < BW / 4; ++j) {
                    const float4 x = sb[j];
                    Sb[4 * j] = x.x, Sb[4 * j + 1] = x.y, Sb[4 * j + 2] = x.z, Sb[4 * j + 3] = x.w;
                }
            }
            load_row(es + tt * BW, e);
            load_row(&s.d[tt][0], dd);
            // o = S'^T q: dS += q do^T, dq = S' do (two partial sums shorten the chain)
            float dq0 = 0.f, dq1 = 0.f;
#pragma unroll
            for (int j = 0; j < BW; j += 2) {
                dS[j] = fmaf(qi, dd[j], dS[j]);
                dS[j + 1] = fmaf(qi, dd[j + 1], dS[j + 1]);
                dq0 = fmaf(fmaf(ki, bt * e[j], Sb[j]), dd[j], dq0);
                dq1 = fmaf(fmaf(ki, bt * e[j + 1], Sb[j + 1]), dd[j + 1], dq1);
            }
            atomicAdd(a.dq + kq, dq0 + dq1);
            // S' = Sb + k u^T
            float x[BW];
#pragma unroll
            for (int j = 0; j < BW; ++j) x[j] = dS[j] * ki;
            column_sums<NWARP>(x, red, tot);
            float dk0 = 0.f, dk1 = 0.f, db0 = 0.f, db1 = 0.f, rg0 = 0.f, rg1 = 0.f;
#pragma unroll
            for (int j = 0; j < BW; j += 2) {
                const float du0 = tot[j], dp0 = -bt * du0, du1 = tot[j + 1], dp1 = -bt * du1;
                dk0 = fmaf(dS[j], bt * e[j], dk0);           // dS u
                dk1 = fmaf(dS[j + 1], bt * e[j + 1], dk1);
                dk0 = fmaf(Sb[j], dp0, dk0);                 // Sb dp
                dk1 = fmaf(Sb[j + 1], dp1, dk1);
                db0 = fmaf(du0, e[j], db0);
                db1 = fmaf(du1, e[j + 1], db1);
                const float dSb0 = fmaf(ki, dp0, dS[j]), dSb1 = fmaf(ki, dp1, dS[j + 1]);
                rg0 = fmaf(dSb0, Sb[j], rg0);
                rg1 = fmaf(dSb1, Sb[j + 1], rg1);
                dS[j] = ai * dSb0;
                dS[j + 1] = ai * dSb1;
            }
            atomicAdd(a.dk + kq, dk0 + dk1);
            if (i == 0) atomicAdd(a.dbeta + tv * a.Hv + h, db0 + db1);
            if (i < BW) a.dv[(tv * a.Hv + h) * Dv + j0 + i] = bt * tot[i];
            float rg = rg0 + rg1;
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

template <typename TIn, int GATE, int DK>
constexpr size_t bwd_smem()
{
    return 2 * sizeof(Stage<TIn, GATE, DK>) +
           ((size_t)BLK * DK * SBLD + BLK * BW + (DK / 32) * BW + BW) * sizeof(float);
}

template <typename TIn, int GATE, int DK>
cudaError_t launch_t(const BwdArgs &a, void *ws, cudaStream_t st)
{
    const dim3 grid(a.Dv / BW, a.B * a.Hv);
    float *ck = reinterpret_cast<float *>(ws);
    bwd_ckpt_kernel<TIn, GATE, DK><<<grid, DK, 0, st>>>(a, ck);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    constexpr size_t smem = bwd_smem<TIn, GATE, DK>();
    e = cudaFuncSetAttribute(bwd_kernel<TIn, GATE, DK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bwd_kernel<TIn, GATE, DK><<<grid, DK, smem, st>>>(a, ck);
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
