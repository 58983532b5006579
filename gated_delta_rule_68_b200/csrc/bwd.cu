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
// The columns of S (value channels) evolve independently, so one CTA of four warps
// takes a (batch row, value head, 16-column slice): each warp owns 4 columns over all
// Dk rows, each lane Dk / 32 consecutive rows of them. The sums over rows (p, du) are
// then sums within a warp (9 shuffles for the 4 columns), and only the sums over
// columns (dq, dk, a per-channel dg) cross warps, once per reverse step through
// shared memory. Two kernels:
//   1. a forward pass that stores the state before every 4th token (workspace, in
//      the kernels' own per-thread order);
//   2. a reverse pass that, per block of 4 tokens, recomputes the decayed states
//      Sb from the block's checkpoint into shared memory, then runs the 4 reverse
//      steps. dv and dh0 belong to one slice and are stored; dq and dk (summed
//      over slices and over the value heads that share a key head), dbeta and dg
//      are accumulated with atomics into zeroed outputs.
// Both kernels stage a block's inputs (k, q, the slice's v and do columns, g, beta)
// in shared memory with asynchronous copies one block ahead, so no token waits on a
// global load.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace gdr {
namespace {

constexpr int NT = 128;     // threads per CTA: four warps
constexpr int CW = 4;       // value columns per warp
constexpr int BW = 16;      // value columns per CTA
constexpr int BLK = 4;      // tokens between checkpoints (50 KB of shared memory: four CTAs per SM)
constexpr unsigned FULL = 0xffffffffu;

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
    for (int c = tid; c < n * CR; c += NT) {
        const int tt = c / CR, x = (c % CR) * E;
        const size_t off = (((size_t)b * a.T + t0 + tt) * a.Hk + hk) * DK + x;
        cp16(&s.k[tt][x], k + off);
        if (REV) cp16(&s.q[tt][x], q + off);
    }
    for (int c = tid; c < n * CV; c += NT) {
        const int tt = c / CV, x = (c % CV) * E;
        const size_t off = (((size_t)b * a.T + t0 + tt) * a.Hv + h) * a.Dv + j0 + x;
        cp16(&s.v[tt][x], v + off);
        if (REV) cp16(&s.d[tt][x], d + off);
    }
    if (GATE) {
        for (int c = tid; c < n * (DK / 4); c += NT) {
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

// N consecutive values as fp32 (N = 2 or 4; a bf16 is the high half of its fp32 value).
template <int N>
__device__ __forceinline__ void load_n(const float *p, float x[N])
{
    if (N == 4) {
        const float4 f = *reinterpret_cast<const float4 *>(p);
        x[0] = f.x, x[1] = f.y, x[2] = f.z, x[3] = f.w;
    } else {
        const float2 f = *reinterpret_cast<const float2 *>(p);
        x[0] = f.x, x[1] = f.y;
    }
}
template <int N>
__device__ __forceinline__ void load_n(const __nv_bfloat16 *p, float x[N])
{
    if (N == 4) {
        const uint2 u = *reinterpret_cast<const uint2 *>(p);
        x[0] = __uint_as_float(u.x << 16), x[1] = __uint_as_float(u.x & 0xffff0000u);
        x[2] = __uint_as_float(u.y << 16), x[3] = __uint_as_float(u.y & 0xffff0000u);
    } else {
        const uint32_t u = *reinterpret_cast<const uint32_t *>(p);
        x[0] = __uint_as_float(u << 16), x[1] = __uint_as_float(u & 0xffff0000u);
    }
}
template <int N>
__device__ __forceinline__ void store_n(float *p, const float x[N])
{
    if (N == 4) *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
    else *reinterpret_cast<float2 *>(p) = make_float2(x[0], x[1]);
}

// Totals over the warp's Dk rows of x[r][c] * y[r] for its 4 columns, returned to every
// lane: the lane's rows first, then a reduce-scatter across lanes (after the xor-1 and xor-2
// exchanges lane l holds column 2 (l & 1) + (l >> 1 & 1)), a sum over the other lanes,
// and an all-gather back to 4 columns.
template <int R>
__device__ __forceinline__ void col_sums(const float x[R][CW], const float y[R], float t[CW])
{
    float v[CW];
#pragma unroll
    for (int c = 0; c < CW; ++c) {
        v[c] = x[0][c] * y[0];
#pragma unroll
        for (int r = 1; r < R; ++r) v[c] = fmaf(x[r][c], y[r], v[c]);
    }
    const int lane = threadIdx.x & 31;
    const bool b0 = lane & 1, b1 = lane & 2;
    const float a0 = (b0 ? v[2] : v[0]) + __shfl_xor_sync(FULL, b0 ? v[0] : v[2], 1);
    const float a1 = (b0 ? v[3] : v[1]) + __shfl_xor_sync(FULL, b0 ? v[1] : v[3], 1);
    float s = (b1 ? a1 : a0) + __shfl_xor_sync(FULL, b1 ? a0 : a1, 2);
    s += __shfl_xor_sync(FULL, s, 4);
    s += __shfl_xor_sync(FULL, s, 8);
    s += __shfl_xor_sync(FULL, s, 16);
    const float o = __shfl_xor_sync(FULL, s, 2);
    const float u0 = b1 ? o : s, u1 = b1 ? s : o;               // columns 2 b0, 2 b0 + 1
    const float p0 = __shfl_xor_sync(FULL, u0, 1), p1 = __shfl_xor_sync(FULL, u1, 1);
    t[0] = b0 ? p0 : u0;
    t[1] = b0 ? p1 : u1;
    t[2] = b0 ? u0 : p0;
    t[3] = b0 ? u1 : p1;
}

// The gate factors a_t of the lane's rows.
template <typename TIn, int GATE, int DK>
__device__ __forceinline__ void gate_rows(const Stage<TIn, GATE, DK> &s, int tt, int row0, float ar[DK / 32])
{
    constexpr int R = DK / 32;
    if (GATE) {
        load_n<R>(&s.g[tt][row0], ar);
#pragma unroll
        for (int r = 0; r < R; ++r) ar[r] = __expf(ar[r]);
    } else {
        const float a0 = __expf(s.g[tt][0]);
#pragma unroll
        for (int r = 0; r < R; ++r) ar[r] = a0;
    }
}

// Offset (floats) of a thread's checkpoint: [unit][block][slice][thread][R rows x 4 columns].
template <int DK>
__device__ __forceinline__ size_t ck_off(int unit, int m, int M, int slice, int nslice)
{
    return (((size_t)unit * M + m) * nslice + slice) * ((size_t)DK * BW) + (size_t)threadIdx.x * (DK / 32) * CW;
}

template <typename TIn, int GATE, int DK>
__global__ void __launch_bounds__(NT)
bwd_ckpt_kernel(BwdArgs a, float *ck)
{
    constexpr int R = DK / 32;
    __shared__ Stage<TIn, GATE, DK> st[2];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int slice = blockIdx.x, j0 = slice * BW, unit = blockIdx.y;
    const int b = unit / a.Hv, h = unit % a.Hv, hk = h / (a.Hv / a.Hk);
    const int T = a.T, M = (T + BLK - 1) / BLK, Dv = a.Dv;
    const int row0 = R * lane, col0 = j0 + CW * w;
    if (M > 0) stage_issue<TIn, GATE, DK, false>(st[0], a, b, h, hk, j0, 0, min(BLK, T));
    float S[R][CW];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        if (a.h0) load_n<CW>(a.h0 + ((size_t)unit * DK + row0 + r) * Dv + col0, S[r]);
        else S[r][0] = S[r][1] = S[r][2] = S[r][3] = 0.f;
    }
    for (int m = 0; m < M; ++m) {
        const int t0 = m * BLK, n = min(BLK, T - t0);
        float *dst = ck + ck_off<DK>(unit, m, M, slice, gridDim.x);
#pragma unroll
        for (int r = 0; r < R; ++r) store_n<CW>(dst + r * CW, S[r]);
        cp_wait_all();
        __syncthreads();   // block m staged; every thread is done with block m - 1's buffer
        if (m + 1 < M)
            stage_issue<TIn, GATE, DK, false>(st[(m + 1) & 1], a, b, h, hk, j0, t0 + BLK, min(BLK, T - t0 - BLK));
        const Stage<TIn, GATE, DK> &s = st[m & 1];
        for (int tt = 0; tt < n; ++tt) {
            float kr[R], ar[R], vc[CW], p[CW];
            load_n<R>(&s.k[tt][row0], kr);
            gate_rows(s, tt, row0, ar);
            const float bt = s.beta[tt];
            load_n<CW>(&s.v[tt][CW * w], vc);
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int c = 0; c < CW; ++c) S[r][c] *= ar[r];
            col_sums<R>(S, kr, p);
#pragma unroll
            for (int c = 0; c < CW; ++c) p[c] = bt * (vc[c] - p[c]);
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int c = 0; c < CW; ++c) S[r][c] = fmaf(kr[r], p[c], S[r][c]);
        }
    }
}

// Shared memory of the reverse kernel (byte offsets; every region 16-byte aligned).
template <typename TIn, int GATE, int DK>
struct RevSmem {
    static constexpr int NV = (DK / 32) * CW;                             // state values per thread
    static constexpr size_t sbs = 2 * sizeof(Stage<TIn, GATE, DK>);       // [BLK][NT][NV] Sb, per thread
    static constexpr size_t es = sbs + (size_t)BLK * NT * NV * 4;         // [BLK][BW] e of the block's tokens
    static constexpr size_t rp = es + (size_t)BLK * BW * 4;               // [2][3][4][DK] row partials
    static constexpr size_t rs = rp + (size_t)2 * 3 * 4 * DK * 4;         // [2][2][4] warp totals
    static constexpr size_t bytes = rs + 2 * 2 * 4 * 4;
};

template <typename TIn, int GATE, int DK>
__global__ void __launch_bounds__(NT)
bwd_kernel(BwdArgs a, const float *ck)
{
    constexpr int R = DK / 32, NV = R * CW;
    using L = RevSmem<TIn, GATE, DK>;
    extern __shared__ __align__(16) unsigned char smraw[];
    Stage<TIn, GATE, DK> *st = reinterpret_cast<Stage<TIn, GATE, DK> *>(smraw);
    float *Sbs = reinterpret_cast<float *>(smraw + L::sbs);
    float *es = reinterpret_cast<float *>(smraw + L::es);
    float *rp = reinterpret_cast<float *>(smraw + L::rp);
    float *rs = reinterpret_cast<float *>(smraw + L::rs);
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int slice = blockIdx.x, j0 = slice * BW, unit = blockIdx.y;
    const int b = unit / a.Hv, h = unit % a.Hv, hk = h / (a.Hv / a.Hk);
    const int T = a.T, M = (T + BLK - 1) / BLK, Dv = a.Dv;
    const int row0 = R * lane, col0 = j0 + CW * w;
    // a thread's Sb rows sit in 16-byte slots r ^ swz, so that the eight lanes of each
    // 128-byte phase of a warp's access hit distinct banks
    const int swz = (lane / (8 / R)) & (R - 1);
    if (M > 0) stage_issue<TIn, GATE, DK, true>(st[(M - 1) & 1], a, b, h, hk, j0, (M - 1) * BLK, T - (M - 1) * BLK);
    float dS[R][CW];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        if (a.dhT) load_n<CW>(a.dhT + ((size_t)unit * DK + row0 + r) * Dv + col0, dS[r]);
        else dS[r][0] = dS[r][1] = dS[r][2] = dS[r][3] = 0.f;
    }
    for (int m = M - 1; m >= 0; --m) {
        const int t0 = m * BLK, n = min(BLK, T - t0);
        float S[R][CW];
        {
            const float *src = ck + ck_off<DK>(unit, m, M, slice, gridDim.x);
#pragma unroll
            for (int r = 0; r < R; ++r) load_n<CW>(src + r * CW, S[r]);
        }
        cp_wait_all();
        __syncthreads();   // block m staged; every thread is done with block m + 1 (buffer, es)
        if (m > 0) stage_issue<TIn, GATE, DK, true>(st[(m - 1) & 1], a, b, h, hk, j0, t0 - BLK, BLK);
        const Stage<TIn, GATE, DK> &s = st[m & 1];
        // recompute the block's decayed states Sb and e from its checkpoint
        for (int tt = 0; tt < n; ++tt) {
            float kr[R], ar[R], vc[CW], p[CW];
            load_n<R>(&s.k[tt][row0], kr);
            gate_rows(s, tt, row0, ar);
            const float bt = s.beta[tt];
            load_n<CW>(&s.v[tt][CW * w], vc);
            float *sb = Sbs + ((size_t)tt * NT + tid) * NV;
#pragma unroll
            for (int r = 0; r < R; ++r) {
#pragma unroll
                for (int c = 0; c < CW; ++c) S[r][c] *= ar[r];
                store_n<CW>(sb + (r ^ swz) * CW, S[r]);
            }
            col_sums<R>(S, kr, p);
#pragma unroll
            for (int c = 0; c < CW; ++c) p[c] = vc[c] - p[c];        // e
            if (lane == 0) store_n<CW>(es + tt * BW + CW * w, p);
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int c = 0; c < CW; ++c) S[r][c] = fmaf(kr[r] * bt, p[c], S[r][c]);
        }
        __syncwarp();      // e of the warp's columns visible to its lanes
        // reverse the block's steps
        for (int tt = n - 1; tt >= 0; --tt) {
            const int t = t0 + tt, par = t & 1;
            const size_t tv = (size_t)b * T + t;
            float kr[R], qr[R], ar[R], dd[CW], e[CW], Sb[R][CW];
            load_n<R>(&s.k[tt][row0], kr);
            load_n<R>(&s.q[tt][row0], qr);
            gate_rows(s, tt, row0, ar);
            const float bt = s.beta[tt];
            load_n<CW>(&s.d[tt][CW * w], dd);
            load_n<CW>(es + tt * BW + CW * w, e);
            {
                const float *sb = Sbs + ((size_t)tt * NT + tid) * NV;
#pragma unroll
                for (int r = 0; r < R; ++r) load_n<CW>(sb + (r ^ swz) * CW, Sb[r]);
            }
            // o = S'^T q with S' = Sb + k (beta e)^T: dS += q do^T, and
            // dq = S' do = Sb do + k beta (e . do)
            float dq[R], du[CW], ed = 0.f;
#pragma unroll
            for (int c = 0; c < CW; ++c) ed = fmaf(e[c], dd[c], ed);
            ed *= bt;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                float acc = kr[r] * ed;
#pragma unroll
                for (int c = 0; c < CW; ++c) {
                    dS[r][c] = fmaf(qr[r], dd[c], dS[r][c]);
                    acc = fmaf(Sb[r][c], dd[c], acc);
                }
                dq[r] = acc;
            }
            col_sums<R>(dS, kr, du);
            float dk[R], rg[R], dp[CW], db = 0.f;
#pragma unroll
            for (int c = 0; c < CW; ++c) dp[c] = -bt * du[c], db = fmaf(du[c], e[c], db);
#pragma unroll
            for (int r = 0; r < R; ++r) {
                float k0 = 0.f, g0 = 0.f;
#pragma unroll
                for (int c = 0; c < CW; ++c) {
                    k0 = fmaf(dS[r][c], bt * e[c], k0);      // dS u
                    k0 = fmaf(Sb[r][c], dp[c], k0);          // Sb dp
                    const float dSb = fmaf(kr[r], dp[c], dS[r][c]);
                    g0 = fmaf(dSb, Sb[r][c], g0);
                    dS[r][c] = ar[r] * dSb;
                }
                dk[r] = k0, rg[r] = g0;
            }
            if (lane == 0) {
                const float dv4[CW] = {bt * du[0], bt * du[1], bt * du[2], bt * du[3]};
                store_n<CW>(a.dv + (tv * a.Hv + h) * Dv + col0, dv4);
            }
            // row partials of this warp's columns; buffers alternate with the token parity
            float *rpp = rp + (size_t)par * 3 * 4 * DK;
            store_n<R>(rpp + (0 * 4 + w) * DK + row0, dq);
            store_n<R>(rpp + (1 * 4 + w) * DK + row0, dk);
            if (GATE) {
                store_n<R>(rpp + (2 * 4 + w) * DK + row0, rg);
            } else {
                float gs = rg[0];
#pragma unroll
                for (int r = 1; r < R; ++r) gs += rg[r];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) gs += __shfl_xor_sync(FULL, gs, off);
                if (lane == 0) rs[(par * 2 + 1) * 4 + w] = gs;
            }
            if (lane == 0) rs[(par * 2 + 0) * 4 + w] = db;
            __syncthreads();   // every warp's partials written; the other parity's buffers were read
            if (tid < DK) {
                const size_t kq = (tv * a.Hk + hk) * DK + tid;
                const float *q0 = rpp, *q1 = rpp + 4 * DK;
                atomicAdd(a.dq + kq, (q0[tid] + q0[DK + tid]) + (q0[2 * DK + tid] + q0[3 * DK + tid]));
                atomicAdd(a.dk + kq, (q1[tid] + q1[DK + tid]) + (q1[2 * DK + tid] + q1[3 * DK + tid]));
                if (GATE) {
                    const float *q2 = rpp + 8 * DK;
                    atomicAdd(a.dg + (tv * a.Hv + h) * DK + tid,
                              (q2[tid] + q2[DK + tid]) + (q2[2 * DK + tid] + q2[3 * DK + tid]));
                }
            }
            if (tid == 0) {
                const float *r0 = rs + par * 2 * 4;
                atomicAdd(a.dbeta + tv * a.Hv + h, (r0[0] + r0[1]) + (r0[2] + r0[3]));
                if (!GATE) atomicAdd(a.dg + tv * a.Hv + h, (r0[4] + r0[5]) + (r0[6] + r0[7]));
            }
        }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) store_n<CW>(a.dh0 + ((size_t)unit * DK + row0 + r) * Dv + col0, dS[r]);
}

template <typename TIn, int GATE, int DK>
cudaError_t launch_t(const BwdArgs &a, void *ws, cudaStream_t st)
{
    const dim3 grid(a.Dv / BW, a.B * a.Hv);
    float *ck = reinterpret_cast<float *>(ws);
    bwd_ckpt_kernel<TIn, GATE, DK><<<grid, NT, 0, st>>>(a, ck);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    constexpr size_t smem = RevSmem<TIn, GATE, DK>::bytes;
    e = cudaFuncSetAttribute(bwd_kernel<TIn, GATE, DK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bwd_kernel<TIn, GATE, DK><<<grid, NT, smem, st>>>(a, ck);
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
