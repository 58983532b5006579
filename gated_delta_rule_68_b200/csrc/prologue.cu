// The layer's elementwise stages around the recurrence: the short causal
// convolution with SiLU on the q/k/v projections, and the gated RMSNorm on the
// output (NextTransformer "Source notes", section "Linear attention", rows
// deltanet, kda and gdn; "Backend and numerical limits"; Atlas entry 03, a
// four-token causal convolution). Both are HBM-bound streams: every input
// element is read once and every output element written once.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"

namespace gdr {
namespace {

constexpr int CONV_W = 4;     // taps; tap CONV_W - 1 sits on the current token
constexpr int CONV_RUN = 8;   // tokens loaded together
constexpr int CONV_TOK = 8;   // consecutive tokens per thread
constexpr int CONV_WS = 44;   // shared floats per 8-channel group: 32 taps, 8 biases, 4 pad (conflict-free)
constexpr int CONV_TPB = 256;

struct Vec8 { float v[8]; };

__device__ __forceinline__ Vec8 load8(const __nv_bfloat16 *p)
{
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
    Vec8 r;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        r.v[2 * i] = f.x;
        r.v[2 * i + 1] = f.y;
    }
    return r;
}
__device__ __forceinline__ Vec8 load8(const float *p)
{
    const float4 a = *reinterpret_cast<const float4 *>(p), b = *reinterpret_cast<const float4 *>(p + 4);
    Vec8 r = {{a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w}};
    return r;
}
__device__ __forceinline__ void store8(__nv_bfloat16 *p, const Vec8 &x)
{
    uint4 u;
    __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(x.v[2 * i], x.v[2 * i + 1]);
    *reinterpret_cast<uint4 *>(p) = u;
}
__device__ __forceinline__ void store8(float *p, const Vec8 &x)
{
    *reinterpret_cast<float4 *>(p) = make_float4(x.v[0], x.v[1], x.v[2], x.v[3]);
    *reinterpret_cast<float4 *>(p + 4) = make_float4(x.v[4], x.v[5], x.v[6], x.v[7]);
}
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ void from_f(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }
__device__ __forceinline__ void from_f(float *p, float x) { *p = x; }

__device__ __forceinline__ float silu(float y) { return __fdividef(y, 1.f + __expf(-y)); }

// Sequence n of the token axis: [s0, s1). Without cu_seqlens, sequence n is
// tokens n*T .. n*T + T - 1.
struct Seqs {
    const int *cu;
    int n, T;
    __device__ int start(int i) const { return cu ? cu[i] : i * T; }
};

// 8 channels of one token as loaded (bf16: one 16-byte word; fp32: two), unpacked on use.
template <typename T_> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
    uint4 u;
    __device__ void load(const __nv_bfloat16 *p) { u = *reinterpret_cast<const uint4 *>(p); }
    __device__ void gather(const __nv_bfloat16 *p, int stride)   // p[0], p[stride], ..., or zeros
    {
        __nv_bfloat16 *e = reinterpret_cast<__nv_bfloat16 *>(&u);
#pragma unroll
        for (int i = 0; i < 8; ++i) e[i] = p ? p[i * stride] : __float2bfloat16_rn(0.f);
    }
    __device__ __nv_bfloat16 raw(int i) const { return reinterpret_cast<const __nv_bfloat16 *>(&u)[i]; }
    __device__ float get(int i) const
    {
        const __nv_bfloat162 h = reinterpret_cast<const __nv_bfloat162 *>(&u)[i >> 1];
        return (i & 1) ? __high2float(h) : __low2float(h);
    }
};
template <> struct Raw8<float> {
    float4 a, b;
    __device__ void load(const float *p)
    {
        a = *reinterpret_cast<const float4 *>(p);
        b = *reinterpret_cast<const float4 *>(p + 4);
    }
    __device__ void gather(const float *p, int stride)
    {
        a = p ? make_float4(p[0], p[stride], p[2 * stride], p[3 * stride]) : make_float4(0.f, 0.f, 0.f, 0.f);
        b = p ? make_float4(p[4 * stride], p[5 * stride], p[6 * stride], p[7 * stride]) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __device__ float raw(int i) const { return get(i); }
    __device__ float get(int i) const
    {
        const float4 &q = i < 4 ? a : b;
        const int j = i & 3;
        return j == 0 ? q.x : j == 1 ? q.y : j == 2 ? q.z : q.w;
    }
};

// Thread (span, group): channels 8 group .. 8 group + 7 of CONV_TOK consecutive
// tokens of the flattened token axis, in runs of CONV_RUN. A run's inputs are
// loaded first (all loads in flight together), together with the CONV_W - 1
// before it (for later runs, the previous run's tail, already in registers);
// the taps then walk the run in registers. At a sequence's first token the
// history comes from state_in (or is zero).
template <typename T_>
__global__ void __launch_bounds__(CONV_TPB)
conv_silu_kernel(const T_ *__restrict__ x, const float *__restrict__ w, const float *__restrict__ bias,
                 const T_ *__restrict__ state_in, T_ *__restrict__ state_out, T_ *__restrict__ y, Seqs sq,
                 long rows, int Ch)
{
    constexpr int H = CONV_W - 1;
    // Block: 32 channel groups (one per lane) x CONV_TPB / 32 runs of CONV_TOK tokens
    // (one per warp); the 32 groups' taps and biases are staged once, coalesced.
    __shared__ __align__(16) float sw[32 * CONV_WS];
    const int ngroups = Ch / 8, gblocks = (ngroups + 31) / 32;
    const int gb = (int)(blockIdx.x % gblocks), lane = threadIdx.x & 31;
    const long rb = blockIdx.x / gblocks;
    const int grp = gb * 32 + lane;
    const long tb = (rb * (CONV_TPB / 32) + (threadIdx.x >> 5)) * CONV_TOK;
    const int c0 = 8 * grp;
    const bool active = grp < ngroups && tb < rows;
    Raw8<T_> xr[H + CONV_RUN];   // tokens t0 - H .. t0 + RUN - 1 of the current run (addresses clamped)
    if (active) {   // the first run's loads go out before the taps are staged
#pragma unroll
        for (int i = 0; i < H; ++i) xr[i].load(x + (size_t)max(tb - H + i, 0L) * Ch + c0);
#pragma unroll
        for (int i = 0; i < CONV_RUN; ++i) xr[H + i].load(x + (size_t)min(tb + i, rows - 1) * Ch + c0);
    }
    {
        const int slot = threadIdx.x >> 3, ch = threadIdx.x & 7, gg = gb * 32 + slot;   // 256 threads: 32 x 8
        if (gg < ngroups) {
            *reinterpret_cast<float4 *>(sw + slot * CONV_WS + ch * 4) =
                *reinterpret_cast<const float4 *>(w + ((size_t)gg * 8 + ch) * CONV_W);
            sw[slot * CONV_WS + 32 + ch] = bias ? bias[(size_t)gg * 8 + ch] : 0.f;
        }
    }
    __syncthreads();
    if (!active) return;
    float wt[8][CONV_W], bs[8];
    {
        const float *ws = sw + lane * CONV_WS;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 q = *reinterpret_cast<const float4 *>(ws + i * 4);
            wt[i][0] = q.x; wt[i][1] = q.y; wt[i][2] = q.z; wt[i][3] = q.w;
            bs[i] = ws[32 + i];
        }
    }
    // the sequence holding tb: the last n with start(n) <= tb (empty sequences skipped)
    int lo = 0, hi = sq.n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (sq.start(mid) <= tb) lo = mid; else hi = mid - 1;
    }
    int n = lo;
    long s0 = sq.start(n), s1 = sq.start(n + 1);
#pragma unroll 1
    for (long t0 = tb; t0 < min(tb + CONV_TOK, rows); t0 += CONV_RUN) {
        const int nt = (int)min((long)CONV_RUN, rows - t0);
        if (t0 != tb) {
#pragma unroll
            for (int i = 0; i < CONV_RUN; ++i) xr[H + i].load(x + (size_t)min(t0 + i, rows - 1) * Ch + c0);
        }
        // The taps of token t0 + u read xr[u .. u + H]. Where those history slots precede
        // the sequence's first token they take state_in (or zero) instead: the sequence's
        // virtual axis is [state_in (oldest first) ; x[s0] ; x[s0 + 1] ; ...].
        auto fix_history = [&](int u) {   // u a compile-time index
#pragma unroll
            for (int j = 0; j < H; ++j) {
                const long vt = t0 + u - s0 + j;
                if (vt < H) xr[u + j].gather(state_in ? state_in + ((size_t)n * Ch + c0) * H + vt : nullptr, H);
            }
        };
        if (t0 == tb) fix_history(0);
#pragma unroll
        for (int u = 0; u < CONV_RUN; ++u) {
            if (u >= nt) break;
            const long t = t0 + u;
            while (t >= s1) {   // next sequence (skipping empty ones)
                ++n;
                s0 = s1;
                s1 = sq.start(n + 1);
                if (t < s1) fix_history(u);
            }
            Vec8 o;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float acc = bs[i];
#pragma unroll
                for (int j = 0; j <= H; ++j) acc = fmaf(wt[i][j], xr[u + j].get(i), acc);
                o.v[i] = silu(acc);
            }
            store8(y + (size_t)t * Ch + c0, o);
            if (state_out && t == s1 - 1) {   // the sequence's last H inputs, as given
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int j = 0; j < H; ++j) state_out[((size_t)n * Ch + c0 + i) * H + j] = xr[u + 1 + j].raw(i);
            }
        }
#pragma unroll
        for (int i = 0; i < H; ++i) xr[i] = xr[CONV_RUN + i];   // the next run's halo
    }
}

// Sequences with no tokens pass their state through (zero without state_in).
template <typename T_>
__global__ void conv_state_empty_kernel(const T_ *__restrict__ state_in, T_ *__restrict__ state_out, Seqs sq,
                                        int Ch)
{
    const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
    const long per = (long)Ch * (CONV_W - 1);
    if (i >= (long)sq.n * per) return;
    const int n = (int)(i / per);
    if (sq.start(n + 1) != sq.start(n)) return;
    state_out[i] = state_in ? state_in[i] : T_(0.f);
}

// One warp per row of D = 32 * PER elements; lane l owns elements PER l .. PER l + PER - 1.
template <typename T_, int PER> struct RowVec;
template <> struct RowVec<__nv_bfloat16, 4> {
    static __device__ void load(const __nv_bfloat16 *p, float *v)
    {
        const uint2 u = *reinterpret_cast<const uint2 *>(p);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
        v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
    }
    static __device__ void store(__nv_bfloat16 *p, const float *v)
    {
        const __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
        uint2 u;
        u.x = *reinterpret_cast<const uint32_t *>(&a);
        u.y = *reinterpret_cast<const uint32_t *>(&b);
        *reinterpret_cast<uint2 *>(p) = u;
    }
};
template <> struct RowVec<__nv_bfloat16, 2> {
    static __device__ void load(const __nv_bfloat16 *p, float *v)
    {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
        v[0] = a.x; v[1] = a.y;
    }
    static __device__ void store(__nv_bfloat16 *p, const float *v)
    {
        *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(v[0], v[1]);
    }
};
template <> struct RowVec<float, 4> {
    static __device__ void load(const float *p, float *v)
    {
        const float4 a = *reinterpret_cast<const float4 *>(p);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    }
    static __device__ void store(float *p, const float *v)
    {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
};
template <> struct RowVec<float, 2> {
    static __device__ void load(const float *p, float *v)
    {
        const float2 a = *reinterpret_cast<const float2 *>(p);
        v[0] = a.x; v[1] = a.y;
    }
    static __device__ void store(float *p, const float *v) { *reinterpret_cast<float2 *>(p) = make_float2(v[0], v[1]); }
};

template <typename T_, int PER>
__global__ void __launch_bounds__(256)
rmsnorm_gated_kernel(const T_ *__restrict__ o, const T_ *__restrict__ z, const float *__restrict__ wt,
                     T_ *__restrict__ y, long rows, float eps)
{
    const long row = (long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    constexpr int D = 32 * PER;
    const size_t base = (size_t)row * D + lane * PER;
    float ov[PER], zv[PER];
    RowVec<T_, PER>::load(o + base, ov);
    RowVec<T_, PER>::load(z + base, zv);
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) ss = fmaf(ov[i], ov[i], ss);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float rstd = rsqrtf(ss / D + eps);
#pragma unroll
    for (int i = 0; i < PER; ++i) ov[i] = ov[i] * rstd * wt[lane * PER + i] * silu(zv[i]);
    RowVec<T_, PER>::store(y + base, ov);
}

template <typename T_>
cudaError_t conv_t(const ConvArgs &a, cudaStream_t st)
{
    const Seqs sq{a.cu_seqlens, a.nseq, a.T};
    const long rows = a.rows;
    if (rows > 0) {
        const long runs = (rows + CONV_TOK - 1) / CONV_TOK, per_block = CONV_TPB / 32;
        const long blocks = ((a.Ch / 8 + 31) / 32) * ((runs + per_block - 1) / per_block);
        conv_silu_kernel<T_><<<(unsigned)blocks, CONV_TPB, 0, st>>>(
            static_cast<const T_ *>(a.x), a.w, a.bias, static_cast<const T_ *>(a.state_in),
            static_cast<T_ *>(a.state_out), static_cast<T_ *>(a.y), sq, rows, a.Ch);
    }
    if (a.state_out && (a.cu_seqlens || rows == 0)) {
        const long n = (long)a.nseq * a.Ch * (CONV_W - 1);
        if (n > 0)
            conv_state_empty_kernel<T_><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
                static_cast<const T_ *>(a.state_in), static_cast<T_ *>(a.state_out), sq, a.Ch);
    }
    return cudaGetLastError();
}

template <typename T_>
cudaError_t norm_t(const NormArgs &a, cudaStream_t st)
{
    const unsigned grid = (unsigned)((a.rows + 7) / 8);
    if (a.D == 128)
        rmsnorm_gated_kernel<T_, 4><<<grid, 256, 0, st>>>(static_cast<const T_ *>(a.o), static_cast<const T_ *>(a.z),
                                                          a.w, static_cast<T_ *>(a.y), a.rows, a.eps);
    else
        rmsnorm_gated_kernel<T_, 2><<<grid, 256, 0, st>>>(static_cast<const T_ *>(a.o), static_cast<const T_ *>(a.z),
                                                          a.w, static_cast<T_ *>(a.y), a.rows, a.eps);
    return cudaGetLastError();
}

}  // namespace

int conv_launches(const ConvArgs &a)
{
    return (a.rows > 0 ? 1 : 0) + ((a.state_out && (a.cu_seqlens || a.rows == 0) && a.nseq > 0) ? 1 : 0);
}

cudaError_t launch_conv_silu(const ConvArgs &a, cudaStream_t st)
{
    return a.fp32 ? conv_t<float>(a, st) : conv_t<__nv_bfloat16>(a, st);
}

cudaError_t launch_rmsnorm_gated(const NormArgs &a, cudaStream_t st)
{
    if (a.rows <= 0) return cudaSuccess;
    return a.fp32 ? norm_t<float>(a, st) : norm_t<__nv_bfloat16>(a, st);
}

}  // namespace gdr
