// Single-token decode step of the gated delta rule (bandwidth-bound; CUDA cores).
//
// Per (batch row, value head) the step reads the fp32 state S [Dk][Dv] once
// and writes it once:
//   S' = diag(exp(g)) S            decay (scalar per head or per key channel)
//   u  = beta (v - S'^T k)         memory prediction and delta correction
//   S  = S' + k u^T
//   o  = S^T q = S'^T q + (q.k) u  recurrent read after the update
// (Frontier-model atlas, item 03: state decay, memory prediction, delta
// correction, recurrent read; NextTransformer "Source notes", "Linear
// attention", rows gdn/kda: decay before the delta update, readout y = q^T S.)
//
// One CTA of 8 warps owns one (b, h). Warp w holds rows [w*Dk/8, (w+1)*Dk/8)
// and lane l columns [l*Dv/32, (l+1)*Dv/32): a warp reads whole 512-byte rows
// with 128-bit loads, the reductions over Dk are per-thread sums followed by
// one 8-way shared-memory reduction, and the state never leaves registers
// between its load and its store.
#include "common.cuh"
#include "kernels.h"

namespace gdr {

template <int CL> struct Vec;
template <> struct Vec<4> { using T = float4; };
template <> struct Vec<2> { using T = float2; };

template <typename TIn, typename TOut, int DK, int DV, int GATE>
__global__ void __launch_bounds__(256) decode_kernel(DecodeArgs a)
{
    constexpr int NW = 8, RW = DK / NW, CL = DV / 32;
    using V = typename Vec<CL>::T;
    __shared__ float qs[DK], ks[DK], ds[DK], vs[DV], us[DV];
    __shared__ float red_k[NW][DV], red_q[NW][DV];
    __shared__ float qk_s;

    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
    const long bh = blockIdx.x;
    const int b = (int)(bh / a.Hv), h = (int)(bh % a.Hv);
    const int hk = h / (a.Hv / a.Hk);
    const TIn *q = (const TIn *)a.q + ((long)b * a.Hk + hk) * DK;
    const TIn *k = (const TIn *)a.k + ((long)b * a.Hk + hk) * DK;
    const TIn *v = (const TIn *)a.v + bh * DV;
    const float beta = a.beta[bh];

    if (tid < DK) {
        qs[tid] = In<TIn>::load(q + tid);
        ks[tid] = In<TIn>::load(k + tid);
        ds[tid] = GATE == 0 ? expf(a.g[bh]) : expf(a.g[bh * DK + tid]);
    }
    if (tid < DV) vs[tid] = In<TIn>::load(v + tid);

    float *S = a.state + bh * (long)DK * DV;
    float s[RW][CL];
#pragma unroll
    for (int i = 0; i < RW; ++i) {
        V x = __ldcs(reinterpret_cast<const V *>(S + (long)(w * RW + i) * DV) + l);
        const float *xf = reinterpret_cast<const float *>(&x);
#pragma unroll
        for (int j = 0; j < CL; ++j) s[i][j] = xf[j];
    }
    __syncthreads();
    if (w == 0) {
        float acc = 0.f;
        for (int c = l; c < DK; c += 32) acc += qs[c] * ks[c];
#pragma unroll
        for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (l == 0) qk_s = acc;
    }
    float pk[CL], pq[CL];
#pragma unroll
    for (int j = 0; j < CL; ++j) pk[j] = pq[j] = 0.f;
#pragma unroll
    for (int i = 0; i < RW; ++i) {
        const int r = w * RW + i;
        const float d = ds[r], kr = ks[r], qr = qs[r];
#pragma unroll
        for (int j = 0; j < CL; ++j) {
            s[i][j] *= d;
            pk[j] += kr * s[i][j];
            pq[j] += qr * s[i][j];
        }
    }
#pragma unroll
    for (int j = 0; j < CL; ++j) {
        red_k[w][l * CL + j] = pk[j];
        red_q[w][l * CL + j] = pq[j];
    }
    __syncthreads();
    if (tid < DV) {
        float kS = 0.f, qS = 0.f;
#pragma unroll
        for (int ww = 0; ww < NW; ++ww) { kS += red_k[ww][tid]; qS += red_q[ww][tid]; }
        const float u = beta * (vs[tid] - kS);
        us[tid] = u;
        In<TOut>::store((TOut *)a.o + bh * DV + tid, qS + qk_s * u);
    }
    __syncthreads();
    float u[CL];
#pragma unroll
    for (int j = 0; j < CL; ++j) u[j] = us[l * CL + j];
#pragma unroll
    for (int i = 0; i < RW; ++i) {
        const float kr = ks[w * RW + i];
        V x;
        float *xf = reinterpret_cast<float *>(&x);
#pragma unroll
        for (int j = 0; j < CL; ++j) xf[j] = s[i][j] + kr * u[j];
        __stcs(reinterpret_cast<V *>(S + (long)(w * RW + i) * DV) + l, x);
    }
}

template <typename TIn, typename TOut, int DK, int DV>
static cudaError_t launch_decode_t(const DecodeArgs &a, cudaStream_t st)
{
    dim3 grid((unsigned)((long)a.B * a.Hv));
    if (a.gate_mode == 0) decode_kernel<TIn, TOut, DK, DV, 0><<<grid, 256, 0, st>>>(a);
    else decode_kernel<TIn, TOut, DK, DV, 1><<<grid, 256, 0, st>>>(a);
    return cudaGetLastError();
}

template <typename TIn, typename TOut>
static cudaError_t launch_decode_d(const DecodeArgs &a, cudaStream_t st)
{
    if (a.Dk == 128 && a.Dv == 128) return launch_decode_t<TIn, TOut, 128, 128>(a, st);
    if (a.Dk == 128 && a.Dv == 64) return launch_decode_t<TIn, TOut, 128, 64>(a, st);
    if (a.Dk == 64 && a.Dv == 128) return launch_decode_t<TIn, TOut, 64, 128>(a, st);
    return launch_decode_t<TIn, TOut, 64, 64>(a, st);
}

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t st)
{
    if (!in_bf16(a.dtype)) return launch_decode_d<float, float>(a, st);
    return out_f32(a.dtype) ? launch_decode_d<__nv_bfloat16, float>(a, st)
                            : launch_decode_d<__nv_bfloat16, __nv_bfloat16>(a, st);
}

}  // namespace gdr
