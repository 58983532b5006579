// Chunked backward of the gated delta rule on tensor cores (scalar gate, bf16 inputs,
// Dk = Dv = 128, chunks of 64 tokens).
//
// NextTransformer docs, "Source notes", "Linear attention": the gdn update and its
// first-order backward. The chunk's forward map is affine in the entering state S,
//     S_next = Gamma_C S + P S + R,     O = Qh S + Uh,
// so its adjoint is the transposed map,
//     dS = Gamma_C dS_next + P^T dS_next + Qh^T dO,
// and the gradients of the chunk's own inputs depend only on S, dS_next, dO and the
// chunk's inputs. Three passes:
//   1. the tcgen05 forward (chunk_tc.cu, its SAVE instance) stores, per chunk, the
//      entering state S^T, P, Qh^T and T = (I + A)^-1 in fp16;
//   2. bwdc_scan_kernel: per (batch row, value head), the chunks in reverse; dS^T is
//      carried in fp32 warp-MMA accumulators and stored per chunk (as dS_next of that
//      chunk) in fp16; the last one is dh0;
//   3. bwdc_chunk_kernel: one CTA per (unit, chunk), all chunks at once. With the
//      in-chunk decays D_ri = exp(G_r - G_i) (r >= i) and f = Gamma_C / Gamma:
//        W = T diag(beta Gamma) K,  U = T diag(beta) V,  U' = U - W S
//        dU' = M^T dO + diag(f) K dS_next,       M = tril(Q K^T * D)
//        dM = tril(dO U'^T),                     dQ = diag(Gamma) dO S^T + (dM * D) K
//        dK3 = diag(f) U' dS_next^T,             dW = -dU' S^T
//        dV = diag(beta) T^T dU',                dK1 = diag(Gamma beta) T^T dW + (dB * D) K
//        dT = dU' V^T diag(beta) + dW K^T diag(beta Gamma)
//        dA = strict tril(-T^T dT T^T),          dB = diag(beta) dA
//        dK2 = (dM * D)^T Q + (dB * D)^T K,      dK = dK1 + dK2 + dK3
//        dbeta = rowsum(V * T^T dU') + rowsum(Gamma K * T^T dW) + rowsum(dA * tril(K K^T * D, -1))
//        dG = rowsum((dK1 - dK2 - dK3) * K + dQ * Q), and its last row adds
//             sum(dK3 * K) + Gamma_C sum(dS_next * S); dg = reverse cumulative sum of dG.
//      Every factor is relative (at most 1), as in the forward.
// Products are warp-level mma.sync (fp16 operands, fp32 accumulation).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"
#include "mma_util.cuh"

namespace gdr {
namespace {

using namespace mmau;

constexpr int NT = 256;   // 8 warps

// The per-(unit, chunk) fp16 buffers of the three passes, in the caller's workspace.
struct BwdcWs {
    __half *s, *p, *qh, *t, *ds;   // S^T [Dv][Dk], P [Dk][Dk], Qh^T [Dk][64], T [64][64], dS_next^T [Dv][Dk]
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_h2f(float x, float y)
{
    const __half2 h = __floats2half2_rn(x, y);
    return *reinterpret_cast<const uint32_t *>(&h);
}
// 8 bf16 values at p, rewritten as fp16 in place.
__device__ __forceinline__ void bf16_to_fp16_16B(uint8_t *p)
{
    uint4 u = *reinterpret_cast<const uint4 *>(p);
    uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[k]));
        w[k] = pack_h2f(f.x, f.y);
    }
    *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}
__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}
__device__ __forceinline__ void hmul_frag(uint32_t &r, __half2 s)
{
    __half2 h = *reinterpret_cast<__half2 *>(&r);
    h = __hmul2(h, s);
    r = *reinterpret_cast<uint32_t *>(&h);
}

// acc[2 NP][4] += A (16 rows from r0, K = 16 KS) B (columns n0 .. n0 + 16 NP).
// A: row-major [m][k] (AT false) or stored transposed [k][m] (AT true);
// B: stored [n][k] (BT false) or [k][n] (BT true). ascale(af, j) may rescale the A
// fragment of k-step j in registers.
template <int KS, int NP, bool AT, bool BT, typename AS>
__device__ __forceinline__ void wgemm(float (*acc)[4], uint32_t aB, int lda, int r0, uint32_t bB, int ldb, int n0,
                                      int lane, AS ascale)
{
#pragma unroll
    for (int j = 0; j < KS; ++j) {
        uint32_t af[4];
        if (AT) ldsm_t(af, a_tr(aB, lda, r0, 16 * j, lane));
        else ldsm(af, a_rm(aB, lda, r0, 16 * j, lane));
        ascale(af, j);
#pragma unroll
        for (int np = 0; np < NP; ++np) {
            uint32_t bf[4];
            if (BT) ldsm_t(bf, b_kn(bB, ldb, n0 + 16 * np, 16 * j, lane));
            else ldsm(bf, b_nk(bB, ldb, n0 + 16 * np, 16 * j, lane));
            mma(acc[2 * np], af, bf[0], bf[1]);
            mma(acc[2 * np + 1], af, bf[2], bf[3]);
        }
    }
}
struct NoScale {
    __device__ __forceinline__ void operator()(uint32_t *, int) const {}
};
template <int N>
__device__ __forceinline__ void zero_acc(float (*acc)[4])
{
#pragma unroll
    for (int i = 0; i < N; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
}

// ------------------------------------------------------------------ pass 2: the reverse scan
constexpr uint32_t SB_P = 0;                                 // P [128][LDD] fp16
constexpr uint32_t SB_QH = D * LDD * 2;                      // Qh^T [128][LDC] fp16
constexpr uint32_t SB_DO = SB_QH + D * LDC * 2;              // dO [64][LDD] fp16
constexpr uint32_t SB_BUF = SB_DO + C * LDD * 2;
constexpr uint32_t SMEM_SCAN = 2 * SB_BUF;

// Warp w carries rows 16 w .. 16 w + 15 of dS^T ([Dv][Dk]) in acc[16][4]: tile nt holds
// columns 8 nt .. 8 nt + 7 (the m16n8 accumulator layout), so the fp16 A fragment of
// dS^T for k-step j is tiles 2 j and 2 j + 1 repacked.
__global__ void __launch_bounds__(NT, 1) bwdc_scan_kernel(BwdArgs a, BwdcWs ws)
{
    extern __shared__ __align__(128) uint8_t sm[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g8 = lane >> 2, t4 = lane & 3;
    const int unit = blockIdx.x, b = unit / a.Hv, h = unit % a.Hv;
    const int NC = (a.T + C - 1) / C;
    const uint32_t sb = smem_u32(sm);
    float acc[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int dv = 16 * warp + g8 + 8 * (e >> 1), dk = 8 * nt + 2 * t4 + (e & 1);
            acc[nt][e] = a.dhT ? a.dhT[((size_t)unit * D + dk) * D + dv] : 0.f;
        }
    auto load = [&](int c, int buf) {
        const uint32_t base = sb + buf * SB_BUF;
        const __half *P = ws.p + ((size_t)unit * NC + c) * D * D;
        for (int i = tid; i < D * 16; i += NT) {
            const int r = i >> 4, j = i & 15;
            cp_async16(base + SB_P + (r * LDD + 8 * j) * 2, P + r * D + 8 * j, 16);
        }
        const __half *Qh = ws.qh + ((size_t)unit * NC + c) * D * C;
        for (int i = tid; i < D * 8; i += NT) {
            const int r = i >> 3, j = i & 7;
            cp_async16(base + SB_QH + (r * LDC + 8 * j) * 2, Qh + r * C + 8 * j, 16);
        }
        const __nv_bfloat16 *dO = reinterpret_cast<const __nv_bfloat16 *>(a.dout);
        for (int i = tid; i < C * 16; i += NT) {
            const int r = i >> 4, j = i & 15, t = c * C + r;
            const bool ok = t < a.T;
            cp_async16(base + SB_DO + (r * LDD + 8 * j) * 2,
                       dO + (((size_t)b * a.T + (ok ? t : 0)) * a.Hv + h) * D + 8 * j, ok ? 16 : 0);
        }
        cp_async_commit();
    };
    load(NC - 1, 0);
    for (int c = NC - 1; c >= 0; --c) {
        const int buf = (NC - 1 - c) & 1;
        if (c > 0) {
            load(c - 1, buf ^ 1);
            cp_async_wait1();
        } else {
            cp_async_wait_all();
        }
        for (int i = tid; i < C * 16; i += NT) {   // this thread's dO copies, to fp16
            const int r = i >> 4, j = i & 15;
            bf16_to_fp16_16B(sm + buf * SB_BUF + SB_DO + (r * LDD + 8 * j) * 2);
        }
        float gsum = 0.f;   // Gamma_C of chunk c: exp of the sum of its g
        for (int r = lane; r < C; r += 32) {
            const int t = c * C + r;
            if (t < a.T) gsum += a.g[((size_t)b * a.T + t) * a.Hv + h];
        }
        const float gC = __expf(warp_sum(gsum));
        __syncthreads();
        // dS_next of chunk c, as fp16 [Dv][Dk]
        __half *dsg = ws.ds + ((size_t)unit * NC + c) * D * D;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
            const int r0 = 16 * warp + g8, col = 8 * nt + 2 * t4;
            *reinterpret_cast<uint32_t *>(dsg + (size_t)r0 * D + col) = pack_h2f(acc[nt][0], acc[nt][1]);
            *reinterpret_cast<uint32_t *>(dsg + (size_t)(r0 + 8) * D + col) = pack_h2f(acc[nt][2], acc[nt][3]);
        }
        uint32_t af[8][4];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            af[j][0] = pack_h2f(acc[2 * j][0], acc[2 * j][1]);
            af[j][1] = pack_h2f(acc[2 * j][2], acc[2 * j][3]);
            af[j][2] = pack_h2f(acc[2 * j + 1][0], acc[2 * j + 1][1]);
            af[j][3] = pack_h2f(acc[2 * j + 1][2], acc[2 * j + 1][3]);
        }
#pragma unroll
        for (int nt = 0; nt < 16; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nt][e] *= gC;
        const uint32_t base = sb + buf * SB_BUF;
        // dS^T P: B = P stored [dk_out = k][dk_in = n]
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                uint32_t bf[4];
                ldsm_t(bf, b_kn(base + SB_P, LDD, 16 * np, 16 * j, lane));
                mma(acc[2 * np], af[j], bf[0], bf[1]);
                mma(acc[2 * np + 1], af[j], bf[2], bf[3]);
            }
        // dO^T Qh: A = dO^T (dO stored [token][dv]), B = Qh stored as Qh^T [dk = n][token = k]
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t a4[4];
            ldsm_t(a4, a_tr(base + SB_DO, LDD, 16 * warp, 16 * j, lane));
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                uint32_t bf[4];
                ldsm(bf, b_nk(base + SB_QH, LDC, 16 * np, 16 * j, lane));
                mma(acc[2 * np], a4, bf[0], bf[1]);
                mma(acc[2 * np + 1], a4, bf[2], bf[3]);
            }
        }
        __syncthreads();   // the buffer is read before the next iteration's loads refill it
    }
#pragma unroll
    for (int nt = 0; nt < 16; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int dv = 16 * warp + g8 + 8 * (e >> 1), dk = 8 * nt + 2 * t4 + (e & 1);
            a.dh0[((size_t)unit * D + dk) * D + dv] = acc[nt][e];
        }
}

// ------------------------------------------------------------------ pass 3: per-chunk gradients
constexpr uint32_t SZ_DT = C * LDD * 2;     // [64][136] fp16
constexpr uint32_t SZ_ST = D * LDD * 2;     // [128][136] fp16
constexpr uint32_t SZ_CT = C * LDC * 2;     // [64][72] fp16
constexpr uint32_t OC_Q = 0, OC_K = SZ_DT, OC_V = 2 * SZ_DT, OC_DO = 3 * SZ_DT;
constexpr uint32_t OC_S = 4 * SZ_DT;          // S^T [dv][dk]; later X = T^T dT [64][LDC]
constexpr uint32_t OC_DS = OC_S + SZ_ST;      // dS_next^T [dv][dk]; later dW [64][LDD]
constexpr uint32_t OC_T = OC_DS + SZ_ST;      // T [64][LDC]
constexpr uint32_t OC_M = OC_T + SZ_CT;       // M, then dM * D [64][LDC]
constexpr uint32_t OC_W = OC_M + SZ_CT;       // W, then dU' [64][LDD]
constexpr uint32_t OC_U = OC_W + SZ_DT;       // U', then dT, then dB * D [64][LDC]
constexpr uint32_t OC_VEC = OC_U + SZ_DT;     // vectors: G, Gamma, beta, f, dG, dbeta [64] each; scalars
// vectors: G, Gamma, beta, f [64]; per column half of the warps, the row sums of dG and dbeta
// [2][64] each; per warp, sum(dK3 * K) and sum(dS_next * S) [8] each (summed in a fixed order,
// so that dg and dbeta repeat bit for bit)
constexpr int VG = 0, VGAM = 64, VBETA = 128, VF = 192, VDG = 256, VDB = 384, VT3 = 512, VSS = 520;
constexpr uint32_t SMEM_CHUNK = OC_VEC + (VSS + 8) * 4;
static_assert(SMEM_CHUNK <= 227 * 1024, "shared memory");

__global__ void __launch_bounds__(NT, 1) bwdc_chunk_kernel(BwdArgs a, BwdcWs ws)
{
    extern __shared__ __align__(128) uint8_t sm[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g8 = lane >> 2, t4 = lane & 3;
    const int rw = warp & 3, cw = warp >> 2, r0 = 16 * rw;
    const int NC = (a.T + C - 1) / C;
    const int unit = blockIdx.x / NC, c = blockIdx.x % NC;
    const int b = unit / a.Hv, h = unit % a.Hv, hk = h / (a.Hv / a.Hk);
    const uint32_t sb = smem_u32(sm);
    float *vec = reinterpret_cast<float *>(sm + OC_VEC);
    const size_t cu = (size_t)unit * NC + c;

    // ---- loads: q, k (key head), v, dO (value head) as bf16, rows past T zero; S^T, dS_next^T, T
    {
        const __nv_bfloat16 *src[4] = {reinterpret_cast<const __nv_bfloat16 *>(a.q),
                                       reinterpret_cast<const __nv_bfloat16 *>(a.k),
                                       reinterpret_cast<const __nv_bfloat16 *>(a.v),
                                       reinterpret_cast<const __nv_bfloat16 *>(a.dout)};
        for (int i = tid; i < 4 * C * 16; i += NT) {
            const int m = i >> 10, r = (i >> 4) & 63, j = i & 15, t = c * C + r;
            const bool ok = t < a.T;
            const int H = m < 2 ? a.Hk : a.Hv, hh = m < 2 ? hk : h;
            cp_async16(sb + m * SZ_DT + (r * LDD + 8 * j) * 2,
                       src[m] + (((size_t)b * a.T + (ok ? t : 0)) * H + hh) * D + 8 * j, ok ? 16 : 0);
        }
        const __half *S = ws.s + cu * D * D, *dS = ws.ds + cu * D * D;
        for (int i = tid; i < D * 16; i += NT) {
            const int r = i >> 4, j = i & 15;
            cp_async16(sb + OC_S + (r * LDD + 8 * j) * 2, S + r * D + 8 * j, 16);
            cp_async16(sb + OC_DS + (r * LDD + 8 * j) * 2, dS + r * D + 8 * j, 16);
        }
        const __half *Tg = ws.t + cu * C * C;
        for (int i = tid; i < C * 8; i += NT) {
            const int r = i >> 3, j = i & 7;
            cp_async16(sb + OC_T + (r * LDC + 8 * j) * 2, Tg + r * C + 8 * j, 16);
        }
        cp_async_commit();
        if (tid < C) {
            const int t = c * C + tid;
            const bool ok = t < a.T;
            vec[VG + tid] = ok ? a.g[((size_t)b * a.T + t) * a.Hv + h] : 0.f;
            vec[VBETA + tid] = ok ? a.beta[((size_t)b * a.T + t) * a.Hv + h] : 0.f;
        }
        cp_async_wait_all();
        for (int i = tid; i < 4 * C * 16; i += NT) {
            const int m = i >> 10, r = (i >> 4) & 63, j = i & 15;
            bf16_to_fp16_16B(sm + m * SZ_DT + (r * LDD + 8 * j) * 2);
        }
        // T is lower triangular: clear what the forward left unwritten above the diagonal blocks
        for (int i = tid; i < C * 8; i += NT) {
            const int r = i >> 3, j = i & 7;
            __half *row = reinterpret_cast<__half *>(sm + OC_T) + r * LDC + 8 * j;
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if (8 * j + e > r) row[e] = __float2half(0.f);
        }
    }
    __syncthreads();
    if (warp == 0) {   // in-chunk prefix G, Gamma = exp(G), f = Gamma_C / Gamma
        float x0 = vec[VG + lane], x1 = vec[VG + 32 + lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y0 = __shfl_up_sync(0xffffffffu, x0, o), y1 = __shfl_up_sync(0xffffffffu, x1, o);
            if (lane >= o) x0 += y0, x1 += y1;
        }
        x1 += __shfl_sync(0xffffffffu, x0, 31);
        const float GL = __shfl_sync(0xffffffffu, x1, 31);
        vec[VG + lane] = x0;
        vec[VG + 32 + lane] = x1;
        vec[VGAM + lane] = __expf(x0);
        vec[VGAM + 32 + lane] = __expf(x1);
        vec[VF + lane] = __expf(GL - x0);
        vec[VF + 32 + lane] = __expf(GL - x1);
    }
    {   // sum(dS_next * S) over the whole state
        float s = 0.f;
        for (int i = tid; i < D * 16; i += NT) {
            const int r = i >> 4, j = i & 15;
            const __half2 *x = reinterpret_cast<const __half2 *>(sm + OC_S + (r * LDD + 8 * j) * 2);
            const __half2 *y = reinterpret_cast<const __half2 *>(sm + OC_DS + (r * LDD + 8 * j) * 2);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 fx = __half22float2(x[e]), fy = __half22float2(y[e]);
                s = fmaf(fx.x, fy.x, fmaf(fx.y, fy.y, s));
            }
        }
        s = warp_sum(s);
        if (lane == 0) vec[VSS + warp] = s;
    }
    __syncthreads();

    const float *G = vec + VG, *Gam = vec + VGAM, *beta = vec + VBETA, *fv = vec + VF;
    const int ra = r0 + g8, rb = ra + 8;   // this thread's two rows in every row block
    auto dec = [&](int r, int i) { return r >= i ? __expf(G[r] - G[i]) : 0.f; };
    // per-row partial sums of this thread (rows ra, rb), added to dG / dbeta at the end
    float pg0 = 0.f, pg1 = 0.f, pb0 = 0.f, pb1 = 0.f, tot3 = 0.f;
    auto rowdot = [&](const float (*acc)[4], uint32_t tile, int n0, float &s0, float &s1) {
        // sum over this thread's columns of acc * tile (fp16 [64][LDD]) on rows ra and rb
        const __half *tp = reinterpret_cast<const __half *>(sm + tile);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            const int col = n0 + 8 * nt + 2 * t4;
            const float2 x = __half22float2(*reinterpret_cast<const __half2 *>(tp + ra * LDD + col));
            const float2 y = __half22float2(*reinterpret_cast<const __half2 *>(tp + rb * LDD + col));
            s0 = fmaf(acc[nt][0], x.x, fmaf(acc[nt][1], x.y, s0));
            s1 = fmaf(acc[nt][2], y.x, fmaf(acc[nt][3], y.y, s1));
        }
    };
    auto store_h = [&](const float (*acc)[4], int ntn, uint32_t tile, int ld, int n0, float s) {
        __half *tp = reinterpret_cast<__half *>(sm + tile);
        for (int nt = 0; nt < ntn; ++nt) {
            const int col = n0 + 8 * nt + 2 * t4;
            *reinterpret_cast<uint32_t *>(tp + ra * ld + col) = pack_h2f(s * acc[nt][0], s * acc[nt][1]);
            *reinterpret_cast<uint32_t *>(tp + rb * ld + col) = pack_h2f(s * acc[nt][2], s * acc[nt][3]);
        }
    };
    const int n128 = 64 * cw, n64 = 32 * cw;   // this warp's columns of 128- and 64-wide outputs

    // ---- a: the Grams, M = tril(Q K^T * D) and Bm = tril(K K^T * D, -1)
    float bm[4][4];
    {
        float qk[4][4], kk[4][4];
        zero_acc<4>(qk);
        zero_acc<4>(kk);
        wgemm<8, 2, false, false>(qk, sb + OC_Q, LDD, r0, sb + OC_K, LDD, n64, lane, NoScale());
        wgemm<8, 2, false, false>(kk, sb + OC_K, LDD, r0, sb + OC_K, LDD, n64, lane, NoScale());
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = e < 2 ? ra : rb, i = n64 + 8 * nt + 2 * t4 + (e & 1);
                const float d = dec(r, i);
                qk[nt][e] *= d;
                bm[nt][e] = r > i ? kk[nt][e] * d : 0.f;
            }
        store_h(qk, 4, OC_M, LDC, n64, 1.f);
    }
    // ---- b: W = T diag(beta Gamma) K, U = T diag(beta) V, then U' = U - W S
    {
        float w[8][4], u[8][4];
        zero_acc<8>(w);
        zero_acc<8>(u);
        auto colscale = [&](const float *s1, const float *s2) {
            return [=](uint32_t *af, int j) {
                const int k0 = 16 * j + 2 * t4;
                const __half2 lo = __floats2half2_rn(s1[k0] * (s2 ? s2[k0] : 1.f), s1[k0 + 1] * (s2 ? s2[k0 + 1] : 1.f));
                const __half2 hi =
                    __floats2half2_rn(s1[k0 + 8] * (s2 ? s2[k0 + 8] : 1.f), s1[k0 + 9] * (s2 ? s2[k0 + 9] : 1.f));
                hmul_frag(af[0], lo);
                hmul_frag(af[1], lo);
                hmul_frag(af[2], hi);
                hmul_frag(af[3], hi);
            };
        };
        wgemm<4, 4, false, true>(w, sb + OC_T, LDC, r0, sb + OC_K, LDD, n128, lane, colscale(beta, Gam));
        wgemm<4, 4, false, true>(u, sb + OC_T, LDC, r0, sb + OC_V, LDD, n128, lane, colscale(beta, nullptr));
        store_h(w, 8, OC_W, LDD, n128, 1.f);
        __syncthreads();
        const __half2 neg = __floats2half2_rn(-1.f, -1.f);
        wgemm<8, 4, false, false>(u, sb + OC_W, LDD, r0, sb + OC_S, LDD, n128, lane, [=](uint32_t *af, int) {
            hmul_frag(af[0], neg);
            hmul_frag(af[1], neg);
            hmul_frag(af[2], neg);
            hmul_frag(af[3], neg);
        });
        store_h(u, 8, OC_U, LDD, n128, 1.f);
    }
    __syncthreads();
    // ---- c: dU' = M^T dO + diag(f) K dS_next
    {
        float du[8][4];
        zero_acc<8>(du);
        wgemm<4, 4, true, true>(du, sb + OC_M, LDC, r0, sb + OC_DO, LDD, n128, lane, NoScale());
        const __half2 fa = __float2half2_rn(fv[ra]), fb = __float2half2_rn(fv[rb]);
        wgemm<8, 4, false, false>(du, sb + OC_K, LDD, r0, sb + OC_DS, LDD, n128, lane, [=](uint32_t *af, int) {
            hmul_frag(af[0], fa);
            hmul_frag(af[1], fb);
            hmul_frag(af[2], fa);
            hmul_frag(af[3], fb);
        });
        store_h(du, 8, OC_W, LDD, n128, 1.f);   // W is dead
    }
    __syncthreads();
    // ---- d: dM = tril(dO U'^T), stored as dM * D
    {
        float dm[4][4];
        zero_acc<4>(dm);
        wgemm<8, 2, false, false>(dm, sb + OC_DO, LDD, r0, sb + OC_U, LDD, n64, lane, NoScale());
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = e < 2 ? ra : rb, i = n64 + 8 * nt + 2 * t4 + (e & 1);
                dm[nt][e] *= dec(r, i);
            }
        store_h(dm, 4, OC_M, LDC, n64, 1.f);   // M is dead
    }
    __syncthreads();
    const bool va = c * C + ra < a.T, vb = c * C + rb < a.T;
    const size_t rowq_a = (((size_t)b * a.T + c * C + ra) * a.Hk + hk) * D, rowq_b = rowq_a + (size_t)8 * a.Hk * D;
    // ---- e: dQ = diag(Gamma) dO S^T + (dM * D) K
    {
        float dq[8][4];
        zero_acc<8>(dq);
        wgemm<8, 4, false, true>(dq, sb + OC_DO, LDD, r0, sb + OC_S, LDD, n128, lane, NoScale());
        const float ga = Gam[ra], gb = Gam[rb];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) dq[nt][0] *= ga, dq[nt][1] *= ga, dq[nt][2] *= gb, dq[nt][3] *= gb;
        wgemm<4, 4, false, true>(dq, sb + OC_M, LDC, r0, sb + OC_K, LDD, n128, lane, NoScale());
        rowdot(dq, OC_Q, n128, pg0, pg1);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            const int col = n128 + 8 * nt + 2 * t4;
            if (va) atomicAdd(a.dq + rowq_a + col, dq[nt][0]), atomicAdd(a.dq + rowq_a + col + 1, dq[nt][1]);
            if (vb) atomicAdd(a.dq + rowq_b + col, dq[nt][2]), atomicAdd(a.dq + rowq_b + col + 1, dq[nt][3]);
        }
    }
    // ---- f: dK3 = diag(f) U' dS_next^T (the start of dK)
    float dk[8][4];
    {
        zero_acc<8>(dk);
        wgemm<8, 4, false, true>(dk, sb + OC_U, LDD, r0, sb + OC_DS, LDD, n128, lane, NoScale());
        const float fa = fv[ra], fb = fv[rb];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) dk[nt][0] *= fa, dk[nt][1] *= fa, dk[nt][2] *= fb, dk[nt][3] *= fb;
        float s0 = 0.f, s1 = 0.f;
        rowdot(dk, OC_K, n128, s0, s1);
        pg0 -= s0, pg1 -= s1, tot3 += s0 + s1;
    }
    // ---- g: dW = -dU' S^T, into the dS_next slot once every warp is done with it
    {
        float dw[8][4];
        zero_acc<8>(dw);
        wgemm<8, 4, false, true>(dw, sb + OC_W, LDD, r0, sb + OC_S, LDD, n128, lane, NoScale());
        __syncthreads();
        store_h(dw, 8, OC_DS, LDD, n128, -1.f);
    }
    __syncthreads();
    // ---- h: dV = diag(beta) T^T dU', and dK1's first part diag(Gamma beta) T^T dW
    {
        float y[8][4];
        zero_acc<8>(y);
        wgemm<4, 4, true, true>(y, sb + OC_T, LDC, r0, sb + OC_W, LDD, n128, lane, NoScale());
        rowdot(y, OC_V, n128, pb0, pb1);   // rowsum(V * T^T dU')
        const float ba = beta[ra], bb = beta[rb];
        const size_t rowv_a = (((size_t)b * a.T + c * C + ra) * a.Hv + h) * D, rowv_b = rowv_a + (size_t)8 * a.Hv * D;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            const int col = n128 + 8 * nt + 2 * t4;
            if (va) *reinterpret_cast<float2 *>(a.dv + rowv_a + col) = make_float2(ba * y[nt][0], ba * y[nt][1]);
            if (vb) *reinterpret_cast<float2 *>(a.dv + rowv_b + col) = make_float2(bb * y[nt][2], bb * y[nt][3]);
        }
        zero_acc<8>(y);
        wgemm<4, 4, true, true>(y, sb + OC_T, LDC, r0, sb + OC_DS, LDD, n128, lane, NoScale());
        float s0 = 0.f, s1 = 0.f;
        rowdot(y, OC_K, n128, s0, s1);   // rowsum(K * T^T dW)
        const float ga = Gam[ra], gb = Gam[rb];
        pb0 += ga * s0, pb1 += gb * s1;
        pg0 += ga * ba * s0, pg1 += gb * bb * s1;   // rowsum(dK1a * K)
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            dk[nt][0] += ga * ba * y[nt][0], dk[nt][1] += ga * ba * y[nt][1];
            dk[nt][2] += gb * bb * y[nt][2], dk[nt][3] += gb * bb * y[nt][3];
        }
    }
    // ---- i: dT = dU' V^T diag(beta) + dW K^T diag(beta Gamma), into the U' slot
    {
        float x1[4][4], x2[4][4];
        zero_acc<4>(x1);
        zero_acc<4>(x2);
        wgemm<8, 2, false, false>(x1, sb + OC_W, LDD, r0, sb + OC_V, LDD, n64, lane, NoScale());
        wgemm<8, 2, false, false>(x2, sb + OC_DS, LDD, r0, sb + OC_K, LDD, n64, lane, NoScale());
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = n64 + 8 * nt + 2 * t4 + (e & 1);
                x1[nt][e] = beta[i] * (x1[nt][e] + Gam[i] * x2[nt][e]);
            }
        store_h(x1, 4, OC_U, LDC, n64, 1.f);   // U' is dead (read in d and f)
    }
    __syncthreads();
    // ---- j: X = T^T dT (into the S^T slot), then dA = strict tril(-X T^T)
    {
        float x[4][4];
        zero_acc<4>(x);
        wgemm<4, 2, true, true>(x, sb + OC_T, LDC, r0, sb + OC_U, LDC, n64, lane, NoScale());
        store_h(x, 4, OC_S, LDC, n64, 1.f);
    }
    __syncthreads();
    {
        float y[4][4];
        zero_acc<4>(y);
        wgemm<4, 2, false, false>(y, sb + OC_S, LDC, r0, sb + OC_T, LDC, n64, lane, NoScale());
        const float ba = beta[ra], bb = beta[rb];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = e < 2 ? ra : rb, i = n64 + 8 * nt + 2 * t4 + (e & 1);
                const float dA = r > i ? -y[nt][e] : 0.f;
                if (e < 2) pb0 += dA * bm[nt][e];
                else pb1 += dA * bm[nt][e];
                y[nt][e] = (e < 2 ? ba : bb) * dA * dec(r, i);   // dB * D
            }
        store_h(y, 4, OC_U, LDC, n64, 1.f);   // dT is dead (read for X)
    }
    __syncthreads();
    // ---- k: dK1 += (dB * D) K;  dK2 = (dM * D)^T Q + (dB * D)^T K
    {
        float p[8][4];
        zero_acc<8>(p);
        wgemm<4, 4, false, true>(p, sb + OC_U, LDC, r0, sb + OC_K, LDD, n128, lane, NoScale());
        rowdot(p, OC_K, n128, pg0, pg1);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) dk[nt][e] += p[nt][e];
        zero_acc<8>(p);
        wgemm<4, 4, true, true>(p, sb + OC_M, LDC, r0, sb + OC_Q, LDD, n128, lane, NoScale());
        wgemm<4, 4, true, true>(p, sb + OC_U, LDC, r0, sb + OC_K, LDD, n128, lane, NoScale());
        float s0 = 0.f, s1 = 0.f;
        rowdot(p, OC_K, n128, s0, s1);
        pg0 -= s0, pg1 -= s1;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            const int col = n128 + 8 * nt + 2 * t4;
            const float k0 = dk[nt][0] + p[nt][0], k1 = dk[nt][1] + p[nt][1];
            const float k2 = dk[nt][2] + p[nt][2], k3 = dk[nt][3] + p[nt][3];
            if (va) atomicAdd(a.dk + rowq_a + col, k0), atomicAdd(a.dk + rowq_a + col + 1, k1);
            if (vb) atomicAdd(a.dk + rowq_b + col, k2), atomicAdd(a.dk + rowq_b + col + 1, k3);
        }
    }
    // ---- l: row sums over the warps, then dg (reverse cumulative sum) and dbeta
#pragma unroll
    for (int o = 1; o < 4; o <<= 1) {
        pg0 += __shfl_xor_sync(0xffffffffu, pg0, o);
        pg1 += __shfl_xor_sync(0xffffffffu, pg1, o);
        pb0 += __shfl_xor_sync(0xffffffffu, pb0, o);
        pb1 += __shfl_xor_sync(0xffffffffu, pb1, o);
    }
    if (t4 == 0) {
        vec[VDG + 64 * cw + ra] = pg0;
        vec[VDG + 64 * cw + rb] = pg1;
        vec[VDB + 64 * cw + ra] = pb0;
        vec[VDB + 64 * cw + rb] = pb1;
    }
    tot3 = warp_sum(tot3);
    if (lane == 0) vec[VT3 + warp] = tot3;
    __syncthreads();
    if (warp == 0) {
        float t3 = 0.f, ss = 0.f;
#pragma unroll
        for (int w8 = 0; w8 < 8; ++w8) t3 += vec[VT3 + w8], ss += vec[VSS + w8];
        // rows 63 - lane and 31 - lane: an inclusive scan over the lanes is the reverse sum
        const float extra = t3 + __expf(G[C - 1]) * ss;
        const int rA = 63 - lane, rB = 31 - lane;
        float x0 = vec[VDG + rA] + vec[VDG + 64 + rA] + (lane == 0 ? extra : 0.f);
        float x1 = vec[VDG + rB] + vec[VDG + 64 + rB];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y0 = __shfl_up_sync(0xffffffffu, x0, o), y1 = __shfl_up_sync(0xffffffffu, x1, o);
            if (lane >= o) x0 += y0, x1 += y1;
        }
        x1 += __shfl_sync(0xffffffffu, x0, 31);
        const size_t base = (size_t)b * a.T + c * C;
        if (c * C + rA < a.T) {
            a.dg[(base + rA) * a.Hv + h] = x0;
            a.dbeta[(base + rA) * a.Hv + h] = vec[VDB + rA] + vec[VDB + 64 + rA];
        }
        if (c * C + rB < a.T) {
            a.dg[(base + rB) * a.Hv + h] = x1;
            a.dbeta[(base + rB) * a.Hv + h] = vec[VDB + rB] + vec[VDB + 64 + rB];
        }
    }
}

}  // namespace

bool bwdc_supported(const BwdArgs &a)
{
    return in_bf16(a.dtype) && a.gate_mode == 0 && a.Dk == D && a.Dv == D;
}

size_t bwdc_workspace_size(const BwdArgs &a)
{
    const size_t cu = (size_t)a.B * a.Hv * ((a.T + C - 1) / C);
    // S^T, P, dS_next^T [128][128], Qh^T [128][64], T [64][64], fp16
    return cu * (3 * D * D + D * C + C * C) * sizeof(__half);
}

cudaError_t launch_bwdc(const BwdArgs &a, void *workspace, cudaStream_t st)
{
    const size_t cu = (size_t)a.B * a.Hv * ((a.T + C - 1) / C);
    BwdcWs ws;
    __half *p = reinterpret_cast<__half *>(workspace);
    ws.s = p;
    ws.p = ws.s + cu * D * D;
    ws.ds = ws.p + cu * D * D;
    ws.qh = ws.ds + cu * D * D;
    ws.t = ws.qh + cu * D * C;
    FwdArgs f{};
    f.q = a.q, f.k = a.k, f.v = a.v, f.g = a.g, f.beta = a.beta, f.h0 = a.h0;
    f.o = nullptr, f.hT = nullptr;
    f.B = a.B, f.T = a.T, f.Hk = a.Hk, f.Hv = a.Hv, f.Dk = a.Dk, f.Dv = a.Dv, f.gate_mode = 0, f.dtype = a.dtype;
    f.save_s = ws.s, f.save_p = ws.p, f.save_qh = ws.qh, f.save_t = ws.t;
    cudaError_t e = launch_fwd_tc(f, st);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bwdc_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_SCAN);
    if (e != cudaSuccess) return e;
    bwdc_scan_kernel<<<(unsigned)(a.B * a.Hv), NT, SMEM_SCAN, st>>>(a, ws);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bwdc_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_CHUNK);
    if (e != cudaSuccess) return e;
    bwdc_chunk_kernel<<<(unsigned)cu, NT, SMEM_CHUNK, st>>>(a, ws);
    return cudaGetLastError();
}

}  // namespace gdr
