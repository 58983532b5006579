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
//      entering state S^T, P, Qh^T and T = (I + A)^-1 as fp16 images of 128-byte swizzled
//      tiles;
//   2. bwdc_scan_kernel: per (batch row, value head), the chunks in reverse on tcgen05;
//      dS^T is carried in fp32 registers, its fp16 copy in tensor memory is the products'
//      A operand, and it is stored per chunk (as dS_next of that chunk); the last is dh0;
//   3. bwdc_chunk_kernel: one CTA per (unit, chunk), all chunks at once, on the warp-level
//      MMAs (mma.sync, fp16 operands, fp32 accumulation). With the
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
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"
#include "mma_util.cuh"
#include "tc_util.cuh"

namespace gdr {
namespace {

using namespace mmau;

constexpr int NT = 256;   // 8 warps

// The per-(unit, chunk) fp16 buffers of the three passes, in the caller's workspace.
struct BwdcWs {
    __half *s, *p, *qh, *t, *ds;   // S^T [Dv][Dk], P [Dk][Dk], Qh^T [Dk][64], T [64][64], dS_next^T [Dv][Dk]
};

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

// ------------------------------------------------------------------ pass 2: the reverse scan
// One CTA of 8 warps per (batch row, value head), on tcgen05. Per chunk, in reverse order:
//     D = dO^T Qh + dS^T P          (128 x 128 fp32 accumulator in tensor memory)
//     dS^T <- Gamma_C dS^T + D      (fp32, in registers: thread (p, hf) holds row p of dS^T,
//                                    columns 64 hf .. 64 hf + 63)
// A of the second product is the fp16 copy of dS^T in tensor memory (as the forward's state
// batch reads S^T); P and Qh^T are the forward's 128-byte swizzled operand tiles, bulk-copied
// from the workspace; dO comes by TMA and is converted to fp16 in place.
constexpr uint32_t SC_P = 0;                  // P [dk_out][dk_in], 2 atoms of 16 KB
constexpr uint32_t SC_QH = 32768;             // Qh^T [dk][token], 16 KB
constexpr uint32_t SC_DO = SC_QH + 16384;     // dO [token][dv], 2 atoms of 8 KB
constexpr uint32_t SC_BUF = SC_DO + 16384;    // one chunk's operands (64 KB)
constexpr uint32_t SC_BAR = 2 * SC_BUF;       // mbarriers: loads (2), products, drain; TMEM base
constexpr uint32_t SMEM_SCAN = SC_BAR + 64 + 1024;
constexpr uint32_t TS_D = 0, TS_A = 128;      // tensor-memory columns: accumulator, fp16 copy of dS^T
constexpr uint32_t ID_SQ = tcu::idesc_f16(128, 128, false, true, false);   // dO^T Qh
constexpr uint32_t ID_SP = tcu::idesc_f16(128, 128, false, false, true);   // dS^T P

__device__ unsigned int g_bwdc_timeouts;

// Global -> L2 prefetches: a 16-byte aligned span of a multiple of 16 bytes.
__device__ __forceinline__ void prefetch_l2_bulk(const void *src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
// One TMA box into L2 (no shared-memory destination).
__device__ __forceinline__ void prefetch_tma_4d(const CUtensorMap *map, int c0, int c1, int c2, int c3)
{
    asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3) : "memory");
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

__global__ void __launch_bounds__(NT, 1) bwdc_scan_kernel(BwdArgs a, BwdcWs ws, const __grid_constant__ CUtensorMap map_do)
{
    using namespace tcu;
    extern __shared__ __align__(1024) uint8_t sm_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q4 = warp & 3, hf = warp >> 2, p = 32 * q4 + lane;
    const int unit = blockIdx.x, b = unit / a.Hv, h = unit % a.Hv;
    const int NC = (a.T + C - 1) / C;
    auto bar = [&](int i) { return sb + SC_BAR + 8 * i; };   // 0, 1: loads; 2: products; 3: drain
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + SC_BAR + 32);
    __shared__ int abort_sh;
    if (tid == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(bar(i), 1);
        abort_sh = 0;
    }
    if (warp == 0) tmem_alloc(smem_u32(tmem_slot), 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = *tmem_slot;
    auto wait = [&](int i, uint32_t parity) {
        if (*reinterpret_cast<volatile int *>(&abort_sh)) return;
        if (!mbar_wait_bounded(bar(i), parity)) {
            *reinterpret_cast<volatile int *>(&abort_sh) = 1;
            atomicAdd(&g_bwdc_timeouts, 1u);
        }
    };
    auto issue_loads = [&](int c, int buf) {   // chunk c's operands into buffer buf
        const uint32_t base = sb + buf * SC_BUF, bl = bar(buf);
        const size_t cu = (size_t)unit * NC + c;
        mbar_expect_tx(bl, SC_BUF);
        bulk_g2s(base + SC_P, ws.p + cu * D * D, 32768, bl);
        bulk_g2s(base + SC_QH, ws.qh + cu * D * C, 16384, bl);
        tma_load_4d(base + SC_DO, &map_do, 0, h, c * C, b, bl);
        tma_load_4d(base + SC_DO + 8192, &map_do, 64, h, c * C, b, bl);
    };

    // dS^T entering the reverse scan: dhT^T
    float dS[64];
    {
        const float *src = a.dhT ? a.dhT + (size_t)unit * D * D + (size_t)(64 * hf) * D + p : nullptr;
#pragma unroll
        for (int i = 0; i < 64; ++i) dS[i] = src ? __ldg(src + (size_t)i * D) : 0.f;
    }
    auto store_copy = [&]() {   // the fp16 copy of dS^T in tensor memory, the next products' A
        uint32_t w[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) w[j] = pack_h2f(dS[2 * j], dS[2 * j + 1]);
        tmem_st32(tmem_addr(tb, q4, TS_A + 32 * hf), w);
        tmem_wait_st();
    };
    store_copy();
    if (tid == 0) {
        issue_loads(NC - 1, 0);
        if (NC > 1) issue_loads(NC - 2, 1);
    }
    // g of a chunk, two values per lane (summed over the warp when needed), loaded one chunk ahead
    auto load_g = [&](int c, float &g0, float &g1) {
        const int t0 = c * C + lane, t1 = t0 + 32;
        g0 = (c >= 0 && t0 < a.T) ? a.g[((size_t)b * a.T + t0) * a.Hv + h] : 0.f;
        g1 = (c >= 0 && t1 < a.T) ? a.g[((size_t)b * a.T + t1) * a.Hv + h] : 0.f;
    };
    auto convert_do = [&](int buf) {   // this thread's 64 bytes of dO to fp16 (rows past T are zeros)
        uint8_t *d = sm + buf * SC_BUF + SC_DO + tid * 64;
#pragma unroll
        for (int k = 0; k < 4; ++k) bf16_to_fp16_16B(d + 16 * k);
    };
    float ga, gb;
    load_g(NC - 1, ga, gb);
    wait(0, 0);
    convert_do(0);
    for (int s = 0; s < NC; ++s) {
        const int c = NC - 1 - s, buf = s & 1;
        const float gC = __expf(warp_sum(ga + gb));   // Gamma_C of chunk c
        load_g(c - 1, ga, gb);
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();   // dO of chunk c converted, the copy of dS^T written
        if (tid == 0) {
            tc_fence_after();
            const uint32_t base = sb + buf * SC_BUF;
#pragma unroll
            for (int k = 0; k < 4; ++k)
                mma_ss(tb + TS_D, sdesc(base + SC_DO + k * 2048, 8192, 1024), sdesc(base + SC_QH + k * 32, 16, 1024),
                       ID_SQ, k > 0);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                mma_ts(tb + TS_D, tb + TS_A + 8 * k, sdesc(base + SC_P + k * 2048, 16384, 1024), ID_SP, true);
            mma_commit(bar(2));
        }
        {   // while the products run: dS_next of chunk c (row p of dS^T, columns 64 hf .., as the
            // fp16 image of a 128-byte swizzled tile) ...
            uint8_t *dst = reinterpret_cast<uint8_t *>(ws.ds + ((size_t)unit * NC + c) * D * D);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint4 *>(dst + swz_chunk(p, j, hf * 16384)) =
                    make_uint4(pack_h2f(dS[8 * j], dS[8 * j + 1]), pack_h2f(dS[8 * j + 2], dS[8 * j + 3]),
                               pack_h2f(dS[8 * j + 4], dS[8 * j + 5]), pack_h2f(dS[8 * j + 6], dS[8 * j + 7]));
        }
        if (s + 1 < NC) {   // ... and the next chunk's dO
            wait(buf ^ 1, ((s + 1) >> 1) & 1);
            convert_do(buf ^ 1);
        }
        wait(2, s & 1);
        tc_fence_after();
        if (tid == 0 && s + 2 < NC) issue_loads(c - 2, buf);   // the products are done with buf
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            float v[32];
            tmem_ld32(tmem_addr(tb, q4, TS_D + 64 * hf + 32 * h2), v);
            uint32_t w[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                dS[32 * h2 + 2 * j] = fmaf(gC, dS[32 * h2 + 2 * j], v[2 * j]);
                dS[32 * h2 + 2 * j + 1] = fmaf(gC, dS[32 * h2 + 2 * j + 1], v[2 * j + 1]);
                w[j] = pack_h2f(dS[32 * h2 + 2 * j], dS[32 * h2 + 2 * j + 1]);
            }
            tmem_st16(tmem_addr(tb, q4, TS_A + 32 * hf + 16 * h2), w);
        }
        tmem_wait_st();
    }
    {   // dh0 = dS entering chunk 0
        float *dst = a.dh0 + (size_t)unit * D * D + (size_t)(64 * hf) * D + p;
#pragma unroll
        for (int i = 0; i < 64; ++i) dst[(size_t)i * D] = dS[i];
    }
    if (tid == 0) {   // every product this thread issued has completed before the memory is freed
        tc_fence_after();
        mma_commit(bar(3));
        mbar_wait_bounded(bar(3), 0);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tb, 256);
    }
}

// ------------------------------------------------------------------ pass 3: per-chunk gradients
// 8 warps; warp (rw, cw) = (warp & 1, warp >> 1) computes rows 32 rw .. 32 rw + 31 of every
// product (two m16 blocks, mi = 0, 1) and columns 32 cw .. of the 128-wide ones, 16 cw .. of
// the 64-wide ones: each fragment loaded from shared memory feeds two to four MMAs.
constexpr int NTC = 256;
// Input tiles are 128-byte swizzled images (64-column atoms, 1024-byte aligned), loaded by TMA
// (q, k, v, dO) and bulk copies (S^T, dS_next^T, T); the tiles the kernel writes itself are
// plain rows padded to LDD / LDC halves. A tile's "ld" below is its padded row stride in
// halves, or minus its atom stride in bytes for a swizzled image.
constexpr uint32_t SZ_DT = C * LDD * 2;     // padded [64][136] fp16
constexpr uint32_t SZ_CT = C * LDC * 2;     // padded [64][72] fp16
constexpr int LQ = -8192, LS = -16384, LT = -8192;   // swizzled [64][128], [128][128], [64][64]
constexpr uint32_t OC_Q = 0, OC_K = 16384, OC_V = 32768, OC_DO = 49152;
constexpr uint32_t OC_S = 65536;              // S^T [dv][dk]; later X = T^T dT [64][LDC]
constexpr uint32_t OC_DS = OC_S + 32768;      // dS_next^T [dv][dk]; later dW [64][LDD]
constexpr uint32_t OC_T = OC_DS + 32768;      // T [64][64]
constexpr uint32_t OC_M = OC_T + 8192;        // M, then dM * D [64][LDC]
constexpr uint32_t OC_W = OC_M + SZ_CT;       // W, then dU' [64][LDD]
constexpr uint32_t OC_U = OC_W + SZ_DT;       // U', then dT, then dB * D [64][LDC]
constexpr uint32_t OC_DEC = OC_U + SZ_DT;     // D_ri = exp(G_r - G_i) (r >= i, else 0) [64][LDC] fp16
constexpr uint32_t OC_BM = OC_DEC + SZ_CT;    // Bm = tril(K K^T * D, -1) [64][LDC] fp16
constexpr uint32_t OC_BAR = OC_BM + SZ_CT;    // two mbarriers: inputs, then S^T and dS_next^T
constexpr uint32_t OC_VEC = OC_BAR + 16;
// vectors: G, Gamma, beta, f [64]; per column quarter of the warps, the row sums of dG and dbeta
// [4][64] each; per warp, sum(dK3 * K) and sum(dS_next * S) [8] each (summed in a fixed order,
// so that dg and dbeta repeat bit for bit)
constexpr int VG = 0, VGAM = 64, VBETA = 128, VF = 192, VDG = 256, VDB = 512, VT3 = 768, VSS = 776;
constexpr uint32_t SMEM_CHUNK = OC_VEC + (VSS + 8) * 4 + 1024;   // + alignment of the base
static_assert(SMEM_CHUNK <= 227 * 1024, "shared memory");

// Byte address of element (row, col) of a tile with the given ld (see above).
__device__ __forceinline__ uint32_t taddr(uint32_t base, int ld, int row, int col)
{
    if (ld > 0) return base + (uint32_t)(row * ld + col) * 2u;
    return base + (uint32_t)(col >> 6) * (uint32_t)(-ld) + (uint32_t)(row >> 3) * 1024u + (uint32_t)(row & 7) * 128u +
           (((uint32_t)((col & 63) >> 3) ^ (uint32_t)(row & 7)) << 4) + (uint32_t)(col & 7) * 2u;
}
// acc[2][2 NP][4] += A (rows r0 .. r0 + 31, K = 16 KS) B (columns n0 .. n0 + 16 NP) on the
// warp-level MMAs (m16n8k16, fp16 operands, fp32 accumulators in the m16n8 layout).
// A: [m][k] (AT false) or stored transposed [k][m] (AT true); B: stored [n][k] (BT false) or
// [k][n] (BT true); each tile by its ld (see taddr). ascale(af, j, mi) may rescale the A
// fragment of k-step j, row block mi, in registers.
template <int KS, int NP, bool AT, bool BT, typename AS>
__device__ __forceinline__ void wgemm2(float (*acc)[2 * NP][4], uint32_t aB, int lda, int r0, uint32_t bB, int ldb,
                                       int n0, int lane, AS ascale)
{
#pragma unroll 4
    for (int j = 0; j < KS; ++j) {
        uint32_t af[2][4];
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) {
            const int m0 = r0 + 16 * mi, k0 = 16 * j;
            if (AT) ldsm_t(af[mi], taddr(aB, lda, k0 + (lane & 7) + (lane >> 4) * 8, m0 + ((lane >> 3) & 1) * 8));
            else ldsm(af[mi], taddr(aB, lda, m0 + (lane & 7) + ((lane >> 3) & 1) * 8, k0 + (lane >> 4) * 8));
            ascale(af[mi], j, mi);
        }
#pragma unroll
        for (int np = 0; np < NP; ++np) {
            uint32_t bf[4];
            const int nn = n0 + 16 * np, k0 = 16 * j;
            if (BT) ldsm_t(bf, taddr(bB, ldb, k0 + (lane & 7) + ((lane >> 3) & 1) * 8, nn + (lane >> 4) * 8));
            else ldsm(bf, taddr(bB, ldb, nn + (lane & 7) + (lane >> 4) * 8, k0 + ((lane >> 3) & 1) * 8));
#pragma unroll
            for (int mi = 0; mi < 2; ++mi) {
                mma(acc[mi][2 * np], af[mi], bf[0], bf[1]);
                mma(acc[mi][2 * np + 1], af[mi], bf[2], bf[3]);
            }
        }
    }
}
// Two products of the same shape in lockstep (twice the independent MMAs per k-step):
// acc1 += A1 B1, acc2 += A2 B2. SA: A2 is A1's tile (loaded once, then scaled by each
// product's ascale); SB: B2 is B1's tile (loaded once).
template <int KS, int NP, bool AT1, bool BT1, bool AT2, bool BT2, bool SA, bool SB, typename AS1, typename AS2>
__device__ __forceinline__ void wgemm2_pair(float (*acc1)[2 * NP][4], uint32_t a1, int lda1, uint32_t b1, int ldb1,
                                            AS1 as1, float (*acc2)[2 * NP][4], uint32_t a2, int lda2, uint32_t b2,
                                            int ldb2, AS2 as2, int r0, int n0, int lane)
{
    auto lda_ = [&](uint32_t *f, uint32_t aB, int lda, bool at, int m0, int k0) {
        if (at) ldsm_t(f, taddr(aB, lda, k0 + (lane & 7) + (lane >> 4) * 8, m0 + ((lane >> 3) & 1) * 8));
        else ldsm(f, taddr(aB, lda, m0 + (lane & 7) + ((lane >> 3) & 1) * 8, k0 + (lane >> 4) * 8));
    };
    auto ldb_ = [&](uint32_t *f, uint32_t bB, int ldb, bool bt, int nn, int k0) {
        if (bt) ldsm_t(f, taddr(bB, ldb, k0 + (lane & 7) + ((lane >> 3) & 1) * 8, nn + (lane >> 4) * 8));
        else ldsm(f, taddr(bB, ldb, nn + (lane & 7) + (lane >> 4) * 8, k0 + ((lane >> 3) & 1) * 8));
    };
#pragma unroll 2
    for (int j = 0; j < KS; ++j) {
        uint32_t f1[2][4], f2[2][4];
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) {
            lda_(f1[mi], a1, lda1, AT1, r0 + 16 * mi, 16 * j);
            if (SA) {
#pragma unroll
                for (int e = 0; e < 4; ++e) f2[mi][e] = f1[mi][e];
            } else {
                lda_(f2[mi], a2, lda2, AT2, r0 + 16 * mi, 16 * j);
            }
            as1(f1[mi], j, mi);
            as2(f2[mi], j, mi);
        }
#pragma unroll
        for (int np = 0; np < NP; ++np) {
            uint32_t g1[4], g2[4];
            ldb_(g1, b1, ldb1, BT1, n0 + 16 * np, 16 * j);
            if (SB) {
#pragma unroll
                for (int e = 0; e < 4; ++e) g2[e] = g1[e];
            } else {
                ldb_(g2, b2, ldb2, BT2, n0 + 16 * np, 16 * j);
            }
#pragma unroll
            for (int mi = 0; mi < 2; ++mi) {
                mma(acc1[mi][2 * np], f1[mi], g1[0], g1[1]);
                mma(acc2[mi][2 * np], f2[mi], g2[0], g2[1]);
                mma(acc1[mi][2 * np + 1], f1[mi], g1[2], g1[3]);
                mma(acc2[mi][2 * np + 1], f2[mi], g2[2], g2[3]);
            }
        }
    }
}
struct NoScale2 {
    __device__ __forceinline__ void operator()(uint32_t *, int, int) const {}
};
template <int N>
__device__ __forceinline__ void zero2(float (*acc)[N][4])
{
#pragma unroll
    for (int mi = 0; mi < 2; ++mi)
#pragma unroll
        for (int i = 0; i < N; ++i) acc[mi][i][0] = acc[mi][i][1] = acc[mi][i][2] = acc[mi][i][3] = 0.f;
}

// pf: the CTA that runs pf launches later on this SM (the resident CTA count) gets its inputs
// prefetched into L2 by this one; sole: every key head has one value head, so dq and dk rows
// have one writer and take plain stores.
__global__ void __launch_bounds__(NTC, 1)
bwdc_chunk_kernel(BwdArgs a, BwdcWs ws, int pf, int sole, const __grid_constant__ CUtensorMap map_q,
                  const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                  const __grid_constant__ CUtensorMap map_do)
{
    extern __shared__ __align__(1024) uint8_t sm_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g8 = lane >> 2, t4 = lane & 3;
    const int rw = warp & 1, cw = warp >> 1, r0 = 32 * rw;
    const int NC = (a.T + C - 1) / C;
    const int unit = blockIdx.x / NC, c = blockIdx.x % NC;
    const int b = unit / a.Hv, h = unit % a.Hv, hk = h / (a.Hv / a.Hk);
    const uint32_t sb = smem_u32(sm);
    float *vec = reinterpret_cast<float *>(sm + OC_VEC);
    const size_t cu = (size_t)unit * NC + c;

    // ---- loads, on two mbarriers: q, k (key head), v, dO (value head) by TMA (bf16, rows past T
    // zero) and T; then S^T and dS_next^T, which arrive while the Grams, W and U are formed
    __shared__ int abort_sh;
    const uint32_t bar0 = sb + OC_BAR, bar1 = bar0 + 8;
    if (tid == 0) {
        mbar_init(bar0, 1);
        mbar_init(bar1, 1);
        abort_sh = 0;
    }
    __syncthreads();
    if (tid == 0) {
        const int t0 = c * C;
        mbar_expect_tx(bar0, 4 * 16384 + 8192);
        tma_load_4d(sb + OC_Q, &map_q, 0, hk, t0, b, bar0);
        tma_load_4d(sb + OC_Q + 8192, &map_q, 64, hk, t0, b, bar0);
        tma_load_4d(sb + OC_K, &map_k, 0, hk, t0, b, bar0);
        tma_load_4d(sb + OC_K + 8192, &map_k, 64, hk, t0, b, bar0);
        tma_load_4d(sb + OC_V, &map_v, 0, h, t0, b, bar0);
        tma_load_4d(sb + OC_V + 8192, &map_v, 64, h, t0, b, bar0);
        tma_load_4d(sb + OC_DO, &map_do, 0, h, t0, b, bar0);
        tma_load_4d(sb + OC_DO + 8192, &map_do, 64, h, t0, b, bar0);
        bulk_g2s(sb + OC_T, ws.t + cu * C * C, 8192, bar0);
        mbar_expect_tx(bar1, 2 * 32768);
        bulk_g2s(sb + OC_S, ws.s + cu * D * D, 32768, bar1);
        bulk_g2s(sb + OC_DS, ws.ds + cu * D * D, 32768, bar1);
    }
    auto wait = [&](uint32_t bar) {
        if (*reinterpret_cast<volatile int *>(&abort_sh)) return;
        if (!mbar_wait_bounded(bar, 0)) {
            *reinterpret_cast<volatile int *>(&abort_sh) = 1;
            atomicAdd(&g_bwdc_timeouts, 1u);
        }
    };
    if (tid < C) {
        const int t = c * C + tid;
        const bool ok = t < a.T;
        vec[VG + tid] = ok ? a.g[((size_t)b * a.T + t) * a.Hv + h] : 0.f;
        vec[VBETA + tid] = ok ? a.beta[((size_t)b * a.T + t) * a.Hv + h] : 0.f;
    }
    wait(bar0);
    for (int i = tid; i < 2 * C * 16; i += NTC) bf16_to_fp16_16B(sm + OC_Q + 16 * i);   // q, k to fp16
    // T is lower triangular: clear what the forward left unwritten above the diagonal blocks
    for (int i = tid; i < C * 8; i += NTC) {
        const int r = i >> 3, j = i & 7;
        __half *row = reinterpret_cast<__half *>(sm + OC_T + tcu::swz_chunk(r, j, 0));
#pragma unroll
        for (int e = 0; e < 8; ++e)
            if (8 * j + e > r) row[e] = __float2half(0.f);
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
    __syncthreads();

    const float *G = vec + VG, *Gam = vec + VGAM, *beta = vec + VBETA, *fv = vec + VF;
    // this thread's rows: row(mi, hi) = r0 + 16 mi + 8 hi + g8 (accumulator elements 2 hi, 2 hi + 1)
    auto row = [&](int mi, int e) { return r0 + 16 * mi + g8 + 8 * (e >> 1); };
    auto dec = [&](int r, int i) { return r >= i ? __expf(G[r] - G[i]) : 0.f; };
    // D and Bm, written in a and read back by the same thread (same warp tiles) in d and j
    __half *decm = reinterpret_cast<__half *>(sm + OC_DEC), *bmm = reinterpret_cast<__half *>(sm + OC_BM);
    // per-row partial sums of this thread, [mi][hi], added to dG / dbeta at the end
    float pg[2][2] = {{0.f, 0.f}, {0.f, 0.f}}, pb[2][2] = {{0.f, 0.f}, {0.f, 0.f}}, tot3 = 0.f;
    auto rowdot = [&](const float (*acc)[4][4], uint32_t tile, int n0, float (*s)[2]) {
        // sum over this thread's columns of acc * tile (a swizzled [64][128] input) on its rows
#pragma unroll
        for (int mi = 0; mi < 2; ++mi)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const int col = n0 + 8 * nt + 2 * t4;
                const float2 x = __half22float2(*reinterpret_cast<const __half2 *>(sm + (taddr(tile, LQ, row(mi, 0), col))));
                const float2 y = __half22float2(*reinterpret_cast<const __half2 *>(sm + (taddr(tile, LQ, row(mi, 2), col))));
                s[mi][0] = fmaf(acc[mi][nt][0], x.x, fmaf(acc[mi][nt][1], x.y, s[mi][0]));
                s[mi][1] = fmaf(acc[mi][nt][2], y.x, fmaf(acc[mi][nt][3], y.y, s[mi][1]));
            }
    };
    auto store_h = [&](const float (*acc)[4], int mi, int ntn, uint32_t tile, int ld, int n0, float sc) {
        __half *tp = reinterpret_cast<__half *>(sm + tile);
        for (int nt = 0; nt < ntn; ++nt) {
            const int col = n0 + 8 * nt + 2 * t4;
            *reinterpret_cast<uint32_t *>(tp + row(mi, 0) * ld + col) = pack_h2f(sc * acc[nt][0], sc * acc[nt][1]);
            *reinterpret_cast<uint32_t *>(tp + row(mi, 2) * ld + col) = pack_h2f(sc * acc[nt][2], sc * acc[nt][3]);
        }
    };
    const int n128 = 32 * cw, n64 = 16 * cw;   // this warp's columns of 128- and 64-wide outputs
    // per-row scalings of A fragments (rows g8 and g8 + 8 of block mi)
    auto rowscale = [&](const float *v) {
        return [=](uint32_t *af, int, int mi) {
            const __half2 sa = __float2half2_rn(v[r0 + 16 * mi + g8]), sb2 = __float2half2_rn(v[r0 + 16 * mi + g8 + 8]);
            hmul_frag(af[0], sa);
            hmul_frag(af[1], sb2);
            hmul_frag(af[2], sa);
            hmul_frag(af[3], sb2);
        };
    };

    // ---- a: the Grams, M = tril(Q K^T * D) and Bm = tril(K K^T * D, -1)
    {
        float qk[2][2][4], kk[2][2][4];
        zero2<2>(qk);
        zero2<2>(kk);
        wgemm2_pair<8, 1, false, false, false, false, false, true>(qk, sb + OC_Q, LQ, sb + OC_K, LQ, NoScale2(), kk,
                                                                   sb + OC_K, LQ, sb + OC_K, LQ, NoScale2(), r0, n64, lane);
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = row(mi, 2 * hi), i = n64 + 8 * nt + 2 * t4;
                    const float d0 = dec(r, i), d1 = dec(r, i + 1);
                    *reinterpret_cast<__half2 *>(decm + r * LDC + i) = __floats2half2_rn(d0, d1);
                    *reinterpret_cast<__half2 *>(bmm + r * LDC + i) =
                        __floats2half2_rn(r > i ? kk[mi][nt][2 * hi] * d0 : 0.f, r > i + 1 ? kk[mi][nt][2 * hi + 1] * d1 : 0.f);
                    qk[mi][nt][2 * hi] *= d0;
                    qk[mi][nt][2 * hi + 1] *= d1;
                }
            store_h(qk[mi], mi, 2, OC_M, LDC, n64, 1.f);
        }
    }
    // ---- b: W = T diag(beta Gamma) K, U = T diag(beta) V, then U' = U - W S
    {
        float u[2][4][4];
        auto colscale = [&](const float *s1, const float *s2) {
            return [=](uint32_t *af, int j, int) {
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
        // v and dO to fp16 (v for U, dO from c on)
        for (int i = tid; i < 2 * C * 16; i += NTC) bf16_to_fp16_16B(sm + OC_V + 16 * i);
        __syncthreads();
        {
            float w[2][4][4];
            zero2<4>(w);
            zero2<4>(u);
            wgemm2_pair<4, 2, false, true, false, true, true, false>(w, sb + OC_T, LT, sb + OC_K, LQ, colscale(beta, Gam), u,
                                                                     sb + OC_T, LT, sb + OC_V, LQ, colscale(beta, nullptr),
                                                                     r0, n128, lane);
#pragma unroll
            for (int mi = 0; mi < 2; ++mi) store_h(w[mi], mi, 4, OC_W, LDD, n128, 1.f);
        }
        wait(bar1);   // S^T and dS_next^T
        __syncthreads();
        if (tid == 0 && pf > 0 && (long)blockIdx.x + pf < (long)gridDim.x) {
            // the inputs of the CTA pf launches later, into L2 while this one computes (its own
            // loads have landed, so the two do not compete): eight TMA boxes and three spans
            const long nbk = (long)blockIdx.x + pf;
            const int nu = (int)(nbk / NC), ncc = (int)(nbk % NC);
            const int n_b = nu / a.Hv, n_h = nu % a.Hv, n_hk = n_h / (a.Hv / a.Hk), nt0 = ncc * C;
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                prefetch_tma_4d(&map_q, 64 * x, n_hk, nt0, n_b);
                prefetch_tma_4d(&map_k, 64 * x, n_hk, nt0, n_b);
                prefetch_tma_4d(&map_v, 64 * x, n_h, nt0, n_b);
                prefetch_tma_4d(&map_do, 64 * x, n_h, nt0, n_b);
            }
            const size_t ncu = (size_t)nu * NC + ncc;
            prefetch_l2_bulk(ws.s + ncu * D * D, D * D * 2);
            prefetch_l2_bulk(ws.ds + ncu * D * D, D * D * 2);
            prefetch_l2_bulk(ws.t + ncu * C * C, C * C * 2);
        }
        {   // sum(dS_next * S) over the whole state
            float s = 0.f;
            for (int i = tid; i < D * 16; i += NTC) {   // the two images share one layout
                const __half2 *x = reinterpret_cast<const __half2 *>(sm + OC_S + 16 * i);
                const __half2 *y = reinterpret_cast<const __half2 *>(sm + OC_DS + 16 * i);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 fx = __half22float2(x[e]), fy = __half22float2(y[e]);
                    s = fmaf(fx.x, fy.x, fmaf(fx.y, fy.y, s));
                }
            }
            s = warp_sum(s);
            if (lane == 0) vec[VSS + warp] = s;
        }
        const __half2 neg = __floats2half2_rn(-1.f, -1.f);
        wgemm2<8, 2, false, false>(u, sb + OC_W, LDD, r0, sb + OC_S, LS, n128, lane, [=](uint32_t *af, int, int) {
            hmul_frag(af[0], neg);
            hmul_frag(af[1], neg);
            hmul_frag(af[2], neg);
            hmul_frag(af[3], neg);
        });
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) store_h(u[mi], mi, 4, OC_U, LDD, n128, 1.f);
    }
    __syncthreads();
    // ---- c: dU' = M^T dO + diag(f) K dS_next
    {
        float du[2][4][4];
        zero2<4>(du);
        wgemm2<4, 2, true, true>(du, sb + OC_M, LDC, r0, sb + OC_DO, LQ, n128, lane, NoScale2());
        wgemm2<8, 2, false, false>(du, sb + OC_K, LQ, r0, sb + OC_DS, LS, n128, lane, rowscale(fv));
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) store_h(du[mi], mi, 4, OC_W, LDD, n128, 1.f);   // W is dead
    }
    __syncthreads();
    // ---- d: dM = tril(dO U'^T), stored as dM * D
    {
        float dm[2][2][4];
        zero2<2>(dm);
        wgemm2<8, 1, false, false>(dm, sb + OC_DO, LQ, r0, sb + OC_U, LDD, n64, lane, NoScale2());
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) dm[mi][nt][e] *= __half2float(decm[row(mi, e) * LDC + n64 + 8 * nt + 2 * t4 + (e & 1)]);
            store_h(dm[mi], mi, 2, OC_M, LDC, n64, 1.f);   // M is dead
        }
    }
    __syncthreads();
    // ---- e: dQ = diag(Gamma) dO S^T + (dM * D) K
    {
        float dq[2][4][4];
        zero2<4>(dq);
        wgemm2<8, 2, false, true>(dq, sb + OC_DO, LQ, r0, sb + OC_S, LS, n128, lane, NoScale2());
#pragma unroll
        for (int mi = 0; mi < 2; ++mi)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) dq[mi][nt][e] *= Gam[row(mi, e)];
        wgemm2<4, 2, false, true>(dq, sb + OC_M, LDC, r0, sb + OC_K, LQ, n128, lane, NoScale2());
        rowdot(dq, OC_Q, n128, pg);
#pragma unroll
        for (int mi = 0; mi < 2; ++mi)
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) {
                const int r = row(mi, 2 * hi);
                if (c * C + r >= a.T) continue;
                float *dst = a.dq + (((size_t)b * a.T + c * C + r) * a.Hk + hk) * D + n128 + 2 * t4;
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    if (sole) {
                        *reinterpret_cast<float2 *>(dst + 8 * nt) = make_float2(dq[mi][nt][2 * hi], dq[mi][nt][2 * hi + 1]);
                    } else {
                        atomicAdd(dst + 8 * nt, dq[mi][nt][2 * hi]);
                        atomicAdd(dst + 8 * nt + 1, dq[mi][nt][2 * hi + 1]);
                    }
                }
            }
    }
    // ---- f: dK3 = diag(f) U' dS_next^T (the start of dK)
    float dk[2][4][4];
    {
        zero2<4>(dk);
        wgemm2<8, 2, false, true>(dk, sb + OC_U, LDD, r0, sb + OC_DS, LS, n128, lane, NoScale2());
#pragma unroll
        for (int mi = 0; mi < 2; ++mi)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) dk[mi][nt][e] *= fv[row(mi, e)];
        float s[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
        rowdot(dk, OC_K, n128, s);
#pragma unroll
        for (int mi = 0; mi < 2; ++mi)
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) pg[mi][hi] -= s[mi][hi], tot3 += s[mi][hi];
    }
    // ---- g: dW = -dU' S^T, into the dS_next slot once every warp is done with it
    {
        float dw[2][4][4];
        zero2<4>(dw);
        wgemm2<8, 2, false, true>(dw, sb + OC_W, LDD, r0, sb + OC_S, LS, n128, lane, NoScale2());
        __syncthreads();
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) store_h(dw[mi], mi, 4, OC_DS, LDD, n128, -1.f);
    }
    __syncthreads();
    // ---- h: dV = diag(beta) T^T dU', and dK1's first part diag(Gamma beta) T^T dW
    {
        float y[2][4][4], y2[2][4][4];
        zero2<4>(y);
        zero2<4>(y2);
        wgemm2_pair<4, 2, true, true, true, true, true, false>(y, sb + OC_T, LT, sb + OC_W, LDD, NoScale2(), y2,
                                                               sb + OC_T, LT, sb + OC_DS, LDD, NoScale2(), r0, n128, lane);
        rowdot(y, OC_V, n128, pb);   // rowsum(V * T^T dU')
#pragma unroll
        for (int mi = 0; mi < 2; ++mi)
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) {
                const int r = row(mi, 2 * hi);
                if (c * C + r >= a.T) continue;
                const float br = beta[r];
                float *dst = a.dv + (((size_t)b * a.T + c * C + r) * a.Hv + h) * D + n128 + 2 * t4;
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
                    *reinterpret_cast<float2 *>(dst + 8 * nt) = make_float2(br * y[mi][nt][2 * hi], br * y[mi][nt][2 * hi + 1]);
            }
        float s[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
        rowdot(y2, OC_K, n128, s);   // rowsum(K * T^T dW)
#pragma unroll
        for (int mi = 0; mi < 2; ++mi)
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) {
                const int r = row(mi, 2 * hi);
                const float gr = Gam[r], gbr = gr * beta[r];
                pb[mi][hi] += gr * s[mi][hi];
                pg[mi][hi] += gbr * s[mi][hi];   // rowsum(dK1a * K)
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    dk[mi][nt][2 * hi] += gbr * y2[mi][nt][2 * hi];
                    dk[mi][nt][2 * hi + 1] += gbr * y2[mi][nt][2 * hi + 1];
                }
            }
    }
    // ---- i: dT = dU' V^T diag(beta) + dW K^T diag(beta Gamma), into the U' slot (dead after f)
    {
        float x1[2][2][4], x2[2][2][4];
        zero2<2>(x1);
        zero2<2>(x2);
        wgemm2_pair<8, 1, false, false, false, false, false, false>(x1, sb + OC_W, LDD, sb + OC_V, LQ, NoScale2(), x2,
                                                                    sb + OC_DS, LDD, sb + OC_K, LQ, NoScale2(), r0, n64, lane);
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = n64 + 8 * nt + 2 * t4 + (e & 1);
                    x1[mi][nt][e] = beta[i] * (x1[mi][nt][e] + Gam[i] * x2[mi][nt][e]);
                }
            store_h(x1[mi], mi, 2, OC_U, LDC, n64, 1.f);
        }
    }
    __syncthreads();
    // ---- j: X = T^T dT (into the S^T slot), then dA = strict tril(-X T^T)
    {
        float x[2][2][4];
        zero2<2>(x);
        wgemm2<4, 1, true, true>(x, sb + OC_T, LT, r0, sb + OC_U, LDC, n64, lane, NoScale2());
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) store_h(x[mi], mi, 2, OC_S, LDC, n64, 1.f);
    }
    __syncthreads();
    {
        float y[2][2][4];
        zero2<2>(y);
        wgemm2<4, 1, false, false>(y, sb + OC_S, LDC, r0, sb + OC_T, LT, n64, lane, NoScale2());
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = row(mi, e), i = n64 + 8 * nt + 2 * t4 + (e & 1);
                    const float dA = r > i ? -y[mi][nt][e] : 0.f;
                    pb[mi][e >> 1] += dA * __half2float(bmm[r * LDC + i]);
                    y[mi][nt][e] = beta[r] * dA * __half2float(decm[r * LDC + i]);   // dB * D
                }
            store_h(y[mi], mi, 2, OC_U, LDC, n64, 1.f);   // dT is dead (read for X)
        }
    }
    __syncthreads();
    // ---- k: dK1 += (dB * D) K;  dK2 = (dM * D)^T Q + (dB * D)^T K
    {
        float p[2][4][4];
        zero2<4>(p);
        wgemm2<4, 2, false, true>(p, sb + OC_U, LDC, r0, sb + OC_K, LQ, n128, lane, NoScale2());
        rowdot(p, OC_K, n128, pg);
#pragma unroll
        for (int mi = 0; mi < 2; ++mi)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) dk[mi][nt][e] += p[mi][nt][e];
        zero2<4>(p);
        wgemm2<4, 2, true, true>(p, sb + OC_M, LDC, r0, sb + OC_Q, LQ, n128, lane, NoScale2());
        wgemm2<4, 2, true, true>(p, sb + OC_U, LDC, r0, sb + OC_K, LQ, n128, lane, NoScale2());
        float s[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
        rowdot(p, OC_K, n128, s);
#pragma unroll
        for (int mi = 0; mi < 2; ++mi)
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) {
                pg[mi][hi] -= s[mi][hi];
                const int r = row(mi, 2 * hi);
                if (c * C + r >= a.T) continue;
                float *dst = a.dk + (((size_t)b * a.T + c * C + r) * a.Hk + hk) * D + n128 + 2 * t4;
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    const float k0 = dk[mi][nt][2 * hi] + p[mi][nt][2 * hi], k1 = dk[mi][nt][2 * hi + 1] + p[mi][nt][2 * hi + 1];
                    if (sole) {
                        *reinterpret_cast<float2 *>(dst + 8 * nt) = make_float2(k0, k1);
                    } else {
                        atomicAdd(dst + 8 * nt, k0);
                        atomicAdd(dst + 8 * nt + 1, k1);
                    }
                }
            }
    }
    // ---- l: row sums over the warps, then dg (reverse cumulative sum) and dbeta
#pragma unroll
    for (int mi = 0; mi < 2; ++mi)
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
#pragma unroll
            for (int o = 1; o < 4; o <<= 1) {
                pg[mi][hi] += __shfl_xor_sync(0xffffffffu, pg[mi][hi], o);
                pb[mi][hi] += __shfl_xor_sync(0xffffffffu, pb[mi][hi], o);
            }
            if (t4 == 0) {
                vec[VDG + 64 * cw + row(mi, 2 * hi)] = pg[mi][hi];
                vec[VDB + 64 * cw + row(mi, 2 * hi)] = pb[mi][hi];
            }
        }
    tot3 = warp_sum(tot3);
    if (lane == 0) vec[VT3 + warp] = tot3;
    __syncthreads();
    if (warp == 0) {
        float t3 = 0.f, ss = 0.f;
#pragma unroll
        for (int w8 = 0; w8 < 8; ++w8) t3 += vec[VT3 + w8], ss += vec[VSS + w8];
        auto dgrow = [&](int r) { return ((vec[VDG + r] + vec[VDG + 64 + r]) + vec[VDG + 128 + r]) + vec[VDG + 192 + r]; };
        auto dbrow = [&](int r) { return ((vec[VDB + r] + vec[VDB + 64 + r]) + vec[VDB + 128 + r]) + vec[VDB + 192 + r]; };
        // rows 63 - lane and 31 - lane: an inclusive scan over the lanes is the reverse sum
        const float extra = t3 + __expf(G[C - 1]) * ss;
        const int rA = 63 - lane, rB = 31 - lane;
        float x0 = dgrow(rA) + (lane == 0 ? extra : 0.f), x1 = dgrow(rB);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y0 = __shfl_up_sync(0xffffffffu, x0, o), y1 = __shfl_up_sync(0xffffffffu, x1, o);
            if (lane >= o) x0 += y0, x1 += y1;
        }
        x1 += __shfl_sync(0xffffffffu, x0, 31);
        const size_t base = (size_t)b * a.T + c * C;
        if (c * C + rA < a.T) {
            a.dg[(base + rA) * a.Hv + h] = x0;
            a.dbeta[(base + rA) * a.Hv + h] = dbrow(rA);
        }
        if (c * C + rB < a.T) {
            a.dg[(base + rB) * a.Hv + h] = x1;
            a.dbeta[(base + rB) * a.Hv + h] = dbrow(rB);
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
    CUtensorMap mdo;
    if (!make_map(&mdo, a.dout, a.B, a.T, a.Hv, 64, false, true)) return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(bwdc_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_SCAN);
    if (e != cudaSuccess) return e;
    bwdc_scan_kernel<<<(unsigned)(a.B * a.Hv), NT, SMEM_SCAN, st>>>(a, ws, mdo);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bwdc_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_CHUNK);
    if (e != cudaSuccess) return e;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, a.q, a.B, a.T, a.Hk, 64, false, true) || !make_map(&mk, a.k, a.B, a.T, a.Hk, 64, false, true) ||
        !make_map(&mv, a.v, a.B, a.T, a.Hv, 64, false, true))
        return cudaErrorInvalidValue;
    bwdc_chunk_kernel<<<(unsigned)cu, NTC, SMEM_CHUNK, st>>>(a, ws, sm_count(), a.Hv == a.Hk ? 1 : 0, mq, mk, mv, mdo);
    return cudaGetLastError();
}

}  // namespace gdr
