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
//   3. bwdc_tc_kernel: one CTA per (unit, chunk), all chunks at once, on tcgen05 (fp16
//      operands, fp32 accumulators in tensor memory). With the in-chunk decays
//      D_ri = exp(G_r - G_i) (r >= i) and f = Gamma_C / Gamma:
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
// Work whose gradients came out inf or NaN: scan units (their dh0) and chunk CTAs (their dq,
// dk, dv, dg, dbeta). An fp16 operand that overflowed (an input, a stored chunk map, the
// state gradient's copy or a tile formed from them) leaves every product it enters
// non-finite, and every product reaches a gradient, so checking the gradients finds it.
// Threads fold x * 0 (0 for finite x, NaN otherwise): the scan over the dh0 values it
// stores, the chunk kernel over the row sums of dq * q, dk * k and dv * v that its epilogues
// form (every stored element enters one, and a non-finite term never cancels: inf * 0 and
// inf - inf are NaN) and over dg and dbeta.
__device__ unsigned int g_bwdc_range_errors;

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
    __shared__ int abort_sh, range_sh;
    if (tid == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(bar(i), 1);
        abort_sh = 0;
        range_sh = 0;
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
        float nf = 0.f;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            dst[(size_t)i * D] = dS[i];
            nf = fmaf(dS[i], 0.f, nf);
        }
        if (nf != 0.f) range_sh = 1;
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
    if (tid == 0 && range_sh) atomicAdd(&g_bwdc_range_errors, 1u);
}

// ------------------------------------------------------------------ pass 3: per-chunk gradients
// One CTA of 16 warps per (unit, chunk), all chunks at once, every product on tcgen05: M = 128,
// fp16 operands from shared memory, fp32 accumulators in tensor memory, issued by thread 0.
// Most products are taken transposed, feature index by token (W^T, U'^T, dU'^T, dV^T,
// dQ^T, dK^T, ...), so that the 128 features fill the 128 lanes. The token-by-token
// products (dM, X, Y) fill only lanes 0-63: their A operand's rows 64-127 are whatever
// the neighbouring tile holds, and those accumulator rows are never read. The two dT terms
// run as one product of the stacked [dU'; dW] (A, 128 rows) with the stacked [V; K]
// (B, 128 rows), of which two diagonal 64 x 64 blocks are used.
// Warp w reads tensor-memory lanes 32 (w % 4) .. + 31 (thread p = its lane there) and
// columns 16 (w / 4) .. + 15 of each 64-column accumulator.
constexpr int NTT = 512;
constexpr uint32_t QKV_AS = 24576;                    // per 64-feature atom x: V, K, Q tiles at 24576 x + 0, 8192, 16384
constexpr uint32_t O_V = 0, O_K = 8192, O_Q = 16384;  // [64 tokens][64 features] each
constexpr uint32_t O_DO = 49152;                      // dO [token][dv], atoms 8192 apart
constexpr uint32_t O_S = 65536;                       // S^T [dv][dk], atoms 16384 apart; later dB * D [r][i]
constexpr uint32_t O_DS = 98304;                      // dS_next^T [dv][dk]; later fp32 [i][r] hand-over for dT
constexpr uint32_t O_T = 131072;                      // T [r][i]
constexpr uint32_t O_TP = 139264, O_TPP = 147456;     // T diag(beta Gamma), T diag(beta); later dU'^T [dv][r]
constexpr uint32_t O_M = 155648;                      // M [r][i]; later dM * D
constexpr uint32_t O_W = 163840;                      // W^T [dk][r]; later dT [r][i] and X [m][n]
constexpr uint32_t O_U = 180224;                      // U'^T [dv][r]; later dW^T [dk][r]
constexpr uint32_t O_DU = O_TP, O_DW = O_U, O_DMD = O_M, O_DT = O_W, O_X = O_W + 8192, O_DBD = O_S, O_XCH = O_DS;
constexpr uint32_t O_VEC = 196608;
// floats: G, Gamma, beta, f [64]; per lane quarter, the row partial sums of dG and dbeta
// [4][64]; per column quarter, dbeta's dA term [4][64]; per warp, sum(dK3 * K) and
// sum(dS_next * S) [16]
constexpr int W_G = 0, W_GAM = 64, W_BETA = 128, W_F = 192, W_DG = 256, W_DB = 512, W_DA = 768, W_T3 = 1024,
              W_SS = 1040, W_END = 1056;
constexpr uint32_t O_BAR = O_VEC + W_END * 4;         // mbarriers: two loads, seven product batches, drain
constexpr int NB_TC = 10;
constexpr uint32_t SMEM_TC = O_BAR + NB_TC * 8 + 1024;
static_assert(SMEM_TC <= 227 * 1024, "shared memory");
static_assert(O_DW > O_DU, "the stacked [dU'; dW] operand needs a positive atom stride");
// tensor-memory columns (512)
constexpr uint32_t C_G = 0;     // [K; Q] K^T: KK^T (lanes 0-63, kept for dbeta), QK^T (lanes 64-127)
constexpr uint32_t C_A = 64;    // W^T, then dM, then the dT stack (128 columns), then X, then dK1b^T
constexpr uint32_t C_B = 128;   // U'^T, then dW^T, then Y
constexpr uint32_t C_QA = 192;  // S dO^T
constexpr uint32_t C_C = 256;   // dSn^T K^T, then dV^T, then K^T (dM * D)^T
constexpr uint32_t C_D = 320;   // dO^T M, then dK3^T
constexpr uint32_t C_K1A = 384; // dW^T T
constexpr uint32_t C_K2 = 448;  // Q^T (dM * D) + K^T (dB * D)
constexpr uint32_t I_KK = tcu::idesc_f16(128, 64, false, false, false);
constexpr uint32_t I_MK = tcu::idesc_f16(128, 64, false, true, false);
constexpr uint32_t I_KM = tcu::idesc_f16(128, 64, false, false, true);
constexpr uint32_t I_MM = tcu::idesc_f16(128, 64, false, true, true);
constexpr uint32_t I_KM_NEG = tcu::idesc_f16(128, 64, false, false, true, true);
constexpr uint32_t I_MM_NEG = tcu::idesc_f16(128, 64, false, true, true, true);
constexpr uint32_t I_MK_N128 = tcu::idesc_f16(128, 128, false, true, false);

__device__ __forceinline__ void st_h8(uint32_t addr, const float *x)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pack_h2f(x[0], x[1])),
                 "r"(pack_h2f(x[2], x[3])), "r"(pack_h2f(x[4], x[5])), "r"(pack_h2f(x[6], x[7]))
                 : "memory");
}
// 16 consecutive fp32 columns of this thread's lane (32x32b shape) at a0 (and a1), one wait.
__device__ __forceinline__ void tmem_ld16(uint32_t a0, float *v)
{
    uint32_t r[16];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
                 "tcgen05.wait::ld.sync.aligned;"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                   "=r"(r[15])
                 : "r"(a0)
                 : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld16x2(uint32_t a0, uint32_t a1, float *v)
{
    uint32_t r[32];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%32];\n\t"
                 "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%33];\n\t"
                 "tcgen05.wait::ld.sync.aligned;"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                   "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
                   "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
                   "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(a0), "r"(a1)
                 : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// One step of a butterfly reduce-scatter over the warp: lanes with bit W set keep the upper
// W of their first 2W values, the others the lower W, each adding its partner's copy.
template <int W>
__device__ __forceinline__ void rs_step(float *x, int lane)
{
    const bool up = (lane & W) != 0;
#pragma unroll
    for (int j = 0; j < W; ++j) {
        const float send = up ? x[j] : x[j + W];
        const float keep = up ? x[j + W] : x[j];
        x[j] = keep + __shfl_xor_sync(0xffffffffu, send, W);
    }
}
// x[16] per lane; returns, in lanes l and l + 16, the sum of x[l % 16] over the warp's 32
// lanes (16 shuffles, in a fixed order).
__device__ __forceinline__ float warp_rs16(float *x, int lane)
{
    rs_step<8>(x, lane);
    rs_step<4>(x, lane);
    rs_step<2>(x, lane);
    rs_step<1>(x, lane);
    return x[0] + __shfl_xor_sync(0xffffffffu, x[0], 16);
}
__device__ __forceinline__ void prefetch_l2_line(const void *p)
{
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// pf: the CTA that runs pf launches later on this SM (the resident CTA count) gets its inputs
// prefetched into L2 by this one; sole: every key head has one value head, so dq and dk rows
// have one writer and take plain stores.
__global__ void __launch_bounds__(NTT, 1)
bwdc_tc_kernel(BwdArgs a, BwdcWs ws, int pf, int sole, const __grid_constant__ CUtensorMap map_q,
               const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
               const __grid_constant__ CUtensorMap map_do)
{
    using namespace tcu;
    extern __shared__ __align__(1024) uint8_t sm_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q4 = warp & 3, cq = warp >> 2, p = 32 * q4 + lane;
    const int col0 = 16 * cq;   // this thread's first column of a 64-column accumulator
    const int NC = (a.T + C - 1) / C;
    const int unit = blockIdx.x / NC, c = blockIdx.x % NC;
    const int b = unit / a.Hv, h = unit % a.Hv, hk = h / (a.Hv / a.Hk);
    const size_t cu = (size_t)unit * NC + c;
    const int nvalid = min(C, a.T - c * C);
    float *vec = reinterpret_cast<float *>(sm + O_VEC);
    auto bar = [&](int i) { return sb + O_BAR + 8 * i; };   // 0, 1: loads; 2-8: products; 9: drain
    __shared__ uint32_t tmem_sh;
    __shared__ int abort_sh, range_sh;
    if (tid == 0) {
        for (int i = 0; i < NB_TC; ++i) mbar_init(bar(i), 1);
        abort_sh = 0;
        range_sh = 0;
    }
    float nf = 0.f;   // x * 0 folded over the gradients this thread stores (NaN if one is not finite)
    if (warp == 0) tmem_alloc(smem_u32(&tmem_sh), 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = tmem_sh;
    if (tid == 0) {
        const int t0 = c * C;
        mbar_expect_tx(bar(0), 8 * 8192 + 8192);
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            tma_load_4d(sb + O_V + x * QKV_AS, &map_v, 64 * x, h, t0, b, bar(0));
            tma_load_4d(sb + O_K + x * QKV_AS, &map_k, 64 * x, hk, t0, b, bar(0));
            tma_load_4d(sb + O_Q + x * QKV_AS, &map_q, 64 * x, hk, t0, b, bar(0));
            tma_load_4d(sb + O_DO + x * 8192, &map_do, 64 * x, h, t0, b, bar(0));
        }
        bulk_g2s(sb + O_T, ws.t + cu * C * C, 8192, bar(0));
        mbar_expect_tx(bar(1), 2 * 32768);
        bulk_g2s(sb + O_S, ws.s + cu * D * D, 32768, bar(1));
        bulk_g2s(sb + O_DS, ws.ds + cu * D * D, 32768, bar(1));
    }
    auto wait = [&](int i) {
        if (*reinterpret_cast<volatile int *>(&abort_sh)) return;
        if (!mbar_wait_bounded(bar(i), 0)) {
            *reinterpret_cast<volatile int *>(&abort_sh) = 1;
            atomicAdd(&g_bwdc_timeouts, 1u);
        }
    };
    // Every product batch: the operand tiles written by all threads are made visible to the
    // tensor core, the tensor-memory reads of the previous epilogue are ordered before it.
    auto to_issue = [&]() {
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    };
    if (tid >= 64 && tid < 64 + C) {   // (not the warp that issues the copies)
        const int t = c * C + tid - 64;
        const bool ok = t < a.T;
        vec[W_G + tid - 64] = ok ? a.g[((size_t)b * a.T + t) * a.Hv + h] : 0.f;
        vec[W_BETA + tid - 64] = ok ? a.beta[((size_t)b * a.T + t) * a.Hv + h] : 0.f;
    }
    __syncthreads();
    if (warp == 2) {   // in-chunk prefix G, Gamma = exp(G), f = Gamma_C / Gamma
        float x0 = vec[W_G + lane], x1 = vec[W_G + 32 + lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y0 = __shfl_up_sync(0xffffffffu, x0, o), y1 = __shfl_up_sync(0xffffffffu, x1, o);
            if (lane >= o) x0 += y0, x1 += y1;
        }
        x1 += __shfl_sync(0xffffffffu, x0, 31);
        const float GL = __shfl_sync(0xffffffffu, x1, 31);
        vec[W_G + lane] = x0;
        vec[W_G + 32 + lane] = x1;
        vec[W_GAM + lane] = __expf(x0);
        vec[W_GAM + 32 + lane] = __expf(x1);
        vec[W_F + lane] = __expf(GL - x0);
        vec[W_F + 32 + lane] = __expf(GL - x1);
    }
    __syncthreads();
    const float *G = vec + W_G, *Gam = vec + W_GAM, *beta = vec + W_BETA, *fv = vec + W_F;
    // Element (token col0 + j, feature p) of the V, K and Q tiles: byte offset pbase + (j / 8) 1024
    // + xo[j % 8] from the tile's first atom (the 128-byte swizzle of swz_off, with col0 a multiple
    // of 16).
    const uint32_t pbase = (uint32_t)(p >> 6) * QKV_AS + (uint32_t)cq * 2048u + (uint32_t)(p & 7) * 2u;
    uint32_t xo[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) xo[k] = (uint32_t)k * 128u + ((((uint32_t)(p & 63) >> 3) ^ (uint32_t)k) << 4);
    auto colrd = [&](uint32_t tile, int j) {
        return __half2float(*reinterpret_cast<const __half *>(sm + tile + pbase + (uint32_t)(j >> 3) * 1024u + xo[j & 7]));
    };

    // ---- inputs to fp16 in place (V, K, Q, dO: 4096 16-byte words, four loads in flight);
    // T's entries above the diagonal blocks cleared (the forward leaves them unwritten), and
    // T' = T diag(beta Gamma), T'' = T diag(beta)
    wait(0);
#pragma unroll
    for (int j0 = 0; j0 < 8; j0 += 4) {
        uint4 u[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) u[j] = reinterpret_cast<const uint4 *>(sm)[tid + NTT * (j0 + j)];
#pragma unroll
        for (int j = 0; j < 4; ++j) reinterpret_cast<uint4 *>(sm)[tid + NTT * (j0 + j)] = bf16x8_to_f16x8(u[j]);
    }
    {
        const int r = tid >> 3, j = tid & 7;
        uint4 u = *reinterpret_cast<const uint4 *>(sm + swz_chunk(r, j, O_T));
        __half2 *hh = reinterpret_cast<__half2 *>(&u);
        float x[8], y[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = __half22float2(hh[k]);
            x[2 * k] = 8 * j + 2 * k > r ? 0.f : f.x;
            x[2 * k + 1] = 8 * j + 2 * k + 1 > r ? 0.f : f.y;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) y[k] = x[k] * beta[8 * j + k];
        st_h8(sb + swz_chunk(r, j, O_TPP), y);
#pragma unroll
        for (int k = 0; k < 8; ++k) y[k] *= Gam[8 * j + k];
        st_h8(sb + swz_chunk(r, j, O_TP), y);
        st_h8(sb + swz_chunk(r, j, O_T), x);
    }
    to_issue();
    // ---- batch 1: [K; Q] K^T, W^T = K^T T'^T, U^T = V^T T''^T; then (once S and dS_next have
    // landed) S dO^T and dS_next^T K^T
    if (tid == 0) {
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            const uint32_t ko = (s >> 2) * QKV_AS + (s & 3) * 32;
            mma_ss(tb + C_G, sdesc(sb + O_K + ko, 16, 1024), sdesc(sb + O_K + ko, 16, 1024), I_KK, s > 0);
        }
#pragma unroll
        for (int s = 0; s < 4; ++s)
            mma_ss(tb + C_A, sdesc(sb + O_K + s * 2048, QKV_AS, 1024), sdesc(sb + O_TP + s * 32, 16, 1024), I_MK, s > 0);
#pragma unroll
        for (int s = 0; s < 4; ++s)
            mma_ss(tb + C_B, sdesc(sb + O_V + s * 2048, QKV_AS, 1024), sdesc(sb + O_TPP + s * 32, 16, 1024), I_MK, s > 0);
        mma_commit(bar(2));
    }
    wait(1);
    if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int s = 0; s < 8; ++s)
            mma_ss(tb + C_QA, sdesc(sb + O_S + s * 2048, 16384, 1024),
                   sdesc(sb + O_DO + (s >> 2) * 8192 + (s & 3) * 32, 16, 1024), I_MK, s > 0);
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            const uint32_t ko = (s >> 2) * 16384 + (s & 3) * 32;
            mma_ss(tb + C_C, sdesc(sb + O_DS + ko, 16, 1024), sdesc(sb + O_K + (s >> 2) * QKV_AS + (s & 3) * 32, 16, 1024),
                   I_KK, s > 0);
        }
    }
    const long nbk = (long)blockIdx.x + pf;
    if (pf > 0 && nbk < (long)gridDim.x && warp == 1) {
        // the inputs of the CTA pf launches later, into L2 while this one computes (its own
        // loads have landed, so the two do not compete)
        const int nu = (int)(nbk / NC), ncc = (int)(nbk % NC);
        const int n_b = nu / a.Hv, n_h = nu % a.Hv, n_hk = n_h / (a.Hv / a.Hk), nt0 = ncc * C;
        if (lane == 0) {
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
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int t = nt0 + lane + 32 * e;
            if (t < a.T) {
                const size_t ix = ((size_t)n_b * a.T + t) * a.Hv + n_h;
                prefetch_l2_line(a.g + ix);
                prefetch_l2_line(a.beta + ix);
            }
        }
    }
    {   // sum(dS_next * S) over the whole state, while the products run
        float s = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {   // the two images share one layout
            const int i = tid + NTT * k;
            const uint4 ux = *reinterpret_cast<const uint4 *>(sm + O_S + 16 * i);
            const uint4 uy = *reinterpret_cast<const uint4 *>(sm + O_DS + 16 * i);
            const __half2 *x = reinterpret_cast<const __half2 *>(&ux), *y = reinterpret_cast<const __half2 *>(&uy);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 fx = __half22float2(x[e]), fy = __half22float2(y[e]);
                s = fmaf(fx.x, fy.x, fmaf(fx.y, fy.y, s));
            }
        }
        s = warp_sum(s);
        if (lane == 0) vec[W_SS + warp] = s;
    }
    // ---- epilogue 1: M = tril(Q K^T * D) (lanes 64-127), W^T
    wait(2);
    tc_fence_after();
    {
        float v[16];
        if (p >= 64) {
            tmem_ld16(tmem_addr(tb, q4, C_G + col0), v);
            const int r = p - 64;
            const float gr = G[r];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = col0 + j <= r ? v[j] * __expf(gr - G[col0 + j]) : 0.f;
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) st_h8(sb + swz_chunk(r, 2 * cq + jj, O_M), v + 8 * jj);
        }
        tmem_ld16(tmem_addr(tb, q4, C_A + col0), v);
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) st_h8(sb + swz_chunk(p, 2 * cq + jj, O_W), v + 8 * jj);
    }
    to_issue();
    // ---- batch 2: U'^T = U^T - S^T W^T, dO^T M
    if (tid == 0) {
#pragma unroll
        for (int s = 0; s < 8; ++s)
            mma_ss(tb + C_B, sdesc(sb + O_S + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024),
                   sdesc(sb + O_W + s * 2048, 8192, 1024), I_KM_NEG, true);
#pragma unroll
        for (int s = 0; s < 4; ++s)
            mma_ss(tb + C_D, sdesc(sb + O_DO + s * 2048, 8192, 1024), sdesc(sb + O_M + s * 2048, 8192, 1024), I_MM, s > 0);
        mma_commit(bar(3));
    }
    // ---- epilogue 2: U'^T; dU'^T = dO^T M + (dS_next^T K^T) diag(f)
    wait(3);
    tc_fence_after();
    {
        float v[32];
        tmem_ld16(tmem_addr(tb, q4, C_B + col0), v);
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) st_h8(sb + swz_chunk(p, 2 * cq + jj, O_U), v + 8 * jj);
        tmem_ld16x2(tmem_addr(tb, q4, C_D + col0), tmem_addr(tb, q4, C_C + col0), v);
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = fmaf(fv[col0 + j], v[16 + j], v[j]);
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) st_h8(sb + swz_chunk(p, 2 * cq + jj, O_DU), v + 8 * jj);
    }
    to_issue();
    // ---- batch 3: dM = dO U'^T (lanes 0-63), dK3^T = dS_next U'^T, dW^T = -S dU'^T, dV^T = dU'^T T
    if (tid == 0) {
#pragma unroll
        for (int s = 0; s < 8; ++s)
            mma_ss(tb + C_A, sdesc(sb + O_DO + (s >> 2) * 8192 + (s & 3) * 32, 16, 1024),
                   sdesc(sb + O_U + s * 2048, 8192, 1024), I_KM, s > 0);
#pragma unroll
        for (int s = 0; s < 8; ++s)
            mma_ss(tb + C_D, sdesc(sb + O_DS + s * 2048, 16384, 1024), sdesc(sb + O_U + s * 2048, 8192, 1024), I_MM, s > 0);
#pragma unroll
        for (int s = 0; s < 8; ++s)
            mma_ss(tb + C_B, sdesc(sb + O_S + s * 2048, 16384, 1024), sdesc(sb + O_DU + s * 2048, 8192, 1024), I_MM_NEG,
                   s > 0);
#pragma unroll
        for (int s = 0; s < 4; ++s)
            mma_ss(tb + C_C, sdesc(sb + O_DU + s * 32, 16, 1024), sdesc(sb + O_T + s * 2048, 8192, 1024), I_KM, s > 0);
        mma_commit(bar(4));
    }
    // ---- epilogue 3: dM * D (lanes 0-63), dW^T; dV and rowsum(V * T^T dU') once batch 4 is issued
    wait(4);
    tc_fence_after();
    float dv[16];
    {
        float v[16];
        if (p < 64) {
            tmem_ld16(tmem_addr(tb, q4, C_A + col0), v);
            const float gr = G[p];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = col0 + j <= p ? v[j] * __expf(gr - G[col0 + j]) : 0.f;
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) st_h8(sb + swz_chunk(p, 2 * cq + jj, O_DMD), v + 8 * jj);
        }
        tmem_ld16(tmem_addr(tb, q4, C_B + col0), v);
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) st_h8(sb + swz_chunk(p, 2 * cq + jj, O_DW), v + 8 * jj);
        tmem_ld16(tmem_addr(tb, q4, C_C + col0), dv);   // (T^T dU')^T [dv = p][i]
    }
    to_issue();
    // ---- batch 4: dQb^T = K^T (dM * D)^T, dK2^T = Q^T (dM * D), dK1a^T = dW^T T, and the dT stack
    if (tid == 0) {
#pragma unroll
        for (int s = 0; s < 4; ++s)
            mma_ss(tb + C_C, sdesc(sb + O_K + s * 2048, QKV_AS, 1024), sdesc(sb + O_DMD + s * 32, 16, 1024), I_MK, s > 0);
#pragma unroll
        for (int s = 0; s < 4; ++s)
            mma_ss(tb + C_K2, sdesc(sb + O_Q + s * 2048, QKV_AS, 1024), sdesc(sb + O_DMD + s * 2048, 8192, 1024), I_MM,
                   s > 0);
#pragma unroll
        for (int s = 0; s < 4; ++s)
            mma_ss(tb + C_K1A, sdesc(sb + O_DW + s * 32, 16, 1024), sdesc(sb + O_T + s * 2048, 8192, 1024), I_KM, s > 0);
#pragma unroll
        for (int s = 0; s < 8; ++s)
            mma_ss(tb + C_A, sdesc(sb + O_DU + s * 2048, O_DW - O_DU, 1024),
                   sdesc(sb + O_V + (s >> 2) * QKV_AS + (s & 3) * 32, 16, 1024), I_MK_N128, s > 0);
        mma_commit(bar(5));
    }
    {
        float *dst = a.dv + (((size_t)b * a.T + c * C + col0) * a.Hv + h) * D + p;
        const size_t stride = (size_t)a.Hv * D;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int i = col0 + j;
            if (i < nvalid) dst[j * stride] = beta[i] * dv[j];
            dv[j] *= colrd(O_V, j);
        }
        const float s = warp_rs16(dv, lane);
        if (lane < 16) vec[W_DB + 64 * q4 + col0 + lane] = s;
        nf = fmaf(s, 0.f, nf);
    }
    // dQ = diag(Gamma) dO S^T + (dM * D) K (from the two accumulators, which no later batch
    // overwrites) and rowsum(dQ * Q)
    auto dq_out = [&]() {
        float v[32];
        tmem_ld16x2(tmem_addr(tb, q4, C_QA + col0), tmem_addr(tb, q4, C_C + col0), v);
        float *dst = a.dq + (((size_t)b * a.T + c * C + col0) * a.Hk + hk) * D + p;
        const size_t stride = (size_t)a.Hk * D;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int r = col0 + j;
            const float x = fmaf(Gam[r], v[j], v[16 + j]);
            if (r < nvalid) {
                if (sole) dst[j * stride] = x;
                else atomicAdd(dst + j * stride, x);
            }
            v[j] = x * colrd(O_Q, j);
        }
        const float s = warp_rs16(v, lane);
        if (lane < 16) vec[W_DG + 64 * q4 + col0 + lane] = s;
        nf = fmaf(s, 0.f, nf);
    };
    // ---- epilogue 4: dT = (dU' V^T + dW K^T diag(Gamma)) diag(beta). The dW K^T block sits on
    // lanes 64-127, columns 64-127 of the stack, and goes to the dU' V^T block's threads through
    // shared memory. From here the token-by-token chain (X, Y, dA, dB) runs on the warps of
    // lanes 0-63 alone, synchronised among themselves (named barrier 1), while the others write
    // their dQ; the chain's warps write theirs once batch 7 is issued.
    wait(5);
    tc_fence_after();
    float *xch = reinterpret_cast<float *>(sm + O_XCH);   // [i][r]
    if (p >= 64) {
        float v[16];
        tmem_ld16(tmem_addr(tb, q4, C_A + 64 + col0), v);
#pragma unroll
        for (int j = 0; j < 16; ++j) xch[(col0 + j) * C + (p - 64)] = Gam[col0 + j] * v[j];
    }
    tc_fence_before();
    __syncthreads();
    // the chain: fence the written tiles and tensor-memory reads, then sync its 8 warps
    auto chain_sync = [&]() {
        fence_proxy_async();
        tc_fence_before();
        named_bar_sync(1, NTT / 2);
        tc_fence_after();
    };
    if (p < 64) {
        {
            float v[16];
            tmem_ld16(tmem_addr(tb, q4, C_A + col0), v);
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = beta[col0 + j] * (v[j] + xch[(col0 + j) * C + p]);
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) st_h8(sb + swz_chunk(p, 2 * cq + jj, O_DT), v + 8 * jj);
        }
        chain_sync();
        // ---- batch 5: X = T^T dT (lanes 0-63)
        if (tid == 0) {
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_ss(tb + C_A, sdesc(sb + O_T + s * 2048, 8192, 1024), sdesc(sb + O_DT + s * 2048, 8192, 1024), I_MM,
                       s > 0);
            mma_commit(bar(6));
        }
        wait(6);
        tc_fence_after();
        {
            float v[16];
            tmem_ld16(tmem_addr(tb, q4, C_A + col0), v);
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) st_h8(sb + swz_chunk(p, 2 * cq + jj, O_X), v + 8 * jj);
        }
        chain_sync();
        // ---- batch 6: Y = X T^T (lanes 0-63)
        if (tid == 0) {
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_ss(tb + C_B, sdesc(sb + O_X + s * 32, 16, 1024), sdesc(sb + O_T + s * 32, 16, 1024), I_KK, s > 0);
            mma_commit(bar(7));
        }
        // ---- epilogue 6: dA = strict tril(-Y), rowsum(dA * tril(K K^T * D, -1)), dB * D = diag(beta) dA * D
        wait(7);
        tc_fence_after();
        {
            float v[32];
            tmem_ld16x2(tmem_addr(tb, q4, C_B + col0), tmem_addr(tb, q4, C_G + col0), v);
            const float gr = G[p], br = beta[p];
            float s = 0.f;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int i = col0 + j;
                const float d = i < p ? __expf(gr - G[i]) : 0.f;
                const float dA = -v[j];
                s = fmaf(dA * d, v[16 + j], s);
                v[j] = br * dA * d;
            }
            vec[W_DA + 64 * cq + p] = s;
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) st_h8(sb + swz_chunk(p, 2 * cq + jj, O_DBD), v + 8 * jj);
        }
        chain_sync();
        // ---- batch 7: dK1b^T = K^T (dB * D)^T, dK2^T += K^T (dB * D)
        if (tid == 0) {
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_ss(tb + C_A, sdesc(sb + O_K + s * 2048, QKV_AS, 1024), sdesc(sb + O_DBD + s * 32, 16, 1024), I_MK,
                       s > 0);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_ss(tb + C_K2, sdesc(sb + O_K + s * 2048, QKV_AS, 1024), sdesc(sb + O_DBD + s * 2048, 8192, 1024),
                       I_MM, true);
            mma_commit(bar(8));
        }
    }
    dq_out();
    // ---- epilogue 7: dK = diag(f) dK3 + diag(Gamma beta) T^T dW + dK1b + dK2, with the row sums
    // of dG, dbeta and the total sum(dK3 * K)
    wait(8);
    tc_fence_after();
    {
        float v[32], kd[16], gs[16], kv[16], t3 = 0.f;
        tmem_ld16x2(tmem_addr(tb, q4, C_D + col0), tmem_addr(tb, q4, C_K1A + col0), v);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int i = col0 + j;
            kv[j] = colrd(O_K, j);
            const float k3 = fv[i] * v[j], k1 = Gam[i] * beta[i] * v[16 + j];
            kd[j] = k3 + k1;
            gs[j] = kv[j] * (k1 - k3);
            t3 = fmaf(k3, kv[j], t3);
            v[j] = Gam[i] * kv[j] * v[16 + j];   // K * T^T dW, for dbeta
        }
        const float sb_ = warp_rs16(v, lane);
        if (lane < 16) vec[W_DB + 64 * q4 + col0 + lane] += sb_;
        tmem_ld16x2(tmem_addr(tb, q4, C_A + col0), tmem_addr(tb, q4, C_K2 + col0), v);
        float *dst = a.dk + (((size_t)b * a.T + c * C + col0) * a.Hk + hk) * D + p;
        const size_t stride = (size_t)a.Hk * D;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int i = col0 + j;
            const float x = kd[j] + v[j] + v[16 + j];
            gs[j] = fmaf(kv[j], v[j] - v[16 + j], gs[j]);
            if (i < nvalid) {
                if (sole) dst[j * stride] = x;
                else atomicAdd(dst + j * stride, x);
            }
        }
        const float sg = warp_rs16(gs, lane);
        if (lane < 16) vec[W_DG + 64 * q4 + col0 + lane] += sg;
        nf = fmaf(sg, 0.f, fmaf(sb_, 0.f, nf));
        t3 = warp_sum(t3);
        if (lane == 0) vec[W_T3 + warp] = t3;
    }
    tc_fence_before();
    __syncthreads();
    // ---- dg (reverse cumulative sum of the row sums of dG) and dbeta
    if (warp == 0) {
        float t3 = 0.f, ss = 0.f;
#pragma unroll
        for (int w = 0; w < NTT / 32; ++w) t3 += vec[W_T3 + w], ss += vec[W_SS + w];
        auto dgrow = [&](int r) {
            return ((vec[W_DG + r] + vec[W_DG + 64 + r]) + vec[W_DG + 128 + r]) + vec[W_DG + 192 + r];
        };
        auto dbrow = [&](int r) {
            return (((vec[W_DB + r] + vec[W_DB + 64 + r]) + vec[W_DB + 128 + r]) + vec[W_DB + 192 + r]) +
                   (((vec[W_DA + r] + vec[W_DA + 64 + r]) + vec[W_DA + 128 + r]) + vec[W_DA + 192 + r]);
        };
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
        if (rA < nvalid) {
            a.dg[(base + rA) * a.Hv + h] = x0;
            a.dbeta[(base + rA) * a.Hv + h] = dbrow(rA);
            nf = fmaf(x0, 0.f, fmaf(dbrow(rA), 0.f, nf));
        }
        if (rB < nvalid) {
            a.dg[(base + rB) * a.Hv + h] = x1;
            a.dbeta[(base + rB) * a.Hv + h] = dbrow(rB);
            nf = fmaf(x1, 0.f, fmaf(dbrow(rB), 0.f, nf));
        }
    }
    if (nf != 0.f) range_sh = 1;
    if (tid == 0) {   // every product this thread issued has completed before the memory is freed
        tc_fence_after();
        mma_commit(bar(9));
        mbar_wait_bounded(bar(9), 0);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tb, 512);
    }
    if (tid == 0 && range_sh) atomicAdd(&g_bwdc_range_errors, 1u);
}

}  // namespace

unsigned int bwdc_error_counts(unsigned int *timeouts, unsigned int *range_errors)
{
    unsigned int t = 0, r = 0;
    cudaMemcpyFromSymbol(&t, g_bwdc_timeouts, sizeof(t));
    cudaMemcpyFromSymbol(&r, g_bwdc_range_errors, sizeof(r));
    if (timeouts) *timeouts = t;
    if (range_errors) *range_errors = r;
    return t + r;
}

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
    e = cudaFuncSetAttribute(bwdc_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_TC);
    if (e != cudaSuccess) return e;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, a.q, a.B, a.T, a.Hk, 64, false, true) || !make_map(&mk, a.k, a.B, a.T, a.Hk, 64, false, true) ||
        !make_map(&mv, a.v, a.B, a.T, a.Hv, 64, false, true))
        return cudaErrorInvalidValue;
    bwdc_tc_kernel<<<(unsigned)cu, NTT, SMEM_TC, st>>>(a, ws, sm_count(), a.Hv == a.Hk ? 1 : 0, mq, mk, mv, mdo);
    return cudaGetLastError();
}

}  // namespace gdr
