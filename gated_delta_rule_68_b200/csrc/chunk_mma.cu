// Fused chunked forward of the gated delta rule on the warp-level tensor cores:
// mma.sync m16n8k16 with fp16 operands and fp32 accumulators, bf16 inputs,
// Dk = Dv = 128, chunks of C = 64 tokens, for a scalar decay per head (Gated
// DeltaNet) or one per key channel (Kimi Delta Attention). One CTA (8 warps) per
// (batch row, value head), or two splitting the value columns when that still
// fills the SMs in one wave, walks the whole sequence; the fp32 state lives in
// the warps' accumulator registers and never leaves the SM until the final state
// is written.
//
// Method: the exact chunkwise form of
//   S_t = (I - beta_t k_t k_t^T) diag(exp g_t) S_{t-1} + beta_t k_t v_t^T,   o_t = S_t^T q_t
// (NextTransformer, "Source notes", "Linear attention", rows gdn and kda;
// SinkProbe (Attention-Sink) README: its delta-rule layer, evaluated chunk by chunk).
// With G_r = sum_{j<=r} g_j inside the chunk (per channel for the channel gate),
// Gamma_r = exp(G_r), Gamma_C = Gamma_63:
//   A_ri = beta_r sum_c k_rc k_ic exp(G_rc - G_ic)  (i < r),   T = (I + A)^-1
//   W = T diag(beta) (K o Gamma),   U = T diag(beta) V,   U' = U - W S
//   O = (Q o Gamma) S + M U',   M_ri = sum_c q_rc k_ic exp(G_rc - G_ic)  (i <= r)
//   S_next = diag(Gamma_C) S + (K o Gamma_C / Gamma)^T U'
// Scalar gate: the exp factors are per row and fold into the Gram epilogue, into
// T diag(beta Gamma) and into row scalings, all at most 1. Channel gate: the
// Gram's operands carry them, rows of K and Q scaled by exp(G_r - G_31) and rows
// of K by exp(G_31 - G_i), so each factor spans at most 32 tokens of decay (a
// factor outside fp16's range is counted, see gdr_fused_error_counts); the other
// operands carry factors at most 1. The products run on tensor cores; A, the
// diagonal blocks of the inverse and the gate factors are fp32 on CUDA cores.
// fp16 operands (bf16 inputs convert exactly in fp16's normal range) keep the
// result within 2e-2 of the fp64 recurrence by max |error| / rms; inputs and
// states must stay inside the fp16 range (|x| < 6.5e4).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"
#include "mma_util.cuh"

namespace gdr {
namespace {

using namespace mmau;

constexpr int NW = 16;           // warps per CTA
constexpr int NT = 32 * NW;
constexpr int NCB = NW / 4;      // column blocks of the [64 x n] products (4 row blocks of 16)
constexpr int NCS = NW / 8;      // column blocks of the [128 x n] products (8 row blocks of 16)
constexpr int NQ = NT / 64;      // row groups of the per-channel gate pass (one thread per channel pair and group)

// Shared-memory layout (bytes).
constexpr int OFF_K = 0;                        // K [i][dk]
constexpr int OFF_Q = OFF_K + SZ_D;             // Q [r][dk]
constexpr int OFF_V = OFF_Q + SZ_D;             // V [i][dv]
constexpr int OFF_W = OFF_V + SZ_D;             // -W [r][dk]
constexpr int OFF_U = OFF_W + SZ_D;             // U' [i][dv]
constexpr int OFF_UE = OFF_U + SZ_D;            // diag(e) U' [i][dv]
constexpr int OFF_S = OFF_UE + SZ_D;            // S [dk][dv] fp16 copy of the state
constexpr int OFF_M = OFF_S + D * LDD * 2;      // M [r][i]
constexpr int OFF_TB = OFF_M + SZ_C;            // T diag(beta) [r][i]
constexpr int OFF_TG = OFF_TB + SZ_C;           // T diag(beta Gamma) [r][i]
constexpr int OFF_STG = OFF_TG + SZ_C;          // next chunk's K, Q, V as loaded (bf16 [3][64][128])
constexpr int OFF_GST = OFF_STG + 3 * C * D * 2;// next chunk's g and beta (fp32 [2][64])
constexpr int OFF_VEC = OFF_GST + 2 * C * 4;    // G, exp(G), exp(G_C - G), beta (64 fp32 each); NQ x 128 fp32 sums
constexpr int SMEM_BYTES = OFF_VEC + (256 + NQ * 128 + 128 + 256) * 4;
// The scratch of the inverse reuses tiles that are dead while it is live: the
// fp32 diagonal blocks of A sit in the U' tile, the fp16 inverse T in the diag(e)
// U' tile, and the fp16 copy of A (an operand of the block-row products) after
// each warp's 16 x 16 block-row product in the -W tile.
constexpr int LDT = 20;                         // fp32 stride of a transposed 16 x 16 block (conflict-free stores)
constexpr int OFF_A = OFF_U;                    // fp32 [4 blocks][16][LDT], block b holds A_bb transposed
constexpr int OFF_TH = OFF_UE;                  // fp16 T [64][72]
constexpr int OFF_X = OFF_W;                    // fp16 [8 warps][16][24]
constexpr int OFF_AH = OFF_X + 8 * 16 * LDX * 2;// fp16 A [64][72]
static_assert(4 * 16 * LDT * 4 <= SZ_D, "the diagonal blocks of A must fit in the U' tile");
static_assert(C * LDC * 2 <= SZ_D, "T must fit in the diag(e) U' tile");
static_assert(8 * 16 * LDX * 2 + C * LDC * 2 <= SZ_D, "block-row products and A must fit in the W tile");
static_assert(SMEM_BYTES + 1024 <= 227 * 1024, "shared memory");
static_assert(OFF_STG % 128 == 0 && OFF_V % 1024 == 0, "TMA shared-memory alignment (1024 B for the swizzled o tile)");
static_assert(C * D * 4 <= 2 * SZ_D, "an fp32 o tile must fit in the V and W tiles");

// Chunk loads that never completed (each abandons its CTA's remaining chunks), and
// per-channel gate factors that left the fp16 range (their chunk's results are not valid).
__device__ unsigned int g_fused_load_timeouts;
__device__ unsigned int g_fused_range_errors;

// One CTA's part of unit bh = (b, h). GATE 0: one decay per (token, head); GATE 1: one
// per (token, head, key channel). NS: the unit's value columns are split over NS CTAs,
// CTA `split` owning D / NS of them (its part of the state, U, U', O); the Gram, the
// inverse and W are computed by each.
template <typename TOut, int GATE, int NS, bool NORM>
__device__ __forceinline__ void fused_unit(const FwdArgs &a, const CUtensorMap *map_q, const CUtensorMap *map_k,
                                           const CUtensorMap *map_v, const CUtensorMap *map_o,
                                           const CUtensorMap *map_z, int bh, int split)
{
    constexpr int DVC = D / NS;      // value columns of this CTA
    constexpr int NJ = DVC / NCB / 8;   // n8 tiles of a warp in the [64 x DVC] products
    constexpr int NJS = DVC / 4 / 8;    // n8 tiles of a warp's state block (32 rows x DVC / 4)
    constexpr int NJW = D / NCB / 8;    // n8 tiles of a warp in W [64 x 128]
    constexpr int NJG = C / NCS / 8;    // n8 tiles of a warp in the Gram [128 x 64]
    constexpr int RPT = C / NQ;         // GATE 1: rows per thread in the per-channel pass
    extern __shared__ __align__(16) uint8_t smem_raw[];
    // 1024-byte aligned base: the TMA tiles need 128 B, the swizzled o tile 1024 B. An offset
    // into the __shared__ array (not an integer round trip), so that accesses through it stay
    // shared-memory instructions.
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __half *sK = reinterpret_cast<__half *>(sm + OFF_K), *sQ = reinterpret_cast<__half *>(sm + OFF_Q);
    __half *sV = reinterpret_cast<__half *>(sm + OFF_V), *sW = reinterpret_cast<__half *>(sm + OFF_W);
    __half *sU = reinterpret_cast<__half *>(sm + OFF_U), *sUE = reinterpret_cast<__half *>(sm + OFF_UE);
    __half *sS = reinterpret_cast<__half *>(sm + OFF_S), *sM = reinterpret_cast<__half *>(sm + OFF_M);
    __half *sTB = reinterpret_cast<__half *>(sm + OFF_TB), *sTG = reinterpret_cast<__half *>(sm + OFF_TG);
    float *sA = reinterpret_cast<float *>(sm + OFF_A);
    // The per-channel gate needs no T diag(beta Gamma) (Gamma rides on K), and its
    // diag(e) U' tile holds K diag(Gamma_C / Gamma): T goes to the T diag(beta Gamma) tile.
    __half *sAh = reinterpret_cast<__half *>(sm + OFF_AH);
    __half *sTh = reinterpret_cast<__half *>(sm + (GATE ? OFF_TG : OFF_TH));
    float *sG = reinterpret_cast<float *>(sm + OFF_VEC);  // [64] G_r           | GATE 1: [128] exp(G_31)
    float *sEg = sG + 64;                                  // [64] exp(G_r)      |
    float *sEt = sG + 128;                                 // [64] exp(G_C - G_r)
    float *sBeta = sG + 192;                               // [64]
    float *sTot = sG + 256;                                // GATE 1: [NQ][128] per-channel sums of each row group
    float *sP2 = sG + 256 + NQ * 128;                      // GATE 1: [128] exp(G_C - G_31)
    float *sRstd = sP2 + 128;                              // GATE 1, q/k L2 norm: [K rows; Q rows] 1 / |row|
    float *sNW = sRstd + 128;                              // gated output norm: [128] weight
    float *sRowSS = sTot;                                  // gated output norm: [64 rows][4] sums of squares
    float *sColf = sG + 256;                               // GATE 0: [4][64] exp(G_16R - G_i)
    const uint32_t aK = smem_u32(sK), aQ = smem_u32(sQ), aV = smem_u32(sV), aW = smem_u32(sW);
    const uint32_t aU = smem_u32(sU), aUE = smem_u32(sUE), aS = smem_u32(sS), aM = smem_u32(sM);
    const uint32_t aTB = smem_u32(sTB), aTG = smem_u32(sTG), aAh = smem_u32(sAh), aTh = smem_u32(sTh);
    const uint4 *sStg = reinterpret_cast<const uint4 *>(sm + OFF_STG);
    const __nv_bfloat16 *sStgH = reinterpret_cast<const __nv_bfloat16 *>(sm + OFF_STG);
    const float *sGst = reinterpret_cast<const float *>(sm + OFF_GST);   // [64] g, then [64] beta
    const uint32_t aStg = smem_u32(sm + OFF_STG), aGst = smem_u32(sm + OFF_GST);

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31, g = lane >> 2, t4 = lane & 3;
    __half *sXw = reinterpret_cast<__half *>(sm + OFF_X) + w * 16 * LDX;   // this warp's 16 x 16 tile
    const uint32_t aXw = smem_u32(sXw);
    const int dv0 = split * DVC;
    const int b = bh / a.Hv, h = bh % a.Hv, hk = h / (a.Hv / a.Hk);
    // This unit's sequence: tokens tok0 .. tok0 + T - 1 of the token axis; in the tensor
    // maps, batch index tb and token offset tt0. Packed input: sequence b of cu_seqlens
    // (clamped into the token axis), with rows past its end masked below.
    int T = a.T, tb = b, tt0 = 0;
    long tok0 = (long)b * a.T;
    if (a.cu_seqlens) {
        const int s0 = min(max(a.cu_seqlens[b], 0), a.T), s1 = min(max(a.cu_seqlens[b + 1], s0), a.T);
        T = s1 - s0, tb = 0, tt0 = s0, tok0 = s0;
    }
    const int NC = (T + C - 1) / C;

    // Row block (16 rows) and column block of this warp in the [64 x DVC] products,
    // and its 32 x DVC / 4 block of the [128 x DVC] state.
    const int rw0 = 16 * (w & 3), cw0 = (DVC / NCB) * (w >> 2);
    const int rs0 = 32 * (w & 3), cs0 = (DVC / 4) * (w >> 2);

    // State S[:, dv0 .. dv0 + DVC) in registers: warp w holds dk rows rs0 .. rs0 + 31
    // as two m16 tiles; n8 tile j holds local columns cs0 + 8j .. cs0 + 8j + 7.
    float accS[2][NJS][4];
    {
        const float *h0 = a.h0 ? a.h0 + (size_t)bh * D * D + dv0 : nullptr;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            const int r0 = rs0 + 16 * mt + g;
#pragma unroll
            for (int j = 0; j < NJS; ++j) {
                const int c = cs0 + 8 * j + 2 * t4;
                float2 x0 = make_float2(0.f, 0.f), x1 = x0;
                if (h0) {
                    x0 = *reinterpret_cast<const float2 *>(h0 + (size_t)r0 * D + c);
                    x1 = *reinterpret_cast<const float2 *>(h0 + (size_t)(r0 + 8) * D + c);
                }
                float *x = accS[mt][j];
                x[0] = x0.x; x[1] = x0.y; x[2] = x1.x; x[3] = x1.y;
                if (GATE == 0) {   // GATE 1 writes its scaled copy in each chunk's gate pass
                    st_h2(sS + r0 * LDD + c, x0.x, x0.y);
                    st_h2(sS + (r0 + 8) * LDD + c, x1.x, x1.y);
                }
            }
        }
    }

    // Chunk c's K, Q tiles and this CTA's V columns -> bf16 staging by three TMA box
    // loads that complete on ld_bar (tokens past T read as zero); beta, and the
    // scalar gate, by 4-byte asynchronous copies.
    __shared__ uint64_t ld_bar, z_bar;
    const uint32_t aBar = smem_u32(&ld_bar), aZBar = smem_u32(&z_bar);
    if (tid == 0) {
        mbar_init(aBar, 1);
        mbar_init(aZBar, 1);
    }
    if (NORM && a.z && tid < D) sNW[tid] = a.norm_w[tid];
    __syncthreads();
    auto issue_loads = [&](int c) {
        const int t0 = c * C, n = min(C, T - t0);
        // issued by the last warps: warps 0-2 run the inverse right after this
        if (tid == NT - 32) {
            mbar_expect_tx(aBar, (2u * C * D + C * DVC) * 2);
            tma_load_4d(aStg, map_k, 0, hk, tt0 + t0, tb, aBar);
            tma_load_4d(aStg + C * D * 2, map_q, 0, hk, tt0 + t0, tb, aBar);
            tma_load_4d(aStg + 2 * C * D * 2, map_v, dv0, h, tt0 + t0, tb, aBar);
        }
        const int u = tid - (NT - 2 * C);   // [0, C): g of row u, [C, 2C): beta of row u - C
        if (u >= 0 && (GATE == 0 || u >= C)) {
            const int r = u & (C - 1);
            const float *src = u < C ? a.g : a.beta;
            if (r < n) src += (tok0 + t0 + r) * a.Hv + h;
            cp_async4(aGst + u * 4, src, r < n ? 4u : 0u);
        }
        cp_async_commit();
    };
    if (NC > 0) issue_loads(0);
    // GATE 1: this thread's per-channel gates of the next chunk, loaded into registers
    // a chunk ahead so their latency hides behind the current chunk's work.
    float2 gnext[GATE ? RPT : 1];
    auto load_gates = [&](int c) {
        if (GATE) {
            const int t0 = c * C, n = min(C, T - t0), q = tid >> 6;
            const float *gp = a.g + ((tok0 + t0 + RPT * q) * a.Hv + h) * D + 2 * (tid & 63);
            const long gstride = (long)a.Hv * D;
#pragma unroll
            for (int r = 0; r < RPT; ++r)   // rows past the end re-read the last row; the consumer masks them
                gnext[r] = __ldg(reinterpret_cast<const float2 *>(gp + min(r, n - 1 - RPT * q) * gstride));
        }
    };
    if (NC > 0) load_gates(0);

#pragma unroll 1
    for (int ch = 0; ch < NC; ++ch) {
        const int t0 = ch * C, n = min(C, T - t0);
        cp_async_wait_all();
        // The previous chunk's o tile (in the V tile, and for fp32 o also in W) must have
        // been read out before those tiles are rewritten, which first happens in the Gram
        // epilogue: the wait comes just before the barrier that ends the gate pass.
        if (!__syncthreads_and(mbar_wait_bounded(aBar, ch & 1))) {
            if (tid == 0) atomicAdd(&g_fused_load_timeouts, 1u);
            return;
        }

        // ---------------- gates and fp16 operand tiles
        // GATE 1 keeps the prefix G of two channels over RPT rows in registers: thread
        // (p, q) owns key channels 2p, 2p + 1 (p = tid % 64) and rows RPT q .. RPT q + RPT - 1.
        float2 Gv[GATE ? RPT : 1];
        float2 gm = make_float2(0.f, 0.f), gcs = gm;   // GATE 1: G at row 31 and at row 63
        bool bad = false;                              // GATE 1: an operand left the fp16 range
        const int ch_p = tid & 63, ch_h = tid >> 6;
        if (GATE == 0) {
            if (w == 0) {   // G, exp(G), exp(G_C - G)
                const float x0 = sGst[2 * lane], x1 = sGst[2 * lane + 1];
                float s = x0 + x1;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, s, off);
                    if (lane >= off) s += y;
                }
                const float e0 = s - x1, e1 = s;
                const float gc = __shfl_sync(0xffffffffu, s, 31);
                sG[2 * lane] = e0;
                sG[2 * lane + 1] = e1;
                sEg[2 * lane] = __expf(e0);
                sEg[2 * lane + 1] = __expf(e1);
                sEt[2 * lane] = __expf(gc - e0);
                sEt[2 * lane + 1] = __expf(gc - e1);
                // column factors exp(G_16R - G_i) for the Gram rows of block R (i < 16R + 16)
#pragma unroll
                for (int R = 0; R < 4; ++R) {
                    const float gR = __shfl_sync(0xffffffffu, e0, 8 * R);
                    sColf[R * C + 2 * lane] = 2 * lane < 16 * R + 16 ? __expf(gR - e0) : 0.f;
                    sColf[R * C + 2 * lane + 1] = 2 * lane + 1 < 16 * R + 16 ? __expf(gR - e1) : 0.f;
                }
            } else if (w == 2 || w == 3) {
                sBeta[tid - 64] = sGst[C + tid - 64];
            }
#pragma unroll 4
            for (int idx = tid; idx < 2 * C * 16; idx += NT) {   // K and Q (a half warp per row)
                const int which = idx / (C * 16), rem = idx % (C * 16), r = rem >> 4, c16 = rem & 15;
                const uint4 u = sStg[idx];
                uint4 h;
                if (NORM && a.qk_l2norm) {
                    const float ss = halfwarp_sum(bf16x8_sumsq(u));
                    h = bf16x8_scaled_f16x8(u, rsqrtf(ss + 1e-6f));
                } else {
                    h = bf16x8_to_f16x8(u);
                }
                *reinterpret_cast<uint4 *>((which ? sQ : sK) + r * LDD + c16 * 8) = r < n ? h : make_uint4(0, 0, 0, 0);
            }
        } else {
            float2 s = make_float2(0.f, 0.f);
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                if (RPT * ch_h + r < n) { s.x += gnext[r].x; s.y += gnext[r].y; }
                Gv[r] = s;
            }
            *reinterpret_cast<float2 *>(sTot + ch_h * D + 2 * ch_p) = s;
            if (w == 2 || w == 3) sBeta[tid - 64] = sGst[C + tid - 64];
            if (NORM && a.qk_l2norm) {   // 1 / |row| of the 64 K rows and 64 Q rows, a half warp per row
#pragma unroll
                for (int rr = 0; rr < 2 * C / (NT / 16); ++rr) {
                    const int R = (tid >> 4) + rr * (NT / 16);
                    const float ss = halfwarp_sum(bf16x8_sumsq(sStg[R * 16 + (tid & 15)]));
                    if ((tid & 15) == 0) sRstd[R] = rsqrtf(ss + 1e-6f);
                }
            }
            __syncthreads();
            float2 off = make_float2(0.f, 0.f);
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
                const float2 tq = *reinterpret_cast<const float2 *>(sTot + q * D + 2 * ch_p);
                if (q < ch_h) { off.x += tq.x; off.y += tq.y; }
                if (q < NQ / 2) { gm.x += tq.x; gm.y += tq.y; }
                gcs.x += tq.x; gcs.y += tq.y;
            }
#pragma unroll
            for (int r = 0; r < RPT; ++r) { Gv[r].x += off.x; Gv[r].y += off.y; }
            if (ch_h == 0) {   // the state's row factors of these channels (their product is Gamma_C)
                *reinterpret_cast<float2 *>(sG + 2 * ch_p) = make_float2(__expf(gm.x), __expf(gm.y));
                *reinterpret_cast<float2 *>(sP2 + 2 * ch_p) = make_float2(__expf(gcs.x - gm.x), __expf(gcs.y - gm.y));
            }
            // Operands about the reference row 31: rows of K and Q scaled by
            // f1 = exp(G_r - G_31), K by f2 = exp(G_31 - G_r). Each factor spans at most
            // 32 tokens of decay; a product over a pair i <= r is exp(G_r - G_i). The same
            // tiles serve every product of the chunk, with the channel constants moved onto
            // the state: K diag(Gamma) = (K diag f1) diag(exp G_31), Q likewise, and
            // K diag(Gamma_C / Gamma) = (K diag f2) diag(exp(G_C - G_31)). So W is formed
            // from K diag f1, O1 and W S use S' = diag(exp G_31) S, and the state update
            // is S <- diag(exp(G_C - G_31)) (S' + (K diag f2)^T U').
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const int row = RPT * ch_h + r;
                const float2 f1 = make_float2(__expf(Gv[r].x - gm.x), __expf(Gv[r].y - gm.y));
                const float2 f2 = make_float2(__expf(gm.x - Gv[r].x), __expf(gm.y - Gv[r].y));
                float2 kv = make_float2(0.f, 0.f), qv = kv;
                if (row < n) {
                    kv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(sStgH + row * D + 2 * ch_p));
                    qv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(sStgH + C * D + row * D + 2 * ch_p));
                    if (NORM && a.qk_l2norm) {
                        const float rk = sRstd[row], rq = sRstd[C + row];
                        kv.x *= rk; kv.y *= rk; qv.x *= rq; qv.y *= rq;
                    }
                }
                const float2 kr = make_float2(kv.x * f1.x, kv.y * f1.y), qr = make_float2(qv.x * f1.x, qv.y * f1.y);
                const float2 kc = make_float2(kv.x * f2.x, kv.y * f2.y);
                bad |= fmaxf(fmaxf(fabsf(kr.x), fabsf(kr.y)), fmaxf(fmaxf(fabsf(qr.x), fabsf(qr.y)),
                                                                   fmaxf(fabsf(kc.x), fabsf(kc.y)))) > 65504.f;
                *reinterpret_cast<__half2 *>(sK + row * LDD + 2 * ch_p) = __floats2half2_rn(kr.x, kr.y);
                *reinterpret_cast<__half2 *>(sQ + row * LDD + 2 * ch_p) = __floats2half2_rn(qr.x, qr.y);
                *reinterpret_cast<__half2 *>(sUE + row * LDD + 2 * ch_p) = __floats2half2_rn(kc.x, kc.y);
            }
        }
        if (tid == 0) tma_store_wait_read();
        __syncthreads();
        if (GATE) {   // S' = diag(exp G_31) S, this warp's block, as the fp16 operand
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                const int r0 = rs0 + 16 * mt + g;
                const float p0 = sG[r0], p1 = sG[r0 + 8];
#pragma unroll
                for (int j = 0; j < NJS; ++j) {
                    const int c = cs0 + 8 * j + 2 * t4;
                    st_h2(sS + r0 * LDD + c, accS[mt][j][0] * p0, accS[mt][j][1] * p0);
                    st_h2(sS + (r0 + 8) * LDD + c, accS[mt][j][2] * p1, accS[mt][j][3] * p1);
                }
            }
        }

        // ---------------- Gram: warps 0-3 rows of K, warps 4-7 rows of Q, against the
        // 64 key rows (GATE 1: the scaled row and column operands)
        {
            // warp tile: rows 16 (w & 7) of [K ; Q], key rows cg0 .. cg0 + 64 / NCS - 1
            float acc[NJG][4];
#pragma unroll
            for (int j = 0; j < NJG; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
            const bool krow = (w & 7) < 4;
            const int cg0 = (C / NCS) * (w >> 3);
            const uint32_t abase = krow ? aK : aQ, bbase = GATE ? aUE : aK;
            // Only key blocks at or left of the diagonal block are ever used (i <= r).
            if (cg0 <= rw0) {
#pragma unroll
                for (int k0 = 0; k0 < D; k0 += 16) {
                    uint32_t af[4];
                    ldsm(af, a_rm(abase, LDD, rw0, k0, lane));
#pragma unroll
                    for (int np = 0; np < NJG / 2; ++np) {
                        if (cg0 + 16 * np <= rw0) {
                            uint32_t bf[4];
                            ldsm(bf, b_nk(bbase, LDD, cg0 + 16 * np, k0, lane));
                            mma(acc[2 * np], af, bf[0], bf[1]);
                            mma(acc[2 * np + 1], af, bf[2], bf[3]);
                        }
                    }
                }
            }
            // A rows (fp32 and fp16) from warps 0-3; M rows (fp16) from warps 4-7
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int r = rw0 + g + 8 * hh;
                const float rf = GATE ? 1.f : __expf(sG[r] - sG[r & ~15]), br = sBeta[r];
                const float *cf = sColf + (r >> 4) * C;
#pragma unroll
                for (int j = 0; j < NJG; ++j) {
                    const int i = cg0 + 8 * j + 2 * t4;
                    const float d0 = acc[j][2 * hh], d1 = acc[j][2 * hh + 1];
                    const float f0 = GATE ? 1.f : rf * cf[i], f1 = GATE ? 1.f : rf * cf[i + 1];
                    if (krow) {
                        const float x0 = i < r ? br * f0 * d0 : 0.f;
                        const float x1 = i + 1 < r ? br * f1 * d1 : 0.f;
                        if ((i >> 4) == (rw0 >> 4)) {   // diagonal block: fp32, transposed
                            float *at = sA + (rw0 >> 4) * 16 * LDT + (i & 15) * LDT + (r & 15);
                            at[0] = x0;
                            at[LDT] = x1;
                        }
                        st_h2(sAh + r * LDC + i, x0, x1);
                    } else {
                        st_h2(sM + r * LDC + i, i <= r ? f0 * d0 : 0.f, i + 1 <= r ? f1 * d1 : 0.f);
                    }
                }
            }
            if (krow) {
                // T = (I + A)^-1, its 16x16 diagonal block: the warp that holds that block of
                // A solves (I + A_bb) t = e_col by forward substitution in fp32 (lane = column
                // col of the block), column-oriented: once t_i is final, every later t_r
                // takes its A_ri t_i, so the dependent chain is one FMA per pivot.
                const int rb = rw0 >> 4;
                if (rb >= (cg0 >> 4) && rb < (cg0 >> 4) + NJG / 2) {
                    __syncwarp();
                    if (lane < 16) {
                        const int base = 16 * rb, col = lane;
                        const float *at = sA + rb * 16 * LDT;   // at[i * LDT + r] = A[base + r][base + i]
                        float tv[16];
#pragma unroll
                        for (int r = 0; r < 16; ++r) tv[r] = r == col ? 1.f : 0.f;
#pragma unroll
                        for (int i = 0; i < 15; ++i) {
                            float ac[16];
#pragma unroll
                            for (int q4 = i / 4; q4 < 4; ++q4)
                                *reinterpret_cast<float4 *>(ac + 4 * q4) =
                                    *reinterpret_cast<const float4 *>(at + i * LDT + 4 * q4);
#pragma unroll
                            for (int r = i + 1; r < 16; ++r) tv[r] = fmaf(-ac[r], tv[i], tv[r]);
                        }
                        const float bc = sBeta[base + col], bgc = GATE ? 0.f : bc * sEg[base + col];
#pragma unroll
                        for (int r = 0; r < 16; ++r) {
                            const int o = (base + r) * LDC + base + col;
                            sTh[o] = __float2half_rn(tv[r]);
                            sTB[o] = __float2half_rn(tv[r] * bc);
                            if (GATE == 0) sTG[o] = __float2half_rn(tv[r] * bgc);
                        }
                    }
                }
            } else {
                // the Q-row warps: this CTA's V columns to fp16 (the blocks of T above
                // its diagonal are never written: every product skips them)
                const int li = ((w >> 3) * 4 + (w & 7) - 4) * 32 + lane, nli = NT / 2;
                for (int idx = li; idx < C * (DVC / 8); idx += nli) {
                    const int r = idx / (DVC / 8), c8 = idx % (DVC / 8);
                    *reinterpret_cast<uint4 *>(sV + r * LDD + c8 * 8) =
                        r < n ? bf16x8_to_f16x8(sStg[2 * C * 16 + idx]) : make_uint4(0, 0, 0, 0);
                }
            }
        }
        __syncthreads();

        // ---------------- T = (I + A)^-1 (blocks above the diagonal are neither
        // written nor read): the diagonal blocks came with the Gram
        // epilogue; block rows bi = 1..3 on tensor cores, one warp per block (bi, bj):
        //   X = sum_{m=bj}^{bi-1} A_{bi,m} T_{m,bj},   T_{bi,bj} = -T_{bi,bi} X
        // The producers also write T diag(beta) and (GATE 0) T diag(beta Gamma).
        if (ch + 1 < NC) {
            issue_loads(ch + 1);   // the staging area has been consumed
            load_gates(ch + 1);
        }
#pragma unroll 1
        for (int bi = 1; bi < 4; ++bi) {
            if (w < bi) {
                const int bj = w;
                float x[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                for (int m = bj; m < bi; ++m) {
                    uint32_t af[4], bf[4];
                    ldsm(af, a_rm(aAh, LDC, 16 * bi, 16 * m, lane));
                    ldsm_t(bf, b_kn(aTh, LDC, 16 * bj, 16 * m, lane));
                    mma(x[0], af, bf[0], bf[1]);
                    mma(x[1], af, bf[2], bf[3]);
                }
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    st_h2(sXw + g * LDX + 8 * j + 2 * t4, x[j][0], x[j][1]);
                    st_h2(sXw + (g + 8) * LDX + 8 * j + 2 * t4, x[j][2], x[j][3]);
                }
                __syncwarp();
                float y[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                {
                    uint32_t af[4], bf[4];
                    ldsm(af, a_rm(aTh, LDC, 16 * bi, 16 * bi, lane));
                    ldsm_t(bf, b_kn(aXw, LDX, 0, 0, lane));
                    mma(y[0], af, bf[0], bf[1]);
                    mma(y[1], af, bf[2], bf[3]);
                }
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int r0 = 16 * bi + g, c = 16 * bj + 8 * j + 2 * t4;
                    const float b0 = sBeta[c], b1 = sBeta[c + 1];
                    st_h2(sTh + r0 * LDC + c, -y[j][0], -y[j][1]);
                    st_h2(sTh + (r0 + 8) * LDC + c, -y[j][2], -y[j][3]);
                    st_h2(sTB + r0 * LDC + c, -y[j][0] * b0, -y[j][1] * b1);
                    st_h2(sTB + (r0 + 8) * LDC + c, -y[j][2] * b0, -y[j][3] * b1);
                    if (GATE == 0) {
                        const float e0 = b0 * sEg[c], e1 = b1 * sEg[c + 1];
                        st_h2(sTG + r0 * LDC + c, -y[j][0] * e0, -y[j][1] * e1);
                        st_h2(sTG + (r0 + 8) * LDC + c, -y[j][2] * e0, -y[j][3] * e1);
                    }
                }
            }
            __syncthreads();
        }

        // ---------------- W = T diag(beta Gamma) K (GATE 1: T diag(beta) (K diag Gamma)),
        // all 128 key columns, warp tile 16 x 64
        {
            float accW[NJW][4];
#pragma unroll
            for (int j = 0; j < NJW; ++j) accW[j][0] = accW[j][1] = accW[j][2] = accW[j][3] = 0.f;
            const int kw0 = (D / NCB) * (w >> 2);
#pragma unroll
            for (int k0 = 0; k0 < C; k0 += 16) {
                if (k0 > rw0) break;   // T is lower triangular
                uint32_t at[4];
                ldsm(at, a_rm(GATE ? aTB : aTG, LDC, rw0, k0, lane));
#pragma unroll
                for (int np = 0; np < NJW / 2; ++np) {
                    uint32_t bk[4];
                    ldsm_t(bk, b_kn(aK, LDD, kw0 + 16 * np, k0, lane));
                    mma(accW[2 * np], at, bk[0], bk[1]);
                    mma(accW[2 * np + 1], at, bk[2], bk[3]);
                }
            }
#pragma unroll
            for (int j = 0; j < NJW; ++j) {
                const int c = kw0 + 8 * j + 2 * t4;
                if (GATE)   // W carries f1, which can exceed 1
                    bad |= fmaxf(fmaxf(fabsf(accW[j][0]), fabsf(accW[j][1])),
                                 fmaxf(fabsf(accW[j][2]), fabsf(accW[j][3]))) > 65504.f;
                st_h2(sW + (rw0 + g) * LDD + c, -accW[j][0], -accW[j][1]);
                st_h2(sW + (rw0 + g + 8) * LDD + c, -accW[j][2], -accW[j][3]);
            }
        }
        // ---------------- U = T diag(beta) V on this CTA's value columns (warp tile 16 x DVC/2)
        float accU[NJ][4];
#pragma unroll
        for (int j = 0; j < NJ; ++j) accU[j][0] = accU[j][1] = accU[j][2] = accU[j][3] = 0.f;
#pragma unroll
        for (int k0 = 0; k0 < C; k0 += 16) {
            if (k0 > rw0) break;
            uint32_t atb[4];
            ldsm(atb, a_rm(aTB, LDC, rw0, k0, lane));
#pragma unroll
            for (int np = 0; np < NJ / 2; ++np) {
                uint32_t bv[4];
                ldsm_t(bv, b_kn(aV, LDD, cw0 + 16 * np, k0, lane));
                mma(accU[2 * np], atb, bv[0], bv[1]);
                mma(accU[2 * np + 1], atb, bv[2], bv[3]);
            }
        }
        // GATE 1: an fp16 operand of this chunk left the fp16 range (its results are not valid)
        if (__syncthreads_or(bad) && tid == 0 && split == 0)   // once per (unit, chunk)
            atomicAdd(&g_fused_range_errors, 1u);
        // Gated output norm: the chunk's z tile into the V tile (dead from here on), in the
        // 128-byte swizzle of a bf16 o tile, so that each thread later finds its z values
        // where it writes its outputs.
        if (NORM && a.z && tid == NT - 32) {
            mbar_expect_tx(aZBar, C * D * 2);
#pragma unroll
            for (int bx = 0; bx < D / 64; ++bx)
                tma_load_4d(smem_u32(sm + OFF_V + bx * C * 128), map_z, 64 * bx, h, tt0 + t0, tb, aZBar);
        }

        // ---------------- U' = U - W S,  O1 = Q S (GATE 0: then scaled by Gamma_r;
        // GATE 1: Q already carries Gamma), K-dim dk. The fragments of step ks + 1
        // are loaded before the products of step ks.
        float accO[NJ][4];
#pragma unroll
        for (int j = 0; j < NJ; ++j) accO[j][0] = accO[j][1] = accO[j][2] = accO[j][3] = 0.f;
        {
            uint32_t fa[2][2][4], fb[2][NJ / 2][4];   // [buffer][W, Q], [buffer][n16 block]
            auto load = [&](int buf, int k0) {
                ldsm(fa[buf][0], a_rm(aW, LDD, rw0, k0, lane));
                ldsm(fa[buf][1], a_rm(aQ, LDD, rw0, k0, lane));
#pragma unroll
                for (int np = 0; np < NJ / 2; ++np) ldsm_t(fb[buf][np], b_kn(aS, LDD, cw0 + 16 * np, k0, lane));
            };
            load(0, 0);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const int cur = ks & 1;
                if (ks + 1 < D / 16) load(cur ^ 1, 16 * (ks + 1));
#pragma unroll
                for (int np = 0; np < NJ / 2; ++np) {
                    const uint32_t *b = fb[cur][np];
                    mma(accU[2 * np], fa[cur][0], b[0], b[1]);
                    mma(accU[2 * np + 1], fa[cur][0], b[2], b[3]);
                    mma(accO[2 * np], fa[cur][1], b[0], b[1]);
                    mma(accO[2 * np + 1], fa[cur][1], b[2], b[3]);
                }
            }
        }
        {
            const float eg0 = GATE ? 1.f : sEg[rw0 + g], eg1 = GATE ? 1.f : sEg[rw0 + g + 8];
            const float et0 = GATE ? 1.f : sEt[rw0 + g], et1 = GATE ? 1.f : sEt[rw0 + g + 8];
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                accO[j][0] *= eg0; accO[j][1] *= eg0; accO[j][2] *= eg1; accO[j][3] *= eg1;
                const int c = cw0 + 8 * j + 2 * t4;
                st_h2(sU + (rw0 + g) * LDD + c, accU[j][0], accU[j][1]);
                st_h2(sU + (rw0 + g + 8) * LDD + c, accU[j][2], accU[j][3]);
                if (GATE == 0) {
                    st_h2(sUE + (rw0 + g) * LDD + c, accU[j][0] * et0, accU[j][1] * et0);
                    st_h2(sUE + (rw0 + g + 8) * LDD + c, accU[j][2] * et1, accU[j][3] * et1);
                }
            }
        }
        if (NORM && a.z) {   // the barrier also waits for the z tile (issued after W/U)
            if (!__syncthreads_and(mbar_wait_bounded(aZBar, ch & 1))) {
                if (tid == 0) atomicAdd(&g_fused_load_timeouts, 1u);
                return;
            }
        } else {
            __syncthreads();
        }

        // ---------------- O += M U'  and the output rows
#pragma unroll
        for (int k0 = 0; k0 < C; k0 += 16) {
            if (k0 > rw0) break;   // M is lower triangular
            uint32_t am[4];
            ldsm(am, a_rm(aM, LDC, rw0, k0, lane));
#pragma unroll
            for (int np = 0; np < NJ / 2; ++np) {
                uint32_t bu[4];
                ldsm_t(bu, b_kn(aU, LDD, cw0 + 16 * np, k0, lane));
                mma(accO[2 * np], am, bu[0], bu[1]);
                mma(accO[2 * np + 1], am, bu[2], bu[3]);
            }
        }
        if (NORM && a.z) {   // o <- o / sqrt(mean(o^2) + eps) * weight * SiLU(z) per row (the CTA has every column)
            const int r0 = rw0 + g, r1 = rw0 + g + 8;
            uint32_t zr[2][NJ];   // read before the barrier below: an fp32 o tile overwrites other rows' z
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int j = 0; j < NJ; ++j)
                    zr[hh][j] = *reinterpret_cast<const uint32_t *>(
                        sm + OFF_V + o_swz<__nv_bfloat16>(rw0 + g + 8 * hh, cw0 + 8 * j + 2 * t4));
            float ss0 = 0.f, ss1 = 0.f;
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                ss0 = fmaf(accO[j][0], accO[j][0], fmaf(accO[j][1], accO[j][1], ss0));
                ss1 = fmaf(accO[j][2], accO[j][2], fmaf(accO[j][3], accO[j][3], ss1));
            }
#pragma unroll
            for (int off = 1; off < 4; off <<= 1) {
                ss0 += __shfl_xor_sync(0xffffffffu, ss0, off);
                ss1 += __shfl_xor_sync(0xffffffffu, ss1, off);
            }
            if (t4 == 0) {
                sRowSS[r0 * NCB + (w >> 2)] = ss0;
                sRowSS[r1 * NCB + (w >> 2)] = ss1;
            }
            __syncthreads();
            const float4 p0 = *reinterpret_cast<const float4 *>(sRowSS + r0 * NCB);
            const float4 p1 = *reinterpret_cast<const float4 *>(sRowSS + r1 * NCB);
            const float rs[2] = {rsqrtf((p0.x + p0.y + p0.z + p0.w) * (1.f / D) + a.norm_eps),
                                 rsqrtf((p1.x + p1.y + p1.z + p1.w) * (1.f / D) + a.norm_eps)};
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int j = 0; j < NJ; ++j) {
                    const int c = cw0 + 8 * j + 2 * t4;
                    const float2 zf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&zr[hh][j]));
                    accO[j][2 * hh] *= rs[hh] * sNW[c] * __fdividef(zf.x, 1.f + __expf(-zf.x));
                    accO[j][2 * hh + 1] *= rs[hh] * sNW[c + 1] * __fdividef(zf.y, 1.f + __expf(-zf.y));
                }
        }
        {   // o rows -> [DVC / EPB][64 rows][128 B] boxes in the 128-byte swizzle the TMA
            // store expects, over the dead V and W tiles
            const int r0 = rw0 + g, r1 = rw0 + g + 8;
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                const int c = cw0 + 8 * j + 2 * t4;
                store_out2(reinterpret_cast<TOut *>(sm + OFF_V + o_swz<TOut>(r0, c)), accO[j][0], accO[j][1]);
                store_out2(reinterpret_cast<TOut *>(sm + OFF_V + o_swz<TOut>(r1, c)), accO[j][2], accO[j][3]);
            }
            fence_proxy_async();
        }

        // ---------------- S <- Gamma_C S + K^T diag(e) U'  (GATE 1: S <- diag(exp(G_C -
        // G_31)) (diag(exp G_31) S + (K diag f2)^T U')); the warp's 32 x DVC / 4 block
        {
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                const int r0 = rs0 + 16 * mt + g;
                const float gc0 = GATE ? sG[r0] : sEg[C - 1], gc1 = GATE ? sG[r0 + 8] : sEg[C - 1];
#pragma unroll
                for (int j = 0; j < NJS; ++j) {
                    float *x = accS[mt][j];
                    x[0] *= gc0; x[1] *= gc0; x[2] *= gc1; x[3] *= gc1;
                }
            }
            const uint32_t aKs = GATE ? aUE : aK, aUs = GATE ? aU : aUE;
            uint32_t fk[2][2][4], fu[2][NJS / 2][4];   // step ks + 1 loads before step ks products
            auto load = [&](int buf, int k0) {
                ldsm_t(fk[buf][0], a_tr(aKs, LDD, rs0, k0, lane));
                ldsm_t(fk[buf][1], a_tr(aKs, LDD, rs0 + 16, k0, lane));
#pragma unroll
                for (int np = 0; np < NJS / 2; ++np) ldsm_t(fu[buf][np], b_kn(aUs, LDD, cs0 + 16 * np, k0, lane));
            };
            load(0, 0);
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks) {
                const int cur = ks & 1;
                if (ks + 1 < C / 16) load(cur ^ 1, 16 * (ks + 1));
#pragma unroll
                for (int np = 0; np < NJS / 2; ++np) {
                    const uint32_t *b = fu[cur][np];
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt) {
                        mma(accS[mt][2 * np], fk[cur][mt], b[0], b[1]);
                        mma(accS[mt][2 * np + 1], fk[cur][mt], b[2], b[3]);
                    }
                }
            }
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                const int r0 = rs0 + 16 * mt + g;
                const float p0 = GATE ? sP2[r0] : 1.f, p1 = GATE ? sP2[r0 + 8] : 1.f;
#pragma unroll
                for (int j = 0; j < NJS; ++j) {
                    float *x = accS[mt][j];
                    if (GATE) {   // its fp16 copy is written with the next chunk's exp(G_31)
                        x[0] *= p0; x[1] *= p0; x[2] *= p1; x[3] *= p1;
                    } else {
                        const int c = cs0 + 8 * j + 2 * t4;
                        st_h2(sS + r0 * LDD + c, x[0], x[1]);
                        st_h2(sS + (r0 + 8) * LDD + c, x[2], x[3]);
                    }
                }
            }
        }
        __syncthreads();
        if (a.cu_seqlens == nullptr || n == C) {
            if (tid == 0) {
                constexpr int EPB = 128 / sizeof(TOut);   // elements per 128-byte box row
#pragma unroll
                for (int bx = 0; bx < DVC / EPB; ++bx)
                    tma_store_4d(map_o, dv0 + bx * EPB, h, tt0 + t0, tb, smem_u32(sm + OFF_V + bx * C * 128));
            }
        } else {   // the rows after a packed sequence's end belong to the next sequence
            TOut *op = reinterpret_cast<TOut *>(a.o) + ((tok0 + t0) * a.Hv + h) * D + dv0;
            for (int idx = tid; idx < n * DVC; idx += NT) {
                const int r = idx / DVC, c = idx % DVC;
                op[(long)r * a.Hv * D + c] = *reinterpret_cast<const TOut *>(sm + OFF_V + o_swz<TOut>(r, c));
            }
            __syncthreads();
        }
    }
    if (tid == 0) tma_store_wait_all();

    if (a.hT) {
        float *hp = a.hT + (size_t)bh * D * D + dv0;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            const int r0 = rs0 + 16 * mt + g;
#pragma unroll
            for (int j = 0; j < NJS; ++j) {
                const int c = cs0 + 8 * j + 2 * t4;
                const float *x = accS[mt][j];
                *reinterpret_cast<float2 *>(hp + (size_t)r0 * D + c) = make_float2(x[0], x[1]);
                *reinterpret_cast<float2 *>(hp + (size_t)(r0 + 8) * D + c) = make_float2(x[2], x[3]);
            }
        }
    }
}


// Blocks [0, n_whole) each run a whole unit; each later pair of blocks splits one of
// the remaining units by value columns. Whole units are dispatched first, and the
// halves fill the SMs as those free up.
template <typename TOut, int GATE, bool NORM>
__global__ void __launch_bounds__(NT, 1)
fused_fwd_kernel(FwdArgs a, int n_whole, const __grid_constant__ CUtensorMap map_q,
                 const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v1,
                 const __grid_constant__ CUtensorMap map_v2, const __grid_constant__ CUtensorMap map_o,
                 const __grid_constant__ CUtensorMap map_z)
{
    const int blk = blockIdx.x;
    if (blk < n_whole) {
        fused_unit<TOut, GATE, 1, NORM>(a, &map_q, &map_k, &map_v1, &map_o, &map_z, blk, 0);
    } else {
        const int i = blk - n_whole;
        fused_unit<TOut, GATE, 2, NORM>(a, &map_q, &map_k, &map_v2, &map_o, &map_z, n_whole + i / 2, i % 2);
    }
}

// The driver's tensor-map encoder, looked up through the runtime once, so the
// library needs no link-time dependency on the driver library.
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled()
{
    static const EncodeTiledFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return EncodeTiledFn(nullptr);
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// Tensor map of a [B][T][H][128] bf16 (or fp32) tensor for boxes of `cols` channels of 64
// consecutive tokens of one head: dims (d, head, t, b), box (cols, 1, 64, 1).
// Tokens past T read as zero.
bool make_map(CUtensorMap *map, const void *base, int B, int T, int H, int cols, bool f32 = false,
              bool swizzle128 = false)
{
    const cuuint64_t es = f32 ? 4 : 2;
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)D * es, (cuuint64_t)H * D * es, (cuuint64_t)T * H * D * es};
    const cuuint32_t box[4] = {(cuuint32_t)cols, 1, (cuuint32_t)C, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const EncodeTiledFn encode = encode_tiled();
    return encode && encode(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                            const_cast<void *>(base), dims, strides, box,
                            estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess)
        return 0;
    return n;
}

template <typename TOut, int GATE>
cudaError_t launch_g(const FwdArgs &a, cudaStream_t st)
{
    // Whole units while they fit one wave of SMs; when all units fit as halves, every
    // unit is split; when the units past one wave fit as halves in a second, those are.
    const long units = (long)a.B * a.Hv, sms = sm_count();
    long n_whole = units;
    if (a.z) n_whole = units;   // the gated output norm needs every column of a row in one CTA
    else if (2 * units <= sms) n_whole = 0;
    else if (units > sms && 2 * (units - sms) <= sms) n_whole = sms;
    CUtensorMap mq, mk, mv1, mv2, mo, mz;
    const int mb = a.cu_seqlens ? 1 : a.B;   // packed input: one batch row of T tokens
    if (!make_map(&mq, a.q, mb, a.T, a.Hk, D) || !make_map(&mk, a.k, mb, a.T, a.Hk, D) ||
        !make_map(&mv1, a.v, mb, a.T, a.Hv, D) || !make_map(&mv2, a.v, mb, a.T, a.Hv, D / 2) ||
        !make_map(&mo, a.o, mb, a.T, a.Hv, 128 / sizeof(TOut), sizeof(TOut) == 4, true))
        return cudaErrorInvalidValue;
    if (a.z ? !make_map(&mz, a.z, mb, a.T, a.Hv, 64, false, true) : (mz = mo, false))   // z: the bf16 o box
        return cudaErrorInvalidValue;
    const int smem = SMEM_BYTES + 1024;
    // The layer's normalisations are compiled into a separate instance, so a call without
    // them runs the same code as before they existed.
    auto kernel = (a.qk_l2norm || a.z) ? fused_fwd_kernel<TOut, GATE, true> : fused_fwd_kernel<TOut, GATE, false>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const long grid = n_whole + 2 * (units - n_whole);
    kernel<<<(unsigned)grid, NT, smem, st>>>(a, (int)n_whole, mq, mk, mv1, mv2, mo, mz);
    return cudaGetLastError();
}

template <typename TOut>
cudaError_t launch_o(const FwdArgs &a, cudaStream_t st)
{
    return a.gate_mode == 0 ? launch_g<TOut, 0>(a, st) : launch_g<TOut, 1>(a, st);
}

}  // namespace

bool fused_supported(const FwdArgs &a)
{
    return in_bf16(a.dtype) && a.Dk == D && a.Dv == D;
}

cudaError_t launch_fwd_fused(const FwdArgs &a, cudaStream_t st)
{
    return out_f32(a.dtype) ? launch_o<float>(a, st) : launch_o<__nv_bfloat16>(a, st);
}

unsigned int fused_error_counts(unsigned int *load_timeouts, unsigned int *range_errors)
{
    unsigned int t = 0, r = 0;
    cudaMemcpyFromSymbol(&t, g_fused_load_timeouts, sizeof(t));
    cudaMemcpyFromSymbol(&r, g_fused_range_errors, sizeof(r));
    if (load_timeouts) *load_timeouts = t;
    if (range_errors) *range_errors = r;
    return t + r;
}

}  // namespace gdr
