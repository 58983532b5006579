// Chunked forward of the gated delta rule with a scalar decay per head (Gated
// DeltaNet) on the fifth-generation tensor cores: tcgen05.mma with operands in
// shared memory and fp32 accumulators in tensor memory, bf16 inputs,
// Dk = Dv = 128, chunks of C = 64 tokens. One CTA per (batch row, value head).
//
// Method: the exact chunkwise form of
//   S_t = (I - beta_t k_t k_t^T) exp(g_t) S_{t-1} + beta_t k_t v_t^T,   o_t = S_t^T q_t
// (NextTransformer, "Source notes", "Linear attention", row gdn; SinkProbe
// (Attention-Sink) README: its delta-rule layer, evaluated chunk by chunk). Inside a
// chunk, with G_r = sum_{j<=r} g_j, Gamma_r = exp(G_r), Gamma_C = Gamma_63:
//   A_ri = beta_r exp(G_r - G_i) k_r.k_i (i < r),   T = (I + A)^-1
//   W = T diag(beta Gamma) K,   U = T diag(beta) V,   U' = U - W S
//   O = diag(Gamma) Q S + M U',   M_ri = exp(G_r - G_i) q_r.k_i (i <= r)
//   S_next = Gamma_C S + Kt^T U',   Kt = diag(Gamma_C / Gamma) K.
// Substituting U' makes both outputs affine in the entering state S:
//   S_next = Gamma_C S + P S + R,   P = -Kt^T W,  R = Kt^T U
//   O      = Qh S + Uh,             Qh = diag(Gamma) Q - M W,  Uh = M U
// and P, R, Qh, Uh depend on the chunk's inputs alone. So the kernel runs two
// groups of eight warps:
//   - the chunk group (warps 8-15) builds P, R, Qh, Uh for one chunk after the
//     other: the gated Gram epilogue (A and M), the inverse (fp32 16 x 16
//     diagonal blocks, off-diagonal blocks as register-chained warp-level MMAs),
//     then W, U and the four products, all large products on tcgen05;
//   - the state group (warps 0-7) keeps S (fp32 in registers, half a value column
//     per thread) and per chunk issues one batch of MMAs that adds P S to R and
//     Qh S to Uh in tensor memory, then forms S_next = Gamma_C S + (P S + R),
//     writes its fp16 copy (the next batch's operand) and stores o through a
//     swizzled shared-memory tile and TMA. In the rest of its time it readies
//     chunk c + 2: TMA loads, bf16 -> fp16 conversion in place, the gate vectors
//     and the Gram [K; Q] K^T (issued by warp 7).
// The chunk group runs one chunk ahead of the state group, so the inverse and
// the other chunk-local work overlap the state chain, and the state chain of a
// chunk is one MMA batch and two short epilogues.
//
// Per-channel gate (Kimi Delta Attention, "Linear attention", row kda; GATE = 1): G
// and Gamma are per key channel, so the decays no longer factor out of the Gram into
// row and column scalings. Instead the Gram's operands carry them, relative to the
// chunk's row 31 so that each factor spans at most 32 tokens of decay:
//   Ks = K * exp(G - G_31), Qs = Q * exp(G - G_31), Kb = K * exp(G_31 - G),
//   A = tril(diag(beta) Ks Kb^T, -1),  M = tril(Qs Kb^T, 0),  T'' = T diag(beta),
//   W' = T'' Ks (W = W' diag(exp G_31)),  U = T'' V,  Kt = Kb diag(exp(G_C - G_31)),
//   P = -Kt^T W' diag(exp G_31),  R = Kt^T U,  Qh = diag(exp G_31) (Qs - M W')^T ... ^T,
//   S_next = diag(Gamma_C) S + P S + R.
// The column factor of P and the row factor of Qh^T are applied as the state group
// copies them out of tensor memory, and diag(Gamma_C) in its fp32 update. The fp16
// copy of S then lives in tensor memory (the state products read it as their A
// operand there), which frees the shared memory for two Kb tiles.
//
// Precision: products take fp16 operands (bf16 inputs convert exactly inside
// fp16's normal range) with fp32 accumulation; the state carry Gamma_C S is fp32
// and only its product with P uses the fp16 copy of S. q, k, v and the state
// must stay inside the fp16 range (|x| < 6.5e4), and with the per-channel gate
// each factor exp(+-(G - G_31)) too; a unit whose results come out non-finite is counted.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <atomic>
#include <chrono>

#include "common.cuh"
#include "kernels.h"
#include "mma_util.cuh"
#include "tc_util.cuh"

namespace gdr {
namespace {

using namespace mmau;
using namespace tcu;

constexpr int GW = 8;            // warps per group
constexpr int GT = 32 * GW;      // threads per group
constexpr int NTH = 2 * GT;      // warps 0-7: state group, warps 8-15: chunk group

// Shared memory (byte offsets from a 1024-byte aligned base). Operand tiles are
// 128-byte swizzled rows (tc_util.cuh).
constexpr uint32_t STG_BYTES = 49152;           // one chunk's inputs: [K; Q] (2 atoms of 128 rows) and V (2 atoms of 64 rows)
constexpr uint32_t STG_Q = 8192;                //   Q rows start at row 64 of each [K; Q] atom
constexpr uint32_t STG_V = 32768;
constexpr uint32_t OFF_P16 = 2 * STG_BYTES;     // P [dk_out][dk_in] fp16, 2 atoms of 16 KB
constexpr uint32_t OFF_QH16 = OFF_P16 + 32768;  // Qh^T [dk][r] fp16
constexpr uint32_t OFF_ST16 = OFF_QH16 + 16384; // 32 KB: Kt and diag(Gamma), or the per-channel gate's Kb tiles
constexpr uint32_t OFF_R1 = OFF_ST16 + 32768;   // T' and T'' (8 KB each) and the inverse's scratch; then W^T, U^T
constexpr uint32_t OFF_TP = OFF_R1;             // T diag(beta Gamma) [r][i] fp16
constexpr uint32_t OFF_TPP = OFF_R1 + 8192;     // T diag(beta) [r][i] fp16
constexpr uint32_t OFF_W16 = OFF_R1;            // W^T [dk][r] fp16 (written once T', T'' are dead)
constexpr uint32_t OFF_U16 = OFF_R1 + 16384;    // U^T [dv][r] fp16
constexpr uint32_t OFF_INV = OFF_R1 + 16384;    // inverse scratch (dead before U^T is written)
constexpr uint32_t OFF_M16 = OFF_R1 + 32768;    // M [r][i] fp16
constexpr uint32_t OFF_VEC = OFF_M16 + 8192;    // per-chunk vectors (fp32)
// Inverse scratch: fp32 diagonal blocks of A (transposed, [4][16][20]), fp16
// off-diagonal rows 16..63 of A ([48][56]) and fp16 diagonal inverses D_b ([4][16][24]).
constexpr int LDAD = 20, LDA16 = 56, LDT16 = 24;
constexpr uint32_t INV_AD = OFF_INV;
constexpr uint32_t INV_A16 = OFF_INV + 4 * 16 * LDAD * 4;
constexpr uint32_t INV_D = INV_A16 + 48 * LDA16 * 2;
constexpr uint32_t INV_END = INV_D + 4 * 16 * LDT16 * 2;
static_assert(INV_END <= OFF_U16 + 16384, "inverse scratch must fit beside T' and T''");
// vectors
// Per-chunk vectors, two sets (chunk parity): G, Gamma, f = Gamma_C / Gamma, beta,
// beta Gamma, row and column factors of exp(G_r - G_i), Gamma_C.
constexpr int V_G = 0, V_GAM = 64, V_F = 128, V_BETA = 192, V_BG = 256, V_EROW = 320, V_ECOL = 384,
              V_GC = 640, V_SET = 644, V_N = 2 * V_SET;
constexpr uint32_t OFF_NW = OFF_VEC + V_N * 4;    // gated output norm: [128] weight
constexpr uint32_t SMEM_USED = OFF_NW + 128 * 4;
constexpr uint32_t SMEM_TC = SMEM_USED + 1024;
static_assert(SMEM_TC <= 227 * 1024, "shared memory");

// Tensor memory columns (512 allocated): the state product (R, then P S + R), the
// o accumulator (Uh, then Qh S + Uh), the Gram, Qh^T, and W^T / U^T, then P, and
// the fp16 copy of S^T that the state batch reads as its A operand (128 lanes x
// 128 fp16, two per column).
constexpr uint32_t TM_S = 0, TM_O = 128, TM_G = 192, TM_X = 256, TM_Y = 320, TM_S16 = 448;

// Per-channel gate: the S^T region holds the Kb tiles of the two staging buffers
// ([64][128] fp16, two 64-column atoms of 8 KB each), and the vector region per chunk
// parity: beta [64], exp(G_31) [128], Gamma_C [128], exp(G_C - G_31) [128]; then the
// gate pass's per-row-group channel sums [4][128].
constexpr uint32_t OFF_KB = OFF_ST16;
// Scalar gate: the same region holds Kt = diag(Gamma_C / Gamma) K ([64][128] fp16, two 64-column
// atoms of 8 KB) and diag(Gamma) ([64][64] fp16), written while the inverse's chains run.
constexpr uint32_t OFF_KT = OFF_ST16, OFF_DG = OFF_ST16 + 16384;
constexpr int KV_BETA = 0, KV_E31 = 64, KV_GC = 192, KV_ECM = 320, KV_SET = 448, KV_TOT = 2 * KV_SET;
static_assert(OFF_VEC + (KV_TOT + 4 * 128) * 4 <= SMEM_USED, "per-channel vectors must fit the vector region");

// mbarriers
enum {
    B_LD0, B_LD1,   // chunk inputs landed in staging buffer 0 / 1 (TMA)
    B_G0, B_G1,     // Gram of the chunk in staging buffer 0 / 1 done
    B_CV0, B_CV1,   // fp16 tiles and gate vectors of the chunk in buffer 0 / 1 written (128 arrivals)
    B_W,            // W^T, U^T done
    B_P1,           // R, Qh, Uh of a chunk done (M and U^T free)
    B_P,            // P too: all four products of a chunk done (waited on by both groups)
    B_ST,           // state batch done
    B_GE,           // the chunk group has read the Gram out of tensor memory (128 arrivals)
    B_YE,           // the state group has read P and Qh out of Y and X (128 arrivals)
    B_SE,           // the state group has read the state product (128 arrivals)
    B_OE,           // the state group has read the o accumulator (128 arrivals)
    B_DR0, B_DR1, B_DR2,   // end-of-kernel drain of each issuing thread's MMAs
    NBAR
};

constexpr uint32_t ID_GRAM = idesc_f16(128, 64, false, false, false);
constexpr uint32_t ID_WU = idesc_f16(128, 64, false, true, false);
constexpr uint32_t ID_P = idesc_f16(128, 128, false, true, false, true);
constexpr uint32_t ID_R = idesc_f16(128, 128, false, false, true);
constexpr uint32_t ID_X = idesc_f16(128, 64, false, false, false, true);
constexpr uint32_t ID_QG = idesc_f16(128, 64, false, true, false);
constexpr uint32_t ID_UH = idesc_f16(128, 64, false, false, false);
constexpr uint32_t ID_S = idesc_f16(128, 128, false, false, false);
constexpr uint32_t ID_O = idesc_f16(128, 64, false, false, true);

// Waits that timed out (each abandons its CTA's remaining work), and units in which a
// value rounded to an fp16 operand left fp16's range (inf or NaN: that unit's o and hT
// are not valid).
__device__ unsigned int g_tc_timeouts;
__device__ unsigned int g_tc_range_errors;

// Range: an fp16 operand that overflowed (or an inf/NaN input) cannot come out of a tensor-core
// product as a finite value (inf * 0 is NaN, inf + x is inf), and every product feeds either
// the state or o. So a unit whose fp16 operands left the range ends with a non-finite o or
// final state: those are checked (x * 0 is 0 for finite x and NaN otherwise), cheaply and off
// the chunk group's path, and the CTA's flag is raised.
__device__ __forceinline__ bool any_nonfinite32(const float *x)
{
    float z0 = 0.f, z1 = 0.f, z2 = 0.f, z3 = 0.f;
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
        z0 = fmaf(x[i], 0.f, z0);
        z1 = fmaf(x[i + 1], 0.f, z1);
        z2 = fmaf(x[i + 2], 0.f, z2);
        z3 = fmaf(x[i + 3], 0.f, z3);
    }
    return (z0 + z1) + (z2 + z3) != 0.f;
}

__device__ __forceinline__ uint32_t pack_h2(float x, float y)
{
    const __half2 h = __floats2half2_rn(x, y);
    return *reinterpret_cast<const uint32_t *>(&h);
}
// 8 fp32 -> one 16-byte chunk of fp16 at shared address `addr`.
__device__ __forceinline__ void st_chunk8(uint32_t addr, const float *x)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pack_h2(x[0], x[1])),
                 "r"(pack_h2(x[2], x[3])), "r"(pack_h2(x[4], x[5])), "r"(pack_h2(x[6], x[7]))
                 : "memory");
}
// A shared-memory span to global memory by the bulk-copy engine (both 16-byte aligned, a
// multiple of 16 bytes), tracked in this thread's bulk groups.
__device__ __forceinline__ void bulk_s2g(void *gdst, uint32_t ssrc, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(ssrc), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void st_h1(uint8_t *sm, uint32_t off, float x)
{
    *reinterpret_cast<__half *>(sm + off) = __float2half_rn(x);
}

__device__ __forceinline__ void out_store1(float *p, float x) { *p = x; }
__device__ __forceinline__ uint32_t pack_bf2(float x, float y)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
    return *reinterpret_cast<const uint32_t *>(&h);
}
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long *p)
{
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_u64(unsigned long long *p, unsigned long long v)
{
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ void prefetch_l1(const void *p)
{
    asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}
__device__ __forceinline__ void prefetch_l2(const void *p)
{
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}
__device__ __forceinline__ void out_store1(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }
__device__ __forceinline__ void out_store2(float *p, float x, float y) { *reinterpret_cast<float2 *>(p) = make_float2(x, y); }
__device__ __forceinline__ void out_store2(__nv_bfloat16 *p, float x, float y)
{
    *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(x, y);
}

// c (16 x 16, fp32, two n8 tiles) += A (16 x 16 row-major at aA, stride lda) B (16 x 16 stored [k][n] at aB, stride ldb).
__device__ __forceinline__ void mma16(float c0[4], float c1[4], uint32_t aA, int lda, uint32_t aB, int ldb, int lane)
{
    uint32_t af[4], bf[4];
    ldsm(af, a_rm(aA, lda, 0, 0, lane));
    ldsm_t(bf, b_kn(aB, ldb, 0, 0, lane));
    mma(c0, af, bf[0], bf[1]);
    mma(c1, af, bf[2], bf[3]);
}
// The fp32 accumulator of a 16 x 16 product (two n8 tiles) is laid out as the A
// fragment of the next m16n8k16 product: c0 holds columns 0..7, c1 columns 8..15.
__device__ __forceinline__ void acc_to_a(uint32_t a[4], const float c0[4], const float c1[4])
{
    a[0] = pack_h2(c0[0], c0[1]);
    a[1] = pack_h2(c0[2], c0[3]);
    a[2] = pack_h2(c1[0], c1[1]);
    a[3] = pack_h2(c1[2], c1[3]);
}
// c (fresh) = A (fragment in registers) B (16 x 16 stored [k][n] at aB, stride ldb).
__device__ __forceinline__ void mma16r(float c0[4], float c1[4], const uint32_t af[4], uint32_t aB, int ldb, int lane)
{
    uint32_t bf[4];
    ldsm_t(bf, b_kn(aB, ldb, 0, 0, lane));
#pragma unroll
    for (int e = 0; e < 4; ++e) c0[e] = c1[e] = 0.f;
    mma(c0, af, bf[0], bf[1]);
    mma(c1, af, bf[2], bf[3]);
}
// c = (A0 B0) B1 ... : a left-to-right chain; the first factor A0 from shared memory.
__device__ __forceinline__ void chain_start(float c0[4], float c1[4], uint32_t aA, int lda, uint32_t aB, int ldb,
                                            int lane)
{
#pragma unroll
    for (int e = 0; e < 4; ++e) c0[e] = c1[e] = 0.f;
    mma16(c0, c1, aA, lda, aB, ldb, lane);
}
__device__ __forceinline__ void chain_next(float c0[4], float c1[4], uint32_t aB, int ldb, int lane)
{
    uint32_t af[4];
    acc_to_a(af, c0, c1);
    mma16r(c0, c1, af, aB, ldb, lane);
}

// c (16 x 16, two n8 accumulator tiles) (+)= A B, A given by its A fragment and B by the A
// fragment of B^T: the B fragment of columns 8 nt .. 8 nt + 7 of B is registers nt and nt + 2
// of that fragment.
__device__ __forceinline__ void mma16_ff(float c[2][4], const uint32_t a[4], const uint32_t bt[4], bool acc)
{
    if (!acc) {
#pragma unroll
        for (int e = 0; e < 4; ++e) c[0][e] = c[1][e] = 0.f;
    }
    mma(c[0], a, bt[0], bt[2]);
    mma(c[1], a, bt[1], bt[3]);
}

// Writes block (R0.., I0..) of T, given as two n8 tiles times `s`, into T diag(beta Gamma)
// and T diag(beta) (swizzled [r][i] tiles); per-channel gate: T diag(beta) only.
template <int GATE>
__device__ __forceinline__ void st_tblock(uint8_t *sm, int R0, int I0, const float c0[4], const float c1[4], float s,
                                          const float *vec, int lane)
{
    const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const float *c = nt ? c1 : c0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int r = R0 + g + 8 * (e >> 1), i = I0 + 8 * nt + 2 * t4 + (e & 1);
            const float t = s * c[e];
            if (GATE == 0) st_h1(sm, OFF_TP + swz_off(r, i, 0), t * vec[V_BG + i]);
            st_h1(sm, OFF_TPP + swz_off(r, i, 0), t * vec[GATE ? KV_BETA + i : V_BETA + i]);
        }
    }
}

// The backward's forward pass: 8 fp32 values as 8 fp16 at a 16-byte aligned global address.
__device__ __forceinline__ void st_global_h8(void *gp, const float *v)
{
    uint4 u;
    u.x = pack_h2(v[0], v[1]);
    u.y = pack_h2(v[2], v[3]);
    u.z = pack_h2(v[4], v[5]);
    u.w = pack_h2(v[6], v[7]);
    *reinterpret_cast<uint4 *>(gp) = u;
}
// Block (R0.., I0..) of T (two n8 tiles times s) into the chunk's [64][64] fp16 T in global memory,
// as the image of a 128-byte swizzled tile.
__device__ __forceinline__ void st_tglobal(__half *tg, int R0, int I0, const float c0[4], const float c1[4], float s,
                                           int lane)
{
    const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const float *c = nt ? c1 : c0;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int r = R0 + g + 8 * hh, i = I0 + 8 * nt + 2 * t4;
            *reinterpret_cast<uint32_t *>(reinterpret_cast<uint8_t *>(tg) + swz_off(r, i, 0)) =
                pack_h2(s * c[2 * hh], s * c[2 * hh + 1]);
        }
    }
}

// NORM: the layer's options (compiled as a separate instance, so the plain forward runs
// exactly its own code): q and k rows divided by sqrt(sum of squares + 1e-6) as they are
// converted, and o rows replaced by o / sqrt(mean(o^2) + eps) * weight * SiLU(z).
// SAVE (scalar gate, one CTA per unit): the first pass of the chunked backward. Per chunk it
// also writes, as fp16 images of 128-byte swizzled tiles, the entering state S^T, T
// (unscaled; the lower triangle and diagonal blocks) and the P and Qh^T operand tiles to the
// caller's buffers, and stores no o. P, Qh^T and S^T (staged in the P tile once the products
// have read it) go out by bulk copies from shared memory, T from the inverse's registers.
template <typename TOut, bool NORM, int GATE, bool SCHED, bool SAVE = false>
__global__ void __launch_bounds__(NTH, 1)
tc_fwd_kernel(FwdArgs a, const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
              const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_o)
{
    extern __shared__ __align__(16) uint8_t smem_raw[];
    // Offset into the __shared__ array (not an integer round trip), so that accesses
    // through it stay shared-memory instructions.
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sb0 = smem_u32(sm);
    float *vec = reinterpret_cast<float *>(sm + OFF_VEC);
    __shared__ uint64_t bars[NBAR];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;
    __shared__ int range_sh;   // set when this unit's o or final state came out non-finite
    auto bar = [&](int i) { return smem_u32(&bars[i]); };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q4 = warp & 3;          // tensor-memory lane quarter of this warp
    const int p = 32 * q4 + lane;     // row of the 128-row products owned by this thread
    const int hf = (warp >> 2) & 1;   // which half of that row's columns this thread takes
    // Without a schedule the CTA's one unit is blockIdx.x: its batch row, heads, and sequence
    // (tokens tok0 .. tok0 + T - 1 of the token axis; in the tensor maps, batch index tbb
    // and token offset tt0). Packed input: sequence b of cu_seqlens (clamped into the token
    // axis); the rows of its last chunk past its end are zeroed when the chunk is converted,
    // since the loaded tile holds the next sequence there.
    const int u_bh = blockIdx.x, u_b = u_bh / a.Hv, u_h = u_bh % a.Hv, u_hk = u_h / (a.Hv / a.Hk);
    int u_T = a.T, u_tbb = u_b, u_tt0 = 0;
    long u_tok0 = (long)u_b * a.T;
    if (a.cu_seqlens) {
        const int s0 = min(max(a.cu_seqlens[u_b], 0), a.T), s1 = min(max(a.cu_seqlens[u_b + 1], s0), a.T);
        u_T = s1 - s0, u_tbb = 0, u_tt0 = s0, u_tok0 = s0;
    }
    const int u_NC = (u_T + C - 1) / C;
    // The CTA's work, as pieces (unit, chunks [c0, c1)). Without a schedule (a.sched_len == 0)
    // one piece: the whole unit blockIdx.x. With one (fixed-length sequences, more units than
    // SMs), the units' chunks are laid end to end and cut into runs of a.sched_len
    // chunk-steps, run i for CTA i, wrapped as in McNaughton's rule: the unit cut by the end
    // of run i does its first chunks at the start of run i + 1 and its last chunks at the end
    // of run i. The first part leaves its state in the workspace and raises its flag; the
    // last part waits for the flag and starts from that state. A unit has at most sched_len
    // chunks, so its first part always ends before its last part begins. Mbarrier phases and
    // staging buffers follow the CTA's running step count, not the chunk index.
    enum { WHOLE = 0, FIRST = 1, LAST = 2 };
    const int nc_unit = (a.T + C - 1) / C;                 // chunks per unit without cu_seqlens
    const long w_all = (long)a.B * a.Hv * nc_unit;
    // The piece that starts at position pos of this CTA's run (pos < run end): unit, first and
    // end chunk (end -1: the unit's chunk count), kind, and the position after it.
    struct Piece { int u, c0, c1, kind; long next; };
    auto piece_at = [&](long pos) -> Piece {
        Piece pc;
        if (!SCHED) {
            pc.u = blockIdx.x, pc.c0 = 0, pc.c1 = -1, pc.kind = WHOLE, pc.next = 1;
            return pc;
        }
        const long r1 = min((long)(blockIdx.x + 1) * a.sched_len, w_all);
        pc.u = (int)(pos / nc_unit);
        const int cu = (int)(pos % nc_unit);
        pc.next = min(r1, (long)(pc.u + 1) * nc_unit);
        const int len = (int)(pc.next - pos);
        if (cu != 0) pc.c0 = 0, pc.c1 = len, pc.kind = FIRST;
        else if (len < nc_unit) pc.c0 = nc_unit - len, pc.c1 = nc_unit, pc.kind = LAST;
        else pc.c0 = 0, pc.c1 = nc_unit, pc.kind = WHOLE;
        return pc;
    };
    const long run0 = SCHED ? (long)blockIdx.x * a.sched_len : 0;
    const long run1 = SCHED ? min(run0 + a.sched_len, w_all) : 1;
    constexpr int VSET = GATE ? KV_SET : V_SET;   // floats per chunk-parity set of vectors
    static_assert(!(GATE && NORM), "the layer options run on the warp-level kernel with the per-channel gate");

    if (warp == 0) tmem_alloc(smem_u32(&tmem_base_sh), 512);
    if (NORM && a.z && tid < D) reinterpret_cast<float *>(sm + OFF_NW)[tid] = a.norm_w[tid];
    if (tid == 0) {
        const uint32_t counts[NBAR] = {1, 1, 1, 1, GT, GT, 1, 1, 1, 1, GT, GT, GT, GT, 1, 1, 1};
        for (int i = 0; i < NBAR; ++i) mbar_init(bar(i), counts[i]);
        abort_sh = 0;
        range_sh = 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = tmem_base_sh;

    // Bounded wait; after any timeout every later wait of the CTA returns at once, so
    // the two groups still meet at all their barriers and the kernel ends.
    auto wait = [&](int i, uint32_t parity) {
        if (*reinterpret_cast<volatile int *>(&abort_sh)) return;
        if (!mbar_wait_bounded(bar(i), parity)) {
            *reinterpret_cast<volatile int *>(&abort_sh) = 1;
            atomicAdd(&g_tc_timeouts, 1u);
        }
    };

    if (warp >= GW) {
        // ============================ chunk group ============================
        // Per chunk: the gated Gram's epilogue (A, M), the inverse (T diag(beta Gamma),
        // T diag(beta)), W^T and U^T, then P, R, Qh, Uh.
        const int gt = tid - GT;          // 0 .. GT-1
        const int wq = q4;                // warp within a half of the group
        const bool issuer = gt == 0;
        // One piece: unit pu, chunks [pc0, pc1) (pc1 < 0: all of them), the CTA's step count
        // at its first chunk gsb.
        auto chunk_piece = [&](const int pu, const int pc0, const int pc1, const int gsb) {
            // The piece's unit: without a schedule the kernel-level values (computed before the
            // groups split, which keeps the state group's registers within budget); with one,
            // fixed-length sequences.
            const int bh = SCHED ? pu : u_bh;
            const int b = SCHED ? bh / a.Hv : u_b, h = SCHED ? bh % a.Hv : u_h;
            const int hk = SCHED ? h / (a.Hv / a.Hk) : u_hk;
            const int T = SCHED ? a.T : u_T, tbb = SCHED ? b : u_tbb, tt0 = SCHED ? 0 : u_tt0;
            const long tok0 = SCHED ? (long)b * a.T : u_tok0;
            const int NC = SCHED ? nc_unit : u_NC;
            const int c0 = pc0, c1 = pc1 < 0 ? NC : pc1;
            (void)hk, (void)tbb, (void)tt0, (void)tok0, (void)T;
        for (int c = c0; c < c1; ++c) {
            const int gs = gsb + (c - c0);
            const int sb = gs & 1;
            const uint32_t stg = sb0 + sb * STG_BYTES;
            uint8_t *stgp = sm + sb * STG_BYTES;
            const float *vc = vec + sb * VSET;
            __half *tg = SAVE ? reinterpret_cast<__half *>(a.save_t) + ((size_t)bh * NC + c) * (C * C) : nullptr;
            (void)tg;
            wait(B_CV0 + sb, (gs >> 1) & 1);
            // Gram epilogue: A (rows < 64) and M (rows 64..127), columns 32 hf .. 32 hf + 31
            wait(B_G0 + sb, (gs >> 1) & 1);
            tc_fence_after();
            {
                float v[32];
                tmem_ld32(tmem_addr(tb, q4, TM_G + 32 * hf), v);
                tc_fence_before();
                mbar_arrive(bar(B_GE));
                const int r = p & 63, rb = r >> 4;
                const int lim = (p < 64 ? r : r + 1) - 32 * hf;   // A: i < r;  M: i <= r
                if (GATE == 0) {
                    // exp(G_r - G_i) = exp(G_r - G_16R) exp(G_16R - G_i), R = r / 16
                    const float4 *ec4 = reinterpret_cast<const float4 *>(vc + V_ECOL + rb * 64 + 32 * hf);
                    const float rowf = p < 64 ? vc[V_BETA + r] * vc[V_EROW + r] : vc[V_EROW + r];
#pragma unroll
                    for (int i4 = 0; i4 < 8; ++i4) {
                        const float4 e = ec4[i4];
                        const int i = 4 * i4;
                        v[i] = i < lim ? rowf * e.x * v[i] : 0.f;
                        v[i + 1] = i + 1 < lim ? rowf * e.y * v[i + 1] : 0.f;
                        v[i + 2] = i + 2 < lim ? rowf * e.z * v[i + 2] : 0.f;
                        v[i + 3] = i + 3 < lim ? rowf * e.w * v[i + 3] : 0.f;
                    }
                } else {   // the decays ride on the operands: A = beta_r (Ks Kb^T)_ri, M = (Qs Kb^T)_ri
                    const float rowf = p < 64 ? vc[KV_BETA + r] : 1.f;
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = i < lim ? rowf * v[i] : 0.f;
                }
                // The previous chunk's first products are done with M and U^T (the inverse's scratch).
                if (gs >= 1) wait(B_P1, (gs - 1) & 1);
                if (p >= 64) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) st_chunk8(sb0 + swz_chunk(r, 4 * hf + j, OFF_M16), v + 8 * j);
                } else {
                    // fp16 blocks left of the diagonal block (rows 16..63 of A), fp32 diagonal block transposed
                    const uint32_t a16 = sb0 + INV_A16 + (uint32_t)((r - 16) * LDA16) * 2u;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        if (4 * hf + j < 2 * rb) st_chunk8(a16 + 16 * (4 * hf + j), v + 8 * j);
                    if ((rb >> 1) == hf) {
                        float *ad = reinterpret_cast<float *>(sm + INV_AD) + rb * 16 * LDAD + (r - 16 * rb);
                        if (rb & 1) {
#pragma unroll
                            for (int ii = 0; ii < 16; ++ii) ad[ii * LDAD] = v[16 + ii];
                        } else {
#pragma unroll
                            for (int ii = 0; ii < 16; ++ii) ad[ii * LDAD] = v[ii];
                        }
                    }
                }
            }
            fence_proxy_async();
            named_bar_sync(1, GT);

            // ... and with W^T (the tiles of T) before they are rewritten.
            if (gs >= 1) wait(B_P, (gs - 1) & 1);
            // Inverse, level 0: warp wq of the first half inverts the unit lower 16 x 16 block
            // I + N (N = A_bb, b = wq) in the product form
            //   (I + N)^-1 = (I - N)(I + N^2)(I + N^4)(I + N^8)      (N^16 = 0)
            // on the warp-level tensor cores, with the running product carried in fp32. Each
            // power is kept with its transpose: the accumulator of X is the A fragment of X, and
            // the B fragment of X regroups the A fragment of X^T, so no product needs a
            // shared-memory round trip. D_b, the b-th diagonal blocks of T diag(beta Gamma) and
            // T diag(beta) go out as fp16 pairs. The second half zeroes the blocks of T above
            // the diagonal.
            if (hf == 0) {
                const int g8 = lane >> 2, t4 = lane & 3;
                const float *ad = reinterpret_cast<const float *>(sm + INV_AD) + wq * 16 * LDAD;   // ad[i][r] = N[r][i]
                float n[2][4], nt[2][4];
#pragma unroll
                for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int r = g8 + 8 * (e >> 1), col = 8 * tt + 2 * t4 + (e & 1);
                        n[tt][e] = ad[col * LDAD + r];    // N[r][col]
                        nt[tt][e] = ad[r * LDAD + col];   // N^T[r][col]
                    }
                uint32_t aN[4], aNT[4], aP2[4], aP2T[4], aP4[4], aP4T[4], aP8T[4], ax[4];
                acc_to_a(aN, n[0], n[1]);
                acc_to_a(aNT, nt[0], nt[1]);
                float p[2][4], pt[2][4];
                mma16_ff(p, aN, aNT, false);       // N^2
                mma16_ff(pt, aNT, aN, false);      // (N^2)^T
                acc_to_a(aP2, p[0], p[1]);
                acc_to_a(aP2T, pt[0], pt[1]);
                mma16_ff(p, aP2, aP2T, false);     // N^4
                mma16_ff(pt, aP2T, aP2, false);    // (N^4)^T
                acc_to_a(aP4, p[0], p[1]);
                acc_to_a(aP4T, pt[0], pt[1]);
                mma16_ff(pt, aP4T, aP4, false);    // (N^8)^T
                acc_to_a(aP8T, pt[0], pt[1]);
                float x[2][4];                     // X = I - N, then X <- X + X N^(2^j)
#pragma unroll
                for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        x[tt][e] = ((g8 + 8 * (e >> 1)) == (8 * tt + 2 * t4 + (e & 1)) ? 1.f : 0.f) - n[tt][e];
                acc_to_a(ax, x[0], x[1]);
                mma16_ff(x, ax, aP2T, true);
                acc_to_a(ax, x[0], x[1]);
                mma16_ff(x, ax, aP4T, true);
                acc_to_a(ax, x[0], x[1]);
                mma16_ff(x, ax, aP8T, true);
                // x[tt][2h], x[tt][2h + 1] = D_b[r][col], D_b[r][col + 1]: r = g8 + 8h, col = 8tt + 2t4
                const int I0 = 16 * wq;
#pragma unroll
                for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int r = g8 + 8 * hh, col = 8 * tt + 2 * t4, i = I0 + col;
                        const float x0 = x[tt][2 * hh], x1 = x[tt][2 * hh + 1];
                        constexpr int VB = GATE ? KV_BETA : V_BETA;
                        const float w0 = x0 * vc[VB + i], w1 = x1 * vc[VB + i + 1];
                        *reinterpret_cast<uint32_t *>(sm + INV_D + (uint32_t)((wq * 16 + r) * LDT16 + col) * 2u) =
                            pack_h2(x0, x1);
                        *reinterpret_cast<uint32_t *>(sm + OFF_TPP + swz_off(I0 + r, i, 0)) = pack_h2(w0, w1);
                        if (SAVE) *reinterpret_cast<uint32_t *>(reinterpret_cast<uint8_t *>(tg) + swz_off(I0 + r, i, 0)) = pack_h2(x0, x1);
                        if (GATE == 0) {
                            const float u0 = x0 * vc[V_BG + i], u1 = x1 * vc[V_BG + i + 1];
                            *reinterpret_cast<uint32_t *>(sm + OFF_TP + swz_off(I0 + r, i, 0)) = pack_h2(u0, u1);
                        }
                    }
            } else {
                // zero chunks: row u of block R = u / 16, 16-byte chunks 2(R+1) .. 7, of one of the two tiles
                const int u = (gt - GT / 2) & 63, R = u >> 4;
                const uint32_t tile = (gt - GT / 2) < 64 ? OFF_TP : OFF_TPP;
                const uint4 z = make_uint4(0, 0, 0, 0);
                for (int j = 2 * (R + 1); j < 8; ++j) *reinterpret_cast<uint4 *>(sm + swz_chunk(u, j, tile)) = z;
                if (GATE == 0) {   // and diag(Gamma) [r][j] for the Qh product (its previous reader is done)
                    const int ht = gt - GT / 2;
#pragma unroll
                    for (int jj = 0; jj < 512 / (GT / 2); ++jj) {
                        const int e = ht + (GT / 2) * jj, r = e >> 3, j = e & 7;
                        float x[8];
#pragma unroll
                        for (int k = 0; k < 8; ++k) x[k] = (8 * j + k == r) ? vc[V_GAM + r] : 0.f;
                        st_chunk8(sb0 + swz_chunk(r, j, OFF_DG), x);
                    }
                }
            }
            named_bar_sync(1, GT);

            // Off-diagonal blocks of T = (I + A)^-1 (D_b the diagonal inverses): expanding
            //   T_ij = -D_i sum_{j <= m < i} A_im T_mj
            // gives sums of alternating chains D A D A ... D, each evaluated left to right so
            // that every right factor is a D or A tile in shared memory and every partial
            // product stays in registers (the accumulator is the next A fragment).
            //   warp 0: T_10 = -D1 A10 D0,  T_21 = -D2 A21 D1
            //   warp 1: T_32 = -D3 A32 D2,  T_20 = (D2 A21 D1 A10 - D2 A20) D0
            //   warp 2: T_31 = (D3 A32 D2 A21 - D3 A31) D1
            //   warp 3: T_30 = ((D3 A31 - D3 A32 D2 A21) D1 A10 + D3 A32 D2 A20 - D3 A30) D0
            if (hf == 0) {
                const uint32_t aD = sb0 + INV_D, aA16 = sb0 + INV_A16;
                constexpr uint32_t T16B = 16 * LDT16 * 2;   // bytes of one [16][24] fp16 tile
                auto Dt = [&](int i) { return aD + i * T16B; };
                auto At = [&](int i, int j) { return aA16 + ((16 * (i - 1)) * LDA16 + 16 * j) * 2; };
                float c0[4], c1[4], u0[4], u1[4];
                if (wq == 0) {
                    chain_start(c0, c1, Dt(1), LDT16, At(1, 0), LDA16, lane);
                    chain_next(c0, c1, Dt(0), LDT16, lane);
                    st_tblock<GATE>(sm, 16, 0, c0, c1, -1.f, vc, lane);
                    if (SAVE) st_tglobal(tg, 16, 0, c0, c1, -1.f, lane);
                    chain_start(c0, c1, Dt(2), LDT16, At(2, 1), LDA16, lane);
                    chain_next(c0, c1, Dt(1), LDT16, lane);
                    st_tblock<GATE>(sm, 32, 16, c0, c1, -1.f, vc, lane);
                    if (SAVE) st_tglobal(tg, 32, 16, c0, c1, -1.f, lane);
                } else if (wq == 1) {
                    chain_start(c0, c1, Dt(3), LDT16, At(3, 2), LDA16, lane);
                    chain_next(c0, c1, Dt(2), LDT16, lane);
                    st_tblock<GATE>(sm, 48, 32, c0, c1, -1.f, vc, lane);
                    if (SAVE) st_tglobal(tg, 48, 32, c0, c1, -1.f, lane);
                    chain_start(c0, c1, Dt(2), LDT16, At(2, 1), LDA16, lane);
                    chain_next(c0, c1, Dt(1), LDT16, lane);
                    chain_next(c0, c1, At(1, 0), LDA16, lane);
                    chain_start(u0, u1, Dt(2), LDT16, At(2, 0), LDA16, lane);
#pragma unroll
                    for (int e = 0; e < 4; ++e) c0[e] -= u0[e], c1[e] -= u1[e];
                    chain_next(c0, c1, Dt(0), LDT16, lane);
                    st_tblock<GATE>(sm, 32, 0, c0, c1, 1.f, vc, lane);
                    if (SAVE) st_tglobal(tg, 32, 0, c0, c1, 1.f, lane);
                } else if (wq == 2) {
                    chain_start(c0, c1, Dt(3), LDT16, At(3, 2), LDA16, lane);
                    chain_next(c0, c1, Dt(2), LDT16, lane);
                    chain_next(c0, c1, At(2, 1), LDA16, lane);
                    chain_start(u0, u1, Dt(3), LDT16, At(3, 1), LDA16, lane);
#pragma unroll
                    for (int e = 0; e < 4; ++e) c0[e] -= u0[e], c1[e] -= u1[e];
                    chain_next(c0, c1, Dt(1), LDT16, lane);
                    st_tblock<GATE>(sm, 48, 16, c0, c1, 1.f, vc, lane);
                    if (SAVE) st_tglobal(tg, 48, 16, c0, c1, 1.f, lane);
                } else {
                    float q0[4], q1[4], h0[4], h1[4];
                    chain_start(q0, q1, Dt(3), LDT16, At(3, 2), LDA16, lane);   // Q = D3 A32 D2
                    chain_next(q0, q1, Dt(2), LDT16, lane);
                    uint32_t qf[4];
                    acc_to_a(qf, q0, q1);
                    mma16r(h0, h1, qf, At(2, 1), LDA16, lane);                  // Q A21
                    chain_start(u0, u1, Dt(3), LDT16, At(3, 1), LDA16, lane);   // D3 A31
#pragma unroll
                    for (int e = 0; e < 4; ++e) u0[e] -= h0[e], u1[e] -= h1[e];
                    chain_next(u0, u1, Dt(1), LDT16, lane);                     // (D3 A31 - Q A21) D1 A10
                    chain_next(u0, u1, At(1, 0), LDA16, lane);
                    mma16r(h0, h1, qf, At(2, 0), LDA16, lane);                  // Q A20
                    chain_start(c0, c1, Dt(3), LDT16, At(3, 0), LDA16, lane);   // D3 A30
#pragma unroll
                    for (int e = 0; e < 4; ++e) c0[e] = u0[e] + h0[e] - c0[e], c1[e] = u1[e] + h1[e] - c1[e];
                    chain_next(c0, c1, Dt(0), LDT16, lane);
                    st_tblock<GATE>(sm, 48, 0, c0, c1, 1.f, vc, lane);
                    if (SAVE) st_tglobal(tg, 48, 0, c0, c1, 1.f, lane);
                }
            } else if (GATE == 0) {
                // Meanwhile the other half (CUDA cores only, so the chains keep the tensor pipe):
                // Kt = diag(Gamma_C / Gamma) K into its own tile. The previous chunk's products
                // that read it are done (waited before level 0).
                const int ht = gt - GT / 2;   // 0 .. 127
#pragma unroll
                for (int jj = 0; jj < 1024 / (GT / 2); ++jj) {
                    const int e = ht + (GT / 2) * jj, tok = (e >> 3) & 63;
                    const __half2 f = __float2half2_rn(vc[V_F + tok]);   // the fp16 product of fp16 values is exact
                    uint4 u = *(reinterpret_cast<const uint4 *>(stgp + (e >> 9) * 16384) + (e & 511));
                    __half2 *hh = reinterpret_cast<__half2 *>(&u);
#pragma unroll
                    for (int k = 0; k < 4; ++k) hh[k] = __hmul2(hh[k], f);
                    *(reinterpret_cast<uint4 *>(sm + OFF_KT + (e >> 9) * 8192) + (e & 511)) = u;
                }
            }
            fence_proxy_async();
            named_bar_sync(1, GT);

            // W^T = K^T T'^T -> Y[0:64),  U^T = V^T T''^T -> Y[64:128), once the state
            // group has read the previous chunk's P and Qh out of Y and X.
            if (issuer) {
                if (gs >= 1) wait(B_YE, (gs - 1) & 1);
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    const uint64_t bt = sdesc(sb0 + (GATE ? OFF_TPP : OFF_TP) + s * 32, 16, 1024);
                    mma_ss(tb + TM_Y, sdesc(stg + s * 2048, 16384, 1024), bt, ID_WU, s > 0);
                }
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    const uint64_t bt = sdesc(sb0 + OFF_TPP + s * 32, 16, 1024);
                    mma_ss(tb + TM_Y + 64, sdesc(stg + STG_V + s * 2048, 8192, 1024), bt, ID_WU, s > 0);
                }
                mma_commit(bar(B_W));
            }
            wait(B_W, gs & 1);
            tc_fence_after();
            {
                float v[64];
                tmem_ld32x2(tmem_addr(tb, q4, TM_Y + 32 * hf), tmem_addr(tb, q4, TM_Y + 64 + 32 * hf), v);
#pragma unroll
                for (int j = 0; j < 4; ++j) st_chunk8(sb0 + swz_chunk(p, 4 * hf + j, OFF_W16), v + 8 * j);
#pragma unroll
                for (int j = 0; j < 4; ++j) st_chunk8(sb0 + swz_chunk(p, 4 * hf + j, OFF_U16), v + 32 + 8 * j);
            }
            // Per-channel gate: Kt = Kb diag(exp(G_C - G_31)) into the K slot (the W product is done
            // with Ks), and the identity in diag(Gamma)'s place into the dead V tile. (The scalar
            // gate built Kt and diag(Gamma) during the chains.)
            if (GATE == 1) {
#pragma unroll
                for (int jj = 0; jj < 1024 / GT; ++jj) {
                    const int e = gt + GT * jj, tok = (e >> 3) & 63;
                    uint4 *pch = reinterpret_cast<uint4 *>(stgp + (e >> 9) * 16384) + (e & 511);
                    // physical 16-byte chunk e % 8 of row tok holds key channels 8 ((e % 8) ^ (tok % 8)) ..
                    const int ch0 = 64 * (e >> 9) + 8 * ((e & 7) ^ (tok & 7));
                    uint4 u = *(reinterpret_cast<const uint4 *>(sm + OFF_KB + sb * 16384 + (e >> 9) * 8192) + (e & 511));
                    const float4 f0 = *reinterpret_cast<const float4 *>(vc + KV_ECM + ch0);
                    const float4 f1 = *reinterpret_cast<const float4 *>(vc + KV_ECM + ch0 + 4);
                    const float f[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
                    __half2 *hh = reinterpret_cast<__half2 *>(&u);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float2 x = __half22float2(hh[k]);
                        hh[k] = __floats2half2_rn(x.x * f[2 * k], x.y * f[2 * k + 1]);
                    }
                    *pch = u;
                }
#pragma unroll
                for (int jj = 0; jj < 512 / GT; ++jj) {
                    const int e = gt + GT * jj, r = e >> 3, j = e & 7;
                    float x[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) x[k] = (8 * j + k == r) ? 1.f : 0.f;
                    st_chunk8(stg + STG_V + swz_chunk(r, j, 0), x);
                }
            }
            tc_fence_before();
            fence_proxy_async();
            named_bar_sync(1, GT);

            // R^T = U^T Kt -> state product,  X = Q^T diag(Gamma) - W^T M^T -> X,
            // Uh^T = U^T M^T -> o accumulator (these free M and U^T), then P = -Kt^T W -> Y.
            if (issuer) {
                if (gs >= 1) wait(B_SE, (gs - 1) & 1);
                if (gs >= 1) wait(B_OE, (gs - 1) & 1);
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_ss(tb + TM_S, sdesc(sb0 + OFF_U16 + s * 32, 16, 1024),
                           GATE ? sdesc(stg + s * 2048, 16384, 1024) : sdesc(sb0 + OFF_KT + s * 2048, 8192, 1024), ID_R,
                           s > 0);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_ss(tb + TM_X, sdesc(stg + STG_Q + s * 2048, 16384, 1024),
                           GATE ? sdesc(stg + STG_V + s * 32, 16, 1024) : sdesc(sb0 + OFF_DG + s * 32, 16, 1024), ID_QG,
                           s > 0);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_ss(tb + TM_X, sdesc(sb0 + OFF_W16 + s * 32, 16, 1024), sdesc(sb0 + OFF_M16 + s * 32, 16, 1024),
                           ID_X, true);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_ss(tb + TM_O, sdesc(sb0 + OFF_U16 + s * 32, 16, 1024), sdesc(sb0 + OFF_M16 + s * 32, 16, 1024),
                           ID_UH, s > 0);
                mma_commit(bar(B_P1));
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_ss(tb + TM_Y,
                           GATE ? sdesc(stg + s * 2048, 16384, 1024) : sdesc(sb0 + OFF_KT + s * 2048, 8192, 1024),
                           sdesc(sb0 + OFF_W16 + s * 32, 16, 1024), ID_P, s > 0);
                mma_commit(bar(B_P));
            }
        }
        };
        if constexpr (SCHED) {
            int gsb = 0;
            for (long ppos = run0; ppos < run1;) {
                const Piece pcs = piece_at(ppos);
                ppos = pcs.next;
                chunk_piece(pcs.u, pcs.c0, pcs.c1, gsb);
                gsb += pcs.c1 - pcs.c0;
            }
        } else {
            chunk_piece(blockIdx.x, 0, -1, 0);
        }
        if (issuer) {
            mma_commit(bar(B_DR1));
            mbar_wait_bounded(bar(B_DR1), 0);
        }
    } else {
        // ============================ state group ============================
        // Thread (p, hf) owns rows dk = 64 hf .. 64 hf + 63 of value column p of S, in fp32
        // registers. Besides the state step of chunk c, the group readies chunk c + 2: its
        // TMA loads, the bf16 -> fp16 conversion of K, Q and V in place, the gate vectors
        // and the Gram.
        const bool issuer = tid == 0;
        const bool gissuer = tid == 7 * 32;   // the Gram's issuer: warp 7 has no gate-vector work
        // One piece: unit pu, chunks [pc0, pc1) (pc1 < 0: all of them), its kind, and the CTA's
        // step count at its first chunk gsb.
        auto state_piece = [&](const int pu, const int pc0, const int pc1, const int pkind, const int gsb) {
            // The piece's unit: without a schedule the kernel-level values (computed before the
            // groups split, which keeps the state group's registers within budget); with one,
            // fixed-length sequences.
            const int bh = SCHED ? pu : u_bh;
            const int b = SCHED ? bh / a.Hv : u_b, h = SCHED ? bh % a.Hv : u_h;
            const int hk = SCHED ? h / (a.Hv / a.Hk) : u_hk;
            const int T = SCHED ? a.T : u_T, tbb = SCHED ? b : u_tbb, tt0 = SCHED ? 0 : u_tt0;
            const long tok0 = SCHED ? (long)b * a.T : u_tok0;
            const int NC = SCHED ? nc_unit : u_NC;
            const int c0 = pc0, c1 = pc1 < 0 ? NC : pc1;
            (void)hk, (void)tbb, (void)tt0, (void)tok0, (void)T;
        auto issue_loads = [&](int c, int gs) {
            const int sb = gs & 1;
            const uint32_t stg = sb0 + sb * STG_BYTES, bl = bar(B_LD0 + sb);
            const int t0 = tt0 + c * C;
            mbar_expect_tx(bl, STG_BYTES);
            tma_load_4d(stg, &map_k, 0, hk, t0, tbb, bl);
            tma_load_4d(stg + 16384, &map_k, 64, hk, t0, tbb, bl);
            tma_load_4d(stg + STG_Q, &map_q, 0, hk, t0, tbb, bl);
            tma_load_4d(stg + 16384 + STG_Q, &map_q, 64, hk, t0, tbb, bl);
            tma_load_4d(stg + STG_V, &map_v, 0, h, t0, tbb, bl);
            tma_load_4d(stg + STG_V + 8192, &map_v, 64, h, t0, tbb, bl);
        };
        // g and beta of chunk c (zero past T), read by warp 0: lane l has rows l and l + 32.
        auto load_gb = [&](int c, float gb[4]) {
            const int t0 = c * C;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int t = t0 + lane + 32 * e;
                const bool ok = t < T;
                const size_t ix = (size_t)(tok0 + t) * a.Hv + h;
                gb[e] = (GATE == 0 && ok) ? a.g[ix] : 0.f;
                gb[2 + e] = ok ? a.beta[ix] : 0.f;
            }
        };
        // Chunk c's tiles to fp16 in place, then its Gram (warp 7) while warps 0 .. 6 write its
        // gate vectors.
        auto ready_chunk = [&](int c, int gs, const float gb[4]) {
            const int sb = gs & 1;
            uint8_t *stgp = sm + sb * STG_BYTES;
            float *vs = vec + sb * V_SET;
            wait(B_LD0 + sb, (gs >> 1) & 1);
            const int nvalid = min(C, T - c * C);
            if (NORM && a.qk_l2norm) {
                // [K; Q] rows: chunks e and e + 1024 are the two halves of one row, and a row's 8
                // chunks of a half sit in 8 adjacent threads
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int e = tid + GT * j, row = (e >> 3) & 63;
                    uint4 *p0 = reinterpret_cast<uint4 *>(stgp) + e, *p1 = p0 + 1024;
                    const uint4 u0 = *p0, u1 = *p1;
                    float ss = bf16x8_sumsq(u0) + bf16x8_sumsq(u1);
                    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
                    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
                    ss += __shfl_xor_sync(0xffffffffu, ss, 4);
                    const float sc = rsqrtf(ss + 1e-6f);
                    *p0 = row < nvalid ? bf16x8_scaled_f16x8(u0, sc) : make_uint4(0, 0, 0, 0);
                    *p1 = row < nvalid ? bf16x8_scaled_f16x8(u1, sc) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int j = 8; j < 3072 / GT; ++j) {
                    const int e = tid + GT * j, row = ((e - 2048) >> 3) & 63;
                    uint4 *pch = reinterpret_cast<uint4 *>(stgp) + e;
                    *pch = row < nvalid ? bf16x8_to_f16x8(*pch) : make_uint4(0, 0, 0, 0);
                }
            } else {
                // all chunks of [K; Q] (2 atoms of 128 rows, Q from row 64) and V (2 atoms of 64
                // rows), four loads in flight before their conversions
#pragma unroll
                for (int j0 = 0; j0 < 3072 / GT; j0 += 4) {
                    uint4 u[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) u[j] = reinterpret_cast<const uint4 *>(stgp)[tid + GT * (j0 + j)];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int e = tid + GT * (j0 + j);
                        const int row = e < 2048 ? ((e >> 3) & 127) & 63 : ((e - 2048) >> 3) & 63;
                        reinterpret_cast<uint4 *>(stgp)[e] = row < nvalid ? bf16x8_to_f16x8(u[j]) : make_uint4(0, 0, 0, 0);
                    }
                }
            }
            fence_proxy_async();
            named_bar_sync(2, GT);   // every tile of the chunk converted
            if (gissuer) {
                const uint32_t stg = sb0 + sb * STG_BYTES;
                if (gs >= 1) wait(B_GE, (gs - 1) & 1);   // the chunk group has read the previous Gram
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const uint32_t ad = stg + (s >> 2) * 16384 + (s & 3) * 32;
                    mma_ss(tb + TM_G, sdesc(ad, 16, 1024), sdesc(ad, 16, 1024), ID_GRAM, s > 0);
                }
                mma_commit(bar(B_G0 + sb));
            }
            // Gate vectors: warps 0 .. 6 scan G (lane l: rows l, l + 32), then write their shares.
            if (warp < 7) {
                float s0 = gb[0], s1 = gb[1];
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y0 = __shfl_up_sync(0xffffffffu, s0, off), y1 = __shfl_up_sync(0xffffffffu, s1, off);
                    if (lane >= off) s0 += y0, s1 += y1;
                }
                s1 += __shfl_sync(0xffffffffu, s0, 31);
                const float GC = __shfl_sync(0xffffffffu, s1, 31);
                const float G[2] = {s0, s1};
                if (warp == 0) {
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int r = lane + 32 * e;
                        vs[V_G + r] = G[e];
                        vs[V_GAM + r] = __expf(G[e]);
                    }
                    if (lane == 0) vs[V_GC] = __expf(GC);
                } else if (warp == 6) {
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int r = lane + 32 * e;
                        const float be = gb[2 + e];
                        vs[V_F + r] = __expf(GC - G[e]);
                        vs[V_BETA + r] = be;
                        vs[V_BG + r] = be * __expf(G[e]);
                    }
                } else if (warp == 1) {   // exp(G_r - G_16R), R = r / 16
                    const float b0 = __shfl_sync(0xffffffffu, s0, lane & ~15), b1 = __shfl_sync(0xffffffffu, s1, lane & ~15);
                    vs[V_EROW + lane] = __expf(s0 - b0);
                    vs[V_EROW + 32 + lane] = __expf(s1 - b1);
                } else {                  // exp(G_16R - G_i) for R = warp - 2
                    const int rb = warp - 2;
                    const float ref = rb < 2 ? __shfl_sync(0xffffffffu, s0, 16 * rb) : __shfl_sync(0xffffffffu, s1, 16 * (rb - 2));
                    vs[V_ECOL + rb * 64 + lane] = __expf(ref - s0);
                    vs[V_ECOL + rb * 64 + 32 + lane] = __expf(ref - s1);
                }
            }
            mbar_arrive(bar(B_CV0 + sb));
        };

        // Per-channel gate: chunk c's gate pass. Thread (cp, rg) = (tid % 64, tid / 64) owns key
        // channels 2 cp, 2 cp + 1 and rows 16 rg .. 16 rg + 15. G is the in-chunk prefix of g per
        // channel (rows past the sequence's end add 0, so G_31 and G_C stop at its last token);
        // K and Q become Ks = K exp(G - G_31) and Qs = Q exp(G - G_31) in place, Kb = K exp(G_31 - G)
        // goes to the buffer's Kb tile, and V is converted to fp16. Then the Gram [Ks; Qs] Kb^T.
        auto ready_chunk_kda = [&](int c, int gs, const float gb[4]) {
            const int sb = gs & 1;
            uint8_t *stgp = sm + sb * STG_BYTES;
            float *vk = vec + sb * KV_SET;
            float *tot = vec + KV_TOT;
            const int nvalid = min(C, T - c * C);
            const int cp = tid & 63, rg = tid >> 6, r0 = 16 * rg;
            float2 gq[16];
            {
                const float *gp = a.g + ((size_t)(tok0 + (long)c * C + r0) * a.Hv + h) * D + 2 * cp;
                const size_t gs = (size_t)a.Hv * D;
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    gq[i] = r0 + i < nvalid ? __ldg(reinterpret_cast<const float2 *>(gp + (size_t)i * gs))
                                            : make_float2(0.f, 0.f);
            }
            wait(B_LD0 + sb, (gs >> 1) & 1);
#pragma unroll
            for (int j = 0; j < 1024 / GT; ++j) {   // V (2 atoms of 64 rows) to fp16, rows past the end zeroed
                const int e = tid + GT * j, row = (e >> 3) & 63;
                uint4 *pch = reinterpret_cast<uint4 *>(stgp + STG_V) + e;
                const uint4 hv = row < nvalid ? bf16x8_to_f16x8(*pch) : make_uint4(0, 0, 0, 0);
                *pch = hv;
            }
            float2 run = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                run.x += gq[i].x;
                run.y += gq[i].y;
                gq[i] = run;
            }
            reinterpret_cast<float2 *>(tot + rg * D)[cp] = run;
            named_bar_sync(2, GT);   // the row groups' sums
            const float2 t0 = reinterpret_cast<const float2 *>(tot)[cp], t1 = reinterpret_cast<const float2 *>(tot + D)[cp],
                         t2 = reinterpret_cast<const float2 *>(tot + 2 * D)[cp];
            const float2 g31 = make_float2(t0.x + t1.x, t0.y + t1.y);
            const float2 off = rg == 0 ? make_float2(0.f, 0.f)
                               : rg == 1 ? t0 : rg == 2 ? g31 : make_float2(g31.x + t2.x, g31.y + t2.y);
            if (rg == 0) {
                const float2 t3 = reinterpret_cast<const float2 *>(tot + 3 * D)[cp];
                const float2 gc = make_float2(g31.x + t2.x + t3.x, g31.y + t2.y + t3.y);
                reinterpret_cast<float2 *>(vk + KV_E31)[cp] = make_float2(__expf(g31.x), __expf(g31.y));
                reinterpret_cast<float2 *>(vk + KV_GC)[cp] = make_float2(__expf(gc.x), __expf(gc.y));
                reinterpret_cast<float2 *>(vk + KV_ECM)[cp] = make_float2(__expf(gc.x - g31.x), __expf(gc.y - g31.y));
            }
            if (warp == 0) {
                vk[KV_BETA + lane] = gb[2];
                vk[KV_BETA + 32 + lane] = gb[3];
            }
            uint8_t *kbp = sm + OFF_KB + sb * 16384;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = r0 + i;
                const float gx = off.x + gq[i].x, gy = off.y + gq[i].y;
                const float e1x = __expf(gx - g31.x), e1y = __expf(gy - g31.y);
                const float e2x = __expf(g31.x - gx), e2y = __expf(g31.y - gy);
                const uint32_t ok = swz_off(r, 2 * cp, 16384), oq = swz_off(64 + r, 2 * cp, 16384);
                const float2 kf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(stgp + ok));
                const float2 qf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(stgp + oq));
                const bool live = r < nvalid;
                const uint32_t ks = live ? pack_h2(kf.x * e1x, kf.y * e1y) : 0u;
                const uint32_t qs = live ? pack_h2(qf.x * e1x, qf.y * e1y) : 0u;
                const uint32_t kb = live ? pack_h2(kf.x * e2x, kf.y * e2y) : 0u;
                *reinterpret_cast<uint32_t *>(stgp + ok) = ks;
                *reinterpret_cast<uint32_t *>(stgp + oq) = qs;
                *reinterpret_cast<uint32_t *>(kbp + swz_off(r, 2 * cp, 8192)) = kb;
            }
            fence_proxy_async();
            named_bar_sync(2, GT);   // every tile of the chunk written
            if (gissuer) {
                const uint32_t stg = sb0 + sb * STG_BYTES, kbs = sb0 + OFF_KB + sb * 16384;
                if (gs >= 1) wait(B_GE, (gs - 1) & 1);   // the chunk group has read the previous Gram
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_ss(tb + TM_G, sdesc(stg + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024),
                           sdesc(kbs + (s >> 2) * 8192 + (s & 3) * 32, 16, 1024), ID_GRAM, s > 0);
                mma_commit(bar(B_G0 + sb));
            }
            mbar_arrive(bar(B_CV0 + sb));
        };
        auto ready = [&](int c, int gs, const float gb[4]) {
            if (GATE) ready_chunk_kda(c, gs, gb);
            else ready_chunk(c, gs, gb);
        };
        float S[64];
        // The fp16 copy of the state S^T [dv][dk]: a shared-memory operand tile, or for the
        // per-channel gate tensor-memory columns TM_S16 + 32 hf .. of lane p (two dk per column).
        // Per-channel gate: the copy read by chunk cn is S~ = diag(exp G_31) S with chunk cn's G_31:
        // then P S = P' S~ and Qh S = X' S~ with P' = -Kt^T W' and X' = (Qs - M W')^T ^T as the chunk
        // group leaves them in tensor memory, so neither needs a scaling on its way out.
        auto store_s16 = [&](int gsn) {
            if (GATE == 0) {
                uint32_t w[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) w[j] = pack_h2(S[2 * j], S[2 * j + 1]);
                tmem_st32(tmem_addr(tb, q4, TM_S16 + 32 * hf), w);
                tmem_wait_st();
            } else {
                const float4 *e4 = reinterpret_cast<const float4 *>(vec + (gsn & 1) * KV_SET + KV_E31 + 64 * hf);
                uint32_t w[32];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float4 e = e4[j];
                    w[2 * j] = pack_h2(S[4 * j] * e.x, S[4 * j + 1] * e.y);
                    w[2 * j + 1] = pack_h2(S[4 * j + 2] * e.z, S[4 * j + 3] * e.w);
                }
                tmem_st32(tmem_addr(tb, q4, TM_S16 + 32 * hf), w);
                tmem_wait_st();
            }
        };
        {
            // The entering state: h0, or for the last part of a cut unit the state its first part
            // left (flag and state of boundary blockIdx.x + 1, written by the next CTA).
            const float *h0 = a.h0 ? a.h0 + (size_t)bh * D * D : nullptr;
            if (SCHED && pkind == LAST) {
                const int bd = blockIdx.x + 1;
                if (tid == 0) {
                    const uint64_t t0 = globaltimer_ns();
                    while (ld_acquire_u64(a.sched_flags + bd) != a.sched_tag)
                        if (globaltimer_ns() - t0 > 1000000000ull) {
                            *reinterpret_cast<volatile int *>(&abort_sh) = 1;
                            atomicAdd(&g_tc_timeouts, 1u);
                            break;
                        }
                }
                named_bar_sync(2, GT);
                h0 = a.sched_states + (size_t)bd * D * D;
            }
            if (h0) h0 += (size_t)(64 * hf) * D + p;
#pragma unroll
            for (int dk = 0; dk < 64; ++dk) S[dk] = h0 ? __ldcg(h0 + (size_t)dk * D) : 0.f;
            if (GATE == 0) store_s16(gsb);
            if (SAVE) {   // the state entering chunk 0: row p of S^T, columns 64 hf ..
                uint8_t *sg = reinterpret_cast<uint8_t *>(a.save_s) + (size_t)bh * NC * (D * D * 2);
#pragma unroll
                for (int j = 0; j < 8; ++j) st_global_h8(sg + swz_chunk(p, j, hf * 16384), S + 8 * j);
            }
        }
        float gbn[4] = {0.f, 0.f, 0.f, 0.f};
        if (issuer && c1 > c0) {
            issue_loads(c0, gsb);
            if (c1 > c0 + 1) issue_loads(c0 + 1, gsb + 1);
        }
        if (c1 > c0) {
            load_gb(c0, gbn);
            ready(c0, gsb, gbn);
        }
        if (c1 > c0 + 1) {
            load_gb(c0 + 1, gbn);
            ready(c0 + 1, gsb + 1, gbn);
        }
        if (GATE && c1 > c0) store_s16(gsb);   // needs the first chunk's exp(G_31)
        tc_fence_before();
        for (int c = c0; c < c1; ++c) {
            const int gs = gsb + (c - c0);
            if (NORM && a.z) {   // this chunk's z row segment (pass B's) into L1
                const int r = 8 * warp + (lane & 7), k = lane >> 3;
                if (c * C + r < T)
                    prefetch_l1(reinterpret_cast<const __nv_bfloat16 *>(a.z) +
                                ((size_t)(tok0 + c * C + r) * a.Hv + h) * D + 32 * k);
            }
            // P and Qh of this chunk, out of tensor memory into the operand tiles
            wait(B_P1, gs & 1);
            tc_fence_after();
            {
                float v[32];
                tmem_ld32(tmem_addr(tb, q4, TM_X + 32 * hf), v);
#pragma unroll
                for (int j = 0; j < 4; ++j) st_chunk8(sb0 + swz_chunk(p, 4 * hf + j, OFF_QH16), v + 8 * j);
            }
            wait(B_P, gs & 1);
            if (issuer && c + 2 < c1) issue_loads(c + 2, gs + 2);   // chunk c's staging buffer is free
            if (c + 2 < c1) load_gb(c + 2, gbn);
            if (GATE && c + 2 < c1 && (c + 2) * C + (tid >> 2) < T)
                prefetch_l2(a.g + ((size_t)(tok0 + (long)(c + 2) * C + (tid >> 2)) * a.Hv + h) * D + 32 * (tid & 3));
            tc_fence_after();
            {
                float v[64];
                tmem_ld32x2(tmem_addr(tb, q4, TM_Y + 64 * hf), tmem_addr(tb, q4, TM_Y + 64 * hf + 32), v);
#pragma unroll
                for (int j = 0; j < 8; ++j) st_chunk8(sb0 + swz_chunk(p, j, OFF_P16 + hf * 16384), v + 8 * j);
            }
            const float gC = GATE ? 0.f : vec[(gs & 1) * V_SET + V_GC];
            tc_fence_before();
            mbar_arrive(bar(B_YE));
            fence_proxy_async();
            named_bar_sync(2, GT);
            if (issuer) {
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const uint32_t koff = (s >> 2) * 16384 + (s & 3) * 32;
                    mma_ts(tb + TM_S, tb + TM_S16 + 8 * s, sdesc(sb0 + OFF_P16 + koff, 16, 1024), ID_S, true);
                }
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    mma_ts(tb + TM_O, tb + TM_S16 + 8 * s, sdesc(sb0 + OFF_QH16 + s * 2048, 8192, 1024), ID_O, true);
                }
                mma_commit(bar(B_ST));
                if (SAVE) {   // the finished P and Qh^T tiles, as they are, to the caller's buffers
                    const size_t cu = (size_t)bh * NC + c;
                    bulk_s2g(reinterpret_cast<uint8_t *>(a.save_p) + cu * 32768, sb0 + OFF_P16, 32768);
                    bulk_s2g(reinterpret_cast<uint8_t *>(a.save_qh) + cu * 16384, sb0 + OFF_QH16, 16384);
                    bulk_commit();
                }
            }
            wait(B_ST, gs & 1);
            tc_fence_after();
            if (SAVE) {   // the copies have read P and Qh^T: the P tile holds the state's image next
                if (issuer) tma_store_wait_read();
                named_bar_sync(2, GT);
            }
            // S <- Gamma_C S + (P S + R), and its fp16 copy for the next batch
            if (GATE == 0 && NORM) {
                // The layer instance's state group is its longer chain: one TMEM wait for all
                // 64 columns (it has the registers for it).
                float v[64];
                tmem_ld32x2(tmem_addr(tb, q4, TM_S + 64 * hf), tmem_addr(tb, q4, TM_S + 64 * hf + 32), v);
#pragma unroll
                for (int i = 0; i < 64; ++i) S[i] = fmaf(gC, S[i], v[i]);
                store_s16(gs + 1);
            } else if (GATE == 0) {
                // In two halves of 32 rows, each written to its 16 columns of the copy as soon as
                // it is done (so the packed copy never sits beside the whole state in registers).
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    float v[32];
                    tmem_ld32(tmem_addr(tb, q4, TM_S + 64 * hf + 32 * h2), v);
                    uint32_t w[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        S[32 * h2 + 2 * j] = fmaf(gC, S[32 * h2 + 2 * j], v[2 * j]);
                        S[32 * h2 + 2 * j + 1] = fmaf(gC, S[32 * h2 + 2 * j + 1], v[2 * j + 1]);
                        w[j] = pack_h2(S[32 * h2 + 2 * j], S[32 * h2 + 2 * j + 1]);
                    }
                    tmem_st16(tmem_addr(tb, q4, TM_S16 + 32 * hf + 16 * h2), w);
                    if (SAVE && c + 1 < c1) {   // the state entering chunk c + 1: its image in the P tile
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            *reinterpret_cast<uint4 *>(sm + swz_chunk(p, 4 * h2 + j, OFF_P16 + hf * 16384)) =
                                make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
                    }
                }
                tmem_wait_st();
                if (SAVE && c + 1 < c1) {   // ... and from there to the caller's buffer
                    fence_proxy_async();
                    named_bar_sync(2, GT);
                    if (issuer) {
                        bulk_s2g(reinterpret_cast<uint8_t *>(a.save_s) + ((size_t)bh * NC + c + 1) * (D * D * 2),
                                 sb0 + OFF_P16, D * D * 2);
                        bulk_commit();
                    }
                }
            } else {   // S <- diag(Gamma_C) S + (P S + R), row dk = 64 hf + i, in two halves of 32
                const float4 *g4 = reinterpret_cast<const float4 *>(vec + (gs & 1) * KV_SET + KV_GC + 64 * hf);
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    float v[32];
                    tmem_ld32(tmem_addr(tb, q4, TM_S + 64 * hf + 32 * h2), v);
#pragma unroll
                    for (int i4 = 0; i4 < 8; ++i4) {
                        const float4 gg = g4[8 * h2 + i4];
                        float *sp = S + 32 * h2 + 4 * i4;
                        sp[0] = fmaf(gg.x, sp[0], v[4 * i4]);
                        sp[1] = fmaf(gg.y, sp[1], v[4 * i4 + 1]);
                        sp[2] = fmaf(gg.z, sp[2], v[4 * i4 + 2]);
                        sp[3] = fmaf(gg.w, sp[3], v[4 * i4 + 3]);
                    }
                }
            }
            if (GATE) store_s16(gs + 1);
            // o rows 32 hf .. 32 hf + 31 of this chunk (column p of Qh S + Uh) into the o tile
            // (the P tile, dead until the next chunk) in the TMA 128-byte swizzle, then out by
            // TMA stores, which clip tokens past T. The partial last chunk of a packed
            // sequence is stored with plain stores instead, so it never touches the next
            // sequence's rows (even lane: row r, columns p and p + 1; odd lane: row r + 1,
            // columns p - 1 and p).
            const int nvalid = min(C, T - c * C);
            const bool tile = !(a.cu_seqlens && nvalid < C);
            if (SAVE) {   // the copy has read the state's image before o is written there
                if (issuer) tma_store_wait_read();
                named_bar_sync(2, GT);
            }
            if (NORM && a.z) {
                // Pass A: fp32 o into the P tile (dead until the next chunk), in the TMA swizzle of
                // an fp32 o tile. Pass B, a row per 4 threads (row r = 8 warp + lane % 8, columns
                // 32 k .. 32 k + 31, k = lane / 8): the row's mean square, then
                // o / sqrt(mean + eps) * weight * SiLU(z) into the o tile (bf16: the Qh tile;
                // fp32: in place), or, for a packed sequence's partial last chunk, to global memory.
                {
                    float o[32];
                    tmem_ld32(tmem_addr(tb, q4, TM_O + 32 * hf), o);
                    tc_fence_before();
                    mbar_arrive(bar(B_SE));
                    mbar_arrive(bar(B_OE));
                    if (any_nonfinite32(o)) *reinterpret_cast<volatile int *>(&range_sh) = 1;
                    const uint32_t byte = (uint32_t)(p & 31) * 4u;
                    uint8_t *base = sm + OFF_P16 + (p >> 5) * C * 128 + (32 * hf) * 128 + (byte & 15);
                    uint32_t xo[8];
#pragma unroll
                    for (int s8 = 0; s8 < 8; ++s8) xo[s8] = ((byte >> 4) ^ s8) << 4;
#pragma unroll
                    for (int i = 0; i < 32; ++i) *reinterpret_cast<float *>(base + i * 128 + xo[i & 7]) = o[i];
                }
                named_bar_sync(2, GT);
                const int r = 8 * warp + (lane & 7), k = lane >> 3;
                float x[32];
                const uint8_t *rowp = sm + OFF_P16 + k * C * 128 + r * 128;
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const float4 v4 = *reinterpret_cast<const float4 *>(rowp + ((jj ^ (r & 7)) << 4));
                    x[4 * jj] = v4.x, x[4 * jj + 1] = v4.y, x[4 * jj + 2] = v4.z, x[4 * jj + 3] = v4.w;
                }
                float ss = 0.f;
#pragma unroll
                for (int i = 0; i < 32; ++i) ss = fmaf(x[i], x[i], ss);
                ss += __shfl_xor_sync(0xffffffffu, ss, 8);
                ss += __shfl_xor_sync(0xffffffffu, ss, 16);
                const float rsd = rsqrtf(ss * (1.f / D) + a.norm_eps);
                const bool rv = r < nvalid;
                const __nv_bfloat16 *zrow =
                    reinterpret_cast<const __nv_bfloat16 *>(a.z) + ((size_t)(tok0 + c * C + r) * a.Hv + h) * D + 32 * k;
                const float *nw = reinterpret_cast<const float *>(sm + OFF_NW) + 32 * k;
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                    const uint4 zz = rv ? *reinterpret_cast<const uint4 *>(zrow + 8 * q8) : make_uint4(0, 0, 0, 0);
                    const __nv_bfloat162 *z2 = reinterpret_cast<const __nv_bfloat162 *>(&zz);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 zf = __bfloat1622float2(z2[e]);
                        const int i = 8 * q8 + 2 * e;
                        x[i] *= rsd * nw[i] * __fdividef(zf.x, 1.f + __expf(-zf.x));
                        x[i + 1] *= rsd * nw[i + 1] * __fdividef(zf.y, 1.f + __expf(-zf.y));
                    }
                }
                if (tile) {
                    if (sizeof(TOut) == 4) {
                        uint8_t *wp = sm + OFF_P16 + k * C * 128 + r * 128;
#pragma unroll
                        for (int jj = 0; jj < 8; ++jj)
                            *reinterpret_cast<float4 *>(wp + ((jj ^ (r & 7)) << 4)) =
                                make_float4(x[4 * jj], x[4 * jj + 1], x[4 * jj + 2], x[4 * jj + 3]);
                    } else {
                        uint8_t *wp = sm + OFF_QH16 + (k >> 1) * C * 128 + r * 128;
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj)
                            *reinterpret_cast<uint4 *>(wp + (((4 * (k & 1) + jj) ^ (r & 7)) << 4)) = make_uint4(
                                pack_bf2(x[8 * jj], x[8 * jj + 1]), pack_bf2(x[8 * jj + 2], x[8 * jj + 3]),
                                pack_bf2(x[8 * jj + 4], x[8 * jj + 5]), pack_bf2(x[8 * jj + 6], x[8 * jj + 7]));
                    }
                    fence_proxy_async();
                } else if (rv) {
                    TOut *orow = reinterpret_cast<TOut *>(a.o) + ((size_t)(tok0 + c * C + r) * a.Hv + h) * D + 32 * k;
#pragma unroll
                    for (int i = 0; i < 32; i += 2) out_store2(orow + i, x[i], x[i + 1]);
                }
            } else {
                float o[32];
                tmem_ld32(tmem_addr(tb, q4, TM_O + 32 * hf), o);
                tc_fence_before();
                mbar_arrive(bar(B_SE));
                mbar_arrive(bar(B_OE));
                float z = 0.f;   // x * 0 is 0 for finite x, NaN otherwise
                if (tile) {
                    constexpr int EPB = 128 / sizeof(TOut);
                    const uint32_t byte = (uint32_t)(p % EPB) * sizeof(TOut);
                    uint8_t *base = sm + OFF_P16 + (p / EPB) * C * 128 + (32 * hf) * 128 + (byte & 15);
                    uint32_t xo[8];
#pragma unroll
                    for (int s8 = 0; s8 < 8; ++s8) xo[s8] = ((byte >> 4) ^ s8) << 4;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        out_store1(reinterpret_cast<TOut *>(base + i * 128 + xo[i & 7]), o[i]);
                        z = fmaf(o[i], 0.f, z);
                    }
                    fence_proxy_async();
                } else {
                    const int nv = nvalid - 32 * hf, odd = p & 1;
                    const size_t rs = (size_t)a.Hv * D;
                    TOut *orow = reinterpret_cast<TOut *>(a.o) + ((size_t)tok0 * a.Hv + h) * D + p +
                                 (size_t)(c * C + 32 * hf + odd) * rs - odd;
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        const float other = __shfl_xor_sync(0xffffffffu, odd ? o[i] : o[i + 1], 1);
                        if (i + odd < nv) out_store2(orow + (size_t)i * rs, odd ? other : o[i], odd ? o[i + 1] : other);
                        z = fmaf(o[i], 0.f, fmaf(o[i + 1], 0.f, z));
                    }
                }
                if (z != 0.f) *reinterpret_cast<volatile int *>(&range_sh) = 1;
            }
            named_bar_sync(2, GT);
            if (!SAVE && issuer && tile) {
                constexpr int EPB = 128 / sizeof(TOut);
                // the normalised bf16 o tile is in the Qh tile
                const uint32_t src = (NORM && a.z && sizeof(TOut) == 2) ? OFF_QH16 : OFF_P16;
#pragma unroll
                for (int k = 0; k < D / EPB; ++k)
                    tma_store_4d(&map_o, k * EPB, h, tt0 + c * C, tbb, sb0 + src + k * C * 128);
            }
            if (c + 2 < c1) ready(c + 2, gs + 2, gbn);
            if (!SAVE && issuer) tma_store_wait_read();   // the o tile is read before the next P tile is written
            named_bar_sync(2, GT);
        }
        if (issuer) tma_store_wait_all();
        if (any_nonfinite32(S) || any_nonfinite32(S + 32)) *reinterpret_cast<volatile int *>(&range_sh) = 1;
        // The state after the piece: the final state to hT, or, after a first part, to this
        // CTA's boundary (blockIdx.x) in the workspace, then the boundary's flag.
        float *hout = SCHED && pkind == FIRST ? a.sched_states + (size_t)blockIdx.x * D * D : a.hT ? a.hT + (size_t)bh * D * D
                                                                                          : nullptr;
        if (hout) {
            float *hp = hout + (size_t)(64 * hf) * D + p;
#pragma unroll
            for (int dk = 0; dk < 64; ++dk) hp[(size_t)dk * D] = S[dk];
        }
        named_bar_sync(2, GT);
        if (tid == 0) {
            if (SCHED && pkind == FIRST) {
                __threadfence();
                st_release_u64(a.sched_flags + blockIdx.x, a.sched_tag);
            }
            if (range_sh) {
                atomicAdd(&g_tc_range_errors, 1u);
                range_sh = 0;
            }
        }
        };
        if constexpr (SCHED) {
            int gsb = 0;
            for (long ppos = run0; ppos < run1;) {
                const Piece pcs = piece_at(ppos);
                ppos = pcs.next;
                state_piece(pcs.u, pcs.c0, pcs.c1, pcs.kind, gsb);
                gsb += pcs.c1 - pcs.c0;
            }
        } else {
            state_piece(blockIdx.x, 0, -1, WHOLE, 0);
        }
        if (issuer) {
            mma_commit(bar(B_DR0));
            mbar_wait_bounded(bar(B_DR0), 0);
        }
        if (gissuer) {
            mma_commit(bar(B_DR2));
            mbar_wait_bounded(bar(B_DR2), 0);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tb, 512);
    }
}

template <typename TOut>
cudaError_t launch_tc_t(const FwdArgs &a, cudaStream_t st)
{
    CUtensorMap mq, mk, mv, mo;
    const int mb = a.cu_seqlens ? 1 : a.B;   // packed input: one batch row of T tokens
    if (!make_map(&mq, a.q, mb, a.T, a.Hk, 64, false, true) || !make_map(&mk, a.k, mb, a.T, a.Hk, 64, false, true) ||
        !make_map(&mv, a.v, mb, a.T, a.Hv, 64, false, true))
        return cudaErrorInvalidValue;
    if (a.save_s) mo = mq;   // the backward's forward pass stores no o (the map is never used)
    else if (!make_map(&mo, a.o, mb, a.T, a.Hv, 128 / sizeof(TOut), sizeof(TOut) == 4, true))
        return cudaErrorInvalidValue;
    // The layer's options and the per-channel gate are separate instances, and so is the
    // wrap-around schedule, so that a call without them runs the same code as before they existed.
    auto kernel = a.sched_len ? (a.gate_mode ? tc_fwd_kernel<TOut, false, 1, true> : tc_fwd_kernel<TOut, false, 0, true>)
                  : a.gate_mode ? tc_fwd_kernel<TOut, false, 1, false>
                  : (a.qk_l2norm || a.z) ? tc_fwd_kernel<TOut, true, 0, false>
                  : a.save_s             ? tc_fwd_kernel<TOut, false, 0, false, true>
                                         : tc_fwd_kernel<TOut, false, 0, false>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_TC);
    if (e != cudaSuccess) return e;
    const long units = (long)a.B * a.Hv, steps = units * ((a.T + C - 1) / C);
    const long grid = a.sched_len ? (steps + a.sched_len - 1) / a.sched_len : units;
    kernel<<<(unsigned)grid, NTH, SMEM_TC, st>>>(a, mq, mk, mv, mo);
    return cudaGetLastError();
}

}  // namespace

// The wrap-around schedule: with U units of n chunks on S SMs (U > S, fixed length) each
// CTA takes ceil(U n / S) chunk-steps; the cuts between CTAs need a 64-bit flag and a
// [Dk][Dv] fp32 state each.
static bool sched_shape(const FwdArgs &a, long *len, long *grid)
{
    const long units = (long)a.B * a.Hv, nc = (a.T + C - 1) / C, sms = sm_count();
    if (a.cu_seqlens || nc == 0 || sms <= 0 || units <= sms) return false;
    *len = (units * nc + sms - 1) / sms;
    *grid = (units * nc + *len - 1) / *len;
    return true;
}
size_t tc_sched_bytes(const FwdArgs &a)
{
    long len, grid;
    if (a.qk_l2norm || a.z || !sched_shape(a, &len, &grid)) return 0;
    return (size_t)((grid * 8 + 255) / 256 * 256) + (size_t)grid * D * D * sizeof(float);
}
void tc_set_sched(FwdArgs &a, void *workspace)
{
    long len, grid;
    if (!workspace || a.qk_l2norm || a.z || !sched_shape(a, &len, &grid)) return;
    // A tag per launch, unlike any earlier one in this process and not 0: whatever a flag holds
    // from before never reads as this launch's.
    static std::atomic<unsigned long long> counter{0};
    static const unsigned long long base =
        (unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count() << 20;
    a.sched_len = (int)len;
    a.sched_tag = (base + ++counter) | 1ull;
    a.sched_flags = reinterpret_cast<unsigned long long *>(workspace);
    a.sched_states = reinterpret_cast<float *>(reinterpret_cast<char *>(workspace) + (grid * 8 + 255) / 256 * 256);
}

bool tc_supported(const FwdArgs &a)
{
    // The per-channel gate with the layer's options stays on the warp-level kernel.
    return in_bf16(a.dtype) && a.Dk == D && a.Dv == D && (a.gate_mode == 0 || (!a.qk_l2norm && !a.z));
}

cudaError_t launch_fwd_tc(const FwdArgs &a, cudaStream_t st)
{
    return out_f32(a.dtype) ? launch_tc_t<float>(a, st) : launch_tc_t<__nv_bfloat16>(a, st);
}

unsigned int tc_error_count()
{
    unsigned int t = 0;
    cudaMemcpyFromSymbol(&t, g_tc_timeouts, sizeof(t));
    return t;
}

unsigned int tc_range_error_count()
{
    unsigned int r = 0;
    cudaMemcpyFromSymbol(&r, g_tc_range_errors, sizeof(r));
    return r;
}

}  // namespace gdr
