// Fused chunked forward of the gated delta rule with a scalar per-head gate
// (Gated DeltaNet) on the warp-level tensor cores: mma.sync m16n8k16 with fp16
// operands and fp32 accumulators, bf16 inputs, Dk = Dv = 128, chunks of C = 64
// tokens. One CTA (8 warps) per (batch row, value head) walks the whole
// sequence; the fp32 state lives in the warps' accumulator registers and never
// leaves the SM until the final state is written.
//
// Method: the exact chunkwise form of
//   S_t = (I - beta_t k_t k_t^T) exp(g_t) S_{t-1} + beta_t k_t v_t^T,   o_t = S_t^T q_t
// (NextTransformer, "Source notes", "Linear attention", row gdn; SinkProbe
// (Attention-Sink) README: delta-rule layer in exact chunkwise form). With
// G_r = sum_{j<=r} g_j inside the chunk, Gamma_r = exp(G_r), Gamma_C = Gamma_63:
//   A_ri = beta_r exp(G_r - G_i) k_r.k_i  (i < r),   T = (I + A)^-1
//   W = T diag(beta Gamma) K,   U = T diag(beta) V,   U' = U - W S
//   O_r = Gamma_r (Q S)_r + (M U')_r,   M_ri = exp(G_r - G_i) q_r.k_i  (i <= r)
//   S_next = Gamma_C S + K^T diag(e) U',   e_i = exp(G_C - G_i)
// Every gate factor is folded where it is at most 1, so no operand grows past
// the size of its inputs. The products run on tensor cores; A, the inverse T
// and the gate factors are fp32 on CUDA cores. fp16 operands (bf16 inputs
// convert exactly in fp16's normal range) keep the result within 2e-2 of the
// fp64 recurrence by max |error| / rms; inputs and states must stay inside the
// fp16 range (|x| < 6.5e4).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"

namespace gdr {
namespace {

constexpr int C = 64;
constexpr int D = 128;
constexpr int NT = 256;          // 8 warps
constexpr int LDD = D + 8;       // fp16 row stride of 128-wide tiles (272 B: ldmatrix rows hit distinct banks)
constexpr int LDC = C + 8;       // fp16 row stride of 64-wide tiles (144 B)
constexpr int LDF = C + 1;       // fp32 row stride of the 64 x 64 scratch

// Shared-memory layout (bytes).
constexpr int SZ_D = C * LDD * 2;               // one [64][128] fp16 tile
constexpr int OFF_K = 0;                        // K [i][dk]
constexpr int OFF_Q = OFF_K + SZ_D;             // Q [r][dk]
constexpr int OFF_V = OFF_Q + SZ_D;             // V [i][dv]
constexpr int OFF_W = OFF_V + SZ_D;             // -W [r][dk]
constexpr int OFF_U = OFF_W + SZ_D;             // U' [i][dv]
constexpr int OFF_UE = OFF_U + SZ_D;            // diag(e) U' [i][dv]
constexpr int OFF_S = OFF_UE + SZ_D;            // S [dk][dv] fp16 copy of the state
constexpr int SZ_C = C * LDC * 2;               // one [64][64] fp16 tile
constexpr int OFF_M = OFF_S + D * LDD * 2;      // M [r][i]
constexpr int OFF_TB = OFF_M + SZ_C;            // T diag(beta) [r][i]
constexpr int OFF_TG = OFF_TB + SZ_C;           // T diag(beta Gamma) [r][i]
constexpr int OFF_STG = OFF_TG + SZ_C;          // next chunk's K, Q, V as loaded (bf16 [3][64][128])
constexpr int OFF_GST = OFF_STG + 3 * C * D * 2;// next chunk's g and beta (fp32 [2][64])
constexpr int OFF_VEC = OFF_GST + 2 * C * 4;    // G, exp(G), exp(G_C - G), beta: 64 fp32 each
constexpr int SMEM_BYTES = OFF_VEC + 4 * 64 * 4;
// The scratch of the inverse reuses tiles that are dead while it is live: fp32
// A sits in the U' tile, the fp16 inverse T in the diag(e) U' tile, and the
// fp16 copy of A (an operand of the block-row products) after each warp's
// 16 x 16 block-row product in the -W tile.
constexpr int OFF_A = OFF_U;                    // fp32 A [64][65]
constexpr int OFF_TH = OFF_UE;                  // fp16 T [64][72]
constexpr int LDX = 24;                         // fp16 row stride of a warp's 16 x 16 product
constexpr int OFF_X = OFF_W;                    // fp16 [8 warps][16][24]
constexpr int OFF_AH = OFF_X + 8 * 16 * LDX * 2;// fp16 A [64][72]
static_assert(C * LDF * 4 <= SZ_D, "A must fit in the U' tile");
static_assert(C * LDC * 2 <= SZ_D, "T must fit in the diag(e) U' tile");
static_assert(8 * 16 * LDX * 2 + C * LDC * 2 <= SZ_D, "block-row products and A must fit in the W tile");
static_assert(SMEM_BYTES + 128 <= 227 * 1024, "shared memory");
static_assert(OFF_STG % 128 == 0, "TMA destination alignment");

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void ldsm(uint32_t r[4], uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr) : "memory");
}
__device__ __forceinline__ void ldsm_t(uint32_t r[4], uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr) : "memory");
}
// c (16x8, fp32) += a (16x16, fp16, row) * b (16x8, fp16, col)
__device__ __forceinline__ void mma(float c[4], const uint32_t a[4], uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
                 "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Fragment addresses for ldmatrix.x4 (lane supplies one row address).
// A tile (16 x 16) at rows r0.., cols k0.. of a row-major tile.
__device__ __forceinline__ uint32_t a_rm(uint32_t base, int ld, int r0, int k0, int lane)
{
    return base + ((r0 + (lane & 7) + ((lane >> 3) & 1) * 8) * ld + k0 + (lane >> 4) * 8) * 2;
}
// A tile (16 x 16) whose element (m, k) is St[k0 + k][m0 + m] of a row-major St (load with .trans).
__device__ __forceinline__ uint32_t a_tr(uint32_t base, int ld, int m0, int k0, int lane)
{
    return base + ((k0 + (lane & 7) + (lane >> 4) * 8) * ld + m0 + ((lane >> 3) & 1) * 8) * 2;
}
// B tiles for n0..n0+15 (two n8 tiles) and k0..k0+15 of a tile stored [n][k] (plain load).
__device__ __forceinline__ uint32_t b_nk(uint32_t base, int ld, int n0, int k0, int lane)
{
    return base + ((n0 + (lane & 7) + (lane >> 4) * 8) * ld + k0 + ((lane >> 3) & 1) * 8) * 2;
}
// B tiles for n0..n0+15 and k0..k0+15 of a tile stored [k][n] (load with .trans).
__device__ __forceinline__ uint32_t b_kn(uint32_t base, int ld, int n0, int k0, int lane)
{
    return base + ((k0 + (lane & 7) + ((lane >> 3) & 1) * 8) * ld + n0 + (lane >> 4) * 8) * 2;
}

// Asynchronous 4-byte global -> shared copy; bytes past src_bytes are filled with zeros.
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" :: "r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
// mbarrier-tracked bulk copies (whole rows, global -> shared) and a bounded wait.
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(bytes) : "memory");
}
// One 4-d box of a tensor map (TMA tiled load) into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *map, int c0, int c1, int c2, int c3,
                                            uint32_t bar)
{
    asm volatile("cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
                 "[%0], [%1, {%2, %3, %4, %5}], [%6];"
                 :: "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t done;
    asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}\n" : "=r"(done) : "r"(bar), "r"(parity) : "memory");
    return done != 0;
}
__device__ __forceinline__ uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Waits for phase `parity` of `bar` for at most one second; false if it gave up.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer_ns() - t0 > 1000000000ull) return false;
    return true;
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void st_h2(__half *p, float x, float y)
{
    *reinterpret_cast<__half2 *>(p) = __floats2half2_rn(x, y);
}

__device__ __forceinline__ void store_out2(float *p, float x, float y)
{
    *reinterpret_cast<float2 *>(p) = make_float2(x, y);
}
__device__ __forceinline__ void store_out2(__nv_bfloat16 *p, float x, float y)
{
    *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(x, y);
}

// 8 bf16 -> 8 fp16 in one 16-byte word.
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 u)
{
    const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&u);
    uint4 r;
    uint32_t *q = reinterpret_cast<uint32_t *>(&r);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(p[e]);
        const __half2 hh = __floats2half2_rn(f.x, f.y);
        q[e] = *reinterpret_cast<const uint32_t *>(&hh);
    }
    return r;
}

// Chunk loads that never completed (each abandons its CTA's remaining chunks).
__device__ unsigned int g_fused_load_timeouts;

template <typename TOut>
__global__ void __launch_bounds__(NT, 1)
fused_fwd_gdn_kernel(FwdArgs a, const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                     const __grid_constant__ CUtensorMap map_v)
{
    extern __shared__ __align__(16) uint8_t smem_raw[];
    // 128-byte aligned base: the TMA destination tiles need it.
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    __half *sK = reinterpret_cast<__half *>(sm + OFF_K), *sQ = reinterpret_cast<__half *>(sm + OFF_Q);
    __half *sV = reinterpret_cast<__half *>(sm + OFF_V), *sW = reinterpret_cast<__half *>(sm + OFF_W);
    __half *sU = reinterpret_cast<__half *>(sm + OFF_U), *sUE = reinterpret_cast<__half *>(sm + OFF_UE);
    __half *sS = reinterpret_cast<__half *>(sm + OFF_S), *sM = reinterpret_cast<__half *>(sm + OFF_M);
    __half *sTB = reinterpret_cast<__half *>(sm + OFF_TB), *sTG = reinterpret_cast<__half *>(sm + OFF_TG);
    float *sA = reinterpret_cast<float *>(sm + OFF_A);
    __half *sAh = reinterpret_cast<__half *>(sm + OFF_AH), *sTh = reinterpret_cast<__half *>(sm + OFF_TH);
    float *sG = reinterpret_cast<float *>(sm + OFF_VEC);  // [64] G_r
    float *sEg = sG + 64;                                  // [64] exp(G_r)
    float *sEt = sG + 128;                                 // [64] exp(G_C - G_r)
    float *sBeta = sG + 192;                               // [64]
    const uint32_t aK = smem_u32(sK), aQ = smem_u32(sQ), aV = smem_u32(sV), aW = smem_u32(sW);
    const uint32_t aU = smem_u32(sU), aUE = smem_u32(sUE), aS = smem_u32(sS), aM = smem_u32(sM);
    const uint32_t aTB = smem_u32(sTB), aTG = smem_u32(sTG), aAh = smem_u32(sAh), aTh = smem_u32(sTh);
    const uint4 *sStg = reinterpret_cast<const uint4 *>(sm + OFF_STG);
    const float *sGst = reinterpret_cast<const float *>(sm + OFF_GST);   // [64] g, then [64] beta
    const uint32_t aStg = smem_u32(sm + OFF_STG), aGst = smem_u32(sm + OFF_GST);

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31, g = lane >> 2, t4 = lane & 3;
    __half *sXw = reinterpret_cast<__half *>(sm + OFF_X) + w * 16 * LDX;   // this warp's 16 x 16 tile
    const uint32_t aXw = smem_u32(sXw);
    const int bh = blockIdx.x;
    const int b = bh / a.Hv, h = bh % a.Hv, hk = h / (a.Hv / a.Hk);
    const int T = a.T, NC = (T + C - 1) / C;

    // Row block (16 rows) and column half (64 columns) of this warp in the [64 x 128] products.
    const int rw0 = 16 * (w & 3), cw0 = 64 * (w >> 2);

    // State S [dk][dv] in registers: warp w holds dk rows 16w..16w+15; n8 tile j holds dv 8j..8j+7.
    float accS[16][4];
    {
        const float *h0 = a.h0 ? a.h0 + (size_t)bh * D * D : nullptr;
        const int r0 = 16 * w + g;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int c = 8 * j + 2 * t4;
            float2 x0 = make_float2(0.f, 0.f), x1 = x0;
            if (h0) {
                x0 = *reinterpret_cast<const float2 *>(h0 + (size_t)r0 * D + c);
                x1 = *reinterpret_cast<const float2 *>(h0 + (size_t)(r0 + 8) * D + c);
            }
            accS[j][0] = x0.x; accS[j][1] = x0.y; accS[j][2] = x1.x; accS[j][3] = x1.y;
            st_h2(sS + r0 * LDD + c, x0.x, x0.y);
            st_h2(sS + (r0 + 8) * LDD + c, x1.x, x1.y);
        }
    }

    // Chunk c's K, Q, V rows, g and beta -> staging buffers, asynchronously (rows past
    // the end of the sequence are zero-filled).
    // Chunk c's K, Q, V tiles -> bf16 staging by three TMA box loads that
    // complete on ld_bar (rows past the end of the sequence read as zero); g and
    // beta by 4-byte asynchronous copies.
    __shared__ uint64_t ld_bar;
    const uint32_t aBar = smem_u32(&ld_bar);
    if (tid == 0) mbar_init(aBar, 1);
    __syncthreads();
    auto issue_loads = [&](int c) {
        const int t0 = c * C, n = min(C, T - t0);
        if (tid == 0) {
            mbar_expect_tx(aBar, 3u * C * D * 2);
            tma_load_4d(aStg, &map_k, 0, hk, t0, b, aBar);
            tma_load_4d(aStg + C * D * 2, &map_q, 0, hk, t0, b, aBar);
            tma_load_4d(aStg + 2 * C * D * 2, &map_v, 0, h, t0, b, aBar);
        }
        if (tid < 2 * C) {
            const int r = tid & (C - 1);
            const float *src = tid < C ? a.g : a.beta;
            if (r < n) src += ((long)b * T + t0 + r) * a.Hv + h;
            cp_async4(aGst + tid * 4, src, r < n ? 4u : 0u);
        }
        cp_async_commit();
    };
    if (NC > 0) issue_loads(0);

#pragma unroll 1
    for (int ch = 0; ch < NC; ++ch) {
        const int t0 = ch * C, n = min(C, T - t0);
        cp_async_wait_all();
        if (!__syncthreads_and(mbar_wait_bounded(aBar, ch & 1))) {
            if (tid == 0) atomicAdd(&g_fused_load_timeouts, 1u);
            return;
        }

        // ---------------- gate prefix G, exp(G), exp(G_C - G) (warp 0); beta (warps 2, 3)
        if (w == 0) {
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
        } else if (w == 2 || w == 3) {
            sBeta[tid - 64] = sGst[C + tid - 64];
        }

        // ---------------- staged bf16 K, Q, V -> fp16 tiles
#pragma unroll 4
        for (int idx = tid; idx < 3 * C * 16; idx += NT) {
            const int which = idx / (C * 16), rem = idx % (C * 16), r = rem >> 4, c16 = rem & 15;
            __half *dst = which == 0 ? sK : (which == 1 ? sQ : sV);
            *reinterpret_cast<uint4 *>(dst + r * LDD + c16 * 8) = bf16x8_to_f16x8(sStg[idx]);
        }
        __syncthreads();
        if (ch + 1 < NC) issue_loads(ch + 1);

        // ---------------- Gram [K ; Q] K^T: warps 0-3 rows of K, warps 4-7 rows of Q
        {
            float acc[8][4];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
            const uint32_t abase = w < 4 ? aK : aQ;
#pragma unroll
            for (int k0 = 0; k0 < D; k0 += 16) {
                uint32_t af[4];
                ldsm(af, a_rm(abase, LDD, rw0, k0, lane));
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t bf[4];
                    ldsm(bf, b_nk(aK, LDD, 16 * np, k0, lane));
                    mma(acc[2 * np], af, bf[0], bf[1]);
                    mma(acc[2 * np + 1], af, bf[2], bf[3]);
                }
            }
            // A rows (fp32) from warps 0-3; M rows (fp16) from warps 4-7
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int r = rw0 + g + 8 * hh;
                const float gr = sG[r], br = sBeta[r];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int i = 8 * j + 2 * t4;
                    const float d0 = acc[j][2 * hh], d1 = acc[j][2 * hh + 1];
                    if (w < 4) {
                        const float x0 = i < r ? br * __expf(gr - sG[i]) * d0 : 0.f;
                        const float x1 = i + 1 < r ? br * __expf(gr - sG[i + 1]) * d1 : 0.f;
                        sA[r * LDF + i] = x0;
                        sA[r * LDF + i + 1] = x1;
                        st_h2(sAh + r * LDC + i, x0, x1);
                    } else {
                        st_h2(sM + r * LDC + i, i <= r ? __expf(gr - sG[i]) * d0 : 0.f,
                              i + 1 <= r ? __expf(gr - sG[i + 1]) * d1 : 0.f);
                    }
                }
            }
        }
        __syncthreads();

        // ---------------- T = (I + A)^-1 (entries above the diagonal are never
        // written and read as zero). The 16x16 diagonal blocks by forward
        // substitution in fp32; then block rows bi = 1..3 on tensor cores, one
        // warp per block (bi, bj):
        //   X = sum_{m=bj}^{bi-1} A_{bi,m} T_{m,bj},   T_{bi,bj} = -T_{bi,bi} X
        if (tid < 64) {
            const int base = (tid >> 4) * 16, col = tid & 15;
            float tv[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float s0 = 0.f, s1 = 0.f;
#pragma unroll
                for (int i = 0; i < r; i += 2) {
                    s0 += sA[(base + r) * LDF + base + i] * tv[i];
                    if (i + 1 < r) s1 += sA[(base + r) * LDF + base + i + 1] * tv[i + 1];
                }
                tv[r] = (r < col) ? 0.f : (r == col ? 1.f : -(s0 + s1));
            }
            const float bc = sBeta[base + col], bgc = bc * sEg[base + col];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const int o = (base + r) * LDC + base + col;
                sTh[o] = __float2half_rn(tv[r]);
                sTB[o] = __float2half_rn(tv[r] * bc);
                sTG[o] = __float2half_rn(tv[r] * bgc);
            }
        } else {
            // zeros in the six blocks above the diagonal of T diag(beta), T diag(beta Gamma)
            const int e = tid - 64, blk = e >> 5, row = (e >> 1) & 15, hf = e & 1;
            const int bi = blk < 3 ? 0 : (blk < 5 ? 1 : 2), bj = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
            const int o = (16 * bi + row) * LDC + 16 * bj + 8 * hf;
            *reinterpret_cast<uint4 *>(sTB + o) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(sTG + o) = make_uint4(0, 0, 0, 0);
        }
        __syncthreads();
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
                // T_{bi,bj} = -y, and its columns scaled by beta and by beta Gamma
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int r0 = 16 * bi + g, c = 16 * bj + 8 * j + 2 * t4;
                    const float b0 = sBeta[c], b1 = sBeta[c + 1];
                    const float e0 = b0 * sEg[c], e1 = b1 * sEg[c + 1];
                    st_h2(sTh + r0 * LDC + c, -y[j][0], -y[j][1]);
                    st_h2(sTh + (r0 + 8) * LDC + c, -y[j][2], -y[j][3]);
                    st_h2(sTB + r0 * LDC + c, -y[j][0] * b0, -y[j][1] * b1);
                    st_h2(sTB + (r0 + 8) * LDC + c, -y[j][2] * b0, -y[j][3] * b1);
                    st_h2(sTG + r0 * LDC + c, -y[j][0] * e0, -y[j][1] * e1);
                    st_h2(sTG + (r0 + 8) * LDC + c, -y[j][2] * e0, -y[j][3] * e1);
                }
            }
            __syncthreads();
        }

        // ---------------- W = T diag(beta Gamma) K,  U = T diag(beta) V  (warp tile 16 x 64)
        float accU[8][4];
        {
            float accW[8][4];
#pragma unroll
            for (int j = 0; j < 8; ++j)
                accW[j][0] = accW[j][1] = accW[j][2] = accW[j][3] = accU[j][0] = accU[j][1] = accU[j][2] =
                    accU[j][3] = 0.f;
#pragma unroll
            for (int k0 = 0; k0 < C; k0 += 16) {
                uint32_t atg[4], atb[4];
                ldsm(atg, a_rm(aTG, LDC, rw0, k0, lane));
                ldsm(atb, a_rm(aTB, LDC, rw0, k0, lane));
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t bk[4], bv[4];
                    ldsm_t(bk, b_kn(aK, LDD, cw0 + 16 * np, k0, lane));
                    ldsm_t(bv, b_kn(aV, LDD, cw0 + 16 * np, k0, lane));
                    mma(accW[2 * np], atg, bk[0], bk[1]);
                    mma(accW[2 * np + 1], atg, bk[2], bk[3]);
                    mma(accU[2 * np], atb, bv[0], bv[1]);
                    mma(accU[2 * np + 1], atb, bv[2], bv[3]);
                }
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int c = cw0 + 8 * j + 2 * t4;
                st_h2(sW + (rw0 + g) * LDD + c, -accW[j][0], -accW[j][1]);
                st_h2(sW + (rw0 + g + 8) * LDD + c, -accW[j][2], -accW[j][3]);
            }
        }
        __syncthreads();

        // ---------------- U' = U - W S,  O1 = Q S  (K-dim dk)
        float accO[8][4];
#pragma unroll
        for (int j = 0; j < 8; ++j) accO[j][0] = accO[j][1] = accO[j][2] = accO[j][3] = 0.f;
#pragma unroll
        for (int k0 = 0; k0 < D; k0 += 16) {
            uint32_t aw[4], aq[4];
            ldsm(aw, a_rm(aW, LDD, rw0, k0, lane));
            ldsm(aq, a_rm(aQ, LDD, rw0, k0, lane));
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t bs[4];
                ldsm_t(bs, b_kn(aS, LDD, cw0 + 16 * np, k0, lane));
                mma(accU[2 * np], aw, bs[0], bs[1]);
                mma(accU[2 * np + 1], aw, bs[2], bs[3]);
                mma(accO[2 * np], aq, bs[0], bs[1]);
                mma(accO[2 * np + 1], aq, bs[2], bs[3]);
            }
        }
        {
            const float eg0 = sEg[rw0 + g], eg1 = sEg[rw0 + g + 8];
            const float et0 = sEt[rw0 + g], et1 = sEt[rw0 + g + 8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                accO[j][0] *= eg0; accO[j][1] *= eg0; accO[j][2] *= eg1; accO[j][3] *= eg1;
                const int c = cw0 + 8 * j + 2 * t4;
                st_h2(sU + (rw0 + g) * LDD + c, accU[j][0], accU[j][1]);
                st_h2(sU + (rw0 + g + 8) * LDD + c, accU[j][2], accU[j][3]);
                st_h2(sUE + (rw0 + g) * LDD + c, accU[j][0] * et0, accU[j][1] * et0);
                st_h2(sUE + (rw0 + g + 8) * LDD + c, accU[j][2] * et1, accU[j][3] * et1);
            }
        }
        __syncthreads();

        // ---------------- O += M U'  and the output rows
#pragma unroll
        for (int k0 = 0; k0 < C; k0 += 16) {
            uint32_t am[4];
            ldsm(am, a_rm(aM, LDC, rw0, k0, lane));
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t bu[4];
                ldsm_t(bu, b_kn(aU, LDD, cw0 + 16 * np, k0, lane));
                mma(accO[2 * np], am, bu[0], bu[1]);
                mma(accO[2 * np + 1], am, bu[2], bu[3]);
            }
        }
        {
            TOut *op = reinterpret_cast<TOut *>(a.o) + (((long)b * T + t0) * a.Hv + h) * D + cw0 + 2 * t4;
            const long rs = (long)a.Hv * D;
            const int r0 = rw0 + g, r1 = rw0 + g + 8;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (r0 < n) store_out2(op + r0 * rs + 8 * j, accO[j][0], accO[j][1]);
                if (r1 < n) store_out2(op + r1 * rs + 8 * j, accO[j][2], accO[j][3]);
            }
        }

        // ---------------- S <- Gamma_C S + K^T diag(e) U'  (warp rows dk 16w.., all dv)
        {
            const float gc = sEg[C - 1];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                accS[j][0] *= gc; accS[j][1] *= gc; accS[j][2] *= gc; accS[j][3] *= gc;
            }
#pragma unroll
            for (int k0 = 0; k0 < C; k0 += 16) {
                uint32_t ak[4];
                ldsm_t(ak, a_tr(aK, LDD, 16 * w, k0, lane));
#pragma unroll
                for (int np = 0; np < 8; ++np) {
                    uint32_t bu[4];
                    ldsm_t(bu, b_kn(aUE, LDD, 16 * np, k0, lane));
                    mma(accS[2 * np], ak, bu[0], bu[1]);
                    mma(accS[2 * np + 1], ak, bu[2], bu[3]);
                }
            }
            const int r0 = 16 * w + g;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int c = 8 * j + 2 * t4;
                st_h2(sS + r0 * LDD + c, accS[j][0], accS[j][1]);
                st_h2(sS + (r0 + 8) * LDD + c, accS[j][2], accS[j][3]);
            }
        }
        __syncthreads();
    }

    if (a.hT) {
        float *hp = a.hT + (size_t)bh * D * D;
        const int r0 = 16 * w + g;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int c = 8 * j + 2 * t4;
            *reinterpret_cast<float2 *>(hp + (size_t)r0 * D + c) = make_float2(accS[j][0], accS[j][1]);
            *reinterpret_cast<float2 *>(hp + (size_t)(r0 + 8) * D + c) = make_float2(accS[j][2], accS[j][3]);
        }
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

// Tensor map of a [B][T][H][128] bf16 tensor for boxes of 64 consecutive
// tokens of one head: dims (d, head, t, b), box (128, 1, 64, 1). Tokens past T
// read as zero.
bool make_map(CUtensorMap *map, const void *base, int B, int T, int H)
{
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)T * H * D * 2};
    const cuuint32_t box[4] = {(cuuint32_t)D, 1, (cuuint32_t)C, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const EncodeTiledFn encode = encode_tiled();
    return encode && encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box,
                            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename TOut>
cudaError_t launch_t(const FwdArgs &a, cudaStream_t st)
{
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, a.q, a.B, a.T, a.Hk) || !make_map(&mk, a.k, a.B, a.T, a.Hk) ||
        !make_map(&mv, a.v, a.B, a.T, a.Hv))
        return cudaErrorInvalidValue;
    const int smem = SMEM_BYTES + 128;
    cudaError_t e = cudaFuncSetAttribute(fused_fwd_gdn_kernel<TOut>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    fused_fwd_gdn_kernel<TOut><<<(unsigned)((long)a.B * a.Hv), NT, smem, st>>>(a, mq, mk, mv);
    return cudaGetLastError();
}

}  // namespace

bool fused_supported(const FwdArgs &a)
{
    return in_bf16(a.dtype) && a.gate_mode == 0 && a.Dk == D && a.Dv == D;
}

cudaError_t launch_fwd_fused(const FwdArgs &a, cudaStream_t st)
{
    return out_f32(a.dtype) ? launch_t<float>(a, st) : launch_t<__nv_bfloat16>(a, st);
}

}  // namespace gdr
