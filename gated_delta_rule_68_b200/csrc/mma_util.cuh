// Building blocks shared by the tensor-core chunked-forward kernels: the tile
// geometry, mma.sync m16n8k16 and ldmatrix fragment addressing, asynchronous
// copies (cp.async, TMA, bulk copies on mbarriers with a bounded wait), and the
// host-side tensor-map construction.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace gdr {
namespace mmau {

constexpr int C = 64;            // tokens per chunk
constexpr int D = 128;           // key and value width
constexpr int LDD = D + 8;       // fp16 row stride of 128-wide tiles (272 B: ldmatrix rows hit distinct banks)
constexpr int LDC = C + 8;       // fp16 row stride of 64-wide tiles (144 B)
constexpr int LDX = 24;          // fp16 row stride of a warp's 16 x 16 product
constexpr int SZ_D = C * LDD * 2;  // one [64][128] fp16 tile
constexpr int SZ_C = C * LDC * 2;  // one [64][64] fp16 tile

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
// One 4-d box from shared memory to a tensor (TMA tiled store); coordinates past
// the tensor's end are not written. Completion is tracked per issuing thread.
__device__ __forceinline__ void tma_store_4d(const CUtensorMap *map, int c0, int c1, int c2, int c3, uint32_t src)
{
    asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3, %4}], [%5];"
                 :: "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(src) : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void tma_store_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void tma_store_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

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

// Barrier `id` over the first `nthreads` threads that reach it (a multiple of 32).
__device__ __forceinline__ void named_bar_sync(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
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

// Byte offset of element (r, c) of an o tile held as 128-byte-wide boxes of 64
// rows in the TMA 128-byte swizzle (16-byte chunk j of row r sits at j ^ (r % 8)).
template <typename TOut>
__device__ __forceinline__ int o_swz(int r, int c)
{
    constexpr int EPB = 128 / sizeof(TOut);
    const int byte = (c % EPB) * (int)sizeof(TOut);
    return (c / EPB) * C * 128 + r * 128 + ((((byte >> 4) ^ (r & 7))) << 4) + (byte & 15);
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

// Sum of squares of 8 bf16 values.
__device__ __forceinline__ float bf16x8_sumsq(uint4 u)
{
    const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&u);
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(p[e]);
        s = fmaf(f.x, f.x, fmaf(f.y, f.y, s));
    }
    return s;
}

// 8 bf16 values times `scale`, rounded to fp16.
__device__ __forceinline__ uint4 bf16x8_scaled_f16x8(uint4 u, float scale)
{
    const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&u);
    uint4 r;
    uint32_t *q = reinterpret_cast<uint32_t *>(&r);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(p[e]);
        const __half2 hh = __floats2half2_rn(f.x * scale, f.y * scale);
        q[e] = *reinterpret_cast<const uint32_t *>(&hh);
    }
    return r;
}

// Sum over the 16 lanes of a half warp (all 32 lanes take part).
__device__ __forceinline__ float halfwarp_sum(float s)
{
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    return s;
}

// The driver's tensor-map encoder, looked up through the runtime once, so the
// library needs no link-time dependency on the driver library.
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
inline EncodeTiledFn encode_tiled()
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
inline bool make_map(CUtensorMap *map, const void *base, int B, int T, int H, int cols, bool f32 = false,
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

inline int sm_count()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess)
        return 0;
    return n;
}

}  // namespace mmau
}  // namespace gdr
