// Shared device helpers for libgdr kernels.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdr {

constexpr int kChunk = 64;  // tokens per chunk of the chunked forward

template <typename T> struct In;
template <> struct In<float> {
    static __device__ __forceinline__ float load(const float *p) { return *p; }
    static __device__ __forceinline__ void store(float *p, float x) { *p = x; }
};
template <> struct In<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }
};

// Launch helper status (host side).
struct LaunchStatus {
    cudaError_t err = cudaSuccess;
};

}  // namespace gdr
