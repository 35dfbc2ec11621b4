// Shared device helpers for the GLA kernels: typed loads/stores, launch checks.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace gla {

typedef __nv_bfloat16 bf16;

__device__ __forceinline__ float ldf(const float* p) { return *p; }
__device__ __forceinline__ float ldf(const bf16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void stf(float* p, float x) { *p = x; }
__device__ __forceinline__ void stf(bf16* p, float x) { *p = __float2bfloat16_rn(x); }

// Number of chunks covering T tokens.
__host__ __device__ __forceinline__ int num_chunks(int T, int C) { return (T + C - 1) / C; }

// Round a byte count up to the 256-byte workspace granularity.
__host__ __device__ __forceinline__ size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

}  // namespace gla
