// Column-block helpers for split shapes (see split.cuh).  HBM-bound copies: one thread per
// 16-byte vector (8 bf16), grid-stride over a few waves of the SMs.
#include "split.cuh"

namespace gla {
namespace split {
namespace {

__global__ void gather_kernel(const bf16* __restrict__ src, bf16* __restrict__ dst, long long rows, int pitch,
                              int col0, int ncols) {
  const int vpr = ncols / 8;
  const long long n = rows * vpr;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
    const long long r = e / vpr;
    const int c = (int)(e % vpr) * 8;
    *reinterpret_cast<uint4*>(dst + r * ncols + c) = *reinterpret_cast<const uint4*>(src + r * pitch + col0 + c);
  }
}

__global__ void add_kernel(const float* __restrict__ part, float* __restrict__ acc, long long rows, int ncols,
                           int acc_pitch, int col0) {
  const int vpr = ncols / 4;
  const long long n = rows * vpr;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
    const long long r = e / vpr;
    const int c = (int)(e % vpr) * 4;
    const float4 u = *reinterpret_cast<const float4*>(part + r * ncols + c);
    float4* a = reinterpret_cast<float4*>(acc + r * acc_pitch + col0 + c);
    float4 x = *a;
    x.x += u.x;
    x.y += u.y;
    x.z += u.z;
    x.w += u.w;
    *a = x;
  }
}

__global__ void to_bf16_kernel(const float* __restrict__ src, bf16* __restrict__ dst, long long n) {
  const long long nv = n / 8;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < nv; e += (long long)gridDim.x * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(src)[2 * e], b = reinterpret_cast<const float4*>(src)[2 * e + 1];
    __nv_bfloat162 h[4] = {__floats2bfloat162_rn(a.x, a.y), __floats2bfloat162_rn(a.z, a.w),
                           __floats2bfloat162_rn(b.x, b.y), __floats2bfloat162_rn(b.z, b.w)};
    reinterpret_cast<uint4*>(dst)[e] = *reinterpret_cast<const uint4*>(h);
  }
}

// dst[r][c] = src[r][c] for c < ncols, 0 for ncols <= c < dst_cols (16-byte vectors of 8 bf16 / 4 fp32)
template <typename T>
__global__ void copy_kernel(const T* __restrict__ src, long long src_pitch, T* __restrict__ dst, long long dst_pitch,
                            long long rows, long long ncols, long long dst_cols) {
  constexpr int V = 16 / sizeof(T);
  const long long vpr = dst_cols / V, n = rows * vpr;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
    const long long r = e / vpr, c = (e % vpr) * V;
    uint4 x = make_uint4(0u, 0u, 0u, 0u);
    if (c < ncols) x = *reinterpret_cast<const uint4*>(src + r * src_pitch + c);
    *reinterpret_cast<uint4*>(dst + r * dst_pitch + c) = x;
  }
}

int grid_for(long long items) {
  const long long blocks = (items + 255) / 256, cap = 148LL * 16;
  return (int)(blocks < 1 ? 1 : blocks > cap ? cap : blocks);
}

}  // namespace

cudaError_t gather_cols(const bf16* src, bf16* dst, long long rows, int pitch, int col0, int ncols,
                        cudaStream_t st) {
  gather_kernel<<<grid_for(rows * (ncols / 8)), 256, 0, st>>>(src, dst, rows, pitch, col0, ncols);
  return cudaGetLastError();
}

cudaError_t add_cols(const float* part, float* acc, long long rows, int ncols, int acc_pitch, int col0,
                     cudaStream_t st) {
  add_kernel<<<grid_for(rows * (ncols / 4)), 256, 0, st>>>(part, acc, rows, ncols, acc_pitch, col0);
  return cudaGetLastError();
}

cudaError_t copy_cols(const bf16* src, long long src_pitch, bf16* dst, long long dst_pitch, long long rows,
                      long long ncols, long long dst_cols, cudaStream_t st) {
  copy_kernel<bf16><<<grid_for(rows * (dst_cols / 8)), 256, 0, st>>>(src, src_pitch, dst, dst_pitch, rows, ncols,
                                                                     dst_cols);
  return cudaGetLastError();
}

cudaError_t copy_cols(const float* src, long long src_pitch, float* dst, long long dst_pitch, long long rows,
                      long long ncols, long long dst_cols, cudaStream_t st) {
  copy_kernel<float><<<grid_for(rows * (dst_cols / 4)), 256, 0, st>>>(src, src_pitch, dst, dst_pitch, rows, ncols,
                                                                      dst_cols);
  return cudaGetLastError();
}

cudaError_t to_bf16(const float* src, bf16* dst, long long n, cudaStream_t st) {
  to_bf16_kernel<<<grid_for(n / 8), 256, 0, st>>>(src, dst, n);
  return cudaGetLastError();
}

}  // namespace split
}  // namespace gla
