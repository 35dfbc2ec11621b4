// Column-block helpers for split shapes (see split.cuh).  HBM-bound copies: one thread per
// 16-byte vector (8 bf16), grid-stride over a few waves of the SMs.
#include "split.cuh"

namespace gla {
namespace split {
namespace {

__global__ void to_bf16_kernel(const float* __restrict__ src, bf16* __restrict__ dst, long long n) {
  const long long nv = n / 8;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < nv; e += (long long)gridDim.x * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(src)[2 * e], b = reinterpret_cast<const float4*>(src)[2 * e + 1];
    __nv_bfloat162 h[4] = {__floats2bfloat162_rn(a.x, a.y), __floats2bfloat162_rn(a.z, a.w),
                           __floats2bfloat162_rn(b.x, b.y), __floats2bfloat162_rn(b.z, b.w)};
    reinterpret_cast<uint4*>(dst)[e] = *reinterpret_cast<const uint4*>(h);
  }
}

// dst[r][col0 + c] (row pitch dst_pitch), c < nblocks * W, = sum over j < nparts of the slice
// (b * bstride + j * jstride) at [r][c % W], b = c / W; slices are [rows][W] fp32, consecutive.
__global__ void sum_blocks_kernel(const float* __restrict__ parts, long long rows, int W, int nblocks, int nparts,
                                  int bstride, int jstride, bf16* __restrict__ dst, long long dst_pitch) {
  const int vpr = nblocks * W / 8;
  const long long n = rows * vpr, slice = rows * W;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
    const long long r = e / vpr;
    const int c = (int)(e % vpr) * 8, b = c / W, cc = c - b * W;
    const float* src = parts + (long long)b * bstride * slice + r * W + cc;
    float4 a = *reinterpret_cast<const float4*>(src), u = *reinterpret_cast<const float4*>(src + 4);
    for (int j = 1; j < nparts; ++j) {
      const float* s2 = src + (long long)j * jstride * slice;
      const float4 x = *reinterpret_cast<const float4*>(s2), y = *reinterpret_cast<const float4*>(s2 + 4);
      a.x += x.x, a.y += x.y, a.z += x.z, a.w += x.w;
      u.x += y.x, u.y += y.y, u.z += y.z, u.w += y.w;
    }
    __nv_bfloat162 h[4] = {__floats2bfloat162_rn(a.x, a.y), __floats2bfloat162_rn(a.z, a.w),
                           __floats2bfloat162_rn(u.x, u.y), __floats2bfloat162_rn(u.z, u.w)};
    *reinterpret_cast<uint4*>(dst + r * dst_pitch + c) = *reinterpret_cast<const uint4*>(h);
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

cudaError_t sum_blocks_to_bf16(const float* parts, long long rows, int W, int nblocks, int nparts, int bstride,
                               int jstride, bf16* dst, long long dst_pitch, cudaStream_t st) {
  if (W % 8 || dst_pitch % 8 || nblocks < 1 || nparts < 1 || (long long)nblocks * W > dst_pitch)
    return cudaErrorInvalidValue;
  sum_blocks_kernel<<<grid_for(rows * (nblocks * W / 8)), 256, 0, st>>>(parts, rows, W, nblocks, nparts, bstride,
                                                                         jstride, dst, dst_pitch);
  return cudaGetLastError();
}

cudaError_t to_bf16(const float* src, bf16* dst, long long n, cudaStream_t st) {
  to_bf16_kernel<<<grid_for(n / 8), 256, 0, st>>>(src, dst, n);
  return cudaGetLastError();
}

}  // namespace split
}  // namespace gla
