// Column-block helpers for running a wide GLA shape as sub-problems on the fused kernels.
#pragma once

#include "common.cuh"

namespace gla {
namespace split {

// dst[r][c] = src[r][col0 + c] for r < rows, c < ncols (bf16; ncols and pitch multiples of 8).
cudaError_t gather_cols(const bf16* src, bf16* dst, long long rows, int pitch, int col0, int ncols,
                        cudaStream_t st);
// acc[r][col0 + c] += part[r][c] (fp32; ncols a multiple of 4).
cudaError_t add_cols(const float* part, float* acc, long long rows, int ncols, int acc_pitch, int col0,
                     cudaStream_t st);
// dst[r][c] = src[r][c] for c < ncols and 0 for ncols <= c < dst_cols, r < rows: pads (dst_cols >
// ncols) or crops (a narrower dst) rows.  ncols and dst_cols multiples of 8 (bf16) / 4 (fp32),
// pitches in elements, 16-byte aligned rows.
cudaError_t copy_cols(const bf16* src, long long src_pitch, bf16* dst, long long dst_pitch, long long rows,
                      long long ncols, long long dst_cols, cudaStream_t st);
cudaError_t copy_cols(const float* src, long long src_pitch, float* dst, long long dst_pitch, long long rows,
                      long long ncols, long long dst_cols, cudaStream_t st);
// dst = bf16(src), n values (n a multiple of 8).
cudaError_t to_bf16(const float* src, bf16* dst, long long n, cudaStream_t st);

}  // namespace split
}  // namespace gla
