// Column-block helpers for running a wide GLA shape as sub-problems on the fused kernels.
#pragma once

#include "common.cuh"

namespace gla {
namespace split {

// dst[r][c] = src[r][c] for c < ncols and 0 for ncols <= c < dst_cols, r < rows: pads (dst_cols >
// ncols) or crops (a narrower dst) rows.  ncols and dst_cols multiples of 8 (bf16) / 4 (fp32),
// pitches in elements, 16-byte aligned rows.
cudaError_t copy_cols(const bf16* src, long long src_pitch, bf16* dst, long long dst_pitch, long long rows,
                      long long ncols, long long dst_cols, cudaStream_t st);
cudaError_t copy_cols(const float* src, long long src_pitch, float* dst, long long dst_pitch, long long rows,
                      long long ncols, long long dst_cols, cudaStream_t st);
// Sums of fp32 column-block slices into a bf16 array: dst rows have pitch dst_pitch (elements, a
// multiple of 8, dst 16-byte aligned); their columns b*W .. b*W + W - 1, b < nblocks, are the sum
// over j < nparts of slice b * bstride + j * jstride, where slices are consecutive [rows][W] fp32
// arrays from parts.  W a multiple of 8, parts 16-byte aligned.
cudaError_t sum_blocks_to_bf16(const float* parts, long long rows, int W, int nblocks, int nparts, int bstride,
                               int jstride, bf16* dst, long long dst_pitch, cudaStream_t st);
// dst = bf16(src), n values (n a multiple of 8).
cudaError_t to_bf16(const float* src, bf16* dst, long long n, cudaStream_t st);

}  // namespace split
}  // namespace gla
