// Fused sm_100a kernels of Gated Slot Attention's first pass and the glue around the two GLA
// passes (bf16, chunk 64, d_k = 128, m = 64 slots).  The API layer asks pass1_supported() first and
// otherwise runs the generic kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "common.cuh"

namespace gla {
namespace gsa {

constexpr int kSlots = 64;

bool pass1_supported(int BH, int T, int dk, int m, int chunk, int dtype);
size_t pass1_workspace(int BH, int T, int dk);

// First pass and slot softmax: p = softmax over the slots of o1, o1_t = q_t S1_t with
// S1_t = S1_{t-1} diag(e^{g_t}) + k_t^T phi_t (S1_0 = h0 or zeros).  q, k [BH][T][dk], phi, g
// [BH][T][64], p [BH][T][64] (bf16; or, with p32 set, p32 [BH][T][64] in fp32 in its place);
// h0, hT [BH][dk][64] fp32 (optional).
cudaError_t pass1_fwd(const void* q, const void* k, const void* phi, const void* g, const float* h0, void* p,
                      float* hT, int BH, int T, int dk, void* ws, cudaStream_t st, float* p32 = nullptr);

// Softmax Jacobian over the slots: do1 = p (dp - <p, dp>) per token, from p (fp32 [rows][m]) and dp
// (fp32, row pitch dp_pitch); do1 is stored as bf16 rows [hi | lo] of 2m.
cudaError_t softmax_jacobian(const float* p, const float* dp, int dp_pitch, void* do1, long long rows, int m,
                             cudaStream_t st);

// Rows of 2m bf16 from rows of m: [hi | lo] of fp32 values (hilo) or two copies of bf16 values.
cudaError_t widen(const void* src, void* dst, long long rows, int m, bool hilo, cudaStream_t st);

// Transpose fp32 states: dst [nb][Cp][R] with dst[b][c][r] = src[b * src_bstride + r * Cc + c] for
// c < Cc and zeros for Cc <= c < Cp; with fold, plus the row r + R of src (a second copy's rows).
cudaError_t transpose_states(const float* src, long long src_bstride, float* dst, int nb, int R, int Cc, int Cp,
                             cudaStream_t st, bool fold = false);

// dst [nb][R][Cc] = src rows 0..R-1 + rows R..2R-1 of src [nb][2R][Cc].
cudaError_t fold_rows(const float* src, float* dst, int nb, int R, int Cc, cudaStream_t st);

// out [rows][m] bf16 = a[:, c] + a[:, m + c] + b[:, c] + b[:, m + c] (a, b fp32 rows of 2m).
cudaError_t fold_add_bf16(const float* a, const float* b, void* out, long long rows, int m, cudaStream_t st);

}  // namespace gsa
}  // namespace gla
