// Launchers of the generic chunkwise kernels (see generic_kernels.cu for the algorithm).
#pragma once

#include "common.cuh"

namespace gla {
namespace generic {

// BH = B*H flattened heads; T tokens; DK = gated (row) dimension of the state; DV = the other
// (column) dimension; C = chunk length.
struct Shape {
  int BH, T, DK, DV, C;
};

template <typename TI>
cudaError_t state_fwd(const Shape& s, const TI* k, const TI* v, const TI* g, const float* h0, int h0_trans,
                      float* states, float* hT, int hT_trans, cudaStream_t st);

template <typename TQ, typename TI>
cudaError_t dstate_bwd(const Shape& s, const TQ* q, const TI* g, const TI* dO, const float* dhT, int dhT_trans,
                       float* dstates, float* dh0, int dh0_trans, cudaStream_t st);

template <typename TQ, typename TI, typename TO>
cudaError_t out(const Shape& s, const TQ* q, const TI* k, const TI* v, const TI* g, const float* states, TO* o,
                cudaStream_t st);

template <typename TQ, typename TI, typename TO>
cudaError_t bwd_dqdk(const Shape& s, const TQ* q, const TI* k, const TI* v, const TI* g, const TI* dO,
                     const float* states, const float* dstates, TO* dq, TO* dk, const float* dk_addend, float* db,
                     cudaStream_t st);

template <typename TQ, typename TI, typename TO>
cudaError_t bwd_dv(const Shape& s, const TQ* q, const TI* k, const TI* g, const TI* dO, const float* dstates, TO* dv,
                   cudaStream_t st);

template <typename TO>
cudaError_t dg(const Shape& s, const float* db, const float* hT, const float* dhT, int dhT_trans,
               const float* addend, TO* dg_out, cudaStream_t st);

template <typename TP>
cudaError_t softmax_fwd(const float* x, TP* p, TP* p2, long rows, int m, cudaStream_t st);

cudaError_t softmax_bwd(const float* x, const float* dp, float* dx, long rows, int m, cudaStream_t st);

template <typename TI>
cudaError_t decode(int BH, int DK, int DV, const TI* q, const TI* k, const TI* v, const TI* g, float* S, TI* o,
                   cudaStream_t st);

template <typename TI>
cudaError_t gsa_decode(int BH, int DK, int DV, int M, const TI* q, const TI* k, const TI* v, const TI* phi,
                       const TI* g, float* S1, float* S2, TI* o, cudaStream_t st);

}  // namespace generic
}  // namespace gla
