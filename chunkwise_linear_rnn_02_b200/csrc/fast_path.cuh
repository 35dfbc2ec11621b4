// Fused sm_100a (tcgen05 / TMEM / TMA) chunkwise kernels for the bf16 GLA shapes they cover.
// The API layer asks *_supported() first and otherwise runs the generic kernels.
#pragma once

#include "common.cuh"

namespace gla {

// Address of the device-side error latch (defined with the C ABI).
unsigned int* device_error_latch();

namespace fast {

bool fwd_supported(int BH, int T, int dk, int dv, int chunk, int dtype);
size_t fwd_workspace(int BH, int T, int dk, int dv);
cudaError_t fwd(const void* q, const void* k, const void* v, const void* g, const float* h0, void* o, float* hT,
                int BH, int T, int dk, int dv, void* ws, cudaStream_t st);

bool bwd_supported(int BH, int T, int dk, int dv, int chunk, int dtype);
size_t bwd_workspace(int BH, int T, int dk, int dv);
cudaError_t bwd(const void* q, const void* k, const void* v, const void* g, const float* h0, const void* dO,
                const float* dhT, void* dq, void* dk, void* dv, void* dg, float* dh0, int BH, int T, int dkd,
                int dvd, void* ws, cudaStream_t st);

}  // namespace fast
}  // namespace gla
