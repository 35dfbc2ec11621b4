// Fused sm_100a chunkwise kernels: not yet covering any shape; every call takes the generic path.
#include "fast_path.cuh"

namespace gla {
namespace fast {

bool fwd_supported(int, int, int, int, int, int) { return false; }
size_t fwd_workspace(int, int, int, int) { return 0; }
cudaError_t fwd(const void*, const void*, const void*, const void*, const float*, void*, float*, int, int, int, int,
                void*, cudaStream_t) {
  return cudaErrorNotSupported;
}
bool bwd_supported(int, int, int, int, int, int) { return false; }
size_t bwd_workspace(int, int, int, int) { return 0; }
cudaError_t bwd(const void*, const void*, const void*, const void*, const float*, const void*, const float*, void*,
                void*, void*, void*, float*, int, int, int, int, void*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace fast
}  // namespace gla
