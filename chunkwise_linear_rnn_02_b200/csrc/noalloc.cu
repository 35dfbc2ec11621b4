// gla_chunk_bwd_noalloc: the fused backward for callers that cannot hand the library a workspace.
//
// Some callers have no way to obtain device memory for a workspace: a plain C host with no device
// allocator of its own, a runtime whose device memory is carved up up front and handed out only
// for tensors, or code that must not call cudaMalloc because that call may synchronise the device
// in the middle of its work.  This entry point needs nothing from them but the inputs and outputs:
// its scratch is a fixed array in this file, reserved on each device that loads the library's code
// for this file and kept there until the process exits.
//
// Set-up: the first call on a device looks up the array's device address with
// cudaGetSymbolAddress (the array's name is only a host-side stand-in in host code) and caches it;
// that first call on each device should therefore come before any stream capture.  Every call
// shares the one array, so calls that overlap on the GPU (two streams, or two threads) race on it.
// Nothing in it has to start at zero: every value is written before it is read in the same call.
// It allocates nothing: no cudaMalloc, no cudaFree, no allocating library routine.
#include <limits.h>

#include <mutex>

#include "../../include/gla.h"
#include "common.cuh"
#include "fast_path.cuh"

namespace {

constexpr size_t kScratchBytes = size_t(128) << 20;  // 128 MiB
__device__ __align__(256) unsigned char g_bwd_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once per device).
int scratch_on_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return GLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || !p) return GLA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return GLA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int gla_chunk_bwd_noalloc(const void* q, const void* k, const void* v, const void* g, const float* h0,
                                     const void* dO, const float* dhT, void* dq, void* dk, void* dv, void* dg,
                                     float* dh0, int B, int H, int T, int dk_dim, int dv_dim, int chunk, int dtype,
                                     void* stream) {
  if (B <= 0 || H <= 0 || T <= 0 || (long long)B * H > INT_MAX) return GLA_ERR_INVALID_ARG;
  if (dtype != GLA_DTYPE_BF16 || chunk != 64 || dk_dim != 128 || (dv_dim != 128 && dv_dim != 256))
    return GLA_ERR_UNSUPPORTED;
  const void* req[] = {q, k, v, g, dO, dq, dk, dv, dg};
  for (const void* p : req)
    if (!p || !aligned16(p)) return GLA_ERR_INVALID_ARG;
  const void* opt[] = {h0, dhT, dh0};
  for (const void* p : opt)
    if (p && !aligned16(p)) return GLA_ERR_INVALID_ARG;
  const int BH = B * H;
  // The size limit is plain host arithmetic on the sizes, so it is checked before anything that
  // needs the driver.
  if (gla::fast::bwd_workspace(BH, T, dk_dim, dv_dim) > kScratchBytes) return GLA_ERR_WORKSPACE;
  if (!gla::fast::bwd_supported(BH, T, dk_dim, dv_dim, chunk, dtype)) return GLA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const int st = scratch_on_current_device(&scratch);
  if (st != GLA_OK) return st;
  return gla::fast::bwd(q, k, v, g, h0, dO, dhT, dq, dk, dv, dg, dh0, BH, T, dk_dim, dv_dim, scratch,
                        static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? GLA_OK
             : GLA_ERR_CUDA;
}
