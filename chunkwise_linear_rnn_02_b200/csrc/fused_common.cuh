// Helpers shared by the fused sm_100a forward and backward kernels: TMA tensor maps, bf16
// packing, swizzled row stores, and the run-product gate math.
#pragma once

#include <cudaTypedefs.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>

#include "common.cuh"
#include "sm100.cuh"

namespace gla {
namespace fast {

constexpr int C = 64;  // chunk length of the fused kernels
constexpr float kLog2e = 1.4426950408889634f;
// Smallest chunk decay e^{gamma} handled by the scaled operand forms: e^-40.  A chunk that keeps
// less of its state in some key dimension (near-reset gates) takes the exact fp32 path.
constexpr float kMinDecay = 4.248354255291589e-18f;

// ------------------------------------------------------------------------------------------
// Host
// ------------------------------------------------------------------------------------------
inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  // Function-local static: initialised once, thread-safe.
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    return nullptr;
  }();
  return fn;
}

// Raise a kernel's dynamic shared-memory limit to `bytes`, once per device (the attribute belongs
// to the kernel as loaded on the current device; `done` holds one flag per device ordinal).  Two
// host threads may race here: both then set the same attribute, which is harmless, and the flag is
// atomic.
template <typename K>
inline cudaError_t ensure_smem_attr(K kern, uint32_t bytes, std::atomic<bool> (&done)[64]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev].store(true, std::memory_order_release);
  return e;
}

// 3-D map over a [BH, T, D] bf16 tensor with box (box_d, 64 tokens, 1 head); tokens past T read
// as zeros.
inline bool make_map(CUtensorMap* m, const void* base, int BH, int T, int D, int box_d, bool swizzle128) {
  auto fn = encode_fn();
  if (!fn) return false;
  memset(m, 0, sizeof(*m));
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)D * 2 * (cuuint64_t)T};
  cuuint32_t box[3] = {(cuuint32_t)box_d, (cuuint32_t)C, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------------------------------------
// Device
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ float bf2f(const uint8_t* p) {
  return __uint_as_float(static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(p)) << 16);
}
__device__ __forceinline__ float bf_round(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }
// The value a bf16 hi + lo pair represents: bf16(x) + bf16(x - bf16(x)).
__device__ __forceinline__ float bf_split_sum(float x) {
  const float h = bf_round(x);
  return h + bf_round(x - h);
}
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void fence_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Store n (a multiple of 8) fp32 values times s as bf16 into swizzled 128-byte row r of a tile;
// values 64b..64b+63 go to the 64-column block at tile + b * block_stride.
template <int N>
__device__ __forceinline__ void store_row_sw128(uint8_t* tile, int r, const float* v, float s = 1.f,
                                                uint32_t block_stride = 0) {
#pragma unroll
  for (int cc = 0; cc < N / 8; ++cc) {
    uint4 w;
    w.x = pack2(s * v[8 * cc + 0], s * v[8 * cc + 1]);
    w.y = pack2(s * v[8 * cc + 2], s * v[8 * cc + 3]);
    w.z = pack2(s * v[8 * cc + 4], s * v[8 * cc + 5]);
    w.w = pack2(s * v[8 * cc + 6], s * v[8 * cc + 7]);
    uint8_t* blk = tile + (cc >> 3) * block_stride;
    *reinterpret_cast<uint4*>(blk + r * 128 + (((cc & 7) ^ (r & 7)) << 4)) = w;
  }
}

// hi + lo bf16 split of a pair of fp32 values: hi = bf16(x), lo = bf16(x - hi).
__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
  hi = pack2(a, b);
  lo = pack2(a - bf_lo(hi), b - bf_hi(hi));
}
// Store 64 fp32 values (times s) as hi and lo bf16 rows r of two swizzled tiles.
__device__ __forceinline__ void store_row_split(uint8_t* th, uint8_t* tl, int r, const float* v, float s) {
#pragma unroll
  for (int cc = 0; cc < 8; ++cc) {
    uint4 h, l;
    split2(s * v[8 * cc + 0], s * v[8 * cc + 1], h.x, l.x);
    split2(s * v[8 * cc + 2], s * v[8 * cc + 3], h.y, l.y);
    split2(s * v[8 * cc + 4], s * v[8 * cc + 5], h.z, l.z);
    split2(s * v[8 * cc + 6], s * v[8 * cc + 7], h.w, l.w);
    const uint32_t off = r * 128 + ((cc ^ (r & 7)) << 4);
    *reinterpret_cast<uint4*>(th + off) = h;
    *reinterpret_cast<uint4*>(tl + off) = l;
  }
}

// Store 32 fp32 values as hi / lo bf16 into columns 32*hb .. 32*hb+31 of swizzled 64-column row r.
__device__ __forceinline__ void store_half_split(uint8_t* th, uint8_t* tl, int r, const float* v, int hb) {
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    uint4 h, l;
    split2(v[8 * cc + 0], v[8 * cc + 1], h.x, l.x);
    split2(v[8 * cc + 2], v[8 * cc + 3], h.y, l.y);
    split2(v[8 * cc + 4], v[8 * cc + 5], h.z, l.z);
    split2(v[8 * cc + 6], v[8 * cc + 7], h.w, l.w);
    const uint32_t off = r * 128 + ((((4 * hb + cc) ^ (r & 7)) & 7) << 4);
    *reinterpret_cast<uint4*>(th + off) = h;
    *reinterpret_cast<uint4*>(tl + off) = l;
  }
}
// Store 16 fp32 values as hi / lo bf16 into columns 16*qb .. 16*qb+15 of swizzled 64-column row r.
__device__ __forceinline__ void store_quarter_split(uint8_t* th, uint8_t* tl, int r, const float* v, int qb) {
#pragma unroll
  for (int cc = 0; cc < 2; ++cc) {
    uint4 h, l;
    split2(v[8 * cc + 0], v[8 * cc + 1], h.x, l.x);
    split2(v[8 * cc + 2], v[8 * cc + 3], h.y, l.y);
    split2(v[8 * cc + 4], v[8 * cc + 5], h.z, l.z);
    split2(v[8 * cc + 6], v[8 * cc + 7], h.w, l.w);
    const uint32_t off = r * 128 + ((((2 * qb + cc) ^ (r & 7)) & 7) << 4);
    *reinterpret_cast<uint4*>(th + off) = h;
    *reinterpret_cast<uint4*>(tl + off) = l;
  }
}
// Store 32 fp32 values as bf16 to global (16-byte aligned destination).
__device__ __forceinline__ void store_half_global_bf16(__nv_bfloat16* dst, const float* v) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    uint4 w;
    w.x = pack2(v[8 * cc + 0], v[8 * cc + 1]);
    w.y = pack2(v[8 * cc + 2], v[8 * cc + 3]);
    w.z = pack2(v[8 * cc + 4], v[8 * cc + 5]);
    w.w = pack2(v[8 * cc + 6], v[8 * cc + 7]);
    d[cc] = w;
  }
}


// Named barriers (id 0 is __syncthreads).  bar_sync waits; bar_arrive signals without waiting (a
// producer warp syncs on a barrier that the consumer threads only arrive at); bar_or is a barrier
// that also ORs a predicate over the participating threads.  Counts are in threads; every warp
// taking part executes the instruction with all its lanes.
__device__ __forceinline__ void bar_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
__device__ __forceinline__ void bar_arrive(int id, int n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ int bar_or(int id, int n, int pred) {
  int r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.s32 p, %3, 0;\n\tbar.red.or.pred q, %1, %2, p;\n\tselp.s32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(id), "r"(n), "r"(pred)
      : "memory");
  return r;
}
constexpr int kBarCompute = 1;  // named barrier of the threads that run the gate math

// Gate math shared by the fused kernels.  The CTA's NTH threads cover ND key dimensions of one
// chunk: thread t owns dimensions (2p, 2p+1), p = t % (ND/2), and the run of TS = 64 * (ND/2) / NTH
// tokens starting at h * TS, h = t / (ND/2).  It loads the raw log-gates g (row-major [64][gstride]
// bf16 at `graw`, columns col0..), computes alpha = e^g with one ex2 per value, and leaves in
// registers the run's alphas and, via the shared buffer `tot` (NSPLIT x ND floats), the products of
// the other runs: pre = prod of earlier runs, suf = prod of later runs, dec = e^{gamma}.  `tot` and
// the decay arrays given to store_decay are 8-byte aligned (each thread moves its pair as a float2).
//
// Raw-logit gates (LOGIT builds): with inv_tau > 0 the tile holds logits x instead of log-gates, and
// the run first replaces every element of it, in place, by g = bf16(logsigmoid(x) * inv_tau) (0 for
// the tokens at or past `valid`, which lie beyond the end of the sequence), the values the
// standalone gate entry would store; everything that reads the tile afterwards sees those
// log-gates.  The caller runs exactly one gate run per loaded tile, before any other reader of it.
// The transform is a loop of its own ahead of the gate loop, so builds without it compile the gate
// loop unchanged.
__device__ __forceinline__ float logsigmoid_scaled(float x, float inv_tau) {
  return (fminf(x, 0.f) - log1pf(expf(-fabsf(x)))) * inv_tau;
}

template <int ND, int NTH, bool LOGIT = false>
struct GateRun {
  static constexpr int NPAIR = ND / 2;
  static constexpr int NSPLIT = NTH / NPAIR;
  static constexpr int TS = C / NSPLIT;
  static_assert(NSPLIT * NPAIR == NTH && NSPLIT * TS == C, "gate thread split");
  float a0[TS], a1[TS];
  float pre0, pre1, suf0, suf1, dec0, dec1;
  int p, h, d;
  float inv_tau = 0.f;  // > 0: the tile holds raw logits (see above)
  int valid = C;        // tokens of the tile inside the sequence (raw-logit mode)

  __device__ __forceinline__ void set_logit(float inv_tau_, int tokens_left) {
    inv_tau = inv_tau_;
    valid = tokens_left < C ? tokens_left : C;
  }

  // Returns true when this thread's dimensions keep less than kMinDecay of the state.
  __device__ __forceinline__ bool run(const uint8_t* graw, int gstride, float* tot) {
    return run_impl(graw, gstride, tot, false);
  }
  // Same for a [64][64] tile stored with the 128-byte swizzle (ND == 64).
  __device__ __forceinline__ bool run_swizzled(const uint8_t* graw, float* tot) {
    return run_impl(graw, 64, tot, true);
  }
  __device__ __forceinline__ bool run_impl(const uint8_t* graw, int gstride, float* tot, bool swz) {
    const int tid = threadIdx.x;
    p = tid % NPAIR;
    h = tid / NPAIR;
    d = 2 * p;
    if (LOGIT && inv_tau > 0.f) {
#pragma unroll 1
      for (int u = 0; u < TS; ++u) {
        const int j = h * TS + u;
        uint32_t* ptr = reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(graw) +
                                                    (swz ? sm100::sw128(j, d) : (j * gstride + d) * 2));
        const uint32_t w = *ptr;
        *ptr = j < valid ? pack2(logsigmoid_scaled(bf_lo(w), inv_tau), logsigmoid_scaled(bf_hi(w), inv_tau)) : 0u;
      }
    }
    float r0 = 1.f, r1 = 1.f;
#pragma unroll
    for (int u = 0; u < TS; ++u) {
      const int j = h * TS + u;
      const uint32_t w = *reinterpret_cast<const uint32_t*>(graw + (swz ? sm100::sw128(j, d) : (j * gstride + d) * 2));
      a0[u] = ex2(bf_lo(w) * kLog2e);
      a1[u] = ex2(bf_hi(w) * kLog2e);
      r0 *= a0[u];
      r1 *= a1[u];
    }
    // one float2 per thread (tot is 8-byte aligned): a warp's 32 pairs take two wavefronts, where
    // two scalar accesses of stride 8 bytes would each meet a 2-way bank conflict
    *reinterpret_cast<float2*>(tot + h * ND + d) = make_float2(r0, r1);
    bar_sync(kBarCompute, NTH);  // the NTH threads running the gate math
    pre0 = pre1 = suf0 = suf1 = 1.f;
#pragma unroll
    for (int hh = 0; hh < NSPLIT; ++hh) {
      const float2 t = *reinterpret_cast<const float2*>(tot + hh * ND + d);
      if (hh < h) {
        pre0 *= t.x;
        pre1 *= t.y;
      } else if (hh > h) {
        suf0 *= t.x;
        suf1 *= t.y;
      }
    }
    dec0 = pre0 * r0 * suf0;
    dec1 = pre1 * r1 * suf1;
    return !(dec0 >= kMinDecay && dec1 >= kMinDecay);
  }

  // dec0, dec1 into dst[d], dst[d + 1].
  __device__ __forceinline__ void store_decay(float* dst) const {
    *reinterpret_cast<float2*>(dst + d) = make_float2(dec0, dec1);
  }

  // The thread's pair of bf16 values for every token of its run, from a [64][ND] tile (row stride
  // `stride` elements, or the 128-byte swizzle), all loaded before any is used: the loops that
  // consume them store to shared memory, and a load cannot move above such a store.
  __device__ __forceinline__ void load_pairs(const uint8_t* src, int stride, bool swz, uint32_t (&w)[TS]) const {
#pragma unroll
    for (int u = 0; u < TS; ++u) {
      const int j = h * TS + u;
      w[u] = *reinterpret_cast<const uint32_t*>(src + (swz ? sm100::sw128(j, d) : (j * stride + d) * 2));
    }
  }

  // For each token j of the run: f(j, E1_0, E1_1) with E1 = e^{B_j} (inclusive products).
  template <typename F>
  __device__ __forceinline__ void forward(F f) const {
    float e0 = pre0, e1 = pre1;
#pragma unroll
    for (int u = 0; u < TS; ++u) {
      e0 *= a0[u];
      e1 *= a1[u];
      f(h * TS + u, e0, e1);
    }
  }
  // For each token j of the run (in reverse): f(j, E2_0, E2_1) with E2 = e^{gamma - B_j}.
  template <typename F>
  __device__ __forceinline__ void backward(F f) const {
    float e0 = suf0, e1 = suf1;
#pragma unroll
    for (int u = TS - 1; u >= 0; --u) {
      f(h * TS + u, e0, e1);
      e0 *= a0[u];
      e1 *= a1[u];
    }
  }
};

}  // namespace fast
}  // namespace gla
