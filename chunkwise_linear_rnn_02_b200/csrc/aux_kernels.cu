// Elementwise pieces around the GLA operator: the raw-logit gate entry and the MS-GLA temporal
// pooling / causal hold (C ABI in include/gla.h).  All are HBM-bound: every thread moves 16-byte
// vectors (8 bf16 or 4 fp32 values), accumulates in fp32 and the grids are grid-stride loops
// sized to a few waves of the SMs.
//
//   gate   g = logsigmoid(x) / tau,  dx = dg * sigmoid(-x) / tau
//          ("MS-GLA: Multi-Scale Gated Linear Attention ...", section 2.1: data-dependent forget
//          gate in log space; "Gated Slot Attention ...", "Approach": sigmoid forget gates).
//   pool   y_p = mean of tokens p*s .. min(T, (p+1)*s) - 1  ("MS-GLA", section 3.1: non-overlapping
//          average pooling, padding positions masked out of the mean), ceil(T/s) outputs.
//   hold   out_t = y_{(t+1)/s - 1}, zeros while no block has completed ("MS-GLA", section 3.3: a
//          block's output is held back until every token of the block has been observed).
//   The backward passes are the transposes of pool and hold.
#include <limits.h>
#include <math.h>

#include "../../include/gla.h"
#include "common.cuh"

namespace {

using gla::bf16;

// 16-byte vector of N = 16 / sizeof(T) values, widened to fp32.
template <typename T>
struct Vec {
  static constexpr int N = 16 / sizeof(T);
  float v[N];
  __device__ __forceinline__ void load(const T* p) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    if constexpr (sizeof(T) == 4) {
      v[0] = __uint_as_float(u.x);
      v[1] = __uint_as_float(u.y);
      v[2] = __uint_as_float(u.z);
      v[3] = __uint_as_float(u.w);
    } else {
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
    }
  }
  __device__ __forceinline__ void store(T* p) const {
    uint4 u;
    if constexpr (sizeof(T) == 4) {
      u.x = __float_as_uint(v[0]);
      u.y = __float_as_uint(v[1]);
      u.z = __float_as_uint(v[2]);
      u.w = __float_as_uint(v[3]);
    } else {
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t*>(&h);
      }
      u = make_uint4(w[0], w[1], w[2], w[3]);
    }
    *reinterpret_cast<uint4*>(p) = u;
  }
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = 0.f;
  }
};

__device__ __forceinline__ float logsigmoid(float x) { return fminf(x, 0.f) - log1pf(expf(-fabsf(x))); }
__device__ __forceinline__ float sigmoid_neg(float x) {  // sigmoid(-x), without overflow
  const float e = expf(-fabsf(x));
  return x >= 0.f ? e / (1.f + e) : 1.f / (1.f + e);
}

template <typename T>
__global__ void gate_fwd_kernel(const T* __restrict__ x, T* g, size_t n, float inv_tau) {
  constexpr int N = Vec<T>::N;
  const size_t nv = n / N, stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < nv; i += stride) {
    Vec<T> a;
    a.load(x + i * N);
#pragma unroll
    for (int j = 0; j < N; ++j) a.v[j] = logsigmoid(a.v[j]) * inv_tau;
    a.store(g + i * N);
  }
  for (size_t i = nv * N + (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    gla::stf(g + i, logsigmoid(gla::ldf(x + i)) * inv_tau);
}

template <typename T>
__global__ void gate_bwd_kernel(const T* __restrict__ x, const T* dg, T* dx, size_t n, float inv_tau) {
  constexpr int N = Vec<T>::N;
  const size_t nv = n / N, stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < nv; i += stride) {
    Vec<T> a, d;
    a.load(x + i * N);
    d.load(dg + i * N);
#pragma unroll
    for (int j = 0; j < N; ++j) d.v[j] = d.v[j] * sigmoid_neg(a.v[j]) * inv_tau;
    d.store(dx + i * N);
  }
  for (size_t i = nv * N + (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    gla::stf(dx + i, gla::ldf(dg + i) * sigmoid_neg(gla::ldf(x + i)) * inv_tau);
}

// One thread per 16-byte vector of one pooled row: y_p = mean of the block's rows.
template <typename T>
__global__ void pool_kernel(const T* __restrict__ x, T* __restrict__ y, long long BH, int T_, int D, int s) {
  constexpr int N = Vec<T>::N;
  const int P = (T_ + s - 1) / s, vpr = D / N;
  const long long total = BH * P * vpr;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(e % vpr);
    const long long row = e / vpr;  // bh * P + p
    const int p = (int)(row % P);
    const long long bh = row / P;
    const int a = p * s, b = min(T_, a + s);
    Vec<T> acc, t;
    acc.zero();
    for (int r = a; r < b; ++r) {
      t.load(x + ((size_t)bh * T_ + r) * D + c * N);
#pragma unroll
      for (int j = 0; j < N; ++j) acc.v[j] += t.v[j];
    }
    const float inv = 1.f / (float)(b - a);
#pragma unroll
    for (int j = 0; j < N; ++j) acc.v[j] *= inv;
    acc.store(y + (size_t)row * D + c * N);
  }
}

// dx_t = dy_{t/s} / (rows in block t/s).
template <typename T>
__global__ void pool_bwd_kernel(const T* __restrict__ dy, T* __restrict__ dx, long long BH, int T_, int D, int s) {
  constexpr int N = Vec<T>::N;
  const int P = (T_ + s - 1) / s, vpr = D / N;
  const long long total = BH * T_ * vpr;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(e % vpr);
    const long long row = e / vpr;  // bh * T + t
    const int t = (int)(row % T_);
    const long long bh = row / T_;
    const int p = t / s;
    const float inv = 1.f / (float)(min(T_, p * s + s) - p * s);
    Vec<T> a;
    a.load(dy + ((size_t)bh * P + p) * D + c * N);
#pragma unroll
    for (int j = 0; j < N; ++j) a.v[j] *= inv;
    a.store(dx + (size_t)row * D + c * N);
  }
}

// out_t = y_{(t+1)/s - 1}, or zeros.
template <typename T>
__global__ void hold_kernel(const T* __restrict__ y, T* __restrict__ out, long long BH, int T_, int D, int s) {
  constexpr int N = Vec<T>::N;
  const int P = (T_ + s - 1) / s, vpr = D / N;
  const long long total = BH * T_ * vpr;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(e % vpr);
    const long long row = e / vpr;
    const int t = (int)(row % T_);
    const long long bh = row / T_;
    const int p = (t + 1) / s - 1;
    Vec<T> a;
    if (p >= 0)
      a.load(y + ((size_t)bh * P + p) * D + c * N);
    else
      a.zero();
    a.store(out + (size_t)row * D + c * N);
  }
}

// dy_p = sum of dout_t over the tokens t that read block p: t = (p+1)s - 1 .. (p+2)s - 2.
template <typename T>
__global__ void hold_bwd_kernel(const T* __restrict__ dout, T* __restrict__ dy, long long BH, int T_, int D, int s) {
  constexpr int N = Vec<T>::N;
  const int P = (T_ + s - 1) / s, vpr = D / N;
  const long long total = BH * P * vpr;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(e % vpr);
    const long long row = e / vpr;
    const int p = (int)(row % P);
    const long long bh = row / P;
    const int a = (p + 1) * s - 1, b = min(T_, (p + 2) * s - 1);
    Vec<T> acc, t;
    acc.zero();
    for (int r = a; r < b; ++r) {
      t.load(dout + ((size_t)bh * T_ + r) * D + c * N);
#pragma unroll
      for (int j = 0; j < N; ++j) acc.v[j] += t.v[j];
    }
    acc.store(dy + (size_t)row * D + c * N);
  }
}

int grid_for(long long items) {
  // Function-local static: looked up once (thread-safe initialisation).
  static const int sms = []() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
        n > 0)
      return n;
    return 148;
  }();
  const long long blocks = (items + 255) / 256, cap = (long long)sms * 8;
  return (int)(blocks < 1 ? 1 : blocks > cap ? cap : blocks);
}

bool aligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int need(const void* p) { return p && aligned(p) ? GLA_OK : GLA_ERR_INVALID_ARG; }

int check_tau(float tau, int dtype) {
  if (!(tau > 0.f) || !isfinite(tau)) return GLA_ERR_INVALID_ARG;
  if (dtype != GLA_DTYPE_F32 && dtype != GLA_DTYPE_BF16) return GLA_ERR_UNSUPPORTED;
  return GLA_OK;
}

int check_pool(int B, int H, int T, int D, int s, int dtype) {
  if (B <= 0 || H <= 0 || T < 0 || D <= 0 || s <= 0) return GLA_ERR_INVALID_ARG;
  if ((long long)B * H > INT_MAX || (long long)B * H * (long long)(T > 0 ? T : 1) > (1LL << 40))
    return GLA_ERR_INVALID_ARG;
  if (D > 512 || D % 8 != 0) return GLA_ERR_UNSUPPORTED;
  if (dtype != GLA_DTYPE_F32 && dtype != GLA_DTYPE_BF16) return GLA_ERR_UNSUPPORTED;
  return GLA_OK;
}

#define AUX_TRY(expr)            \
  do {                           \
    const int _s = (expr);       \
    if (_s != GLA_OK) return _s; \
  } while (0)

int launched() { return cudaGetLastError() == cudaSuccess ? GLA_OK : GLA_ERR_CUDA; }

}  // namespace

extern "C" int gla_gate_logsigmoid(const void* x, void* g, size_t n, float tau, int dtype, void* stream) {
  AUX_TRY(check_tau(tau, dtype));
  if (n == 0) return GLA_OK;
  AUX_TRY(need(x));
  AUX_TRY(need(g));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int grid = grid_for((long long)(n / 4 + 1));
  if (dtype == GLA_DTYPE_BF16)
    gate_fwd_kernel<bf16><<<grid, 256, 0, st>>>((const bf16*)x, (bf16*)g, n, 1.f / tau);
  else
    gate_fwd_kernel<float><<<grid, 256, 0, st>>>((const float*)x, (float*)g, n, 1.f / tau);
  return launched();
}

extern "C" int gla_gate_logsigmoid_bwd(const void* x, const void* dg, void* dx, size_t n, float tau, int dtype,
                                       void* stream) {
  AUX_TRY(check_tau(tau, dtype));
  if (n == 0) return GLA_OK;
  AUX_TRY(need(x));
  AUX_TRY(need(dg));
  AUX_TRY(need(dx));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int grid = grid_for((long long)(n / 4 + 1));
  if (dtype == GLA_DTYPE_BF16)
    gate_bwd_kernel<bf16><<<grid, 256, 0, st>>>((const bf16*)x, (const bf16*)dg, (bf16*)dx, n, 1.f / tau);
  else
    gate_bwd_kernel<float><<<grid, 256, 0, st>>>((const float*)x, (const float*)dg, (float*)dx, n, 1.f / tau);
  return launched();
}

// Shared driver of the four MS-GLA maps: `rows_out` rows of D values are written.
#define MSGLA_ENTRY(name, kernel, rows_out)                                                                  \
  extern "C" int name(const void* in, void* out, int B, int H, int T, int D, int s, int dtype, void* stream) { \
    AUX_TRY(check_pool(B, H, T, D, s, dtype));                                                               \
    if (T == 0) return GLA_OK;                                                                               \
    AUX_TRY(need(in));                                                                                       \
    AUX_TRY(need(out));                                                                                      \
    const long long BH = (long long)B * H, P = (T + s - 1) / s;                                              \
    (void)P;                                                                                                 \
    cudaStream_t st = static_cast<cudaStream_t>(stream);                                                     \
    const long long items = BH * (rows_out) * (D / (dtype == GLA_DTYPE_BF16 ? 8 : 4));                       \
    const int grid = grid_for(items);                                                                        \
    if (dtype == GLA_DTYPE_BF16)                                                                             \
      kernel<bf16><<<grid, 256, 0, st>>>((const bf16*)in, (bf16*)out, BH, T, D, s);                          \
    else                                                                                                     \
      kernel<float><<<grid, 256, 0, st>>>((const float*)in, (float*)out, BH, T, D, s);                       \
    return launched();                                                                                       \
  }

MSGLA_ENTRY(gla_msgla_pool, pool_kernel, P)
MSGLA_ENTRY(gla_msgla_pool_bwd, pool_bwd_kernel, T)
MSGLA_ENTRY(gla_msgla_hold, hold_kernel, T)
MSGLA_ENTRY(gla_msgla_hold_bwd, hold_bwd_kernel, P)
