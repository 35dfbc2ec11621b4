// Generic chunkwise GLA kernels (CUDA cores, fp32 arithmetic, any supported shape).
//
// These kernels implement the chunkwise form of the key-gated recurrence
//     S_t = diag(exp g_t) S_{t-1} + k_t^T v_t ,   o_t = q_t S_t
// ("MS-GLA: Multi-Scale Gated Linear Attention ...", section 2.1: sequential inter-chunk state
// updates, parallel intra-chunk work) as a set of chunk-parallel passes that exchange the
// per-chunk states through the workspace:
//
//   state_fwd   S_i (state entering chunk i) for every chunk, and S_N = hT     (sequential in i)
//   out         o = (q * e^B) S_i + A v, A = gated causal q k^T inside a chunk    (parallel in i)
//   dstate_bwd  G_{i+1} = dL/dS_{i+1} for every chunk, and dh0                   (sequential, reversed)
//   bwd_dqdk    dq, dk and db = q*dq - k*dk for a block of key dimensions          (parallel in i)
//   bwd_dv      dv for a block of value dimensions                                (parallel in i)
//   dg          dg = reverse cumulative sum over t of db, plus the hT term
//
// Inside a chunk, B_j is the inclusive fp32 cumulative sum of g over the chunk.  The intra-chunk
// decay exp(B_j - B_r) (r <= j) is evaluated with secondary 16-token sub-chunks so that no
// exponential can overflow: for r in an earlier sub-chunk than j it is split as
// exp(B_j - rho) * exp(rho - B_r) with rho = B at the last token before j's sub-chunk (both
// exponents <= 0 because g <= 0); inside the diagonal sub-chunk it is evaluated exactly per
// element.  Tail positions t >= T behave as g = 0, k = v = q = 0.
//
// The same kernels serve GSA: its slot-gated first pass is the key-gated pass with roles
// exchanged (see gla_api.cu), so every kernel takes the "query" operand type TQ, the type TI
// of the other inputs and the output type TO as template parameters.
#include "common.cuh"
#include "generic_kernels.cuh"

namespace gla {
namespace generic {

constexpr int TB = 64;    // tile width along d_k / d_v
constexpr int LD = 65;    // padded leading dimension of shared tiles
constexpr int NT = 256;   // threads per CTA
constexpr int SUB = 16;   // secondary sub-chunk length

template <int C>
struct Geo {
  static constexpr int NSUB = C / SUB;
  static constexpr int KF_ROWS = SUB * NSUB * (NSUB - 1) / 2;  // key rows scaled per query sub-chunk
  static constexpr int EPT = C * C / NT;                        // A entries per thread
  static constexpr int OPT = C * TB / NT;                       // output entries per thread
};

__host__ __device__ __forceinline__ int kf_offset(int I) { return SUB * I * (I - 1) / 2; }

// Load a [C x TB] tile of a [BH, T, D] tensor (rows t0.., columns c0..) into shared memory
// with leading dimension LD, zero-filling rows >= T and columns >= D.
template <int C, typename T>
__device__ __forceinline__ void load_tile(float* dst, const T* __restrict__ src, int bh, int t0,
                                          int T_len, int D, int c0) {
  for (int e = threadIdx.x; e < C * TB; e += NT) {
    const int j = e / TB, c = e % TB;
    const int t = t0 + j, cc = c0 + c;
    float x = 0.f;
    if (t < T_len && cc < D) x = ldf(src + ((size_t)bh * T_len + t) * D + cc);
    dst[j * LD + c] = x;
  }
}

// Load a [TB x TB] block (rows r0.., cols c0..) of a [rows x cols] fp32 matrix.
__device__ __forceinline__ void load_state_block(float* dst, const float* __restrict__ src,
                                                 int rows, int cols, int r0, int c0) {
  for (int e = threadIdx.x; e < TB * TB; e += NT) {
    const int r = e / TB, c = e % TB;
    float x = 0.f;
    if (r0 + r < rows && c0 + c < cols) x = src[(size_t)(r0 + r) * cols + c0 + c];
    dst[r * LD + c] = x;
  }
}

// In-place inclusive cumulative sum of a [C x TB] gate tile along rows (one thread per column).
template <int C>
__device__ __forceinline__ void cumsum_cols(float* Bs) {
  if (threadIdx.x < TB) {
    float b = 0.f;
    for (int j = 0; j < C; ++j) {
      b += Bs[j * LD + threadIdx.x];
      Bs[j * LD + threadIdx.x] = b;
    }
  }
}

// Sub-chunk reference points rho[I][d] = B[16I-1][d] (I >= 1), query factors
// qf[j] = q[j] exp(B[j] - rho_{I(j)}) and key factors kf_I[r] = k[r] exp(rho_I - B[r]), r < 16I.
template <int C>
__device__ __forceinline__ void subchunk_factors(const float* qs, const float* ks, const float* Bs,
                                                 float* qf, float* kf, float* rho) {
  using G = Geo<C>;
  for (int e = threadIdx.x; e < G::NSUB * TB; e += NT) {
    const int I = e / TB, d = e % TB;
    rho[I * TB + d] = (I == 0) ? 0.f : Bs[(SUB * I - 1) * LD + d];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < C * TB; e += NT) {
    const int j = e / TB, d = e % TB;
    const int I = j / SUB;
    qf[j * LD + d] = (I == 0) ? 0.f : qs[j * LD + d] * expf(Bs[j * LD + d] - rho[I * TB + d]);
  }
  for (int e = threadIdx.x; e < G::KF_ROWS * TB; e += NT) {
    const int row = e / TB, d = e % TB;
    int I = 1;
    while (kf_offset(I + 1) <= row) ++I;
    const int r = row - kf_offset(I);
    kf[row * LD + d] = ks[r * LD + d] * expf(rho[I * TB + d] - Bs[r * LD + d]);
  }
}

// Accumulate this thread's A[j][r0 .. r0+EPT) over one block of TB key dimensions:
// A[j][r] = sum_d q[j][d] k[r][d] exp(B[j][d] - B[r][d]) for r <= j (0 above the diagonal).
template <int C>
__device__ __forceinline__ void accumulate_A(float* acc, int j, int r0, const float* qs,
                                             const float* ks, const float* Bs, const float* qf,
                                             const float* kf) {
  using G = Geo<C>;
  const int I = j / SUB;
  for (int u = 0; u < G::EPT; ++u) {
    const int r = r0 + u;
    if (r > j) continue;
    float s = 0.f;
    if (r / SUB == I) {
      for (int d = 0; d < TB; ++d)
        s += qs[j * LD + d] * ks[r * LD + d] * expf(Bs[j * LD + d] - Bs[r * LD + d]);
    } else {
      const float* kr = kf + (kf_offset(I) + r) * LD;
      for (int d = 0; d < TB; ++d) s += qf[j * LD + d] * kr[d];
    }
    acc[u] += s;
  }
}

// ---------------------------------------------------------------------------------------------
// state_fwd: grid (ceil(DV/64), ceil(DK/64), BH).  S tile [64 x 64] in registers, 16 per thread.
// ---------------------------------------------------------------------------------------------
template <int C, typename TI>
__global__ void __launch_bounds__(NT) state_fwd_kernel(const TI* __restrict__ k, const TI* __restrict__ v,
                                                       const TI* __restrict__ g, const float* __restrict__ h0,
                                                       int h0_trans, float* __restrict__ states,
                                                       float* __restrict__ hT, int hT_trans, int T, int DK,
                                                       int DV) {
  extern __shared__ float smem[];
  float* Bs = smem;
  float* ks = Bs + C * LD;
  float* vs = ks + C * LD;
  float* decay = vs + C * LD;
  const int bh = blockIdx.z, d0 = blockIdx.y * TB, c0 = blockIdx.x * TB;
  const int r = threadIdx.x / 4, cb = (threadIdx.x % 4) * 16;
  const int NC = num_chunks(T, C);
  const size_t sz = (size_t)DK * DV;
  float S[16];
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const int d = d0 + r, c = c0 + cb + u;
    float x = 0.f;
    if (h0 && d < DK && c < DV)
      x = h0_trans ? h0[bh * sz + (size_t)c * DK + d] : h0[bh * sz + (size_t)d * DV + c];
    S[u] = x;
  }
  for (int i = 0; i < NC; ++i) {
    load_tile<C>(Bs, g, bh, i * C, T, DK, d0);
    load_tile<C>(ks, k, bh, i * C, T, DK, d0);
    load_tile<C>(vs, v, bh, i * C, T, DV, c0);
    __syncthreads();
    cumsum_cols<C>(Bs);
    if (threadIdx.x < TB) {
      const float gam = Bs[(C - 1) * LD + threadIdx.x];
      for (int j = 0; j < C; ++j) ks[j * LD + threadIdx.x] *= expf(gam - Bs[j * LD + threadIdx.x]);
      decay[threadIdx.x] = expf(gam);
    }
    __syncthreads();
    if (states && d0 + r < DK) {
      float* dst = states + ((size_t)bh * NC + i) * sz + (size_t)(d0 + r) * DV + c0 + cb;
#pragma unroll
      for (int u = 0; u < 16; ++u)
        if (c0 + cb + u < DV) dst[u] = S[u];
    }
    const float dr = decay[r];
#pragma unroll
    for (int u = 0; u < 16; ++u) S[u] *= dr;
    for (int j = 0; j < C; ++j) {
      const float kv = ks[j * LD + r];
#pragma unroll
      for (int u = 0; u < 16; ++u) S[u] += kv * vs[j * LD + cb + u];
    }
    __syncthreads();
  }
  if (hT && d0 + r < DK) {
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int c = c0 + cb + u;
      if (c < DV) {
        if (hT_trans)
          hT[bh * sz + (size_t)c * DK + d0 + r] = S[u];
        else
          hT[bh * sz + (size_t)(d0 + r) * DV + c] = S[u];
      }
    }
  }
}

// ---------------------------------------------------------------------------------------------
// dstate_bwd: reverse walk.  G_N = dhT; store G_{i+1} for chunk i; G_i = e^gamma G_{i+1} + Qt^T dO.
// ---------------------------------------------------------------------------------------------
template <int C, typename TQ, typename TI>
__global__ void __launch_bounds__(NT) dstate_bwd_kernel(const TQ* __restrict__ q, const TI* __restrict__ g,
                                                        const TI* __restrict__ dO, const float* __restrict__ dhT,
                                                        int dhT_trans, float* __restrict__ dstates,
                                                        float* __restrict__ dh0, int dh0_trans, int T, int DK,
                                                        int DV) {
  extern __shared__ float smem[];
  float* Bs = smem;
  float* qs = Bs + C * LD;
  float* ds = qs + C * LD;
  float* decay = ds + C * LD;
  const int bh = blockIdx.z, d0 = blockIdx.y * TB, c0 = blockIdx.x * TB;
  const int r = threadIdx.x / 4, cb = (threadIdx.x % 4) * 16;
  const int NC = num_chunks(T, C);
  const size_t sz = (size_t)DK * DV;
  float D[16];
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const int d = d0 + r, c = c0 + cb + u;
    float x = 0.f;
    if (dhT && d < DK && c < DV)
      x = dhT_trans ? dhT[bh * sz + (size_t)c * DK + d] : dhT[bh * sz + (size_t)d * DV + c];
    D[u] = x;
  }
  for (int i = NC - 1; i >= 0; --i) {
    load_tile<C>(Bs, g, bh, i * C, T, DK, d0);
    load_tile<C>(qs, q, bh, i * C, T, DK, d0);
    load_tile<C>(ds, dO, bh, i * C, T, DV, c0);
    __syncthreads();
    cumsum_cols<C>(Bs);
    if (threadIdx.x < TB) {
      for (int j = 0; j < C; ++j) qs[j * LD + threadIdx.x] *= expf(Bs[j * LD + threadIdx.x]);
      decay[threadIdx.x] = expf(Bs[(C - 1) * LD + threadIdx.x]);
    }
    __syncthreads();
    if (dstates && d0 + r < DK) {
      float* dst = dstates + ((size_t)bh * NC + i) * sz + (size_t)(d0 + r) * DV + c0 + cb;
#pragma unroll
      for (int u = 0; u < 16; ++u)
        if (c0 + cb + u < DV) dst[u] = D[u];
    }
    const float dr = decay[r];
#pragma unroll
    for (int u = 0; u < 16; ++u) D[u] *= dr;
    for (int j = 0; j < C; ++j) {
      const float qv = qs[j * LD + r];
#pragma unroll
      for (int u = 0; u < 16; ++u) D[u] += qv * ds[j * LD + cb + u];
    }
    __syncthreads();
  }
  if (dh0 && d0 + r < DK) {
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int c = c0 + cb + u;
      if (c < DV) {
        if (dh0_trans)
          dh0[bh * sz + (size_t)c * DK + d0 + r] = D[u];
        else
          dh0[bh * sz + (size_t)(d0 + r) * DV + c] = D[u];
      }
    }
  }
}

// ---------------------------------------------------------------------------------------------
// out: grid (ceil(DV/64), NC, BH).  o = (q * e^B) S_i + A v for one chunk and 64 value columns.
// ---------------------------------------------------------------------------------------------
template <int C>
struct OutSmem {
  static constexpr int floats = 4 * C * LD + Geo<C>::KF_ROWS * LD + TB * LD + C * (C + 1) + C * LD +
                                Geo<C>::NSUB * TB;
};

template <int C, typename TQ, typename TI, typename TO>
__global__ void __launch_bounds__(NT) out_kernel(const TQ* __restrict__ q, const TI* __restrict__ k,
                                                 const TI* __restrict__ v, const TI* __restrict__ g,
                                                 const float* __restrict__ states, TO* __restrict__ o, int T,
                                                 int DK, int DV) {
  using G = Geo<C>;
  extern __shared__ float smem[];
  float* qs = smem;
  float* ks = qs + C * LD;
  float* Bs = ks + C * LD;
  float* qf = Bs + C * LD;
  float* kf = qf + C * LD;
  float* Ss = kf + G::KF_ROWS * LD;
  float* As = Ss + TB * LD;
  float* vs = As + C * (C + 1);
  float* rho = vs + C * LD;
  const int bh = blockIdx.z, i = blockIdx.y, c0 = blockIdx.x * TB;
  const int NC = num_chunks(T, C);
  const int ja = (threadIdx.x * G::EPT) / C, ra = (threadIdx.x * G::EPT) % C;
  const int jo = (threadIdx.x * G::OPT) / TB, co = (threadIdx.x * G::OPT) % TB;
  float accA[G::EPT];
  float accO[G::OPT];
#pragma unroll
  for (int u = 0; u < G::EPT; ++u) accA[u] = 0.f;
#pragma unroll
  for (int u = 0; u < G::OPT; ++u) accO[u] = 0.f;
  const float* Si = states + ((size_t)bh * NC + i) * DK * DV;
  for (int d0 = 0; d0 < DK; d0 += TB) {
    load_tile<C>(qs, q, bh, i * C, T, DK, d0);
    load_tile<C>(ks, k, bh, i * C, T, DK, d0);
    load_tile<C>(Bs, g, bh, i * C, T, DK, d0);
    load_state_block(Ss, Si, DK, DV, d0, c0);
    __syncthreads();
    cumsum_cols<C>(Bs);
    __syncthreads();
    subchunk_factors<C>(qs, ks, Bs, qf, kf, rho);
    __syncthreads();
    accumulate_A<C>(accA, ja, ra, qs, ks, Bs, qf, kf);
    // inter-chunk term: (q * e^B) S_i
    for (int d = 0; d < TB; ++d) {
      const float qe = qs[jo * LD + d] * expf(Bs[jo * LD + d]);
#pragma unroll
      for (int u = 0; u < G::OPT; ++u) accO[u] += qe * Ss[d * LD + co + u];
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < G::EPT; ++u) As[ja * (C + 1) + ra + u] = accA[u];
  load_tile<C>(vs, v, bh, i * C, T, DV, c0);
  __syncthreads();
  for (int r = 0; r <= jo; ++r) {
    const float a = As[jo * (C + 1) + r];
#pragma unroll
    for (int u = 0; u < G::OPT; ++u) accO[u] += a * vs[r * LD + co + u];
  }
  const int t = i * C + jo;
  if (t < T) {
#pragma unroll
    for (int u = 0; u < G::OPT; ++u)
      if (c0 + co + u < DV) stf(o + ((size_t)bh * T + t) * DV + c0 + co + u, accO[u]);
  }
}

// ---------------------------------------------------------------------------------------------
// bwd_dqdk: grid (ceil(DK/64), NC, BH).  For 64 key dimensions of one chunk:
//   dA[j][r] = dO_j . v_r (r <= j)
//   dq_j = e^{B_j} (dO_j S_i^T) + sum_{r<=j} dA[j][r] k_r e^{B_j - B_r}
//   dk_r = e^{gamma - B_r} (v_r G_{i+1}^T) + sum_{j>=r} dA[j][r] q_j e^{B_j - B_r}
//   db   = q dq - k dk
// ---------------------------------------------------------------------------------------------
template <int C>
struct DqdkSmem {
  static constexpr int floats = 4 * C * LD + Geo<C>::KF_ROWS * LD + Geo<C>::NSUB * TB + 2 * C * LD +
                                2 * TB * LD + C * (C + 1);
};

template <int C, typename TQ, typename TI, typename TO>
__global__ void __launch_bounds__(NT) bwd_dqdk_kernel(
    const TQ* __restrict__ q, const TI* __restrict__ k, const TI* __restrict__ v, const TI* __restrict__ g,
    const TI* __restrict__ dO, const float* __restrict__ states, const float* __restrict__ dstates,
    TO* __restrict__ dq, TO* __restrict__ dk, const float* __restrict__ dk_addend, float* __restrict__ db,
    int T, int DK, int DV) {
  using G = Geo<C>;
  extern __shared__ float smem[];
  float* qs = smem;
  float* ks = qs + C * LD;
  float* Bs = ks + C * LD;
  float* qf = Bs + C * LD;
  float* kf = qf + C * LD;
  float* rho = kf + G::KF_ROWS * LD;
  float* vs = rho + G::NSUB * TB;
  float* ds = vs + C * LD;
  float* Ss = ds + C * LD;
  float* Gs = Ss + TB * LD;
  float* dAs = Gs + TB * LD;
  const int bh = blockIdx.z, i = blockIdx.y, d0 = blockIdx.x * TB;
  const int NC = num_chunks(T, C);
  const int ja = (threadIdx.x * G::EPT) / C, ra = (threadIdx.x * G::EPT) % C;
  const int jo = (threadIdx.x * G::OPT) / TB, co = (threadIdx.x * G::OPT) % TB;  // co: key-dim offset
  load_tile<C>(qs, q, bh, i * C, T, DK, d0);
  load_tile<C>(ks, k, bh, i * C, T, DK, d0);
  load_tile<C>(Bs, g, bh, i * C, T, DK, d0);
  __syncthreads();
  cumsum_cols<C>(Bs);
  __syncthreads();
  subchunk_factors<C>(qs, ks, Bs, qf, kf, rho);
  float accA[G::EPT], dqi[G::OPT], dki[G::OPT];
#pragma unroll
  for (int u = 0; u < G::EPT; ++u) accA[u] = 0.f;
#pragma unroll
  for (int u = 0; u < G::OPT; ++u) dqi[u] = dki[u] = 0.f;
  const size_t sz = (size_t)DK * DV;
  const float* Si = states ? states + ((size_t)bh * NC + i) * sz : nullptr;
  const float* Gi = dstates ? dstates + ((size_t)bh * NC + i) * sz : nullptr;
  for (int c0 = 0; c0 < DV; c0 += TB) {
    __syncthreads();
    load_tile<C>(vs, v, bh, i * C, T, DV, c0);
    load_tile<C>(ds, dO, bh, i * C, T, DV, c0);
    if (Si) load_state_block(Ss, Si, DK, DV, d0, c0);
    if (Gi) load_state_block(Gs, Gi, DK, DV, d0, c0);
    __syncthreads();
#pragma unroll
    for (int u = 0; u < G::EPT; ++u) {
      const int r = ra + u;
      if (r > ja) continue;
      float s = 0.f;
      for (int c = 0; c < TB; ++c) s += ds[ja * LD + c] * vs[r * LD + c];
      accA[u] += s;
    }
    for (int c = 0; c < TB; ++c) {
      const float dov = ds[jo * LD + c], vv = vs[jo * LD + c];
#pragma unroll
      for (int u = 0; u < G::OPT; ++u) {
        if (Si) dqi[u] += dov * Ss[(co + u) * LD + c];
        if (Gi) dki[u] += vv * Gs[(co + u) * LD + c];
      }
    }
  }
#pragma unroll
  for (int u = 0; u < G::EPT; ++u) dAs[ja * (C + 1) + ra + u] = accA[u];
  __syncthreads();
  const int I = jo / SUB;
  const int t = i * C + jo;
  float outq[G::OPT], outk[G::OPT];
#pragma unroll
  for (int u = 0; u < G::OPT; ++u) {
    const int d = co + u;
    const float bj = Bs[jo * LD + d];
    // dq: inter + diagonal sub-chunk (exact) + earlier sub-chunks (factored through rho_I)
    float sq = expf(bj) * dqi[u];
    for (int r = I * SUB; r <= jo; ++r) sq += dAs[jo * (C + 1) + r] * ks[r * LD + d] * expf(bj - Bs[r * LD + d]);
    if (I > 0) {
      float so = 0.f;
      const float* kI = kf + kf_offset(I) * LD;
      for (int r = 0; r < I * SUB; ++r) so += dAs[jo * (C + 1) + r] * kI[r * LD + d];
      sq += expf(bj - rho[I * TB + d]) * so;
    }
    // dk (row jo plays the key position r): inter + diagonal + later sub-chunks
    const float gam = Bs[(C - 1) * LD + d];
    float sk = expf(gam - bj) * dki[u];
    const int Iend = min((I + 1) * SUB, C);
    for (int jj = jo; jj < Iend; ++jj) sk += dAs[jj * (C + 1) + jo] * qs[jj * LD + d] * expf(Bs[jj * LD + d] - bj);
    for (int I2 = I + 1; I2 < G::NSUB; ++I2) {
      float so = 0.f;
      for (int jj = I2 * SUB; jj < (I2 + 1) * SUB; ++jj) so += dAs[jj * (C + 1) + jo] * qf[jj * LD + d];
      sk += expf(rho[I2 * TB + d] - bj) * so;
    }
    outq[u] = sq;
    outk[u] = sk;
  }
  if (t < T) {
    const size_t row = ((size_t)bh * T + t) * DK + d0 + co;
#pragma unroll
    for (int u = 0; u < G::OPT; ++u) {
      if (d0 + co + u >= DK) continue;
      float kk = outk[u];
      if (dk_addend) kk += dk_addend[row + u];
      if (dq) stf(dq + row + u, outq[u]);
      if (dk) stf(dk + row + u, kk);
      // The r = j = t terms of dq_t and dk_t (dA[t][t] k_t and dA[t][t] q_t) cancel exactly in
      // q*dq - k*dk; leaving them out avoids cancellation when the gates decay strongly.
      if (db) {
        const float a = dAs[jo * (C + 1) + jo], qv = qs[jo * LD + co + u], kv = ks[jo * LD + co + u];
        db[row + u] = qv * (outq[u] - a * kv) - kv * (outk[u] - a * qv);
      }
    }
  }
}

// ---------------------------------------------------------------------------------------------
// bwd_dv: grid (ceil(DV/64), NC, BH).  dv_r = (k_r e^{gamma - B_r}) G_{i+1} + sum_{j>=r} A[j][r] dO_j.
// ---------------------------------------------------------------------------------------------
template <int C, typename TQ, typename TI, typename TO>
__global__ void __launch_bounds__(NT) bwd_dv_kernel(const TQ* __restrict__ q, const TI* __restrict__ k,
                                                    const TI* __restrict__ g, const TI* __restrict__ dO,
                                                    const float* __restrict__ dstates, TO* __restrict__ dv, int T,
                                                    int DK, int DV) {
  using G = Geo<C>;
  extern __shared__ float smem[];
  float* qs = smem;
  float* ks = qs + C * LD;
  float* Bs = ks + C * LD;
  float* qf = Bs + C * LD;
  float* kf = qf + C * LD;
  float* Gs = kf + G::KF_ROWS * LD;
  float* As = Gs + TB * LD;
  float* ds = As + C * (C + 1);
  float* rho = ds + C * LD;
  const int bh = blockIdx.z, i = blockIdx.y, c0 = blockIdx.x * TB;
  const int NC = num_chunks(T, C);
  const int ja = (threadIdx.x * G::EPT) / C, ra = (threadIdx.x * G::EPT) % C;
  const int jo = (threadIdx.x * G::OPT) / TB, co = (threadIdx.x * G::OPT) % TB;
  float accA[G::EPT], acc[G::OPT];
#pragma unroll
  for (int u = 0; u < G::EPT; ++u) accA[u] = 0.f;
#pragma unroll
  for (int u = 0; u < G::OPT; ++u) acc[u] = 0.f;
  const float* Gi = dstates + ((size_t)bh * NC + i) * DK * DV;
  for (int d0 = 0; d0 < DK; d0 += TB) {
    load_tile<C>(qs, q, bh, i * C, T, DK, d0);
    load_tile<C>(ks, k, bh, i * C, T, DK, d0);
    load_tile<C>(Bs, g, bh, i * C, T, DK, d0);
    load_state_block(Gs, Gi, DK, DV, d0, c0);
    __syncthreads();
    cumsum_cols<C>(Bs);
    __syncthreads();
    subchunk_factors<C>(qs, ks, Bs, qf, kf, rho);
    __syncthreads();
    accumulate_A<C>(accA, ja, ra, qs, ks, Bs, qf, kf);
    for (int d = 0; d < TB; ++d) {
      const float kh = ks[jo * LD + d] * expf(Bs[(C - 1) * LD + d] - Bs[jo * LD + d]);
#pragma unroll
      for (int u = 0; u < G::OPT; ++u) acc[u] += kh * Gs[d * LD + co + u];
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < G::EPT; ++u) As[ja * (C + 1) + ra + u] = accA[u];
  load_tile<C>(ds, dO, bh, i * C, T, DV, c0);
  __syncthreads();
  for (int j = jo; j < C; ++j) {
    const float a = As[j * (C + 1) + jo];
#pragma unroll
    for (int u = 0; u < G::OPT; ++u) acc[u] += a * ds[j * LD + co + u];
  }
  const int t = i * C + jo;
  if (t < T) {
#pragma unroll
    for (int u = 0; u < G::OPT; ++u)
      if (c0 + co + u < DV) stf(dv + ((size_t)bh * T + t) * DV + c0 + co + u, acc[u]);
  }
}

// ---------------------------------------------------------------------------------------------
// dg: one thread per (bh, d).  dg_t = sum_{s>=t} db_s + sum_c dhT[d][c] hT[d][c] (+ addend_t).
// ---------------------------------------------------------------------------------------------
template <typename TO>
__global__ void dg_kernel(const float* __restrict__ db, const float* __restrict__ hT,
                          const float* __restrict__ dhT, int dhT_trans, const float* __restrict__ addend,
                          TO* __restrict__ dg, int BH, int T, int DK, int DV) {
  const int bh = blockIdx.y, d = blockIdx.x * blockDim.x + threadIdx.x;
  if (d >= DK || bh >= BH) return;
  float acc = 0.f;
  if (dhT && hT) {
    const size_t base = (size_t)bh * DK * DV;
    for (int c = 0; c < DV; ++c) {
      const float a = dhT_trans ? dhT[base + (size_t)c * DK + d] : dhT[base + (size_t)d * DV + c];
      acc += a * hT[base + (size_t)d * DV + c];
    }
  }
  for (int t = T - 1; t >= 0; --t) {
    const size_t idx = ((size_t)bh * T + t) * DK + d;
    acc += db[idx];
    float out = acc;
    if (addend) out += addend[idx];
    stf(dg + idx, out);
  }
}

// ---------------------------------------------------------------------------------------------
// Slot softmax over the last dimension (one warp per row), forward and backward.
// ---------------------------------------------------------------------------------------------
template <typename TP>
__global__ void softmax_fwd_kernel(const float* __restrict__ x, TP* __restrict__ p, TP* __restrict__ p2,
                                   long rows, int m) {
  const long row = (long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  const float* xr = x + row * m;
  float mx = -INFINITY;
  for (int s = lane; s < m; s += 32) mx = fmaxf(mx, xr[s]);
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float sum = 0.f;
  for (int s = lane; s < m; s += 32) sum += expf(xr[s] - mx);
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float inv = 1.f / sum;
  for (int s = lane; s < m; s += 32) {
    const float e = expf(xr[s] - mx) * inv;
    stf(p + row * m + s, e);
    if (p2) stf(p2 + row * m + s, e);
  }
}

// do1 = p * (dp - <p, dp>) with p = softmax(o1) recomputed in fp32.
__global__ void softmax_bwd_kernel(const float* __restrict__ x, const float* __restrict__ dp,
                                   float* __restrict__ dx, long rows, int m) {
  const long row = (long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  const float* xr = x + row * m;
  const float* dr = dp + row * m;
  float mx = -INFINITY;
  for (int s = lane; s < m; s += 32) mx = fmaxf(mx, xr[s]);
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float sum = 0.f, dot = 0.f;
  for (int s = lane; s < m; s += 32) {
    const float e = expf(xr[s] - mx);
    sum += e;
    dot += e * dr[s];
  }
  for (int o = 16; o > 0; o >>= 1) {
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
    dot += __shfl_xor_sync(0xffffffffu, dot, o);
  }
  const float inv = 1.f / sum;
  dot *= inv;
  for (int s = lane; s < m; s += 32) dx[row * m + s] = expf(xr[s] - mx) * inv * (dr[s] - dot);
}

// ---------------------------------------------------------------------------------------------
// Recurrent decode step: grid (ceil(DV/32), BH), block (32, 8).  Columns across lanes (coalesced
// state rows), key rows split over the 8 warps and reduced through shared memory.
// ---------------------------------------------------------------------------------------------
template <typename TI>
__global__ void decode_kernel(const TI* __restrict__ q, const TI* __restrict__ k, const TI* __restrict__ v,
                              const TI* __restrict__ g, float* __restrict__ S, TI* __restrict__ o, int DK,
                              int DV) {
  __shared__ float part[8][32];
  const int bh = blockIdx.y, c = blockIdx.x * 32 + threadIdx.x;
  float acc = 0.f;
  if (c < DV) {
    const float vc = ldf(v + (size_t)bh * DV + c);
    float* Sb = S + (size_t)bh * DK * DV;
    constexpr int R = 16;  // rows per thread held in registers (d_k <= 128): all loads in flight at once
    if (DK <= 8 * R) {
      float sv[R];
#pragma unroll
      for (int j = 0; j < R; ++j) {
        const int d = threadIdx.y + 8 * j;
        sv[j] = d < DK ? Sb[(size_t)d * DV + c] : 0.f;
      }
#pragma unroll
      for (int j = 0; j < R; ++j) {
        const int d = threadIdx.y + 8 * j;
        if (d < DK) {
          const size_t qi = (size_t)bh * DK + d;
          const float s = expf(ldf(g + qi)) * sv[j] + ldf(k + qi) * vc;
          Sb[(size_t)d * DV + c] = s;
          acc += ldf(q + qi) * s;
        }
      }
    } else {
      for (int d = threadIdx.y; d < DK; d += 8) {
        const size_t qi = (size_t)bh * DK + d;
        const float s = expf(ldf(g + qi)) * Sb[(size_t)d * DV + c] + ldf(k + qi) * vc;
        Sb[(size_t)d * DV + c] = s;
        acc += ldf(q + qi) * s;
      }
    }
  }
  part[threadIdx.y][threadIdx.x] = acc;
  __syncthreads();
  if (threadIdx.y == 0 && c < DV) {
    float s = 0.f;
#pragma unroll
    for (int y = 0; y < 8; ++y) s += part[y][threadIdx.x];
    stf(o + (size_t)bh * DV + c, s);
  }
}

// GSA decode: one CTA per (b,h); m <= 512, dk, dv <= 512.  Shared: p[m].
template <typename TI>
__global__ void gsa_decode_kernel(const TI* __restrict__ q, const TI* __restrict__ k, const TI* __restrict__ v,
                                  const TI* __restrict__ phi, const TI* __restrict__ g, float* __restrict__ S1,
                                  float* __restrict__ S2, TI* __restrict__ o, int DK, int DV, int M) {
  extern __shared__ float sm[];
  float* o1 = sm;        // [M]
  float* red = sm + M;   // [2]
  const int bh = blockIdx.x;
  float* S1b = S1 + (size_t)bh * DK * M;
  float* S2b = S2 + (size_t)bh * M * DV;
  // pass 1: S1 <- S1 diag(e^g) + k^T phi ; o1 = q S1   (threads over slots s)
  for (int s = threadIdx.x; s < M; s += blockDim.x) {
    const float a = expf(ldf(g + (size_t)bh * M + s)), ph = ldf(phi + (size_t)bh * M + s);
    float acc = 0.f;
    for (int i = 0; i < DK; ++i) {
      const float x = S1b[(size_t)i * M + s] * a + ldf(k + (size_t)bh * DK + i) * ph;
      S1b[(size_t)i * M + s] = x;
      acc += ldf(q + (size_t)bh * DK + i) * x;
    }
    o1[s] = acc;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float mx = -INFINITY;
    for (int s = 0; s < M; ++s) mx = fmaxf(mx, o1[s]);
    float sum = 0.f;
    for (int s = 0; s < M; ++s) sum += expf(o1[s] - mx);
    red[0] = mx;
    red[1] = 1.f / sum;
  }
  __syncthreads();
  for (int s = threadIdx.x; s < M; s += blockDim.x) o1[s] = expf(o1[s] - red[0]) * red[1];
  __syncthreads();
  // pass 2: S2 <- diag(e^g) S2 + phi^T v ; o = p S2   (threads over value columns)
  for (int c = threadIdx.x; c < DV; c += blockDim.x) {
    const float vc = ldf(v + (size_t)bh * DV + c);
    float acc = 0.f;
    for (int s = 0; s < M; ++s) {
      const float a = expf(ldf(g + (size_t)bh * M + s));
      const float x = a * S2b[(size_t)s * DV + c] + ldf(phi + (size_t)bh * M + s) * vc;
      S2b[(size_t)s * DV + c] = x;
      acc += o1[s] * x;
    }
    stf(o + (size_t)bh * DV + c, acc);
  }
}

// ---------------------------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------------------------
static inline int cdiv(int a, int b) { return (a + b - 1) / b; }

template <typename F>
static cudaError_t set_smem(F* f, size_t bytes) {
  return cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int C, typename TI>
static cudaError_t state_fwd_c(const Shape& s, const TI* k, const TI* v, const TI* g, const float* h0, int h0t,
                               float* states, float* hT, int hTt, cudaStream_t st) {
  const size_t smem = (3 * C * LD + TB) * sizeof(float);
  auto f = state_fwd_kernel<C, TI>;
  cudaError_t e = set_smem(f, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(cdiv(s.DV, TB), cdiv(s.DK, TB), s.BH);
  f<<<grid, NT, smem, st>>>(k, v, g, h0, h0t, states, hT, hTt, s.T, s.DK, s.DV);
  return cudaGetLastError();
}

template <typename TI>
cudaError_t state_fwd(const Shape& s, const TI* k, const TI* v, const TI* g, const float* h0, int h0_trans,
                      float* states, float* hT, int hT_trans, cudaStream_t st) {
  switch (s.C) {
    case 16: return state_fwd_c<16>(s, k, v, g, h0, h0_trans, states, hT, hT_trans, st);
    case 32: return state_fwd_c<32>(s, k, v, g, h0, h0_trans, states, hT, hT_trans, st);
    case 64: return state_fwd_c<64>(s, k, v, g, h0, h0_trans, states, hT, hT_trans, st);
  }
  return cudaErrorInvalidValue;
}

template <int C, typename TQ, typename TI>
static cudaError_t dstate_bwd_c(const Shape& s, const TQ* q, const TI* g, const TI* dO, const float* dhT, int dhTt,
                                float* dstates, float* dh0, int dh0t, cudaStream_t st) {
  const size_t smem = (3 * C * LD + TB) * sizeof(float);
  auto f = dstate_bwd_kernel<C, TQ, TI>;
  cudaError_t e = set_smem(f, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(cdiv(s.DV, TB), cdiv(s.DK, TB), s.BH);
  f<<<grid, NT, smem, st>>>(q, g, dO, dhT, dhTt, dstates, dh0, dh0t, s.T, s.DK, s.DV);
  return cudaGetLastError();
}

template <typename TQ, typename TI>
cudaError_t dstate_bwd(const Shape& s, const TQ* q, const TI* g, const TI* dO, const float* dhT, int dhT_trans,
                       float* dstates, float* dh0, int dh0_trans, cudaStream_t st) {
  switch (s.C) {
    case 16: return dstate_bwd_c<16>(s, q, g, dO, dhT, dhT_trans, dstates, dh0, dh0_trans, st);
    case 32: return dstate_bwd_c<32>(s, q, g, dO, dhT, dhT_trans, dstates, dh0, dh0_trans, st);
    case 64: return dstate_bwd_c<64>(s, q, g, dO, dhT, dhT_trans, dstates, dh0, dh0_trans, st);
  }
  return cudaErrorInvalidValue;
}

template <int C, typename TQ, typename TI, typename TO>
static cudaError_t out_c(const Shape& s, const TQ* q, const TI* k, const TI* v, const TI* g, const float* states,
                         TO* o, cudaStream_t st) {
  const size_t smem = OutSmem<C>::floats * sizeof(float);
  auto f = out_kernel<C, TQ, TI, TO>;
  cudaError_t e = set_smem(f, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(cdiv(s.DV, TB), num_chunks(s.T, C), s.BH);
  f<<<grid, NT, smem, st>>>(q, k, v, g, states, o, s.T, s.DK, s.DV);
  return cudaGetLastError();
}

template <typename TQ, typename TI, typename TO>
cudaError_t out(const Shape& s, const TQ* q, const TI* k, const TI* v, const TI* g, const float* states, TO* o,
                cudaStream_t st) {
  switch (s.C) {
    case 16: return out_c<16>(s, q, k, v, g, states, o, st);
    case 32: return out_c<32>(s, q, k, v, g, states, o, st);
    case 64: return out_c<64>(s, q, k, v, g, states, o, st);
  }
  return cudaErrorInvalidValue;
}

template <int C, typename TQ, typename TI, typename TO>
static cudaError_t dqdk_c(const Shape& s, const TQ* q, const TI* k, const TI* v, const TI* g, const TI* dO,
                          const float* states, const float* dstates, TO* dq, TO* dk, const float* dk_addend,
                          float* db, cudaStream_t st) {
  const size_t smem = DqdkSmem<C>::floats * sizeof(float);
  auto f = bwd_dqdk_kernel<C, TQ, TI, TO>;
  cudaError_t e = set_smem(f, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(cdiv(s.DK, TB), num_chunks(s.T, C), s.BH);
  f<<<grid, NT, smem, st>>>(q, k, v, g, dO, states, dstates, dq, dk, dk_addend, db, s.T, s.DK, s.DV);
  return cudaGetLastError();
}

template <typename TQ, typename TI, typename TO>
cudaError_t bwd_dqdk(const Shape& s, const TQ* q, const TI* k, const TI* v, const TI* g, const TI* dO,
                     const float* states, const float* dstates, TO* dq, TO* dk, const float* dk_addend, float* db,
                     cudaStream_t st) {
  switch (s.C) {
    case 16: return dqdk_c<16>(s, q, k, v, g, dO, states, dstates, dq, dk, dk_addend, db, st);
    case 32: return dqdk_c<32>(s, q, k, v, g, dO, states, dstates, dq, dk, dk_addend, db, st);
    case 64: return dqdk_c<64>(s, q, k, v, g, dO, states, dstates, dq, dk, dk_addend, db, st);
  }
  return cudaErrorInvalidValue;
}

template <int C, typename TQ, typename TI, typename TO>
static cudaError_t dv_c(const Shape& s, const TQ* q, const TI* k, const TI* g, const TI* dO, const float* dstates,
                        TO* dv, cudaStream_t st) {
  const size_t smem = OutSmem<C>::floats * sizeof(float);
  auto f = bwd_dv_kernel<C, TQ, TI, TO>;
  cudaError_t e = set_smem(f, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(cdiv(s.DV, TB), num_chunks(s.T, C), s.BH);
  f<<<grid, NT, smem, st>>>(q, k, g, dO, dstates, dv, s.T, s.DK, s.DV);
  return cudaGetLastError();
}

template <typename TQ, typename TI, typename TO>
cudaError_t bwd_dv(const Shape& s, const TQ* q, const TI* k, const TI* g, const TI* dO, const float* dstates, TO* dv,
                   cudaStream_t st) {
  switch (s.C) {
    case 16: return dv_c<16>(s, q, k, g, dO, dstates, dv, st);
    case 32: return dv_c<32>(s, q, k, g, dO, dstates, dv, st);
    case 64: return dv_c<64>(s, q, k, g, dO, dstates, dv, st);
  }
  return cudaErrorInvalidValue;
}

template <typename TO>
cudaError_t dg(const Shape& s, const float* db, const float* hT, const float* dhT, int dhT_trans,
               const float* addend, TO* dgo, cudaStream_t st) {
  dim3 grid(cdiv(s.DK, 128), s.BH);
  dg_kernel<TO><<<grid, 128, 0, st>>>(db, hT, dhT, dhT_trans, addend, dgo, s.BH, s.T, s.DK, s.DV);
  return cudaGetLastError();
}

template <typename TP>
cudaError_t softmax_fwd(const float* x, TP* p, TP* p2, long rows, int m, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  softmax_fwd_kernel<TP><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(x, p, p2, rows, m);
  return cudaGetLastError();
}

cudaError_t softmax_bwd(const float* x, const float* dp, float* dx, long rows, int m, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  softmax_bwd_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(x, dp, dx, rows, m);
  return cudaGetLastError();
}

template <typename TI>
cudaError_t decode(int BH, int DK, int DV, const TI* q, const TI* k, const TI* v, const TI* g, float* S, TI* o,
                   cudaStream_t st) {
  dim3 grid(cdiv(DV, 32), BH);
  decode_kernel<TI><<<grid, dim3(32, 8), 0, st>>>(q, k, v, g, S, o, DK, DV);
  return cudaGetLastError();
}

template <typename TI>
cudaError_t gsa_decode(int BH, int DK, int DV, int M, const TI* q, const TI* k, const TI* v, const TI* phi,
                       const TI* g, float* S1, float* S2, TI* o, cudaStream_t st) {
  gsa_decode_kernel<TI><<<BH, 256, (M + 2) * sizeof(float), st>>>(q, k, v, phi, g, S1, S2, o, DK, DV, M);
  return cudaGetLastError();
}

// Explicit instantiations used by the API layer.
#define GLA_INST_TI(TI)                                                                                         \
  template cudaError_t state_fwd<TI>(const Shape&, const TI*, const TI*, const TI*, const float*, int, float*, \
                                     float*, int, cudaStream_t);                                               \
  template cudaError_t decode<TI>(int, int, int, const TI*, const TI*, const TI*, const TI*, float*, TI*,       \
                                  cudaStream_t);                                                               \
  template cudaError_t gsa_decode<TI>(int, int, int, int, const TI*, const TI*, const TI*, const TI*,           \
                                      const TI*, float*, float*, TI*, cudaStream_t);

#define GLA_INST_D(TQ, TI)                                                                                     \
  template cudaError_t dstate_bwd<TQ, TI>(const Shape&, const TQ*, const TI*, const TI*, const float*, int,    \
                                          float*, float*, int, cudaStream_t);

#define GLA_INST_Q(TQ, TI, TO)                                                                                 \
  template cudaError_t out<TQ, TI, TO>(const Shape&, const TQ*, const TI*, const TI*, const TI*, const float*, \
                                       TO*, cudaStream_t);                                                     \
  template cudaError_t bwd_dqdk<TQ, TI, TO>(const Shape&, const TQ*, const TI*, const TI*, const TI*,          \
                                            const TI*, const float*, const float*, TO*, TO*, const float*,     \
                                            float*, cudaStream_t);                                             \
  template cudaError_t bwd_dv<TQ, TI, TO>(const Shape&, const TQ*, const TI*, const TI*, const TI*,            \
                                          const float*, TO*, cudaStream_t);

GLA_INST_TI(float)
GLA_INST_TI(bf16)
GLA_INST_D(float, float)
GLA_INST_D(bf16, bf16)
GLA_INST_D(float, bf16)
GLA_INST_Q(float, float, float)
GLA_INST_Q(bf16, bf16, bf16)
GLA_INST_Q(bf16, bf16, float)
GLA_INST_Q(float, bf16, bf16)
GLA_INST_Q(float, bf16, float)

template cudaError_t dg<float>(const Shape&, const float*, const float*, const float*, int, const float*, float*,
                               cudaStream_t);
template cudaError_t dg<bf16>(const Shape&, const float*, const float*, const float*, int, const float*, bf16*,
                              cudaStream_t);
template cudaError_t softmax_fwd<float>(const float*, float*, float*, long, int, cudaStream_t);
template cudaError_t softmax_fwd<bf16>(const float*, bf16*, bf16*, long, int, cudaStream_t);

}  // namespace generic
}  // namespace gla
