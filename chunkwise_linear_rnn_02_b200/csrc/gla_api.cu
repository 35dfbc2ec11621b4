// C ABI of the library (declared in include/gla.h): argument checks, workspace layout and the
// sequence of kernel launches for each operator.  Every check runs on the host before anything
// is enqueued; nothing here allocates, frees or synchronises (except gla_device_error).
#include <limits.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "../../include/gla.h"
#include "common.cuh"
#include "fast_path.cuh"
#include "split.cuh"
#include "generic_kernels.cuh"
#include "gsa_fused.cuh"

using gla::bf16;
namespace gk = gla::generic;

// Device-side error latch written by bounded waits that run out (see gla_device_error).
__device__ unsigned int g_gla_device_error = 0;

namespace {

constexpr int kVersion = 10000;  // 1.0.0

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Pointer rule: required pointers must be non-NULL; every non-NULL pointer 16-byte aligned.
int check_ptr(const void* p, bool required) {
  if (!p) return required ? GLA_ERR_INVALID_ARG : GLA_OK;
  return aligned16(p) ? GLA_OK : GLA_ERR_INVALID_ARG;
}

int check_dim(int d) {
  if (d <= 0) return GLA_ERR_INVALID_ARG;
  if (d > 512 || d % 8 != 0) return GLA_ERR_UNSUPPORTED;
  return GLA_OK;
}

int check_common(int B, int H, int T, int chunk, int dtype) {
  if (B <= 0 || H <= 0 || T < 0) return GLA_ERR_INVALID_ARG;
  if ((long long)B * H > INT_MAX) return GLA_ERR_INVALID_ARG;
  if ((long long)B * H * (long long)(T > 0 ? T : 1) > (1LL << 40)) return GLA_ERR_INVALID_ARG;
  if (dtype != GLA_DTYPE_F32 && dtype != GLA_DTYPE_BF16) return GLA_ERR_UNSUPPORTED;
  if (chunk != 16 && chunk != 32 && chunk != 64) return GLA_ERR_UNSUPPORTED;
  return GLA_OK;
}

#define GLA_TRY(expr)              \
  do {                             \
    int _s = (expr);               \
    if (_s != GLA_OK) return _s;   \
  } while (0)

#define GLA_CUDA(expr)                          \
  do {                                          \
    if ((expr) != cudaSuccess) return GLA_ERR_CUDA; \
  } while (0)

size_t esize(int dtype) { return dtype == GLA_DTYPE_BF16 ? 2 : 4; }

// Bump allocator over the caller's workspace (or a dry run that only counts bytes).
struct Carve {
  char* base;
  size_t used = 0;
  explicit Carve(void* b) : base(static_cast<char*>(b)) {}
  template <typename T>
  T* take(size_t count) {
    T* p = base ? reinterpret_cast<T*>(base + used) : nullptr;
    used += gla::align256(count * sizeof(T));
    return p;
  }
};

// ----------------------------------------------------------------------------------------
// Wide bf16 shapes as sub-problems of the fused kernels
//
// The recurrence decays every row of S on its own, so the forward is linear in a split of the key
// dimension: o = sum over key blocks of the output of the key block alone, and each block's hT is
// its rows of hT.  The loss <dO, o> is a sum over value columns, so the backward is also a sum of
// sub-problems over value blocks: dq, dk, dg of a key block sum over the value blocks, dv of a
// value block sums over the key blocks, and dh0 / dhT are the (key, value) blocks of the state.
// Key blocks are 128 wide; value blocks 256 (or 128) wide for the backward.  The kernels read
// their blocks of q, k, g, v, dO in place (the tile loads take the block's first column); every
// sub-problem but the last of an output block leaves an fp32 partial sum, which the next one adds
// in its epilogue; the last writes the bf16 result.
// ----------------------------------------------------------------------------------------
constexpr int kSplitK = 128;
int split_vblock(int dv) { return dv % 256 == 0 ? 256 : 128; }

bool split_fwd_ok(int BH, int T, int dk, int dv, int chunk, int dtype) {
  if (gla::fast::fwd_supported(BH, T, dk, dv, chunk, dtype)) return false;  // served directly
  return dk > kSplitK && dk % kSplitK == 0 && gla::fast::fwd_supported(BH, T, kSplitK, dv, chunk, dtype);
}
bool split_bwd_ok(int BH, int T, int dk, int dv, int chunk, int dtype) {
  if (gla::fast::bwd_supported(BH, T, dk, dv, chunk, dtype)) return false;
  if (dk % kSplitK != 0 || dv % 128 != 0) return false;
  return gla::fast::bwd_supported(BH, T, kSplitK, split_vblock(dv), chunk, dtype);
}

struct SplitFwdWs {
  float* acc;  // [BH*T][dv] partial output of the key blocks so far
  void* fws;
};
size_t carve_split_fwd(Carve& c, int BH, int T, int dk, int dv, SplitFwdWs* w) {
  (void)dk;
  SplitFwdWs x;
  x.acc = c.take<float>((size_t)BH * T * dv);
  x.fws = c.take<char>(gla::fast::fwd_workspace(BH, T, kSplitK, dv));
  if (w) *w = x;
  return c.used;
}

int split_fwd(const bf16* q, const bf16* k, const bf16* v, const bf16* g, const float* h0, bf16* o, float* hT,
              int BH, int T, int dk, int dv, void* ws, cudaStream_t st, float inv_tau = 0.f) {
  Carve c(ws);
  SplitFwdWs w;
  carve_split_fwd(c, BH, T, dk, dv, &w);
  const int nk = dk / kSplitK;
  for (int kb = 0; kb < nk; ++kb) {
    const int c0 = kb * kSplitK;
    GLA_CUDA(gla::fast::fwd(q, k, v, g, h0 ? h0 + (size_t)c0 * dv : nullptr, o, hT ? hT + (size_t)c0 * dv : nullptr, BH,
                            T, kSplitK, dv, w.fws, st, (long long)dk * dv, dv, kb < nk - 1 ? w.acc : nullptr, inv_tau,
                            dk, c0, kb > 0 ? w.acc : nullptr));
  }
  return GLA_OK;
}

struct SplitBwdWs {
  float *aq, *ak, *ag;  // [nk][nv] slices [BH*T][128]: each sub-problem's key-side gradients
  float* av;            // [nk][nv] slices [BH*T][vb]: each sub-problem's dv (none with one key block)
  void* bws[2];         // the fused kernels' workspace, one per stream
};
size_t carve_split_bwd(Carve& c, int BH, int T, int dk, int dv, SplitBwdWs* w) {
  const size_t rows = (size_t)BH * T;
  const int vb = split_vblock(dv), nv = dv / vb, nk = dk / kSplitK;
  SplitBwdWs x;
  x.aq = c.take<float>(nv * rows * dk);
  x.ak = c.take<float>(nv * rows * dk);
  x.ag = c.take<float>(nv * rows * dk);
  x.av = nk > 1 ? c.take<float>(nk * rows * dv) : nullptr;
  for (int j = 0; j < 2; ++j) x.bws[j] = c.take<char>(gla::fast::bwd_workspace(BH, T, kSplitK, vb));
  if (w) *w = x;
  return c.used;
}

int split_bwd(const bf16* q, const bf16* k, const bf16* v, const bf16* g, const float* h0, const bf16* dO,
              const float* dhT, bf16* dq, bf16* dk, bf16* dv, bf16* dg, float* dh0, int BH, int T, int dkd, int dvd,
              void* ws, cudaStream_t st, float inv_tau = 0.f) {
  Carve c(ws);
  SplitBwdWs w;
  carve_split_bwd(c, BH, T, dkd, dvd, &w);
  const int vb = split_vblock(dvd), nv = dvd / vb, nk = dkd / kSplitK;
  const long long rows = (long long)BH * T, ks = rows * kSplitK, vs = rows * vb;
  // The sub-problems write disjoint slices, so they run on two streams (the caller's and a side
  // stream, sub-problem s on stream s & 1): the CTAs of one sub-problem's chunk-parallel launch fill
  // the SMs that the other's walks leave idle.  Each summing pass is enqueued as soon as its slices
  // are: a key block's after its last sub-problem (waiting for the other stream's part of the block),
  // a value block's at the end of the stream that ran all its sub-problems (nv even) or after the
  // join.
  gla::fast::SideStream* side = nullptr;
  GLA_CUDA(gla::fast::side_stream(0, &side));
  std::lock_guard<std::mutex> lock(side->mu);
  cudaStream_t sts[2] = {st, side->s};
  GLA_CUDA(cudaEventRecord(side->fork, st));
  GLA_CUDA(cudaStreamWaitEvent(side->s, side->fork, 0));
  for (int kb = 0; kb < nk; ++kb) {
    const int k0 = kb * kSplitK;
    for (int vi = 0; vi < nv; ++vi) {
      const int v0 = vi * vb, s = kb * nv + vi;
      const size_t so = (size_t)k0 * dvd + v0;  // state block (k0.., v0..) of every head
      // key-side gradients sum over the value blocks, dv over the key blocks: each sub-problem writes
      // its fp32 part into compact slices of its own (with one key block dv goes straight to bf16),
      // and the summing passes add the slices into the bf16 columns
      const gla::fast::BwdAccum out{w.aq + s * ks, w.ak + s * ks, w.ag + s * ks, w.av ? w.av + s * vs : nullptr,
                                    dkd, k0, dvd, v0};
      GLA_CUDA(gla::fast::bwd(q, k, v, g, h0 ? h0 + so : nullptr, dO, dhT ? dhT + so : nullptr, dq, dk, dv, dg,
                              dh0 ? dh0 + so : nullptr, BH, T, kSplitK, vb, w.bws[s & 1], sts[s & 1],
                              (long long)dkd * dvd, dvd, &out, inv_tau));
    }
    // key block kb is complete once both streams are past its sub-problems
    const int last = (kb * nv + nv - 1) & 1;
    cudaStream_t ks_st = sts[last];
    if (nv > 1) {
      GLA_CUDA(cudaEventRecord(side->join, sts[last ^ 1]));
      GLA_CUDA(cudaStreamWaitEvent(ks_st, side->join, 0));
    }
    const float* base[3] = {w.aq, w.ak, w.ag};
    bf16* outs[3] = {dq, dk, dg};
    for (int j = 0; j < 3; ++j)
      GLA_CUDA(gla::split::sum_blocks_to_bf16(base[j] + (size_t)kb * nv * ks, rows, kSplitK, 1, nv, 0, 1,
                                              outs[j] + k0, dkd, ks_st));
  }
  if (w.av && nv % 2 == 0) {  // value block vi ran on stream vi & 1 for every key block
    for (int vi = 0; vi < nv; ++vi)
      GLA_CUDA(gla::split::sum_blocks_to_bf16(w.av + (size_t)vi * vs, rows, vb, 1, nk, 0, nv, dv + vi * vb, dvd,
                                              sts[vi & 1]));
  }
  GLA_CUDA(cudaEventRecord(side->join, side->s));
  GLA_CUDA(cudaStreamWaitEvent(st, side->join, 0));
  if (w.av && nv % 2 != 0) GLA_CUDA(gla::split::sum_blocks_to_bf16(w.av, rows, vb, nv, nk, 1, nv, dv, dvd, st));
  return GLA_OK;
}

// ----------------------------------------------------------------------------------------
// GLA forward / backward (generic chunk-parallel passes)
// ----------------------------------------------------------------------------------------
struct GlaFwdWs {
  float* states;
};
size_t carve_gla_fwd(Carve& c, int BH, int T, int dk, int dv, int chunk, GlaFwdWs* w) {
  const size_t NC = gla::num_chunks(T, chunk);
  float* s = c.take<float>((size_t)BH * NC * dk * dv);
  if (w) w->states = s;
  return c.used;
}

struct GlaBwdWs {
  float *states, *dstates, *db, *hT;
};
size_t carve_gla_bwd(Carve& c, int BH, int T, int dk, int dv, int chunk, GlaBwdWs* w) {
  const size_t NC = gla::num_chunks(T, chunk);
  GlaBwdWs x;
  x.states = c.take<float>((size_t)BH * NC * dk * dv);
  x.dstates = c.take<float>((size_t)BH * NC * dk * dv);
  x.db = c.take<float>((size_t)BH * T * dk);
  x.hT = c.take<float>((size_t)BH * dk * dv);
  if (w) *w = x;
  return c.used;
}

template <typename TI>
int gla_fwd_generic(const TI* q, const TI* k, const TI* v, const TI* g, const float* h0, TI* o, float* hT,
                    gk::Shape s, void* ws, cudaStream_t st) {
  Carve c(ws);
  GlaFwdWs w;
  carve_gla_fwd(c, s.BH, s.T, s.DK, s.DV, s.C, &w);
  GLA_CUDA(gk::state_fwd<TI>(s, k, v, g, h0, 0, w.states, hT, 0, st));
  GLA_CUDA((gk::out<TI, TI, TI>(s, q, k, v, g, w.states, o, st)));
  return GLA_OK;
}

template <typename TI>
int gla_bwd_generic(const TI* q, const TI* k, const TI* v, const TI* g, const float* h0, const TI* dO,
                    const float* dhT, TI* dq, TI* dk, TI* dv, TI* dg, float* dh0, gk::Shape s, void* ws,
                    cudaStream_t st) {
  Carve c(ws);
  GlaBwdWs w;
  carve_gla_bwd(c, s.BH, s.T, s.DK, s.DV, s.C, &w);
  GLA_CUDA(gk::state_fwd<TI>(s, k, v, g, h0, 0, w.states, w.hT, 0, st));
  GLA_CUDA((gk::dstate_bwd<TI, TI>(s, q, g, dO, dhT, 0, w.dstates, dh0, 0, st)));
  GLA_CUDA((gk::bwd_dqdk<TI, TI, TI>(s, q, k, v, g, dO, w.states, w.dstates, dq, dk, nullptr, w.db, st)));
  GLA_CUDA((gk::bwd_dv<TI, TI, TI>(s, q, k, g, dO, w.dstates, dv, st)));
  GLA_CUDA(gk::dg<TI>(s, w.db, w.hT, dhT, 0, nullptr, dg, st));
  return GLA_OK;
}

// Copy src (or zeros when NULL) into dst, n floats; used for T == 0.
int copy_or_zero(float* dst, const float* src, size_t n, cudaStream_t st) {
  if (!dst) return GLA_OK;
  if (src)
    GLA_CUDA(cudaMemcpyAsync(dst, src, n * sizeof(float), cudaMemcpyDeviceToDevice, st));
  else
    GLA_CUDA(cudaMemsetAsync(dst, 0, n * sizeof(float), st));
  return GLA_OK;
}

// ----------------------------------------------------------------------------------------
// GSA.  Pass 1 runs on the generic kernels as the key-gated pass with roles exchanged (its state
// kept transposed, [m x dk], so that the slot axis is the gated row axis); pass 2, a plain
// key-gated GLA, runs on the fused kernels where they serve the shape, else on the generic ones.
// ----------------------------------------------------------------------------------------
struct GsaFwdWs {
  float *S1, *o1, *S2;
  void* p;
};
size_t carve_gsa_fwd(Carve& c, int BH, int T, int dk, int dv, int m, int chunk, int dtype, bool need_p,
                     GsaFwdWs* w) {
  const size_t NC = gla::num_chunks(T, chunk);
  GsaFwdWs x;
  x.S1 = c.take<float>((size_t)BH * NC * m * dk);
  x.o1 = c.take<float>((size_t)BH * T * m);
  // pass 2 is a plain key-gated GLA: per-chunk states for the generic kernels, or the fused
  // forward's workspace when it serves the shape
  size_t s2 = (size_t)BH * NC * m * dv;
  if (gla::fast::fwd_supported(BH, T, m, dv, chunk, dtype)) {
    const size_t fw = (gla::fast::fwd_workspace(BH, T, m, dv) + sizeof(float) - 1) / sizeof(float);
    if (fw > s2) s2 = fw;
  }
  x.S2 = c.take<float>(s2);
  x.p = need_p ? (void*)c.take<char>((size_t)BH * T * m * esize(dtype)) : nullptr;
  if (w) *w = x;
  return c.used;
}

// GSA's second pass (queries p, keys phi, values v, slot gates on its key axis) on the fused
// backward: the m slots zero-padded to one 128-wide key block.  Exact: padded dimensions have zero
// keys, queries, gates (decay 1) and states, so they add nothing to any output of the m real ones.
bool gsa_pass2_fused_ok(int BH, int T, int m, int dv, int chunk, int dtype) {
  return m <= 128 && m % 8 == 0 && gla::fast::bwd_supported(BH, T, 128, dv, chunk, dtype);
}
struct GsaFusedWs {
  bf16 *p, *phi, *g;                 // [BH*T][128] padded operands
  float *dq, *dk, *dg, *dv;          // fp32 outputs: [BH*T][128] (dp, dphi2, dg2) and [BH*T][dv]
  float *h0, *dhT, *dh0;             // [BH][128][dv] padded states
  void* ws;                          // the fused backward's workspace
};
void carve_gsa_fused(Carve& c, int BH, int T, int dv, GsaFusedWs* w, size_t bwd_ws = 0) {
  const size_t rows = (size_t)BH * T, st = (size_t)BH * 128 * dv;
  GsaFusedWs x;
  x.p = c.take<bf16>(rows * 128);
  x.phi = c.take<bf16>(rows * 128);
  x.g = c.take<bf16>(rows * 128);
  x.dq = c.take<float>(rows * 128);
  x.dk = c.take<float>(rows * 128);
  x.dg = c.take<float>(rows * 128);
  x.dv = c.take<float>(rows * dv);
  x.h0 = c.take<float>(st);
  x.dhT = c.take<float>(st);
  x.dh0 = c.take<float>(st);
  const size_t need = gla::fast::bwd_workspace(BH, T, 128, dv);
  x.ws = c.take<char>(need > bwd_ws ? need : bwd_ws);
  if (w) *w = x;
}

struct GsaBwdWs {
  float *S1, *o1, *S2, *dS2, *hT2, *db, *dp, *dphi2, *dg2, *do1, *dS1, *hT1;
  void* p;
  GsaFusedWs f;
};
size_t carve_gsa_bwd(Carve& c, int BH, int T, int dk, int dv, int m, int chunk, int dtype, GsaBwdWs* w) {
  const size_t NC = gla::num_chunks(T, chunk);
  const size_t tm = (size_t)BH * T * m;
  GsaBwdWs x;
  x.S1 = c.take<float>((size_t)BH * NC * m * dk);
  x.o1 = c.take<float>(tm);
  x.S2 = c.take<float>((size_t)BH * NC * m * dv);
  x.dS2 = c.take<float>((size_t)BH * NC * m * dv);
  x.hT2 = c.take<float>((size_t)BH * m * dv);
  x.db = c.take<float>(tm);
  x.dp = c.take<float>(tm);
  x.dphi2 = c.take<float>(tm);
  x.dg2 = c.take<float>(tm);
  x.do1 = c.take<float>(tm);
  x.dS1 = c.take<float>((size_t)BH * NC * m * dk);
  x.hT1 = c.take<float>((size_t)BH * m * dk);
  x.p = (void*)c.take<char>(tm * esize(dtype));
  if (gsa_pass2_fused_ok(BH, T, m, dv, chunk, dtype)) carve_gsa_fused(c, BH, T, dv, &x.f);
  if (w) *w = x;
  return c.used;
}

// ----------------------------------------------------------------------------------------
// GSA with both passes on the fused kernels (bf16, chunk 64, d_k = 128, m = 64): pass 1 and the
// slot softmax on the pass-1 kernel, pass 2 on the GLA forward.  The backward differentiates pass
// 2 on the GLA backward (slots zero-padded to a 128-wide key block), applies the softmax Jacobian,
// and differentiates pass 1 as a GLA with the roles exchanged: <do1, o1(q, k, phi, g)> equals
// <q, o'> for o' = GLA(queries do1, keys phi, values k, the slot gates on the key axis) with the
// initial state h0_1^T, so pass 1's gradients for phi, k, g and h0_1 are that GLA's gradients for
// its keys, values, gates and initial state with dO' = q, and dq = S1 do1 is that GLA's output.
// ----------------------------------------------------------------------------------------
bool gsa_fused_fwd_ok(int BH, int T, int dk, int dv, int m, int chunk, int dtype) {
  return gla::gsa::pass1_supported(BH, T, dk, m, chunk, dtype) && gla::fast::fwd_supported(BH, T, m, dv, chunk, dtype);
}
bool gsa_fused_bwd_ok(int BH, int T, int dk, int dv, int m, int chunk, int dtype) {
  return gsa_fused_fwd_ok(BH, T, dk, dv, m, chunk, dtype) && 2 * m == 128 &&
         gla::fast::bwd_supported(BH, T, 128, dv, chunk, dtype) && gla::fast::bwd_supported(BH, T, 128, dk, chunk, dtype) &&
         gla::fast::fwd_supported(BH, T, m, dk, chunk, dtype);
}

struct GsaFusedFwdWs {
  bf16* p;
  void *p1ws, *fws;
};
size_t carve_gsa_fused_fwd(Carve& c, int BH, int T, int dk, int dv, int m, bool need_p, GsaFusedFwdWs* w) {
  GsaFusedFwdWs x;
  x.p = need_p ? c.take<bf16>((size_t)BH * T * m) : nullptr;
  x.p1ws = c.take<char>(gla::gsa::pass1_workspace(BH, T, dk));
  x.fws = c.take<char>(gla::fast::fwd_workspace(BH, T, m, dv));
  if (w) *w = x;
  return c.used;
}

struct GsaFusedBwdWs {
  GsaFusedWs f;                    // pass 2: widened operands, fp32 gradients, widened states, bwd workspace
  float* p32;                      // [rows][m] the slot softmax in fp32
  bf16* do1;                       // [rows][128]: do1 [hi | lo]
  float *dq1, *dphi1, *dg1;        // pass-1 backward outputs: [rows][128] x 3
  float *h0p, *dhTp, *dh0p, *h0t;  // [BH][128][dk] x 3, [BH][m][dk]
  float* dqp;                      // [rows][dk] fp32: dq's partial from the queries' hi half
  void *p1ws, *fws;
};
size_t carve_gsa_fused_bwd(Carve& c, int BH, int T, int dk, int dv, int m, GsaFusedBwdWs* w) {
  const size_t rows = (size_t)BH * T, sp = (size_t)BH * 128 * dk;
  GsaFusedBwdWs x;
  carve_gsa_fused(c, BH, T, dv, &x.f, gla::fast::bwd_workspace(BH, T, 128, dk));
  x.p32 = c.take<float>(rows * m);
  x.do1 = c.take<bf16>(rows * 128);
  x.dq1 = c.take<float>(rows * 128);
  x.dphi1 = c.take<float>(rows * 128);
  x.dg1 = c.take<float>(rows * 128);
  x.h0p = c.take<float>(sp);
  x.dhTp = c.take<float>(sp);
  x.dh0p = c.take<float>(sp);
  x.h0t = c.take<float>((size_t)BH * m * dk);
  x.dqp = c.take<float>(rows * dk);
  x.p1ws = c.take<char>(gla::gsa::pass1_workspace(BH, T, dk));
  x.fws = c.take<char>(gla::fast::fwd_workspace(BH, T, m, dk));
  if (w) *w = x;
  return c.used;
}

int gsa_fwd_fused(const bf16* q, const bf16* k, const bf16* v, const bf16* phi, const bf16* g, const float* h01,
                  const float* h02, bf16* o, bf16* p_save, float* hT1, float* hT2, int BH, int T, int dk, int dv,
                  int m, void* ws, cudaStream_t st) {
  Carve c(ws);
  GsaFusedFwdWs w;
  carve_gsa_fused_fwd(c, BH, T, dk, dv, m, p_save == nullptr, &w);
  bf16* p = p_save ? p_save : w.p;
  // Pass 2's segment entry states need phi, g and v, not p: on the side stream, beside pass 1.
  gla::fast::SideStream* side = nullptr;
  GLA_CUDA(gla::fast::side_stream(0, &side));
  {
    std::lock_guard<std::mutex> lock(side->mu);
    GLA_CUDA(cudaEventRecord(side->fork, st));
    GLA_CUDA(cudaStreamWaitEvent(side->s, side->fork, 0));
    GLA_CUDA(gla::fast::fwd(p, phi, v, g, h02, o, hT2, BH, T, m, dv, w.fws, side->s, -1, -1, nullptr, 0.f, -1, 0,
                            nullptr, false, gla::fast::kFwdStates));
    GLA_CUDA(cudaEventRecord(side->join, side->s));
    GLA_CUDA(gla::gsa::pass1_fwd(q, k, phi, g, h01, p, hT1, BH, T, dk, w.p1ws, st));
    GLA_CUDA(cudaStreamWaitEvent(st, side->join, 0));
  }
  GLA_CUDA(gla::fast::fwd(p, phi, v, g, h02, o, hT2, BH, T, m, dv, w.fws, st, -1, -1, nullptr, 0.f, -1, 0, nullptr,
                          false, gla::fast::kFwdWalk));
  return GLA_OK;
}

// Both GLA passes of the backward run on 128-wide key blocks: the m = 64 slots, then a second copy of
// them (same keys and gates) whose queries are the low bf16 parts of the real queries, so that p and
// do1 enter at about 16 mantissa bits (the slot softmax and its Jacobian amplify a bf16 rounding of
// either several times over).  The two copies' gradients add up.
int gsa_bwd_fused(const bf16* q, const bf16* k, const bf16* v, const bf16* phi, const bf16* g, const float* h01,
                  const float* h02, const bf16* dO, const float* dhT1, const float* dhT2, bf16* dq, bf16* dk, bf16* dv,
                  bf16* dphi, bf16* dg, float* dh01, float* dh02, int BH, int T, int dkd, int dvd, int m, void* ws,
                  cudaStream_t st) {
  Carve c(ws);
  GsaFusedBwdWs w;
  carve_gsa_fused_bwd(c, BH, T, dkd, dvd, m, &w);
  const GsaFusedWs& f = w.f;
  const long long rows = (long long)BH * T, sz = (long long)m * dvd, sp = 128LL * dvd, s1 = (long long)dkd * m;
  const long long s1t = (long long)m * dkd, s1p = 128LL * dkd;
  // pass 1 forward again: the slot softmax p, in fp32
  GLA_CUDA(gla::gsa::pass1_fwd(q, k, phi, g, h01, nullptr, nullptr, BH, T, dkd, w.p1ws, st, w.p32));
  // key blocks of 128: queries [p hi | p lo], keys [phi | phi], gates [g | g]
  GLA_CUDA(gla::gsa::widen(w.p32, f.p, rows, m, true, st));
  GLA_CUDA(gla::gsa::widen(phi, f.phi, rows, m, false, st));
  GLA_CUDA(gla::gsa::widen(g, f.g, rows, m, false, st));
  // pass 2 backward (queries p, keys phi, values v): both copies start from h0_2, the first alone
  // carries dhT2
  if (h02) {
    GLA_CUDA(gla::split::copy_cols(h02, sz, f.h0, sp, BH, sz, sz, st));
    GLA_CUDA(gla::split::copy_cols(h02, sz, f.h0 + sz, sp, BH, sz, sz, st));
  }
  if (dhT2) GLA_CUDA(gla::split::copy_cols(dhT2, sz, f.dhT, sp, BH, sz, sp, st));
  const gla::fast::BwdAccum acc2{f.dq, f.dk, f.dg, nullptr, 128, 0, dvd, 0};  // dv straight to bf16
  GLA_CUDA(gla::fast::bwd(f.p, f.phi, v, f.g, h02 ? f.h0 : nullptr, dO, dhT2 ? f.dhT : nullptr, nullptr, nullptr, dv,
                          nullptr, dh02 ? f.dh0 : nullptr, BH, T, 128, dvd, f.ws, st, -1, -1, &acc2));
  if (dh02) GLA_CUDA(gla::gsa::fold_rows(f.dh0, dh02, BH, m, dvd, st));
  // slot softmax Jacobian: do1 = p (dp - <p, dp>), dp = the first copy's query gradient
  GLA_CUDA(gla::gsa::softmax_jacobian(w.p32, f.dq, 128, w.do1, rows, m, st));
  // pass 1 backward as a GLA backward: queries do1, keys phi, values k, dO' = q, states transposed
  if (h01) {
    GLA_CUDA(gla::gsa::transpose_states(h01, s1, w.h0t, BH, dkd, m, m, st));
    GLA_CUDA(gla::split::copy_cols(w.h0t, s1t, w.h0p, s1p, BH, s1t, s1t, st));
    GLA_CUDA(gla::split::copy_cols(w.h0t, s1t, w.h0p + s1t, s1p, BH, s1t, s1t, st));
  }
  if (dhT1) GLA_CUDA(gla::gsa::transpose_states(dhT1, s1, w.dhTp, BH, dkd, m, 128, st));
  // From here the pass-1 backward (caller's stream) and the dq forwards (side stream) read only do1
  // and the inputs, and write disjoint outputs, so they run side by side.
  gla::fast::SideStream* side = nullptr;
  GLA_CUDA(gla::fast::side_stream(0, &side));
  std::lock_guard<std::mutex> lock(side->mu);
  GLA_CUDA(cudaEventRecord(side->fork, st));
  GLA_CUDA(cudaStreamWaitEvent(side->s, side->fork, 0));
  // dq = S1 do1: the output of the GLA with queries do1, keys phi, values k from h0_1^T, as two
  // d_k = 64 forwards over the queries' hi and lo halves (the second adds the first's partial), with
  // the decayed keys as bf16 hi + lo pairs (a single bf16 put dq 2 % off in the emulation)
  GLA_CUDA(gla::fast::fwd(w.do1, f.phi, k, f.g, h01 ? w.h0t : nullptr, nullptr, nullptr, BH, T, m, dkd, w.fws, side->s,
                          -1, -1, w.dqp, 0.f, 128, 0, nullptr, true));
  GLA_CUDA(gla::fast::fwd(w.do1, f.phi, k, f.g, h01 ? w.h0t : nullptr, dq, nullptr, BH, T, m, dkd, w.fws, side->s, -1,
                          -1, nullptr, 0.f, 128, m, w.dqp, true));
  GLA_CUDA(cudaEventRecord(side->join, side->s));
  const gla::fast::BwdAccum acc1{w.dq1, w.dphi1, w.dg1, nullptr, 128, 0, dkd, 0};  // dk (its dv) straight to bf16
  GLA_CUDA(gla::fast::bwd(w.do1, f.phi, k, f.g, h01 ? w.h0p : nullptr, q, dhT1 ? w.dhTp : nullptr, nullptr, nullptr,
                          dk, nullptr, dh01 ? w.dh0p : nullptr, BH, T, 128, dkd, f.ws, st, -1, -1, &acc1));
  // both passes' and both copies' contributions to dphi and dg; dh0_1 back to [dk][m]
  GLA_CUDA(gla::gsa::fold_add_bf16(w.dphi1, f.dk, dphi, rows, m, st));
  GLA_CUDA(gla::gsa::fold_add_bf16(w.dg1, f.dg, dg, rows, m, st));
  if (dh01) GLA_CUDA(gla::gsa::transpose_states(w.dh0p, s1p, dh01, BH, m, dkd, dkd, st, true));
  GLA_CUDA(cudaStreamWaitEvent(st, side->join, 0));
  return GLA_OK;
}

template <typename TI>
int gsa_fwd_impl(const TI* q, const TI* k, const TI* v, const TI* phi, const TI* g, const float* h01,
                 const float* h02, TI* o, TI* p_save, float* hT1, float* hT2, int BH, int T, int dk, int dv, int m,
                 int C, void* ws, cudaStream_t st) {
  Carve c(ws);
  GsaFwdWs w;
  carve_gsa_fwd(c, BH, T, dk, dv, m, C, sizeof(TI) == 2 ? GLA_DTYPE_BF16 : GLA_DTYPE_F32, p_save == nullptr, &w);
  TI* p = p_save ? p_save : static_cast<TI*>(w.p);
  const gk::Shape s1{BH, T, m, dk, C}, s2{BH, T, m, dv, C};
  // pass 1 state (transposed), then o1 = e^B (q S1) + gated intra term, via the dq formula.
  GLA_CUDA(gk::state_fwd<TI>(s1, phi, k, g, h01, 1, w.S1, hT1, 1, st));
  GLA_CUDA((gk::bwd_dqdk<TI, TI, float>(s1, phi, phi, k, g, q, w.S1, nullptr, w.o1, nullptr, nullptr, nullptr,
                                        st)));
  GLA_CUDA(gk::softmax_fwd<TI>(w.o1, p, nullptr, (long)BH * T, m, st));
  // pass 2: GLA with queries p, keys phi, values v and the same slot gates (key axis)
  const int dtype = sizeof(TI) == 2 ? GLA_DTYPE_BF16 : GLA_DTYPE_F32;
  if (gla::fast::fwd_supported(BH, T, m, dv, C, dtype)) {
    GLA_CUDA(gla::fast::fwd(p, phi, v, g, h02, o, hT2, BH, T, m, dv, w.S2, st));
    return GLA_OK;
  }
  GLA_CUDA(gk::state_fwd<TI>(s2, phi, v, g, h02, 0, w.S2, hT2, 0, st));
  GLA_CUDA((gk::out<TI, TI, TI>(s2, p, phi, v, g, w.S2, o, st)));
  return GLA_OK;
}

template <typename TI>
int gsa_bwd_impl(const TI* q, const TI* k, const TI* v, const TI* phi, const TI* g, const float* h01,
                 const float* h02, const TI* dO, const float* dhT1, const float* dhT2, TI* dq, TI* dk, TI* dv,
                 TI* dphi, TI* dg, float* dh01, float* dh02, int BH, int T, int dkd, int dvd, int m, int C,
                 void* ws, cudaStream_t st) {
  Carve c(ws);
  GsaBwdWs w;
  carve_gsa_bwd(c, BH, T, dkd, dvd, m, C, sizeof(TI) == 2 ? GLA_DTYPE_BF16 : GLA_DTYPE_F32, &w);
  TI* p = static_cast<TI*>(w.p);
  const gk::Shape s1{BH, T, m, dkd, C}, s2{BH, T, m, dvd, C};
  // recompute pass 1 and the slot softmax
  GLA_CUDA(gk::state_fwd<TI>(s1, phi, k, g, h01, 1, w.S1, w.hT1, 0, st));
  GLA_CUDA((gk::bwd_dqdk<TI, TI, float>(s1, phi, phi, k, g, q, w.S1, nullptr, w.o1, nullptr, nullptr, nullptr,
                                        st)));
  GLA_CUDA(gk::softmax_fwd<TI>(w.o1, p, nullptr, (long)BH * T, m, st));
  // pass 2 backward (queries p, keys phi, values v)
  bool pass2_done = false;
  if constexpr (sizeof(TI) == 2) {
    if (gsa_pass2_fused_ok(BH, T, m, dvd, C, GLA_DTYPE_BF16)) {
      const GsaFusedWs& f = w.f;
      const long long rows = (long long)BH * T, sz = (long long)m * dvd, sp = 128LL * dvd;
      GLA_CUDA(gla::split::copy_cols(p, m, f.p, 128, rows, m, 128, st));
      GLA_CUDA(gla::split::copy_cols(phi, m, f.phi, 128, rows, m, 128, st));
      GLA_CUDA(gla::split::copy_cols(g, m, f.g, 128, rows, m, 128, st));
      if (h02) GLA_CUDA(gla::split::copy_cols(h02, sz, f.h0, sp, BH, sz, sp, st));
      if (dhT2) GLA_CUDA(gla::split::copy_cols(dhT2, sz, f.dhT, sp, BH, sz, sp, st));
      const gla::fast::BwdAccum acc{f.dq, f.dk, f.dg, f.dv, 128, 0, dvd, 0};
      GLA_CUDA(gla::fast::bwd(f.p, f.phi, v, f.g, h02 ? f.h0 : nullptr, dO, dhT2 ? f.dhT : nullptr, nullptr,
                              nullptr, nullptr, nullptr, dh02 ? f.dh0 : nullptr, BH, T, 128, dvd, f.ws, st, -1, -1,
                              &acc));
      GLA_CUDA(gla::split::copy_cols(f.dq, 128, w.dp, m, rows, m, m, st));
      GLA_CUDA(gla::split::copy_cols(f.dk, 128, w.dphi2, m, rows, m, m, st));
      GLA_CUDA(gla::split::copy_cols(f.dg, 128, w.dg2, m, rows, m, m, st));
      GLA_CUDA(gla::split::to_bf16(f.dv, dv, rows * dvd, st));
      if (dh02) GLA_CUDA(gla::split::copy_cols(f.dh0, sp, dh02, sz, BH, sz, sz, st));
      pass2_done = true;
    }
  }
  if (!pass2_done) {
    GLA_CUDA(gk::state_fwd<TI>(s2, phi, v, g, h02, 0, w.S2, w.hT2, 0, st));
    GLA_CUDA((gk::dstate_bwd<TI, TI>(s2, p, g, dO, dhT2, 0, w.dS2, dh02, 0, st)));
    GLA_CUDA((gk::bwd_dqdk<TI, TI, float>(s2, p, phi, v, g, dO, w.S2, w.dS2, w.dp, w.dphi2, nullptr, w.db, st)));
    GLA_CUDA((gk::bwd_dv<TI, TI, TI>(s2, p, phi, g, dO, w.dS2, dv, st)));
    GLA_CUDA(gk::dg<float>(s2, w.db, w.hT2, dhT2, 0, nullptr, w.dg2, st));
  }
  // slot softmax Jacobian
  GLA_CUDA(gk::softmax_bwd(w.o1, w.dp, w.do1, (long)BH * T, m, st));
  // pass 1 backward with roles exchanged
  GLA_CUDA((gk::dstate_bwd<float, TI>(s1, w.do1, g, q, dhT1, 1, w.dS1, dh01, 1, st)));
  GLA_CUDA((gk::out<float, TI, TI>(s1, w.do1, phi, k, g, w.S1, dq, st)));
  GLA_CUDA((gk::bwd_dv<float, TI, TI>(s1, w.do1, phi, g, q, w.dS1, dk, st)));
  GLA_CUDA((gk::bwd_dqdk<float, TI, TI>(s1, w.do1, phi, k, g, q, w.S1, w.dS1, nullptr, dphi, w.dphi2, w.db, st)));
  GLA_CUDA(gk::dg<TI>(s1, w.db, w.hT1, dhT1, 1, w.dg2, dg, st));
  return GLA_OK;
}

}  // namespace

// =========================================================================================
// C ABI
// =========================================================================================
extern "C" {

const char* gla_status_string(int status) {
  switch (status) {
    case GLA_OK: return "GLA_OK";
    case GLA_ERR_INVALID_ARG: return "GLA_ERR_INVALID_ARG: NULL, misaligned or out-of-range argument";
    case GLA_ERR_UNSUPPORTED: return "GLA_ERR_UNSUPPORTED: dtype, chunk or dimension not supported";
    case GLA_ERR_WORKSPACE: return "GLA_ERR_WORKSPACE: workspace missing or too small";
    case GLA_ERR_CUDA: return "GLA_ERR_CUDA: a CUDA call or kernel launch failed";
    case GLA_ERR_TIMEOUT: return "GLA_ERR_TIMEOUT: a bounded device-side wait ran out";
  }
  return "unknown gla_status";
}

int gla_version(void) { return kVersion; }

size_t gla_chunk_fwd_workspace(int B, int H, int T, int dk, int dv, int chunk, int dtype) {
  if (check_common(B, H, T, chunk, dtype) || check_dim(dk) || check_dim(dv)) return 0;
  if (T == 0) return 0;
  if (gla::fast::fwd_supported(B * H, T, dk, dv, chunk, dtype)) return gla::fast::fwd_workspace(B * H, T, dk, dv);
  Carve c(nullptr);
  if (split_fwd_ok(B * H, T, dk, dv, chunk, dtype)) return carve_split_fwd(c, B * H, T, dk, dv, nullptr);
  return carve_gla_fwd(c, B * H, T, dk, dv, chunk, nullptr);
}

size_t gla_chunk_bwd_workspace(int B, int H, int T, int dk, int dv, int chunk, int dtype) {
  if (check_common(B, H, T, chunk, dtype) || check_dim(dk) || check_dim(dv)) return 0;
  if (T == 0) return 0;
  if (gla::fast::bwd_supported(B * H, T, dk, dv, chunk, dtype)) return gla::fast::bwd_workspace(B * H, T, dk, dv);
  Carve c(nullptr);
  if (split_bwd_ok(B * H, T, dk, dv, chunk, dtype)) return carve_split_bwd(c, B * H, T, dk, dv, nullptr);
  return carve_gla_bwd(c, B * H, T, dk, dv, chunk, nullptr);
}

// Raw-logit entries: the fused and blocked paths form g = logsigmoid(x) / tau inside their gate
// runs; the generic kernels take g from the standalone gate pass, written behind their workspace.
size_t gla_chunk_fwd_logit_workspace(int B, int H, int T, int dk, int dv, int chunk, int dtype) {
  const size_t base = gla_chunk_fwd_workspace(B, H, T, dk, dv, chunk, dtype);
  if (T <= 0 || check_common(B, H, T, chunk, dtype) || check_dim(dk) || check_dim(dv)) return base;
  if (gla::fast::fwd_supported(B * H, T, dk, dv, chunk, dtype) || split_fwd_ok(B * H, T, dk, dv, chunk, dtype))
    return base;
  return gla::align256(base) + gla::align256((size_t)B * H * T * dk * esize(dtype));
}

size_t gla_chunk_bwd_logit_workspace(int B, int H, int T, int dk, int dv, int chunk, int dtype) {
  const size_t base = gla_chunk_bwd_workspace(B, H, T, dk, dv, chunk, dtype);
  if (T <= 0 || check_common(B, H, T, chunk, dtype) || check_dim(dk) || check_dim(dv)) return base;
  if (gla::fast::bwd_supported(B * H, T, dk, dv, chunk, dtype) || split_bwd_ok(B * H, T, dk, dv, chunk, dtype))
    return base;
  return gla::align256(base) + gla::align256((size_t)B * H * T * dk * esize(dtype));
}

}  // extern "C"

namespace {

// tau == 0: g holds log-gates; tau > 0: g holds raw logits x and the operator uses logsigmoid(x) / tau.
int chunk_fwd_entry(const void* q, const void* k, const void* v, const void* g, float tau, const float* h0, void* o,
                    float* hT, int B, int H, int T, int dk, int dv, int chunk, int dtype, void* ws, size_t ws_bytes,
                    void* stream) {
  GLA_TRY(check_common(B, H, T, chunk, dtype));
  GLA_TRY(check_dim(dk));
  GLA_TRY(check_dim(dv));
  const bool tok = T > 0;
  GLA_TRY(check_ptr(q, tok));
  GLA_TRY(check_ptr(k, tok));
  GLA_TRY(check_ptr(v, tok));
  GLA_TRY(check_ptr(g, tok));
  GLA_TRY(check_ptr(o, tok));
  GLA_TRY(check_ptr(h0, false));
  GLA_TRY(check_ptr(hT, false));
  const bool logit = tau != 0.f;
  if (logit && !(tau > 0.f && tau < 3.0e38f)) return GLA_ERR_INVALID_ARG;
  const size_t need = logit ? gla_chunk_fwd_logit_workspace(B, H, T, dk, dv, chunk, dtype)
                            : gla_chunk_fwd_workspace(B, H, T, dk, dv, chunk, dtype);
  if (need > 0 && (!ws || ws_bytes < need || !aligned16(ws))) return GLA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
  if (T == 0) return copy_or_zero(hT, h0, (size_t)BH * dk * dv, st);
  const float inv_tau = logit ? 1.f / tau : 0.f;
  if (gla::fast::fwd_supported(BH, T, dk, dv, chunk, dtype))
    return gla::fast::fwd(q, k, v, g, h0, o, hT, BH, T, dk, dv, ws, st, -1, -1, nullptr, inv_tau) == cudaSuccess
               ? GLA_OK
               : GLA_ERR_CUDA;
  if (split_fwd_ok(BH, T, dk, dv, chunk, dtype))
    return split_fwd((const bf16*)q, (const bf16*)k, (const bf16*)v, (const bf16*)g, h0, (bf16*)o, hT, BH, T, dk, dv,
                     ws, st, inv_tau);
  if (logit) {  // the standalone gate pass into the space behind the generic kernels' workspace
    void* gbuf = static_cast<char*>(ws) + gla::align256(gla_chunk_fwd_workspace(B, H, T, dk, dv, chunk, dtype));
    GLA_TRY(gla_gate_logsigmoid(g, gbuf, (size_t)BH * T * dk, tau, dtype, stream));
    g = gbuf;
  }
  const gk::Shape s{BH, T, dk, dv, chunk};
  if (dtype == GLA_DTYPE_BF16)
    return gla_fwd_generic<bf16>((const bf16*)q, (const bf16*)k, (const bf16*)v, (const bf16*)g, h0, (bf16*)o, hT,
                                 s, ws, st);
  return gla_fwd_generic<float>((const float*)q, (const float*)k, (const float*)v, (const float*)g, h0, (float*)o,
                                hT, s, ws, st);
}

int chunk_bwd_entry(const void* q, const void* k, const void* v, const void* g, float tau, const float* h0,
                    const void* dO, const float* dhT, void* dq, void* dk, void* dv, void* dg, float* dh0, int B, int H,
                    int T, int dkd, int dvd, int chunk, int dtype, void* ws, size_t ws_bytes, void* stream) {
  GLA_TRY(check_common(B, H, T, chunk, dtype));
  GLA_TRY(check_dim(dkd));
  GLA_TRY(check_dim(dvd));
  const bool tok = T > 0;
  const void* req[] = {q, k, v, g, dO, dq, dk, dv, dg};
  for (const void* p : req) GLA_TRY(check_ptr(p, tok));
  GLA_TRY(check_ptr(h0, false));
  GLA_TRY(check_ptr(dhT, false));
  GLA_TRY(check_ptr(dh0, false));
  const bool logit = tau != 0.f;
  if (logit && !(tau > 0.f && tau < 3.0e38f)) return GLA_ERR_INVALID_ARG;
  const size_t need = logit ? gla_chunk_bwd_logit_workspace(B, H, T, dkd, dvd, chunk, dtype)
                            : gla_chunk_bwd_workspace(B, H, T, dkd, dvd, chunk, dtype);
  if (need > 0 && (!ws || ws_bytes < need || !aligned16(ws))) return GLA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
  if (T == 0) return copy_or_zero(dh0, dhT, (size_t)BH * dkd * dvd, st);
  const float inv_tau = logit ? 1.f / tau : 0.f;
  if (gla::fast::bwd_supported(BH, T, dkd, dvd, chunk, dtype))
    return gla::fast::bwd(q, k, v, g, h0, dO, dhT, dq, dk, dv, dg, dh0, BH, T, dkd, dvd, ws, st, -1, -1, nullptr,
                          inv_tau) == cudaSuccess
               ? GLA_OK
               : GLA_ERR_CUDA;
  if (split_bwd_ok(BH, T, dkd, dvd, chunk, dtype))
    return split_bwd((const bf16*)q, (const bf16*)k, (const bf16*)v, (const bf16*)g, h0, (const bf16*)dO, dhT,
                     (bf16*)dq, (bf16*)dk, (bf16*)dv, (bf16*)dg, dh0, BH, T, dkd, dvd, ws, st, inv_tau);
  const void* x = g;
  if (logit) {
    void* gbuf = static_cast<char*>(ws) + gla::align256(gla_chunk_bwd_workspace(B, H, T, dkd, dvd, chunk, dtype));
    GLA_TRY(gla_gate_logsigmoid(x, gbuf, (size_t)BH * T * dkd, tau, dtype, stream));
    g = gbuf;
  }
  const gk::Shape s{BH, T, dkd, dvd, chunk};
  int r;
  if (dtype == GLA_DTYPE_BF16)
    r = gla_bwd_generic<bf16>((const bf16*)q, (const bf16*)k, (const bf16*)v, (const bf16*)g, h0, (const bf16*)dO, dhT,
                              (bf16*)dq, (bf16*)dk, (bf16*)dv, (bf16*)dg, dh0, s, ws, st);
  else
    r = gla_bwd_generic<float>((const float*)q, (const float*)k, (const float*)v, (const float*)g, h0,
                               (const float*)dO, dhT, (float*)dq, (float*)dk, (float*)dv, (float*)dg, dh0, s, ws, st);
  if (r != GLA_OK || !logit) return r;
  return gla_gate_logsigmoid_bwd(x, dg, dg, (size_t)BH * T * dkd, tau, dtype, stream);  // dx = dg sigmoid(-x) / tau
}

}  // namespace

extern "C" {

int gla_chunk_fwd(const void* q, const void* k, const void* v, const void* g, const float* h0, void* o, float* hT,
                  int B, int H, int T, int dk, int dv, int chunk, int dtype, void* ws, size_t ws_bytes,
                  void* stream) {
  return chunk_fwd_entry(q, k, v, g, 0.f, h0, o, hT, B, H, T, dk, dv, chunk, dtype, ws, ws_bytes, stream);
}

int gla_chunk_fwd_logit(const void* q, const void* k, const void* v, const void* x, float tau, const float* h0,
                        void* o, float* hT, int B, int H, int T, int dk, int dv, int chunk, int dtype, void* ws,
                        size_t ws_bytes, void* stream) {
  if (!(tau > 0.f)) return GLA_ERR_INVALID_ARG;
  return chunk_fwd_entry(q, k, v, x, tau, h0, o, hT, B, H, T, dk, dv, chunk, dtype, ws, ws_bytes, stream);
}

int gla_chunk_bwd(const void* q, const void* k, const void* v, const void* g, const float* h0, const void* dO,
                  const float* dhT, void* dq, void* dk, void* dv, void* dg, float* dh0, int B, int H, int T,
                  int dkd, int dvd, int chunk, int dtype, void* ws, size_t ws_bytes, void* stream) {
  return chunk_bwd_entry(q, k, v, g, 0.f, h0, dO, dhT, dq, dk, dv, dg, dh0, B, H, T, dkd, dvd, chunk, dtype, ws,
                         ws_bytes, stream);
}

int gla_chunk_bwd_logit(const void* q, const void* k, const void* v, const void* x, float tau, const float* h0,
                        const void* dO, const float* dhT, void* dq, void* dk, void* dv, void* dx, float* dh0, int B,
                        int H, int T, int dkd, int dvd, int chunk, int dtype, void* ws, size_t ws_bytes,
                        void* stream) {
  if (!(tau > 0.f)) return GLA_ERR_INVALID_ARG;
  return chunk_bwd_entry(q, k, v, x, tau, h0, dO, dhT, dq, dk, dv, dx, dh0, B, H, T, dkd, dvd, chunk, dtype, ws,
                         ws_bytes, stream);
}

int gla_recurrent_step(const void* q, const void* k, const void* v, const void* g, float* S, void* o, int B, int H,
                       int dk, int dv, int dtype, void* stream) {
  GLA_TRY(check_common(B, H, 1, 64, dtype));
  GLA_TRY(check_dim(dk));
  GLA_TRY(check_dim(dv));
  const void* req[] = {q, k, v, g, S, o};
  for (const void* p : req) GLA_TRY(check_ptr(p, true));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
  if (dtype == GLA_DTYPE_BF16)
    GLA_CUDA(gk::decode<bf16>(BH, dk, dv, (const bf16*)q, (const bf16*)k, (const bf16*)v, (const bf16*)g, S,
                              (bf16*)o, st));
  else
    GLA_CUDA(gk::decode<float>(BH, dk, dv, (const float*)q, (const float*)k, (const float*)v, (const float*)g, S,
                               (float*)o, st));
  return GLA_OK;
}

size_t gsa_fwd_workspace(int B, int H, int T, int dk, int dv, int m, int chunk, int dtype) {
  if (check_common(B, H, T, chunk, dtype) || check_dim(dk) || check_dim(dv) || check_dim(m)) return 0;
  if (T == 0) return 0;
  Carve c(nullptr);
  if (gsa_fused_fwd_ok(B * H, T, dk, dv, m, chunk, dtype))
    return carve_gsa_fused_fwd(c, B * H, T, dk, dv, m, true, nullptr);
  return carve_gsa_fwd(c, B * H, T, dk, dv, m, chunk, dtype, true, nullptr);
}

int gsa_fwd(const void* q, const void* k, const void* v, const void* phi, const void* g, const float* h0_1,
            const float* h0_2, void* o, void* p_save, float* hT1, float* hT2, int B, int H, int T, int dk, int dv,
            int m, int chunk, int dtype, void* ws, size_t ws_bytes, void* stream) {
  GLA_TRY(check_common(B, H, T, chunk, dtype));
  GLA_TRY(check_dim(dk));
  GLA_TRY(check_dim(dv));
  GLA_TRY(check_dim(m));
  const bool tok = T > 0;
  const void* req[] = {q, k, v, phi, g, o};
  for (const void* p : req) GLA_TRY(check_ptr(p, tok));
  const void* opt[] = {h0_1, h0_2, p_save, hT1, hT2};
  for (const void* p : opt) GLA_TRY(check_ptr(p, false));
  const size_t need = gsa_fwd_workspace(B, H, T, dk, dv, m, chunk, dtype);
  if (need > 0 && (!ws || ws_bytes < need || !aligned16(ws))) return GLA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
  if (T == 0) {
    GLA_TRY(copy_or_zero(hT1, h0_1, (size_t)BH * dk * m, st));
    return copy_or_zero(hT2, h0_2, (size_t)BH * m * dv, st);
  }
  if (gsa_fused_fwd_ok(BH, T, dk, dv, m, chunk, dtype))
    return gsa_fwd_fused((const bf16*)q, (const bf16*)k, (const bf16*)v, (const bf16*)phi, (const bf16*)g, h0_1, h0_2,
                         (bf16*)o, (bf16*)p_save, hT1, hT2, BH, T, dk, dv, m, ws, st);
  if (dtype == GLA_DTYPE_BF16)
    return gsa_fwd_impl<bf16>((const bf16*)q, (const bf16*)k, (const bf16*)v, (const bf16*)phi, (const bf16*)g,
                              h0_1, h0_2, (bf16*)o, (bf16*)p_save, hT1, hT2, BH, T, dk, dv, m, chunk, ws, st);
  return gsa_fwd_impl<float>((const float*)q, (const float*)k, (const float*)v, (const float*)phi,
                             (const float*)g, h0_1, h0_2, (float*)o, (float*)p_save, hT1, hT2, BH, T, dk, dv, m,
                             chunk, ws, st);
}

size_t gsa_bwd_workspace(int B, int H, int T, int dk, int dv, int m, int chunk, int dtype) {
  if (check_common(B, H, T, chunk, dtype) || check_dim(dk) || check_dim(dv) || check_dim(m)) return 0;
  if (T == 0) return 0;
  Carve c(nullptr);
  if (gsa_fused_bwd_ok(B * H, T, dk, dv, m, chunk, dtype)) return carve_gsa_fused_bwd(c, B * H, T, dk, dv, m, nullptr);
  return carve_gsa_bwd(c, B * H, T, dk, dv, m, chunk, dtype, nullptr);
}

int gsa_bwd(const void* q, const void* k, const void* v, const void* phi, const void* g, const float* h0_1,
            const float* h0_2, const void* dO, const float* dhT1, const float* dhT2, void* dq, void* dk, void* dv,
            void* dphi, void* dg, float* dh0_1, float* dh0_2, int B, int H, int T, int dkd, int dvd, int m,
            int chunk, int dtype, void* ws, size_t ws_bytes, void* stream) {
  GLA_TRY(check_common(B, H, T, chunk, dtype));
  GLA_TRY(check_dim(dkd));
  GLA_TRY(check_dim(dvd));
  GLA_TRY(check_dim(m));
  const bool tok = T > 0;
  const void* req[] = {q, k, v, phi, g, dO, dq, dk, dv, dphi, dg};
  for (const void* p : req) GLA_TRY(check_ptr(p, tok));
  const void* opt[] = {h0_1, h0_2, dhT1, dhT2, dh0_1, dh0_2};
  for (const void* p : opt) GLA_TRY(check_ptr(p, false));
  const size_t need = gsa_bwd_workspace(B, H, T, dkd, dvd, m, chunk, dtype);
  if (need > 0 && (!ws || ws_bytes < need || !aligned16(ws))) return GLA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
  if (T == 0) {
    GLA_TRY(copy_or_zero(dh0_1, dhT1, (size_t)BH * dkd * m, st));
    return copy_or_zero(dh0_2, dhT2, (size_t)BH * m * dvd, st);
  }
  if (gsa_fused_bwd_ok(BH, T, dkd, dvd, m, chunk, dtype))
    return gsa_bwd_fused((const bf16*)q, (const bf16*)k, (const bf16*)v, (const bf16*)phi, (const bf16*)g, h0_1, h0_2,
                         (const bf16*)dO, dhT1, dhT2, (bf16*)dq, (bf16*)dk, (bf16*)dv, (bf16*)dphi, (bf16*)dg, dh0_1,
                         dh0_2, BH, T, dkd, dvd, m, ws, st);
  if (dtype == GLA_DTYPE_BF16)
    return gsa_bwd_impl<bf16>((const bf16*)q, (const bf16*)k, (const bf16*)v, (const bf16*)phi, (const bf16*)g,
                              h0_1, h0_2, (const bf16*)dO, dhT1, dhT2, (bf16*)dq, (bf16*)dk, (bf16*)dv, (bf16*)dphi,
                              (bf16*)dg, dh0_1, dh0_2, BH, T, dkd, dvd, m, chunk, ws, st);
  return gsa_bwd_impl<float>((const float*)q, (const float*)k, (const float*)v, (const float*)phi,
                             (const float*)g, h0_1, h0_2, (const float*)dO, dhT1, dhT2, (float*)dq, (float*)dk,
                             (float*)dv, (float*)dphi, (float*)dg, dh0_1, dh0_2, BH, T, dkd, dvd, m, chunk, ws, st);
}

int gsa_recurrent_step(const void* q, const void* k, const void* v, const void* phi, const void* g, float* S1,
                       float* S2, void* o, int B, int H, int dk, int dv, int m, int dtype, void* stream) {
  GLA_TRY(check_common(B, H, 1, 64, dtype));
  GLA_TRY(check_dim(dk));
  GLA_TRY(check_dim(dv));
  GLA_TRY(check_dim(m));
  const void* req[] = {q, k, v, phi, g, S1, S2, o};
  for (const void* p : req) GLA_TRY(check_ptr(p, true));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
  if (dtype == GLA_DTYPE_BF16)
    GLA_CUDA(gk::gsa_decode<bf16>(BH, dk, dv, m, (const bf16*)q, (const bf16*)k, (const bf16*)v,
                                  (const bf16*)phi, (const bf16*)g, S1, S2, (bf16*)o, st));
  else
    GLA_CUDA(gk::gsa_decode<float>(BH, dk, dv, m, (const float*)q, (const float*)k, (const float*)v,
                                   (const float*)phi, (const float*)g, S1, S2, (float*)o, st));
  return GLA_OK;
}

int gla_device_error(void* stream, int reset, int* code) {
  if (!code) return GLA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned int v = 0;
  GLA_CUDA(cudaMemcpyFromSymbolAsync(&v, g_gla_device_error, sizeof(v), 0, cudaMemcpyDeviceToHost, st));
  GLA_CUDA(cudaStreamSynchronize(st));
  if (reset) {
    const unsigned int zero = 0;
    GLA_CUDA(cudaMemcpyToSymbolAsync(g_gla_device_error, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, st));
    GLA_CUDA(cudaStreamSynchronize(st));
  }
  *code = v == 0 ? GLA_OK : (int)v;
  return GLA_OK;
}

}  // extern "C"

// Address of the device error latch for kernels in other translation units.
namespace gla {
unsigned int* device_error_latch() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_gla_device_error) != cudaSuccess) return nullptr;
  return static_cast<unsigned int*>(p);
}
}  // namespace gla
