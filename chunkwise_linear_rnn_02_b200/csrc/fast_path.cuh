// Fused sm_100a (tcgen05 / TMEM / TMA) chunkwise kernels for the bf16 GLA shapes they cover.
// The API layer asks *_supported() first and otherwise runs the generic kernels.
#pragma once

#include <mutex>

#include <cuda.h>

#include "common.cuh"

namespace gla {

// Address of the device-side error latch (defined with the C ABI).
unsigned int* device_error_latch();

namespace fast {

bool fwd_supported(int BH, int T, int dk, int dv, int chunk, int dtype);
size_t fwd_workspace(int BH, int T, int dk, int dv);
// st_bh / st_row: element strides of the fp32 states per head and per row (defaults, when
// negative: dk*dv and dv).  A split shape passes a sub-block of the caller's states this way, and
// an fp32 array acc_o [BH*T][dv] that receives o in place of the bf16 output.  inv_tau > 0: g holds
// raw logits x and the kernels use g = bf16(logsigmoid(x) * inv_tau).  A key block of wider
// tensors: q, k, g are [BH][T][dk_total] and the call uses columns k0 .. k0+dk-1 (read in place by
// the tile loads); add_o ([BH*T][dv] fp32) is added to o before it is stored (to acc_o or as bf16).
// kh_hilo (d_k = 64 only): the decayed keys enter the MMAs as bf16 hi + lo pairs too.
// phase: kFwdAll runs the whole forward; with a sequence split, kFwdStates runs only the segment
// entry states (state pass and scan, into ws; they need k, g, v and h0, not q) and kFwdWalk only the
// walks, from entry states an earlier kFwdStates call with the same arguments left in ws.  Without a
// split kFwdStates does nothing and kFwdWalk is kFwdAll.
enum FwdPhase { kFwdAll = 0, kFwdStates = 1, kFwdWalk = 2 };
cudaError_t fwd(const void* q, const void* k, const void* v, const void* g, const float* h0, void* o, float* hT,
                int BH, int T, int dk, int dv, void* ws, cudaStream_t st, long long st_bh = -1,
                long long st_row = -1, float* acc_o = nullptr, float inv_tau = 0.f, int dk_total = -1, int k0 = 0,
                const float* add_o = nullptr, bool kh_hilo = false, int phase = kFwdAll);

// A backward sub-problem inside wider tensors (split shapes, padded operands): its key dimensions
// are columns ck.. of the [BH*T][pk] inputs q, k, g, its value columns cv.. of the [BH*T][pv] inputs
// v and dO.  The key-side gradients go in fp32 to q / k / g (all required, [BH*T][dk] each) in place
// of the bf16 outputs; dv goes in fp32 to v ([BH*T][dv]), or, with v null, in bf16 to the dv output,
// then [BH*T][pv] and written at columns cv...
struct BwdAccum {
  float *q, *k, *g, *v;
  int pk, ck, pv, cv;
};

// Sequence split of the backward (d_k = 128): segment count and length, and the segment states
// (fp32 [BH][nseg][DK][DV]): sbuf[s-1] = the forward state entering segment s (s >= 1, from h0),
// gbuf[s] = dL/dS at the end of segment s (s <= nseg-2, from dhT), gam[s] = the decay product of
// segment s (s <= nseg-2).  Maps: q, k, g as [64 x DK] row tiles, v and dO as 64-column tiles.
void plan_bwd_segments(int ctas_per_seg, int T, int* nseg, int* seg_chunks);
cudaError_t segment_states(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mg,
                           const CUtensorMap& mv, const CUtensorMap& mdo, const float* h0, const float* dhT,
                           float* sbuf, float* gbuf, float* gam, int BH, int T, int dk, int dv, int nseg,
                           int seg_chunks, long long st_bh, long long st_row, cudaStream_t st, float inv_tau, int ck,
                           int cv);

// SM count of the current device (cached per device).
int sm_count();

// A second stream per device and pool, with fork / join events, for launches that need not run after
// one another; made on first use.  Its mutex is held while a call enqueues its work there, so that
// the event records and waits of concurrent callers do not interleave.  Pool 0 serves the API layer
// (wide-shape sub-problems, GSA), pool 1 the launches inside one fused call (the backward's segment
// state passes), so that a call made while pool 0 is held never waits for it again.
struct SideStream {
  cudaStream_t s;
  cudaEvent_t fork, join;
  std::mutex mu;
};
cudaError_t side_stream(int pool, SideStream** out);

// Sequence split of a key-gated recurrence S <- diag(e^{g_t}) S + k_t^T v_t with d_k = 64 rows
// (k, g: bf16 [BH][T][64]; v: bf16 [BH][T][dv], dv a multiple of 64), for a caller that walks the
// segments itself: sbuf [BH][nseg][64][dv] receives in entry s-1 the state entering segment s
// (s >= 1; the first segment starts from h0 [BH][64][dv] or zeros), gam [BH][nseg][64] the
// segments' decay products.
cudaError_t segment_entry_states(const void* k, const void* g, const void* v, const float* h0, float* sbuf,
                                 float* gam, int BH, int T, int dk, int dv, int nseg, int seg_chunks,
                                 cudaStream_t st);

bool bwd_supported(int BH, int T, int dk, int dv, int chunk, int dtype);
size_t bwd_workspace(int BH, int T, int dk, int dv);
// inv_tau > 0: g holds raw logits x (as for fwd) and dg receives dx = dg * sigmoid(-x) / tau.
cudaError_t bwd(const void* q, const void* k, const void* v, const void* g, const float* h0, const void* dO,
                const float* dhT, void* dq, void* dk, void* dv, void* dg, float* dh0, int BH, int T, int dkd,
                int dvd, void* ws, cudaStream_t st, long long st_bh = -1, long long st_row = -1,
                const BwdAccum* acc = nullptr, float inv_tau = 0.f);

}  // namespace fast
}  // namespace gla
