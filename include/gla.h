/*
 * gla.h - C ABI of the B200 (sm_100a) chunkwise Gated Linear Attention library.
 *
 * Operators
 * ---------
 * GLA (key-gated linear recurrence over a matrix memory, one head):
 *     S_t = diag(exp g_t) . S_{t-1} + k_t^T v_t ,      o_t = q_t . S_t
 *   q_t, k_t, g_t in R^dk, v_t in R^dv, S_t in R^{dk x dv}.
 *   Described in words by "Gated Linear Attention for Efficient Long Sequences" (panels "Core
 *   move" and "Step-by-step memory update") and by "MS-GLA: Multi-Scale Gated Linear
 *   Attention ...", section 2.1 (data-dependent forget gate that scales rows of the memory;
 *   chunkwise training with sequential inter-chunk and parallel intra-chunk work).
 * GSA (Gated Slot Attention, m memory slots):
 *     o1 = GLA_v(q, k, phi, g)  (pass 1: gate on the slot axis, which is the value axis)
 *     p  = softmax over the m slots of o1
 *     o  = GLA(p, phi, v, g)    (pass 2: keys phi, the same slot gates, now on the key axis)
 *   "Gated Slot Attention for Efficient Linear-Time Sequence Modeling", abstract (two-layer
 *   GLA linked via softmax) and "Approach" (two-pass linear attention, per-slot forget gates).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout      Per-token tensors are contiguous [B, H, T, D] (D fastest).  States and their
 *             gradients (h0, hT, dhT, dh0, S) are contiguous float32 [B, H, rows, cols]:
 *             GLA [B,H,dk,dv]; GSA pass 1 [B,H,dk,m]; GSA pass 2 [B,H,m,dv].
 * dtype       GLA_DTYPE_BF16: q, k, v, g, phi, o, p and all per-token gradients are bf16;
 *             arithmetic accumulates in fp32.  GLA_DTYPE_F32: all of them are fp32 and no
 *             reduced-precision (bf16 or TF32) arithmetic is used anywhere.
 * Gate        g is the log of the decay (alpha = exp g).  It must be finite and <= 0;
 *             g = 0 means "keep", very negative g means "forget".  No scale is applied to q.
 * chunk       Chunk length of the chunkwise algorithm: 16, 32 or 64.  It changes rounding
 *             only, never the mathematical result.
 * Tails       T need not be a multiple of chunk.  T == 0 is allowed: per-token pointers may
 *             then be NULL, hT is set to h0 (or zeros) and dh0 to dhT (or zeros).
 * Optional    A NULL optional input means zeros (h0, dhT).  A NULL optional output is not
 *             written (hT, dh0, p_save).
 * Ownership   The caller owns every buffer, including the workspace; nothing is allocated,
 *             freed or retained by the library between calls.  Device pointers must be
 *             16-byte aligned.  Buffers of one call must not overlap, except where stated.
 * Streams     All work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is the
 *             legacy default stream).  Calls return once the work is enqueued.
 * Workspace   `*_workspace()` returns the bytes the matching call needs for those sizes (0 is
 *             possible).  Pass at least that many bytes, 256-byte aligned.  The workspace
 *             contents on entry do not matter; on exit they are unspecified.
 * Errors      Invalid arguments are rejected before anything is enqueued:
 *               GLA_ERR_INVALID_ARG   NULL required pointer, negative or zero size where a
 *                                     positive one is required, misaligned pointer
 *               GLA_ERR_UNSUPPORTED   dtype, chunk or a dimension outside the supported set
 *               GLA_ERR_WORKSPACE     workspace NULL or smaller than *_workspace() returned
 *             A failed kernel launch returns GLA_ERR_CUDA.  Kernels never trap: every wait on
 *             an mbarrier is bounded, and a wait that runs out records GLA_ERR_TIMEOUT in a
 *             device-side latch that gla_device_error() reads.
 * Supported   1 <= dk, dv, m <= 512; dk, dv, m multiples of 8; B*H <= 2^31-1.
 */
#ifndef GLA_B200_H
#define GLA_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GLA_OK = 0,
  GLA_ERR_INVALID_ARG = 1,
  GLA_ERR_UNSUPPORTED = 2,
  GLA_ERR_WORKSPACE = 3,
  GLA_ERR_CUDA = 4,
  GLA_ERR_TIMEOUT = 5
} gla_status;

typedef enum { GLA_DTYPE_F32 = 0, GLA_DTYPE_BF16 = 1 } gla_dtype;

/* Human-readable name of a status code (static string, never NULL). */
const char* gla_status_string(int status);

/* Library ABI version: major * 10000 + minor * 100 + patch. */
int gla_version(void);

/* ---------------------------------------------------------------------------------------
 * gla_chunk_fwd - chunkwise GLA forward.
 *   in : q, k, g [B,H,T,dk]; v [B,H,T,dv]; h0 [B,H,dk,dv] fp32 (optional, NULL = zeros)
 *   out: o [B,H,T,dv]; hT = S_T [B,H,dk,dv] fp32 (optional)
 * Chunkwise form ("MS-GLA", section 2.1): the state is carried chunk to chunk; inside a chunk
 * the output is the inter-chunk term (q * exp(b)) S_in plus the gated causal intra-chunk term.
 * ------------------------------------------------------------------------------------- */
size_t gla_chunk_fwd_workspace(int B, int H, int T, int dk, int dv, int chunk, int dtype);
int gla_chunk_fwd(const void* q, const void* k, const void* v, const void* g, const float* h0,
                  void* o, float* hT, int B, int H, int T, int dk, int dv, int chunk, int dtype,
                  void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * gla_chunk_bwd - gradients of L(o, hT) for the same inputs as gla_chunk_fwd.
 *   in : q, k, g, v, h0 (optional) as in gla_chunk_fwd; dO [B,H,T,dv];
 *        dhT [B,H,dk,dv] fp32 (optional, NULL = zeros)
 *   out: dq, dk, dg [B,H,T,dk]; dv [B,H,T,dv]; dh0 [B,H,dk,dv] fp32 (optional)
 * The reverse-mode recurrence is derived from the forward recurrence; dg is the reverse
 * cumulative sum over t of q*dq - k*dk plus, for every t, sum_j dhT[i,j] hT[i,j].
 * It is the gradient of the same chunkwise form ("MS-GLA", section 2.1: chunkwise parallel
 * training of the gated recurrence, sequential across chunks and parallel inside a chunk),
 * evaluated chunk by chunk in reverse with the state gradient kept on chip ("Gated Linear
 * Attention for Efficient Long Sequences", "Why chunking and SRAM locality matter": only
 * inputs and gradients cross HBM, no per-step state is written).
 * ------------------------------------------------------------------------------------- */
size_t gla_chunk_bwd_workspace(int B, int H, int T, int dk, int dv, int chunk, int dtype);
int gla_chunk_bwd(const void* q, const void* k, const void* v, const void* g, const float* h0,
                  const void* dO, const float* dhT, void* dq, void* dk, void* dv, void* dg,
                  float* dh0, int B, int H, int T, int dk_dim, int dv_dim, int chunk, int dtype,
                  void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * gla_chunk_fwd_logit / gla_chunk_bwd_logit - gla_chunk_fwd / gla_chunk_bwd with the gate given
 * as raw logits: x [B,H,T,dk] in place of g, with g = logsigmoid(x) / tau formed inside the
 * kernels' gate runs ("MS-GLA", section 2.1: a data-dependent forget gate; "Gated Slot
 * Attention ...", "Approach": sigmoid forget gates, alpha = sigmoid(x)^(1/tau)).  The log-gates
 * equal, value for value, what gla_gate_logsigmoid stores for x (so these calls return exactly
 * what gla_gate_logsigmoid followed by gla_chunk_fwd / gla_chunk_bwd returns), without that
 * pass's trip through memory.  The backward writes dx = dg * sigmoid(-x) / tau into `dx` in
 * place of dg.  tau > 0 and finite (else GLA_ERR_INVALID_ARG).  Everything else, including the
 * errors, as for gla_chunk_fwd / gla_chunk_bwd; the workspace is what the *_logit_workspace()
 * query returns (the shapes the generic kernels serve need room for g behind their own).
 * ------------------------------------------------------------------------------------- */
size_t gla_chunk_fwd_logit_workspace(int B, int H, int T, int dk, int dv, int chunk, int dtype);
int gla_chunk_fwd_logit(const void* q, const void* k, const void* v, const void* x, float tau,
                        const float* h0, void* o, float* hT, int B, int H, int T, int dk, int dv,
                        int chunk, int dtype, void* workspace, size_t workspace_bytes, void* stream);
size_t gla_chunk_bwd_logit_workspace(int B, int H, int T, int dk, int dv, int chunk, int dtype);
int gla_chunk_bwd_logit(const void* q, const void* k, const void* v, const void* x, float tau,
                        const float* h0, const void* dO, const float* dhT, void* dq, void* dk,
                        void* dv, void* dx, float* dh0, int B, int H, int T, int dk_dim,
                        int dv_dim, int chunk, int dtype, void* workspace, size_t workspace_bytes,
                        void* stream);

/* ---------------------------------------------------------------------------------------
 * gla_recurrent_step - one token of recurrent inference, in place on the state.
 *   in : q, k, g [B,H,dk]; v [B,H,dv]; S [B,H,dk,dv] fp32 (read, then overwritten)
 *   out: o [B,H,dv];  S <- diag(exp g) S + k^T v ; o = q S
 * "MS-GLA", section 1 (O(1) inference memory per token).  No workspace.  S may not alias
 * any other argument.
 * ------------------------------------------------------------------------------------- */
int gla_recurrent_step(const void* q, const void* k, const void* v, const void* g, float* S,
                       void* o, int B, int H, int dk, int dv, int dtype, void* stream);

/* ---------------------------------------------------------------------------------------
 * gsa_fwd - Gated Slot Attention forward.
 *   in : q, k [B,H,T,dk]; v [B,H,T,dv]; phi, g [B,H,T,m] (g: per-slot log forget gate);
 *        h0_1 [B,H,dk,m], h0_2 [B,H,m,dv] fp32 (optional)
 *   out: o [B,H,T,dv]; p_save [B,H,T,m] (optional: the slot softmax p, in dtype);
 *        hT1 [B,H,dk,m], hT2 [B,H,m,dv] fp32 (optional)
 * "Gated Slot Attention ...", abstract (a two-layer GLA linked via softmax) and "Approach"
 * (two-pass linear attention with a softmax in between; a data-dependent forget gate per
 * slot; reuses GLA's chunkwise training form): pass 1 writes k into the m slots weighted by
 * phi under the slot gates and reads them with q; the softmax over the slots gives p; pass 2
 * reads the values written under the same gates with p.
 * ------------------------------------------------------------------------------------- */
size_t gsa_fwd_workspace(int B, int H, int T, int dk, int dv, int m, int chunk, int dtype);
int gsa_fwd(const void* q, const void* k, const void* v, const void* phi, const void* g,
            const float* h0_1, const float* h0_2, void* o, void* p_save, float* hT1, float* hT2,
            int B, int H, int T, int dk, int dv, int m, int chunk, int dtype, void* workspace,
            size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * gsa_bwd - gradients of L(o, hT1, hT2) for the inputs of gsa_fwd.
 *   in : as gsa_fwd, plus dO [B,H,T,dv]; dhT1 [B,H,dk,m], dhT2 [B,H,m,dv] fp32 (optional)
 *   out: dq, dk [B,H,T,dk]; dv [B,H,T,dv]; dphi, dg [B,H,T,m];
 *        dh0_1 [B,H,dk,m], dh0_2 [B,H,m,dv] fp32 (optional)
 * Pass 2 is differentiated first, then the softmax Jacobian do1 = p * (dp - <p, dp>), then
 * pass 1; dphi and dg sum the contributions of both passes.  The reverse mode of the two-pass
 * form of "Gated Slot Attention ...", "Approach" (two GLA passes sharing the per-slot forget
 * gates, joined by a softmax over the slots); each pass's gradient is that of a chunkwise GLA
 * ("MS-GLA", section 2.1).
 * ------------------------------------------------------------------------------------- */
size_t gsa_bwd_workspace(int B, int H, int T, int dk, int dv, int m, int chunk, int dtype);
int gsa_bwd(const void* q, const void* k, const void* v, const void* phi, const void* g,
            const float* h0_1, const float* h0_2, const void* dO, const float* dhT1,
            const float* dhT2, void* dq, void* dk, void* dv, void* dphi, void* dg, float* dh0_1,
            float* dh0_2, int B, int H, int T, int dk_dim, int dv_dim, int m, int chunk,
            int dtype, void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * gsa_recurrent_step - one token of GSA recurrent inference, in place on both states.
 *   in : q, k [B,H,dk]; v [B,H,dv]; phi, g [B,H,m];
 *        S1 [B,H,dk,m], S2 [B,H,m,dv] fp32 (read, then overwritten)
 *   out: o [B,H,dv]
 *   S1 <- S1 diag(exp g) + k^T phi ; p = softmax(q S1) ; S2 <- diag(exp g) S2 + phi^T v ;
 *   o = p S2.  "Gated Slot Attention ...", abstract (efficient recurrent inference with a
 *   small state).  No workspace.
 * ------------------------------------------------------------------------------------- */
int gsa_recurrent_step(const void* q, const void* k, const void* v, const void* phi,
                       const void* g, float* S1, float* S2, void* o, int B, int H, int dk,
                       int dv, int m, int dtype, void* stream);

/* ---------------------------------------------------------------------------------------
 * gla_chunk_bwd_noalloc - gla_chunk_bwd without a workspace argument, for callers that cannot
 * provide one.  (A library entry point only; the source pages have no counterpart of it.)
 *
 * Who needs it: callers that have no means to obtain device memory for a workspace, such as a
 * plain C host without a device allocator, a runtime that has carved up device memory in advance
 * and hands it out only for tensors, or code that must not call cudaMalloc because that call may
 * synchronise the device while its work is in flight.
 * What it uses instead: a fixed 128 MiB scratch array compiled into the library, reserved on
 * every device that loads this part of the library and held until the process exits.  The first
 * call on a device looks up that array's device address (cudaGetSymbolAddress); make the first
 * call on each device before any stream capture.  All calls share the array: calls that overlap
 * on the GPU (different streams or host threads) race on it.  Nothing in it needs to start at zero.
 * Arguments, layouts and outputs are those of gla_chunk_bwd.  Supported: bf16, chunk 64,
 * d_k = 128, d_v in {128, 256}, T >= 1 (else GLA_ERR_UNSUPPORTED / GLA_ERR_INVALID_ARG), and
 * scratch within the 128 MiB (else GLA_ERR_WORKSPACE): the bytes gla_chunk_bwd_workspace()
 * reports for the same sizes, (66 + d_v/2 + d_v/64)*B*H*ceil(T/64)*d_k*4 + nseg*B*H*d_k*4 +
 * 16640*B*H*ceil(T/64) (seven parts, each rounded up to 256 bytes), plus 2*nseg*B*H*d_k*d_v*4 +
 * nseg*B*H*d_k*4 when few heads leave SMs idle and the sequence is split into nseg segments.
 * It allocates nothing.
 * ------------------------------------------------------------------------------------- */
int gla_chunk_bwd_noalloc(const void* q, const void* k, const void* v, const void* g, const float* h0,
                          const void* dO, const float* dhT, void* dq, void* dk, void* dv, void* dg,
                          float* dh0, int B, int H, int T, int dk_dim, int dv_dim, int chunk, int dtype,
                          void* stream);

/* ---------------------------------------------------------------------------------------
 * gla_gate_logsigmoid - raw-logit gate entry: g = logsigmoid(x) / tau, element by element.
 * The operators take the log-gate g (alpha = exp g <= 1); models build it from a logit x as
 * log(sigmoid(x)) / tau ("MS-GLA ...", section 2.1: data-dependent forget gate; "Gated Slot
 * Attention ...", "Approach": sigmoid forget gates, alpha = sigmoid(x)^(1/tau)).
 *   x, g   n values of `dtype` (any layout; g may alias x).  tau > 0 and finite.
 * n == 0 enqueues nothing.  Errors: GLA_ERR_INVALID_ARG (NULL or misaligned pointer with
 * n > 0, tau not positive), GLA_ERR_UNSUPPORTED (dtype).  No workspace.
 * ------------------------------------------------------------------------------------- */
int gla_gate_logsigmoid(const void* x, void* g, size_t n, float tau, int dtype, void* stream);

/* gla_gate_logsigmoid_bwd - its backward: dx = dg * sigmoid(-x) / tau (dx may alias dg). */
int gla_gate_logsigmoid_bwd(const void* x, const void* dg, void* dx, size_t n, float tau, int dtype,
                            void* stream);

/* ---------------------------------------------------------------------------------------
 * MS-GLA temporal pooling and causal hold ("MS-GLA: Multi-Scale Gated Linear Attention ...",
 * sections 3.1 and 3.3), the reshaping around a GLA branch that runs at scale s.
 *   gla_msgla_pool       x [B,H,T,D] -> y [B,H,P,D], P = ceil(T/s): y_p is the mean of tokens
 *                        p*s .. min(T,(p+1)*s)-1 (a short last block averages only its tokens).
 *   gla_msgla_pool_bwd   dy [B,H,P,D] -> dx [B,H,T,D]: dx_t = dy_{t/s} / (tokens in block t/s).
 *   gla_msgla_hold       y [B,H,P,D] -> out [B,H,T,D]: out_t = y_{(t+1)/s - 1}, zeros while
 *                        (t+1)/s = 0 (a block is visible from its last token on).
 *   gla_msgla_hold_bwd   dout [B,H,T,D] -> dy [B,H,P,D]: the transpose (sum over the tokens that
 *                        read block p).
 * Arguments are (in, out, B, H, T, D, s, dtype, stream) for all four; in and out must not
 * overlap.  D in 8..512, a multiple of 8; s >= 1; T == 0 enqueues nothing.  Errors as for the
 * operators.  No workspace.
 * ------------------------------------------------------------------------------------- */
int gla_msgla_pool(const void* x, void* y, int B, int H, int T, int D, int s, int dtype, void* stream);
int gla_msgla_pool_bwd(const void* dy, void* dx, int B, int H, int T, int D, int s, int dtype, void* stream);
int gla_msgla_hold(const void* y, void* out, int B, int H, int T, int D, int s, int dtype, void* stream);
int gla_msgla_hold_bwd(const void* dout, void* dy, int B, int H, int T, int D, int s, int dtype,
                       void* stream);

/* ---------------------------------------------------------------------------------------
 * gla_device_error - read (and optionally clear) the device-side error latch.
 * Synchronises `stream`, then stores GLA_OK or the first error a kernel recorded since the
 * last reset (GLA_ERR_TIMEOUT: a bounded wait ran out) in *code.  Returns GLA_ERR_CUDA if
 * the copy fails, GLA_ERR_INVALID_ARG if code is NULL, else GLA_OK.
 * ------------------------------------------------------------------------------------- */
int gla_device_error(void* stream, int reset, int* code);

#ifdef __cplusplus
}
#endif

#endif /* GLA_B200_H */
