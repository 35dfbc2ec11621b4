// Fused sm_100a chunkwise GLA kernels (bf16 in, fp32 accumulate, chunk 64).
//
// Forward, one CTA per (head, 64 value columns, sequence segment); the CTA walks the chunks of its
// segment in order and keeps the recurrent state on chip ("MS-GLA ...", section 2.1: sequential inter-chunk
// updates, parallel intra-chunk work; "Gated Linear Attention for Efficient Long Sequences":
// chunking with on-chip reuse so that only inputs and outputs cross HBM).
//
// Per chunk of 64 tokens, with alpha_t = e^{g_t}, E1_j = prod_{t<=j} alpha_t = e^{B_j} and
// E2_j = prod_{t>j} alpha_t = e^{gamma - B_j} (B_j the inclusive cumulative log-gate of the chunk,
// gamma = B_63), everything is built from ONE exponential per (token, key dimension):
//
//   gate math (CUDA cores; each thread owns 2 adjacent key dimensions and a run of tokens):
//     Qs = q E1 / e^{gamma} = q e^{B - gamma}     Kh = k E2 = k e^{gamma - B}
//   tcgen05.mma (operands in shared memory, accumulators in TMEM):
//     A   = Qs Kh^T                   [64 x 64]   = sum_d q_jd k_rd e^{B_jd - B_rd}, masked to r <= j
//     O   = Qs (e^{gamma} S_i)        [64 x 64]   = (q e^{B}) S_i  (state copy pre-scaled by e^{gamma})
//     dS  = Kh^T V                    [dk x 64]
//     O  += A V
//   state (fp32 registers; a thread holds half a row d):   S_{i+1} = e^{gamma} S_i + dS
//
// Qs carries e^{B - gamma} <= e^{|gamma|}; it stays finite (and e^{gamma} S_i stays normal) while
// the chunk keeps at least e^-40 of its state in every key dimension.  A chunk below that bound
// (near-reset gates) switches to a safe form for that chunk: Qs = q e^{B} with an unscaled state
// copy, and the intra-chunk matrix recomputed exactly in fp32 from e^{B_j - B_r} (r <= j).
//
// Operand layouts are the 128-byte-swizzled forms described in sm100.cuh; V comes straight from a
// TMA tile load and serves as the MN-major B operand of two MMAs; Kh, stored [token][dim], is the
// K-major B operand of A and the MN-major A operand of dS.
//
// Sequence split.  When the (head, value tile) CTAs alone would leave most SMs idle (few heads, long
// sequences), the chunks are cut into nseg segments and the state recurrence is evaluated as an
// affine scan over them ("MS-GLA ...", section 2.1: the state update S <- diag(decay) S + dS is an
// affine map, so maps compose): (1) a state-only pass gives, per segment, the end state reached from
// zero (from h0 for the first segment) and the segment's decay product Gamma; (2) a scan
// S_in(s+1) = Gamma_s * S_in(s) + S_local(s) gives every segment's entry state; (3) the full kernel
// runs each segment from its entry state.  Nothing else changes: the per-chunk arithmetic of (3)
// is the one above, so the outputs differ from the unsplit run only by rounding.
#include "fast_path.cuh"
#include "fused_common.cuh"

namespace gla {
namespace fast {

using namespace sm100;

constexpr int DVT = 64;      // value columns per CTA
constexpr int NTHREADS = 256;  // warps w and w+4 share TMEM lanes and split accumulator columns

// ------------------------------------------------------------------------------------------
// Arguments of the forward passes
// ------------------------------------------------------------------------------------------
struct FwdArgs {
  const float* h0;     // [BH][DK][DV] or null (zeros); element strides st_bh (head), st_row (row)
  float* sbuf;         // [BH][nseg][DK][DV]: segment end states (state-only pass), then entry states
  float* gam;          // [BH][nseg][DK]: segment decay products
  __nv_bfloat16* o;
  float* hT;           // [BH][DK][DV] or null
  int T, DV, seg_chunks, nseg;
  long long st_bh, st_row;  // h0 / hT strides (a sub-block of a larger state when the shape is split)
  float* acc_o;             // optional fp32 output [BH*T][DV] in place of o (split shapes)
  const float* add_o;       // optional fp32 [BH*T][DV] added to o before it is stored (split shapes)
  int ck, cv;               // first column of the CTA's key block in q / k / g and of v (wider tensors)
  float inv_tau;            // > 0: the gate tensor holds raw logits x, g = logsigmoid(x) / tau
  unsigned int* latch;
};

// ------------------------------------------------------------------------------------------
// State-only pass of the sequence split: one CTA per (64 value columns, head, segment) runs the
// state recurrence alone (gates, Kh, dS = Kh^T V, S = e^{gamma} S + dS; no queries, no outputs)
// and writes the segment's end state and decay product.  Kh is finite for every gate (E2 <= 1),
// so this pass needs no exact path.
//
// REV: the same pass for the backward's state gradient G = dL/dS, which runs the other way:
// G_i = e^{gamma} G_{i+1} + Qt^T dO with Qt = q e^{B} (E1 <= 1, again finite for every gate).  Its
// CTAs take segments 1 .. nseg-1, walk their chunks last to first, start the last segment from
// dhT (args.h0) and write the G at each segment's start from its end G of zero (from dhT).
// HILO: the operand enters the MMA as a bf16 hi + lo pair (the backward's gate gradient takes
// sums several times larger than itself from these states).
// ------------------------------------------------------------------------------------------
template <int DK, bool HILO>
struct StateLayout {
  static constexpr uint32_t RAW = C * DK * 2;          // one raw k / g tile
  static constexpr uint32_t STAGE = 2 * RAW + C * DVT * 2;  // k, g, v
  static constexpr uint32_t KH = 2 * STAGE;            // Kh [64 x DK], MN-major A operand of dS (hi part)
  static constexpr uint32_t KH_LO = KH + C * DK * 2;   // its lo part (HILO)
  static constexpr uint32_t DECAY = KH + (HILO ? 2 : 1) * C * DK * 2;
  static constexpr uint32_t TOT = DECAY + DK * 4;
  static constexpr uint32_t TOTAL = TOT + GateRun<DK, NTHREADS>::NSPLIT * DK * 4;
  static_assert(TOT % 8 == 0 && DECAY % 8 == 0, "gate tables are read as float2");
  static constexpr uint32_t ALLOC = TOTAL + 1024;
  static_assert(STAGE % 1024 == 0 && RAW % 1024 == 0, "stage alignment");
};

template <int DK, bool HILO, bool REV, bool FLEX, bool LOGIT>
__global__ void __launch_bounds__(NTHREADS, 1)
    fwd_state_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_g,
                     const __grid_constant__ CUtensorMap tm_v, const FwdArgs args) {
  using L = StateLayout<DK, HILO>;
  using Gate = GateRun<DK, NTHREADS, LOGIT>;
  const int ck = FLEX ? args.ck : 0, cv = FLEX ? args.cv : 0;  // column offsets into wider tensors
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_load[2], bar_mma;
  __shared__ uint32_t tmem_base_sh;
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3, half = warp >> 2;
  const int dv0 = blockIdx.x * DVT, bh = blockIdx.y, seg = REV ? blockIdx.z + 1 : blockIdx.z;
  const int T = args.T, DV = args.DV, NC = (T + C - 1) / C;
  const int c_begin = seg * args.seg_chunks;
  const int c_end = min(NC, c_begin + args.seg_chunks);
  const int nloc = c_end - c_begin;
  float* decay_sm = reinterpret_cast<float*>(sm + L::DECAY);
  float* tot_sm = reinterpret_cast<float*>(sm + L::TOT);
  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, 64);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar_load[0], 1);
    mbar_init(&bar_load[1], 1);
    mbar_init(&bar_mma, 1);
    fence_mbar_init();
  }
  __syncthreads();
  auto issue_load = [&](int li) {
    const int s = li & 1, chunk = REV ? c_end - 1 - li : c_begin + li;
    uint8_t* st = sm + s * L::STAGE;
    mbar_arrive_expect_tx(&bar_load[s], L::STAGE);
    tma_load_3d(st, &tm_k, &bar_load[s], ck, chunk * C, bh);
    tma_load_3d(st + L::RAW, &tm_g, &bar_load[s], ck, chunk * C, bh);
    tma_load_3d(st + 2 * L::RAW, &tm_v, &bar_load[s], cv + dv0, chunk * C, bh);
  };
  if (tid == 0) {
    issue_load(0);
    if (nloc > 1) issue_load(1);
  }
  constexpr int SW = DVT / 2;
  const bool s_owner = (DK == 128) ? true : (lane < 16);
  const int s_row = (DK == 128) ? (q4 * 32 + lane) : (q4 * 16 + lane);
  const int sc0 = half * SW;
  float S[SW];
#pragma unroll
  for (int c = 0; c < SW; ++c) S[c] = 0.f;
  if (seg == (REV ? args.nseg - 1 : 0) && s_owner && args.h0) {
    const float4* src = reinterpret_cast<const float4*>(args.h0 + bh * args.st_bh + s_row * args.st_row + dv0 + sc0);
#pragma unroll
    for (int c = 0; c < SW / 4; ++c) {
      const float4 x = src[c];
      S[4 * c] = x.x;
      S[4 * c + 1] = x.y;
      S[4 * c + 2] = x.z;
      S[4 * c + 3] = x.w;
    }
  }
  float gamma_acc = 1.f;  // decay product of the segment for row s_row
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t t_dS = tmem_base_sh;
  const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
  for (int li = 0; li < nloc; ++li) {
    const int s = li & 1;
    uint8_t* st = sm + s * L::STAGE;
    mbar_wait(&bar_load[s], (li >> 1) & 1, args.latch);
    Gate gr;
    gr.set_logit(args.inv_tau, T - (REV ? c_end - 1 - li : c_begin + li) * C);
    gr.run(st + L::RAW, DK, tot_sm);
    if (gr.h == 0) gr.store_decay(decay_sm);
    {
      const uint32_t blk = (gr.d >> 6) * (C * 128), col = gr.d & 63;
      uint32_t w[Gate::TS];
      gr.load_pairs(st, DK, false, w);
      auto put = [&](int j, float e0, float e1) {  // Kh = k E2, or Qt = q E1 (REV)
        const uint32_t wk = w[j - gr.h * Gate::TS];
        if (HILO) {
          uint32_t hi, lo;
          split2(bf_lo(wk) * e0, bf_hi(wk) * e1, hi, lo);
          *reinterpret_cast<uint32_t*>(sm + L::KH + blk + sw128(j, col)) = hi;
          *reinterpret_cast<uint32_t*>(sm + L::KH_LO + blk + sw128(j, col)) = lo;
        } else {
          *reinterpret_cast<uint32_t*>(sm + L::KH + blk + sw128(j, col)) = pack2(bf_lo(wk) * e0, bf_hi(wk) * e1);
        }
      };
      if (REV)
        gr.forward(put);
      else
        gr.backward(put);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      const uint32_t base = smem_u32(sm);
      const uint32_t vbase = base + s * L::STAGE + 2 * L::RAW;
      constexpr uint32_t id_S = idesc_bf16_f32(DK, DVT, true, true);
#pragma unroll
      for (int k = 0; k < C / 16; ++k) {
        const uint64_t vd = desc_sw128(vbase + k * 2048, 16, 1024);
        umma_bf16(t_dS, desc_sw128(base + L::KH + k * 2048, C * 128, 1024), vd, id_S, k > 0);
        if (HILO) umma_bf16(t_dS, desc_sw128(base + L::KH_LO + k * 2048, C * 128, 1024), vd, id_S, 1);
      }
      umma_commit(&bar_mma);
    }
    __syncwarp();
    mbar_wait(&bar_mma, li & 1, args.latch);
    tc_fence_after();
    float ds[SW];
    tmem_ld32(t_dS + lane_off + sc0, ds);
    tmem_ld_wait();
    if (s_owner) {
      const float dec = decay_sm[s_row];
      gamma_acc *= dec;
#pragma unroll
      for (int c = 0; c < SW; ++c) S[c] = dec * S[c] + ds[c];
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && li + 2 < nloc) issue_load(li + 2);
  }
  float* out = args.sbuf + ((size_t)bh * args.nseg + (REV ? seg - 1 : seg)) * DK * DV;
  if (s_owner) {
    float4* dst = reinterpret_cast<float4*>(out + (size_t)s_row * DV + dv0 + sc0);
#pragma unroll
    for (int c = 0; c < SW / 4; ++c) dst[c] = make_float4(S[4 * c], S[4 * c + 1], S[4 * c + 2], S[4 * c + 3]);
    if (!REV && half == 0 && blockIdx.x == 0) args.gam[((size_t)bh * args.nseg + seg) * DK + s_row] = gamma_acc;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(t_dS, 64);
}

// ------------------------------------------------------------------------------------------
// Pipelined forward (the full pass).  Per chunk i the two MMA groups run while the CTA works on
// its neighbours.  Group 1 is A = Qs Kh^T and dS = Kh^T V (first commit), then O_i = Qs S'
// (second commit).  During group 1 the threads store the outputs of chunk i-1; once A and dS are
// done they form A's operand and update the state while the O MMAs still run, hand A over for
// group 2 (O_i += A V), and run the gate math of chunk i+1 into registers; once group 1 is done
// they store chunk i+1's operands (Qs, Kh, the scaled state copy) and group 1 of chunk i+1 is
// issued right behind group 2.  O is double-buffered in TMEM; q/k/g come through a
// two-stage ring and v through a three-deep ring, so a raw tile is free as soon as its own
// chunk's math is done.  MMAs issued by one thread complete in order, so waiting for group 1 of
// chunk i+1 also covers group 2 of chunk i.
//
// A ninth warp issues the TMA loads and the MMAs.  tcgen05.mma issue proceeds at the rate the
// tensor pipe executes (about 48 cycles per 64-wide MMA), so the issuing thread is held for a
// group's whole duration; in its own warp it holds up no other work.  The 256 compute threads
// hand over with named barriers: they arrive at kBarOps once a chunk's group-1 operands are in
// shared memory and at kBarAB once its A operand is, and the producer waits at both.
// ------------------------------------------------------------------------------------------
template <int DK, bool KHILO = false>
struct FwdPipeLayout {
  static constexpr uint32_t RAW = C * DK * 2;               // one raw q / k / g tile
  static constexpr uint32_t QKG = 3 * RAW;                  // a q/k/g stage (two stages)
  static constexpr uint32_t VTB = C * DVT * 2;              // a v tile (three buffers)
  static constexpr uint32_t V0 = 2 * QKG;
  static constexpr uint32_t QS_HI = V0 + 3 * VTB;           // Qs hi / lo [64 x DK]  K-major
  static constexpr uint32_t QS_LO = QS_HI + C * DK * 2;
  static constexpr uint32_t KH = QS_LO + C * DK * 2;        // Kh [64 x DK]  K-major B / MN-major A
  static constexpr uint32_t KH_LO = KH + C * DK * 2;        // its lo part (KHILO builds)
  static constexpr uint32_t SB_HI = KH_LO + (KHILO ? C * DK * 2 : 0);  // scaled state copy hi / lo [DK x 64]
  static constexpr uint32_t SB_LO = SB_HI + DK * DVT * 2;
  static constexpr uint32_t AB_HI = SB_LO + DK * DVT * 2;   // A hi / lo [64 x 64] K-major
  static constexpr uint32_t AB_LO = AB_HI + C * C * 2;
  static constexpr uint32_t DECAY = AB_LO + C * C * 2;      // float[2][DK]: e^{gamma_d} per chunk parity
  static constexpr int NS = GateRun<DK, NTHREADS>::NSPLIT;
  static constexpr uint32_t TOT = DECAY + 2 * DK * 4;       // float[NS][DK] run products
  static constexpr uint32_t TOTAL = TOT + NS * DK * 4;
  static_assert(TOT % 8 == 0 && DECAY % 8 == 0, "gate tables are read as float2");
  static constexpr uint32_t ALLOC = TOTAL + 1024;
  // Exact-path scratch during the A epilogue of a chunk (its Qs / Kh are consumed by then, the
  // next chunk's are still in registers): cumulative log-gates over QS_HI.., exact A over KH..
  static constexpr uint32_t XB = QS_HI, XA = KH;
  static_assert(QKG % 1024 == 0 && VTB % 1024 == 0 && QS_HI % 1024 == 0, "alignment");
  static_assert(ALLOC <= 227 * 1024, "shared memory");
  static_assert(C * DK * 4 <= KH - QS_HI && C * C * 4 <= SB_LO - KH, "exact-path scratch");
};

constexpr int PIPE_THREADS = NTHREADS + 32;  // 8 compute warps + the producer warp
constexpr int kBarOps = 2, kBarAB = 3;       // compute threads -> producer handoffs

// FLEX: the build for wider tensors (column offsets, fp32 partial outputs with an added partial) and
// raw-logit gates; the plain build has none of that code.  KHILO: Kh enters the MMAs as a bf16
// hi + lo pair as well (for a caller whose output needs it, at the price of three more MMAs per
// 16 keys in A and one more per 16 tokens in dS).
template <int DK, bool FLEX, bool KHILO, bool LOGIT>
__global__ void __launch_bounds__(PIPE_THREADS, 1)
    fwd_pipe_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_v,
                    const FwdArgs args) {
  using L = FwdPipeLayout<DK, KHILO>;
  using Gate = GateRun<DK, NTHREADS, LOGIT>;
  const int ck = FLEX ? args.ck : 0, cv = FLEX ? args.cv : 0;  // column offsets into wider tensors
  constexpr int TS = Gate::TS;
  constexpr int NHAND = NTHREADS + 32;  // threads taking part in a handoff barrier
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_qkg[2], bar_v[3], bar_mmaA, bar_mma1, bar_mma2;
  __shared__ uint32_t tmem_base_sh;
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const uint32_t base = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3, half = (warp >> 2) & 1;  // TMEM lane quarter, column half
  const int dv0 = blockIdx.x * DVT, bh = blockIdx.y, seg = blockIdx.z;
  const int T = args.T, DV = args.DV, NC = (T + C - 1) / C;
  const int c_begin = seg * args.seg_chunks;
  const int nloc = min(NC, c_begin + args.seg_chunks) - c_begin;
  unsigned int* latch = args.latch;
  float* decay_sm = reinterpret_cast<float*>(sm + L::DECAY);
  float* tot_sm = reinterpret_cast<float*>(sm + L::TOT);

  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, 256);
    tmem_relinquish();
  }
  if (tid == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_g);
    prefetch_tmap(&tm_v);
    for (int b = 0; b < 2; ++b) mbar_init(&bar_qkg[b], 1);
    for (int b = 0; b < 3; ++b) mbar_init(&bar_v[b], 1);
    mbar_init(&bar_mmaA, 1);
    mbar_init(&bar_mma1, 1);
    mbar_init(&bar_mma2, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t t_A = tmem, t_O0 = tmem + 64, t_dS = tmem + 192;
  const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;

  if (warp == NTHREADS / 32) {
    // ------------------------------ producer warp ------------------------------
    auto load_qkg = [&](int li) {
      const int s = li & 1, chunk = c_begin + li;
      uint8_t* st = sm + s * L::QKG;
      mbar_arrive_expect_tx(&bar_qkg[s], L::QKG);
      tma_load_3d(st, &tm_q, &bar_qkg[s], ck, chunk * C, bh);
      tma_load_3d(st + L::RAW, &tm_k, &bar_qkg[s], ck, chunk * C, bh);
      tma_load_3d(st + 2 * L::RAW, &tm_g, &bar_qkg[s], ck, chunk * C, bh);
    };
    auto load_v = [&](int li) {
      const int b = li % 3;
      mbar_arrive_expect_tx(&bar_v[b], L::VTB);
      tma_load_3d(sm + L::V0 + b * L::VTB, &tm_v, &bar_v[b], cv + dv0, (c_begin + li) * C, bh);
    };
    if (lane == 0) {
      load_qkg(0);
      load_v(0);
      if (nloc > 1) {
        load_qkg(1);
        load_v(1);
      }
      if (nloc > 2) load_v(2);
    }
    for (int li = 0; li < nloc; ++li) {
      bar_sync(kBarOps, NHAND);  // chunk li's Qs, Kh and state copy are in shared memory
      if (lane == 0) {
        // group 1: A = Qs Kh^T and dS = Kh^T V (first commit: the A epilogue and the state update
        // need only these), then O_li = Qs S' (second commit)
        mbar_wait(&bar_v[li % 3], (li / 3) & 1, latch);
        tc_fence_after();
        const uint32_t vbase = base + L::V0 + (li % 3) * L::VTB;
        const uint32_t t_O = t_O0 + (li & 1) * 64;
        constexpr uint32_t id_A = idesc_bf16_f32(C, C, false, false);
        constexpr uint32_t id_O = idesc_bf16_f32(C, DVT, false, true);
        constexpr uint32_t id_S = idesc_bf16_f32(DK, DVT, true, true);
#pragma unroll
        for (int k = 0; k < DK / 16; ++k) {
          const uint32_t koff = (k >> 2) * (C * 128) + (k & 3) * 32;
          const uint64_t kd = desc_sw128(base + L::KH + koff, 16, 1024);
          const uint64_t qh_d = desc_sw128(base + L::QS_HI + koff, 16, 1024);
          const uint64_t ql_d = desc_sw128(base + L::QS_LO + koff, 16, 1024);
          umma_bf16(t_A, qh_d, kd, id_A, k > 0);
          umma_bf16(t_A, ql_d, kd, id_A, 1);
          if (KHILO) umma_bf16(t_A, qh_d, desc_sw128(base + L::KH_LO + koff, 16, 1024), id_A, 1);
        }
#pragma unroll
        for (int k = 0; k < C / 16; ++k) {
          const uint64_t vd = desc_sw128(vbase + k * 2048, 16, 1024);
          umma_bf16(t_dS, desc_sw128(base + L::KH + k * 2048, C * 128, 1024), vd, id_S, k > 0);
          if (KHILO) umma_bf16(t_dS, desc_sw128(base + L::KH_LO + k * 2048, C * 128, 1024), vd, id_S, 1);
        }
        umma_commit(&bar_mmaA);
#pragma unroll
        for (int k = 0; k < DK / 16; ++k) {
          const uint32_t koff = (k >> 2) * (C * 128) + (k & 3) * 32;
          const uint64_t qh_d = desc_sw128(base + L::QS_HI + koff, 16, 1024);
          const uint64_t sh = desc_sw128(base + L::SB_HI + k * 2048, 16, 1024);
          umma_bf16(t_O, qh_d, sh, id_O, k > 0);
          umma_bf16(t_O, qh_d, desc_sw128(base + L::SB_LO + k * 2048, 16, 1024), id_O, 1);
          umma_bf16(t_O, desc_sw128(base + L::QS_LO + koff, 16, 1024), sh, id_O, 1);
        }
        umma_commit(&bar_mma1);
      }
      bar_sync(kBarAB, NHAND);  // chunk li's A operand is in shared memory; its raw tiles are free
      if (lane == 0) {
        // group 2: O_li += A V
        tc_fence_after();
        const uint32_t vbase = base + L::V0 + (li % 3) * L::VTB;
        const uint32_t t_O = t_O0 + (li & 1) * 64;
        constexpr uint32_t id_O = idesc_bf16_f32(C, DVT, false, true);
#pragma unroll
        for (int k = 0; k < C / 16; ++k) {
          const uint64_t vd = desc_sw128(vbase + k * 2048, 16, 1024);
          umma_bf16(t_O, desc_sw128(base + L::AB_HI + k * 32, 16, 1024), vd, id_O, 1);
          umma_bf16(t_O, desc_sw128(base + L::AB_LO + k * 32, 16, 1024), vd, id_O, 1);
        }
        umma_commit(&bar_mma2);
        if (li + 2 < nloc) {
          load_qkg(li + 2);
          if (li >= 1) {
            // The v buffer of chunk li+2 held chunk li-1's v, read by its group 2.  Group 1 of
            // chunk li was issued after that group 2 and MMAs complete in order, so its completion
            // frees the buffer.  (A parity wait on group 2's barrier could be two phases behind
            // here, since group 2 of chunk li may already have completed; group 1 of chunk li+1
            // has not been issued yet, so this wait is at most one phase behind.)
            mbar_wait(&bar_mma1, li & 1, latch);
            load_v(li + 2);
          }
        }
      }
      __syncwarp();
    }
  } else {
    // ------------------------------ compute warps ------------------------------
    // State owned by this thread: row s_row (lane layout of the dS accumulator, M = DK), columns
    // sc0 .. sc0+31 of the CTA's 64.
    constexpr int SW = DVT / 2;
    const bool s_owner = (DK == 128) ? true : (lane < 16);
    const int s_row = (DK == 128) ? (q4 * 32 + lane) : (q4 * 16 + lane);
    const int sc0 = half * SW;
    float S[SW];
#pragma unroll
    for (int c = 0; c < SW; ++c) S[c] = 0.f;
    const float* init = seg == 0 ? (args.h0 ? args.h0 + bh * args.st_bh : nullptr)
                                 : args.sbuf + ((size_t)bh * args.nseg + seg - 1) * DK * DV;
    const long long ipitch = seg == 0 ? args.st_row : DV;
    if (s_owner && init) {
      const float4* src = reinterpret_cast<const float4*>(init + s_row * ipitch + dv0 + sc0);
#pragma unroll
      for (int c = 0; c < SW / 4; ++c) {
        const float4 x = src[c];
        S[4 * c] = x.x;
        S[4 * c + 1] = x.y;
        S[4 * c + 2] = x.z;
        S[4 * c + 3] = x.w;
      }
    }

    // Gate math of local chunk li (stage li & 1) into registers: Qs hi / lo and Kh for the two
    // dims gd, gd+1 and the tokens gh*TS .. gh*TS+TS-1 owned by this thread.  Returns the chunk's
    // exact-path flag (CTA-uniform).
    uint32_t qh[TS], ql[TS], kh[TS], kl[KHILO ? TS : 1];
    int gd = 0, gh = 0;
    auto gate_regs = [&](int li) {
      const uint8_t* st = sm + (li & 1) * L::QKG;
      Gate gr;
      gr.set_logit(args.inv_tau, T - (c_begin + li) * C);
      const bool weak = gr.run(st + 2 * L::RAW, DK, tot_sm);
      float* dec = decay_sm + (li & 1) * DK;
      if (gr.h == 0) gr.store_decay(dec);
      const int safe = bar_or(kBarCompute, NTHREADS, weak);
      gd = gr.d;
      gh = gr.h;
      float e0 = gr.pre0 * (safe ? 1.f : 1.f / gr.dec0), e1 = gr.pre1 * (safe ? 1.f : 1.f / gr.dec1);
#pragma unroll
      for (int u = 0; u < TS; ++u) {
        e0 *= gr.a0[u];
        e1 *= gr.a1[u];
        const uint32_t wq = *reinterpret_cast<const uint32_t*>(st + ((gh * TS + u) * DK + gd) * 2);
        split2(bf_lo(wq) * e0, bf_hi(wq) * e1, qh[u], ql[u]);
      }
      float f0 = gr.suf0, f1 = gr.suf1;
#pragma unroll
      for (int u = TS - 1; u >= 0; --u) {
        const uint32_t wk = *reinterpret_cast<const uint32_t*>(st + L::RAW + ((gh * TS + u) * DK + gd) * 2);
        if (KHILO)
          split2(bf_lo(wk) * f0, bf_hi(wk) * f1, kh[u], kl[KHILO ? u : 0]);
        else
          kh[u] = pack2(bf_lo(wk) * f0, bf_hi(wk) * f1);
        f0 *= gr.a0[u];
        f1 *= gr.a1[u];
      }
      return safe;
    };
    // Operands of local chunk li into shared memory (Qs, Kh from registers; the state copy), then
    // hand them to the producer.
    auto store_ops = [&](int li, int safe) {
      const uint32_t blk = (gd >> 6) * (C * 128), col = gd & 63;
#pragma unroll
      for (int u = 0; u < TS; ++u) {
        const uint32_t off = blk + sw128(gh * TS + u, col);
        *reinterpret_cast<uint32_t*>(sm + L::QS_HI + off) = qh[u];
        *reinterpret_cast<uint32_t*>(sm + L::QS_LO + off) = ql[u];
        *reinterpret_cast<uint32_t*>(sm + L::KH + off) = kh[u];
        if (KHILO) *reinterpret_cast<uint32_t*>(sm + L::KH_LO + off) = kl[KHILO ? u : 0];
      }
      if (s_owner) {
        const float sc = safe ? 1.f : decay_sm[(li & 1) * DK + s_row];
        float sv[SW];
#pragma unroll
        for (int c = 0; c < SW; ++c) sv[c] = S[c] * sc;
        store_half_split(sm + L::SB_HI, sm + L::SB_LO, s_row, sv, half);
      }
      fence_async_smem();
      tc_fence_before();
      bar_arrive(kBarOps, NHAND);
    };
    // O rows of local chunk li (after its group 2): bf16 straight to global.  The tile is read with
    // the 16-lane TMEM shape, so each thread holds two rows x four column pairs and a warp's access
    // covers 8 rows x 32 contiguous bytes (fp32) instead of 16 rows x 16 bytes.
    const int cb_o = half * 32, r0_o = q4 * 16 + (lane >> 2), cq_o = 2 * (lane & 3);
    // The partial output of earlier key blocks for chunk li's rows as this thread adds them (see
    // store_o), loaded a whole chunk step before it is used.
    auto load_add = [&](int li, float2 (&ad)[8]) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int t = (c_begin + li) * C + r0_o + 8 * h;
        const size_t off = ((size_t)bh * T + (t < T ? t : 0)) * DV + dv0 + cb_o + cq_o;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          ad[4 * h + k] = t < T ? *reinterpret_cast<const float2*>(args.add_o + off + 8 * k) : make_float2(0.f, 0.f);
      }
    };
    auto store_o = [&](int li, const float2 (&ad)[8]) {
      mbar_wait(&bar_mma2, li & 1, latch);
      tc_fence_after();
      const int cb = cb_o, r0 = r0_o, cq = cq_o;
      float ov[16];  // register 4k + 2h + e: row r0 + 8h, column cb + 8k + cq + e
      tmem_ld16x32(t_O0 + (li & 1) * 64 + lane_off + cb, ov);
      tmem_ld_wait();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int t = (c_begin + li) * C + r0 + 8 * h;
        if (t >= T) continue;
        const size_t off = ((size_t)bh * T + t) * DV + dv0 + cb + cq;
        float2 o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) o[k] = make_float2(ov[4 * k + 2 * h], ov[4 * k + 2 * h + 1]);
        if (FLEX && args.add_o) {  // a partial output of earlier key blocks
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            o[k].x += ad[4 * h + k].x;
            o[k].y += ad[4 * h + k].y;
          }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (FLEX && args.acc_o)
            *reinterpret_cast<float2*>(args.acc_o + off + 8 * k) = o[k];
          else
            *reinterpret_cast<__nv_bfloat162*>(args.o + off + 8 * k) = __floats2bfloat162_rn(o[k].x, o[k].y);
        }
      }
    };

    mbar_wait(&bar_qkg[0], 0, latch);
    int safe = gate_regs(0);
    store_ops(0, safe);
    float2 ad_cur[8], ad_next[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) ad_cur[k] = ad_next[k] = make_float2(0.f, 0.f);
    for (int li = 0; li < nloc; ++li) {
      const uint8_t* st = sm + (li & 1) * L::QKG;
      if (FLEX && args.add_o) load_add(li, ad_next);  // used by store_o(li), one step later
      // ---- while group 1 of chunk li runs: outputs of chunk li-1 ----
      if (li > 0) store_o(li - 1, ad_cur);
      // ---- A and dS done (O may still run): exact A if needed, A epilogue, state update ----
      mbar_wait(&bar_mmaA, li & 1, latch);
      // the exact path's scratch lies over Qs and Kh, which the O MMAs read
      if (safe) mbar_wait(&bar_mma1, li & 1, latch);
      tc_fence_after();
      float* Aex = reinterpret_cast<float*>(sm + L::XA);
      if (safe) {
        float* Bf = reinterpret_cast<float*>(sm + L::XB);
        if (tid < DK) {
          float b = 0.f;
          for (int j = 0; j < C; ++j) {
            b += bf2f(st + 2 * L::RAW + (j * DK + tid) * 2);
            Bf[j * DK + tid] = b;
          }
        }
        bar_sync(kBarCompute, NTHREADS);
        for (int e = tid; e < C * C; e += NTHREADS) {
          const int j = e / C, r = e % C;
          float acc = 0.f;
          if (r <= j)
            for (int d = 0; d < DK; ++d)
              acc += bf2f(st + (j * DK + d) * 2) * bf2f(st + L::RAW + (r * DK + d) * 2) *
                     __expf(Bf[j * DK + d] - Bf[r * DK + d]);
          Aex[e] = acc;
        }
        bar_sync(kBarCompute, NTHREADS);
      }
      {
        const int j = q4 * 16 + lane, cb = half * 32;
        float a[32];
        tmem_ld32(t_A + lane_off + cb, a);
        tmem_ld_wait();
        if (lane < 16) {
          if (safe) {
#pragma unroll
            for (int c = 0; c < 32; ++c) a[c] = Aex[j * C + cb + c];
          }
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (cb + c > j) a[c] = 0.f;
          store_half_split(sm + L::AB_HI, sm + L::AB_LO, j, a, half);
        }
        float ds[SW];
        tmem_ld32(t_dS + lane_off + sc0, ds);
        tmem_ld_wait();
        if (s_owner) {
          const float dec = decay_sm[(li & 1) * DK + s_row];
#pragma unroll
          for (int c = 0; c < SW; ++c) S[c] = dec * S[c] + ds[c];
        }
      }
      fence_async_smem();
      tc_fence_before();
      bar_arrive(kBarAB, NHAND);
      // ---- while the O MMAs and group 2 of chunk li run: gate math of chunk li+1 ----
      int safe_next = 0;
      if (li + 1 < nloc) {
        mbar_wait(&bar_qkg[(li + 1) & 1], ((li + 1) >> 1) & 1, latch);
        safe_next = gate_regs(li + 1);
      }
      // ---- group 1 done (O read Qs and the state copy): operands of chunk li+1 (group 1 follows) ----
      if (!safe) {
        mbar_wait(&bar_mma1, li & 1, latch);
        tc_fence_after();
      }
      // Exact-path scratch over Qs / Kh: every compute thread has finished with it before any
      // thread stores chunk li+1's operands.
      if (safe) bar_sync(kBarCompute, NTHREADS);
      if (li + 1 < nloc) store_ops(li + 1, safe_next);
      safe = safe_next;
#pragma unroll
      for (int k = 0; k < 8; ++k) ad_cur[k] = ad_next[k];
    }
    store_o(nloc - 1, ad_cur);

    float* out = (seg == args.nseg - 1 && args.hT) ? args.hT + bh * args.st_bh : nullptr;
    if (s_owner && out) {
      float4* dst = reinterpret_cast<float4*>(out + s_row * args.st_row + dv0 + sc0);
#pragma unroll
      for (int c = 0; c < SW / 4; ++c) dst[c] = make_float4(S[4 * c], S[4 * c + 1], S[4 * c + 2], S[4 * c + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

// ------------------------------------------------------------------------------------------
// Host entry points
// ------------------------------------------------------------------------------------------
bool fwd_supported(int BH, int T, int dk, int dv, int chunk, int dtype) {
  if (dtype != 1 || chunk != C || T < 1 || BH < 1 || BH > 65535) return false;
  if (dk != 64 && dk != 128) return false;
  if (dv % DVT != 0) return false;
  return encode_fn() != nullptr;
}

// Entry states of segments 1 .. nseg-1, in place: entry s-1 of sbuf holds S_local(s-1) on input and
// the state entering segment s on output, S_in(s) = Gamma_{s-1} * S_in(s-1) + S_local(s-1) per row.
__global__ void segment_scan_kernel(float* __restrict__ sbuf, const float* __restrict__ gam, int BH, int DK, int DV,
                                    int nseg) {
  const size_t per = (size_t)DK * DV, n = (size_t)BH * per;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
    const size_t bh = e / per, rem = e % per;
    const int d = (int)(rem / DV);
    float* p = sbuf + bh * nseg * per + rem;
    float acc = p[0];
    for (int sg = 1; sg < nseg - 1; ++sg) {
      acc = gam[(bh * nseg + sg) * DK + d] * acc + p[sg * per];
      p[sg * per] = acc;
    }
  }
}

cudaError_t side_stream(int pool, SideStream** out) {
  static std::mutex make_mu;
  static SideStream per_dev[2][64];
  static bool made[2][64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || pool < 0 || pool > 1) return cudaErrorInvalidValue;
  std::lock_guard<std::mutex> g(make_mu);
  SideStream& x = per_dev[pool][dev];
  if (!made[pool][dev]) {
    if ((e = cudaStreamCreateWithFlags(&x.s, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&x.fork, cudaEventDisableTiming)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&x.join, cudaEventDisableTiming)) != cudaSuccess) return e;
    made[pool][dev] = true;
  }
  *out = &x;
  return cudaSuccess;
}

int sm_count() {
  static std::atomic<int> cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (!n) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// Segments of the sequence split: as many as fill the SMs once with (head, value tile, segment)
// CTAs; 1 (no split) when the heads alone fill at least half of them.
static void plan_segments(int BH, int T, int dv, int* nseg, int* seg_chunks) {
  const int NC = (T + C - 1) / C, base = BH * (dv / DVT), sms = sm_count();
  int n = 1;
  if (2 * base <= sms) n = sms / base;
  if (n > NC) n = NC;
  if (n < 1) n = 1;
  const int per = (NC + n - 1) / n;
  *seg_chunks = per;
  *nseg = (NC + per - 1) / per;
}

size_t fwd_workspace(int BH, int T, int dk, int dv) {
  int nseg, per;
  plan_segments(BH, T, dv, &nseg, &per);
  if (nseg == 1) return 0;
  return align256((size_t)BH * nseg * dk * dv * sizeof(float)) + align256((size_t)BH * nseg * dk * sizeof(float));
}

// m: maps of the operand ([64 x DK] rows), the gates, and the 64-column value tiles.
template <int DK, bool HILO, bool REV, bool FLEX>
static cudaError_t launch_state_pass(const CUtensorMap& mk, const CUtensorMap& mg, const CUtensorMap& mv,
                                     const FwdArgs& args, int BH, int dv, cudaStream_t st) {
  // raw-logit gates only in a build of their own
  auto kern = args.inv_tau > 0.f ? fwd_state_kernel<DK, HILO, REV, FLEX, FLEX>
                                 : fwd_state_kernel<DK, HILO, REV, FLEX, false>;
  static std::atomic<bool> attr_set[2][64] = {};
  const cudaError_t e = ensure_smem_attr(kern, StateLayout<DK, HILO>::ALLOC, attr_set[args.inv_tau > 0.f ? 1 : 0]);
  if (e != cudaSuccess) return e;
  dim3 grid(dv / DVT, BH, args.nseg - 1);
  kern<<<grid, NTHREADS, StateLayout<DK, HILO>::ALLOC, st>>>(mk, mg, mv, args);
  return cudaGetLastError();
}

template <int DK>
static cudaError_t launch_fwd(const void* q, const void* k, const void* v, const void* g, const float* h0, void* o,
                              float* hT, int BH, int T, int dv, long long st_bh, long long st_row, float* acc_o,
                              void* ws, cudaStream_t st, float inv_tau, int dk_total, int k0, const float* add_o,
                              bool kh_hilo, int phase) {
  CUtensorMap m[4];
  if (!make_map(&m[0], q, BH, T, dk_total, DK, false) || !make_map(&m[1], k, BH, T, dk_total, DK, false) ||
      !make_map(&m[2], g, BH, T, dk_total, DK, false) || !make_map(&m[3], v, BH, T, dv, DVT, true))
    return cudaErrorInvalidValue;
  FwdArgs a;
  a.h0 = h0;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.hT = hT;
  a.T = T;
  a.DV = dv;
  a.st_bh = st_bh;
  a.st_row = st_row;
  a.acc_o = acc_o;
  a.add_o = add_o;
  a.ck = k0;
  a.cv = 0;
  a.inv_tau = inv_tau;
  a.latch = device_error_latch();
  const bool flex = inv_tau > 0.f || acc_o || add_o || k0 != 0 || dk_total != DK || kh_hilo;
  plan_segments(BH, T, dv, &a.nseg, &a.seg_chunks);
  a.sbuf = nullptr;
  a.gam = nullptr;
  if (a.nseg > 1) {
    if (!ws) return cudaErrorInvalidValue;
    a.sbuf = static_cast<float*>(ws);
    a.gam = a.sbuf + align256((size_t)BH * a.nseg * DK * dv * sizeof(float)) / sizeof(float);
  }
  if (a.nseg > 1 && phase != kFwdWalk) {
    cudaError_t e = kh_hilo ? launch_state_pass<DK, true, false, true>(m[1], m[2], m[3], a, BH, dv, st)
                    : flex  ? launch_state_pass<DK, false, false, true>(m[1], m[2], m[3], a, BH, dv, st)
                            : launch_state_pass<DK, false, false, false>(m[1], m[2], m[3], a, BH, dv, st);
    if (e != cudaSuccess) return e;
    if (a.nseg > 2) {
      const size_t n = (size_t)BH * DK * dv;
      const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
      segment_scan_kernel<<<blocks, 256, 0, st>>>(a.sbuf, a.gam, BH, DK, dv, a.nseg);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
  }
  if (phase == kFwdStates) return cudaSuccess;
  // the split-Kh build exists for d_k = 64 only (its extra operand does not fit next to d_k = 128)
  const bool logit = inv_tau > 0.f;
  auto kern = kh_hilo ? fwd_pipe_kernel<DK, true, DK == 64, false>
              : logit ? fwd_pipe_kernel<DK, true, false, true>
              : flex  ? fwd_pipe_kernel<DK, true, false, false>
                      : fwd_pipe_kernel<DK, false, false, false>;
  const uint32_t alloc = kh_hilo ? FwdPipeLayout<DK, DK == 64>::ALLOC : FwdPipeLayout<DK>::ALLOC;
  static std::atomic<bool> attr_set[4][64] = {};
  {
    const cudaError_t e = ensure_smem_attr(kern, alloc, attr_set[kh_hilo ? 3 : logit ? 2 : flex ? 1 : 0]);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(dv / DVT, BH, a.nseg);
  kern<<<grid, PIPE_THREADS, alloc, st>>>(m[0], m[1], m[2], m[3], a);
  return cudaGetLastError();
}

// Segments of the backward's sequence split: as many as fill the SMs once when each segment takes
// ctas_per_seg CTAs of the backward's first launch; 1 when those alone fill half of the SMs.
void plan_bwd_segments(int ctas_per_seg, int T, int* nseg, int* seg_chunks) {
  const int NC = (T + C - 1) / C, sms = sm_count();
  int n = 1;
  if (2 * ctas_per_seg <= sms) n = sms / ctas_per_seg;
  if (n > NC) n = NC;
  if (n < 1) n = 1;
  const int per = (NC + n - 1) / n;
  *seg_chunks = per;
  *nseg = (NC + per - 1) / per;
}

// End gradients of segments nseg-3 .. 0, in place: entry s of gbuf holds the gradient at the start
// of segment s+1 reached from a zero end gradient (from dhT for the last segment) on input, and
// the gradient at the end of segment s on output: G_end(s) = Gamma_{s+1} * G_end(s+1) + entry s.
__global__ void segment_scan_rev_kernel(float* __restrict__ gbuf, const float* __restrict__ gam, int BH, int DK,
                                        int DV, int nseg) {
  const size_t per = (size_t)DK * DV, n = (size_t)BH * per;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
    const size_t bh = e / per, rem = e % per;
    const int d = (int)(rem / DV);
    float* p = gbuf + bh * nseg * per + rem;
    float acc = p[(nseg - 2) * per];
    for (int sg = nseg - 3; sg >= 0; --sg) {
      acc = gam[(bh * nseg + sg + 1) * DK + d] * acc + p[sg * per];
      p[sg * per] = acc;
    }
  }
}

cudaError_t segment_states(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mg,
                           const CUtensorMap& mv, const CUtensorMap& mdo, const float* h0, const float* dhT,
                           float* sbuf, float* gbuf, float* gam, int BH, int T, int dk, int dv, int nseg,
                           int seg_chunks, long long st_bh, long long st_row, cudaStream_t st, float inv_tau, int ck,
                           int cv) {
  if (dk != 128 || nseg < 2) return cudaErrorNotSupported;
  FwdArgs a = {};
  a.inv_tau = inv_tau;
  a.ck = ck;
  a.cv = cv;
  a.T = T;
  a.DV = dv;
  a.seg_chunks = seg_chunks;
  a.nseg = nseg;
  a.st_bh = st_bh;
  a.st_row = st_row;
  a.latch = device_error_latch();
  a.h0 = h0;
  a.sbuf = sbuf;
  a.gam = gam;
  const bool flex = inv_tau > 0.f || ck != 0 || cv != 0;
  // The two passes are independent (only the reverse scan below needs the forward pass's decay
  // products): the reverse pass runs on a side stream, beside the forward one.
  SideStream* side = nullptr;
  cudaError_t e = side_stream(1, &side);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lock(side->mu);
    if ((e = cudaEventRecord(side->fork, st)) != cudaSuccess) return e;
    if ((e = cudaStreamWaitEvent(side->s, side->fork, 0)) != cudaSuccess) return e;
    FwdArgs r = a;
    r.h0 = dhT;
    r.sbuf = gbuf;
    r.gam = nullptr;
    e = flex ? launch_state_pass<128, true, true, true>(mq, mg, mdo, r, BH, dv, side->s)
             : launch_state_pass<128, true, true, false>(mq, mg, mdo, r, BH, dv, side->s);
    if (e != cudaSuccess) return e;
    if ((e = cudaEventRecord(side->join, side->s)) != cudaSuccess) return e;
    e = flex ? launch_state_pass<128, true, false, true>(mk, mg, mv, a, BH, dv, st)
             : launch_state_pass<128, true, false, false>(mk, mg, mv, a, BH, dv, st);
    if (e != cudaSuccess) return e;
    if ((e = cudaStreamWaitEvent(st, side->join, 0)) != cudaSuccess) return e;
  }
  if (nseg > 2) {
    const size_t n = (size_t)BH * dk * dv;
    const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
    segment_scan_kernel<<<blocks, 256, 0, st>>>(sbuf, gam, BH, dk, dv, nseg);
    segment_scan_rev_kernel<<<blocks, 256, 0, st>>>(gbuf, gam, BH, dk, dv, nseg);
    e = cudaGetLastError();
  }
  return e;
}

cudaError_t segment_entry_states(const void* k, const void* g, const void* v, const float* h0, float* sbuf,
                                 float* gam, int BH, int T, int dk, int dv, int nseg, int seg_chunks,
                                 cudaStream_t st) {
  if (dk != 64 || dv % DVT != 0 || nseg < 2) return cudaErrorNotSupported;
  CUtensorMap m[3];
  if (!make_map(&m[0], k, BH, T, dk, dk, false) || !make_map(&m[1], g, BH, T, dk, dk, false) ||
      !make_map(&m[2], v, BH, T, dv, DVT, true))
    return cudaErrorInvalidValue;
  FwdArgs a = {};
  a.h0 = h0;
  a.sbuf = sbuf;
  a.gam = gam;
  a.T = T;
  a.DV = dv;
  a.seg_chunks = seg_chunks;
  a.nseg = nseg;
  a.st_bh = (long long)dk * dv;
  a.st_row = dv;
  a.latch = device_error_latch();
  cudaError_t e = launch_state_pass<64, false, false, false>(m[0], m[1], m[2], a, BH, dv, st);
  if (e != cudaSuccess || nseg < 3) return e;
  const size_t n = (size_t)BH * dk * dv;
  const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  segment_scan_kernel<<<blocks, 256, 0, st>>>(sbuf, gam, BH, dk, dv, nseg);
  return cudaGetLastError();
}

cudaError_t fwd(const void* q, const void* k, const void* v, const void* g, const float* h0, void* o, float* hT,
                int BH, int T, int dk, int dv, void* ws, cudaStream_t st, long long st_bh, long long st_row,
                float* acc_o, float inv_tau, int dk_total, int k0, const float* add_o, bool kh_hilo, int phase) {
  if (st_bh < 0) st_bh = (long long)dk * dv;
  if (st_row < 0) st_row = dv;
  if (dk_total < 0) dk_total = dk;
  if (k0 < 0 || k0 + dk > dk_total || k0 % 8 != 0) return cudaErrorInvalidValue;
  if (kh_hilo && (dk != 64 || inv_tau > 0.f)) return cudaErrorNotSupported;
  if (dk == 64)
    return launch_fwd<64>(q, k, v, g, h0, o, hT, BH, T, dv, st_bh, st_row, acc_o, ws, st, inv_tau, dk_total, k0, add_o,
                          kh_hilo, phase);
  if (dk == 128)
    return launch_fwd<128>(q, k, v, g, h0, o, hT, BH, T, dv, st_bh, st_row, acc_o, ws, st, inv_tau, dk_total, k0,
                           add_o, false, phase);
  return cudaErrorNotSupported;
}

}  // namespace fast
}  // namespace gla
