// Gated Slot Attention's first pass on the tensor cores, with the slot softmax in its epilogue.
//
// Pass 1 of GSA ("Gated Slot Attention for Efficient Linear-Time Sequence Modeling", abstract: a
// two-layer GLA linked via softmax; "Approach": two-pass linear attention with a data-dependent
// forget gate per memory slot) is a GLA whose gate sits on its value axis, the m slots:
//
//     S1_t = S1_{t-1} diag(alpha_t) + k_t^T phi_t ,    o1_t = q_t S1_t ,    p_t = softmax_m(o1_t)
//
// Per chunk of 64 tokens, with B_j[s] the chunk-local inclusive cumulative log-gate of slot s,
// gamma = B_63, dec = e^{gamma} and E2_j = e^{gamma - B_j} (one ex2 per (token, slot), run products
// as in the GLA kernels):
//
//     X        = Q (S1_i diag(dec)) + mask(Q K^T) (Phi o E2)      one TMEM accumulator [64 x 64]
//     o1_j[s]  = e^{B_j[s] - gamma[s]} X_j[s]                      epilogue (fp32)
//     S1_{i+1} = S1_i diag(dec) + K^T (Phi o E2)                   state on chip (fp32 registers)
//
// The gate enters only through column scalings, so q and k feed tcgen05.mma as TMA loads them
// (raw bf16 tiles with the 128-byte swizzle) and A = Q K^T is exact in fp32.  The state copy, the
// masked A and Phi o E2 are bf16 hi + lo pairs: the slot softmax turns absolute errors of o1 into
// relative errors of p, and a single bf16 Phi o E2 alone put the output several percent off.  The epilogue scales X, takes the softmax over the 64 slots of each token
// (the two threads that hold a token's halves exchange the row max and sum in shared memory) and
// stores p in bf16; o1 never reaches HBM.
//
// Exponent safety: e^{B - gamma} <= e^{|gamma|} stays finite while every slot keeps at least e^-40
// of its state over the chunk.  A chunk below that (near-reset gates) takes an exact path: the
// state copy is unscaled, and o1_j[s] = e^{B_j[s]} (Q S1_i)_j[s] + sum_{r<=j} A_jr phi_r[s]
// prod_{t=r+1..j} alpha_t[s] is formed in fp32 on the CUDA cores (the products only shrink, so any
// finite g <= 0 is handled); the chunk then adds nothing through the second MMA group.
//
// One CTA per (head, sequence segment): 8 compute warps and a producer warp that issues the TMA
// loads and the MMAs, with the same hand-over and software pipeline as the GLA forward (while the
// first MMA group of chunk i runs, the compute warps finish chunk i-1's outputs and run chunk
// i+1's gate math).  With few heads the chunks are cut into segments: a state-only pass of the
// transposed recurrence S1^T <- diag(dec) S1^T + (Phi o E2)^T K (a key-gated GLA state with keys
// phi and values k) and a scan over segments give every segment its entry state.
#include "fast_path.cuh"
#include "fused_common.cuh"
#include "gsa_fused.cuh"

namespace gla {
namespace gsa {

using namespace sm100;
using fast::C;
using fast::kBarCompute;
using fast::kLog2e;
using fast::kMinDecay;
using fast::bar_arrive;
using fast::bar_or;
using fast::bar_sync;
using fast::bf2f;
using fast::bf_hi;
using fast::bf_lo;
using fast::ex2;
using fast::pack2;
using fast::store_half_split;

constexpr int M = kSlots;
constexpr int NCOMP = 256;          // compute threads: warps w and w+4 share TMEM lanes
constexpr int NTH = NCOMP + 32;     // and the producer warp
constexpr int kBarOps = 2, kBarAB = 3;

template <int DK>
struct Pass1Layout {
  static constexpr uint32_t QT = C * DK * 2;               // a q or k tile [64 x DK]: DK/64 swizzled boxes
  static constexpr uint32_t ST = C * M * 2;                // a phi or g tile [64 x 64], swizzled
  static constexpr uint32_t Q_OFF = 0, K_OFF = QT, PHI_OFF = 2 * QT, G_OFF = 2 * QT + ST;
  static constexpr uint32_t STAGE = 2 * QT + 2 * ST;       // two stages
  static constexpr uint32_t PH0 = 2 * STAGE;               // Phi o E2 hi / lo [64 x 64], per chunk parity
  static constexpr uint32_t SB_HI = PH0 + 4 * ST;          // state copy hi / lo [DK x 64], MN-major B
  static constexpr uint32_t SB_LO = SB_HI + DK * M * 2;
  static constexpr uint32_t AB_HI = SB_LO + DK * M * 2;    // masked A hi / lo [64 x 64], K-major A
  static constexpr uint32_t AB_LO = AB_HI + C * C * 2;
  static constexpr int EP = 68;                            // row pitch (floats) of the scale table
  static constexpr uint32_t ETAB = AB_LO + C * C * 2;      // float [2][64][EP]: per-token slot scales
  static constexpr uint32_t DECAY = ETAB + 2 * C * EP * 4; // float [2][64]: e^{gamma} per slot
  static constexpr uint32_t SMX = DECAY + 2 * M * 4;       // float [2][64] row maxima, [2][64] row sums
  static constexpr int NS = fast::GateRun<M, NCOMP>::NSPLIT;
  static constexpr uint32_t TOT = SMX + 4 * C * 4;         // float [NS][64]: gate run products
  static constexpr uint32_t TOTAL = TOT + NS * M * 4;
  static_assert(TOT % 8 == 0 && DECAY % 8 == 0, "gate tables are read as float2");
  static constexpr uint32_t ALLOC = TOTAL + 1024;
  // exact-path scratch while the A epilogue of a chunk runs (its state copy has been consumed):
  // A in fp32 and the decays alpha, both [64][64]
  static constexpr uint32_t XA = SB_HI, XAL = SB_HI + C * C * 4;
  static_assert(DK == 128, "the pass-1 kernel covers d_k = 128");
  static_assert(STAGE % 1024 == 0 && QT % 1024 == 0 && PH0 % 1024 == 0 && SB_HI % 1024 == 0 && AB_HI % 1024 == 0,
                "operand alignment");
  static_assert(2 * C * C * 4 <= 2 * DK * M * 2, "exact-path scratch");
  static_assert(ALLOC <= 227 * 1024, "shared memory");
};

struct Pass1Args {
  const float* h0;        // [BH][DK][64] or null (zeros)
  const float* sin;       // [BH][nseg][64][DK]: transposed state entering segment s at entry s-1
  __nv_bfloat16* p;       // [BH][T][64], or
  float* p32;             // [BH][T][64] in fp32 (when set, in place of p)
  float* hT;              // [BH][DK][64] or null
  int T, seg_chunks, nseg;
  unsigned int* latch;
};

template <int DK>
__global__ void __launch_bounds__(NTH, 1)
    pass1_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_phi, const __grid_constant__ CUtensorMap tm_g,
                 const Pass1Args args) {
  using L = Pass1Layout<DK>;
  using Gate = fast::GateRun<M, NCOMP>;
  constexpr int TS = Gate::TS;
  constexpr int NHAND = NCOMP + 32;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_ld[2], bar_mma1, bar_mma2;
  __shared__ uint32_t tmem_base_sh;
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const uint32_t base = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3, half = (warp >> 2) & 1;
  const int bh = blockIdx.x, seg = blockIdx.y;
  const int T = args.T, NC = (T + C - 1) / C;
  const int c_begin = seg * args.seg_chunks;
  const int nloc = min(NC, c_begin + args.seg_chunks) - c_begin;
  unsigned int* latch = args.latch;
  float* decay_sm = reinterpret_cast<float*>(sm + L::DECAY);
  float* tot_sm = reinterpret_cast<float*>(sm + L::TOT);
  float* etab = reinterpret_cast<float*>(sm + L::ETAB);
  float* smx = reinterpret_cast<float*>(sm + L::SMX);

  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, 256);
    tmem_relinquish();
  }
  if (tid == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_phi);
    prefetch_tmap(&tm_g);
    mbar_init(&bar_ld[0], 1);
    mbar_init(&bar_ld[1], 1);
    mbar_init(&bar_mma1, 1);
    mbar_init(&bar_mma2, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t t_A = tmem, t_X0 = tmem + 64, t_dS = tmem + 192;
  const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;

  if (warp == NCOMP / 32) {
    // ------------------------------ producer warp ------------------------------
    auto load_stage = [&](int li) {
      const int s = li & 1, chunk = c_begin + li;
      uint8_t* st = sm + s * L::STAGE;
      mbar_arrive_expect_tx(&bar_ld[s], L::STAGE);
#pragma unroll
      for (int b = 0; b < DK / 64; ++b) {
        tma_load_3d(st + L::Q_OFF + b * (C * 128), &tm_q, &bar_ld[s], b * 64, chunk * C, bh);
        tma_load_3d(st + L::K_OFF + b * (C * 128), &tm_k, &bar_ld[s], b * 64, chunk * C, bh);
      }
      tma_load_3d(st + L::PHI_OFF, &tm_phi, &bar_ld[s], 0, chunk * C, bh);
      tma_load_3d(st + L::G_OFF, &tm_g, &bar_ld[s], 0, chunk * C, bh);
    };
    if (lane == 0) {
      load_stage(0);
      if (nloc > 1) load_stage(1);
    }
    constexpr uint32_t id_A = idesc_bf16_f32(C, C, false, false);
    constexpr uint32_t id_X = idesc_bf16_f32(C, M, false, true);
    constexpr uint32_t id_S = idesc_bf16_f32(DK, M, true, true);
    for (int li = 0; li < nloc; ++li) {
      bar_sync(kBarOps, NHAND);  // chunk li's Phi o E2 and state copy are in shared memory
      if (lane == 0) {
        // group 1: A = Q K^T, X = Q S', dS = K^T (Phi o E2)
        mbar_wait(&bar_ld[li & 1], (li >> 1) & 1, latch);
        tc_fence_after();
        const uint32_t st = base + (li & 1) * L::STAGE;
        const uint32_t ph = base + L::PH0 + (li & 1) * 2 * L::ST;  // hi, then lo at + ST
        const uint32_t t_X = t_X0 + (li & 1) * 64;
#pragma unroll
        for (int k = 0; k < DK / 16; ++k) {
          const uint32_t koff = (k >> 2) * (C * 128) + (k & 3) * 32;
          const uint64_t qd = desc_sw128(st + L::Q_OFF + koff, 16, 1024);
          umma_bf16(t_A, qd, desc_sw128(st + L::K_OFF + koff, 16, 1024), id_A, k > 0);
          umma_bf16(t_X, qd, desc_sw128(base + L::SB_HI + k * 2048, 16, 1024), id_X, k > 0);
          umma_bf16(t_X, qd, desc_sw128(base + L::SB_LO + k * 2048, 16, 1024), id_X, 1);
        }
#pragma unroll
        for (int k = 0; k < C / 16; ++k) {
          const uint64_t kd = desc_sw128(st + L::K_OFF + k * 2048, C * 128, 1024);
          umma_bf16(t_dS, kd, desc_sw128(ph + k * 2048, 16, 1024), id_S, k > 0);
          umma_bf16(t_dS, kd, desc_sw128(ph + L::ST + k * 2048, 16, 1024), id_S, 1);
        }
        umma_commit(&bar_mma1);
      }
      bar_sync(kBarAB, NHAND);  // chunk li's masked A is in shared memory; its stage is free
      if (lane == 0) {
        // group 2: X += mask(A) (Phi o E2)
        tc_fence_after();
        const uint32_t ph = base + L::PH0 + (li & 1) * 2 * L::ST;
        const uint32_t t_X = t_X0 + (li & 1) * 64;
#pragma unroll
        for (int k = 0; k < C / 16; ++k) {
          const uint64_t vh = desc_sw128(ph + k * 2048, 16, 1024), vl = desc_sw128(ph + L::ST + k * 2048, 16, 1024);
          const uint64_t ah = desc_sw128(base + L::AB_HI + k * 32, 16, 1024);
          umma_bf16(t_X, ah, vh, id_X, 1);
          umma_bf16(t_X, desc_sw128(base + L::AB_LO + k * 32, 16, 1024), vh, id_X, 1);
          umma_bf16(t_X, ah, vl, id_X, 1);
        }
        umma_commit(&bar_mma2);
        // the stage of chunk li is read by nothing after its first group and the A epilogue
        if (li + 2 < nloc) load_stage(li + 2);
      }
      __syncwarp();
    }
  } else {
    // ------------------------------ compute warps ------------------------------
    // State owned by this thread: row s_row of S1 (the M = DK lanes of the dS accumulator),
    // slots sc0 .. sc0+31.
    constexpr int SW = M / 2;
    const int s_row = q4 * 32 + lane;
    const int sc0 = half * SW;
    float S[SW];
#pragma unroll
    for (int c = 0; c < SW; ++c) S[c] = 0.f;
    if (seg == 0) {
      if (args.h0) {
        const float4* src = reinterpret_cast<const float4*>(args.h0 + ((size_t)bh * DK + s_row) * M + sc0);
#pragma unroll
        for (int c = 0; c < SW / 4; ++c) {
          const float4 x = src[c];
          S[4 * c] = x.x;
          S[4 * c + 1] = x.y;
          S[4 * c + 2] = x.z;
          S[4 * c + 3] = x.w;
        }
      }
    } else {
      const float* src = args.sin + ((size_t)bh * args.nseg + seg - 1) * M * DK;
#pragma unroll
      for (int c = 0; c < SW; ++c) S[c] = src[(size_t)(sc0 + c) * DK + s_row];
    }

    // Gate math of local chunk li (stage li & 1): decays, Phi o E2 into registers, and the scale
    // table e^{B_j - gamma} (e^{B_j} on the exact path).  Returns the chunk's exact-path flag.
    uint32_t phr[TS], phl[TS];
    int gd = 0, gh = 0;
    auto gate_regs = [&](int li) {
      const uint8_t* st = sm + (li & 1) * L::STAGE;
      Gate gr;
      const bool weak = gr.run_swizzled(st + L::G_OFF, tot_sm);
      float* dec = decay_sm + (li & 1) * M;
      if (gr.h == 0) gr.store_decay(dec);
      const int safe = bar_or(kBarCompute, NCOMP, weak);
      gd = gr.d;
      gh = gr.h;
      uint32_t w[TS];
      gr.load_pairs(st + L::PHI_OFF, M, true, w);
      gr.backward([&](int j, float e0, float e1) {
        const uint32_t x = w[j - gh * TS];
        fast::split2(bf_lo(x) * e0, bf_hi(x) * e1, phr[j - gh * TS], phl[j - gh * TS]);
      });
      // written after the gate run's barrier: every compute thread has finished reading the table
      // of chunk li - 2 (same parity) by then
      float* et = etab + (li & 1) * C * L::EP;
      const float i0 = safe ? 1.f : 1.f / gr.dec0, i1 = safe ? 1.f : 1.f / gr.dec1;
      gr.forward([&](int j, float e0, float e1) {
        et[j * L::EP + gd] = e0 * i0;
        et[j * L::EP + gd + 1] = e1 * i1;
      });
      return safe;
    };
    // Operands of local chunk li into shared memory, then hand them to the producer.
    auto store_ops = [&](int li, int safe) {
      uint8_t* phb = sm + L::PH0 + (li & 1) * 2 * L::ST;
#pragma unroll
      for (int u = 0; u < TS; ++u) {
        *reinterpret_cast<uint32_t*>(phb + sw128(gh * TS + u, gd)) = phr[u];
        *reinterpret_cast<uint32_t*>(phb + L::ST + sw128(gh * TS + u, gd)) = phl[u];
      }
      const float* dec = decay_sm + (li & 1) * M;
      float sv[SW];
#pragma unroll
      for (int c = 0; c < SW; ++c) sv[c] = safe ? S[c] : S[c] * dec[sc0 + c];
      store_half_split(sm + L::SB_HI, sm + L::SB_LO, s_row, sv, half);
      fence_async_smem();
      tc_fence_before();
      bar_arrive(kBarOps, NHAND);
    };
    // Exact path of chunk li (after its first MMA group): o1 in fp32 into the X accumulator, and a
    // zero masked A so that the second group adds nothing.
    auto exact_chunk = [&](int li) {
      const uint8_t* st = sm + (li & 1) * L::STAGE;
      float* XA = reinterpret_cast<float*>(sm + L::XA);
      float* XAL = reinterpret_cast<float*>(sm + L::XAL);
      const int j = q4 * 16 + lane, cb = half * 32;
      const uint32_t t_X = t_X0 + (li & 1) * 64;
      float v[32];
      tmem_ld32(t_A + lane_off + cb, v);
      tmem_ld_wait();
      if (lane < 16) {
#pragma unroll
        for (int c = 0; c < 32; ++c) XA[j * C + cb + c] = v[c];
      }
      for (int e = tid; e < C * M; e += NCOMP) {
        const int t = e / M, s = e % M;
        XAL[e] = ex2(bf2f(st + L::G_OFF + sw128(t, s)) * kLog2e);
      }
      bar_sync(kBarCompute, NCOMP);
      tmem_ld32(t_X + lane_off + cb, v);  // Q S1_i (unscaled state copy)
      tmem_ld_wait();
      if (lane < 16) {
        const float* et = etab + (li & 1) * C * L::EP + j * L::EP + cb;  // e^{B_j}
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {  // two groups of 16 slots keep the register count down
          float acc[16], w[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            acc[c] = 0.f;
            w[c] = 1.f;
          }
          for (int r = j; r >= 0; --r) {
            const float ar = XA[j * C + r];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const int s = cb + 16 * hh + c;
              acc[c] += ar * bf2f(st + L::PHI_OFF + sw128(r, s)) * w[c];
              w[c] *= XAL[r * M + s];
            }
          }
#pragma unroll
          for (int c = 0; c < 16; ++c) v[16 * hh + c] = et[16 * hh + c] * v[16 * hh + c] + acc[c];
        }
      }
      tmem_st32(t_X + lane_off + cb, v);
      tmem_st_wait();
      if (lane < 16) {
        const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const uint32_t off = j * 128 + ((((4 * half + cc) ^ (j & 7)) & 7) << 4);
          *reinterpret_cast<uint4*>(sm + L::AB_HI + off) = zero;
          *reinterpret_cast<uint4*>(sm + L::AB_LO + off) = zero;
        }
      }
    };
    // Outputs of local chunk li (after its second group): scale, slot softmax, p in bf16.
    auto store_o = [&](int li, int safe_li) {
      mbar_wait(&bar_mma2, li & 1, latch);
      tc_fence_after();
      const int j = q4 * 16 + lane, cb = half * 32;
      float x[32];
      tmem_ld32(t_X0 + (li & 1) * 64 + lane_off + cb, x);
      tmem_ld_wait();
      float* smax = smx;
      float* ssum = smx + 2 * C;
      bar_sync(kBarCompute, NCOMP);  // the scale table of chunk li is complete
      if (lane < 16) {
        if (!safe_li) {
          const float* et = etab + (li & 1) * C * L::EP + j * L::EP + cb;
#pragma unroll
          for (int c = 0; c < 32; ++c) x[c] *= et[c];
        }
        float mx = x[0];
#pragma unroll
        for (int c = 1; c < 32; ++c) mx = fmaxf(mx, x[c]);
        smax[half * C + j] = mx;
      }
      bar_sync(kBarCompute, NCOMP);
      if (lane < 16) {
        const float mx = fmaxf(smax[j], smax[C + j]);
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          x[c] = ex2((x[c] - mx) * kLog2e);
          sum += x[c];
        }
        ssum[half * C + j] = sum;
      }
      bar_sync(kBarCompute, NCOMP);
      const int t = (c_begin + li) * C + j;
      if (lane < 16 && t < T) {
        const float inv = 1.f / (ssum[j] + ssum[C + j]);
#pragma unroll
        for (int c = 0; c < 32; ++c) x[c] *= inv;
        if (args.p32) {
          float4* dst = reinterpret_cast<float4*>(args.p32 + ((size_t)bh * T + t) * M + cb);
#pragma unroll
          for (int c = 0; c < 8; ++c) dst[c] = make_float4(x[4 * c], x[4 * c + 1], x[4 * c + 2], x[4 * c + 3]);
        } else {
          fast::store_half_global_bf16(args.p + ((size_t)bh * T + t) * M + cb, x);
        }
      }
    };

    mbar_wait(&bar_ld[0], 0, latch);
    int safe = gate_regs(0);
    store_ops(0, safe);
    int safe_prev = 0;
    for (int li = 0; li < nloc; ++li) {
      // ---- while group 1 of chunk li runs: outputs of chunk li-1, gate math of chunk li+1 ----
      if (li > 0) store_o(li - 1, safe_prev);
      int safe_next = 0;
      if (li + 1 < nloc) {
        mbar_wait(&bar_ld[(li + 1) & 1], ((li + 1) >> 1) & 1, latch);
        safe_next = gate_regs(li + 1);
      }
      // ---- group 1 done: A epilogue (or the exact path), state update; group 2 next ----
      mbar_wait(&bar_mma1, li & 1, latch);
      tc_fence_after();
      if (safe) {
        exact_chunk(li);
      } else {
        const int j = q4 * 16 + lane, cb = half * 32;
        float a[32];
        tmem_ld32(t_A + lane_off + cb, a);
        tmem_ld_wait();
        if (lane < 16) {
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (cb + c > j) a[c] = 0.f;
          store_half_split(sm + L::AB_HI, sm + L::AB_LO, j, a, half);
        }
      }
      {
        float ds[SW];
        tmem_ld32(t_dS + lane_off + sc0, ds);
        tmem_ld_wait();
        const float* dec = decay_sm + (li & 1) * M;
#pragma unroll
        for (int c = 0; c < SW; ++c) S[c] = dec[sc0 + c] * S[c] + ds[c];
      }
      fence_async_smem();
      tc_fence_before();
      bar_arrive(kBarAB, NHAND);
      // ---- while group 2 of chunk li runs: operands of chunk li+1 (group 1 follows) ----
      // The exact path's scratch lies over the state copy: every thread is done with it first.
      if (safe) bar_sync(kBarCompute, NCOMP);
      if (li + 1 < nloc) store_ops(li + 1, safe_next);
      safe_prev = safe;
      safe = safe_next;
    }
    store_o(nloc - 1, safe_prev);
    if (seg == args.nseg - 1 && args.hT) {
      float4* dst = reinterpret_cast<float4*>(args.hT + ((size_t)bh * DK + s_row) * M + sc0);
#pragma unroll
      for (int c = 0; c < SW / 4; ++c) dst[c] = make_float4(S[4 * c], S[4 * c + 1], S[4 * c + 2], S[4 * c + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

// ------------------------------------------------------------------------------------------
// Elementwise glue.  The backward runs both GLA passes on 128-wide key blocks whose first 64 keys
// are the slots; the other 64 carry a second copy of the slots (same keys phi, same gates) whose
// queries are the low bf16 parts of the real queries: with queries [hi | lo] the pass computes
// exactly what queries hi + lo give (the output is linear in the queries), so p and do1 enter with
// about 16 mantissa bits instead of 8.  The gradients of the two copies add up.
// ------------------------------------------------------------------------------------------
// One warp per token: do1 = p (dp - <p, dp>) over the m <= 64 slots (each lane takes two), from
// p in fp32 and dp (fp32, row pitch dp_pitch); do1 goes out as bf16 [hi | lo] rows of 2m.
__global__ void jacobian_kernel(const float* __restrict__ p, const float* __restrict__ dp, int dp_pitch,
                                __nv_bfloat16* __restrict__ do1, long long rows, int m) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const int c = 2 * lane;
    float p0 = 0.f, p1 = 0.f, d0 = 0.f, d1 = 0.f;
    if (c < m) {
      const float2 pp = *reinterpret_cast<const float2*>(p + r * m + c);
      const float2 dd = *reinterpret_cast<const float2*>(dp + r * dp_pitch + c);
      p0 = pp.x;
      p1 = pp.y;
      d0 = dd.x;
      d1 = dd.y;
    }
    float dot = p0 * d0 + p1 * d1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    if (c < m) {
      const float x0 = p0 * (d0 - dot), x1 = p1 * (d1 - dot);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(x0, x1);
      const __nv_bfloat162 lo = __floats2bfloat162_rn(x0 - __low2float(hi), x1 - __high2float(hi));
      *reinterpret_cast<__nv_bfloat162*>(do1 + r * 2 * m + c) = hi;
      *reinterpret_cast<__nv_bfloat162*>(do1 + r * 2 * m + m + c) = lo;
    }
  }
}

// Rows of 2m bf16: [hi | lo] of fp32 rows of m (mode 0), or [x | x] of bf16 rows of m (mode 1).
__global__ void widen_kernel(const void* __restrict__ src, __nv_bfloat16* __restrict__ dst, long long rows, int m,
                             int mode) {
  const int vpr = m / 2;
  const long long n = rows * vpr;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
    const long long r = e / vpr;
    const int c = (int)(e % vpr) * 2;
    __nv_bfloat162 a, b;
    if (mode == 0) {
      const float2 x = *reinterpret_cast<const float2*>(static_cast<const float*>(src) + r * m + c);
      a = __floats2bfloat162_rn(x.x, x.y);
      b = __floats2bfloat162_rn(x.x - __low2float(a), x.y - __high2float(a));
    } else {
      a = b = *reinterpret_cast<const __nv_bfloat162*>(static_cast<const __nv_bfloat16*>(src) + r * m + c);
    }
    *reinterpret_cast<__nv_bfloat162*>(dst + r * 2 * m + c) = a;
    *reinterpret_cast<__nv_bfloat162*>(dst + r * 2 * m + m + c) = b;
  }
}

// dst [nb][Cp][R]: dst[b][c][r] = src[b * sb + r * Cc + c] (+ src[b * sb + (r + R) * Cc + c] when
// fold, the second copy's row) for c < Cc, zeros for Cc <= c < Cp.
__global__ void transpose_kernel(const float* __restrict__ src, long long sb, float* __restrict__ dst, int nb, int R,
                                 int Cc, int Cp, int fold) {
  const long long n = (long long)nb * Cp * R;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(e % R);
    const int c = (int)((e / R) % Cp);
    const long long b = e / ((long long)R * Cp);
    float x = 0.f;
    if (c < Cc) {
      x = src[b * sb + (long long)r * Cc + c];
      if (fold) x += src[b * sb + (long long)(r + R) * Cc + c];
    }
    dst[e] = x;
  }
}

// dst[b][r][c] = src[b][r][c] + src[b][r + R][c]: the two copies' state gradients, [nb][2R][Cc] -> [nb][R][Cc].
__global__ void fold_rows_kernel(const float* __restrict__ src, float* __restrict__ dst, int nb, int R, int Cc) {
  const long long per = (long long)R * Cc, n = (long long)nb * per;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
    const long long b = e / per, i = e % per;
    dst[e] = src[b * 2 * per + i] + src[b * 2 * per + per + i];
  }
}

// out[r][c] = bf16(a[r][c] + a[r][m + c] + b[r][c] + b[r][m + c]) for c < m: both passes, both copies
// (a, b fp32 with rows of 2m).
__global__ void fold_add_kernel(const float* __restrict__ a, const float* __restrict__ b, __nv_bfloat16* __restrict__ out,
                                long long rows, int m) {
  const int vpr = m / 2;
  const long long n = rows * vpr;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
    const long long r = e / vpr;
    const int c = (int)(e % vpr) * 2;
    const float* ar = a + r * 2 * m;
    const float* br = b + r * 2 * m;
    const float2 a0 = *reinterpret_cast<const float2*>(ar + c), a1 = *reinterpret_cast<const float2*>(ar + m + c);
    const float2 b0 = *reinterpret_cast<const float2*>(br + c), b1 = *reinterpret_cast<const float2*>(br + m + c);
    *reinterpret_cast<__nv_bfloat162*>(out + r * m + c) =
        __floats2bfloat162_rn(a0.x + a1.x + b0.x + b1.x, a0.y + a1.y + b0.y + b1.y);
  }
}

int grid_for(long long items, int per_block) {
  const long long blocks = (items + per_block - 1) / per_block, cap = (long long)fast::sm_count() * 8;
  return (int)(blocks < 1 ? 1 : blocks > cap ? cap : blocks);
}

// ------------------------------------------------------------------------------------------
// Host entry points
// ------------------------------------------------------------------------------------------
// Segments: as many as fill the SMs once with one CTA per (head, segment); 1 when the heads alone
// fill at least half of them.
static void plan_pass1(int BH, int T, int* nseg, int* seg_chunks) {
  const int NC = (T + C - 1) / C, sms = fast::sm_count();
  int n = 1;
  if (2 * BH <= sms) n = sms / BH;
  if (n > NC) n = NC;
  if (n < 1) n = 1;
  const int per = (NC + n - 1) / n;
  *seg_chunks = per;
  *nseg = (NC + per - 1) / per;
}

bool pass1_supported(int BH, int T, int dk, int m, int chunk, int dtype) {
  if (dtype != 1 || chunk != C || T < 1 || BH < 1 || BH > 65535) return false;
  if (dk != 128 || m != M) return false;
  return fast::encode_fn() != nullptr;
}

size_t pass1_workspace(int BH, int T, int dk) {
  int nseg, per;
  plan_pass1(BH, T, &nseg, &per);
  if (nseg == 1) return 0;
  return align256((size_t)BH * nseg * M * dk * 4) + align256((size_t)BH * nseg * M * 4) +
         align256((size_t)BH * M * dk * 4);
}

cudaError_t pass1_fwd(const void* q, const void* k, const void* phi, const void* g, const float* h0, void* p,
                      float* hT, int BH, int T, int dk, void* ws, cudaStream_t st, float* p32) {
  if (dk != 128) return cudaErrorNotSupported;
  constexpr int DK = 128;
  using L = Pass1Layout<DK>;
  CUtensorMap mq, mk, mphi, mg;
  if (!fast::make_map(&mq, q, BH, T, DK, 64, true) || !fast::make_map(&mk, k, BH, T, DK, 64, true) ||
      !fast::make_map(&mphi, phi, BH, T, M, 64, true) || !fast::make_map(&mg, g, BH, T, M, 64, true))
    return cudaErrorInvalidValue;
  Pass1Args a;
  a.h0 = h0;
  a.sin = nullptr;
  a.p = static_cast<__nv_bfloat16*>(p);
  a.p32 = p32;
  a.hT = hT;
  a.T = T;
  a.latch = device_error_latch();
  plan_pass1(BH, T, &a.nseg, &a.seg_chunks);
  if (a.nseg > 1) {
    if (!ws) return cudaErrorInvalidValue;
    float* sbuf = static_cast<float*>(ws);
    float* gam = sbuf + align256((size_t)BH * a.nseg * M * DK * 4) / 4;
    float* h0t = gam + align256((size_t)BH * a.nseg * M * 4) / 4;
    if (h0) {
      transpose_kernel<<<grid_for((long long)BH * M * DK, 256), 256, 0, st>>>(h0, (long long)DK * M, h0t, BH, DK,
                                                                            M, M, 0);
      const cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    // transposed recurrence: keys phi (the 64 gated slots), values k
    const cudaError_t e =
        fast::segment_entry_states(phi, g, k, h0 ? h0t : nullptr, sbuf, gam, BH, T, M, DK, a.nseg, a.seg_chunks, st);
    if (e != cudaSuccess) return e;
    a.sin = sbuf;
  }
  auto kern = pass1_kernel<DK>;
  static std::atomic<bool> attr_set[64] = {};
  {
    const cudaError_t e = fast::ensure_smem_attr(kern, L::ALLOC, attr_set);
    if (e != cudaSuccess) return e;
  }
  kern<<<dim3(BH, a.nseg), NTH, L::ALLOC, st>>>(mq, mk, mphi, mg, a);
  return cudaGetLastError();
}

cudaError_t softmax_jacobian(const float* p, const float* dp, int dp_pitch, void* do1, long long rows, int m,
                             cudaStream_t st) {
  if (m > 64 || m % 2 != 0) return cudaErrorNotSupported;
  jacobian_kernel<<<grid_for(rows, 8), 256, 0, st>>>(p, dp, dp_pitch, static_cast<__nv_bfloat16*>(do1), rows, m);
  return cudaGetLastError();
}

cudaError_t widen(const void* src, void* dst, long long rows, int m, bool hilo, cudaStream_t st) {
  if (m % 2 != 0) return cudaErrorNotSupported;
  widen_kernel<<<grid_for(rows * (m / 2), 256), 256, 0, st>>>(src, static_cast<__nv_bfloat16*>(dst), rows, m,
                                                               hilo ? 0 : 1);
  return cudaGetLastError();
}

cudaError_t transpose_states(const float* src, long long src_bstride, float* dst, int nb, int R, int Cc, int Cp,
                             cudaStream_t st, bool fold) {
  transpose_kernel<<<grid_for((long long)nb * Cp * R, 256), 256, 0, st>>>(src, src_bstride, dst, nb, R, Cc, Cp,
                                                                          fold ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t fold_rows(const float* src, float* dst, int nb, int R, int Cc, cudaStream_t st) {
  fold_rows_kernel<<<grid_for((long long)nb * R * Cc, 256), 256, 0, st>>>(src, dst, nb, R, Cc);
  return cudaGetLastError();
}

cudaError_t fold_add_bf16(const float* a, const float* b, void* out, long long rows, int m, cudaStream_t st) {
  if (m % 2 != 0) return cudaErrorNotSupported;
  fold_add_kernel<<<grid_for(rows * (m / 2), 256), 256, 0, st>>>(a, b, static_cast<__nv_bfloat16*>(out), rows, m);
  return cudaGetLastError();
}

}  // namespace gsa
}  // namespace gla
