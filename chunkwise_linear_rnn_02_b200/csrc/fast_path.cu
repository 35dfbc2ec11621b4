// Fused sm_100a chunkwise GLA kernels (bf16 in, fp32 accumulate, chunk 64).
//
// Forward, one CTA per (head, 64 value columns); the CTA walks the chunks of its head in order
// and keeps the recurrent state on chip ("MS-GLA ...", section 2.1: sequential inter-chunk
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
//   state (fp32 registers, one thread per row d):   S_{i+1} = e^{gamma} S_i + dS
//
// Qs carries e^{B - gamma} <= e^{|gamma|}; it stays finite (and e^{gamma} S_i stays normal) while
// the chunk keeps at least e^-80 of its state in every key dimension.  A chunk below that bound
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
// Forward kernel
// ------------------------------------------------------------------------------------------
template <int DK>
struct FwdLayout {
  static constexpr uint32_t RAW = C * DK * 2;               // one raw q / k / g tile
  static constexpr uint32_t RAW_V = C * DVT * 2;            // raw v tile (swizzled)
  static constexpr uint32_t STAGE = 3 * RAW + RAW_V;
  static constexpr uint32_t OPS = 2 * STAGE;                // operand area
  static constexpr uint32_t QS_HI = OPS;                    // Qs hi / lo [64 x DK]  K-major
  static constexpr uint32_t QS_LO = QS_HI + C * DK * 2;
  static constexpr uint32_t KH = QS_LO + C * DK * 2;        // Kh [64 x DK]  K-major B / MN-major A
  static constexpr uint32_t SB_HI = KH + C * DK * 2;        // scaled state copy hi / lo [DK x 64] MN-major
  static constexpr uint32_t SB_LO = SB_HI + DK * DVT * 2;
  static constexpr uint32_t AB_HI = SB_LO + DK * DVT * 2;   // A hi / lo [64 x 64] K-major
  static constexpr uint32_t AB_LO = AB_HI + C * C * 2;
  static constexpr uint32_t DECAY = AB_LO + C * C * 2;      // float[DK]       e^{gamma_d}
  static constexpr uint32_t TOT = DECAY + DK * 4;           // float[NSPLIT][DK] run products
  static constexpr uint32_t TOTAL = TOT + GateRun<DK, NTHREADS>::NSPLIT * DK * 4;
  static constexpr uint32_t ALLOC = TOTAL + 1024;           // slack for 1024-byte alignment
  // Exact-path scratch, used after the first MMA group of a chunk has completed: fp32
  // cumulative log-gates [64 x DK] over QS_HI..QS_LO, exact A [64 x 64] fp32 over KH..SB_HI.
  static constexpr uint32_t XB = QS_HI, XA = KH;
  static_assert(STAGE % 1024 == 0 && RAW % 1024 == 0, "stage alignment");
  static_assert(ALLOC <= 227 * 1024, "shared memory");
  static_assert(C * DK * 4 <= KH - QS_HI && C * C * 4 <= SB_LO - KH, "exact-path scratch");
};

struct FwdArgs {
  const float* h0;     // [BH][DK][DV] or null (zeros)
  float* sbuf;         // [BH][nseg][DK][DV]: segment end states (state-only pass), then entry states
  float* gam;          // [BH][nseg][DK]: segment decay products
  __nv_bfloat16* o;
  float* hT;           // [BH][DK][DV] or null
  int T, DV, seg_chunks, nseg;
  unsigned int* latch;
};

// One CTA per (64 value columns, head, segment).  STATE_ONLY: the state recurrence alone (no
// queries, no outputs), writing the segment's end state and decay product.
template <int DK, bool STATE_ONLY>
__global__ void __launch_bounds__(NTHREADS, 1)
    fwd_fused_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_v,
                     const FwdArgs args) {
  using L = FwdLayout<DK>;
  const float* h0 = args.h0;
  __nv_bfloat16* o = args.o;
  const int T = args.T, DV = args.DV;
  unsigned int* latch = args.latch;
  using Gate = GateRun<DK, NTHREADS>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_load[2], bar_mma1, bar_mma2;
  __shared__ uint32_t tmem_base_sh;
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3, half = warp >> 2;  // TMEM lane quarter, column half
  const int dv0 = blockIdx.x * DVT, bh = blockIdx.y, seg = blockIdx.z;
  const int NC = (T + C - 1) / C;
  const int c_begin = seg * args.seg_chunks;
  const int nloc = min(NC, c_begin + args.seg_chunks) - c_begin;  // chunks of this segment
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
    mbar_init(&bar_load[0], 1);
    mbar_init(&bar_load[1], 1);
    mbar_init(&bar_mma1, 1);
    mbar_init(&bar_mma2, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // Local chunk li of the segment into stage li & 1 (the state-only pass skips q).
  auto issue_load = [&](int li) {
    const int s = li & 1, chunk = c_begin + li;
    uint8_t* st = sm + s * L::STAGE;
    mbar_arrive_expect_tx(&bar_load[s], STATE_ONLY ? L::STAGE - L::RAW : L::STAGE);
    if (!STATE_ONLY) tma_load_3d(st, &tm_q, &bar_load[s], 0, chunk * C, bh);
    tma_load_3d(st + L::RAW, &tm_k, &bar_load[s], 0, chunk * C, bh);
    tma_load_3d(st + 2 * L::RAW, &tm_g, &bar_load[s], 0, chunk * C, bh);
    tma_load_3d(st + 3 * L::RAW, &tm_v, &bar_load[s], dv0, chunk * C, bh);
  };
  if (tid == 0) {
    issue_load(0);
    if (nloc > 1) issue_load(1);
  }

  // State owned by this thread: row s_row (lane layout of the dS accumulator, M = DK), columns
  // sc0 .. sc0+31 of the CTA's 64.
  constexpr int SW = DVT / 2;
  const bool s_owner = (DK == 128) ? true : (lane < 16);
  const int s_row = (DK == 128) ? (q4 * 32 + lane) : (q4 * 16 + lane);
  const int sc0 = half * SW;
  float S[SW];
#pragma unroll
  for (int c = 0; c < SW; ++c) S[c] = 0.f;
  // Entry state: h0 for the first segment; the scanned entry state for the others (full pass).
  const float* init = seg == 0 ? (h0 ? h0 + (size_t)bh * DK * DV : nullptr)
                      : STATE_ONLY ? nullptr
                                   : args.sbuf + ((size_t)bh * args.nseg + seg - 1) * DK * DV;
  float gamma_acc = 1.f;  // decay product of the segment for row s_row (state-only pass)
  if (s_owner && init) {
    const float4* src = reinterpret_cast<const float4*>(init + (size_t)s_row * DV + dv0 + sc0);
#pragma unroll
    for (int c = 0; c < SW / 4; ++c) {
      const float4 x = src[c];
      S[4 * c] = x.x;
      S[4 * c + 1] = x.y;
      S[4 * c + 2] = x.z;
      S[4 * c + 3] = x.w;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t t_A = tmem, t_O = tmem + 64, t_dS = tmem + 128;
  const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;

  for (int li = 0; li < nloc; ++li) {
    const int s = li & 1, i = c_begin + li;
    uint8_t* st = sm + s * L::STAGE;
    mbar_wait(&bar_load[s], (li >> 1) & 1, latch);

    if constexpr (STATE_ONLY) {  // gates, Kh, dS = Kh^T V, S = e^{gamma} S + dS
      Gate gr;
      gr.run(st + 2 * L::RAW, DK, tot_sm);
      if (gr.h == 0) {
        decay_sm[gr.d] = gr.dec0;
        decay_sm[gr.d + 1] = gr.dec1;
      }
      {
        const uint32_t blk = (gr.d >> 6) * (C * 128), col = gr.d & 63;
        gr.backward([&](int j, float e0, float e1) {
          const uint32_t wk = *reinterpret_cast<const uint32_t*>(st + L::RAW + (j * DK + gr.d) * 2);
          *reinterpret_cast<uint32_t*>(sm + L::KH + blk + sw128(j, col)) = pack2(bf_lo(wk) * e0, bf_hi(wk) * e1);
        });
      }
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      if (tid == 0) {
        const uint32_t base = smem_u32(sm);
        const uint32_t vbase = base + s * L::STAGE + 3 * L::RAW;
        constexpr uint32_t id_S = idesc_bf16_f32(DK, DVT, true, true);
#pragma unroll
        for (int k = 0; k < C / 16; ++k)
          umma_bf16(t_dS, desc_sw128(base + L::KH + k * 2048, C * 128, 1024), desc_sw128(vbase + k * 2048, 16, 1024),
                    id_S, k > 0);
        umma_commit(&bar_mma1);
      }
      __syncwarp();
      mbar_wait(&bar_mma1, li & 1, latch);
      tc_fence_after();
      {
        float ds[SW];
        tmem_ld32(t_dS + lane_off + sc0, ds);
        tmem_ld_wait();
        if (s_owner) {
          const float dec = decay_sm[s_row];
          gamma_acc *= dec;
#pragma unroll
          for (int c = 0; c < SW; ++c) S[c] = dec * S[c] + ds[c];
        }
      }
      tc_fence_before();
      __syncthreads();
      if (tid == 0 && li + 2 < nloc) issue_load(li + 2);
      continue;
    }

    // ---------------- gate math: one ex2 per (token, dim); decays from running products -------
    Gate gr;
    const bool weak = gr.run(st + 2 * L::RAW, DK, tot_sm);
    if (gr.h == 0) {
      decay_sm[gr.d] = gr.dec0;
      decay_sm[gr.d + 1] = gr.dec1;
    }
    const int safe = __syncthreads_or(weak);
    {
      const float inv0 = safe ? 1.f : 1.f / gr.dec0, inv1 = safe ? 1.f : 1.f / gr.dec1;
      const uint32_t blk = (gr.d >> 6) * (C * 128), col = gr.d & 63;
      gr.forward([&](int j, float e0, float e1) {
        const uint32_t wq = *reinterpret_cast<const uint32_t*>(st + (j * DK + gr.d) * 2);
        uint32_t hi, lo;
        split2(bf_lo(wq) * e0 * inv0, bf_hi(wq) * e1 * inv1, hi, lo);
        *reinterpret_cast<uint32_t*>(sm + L::QS_HI + blk + sw128(j, col)) = hi;
        *reinterpret_cast<uint32_t*>(sm + L::QS_LO + blk + sw128(j, col)) = lo;
      });
      gr.backward([&](int j, float e0, float e1) {
        const uint32_t wk = *reinterpret_cast<const uint32_t*>(st + L::RAW + (j * DK + gr.d) * 2);
        *reinterpret_cast<uint32_t*>(sm + L::KH + blk + sw128(j, col)) = pack2(bf_lo(wk) * e0, bf_hi(wk) * e1);
      });
    }
    // ---------------- state copy for the inter-chunk term: e^{gamma} S_i (or S_i in safe mode) ----
    if (s_owner) {
      const float sc = safe ? 1.f : decay_sm[s_row];
      float sv[SW];
#pragma unroll
      for (int c = 0; c < SW; ++c) sv[c] = S[c] * sc;
      store_half_split(sm + L::SB_HI, sm + L::SB_LO, s_row, sv, half);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---------------- MMA group 1: A, O = Qs S', dS = Kh^T V ----------------
    if (tid == 0) {
      const uint32_t base = smem_u32(sm);
      const uint32_t vbase = base + s * L::STAGE + 3 * L::RAW;
      constexpr uint32_t id_A = idesc_bf16_f32(C, C, false, false);
      constexpr uint32_t id_O = idesc_bf16_f32(C, DVT, false, true);
      constexpr uint32_t id_S = idesc_bf16_f32(DK, DVT, true, true);
#pragma unroll
      for (int k = 0; k < DK / 16; ++k) {
        const uint32_t koff = (k >> 2) * (C * 128) + (k & 3) * 32;
        const uint64_t kd = desc_sw128(base + L::KH + koff, 16, 1024);
        umma_bf16(t_A, desc_sw128(base + L::QS_HI + koff, 16, 1024), kd, id_A, k > 0);
        umma_bf16(t_A, desc_sw128(base + L::QS_LO + koff, 16, 1024), kd, id_A, 1);
      }
#pragma unroll
      for (int k = 0; k < DK / 16; ++k) {
        const uint32_t koff = (k >> 2) * (C * 128) + (k & 3) * 32;
        const uint64_t qh = desc_sw128(base + L::QS_HI + koff, 16, 1024);
        const uint64_t sh = desc_sw128(base + L::SB_HI + k * 2048, 16, 1024);
        umma_bf16(t_O, qh, sh, id_O, k > 0);
        umma_bf16(t_O, qh, desc_sw128(base + L::SB_LO + k * 2048, 16, 1024), id_O, 1);
        umma_bf16(t_O, desc_sw128(base + L::QS_LO + koff, 16, 1024), sh, id_O, 1);
      }
#pragma unroll
      for (int k = 0; k < C / 16; ++k)
        umma_bf16(t_dS, desc_sw128(base + L::KH + k * 2048, C * 128, 1024), desc_sw128(vbase + k * 2048, 16, 1024),
                  id_S, k > 0);
      umma_commit(&bar_mma1);
    }
    __syncwarp();
    mbar_wait(&bar_mma1, li & 1, latch);
    tc_fence_after();

    // ---------------- safe mode: exact intra-chunk matrix ----------------
    float* Aex = reinterpret_cast<float*>(sm + L::XA);  // 64 x 64 fp32
    if (safe) {
      float* Bf = reinterpret_cast<float*>(sm + L::XB);  // 64 x DK fp32 cumulative log-gates
      if (tid < DK) {
        float b = 0.f;
        for (int j = 0; j < C; ++j) {
          b += bf2f(st + 2 * L::RAW + (j * DK + tid) * 2);
          Bf[j * DK + tid] = b;
        }
      }
      __syncthreads();
      for (int e = tid; e < C * C; e += NTHREADS) {
        const int j = e / C, r = e % C;
        float acc = 0.f;
        if (r <= j)
          for (int d = 0; d < DK; ++d)
            acc += bf2f(st + (j * DK + d) * 2) * bf2f(st + L::RAW + (r * DK + d) * 2) *
                   __expf(Bf[j * DK + d] - Bf[r * DK + d]);
        Aex[e] = acc;
      }
      __syncthreads();
    }

    // ---------------- A epilogue: mask, hi/lo bf16, store as the K-major A operand ----------------
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
    }
    // ---------------- state update: S = e^gamma S + dS (fp32 registers) ----------------
    {
      float ds[SW];
      tmem_ld32(t_dS + lane_off + sc0, ds);
      tmem_ld_wait();
      if (s_owner) {
        const float dec = decay_sm[s_row];
#pragma unroll
        for (int c = 0; c < SW; ++c) S[c] = dec * S[c] + ds[c];
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---------------- MMA group 2: O += A V ----------------
    if (tid == 0) {
      const uint32_t base = smem_u32(sm);
      const uint32_t vbase = base + s * L::STAGE + 3 * L::RAW;
      constexpr uint32_t id_O = idesc_bf16_f32(C, DVT, false, true);
#pragma unroll
      for (int k = 0; k < C / 16; ++k) {
        const uint64_t vd = desc_sw128(vbase + k * 2048, 16, 1024);
        umma_bf16(t_O, desc_sw128(base + L::AB_HI + k * 32, 16, 1024), vd, id_O, 1);
        umma_bf16(t_O, desc_sw128(base + L::AB_LO + k * 32, 16, 1024), vd, id_O, 1);
      }
      umma_commit(&bar_mma2);
    }
    __syncwarp();
    mbar_wait(&bar_mma2, li & 1, latch);
    tc_fence_after();

    // ---------------- O epilogue: bf16 rows straight to global ----------------
    {
      const int j = q4 * 16 + lane, cb = half * 32;
      float ov[32];
      tmem_ld32(t_O + lane_off + cb, ov);
      tmem_ld_wait();
      const int t = i * C + j;
      if (lane < 16 && t < T) store_half_global_bf16(o + ((size_t)bh * T + t) * DV + dv0 + cb, ov);
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && li + 2 < nloc) issue_load(li + 2);
  }

  float* out = STATE_ONLY ? args.sbuf + ((size_t)bh * args.nseg + seg) * DK * DV
                          : (seg == args.nseg - 1 && args.hT ? args.hT + (size_t)bh * DK * DV : nullptr);
  if (s_owner && out) {
    float4* dst = reinterpret_cast<float4*>(out + (size_t)s_row * DV + dv0 + sc0);
#pragma unroll
    for (int c = 0; c < SW / 4; ++c) dst[c] = make_float4(S[4 * c], S[4 * c + 1], S[4 * c + 2], S[4 * c + 3]);
  }
  if (STATE_ONLY && s_owner && half == 0 && blockIdx.x == 0)
    args.gam[((size_t)bh * args.nseg + seg) * DK + s_row] = gamma_acc;
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

// ------------------------------------------------------------------------------------------
// Host entry points
// ------------------------------------------------------------------------------------------
bool fwd_supported(int BH, int T, int dk, int dv, int chunk, int dtype) {
  if (force_generic()) return false;
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

static int sm_count() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
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

template <int DK, bool STATE_ONLY>
static cudaError_t launch_fwd_pass(const CUtensorMap* m, const FwdArgs& args, int BH, int dv, int nz, cudaStream_t st) {
  auto kern = fwd_fused_kernel<DK, STATE_ONLY>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, FwdLayout<DK>::ALLOC);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 grid(dv / DVT, BH, nz);
  kern<<<grid, NTHREADS, FwdLayout<DK>::ALLOC, st>>>(m[0], m[1], m[2], m[3], args);
  return cudaGetLastError();
}

template <int DK>
static cudaError_t launch_fwd(const void* q, const void* k, const void* v, const void* g, const float* h0, void* o,
                              float* hT, int BH, int T, int dv, void* ws, cudaStream_t st) {
  CUtensorMap m[4];
  if (!make_map(&m[0], q, BH, T, DK, DK, false) || !make_map(&m[1], k, BH, T, DK, DK, false) ||
      !make_map(&m[2], g, BH, T, DK, DK, false) || !make_map(&m[3], v, BH, T, dv, DVT, true))
    return cudaErrorInvalidValue;
  FwdArgs a;
  a.h0 = h0;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.hT = hT;
  a.T = T;
  a.DV = dv;
  a.latch = device_error_latch();
  plan_segments(BH, T, dv, &a.nseg, &a.seg_chunks);
  a.sbuf = nullptr;
  a.gam = nullptr;
  if (a.nseg > 1) {
    if (!ws) return cudaErrorInvalidValue;
    a.sbuf = static_cast<float*>(ws);
    a.gam = a.sbuf + align256((size_t)BH * a.nseg * DK * dv * sizeof(float)) / sizeof(float);
    cudaError_t e = launch_fwd_pass<DK, true>(m, a, BH, dv, a.nseg - 1, st);
    if (e != cudaSuccess) return e;
    if (a.nseg > 2) {
      const size_t n = (size_t)BH * DK * dv;
      const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
      segment_scan_kernel<<<blocks, 256, 0, st>>>(a.sbuf, a.gam, BH, DK, dv, a.nseg);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
  }
  return launch_fwd_pass<DK, false>(m, a, BH, dv, a.nseg, st);
}

cudaError_t fwd(const void* q, const void* k, const void* v, const void* g, const float* h0, void* o, float* hT,
                int BH, int T, int dk, int dv, void* ws, cudaStream_t st) {
  if (dk == 64) return launch_fwd<64>(q, k, v, g, h0, o, hT, BH, T, dv, ws, st);
  if (dk == 128) return launch_fwd<128>(q, k, v, g, h0, o, hT, BH, T, dv, ws, st);
  return cudaErrorNotSupported;
}

}  // namespace fast
}  // namespace gla
