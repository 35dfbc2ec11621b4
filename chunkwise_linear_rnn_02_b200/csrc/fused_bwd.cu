// Fused sm_100a chunkwise GLA backward (bf16 in, fp32 accumulate, chunk 64, d_k = 128).
//
// Reverse-mode of the chunkwise recurrence.  With G_{i+1} = dL/dS at the end of chunk i
// (G_N = dhT), per chunk (B_j the inclusive cumulative log-gate, gamma = B_63, E1 = e^{B},
// E2 = e^{gamma - B}, dec = e^{gamma}, Kh = k E2, Qt = q E1, Qs = Qt / dec):
//
//   dA  = mask(dO V^T)                        A = mask(Qs Kh^T)
//   dq  = E1 (dO S_i^T) + (E1 / dec) (dA Kh)
//   dk  = E2 (V G_{i+1}^T) + (E2 / dec) (dA^T Qt)
//   dv  = Kh G_{i+1} + A^T dO
//   G_i = dec G_{i+1} + Qt^T dO               S_{i+1} = dec S_i + Kh^T V
//   dg: chunk-local parts plus a carry across chunk boundaries (the carry scan below), so that
//       no rounding accumulates over the sequence.
//
// Three launches on the caller's stream:
//   1. two kinds of CTA, independent of each other:
//      * key-tile CTAs, one per (head, 64 key dimensions): a forward walk that rebuilds S on chip
//        and writes dq, the forward part of dg and the chunk sums of Qt X (fp32, workspace), the
//        carry's start value rowsum(dhT * hT), and (the first key tile of a head) each chunk's
//        masked dA for the third launch;
//      * value-tile CTAs, one per (head, 128 value columns): a reverse walk carrying G[:, tile]
//        that writes dv, dh0[:, tile], and for every chunk this tile's part of Z^T = G V^T and of
//        the chunk sums of Kh Z (fp32, workspace; both are summed over the value tiles later);
//   2. a scan over chunks per (head, key dim) that turns the chunk sums into the carry c_i of
//      every chunk;
//   3. one CTA per (head, 64 key dimensions, chunk), all independent: dk and the rest of dg
//      from Z, the key tile's dA, the forward walk's part and c_i.
// Each CTA of the first launch has 8 compute warps and a ninth warp that issues its MMA groups.
// With few heads the chunks are cut into segments, each walked by its own key and value tiles:
// state-only passes and scans first give every segment its entry state S and its end gradient G
// (segment_states), and each segment's carry starts from rowsum(G_end * S_end) of the states its
// own walks used.
// States live in TMEM as fp32 accumulators; their bf16 hi / lo copies in shared memory feed the
// MMAs.  A chunk that keeps less than e^-40 of its state in some dimension computes its
// intra-chunk terms exactly in fp32 (CUDA cores) instead of through the scaled operands.  A
// compile-time variant reads column blocks of wider tensors and writes fp32 outputs (wide shapes
// run as blocks whose results are added afterwards).
#include "fast_path.cuh"
#include "fused_common.cuh"

namespace gla {
namespace fast {

using namespace sm100;

constexpr int BT = 256;  // compute threads per CTA: warps w and w+4 share TMEM lanes and split columns
// The walk kernel adds a ninth warp that issues the MMAs: tcgen05.mma issue holds the issuing thread
// for the group's execution, so the compute warps only hand over (named barriers kBarH1 / kBarH2:
// the compute threads arrive, the producer warp syncs) and wait for the groups' mbarriers.
constexpr int BTP = BT + 32;
constexpr int kBarH1 = 2, kBarH2 = 3, kBarH0 = 4;
constexpr int KT = 64;   // key dimensions per key-tile CTA
constexpr int VT = 128;  // value columns per value-tile CTA
// Per (head, chunk): the masked dA as the MMAs take it (bf16 hi and lo [64 x 64] tiles, 128-byte
// swizzled) and its fp32 diagonal, written by the first key tile for the chunk kernel.
constexpr uint32_t kDaBytes = 2 * C * KT * 2 + C * 4;

struct BwdMaps {
  CUtensorMap v, dO;                 // box (64 cols, 64 tokens), 128-byte swizzle
  CUtensorMap k64, g64, q64;         // box (64 dims, 64 tokens), 128-byte swizzle
  CUtensorMap q_all, k_all, g_all;   // box (DK dims, 64 tokens), plain
};

struct BwdArgs {
  const float* h0;
  const float* dhT;
  __nv_bfloat16 *dq, *dk, *dv, *dg;
  float* dh0;
  float* ws_qx;    // [BH][NC][DK] chunk sums of Qt X
  float* ws_carry; // [BH][nseg][DK] rowsum(G_end * S_end) per segment: where the dg carry starts
  float* ws_z;     // [BH][DV/VT][NC][64][DK] value tiles' parts of Z (token rows of DK dims)
  float* ws_kz;    // [BH][DV/VT][NC][2][DK] value tiles' parts of the chunk sums of Kh Z (per token half)
  float* ws_c;     // [BH][NC][DK] the dg carry c_i of every chunk
  float* ws_part;  // [BH][NC][64][DK] forward-walk part of dg, one row of DK dims per token
  uint8_t* ws_da;  // [BH][NC] blocks of kDaBytes: masked dA hi / lo tiles and diagonal
  int T;
  // Sequence split: nseg segments of seg_chunks chunks; s_in / g_end hold the segment states
  // ([BH][nseg][DK][DV] fp32: s_in[s-1] enters segment s, g_end[s] = dL/dS at the end of s).
  int nseg, seg_chunks, n_bh;
  const float *s_in, *g_end;
  long long st_bh, st_row;  // h0 / dhT / dh0 strides (a sub-block of a larger state when split)
  // FLEX builds: the inputs are column blocks of wider arrays, read in place by the tile loads: q,
  // k, g are [BH*T][pk] with this call's key dimensions from column ck, v and dO [BH*T][pv] with its
  // value columns from cv.  The gradients go in fp32 to acc_q / acc_k / acc_g ([BH*T][DK] each) and
  // acc_v ([BH*T][DV]) in place of the bf16 outputs; with acc_v null, dv goes in bf16 to the value
  // columns of dv, [BH*T][pv].
  float *acc_q, *acc_k, *acc_g, *acc_v;
  int pk, ck, pv, cv;
  // > 0: the gate tensor holds raw logits x (g = logsigmoid(x) / tau) and the gate-gradient output
  // receives dx = dg sigmoid(-x) / tau in place of dg
  float inv_tau;
  unsigned int* latch;
};


// ------------------------------------------------------------------------------------------
// Key-tile CTA
//
// Gate gradient, evaluated chunk by chunk so that rounding never accumulates over the sequence:
// for token t at local position tau of chunk i (Qt = q E1, Kh = k E2, X = dO S_i^T, Z = V G_{i+1}^T),
//   dg_t = c_i + sum_{r<tau} Kh_r Z_r + sum_{j>=tau} Qt_j X_j
//              + sum_{r<tau} ( k_r dk^intra_r - q_r dq^intra_r )        (intra terms without j = r)
//   c_i  = e^{gamma_i} rowsum(G_{i+1} * S_i), carried backwards over chunk boundaries as
//   c_{N-1} = rowsum(dhT * hT) - sum_r (Kh Z)_{N-1},  c_i = c_{i+1} + sum_j (Qt X)_{i+1} - sum_r (Kh Z)_i
//   (per segment when the sequence is split: G_end * S_end of the segment in place of dhT * hT).
// The forward walk writes the Qt X and q dq^intra parts (chunk-local, fp32) and the chunk sums of
// Qt X into the workspace; the value tiles write the chunk sums of Kh Z, the carry scan forms every
// c_i and the chunk kernel adds the rest.  The chunk sums use Qt and Kh as the G and S updates see
// them (bf16 hi + lo), so the recurrence for c telescopes for the states the kernels carry and its
// rounding does not accumulate over chunks.  Because the four parts of dg are several times
// larger than dg, every MMA operand is a bf16 hi + lo pair (three products per MMA, two where one
// side is exact), which keeps them near fp32 accuracy; the state copies feeding X and Z are split
// the same way, because the chunk sums they produce are carried over the whole sequence.
// ------------------------------------------------------------------------------------------
template <int DK, int DV>
struct KeyLayout {
  static constexpr uint32_t VB = C * DV * 2;        // a v or dO tile [64 x DV] (DV/64 swizzled boxes)
  static constexpr uint32_t TILE = C * KT * 2;      // a [64 x 64] bf16 tile
  static constexpr uint32_t PA_V = 0, PA_DO = VB;   // part A: v, dO (one buffer)
  static constexpr uint32_t PB = 2 * VB;            // part B: k, g, q tiles (two buffers)
  static constexpr uint32_t PB_STAGE = 3 * TILE;
  static constexpr uint32_t PB_K = 0, PB_G = TILE, PB_Q = 2 * TILE;  // offsets inside a part-B buffer
  static constexpr uint32_t KQ_HI = PB + 2 * PB_STAGE;  // Kh hi / lo
  static constexpr uint32_t KQ_LO = KQ_HI + TILE;
  static constexpr uint32_t SG_HI = KQ_LO + TILE;   // bf16 hi / lo copies of the S rows [64 x DV], K-major
  static constexpr uint32_t SG_LO = SG_HI + KT * DV * 2;
  static constexpr uint32_t DA_HI = SG_LO + KT * DV * 2;  // masked dA, bf16 hi / lo [64 x 64]
  static constexpr uint32_t DA_LO = DA_HI + TILE;
  static constexpr int NS = GateRun<KT, BT>::NSPLIT;
  static constexpr uint32_t XCH = DA_LO + TILE;         // float2 [2][64]: token-half sums exchanged per dim
  static constexpr uint32_t DEC = XCH + 2 * KT * 8;     // float [2][64]: chunk decays, per part-B buffer
  static constexpr uint32_t TOT = DEC + 2 * KT * 4;     // float [2][NS][64]: gate run products, per buffer
  static constexpr uint32_t DIAG = TOT + 2 * NS * KT * 4;
  static constexpr uint32_t CARRYP = DIAG + C * 4;      // [2][64] per-column-half partial row sums
  static constexpr uint32_t PRE = CARRYP + 2 * KT * 4;  // float [2][NS][64]: prefix products of TOT
  static constexpr uint32_t TOTAL = PRE + 2 * NS * KT * 4;
  static_assert(TOT % 8 == 0 && DEC % 8 == 0, "gate tables are read as float2");
  // TMEM columns
  static constexpr uint32_t T_SG = 0, T_DA = DV, T_X = DV + 64, T_Y = DV + 128;
  static_assert(DV + 192 <= 512, "TMEM columns");
  static_assert(PB % 1024 == 0 && PB_STAGE % 1024 == 0 && KQ_HI % 1024 == 0 && SG_HI % 1024 == 0 &&
                    DA_HI % 1024 == 0,
                "operand alignment");
};

// Key-tile schedule: chunk i's epilogue runs while chunk i+1's first MMA group is on the tensor
// pipe.  Per chunk step: wait for MMA group 1 of chunk i, move its dA and X^T rows into
// registers, issue group 2 (Y^T); then prepare chunk i+1 (gate run from the second part-B
// buffer, Kh operand, state copy and rescale) and issue its group 1; then finish chunk i's
// outputs.  The epilogue forms E1 / E2 itself from the raw gates and the run products of the gate
// run, multiplying in the same order, so its values equal the ones behind the MMA operands.
template <int DK, int DV, bool FLEX, bool LOGIT>
__device__ void key_tile_body(uint8_t* sm, const BwdMaps& mp, const BwdArgs& a, int bh, int tau, int seg,
                              uint64_t* bars, uint32_t tmem, int* safe_flag) {
  using L = KeyLayout<DK, DV>;
  using Gate = GateRun<KT, BT, LOGIT>;
  constexpr int NS = L::NS, TS = Gate::TS;
  static_assert(TS % 4 == 0, "token pairs u, u ^ 2 of the epilogue loads lie in one group");
  // column offsets into wider input tensors (FLEX builds only)
  const int col_k = FLEX ? a.ck : 0, col_v = FLEX ? a.cv : 0;
  static_assert(TS == 8 && NS == 8, "epilogue runs: four gate runs of eight tokens per token half");
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3, half = warp >> 2;  // TMEM lane quarter, column half
  const int T = a.T, NC = (T + C - 1) / C, d0 = tau * KT;
  const int ch0 = seg * a.seg_chunks, ch1 = min(NC, ch0 + a.seg_chunks);  // this segment's chunks
  const uint32_t base = smem_u32(sm);
  const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
  const bool row_owner = lane < 16;
  const int row = q4 * 16 + lane;  // row of an M=64 accumulator owned by this thread
  const int tb = half * 32;        // first column (token) of this thread's half
  constexpr int HV = DV / 2;       // state columns per warp
  uint64_t* bar_pa = bars + 0;
  uint64_t* bar_pb = bars + 1;     // two barriers, one per part-B buffer
  uint64_t* bar_m1 = bars + 3;
  uint64_t* bar_m2 = bars + 4;
  uint32_t ph_pa = 0, ph_pb = 0, ph_m1 = 0, ph_m2 = 0;
  float* DEC = reinterpret_cast<float*>(sm + L::DEC);
  float* TOT = reinterpret_cast<float*>(sm + L::TOT);
  float* PRE = reinterpret_cast<float*>(sm + L::PRE);
  float2* XCH = reinterpret_cast<float2*>(sm + L::XCH);
  float* DIAG = reinterpret_cast<float*>(sm + L::DIAG);
  float* qx_sums = a.ws_qx + (size_t)bh * NC * DK + d0;          // [NC][DK] slice of this head and key tile
  float* part = a.ws_part + (size_t)bh * NC * C * DK + d0;  // [NC][64][DK] slice: forward-walk part of dg

  auto pbo = [&](int b) { return L::PB + (uint32_t)b * L::PB_STAGE; };
  auto load_a = [&](int chunk) {
    mbar_arrive_expect_tx(bar_pa, 2 * L::VB);
    for (int bb = 0; bb < DV / 64; ++bb) {
      tma_load_3d(sm + L::PA_V + bb * (C * 128), &mp.v, bar_pa, col_v + bb * 64, chunk * C, bh);
      tma_load_3d(sm + L::PA_DO + bb * (C * 128), &mp.dO, bar_pa, col_v + bb * 64, chunk * C, bh);
    }
  };
  auto load_b = [&](int chunk, int b) {
    uint8_t* pb = sm + pbo(b);
    mbar_arrive_expect_tx(bar_pb + b, L::PB_STAGE);
    tma_load_3d(pb + L::PB_K, &mp.k64, bar_pb + b, col_k + d0, chunk * C, bh);
    tma_load_3d(pb + L::PB_G, &mp.g64, bar_pb + b, col_k + d0, chunk * C, bh);
    tma_load_3d(pb + L::PB_Q, &mp.q64, bar_pb + b, col_k + d0, chunk * C, bh);
  };
  auto wait_b = [&](int b) {
    mbar_wait(bar_pb + b, (ph_pb >> b) & 1u, a.latch);
    ph_pb ^= 1u << b;
  };
  // operands in shared memory / TMEM are complete: hand them to the producer warp
  auto handoff = [&](int id) {
    fence_async_smem();
    tc_fence_before();
    bar_arrive(id, BTP);
  };
  // Element (token j, dim d) of a raw tile at shared-memory offset off (TMA 128-byte swizzle).
  auto raw = [&](uint32_t off, int j, int d) { return bf2f(sm + off + sw128(j, d)); };
  // dA (masked, as the MMAs see it: hi + lo) at (j, r).
  auto dA_at = [&](int j, int r) { return raw(L::DA_HI, j, r) + raw(L::DA_LO, j, r); };
  // Gate run of the chunk in part-B buffer b: run products into TOT[b], decays into DEC[b].
  auto gate = [&](Gate& gr, int b, int chunk) {
    if constexpr (LOGIT) gr.set_logit(a.inv_tau, T - chunk * C);
    const bool weak = gr.run_swizzled(sm + pbo(b) + L::PB_G, TOT + b * NS * KT);
    if (gr.h == 0) gr.store_decay(DEC + b * KT);
    return bar_or(kBarCompute, BT, weak);
  };
  auto write_kq = [&](uint32_t w, int j, int d, float e0, float e1) {
    uint32_t hi, lo;
    split2(bf_lo(w) * e0, bf_hi(w) * e1, hi, lo);
    *reinterpret_cast<uint32_t*>(sm + L::KQ_HI + sw128(j, d)) = hi;
    *reinterpret_cast<uint32_t*>(sm + L::KQ_LO + sw128(j, d)) = lo;
  };
  // Initialise the TMEM state rows from a [DK x DV] fp32 source with row stride srow (or zeros).
  auto init_state = [&](const float* src, long long srow) {
    float v[64];
    for (int c0 = half * HV; c0 < (half + 1) * HV; c0 += 64) {
#pragma unroll
      for (int c = 0; c < 64; ++c) v[c] = (src && row_owner) ? src[(d0 + row) * srow + c0 + c] : 0.f;
      tmem_st32(tmem + L::T_SG + lane_off + c0, v);
      tmem_st32(tmem + L::T_SG + lane_off + c0 + 32, v + 32);
    }
    tmem_st_wait();
  };
  // TMEM state rows -> hi/lo bf16 K-major operand copy; then the rows scaled by DEC[b] (all lanes
  // take part; only owners' rows matter).
  // The copy uses all 32 lanes, 32 columns at a time: lane l < 16 stores columns 0-15 of its row's
  // piece, lane l + 16 columns 16-31 of the same row, received by shuffle (the M = 64 accumulator
  // leaves TMEM lanes 16-31 empty, so those lanes' own values are unused).
  auto state_pass = [&](int b) {
    const float sc = row_owner ? DEC[b * KT + row] : 0.f;
    const int sub = lane >> 4, srow = q4 * 16 + (lane & 15);
    float v[32];
    for (int c0 = half * HV; c0 < (half + 1) * HV; c0 += 32) {
      tmem_ld32(tmem + L::T_SG + lane_off + c0, v);
      tmem_ld_wait();
      float u[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float x = __shfl_sync(0xffffffffu, v[16 + c], lane & 15);
        u[c] = sub ? x : v[c];
      }
      store_quarter_split(sm + L::SG_HI + (c0 / 64) * (KT * 128), sm + L::SG_LO + (c0 / 64) * (KT * 128), srow, u,
                          ((c0 & 63) >> 4) + sub);
#pragma unroll
      for (int c = 0; c < 32; ++c) v[c] *= sc;
      tmem_st32(tmem + L::T_SG + lane_off + c0, v);
    }
    tmem_st_wait();
  };
  // dA epilogue: masked bf16 hi / lo operand and its diagonal.
  auto dA_epilogue = [&]() {
    float v[32];
    tmem_ld32(tmem + L::T_DA + lane_off + tb, v);
    tmem_ld_wait();
    if (row_owner) {
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        if (tb + c > row) v[c] = 0.f;
        if (tb + c == row) DIAG[row] = v[c];
      }
      store_half_split(sm + L::DA_HI, sm + L::DA_LO, row, v, half);
    }
  };
  // MMA group 1 (producer lane 0): dA = dO V^T, X^T = S dO^T and the state update S += Kh^T V.
  auto issue_m1 = [&]() {
    mbar_wait(bar_pa, ph_pa, a.latch);
    ph_pa ^= 1;
    tc_fence_after();
    constexpr uint32_t id_dA = idesc_bf16_f32(C, C, false, false);
    constexpr uint32_t id_X = idesc_bf16_f32(KT, C, false, false);
    constexpr uint32_t id_S = idesc_bf16_f32(KT, DV, true, true);
#pragma unroll
    for (int k = 0; k < DV / 16; ++k) {
      const uint32_t ko = (k >> 2) * (C * 128) + (k & 3) * 32;
      const uint64_t bd = desc_sw128(base + L::PA_DO + ko, 16, 1024);
      umma_bf16(tmem + L::T_DA, desc_sw128(base + L::PA_DO + ko, 16, 1024),
                desc_sw128(base + L::PA_V + ko, 16, 1024), id_dA, k > 0);
      umma_bf16(tmem + L::T_X, desc_sw128(base + L::SG_HI + ko, 16, 1024), bd, id_X, k > 0);
      umma_bf16(tmem + L::T_X, desc_sw128(base + L::SG_LO + ko, 16, 1024), bd, id_X, 1);
    }
#pragma unroll
    for (int k = 0; k < C / 16; ++k) {
      const uint64_t dd = desc_sw128(base + L::PA_V + k * 2048, C * 128, 1024);
      umma_bf16(tmem + L::T_SG, desc_sw128(base + L::KQ_HI + k * 2048, C * 128, 1024), dd, id_S, 1);
      umma_bf16(tmem + L::T_SG, desc_sw128(base + L::KQ_LO + k * 2048, C * 128, 1024), dd, id_S, 1);
    }
    umma_commit(bar_m1);
  };
  // MMA group 2 (producer lane 0): Y^T = Kh^T dA^T.
  auto issue_m2 = [&]() {
    constexpr uint32_t id_Y = idesc_bf16_f32(KT, C, true, false);
#pragma unroll
    for (int k = 0; k < C / 16; ++k) {
      const uint64_t ah = desc_sw128(base + L::KQ_HI + k * 2048, C * 128, 1024);
      const uint64_t al = desc_sw128(base + L::KQ_LO + k * 2048, C * 128, 1024);
      const uint64_t bh = desc_sw128(base + L::DA_HI + k * 32, 16, 1024);
      const uint64_t bl = desc_sw128(base + L::DA_LO + k * 32, 16, 1024);
      umma_bf16(tmem + L::T_Y, ah, bh, id_Y, k > 0);
      umma_bf16(tmem + L::T_Y, al, bh, id_Y, 1);
      umma_bf16(tmem + L::T_Y, ah, bl, id_Y, 1);
    }
    umma_commit(bar_m2);
  };
  auto wait_m2 = [&]() {
    mbar_wait(bar_m2, ph_m2, a.latch);
    ph_m2 ^= 1;
    tc_fence_after();
  };
  // Chunk i+1: gate run from buffer nb, Kh operand, state copy + rescale, then group 1 (handed to
  // the producer with the chunk's exact-path flag).  The operand area KQ is free once group 2 of
  // the current chunk has completed.
  auto prepare = [&](int nb, int m2_pending, int chunk) {
    wait_b(nb);
    Gate gr;
    const int safe = gate(gr, nb, chunk);
    if (tid < KT) {  // E1 at each token group's start, multiplied in the order the epilogue used
      float* pre = PRE + nb * NS * KT;
      const float* tot = TOT + nb * NS * KT;
      float e = 1.f;
#pragma unroll
      for (int hh = 0; hh < NS; ++hh) {
        pre[hh * KT + tid] = e;
        e *= tot[hh * KT + tid];
      }
    }
    uint32_t w[Gate::TS];
    gr.load_pairs(sm + pbo(nb) + L::PB_K, KT, true, w);
    if (m2_pending) wait_m2();
    gr.backward([&](int j, float e0, float e1) { write_kq(w[j - gr.h * Gate::TS], j, gr.d, e0, e1); });
    state_pass(nb);
    if (tid == 0) safe_flag[nb] = safe;
    handoff(kBarH1);
    return safe;
  };

  if (tid >= BT) {  // ======== producer warp: the MMA groups, in the order the compute threads hand over
    bar_sync(kBarH1, BTP);
    tc_fence_after();
    if (lane == 0) issue_m1();
    __syncwarp();
    for (int i = ch0; i < ch1; ++i) {
      const int b = (i - ch0) & 1;
      bar_sync(kBarH2, BTP);  // chunk i's dA operand is in shared memory
      tc_fence_after();
      if (lane == 0) {
        if (!safe_flag[b]) issue_m2();
        if (tau == 0) {  // dA and its diagonal for the chunk kernel (one key tile per head writes)
          uint8_t* dst = a.ws_da + ((size_t)bh * NC + i) * kDaBytes;
          bulk_s2g(dst, sm + L::DA_HI, 2 * L::TILE);
          bulk_s2g(dst + 2 * L::TILE, sm + L::DIAG, C * 4);
          tma_store_commit();
        }
      }
      __syncwarp();
      if (i + 1 < ch1) {
        bar_sync(kBarH1, BTP);  // chunk i+1's Kh and state copy are in shared memory
        tc_fence_after();
        if (lane == 0) {
          // the copies have read dA before group 1 of chunk i+1 is issued, whose completion the
          // compute threads wait for before they write chunk i+1's dA
          if (tau == 0) tma_store_wait_read_all();
          issue_m1();
        }
        __syncwarp();
      }
    }
    if (lane == 0 && tau == 0) tma_store_wait_all();  // written before the CTA exits
    return;
  }

  // ================================ forward walk: dq, first part of dg ================================
  if (tid == 0) {
    load_a(ch0);
    load_b(ch0, 0);
    if (ch1 - ch0 > 1) load_b(ch0 + 1, 1);
  }
  if (seg == 0)
    init_state(a.h0 ? a.h0 + bh * a.st_bh : nullptr, a.st_row);
  else
    init_state(a.s_in + ((size_t)bh * a.nseg + seg - 1) * DK * DV, DV);
  int safe_next = prepare(0, 0, ch0);
  for (int i = ch0; i < ch1; ++i) {
    const int b = (i - ch0) & 1, safe = safe_next;
    mbar_wait(bar_m1, ph_m1, a.latch);
    ph_m1 ^= 1;
    tc_fence_after();
    if (tid == 0 && i + 1 < ch1) load_a(i + 1);
    float x[32];  // this thread's row of X^T: key dim d = row, tokens tb .. tb+31
    tmem_ld32(tmem + L::T_X + lane_off + tb, x);
    dA_epilogue();
    handoff(kBarH2);  // group 2 (chunk off the exact path)
    // dA and DIAG of every thread are read below: the gate run's barrier in prepare orders them, or
    // this one after the last chunk
    if (i + 1 < ch1) {
      safe_next = prepare(b ^ 1, !safe, i + 1);
    } else {
      bar_sync(kBarCompute, BT);
      if (!safe) wait_m2();
    }
    float y[32];  // this thread's row of Y^T
    if (!safe) {
      tmem_ld32(tmem + L::T_Y + lane_off + tb, y);
      tmem_ld_wait();
    }
    // The M = 64 accumulators sit in TMEM lanes 0-15 of each quarter.  Split the row's 32 tokens
    // over the warp: lane l < 16 keeps tokens tb .. tb+15 of key dim q4*16 + l, lane l + 16 takes
    // tokens tb+16 .. tb+31 of the same dim (by shuffle), so that every lane works on 16 tokens.
    const int sub = lane >> 4, tq = tb + sub * 16, d = q4 * 16 + (lane & 15);
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const float xv = __shfl_sync(0xffffffffu, x[16 + c], lane & 15);
      if (sub) x[c] = xv;
    }
    if (!safe) {  // (on the exact path y is formed below, per token)
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float yv = __shfl_sync(0xffffffffu, y[16 + c], lane & 15);
        if (sub) y[c] = yv;
      }
    }
    float tot_s = 0.f, tot_e = 0.f;
    {  // dq; per-token terms Qt X (-> x) and q dq^intra without j = r (-> y)
      const uint32_t pk = pbo(b) + L::PB_K, pg = pbo(b) + L::PB_G, pq = pbo(b) + L::PB_Q;
      if (safe) {  // exact intra term y_j = sum_{r<=j} dA_jr k_r e^{B_j - B_r}
        float bj = 0.f;
        for (int t = 0; t < tq; ++t) bj += raw(pg, t, d);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          bj += raw(pg, tq + c, d);
          float acc = 0.f, br = 0.f;
          for (int r = 0; r <= tq + c; ++r) {
            br += raw(pg, r, d);
            acc += dA_at(tq + c, r) * raw(pk, r, d) * __expf(bj - br);
          }
          y[c] = acc;
        }
      }
      const float inv = 1.f / DEC[b * KT + d];
      __nv_bfloat16* dst = a.dq + ((size_t)bh * T + i * C + tq) * DK + d0 + d;
      float* dst32 = FLEX ? a.acc_q + ((size_t)bh * T + i * C + tq) * DK + d0 + d : nullptr;
#pragma unroll
      for (int rr = 0; rr < 16 / TS; ++rr) {
        // The group's raw g, q and k values.  Lanes 16-31 read token rows 16 below those of lanes
        // 0-15, which the 128-byte swizzle puts on the same banks; so at load step u they read
        // token u ^ 2 of their group (the other 32-byte half of the row), and the values are put
        // back in token order once loaded.
        float gl[TS], ql[TS], kl[TS];
#pragma unroll
        for (int u = 0; u < TS; ++u) {
          const int j = tq + rr * TS + (u ^ (2 * sub));
          gl[u] = raw(pg, j, d);
          ql[u] = raw(pq, j, d);
          kl[u] = raw(pk, j, d);
        }
        // E1 = e^{B_j}, formed as GateRun::forward forms it: the earlier groups' run products, then
        // this group's factors one token at a time
        float e = PRE[(b * NS + tq / TS + rr) * KT + d];
#pragma unroll
        for (int u = 0; u < TS; ++u) {
          const int c = rr * TS + u, j = tq + c;
          e *= ex2((sub ? gl[u ^ 2] : gl[u]) * kLog2e);
          if (!safe) y[c] *= e * inv;
          const float qv = sub ? ql[u ^ 2] : ql[u], kv = sub ? kl[u ^ 2] : kl[u];
          if (i * C + j < T) {
            if constexpr (FLEX)
              dst32[(size_t)c * DK] = e * x[c] + y[c];
            else
              dst[(size_t)c * DK] = __float2bfloat16_rn(e * x[c] + y[c]);
          }
          x[c] = bf_split_sum(qv * e) * x[c];  // Qt X, with Qt as the G update sees it
          y[c] = qv * (y[c] - DIAG[j] * kv);   // q dq^intra without j = r
          tot_s += x[c];
          tot_e += y[c];
        }
      }
    }
    // sums over the other 16 tokens of this half (the partner lane) and over the other half (XCH)
    const float part_s = __shfl_xor_sync(0xffffffffu, tot_s, 16), part_e = __shfl_xor_sync(0xffffffffu, tot_e, 16);
    if (!sub) XCH[half * KT + d] = make_float2(tot_s + part_s, tot_e + part_e);
    bar_sync(kBarCompute, BT);
    if (tid == 0 && i + 2 < ch1) load_b(i + 2, b);
    {  // part = suffix (inclusive) of Qt X minus prefix (exclusive) of q dq^intra
      const float2 o = XCH[(half ^ 1) * KT + d];
      float suf = (half == 0 ? o.x : 0.f) + (sub == 0 ? part_s : 0.f);
      float pre = (half == 1 ? o.y : 0.f) + (sub == 1 ? part_e : 0.f);
#pragma unroll
      for (int c = 15; c >= 0; --c) {
        suf += x[c];
        x[c] = suf;
      }
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        x[c] -= pre;
        pre += y[c];
      }
      // token-major rows: the lanes (consecutive dims) store adjacent words
      float* dst = part + ((size_t)i * C + tq) * DK + d;
#pragma unroll
      for (int c = 0; c < 16; ++c) dst[(size_t)c * DK] = x[c];
      if (half == 0 && sub == 0) qx_sums[(size_t)i * DK + d] = suf;
    }
  }

  // rowsum(G_end * S_end): S_end rows = the state after this segment's walk, G_end = dhT for the
  // last segment, else the gradient at the segment's end from the segment scan
  {
    float* CARRYP = reinterpret_cast<float*>(sm + L::CARRYP);
    const bool last = seg == a.nseg - 1;
    const float* gsrc = last ? (a.dhT ? a.dhT + bh * a.st_bh : nullptr)
                             : a.g_end + ((size_t)bh * a.nseg + seg) * DK * DV;
    const long long grs = last ? a.st_row : DV;
    float v[32];
    float acc = 0.f;
    for (int c0 = half * HV; c0 < (half + 1) * HV; c0 += 32) {
      tmem_ld32(tmem + L::T_SG + lane_off + c0, v);
      tmem_ld_wait();
      if (row_owner && gsrc) {
        const float* src = gsrc + (d0 + row) * grs + c0;
#pragma unroll
        for (int c = 0; c < 32; ++c) acc += src[c] * v[c];
      }
    }
    if (row_owner) CARRYP[half * KT + row] = acc;
    bar_sync(kBarCompute, BT);
    if (tid < KT) a.ws_carry[((size_t)bh * a.nseg + seg) * DK + d0 + tid] = CARRYP[tid] + CARRYP[KT + tid];
  }
}

// ------------------------------------------------------------------------------------------
// Value-tile CTA: reverse walk carrying G[:, tile] (fp32, TMEM); dv = Kh G_{i+1} + A^T dO, formed
// transposed (dv^T = G^T Kh^T + dO^T A: 128 value columns on the MMA's M axis, 64 tokens on N,
// because an M = 64 MMA takes as long as an M = 128 one).
// Qs, Kh, the G copy and A enter the MMAs as bf16 hi + lo pairs.  One array holds the queries of
// both A and the G update: Qs = Qt / dec (then G <- dec (G + Qs^T dO)), or Qt itself in a chunk on
// the exact path (then G <- dec G + Qt^T dO, the intra-chunk A computed exactly in fp32).
// ------------------------------------------------------------------------------------------
template <int DK>
struct ValLayout {
  static constexpr uint32_t RAW = C * DK * 2;       // q, k, g [64][DK] row-major
  static constexpr uint32_t DOT = C * VT * 2;       // dO tile, VT/64 swizzled boxes
  static constexpr uint32_t STAGE = 3 * RAW + DOT;  // single-buffered
  static constexpr uint32_t QP_HI = STAGE;          // Qs (or Qt) hi / lo [64 x DK] K-major
  static constexpr uint32_t QP_LO = QP_HI + C * DK * 2;
  static constexpr uint32_t KH_HI = QP_LO + C * DK * 2;  // Kh hi / lo [64 x DK] K-major
  static constexpr uint32_t KH_LO = KH_HI + C * DK * 2;
  static constexpr uint32_t GC_HI = KH_LO + C * DK * 2;  // G[:, tile] copy hi / lo [DK rows x VT] MN-major
  static constexpr uint32_t GC_LO = GC_HI + DK * VT * 2;
  static constexpr uint32_t AB_HI = GC_LO + DK * VT * 2;  // A hi / lo [64 x 64]
  static constexpr uint32_t AB_LO = AB_HI + C * C * 2;
  static constexpr uint32_t DEC = AB_LO + C * C * 2;
  static constexpr uint32_t TOT = DEC + DK * 4;
  static constexpr uint32_t TOTAL = TOT + GateRun<DK, BT>::NSPLIT * DK * 4;
  static_assert(TOT % 8 == 0 && DEC % 8 == 0, "gate tables are read as float2");
  static constexpr uint32_t XB = QP_HI, XA = KH_HI;  // exact-path scratch (after the first MMA group)
  // v tile [64 x VT] for Z^T = G V^T: read by the Z^T MMAs only, which complete before the A
  // commit (MMAs of one thread complete in order), so it shares A's space
  static constexpr uint32_t VZ = AB_HI;
  // dv^T takes 64 columns, double-buffered by chunk parity (its epilogue runs during the next chunk)
  static constexpr uint32_t T_G = 0, T_A = VT, T_DV = VT + 64, T_Z = 2 * VT + 64;
  static_assert(T_DV + 128 <= T_Z, "two dv^T buffers");
  static_assert(C * VT * 2 <= DEC - AB_HI && T_Z + 64 <= 512, "v tile / TMEM columns");
  static_assert(STAGE % 1024 == 0, "stage alignment");
  static_assert(C * DK * 4 <= KH_HI - QP_HI && C * C * 4 <= GC_HI - KH_HI, "exact-path scratch");
};

template <int DK, bool FLEX, bool LOGIT>
__device__ void val_tile_body(uint8_t* sm, const BwdMaps& mp, const BwdArgs& a, int bh, int vt, int DV, int seg,
                              uint64_t* bars, uint32_t tmem, int* safe_flag) {
  using L = ValLayout<DK>;
  using Gate = GateRun<DK, BT, LOGIT>;
  // column offsets into wider tensors and the value-side row pitch (FLEX builds only)
  const int col_k = FLEX ? a.ck : 0, col_v = FLEX ? a.cv : 0, pitch_v = FLEX ? a.pv : DV;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = a.T, NC = (T + C - 1) / C, c0 = vt * VT;
  const int ch0 = seg * a.seg_chunks, ch1 = min(NC, ch0 + a.seg_chunks), nl = ch1 - ch0;  // segment
  const uint32_t base = smem_u32(sm);
  const int q4 = warp & 3, half = warp >> 2;  // TMEM lane quarter, column half
  const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
  const bool row_owner = lane < 16;
  const int row = q4 * 16 + lane;   // row of an M=64 accumulator
  const int grow = q4 * 32 + lane;  // row of the M=128 G accumulator
  constexpr int HT = VT / 2;        // G columns per warp
  uint64_t* bar_ld = bars + 0;  // q, k, g of a chunk
  uint64_t* bar_dv = bars + 1;  // dO, v of a chunk
  uint64_t* bar_m1 = bars + 3;
  uint64_t* bar_m2 = bars + 4;
  uint64_t* bar_mA = bars + 5;  // the A MMAs (and, completing before them, the Z^T part)
  uint64_t* bar_mZ = bars + 6;  // the Z^T part alone
  uint32_t ph_ld = 0, ph_dv = 0, ph_m1 = 0, ph_m2 = 0, ph_mA = 0, ph_mZ = 0;
  float* DEC = reinterpret_cast<float*>(sm + L::DEC);
  float* TOT = reinterpret_cast<float*>(sm + L::TOT);

  // q, k, g are read only by the gate run (and the exact path), so the next chunk's copies are
  // issued as soon as those reads are done; dO and v once the second MMA group has completed.
  auto load_qkg = [&](int chunk) {
    mbar_arrive_expect_tx(bar_ld, 3 * L::RAW);
    tma_load_3d(sm, &mp.q_all, bar_ld, col_k, chunk * C, bh);
    tma_load_3d(sm + L::RAW, &mp.k_all, bar_ld, col_k, chunk * C, bh);
    tma_load_3d(sm + 2 * L::RAW, &mp.g_all, bar_ld, col_k, chunk * C, bh);
  };
  auto load_dov = [&](int chunk) {
    mbar_arrive_expect_tx(bar_dv, L::DOT + C * VT * 2);
    for (int b = 0; b < VT / 64; ++b) {
      tma_load_3d(sm + 3 * L::RAW + b * (C * 128), &mp.dO, bar_dv, col_v + c0 + b * 64, chunk * C, bh);
      tma_load_3d(sm + L::VZ + b * (C * 128), &mp.v, bar_dv, col_v + c0 + b * 64, chunk * C, bh);
    }
  };
  // operands in shared memory / TMEM are complete: hand them to the producer warp
  auto handoff = [&](int id) {
    fence_async_smem();
    tc_fence_before();
    bar_arrive(id, BTP);
  };
  // G <- DEC[row] * G for this thread's row of the M=128 accumulator.
  auto rescale_G = [&]() {
    const float sc = DEC[grow];
    float v[32];
    for (int cb = half * HT; cb < (half + 1) * HT; cb += 32) {
      tmem_ld32(tmem + L::T_G + lane_off + cb, v);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 32; ++c) v[c] *= sc;
      tmem_st32(tmem + L::T_G + lane_off + cb, v);
    }
    tmem_st_wait();
  };
  // Z^T part of this value tile (producer lane 0): G_{i+1}[:, tile] V[:, tile]^T with the G copy
  // hi + lo.  It needs only the G copy and the v tile, so it is issued as soon as the previous
  // chunk's G pass has handed over; the A commit that follows covers it (MMAs of one thread
  // complete in order), which matters because the v tile shares A's space.
  auto issue_z = [&]() {
    constexpr uint32_t id_Z = idesc_bf16_f32(DK, C, false, false);
#pragma unroll
    for (int k = 0; k < VT / 16; ++k) {
      const uint32_t ko = (k >> 2) * (DK * 128) + (k & 3) * 32;
      const uint64_t vd = desc_sw128(base + L::VZ + (k >> 2) * (C * 128) + (k & 3) * 32, 16, 1024);
      umma_bf16(tmem + L::T_Z, desc_sw128(base + L::GC_HI + ko, 16, 1024), vd, id_Z, k > 0);
      umma_bf16(tmem + L::T_Z, desc_sw128(base + L::GC_LO + ko, 16, 1024), vd, id_Z, 1);
    }
    umma_commit(bar_mZ);
  };
  // MMA group 1 (producer lane 0): A (first commit, with the Z^T part before it), dv^T = G^T Kh^T
  // and the G update
  auto issue_g1 = [&](int n) {
    const uint32_t dob = base + 3 * L::RAW, t_dv = tmem + L::T_DV + (n & 1) * 64;
    constexpr uint32_t id_A = idesc_bf16_f32(C, C, false, false);
    constexpr uint32_t id_dv = idesc_bf16_f32(VT, C, true, false);  // dv^T = G^T Kh^T: value columns on M
    constexpr uint32_t id_G = idesc_bf16_f32(DK, VT, true, true);
#pragma unroll
    for (int k = 0; k < DK / 16; ++k) {
      const uint32_t ko = (k >> 2) * (C * 128) + (k & 3) * 32;
      const uint64_t qh = desc_sw128(base + L::QP_HI + ko, 16, 1024), ql = desc_sw128(base + L::QP_LO + ko, 16, 1024);
      const uint64_t kh = desc_sw128(base + L::KH_HI + ko, 16, 1024), kl = desc_sw128(base + L::KH_LO + ko, 16, 1024);
      umma_bf16(tmem + L::T_A, qh, kh, id_A, k > 0);
      umma_bf16(tmem + L::T_A, qh, kl, id_A, 1);
      umma_bf16(tmem + L::T_A, ql, kh, id_A, 1);
    }
    umma_commit(bar_mA);
    // dv^T = G^T Kh^T and the G update: the A epilogue runs while they execute
#pragma unroll
    for (int k = 0; k < DK / 16; ++k) {
      const uint32_t ko = (k >> 2) * (C * 128) + (k & 3) * 32;
      const uint64_t kh = desc_sw128(base + L::KH_HI + ko, 16, 1024), kl = desc_sw128(base + L::KH_LO + ko, 16, 1024);
      const uint64_t gh = desc_sw128(base + L::GC_HI + k * 2048, DK * 128, 1024);
      umma_bf16(t_dv, gh, kh, id_dv, k > 0);
      umma_bf16(t_dv, desc_sw128(base + L::GC_LO + k * 2048, DK * 128, 1024), kh, id_dv, 1);
      umma_bf16(t_dv, gh, kl, id_dv, 1);
    }
#pragma unroll
    for (int k = 0; k < C / 16; ++k) {
      const uint64_t dd = desc_sw128(dob + k * 2048, C * 128, 1024);
      umma_bf16(tmem + L::T_G, desc_sw128(base + L::QP_HI + k * 2048, C * 128, 1024), dd, id_G, 1);
      umma_bf16(tmem + L::T_G, desc_sw128(base + L::QP_LO + k * 2048, C * 128, 1024), dd, id_G, 1);
    }
    umma_commit(bar_m1);
  };
  // MMA group 2 (producer lane 0): dv^T += dO^T A
  auto issue_g2 = [&](int n) {
    const uint32_t dob = base + 3 * L::RAW, t_dv = tmem + L::T_DV + (n & 1) * 64;
    constexpr uint32_t id_dv2 = idesc_bf16_f32(VT, C, true, true);  // dv^T += dO^T A
#pragma unroll
    for (int k = 0; k < C / 16; ++k) {
      const uint64_t dd = desc_sw128(dob + k * 2048, C * 128, 1024);
      umma_bf16(t_dv, dd, desc_sw128(base + L::AB_HI + k * 2048, C * 128, 1024), id_dv2, 1);
      umma_bf16(t_dv, dd, desc_sw128(base + L::AB_LO + k * 2048, C * 128, 1024), id_dv2, 1);
    }
    umma_commit(bar_m2);
  };

  if (tid >= BT) {  // ======== producer warp: the MMA groups and the loads that wait for a handoff
    // the Z^T part of chunk i: after the G copy's handoff (H0) and the arrival of chunk i's v tile
    auto z_part = [&]() {
      bar_sync(kBarH0, BTP);
      tc_fence_after();
      if (lane == 0) {
        mbar_wait(bar_dv, ph_dv, a.latch);
        ph_dv ^= 1;
        tc_fence_after();
        issue_z();
      }
      __syncwarp();
    };
    if (nl > 0) z_part();
    for (int n = 0; n < nl; ++n) {
      const int i = ch1 - 1 - n;
      bar_sync(kBarH1, BTP);  // chunk i's Qs, Kh (and rescaled G) are ready
      tc_fence_after();
      const int safe = safe_flag[0];
      if (lane == 0) {
        issue_g1(n);
        if (!safe && n + 1 < nl) load_qkg(i - 1);  // the raw q, k, g tiles have been read
      }
      __syncwarp();
      bar_sync(kBarH2, BTP);  // chunk i's A operand is in shared memory
      tc_fence_after();
      if (lane == 0) {
        if (safe && n + 1 < nl) load_qkg(i - 1);  // the exact path has read the raw tiles
        issue_g2(n);
        if (n + 1 < nl) {  // dO and v (over A) are free once group 2 has completed
          mbar_wait(bar_m2, ph_m2, a.latch);
          ph_m2 ^= 1;
          load_dov(i - 1);
        }
      }
      __syncwarp();
      if (n + 1 < nl) z_part();  // chunk i-1's Z^T part, after chunk i's G pass
    }
    return;
  }
  // G rows (this thread owns row grow of the M=128 accumulator): init from dhT[:, tile] (last
  // segment) or from the gradient at the segment's end
  {
    const bool last = seg == a.nseg - 1;
    const float* gsrc = last ? (a.dhT ? a.dhT + bh * a.st_bh + grow * a.st_row : nullptr)
                             : a.g_end + (((size_t)bh * a.nseg + seg) * DK + grow) * DV;
    float v[64];
    for (int cb = half * HT; cb < (half + 1) * HT; cb += 64) {
#pragma unroll
      for (int c = 0; c < 64; ++c) v[c] = gsrc ? gsrc[c0 + cb + c] : 0.f;
      tmem_st32(tmem + L::T_G + lane_off + cb, v);
      tmem_st32(tmem + L::T_G + lane_off + cb + 32, v + 32);
      store_row_split(sm + L::GC_HI + (cb / 64) * (DK * 128), sm + L::GC_LO + (cb / 64) * (DK * 128), grow, v, 1.f);
    }
    tmem_st_wait();
  }
  if (tid == 0) {
    load_qkg(ch1 - 1);
    load_dov(ch1 - 1);
  }
  if (nl > 0) handoff(kBarH0);  // the G copy: the first chunk's Z^T part
  // dv epilogue of chunk ic from dv^T buffer buf (its group 2 has completed): row vcol of dv^T (value
  // column c0 + vcol), tokens half*32 .. half*32+31; a warp's store covers 32 adjacent value columns
  // of one token.  It runs during the next chunk's first MMA group.
  auto dv_epilogue = [&](int ic, int buf) {
    tc_fence_after();
    float v[32];
    const int vcol = q4 * 32 + lane, t0 = ic * C + half * 32;
    tmem_ld32(tmem + L::T_DV + buf * 64 + lane_off + half * 32, v);
    tmem_ld_wait();
    if (FLEX && a.acc_v) {
      float* p = a.acc_v + ((size_t)bh * T + t0) * DV + c0 + vcol;
#pragma unroll
      for (int c = 0; c < 32; ++c)
        if (t0 + c < T) p[(size_t)c * DV] = v[c];
    } else if (FLEX) {  // dv in bf16 at the value columns of a [BH*T][pv] array
      __nv_bfloat16* p = a.dv + ((size_t)bh * T + t0) * pitch_v + col_v + c0 + vcol;
#pragma unroll
      for (int c = 0; c < 32; ++c)
        if (t0 + c < T) p[(size_t)c * pitch_v] = __float2bfloat16_rn(v[c]);
    } else {
      __nv_bfloat16* p = a.dv + ((size_t)bh * T + t0) * DV + c0 + vcol;
#pragma unroll
      for (int c = 0; c < 32; ++c)
        if (t0 + c < T) p[(size_t)c * DV] = __float2bfloat16_rn(v[c]);
    }
  };
  for (int n = 0; n < nl; ++n) {
    const int i = ch1 - 1 - n;
    mbar_wait(bar_ld, ph_ld, a.latch);
    ph_ld ^= 1;
    Gate gr;
    if constexpr (LOGIT) gr.set_logit(a.inv_tau, T - i * C);
    const bool weak = gr.run(sm + 2 * L::RAW, DK, TOT);
    if (gr.h == 0) gr.store_decay(DEC);
    const int safe = bar_or(kBarCompute, BT, weak);
    {
      const float inv0 = safe ? 1.f : 1.f / gr.dec0, inv1 = safe ? 1.f : 1.f / gr.dec1;
      const uint32_t blk = (gr.d >> 6) * (C * 128), col = gr.d & 63;
      uint32_t w[Gate::TS];
      gr.load_pairs(sm, DK, false, w);
      gr.forward([&](int j, float e0, float e1) {
        const uint32_t wq = w[j - gr.h * Gate::TS];
        uint32_t hi, lo;
        split2(bf_lo(wq) * e0 * inv0, bf_hi(wq) * e1 * inv1, hi, lo);
        *reinterpret_cast<uint32_t*>(sm + L::QP_HI + blk + sw128(j, col)) = hi;
        *reinterpret_cast<uint32_t*>(sm + L::QP_LO + blk + sw128(j, col)) = lo;
      });
      gr.load_pairs(sm + L::RAW, DK, false, w);
      gr.backward([&](int j, float e0, float e1) {
        const uint32_t wk = w[j - gr.h * Gate::TS];
        uint32_t hi, lo;
        split2(bf_lo(wk) * e0, bf_hi(wk) * e1, hi, lo);
        *reinterpret_cast<uint32_t*>(sm + L::KH_HI + blk + sw128(j, col)) = hi;
        *reinterpret_cast<uint32_t*>(sm + L::KH_LO + blk + sw128(j, col)) = lo;
      });
    }
    if (safe) rescale_G();
    // this tile's part of Z^T for chunk i: row grow of the M=128 accumulator, 32 tokens
    auto z_epilogue = [&]() {
      float zv[32];
      tmem_ld32(tmem + L::T_Z + lane_off + half * 32, zv);
      tmem_ld_wait();
      // token-major rows: the lanes (consecutive key dims) store adjacent words
      float* dst = a.ws_z + ((((size_t)bh * (DV / VT) + vt) * NC + i) * C + half * 32) * DK + grow;
#pragma unroll
      for (int c = 0; c < 32; ++c) dst[(size_t)c * DK] = zv[c];
      // this tile's part of sum_r Kh_r Z_r over the thread's 32 tokens (Kh as hi + lo)
      const uint32_t kblk = (grow >> 6) * (C * 128), kcol = grow & 63;
      float kz = 0.f;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const uint32_t off = kblk + sw128(half * 32 + c, kcol);
        kz += (bf2f(sm + L::KH_HI + off) + bf2f(sm + L::KH_LO + off)) * zv[c];
      }
      a.ws_kz[((((size_t)bh * (DV / VT) + vt) * NC + i) * 2 + half) * DK + grow] = kz;
    };
    if (tid == 0) safe_flag[0] = safe;
    handoff(kBarH1);  // group 1
    bar_sync(kBarCompute, BT);  // every thread's Kh is in shared memory (the Z^T epilogue reads it)
    if (n > 0) dv_epilogue(i + 1, (n - 1) & 1);  // the previous chunk's dv, while group 1 runs
    mbar_wait(bar_mZ, ph_mZ, a.latch);
    ph_mZ ^= 1;
    tc_fence_after();
    if (!safe) z_epilogue();  // its part was issued after the previous chunk's G pass
    __syncwarp();
    mbar_wait(bar_mA, ph_mA, a.latch);
    ph_mA ^= 1;
    if (safe) {  // the exact path overwrites Qs / Kh, which the rest of group 1 reads
      mbar_wait(bar_m1, ph_m1, a.latch);
      ph_m1 ^= 1;
    }
    tc_fence_after();
    if (safe) z_epilogue();  // the exact path below overwrites Kh
    float* XA = reinterpret_cast<float*>(sm + L::XA);
    if (safe) {  // exact A = sum_d q_jd k_rd e^{B_jd - B_rd}, r <= j
      float* XB = reinterpret_cast<float*>(sm + L::XB);
      if (tid < DK) {
        float b = 0.f;
        for (int j = 0; j < C; ++j) {
          b += bf2f(sm + 2 * L::RAW + (j * DK + tid) * 2);
          XB[j * DK + tid] = b;
        }
      }
      bar_sync(kBarCompute, BT);
      for (int e = tid; e < C * C; e += BT) {
        const int j = e / C, r = e % C;
        float acc = 0.f;
        if (r <= j)
          for (int d = 0; d < DK; ++d)
            acc += bf2f(sm + (j * DK + d) * 2) * bf2f(sm + L::RAW + (r * DK + d) * 2) *
                   __expf(XB[j * DK + d] - XB[r * DK + d]);
        XA[e] = acc;
      }
      bar_sync(kBarCompute, BT);
    }
    {  // A epilogue
      float v[32];
      tmem_ld32(tmem + L::T_A + lane_off + half * 32, v);
      tmem_ld_wait();
      if (row_owner) {
        if (safe) {
#pragma unroll
          for (int c = 0; c < 32; ++c) v[c] = XA[row * C + half * 32 + c];
        }
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (half * 32 + c > row) v[c] = 0.f;
        store_half_split(sm + L::AB_HI, sm + L::AB_LO, row, v, half);
      }
    }
    handoff(kBarH2);  // group 2
    // group 1 complete: the G pass (it touches neither A, dO nor dv)
    if (!safe) {
      mbar_wait(bar_m1, ph_m1, a.latch);
      ph_m1 ^= 1;
      tc_fence_after();
    }
    {  // G_i = dec * G (chunks off the exact path, whose rescale came first) and its hi / lo copy
      const float sc = safe ? 1.f : DEC[grow];
      float v[64];
      for (int cb = half * HT; cb < (half + 1) * HT; cb += 64) {
        tmem_ld32(tmem + L::T_G + lane_off + cb, v);
        tmem_ld32(tmem + L::T_G + lane_off + cb + 32, v + 32);
        tmem_ld_wait();
        if (!safe) {
#pragma unroll
          for (int c = 0; c < 64; ++c) v[c] *= sc;
          tmem_st32(tmem + L::T_G + lane_off + cb, v);
          tmem_st32(tmem + L::T_G + lane_off + cb + 32, v + 32);
        }
        store_row_split(sm + L::GC_HI + (cb / 64) * (DK * 128), sm + L::GC_LO + (cb / 64) * (DK * 128), grow, v, 1.f);
      }
      tmem_st_wait();
    }
    if (n + 1 < nl) handoff(kBarH0);  // the G copy: the next chunk's Z^T part
    __syncwarp();
    mbar_wait(bar_m2, ph_m2, a.latch);
    ph_m2 ^= 1;
    tc_fence_after();
    tc_fence_before();
    bar_sync(kBarCompute, BT);
  }
  if (nl > 0) dv_epilogue(ch0, (nl - 1) & 1);
  // dh0[:, tile] = G_0
  if (a.dh0 && seg == 0) {
    tc_fence_after();
    float dv0v[32];
    for (int cb = half * HT; cb < (half + 1) * HT; cb += 32) {
      tmem_ld32(tmem + L::T_G + lane_off + cb, dv0v);
      tmem_ld_wait();
      float4* dst = reinterpret_cast<float4*>(a.dh0 + bh * a.st_bh + grow * a.st_row + c0 + cb);
#pragma unroll
      for (int c = 0; c < 8; ++c) dst[c] = make_float4(dv0v[4 * c], dv0v[4 * c + 1], dv0v[4 * c + 2], dv0v[4 * c + 3]);
    }
  }
}

// ------------------------------------------------------------------------------------------
// Carry scan: per (head, key dim), c_{N-1} = rowsum(dhT * hT) - K_{N-1} and
// c_i = c_{i+1} + Q_{i+1} - K_i, with Q the forward walk's chunk sums of Qt X and K the chunk
// sums of Kh Z (summed over value tiles and token halves).
// ------------------------------------------------------------------------------------------
// One block per (head, 32 key dims, segment); its 8 warps each take a slice of the segment's
// chunks: the slice sums are exchanged in shared memory, then every warp walks its own slice from
// the right start.  Each segment's carry starts at its last chunk from rowsum(G_end * S_end) of
// the states its walks used, so the recurrence telescopes within the segment.
template <int NVT>
__global__ void __launch_bounds__(256) carry_scan_kernel(const float* __restrict__ carry, const float* __restrict__ qx,
                                                         const float* __restrict__ kz, float* __restrict__ cout,
                                                         int DK, int NC, int seg_chunks) {
  __shared__ float slice_sum[8][32];
  const int dl = threadIdx.x & 31, s = threadIdx.x >> 5;
  const int bh = blockIdx.x / (DK / 32), d = (blockIdx.x % (DK / 32)) * 32 + dl;
  const int seg = blockIdx.y, nseg = gridDim.y;
  const int ch0 = seg * seg_chunks, ch1 = min(NC, ch0 + seg_chunks);
  const int G = (ch1 - ch0 + 7) / 8, top = ch1 - 1 - s * G;  // slice s: chunks top, top - 1, ... (>= ch0)
  // change of the carry from chunk i + 1 to chunk i (none from beyond the segment)
  auto delta = [&](int i) {
    float v = i < ch1 - 1 ? qx[((size_t)bh * NC + i + 1) * DK + d] : 0.f;
#pragma unroll
    for (int h = 0; h < 2 * NVT; ++h) v -= kz[(((size_t)bh * NVT * NC + (h >> 1) * NC + i) * 2 + (h & 1)) * DK + d];
    return v;
  };
  float sum = 0.f;
#pragma unroll 4
  for (int u = 0; u < G; ++u)
    if (top - u >= ch0) sum += delta(top - u);
  slice_sum[s][dl] = sum;
  __syncthreads();
  float c = carry[((size_t)bh * nseg + seg) * DK + d];
  for (int t = 0; t < s; ++t) c += slice_sum[t][dl];
  for (int u = 0; u < G; ++u)
    if (top - u >= ch0) {
      c += delta(top - u);
      cout[((size_t)bh * NC + top - u) * DK + d] = c;
    }
}

// ------------------------------------------------------------------------------------------
// Third launch: one CTA per (head, 64 key dimensions, chunk).  Gate run of the key slab (Qt, E2,
// decays), the masked dA of the chunk as the first key tile wrote it (hi / lo operand tiles and the
// diagonal, one bulk copy), W^T = Qt^T dA, and the epilogue
//   dk = E2 Z + (E2 / dec) W,   dg = c_i + prefix(Kh Z + k dk^intra) + the forward walk's part,
// with Z^T summed over the value tiles' parts.  No state: every chunk is independent.
// ------------------------------------------------------------------------------------------
template <int DK, int DV>
struct ChunkLayout {
  static constexpr uint32_t TILE = C * KT * 2;      // a [64 x 64] bf16 tile
  static constexpr uint32_t PB_K = 0, PB_G = TILE, PB_Q = 2 * TILE;  // k, g, q tiles
  static constexpr uint32_t KQ_HI = 3 * TILE;       // Qt hi / lo
  static constexpr uint32_t KQ_LO = KQ_HI + TILE;
  static constexpr uint32_t DA_HI = KQ_LO + TILE;   // masked dA hi / lo, then its diagonal: one
  static constexpr uint32_t DA_LO = DA_HI + TILE;   // kDaBytes block as the key tile wrote it
  static constexpr uint32_t DIAG = DA_LO + TILE;
  static constexpr int NS = GateRun<KT, BT>::NSPLIT;
  static constexpr uint32_t XCH = DIAG + C * 4;
  static constexpr uint32_t DEC = XCH + 2 * KT * 8;
  static constexpr uint32_t TOT = DEC + KT * 4;
  static constexpr uint32_t TOTAL = TOT + NS * KT * 4;
  static_assert(TOT % 8 == 0 && DEC % 8 == 0, "gate tables are read as float2");
  static constexpr uint32_t T_Y = 0;  // TMEM columns (64 allocated)
  static_assert(KQ_HI % 1024 == 0 && DA_HI % 1024 == 0 && DIAG == DA_HI + 2 * TILE &&
                    DIAG + C * 4 - DA_HI == kDaBytes,
                "operand layout");
};

template <int DK, int DV, bool FLEX, bool LOGIT>
__global__ void __launch_bounds__(BT, 2) bwd_chunk_kernel(const __grid_constant__ BwdMaps mp, const BwdArgs a) {
  using L = ChunkLayout<DK, DV>;
  using Gate = GateRun<KT, BT, LOGIT>;
  // column offset into wider input tensors (FLEX builds only)
  const int col_k = FLEX ? a.ck : 0;
  constexpr int NS = L::NS, TS = Gate::TS, NVT = DV / VT;
  static_assert(TS % 4 == 0, "token pairs u, u ^ 2 of the epilogue loads lie in one group");
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_ld, bar_m2;
  __shared__ uint32_t tmem_base_sh;
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const uint32_t base = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3, half = warp >> 2;
  const int T = a.T, NC = (T + C - 1) / C;
  const int i = blockIdx.x % NC, slab = blockIdx.x / NC;
  const int tau = slab % (DK / KT), bh = slab / (DK / KT), d0 = tau * KT;
  const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
  const int tb = half * 32;
  float* DEC = reinterpret_cast<float*>(sm + L::DEC);
  float* TOT = reinterpret_cast<float*>(sm + L::TOT);
  float* DIAG = reinterpret_cast<float*>(sm + L::DIAG);

  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, 64);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar_ld, 1);
    mbar_init(&bar_m2, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  if (tid == 0) {
    mbar_arrive_expect_tx(&bar_ld, 3 * L::TILE + kDaBytes);
    bulk_g2s(sm + L::DA_HI, a.ws_da + ((size_t)bh * NC + i) * kDaBytes, kDaBytes, &bar_ld);
    tma_load_3d(sm + L::PB_K, &mp.k64, &bar_ld, col_k + d0, i * C, bh);
    tma_load_3d(sm + L::PB_G, &mp.g64, &bar_ld, col_k + d0, i * C, bh);
    tma_load_3d(sm + L::PB_Q, &mp.q64, &bar_ld, col_k + d0, i * C, bh);
  }
  // The epilogue runs on all 32 lanes: lane l < 16 owns key dim row = q4 * 16 + l for tokens
  // tb .. tb + 15, lane l + 16 the same dim for tokens tb + 16 .. tb + 31 (the M = 64 accumulators
  // sit in TMEM lanes 0-15 of each quarter, so those values reach the upper lanes by shuffle).
  const int sub = lane >> 4, tq = tb + sub * 16, qi = half * 2 + sub;
  const int erow = q4 * 16 + (lane & 15);
  // global inputs of the epilogue, loaded while the tiles arrive
  float pv[16], z[16];
  {  // token-major rows: for each token the lanes read adjacent words (two runs of 16 dims)
    const float* src = a.ws_part + (((size_t)bh * NC + i) * C + tq) * DK + d0 + erow;
    float zz[NVT][16];
#pragma unroll
    for (int c = 0; c < 16; ++c) pv[c] = src[(size_t)c * DK];
#pragma unroll
    for (int vt = 0; vt < NVT; ++vt) {
      const float* zs = a.ws_z + ((((size_t)bh * NVT + vt) * NC + i) * C + tq) * DK + d0 + erow;
#pragma unroll
      for (int c = 0; c < 16; ++c) zz[vt][c] = zs[(size_t)c * DK];
    }
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      z[c] = 0.f;
#pragma unroll
      for (int vt = 0; vt < NVT; ++vt) z[c] += zz[vt][c];
    }
  }
  const float ci = a.ws_c[((size_t)bh * NC + i) * DK + d0 + erow];
  auto raw = [&](uint32_t off, int j, int d) { return bf2f(sm + off + sw128(j, d)); };
  auto dA_at = [&](int j, int r) { return raw(L::DA_HI, j, r) + raw(L::DA_LO, j, r); };

  mbar_wait(&bar_ld, 0, a.latch);
  // gate run of the key slab: Qt hi / lo, decays, run products
  Gate gr;
  if constexpr (LOGIT) gr.set_logit(a.inv_tau, T - i * C);
  const bool weak = gr.run_swizzled(sm + L::PB_G, TOT);
  if (gr.h == 0) gr.store_decay(DEC);
  const int safe = __syncthreads_or(weak);
  uint32_t wq[Gate::TS];
  gr.load_pairs(sm + L::PB_Q, KT, true, wq);
  gr.forward([&](int j, float e0, float e1) {
    const uint32_t w = wq[j - gr.h * Gate::TS];
    uint32_t hi, lo;
    split2(bf_lo(w) * e0, bf_hi(w) * e1, hi, lo);
    *reinterpret_cast<uint32_t*>(sm + L::KQ_HI + sw128(j, gr.d)) = hi;
    *reinterpret_cast<uint32_t*>(sm + L::KQ_LO + sw128(j, gr.d)) = lo;
  });
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid == 0 && !safe) {  // W^T = Qt^T dA
    constexpr uint32_t id_W = idesc_bf16_f32(KT, C, true, true);
#pragma unroll
    for (int k = 0; k < C / 16; ++k) {
      const uint64_t ah = desc_sw128(base + L::KQ_HI + k * 2048, C * 128, 1024);
      const uint64_t bh2 = desc_sw128(base + L::DA_HI + k * 2048, C * 128, 1024);
      umma_bf16(tmem + L::T_Y, ah, bh2, id_W, k > 0);
      umma_bf16(tmem + L::T_Y, desc_sw128(base + L::KQ_LO + k * 2048, C * 128, 1024), bh2, id_W, 1);
      umma_bf16(tmem + L::T_Y, ah, desc_sw128(base + L::DA_LO + k * 2048, C * 128, 1024), id_W, 1);
    }
    umma_commit(&bar_m2);
  }
  const int d = erow;
  float w[16];
  if (!safe) {
    float wr[32];
    __syncwarp();
    mbar_wait(&bar_m2, 0, a.latch);
    tc_fence_after();
    tmem_ld32(tmem + L::T_Y + lane_off + tb, wr);
    tmem_ld_wait();
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const float x = __shfl_sync(0xffffffffu, wr[16 + c], lane & 15);
      w[c] = sub ? x : wr[c];
    }
  } else {  // exact intra term w_r = sum_{j>=r} dA_jr q_j e^{B_j - B_r}
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const int r = tq + c;
      float acc = dA_at(r, r) * raw(L::PB_Q, r, d), bd = 0.f;
      for (int j = r + 1; j < C; ++j) {
        bd += raw(L::PB_G, j, d);
        acc += dA_at(j, r) * raw(L::PB_Q, j, d) * __expf(bd);
      }
      w[c] = acc;
    }
  }
  float tot_s = 0.f;
  {  // dk; per-token terms Kh Z + k dk^intra without j = r (-> w)
    const float inv = 1.f / DEC[d];
    __nv_bfloat16* dst = a.dk + ((size_t)bh * T + i * C + tq) * DK + d0 + d;
    float* dst32 = FLEX ? a.acc_k + ((size_t)bh * T + i * C + tq) * DK + d0 + d : nullptr;
#pragma unroll
    for (int rr = 0; rr < 16 / TS; ++rr) {
      const int h = tq / TS + rr;
      // the group's raw g, q and k values; lanes 16-31 read token u ^ 2 at load step u, off the
      // banks of lanes 0-15 (as in the key tile's dq epilogue), and take them back in token order
      float gl[TS], ql[TS], kl[TS];
#pragma unroll
      for (int u = 0; u < TS; ++u) {
        const int r = h * TS + (u ^ (2 * sub));
        gl[u] = raw(L::PB_G, r, d);
        ql[u] = raw(L::PB_Q, r, d);
        kl[u] = raw(L::PB_K, r, d);
      }
      float al[TS], e2[TS];
#pragma unroll
      for (int u = 0; u < TS; ++u) al[u] = ex2((sub ? gl[u ^ 2] : gl[u]) * kLog2e);
      float e = 1.f;  // E2 = e^{gamma - B_r}, formed as GateRun::backward forms it
      for (int hh = h + 1; hh < NS; ++hh) e *= TOT[hh * KT + d];
#pragma unroll
      for (int u = TS - 1; u >= 0; --u) {
        e2[u] = e;
        e *= al[u];
      }
#pragma unroll
      for (int u = 0; u < TS; ++u) {
        const int c = rr * TS + u, r = tq + c;
        const float ev = e2[u];
        if (!safe) w[c] *= ev * inv;
        const float qv = sub ? ql[u ^ 2] : ql[u], kv = sub ? kl[u ^ 2] : kl[u];
        if (i * C + r < T) {
          if constexpr (FLEX)
            dst32[(size_t)c * DK] = ev * z[c] + w[c];
          else
            dst[(size_t)c * DK] = __float2bfloat16_rn(ev * z[c] + w[c]);
        }
        const float kz = bf_split_sum(kv * ev) * z[c];  // Kh Z, with Kh as the S update sees it
        w[c] = kz + kv * (w[c] - DIAG[r] * qv);        // plus k dk^intra without j = r
        tot_s += w[c];
      }
    }
  }
  float* XQ = reinterpret_cast<float*>(sm + L::XCH);  // [4 token quarters][KT] sums of w
  XQ[qi * KT + d] = tot_s;
  __syncthreads();
  {  // dg = c_i + prefix (exclusive) of (Kh Z + k dk^intra) + the forward walk's part
    float pre = 0.f;
    for (int t = 0; t < qi; ++t) pre += XQ[t * KT + d];
    __nv_bfloat16* dst = a.dg + ((size_t)bh * T + i * C + tq) * DK + d0 + d;
    float* dst32 = FLEX ? a.acc_g + ((size_t)bh * T + i * C + tq) * DK + d0 + d : nullptr;
    const float tau = LOGIT ? 1.f / a.inv_tau : 0.f;
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      if (i * C + tq + c < T) {
        float dgv = ci + pre + pv[c];
        // raw logits: dx = dg sigmoid(-x) / tau, with sigmoid(-x) = 1 - e^{tau g} = -expm1(tau g)
        if constexpr (LOGIT) dgv *= -expm1f(tau * raw(L::PB_G, tq + c, d)) * a.inv_tau;
        if constexpr (FLEX)
          dst32[(size_t)c * DK] = dgv;
        else
          dst[(size_t)c * DK] = __float2bfloat16_rn(dgv);
      }
      pre += w[c];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 64);
}

// ------------------------------------------------------------------------------------------
// Kernel and host entry points
// ------------------------------------------------------------------------------------------
template <int DK, int DV>
struct BwdSmem {
  static constexpr uint32_t K = KeyLayout<DK, DV>::TOTAL, V = ValLayout<DK>::TOTAL;
  static constexpr uint32_t ALLOC = (K > V ? K : V) + 1024;
  static_assert(ALLOC <= 227 * 1024, "shared memory");
};

template <int DK, int DV, bool FLEX, bool LOGIT>
__global__ void __launch_bounds__(BTP, 1) bwd_fused_kernel(const __grid_constant__ BwdMaps mp, const BwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bars[7];
  __shared__ int safe_flag[2];  // exact-path flag of a chunk, compute threads -> producer warp
  __shared__ uint32_t tmem_base_sh;
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const int warp = threadIdx.x >> 5;
  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int b = 0; b < 7; ++b) mbar_init(&bars[b], 1);
    fence_mbar_init();
  }
  if (threadIdx.x == BT) {  // the tensor maps, ahead of the first loads
    prefetch_tmap(&mp.v);
    prefetch_tmap(&mp.dO);
    prefetch_tmap(&mp.k64);
    prefetch_tmap(&mp.g64);
    prefetch_tmap(&mp.q64);
    prefetch_tmap(&mp.q_all);
    prefetch_tmap(&mp.k_all);
    prefetch_tmap(&mp.g_all);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  constexpr int per_head = DK / KT + DV / VT;
  const int per_seg = a.n_bh * per_head;
  const int seg = blockIdx.x / per_seg, bh = (blockIdx.x % per_seg) / per_head, role = blockIdx.x % per_head;
  if (role < DK / KT)
    key_tile_body<DK, DV, FLEX, LOGIT>(sm, mp, a, bh, role, seg, bars, tmem, safe_flag);
  else
    val_tile_body<DK, FLEX, LOGIT>(sm, mp, a, bh, role - DK / KT, DV, seg, bars, tmem, safe_flag);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int DK, int DV, bool FLEX, bool LOGIT>
static cudaError_t launch_all(const BwdMaps& mp, const BwdArgs& a, int BH, cudaStream_t st) {
  constexpr uint32_t CHK = ChunkLayout<DK, DV>::TOTAL + 1024;
  static_assert(2 * CHK <= 228 * 1024, "two chunk CTAs per SM");
  auto k1 = bwd_fused_kernel<DK, DV, FLEX, LOGIT>;
  auto k3 = bwd_chunk_kernel<DK, DV, FLEX, LOGIT>;
  static std::atomic<bool> attr1[64] = {}, attr3[64] = {};
  {
    cudaError_t e = ensure_smem_attr(k1, BwdSmem<DK, DV>::ALLOC, attr1);
    if (e == cudaSuccess) e = ensure_smem_attr(k3, CHK, attr3);
    if (e != cudaSuccess) return e;
  }
  k1<<<BH * (DK / KT + DV / VT) * a.nseg, BTP, BwdSmem<DK, DV>::ALLOC, st>>>(mp, a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int NC = (a.T + C - 1) / C;
  carry_scan_kernel<DV / VT><<<dim3(BH * (DK / 32), a.nseg), 256, 0, st>>>(a.ws_carry, a.ws_qx, a.ws_kz, a.ws_c, DK,
                                                                          NC, a.seg_chunks);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k3<<<BH * (DK / KT) * NC, BT, CHK, st>>>(mp, a);
  return cudaGetLastError();
}

bool bwd_supported(int BH, int T, int dk, int dv, int chunk, int dtype) {
  if (dtype != 1 || chunk != C || T < 1 || BH < 1) return false;
  if (dk != 128 || (dv != 128 && dv != 256)) return false;
  return encode_fn() != nullptr;
}

// Workspace parts, in order: Qt X chunk sums, forward part of dg, carry starts, Z parts, Kh Z chunk
// sums, carries; with a sequence split the segment states (forward, gradient) and the segment decay
// products; the masked dA blocks.
static void bwd_parts(int BH, int T, int dk, int dv, size_t* sz, int* nseg, int* seg_chunks) {
  plan_bwd_segments(BH * (dk / KT + dv / VT), T, nseg, seg_chunks);
  const size_t NC = (T + C - 1) / C, ns = *nseg, f = sizeof(float);
  sz[0] = align256((size_t)BH * NC * dk * f);
  sz[1] = align256((size_t)BH * NC * C * dk * f);
  sz[2] = align256((size_t)BH * ns * dk * f);
  sz[3] = align256((size_t)BH * (dv / VT) * NC * dk * C * f);
  sz[4] = align256((size_t)BH * (dv / VT) * NC * 2 * dk * f);
  sz[5] = align256((size_t)BH * NC * dk * f);
  sz[6] = ns > 1 ? align256((size_t)BH * ns * dk * dv * f) : 0;
  sz[7] = sz[6];
  sz[8] = ns > 1 ? align256((size_t)BH * ns * dk * f) : 0;
  sz[9] = align256((size_t)BH * NC * kDaBytes);
}

size_t bwd_workspace(int BH, int T, int dk, int dv) {
  size_t sz[10];
  int nseg, per;
  bwd_parts(BH, T, dk, dv, sz, &nseg, &per);
  size_t n = 0;
  for (size_t x : sz) n += x;
  return n;
}

template <int DK, int DV>
static cudaError_t launch_bwd(const void* q, const void* k, const void* v, const void* g, const float* h0,
                              const void* dO, const float* dhT, void* dq, void* dk, void* dv, void* dg, float* dh0,
                              int BH, int T, void* ws, cudaStream_t st, long long st_bh, long long st_row,
                              const BwdAccum* acc, float inv_tau) {
  // pitch and first column of this sub-problem's key dims and value columns in the tensors given
  const int PK = acc ? acc->pk : DK, CK = acc ? acc->ck : 0, PV = acc ? acc->pv : DV, CV = acc ? acc->cv : 0;
  if (CK < 0 || CK + DK > PK || CK % 8 || CV < 0 || CV + DV > PV || CV % 8) return cudaErrorInvalidValue;
  if (acc && (!acc->q || !acc->k || !acc->g || (!acc->v && !dv))) return cudaErrorInvalidValue;
  BwdMaps mp;
  if (!make_map(&mp.v, v, BH, T, PV, 64, true) || !make_map(&mp.dO, dO, BH, T, PV, 64, true) ||
      !make_map(&mp.k64, k, BH, T, PK, KT, true) || !make_map(&mp.g64, g, BH, T, PK, KT, true) ||
      !make_map(&mp.q64, q, BH, T, PK, KT, true) ||
      !make_map(&mp.q_all, q, BH, T, PK, DK, false) || !make_map(&mp.k_all, k, BH, T, PK, DK, false) ||
      !make_map(&mp.g_all, g, BH, T, PK, DK, false))
    return cudaErrorInvalidValue;
  BwdArgs a;
  a.h0 = h0;
  a.dhT = dhT;
  a.dq = static_cast<__nv_bfloat16*>(dq);
  a.dk = static_cast<__nv_bfloat16*>(dk);
  a.dv = static_cast<__nv_bfloat16*>(dv);
  a.dg = static_cast<__nv_bfloat16*>(dg);
  a.dh0 = dh0;
  a.T = T;
  a.st_bh = st_bh;
  a.st_row = st_row;
  a.acc_q = acc ? acc->q : nullptr;
  a.acc_k = acc ? acc->k : nullptr;
  a.acc_g = acc ? acc->g : nullptr;
  a.acc_v = acc ? acc->v : nullptr;
  a.pk = PK;
  a.ck = CK;
  a.pv = PV;
  a.cv = CV;
  a.inv_tau = inv_tau;
  size_t sz[10];
  bwd_parts(BH, T, DK, DV, sz, &a.nseg, &a.seg_chunks);
  float* p[10];
  p[0] = static_cast<float*>(ws);
  for (int j = 1; j < 10; ++j) p[j] = p[j - 1] + sz[j - 1] / sizeof(float);
  a.ws_qx = p[0];
  a.ws_part = p[1];
  a.ws_carry = p[2];
  a.ws_z = p[3];
  a.ws_kz = p[4];
  a.ws_c = p[5];
  a.s_in = a.nseg > 1 ? p[6] : nullptr;
  a.g_end = a.nseg > 1 ? p[7] : nullptr;
  a.ws_da = reinterpret_cast<uint8_t*>(p[9]);
  a.n_bh = BH;
  a.latch = device_error_latch();
  if (a.nseg > 1) {
    const cudaError_t e = segment_states(mp.q_all, mp.k_all, mp.g_all, mp.v, mp.dO, h0, dhT, p[6], p[7], p[8], BH, T,
                                         DK, DV, a.nseg, a.seg_chunks, st_bh, st_row, st, inv_tau, CK, CV);
    if (e != cudaSuccess) return e;
  }
  // the plain build unless the call needs offsets and fp32 outputs (FLEX) or raw-logit gates (LOGIT);
  // each build carries only its own code
  const bool logit = inv_tau > 0.f;
  if (acc) return logit ? launch_all<DK, DV, true, true>(mp, a, BH, st) : launch_all<DK, DV, true, false>(mp, a, BH, st);
  return logit ? launch_all<DK, DV, false, true>(mp, a, BH, st) : launch_all<DK, DV, false, false>(mp, a, BH, st);
}

cudaError_t bwd(const void* q, const void* k, const void* v, const void* g, const float* h0, const void* dO,
                const float* dhT, void* dq, void* dk, void* dv, void* dg, float* dh0, int BH, int T, int dkd, int dvd,
                void* ws, cudaStream_t st, long long st_bh, long long st_row, const BwdAccum* acc, float inv_tau) {
  if (st_bh < 0) st_bh = (long long)dkd * dvd;
  if (st_row < 0) st_row = dvd;
  if (dkd == 128 && dvd == 256)
    return launch_bwd<128, 256>(q, k, v, g, h0, dO, dhT, dq, dk, dv, dg, dh0, BH, T, ws, st, st_bh, st_row, acc,
                                inv_tau);
  if (dkd == 128 && dvd == 128)
    return launch_bwd<128, 128>(q, k, v, g, h0, dO, dhT, dq, dk, dv, dg, dh0, BH, T, ws, st, st_bh, st_row, acc,
                                inv_tau);
  return cudaErrorNotSupported;
}

}  // namespace fast
}  // namespace gla
