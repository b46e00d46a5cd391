// Fused attention forward for sm_100a: O = softmax(scale Q K^T [+ causal mask]) V and LSE.
//
// Method: the tiled forward of "Transformer、注意力机制与优化" (section FlashAttention-2 算法):
// a block of query rows stays on chip while key/value blocks stream past it; each row keeps
// a running max m and running sum l (section 安全 Softmax 与在线 Softmax, two-block identity)
// and a running output accumulator that is rescaled when m grows ("FlashAttention 的基本原理",
// section 2.3 前向传播).  Normalisation by l is deferred to the end and only
// L = m + log(l) is saved for the backward pass ("FlashAttention 系列技术详解", section
// 具体优化策略).  The score matrix exists only in tensor memory, one 128 x 128 tile at a time.
//
// B200 design (not the pages' A100/H100 kernels):
//  * one CTA owns two 128-row query tiles (Q0, Q1) of one (batch, head) and streams 128-key
//    K and V tiles through a shared-memory ring filled by TMA (128-byte swizzle);
//  * tcgen05 MMAs: S_t = Q_t K^T (both operands in shared memory) and O_t += P_t V (P_t read
//    from tensor memory, V from shared memory), fp32 accumulators in TMEM:
//    S0 | S1 | O0 | O1 = 128 + 128 + d + d columns;
//  * one issuing thread for both tiles, in the order S0 S1 PV0 S0' PV1 S1' ..., which staggers
//    the two softmax groups (measured on B200: two independent issuers, one per tile, ran the
//    groups in lockstep and were ~17% slower, although a lone thread issues a 128 x 128 x 16
//    MMA only every ~115 cycles);
//  * two softmax warpgroups, one per query tile, each thread owning one row (= one TMEM
//    lane): while one group exponentiates its S tile, the tensor core runs the other tile's
//    MMAs;
//  * exp2 with scale*log2(e) folded into one packed FMA; the running max is only moved (and O
//    and l rescaled) when a row's max grows by more than 2^8, which keeps P <= 256 and is exact
//    because O, l and LSE all use the same stale max;
//  * P is rounded to bf16 and written over the first half of its own S columns; O is normalised
//    by the sum of those rounded weights, LSE by the exact fp32 sum.
#pragma once

#include "dropout_sm100.cuh"

namespace fa {

constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D, bool F8 = false, bool EXT = false>
struct FwdTraits {
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(!F8 || D == 128, "FP8 operands: d = 128");
  static constexpr int EB = F8 ? 1 : 2;                // bytes per Q/K/V element (E4M3 or bf16)
  static constexpr int BM = 128;                       // query rows per tile
  static constexpr int BN = 128;                       // keys per tile
  static constexpr int BOX_COLS = 128 / EB;            // elements per 128-byte swizzle row
  static constexpr int NBOX = D * EB / 128;            // 128-byte-wide TMA boxes per tile
  static constexpr int BOX_BYTES = 128 * 128;          // 128 rows x 128 bytes = 16 KB
  static constexpr int TILE_BYTES = NBOX * BOX_BYTES;  // one 128 x D tile
  static constexpr int KSTEP = 32 / EB;                // MMA K per instruction (32 bytes of operand)
  static constexpr int NS = F8 ? 8 : ((D == 64) ? 6 : 3);  // K/V ring stages
  // Q slots (work items alternate between them, so the next item's Q loads while the current one
  // runs), each holding the item's two 128-row tiles: slot s, tile t at OFF_Q + (2 s + t) TILE_BYTES.
  // The bias instantiation keeps one slot and spends the space on two bias tiles (one per softmax
  // group: 128 rows x 128 keys bf16, two 64-key TMA boxes with the 128-byte swizzle).
  static constexpr int QSLOTS = EXT ? 1 : 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = 2 * QSLOTS * TILE_BYTES;
  static constexpr int BIAS_TILE = 128 * 128 * 2;
  static constexpr int OFF_BIAS = OFF_KV + NS * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_BIAS + (EXT ? 2 * BIAS_TILE : 0);
  // barriers: q_full[2] | q_empty[2] | kv_full[NS] | kv_empty[NS] | s_full[2] | p_ready[2][2] | o_done[2] |
  //           o_free[2] | drain | merge | bias_full[2] | bias_empty[2]
  static constexpr int BAR_Q_FULL = 0;
  static constexpr int BAR_Q_EMPTY = 2;
  static constexpr int BAR_KV_FULL = 4;
  static constexpr int BAR_KV_EMPTY = 4 + NS;
  static constexpr int BAR_S_FULL = 4 + 2 * NS;
  // p_ready[t][half]: group t has written the softmax weights of keys [64 half, 64 half + 64) of
  // its current tile (the P V product starts on the first half while the second is computed).
  static constexpr int BAR_P_READY = BAR_S_FULL + 2;
  static constexpr int BAR_O_DONE = BAR_P_READY + 4;
  static constexpr int BAR_O_FREE = BAR_O_DONE + 2;  // group t has read O_t out: the next item may overwrite it
  static constexpr int BAR_DRAIN = BAR_O_FREE + 2;
  static constexpr int BAR_MERGE = BAR_DRAIN + 1;  // split mode: group 1's row statistics published
  static constexpr int BAR_BIAS_FULL = BAR_MERGE + 1;       // group t's bias tile has landed
  static constexpr int BAR_BIAS_EMPTY = BAR_BIAS_FULL + 2;  // group t has read its bias tile
  static constexpr int NBAR = BAR_BIAS_EMPTY + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base (u32), abort flag (int)
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack for 1024-byte alignment
  static constexpr uint32_t TMEM_COLS = 512;
  // TMEM columns: S_t at 128 t, O_t at 256 + D t.
  static __host__ __device__ constexpr uint32_t col_s(int t) { return 128u * t; }
  static __host__ __device__ constexpr uint32_t col_o(int t) { return 256u + (uint32_t)D * t; }
  // Warps 0-7 softmax, 8 MMA issuer, 9 TMA (Q, K, V), 10 (bias instantiation) TMA of the bias tiles.
  static constexpr int WARP_BIAS = 10;
  static constexpr int THREADS = EXT ? 352 : 320;
  static constexpr uint32_t IDESC_QK = F8 ? make_idesc_e4m3(128, 128, false, false) : make_idesc_bf16(128, 128, false, false);
  static constexpr uint32_t IDESC_PV = F8 ? make_idesc_e4m3(128, D, false, true) : make_idesc_bf16(128, D, false, true);
};

struct FwdParams {
  __nv_bfloat16* o;
  float* lse;
  int Nq, Nk, BH;
  int nunits;        // query units per (batch, head): ceil(Nq / (128 * tiles))
  int tiles;         // 128-row query tiles per unit: 2 (ping-pong), or 1 when there are fewer units than
                     // SMs (then each CTA takes one unit and the two softmax groups split its key tiles:
                     // even / odd)
  float scale_log2;  // scale * log2(e)
  int causal;
  // FP8 operands only: per-(batch, head) dequantisation factors (x = x8 * descale).
  const float* descale_q;
  const float* descale_k;
  const float* descale_v;
  // Bias and dropout instantiation only.  bias: [Bb, Hb, Nq, Nk] bf16 or null, b / h element
  // strides bias_sb / bias_sh (0 where broadcast), and b / h strides bias_pb / bias_ph in [Nq, Nk]
  // planes (the third coordinate of the bias tensor map); H splits the (batch, head) index.
  const __nv_bfloat16* bias;
  long long bias_sb, bias_sh;
  int bias_pb, bias_ph;
  int H;
  DropoutCfg drop;
};

// One work item: the query unit of rows [q0, q0 + 128 tiles) of (batch, head) bh.  n0 / n1: key tiles
// query tile 0 / 1 must visit (under the causal mask the last key tile of the unit is hidden from
// tile 0 entirely, so tile 0 skips it); n_kv = max(n0, n1) K/V tiles are streamed.
struct FwdItem {
  int bh, q0, n0, n1, n_kv;
};

// Number of 128-key tiles the CTA owning query rows [q0, q0 + span) must visit.
__device__ __forceinline__ int fwd_num_kv_tiles(int q0, int span, int Nq, int Nk, int causal) {
  const int nkt = (Nk + 127) / 128;
  if (!causal) return nkt;
  const int last = min(q0 + span - 1, Nq - 1);
  const int kmax = last + Nk - Nq;  // last visible key of the last row
  if (kmax < 0) return 1;           // every row fully masked: one tile, all -inf
  return min(nkt, kmax / 128 + 1);
}

template <int D, bool F8>
__device__ __forceinline__ void fwd_issue_qk(uint32_t tmem_d, uint32_t q_smem, uint32_t k_smem) {
  using T = FwdTraits<D, F8>;
  const uint64_t qd = make_sdesc_sw128(q_smem, 16, 1024), kd = make_sdesc_sw128(k_smem, 16, 1024);
#pragma unroll
  for (int kk = 0; kk < D / T::KSTEP; ++kk) {
    // K advances 32 bytes inside a 128-byte swizzle row; every 4 steps, the next box.
    const uint64_t off = (uint64_t)(((kk / 4) * T::BOX_BYTES + (kk % 4) * 32) >> 4);
    if constexpr (F8)
      mma_ss_w_f8(tmem_d, qd + off, kd + off, T::IDESC_QK, kk > 0 ? 1u : 0u);
    else
      mma_ss_w(tmem_d, qd + off, kd + off, T::IDESC_QK, kk > 0 ? 1u : 0u);
  }
}

// O += P V over keys [64 half, 64 half + 64) of the tile (accumulate: whether O already holds a sum;
// the second half always accumulates).
template <int D, bool F8>
__device__ __forceinline__ void fwd_issue_pv(uint32_t tmem_d, uint32_t tmem_p, uint32_t v_smem, int half,
                                             bool accumulate) {
  using T = FwdTraits<D, F8>;
  const uint64_t vd = make_sdesc_sw128(v_smem, T::BOX_BYTES, 1024);
  accumulate = accumulate || half > 0;
  constexpr int NK = 128 / T::KSTEP;
#pragma unroll
  for (int kk = half * NK / 2; kk < (half + 1) * NK / 2; ++kk) {
    // KSTEP keys per step: P advances 8 32-bit columns (two bf16 or four E4M3 per column), V rows
    // by KSTEP x 128 bytes.
    const uint64_t voff = (uint64_t)((kk * T::KSTEP * 128) >> 4);
    if constexpr (F8)
      mma_ts_w_f8(tmem_d, tmem_p + kk * 8, vd + voff, T::IDESC_PV, (accumulate || kk > 0) ? 1u : 0u);
    else
      mma_ts_w(tmem_d, tmem_p + kk * 8, vd + voff, T::IDESC_PV, (accumulate || kk > 0) ? 1u : 0u);
  }
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Max over 64 values with short dependency chains (three-input max, four partial chains).
__device__ __forceinline__ float max64(const float* s) {
  float m0 = fmax3(s[0], s[1], s[2]), m1 = fmax3(s[3], s[4], s[5]);
  float m2 = fmax3(s[6], s[7], s[8]), m3 = fmax3(s[9], s[10], s[11]);
#pragma unroll
  for (int c = 12; c < 60; c += 8) {
    m0 = fmax3(m0, s[c], s[c + 1]);
    m1 = fmax3(m1, s[c + 2], s[c + 3]);
    m2 = fmax3(m2, s[c + 4], s[c + 5]);
    m3 = fmax3(m3, s[c + 6], s[c + 7]);
  }
  m0 = fmax3(m0, s[60], s[61]);
  m1 = fmax3(m1, s[62], s[63]);
  return fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
}

// Bias step of the EXT forward for the 64 keys of one row held in a staged bias box:
// s <- s + bias / scale (in pairs, one fused multiply-add each): the scores stay unscaled, as without
// a bias, and scale * log2(e) enters with the row maximum in the exponent's multiply-add, so that
// exp2((s + bias / scale) * scale * log2(e) - m) = exp(scale * s + bias) / 2^m.  The box is 128 rows of
// 128 bytes with 16-byte chunk c of row r at ((c ^ (r % 8)) * 16) (the 128-byte swizzle of the TMA
// box); keys past Nk and rows past Nq were filled with zeros by the TMA (those scores are -inf or
// never stored).
__device__ __forceinline__ void fwd_apply_bias_smem(float* s, const uint8_t* box, int r, float inv_scale) {
  const float2 inv2 = make_float2(inv_scale, inv_scale);
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    const uint4 raw = *reinterpret_cast<const uint4*>(box + r * 128 + ((g ^ (r & 7)) << 4));
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 v = ffma2(make_float2(bf16lo_to_f32(w[i]), bf16hi_to_f32(w[i])), inv2,
                             make_float2(s[8 * g + 2 * i], s[8 * g + 2 * i + 1]));
      s[8 * g + 2 * i] = v.x;
      s[8 * g + 2 * i + 1] = v.y;
    }
  }
}

// EXT: the scores get an additive bias (p.bias) and the weights dropout (p.drop) before P V.
template <int D, bool F8 = false, bool EXT = false>
__global__ void __launch_bounds__(FwdTraits<D, F8, EXT>::THREADS, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmB,
                  const FwdParams p) {
  static_assert(!(F8 && EXT), "bias and dropout are not combined with FP8 operands");
  using T = FwdTraits<D, F8, EXT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + T::OFF_BAR + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + T::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + T::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool two = p.tiles == 2;
  // Work items (query units of one (batch, head)), numbered heaviest first under the causal mask.
  // A CTA takes one item per round of gridDim.x items, in a snake order over the CTAs (forward in
  // even rounds, backward in odd ones), which evens out the causal work per CTA; with fewer items
  // than CTAs (the split mode) every CTA has exactly one.  Every role walks the same list, and the
  // K/V ring, the Q slots and all barrier phases run on across items.
  const int n_items = p.nunits * p.BH;
  const int G = gridDim.x;
  auto item_at = [&](int r) -> int { return r * G + ((r & 1) ? (G - 1 - (int)blockIdx.x) : (int)blockIdx.x); };
  auto decode = [&](int i) -> FwdItem {
    FwdItem w;
    w.bh = i % p.BH;
    const int rank = i / p.BH;
    const int unit = p.causal ? (p.nunits - 1 - rank) : rank;
    w.q0 = unit * 128 * p.tiles;
    w.n0 = fwd_num_kv_tiles(w.q0, 128, p.Nq, p.Nk, p.causal);
    w.n1 = two ? fwd_num_kv_tiles(w.q0 + 128, 128, p.Nq, p.Nk, p.causal) : w.n0;
    w.n_kv = max(w.n0, w.n1);
    return w;
  };
  int my_items = 0, total_loads = 0;
  for (int r = 0; item_at(r) < n_items; ++r) {
    ++my_items;
    total_loads += 2 * decode(item_at(r)).n_kv;
  }
  int issued = 0;           // K/V loads started by the TMA producer (its lane 0), for the teardown
  int q_fills[2] = {0, 0};  // Q loads per slot started by the TMA producer, for the teardown
  int b_fills[2] = {0, 0};  // bias tiles per group started by the bias loader, for the teardown
  const bool staged_bias = EXT && p.bias != nullptr;
  // Bias tiles group t consumes in item w, in its order: its key tiles j (two tiles: 0 .. n_t - 1;
  // split: t, t + 2, ...).
  auto n_bias = [&](const FwdItem& w, int t) { return two ? (t ? w.n1 : w.n0) : (w.n_kv + 1 - t) / 2; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(T::BAR_Q_FULL + s), 1);
      mbar_init(bar(T::BAR_Q_EMPTY + s), 1);
    }
    for (int s = 0; s < T::NS; ++s) {
      mbar_init(bar(T::BAR_KV_FULL + s), 1);
      mbar_init(bar(T::BAR_KV_EMPTY + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(T::BAR_S_FULL + t), 1);
      mbar_init(bar(T::BAR_P_READY + 2 * t), 128);
      mbar_init(bar(T::BAR_P_READY + 2 * t + 1), 128);
      mbar_init(bar(T::BAR_O_DONE + t), 1);
      mbar_init(bar(T::BAR_O_FREE + t), 128);
    }
    mbar_init(bar(T::BAR_DRAIN), 1);
    mbar_init(bar(T::BAR_MERGE), 128);
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(T::BAR_BIAS_FULL + t), 1);
      mbar_init(bar(T::BAR_BIAS_EMPTY + t), 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(tmem_slot), T::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 9 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == T::WARP_BIAS && lane == 0 && staged_bias) tma_prefetch_desc(&tmB);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 8) {
    // ------------------------------------------------------------------ softmax warpgroups
    // Two tiles: group t owns query tile t of each item.  Split (one query tile): group t visits
    // the item's key tiles t, t + 2, ... with its own running (m, l, O_t); group 0 merges.
    const int t = warp >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // row in the tile == TMEM lane
    const uint32_t lane_addr = tmem_base + ((uint32_t)(quarter * 32) << 16);
    const uint32_t colS = T::col_s(t), colO = T::col_o(t);
    bool ok = true;
    int cnt = 0;   // S tiles this group has processed in earlier items (barrier phases run on)
    int bcnt = 0;  // staged bias tiles this group has consumed
    for (int it = 0; ok && item_at(it) < n_items; ++it) {
      const FwdItem w = decode(item_at(it));
      const int bh = w.bh;
      const int row = w.q0 + (two ? 128 * t : 0) + r;  // query index within the head
      const int n_own = two ? (t ? w.n1 : w.n0) : (w.n_kv + 1 - t) / 2;  // key tiles this group visits
      int kmax = p.Nk - 1;  // last visible key of this row (inclusive)
      if (p.causal) kmax = min(kmax, row + p.Nk - p.Nq);
      float m_run = -INFINITY, l_run = 0.f, lr_run = 0.f;
      float scale_log2 = p.scale_log2;
      if constexpr (F8) scale_log2 *= __ldg(p.descale_q + bh) * __ldg(p.descale_k + bh);
      // EXT: the scores are turned into log2-domain logits s * scale * log2(e) + bias * log2(e) in
      // place, so the exponent step below multiplies by 1.
      const float2 sc2 = make_float2(scale_log2, scale_log2);
      [[maybe_unused]] const float inv_scale = 1.4426950408889634f / scale_log2;  // EXT: 1 / scale
      // EXT with a bias: this group's staged bias tile, one 64-key box per half of the scores.
      const uint8_t* bias_box = smem + T::OFF_BIAS + t * T::BIAS_TILE;
      for (int step = 0; step < n_own; ++step) {
        const int j = two ? step : 2 * step + t;  // key tile
        ok = __all_sync(0xffffffffu, mbar_wait(bar(T::BAR_S_FULL + t), (cnt + step) & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
        // Load the S row in two halves; the second half's load overlaps the first half's max.
        uint32_t sa[64], sb[64];
        tmem_ld32x32b_x64_nowait(lane_addr + colS, sa);
        tmem_wait_ld_x64(sa);
        tmem_ld32x32b_x64_nowait(lane_addr + colS + 64, sb);
        float* s = reinterpret_cast<float*>(sa);
        float* s2 = reinterpret_cast<float*>(sb);
        const int lim = kmax - 128 * j;  // keys [0, lim] of this tile are visible
        const bool masked = __any_sync(0xffffffffu, lim < 127);
        if (masked) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c > lim) s[c] = -INFINITY;
        }
        if constexpr (EXT) {
          if (staged_bias) {
            ok = __all_sync(0xffffffffu, mbar_wait(bar(T::BAR_BIAS_FULL + t), bcnt & 1, abort_flag));
            if (!ok) break;
            fwd_apply_bias_smem(s, bias_box, r, inv_scale);
          }
        }
        const float mx_a = max64(s);
        tmem_wait_ld_x64(sb);
        if (masked) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c + 64 > lim) s2[c] = -INFINITY;
        }
        if constexpr (EXT) {
          if (staged_bias) {
            fwd_apply_bias_smem(s2, bias_box + T::BIAS_TILE / 2, r, inv_scale);
            mbar_arrive(bar(T::BAR_BIAS_EMPTY + t));  // this tile's bias has been read
            ++bcnt;
          }
        }
        const float mx = fmaxf(mx_a, max64(s2));
        const float m_tile = mx * scale_log2;
        float alpha = 1.f;
        bool resc = false;
        if (m_tile > m_run + kRescaleThreshold) {
          alpha = ex2_approx(m_run - m_tile);
          resc = (step > 0) && (m_run != -INFINITY);
          m_run = m_tile;
        }
        const float base = (m_run == -INFINITY) ? 0.f : m_run;
        const float2 nb2 = make_float2(-base, -base);
        // O_t still holds the sum through this group's previous tile: when the max moved, it is
        // scaled before the first key half of this tile is published (after that half's weights,
        // when the first 64 scores are no longer needed).  That P V has completed already (it was
        // issued before this tile's S, whose completion this group has seen); the wait confirms it.
        const bool any_resc = __any_sync(0xffffffffu, resc);
        auto rescale_o = [&]() -> bool {
          if (!__all_sync(0xffffffffu, mbar_wait(bar(T::BAR_O_DONE + t), (cnt + step - 1) & 1, abort_flag)))
            return false;
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < D / 16; ++c) {
            uint32_t o[16];
            tmem_ld32x32b_x16_wait(lane_addr + colO + 16 * c, o);
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32x32b_x16(lane_addr + colO + 16 * c, o);
          }
          return true;
        };
        // Exponentials in four chunks of 32 keys; each chunk of P is stored to TMEM as soon as it is
        // ready, and each key half (two chunks) is published on its own barrier so that its P V
        // starts while the next half is computed.  Two row sums: exact (for LSE) and of the rounded
        // weights (normalises O so it stays a convex combination of V rows).
        float2 sum_e[2], sum_r[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) sum_e[i] = sum_r[i] = make_float2(0.f, 0.f);
        if constexpr (F8) {
          // E4M3 weights, four per 32-bit column (P <= 2^8 stays inside the format's 448).
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            const float* src = (ch < 2) ? s + 32 * ch : s2 + 32 * (ch - 2);
            uint32_t pk[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const float2 x0 = ffma2(make_float2(src[4 * c], src[4 * c + 1]), sc2, nb2);
              const float2 x1 = ffma2(make_float2(src[4 * c + 2], src[4 * c + 3]), sc2, nb2);
              const float2 e0 = make_float2(ex2_approx(x0.x), ex2_approx(x0.y));
              const float2 e1 = make_float2(ex2_approx(x1.x), ex2_approx(x1.y));
              const uint32_t lo = f32x2_to_e4m3x2(e0.x, e0.y), hi = f32x2_to_e4m3x2(e1.x, e1.y);
              pk[c] = lo | (hi << 16);
              sum_e[0] = fadd2(sum_e[0], e0);
              sum_e[1] = fadd2(sum_e[1], e1);
              sum_r[0] = fadd2(sum_r[0], e4m3x2_to_f32x2(lo));
              sum_r[1] = fadd2(sum_r[1], e4m3x2_to_f32x2(hi));
            }
            tmem_st32x32b_x8(lane_addr + colS + 8 * ch, pk);
            if (ch == 1 && any_resc && !(ok = rescale_o())) break;
            if (ch & 1) {
              tmem_st_wait();
              tc_fence_before();
              mbar_arrive(bar(T::BAR_P_READY + 2 * t + (ch >> 1)));
            }
          }
        } else {
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            const float* src = (ch < 2) ? s + 32 * ch : s2 + 32 * (ch - 2);
            uint32_t pk[16];
            uint32_t keep[8];  // EXT with dropout: 0xff per kept key of this chunk's 8 key quads
            if constexpr (EXT) {
              if (p.drop.p8 != 0)
                dropout_keep_rowwise(p.drop, (uint32_t)(32 * j + 8 * ch), (uint32_t)row, (uint32_t)bh, lane, keep);
            }
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const float2 x = ffma2(make_float2(src[2 * c], src[2 * c + 1]), sc2, nb2);
              const float2 e = make_float2(ex2_approx(x.x), ex2_approx(x.y));
              pk[c] = pack_bf16x2(e.x, e.y);
              sum_e[c & 1] = fadd2(sum_e[c & 1], e);
              sum_r[c & 1] = fadd2(sum_r[c & 1], make_float2(bf16lo_to_f32(pk[c]), bf16hi_to_f32(pk[c])));
              if constexpr (EXT) {
                // Dropped weights leave the normalising sums untouched and enter P V as +0.
                if (p.drop.p8 != 0) pk[c] &= __byte_perm(keep[c >> 1], 0u, (c & 1) ? 0x3322u : 0x1100u);
              }
            }
            tmem_st32x32b_x16(lane_addr + colS + 16 * ch, pk);
            if (ch == 1 && any_resc && !(ok = rescale_o())) break;
            if (ch & 1) {
              tmem_st_wait();
              tc_fence_before();
              mbar_arrive(bar(T::BAR_P_READY + 2 * t + (ch >> 1)));
            }
          }
        }
        if (!ok) break;
        const float2 tot_e = fadd2(sum_e[0], sum_e[1]);
        const float2 tot_r = fadd2(sum_r[0], sum_r[1]);
        l_run = l_run * alpha + (tot_e.x + tot_e.y);
        lr_run = lr_run * alpha + (tot_r.x + tot_r.y);
      }
      if (!ok) break;
      // This group's accumulator is complete once its last PV has landed.
      ok = __all_sync(0xffffffffu, mbar_wait(bar(T::BAR_O_DONE + t), (cnt + n_own - 1) & 1, abort_flag));
      cnt += n_own;
      float* merge_stats = reinterpret_cast<float*>(smem + T::OFF_Q + T::TILE_BYTES);  // split: slot 0 tile 1 unused
      if (ok && !two && t == 1) {
        // Split: publish (m, l, l of the rounded weights) for group 0, which merges both halves.
        merge_stats[r] = m_run;
        merge_stats[128 + r] = l_run;
        merge_stats[256 + r] = lr_run;
        mbar_arrive(bar(T::BAR_MERGE));
      }
      // Weights of O_0 and O_1 in the merged sum: the two-block identity of the online softmax (each
      // group's sums are relative to its own running maximum).
      float a0 = 1.f, a1 = 0.f;
      bool use1 = false;
      if (ok && !two && t == 0) {
        // Split (one item per CTA): group 1's statistics and (if it visited any key tile) its
        // accumulator.
        const int n1 = w.n_kv / 2;
        ok = __all_sync(0xffffffffu, mbar_wait(bar(T::BAR_MERGE), 0, abort_flag));
        if (ok && n1 > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar(T::BAR_O_DONE + 1), (n1 - 1) & 1, abort_flag));
        if (ok) {
          const float m1 = merge_stats[r], l1 = merge_stats[128 + r], lr1 = merge_stats[256 + r];
          const float m = fmaxf(m_run, m1);
          a0 = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - m);
          a1 = (m1 == -INFINITY) ? 0.f : ex2_approx(m1 - m);
          l_run = a0 * l_run + a1 * l1;
          lr_run = a0 * lr_run + a1 * lr1;
          m_run = m;
          use1 = n1 > 0;
        }
      }
      if (ok && (two || t == 0)) {
        tc_fence_after();
        float num = 1.f;
        if constexpr (F8) num = __ldg(p.descale_v + bh);
        if constexpr (EXT) num = p.drop.scale;
        const float inv = lr_run > 0.f ? num / lr_run : 0.f;
        const bool in_range = row < p.Nq;
        __nv_bfloat16* orow = p.o + ((size_t)bh * p.Nq + (in_range ? row : 0)) * D;
        // O chunk c (32 columns, already combined) / l -> bf16 -> the output row.
        auto put = [&](const uint32_t (&o)[32], int c) {
          uint32_t wv[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            wv[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
          if (in_range) {
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(wv[4 * i], wv[4 * i + 1], wv[4 * i + 2], wv[4 * i + 3]);
          }
        };
        bool released = false;  // O_FREE already signalled
        if constexpr (F8) {
          if (two) {
            // FP8, two-tile mode (measured faster there, not with bf16 operands): the four 32-column
            // chunks of O_t with loads in flight while earlier chunks are stored (a TMEM load wait
            // covers every load in flight), and the columns released as soon as the last chunk is in
            // registers.
            uint32_t oa[32], ob[32], oc[32];
            tmem_ld32x32b_x32_nowait(lane_addr + colO, oa);
            tmem_ld32x32b_x32_nowait(lane_addr + colO + 32, ob);
            tmem_wait_ld_2x32(oa, ob);
            tmem_ld32x32b_x32_nowait(lane_addr + colO + 64, oc);
            put(oa, 0);
            tmem_ld32x32b_x32_nowait(lane_addr + colO + 96, oa);
            put(ob, 1);
            tmem_wait_ld_2x32(oc, oa);
            tc_fence_before();
            mbar_arrive(bar(T::BAR_O_FREE + t));
            released = true;
            put(oc, 2);
            put(oa, 3);
          }
        }
        if (!released) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32x32b_x32_wait(lane_addr + colO + 32 * c, o);
            if (use1) {
              uint32_t o1[32];
              tmem_ld32x32b_x32_wait(lane_addr + T::col_o(1) + 32 * c, o1);
#pragma unroll
              for (int i = 0; i < 32; ++i)
                o[i] = __float_as_uint(a0 * __uint_as_float(o[i]) + a1 * __uint_as_float(o1[i]));
            } else if (!two) {
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(a0 * __uint_as_float(o[i]));
            }
            put(o, c);
          }
          // O_t is in registers and on its way out: the next item's first P V may overwrite it.
          tc_fence_before();
          mbar_arrive(bar(T::BAR_O_FREE + t));
        }
        if (in_range) p.lse[(size_t)bh * p.Nq + row] = l_run > 0.f ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
      }
    }
    if (!ok) *abort_flag = 1;
  } else if (warp == 8) {
    // ------------------------------------------------------------------ MMA issuer
    {  // the whole warp, converged: one elected lane issues
      auto release = [&](int load_idx) {
        // Only stages the producer will refill get an "empty" arrival.
        if (load_idx + T::NS < total_loads) mma_commit_w(bar(T::BAR_KV_EMPTY + load_idx % T::NS));
      };
      auto kv_smem = [&](int load_idx) { return sbase + T::OFF_KV + (load_idx % T::NS) * T::TILE_BYTES; };
      auto kv_wait = [&](int load_idx) {
        return warp_wait(bar(T::BAR_KV_FULL + load_idx % T::NS), (load_idx / T::NS) & 1, abort_flag);
      };
      const uint32_t tS[2] = {tmem_base + T::col_s(0), tmem_base + T::col_s(1)};
      const uint32_t tO[2] = {tmem_base + T::col_o(0), tmem_base + T::col_o(1)};
      // O_t += P_t V (V of load v_load): the first key half as soon as group t has published it, then
      // the second; c counts group t's tiles (barrier phase), acc: whether O_t already holds a sum.
      auto pv = [&](int t, int c, int v_load, bool acc) -> bool {
        for (int half = 0; half < 2; ++half) {
          if (!warp_wait(bar(T::BAR_P_READY + 2 * t + half), c & 1, abort_flag)) return false;
          tc_fence_after();
          fwd_issue_pv<D, F8>(tO[t], tS[t], kv_smem(v_load), half, acc);
        }
        mma_commit_w(bar(T::BAR_O_DONE + t));
        return true;
      };
      bool ok = true;
      int L = 0;                // global index of the item's first K/V load
      int cnt0 = 0, cnt1 = 0;   // S tiles of groups 0 / 1 in earlier items (barrier phases run on)
      for (int k = 0; ok && item_at(k) < n_items; ++k) {
        const FwdItem w = decode(item_at(k));
        const int slot = k % T::QSLOTS;
        const uint32_t q_smem[2] = {sbase + T::OFF_Q + (2 * slot) * T::TILE_BYTES,
                                    sbase + T::OFF_Q + (2 * slot + 1) * T::TILE_BYTES};
        if (!(ok = warp_wait(bar(T::BAR_Q_FULL + slot), (k / T::QSLOTS) & 1, abort_flag))) break;
        // The first P V of group t in this item overwrites O_t: group t must have read out the
        // previous item's output (two-tile mode; the split mode has one item per CTA).
        auto o_free = [&](int t) {
          return k == 0 || warp_wait(bar(T::BAR_O_FREE + t), (k - 1) & 1, abort_flag);
        };
        if (!two) {
          // Split: step i computes S_0 = Q K(2i)^T and S_1 = Q K(2i+1)^T, then O_0 += P_0 V(2i) and
          // (one step later, like the two-tile order) O_1 += P_1 V(2i+1).  Loads arrive in the ring
          // order K(j), V(j), K(j+1), V(j+1), ...
          const int n_kv = w.n_kv;
          const int nsteps = (n_kv + 1) / 2;
          int v1_prev = -1;  // load index of the V tile of group 1's pending PV
          for (int i = 0; ok && i < nsteps; ++i) {
            const int ik0 = L + 4 * i, iv0 = ik0 + 1, ik1 = ik0 + 2, iv1 = ik0 + 3;
            const bool has1 = 2 * i + 1 < n_kv;
            if (!(ok = kv_wait(ik0))) break;
            tc_fence_after();
            fwd_issue_qk<D, F8>(tS[0], q_smem[0], kv_smem(ik0));
            mma_commit_w(bar(T::BAR_S_FULL + 0));
            release(ik0);
            if (v1_prev >= 0) {
              if (!(ok = kv_wait(v1_prev))) break;
              if (!(ok = pv(1, cnt1 + i - 1, v1_prev, i - 1 > 0))) break;
              release(v1_prev);
              v1_prev = -1;
            }
            if (has1) {
              if (!(ok = kv_wait(ik1))) break;
              tc_fence_after();
              fwd_issue_qk<D, F8>(tS[1], q_smem[0], kv_smem(ik1));
              mma_commit_w(bar(T::BAR_S_FULL + 1));
              release(ik1);
              v1_prev = iv1;
            }
            if (!(ok = kv_wait(iv0))) break;
            if (!(ok = pv(0, cnt0 + i, iv0, i > 0))) break;
            release(iv0);
          }
          if (ok && v1_prev >= 0) {
            const int i = nsteps - 1;
            if ((ok = kv_wait(v1_prev)) && (ok = pv(1, cnt1 + i, v1_prev, i > 0))) release(v1_prev);
          }
          cnt0 += (n_kv + 1) / 2;
          cnt1 += n_kv / 2;
        } else {
          // Two tiles, in the order S0 S1 PV0 S0' PV1 S1' ...; query tile 0 skips the key tiles it
          // cannot see (j >= n0), tile 1 visits all n_kv = n1.
          int v_prev = -1;
          for (int j = 0; ok && j < w.n_kv; ++j) {
            const int ik = L + 2 * j, iv = ik + 1;
            if (!(ok = kv_wait(ik))) break;
            tc_fence_after();
            if (j < w.n0) {
              fwd_issue_qk<D, F8>(tS[0], q_smem[0], kv_smem(ik));
              mma_commit_w(bar(T::BAR_S_FULL + 0));
            }
            if (j > 0) {
              if (j == 1 && !(ok = o_free(1))) break;
              if (!(ok = pv(1, cnt1 + j - 1, v_prev, j - 1 > 0))) break;
              release(v_prev);
            }
            fwd_issue_qk<D, F8>(tS[1], q_smem[1], kv_smem(ik));
            mma_commit_w(bar(T::BAR_S_FULL + 1));
            release(ik);
            if (!(ok = kv_wait(iv))) break;
            if (j < w.n0) {
              if (j == 0 && !(ok = o_free(0))) break;
              if (!(ok = pv(0, cnt0 + j, iv, j > 0))) break;
            }
            v_prev = iv;
          }
          if (ok && w.n_kv == 1) ok = o_free(1);
          if (ok && (ok = pv(1, cnt1 + w.n_kv - 1, v_prev, w.n_kv - 1 > 0))) release(v_prev);
          cnt0 += w.n0;
          cnt1 += w.n1;
        }
        // Every S MMA of this item has been issued: its Q slot is free once they complete (the
        // commit tracks all earlier MMAs of this thread).  Only slots the producer refills.
        if (ok && k + T::QSLOTS < my_items) mma_commit_w(bar(T::BAR_Q_EMPTY + slot));
        L += 2 * w.n_kv;
      }
      if (!ok) *abort_flag = 1;
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      bool ok = true;
      int L = 0;  // global index of the item's first K/V load
      for (int k = 0; ok && item_at(k) < n_items; ++k) {
        const FwdItem w = decode(item_at(k));
        const int slot = k % T::QSLOTS;
        // The slot's previous item (k - QSLOTS) must have finished its S MMAs.
        if (k >= T::QSLOTS &&
            !(ok = mbar_wait(bar(T::BAR_Q_EMPTY + slot), ((k - T::QSLOTS) / T::QSLOTS) & 1, abort_flag)))
          break;
        mbar_arrive_expect_tx(bar(T::BAR_Q_FULL + slot), p.tiles * T::TILE_BYTES);
        for (int t = 0; t < p.tiles; ++t)
          for (int b = 0; b < T::NBOX; ++b)
            tma_load_3d(sbase + T::OFF_Q + (2 * slot + t) * T::TILE_BYTES + b * T::BOX_BYTES, &tmQ,
                        bar(T::BAR_Q_FULL + slot), T::BOX_COLS * b, w.q0 + 128 * t, w.bh);
        ++q_fills[slot];
        for (int idx = 0; idx < 2 * w.n_kv; ++idx) {
          const int g = L + idx;
          const int s = g % T::NS;
          if (!(ok = mbar_wait(bar(T::BAR_KV_EMPTY + s), ((g / T::NS) & 1) ^ 1, abort_flag))) break;
          mbar_arrive_expect_tx(bar(T::BAR_KV_FULL + s), T::TILE_BYTES);
          const CUtensorMap* map = (idx & 1) ? &tmV : &tmK;
          for (int b = 0; b < T::NBOX; ++b)
            tma_load_3d(sbase + T::OFF_KV + s * T::TILE_BYTES + b * T::BOX_BYTES, map, bar(T::BAR_KV_FULL + s),
                        T::BOX_COLS * b, 128 * (idx >> 1), w.bh);
          issued = g + 1;
        }
        L += 2 * w.n_kv;
      }
      if (!ok) *abort_flag = 1;
    }
    __syncwarp();
  } else if (EXT && warp == T::WARP_BIAS) {
    // ------------------------------------------------------------------ bias tiles (TMA)
    // Group t's next bias tile goes into its buffer as soon as the group has read the previous one;
    // the tiles follow each group's own order of key tiles, the two groups interleaved.  A group
    // releases a tile using only tiles loaded before it, so the interleaving cannot deadlock.
    if (lane == 0 && staged_bias) {
      bool ok = true;
      for (int k = 0; ok && item_at(k) < n_items; ++k) {
        const FwdItem w = decode(item_at(k));
        const int plane = (w.bh / p.H) * p.bias_pb + (w.bh % p.H) * p.bias_ph;
        const int nb0 = n_bias(w, 0), nb1 = n_bias(w, 1);
        for (int st = 0; ok && st < max(nb0, nb1); ++st) {
          for (int t = 0; t < 2; ++t) {
            if (st >= (t ? nb1 : nb0)) continue;
            const int j = two ? st : 2 * st + t;  // key tile
            const int row0 = w.q0 + (two ? 128 * t : 0);
            if (b_fills[t] > 0 &&
                !(ok = mbar_wait(bar(T::BAR_BIAS_EMPTY + t), (b_fills[t] - 1) & 1, abort_flag)))
              break;
            mbar_arrive_expect_tx(bar(T::BAR_BIAS_FULL + t), T::BIAS_TILE);
            for (int b = 0; b < 2; ++b)
              tma_load_3d(sbase + T::OFF_BIAS + t * T::BIAS_TILE + b * (T::BIAS_TILE / 2), &tmB,
                          bar(T::BAR_BIAS_FULL + t), 128 * j + 64 * b, row0, plane);
            ++b_fills[t];
          }
        }
      }
      if (!ok) *abort_flag = 1;
    }
    __syncwarp();
  }

  // Teardown.  On the normal path every copy and MMA has been consumed by now.  If any warp gave
  // up, the others have stopped too (they poll the abort flag); then the CTA still waits for its
  // own work in flight (fixed-limit waits): the MMAs before tensor memory is freed, the copies
  // before shared memory is given back with the CTA's exit.
  if (warp < 8) tmem_st_wait();
  tc_fence_before();
  __syncthreads();
  const bool aborted = *abort_flag != 0;
  if (warp == 8) {
    if (aborted) {
      mma_commit_w(bar(T::BAR_DRAIN));
      warp_drain_wait(bar(T::BAR_DRAIN), 0);
    }
    tc_fence_after();
    tmem_dealloc(tmem_base, T::TMEM_COLS);
  } else if (warp == 9 && lane == 0 && aborted) {
    for (int idx = max(0, issued - T::NS); idx < issued; ++idx)
      drain_wait(bar(T::BAR_KV_FULL + idx % T::NS), (idx / T::NS) & 1);
    for (int slot = 0; slot < 2; ++slot)
      if (q_fills[slot] > 0) drain_wait(bar(T::BAR_Q_FULL + slot), (q_fills[slot] - 1) & 1);
  } else if (EXT && warp == T::WARP_BIAS && lane == 0 && aborted) {
    for (int t = 0; t < 2; ++t)
      if (b_fills[t] > 0) drain_wait(bar(T::BAR_BIAS_FULL + t), (b_fills[t] - 1) & 1);
  }
}

// Nk == 0: every row sees no key.
__global__ void fa_fwd_empty_kernel(__nv_bfloat16* o, float* lse, long long rows, int D) {
  const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (i < rows * D) o[i] = __float2bfloat16(0.f);
  if (i < rows) lse[i] = -INFINITY;
}

}  // namespace fa
