// Deterministic dQ for the backward pass (sm_100a): dQ_i = scale * sum_j dS_ij K_j with the
// query block stationary.
//
// Method: the recomputation backward of "FlashAttention 的基本原理" (section 2.4 反向传播) —
// P rebuilt from the saved LSE, dP = dO V^T, dS = P * (dP - D), dQ = dS K — scheduled the other
// way round from fa_bwd_main_kernel: one CTA owns a 128-row query block and key / value blocks
// stream past it, as in the forward.  No two CTAs write the same dQ row, so dQ needs no
// atomics and is bitwise reproducible; the price is computing S and dP a second time (they are
// also computed by the dK / dV kernel).  The pages name the atomic adds of the key-block
// schedule as the source of the nondeterminism ("Transformer、注意力机制与优化", section
// 为什么前向传播和反向传播的并行化策略不同).
//
// B200 design:
//  * TMA: Q and dO once, K and V tiles through a shared-memory ring (128-byte swizzle);
//  * tcgen05: S = Q K^T and dP = dO V^T (both operands in shared memory) into TMEM, then
//    dQ += dS K with dS (bf16) staged in shared memory; TMEM: S | dP | dQ = 128 + 128 + d;
//  * two compute warpgroups split each S / dP tile by keys (group g: keys 64 g .. 64 g + 63),
//    thread = query row = TMEM lane; the next tile's S and dP are issued as soon as both groups
//    hold the current ones in registers, so the recomputation overlaps the dS arithmetic;
//  * one converged MMA-issuing warp, one TMA warp.
#pragma once

#include "bwd_sm100.cuh"  // kLog2e

namespace fa {

template <int D>
struct DqTraits {
  static_assert(D == 64 || D == 128, "head dim");
  static constexpr int NBOX = D / 64;
  static constexpr int BOX_BYTES = 128 * 64 * 2;       // 16 KB
  static constexpr int TILE_BYTES = NBOX * BOX_BYTES;  // one 128 x D bf16 tile
  static constexpr int NS = (D == 64) ? 8 : 4;         // K/V ring stages (>= 4: see the issuer)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = TILE_BYTES;
  static constexpr int OFF_DS = 2 * TILE_BYTES;             // 128 rows x 128 keys bf16, two 64-key boxes
  static constexpr int OFF_KV = OFF_DS + 2 * BOX_BYTES;
  static constexpr int OFF_BAR = OFF_KV + NS * TILE_BYTES;
  // barriers: qd | kv_full[NS] | kv_empty[NS] | sd_full | sd_used | ds_ready | ds_free | dq_done | drain
  static constexpr int BAR_QD = 0;
  static constexpr int BAR_KV_FULL = 1;
  static constexpr int BAR_KV_EMPTY = 1 + NS;
  static constexpr int BAR_SD_FULL = 1 + 2 * NS;     // S_j and dP_j are in TMEM
  static constexpr int BAR_SD_USED = BAR_SD_FULL + 1;  // both groups hold S_j and dP_j in registers
  static constexpr int BAR_DS_READY = BAR_SD_FULL + 2; // dS_j staged in shared memory
  static constexpr int BAR_DS_FREE = BAR_SD_FULL + 3;  // the dQ MMA of key block j has read dS_j
  static constexpr int BAR_DQ_DONE = BAR_SD_FULL + 4;
  static constexpr int BAR_DRAIN = BAR_SD_FULL + 5;
  static constexpr int NBAR = BAR_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base (u32), abort flag (int)
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DQ = 256;
  static constexpr int THREADS = 320;  // warps 0-7 compute (group = warp / 4), 8 MMA issuer, 9 TMA
  static constexpr uint32_t IDESC_QK = make_idesc_bf16(128, 128, false, false);  // Q K^T, dO V^T
  static constexpr uint32_t IDESC_DQ = make_idesc_bf16(128, D, false, true);     // dS (K-major) K (MN-major)
};

struct DqParams {
  __nv_bfloat16* dq;  // [BH, Nq, D], written
  const float* lse;   // [BH, Nq]
  const float* dvec;  // [BH, Nq]
  int Nq, Nk, BH, nqt;
  float scale, scale_log2;
  int causal;
};

// Key blocks the query block [q0, q0 + 128) sees (bottom-right causal alignment); at least one.
__device__ __forceinline__ int dq_num_kv_tiles(int q0, int Nq, int Nk, int causal) {
  const int nkt = (Nk + 127) / 128;
  if (!causal) return nkt;
  const int kmax = min(q0 + 127, Nq - 1) + Nk - Nq;
  if (kmax < 0) return 1;
  return min(nkt, kmax / 128 + 1);
}

template <int D>
__device__ __forceinline__ void dq_issue_kmajor(uint32_t tmem_d, uint32_t a_smem, uint32_t b_smem) {
  using T = DqTraits<D>;
  const uint64_t ad = make_sdesc_sw128(a_smem, 16, 1024), bd = make_sdesc_sw128(b_smem, 16, 1024);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint64_t off = (uint64_t)(((kk / 4) * T::BOX_BYTES + (kk % 4) * 32) >> 4);
    mma_ss_w(tmem_d, ad + off, bd + off, T::IDESC_QK, kk > 0 ? 1u : 0u);
  }
}

template <int D>
__global__ void __launch_bounds__(DqTraits<D>::THREADS, 1)
    fa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                     const DqParams p) {
  using T = DqTraits<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + T::OFF_BAR + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + T::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + T::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x % p.BH;
  const int rank = blockIdx.x / p.BH;
  const int q0 = (p.causal ? (p.nqt - 1 - rank) : rank) * 128;  // causal: heaviest blocks first
  const int n_kv = dq_num_kv_tiles(q0, p.Nq, p.Nk, p.causal);

  if (threadIdx.x == 0) {
    mbar_init(bar(T::BAR_QD), 1);
    for (int s = 0; s < T::NS; ++s) {
      mbar_init(bar(T::BAR_KV_FULL + s), 1);
      mbar_init(bar(T::BAR_KV_EMPTY + s), 1);
    }
    mbar_init(bar(T::BAR_SD_FULL), 1);
    mbar_init(bar(T::BAR_SD_USED), 256);
    mbar_init(bar(T::BAR_DS_READY), 256);
    mbar_init(bar(T::BAR_DS_FREE), 1);
    mbar_init(bar(T::BAR_DQ_DONE), 1);
    mbar_init(bar(T::BAR_DRAIN), 1);
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
    tma_prefetch_desc(&tmDO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 8) {
    // ------------------------------------------------------------------ compute warpgroups
    const int g = warp >> 2;  // keys 64 g .. 64 g + 63 of every key block
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // query row in the block == TMEM lane
    const int row = q0 + r;
    const bool in = row < p.Nq;
    const uint32_t lane_addr = tmem_base + ((uint32_t)(quarter * 32) << 16);
    // This row's statistics, negated: -LSE in log2 units (-inf past Nq: P = 0) and -D.
    const size_t gi = (size_t)bh * p.Nq + (in ? row : 0);
    const float2 nl2 = make_float2(in ? -p.lse[gi] * kLog2e : -INFINITY, in ? -p.lse[gi] * kLog2e : -INFINITY);
    const float2 nd2 = make_float2(in ? -p.dvec[gi] : 0.f, in ? -p.dvec[gi] : 0.f);
    int kmax = p.Nk - 1;
    if (p.causal) kmax = min(kmax, row + p.Nk - p.Nq);
    const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
    const uint32_t ds_row = sbase + T::OFF_DS + g * T::BOX_BYTES + r * 128;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar(T::BAR_SD_FULL), j & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[64], dpv[64];
      tmem_ld32x32b_x64_nowait(lane_addr + T::COL_S + 64 * g, sv);
      tmem_ld32x32b_x64_nowait(lane_addr + T::COL_DP + 64 * g, dpv);
      tmem_wait_ld_2x64(sv, dpv);
      // S_j and dP_j are in registers: the issuer may compute the next key block's.
      tc_fence_before();
      mbar_arrive(bar(T::BAR_SD_USED));
      const int lim = kmax - 128 * j - 64 * g;  // own keys [0, lim] of this block are visible
      const bool masked = __any_sync(0xffffffffu, lim < 63);
      uint32_t dk[32];
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        const float2 x = ffma2(make_float2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), sc2, nl2);
        float2 pr = make_float2(ex2_approx(x.x), ex2_approx(x.y));
        if (masked) {
          pr.x = (c > lim) ? 0.f : pr.x;
          pr.y = (c + 1 > lim) ? 0.f : pr.y;
        }
        const float2 t = fadd2(make_float2(__uint_as_float(dpv[c]), __uint_as_float(dpv[c + 1])), nd2);
        const float2 ds = fmul2(pr, t);
        dk[c / 2] = pack_bf16x2(ds.x, ds.y);
      }
      // dS_{j-1} must have been read by its dQ MMA before this block's overwrites it.
      if (j > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(T::BAR_DS_FREE), (j - 1) & 1, abort_flag));
        if (!ok) break;
      }
      // dS row r, this group's 64 keys: K-major with 128-byte swizzle (16-byte chunk c of the row
      // at (c ^ r mod 8) * 16), the layout of the dQ MMA's A operand.
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t addr = ds_row + ((c ^ (r & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(dk[4 * c]), "r"(dk[4 * c + 1]),
                     "r"(dk[4 * c + 2]), "r"(dk[4 * c + 3])
                     : "memory");
      }
      fence_proxy_async_smem();
      mbar_arrive(bar(T::BAR_DS_READY));
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(T::BAR_DQ_DONE), 0, abort_flag));
    if (ok) {
      tc_fence_after();
      // Each group writes half of the row's dQ columns, scaled.
      __nv_bfloat16* out = p.dq + gi * D + (D / 2) * g;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t v[32];
        tmem_ld32x32b_x32_wait(lane_addr + T::COL_DQ + (D / 2) * g + 32 * c, v);
        if (in) {
          uint4* dst = reinterpret_cast<uint4*>(out + 32 * c);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * i]) * p.scale, __uint_as_float(v[8 * i + 1]) * p.scale),
                                pack_bf16x2(__uint_as_float(v[8 * i + 2]) * p.scale, __uint_as_float(v[8 * i + 3]) * p.scale),
                                pack_bf16x2(__uint_as_float(v[8 * i + 4]) * p.scale, __uint_as_float(v[8 * i + 5]) * p.scale),
                                pack_bf16x2(__uint_as_float(v[8 * i + 6]) * p.scale, __uint_as_float(v[8 * i + 7]) * p.scale));
        }
      }
    } else {
      *abort_flag = 1;
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------------ MMA issuer
    // The whole warp, converged; one elected lane issues.  Ring order: K_0, V_0, K_1, V_1, ...;
    // V_j is released after dP_j, K_j after dQ_j.  While the issuer waits for K_{j+1} and V_{j+1},
    // K_j is the only load it holds, so NS >= 4 stages cannot deadlock the producer.
    const int total_loads = 2 * n_kv;
    auto release = [&](int li) {
      if (li + T::NS < total_loads) mma_commit_w(bar(T::BAR_KV_EMPTY + li % T::NS));
    };
    auto stage = [&](int li) { return sbase + T::OFF_KV + (li % T::NS) * T::TILE_BYTES; };
    auto wait_load = [&](int li) {
      return warp_wait(bar(T::BAR_KV_FULL + li % T::NS), (li / T::NS) & 1, abort_flag);
    };
    auto issue_sd = [&](int j) {  // S_j = Q K_j^T, dP_j = dO V_j^T
      const bool w = wait_load(2 * j) && wait_load(2 * j + 1);
      if (w) {
        tc_fence_after();
        dq_issue_kmajor<D>(tmem_base + T::COL_S, sbase + T::OFF_Q, stage(2 * j));
        dq_issue_kmajor<D>(tmem_base + T::COL_DP, sbase + T::OFF_DO, stage(2 * j + 1));
        mma_commit_w(bar(T::BAR_SD_FULL));
        release(2 * j + 1);
      }
      return w;
    };
    const uint64_t ds_kmaj = make_sdesc_sw128(sbase + T::OFF_DS, 16, 1024);  // dS as A, K-major
    bool ok = warp_wait(bar(T::BAR_QD), 0, abort_flag) && issue_sd(0);
    for (int j = 0; ok && j < n_kv; ++j) {
      if (!(ok = warp_wait(bar(T::BAR_SD_USED), j & 1, abort_flag))) break;
      if (j + 1 < n_kv && !(ok = issue_sd(j + 1))) break;
      if (!(ok = warp_wait(bar(T::BAR_DS_READY), j & 1, abort_flag))) break;
      tc_fence_after();
      // dQ += dS_j K_j: K runs over the block's 128 keys (two 64-key boxes of dS; K rows
      // 16 keys = 2048 bytes per step in the MN-major view of the K tile).
      const uint64_t k_mn = make_sdesc_sw128(stage(2 * j), T::BOX_BYTES, 1024);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ss_w(tmem_base + T::COL_DQ, ds_kmaj + (uint64_t)(((kk / 4) * T::BOX_BYTES + (kk % 4) * 32) >> 4),
                 k_mn + (uint64_t)((kk * 2048) >> 4), T::IDESC_DQ, (j > 0 || kk > 0) ? 1u : 0u);
      mma_commit_w(bar(T::BAR_DS_FREE));
      release(2 * j);
    }
    if (ok) mma_commit_w(bar(T::BAR_DQ_DONE));
    if (!ok) {
      *abort_flag = 1;
      mma_commit_w(bar(T::BAR_DRAIN));
      warp_drain_wait(bar(T::BAR_DRAIN), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_arrive_expect_tx(bar(T::BAR_QD), 2 * T::TILE_BYTES);
      for (int b = 0; b < T::NBOX; ++b) {
        tma_load_3d(sbase + T::OFF_Q + b * T::BOX_BYTES, &tmQ, bar(T::BAR_QD), 64 * b, q0, bh);
        tma_load_3d(sbase + T::OFF_DO + b * T::BOX_BYTES, &tmDO, bar(T::BAR_QD), 64 * b, q0, bh);
      }
      const int total_loads = 2 * n_kv;
      bool ok = true;
      int issued = 0;
      for (int idx = 0; idx < total_loads; ++idx) {
        const int s = idx % T::NS;
        if (!(ok = mbar_wait(bar(T::BAR_KV_EMPTY + s), ((idx / T::NS) & 1) ^ 1, abort_flag))) break;
        mbar_arrive_expect_tx(bar(T::BAR_KV_FULL + s), T::TILE_BYTES);
        const CUtensorMap* map = (idx & 1) ? &tmV : &tmK;
        for (int b = 0; b < T::NBOX; ++b)
          tma_load_3d(sbase + T::OFF_KV + s * T::TILE_BYTES + b * T::BOX_BYTES, map, bar(T::BAR_KV_FULL + s),
                      64 * b, 128 * (idx >> 1), bh);
        issued = idx + 1;
      }
      if (!ok) {
        *abort_flag = 1;
        for (int idx = max(0, issued - T::NS); idx < issued; ++idx)
          drain_wait(bar(T::BAR_KV_FULL + idx % T::NS), (idx / T::NS) & 1);
        drain_wait(bar(T::BAR_QD), 0);
      }
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem_base, T::TMEM_COLS);
  }
}

}  // namespace fa
