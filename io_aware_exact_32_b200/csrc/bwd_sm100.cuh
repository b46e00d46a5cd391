// Attention backward for sm_100a by recomputation.
//
// Method ("FlashAttention 的基本原理", section 2.4 反向传播; "FlashAttention 系列技术详解",
// sections 反向传播步骤 and 具体优化策略): the forward saved only O and L = logsumexp.  For
// every (query block i, key block j) the scores are recomputed, P = exp(scale S - L), and
//   dV_j += P^T dO_i,  dP = dO_i V_j^T,  dS = P * (dP - D_i),  dK_j += scale dS^T Q_i,
//   dQ_i += scale dS K_j,  with D_i = rowsum(dO_i * O_i).
// Work is split over key/value blocks ("Transformer、注意力机制与优化", section 为什么前向
// 传播和反向传播的并行化策略不同): each CTA owns one key block, keeps dK_j and dV_j on chip, and
// adds its dQ_i contributions to an fp32 accumulator in device memory with TMA bulk reduce-adds.
//
// Kernels:
//   fa_bwd_preprocess_kernel  D = rowsum(dO * O) (fp32) and zero the dQ accumulator
//   fa_bwd_main_kernel        the loop above for one 128-key block per CTA (tcgen05 + TMA)
//   fa_bwd_dq_convert_kernel  dQ accumulator (fp32) -> dQ (bf16)
//
// Main-kernel layout (computed transposed, keys on TMEM lanes, so that dK/dV rows and the
// P^T operand of dV = P^T dO live on the lane that owns the key):
//   TMEM: S^T (128 cols) | dP^T (128 cols) | dV (d) | dK (d) | dQ (d = 64 only; at d = 128 the
//         dQ block reuses the dP^T columns once dP^T has been consumed)
//   SMEM: K_j, V_j (resident), a ring of (Q_i, dO_i) stages, dS^T (bf16, 128-byte swizzle),
//         and at d = 64 an fp32 staging tile for the dQ block
//   P/dS warpgroups: one thread per key row, two groups of 64 query columns each: P, dS (the
//              critical path); group 0 also runs the dK/dV epilogue
//   dQ warpgroup: one thread per query row of the dQ block: read it out of TMEM, release the
//              columns, then add it into the fp32 accumulator with TMA bulk reduce-adds of a staged
//              tile (d = 64: its own staging buffer; d = 128: the block's dO tile once dV has read it)
//   MMA issuer A (S^T, dV: the users of the S^T/P^T columns), MMA issuer B (dP^T, dQ, dK),
//   and a TMA producer warp.
// Two issuers because one thread issues at most one 128 x N x 16 MMA every ~115 cycles
// (measured on B200), about half the tensor-core rate at N = 128.  Each issuer runs one
// iteration ahead: right after the MMAs that consume block i it issues the next block's S^T /
// dP^T, so the compute warps wait only for those.  Barriers that must see both issuers' work
// (S^T and dP^T ready, a Q/dO stage free, final dK/dV) count two commits.
#pragma once

#include <type_traits>

#include "dropout_sm100.cuh"

namespace fa {

constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct BwdTraits {
  static_assert(D == 64 || D == 128, "head dim");
  static constexpr bool SEP_DQ = (D == 64);            // dQ block has its own TMEM columns + TMA reduce
  static constexpr int NBOX = D / 64;
  static constexpr int BOX_BYTES = 128 * 64 * 2;       // 16 KB
  static constexpr int TILE_BYTES = NBOX * BOX_BYTES;  // 128 x D bf16
  static constexpr int NS = (D == 64) ? 3 : 2;         // (Q, dO) stages
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = TILE_BYTES;
  static constexpr int OFF_QD = 2 * TILE_BYTES;              // stage s: Q at +0, dO at +TILE_BYTES
  static constexpr int OFF_DS = OFF_QD + NS * 2 * TILE_BYTES;  // 128 keys x 128 queries bf16 = 32 KB
  static constexpr int OFF_STG = OFF_DS + 2 * BOX_BYTES;       // dQ staging, 2 x (128 rows x 32 fp32) (d = 64)
  static constexpr int STG_BYTES = SEP_DQ ? 128 * 64 * 4 : 0;
  static constexpr int OFF_STAT = OFF_STG + STG_BYTES;         // [2][128] fp32: LSE*log2e, D
  static constexpr int OFF_BAR = OFF_STAT + 2 * 128 * 4;
  // barriers: kv_full | qd_full[NS] | qd_empty[NS] | s_full | ds_ready | ds_free | dq_full | dq_free |
  //           acc_done | drain A | drain B | sd_used | p_free
  static constexpr int BAR_KV = 0;
  static constexpr int BAR_QD_FULL = 1;
  static constexpr int BAR_QD_EMPTY = 1 + NS;
  static constexpr int BAR_S_FULL = 1 + 2 * NS;
  static constexpr int BAR_DS_READY = BAR_S_FULL + 1;
  static constexpr int BAR_DS_FREE = BAR_S_FULL + 2;
  static constexpr int BAR_DQ_FULL = BAR_S_FULL + 3;
  static constexpr int BAR_DQ_FREE = BAR_S_FULL + 4;
  static constexpr int BAR_ACC_DONE = BAR_S_FULL + 5;
  static constexpr int BAR_DRAIN = BAR_S_FULL + 6;
  static constexpr int BAR_DRAIN2 = BAR_S_FULL + 7;
  static constexpr int BAR_SD_USED = BAR_S_FULL + 8;  // S^T/dP^T of block i are in registers
  static constexpr int BAR_P_FREE = BAR_S_FULL + 9;   // dV(i) has read P^T(i)
  static constexpr int BAR_DO_FREE = BAR_S_FULL + 10; // dV(i) has read dO(i) (d = 128: staging)
  static constexpr int BAR_DQ_ISSUED = BAR_S_FULL + 11;  // issuer B has issued dQ(i): issuer A may issue dV(i)
  static constexpr int NBAR = BAR_DQ_ISSUED + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DV = 256, COL_DK = 256 + D;
  static constexpr uint32_t COL_DQ = SEP_DQ ? 256 + 2 * D : COL_DP;
  // Two P/dS warpgroups split the 128 query columns of every key row (the per-row chain of TMEM
  // loads and exponentials is the critical path); each writes its 64 columns of P^T (32 TMEM
  // columns of bf16 pairs).  d = 64: P^T has its own 64 columns, so the next block's S^T can be
  // computed while this block's P^T still feeds dV.  d = 128: no room; each group's P^T
  // overwrites the start of its own, already read, half of S^T.
  static constexpr bool EARLY = SEP_DQ;
  static constexpr uint32_t COL_P = EARLY ? 256 + 3 * D : COL_S;
  static constexpr uint32_t P_WG_STRIDE = EARLY ? 32 : 64;  // TMEM columns between the groups' P^T
  static __host__ __device__ constexpr uint32_t p_col(int kk) {  // P^T columns of K-step kk (16 queries)
    return COL_P + (uint32_t)(kk / 4) * P_WG_STRIDE + (uint32_t)(kk % 4) * 8;
  }
  static constexpr int NCWG = 2;
  static constexpr int CW = 128 / NCWG;                 // query columns per P/dS warpgroup
  static constexpr int WARP_DQ = 4 * NCWG;              // first warp of the dQ warpgroup
  static constexpr int WARP_A = WARP_DQ + 4, WARP_B = WARP_DQ + 5, WARP_TMA = WARP_DQ + 6;
  static constexpr int THREADS = 32 * (WARP_TMA + 1);
  static constexpr uint32_t IDESC_SQ = make_idesc_bf16(128, 128, false, false);  // K Q^T, V dO^T
  static constexpr uint32_t IDESC_DVK = make_idesc_bf16(128, D, false, true);    // P^T dO, dS^T Q
  static constexpr uint32_t IDESC_DQ = make_idesc_bf16(128, D, true, true);      // dS K
};

struct BwdParams {
  const float* lse;   // [BH, Nq]
  const float* dvec;  // [BH, Nq]
  float* dq_acc;      // [BH, Nq, D]
  __nv_bfloat16* dk;  // [BH, Nk, D]
  __nv_bfloat16* dv;  // [BH, Nk, D]
  int Nq, Nk, BH, nkt;
  int hgroup;         // heads per scheduling group (1 <= hgroup <= BH)
  float scale, scale_log2;
  int causal;
  // Bias and dropout instantiation only (as in FwdParams).
  const __nv_bfloat16* bias;
  long long bias_sb, bias_sh;
  int bias_pb, bias_ph;
  int H;
  DropoutCfg drop;
};

// ---------------------------------------------------------------------------------------------
// D_i = sum_k dO_ik O_ik and dQ accumulator zeroing.  One warp per query row.
// ---------------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_preprocess_kernel(const __nv_bfloat16* __restrict__ o,
                                                                const __nv_bfloat16* __restrict__ dout,
                                                                float* __restrict__ dvec,
                                                                float* __restrict__ dq_acc, long long rows) {
  const long long row = blockIdx.x * 8ll + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  constexpr int PER = D / 32;  // elements per lane (2 or 4)
  const __nv_bfloat16* orow = o + row * D + lane * PER;
  const __nv_bfloat16* drow = dout + row * D + lane * PER;
  float acc = 0.f;
  if constexpr (PER == 4) {
    const uint2 a = *reinterpret_cast<const uint2*>(orow);
    const uint2 b = *reinterpret_cast<const uint2*>(drow);
    acc = bf16lo_to_f32(a.x) * bf16lo_to_f32(b.x) + bf16hi_to_f32(a.x) * bf16hi_to_f32(b.x) +
          bf16lo_to_f32(a.y) * bf16lo_to_f32(b.y) + bf16hi_to_f32(a.y) * bf16hi_to_f32(b.y);
  } else {
    const uint32_t a = *reinterpret_cast<const uint32_t*>(orow);
    const uint32_t b = *reinterpret_cast<const uint32_t*>(drow);
    acc = bf16lo_to_f32(a) * bf16lo_to_f32(b) + bf16hi_to_f32(a) * bf16hi_to_f32(b);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) dvec[row] = acc;
  if (dq_acc) {  // null in the deterministic backward, which has no accumulator
    float* qrow = dq_acc + row * D + lane * PER;
#pragma unroll
    for (int i = 0; i < PER; ++i) qrow[i] = 0.f;
  }
}

// dQ accumulator (already scaled) -> bf16, 8 elements per thread.
__global__ void __launch_bounds__(256) fa_bwd_dq_convert_kernel(const float* __restrict__ acc,
                                                                __nv_bfloat16* __restrict__ dq, long long n8) {
  const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
  const float4 b = reinterpret_cast<const float4*>(acc)[2 * i + 1];
  reinterpret_cast<uint4*>(dq)[i] =
      make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
}

// First query block that sees key k0, under the bottom-right causal alignment.
__device__ __forceinline__ int bwd_first_q_tile(int k0, int Nq, int Nk, int causal) {
  if (!causal) return 0;
  const int qmin = k0 - (Nk - Nq);
  return qmin <= 0 ? 0 : qmin / 128;
}

template <int D>
__device__ __forceinline__ void bwd_issue_ss_kmajor(uint32_t tmem_d, uint32_t a_smem, uint32_t b_smem) {
  using T = BwdTraits<D>;
  const uint64_t ad = make_sdesc_sw128(a_smem, 16, 1024), bd = make_sdesc_sw128(b_smem, 16, 1024);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint64_t off = (uint64_t)(((kk / 4) * T::BOX_BYTES + (kk % 4) * 32) >> 4);
    mma_ss_w(tmem_d, ad + off, bd + off, T::IDESC_SQ, kk > 0 ? 1u : 0u);
  }
}


// DQ = false (the deterministic backward): dK and dV only; dQ comes from fa_bwd_dq_kernel.
// EXT: the forward had an additive bias (p.bias) and dropout (p.drop): P is recomputed with the
// bias, dV uses the dropped and rescaled weights P o Z, and dS = P o (dP o Z - D).
template <int D, bool DQ = true, bool EXT = false>
__global__ void __launch_bounds__(BwdTraits<D>::THREADS, 1)
    fa_bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                       const __grid_constant__ CUtensorMap tmDQ, const __grid_constant__ CUtensorMap tmB,
                       const BwdParams p) {
  using T = BwdTraits<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + T::OFF_BAR + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + T::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + T::OFF_MISC + 4);
  float* stat = reinterpret_cast<float*>(smem + T::OFF_STAT);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Blocks run in groups of hgroup heads; inside a group, every key tile of those heads, the
  // heaviest (causal) first.  The group's Q, dO and dQ accumulator then stay in L2 while its
  // blocks sweep them, each block starting at its own query tile.
  const int grp = blockIdx.x / (p.hgroup * p.nkt);
  const int gsz = min(p.hgroup, p.BH - grp * p.hgroup);
  const int r_in = blockIdx.x - grp * p.hgroup * p.nkt;
  const int bh = grp * p.hgroup + r_in % gsz;
  const int jt = r_in / gsz;
  const int k0 = jt * 128;
  const int nqt = (p.Nq + 127) / 128;
  const int i0 = bwd_first_q_tile(k0, p.Nq, p.Nk, p.causal);
  const int n_q = max(0, nqt - i0);

  if (threadIdx.x == 0) {
    mbar_init(bar(T::BAR_KV), 1);
    for (int s = 0; s < T::NS; ++s) {
      mbar_init(bar(T::BAR_QD_FULL + s), 1);
      // issuer B after dK; issuer A after dV (d = 64) or the dQ warpgroup once its staging in the
      // dO tile is read out (d = 128)
      mbar_init(bar(T::BAR_QD_EMPTY + s), 2);
    }
    mbar_init(bar(T::BAR_S_FULL), 2);  // issuer A after S^T, issuer B after dP^T
    mbar_init(bar(T::BAR_DS_READY), 128 * T::NCWG);
    mbar_init(bar(T::BAR_DS_FREE), 1);  // issuer B after dQ and dK (the readers of dS^T)
    mbar_init(bar(T::BAR_DQ_FULL), 1);
    mbar_init(bar(T::BAR_DQ_FREE), 128);
    mbar_init(bar(T::BAR_ACC_DONE), 2);
    mbar_init(bar(T::BAR_DRAIN), 1);
    mbar_init(bar(T::BAR_DRAIN2), 1);
    mbar_init(bar(T::BAR_SD_USED), 128 * T::NCWG);
    mbar_init(bar(T::BAR_P_FREE), 1);
    mbar_init(bar(T::BAR_DO_FREE), 1);
    mbar_init(bar(T::BAR_DQ_ISSUED), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == T::WARP_A) {
    tmem_alloc(smem_u32(tmem_slot), T::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == T::WARP_TMA && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmDO);
    if (T::SEP_DQ) tma_prefetch_desc(&tmDQ);
    if (EXT && p.bias != nullptr) tma_prefetch_desc(&tmB);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < T::WARP_DQ) {
    // ------------------------------------------------------------------ P / dS warpgroup(s)
    const int wg = warp >> 2;            // which half of the query columns
    const int cb = wg * T::CW;           // first query column of this group
    const int r = (warp & 3) * 32 + lane;  // key row in the block == TMEM lane
    const int key = k0 + r;
    const bool key_ok = key < p.Nk;
    const uint32_t lane_addr = tmem_base + ((uint32_t)((warp & 3) * 32) << 16);
    // Query column c of block i sees this key iff c >= cmin (bottom-right causal alignment).
    const int shift = key - (p.Nk - p.Nq);
    const uint32_t ds_row = sbase + T::OFF_DS + r * 128;
    // EXT: this key's column of the bias (element (q, key) at bias_col[q * Nk]).  A key past Nk reads
    // key 0's column instead (its weights are masked to 0), so the loads need no per-thread guard.
    [[maybe_unused]] const bool has_bias = EXT && p.bias != nullptr;  // uniform over the CTA
    const __nv_bfloat16* bias_col = nullptr;
    if constexpr (EXT) {
      if (has_bias) bias_col = p.bias + (bh / p.H) * p.bias_sb + (bh % p.H) * p.bias_sh + (key_ok ? key : 0);
    }
    // EXT: the bias entries (q, key) of one 16-column chunk of this group as packed bf16 pairs, loaded
    // one chunk ahead of their use (the first chunk before the block's waits) so that their latency
    // stays off the P/dS chain.  A query row past Nq reads row Nq - 1 instead: its LSE is -inf, so its
    // weight is 0 whatever the bias (never +inf, so no NaN).
    auto load_bias = [&](int q0, int ch, uint32_t (&dst)[8]) {
      const int qc = q0 + cb + 16 * ch;
#pragma unroll
      for (int e = 0; e < 16; e += 2) {
        const int qa = min(qc + e, p.Nq - 1), qb = min(qc + e + 1, p.Nq - 1);
        const uint32_t lo = __ldg(reinterpret_cast<const unsigned short*>(bias_col + (size_t)qa * p.Nk));
        const uint32_t hi = __ldg(reinterpret_cast<const unsigned short*>(bias_col + (size_t)qb * p.Nk));
        dst[e / 2] = lo | (hi << 16);
      }
    };
    bool ok = true;
    for (int it = 0; it < n_q; ++it) {
      const int q0 = (i0 + it) * 128;
      [[maybe_unused]] uint32_t braw[2][8];
      if constexpr (EXT) {
        if (has_bias) load_bias(q0, 0, braw[0]);
      }
      // Per-block statistics, stored negated: -LSE in log2 units (-inf past Nq) and -D.  The
      // first barrier keeps the previous block's readers ahead of the overwrite, the second
      // publishes the new values.
      {
        const int q = q0 + r;
        const bool in = q < p.Nq;
        const size_t gi = (size_t)bh * p.Nq + (in ? q : 0);
        float nlse2 = in ? -p.lse[gi] * kLog2e : -INFINITY;
        // EXT: a row the bias hides entirely has LSE = -inf; keep its weights at 0 (a -inf bias
        // entry plus +inf would be NaN).
        if constexpr (EXT) nlse2 = (nlse2 == INFINITY) ? -INFINITY : nlse2;
        const float nd = in ? -p.dvec[gi] : 0.f;
        asm volatile("bar.sync 1, %0;" ::"n"(128 * T::NCWG) : "memory");
        if (wg == 0) {
          stat[r] = nlse2;
          stat[128 + r] = nd;
        }
      }
      // The second barrier is also where the groups agree to go on: a wait that gave up in any of
      // their warps ends the loop for all of them, so none is left at a later named barrier.
      if (!bar_sync_all(1, 128 * T::NCWG, ok)) {
        ok = false;
        break;
      }
      ok = __all_sync(0xffffffffu, mbar_wait(bar(T::BAR_S_FULL), it & 1, abort_flag));
      if (!ok) {
        *abort_flag = 1;  // the other warps' waits give up at once
        continue;         // to the agreement at the next block's barrier
      }
      tc_fence_after();
      const int cmin = p.causal ? shift - q0 : -1;
      // Masking is needed only where this warp holds a key past Nk or a causally hidden entry.
      const bool masked = __any_sync(0xffffffffu, !key_ok || cmin > cb);
      const float4* st4 = reinterpret_cast<const float4*>(stat);
      const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
      [[maybe_unused]] const float2 inv2 = make_float2(kLog2e / p.scale_log2, kLog2e / p.scale_log2);  // 1 / scale
      [[maybe_unused]] const float zscale = p.drop.p8 != 0 ? p.drop.scale : 1.f;
      // 16-column chunks, double-buffered: the load of chunk c+1 is issued right after chunk c
      // has arrived and overlaps its arithmetic (a TMEM load wait covers every load in flight).
      constexpr int NCH = T::CW / 16;  // 16-column chunks of this group
      uint32_t sv[2][16], dpv[2][16];
      tmem_ld32x32b_x16_nowait(lane_addr + T::COL_S + cb, sv[0]);
      tmem_ld32x32b_x16_nowait(lane_addr + T::COL_DP + cb, dpv[0]);
      tmem_wait_ld_2x16(sv[0], dpv[0]);
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch) {
        const int cur = ch & 1;
        if (ch < NCH - 1) {
          tmem_ld32x32b_x16_nowait(lane_addr + T::COL_S + cb + 16 * (ch + 1), sv[cur ^ 1]);
          tmem_ld32x32b_x16_nowait(lane_addr + T::COL_DP + cb + 16 * (ch + 1), dpv[cur ^ 1]);
        }
        uint32_t pk[8], dk[8];
        // EXT: bias and dropout decisions (bit e: column 16 ch + e kept) of this chunk's 16 query
        // columns.  The bias enters the unscaled score, s + bias / scale, so that the exponent's
        // multiply-add by scale * log2(e) covers both.
        [[maybe_unused]] uint32_t keepm = 0xffffu;
        if constexpr (EXT) {
          const int qc = q0 + cb + 16 * ch;
          if (has_bias && ch < NCH - 1) load_bias(q0, ch + 1, braw[cur ^ 1]);
          if (p.drop.p8 != 0) keepm = dropout_keep_colwise(p.drop, (uint32_t)(qc >> 2), (uint32_t)key, (uint32_t)bh, lane);
        }
#pragma unroll
        for (int i = 0; i < 16; i += 4) {
          const int c = cb + 16 * ch + i;
          const float4 nl = st4[c >> 2];  // broadcast: every lane reads the same address
          const float4 nd = st4[32 + (c >> 2)];
          float2 s01 = make_float2(__uint_as_float(sv[cur][i]), __uint_as_float(sv[cur][i + 1]));
          float2 s23 = make_float2(__uint_as_float(sv[cur][i + 2]), __uint_as_float(sv[cur][i + 3]));
          if constexpr (EXT) {
            if (has_bias) {
              const uint32_t b01 = braw[cur][i / 2], b23 = braw[cur][i / 2 + 1];
              s01 = ffma2(make_float2(__uint_as_float(b01 << 16), __uint_as_float(b01 & 0xffff0000u)), inv2, s01);
              s23 = ffma2(make_float2(__uint_as_float(b23 << 16), __uint_as_float(b23 & 0xffff0000u)), inv2, s23);
            }
          }
          const float2 x01 = ffma2(s01, sc2, make_float2(nl.x, nl.y));
          const float2 x23 = ffma2(s23, sc2, make_float2(nl.z, nl.w));
          float2 p01 = make_float2(ex2_approx(x01.x), ex2_approx(x01.y));
          float2 p23 = make_float2(ex2_approx(x23.x), ex2_approx(x23.y));
          if (masked) {
            p01.x = (key_ok && c >= cmin) ? p01.x : 0.f;
            p01.y = (key_ok && c + 1 >= cmin) ? p01.y : 0.f;
            p23.x = (key_ok && c + 2 >= cmin) ? p23.x : 0.f;
            p23.y = (key_ok && c + 3 >= cmin) ? p23.y : 0.f;
          }
          float2 t01, t23;
          [[maybe_unused]] float2 z01, z23;  // EXT: dropout factors (kept: 1 / (1 - p), dropped: 0)
          if constexpr (EXT) {
            z01 = make_float2(((keepm >> i) & 1u) ? zscale : 0.f, ((keepm >> (i + 1)) & 1u) ? zscale : 0.f);
            z23 = make_float2(((keepm >> (i + 2)) & 1u) ? zscale : 0.f, ((keepm >> (i + 3)) & 1u) ? zscale : 0.f);
            t01 = ffma2(make_float2(__uint_as_float(dpv[cur][i]), __uint_as_float(dpv[cur][i + 1])), z01,
                        make_float2(nd.x, nd.y));
            t23 = ffma2(make_float2(__uint_as_float(dpv[cur][i + 2]), __uint_as_float(dpv[cur][i + 3])), z23,
                        make_float2(nd.z, nd.w));
          } else {
            t01 = fadd2(make_float2(__uint_as_float(dpv[cur][i]), __uint_as_float(dpv[cur][i + 1])),
                        make_float2(nd.x, nd.y));
            t23 = fadd2(make_float2(__uint_as_float(dpv[cur][i + 2]), __uint_as_float(dpv[cur][i + 3])),
                        make_float2(nd.z, nd.w));
          }
          const float2 d01 = fmul2(p01, t01), d23 = fmul2(p23, t23);
          if constexpr (EXT) {
            const float2 pz01 = fmul2(p01, z01);
            const float2 pz23 = fmul2(p23, z23);
            pk[i / 2] = pack_bf16x2(pz01.x, pz01.y);
            pk[i / 2 + 1] = pack_bf16x2(pz23.x, pz23.y);
          } else {
            pk[i / 2] = pack_bf16x2(p01.x, p01.y);
            pk[i / 2 + 1] = pack_bf16x2(p23.x, p23.y);
          }
          dk[i / 2] = pack_bf16x2(d01.x, d01.y);
          dk[i / 2 + 1] = pack_bf16x2(d23.x, d23.y);
        }
        if (ch == 0 && it > 0) {
          // d = 64: P^T(it-1) must have been read by dV(it-1).  Both: dS^T(it-1) must have been
          // read by dQ(it-1) and dK(it-1) before it is overwritten.
          if (T::EARLY) ok = __all_sync(0xffffffffu, mbar_wait(bar(T::BAR_P_FREE), (it - 1) & 1, abort_flag));
          if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(T::BAR_DS_FREE), (it - 1) & 1, abort_flag));
          tc_fence_after();
        }
        // P^T chunk -> TMEM (bf16 pairs).  d = 128: over the consumed first half of S^T (S_FULL
        // also covers issuer A's dV(it-1)); d = 64: into its own columns.
        tmem_st32x32b_x8(lane_addr + T::COL_P + wg * T::P_WG_STRIDE + 8 * ch, pk);
        // dS^T chunk (16 query columns = two 16-byte chunks) -> shared memory, K-major with
        // 128-byte swizzle (box = 64 query columns).
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          const int kc = cb / 8 + 2 * ch + m;  // 16-byte chunk index along the 128 query columns
          const uint32_t addr = ds_row + (kc >> 3) * T::BOX_BYTES + (((kc & 7) ^ (r & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(dk[4 * m]), "r"(dk[4 * m + 1]),
                       "r"(dk[4 * m + 2]), "r"(dk[4 * m + 3])
                       : "memory");
        }
        if (ch < NCH - 1) {
          tmem_wait_ld_2x16(sv[cur ^ 1], dpv[cur ^ 1]);
          if (T::EARLY && ch == NCH - 2) {
            // Both blocks of this iteration are now in registers: the issuers may overwrite them.
            tc_fence_before();
            mbar_arrive(bar(T::BAR_SD_USED));
          }
        }
      }
      tmem_st_wait();  // also on the give-up path: no TMEM store is left in flight at teardown
      if (!ok) {
        *abort_flag = 1;
        continue;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(T::BAR_DS_READY));
    }
    // dK, dV epilogue (group 0 owns it; both groups hold the same key rows).
    if (ok && wg == 0 && n_q > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar(T::BAR_ACC_DONE), 0, abort_flag));
    if (!ok) {
      *abort_flag = 1;
    } else if (wg == 0) {
      tc_fence_after();
      const size_t off = ((size_t)bh * p.Nk + (key_ok ? key : 0)) * D;
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        __nv_bfloat16* out = (which ? p.dk : p.dv) + off;
        const float mul = which ? p.scale : 1.f;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          if (n_q > 0) {
            tmem_ld32x32b_x32_wait(lane_addr + (which ? T::COL_DK : T::COL_DV) + 32 * c, v);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0u;
          }
          if (key_ok) {
            uint4* dst = reinterpret_cast<uint4*>(out + 32 * c);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * i]) * mul, __uint_as_float(v[8 * i + 1]) * mul),
                                  pack_bf16x2(__uint_as_float(v[8 * i + 2]) * mul, __uint_as_float(v[8 * i + 3]) * mul),
                                  pack_bf16x2(__uint_as_float(v[8 * i + 4]) * mul, __uint_as_float(v[8 * i + 5]) * mul),
                                  pack_bf16x2(__uint_as_float(v[8 * i + 6]) * mul, __uint_as_float(v[8 * i + 7]) * mul));
          }
        }
      }
    }
  } else if (warp < T::WARP_DQ + 4) {
    // ------------------------------------------------------------------ dQ warpgroup
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // query row of the dQ block == TMEM lane
    const uint32_t lane_addr = tmem_base + ((uint32_t)(quarter * 32) << 16);
    const bool leader = (warp == T::WARP_DQ && lane == 0);
    const uint32_t stg_row = sbase + T::OFF_STG + r * 128;
    bool ok = true;
    // A warp whose wait gave up skips the data steps but still takes the first named barrier of
    // the block, where the group decides whether to go on (so that no warp is left at a barrier
    // the others never reach).
    for (int it = 0; it < (DQ ? n_q : 0); ++it) {
      const int q0 = (i0 + it) * 128;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(T::BAR_DQ_FULL), it & 1, abort_flag));
      if constexpr (T::SEP_DQ) {
        uint32_t v[D];
        if (ok) {
          tc_fence_after();
          tmem_ld32x32b_x64_nowait(lane_addr + T::COL_DQ, v);
          tmem_wait_ld_x64(v);
          // The dQ columns are free as soon as they are in registers.
          tc_fence_before();
          mbar_arrive(bar(T::BAR_DQ_FREE));
        }
        // Stage the scaled block as two 32-column fp32 boxes in the 128-byte-swizzle layout (row r
        // at r*128 bytes of each box, 16-byte chunk c at (c ^ r%8)*16: a quarter-warp hits
        // distinct banks), then bulk reduce-add both boxes.
        if (leader && it > 0) bulk_wait_group_read0();  // previous tile read out of the staging buffer
        if (!bar_sync_all(2, 128, ok)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const uint32_t addr = stg_row + (c >> 3) * (128 * 128) + (((c & 7) ^ (r & 7)) << 4);
          asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                       "f"(__uint_as_float(v[4 * c]) * p.scale), "f"(__uint_as_float(v[4 * c + 1]) * p.scale),
                       "f"(__uint_as_float(v[4 * c + 2]) * p.scale), "f"(__uint_as_float(v[4 * c + 3]) * p.scale)
                       : "memory");
        }
        fence_proxy_async_smem();
        asm volatile("bar.sync 2, 128;" ::: "memory");
        if (leader) {
          // Rows past Nq fall outside the tensor map and are not written.
          tma_reduce_add_3d(&tmDQ, sbase + T::OFF_STG, 0, q0, bh);
          tma_reduce_add_3d(&tmDQ, sbase + T::OFF_STG + 128 * 128, 32, q0, bh);
          bulk_commit_group();
        }
      } else {
        // d = 128: no shared memory is left for a separate staging buffer.  The dO tile of this
        // block's stage is free once dV(it) has read it; it takes the scaled dQ block in two
        // 64-column halves (two 32-column fp32 boxes each), bulk reduce-added one after the other.
        // The 128 TMEM columns are read as four 32-column chunks, two loads in flight, and are
        // released once the last chunk is in registers.
        const int s = it % T::NS;
        const uint32_t stg = sbase + T::OFF_QD + s * 2 * T::TILE_BYTES + T::TILE_BYTES;
        auto stage = [&](const uint32_t (&v)[32], int box) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint32_t addr = stg + box * (128 * 128) + r * 128 + ((c ^ (r & 7)) << 4);
            asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                         "f"(__uint_as_float(v[4 * c]) * p.scale), "f"(__uint_as_float(v[4 * c + 1]) * p.scale),
                         "f"(__uint_as_float(v[4 * c + 2]) * p.scale), "f"(__uint_as_float(v[4 * c + 3]) * p.scale)
                         : "memory");
          }
        };
        auto reduce_half = [&](int h) {  // after the barrier that follows the half's staging
          if (leader) {
            // Rows past Nq fall outside the tensor map and are not written.
            tma_reduce_add_3d(&tmDQ, stg, 64 * h, q0, bh);
            tma_reduce_add_3d(&tmDQ, stg + 128 * 128, 64 * h + 32, q0, bh);
            bulk_commit_group();
            bulk_wait_group_read0();  // the staging buffer is read out
          }
          asm volatile("bar.sync 2, 128;" ::: "memory");
        };
        uint32_t va[32], vb[32];
        if (ok) {
          tc_fence_after();
          tmem_ld32x32b_x32_nowait(lane_addr + T::COL_DQ, va);
          tmem_ld32x32b_x32_nowait(lane_addr + T::COL_DQ + 32, vb);
          tmem_wait_ld_2x32(va, vb);
          ok = __all_sync(0xffffffffu, mbar_wait(bar(T::BAR_DO_FREE), it & 1, abort_flag));
        }
        if (ok) {
          stage(va, 0);
          stage(vb, 1);
          tmem_ld32x32b_x32_nowait(lane_addr + T::COL_DQ + 64, va);
          tmem_ld32x32b_x32_nowait(lane_addr + T::COL_DQ + 96, vb);
          tmem_wait_ld_2x32(va, vb);
          tc_fence_before();
          mbar_arrive(bar(T::BAR_DQ_FREE));
          fence_proxy_async_smem();
        }
        if (!bar_sync_all(2, 128, ok)) {
          ok = false;
          break;
        }
        reduce_half(0);
        stage(va, 0);
        stage(vb, 1);
        fence_proxy_async_smem();
        asm volatile("bar.sync 2, 128;" ::: "memory");
        reduce_half(1);
        if (leader && it + T::NS < n_q) mbar_arrive(bar(T::BAR_QD_EMPTY + s));
      }
    }
    if (!ok) *abort_flag = 1;
    if (leader) bulk_wait_group0();  // every reduce-add complete before the CTA exits
  } else if (warp == T::WARP_A || warp == T::WARP_B) {
    // ------------------------------------------------------------------ MMA issuers A and B
    // Each issuer is a whole converged warp (one elected lane issues), and each runs its own
    // specialised loop: no per-MMA branch on the issuer's role.
    auto issuer = [&](auto role) {
      constexpr bool is_a = decltype(role)::value;
      const uint32_t k_smem = sbase + T::OFF_K, v_smem = sbase + T::OFF_V, ds_smem = sbase + T::OFF_DS;
      const uint32_t tS = tmem_base + T::COL_S, tDP = tmem_base + T::COL_DP;
      [[maybe_unused]] const uint32_t tDQ = tmem_base + T::COL_DQ;
      const uint32_t tDV = tmem_base + T::COL_DV, tDK = tmem_base + T::COL_DK;
      auto q_smem = [&](int it) { return sbase + T::OFF_QD + (it % T::NS) * 2 * T::TILE_BYTES; };
      auto wait_qd = [&](int it) { return warp_wait(bar(T::BAR_QD_FULL + it % T::NS), (it / T::NS) & 1, abort_flag); };
      // The first operand block of this issuer's recomputed product: S^T = K Q^T (A) or dP^T = V dO^T (B).
      auto issue_first = [&](int it) {
        if constexpr (is_a) bwd_issue_ss_kmajor<D>(tS, k_smem, q_smem(it));
        else bwd_issue_ss_kmajor<D>(tDP, v_smem, q_smem(it) + T::TILE_BYTES);
        mma_commit_w(bar(T::BAR_S_FULL));
      };
      const uint64_t ds_kmaj = make_sdesc_sw128(ds_smem, 16, 1024);           // dS^T as A, K-major
      const uint64_t ds_mn = make_sdesc_sw128(ds_smem, T::BOX_BYTES, 1024);    // dS as A, MN-major
      const uint64_t k_mn = make_sdesc_sw128(k_smem, T::BOX_BYTES, 1024);      // K as B, MN-major
      bool ok = warp_wait(bar(T::BAR_KV), 0, abort_flag) && wait_qd(0);
      if (ok) {
        tc_fence_after();
        issue_first(0);
      }
      for (int it = 0; ok && it < n_q; ++it) {
        const uint32_t qs = q_smem(it), dos = qs + T::TILE_BYTES;
        const bool more = it + 1 < n_q;
        if (T::EARLY && more) {
          // d = 64: the next block's S^T / dP^T as soon as this block's are in registers.
          if (!(ok = warp_wait(bar(T::BAR_SD_USED), it & 1, abort_flag))) break;
          if (!(ok = wait_qd(it + 1))) break;
          tc_fence_after();
          issue_first(it + 1);
        }
        if (!(ok = warp_wait(bar(T::BAR_DS_READY), it & 1, abort_flag))) break;
        tc_fence_after();
        if constexpr (is_a) {
          // dQ(i) goes to the tensor pipe first: its read-out gates the next block's dP^T, while dV(i)
          // only has to precede the next S^T, which this issuer sends after it anyway.
          if (DQ && !(ok = warp_wait(bar(T::BAR_DQ_ISSUED), it & 1, abort_flag))) break;
          // dV_j += P^T dO_i  (P^T from TMEM, dO MN-major).
          const uint64_t do_mn = make_sdesc_sw128(dos, T::BOX_BYTES, 1024);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts_w(tDV, tmem_base + T::p_col(kk), do_mn + (uint64_t)((kk * 2048) >> 4), T::IDESC_DVK,
                     (it > 0 || kk > 0) ? 1u : 0u);
          if (T::EARLY) mma_commit_w(bar(T::BAR_P_FREE));
          if constexpr (T::SEP_DQ || !DQ) {
            if (it + T::NS < n_q) mma_commit_w(bar(T::BAR_QD_EMPTY + it % T::NS));
          } else {
            // d = 128: dO(it) becomes the dQ staging buffer; the dQ warpgroup frees the stage.
            mma_commit_w(bar(T::BAR_DO_FREE));
          }
          if (!T::EARLY && more) {
            // d = 128: the next S^T overwrites P^T(it) only after dV(it) (same thread, in order).
            if (!(ok = wait_qd(it + 1))) break;
            tc_fence_after();
            issue_first(it + 1);
          }
        } else {
          if constexpr (DQ) {
            // dQ_i = dS K_j (A = dS, the MN-major view of dS^T), once the dQ columns are free.
            if (T::SEP_DQ && it > 0 && !(ok = warp_wait(bar(T::BAR_DQ_FREE), (it - 1) & 1, abort_flag))) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ss_w(tDQ, ds_mn + (uint64_t)((kk * 2048) >> 4), k_mn + (uint64_t)((kk * 2048) >> 4), T::IDESC_DQ,
                       kk > 0 ? 1u : 0u);
            mma_commit_w(bar(T::BAR_DQ_FULL));
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(T::BAR_DQ_ISSUED));
          }
          // d = 128: the next block's dP^T reuses the dQ columns, once dQ(it) is read out.
          if (!T::EARLY && more) {
            if (!(ok = wait_qd(it + 1))) break;
            if (DQ && !(ok = warp_wait(bar(T::BAR_DQ_FREE), it & 1, abort_flag))) break;
            tc_fence_after();
            issue_first(it + 1);
          }
          // dK_j += dS^T Q_i  (dS^T K-major, Q MN-major); scale is applied in the epilogue.
          const uint64_t q_mn = make_sdesc_sw128(qs, T::BOX_BYTES, 1024);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss_w(tDK, ds_kmaj + (uint64_t)(((kk / 4) * T::BOX_BYTES + (kk % 4) * 32) >> 4),
                     q_mn + (uint64_t)((kk * 2048) >> 4), T::IDESC_DVK, (it > 0 || kk > 0) ? 1u : 0u);
          mma_commit_w(bar(T::BAR_DS_FREE));
          if (it + T::NS < n_q) mma_commit_w(bar(T::BAR_QD_EMPTY + it % T::NS));
        }
      }
      if (ok) mma_commit_w(bar(T::BAR_ACC_DONE));
      if (!ok) {
        *abort_flag = 1;
        const int drain = is_a ? T::BAR_DRAIN : T::BAR_DRAIN2;
        mma_commit_w(bar(drain));
        warp_drain_wait(bar(drain), 0);
      }
    };
    if (n_q > 0) {
      if (warp == T::WARP_A) issuer(std::true_type{});
      else issuer(std::false_type{});
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && n_q > 0) {
      mbar_arrive_expect_tx(bar(T::BAR_KV), 2 * T::TILE_BYTES);
      for (int b = 0; b < T::NBOX; ++b) {
        tma_load_3d(sbase + T::OFF_K + b * T::BOX_BYTES, &tmK, bar(T::BAR_KV), 64 * b, k0, bh);
        tma_load_3d(sbase + T::OFF_V + b * T::BOX_BYTES, &tmV, bar(T::BAR_KV), 64 * b, k0, bh);
      }
      bool ok = true;
      int issued = 0;
      for (int it = 0; it < n_q; ++it) {
        const int s = it % T::NS;
        if (!(ok = mbar_wait(bar(T::BAR_QD_EMPTY + s), ((it / T::NS) & 1) ^ 1, abort_flag))) break;
        mbar_arrive_expect_tx(bar(T::BAR_QD_FULL + s), 2 * T::TILE_BYTES);
        const uint32_t dst = sbase + T::OFF_QD + s * 2 * T::TILE_BYTES;
        const int q0 = (i0 + it) * 128;
        for (int b = 0; b < T::NBOX; ++b) {
          tma_load_3d(dst + b * T::BOX_BYTES, &tmQ, bar(T::BAR_QD_FULL + s), 64 * b, q0, bh);
          tma_load_3d(dst + T::TILE_BYTES + b * T::BOX_BYTES, &tmDO, bar(T::BAR_QD_FULL + s), 64 * b, q0, bh);
        }
        issued = it + 1;
        if constexpr (EXT) {
          // Warm the L2 with this block's bias tile (the P/dS threads read its key columns with plain
          // loads once the block's stage is consumed).
          if (p.bias != nullptr) {
            const int plane = (bh / p.H) * p.bias_pb + (bh % p.H) * p.bias_ph;
            for (int b = 0; b < 2; ++b) tma_prefetch_l2_3d(&tmB, k0 + 64 * b, q0, plane);
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        for (int it = max(0, issued - T::NS); it < issued; ++it)
          drain_wait(bar(T::BAR_QD_FULL + it % T::NS), (it / T::NS) & 1);
        drain_wait(bar(T::BAR_KV), 0);
      }
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == T::WARP_A) {
    tc_fence_after();
    tmem_dealloc(tmem_base, T::TMEM_COLS);
  }
}

}  // namespace fa
