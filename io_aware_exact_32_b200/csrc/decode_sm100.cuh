// Split-KV decode for sm_100a (one query per (batch, head), ragged KV-cache lengths).
//
// Method ("Transformer、注意力机制与优化", section Flash-Decoding): attention is associative, so
// the keys/values of one sequence are cut into chunks, each chunk is attended to in parallel,
// and the partial results are reduced.  Each chunk produces (m, l, O~) with
// O~ = sum_k exp(s_k - m) v_k; the reduction is the two-block identity for m and l of the same
// page (section 安全 Softmax 与在线 Softmax) applied to all chunks at once.
//
// The pass is bound by HBM bandwidth (each K/V byte is used for one multiply-add), so it runs on
// the CUDA cores: a producer warp streams 16-key K and V blocks into a shared-memory ring with
// plain bulk copies (exactly the visible rows, nothing past seqlens[b] is read); four consumer
// warps each take every fourth block, two lanes per key for q.k and one lane per 4 (or 2) output
// dims for P V, each warp with its own running (m, l, acc); the four are merged in shared memory.
// Block i lives in ring stage i % NS with NS a multiple of the consumer-warp count, so every
// stage belongs to one warp and is consumed in order (each wait is at most one phase ahead).
#pragma once

#include "sm100_ptx.cuh"

namespace fa {

template <int D>
struct DecTraits {
  static_assert(D == 64 || D == 128, "head dim");
  static constexpr int KB = 16;  // keys per block
  static constexpr int ROW_BYTES = D * 2;
  static constexpr int BLK_BYTES = KB * ROW_BYTES;  // 4 KB at D = 128
  static constexpr int NCW = 4;                     // consumer warps
  static constexpr int NS = 2 * NCW;                // ring stages (each holds a K and a V block)
  static_assert(NS % NCW == 0, "each stage must belong to one consumer warp");
  static constexpr int THREADS = 32 * (NCW + 1);
  static constexpr int NCHUNK = D / 8;  // 16-byte chunks per row
  static constexpr int PER = D / 32;    // output dims per lane
  static constexpr int OFF_STAGE = 0;
  static constexpr int OFF_Q = NS * 2 * BLK_BYTES;
  static constexpr int Q_BYTES = NCHUNK * 48;  // 8 fp32 per chunk + 16 bytes of padding
  static constexpr int OFF_MERGE = OFF_Q + Q_BYTES;
  static constexpr int MERGE_STRIDE = D + 4;  // floats per warp: acc[D], m, l, pad
  static constexpr int OFF_BAR = OFF_MERGE + NCW * MERGE_STRIDE * 4;
  static constexpr int SMEM_BYTES = OFF_BAR + 2 * NS * 8 + 16 + 128;
};

struct DecParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* kc;
  const __nv_bfloat16* vc;
  const int* seqlens;
  float* part_o;   // [BH * S, D]
  float* part_ml;  // [BH * S, 2]  (m in log2 units, l)
  int Lmax, H, S, C;
  float scale_log2;
};

template <int D>
__global__ void __launch_bounds__(DecTraits<D>::THREADS) fa_decode_split_kernel(const DecParams p) {
  using T = DecTraits<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const uint32_t sbase = smem_u32(smem);
  auto full = [&](int s) -> uint32_t { return sbase + T::OFF_BAR + 8 * s; };
  auto empty = [&](int s) -> uint32_t { return sbase + T::OFF_BAR + 8 * (T::NS + s); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + T::OFF_BAR + 16 * T::NS);

  const int unit = blockIdx.x;
  const int s_idx = unit % p.S;
  const int bh = unit / p.S;
  const int b = bh / p.H;
  const int L = min(max(p.seqlens[b], 0), p.Lmax);
  const int k_begin = s_idx * p.C;
  const int nkeys = max(0, min(k_begin + p.C, L) - k_begin);
  const int nblk = (nkeys + T::KB - 1) / T::KB;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (nblk == 0) {
    for (int i = threadIdx.x; i < D; i += blockDim.x) p.part_o[(size_t)unit * D + i] = 0.f;
    if (threadIdx.x == 0) {
      p.part_ml[2 * (size_t)unit] = -INFINITY;
      p.part_ml[2 * (size_t)unit + 1] = 0.f;
    }
    return;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < T::NS; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  // q, pre-multiplied by scale*log2(e), as fp32 in padded 32-byte chunks (conflict-free reads).
  float* qs = reinterpret_cast<float*>(smem + T::OFF_Q);
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    const float qv = __bfloat162float(p.q[(size_t)bh * D + i]);
    qs[(i >> 3) * 12 + (i & 7)] = qv * p.scale_log2;
  }
  __syncthreads();

  const size_t row0 = (size_t)bh * p.Lmax + k_begin;
  if (warp == T::NCW) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      bool ok = true;
      int issued = 0;
      for (int i = 0; i < nblk; ++i) {
        const int s = i % T::NS;
        if (!(ok = mbar_wait(empty(s), ((i / T::NS) & 1) ^ 1, abort_flag))) break;
        const int nk = min(T::KB, nkeys - i * T::KB);
        const uint32_t bytes = (uint32_t)nk * T::ROW_BYTES;
        mbar_arrive_expect_tx(full(s), 2 * bytes);
        const size_t off = (row0 + (size_t)i * T::KB) * D;
        bulk_load(sbase + T::OFF_STAGE + s * 2 * T::BLK_BYTES, p.kc + off, bytes, full(s));
        bulk_load(sbase + T::OFF_STAGE + s * 2 * T::BLK_BYTES + T::BLK_BYTES, p.vc + off, bytes, full(s));
        issued = i + 1;
      }
      if (!ok) {
        *abort_flag = 1;
        for (int i = max(0, issued - T::NS); i < issued; ++i) drain_wait(full(i % T::NS), (i / T::NS) & 1);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ consumers
    float m = -INFINITY, l = 0.f;
    float acc[T::PER];
#pragma unroll
    for (int i = 0; i < T::PER; ++i) acc[i] = 0.f;
    bool ok = true;
    for (int i = warp; i < nblk; i += T::NCW) {
      const int s = i % T::NS;
      ok = __all_sync(0xffffffffu, mbar_wait(full(s), (i / T::NS) & 1, abort_flag));
      if (!ok) break;
      const int nk = min(T::KB, nkeys - i * T::KB);
      const uint8_t* kblk = smem + T::OFF_STAGE + s * 2 * T::BLK_BYTES;
      const uint8_t* vblk = kblk + T::BLK_BYTES;
      // Score of key (lane & 15) in log2 units: lanes l and l + 16 each take half of the row;
      // chunks are visited in a key-rotated order so a quarter-warp hits distinct banks.
      const int key = lane & 15;
      const int half = lane >> 4;
      float dot = 0.f;
      if (key < nk) {
        const uint8_t* krow = kblk + key * T::ROW_BYTES;
#pragma unroll
        for (int c = 0; c < T::NCHUNK / 2; ++c) {
          const int ch = ((c + key) & (T::NCHUNK / 2 - 1)) + half * (T::NCHUNK / 2);
          const uint4 kv = *reinterpret_cast<const uint4*>(krow + ch * 16);
          const float4 qa = *reinterpret_cast<const float4*>(qs + ch * 12);
          const float4 qb = *reinterpret_cast<const float4*>(qs + ch * 12 + 4);
          dot = fmaf(bf16lo_to_f32(kv.x), qa.x, dot);
          dot = fmaf(bf16hi_to_f32(kv.x), qa.y, dot);
          dot = fmaf(bf16lo_to_f32(kv.y), qa.z, dot);
          dot = fmaf(bf16hi_to_f32(kv.y), qa.w, dot);
          dot = fmaf(bf16lo_to_f32(kv.z), qb.x, dot);
          dot = fmaf(bf16hi_to_f32(kv.z), qb.y, dot);
          dot = fmaf(bf16lo_to_f32(kv.w), qb.z, dot);
          dot = fmaf(bf16hi_to_f32(kv.w), qb.w, dot);
        }
      }
      dot += __shfl_xor_sync(0xffffffffu, dot, 16);
      const float sc = (key < nk) ? dot : -INFINITY;  // lanes l and l + 16 hold the same score
      float mb = sc;
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, off));
      const float m_new = fmaxf(m, mb);  // finite: the block has at least one key
      const float alpha = ex2_approx(m - m_new);
      const float pl = (key < nk) ? ex2_approx(sc - m_new) : 0.f;
      float ps = pl;
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l = l * alpha + ps;
#pragma unroll
      for (int e = 0; e < T::PER; ++e) acc[e] *= alpha;
      m = m_new;
      for (int k = 0; k < nk; ++k) {
        const float pk = __shfl_sync(0xffffffffu, pl, k);
        const uint8_t* vrow = vblk + k * T::ROW_BYTES + lane * T::PER * 2;
        if constexpr (T::PER == 4) {
          const uint2 vv = *reinterpret_cast<const uint2*>(vrow);
          acc[0] = fmaf(pk, bf16lo_to_f32(vv.x), acc[0]);
          acc[1] = fmaf(pk, bf16hi_to_f32(vv.x), acc[1]);
          acc[2] = fmaf(pk, bf16lo_to_f32(vv.y), acc[2]);
          acc[3] = fmaf(pk, bf16hi_to_f32(vv.y), acc[3]);
        } else {
          const uint32_t vv = *reinterpret_cast<const uint32_t*>(vrow);
          acc[0] = fmaf(pk, bf16lo_to_f32(vv), acc[0]);
          acc[1] = fmaf(pk, bf16hi_to_f32(vv), acc[1]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty(s));
    }
    if (!ok) *abort_flag = 1;
    float* mg = reinterpret_cast<float*>(smem + T::OFF_MERGE) + warp * T::MERGE_STRIDE;
#pragma unroll
    for (int e = 0; e < T::PER; ++e) mg[lane * T::PER + e] = acc[e];
    if (lane == 0) {
      mg[D] = m;
      mg[D + 1] = l;
    }
  }
  __syncthreads();
  // Merge the consumer warps' (m, l, acc) with the two-block identity.
  const float* mg = reinterpret_cast<const float*>(smem + T::OFF_MERGE);
  float mt = -INFINITY;
#pragma unroll
  for (int w = 0; w < T::NCW; ++w) mt = fmaxf(mt, mg[w * T::MERGE_STRIDE + D]);
  const float base = (mt == -INFINITY) ? 0.f : mt;
  for (int i = threadIdx.x; i < D + 1; i += blockDim.x) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < T::NCW; ++w) {
      const float mw = mg[w * T::MERGE_STRIDE + D];
      const float wgt = (mw == -INFINITY) ? 0.f : ex2_approx(mw - base);
      v += wgt * mg[w * T::MERGE_STRIDE + (i < D ? i : D + 1)];
    }
    if (i < D) {
      p.part_o[(size_t)unit * D + i] = v;
    } else {
      p.part_ml[2 * (size_t)unit] = mt;
      p.part_ml[2 * (size_t)unit + 1] = v;
    }
  }
}

// Reduce the S partials of each (batch, head): one warp per (batch, head).
template <int D>
// Partials come in R groups (R = 1 for one device; R ranks after an all-gather of per-rank
// partials in sequence-parallel decode): partial s of group r for (b, h) sits at row
// (r * BH + bh) * S + s.
__global__ void __launch_bounds__(128) fa_decode_merge_kernel(const float* __restrict__ part_o,
                                                              const float* __restrict__ part_ml,
                                                              __nv_bfloat16* __restrict__ o, float* __restrict__ lse,
                                                              int BH, int S, int R = 1) {
  constexpr int PER = D / 32;
  const int bh = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (bh >= BH) return;
  auto row = [&](int i) { return ((size_t)(i / S) * BH + bh) * S + i % S; };  // i = r * S + s
  const int n = R * S;
  float mt = -INFINITY;
  for (int i = lane; i < n; i += 32) mt = fmaxf(mt, part_ml[2 * row(i)]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
  const float base = (mt == -INFINITY) ? 0.f : mt;
  float l = 0.f, acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  for (int i = 0; i < n; ++i) {
    const size_t ri = row(i);
    const float ms = part_ml[2 * ri];
    if (ms == -INFINITY) continue;
    const float w = ex2_approx(ms - base);
    l += w * part_ml[2 * ri + 1];
    const float* po = part_o + ri * D + lane * PER;
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = fmaf(w, po[e], acc[e]);
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  __nv_bfloat16* orow = o + (size_t)bh * D + lane * PER;
#pragma unroll
  for (int e = 0; e < PER; ++e) orow[e] = __float2bfloat16(acc[e] * inv);
  if (lse != nullptr && lane == 0) lse[bh] = l > 0.f ? (mt + log2f(l)) * 0.6931471805599453f : -INFINITY;
}

}  // namespace fa
