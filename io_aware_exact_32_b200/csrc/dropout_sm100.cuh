// Additive bias and dropout for the attention kernels: the counter-based random numbers and
// the lane exchanges that hand them out.
//
// "优化的注意力实现 (FlashAttention)", section 优势与集成: the scores get an additive bias
// (-inf where masked) before the row softmax, and dropout is applied to the softmax weights
// before they multiply V; "FlashAttention 的基本原理", section 2.4 反向传播: the backward of
// the paper's algorithm covers masking and dropout too.
//
// Dropout decisions are regenerated, not stored: Philox4x32-10 (Salmon, Moraes, Dror, Shaw,
// "Parallel random numbers: as easy as 1, 2, 3", SC 2011) keyed by the 64-bit seed.  One call
// covers 4 queries x 4 keys of one (batch, head): counter = (key / 4, query / 4, b * H + h,
// offset); byte (key % 4) of word (query % 4) is the entry's random byte u, and the entry is
// kept iff u >= p8 (p8 = floor(256 p + 1/2)).  Kept weights are scaled by 256 / (256 - p8).
//
// Lane layout: in the forward a thread owns a query row (4 consecutive lanes = one query quad);
// in the backward a thread owns a key row (4 consecutive lanes = one key quad).  Each lane of a
// quad computes one call in four and the lanes exchange words with shuffles.
#pragma once

#include "sm100_ptx.cuh"

namespace fa {

struct DropoutCfg {
  uint32_t p8;       // keep iff random byte >= p8 (0: no dropout)
  float scale;       // 256 / (256 - p8)
  uint32_t seed_lo, seed_hi, offset;
};

// Philox4x32-10: four 32-bit outputs for counter (c0, c1, c2, c3) and key (k0, k1).
__device__ __forceinline__ uint4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, uint32_t k0,
                                               uint32_t k1) {
  constexpr uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u, W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t hi0 = __umulhi(M0, c0), lo0 = M0 * c0;
    const uint32_t hi1 = __umulhi(M1, c2), lo1 = M1 * c2;
    c0 = hi1 ^ c1 ^ k0;
    c1 = lo1;
    c2 = hi0 ^ c3 ^ k1;
    c3 = lo0;
    k0 += W0;
    k1 += W1;
  }
  return make_uint4(c0, c1, c2, c3);
}

__device__ __forceinline__ uint32_t u4_at(const uint4& w, int i) {
  return i == 0 ? w.x : (i == 1 ? w.y : (i == 2 ? w.z : w.w));
}

// w'[i] = w[i ^ s] for a lane-dependent s in [0, 4): two conditional swap stages.
__device__ __forceinline__ uint4 xor_permute(uint4 w, int s) {
  if (s & 1) w = make_uint4(w.y, w.x, w.w, w.z);
  if (s & 2) w = make_uint4(w.z, w.w, w.x, w.y);
  return w;
}

// Forward: the keep words of query row `row` (lane = row % 4 within its quad) for the 8 key quads
// [J0, J0 + 8): out[t] holds the random bytes of keys 4 (J0 + t) + 0..3 (byte i = key 4 (J0 + t) + i),
// already compared: 0xff where kept, 0x00 where dropped.  All 32 lanes must call it together.
__device__ __forceinline__ void dropout_keep_rowwise(const DropoutCfg& dc, uint32_t J0, uint32_t row, uint32_t bh,
                                                     int lane, uint32_t (&out)[8]) {
  const int m = lane & 3;
  const uint32_t thr = dc.p8 * 0x01010101u;
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    // This lane's call: key quad J0 + 4u + m, query quad row / 4.
    uint4 w = philox4x32_10(J0 + 4 * u + m, row >> 2, bh, dc.offset, dc.seed_lo, dc.seed_hi);
    // Lane m needs word m of each of the four calls of its quad: a 4 x 4 transpose over the lanes.
    // Round r: read from lane m ^ r, which sends its word (m ^ r) ^ r = m.
    const uint4 sendw = xor_permute(w, m);  // sendw[r] = w[m ^ r]
    uint4 recv;
    recv.x = sendw.x;                                     // r = 0: own call, quad J0 + 4u + m
    recv.y = __shfl_xor_sync(0xffffffffu, sendw.y, 1);    // r = 1: quad J0 + 4u + (m ^ 1)
    recv.z = __shfl_xor_sync(0xffffffffu, sendw.z, 2);    // r = 2
    recv.w = __shfl_xor_sync(0xffffffffu, sendw.w, 3);    // r = 3
    // recv[r] belongs to quad slot m ^ r; reorder so that slot t sits at index t.
    const uint4 bys = xor_permute(recv, m);
    out[4 * u + 0] = __vcmpgeu4(bys.x, thr);
    out[4 * u + 1] = __vcmpgeu4(bys.y, thr);
    out[4 * u + 2] = __vcmpgeu4(bys.z, thr);
    out[4 * u + 3] = __vcmpgeu4(bys.w, thr);
  }
}

// Backward: the keep decisions of key row `key` (lane = key % 4 within its quad) for the 16 query
// rows [4 I0, 4 I0 + 16), as a mask: bit 4 u + m is set if (query 4 (I0 + u) + m, key) is kept.
// All 32 lanes must call it together.
__device__ __forceinline__ uint32_t dropout_keep_colwise(const DropoutCfg& dc, uint32_t I0, uint32_t key, uint32_t bh,
                                                         int lane) {
  const int t = lane & 3;
  const uint4 w = philox4x32_10(key >> 2, I0 + t, bh, dc.offset, dc.seed_lo, dc.seed_hi);
  const uint32_t thr = dc.p8 * 0x01010101u;
  const int sh = 8 * t;
  uint32_t mask = 0u;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int owner = (lane & ~3) | u;  // the lane that computed query quad I0 + u
    const uint32_t w0 = __shfl_sync(0xffffffffu, w.x, owner);
    const uint32_t w1 = __shfl_sync(0xffffffffu, w.y, owner);
    const uint32_t w2 = __shfl_sync(0xffffffffu, w.z, owner);
    const uint32_t w3 = __shfl_sync(0xffffffffu, w.w, owner);
    // Byte t of each word -> one word of four bytes (query m in byte m), then compare: byte m of k
    // is 0xff where kept; its top bit (bit 8 m + 7) goes to bit 4 u + m of the mask.
    const uint32_t packed = ((w0 >> sh) & 0xffu) | (((w1 >> sh) & 0xffu) << 8) | (((w2 >> sh) & 0xffu) << 16) |
                            (((w3 >> sh) & 0xffu) << 24);
    const uint32_t k = __vcmpgeu4(packed, thr);
    const uint32_t m4 = ((k >> 7) & 1u) | ((k >> 14) & 2u) | ((k >> 21) & 4u) | ((k >> 28) & 8u);
    mask |= m4 << (4 * u);
  }
  return mask;
}

}  // namespace fa
