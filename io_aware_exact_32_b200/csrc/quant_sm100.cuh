// Incoherent processing and FP8 quantisation of one attention operand.
//
// "FlashAttention 系列技术详解", section 具体技术 (FlashAttention-3): the GEMMs can run on FP8
// tensor cores; to limit the quantisation error, Q and K are first multiplied by a random
// orthogonal matrix -- a Hadamard transform, O(d log d) per row -- which spreads outlier
// channels over all coordinates.  Q M (K M)^T = Q K^T, so the scores are unchanged.
//
// Here M = diag(s) H_d / sqrt(d) (s: random signs supplied by the caller, H_d the Sylvester
// Hadamard matrix); V is quantised without rotation.  Each (batch, head) gets one scale:
// x8 = rn_e4m3(y * 448 / amax), descale = (amax / 448) / sqrt(d) (no 1 / sqrt(d) without rotation),
// so that x M ~= x8 * descale.
//
// B200 layout: 32 consecutive elements per lane (four 16-byte loads), d / 32 lanes per row.  The
// butterflies of the transform run in stages h = 1, 2, 4, ...: inside a lane while h < 32, then
// across lanes with shuffles; every butterfly maps (a, b) at indices (i, i + h) to (a + b, a - b)
// with one float32 rounding, so the result does not depend on how the row is spread over the
// lanes.  The kernels are bound by this arithmetic, not by memory, so the layout keeps most stages
// inside the lane (packed float32 pairs) and needs only log2(d / 32) shuffle stages.  Three
// launches: the per-head amax (block max, one atomicMax per block on the non-negative float bits,
// stored in the descale buffer), the quantisation (recomputing the transform, which is cheaper than
// storing it), and the descale finish.
#pragma once

#include "sm100_ptx.cuh"

namespace fa {

constexpr float kE4M3Max = 448.f;

// Lane layout: every lane holds 32 consecutive elements of one row (four 16-byte loads), D / 32
// lanes hold a row, a warp holds 32 / (D / 32) rows and a block of 8 warps kQuantRows<D> rows.
template <int D>
struct QuantLayout {
  static constexpr int LPR = D / 32;         // lanes per row
  static constexpr int RPW = 32 / LPR;       // rows per warp
  static constexpr int ROWS = 8 * RPW;       // rows per block
};
template <int D>
constexpr int kQuantRows = QuantLayout<D>::ROWS;

// 32 bf16 at p (16-byte aligned) to float32 (exact).
__device__ __forceinline__ void quant_load32(const __nv_bfloat16* p, float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 u = *reinterpret_cast<const uint4*>(p + 8 * q);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[8 * q + 2 * i] = __uint_as_float(w[i] << 16);
      v[8 * q + 2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
}

// y = H_D (s o x) for the rows held by the warp (lane li of a row owns elements [32 li, 32 li + 32);
// sg: this lane's 32 signs, already loaded).  Butterfly stages h = 1, 2, 4, ... in that order, each
// mapping (a, b) at indices (i, i + h) to (a + b, a - b) in float32 with round to nearest: inside
// the lane while h < 32 (stages h >= 2 on register pairs with the packed f32x2 add / subtract,
// which rounds each element like the scalar operation), then across lanes, where the lane holding
// index i + h forms o - v as fma(v, -1, o) and its partner v + o as fma(v, 1, o) (the product by
// +-1 is exact, so each is the same single rounding as the add or subtract).
template <int D>
__device__ __forceinline__ void quant_rotate32(float (&v)[32], const float (&sg)[32], bool signed_, int li) {
  if (signed_) {
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const float2 r = fmul2(make_float2(v[i], v[i + 1]), make_float2(sg[i], sg[i + 1]));
      v[i] = r.x;
      v[i + 1] = r.y;
    }
  }
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const float a = v[i], b = v[i + 1];
    v[i] = __fadd_rn(a, b);
    v[i + 1] = __fsub_rn(a, b);
  }
#pragma unroll
  for (int h = 2; h < 32; h *= 2) {
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      if (!(i & h)) {
        const float2 a = make_float2(v[i], v[i + 1]), b = make_float2(v[i + h], v[i + h + 1]);
        const float2 sum = fadd2(a, b);
        const float2 dif = fadd2(a, make_float2(-b.x, -b.y));
        v[i] = sum.x;
        v[i + 1] = sum.y;
        v[i + h] = dif.x;
        v[i + h + 1] = dif.y;
      }
    }
  }
#pragma unroll
  for (int m = 1; m < QuantLayout<D>::LPR; m *= 2) {
    const float sgn = (li & m) ? -1.f : 1.f;  // the lane holding index i + h of each butterfly: o - v
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const float o0 = __shfl_xor_sync(0xffffffffu, v[i], m);
      const float o1 = __shfl_xor_sync(0xffffffffu, v[i + 1], m);
      const float2 r = ffma2(make_float2(v[i], v[i + 1]), make_float2(sgn, sgn), make_float2(o0, o1));
      v[i] = r.x;
      v[i + 1] = r.y;
    }
  }
}

// This lane's 32 signs (all +1 without a sign vector or without the rotation).
template <int D>
__device__ __forceinline__ bool quant_signs(const float* signs, int hadamard, int li, float (&sg)[32]) {
  const bool use = hadamard && signs != nullptr;
#pragma unroll
  for (int i = 0; i < 32; ++i) sg[i] = use ? __ldg(signs + 32 * li + i) : 1.f;
  return use;
}

// Per-head max |y| into amax_bits (non-negative floats order like their bit patterns).
template <int D>
__global__ void __launch_bounds__(256) fa_quant_amax_kernel(const __nv_bfloat16* __restrict__ x,
                                                            const float* __restrict__ signs,
                                                            unsigned int* __restrict__ amax_bits, int N, int chunks,
                                                            int hadamard) {
  using L = QuantLayout<D>;
  __shared__ float red[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int li = lane % L::LPR;
  const long long bh = blockIdx.x / chunks;
  const int r = (blockIdx.x % chunks) * L::ROWS + warp * L::RPW + lane / L::LPR;
  float sg[32];
  const bool signed_ = quant_signs<D>(signs, hadamard, li, sg);
  float v[32];
  if (r < N) {
    quant_load32(x + ((size_t)bh * N + r) * D + 32 * li, v);
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = 0.f;  // rows past N still take part in the shuffles
  }
  if (hadamard) quant_rotate32<D>(v, sg, signed_, li);
  float mx = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) mx = fmaxf(mx, fabsf(v[i]));
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) b = fmaxf(b, red[w]);
    atomicMax(amax_bits + bh, __float_as_uint(b));
  }
}

template <int D>
__global__ void __launch_bounds__(256) fa_quant_store_kernel(const __nv_bfloat16* __restrict__ x,
                                                            const float* __restrict__ signs,
                                                            const float* __restrict__ amax,
                                                            uint8_t* __restrict__ x8, int N, int chunks,
                                                            int hadamard) {
  using L = QuantLayout<D>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int li = lane % L::LPR;
  const long long bh = blockIdx.x / chunks;
  const int r = (blockIdx.x % chunks) * L::ROWS + warp * L::RPW + lane / L::LPR;
  const float a = amax[bh];
  const float qs = a > 0.f ? __fdiv_rn(kE4M3Max, a) : 1.f;
  float sg[32];
  const bool signed_ = quant_signs<D>(signs, hadamard, li, sg);
  float v[32];
  const size_t off = ((size_t)bh * N + (r < N ? r : 0)) * D + 32 * li;
  if (r < N) {
    quant_load32(x + off, v);
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = 0.f;
  }
  if (hadamard) quant_rotate32<D>(v, sg, signed_, li);
  if (r < N) {
    uint32_t c[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 s0 = fmul2(make_float2(v[4 * i], v[4 * i + 1]), make_float2(qs, qs));
      const float2 s1 = fmul2(make_float2(v[4 * i + 2], v[4 * i + 3]), make_float2(qs, qs));
      c[i] = f32x2_to_e4m3x2(s0.x, s0.y) | (f32x2_to_e4m3x2(s1.x, s1.y) << 16);
    }
    uint4* dst = reinterpret_cast<uint4*>(x8 + off);
    dst[0] = make_uint4(c[0], c[1], c[2], c[3]);
    dst[1] = make_uint4(c[4], c[5], c[6], c[7]);
  }
}

// descale = (amax / 448) * r, in place over the amax values.
__global__ void fa_quant_descale_kernel(float* __restrict__ descale, long long BH, float r) {
  const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (i < BH) descale[i] = __fmul_rn(__fdiv_rn(descale[i], kE4M3Max), r);
}

}  // namespace fa
