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
// B200 layout: one warp per row, d / 32 consecutive elements per lane (one 4- or 8-byte load, a
// 128- or 256-byte coalesced row).  The butterflies of the transform run in stages h = 1, 2, 4,
// ...: inside a lane while h < d / 32, then across lanes with shuffles; every butterfly maps
// (a, b) at indices (i, i + h) to (a + b, a - b), so the float32 result does not depend on how
// the row is spread over the lanes.  Three launches: the per-head amax (block max, one atomicMax
// per block on the non-negative float bits, stored in the descale buffer), the quantisation
// (recomputing the transform, which is cheaper than storing it), and the descale finish.
#pragma once

#include "sm100_ptx.cuh"

namespace fa {

constexpr int kQuantRowsPerBlock = 64;  // rows of one head per block (8 warps x 8 rows)
constexpr float kE4M3Max = 448.f;

template <int D>
__device__ __forceinline__ void quant_load_row(const __nv_bfloat16* row, int lane, float (&v)[D / 32]) {
  constexpr int E = D / 32;
  if constexpr (E == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(row + 4 * lane);
    v[0] = __uint_as_float(u.x << 16);
    v[1] = __uint_as_float(u.x & 0xffff0000u);
    v[2] = __uint_as_float(u.y << 16);
    v[3] = __uint_as_float(u.y & 0xffff0000u);
  } else {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(row + 2 * lane);
    v[0] = __uint_as_float(u << 16);
    v[1] = __uint_as_float(u & 0xffff0000u);
  }
}

// y = H_D (s o x) for the row held by the warp (lane owns elements [E lane, E lane + E)).
template <int D>
__device__ __forceinline__ void quant_rotate_row(float (&v)[D / 32], const float* signs, int lane) {
  constexpr int E = D / 32;
  if (signs != nullptr) {
#pragma unroll
    for (int i = 0; i < E; ++i) v[i] = __fmul_rn(v[i], __ldg(signs + E * lane + i));
  }
#pragma unroll
  for (int h = 1; h < E; h *= 2) {
#pragma unroll
    for (int i = 0; i < E; ++i) {
      if (!(i & h)) {
        const float a = v[i], b = v[i + h];
        v[i] = __fadd_rn(a, b);
        v[i + h] = __fsub_rn(a, b);
      }
    }
  }
#pragma unroll
  for (int m = 1; m < 32; m *= 2) {
    const bool upper = (lane & m) != 0;  // holds index i + h of each butterfly, h = E m
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, v[i], m);
      v[i] = upper ? __fsub_rn(o, v[i]) : __fadd_rn(v[i], o);
    }
  }
}

// Per-head max |y| into amax_bits (non-negative floats order like their bit patterns).
template <int D>
__global__ void __launch_bounds__(256) fa_quant_amax_kernel(const __nv_bfloat16* __restrict__ x,
                                                            const float* __restrict__ signs,
                                                            unsigned int* __restrict__ amax_bits, int N, int chunks,
                                                            int hadamard) {
  constexpr int E = D / 32;
  __shared__ float red[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long bh = blockIdx.x / chunks;
  const int r0 = (blockIdx.x % chunks) * kQuantRowsPerBlock;
  float mx = 0.f;
#pragma unroll 2
  for (int rr = warp; rr < kQuantRowsPerBlock; rr += 8) {
    const int r = r0 + rr;
    if (r >= N) break;
    float v[E];
    quant_load_row<D>(x + ((size_t)bh * N + r) * D, lane, v);
    if (hadamard) quant_rotate_row<D>(v, signs, lane);
#pragma unroll
    for (int i = 0; i < E; ++i) mx = fmaxf(mx, fabsf(v[i]));
  }
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
  constexpr int E = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long bh = blockIdx.x / chunks;
  const int r0 = (blockIdx.x % chunks) * kQuantRowsPerBlock;
  const float a = amax[bh];
  const float qs = a > 0.f ? __fdiv_rn(kE4M3Max, a) : 1.f;
#pragma unroll 2
  for (int rr = warp; rr < kQuantRowsPerBlock; rr += 8) {
    const int r = r0 + rr;
    if (r >= N) break;
    float v[E];
    const size_t off = ((size_t)bh * N + r) * D;
    quant_load_row<D>(x + off, lane, v);
    if (hadamard) quant_rotate_row<D>(v, signs, lane);
    if constexpr (E == 4) {
      const uint32_t lo = f32x2_to_e4m3x2(__fmul_rn(v[0], qs), __fmul_rn(v[1], qs));
      const uint32_t hi = f32x2_to_e4m3x2(__fmul_rn(v[2], qs), __fmul_rn(v[3], qs));
      *reinterpret_cast<uint32_t*>(x8 + off + 4 * lane) = lo | (hi << 16);
    } else {
      *reinterpret_cast<uint16_t*>(x8 + off + 2 * lane) = (uint16_t)f32x2_to_e4m3x2(__fmul_rn(v[0], qs), __fmul_rn(v[1], qs));
    }
  }
}

// descale = (amax / 448) * r, in place over the amax values.
__global__ void fa_quant_descale_kernel(float* __restrict__ descale, long long BH, float r) {
  const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (i < BH) descale[i] = __fmul_rn(__fdiv_rn(descale[i], kE4M3Max), r);
}

}  // namespace fa
