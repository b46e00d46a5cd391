// C-ABI entry points (declared in include/fa.h): argument validation, TMA tensor-map encoding
// and kernel launches on the caller's stream.  Nothing here allocates device memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/fa.h"
#include "bwd_dq_sm100.cuh"
#include "bwd_sm100.cuh"
#include "decode_sm100.cuh"
#include "fwd_sm100.cuh"
#include "quant_sm100.cuh"

namespace {

constexpr int kMaxSeq = 1 << 24;
constexpr int kMaxSplits = 256;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [BH, N, D] bf16 (or 1-byte E4M3 when f8) viewed as a 3-D tensor {D, N, BH}; box = one 128-byte
// row segment (64 bf16 or 128 E4M3 columns) x 128 rows x 1, 128-byte swizzle.  Rows past N read
// as zero.
bool make_map_3d(CUtensorMap* map, const void* base, int D, int N, long long BH, bool f8 = false) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t eb = f8 ? 1 : 2;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)D * eb, (cuuint64_t)N * D * eb};
  cuuint32_t box[3] = {(cuuint32_t)(128 / eb), 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, f8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                   const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// [BH, N, D] fp32 viewed as {D, N, BH}; box = 32 columns x 128 rows x 1, 128-byte swizzle (the dQ
// accumulator, target of the backward's bulk reduce-add).  Rows past N are not written.
bool make_map_3d_f32(CUtensorMap* map, void* base, int D, int N, long long BH) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)N * D * 4};
  cuuint32_t box[3] = {32, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// [planes, Nq, Nk] bf16 bias viewed as {Nk, Nq, planes}; box = 64 keys x 128 query rows x 1, 128-byte
// swizzle: the forward stages bias tiles through it, the backward prefetches them into L2.  Rows past
// Nq and keys past Nk read as zero.
bool make_map_bias(CUtensorMap* map, const void* base, int Nk, int Nq, long long planes) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)Nk, (cuuint64_t)Nq, (cuuint64_t)planes};
  cuuint64_t strides[2] = {(cuuint64_t)Nk * 2, (cuuint64_t)Nq * Nk * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Multiprocessor count of the current device (cached per device).
int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

// Opt a kernel into its dynamic shared memory once per device.
template <typename K>
bool set_smem(K kernel, int bytes) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  static std::mutex mu;
  static const void* done[64][16];
  static int ndone[64];
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 0 || dev >= 64) return false;
  for (int i = 0; i < ndone[dev]; ++i)
    if (done[dev][i] == reinterpret_cast<const void*>(kernel)) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  if (ndone[dev] < 16) done[dev][ndone[dev]++] = reinterpret_cast<const void*>(kernel);
  return true;
}

fa_status check_common(int B, int H, int Nq, int Nk, int d, float scale) {
  if (B < 0 || H < 0 || Nq < 0 || Nk < 0) return FA_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (Nq > kMaxSeq || Nk > kMaxSeq) return FA_ERR_UNSUPPORTED;
  if ((long long)B * H > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

int decode_splits(int Lmax, int num_splits) {
  if (num_splits > 0) return num_splits < kMaxSplits ? num_splits : kMaxSplits;
  int s = (Lmax + 1023) / 1024;  // about 1024 keys (512 KB of K+V at d = 128) per chunk
  return s < 1 ? 1 : (s > kMaxSplits ? kMaxSplits : s);
}

int decode_chunk(int Lmax, int S) {
  int c = (Lmax + S - 1) / S;
  return (c + 31) & ~31;
}

// Bias and dropout of the *_ext calls, validated on the host.
struct ExtArgs {
  const __nv_bfloat16* bias;  // null: no bias
  long long sb, sh;           // element strides of b and h in the bias (0 where broadcast)
  int pb, ph;                 // the same strides in [Nq, Nk] planes
  long long planes;           // bias_B * bias_H
  int H;
  fa::DropoutCfg drop;
};

// The bias tensor map of an extended call (all zero when there is no bias: never read then).
bool ext_bias_map(CUtensorMap* map, const ExtArgs* ext, int Nq, int Nk) {
  std::memset(map, 0, sizeof(*map));
  if (!ext || !ext->bias) return true;
  return make_map_bias(map, ext->bias, Nk, Nq, ext->planes);
}

template <typename P>
void set_ext(P& p, const ExtArgs* ext) {
  p.bias = ext ? ext->bias : nullptr;
  p.bias_sb = ext ? ext->sb : 0;
  p.bias_sh = ext ? ext->sh : 0;
  p.bias_pb = ext ? ext->pb : 0;
  p.bias_ph = ext ? ext->ph : 0;
  p.H = ext ? ext->H : 1;
  p.drop = ext ? ext->drop : fa::DropoutCfg{0u, 1.f, 0u, 0u, 0u};
}

// Checks the bias shape and dropout probability and fills ext.
fa_status make_ext(ExtArgs* ext, const void* bias, int bias_B, int bias_H, int B, int H, int Nq, int Nk,
                   float dropout_p, unsigned long long seed, unsigned int offset) {
  if (!(dropout_p >= 0.f && dropout_p < 1.f)) return FA_ERR_INVALID_ARG;
  // p8 = floor(256 p + 1/2): a tie (256 p exactly half-way between two integers) goes up.
  const long r = (long)std::floor(256.0 * (double)dropout_p + 0.5);
  const uint32_t p8 = (uint32_t)(r > 255 ? 255 : r);
  ext->drop = fa::DropoutCfg{p8, (float)(256.0 / (256.0 - (double)p8)), (uint32_t)(seed & 0xffffffffull),
                             (uint32_t)(seed >> 32), offset};
  ext->H = H;
  ext->bias = static_cast<const __nv_bfloat16*>(bias);
  ext->sb = ext->sh = 0;
  ext->pb = ext->ph = 0;
  ext->planes = 1;
  if (bias) {
    if ((bias_B != 1 && bias_B != B) || (bias_H != 1 && bias_H != H)) return FA_ERR_INVALID_ARG;
    if (Nk % 8 != 0) return FA_ERR_UNSUPPORTED;  // bias rows are read in 16-byte chunks
    if (!aligned16(bias)) return FA_ERR_MISALIGNED;
    const long long plane = (long long)Nq * Nk;
    ext->sh = bias_H == 1 ? 0 : plane;
    ext->sb = bias_B == 1 ? 0 : (long long)bias_H * plane;
    ext->ph = bias_H == 1 ? 0 : 1;
    ext->pb = bias_B == 1 ? 0 : bias_H;
    ext->planes = (long long)bias_B * bias_H;
  }
  return FA_OK;
}

template <int D, bool F8 = false, bool EXT = false>
fa_status launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int BH, int Nq, int Nk,
                     float scale, int causal, cudaStream_t stream, const float* descale_q = nullptr,
                     const float* descale_k = nullptr, const float* descale_v = nullptr,
                     const ExtArgs* ext = nullptr) {
  using T = fa::FwdTraits<D, F8, EXT>;
  CUtensorMap mq, mk, mv;
  if (!make_map_3d(&mq, q, D, Nq, BH, F8) || !make_map_3d(&mk, k, D, Nk, BH, F8) ||
      !make_map_3d(&mv, v, D, Nk, BH, F8))
    return FA_ERR_CUDA;
  if (!set_smem(fa::fa_fwd_kernel<D, F8, EXT>, T::SMEM_BYTES)) return FA_ERR_CUDA;
  fa::FwdParams p;
  set_ext(p, ext);
  p.descale_q = descale_q;
  p.descale_k = descale_k;
  p.descale_v = descale_v;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.Nq = Nq;
  p.Nk = Nk;
  p.BH = BH;
  // Two 128-row tiles per work item (softmax / MMA ping-pong) unless there are fewer such items than
  // SMs; then one tile per item and one item per CTA.  With two tiles the grid is persistent: one CTA
  // per SM walks its share of the items.
  const int sms = num_sms();
  p.tiles = ((long long)((Nq + 255) / 256) * BH < sms) ? 1 : 2;
  p.nunits = (Nq + 128 * p.tiles - 1) / (128 * p.tiles);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.causal = causal ? 1 : 0;
  const long long items = (long long)p.nunits * BH;
  if (items > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  const long long blocks = p.tiles == 2 ? (items < sms ? items : sms) : items;
  // The kernel counts K/V loads per CTA in 32-bit integers.
  const long long loads_per_cta = ((items + blocks - 1) / blocks) * 2LL * ((Nk + 127) / 128);
  if (loads_per_cta > (1LL << 30)) return FA_ERR_UNSUPPORTED;
  CUtensorMap mb;
  if (!ext_bias_map(&mb, ext, Nq, Nk)) return FA_ERR_CUDA;
  fa::fa_fwd_kernel<D, F8, EXT><<<(unsigned)blocks, T::THREADS, T::SMEM_BYTES, stream>>>(mq, mk, mv, mb, p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// deterministic: dK/dV from the key-block kernel without its dQ part, and dQ from the
// query-block kernel (no accumulator, no atomics).  With no key at all the regular path runs
// (it only writes zeros).
template <int D>
fa_status launch_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                     void* dq, void* dk, void* dv, void* ws, int BH, int Nq, int Nk, float scale, int causal,
                     cudaStream_t stream, bool deterministic, const ExtArgs* ext = nullptr) {
  if (Nk == 0) deterministic = false;
  using T = fa::BwdTraits<D>;
  const long long rows = (long long)BH * Nq;
  float* dvec = static_cast<float*>(ws);
  float* dq_acc = reinterpret_cast<float*>(static_cast<char*>(ws) + align256((size_t)rows * 4));
  if (rows > 0) {
    fa::fa_bwd_preprocess_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), dvec,
        deterministic ? nullptr : dq_acc, rows);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  if (Nk > 0) {
    CUtensorMap mq, mk, mv, mdo, mdq;
    if (!make_map_3d(&mq, q, D, Nq, BH) || !make_map_3d(&mk, k, D, Nk, BH) || !make_map_3d(&mv, v, D, Nk, BH) ||
        !make_map_3d(&mdo, dO, D, Nq, BH) || !make_map_3d_f32(&mdq, dq_acc, D, Nq > 0 ? Nq : 1, BH))
      return FA_ERR_CUDA;
    if (!set_smem(fa::fa_bwd_main_kernel<D, true>, T::SMEM_BYTES) ||
        !set_smem(fa::fa_bwd_main_kernel<D, false>, T::SMEM_BYTES) ||
        (ext && !set_smem(fa::fa_bwd_main_kernel<D, true, true>, T::SMEM_BYTES)))
      return FA_ERR_CUDA;
    fa::BwdParams p;
    set_ext(p, ext);
    p.lse = lse;
    p.dvec = dvec;
    p.dq_acc = dq_acc;
    p.dk = static_cast<__nv_bfloat16*>(dk);
    p.dv = static_cast<__nv_bfloat16*>(dv);
    p.Nq = Nq;
    p.Nk = Nk;
    p.BH = BH;
    p.nkt = (Nk + 127) / 128;
    // Heads per group: their Q and dO (bf16) and dQ accumulator (fp32), 8 Nq d bytes a head,
    // within ~32 MB of the 126 MB L2, but at least enough heads for the group's key blocks to fill
    // the SMs (one head of a long sequence already does).
    {
      const long long per_head = 8LL * Nq * D;
      long long g = (32LL << 20) / (per_head > 0 ? per_head : 1);
      const long long fill = (num_sms() + p.nkt - 1) / p.nkt;
      g = g < fill ? fill : g;
      g = g < 1 ? 1 : g;
      p.hgroup = (int)(g < BH ? g : BH);
    }
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.causal = causal ? 1 : 0;
    const long long blocks = (long long)p.nkt * BH;
    if (blocks > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
    CUtensorMap mb;
    if (!ext_bias_map(&mb, ext, Nq, Nk)) return FA_ERR_CUDA;
    if (ext)
      fa::fa_bwd_main_kernel<D, true, true><<<(unsigned)blocks, T::THREADS, T::SMEM_BYTES, stream>>>(mq, mk, mv, mdo,
                                                                                                     mdq, mb, p);
    else if (deterministic)
      fa::fa_bwd_main_kernel<D, false><<<(unsigned)blocks, T::THREADS, T::SMEM_BYTES, stream>>>(mq, mk, mv, mdo, mdq,
                                                                                                mb, p);
    else
      fa::fa_bwd_main_kernel<D, true><<<(unsigned)blocks, T::THREADS, T::SMEM_BYTES, stream>>>(mq, mk, mv, mdo, mdq,
                                                                                               mb, p);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    if (deterministic && Nq > 0) {
      using TQ = fa::DqTraits<D>;
      if (!set_smem(fa::fa_bwd_dq_kernel<D>, TQ::SMEM_BYTES)) return FA_ERR_CUDA;
      fa::DqParams pq;
      pq.dq = static_cast<__nv_bfloat16*>(dq);
      pq.lse = lse;
      pq.dvec = dvec;
      pq.Nq = Nq;
      pq.Nk = Nk;
      pq.BH = BH;
      pq.nqt = (Nq + 127) / 128;
      pq.scale = scale;
      pq.scale_log2 = scale * 1.4426950408889634f;
      pq.causal = causal ? 1 : 0;
      const long long qblocks = (long long)pq.nqt * BH;
      if (qblocks > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
      fa::fa_bwd_dq_kernel<D><<<(unsigned)qblocks, TQ::THREADS, TQ::SMEM_BYTES, stream>>>(mq, mk, mv, mdo, pq);
      if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    }
  }
  if (rows > 0 && !deterministic) {
    const long long n8 = rows * D / 8;
    fa::fa_bwd_dq_convert_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, stream>>>(
        dq_acc, static_cast<__nv_bfloat16*>(dq), n8);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  return FA_OK;
}

template <int D>
fa_status launch_decode(const void* q, const void* kc, const void* vc, const int* seqlens, int Lmax, void* o,
                        float* lse, int BH, int H, float scale, int S, void* ws, cudaStream_t stream) {
  using T = fa::DecTraits<D>;
  if (!set_smem(fa::fa_decode_split_kernel<D>, T::SMEM_BYTES)) return FA_ERR_CUDA;
  fa::DecParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.kc = static_cast<const __nv_bfloat16*>(kc);
  p.vc = static_cast<const __nv_bfloat16*>(vc);
  p.seqlens = seqlens;
  p.part_o = static_cast<float*>(ws);
  p.part_ml = reinterpret_cast<float*>(static_cast<char*>(ws) + align256((size_t)BH * S * D * 4));
  p.Lmax = Lmax;
  p.H = H;
  p.S = S;
  p.C = decode_chunk(Lmax, S);
  p.scale_log2 = scale * 1.4426950408889634f;
  const long long units = (long long)BH * S;
  if (units > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  fa::fa_decode_split_kernel<D><<<(unsigned)units, T::THREADS, T::SMEM_BYTES, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  fa::fa_decode_merge_kernel<D><<<(unsigned)((BH + 3) / 4), 128, 0, stream>>>(
      p.part_o, p.part_ml, static_cast<__nv_bfloat16*>(o), lse, BH, S);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <int D>
fa_status launch_decode_partials(const void* q, const void* kc, const void* vc, const int* seqlens, int Lmax,
                                 float* part_o, float* part_ml, int BH, int H, float scale, int S,
                                 cudaStream_t stream) {
  using T = fa::DecTraits<D>;
  if (!set_smem(fa::fa_decode_split_kernel<D>, T::SMEM_BYTES)) return FA_ERR_CUDA;
  fa::DecParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.kc = static_cast<const __nv_bfloat16*>(kc);
  p.vc = static_cast<const __nv_bfloat16*>(vc);
  p.seqlens = seqlens;
  p.part_o = part_o;
  p.part_ml = part_ml;
  p.Lmax = Lmax;
  p.H = H;
  p.S = S;
  p.C = decode_chunk(Lmax, S);
  p.scale_log2 = scale * 1.4426950408889634f;
  const long long units = (long long)BH * S;
  if (units > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  fa::fa_decode_split_kernel<D><<<(unsigned)units, T::THREADS, T::SMEM_BYTES, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

extern "C" {

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq, int Nk,
                 int d, float scale, int causal, void* stream) {
  fa_status st = check_common(B, H, Nq, Nk, d, scale);
  if (st != FA_OK) return st;
  const long long BH = (long long)B * H;
  if (BH == 0 || Nq == 0) return FA_OK;
  if (!q || !o || !lse || (Nk > 0 && (!k || !v))) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || !aligned16(lse) || (Nk > 0 && (!aligned16(k) || !aligned16(v))))
    return FA_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (Nk == 0) {
    const long long rows = BH * Nq;
    const long long n = rows * d;
    fa::fa_fwd_empty_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(static_cast<__nv_bfloat16*>(o), lse, rows,
                                                                         d);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
  }
  return d == 64 ? launch_fwd<64>(q, k, v, o, lse, (int)BH, Nq, Nk, scale, causal, s)
                 : launch_fwd<128>(q, k, v, o, lse, (int)BH, Nq, Nk, scale, causal, s);
}

fa_status fa_quantize_fp8(const void* x, const float* signs, void* x8, float* descale, int B, int H, int N, int d,
                          int hadamard, void* stream) {
  if (B < 0 || H < 0 || N < 0) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (N > kMaxSeq || (long long)B * H > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  const long long BH = (long long)B * H;
  if (BH == 0) return FA_OK;
  if (!descale || (N > 0 && (!x || !x8))) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(descale) & 3u) || (signs && (reinterpret_cast<uintptr_t>(signs) & 3u)) ||
      (N > 0 && (!aligned16(x) || !aligned16(x8))))
    return FA_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The descale buffer first holds the per-head amax (float bits, atomically maximised).
  if (cudaMemsetAsync(descale, 0, (size_t)BH * sizeof(float), s) != cudaSuccess) return FA_ERR_CUDA;
  if (N > 0) {
    const int rows = d == 64 ? fa::kQuantRows<64> : fa::kQuantRows<128>;
    const int chunks = (N + rows - 1) / rows;
    const long long blocks = BH * chunks;
    if (blocks > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
    const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
    uint8_t* out = static_cast<uint8_t*>(x8);
    const int had = hadamard ? 1 : 0;
    if (d == 64) {
      fa::fa_quant_amax_kernel<64><<<(unsigned)blocks, 256, 0, s>>>(xb, signs, reinterpret_cast<unsigned*>(descale), N,
                                                                     chunks, had);
      fa::fa_quant_store_kernel<64><<<(unsigned)blocks, 256, 0, s>>>(xb, signs, descale, out, N, chunks, had);
    } else {
      fa::fa_quant_amax_kernel<128><<<(unsigned)blocks, 256, 0, s>>>(xb, signs, reinterpret_cast<unsigned*>(descale),
                                                                      N, chunks, had);
      fa::fa_quant_store_kernel<128><<<(unsigned)blocks, 256, 0, s>>>(xb, signs, descale, out, N, chunks, had);
    }
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  const float r = hadamard ? (float)(1.0 / std::sqrt((double)d)) : 1.f;
  fa::fa_quant_descale_kernel<<<(unsigned)((BH + 255) / 256), 256, 0, s>>>(descale, BH, r);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* descale_q, const float* descale_k,
                     const float* descale_v, void* o, float* lse, int B, int H, int Nq, int Nk, int d, float scale,
                     int causal, void* stream) {
  fa_status st = check_common(B, H, Nq, Nk, d, scale);
  if (st != FA_OK) return st;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  const long long BH = (long long)B * H;
  if (BH == 0 || Nq == 0) return FA_OK;
  if (!q8 || !o || !lse || !descale_q || (Nk > 0 && (!k8 || !v8 || !descale_k || !descale_v)))
    return FA_ERR_INVALID_ARG;
  if (!aligned16(q8) || !aligned16(o) || !aligned16(lse) || (Nk > 0 && (!aligned16(k8) || !aligned16(v8))) ||
      (reinterpret_cast<uintptr_t>(descale_q) & 3u) || (reinterpret_cast<uintptr_t>(descale_k) & 3u) ||
      (reinterpret_cast<uintptr_t>(descale_v) & 3u))
    return FA_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (Nk == 0) {
    const long long rows = BH * Nq;
    const long long n = rows * d;
    fa::fa_fwd_empty_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(static_cast<__nv_bfloat16*>(o), lse, rows,
                                                                         d);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
  }
  return launch_fwd<128, true>(q8, k8, v8, o, lse, (int)BH, Nq, Nk, scale, causal, s, descale_q, descale_k,
                               descale_v);
}

size_t fa_bwd_workspace_size(int B, int H, int Nq, int d) {
  if (B < 0 || H < 0 || Nq < 0 || (d != 64 && d != 128)) return 0;
  const size_t rows = (size_t)B * H * Nq;
  return align256(rows * 4) + align256(rows * d * 4);
}

static fa_status bwd_entry(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                 void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, int B, int H, int Nq, int Nk, int d,
                 float scale, int causal, void* stream, bool deterministic, const ExtArgs* ext = nullptr) {
  fa_status st = check_common(B, H, Nq, Nk, d, scale);
  if (st != FA_OK) return st;
  const long long BH = (long long)B * H;
  if (BH == 0 || (Nq == 0 && Nk == 0)) return FA_OK;
  const bool has_q = Nq > 0, has_k = Nk > 0;
  if ((has_q && (!q || !o || !dO || !lse || !dq)) || (has_k && (!k || !v || !dk || !dv)))
    return FA_ERR_INVALID_ARG;
  if ((has_q && (!aligned16(q) || !aligned16(o) || !aligned16(dO) || !aligned16(lse) || !aligned16(dq))) ||
      (has_k && (!aligned16(k) || !aligned16(v) || !aligned16(dk) || !aligned16(dv))))
    return FA_ERR_MISALIGNED;
  const size_t need = fa_bwd_workspace_size(B, H, Nq, d);
  if (need > 0 && (!workspace || ws_bytes < need)) return FA_ERR_WORKSPACE;
  if (need > 0 && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return FA_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!has_q) {
    // No query row: no score touches any key, so dK = dV = 0 (nothing else is read or written).
    const size_t bytes = (size_t)BH * Nk * d * sizeof(__nv_bfloat16);
    if (cudaMemsetAsync(dk, 0, bytes, s) != cudaSuccess || cudaMemsetAsync(dv, 0, bytes, s) != cudaSuccess)
      return FA_ERR_CUDA;
    return FA_OK;
  }
  return d == 64 ? launch_bwd<64>(q, k, v, o, dO, lse, dq, dk, dv, workspace, (int)BH, Nq, Nk, scale, causal, s, deterministic,
                                  ext)
                 : launch_bwd<128>(q, k, v, o, dO, lse, dq, dk, dv, workspace, (int)BH, Nq, Nk, scale, causal, s,
                                   deterministic, ext);
}

fa_status fa_fwd_ext(const void* q, const void* k, const void* v, const void* bias, int bias_B, int bias_H, void* o,
                     float* lse, int B, int H, int Nq, int Nk, int d, float scale, int causal, float dropout_p,
                     unsigned long long seed, unsigned int offset, void* stream) {
  fa_status st = check_common(B, H, Nq, Nk, d, scale);
  if (st != FA_OK) return st;
  ExtArgs ext;
  if ((st = make_ext(&ext, bias, bias_B, bias_H, B, H, Nq, Nk, dropout_p, seed, offset)) != FA_OK) return st;
  const long long BH = (long long)B * H;
  if (BH == 0 || Nq == 0) return FA_OK;
  if (!q || !o || !lse || (Nk > 0 && (!k || !v))) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || !aligned16(lse) || (Nk > 0 && (!aligned16(k) || !aligned16(v))))
    return FA_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (Nk == 0) {
    const long long rows = BH * Nq;
    const long long n = rows * d;
    fa::fa_fwd_empty_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(static_cast<__nv_bfloat16*>(o), lse, rows,
                                                                         d);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
  }
  return d == 64 ? launch_fwd<64, false, true>(q, k, v, o, lse, (int)BH, Nq, Nk, scale, causal, s, nullptr, nullptr,
                                               nullptr, &ext)
                 : launch_fwd<128, false, true>(q, k, v, o, lse, (int)BH, Nq, Nk, scale, causal, s, nullptr, nullptr,
                                                nullptr, &ext);
}

fa_status fa_bwd_ext(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                     const void* bias, int bias_B, int bias_H, void* dq, void* dk, void* dv, void* workspace,
                     size_t ws_bytes, int B, int H, int Nq, int Nk, int d, float scale, int causal, float dropout_p,
                     unsigned long long seed, unsigned int offset, void* stream) {
  fa_status st = check_common(B, H, Nq, Nk, d, scale);
  if (st != FA_OK) return st;
  ExtArgs ext;
  if ((st = make_ext(&ext, bias, bias_B, bias_H, B, H, Nq, Nk, dropout_p, seed, offset)) != FA_OK) return st;
  return bwd_entry(q, k, v, o, dO, lse, dq, dk, dv, workspace, ws_bytes, B, H, Nq, Nk, d, scale, causal, stream,
                   false, &ext);
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                 void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, int B, int H, int Nq, int Nk, int d,
                 float scale, int causal, void* stream) {
  return bwd_entry(q, k, v, o, dO, lse, dq, dk, dv, workspace, ws_bytes, B, H, Nq, Nk, d, scale, causal, stream,
                   false);
}

fa_status fa_bwd_deterministic(const void* q, const void* k, const void* v, const void* o, const void* dO,
                               const float* lse, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, int B,
                               int H, int Nq, int Nk, int d, float scale, int causal, void* stream) {
  return bwd_entry(q, k, v, o, dO, lse, dq, dk, dv, workspace, ws_bytes, B, H, Nq, Nk, d, scale, causal, stream,
                   true);
}

size_t fa_decode_workspace_size(int B, int H, int Lmax, int d, int num_splits) {
  if (B < 0 || H < 0 || Lmax < 1 || Lmax > kMaxSeq || (d != 64 && d != 128) || num_splits < 0) return 0;
  const int S = decode_splits(Lmax, num_splits);
  const size_t units = (size_t)B * H * S;
  return align256(units * d * 4) + align256(units * 2 * 4);
}

fa_status fa_decode_splitkv(const void* q, const void* k_cache, const void* v_cache, const int* seqlens, int Lmax,
                            void* o, float* lse, int B, int H, int d, float scale, int num_splits, void* workspace,
                            size_t ws_bytes, void* stream) {
  if (B < 0 || H < 0 || num_splits < 0) return FA_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (Lmax < 1 || Lmax > kMaxSeq) return Lmax < 1 ? FA_ERR_INVALID_ARG : FA_ERR_UNSUPPORTED;
  if (num_splits > kMaxSplits) return FA_ERR_UNSUPPORTED;
  const long long BH = (long long)B * H;
  if (BH > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  if (BH == 0) return FA_OK;
  if (!q || !k_cache || !v_cache || !seqlens || !o) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
      (lse && !aligned16(lse)) || (reinterpret_cast<uintptr_t>(seqlens) & 3u))
    return FA_ERR_MISALIGNED;
  const size_t need = fa_decode_workspace_size(B, H, Lmax, d, num_splits);
  if (!workspace || ws_bytes < need) return FA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return FA_ERR_MISALIGNED;
  const int S = decode_splits(Lmax, num_splits);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d == 64 ? launch_decode<64>(q, k_cache, v_cache, seqlens, Lmax, o, lse, (int)BH, H, scale, S, workspace, s)
                 : launch_decode<128>(q, k_cache, v_cache, seqlens, Lmax, o, lse, (int)BH, H, scale, S, workspace, s);
}

int fa_decode_num_splits(int Lmax, int num_splits) {
  if (Lmax < 1 || Lmax > kMaxSeq || num_splits < 0 || num_splits > kMaxSplits) return 0;
  return decode_splits(Lmax, num_splits);
}

fa_status fa_decode_partials(const void* q, const void* k_cache, const void* v_cache, const int* seqlens, int Lmax,
                             float* part_o, float* part_ml, int B, int H, int d, float scale, int num_splits,
                             void* stream) {
  if (B < 0 || H < 0 || num_splits < 0) return FA_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (Lmax < 1 || Lmax > kMaxSeq) return Lmax < 1 ? FA_ERR_INVALID_ARG : FA_ERR_UNSUPPORTED;
  if (num_splits > kMaxSplits) return FA_ERR_UNSUPPORTED;
  const long long BH = (long long)B * H;
  if (BH > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  if (BH == 0) return FA_OK;
  if (!q || !k_cache || !v_cache || !seqlens || !part_o || !part_ml) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(part_o) || !aligned16(part_ml) ||
      (reinterpret_cast<uintptr_t>(seqlens) & 3u))
    return FA_ERR_MISALIGNED;
  const int S = decode_splits(Lmax, num_splits);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d == 64 ? launch_decode_partials<64>(q, k_cache, v_cache, seqlens, Lmax, part_o, part_ml, (int)BH, H, scale, S, s)
                 : launch_decode_partials<128>(q, k_cache, v_cache, seqlens, Lmax, part_o, part_ml, (int)BH, H, scale, S,
                                               s);
}

fa_status fa_decode_merge(const float* part_o, const float* part_ml, int R, int S, void* o, float* lse, int B, int H,
                          int d, void* stream) {
  if (B < 0 || H < 0 || R < 1 || S < 1) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const long long BH = (long long)B * H;
  if (BH > 0x7fffffffLL || (long long)R * S > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  if (BH == 0) return FA_OK;
  if (!part_o || !part_ml || !o) return FA_ERR_INVALID_ARG;
  if (!aligned16(part_o) || !aligned16(part_ml) || !aligned16(o) || (lse && !aligned16(lse))) return FA_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const unsigned grid = (unsigned)((BH + 3) / 4);
  if (d == 64)
    fa::fa_decode_merge_kernel<64><<<grid, 128, 0, s>>>(part_o, part_ml, static_cast<__nv_bfloat16*>(o), lse,
                                                        (int)BH, S, R);
  else
    fa::fa_decode_merge_kernel<128><<<grid, 128, 0, s>>>(part_o, part_ml, static_cast<__nv_bfloat16*>(o), lse,
                                                         (int)BH, S, R);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_get_device_error(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return FA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, fa::g_status, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(fa::g_status, &zero, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  }
  return v == 0 ? FA_OK : static_cast<fa_status>(v);
}

fa_status fa_debug_set_wait_limit(unsigned long long limit_ns) {
  const unsigned long long lim = limit_ns == 0 ? fa::kWaitLimitNs : limit_ns;
  const uint32_t hint = (uint32_t)(lim < fa::kSuspendHintNs ? lim : fa::kSuspendHintNs);
  if (cudaMemcpyToSymbol(fa::c_wait_limit_ns, &lim, sizeof(lim)) != cudaSuccess) return FA_ERR_CUDA;
  if (cudaMemcpyToSymbol(fa::c_suspend_hint_ns, &hint, sizeof(hint)) != cudaSuccess) return FA_ERR_CUDA;
  return FA_OK;
}

const char* fa_status_string(fa_status status) {
  switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported size or head dimension";
    case FA_ERR_MISALIGNED: return "pointer not 16-byte aligned (workspace: 256-byte)";
    case FA_ERR_WORKSPACE: return "workspace missing or too small";
    case FA_ERR_CUDA: return "CUDA runtime or driver call failed";
    case FA_ERR_TIMEOUT: return "a bounded device-side wait gave up";
  }
  return "unknown status";
}

int fa_version(void) { return 100; }

}  // extern "C"

// ---------------------------------------------------------------------------------------------
// Allocation-free split-KV decode: the partials live in a file-scope device array instead of a
// caller workspace.  Host code must not hand the array's name to a kernel (in host code it is a
// host-side stand-in, not a device address); it looks up each device's address once.
// ---------------------------------------------------------------------------------------------
namespace {

constexpr size_t kNoallocScratchBytes = FA_DECODE_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_decode_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once per device).
fa_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return FA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return FA_OK;
}

}  // namespace

extern "C" fa_status fa_decode_splitkv_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                               const int* seqlens, int Lmax, void* o, float* lse, int B, int H,
                                               int d, float scale, int num_splits, void* stream) {
  if (B < 0 || H < 0 || num_splits < 0) return FA_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (Lmax < 1 || Lmax > kMaxSeq) return Lmax < 1 ? FA_ERR_INVALID_ARG : FA_ERR_UNSUPPORTED;
  if (num_splits > kMaxSplits) return FA_ERR_UNSUPPORTED;
  const long long BH = (long long)B * H;
  if (BH > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  if (BH == 0) return FA_OK;
  if (!q || !k_cache || !v_cache || !seqlens || !o) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
      (lse && !aligned16(lse)) || (reinterpret_cast<uintptr_t>(seqlens) & 3u))
    return FA_ERR_MISALIGNED;
  if (fa_decode_workspace_size(B, H, Lmax, d, num_splits) > kNoallocScratchBytes) return FA_ERR_WORKSPACE;
  void* ws = nullptr;
  const fa_status st = noalloc_scratch(&ws);
  if (st != FA_OK) return st;
  const int S = decode_splits(Lmax, num_splits);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d == 64 ? launch_decode<64>(q, k_cache, v_cache, seqlens, Lmax, o, lse, (int)BH, H, scale, S, ws, s)
                 : launch_decode<128>(q, k_cache, v_cache, seqlens, Lmax, o, lse, (int)BH, H, scale, S, ws, s);
}
