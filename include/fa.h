/*
 * io_aware_exact_32_b200 -- exact IO-aware fused attention for NVIDIA B200 (sm_100a).
 *
 * C ABI.  Plain pointers and sizes only; no C++ or framework types cross it.
 *
 * The operation is exact scaled-dot-product attention,
 *     O = softmax(scale * Q K^T [+ causal mask]) V,
 * with Q in R^{Nq x d} and K, V in R^{Nk x d} per (batch, head)
 * ("Transformer、注意力机制与优化", section 数学公式; the (batch, heads, seq,
 * head_dim) layout of "优化的注意力实现 (FlashAttention)", section 优势与集成).
 *
 * Conventions shared by every call:
 *  - Tensors are contiguous row-major [B, H, N, d] with d innermost, element
 *    type bf16 (IEEE bfloat16, 2 bytes), unless stated otherwise.  LSE, D and
 *    workspaces are fp32.
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *    never allocates, frees or retains device memory at call time; its module
 *    holds one static status word per device (see fa_get_device_error) and the
 *    fixed scratch array of fa_decode_splitkv_noalloc.
 *  - Every tensor pointer must be 16-byte aligned (the TMA engine requires it);
 *    otherwise FA_ERR_MISALIGNED is returned and nothing is launched.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = the legacy default stream).  Arguments are validated on the host
 *    before anything is launched; on any error nothing is launched.
 *  - Supported head dimensions: d = 64 and d = 128 (FA_ERR_UNSUPPORTED otherwise).
 *  - causal != 0 applies the lower-triangle mask aligned to the bottom-right
 *    corner: key j is visible to query i iff j <= i + (Nk - Nq).  For Nq == Nk
 *    this is tril(diagonal=0).  A query row that sees no key gets O = 0 and
 *    LSE = -inf.
 *  - LSE is the natural log of sum_j exp(scale * q_i . k_j) over visible keys.
 *  - Gradients are overwritten, not accumulated.
 *  - No exception, abort or exit crosses this boundary.
 *  - Device-side waits are bounded; a wait that gives up records
 *    FA_ERR_TIMEOUT in the device status word and the kernel returns.
 */
#ifndef IO_AWARE_EXACT_32_B200_FA_H
#define IO_AWARE_EXACT_32_B200_FA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,  /* null pointer, negative size, bad scale */
  FA_ERR_UNSUPPORTED = 2,  /* d not in {64, 128}, or a size beyond the limits below */
  FA_ERR_MISALIGNED = 3,   /* a tensor pointer not 16-byte aligned */
  FA_ERR_WORKSPACE = 4,    /* workspace missing or smaller than the *_workspace_size query */
  FA_ERR_CUDA = 5,         /* a CUDA runtime/driver call failed (launch, tensor map) */
  FA_ERR_TIMEOUT = 6       /* a bounded device wait gave up (reported by fa_get_device_error) */
} fa_status;

/*
 * Forward pass: O and LSE in one fused pass.
 *
 * Follows the tiled forward with the online-softmax recurrence (running max m,
 * running sum l, rescaled output accumulator) of "Transformer、注意力机制与优化",
 * sections 安全 Softmax 与在线 Softmax and FlashAttention-2 算法, with the
 * deferred normalisation and the single saved statistic L = m + log(l) of
 * "FlashAttention 系列技术详解", section 具体优化策略.  The N x N score
 * matrix never reaches device memory.
 *
 *   q    [B, H, Nq, d] bf16, read
 *   k, v [B, H, Nk, d] bf16, read
 *   o    [B, H, Nq, d] bf16, written
 *   lse  [B, H, Nq] fp32, written (natural log; -inf for rows with no visible key)
 *   scale: multiplies q.k before the softmax (finite, > 0); usually 1/sqrt(d)
 * Limits: 0 <= B*H <= 2^31-1, 0 <= Nq, Nk <= 2^24.  Nq == 0 or B*H == 0 is a
 * no-op; Nk == 0 writes O = 0 and LSE = -inf.
 */
FA_API fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int H, int Nq, int Nk, int d, float scale, int causal,
                 void* stream);

/*
 * Additive bias and dropout: O = dropout(softmax(scale * Q K^T + bias
 * [+ causal mask])) V, the manual path of "优化的注意力实现 (FlashAttention)",
 * section 优势与集成 (attn_bias added to the scaled scores, dropout on the
 * weights), and its backward ("FlashAttention 的基本原理", section 2.4 反向传播:
 * the algorithm covers masking and dropout).
 *
 *   bias   [bias_B, bias_H, Nq, Nk] bf16 or NULL; bias_B in {1, B} and
 *          bias_H in {1, H} (size 1 = broadcast).  -inf masks an entry;
 *          +inf and NaN are not allowed.  Requires Nk % 8 == 0
 *          (FA_ERR_UNSUPPORTED otherwise) and a 16-byte aligned pointer.
 *          The bias is a constant: no gradient is computed for it.
 *   dropout_p in [0, 1): each weight is dropped with probability
 *          p8 / 256, p8 = floor(256 p + 1/2) (at most 255; a tie goes
 *          up), and kept weights are scaled by 256 / (256 - p8).  LSE is
 *          that of the weights before dropout.
 *   seed, offset: the dropout decisions are regenerated, not stored:
 *          Philox4x32-10 (Salmon et al., SC 2011) with key (seed low 32
 *          bits, seed high 32 bits) and counter (key / 4, query / 4,
 *          b * H + h, offset); byte (key % 4) of output word (query % 4) is
 *          the entry's random byte u, kept iff u >= p8.  fa_bwd_ext must get
 *          the same bias, dropout_p, seed and offset as the forward.
 * Other arguments, layouts and limits as fa_fwd / fa_bwd (same workspace).
 * dropout_p = 0 and bias = NULL give fa_fwd / fa_bwd's results through the
 * slower extended kernels.  There is no deterministic variant.
 */
FA_API fa_status fa_fwd_ext(const void* q, const void* k, const void* v, const void* bias,
                 int bias_B, int bias_H, void* o, float* lse, int B, int H, int Nq, int Nk,
                 int d, float scale, int causal, float dropout_p, unsigned long long seed,
                 unsigned int offset, void* stream);
FA_API fa_status fa_bwd_ext(const void* q, const void* k, const void* v, const void* o,
                 const void* dO, const float* lse, const void* bias, int bias_B, int bias_H,
                 void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                 int B, int H, int Nq, int Nk, int d, float scale, int causal,
                 float dropout_p, unsigned long long seed, unsigned int offset, void* stream);

/*
 * FP8 (E4M3) operands with incoherent processing ("FlashAttention 系列技术详解",
 * section 具体技术, FlashAttention-3): the score and output GEMMs run on FP8
 * tensor cores, and Q and K are first multiplied by a random orthogonal matrix,
 * a Hadamard transform, to spread outlier channels before quantisation.
 *
 * E4M3 here is the "FN" byte format: 1 sign, 4 exponent bits (bias 7),
 * 3 mantissa bits, largest finite value 448, no infinities; conversions round
 * to nearest even and saturate.
 *
 * fa_quantize_fp8: x8 = rn_e4m3(y * 448 / amax) per (batch, head), where
 *   y = H_d (s o x_row) for every row when hadamard != 0 (H_d the Sylvester
 *   Hadamard matrix, s the signs; all in fp32), y = x_row otherwise, and amax
 *   is the largest |y| of the head.  descale[b, h] = (amax / 448) / sqrt(d)
 *   with the rotation, amax / 448 without, so that x M ~= x8 * descale with
 *   M = diag(s) H_d / sqrt(d) orthogonal.  Rotate Q and K with the same signs
 *   (Q M (K M)^T = Q K^T); quantise V with hadamard = 0.
 *   x       [B, H, N, d] bf16, read
 *   signs   [d] fp32 of +-1, read; NULL = all +1 (plain Hadamard)
 *   x8      [B, H, N, d] E4M3 bytes, written
 *   descale [B, H] fp32, written (also used as scratch during the call)
 *   d in {64, 128}; N == 0 writes descale = 0.  x and x8 16-byte aligned,
 *   signs and descale 4-byte aligned.
 *
 * fa_fwd_fp8: the forward of fa_fwd on E4M3 operands, O = softmax(scale * Qd Kd^T
 *   [+ causal mask]) Vd with Qd = q8 * descale_q[b, h] (likewise K, V).  The
 *   softmax weights are rounded to E4M3 for the P V product and O is normalised
 *   by the sum of the rounded weights; LSE uses the exact fp32 sum.
 *   q8 [B, H, Nq, d], k8 / v8 [B, H, Nk, d] E4M3 bytes; descale_* [B, H] fp32;
 *   o [B, H, Nq, d] bf16 and lse [B, H, Nq] fp32 written as in fa_fwd.
 *   d = 128 only (FA_ERR_UNSUPPORTED otherwise); other limits as fa_fwd.
 */
FA_API fa_status fa_quantize_fp8(const void* x, const float* signs, void* x8, float* descale,
                 int B, int H, int N, int d, int hadamard, void* stream);
FA_API fa_status fa_fwd_fp8(const void* q8, const void* k8, const void* v8,
                 const float* descale_q, const float* descale_k, const float* descale_v,
                 void* o, float* lse, int B, int H, int Nq, int Nk, int d, float scale,
                 int causal, void* stream);

/*
 * Bytes of fp32 workspace fa_bwd needs: D [B, H, Nq] plus the dQ accumulator
 * [B, H, Nq, d], each region 256-byte aligned.  Returns 0 on invalid sizes.
 */
FA_API size_t fa_bwd_workspace_size(int B, int H, int Nq, int d);

/*
 * Backward pass by recomputation: dQ, dK, dV from Q, K, V, O, dO and the
 * saved LSE, never storing the N x N matrices.
 *
 * Follows "FlashAttention 的基本原理", section 2.4 反向传播 (recompute the
 * scores and P from the saved statistics; dV = P^T dO, dP = dO V^T, the
 * row-softmax gradient dS, dQ = dS K, dK = dS^T Q), with D_i = rowsum(dO_i * O_i)
 * and P recomputed from LSE alone ("FlashAttention 系列技术详解", section
 * 具体优化策略), and the column-block parallel schedule whose dQ partial sums
 * meet through reduce-adds in device memory ("Transformer、注意力机制与优化",
 * section 为什么前向传播和反向传播的并行化策略不同; here TMA bulk reduce-adds of
 * shared-memory-staged blocks).  The order of those adds varies, so dQ is not
 * bitwise deterministic run to run (see fa_bwd_deterministic).
 *
 *   q, o, dO [B, H, Nq, d] bf16, read;  k, v [B, H, Nk, d] bf16, read
 *   lse      [B, H, Nq] fp32, read (as written by fa_fwd)
 *   dq       [B, H, Nq, d] bf16, written;  dk, dv [B, H, Nk, d] bf16, written
 *   workspace: device fp32 scratch of at least fa_bwd_workspace_size() bytes,
 *              caller-owned, contents on entry ignored, garbage on exit
 * Same limits and mask convention as fa_fwd.
 */
FA_API fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                 const float* lse, void* dq, void* dk, void* dv,
                 void* workspace, size_t ws_bytes,
                 int B, int H, int Nq, int Nk, int d, float scale, int causal,
                 void* stream);

/*
 * Deterministic backward: the same results as fa_bwd (same arguments, same
 * workspace size query), with dQ bitwise reproducible run to run.
 *
 * dK and dV come from the key-block schedule of fa_bwd without its dQ part;
 * dQ comes from a second pass with the query block stationary, which
 * recomputes S and dP for each (query block, key block) pair and accumulates
 * dQ_i = scale * sum_j dS_ij K_j on chip, so no two blocks add into the same dQ
 * row (the nondeterminism of fa_bwd comes from the order of those adds,
 * "Transformer、注意力机制与优化", section 为什么前向传播和反向传播的并行化策略不同).
 * Costs two extra matrix products per pair (about 40% more tensor work).
 */
FA_API fa_status fa_bwd_deterministic(const void* q, const void* k, const void* v, const void* o,
                 const void* dO, const float* lse, void* dq, void* dk, void* dv,
                 void* workspace, size_t ws_bytes,
                 int B, int H, int Nq, int Nk, int d, float scale, int causal,
                 void* stream);

/*
 * Bytes of workspace fa_decode_splitkv needs for the per-split partial
 * results (m, l, unnormalised O) at the given split count (0 = the automatic
 * choice for this Lmax).  Returns 0 on invalid sizes.
 */
FA_API size_t fa_decode_workspace_size(int B, int H, int Lmax, int d, int num_splits);

/*
 * Split-KV decode: one query per (batch, head) against a KV cache with ragged
 * per-sequence lengths.  The keys of each sequence are cut into chunks that
 * are processed in parallel; each chunk yields partial (m, l, O~) and a second
 * kernel merges the partials with the two-block identity for m and l
 * ("Transformer、注意力机制与优化", sections Flash-Decoding and 安全 Softmax
 * 与在线 Softmax).  The result does not depend on the split count beyond
 * rounding.
 *
 *   q        [B, H, 1, d] bf16, read
 *   k_cache, v_cache [B, H, Lmax, d] bf16, read; slots at or beyond
 *            seqlens[b] are never read
 *   seqlens  [B] int32 DEVICE array, 1 <= seqlens[b] <= Lmax (values outside
 *            are clamped to [0, Lmax]; a length of 0 gives O = 0, LSE = -inf)
 *   o        [B, H, 1, d] bf16, written
 *   lse      [B, H] fp32, written; may be NULL
 *   num_splits: chunks per sequence at Lmax (0 = automatic; at most 256)
 *   workspace: device scratch of at least fa_decode_workspace_size() bytes
 * Limits: 1 <= Lmax <= 2^24, 0 <= B*H <= 2^31-1.
 */
FA_API fa_status fa_decode_splitkv(const void* q, const void* k_cache, const void* v_cache,
                            const int* seqlens, int Lmax, void* o, float* lse,
                            int B, int H, int d, float scale, int num_splits,
                            void* workspace, size_t ws_bytes, void* stream);

/*
 * Capacity of the library's built-in decode scratch (bytes), used only by
 * fa_decode_splitkv_noalloc.
 */
#define FA_DECODE_NOALLOC_SCRATCH_BYTES (8u << 20)

/*
 * Sequence-parallel decode building blocks (several devices each hold a slice
 * of every sequence's KV cache): the per-split partial results of
 * fa_decode_splitkv, unmerged, and their merge.  The merge is the same
 * (m, l, O) recurrence that combines splits on one device ("Transformer、注意力
 * 机制与优化", section Flash-Decoding), so partials from several devices,
 * gathered in one buffer, merge exactly like partials from one device.
 *
 * fa_decode_num_splits: the split count S fa_decode_partials uses for this
 * Lmax and num_splits (0 on invalid arguments).
 *
 * fa_decode_partials: as fa_decode_splitkv for k_cache, v_cache [B, H, Lmax, d]
 * and seqlens (device int32 [B], 0 <= L_b <= Lmax; a slice may be empty), but
 * writes, for every (b, h) and split s, the unnormalised output
 * part_o [B, H, S, d] fp32 and part_ml [B, H, S, 2] fp32 = (running max m in
 * log2 units of scale * q.k, sum l of 2^(x - m)); an empty split gives
 * (m, l) = (-inf, 0).  Buffers caller-owned, 16-byte aligned.
 *
 * fa_decode_merge: merges R groups of S partials (group r at offset r*B*H*S
 * rows: the layout of an all-gather of per-device partials along the first
 * dimension) into o [B, H, 1, d] bf16 and, if lse is not NULL, lse [B, H]
 * fp32.  A (b, h) with no key at all gets o = 0 and lse = -inf.
 */
FA_API int fa_decode_num_splits(int Lmax, int num_splits);
FA_API fa_status fa_decode_partials(const void* q, const void* k_cache, const void* v_cache,
                                    const int* seqlens, int Lmax, float* part_o, float* part_ml,
                                    int B, int H, int d, float scale, int num_splits, void* stream);
FA_API fa_status fa_decode_merge(const float* part_o, const float* part_ml, int R, int S,
                                 void* o, float* lse, int B, int H, int d, void* stream);

/*
 * Split-KV decode that allocates nothing and takes no workspace.
 *
 * The paper has no counterpart: this is an interface convenience for callers
 * that cannot allocate device memory themselves -- for example a plugin whose
 * host framework owns all device memory through its own pool and forbids raw
 * cudaMalloc, or a latency-critical serving loop in which an allocation could
 * synchronise the device.  Such a caller still owns q, the caches, seqlens, o
 * and lse; the per-split partials live instead in one file-scope device array
 * of FA_DECODE_NOALLOC_SCRATCH_BYTES inside this library, which every GPU that
 * loads the library holds until the process exits.
 *
 * Arguments, layouts, results and error codes are those of fa_decode_splitkv
 * without the workspace.  If fa_decode_workspace_size(B, H, Lmax, d,
 * num_splits) exceeds FA_DECODE_NOALLOC_SCRATCH_BYTES the call returns
 * FA_ERR_WORKSPACE and launches nothing.
 *
 * The first call on each device looks up that device's address of the scratch
 * array (cudaGetSymbolAddress, with the device current); make that first call
 * before any stream capture.  The address is kept for the life of the
 * process, so this entry point does not survive a cudaDeviceReset of that
 * device in the same process.  All calls share the one array: calls whose
 * kernels overlap on the GPU (different streams, no ordering between them)
 * race on it and must be serialised by the caller.  Nothing needs clearing
 * between calls: every partial is written before it is read.
 */
FA_API fa_status fa_decode_splitkv_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                           const int* seqlens, int Lmax, void* o, float* lse,
                                           int B, int H, int d, float scale, int num_splits,
                                           void* stream);

/*
 * Synchronises `stream`, then returns and clears the calling device's status
 * word: FA_OK, or FA_ERR_TIMEOUT if a device-side wait gave up since the last
 * call.  Returns FA_ERR_CUDA if the synchronisation itself failed.
 */
FA_API fa_status fa_get_device_error(void* stream);

/*
 * Test hook, not for production use: sets the time after which every pipeline
 * wait of this library's kernels on the current device gives up (default 2 s;
 * limit_ns == 0 restores it), and caps the hardware suspend time of those waits
 * at the same value.  With a limit of a few hundred nanoseconds the waits of a
 * healthy kernel run out: each CTA records FA_ERR_TIMEOUT, stops, waits (with
 * the fixed 2 s limit) for its own copies and MMAs still in flight, frees its
 * tensor memory and returns, so the give-up path can be tested without a
 * fault.  The setting is per device and lasts until changed; the call is
 * synchronous (it copies to device constant memory).  Returns FA_ERR_CUDA if
 * the copy fails.  The pages have no counterpart: this exists for testing.
 */
FA_API fa_status fa_debug_set_wait_limit(unsigned long long limit_ns);

/* Static, NUL-terminated description of a status code. */
FA_API const char* fa_status_string(fa_status status);

/* Library version as 10000*major + 100*minor + patch. */
FA_API int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* IO_AWARE_EXACT_32_B200_FA_H */
