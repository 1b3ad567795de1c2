/*
 * sdpa_b200.h -- C ABI of libsdpa_b200.so: fused scaled-dot-product attention
 * forward (prefill) and split-KV decode for NVIDIA B200 (sm_100a).
 *
 * The operation, for every batch b, query head hq and query row i, with
 * hk = hq / (Hq / Hkv):
 *     x_ij  = scale * sum_c q[b,hq,i,c] * k[b,hk,j,c]           (matmul, scale)
 *     x_ij  = -inf where key j is masked for row i               (masked_fill)
 *     p_ij  = exp(x_ij - max_j x_ij) / sum_j exp(x_ij - max_j x_ij)   (softmax)
 *     o[b,hq,i,:] = sum_j p_ij v[b,hk,j,:]                       (matmul)
 *     lse[b,hq,i] = max_j x_ij + ln sum_j exp(x_ij - max_j x_ij)
 * -- the five naive steps of "PyTorch attention profiling: Flash, cuDNN, Math
 * backends" (section 1), computed the FlashAttention-2 way ("FlashAttention-2"
 * notes, algorithm overview: per query block, online max/sum over key blocks,
 * one final division).  A row with no visible key gets o = 0 and
 * lse = -inf (the no-NaN intent of that page's "_safe_softmax").
 *
 * Masks (`causal`):
 *   ATTN_CAUSAL_NONE          every key visible
 *   ATTN_CAUSAL_TOP_LEFT      key j visible to row i iff j <= i
 *   ATTN_CAUSAL_BOTTOM_RIGHT  key j visible to row i iff j <= i + Sk - Sq
 *                             (query rows sit at the end of the keys)
 * Scale: scale == 0 selects 1/sqrt(d) (the default-alpha rule of the
 * onnxruntime WebGPU decode page, section 2); otherwise it must be finite and
 * > 0.
 *
 * Layout and types: every tensor is contiguous, row-major.
 *   q, o          [B, Hq,  Sq, d]  bf16
 *   k, v          [B, Hkv, Sk, d]  bf16
 *   lse           [B, Hq,  Sq]     fp32 (may be NULL)
 * d must be 64 or 128; Hq must be a multiple of Hkv (GQA: query head hq
 * reads KV head hq / (Hq/Hkv), no expansion).  q, k, v, o must be 16-byte
 * aligned device pointers; lse 4-byte aligned.
 *
 * Ownership: the caller allocates and owns every buffer, including the
 * decode workspace.  The library allocates no device memory per call (its
 * only device memory is a 4-byte error word and the fixed scratch array of
 * attn_decode_splitkv_static, both static) and keeps no per-call search.  Calls are asynchronous on `stream` (a cudaStream_t
 * passed as void*; NULL = legacy default stream) and never synchronize.
 *
 * Errors: argument errors are detected on the host before anything is
 * launched and returned synchronously; ATTN_ERR_CUDA is returned when a
 * CUDA runtime call fails (launch, attribute, tensor-map encoding).  Every
 * wait inside the kernels is bounded (1 s); a wait that gives up records a
 * bit in the device error word and the kernel exits without trapping;
 * attn_check_device_error() reports it as ATTN_ERR_DEVICE_TIMEOUT.
 * No function ever aborts the process.
 */
#ifndef SDPA_B200_H
#define SDPA_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_NULL = 1,           /* a required pointer is NULL */
  ATTN_ERR_SHAPE = 2,          /* negative size, or a size beyond the supported range */
  ATTN_ERR_GQA = 3,            /* Hq is not a multiple of Hkv */
  ATTN_ERR_HEADDIM = 4,        /* d is not 64 or 128 */
  ATTN_ERR_ALIGN = 5,          /* a pointer is not 16-byte (lse: 4-byte) aligned */
  ATTN_ERR_CAUSAL = 6,         /* unknown causal mode, or a mode the entry point lacks */
  ATTN_ERR_WORKSPACE = 7,      /* decode workspace NULL, misaligned or too small */
  ATTN_ERR_CUDA = 8,           /* a CUDA runtime call failed */
  ATTN_ERR_DEVICE_TIMEOUT = 9, /* a bounded wait inside a kernel gave up */
  ATTN_ERR_ARCH = 10,          /* the current device is not compute capability 10.0 */
  ATTN_ERR_SCALE = 11,         /* scale is negative, NaN or infinite */
  ATTN_ERR_SCRATCH_LIMIT = 12, /* attn_decode_splitkv_static: problem needs more than
                                  ATTN_STATIC_SCRATCH_BYTES of scratch */
  ATTN_ERR_SEQLEN = 13         /* reported by attn_check_device_error: a per-batch length read on
                                  the device was outside its valid range and was clamped, or a
                                  position of attn_rope_append was out of range and skipped */
} attn_status_t;

enum { ATTN_CAUSAL_NONE = 0, ATTN_CAUSAL_TOP_LEFT = 1, ATTN_CAUSAL_BOTTOM_RIGHT = 2 };

/*
 * Tensor layouts (attn_extras_t.layout): BHSD is [B, H, S, d] (heads outer,
 * the default everywhere); BSHD is [B, S, H, d] (tokens outer: the
 * non-"BNSH" Q format of the onnxruntime WebGPU decode page, section 2).
 * Both contiguous with d innermost.
 */
enum { ATTN_LAYOUT_BHSD = 0, ATTN_LAYOUT_BSHD = 1 };

/*
 * Optional inputs of attn_fwd_ex and attn_decode_splitkv_ex.  Zero-initialise
 * (memset), then set what is needed; a NULL `extras` argument means none.
 *   seqlens_q, seqlens_k  device int32 [B] per-batch valid query rows / keys
 *                         (as in attn_fwd_varlen / attn_decode_splitkv_varlen;
 *                         seqlens_q is for the forward only); NULL = all.
 *   bias                  device bf16 additive attention bias, laid out
 *                         [bias_b, bias_h, Sq, Sk] row-major, 2-byte aligned,
 *                         with bias_b in {1, B} and bias_h in {1, Hq} (1 =
 *                         broadcast over that dimension).  It is added to the
 *                         scaled scores before the causal mask:
 *                         x_ij = scale * q_i.k_j + bias[b', h', i, j], with
 *                         b' = b unless bias_b == 1 and h' = hq unless
 *                         bias_h == 1 ("[onnxruntime] WebGPU FlashAttention:
 *                         kernel fusion and variable sequence length",
 *                         section 1: the fused decode applies the attention
 *                         bias with the mask; attn_bias_dim0/dim1 broadcast).
 *                         LSE is over these x.  A -inf bias entry masks the
 *                         key.  NULL = no bias.
 *   layout                ATTN_LAYOUT_BHSD (0) or ATTN_LAYOUT_BSHD: the layout
 *                         of q, k, v and o for the forward, of q and o for the
 *                         decode (its K/V cache is always [B, Hkv, S, d]).  lse,
 *                         the lengths and the bias keep their layouts.
 */
typedef struct {
  const int* seqlens_q;
  const int* seqlens_k;
  const void* bias;
  int bias_b;
  int bias_h;
  int layout;
} attn_extras_t;

/*
 * Prefill / general forward.  Computes o (and lse when non-NULL) for any
 * Sq >= 0, Sk >= 0.  Work items are (b, hq, block of 256 query rows); each
 * visits only the key blocks its causal mask leaves visible ("FlashAttention-2"
 * notes, causal masking and sequence-length parallelism).
 */
attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                       int Sq, int Sk, int d, float scale, int causal, void* stream);

/*
 * attn_fwd with the optional inputs of attn_extras_t (per-batch lengths as in
 * attn_fwd_varlen, additive bias; `extras` may be NULL).  With a bias the
 * forward also needs Sk % 8 == 0 and a 16-byte aligned bias (it reads bias
 * rows in 16-byte pieces), else ATTN_ERR_ALIGN; invalid bias dims give
 * ATTN_ERR_SHAPE.
 */
attn_status_t attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                          int Sq, int Sk, int d, float scale, int causal, const attn_extras_t* extras,
                          void* stream);

/*
 * Forward over a batch of sequences of different lengths, held padded:
 *   q, o     [B, Hq,  Sq_max, d] bf16;  k, v [B, Hkv, Sk_max, d] bf16
 *   seqlens_q, seqlens_k  device int32 [B], 4-byte aligned: batch b has
 *            seqlens_q[b] query rows and seqlens_k[b] keys (the leading
 *            rows of its padded tensors); read by the kernels only, so they
 *            may be written by earlier work on `stream`.  A value outside
 *            [0, Sq_max] resp. [0, Sk_max] is clamped and makes
 *            attn_check_device_error() return ATTN_ERR_SEQLEN.
 * Row i < seqlens_q[b] of batch b is attention over keys j < seqlens_k[b]
 * with the mask aligned to the batch's own lengths (bottom-right: j <= i +
 * seqlens_k[b] - seqlens_q[b]).  Padding rows (i >= seqlens_q[b]) of o and
 * lse are not written, except when Sk_max == 0, where every row gets o = 0
 * and lse = -inf.  The work list is built for Sq_max; units past a batch's
 * length finish at once ("FlashAttention-2" notes, sequence-length
 * parallelism; the variable-length decode input of the onnxruntime WebGPU
 * page, section 1, applied to the forward pass).
 */
attn_status_t attn_fwd_varlen(const void* q, const void* k, const void* v, const int* seqlens_q,
                              const int* seqlens_k, void* o, float* lse, int B, int Hq, int Hkv, int Sq_max,
                              int Sk_max, int d, float scale, int causal, void* stream);

/*
 * Number of KV splits attn_decode_splitkv uses for this shape when called
 * with num_splits = 0 (picked to fill the device's SMs).  Needs the current
 * device's SM count; without a device it assumes 148.  Returns 0 for an
 * invalid shape.
 */
int attn_decode_num_splits(int B, int Hq, int Hkv, int Sq, int Sk, int d);

/*
 * Bytes of workspace attn_decode_splitkv needs: B*Hq*Sq*splits fp32 partial
 * output rows of d values plus as many fp32 (max, sum) pairs, with `splits`
 * the effective split count for num_splits (0 = automatic).
 * Returns 0 for an invalid shape.
 */
size_t attn_decode_workspace_size(int B, int Hq, int Hkv, int Sq, int Sk, int d, int num_splits);

/*
 * Split-KV decode ("[onnxruntime] WebGPU FlashAttention: kernel fusion and
 * variable sequence length", section 1): the keys of each (b, kv head) are
 * cut into splits of whole 64-key tiles; one kernel computes, per split, the
 * locally normalised partial output and its (local max, local sum); a
 * second kernel combines the splits by log-sum-exp rescaling into o and lse.
 * The result equals attn_fwd on the same inputs up to rounding.
 *   k_cache, v_cache  [B, Hkv, Sk, d] bf16 (every position valid)
 *   causal            ATTN_CAUSAL_NONE or ATTN_CAUSAL_BOTTOM_RIGHT (rows at
 *                     the end of the cache) or ATTN_CAUSAL_TOP_LEFT
 *   num_splits        0 = automatic; otherwise the requested count, rounded
 *                     to whole 64-key tiles (never more than ceil(Sk/64))
 *   workspace         device buffer of at least
 *                     attn_decode_workspace_size(...) bytes, 16-byte aligned;
 *                     owned by the caller, overwritten by the call.
 * Each CTA serves the G*Sq <= 16 query rows of one KV head at a time (G =
 * Hq/Hkv); larger G*Sq is handled in groups of 16 rows.
 */
attn_status_t attn_decode_splitkv(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                                  int B, int Hq, int Hkv, int Sq, int Sk, int d, float scale, int causal,
                                  int num_splits, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Split-KV decode over a KV cache whose valid length differs per batch and
 * lives in device memory ("[onnxruntime] WebGPU FlashAttention: kernel fusion
 * and variable sequence length", section 1: the decode reads seqlen_k on the
 * GPU, and the launch size must not depend on a host copy of it, or the two
 * race).
 *   k_cache, v_cache  [B, Hkv, Sk_capacity, d] bf16; for batch b only keys
 *                     0 .. seqlens_k[b]-1 are read as keys (the rest of the
 *                     capacity may hold anything)
 *   seqlens_k         device int32 [B], 4-byte aligned; read by the kernels
 *                     only, so it may be written by earlier work on `stream`
 *                     (no host synchronisation is needed or performed).  A
 *                     value outside [0, Sk_capacity] is clamped and makes
 *                     attn_check_device_error() return ATTN_ERR_SEQLEN.
 *   causal            as for attn_decode_splitkv, aligned to each batch's own
 *                     length: with ATTN_CAUSAL_BOTTOM_RIGHT query row i of
 *                     batch b sees key j iff j <= i + seqlens_k[b] - Sq.
 * The grid, the split count and the workspace size depend only on
 * Sk_capacity (attn_decode_workspace_size(B, Hq, Hkv, Sq, Sk_capacity, d,
 * num_splits)).  With more than one split and at most 128 batches, the
 * B * splits CTAs of each kv head are dealt on the device to the batches in
 * proportion to their valid 64-key tiles (every batch gets at least one; the
 * per-CTA tile count is the smallest that lets the deal fit), so a mix of
 * long and short caches keeps the CTAs' work about equal; otherwise each
 * batch's valid tiles are spread evenly over its own splits.
 * A batch with length 0 (or a row that sees no key) gets o = 0 and
 * lse = -inf.  Everything else is as for attn_decode_splitkv.
 */
attn_status_t attn_decode_splitkv_varlen(const void* q, const void* k_cache, const void* v_cache,
                                         const int* seqlens_k, void* o, float* lse, int B, int Hq, int Hkv, int Sq,
                                         int Sk_capacity, int d, float scale, int causal, int num_splits,
                                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_decode_splitkv with the optional inputs of attn_extras_t (per-batch
 * key lengths, additive bias; `extras` may be NULL).  An invalid extras field
 * returns ATTN_ERR_SHAPE (bias dims, or seqlens_q given) or ATTN_ERR_ALIGN.
 */
attn_status_t attn_decode_splitkv_ex(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                                     int B, int Hq, int Hkv, int Sq, int Sk, int d, float scale, int causal,
                                     int num_splits, void* workspace, size_t workspace_bytes,
                                     const attn_extras_t* extras, void* stream);

/*
 * Split-KV decode that allocates nothing and takes no workspace -- for callers
 * that cannot obtain device memory themselves: a plug-in whose host framework
 * owns every device allocation and hands none out, or a service that fixes its
 * memory budget at start-up and may not allocate afterwards.  Such callers
 * cannot provide the workspace attn_decode_splitkv needs.  The pages have no
 * counterpart to this entry point; it exists only for such callers.
 *
 * Same arguments, semantics and result as attn_decode_splitkv minus the
 * workspace: the partial outputs go to a scratch array that the library keeps
 * in device memory for the life of the process, ATTN_STATIC_SCRATCH_BYTES
 * (16 MiB) on every GPU that loads the library.  A problem whose workspace
 * (attn_decode_workspace_size for the same arguments) exceeds that size is
 * rejected with ATTN_ERR_SCRATCH_LIMIT before anything is launched.
 *
 * The first call on each device looks up the scratch array's device address
 * (once per device, with that device current); make that first call before
 * any stream capture.  The address is kept for the life of the process, so a
 * caller that resets a device (cudaDeviceReset) must not use this entry point
 * on it afterwards.  On a device that is not a B200 the call returns
 * ATTN_ERR_ARCH before it looks anything up.  The scratch is shared by every call on a device and
 * keeps the last call's contents; nothing in it needs to start at zero (each
 * call writes every partial it later reads).  Calls that may overlap on the
 * GPU (different streams without ordering between them) race on the scratch:
 * order them, e.g. issue them on one stream.
 */
#define ATTN_STATIC_SCRATCH_BYTES ((size_t)16 << 20)
attn_status_t attn_decode_splitkv_static(const void* q, const void* k_cache, const void* v_cache, void* o,
                                         float* lse, int B, int Hq, int Hkv, int Sq, int Sk, int d, float scale,
                                         int causal, int num_splits, void* stream);

/*
 * Backward pass of attn_fwd: gradients dq, dk, dv of a loss L given
 * dout = dL/do.  "FlashAttention-2" notes report the backward pass's speed
 * but give no algorithm; this library's kernels recompute the probabilities
 * P = exp(scale q.k - lse) tile by tile from the forward's lse (nothing of
 * size Sq x Sk is stored) and apply the chain rule through the forward:
 *   dP = dout v^T,  D_i = dout_i . o_i,  dS = P (dP - D),
 *   dq = scale dS k,  dk = scale dS^T q,  dv = P^T dout,
 * with dk and dv of a KV head summed over the query heads that share it (GQA).
 *
 *   q, o, dout, dq   [B, Hq, Sq, d] bf16 (BHSD), device
 *   k, v, dk, dv     [B, Hkv, Sk, d] bf16, device
 *   lse              [B, Hq, Sq] fp32: the forward's lse (natural log) for the
 *                    same q, k, v, scale and causal mode; o is its output.
 *   workspace        attn_bwd_workspace_size(B, Hq, Sq) bytes, device,
 *                    16-byte aligned, caller-owned; nothing in it needs to be
 *                    initialised.
 * scale and causal as in attn_fwd (causal 0, 1 or 2).  Every output is fully
 * written: rows that saw no key get dq = 0; keys no row sees get dk = dv = 0;
 * Sq == 0 gives dk = dv = 0, Sk == 0 gives dq = 0.  Errors as attn_fwd, plus
 * ATTN_ERR_WORKSPACE.  Three kernels on `stream`, asynchronous.
 */
size_t attn_bwd_workspace_size(int B, int Hq, int Sq);
attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                       const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq, int Sk, int d,
                       float scale, int causal, void* workspace, size_t workspace_bytes, void* stream);

/*
 * The step before a decode: split a packed QKV projection, rotate q and k by
 * the rotary embedding, append k and v to the KV cache -- one streaming kernel.
 * This is the fused "split packed QKV with rotary embedding and copy KV" step
 * of "[onnxruntime] WebGPU FlashAttention: kernel fusion and variable sequence
 * length" (section 2).  The page names the step but gives no formula; this
 * library takes the non-interleaved rotary embedding: for position p and
 * i < d/2 the pair (x_i, x_{i+d/2}) becomes
 *   (x_i cos[p][i] - x_{i+d/2} sin[p][i],  x_{i+d/2} cos[p][i] + x_i sin[p][i]),
 * computed in fp32 and rounded once to bf16.  Token t of batch b sits at the
 * absolute position p = past_lens[b] + t.
 *
 *   packed_qkv  [B, S_new, (Hq + 2*Hkv) * d] bf16, device; each token's row
 *               holds Hq q heads, then Hkv k heads, then Hkv v heads, d each.
 *   cos_table,
 *   sin_table   [max_pos, d/2] fp32, device (the caller picks the frequencies).
 *   past_lens   [B] int32, device: tokens already in the cache per batch.
 *   q_out       rotated q, [B, Hq, S_new, d] bf16 (layout BSHD: [B, S_new, Hq, d]).
 *   k_cache,
 *   v_cache     [B, Hkv, cap, d] bf16 (layout BSHD: [B, cap, Hkv, d]), device,
 *               updated in place: rows past_lens[b] .. past_lens[b] + S_new - 1
 *               receive the rotated k and the unchanged v; no other row is touched.
 *   total_lens  [B] int32, device, or NULL: receives past_lens[b] + S_new, the
 *               key lengths for attn_decode_splitkv_varlen over the updated cache
 *               (saturated at INT_MAX).  It may be past_lens itself (lengths
 *               advanced in place): every token's position is then taken from
 *               the old lengths, and the new ones are written by a second
 *               kernel ordered after the append on `stream`.
 *   layout      ATTN_LAYOUT_BHSD or ATTN_LAYOUT_BSHD, for q_out and both caches.
 *
 * All buffers are the caller's; the library allocates nothing.  Pointers must
 * be 16-byte aligned (past_lens, total_lens: 4 bytes).  Host-side errors:
 * ATTN_ERR_SHAPE (negative size, cap or max_pos < 1, unknown layout),
 * ATTN_ERR_GQA, ATTN_ERR_HEADDIM (d not 64 or 128), ATTN_ERR_NULL,
 * ATTN_ERR_ALIGN.  B == 0 or S_new == 0 writes only total_lens.  A token whose
 * position falls outside [0, min(cap, max_pos)) is skipped (nothing of its row
 * is written) and attn_check_device_error() then returns ATTN_ERR_SEQLEN.
 * Asynchronous on `stream`.
 */
attn_status_t attn_rope_append(const void* packed_qkv, const float* cos_table, const float* sin_table, int max_pos,
                               const int* past_lens, void* q_out, void* k_cache, void* v_cache, int* total_lens,
                               int B, int S_new, int Hq, int Hkv, int cap, int d, int layout, void* stream);

/*
 * Self-test of the bounded-wait contract above (not a computation): runs the
 * split-KV decode of attn_decode_splitkv (bottom-right mask, default scale,
 * automatic split count) with its K/V copies withheld, so every consumer
 * wait in the split kernel gives up after its 1 s limit and the kernel exits
 * through its timeout path -- no trap, no copy in flight, no tensor memory
 * held.  The next attn_check_device_error(stream) must then return
 * ATTN_ERR_DEVICE_TIMEOUT, and the context stays usable.  o and lse receive
 * meaningless values.  Arguments as for attn_decode_splitkv (B, Sq and Sk
 * must be > 0); takes about one second of GPU time.
 */
attn_status_t attn_selftest_decode_wait_timeout(const void* q, const void* k_cache, const void* v_cache, void* o,
                                                float* lse, int B, int Hq, int Hkv, int Sq, int Sk, int d,
                                                void* workspace, size_t workspace_bytes, void* stream);

/* A static, human-readable name for a status code. */
const char* attn_status_string(attn_status_t status);

/*
 * Synchronizes `stream`, then reads and clears the device error word.
 * Returns ATTN_ERR_DEVICE_TIMEOUT if a kernel gave up on a bounded wait since
 * the last check, else ATTN_ERR_SEQLEN if attn_fwd_varlen or
 * attn_decode_splitkv_varlen had to clamp a per-batch length or
 * attn_rope_append skipped a token, ATTN_ERR_CUDA
 * if the synchronization itself failed, else ATTN_OK.
 */
attn_status_t attn_check_device_error(void* stream);

/* Library version as major*10000 + minor*100 + patch. */
int attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SDPA_B200_H */
