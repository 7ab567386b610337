/*
 * fa.h -- C ABI of the io_aware_online_b200 attention library (NVIDIA B200, sm_100a).
 *
 * Exact, IO-aware attention forward: O = softmax(mask(softcap(scale*Q*K^T) + ALiBi)) * V
 * with the per-row log-sum-exp, computed by streaming K/V tiles through on-chip
 * memory with online-softmax rescaling, so that the score matrix never reaches
 * HBM (tag page "flash attention" (xhh.club): tiling plus online softmax, no
 * materialised score matrix).  The argument set follows the problem statement
 * of "FlashAttention common interfaces" (xllm-io blog), sections 3.1-3.4.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Memory: every tensor argument is a DEVICE pointer owned by the caller.  The
 *   library allocates no memory on any call; scratch (the split-KV workspace)
 *   is passed in.  Pointers of 16-bit tensors must be 16-byte aligned.
 * - Execution: every call is asynchronous and stream-ordered on `stream` (a
 *   cudaStream_t; NULL = the legacy default stream).  A nonzero return means
 *   nothing was launched.
 * - Dtypes: FA_FP16 or FA_BF16 for Q, K, V and O (one dtype per call); LSE,
 *   ALiBi slopes and split partials are fp32.  fp32 inputs are not supported
 *   (the pages: fp16/bf16 only).  fa_fwd_fp8 takes E4M3 Q, K, V and writes bf16.
 * - Head dim: 64 or 128.
 * - softmax_scale: a NaN means the default 1/sqrt(head_dim) (section 3.1);
 *   otherwise it must be finite and >= 0.
 * - Masks: the causal mask is aligned bottom-right (changelog post, v2.1): query
 *   row i of a sequence with Sq queries and Sk keys sees key j iff
 *   j <= i + Sk - Sq.  window_size = (left, right), -1 meaning unbounded
 *   (section 3.1): key j is inside iff i + Sk - Sq - left <= j <= i + Sk - Sq + right.
 *   With causal set, the causal bound limits the right side.  A row with no
 *   allowed key gets O = 0 and LSE = -inf.
 * - softcap > 0 replaces each scaled score s by softcap * tanh(s / softcap)
 *   (changelog v2.6, section 5.2); 0 disables it.
 * - alibi_slopes: NULL or fp32 [num_heads]; head h subtracts
 *   slope[h] * |i + Sk - Sq - j| from its scores (changelog v2.4, section 5.1).
 * - GQA/MQA: num_heads must be a multiple of num_heads_k; query head h reads
 *   K/V head h / (num_heads / num_heads_k) (section 4.2).
 * - Errors: functions return FA_OK (0) or an FA_ERR_* code; fa_last_error()
 *   gives a message for the calling thread.  Faults the kernels detect on the
 *   device (a block_table entry outside the pool, a pipeline wait that ran out
 *   of time) set bits of a device status word, read by fa_device_status().
 */
#ifndef IO_AWARE_ONLINE_FA_H
#define IO_AWARE_ONLINE_FA_H

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

enum fa_status {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,  /* null pointer, bad shape/stride/alignment, bad flag value */
    FA_ERR_UNSUPPORTED = 2,  /* head_dim not in {64,128}, dtype not fp16/bf16, too many rows */
    FA_ERR_WORKSPACE = 3,    /* workspace missing or smaller than fa_kvcache_workspace_size() */
    FA_ERR_CUDA = 4,         /* a CUDA runtime/driver call or kernel launch failed */
    FA_ERR_DEVICE = 5        /* fa_device_status(): the device reported a fault */
};

enum fa_dtype { FA_FP16 = 0, FA_BF16 = 1, FA_FP32 = 2 /* fa_combine output only */ };

/* Device status bits (fa_device_status). */
enum fa_device_flag {
    FA_DEV_WAIT_TIMEOUT = 1u,   /* a pipeline wait exceeded its time limit; that CTA stopped */
    FA_DEV_BAD_BLOCK = 2u,      /* a block_table entry was outside [0, num_blocks) */
    FA_DEV_BAD_LENGTH = 4u,     /* a cache length (cache_seqlens[b], plus appended keys)
                                   was negative or beyond the cache's capacity; the
                                   kernel clamped it (attention) or skipped the row
                                   (append) */
    FA_DEV_SMEM_ALIGN = 8u      /* fa_bwd: the dynamic shared memory did not start on a
                                   1 KiB boundary, which the dK/dV kernel's layout needs;
                                   that kernel did nothing and dK, dV are undefined */
};

/*
 * fa_fwd -- dense or variable-length attention forward
 * (section 3.1 flash_attn_func, section 3.2 flash_attn_varlen_func).
 *
 * Dense (cu_seqlens_q == cu_seqlens_k == NULL):
 *   q [batch, seqlen_q, num_heads, head_dim], k/v [batch, seqlen_k, num_heads_k, head_dim],
 *   out like q, lse fp32 [batch, num_heads, seqlen_q] (contiguous).
 * Varlen (both cu_seqlens non-NULL, device int32 [batch + 1], nondecreasing, starting at 0):
 *   q [total_q, num_heads, head_dim], k/v [total_k, num_heads_k, head_dim], out like q,
 *   lse fp32 [num_heads, total_q].  seqlen_q / seqlen_k are then total_q / total_k
 *   (the packed row counts, cu_seqlens_q[batch] and cu_seqlens_k[batch]) and
 *   max_seqlen_q / max_seqlen_k bound every sequence's length.  Sequence b owns
 *   rows cu_seqlens[b] .. cu_seqlens[b+1]-1; its mask offset is
 *   (its key count) - (its query count).
 * Strides: q_strides, k_strides, v_strides, o_strides are int64 [3] element strides
 *   for (batch, seq, head); the head_dim axis must be contiguous.  NULL means the
 *   contiguous layout above.  In varlen mode entry 0 is ignored.  Every stride must
 *   be a multiple of 8 elements (16 bytes) and every pointer 16-byte aligned.
 * lse may be NULL.  The N x N score matrix is never written to memory.
 * Errors: argument errors return FA_ERR_* before anything is launched.  A
 * pipeline wait inside the kernel that runs past its limit (fa_set_wait_timeout_ms)
 * stops that CTA and raises FA_DEV_WAIT_TIMEOUT in the device status word
 * (fa_device_status); out and lse of a call after which that bit is set are
 * undefined: the stopped CTA's rows may hold partial results or stale memory.
 */
FA_API int fa_fwd(const void *q, const void *k, const void *v, void *out, float *lse, int dtype,
           int batch, int seqlen_q, int seqlen_k, int num_heads, int num_heads_k, int head_dim,
           const int64_t *q_strides, const int64_t *k_strides, const int64_t *v_strides,
           const int64_t *o_strides, const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
           int max_seqlen_q, int max_seqlen_k, float softmax_scale, int causal, int window_left,
           int window_right, float softcap, const float *alibi_slopes, void *stream);

/*
 * fa_fwd_host -- fa_fwd (dense, section 3.1 flash_attn_func) on operands in host
 * memory, with the transfers overlapped with the kernels.
 *
 *   q [batch, seqlen_q, num_heads, head_dim], k/v [batch, seqlen_k, num_heads_k,
 *   head_dim], out like q: contiguous, fp16 or bf16 (dtype), in host memory;
 *   lse fp32 [batch, num_heads, seqlen_q] in host memory, or NULL; alibi_slopes
 *   fp32 [num_heads] in host memory, or NULL.  Page-locked memory (cudaHostAlloc,
 *   cudaHostRegister) lets the copies run asynchronously and overlap; pageable
 *   memory works but each copy then waits on the host.
 *   workspace: device memory, 256-byte aligned, at least
 *   fa_fwd_host_workspace_size(batch, seqlen_q, seqlen_k, num_heads, num_heads_k,
 *   head_dim, lse != NULL) bytes; owned by the caller, who keeps it (and the host
 *   buffers) alive until `stream` has passed the call.
 * The batch is cut into at most four chunks of whole sequences that pass through
 * two workspace slots: chunk c+1 is copied in and chunk c-1 copied out while chunk c
 * is computed, on three streams of the library that start after the work already
 * on `stream` and that `stream` waits for at the end of the call.  Results are
 * bit-identical to fa_fwd over the whole batch.  Masks, scale and softcap as for
 * fa_fwd (varlen, strides and FP8 are not offered here).
 * Errors: argument and workspace errors return FA_ERR_* before anything is enqueued;
 * an error from a later step returns after `stream` has been made to wait for what
 * was enqueued, and out / lse are then undefined.  Calls from several host threads
 * are serialised while they enqueue; the streams are created on a device's first
 * call and kept for the life of the process (not valid after a device reset).
 */
FA_API size_t fa_fwd_host_workspace_size(int batch, int seqlen_q, int seqlen_k, int num_heads,
                                         int num_heads_k, int head_dim, int with_lse);
FA_API int fa_fwd_host(const void *q, const void *k, const void *v, void *out, float *lse,
                       int dtype, int batch, int seqlen_q, int seqlen_k, int num_heads,
                       int num_heads_k, int head_dim, float softmax_scale, int causal,
                       int window_left, int window_right, float softcap,
                       const float *alibi_slopes, void *workspace, size_t workspace_bytes,
                       void *stream);

/*
 * fa_fwd_fp8 -- fa_fwd with 8-bit inputs (the "FlashAttention common interfaces"
 * page's workflow three: q, k and v cast to float8 E4M3 and passed to the same
 * call; FlashAttention-3's FP8 path on the tag page).
 *
 *   q, k, v: E4M3 bytes, layouts and strides (in elements, multiples of 16) as for
 *   fa_fwd; head_dim must be 128.  out: bf16, layout as for fa_fwd (strides in
 *   elements, multiples of 8).  lse: fp32 as for fa_fwd, or NULL.
 *   q_descale, k_descale, v_descale: finite, > 0 (1 for a plain cast): the real
 *   inputs are q * q_descale etc.; the scores use softmax_scale * q_descale *
 *   k_descale and O is multiplied by v_descale.
 * Both products run on the tensor cores with 8-bit operands (tcgen05.mma
 * kind::f8f6f4), so P is rounded to E4M3 before P.V: each probability carries a
 * relative error of at most 2^-4, and O differs from exact attention on the
 * dequantised inputs by at most 2^-4 * sum_j w_ij |v_j| per element (w the exact
 * attention weights) plus n_k * 2^-18 * max_j |v_j| (probabilities below 2^-14 of
 * the row's largest can fall in E4M3's subnormal range), plus the bf16 rounding of O.
 * The LSE comes from the exact fp32 sum.  Other arguments, masks and errors as for
 * fa_fwd.
 */
FA_API int fa_fwd_fp8(const void *q, const void *k, const void *v, void *out, float *lse,
                      float q_descale, float k_descale, float v_descale, int batch,
                      int seqlen_q, int seqlen_k, int num_heads, int num_heads_k, int head_dim,
                      const int64_t *q_strides, const int64_t *k_strides,
                      const int64_t *v_strides, const int64_t *o_strides,
                      const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                      int max_seqlen_q, int max_seqlen_k, float softmax_scale, int causal,
                      int window_left, int window_right, float softcap,
                      const float *alibi_slopes, void *stream);

/*
 * fa_kvcache_num_splits -- the split count fa_fwd_kvcache uses for these sizes.
 * num_splits in 1..256 is returned unchanged apart from a clamp to the number of
 * cache pages; 0 asks for the library's heuristic, which depends only on the
 * arguments and on the current device's SM count.  max_seqlen_k is the largest
 * cache length (max_blocks_per_seq * page_size for a paged cache).  Returns <= 0
 * on bad input, including num_splits < 0 or > 256.
 */
FA_API int fa_kvcache_num_splits(int batch, int seqlen_q, int num_heads, int num_heads_k,
                          int head_dim, int max_seqlen_k, int page_size, int num_splits);

/*
 * fa_kvcache_workspace_size -- bytes of device scratch fa_fwd_kvcache needs:
 * 256 (a work-item counter the call resets) plus, when the resolved split count is
 * above 1, splits * batch * seqlen_q * num_heads * (head_dim + 1) * 4 for the fp32
 * split partials.  Same arguments as fa_kvcache_num_splits (which returns 1 when
 * the call runs the tensor-core kernel: more than 16 query rows per KV head).
 */
FA_API size_t fa_kvcache_workspace_size(int batch, int seqlen_q, int num_heads, int num_heads_k,
                                 int head_dim, int max_seqlen_k, int page_size,
                                 int num_splits);

/*
 * fa_fwd_kvcache -- attention of a few new query rows against a KV cache,
 * split along the keys (changelog v2.2 split-KV "flash-decoding"; v2.5 paged KV
 * cache; section 3.3 flash_attn_with_kvcache; the in-place append of new keys is
 * fa_fwd_kvcache_append).
 *
 *   q   [batch, seqlen_q, num_heads, head_dim] contiguous; out like q;
 *   lse fp32 [batch, num_heads, seqlen_q] or NULL.
 * Paged cache (block_table != NULL): k_cache/v_cache are pools
 *   [num_blocks, page_size, num_heads_k, head_dim] contiguous; block_table is
 *   int32 [batch, max_blocks_per_seq]; entry p of sequence b names the pool block
 *   holding its keys p*page_size .. p*page_size + page_size - 1.  page_size must be
 *   a multiple of 64.  Entries past a sequence's last page are never read.
 * Contiguous cache (block_table == NULL): k_cache/v_cache are
 *   [batch, seqlen_k_max, num_heads_k, head_dim] contiguous.
 * cache_seqlens: int32 [batch], the number of keys sequence b attends (its query
 *   rows sit at key positions cache_seqlens[b] - seqlen_q ..).  NULL means
 *   seqlen_k_max for every sequence (contiguous cache only).
 * num_splits: 0 = heuristic; 1..256 (larger counts return FA_ERR_INVALID_ARG:
 *   the combine step weighs at most 256 partials); otherwise the keys of each sequence are cut, at
 *   page granularity (64-token chunks for a contiguous cache), into num_splits
 *   ranges of ceil(pages / num_splits) pages, each computed by its own CTAs, and a
 *   second kernel combines them (fa_combine's arithmetic).  The result does not
 *   depend on num_splits beyond rounding.
 * workspace: device scratch of at least fa_kvcache_workspace_size(...) bytes,
 *   16-byte aligned, required.  It holds the split kernel's work-item counter and
 *   the longest-first order of the sequences (both written by a small kernel the
 *   call launches on `stream` first; the split kernel claims the items of the
 *   longest sequences first) and the fp32 split partials between the kernels of one
 *   call, so calls that share a workspace must be stream-ordered.
 * Up to 16 query rows per KV head ((num_heads / num_heads_k) * seqlen_q) the call
 *   runs the split-KV decode kernel above.  With more (chunked prefill against the
 *   cache: a chunk of new query rows attends everything cached, causal aligned
 *   bottom-right) it runs the tcgen05 prefill kernel of fa_fwd with K/V read from
 *   the cache, one CTA per 256 query rows; num_splits is then ignored.  Keys past
 *   a sequence's length (page tails, unused blocks) are never loaded or are
 *   cleared before use, so their contents cannot reach the output either way.
 */
FA_API int fa_fwd_kvcache(const void *q, const void *k_cache, const void *v_cache, void *out, float *lse,
                   int dtype, int batch, int seqlen_q, int num_heads, int num_heads_k,
                   int head_dim, const int32_t *block_table, int max_blocks_per_seq,
                   int page_size, int num_blocks, int seqlen_k_max,
                   const int32_t *cache_seqlens, float softmax_scale, int causal,
                   int window_left, int window_right, float softcap,
                   const float *alibi_slopes, int num_splits, void *workspace,
                   size_t workspace_bytes, void *stream);

/*
 * fa_kvcache_append -- write new keys and values into a KV cache in place, at the
 * positions after each sequence's cached keys (section 3.3: flash_attn_with_kvcache
 * with k and v given "updates the cache").
 *
 *   k_new, v_new [batch, seqlen_new, num_heads_k, head_dim] contiguous, 16-bit
 *   (dtype as for fa_fwd).  Row t of sequence b goes to key position
 *   cache_seqlens[b] + t of that sequence: cache_seqlens is the number of keys
 *   ALREADY in the cache, before this append (the parameter's description on
 *   the page; its worked example's 128-then-129 values read as lengths after the
 *   append and are not followed).  cache_seqlens is required and is not updated:
 *   the caller advances it by seqlen_new for the next step.
 * Paged cache (block_table != NULL): position x of sequence b is row x % page_size
 *   of pool block block_table[b, x / page_size]; the cache layout and arguments are
 *   those of fa_fwd_kvcache.  Contiguous cache (block_table == NULL): row x of
 *   sequence b of k_cache [batch, seqlen_k_max, num_heads_k, head_dim].
 * A position outside the cache's capacity (max_blocks_per_seq * page_size or
 *   seqlen_k_max) or a block_table entry outside [0, num_blocks) is not written;
 *   the kernel raises FA_DEV_BAD_LENGTH or FA_DEV_BAD_BLOCK (fa_device_status).
 * Writes nothing else.  Asynchronous on `stream`; allocates nothing.
 */
FA_API int fa_kvcache_append(void *k_cache, void *v_cache, const void *k_new, const void *v_new,
                             int dtype, int batch, int seqlen_new, int num_heads_k, int head_dim,
                             const int32_t *block_table, int max_blocks_per_seq, int page_size,
                             int num_blocks, int seqlen_k_max, const int32_t *cache_seqlens,
                             void *stream);

/*
 * fa_fwd_kvcache_append -- fa_kvcache_append followed, on the same stream, by
 * fa_fwd_kvcache over the grown cache (section 3.3 with k and v given): sequence
 * b then attends its cache_seqlens[b] + seqlen_new keys, and with causal the
 * query rows sit at the last seqlen_q of those positions (bottom-right).  The
 * arguments are those of fa_fwd_kvcache (cache_seqlens still counts the keys
 * before the append and is required) plus k_new, v_new and seqlen_new as for
 * fa_kvcache_append; the workspace rule is fa_fwd_kvcache's.
 */
FA_API int fa_fwd_kvcache_append(const void *q, void *k_cache, void *v_cache, const void *k_new,
                                 const void *v_new, int seqlen_new, void *out, float *lse,
                                 int dtype, int batch, int seqlen_q, int num_heads,
                                 int num_heads_k, int head_dim, const int32_t *block_table,
                                 int max_blocks_per_seq, int page_size, int num_blocks,
                                 int seqlen_k_max, const int32_t *cache_seqlens,
                                 float softmax_scale, int causal, int window_left,
                                 int window_right, float softcap, const float *alibi_slopes,
                                 int num_splits, void *workspace, size_t workspace_bytes,
                                 void *stream);

/*
 * fa_bwd_workspace_size -- bytes of device scratch fa_bwd needs: two fp32 arrays
 * (D = rowsum(dO * O) and LSE * log2 e) of batch * num_heads rows of seqlen_q
 * rounded up to 4 values, the total rounded up to 256 bytes.
 */
FA_API size_t fa_bwd_workspace_size(int batch, int seqlen_q, int num_heads);

/*
 * fa_bwd -- gradients of the attention forward (tag page "flash attention": the
 * backward recomputes the attention matrix tile by tile from Q, K and the
 * forward's softmax statistics instead of reading a stored one).
 *
 * Dense (cu_seqlens_q == cu_seqlens_k == NULL):
 *   dout, q, out, dq: [batch, seqlen_q, num_heads, head_dim] contiguous, 16-bit
 *   (dtype as for fa_fwd); k, v, dk, dv: [batch, seqlen_k, num_heads_k, head_dim]
 *   contiguous; lse: fp32 [batch, num_heads, seqlen_q], the forward's LSE.
 * Varlen (both cu_seqlens non-NULL, device int32 [batch + 1] as for fa_fwd,
 *   section 3.2): the same tensors packed along the rows, [total_q, num_heads,
 *   head_dim] and [total_k, num_heads_k, head_dim] with seqlen_q / seqlen_k the
 *   packed totals; lse fp32 [num_heads, total_q] (fa_fwd's varlen layout);
 *   max_seqlen_q / max_seqlen_k bound every sequence's lengths.  Each sequence
 *   is its own problem, its mask aligned bottom-right within it.
 * out: the forward's O.  The mask, scale, window, softcap and ALiBi arguments
 * must be those of the forward call.
 * Computes, with X = scale Q K^T, T = tanh(X / softcap) and S = softcap T
 * (S = X without a softcap; changelog v2.6, section 5.2), P = exp(S + bias - LSE)
 * on the allowed entries and D = rowsum(dout * out): dv = P^T dout,
 * dS = P * (dout v^T - D), dX = dS * (1 - T^2) (dX = dS without a softcap),
 * dq = scale dX k, dk = scale dX^T q; dk and dv sum over the query heads that
 * share a KV head.  Deterministic (no atomics): one pass per key block for dk/dv,
 * one per query block for dq.  P and dX are rounded to the input dtype before
 * their products (fp32 accumulation).
 * workspace: >= fa_bwd_workspace_size(batch, seqlen_q, num_heads) bytes (varlen:
 *   fa_bwd_workspace_size(1, total_q, num_heads)), 16-byte aligned; calls sharing
 *   it must be stream-ordered.
 */
FA_API int fa_bwd(const void *dout, const void *q, const void *k, const void *v,
                  const void *out, const float *lse, void *dq, void *dk, void *dv, int dtype,
                  int batch, int seqlen_q, int seqlen_k, int num_heads, int num_heads_k,
                  int head_dim, const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                  int max_seqlen_q, int max_seqlen_k, float softmax_scale, int causal,
                  int window_left, int window_right, float softcap, const float *alibi_slopes,
                  void *workspace, size_t workspace_bytes, void *stream);

/*
 * fa_selftest_wait_timeout -- a diagnostic of the bounded waits (the pages have no
 * counterpart): launches one CTA that waits, through the library's bounded wait, on
 * a barrier phase nothing ever completes.  After timeout_ms (1..10000) of GPU time
 * the wait gives up and raises FA_DEV_WAIT_TIMEOUT in the device status word, as a
 * stalled pipeline wait of any kernel here would; read it with fa_device_status
 * after synchronising `stream`.  The context stays usable.  Returns FA_OK once
 * launched, FA_ERR_INVALID_ARG for a limit out of range.
 */
FA_API int fa_selftest_wait_timeout(int timeout_ms, void *stream);

/*
 * fa_fwd_kvcache_static -- fa_fwd_kvcache without a workspace argument, for callers
 * that cannot allocate device memory where they run attention (a host framework
 * that owns every device allocation through its own pool, or a serving loop that
 * must not risk the device synchronisation a cudaMalloc can cause).  The pages
 * have no counterpart to this call.  It allocates nothing: its scratch (the
 * work-item counter and the fp32 split partials) is one fixed 24 MiB array in
 * device memory (fa_kvcache_static_scratch_bytes()), present on every GPU that
 * loads the library until the process exits; it holds, for example, the partials
 * of a 64-sequence, 32-head, head-dim-128 single-token decode at up to 23 splits.  Arguments and results are those of
 * fa_fwd_kvcache.  A call whose need (fa_kvcache_workspace_size) exceeds the array
 * returns FA_ERR_WORKSPACE without launching anything.  All calls share the array
 * and it keeps the last call's contents; each call clears the counter on its own
 * stream, so calls that overlap on the GPU race and must be serialised by the
 * caller.  The first call on a device looks the array's address up
 * (cudaGetSymbolAddress) with that device current; make it before any stream
 * capture.  The address stays cached for the life of the process, so after a
 * device reset (cudaDeviceReset, or the primary context released and created
 * again) this call must not be used any more.
 */
FA_API int fa_fwd_kvcache_static(const void *q, const void *k_cache, const void *v_cache,
                                 void *out, float *lse, int dtype, int batch, int seqlen_q,
                                 int num_heads, int num_heads_k, int head_dim,
                                 const int32_t *block_table, int max_blocks_per_seq,
                                 int page_size, int num_blocks, int seqlen_k_max,
                                 const int32_t *cache_seqlens, float softmax_scale, int causal,
                                 int window_left, int window_right, float softcap,
                                 const float *alibi_slopes, int num_splits, void *stream);

/* Size in bytes of the fixed scratch array behind fa_fwd_kvcache_static. */
FA_API size_t fa_kvcache_static_scratch_bytes(void);

/*
 * fa_combine -- LSE-weighted combine of split partial results
 * (section 3.4 flash_attn_combine; changelog v2.2: "an extra kernel reduces").
 *   LSE = log sum_s exp(lse_s);  O = sum_s exp(lse_s - LSE) * O_s
 * out_partial fp32 with logical shape [batch, seqlen, num_heads, head_dim, num_splits]
 *   and element strides op_strides[5] (NULL = that shape, contiguous: the pages' layout);
 * lse_partial fp32 [batch, seqlen, num_heads, num_splits], strides lp_strides[4]
 *   (NULL = contiguous).  A split with lse_s = -inf contributes nothing (its O_s is
 *   not read as a factor); all -inf gives O = 0, LSE = -inf.
 * out [batch, seqlen, num_heads, head_dim] contiguous in out_dtype (FA_FP16, FA_BF16
 *   or FA_FP32); lse fp32 [batch, num_heads, seqlen] or NULL.
 * head_dim: any multiple of 4 up to 256 (inner loops are 16-byte vectors when the
 *   partials are contiguous along head_dim).  num_splits: 1 .. 256.
 */
FA_API int fa_combine(const float *out_partial, const float *lse_partial, void *out, float *lse,
               int out_dtype, int batch, int seqlen, int num_heads, int head_dim,
               int num_splits, const int64_t *op_strides, const int64_t *lp_strides,
               void *stream);

/* Message describing the last error returned on the calling thread ("" if none). */
FA_API const char *fa_last_error(void);

/*
 * fa_device_status -- synchronises the current device, then stores the OR of the
 * FA_DEV_* bits raised by kernels since the last clear into *flags (may be NULL).
 * clear != 0 resets them.  Returns FA_ERR_DEVICE if any bit was set, FA_OK if
 * none, FA_ERR_CUDA if the synchronisation itself failed.
 */
FA_API int fa_device_status(int clear, unsigned int *flags);

/*
 * fa_set_wait_timeout_ms -- time limit of every pipeline wait inside the kernels
 * (default 1000 ms, or the FA_WAIT_TIMEOUT_MS environment variable).  A wait that
 * runs out sets FA_DEV_WAIT_TIMEOUT, and its CTA drains its in-flight copies and
 * MMAs, frees its tensor memory and exits instead of hanging the GPU.  ms >= 1.
 */
FA_API int fa_set_wait_timeout_ms(int ms);

/* Library version: major * 10000 + minor * 100 + patch. */
FA_API int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* IO_AWARE_ONLINE_FA_H */
