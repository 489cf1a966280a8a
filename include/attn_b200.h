/*
 * attn_b200.h -- C ABI of libattn_b200.so: fused scaled-dot-product attention
 * forward with log-sum-exp output on NVIDIA B200 (sm_100a).
 *
 *   O   = softmax(scale * Q K^T + mask) V
 *   LSE = ln sum_{allowed j} exp(scale * q . k_j)        (natural log, scale included)
 *
 * Definition: the FlexAttention forward ("[FlexAttention] Enforce Q,K,V memory
 * layouts for fp8 flex attention", pytorch commit 7e16cb99, flex_attention
 * docstring: shapes (B,Hq,L,E) / (B,Hkv,S,E), default scale 1/sqrt(E),
 * enable_gqa) with the log-sum-exp output and possibly fully masked rows of its
 * lowering ("Cross Attention does not work on CPU and older GPUs", BLT issue 6:
 * OUTPUT_LOGSUMEXP True, ROWS_GUARANTEED_SAFE False).  Varlen batches, the paged
 * KV cache and grouped-query heads follow "[CUDA] PagedAttention: add SM<80
 * fp16 fallback via memory-efficient attention" (onnxruntime PR 28200,
 * Implementation steps 2-3: block_table walk, [total_tokens, num_heads,
 * head_size] packing addressed by cumulative sequence lengths); seqused_k
 * follows "Rope dim" (vllm-project/flash-attention PR 172, the varlen
 * arguments).  fp8 e4m3 operands follow the FlexAttention fp8 commit above
 * (float8_e4m3fn, both GEMMs in the query dtype).
 *
 * Conventions shared by every call:
 *  - Ownership: the caller owns every buffer.  All tensor pointers are DEVICE
 *    pointers (e.g. from torch); scalars are passed by value.  The library never
 *    allocates device memory per call, never synchronises the stream and never
 *    reads device data on the host: calls are asynchronous on `stream`.
 *  - Errors: argument errors are returned synchronously before anything is
 *    launched.  A launch failure (cudaGetLastError) returns ATTN_ERR_CUDA.
 *    No call prints, traps or aborts.
 *  - Device check: each call first checks (once per device, then cached) that
 *    the current device is compute capability 10.0 and that this library's
 *    kernel image loads on it (ATTN_ERR_NO_KERNEL_IMAGE otherwise) -- the
 *    check is made at call time, not deferred to the first launch.
 *  - softmax_scale <= 0 selects the default 1/sqrt(head_dim).
 *  - Element types: ATTN_BF16 tensors are bfloat16; ATTN_FP8_E4M3 tensors are
 *    float8_e4m3fn codes whose real values are code * descale, with the three
 *    descales given as DEVICE pointers to one fp32 each (no host sync).  The
 *    output O is always bfloat16; LSE is fp32.
 *  - Alignment: every tensor pointer and every row stride must be a multiple
 *    of 16 bytes (the TMA rule), otherwise ATTN_ERR_INVALID_ARG.
 *  - Supported: head_dim in {64, 128}; paged block_size == 16.  Anything else
 *    returns ATTN_ERR_UNSUPPORTED.  num_heads_q must be a multiple of
 *    num_heads_kv.
 *  - Masks: ATTN_MASK_CAUSAL allows key j for query i iff j <= i + (Lk - Lq)
 *    (bottom-right aligned; equal to q_idx >= kv_idx when Lq == Lk).
 *    ATTN_MASK_PATCH allows key j for query i iff start_i <= j < end_i, with the
 *    sequence-local interval [start_i, end_i) given per query.  A query with no
 *    allowed key gets O = 0 and LSE = -inf.
 *  - Sliding window and softcap (the "local window on/off" and "softcap 0/50"
 *    options of the parity matrix in "[CUDA] PagedAttention: add SM<80 fp16
 *    fallback via memory-efficient attention", Testing; nanochat's SSSL
 *    window pattern in "FA3 loader reports success on Blackwell (sm_120) then
 *    dies at first kernel launch"):
 *      window_left >= 0 keeps, for the causal mask only, the keys
 *        i' - window_left <= j <= i'   (i' = i + Lk - Lq, the row's diagonal);
 *        a negative window_left means no window; with another mask it
 *        returns ATTN_ERR_UNSUPPORTED.
 *      softcap > 0 replaces each scaled logit s = scale * q.k (for fp8 the
 *        dequantised one) by softcap * tanh(s / softcap) before the softmax
 *        and the LSE; 0 means none; negative or non-finite values return
 *        ATTN_ERR_INVALID_ARG.
 *  - Stream: `stream` is a cudaStream_t (NULL = legacy default stream).
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID_ARG = 1,        /* null/misaligned pointer, bad size or stride */
    ATTN_ERR_UNSUPPORTED = 2,        /* valid but not implemented (head_dim, block_size, ...) */
    ATTN_ERR_NO_KERNEL_IMAGE = 3,    /* device is not sm_100 or the image does not load */
    ATTN_ERR_TMA_ENCODE = 4,         /* cuTensorMapEncodeTiled rejected a descriptor */
    ATTN_ERR_WORKSPACE_TOO_SMALL = 5,
    ATTN_ERR_CUDA = 6,               /* a CUDA runtime call or a launch failed */
    ATTN_ERR_DEVICE_TIMEOUT = 7,     /* a kernel gave up on a bounded wait (see attn_device_error) */
    ATTN_ERR_SCRATCH_LIMIT = 8,      /* attn_decode_paged_noalloc: needs more than its fixed scratch */
    ATTN_ERR_DEVICE_RANGE = 9        /* a kernel met an out-of-range index (see attn_device_error) */
} attn_status_t;

typedef enum { ATTN_MASK_NONE = 0, ATTN_MASK_CAUSAL = 1, ATTN_MASK_PATCH = 2 } attn_mask_t;
typedef enum { ATTN_BF16 = 0, ATTN_FP8_E4M3 = 1 } attn_dtype_t;

/* A cudaStream_t, passed as an opaque pointer so this header needs no CUDA header. */
typedef void *attn_stream_t;

/*
 * Checks that `device` is a compute-capability 10.0 GPU and that this
 * library's kernels load on it.  Returns ATTN_OK, ATTN_ERR_NO_KERNEL_IMAGE or
 * ATTN_ERR_CUDA (no driver / no such device).  Lesson of "FA3 loader reports
 * success on Blackwell (sm_120) then dies at first kernel launch" (nanochat
 * issue 820, Cause): check the architecture at load time, not at first launch.
 */
attn_status_t attn_check_device(int device);

/* Static, NUL-terminated description of a status code (never NULL). */
const char *attn_status_string(attn_status_t status);

/*
 * Reads and clears the two device-side error words of the current device and
 * synchronises `stream` (a debugging aid, not for hot loops).
 *   - A kernel gave up on a bounded wait since the last read: returns
 *     ATTN_ERR_DEVICE_TIMEOUT, *code_out names the wait (101..303 forward,
 *     401..402 decode, 601..604 backward, 901 the test hook below).  While that
 *     word is set, the other kernels' waits give up early.
 *   - Otherwise, a kernel met an index outside its buffers: returns
 *     ATTN_ERR_DEVICE_RANGE, *code_out names it (111 forward and 411 decode: a
 *     block_table entry outside [0, num_blocks), page 0 read in its place;
 *     501/502 KV append: a position past the block table / a page outside the
 *     cache, that token not written).  Nothing else stops on these.
 *   - Neither: ATTN_OK and *code_out = 0.
 */
attn_status_t attn_device_error(int *code_out, attn_stream_t stream);

/*
 * Test hook for the kernels' failure detection: launches one CTA whose thread
 * waits on a shared-memory barrier that nothing ever arrives on, bounded by
 * limit_ns nanoseconds (0 .. 1e10) instead of the kernels' 2 s.  The wait runs
 * out, records code 901 in the device error word and the kernel returns, so
 * the stream completes and the context stays usable; attn_device_error then
 * reports ATTN_ERR_DEVICE_TIMEOUT with that code (and clears it).  Run it with
 * no other kernel of this library in flight: while the word is set, their
 * bounded waits give up early.  No counterpart on the pages: the bounded
 * waits are this library's own protection against hanging the GPU.
 * Returns ATTN_ERR_INVALID_ARG for a limit outside that range.
 */
attn_status_t attn_selftest_wait_expiry(long long limit_ns, attn_stream_t stream);


/*
 * Dense attention forward.
 *   q  [B, Lq, Hq, D], k/v [B, Lk, Hkv, D] with element strides given per
 *      tensor as strides[3] = {batch, token, head}; the head_dim stride is 1.
 *   o  [B, Lq, Hq, D] bf16, contiguous.   lse [B, Hq, Lq] fp32, contiguous, or NULL.
 *   mask: ATTN_MASK_NONE or ATTN_MASK_CAUSAL (PATCH needs the varlen call).
 *   descale_*: fp8 only (device fp32 scalars), ignored for bf16.
 */
attn_status_t attn_fwd_dense(
    const void *q, const void *k, const void *v, void *o, float *lse,
    int B, int Lq, int Lk, int num_heads_q, int num_heads_kv, int head_dim,
    const int64_t *strides_q, const int64_t *strides_k, const int64_t *strides_v,
    float softmax_scale, int mask, int window_left, float softcap, int dtype,
    const float *descale_q, const float *descale_k, const float *descale_v,
    attn_stream_t stream);

/*
 * Varlen attention forward over packed queries and a paged (or packed) KV store.
 *   q            [total_q, Hq, D], contiguous; sequence b owns rows
 *                cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1 (cu_seqlens_q: int32 [B+1]).
 *   k_cache/v_cache
 *     paged  (block_table != NULL): [num_blocks, block_size, Hkv, D], contiguous;
 *            key j of sequence b is row j % block_size of page
 *            block_table[b * max_blocks_per_seq + j / block_size].
 *     packed (block_table == NULL): [total_k, Hkv, D], contiguous; sequence b owns
 *            rows cu_seqlens_k[b] .. ; cu_seqlens_k required.
 *   seqused_k    int32 [B] keys used per sequence, or NULL (then the
 *                difference of cu_seqlens_k, which is then required).
 *   max_seqlen_q upper bound of the per-sequence query lengths (sizes the grid).
 *   patch_kv_range int32 [total_q, 2], PATCH only: per-query [start, end).
 *   o            [total_q, Hq, D] bf16.   lse [Hq, total_q] fp32 or NULL.
 *   workspace    unused by this version; may be NULL with workspace_bytes 0.
 * A used block_table entry outside [0, num_blocks) is a caller error: the
 * kernel reads page 0 in its place and records code 111 for attn_device_error
 * (ATTN_ERR_DEVICE_RANGE); the decode calls do the same with code 411.
 */
attn_status_t attn_fwd_varlen_paged(
    const void *q, const void *k_cache, const void *v_cache,
    const int32_t *block_table, int max_blocks_per_seq, int num_blocks, int block_size,
    const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k, const int32_t *seqused_k,
    int B, int total_q, int total_k, int max_seqlen_q,
    int num_heads_q, int num_heads_kv, int head_dim,
    float softmax_scale, int mask, const int32_t *patch_kv_range,
    int window_left, float softcap,
    int dtype, const float *descale_q, const float *descale_k, const float *descale_v,
    void *o, float *lse, void *workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * Patch-to-byte cross-attention (the patch mask of attn_fwd_varlen_paged) for
 * intervals the caller knows to be short, as in the byte-latent model of "Cross
 * Attention does not work on CPU and older GPUs" (one query per patch, each
 * attending to its own patch's bytes; patches of at most 16 bytes).  Query i of
 * sequence b sees the keys [patch_kv_range[i][0], patch_kv_range[i][1]) of its
 * sequence (clamped to [0, Lk_b)); O and LSE as in attn_fwd_varlen_paged, an
 * empty interval giving O = 0 and LSE = -inf.
 *   q [total_q, Hq, D], k/v packed [total_k, Hkv, D], cu_seqlens_q/k int32 [B+1],
 *   patch_kv_range int32 [total_q, 2], o [total_q, Hq, D] bf16, lse [Hq, total_q] or NULL.
 *   max_interval  the caller's bound on end - start over all queries.  It only
 *                 chooses the kernel, never the result: up to 64 (bf16) CUDA-core
 *                 kernels read each key and value row once per query (with
 *                 Hq == Hkv the rows of consecutive queries stream through
 *                 shared memory; with grouped heads one warp takes a query);
 *                 above that, or for fp8, the tiled tensor-core kernel of
 *                 attn_fwd_varlen_paged runs.
 * Supported: head_dim in {64, 128}.
 */
attn_status_t attn_fwd_patch(
    const void *q, const void *k, const void *v, const int32_t *cu_seqlens_q,
    const int32_t *cu_seqlens_k, const int32_t *patch_kv_range, int B, int total_q, int total_k,
    int max_seqlen_q, int num_heads_q, int num_heads_kv, int head_dim, float softmax_scale,
    int max_interval, int dtype, const float *descale_q, const float *descale_k,
    const float *descale_v, void *o, float *lse, attn_stream_t stream);

/*
 * The forward with the extra Qv score term of "Rope dim" (vllm-project
 * flash-attention PR 172, overview: the Qv GEMM beside the QK GEMM, HasQv): the
 * logit of query i and key j is scale * (q_i . k_j + qv_i . v_j), then softcap,
 * masks, softmax and P.V as in attn_fwd_varlen_paged.
 *   qv           [total_q, Hq, D] bf16, laid out as q, 16-byte aligned; the
 *                value head dimension equals the key one here.
 *   other arguments as attn_fwd_varlen_paged (no descales: bf16 only).
 * Supported: bf16, head_dim in {64, 128}; fp8 gives ATTN_ERR_UNSUPPORTED and
 * qv NULL ATTN_ERR_INVALID_ARG.  The value tile is read once per key tile and
 * feeds both the second score GEMM and the P.V GEMM.
 */
attn_status_t attn_fwd_varlen_paged_qv(
    const void *q, const void *qv, const void *k_cache, const void *v_cache,
    const int32_t *block_table, int max_blocks_per_seq, int num_blocks, int block_size,
    const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k, const int32_t *seqused_k, int B,
    int total_q, int total_k, int max_seqlen_q, int num_heads_q, int num_heads_kv, int head_dim,
    float softmax_scale, int mask, const int32_t *patch_kv_range, int window_left, float softcap,
    int dtype, void *o, float *lse, attn_stream_t stream);

/*
 * The only_qv score path of "Rope dim" (vllm-project flash-attention PR 172,
 * overview: the mode that skips the Q and K loads and the QK GEMM and
 * zero-initialises the score with the Qv GEMM).  The score of query i and key
 * j is scale * (qv_i . v_j): the value rows serve as the score's second
 * operand, and there is no key store.  Everything else (masks, window,
 * softcap, LSE, paging, varlen, fp8) is as in attn_fwd_varlen_paged, with
 *   qv           in place of q: [total_q, Hq, D], the value head dimension.
 *   v_cache      the only KV store, laid out as v_cache there.
 *   descale_qv, descale_v   fp8 only; the score uses descale_qv * descale_v.
 * No key tile is fetched: each value tile is read once and feeds both the
 * score GEMM and the P.V GEMM.
 */
attn_status_t attn_fwd_varlen_paged_only_qv(
    const void *qv, const void *v_cache, const int32_t *block_table, int max_blocks_per_seq,
    int num_blocks, int block_size, const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
    const int32_t *seqused_k, int B, int total_q, int total_k, int max_seqlen_q,
    int num_heads_q, int num_heads_kv, int head_dim, float softmax_scale, int mask,
    const int32_t *patch_kv_range, int window_left, float softcap, int dtype,
    const float *descale_qv, const float *descale_v, void *o, float *lse, attn_stream_t stream);

/*
 * Bytes of workspace attn_decode_paged needs for these sizes (fp32 partial O
 * and LSE per split).  num_splits <= 0 means "as chosen automatically for
 * max_blocks_per_seq".  Returns 0 for invalid sizes.
 */
size_t attn_decode_workspace_size(int B, int num_heads_q, int num_heads_kv, int head_dim,
                                  int max_blocks_per_seq, int block_size, int num_splits);

/*
 * Paged decode: one query token per sequence, split-KV with an LSE-weighted
 * combine.  The query is the newest of the sequence's cached keys and sees
 * all of them, or with window_left >= 0 only keys L-1-window_left .. L-1
 * (L = seqused_k[b]); softcap as above.
 *   q            [B, Hq, D] bf16 (or e4m3), contiguous.
 *   k_cache/v_cache, block_table, block_size: as in attn_fwd_varlen_paged.
 *   seqused_k    int32 [B], keys cached per sequence (0 gives O = 0, LSE = -inf).
 *   num_splits   key-range splits per sequence; <= 0 chooses automatically.
 *   dtype        ATTN_BF16, or ATTN_FP8_E4M3 for an e4m3 q and cache with
 *                descale_q/k/v (device fp32 scalars, all three required):
 *                num_splits <= 0, at most 8 KV heads.
 *   o            [B, Hq, D] bf16.   lse [B, Hq] fp32 or NULL.
 *   workspace    >= attn_decode_workspace_size(...) bytes of device memory,
 *                16-byte aligned; its contents on entry do not matter.
 * Supported: bf16, head_dim in {64, 128}, Hq/Hkv <= 16; e4m3 as above.
 */
attn_status_t attn_decode_paged(
    const void *q, const void *k_cache, const void *v_cache, const int32_t *block_table,
    int max_blocks_per_seq, int num_blocks, int block_size, const int32_t *seqused_k,
    int B, int num_heads_q, int num_heads_kv, int head_dim, float softmax_scale,
    int window_left, float softcap, int num_splits, int dtype,
    const float *descale_q, const float *descale_k, const float *descale_v,
    void *o, float *lse, void *workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * Paged decode with the extra Qv score term of "Rope dim" (vllm-project
 * flash-attention PR 172, overview: the Qv GEMM beside the QK GEMM, HasQv):
 * the logit of key j is scale * (q . k_j + qv . v_j), then softcap, masks,
 * softmax and P.V as in attn_decode_paged.
 *   qv           [B, Hq, D] bf16, contiguous, 16-byte aligned; the value head
 *                dimension equals the key one here.
 *   other arguments as attn_decode_paged (workspace sized by
 *                attn_decode_workspace_size with the same arguments).
 * Supported: bf16, head_dim in {64, 128}, num_splits <= 0 (the automatic
 * split), Hkv <= 8, Hq/Hkv <= 16, B <= 4096; otherwise ATTN_ERR_UNSUPPORTED.
 * qv NULL gives ATTN_ERR_INVALID_ARG.  Each value row is read once per page
 * and feeds both the score and the P.V product.
 */
attn_status_t attn_decode_paged_qv(
    const void *q, const void *qv, const void *k_cache, const void *v_cache,
    const int32_t *block_table, int max_blocks_per_seq, int num_blocks, int block_size,
    const int32_t *seqused_k, int B, int num_heads_q, int num_heads_kv, int head_dim,
    float softmax_scale, int window_left, float softcap, int num_splits, int dtype, void *o,
    float *lse, void *workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * Paged decode with the only_qv score (as attn_fwd_varlen_paged_only_qv): the
 * score of key j is scale * (qv . v_j), read from the one value store; each
 * page of V is fetched once.  Arguments as attn_decode_paged with qv in place
 * of q and without the key store; workspace sized by attn_decode_workspace_size.
 * Supported: bf16, head_dim in {64, 128}, Hq/Hkv <= 16.
 */
attn_status_t attn_decode_paged_only_qv(
    const void *qv, const void *v_cache, const int32_t *block_table, int max_blocks_per_seq,
    int num_blocks, int block_size, const int32_t *seqused_k, int B, int num_heads_q,
    int num_heads_kv, int head_dim, float softmax_scale, int window_left, float softcap,
    int num_splits, int dtype, void *o, float *lse, void *workspace, size_t workspace_bytes,
    attn_stream_t stream);

/*
 * Paged KV append: writes new tokens' keys and values into the paged cache
 * (the ReshapeAndCache step of "[CUDA] PagedAttention: add SM<80 fp16
 * fallback via memory-efficient attention", Implementation step 1; the K_new
 * / AppendKV path of "Rope dim").  Sequence b holds seqused_k[b] cached tokens
 * before the call; its i-th new token (row cu_seqlens_new[b] + i of k_new /
 * v_new) is stored at cache position p = seqused_k[b] + i, i.e. row p % 16 of
 * page block_table[b * max_blocks_per_seq + p / 16].  Nothing else in the
 * cache is written.
 *   k_new/v_new    [total_new, Hkv, D], contiguous, of `dtype` (bf16 or e4m3
 *                  codes; the bytes are copied as they are).
 *   k_cache/v_cache [num_blocks, block_size, Hkv, D], contiguous, same dtype.
 *   cu_seqlens_new int32 [B+1] (NULL: exactly one new token per sequence,
 *                  total_new == B).
 *   seqused_k      int32 [B], lengths before the call (read only).
 *   seqused_k_out  int32 [B] or NULL: receives seqused_k[b] + n_b.  It must
 *                  not be the same buffer as seqused_k (ATTN_ERR_INVALID_ARG).
 * Requirements: block_size == 16; head_dim * element bytes a multiple of 16;
 * 16-byte aligned k_new, v_new and caches.  The appended positions of
 * different sequences must map to different cache rows.  A position past a
 * sequence's block table, or a page index outside [0, num_blocks), is not
 * written: the kernel records code 501 (position) or 502 (page) in the device
 * data-error word (attn_device_error reports ATTN_ERR_DEVICE_RANGE) and copies
 * the remaining tokens.
 */
attn_status_t attn_kv_append_paged(
    const void *k_new, const void *v_new, void *k_cache, void *v_cache,
    const int32_t *block_table, int max_blocks_per_seq, int num_blocks, int block_size,
    const int32_t *cu_seqlens_new, const int32_t *seqused_k, int32_t *seqused_k_out,
    int B, int total_new, int num_heads_kv, int head_dim, int dtype, attn_stream_t stream);

/*
 * One decode step with its KV append in one call: appends one new token per
 * sequence (k_new/v_new [B, Hkv, D]) as attn_kv_append_paged does, then runs
 * attn_decode_paged for q [B, Hq, D] over the updated cache, whose lengths
 * the append writes to seqused_k_out (required; lengths before the call in
 * seqused_k).  The decode is launched as a programmatic dependent of the
 * append, so its launch overlaps the append and it waits for the append's
 * writes on the device.  Arguments otherwise as attn_decode_paged (bf16).
 * The decode's arguments are checked before the append is launched; should
 * the decode still fail to launch, the append has already taken effect.
 */
attn_status_t attn_decode_paged_append(
    const void *q, const void *k_new, const void *v_new, void *k_cache, void *v_cache,
    const int32_t *block_table, int max_blocks_per_seq, int num_blocks, int block_size,
    const int32_t *seqused_k, int32_t *seqused_k_out,
    int B, int num_heads_q, int num_heads_kv, int head_dim, float softmax_scale,
    int window_left, float softcap, int num_splits, int dtype,
    void *o, float *lse, void *workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * Bytes of workspace attn_bwd_varlen needs (fp32 Delta per query row and head).
 * Returns 0 for invalid sizes.
 */
size_t attn_bwd_workspace_size(int num_heads_q, int total_q);

/*
 * Attention backward: the gradients dQ, dK, dV of the varlen forward, for the
 * training path of the pages (BLT trains through the FlexAttention autograd;
 * "Rope dim" lists the FlashAttnVarlenFunc backward).  With
 * P = exp(scale Q K^T - LSE) under the mask and Delta_i = dO_i . O_i:
 *   dV = P^T dO,  dS = P (dO V^T - Delta) scale,  dQ = dS K,  dK = dS^T Q,
 * dK and dV summed over each KV head's query heads.
 *   q, o, dout, dq [total_q, Hq, D] bf16, contiguous (o and lse from the
 *                  forward on the same inputs, lse [Hq, total_q] fp32).
 *   k, v, dk, dv   [total_k, Hkv, D] bf16, contiguous (packed; no paging).
 *   cu_seqlens_q, cu_seqlens_k int32 [B+1]; max_seqlen_q / max_seqlen_k bound
 *                  the per-sequence lengths (they size the grids).
 *   mask           ATTN_MASK_NONE or ATTN_MASK_CAUSAL (bottom-right aligned),
 *                  window_left as in the forward (causal only); no softcap
 *                  and no patch mask (ATTN_ERR_UNSUPPORTED).
 *   workspace      >= attn_bwd_workspace_size(Hq, total_q) bytes, 16-byte
 *                  aligned (receives Delta).
 * Every output row is written (rows whose query saw no key get dQ = 0; keys
 * no query saw get dK = dV = 0).  Supported: head_dim in {64, 128}.
 */
attn_status_t attn_bwd_varlen(
    const void *q, const void *k, const void *v, const void *o, const void *dout,
    const float *lse, void *dq, void *dk, void *dv,
    const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
    int B, int total_q, int total_k, int max_seqlen_q, int max_seqlen_k,
    int num_heads_q, int num_heads_kv, int head_dim, float softmax_scale,
    int mask, int window_left, void *workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_decode_paged without any device allocation by the caller: the same
 * paged decode (automatic split choice), with its scratch taken from a fixed
 * 8 MiB array that this library keeps in device memory.  No counterpart on
 * the pages; it exists for callers that cannot allocate device memory at
 * call time -- e.g. a plug-in loaded into a host program that owns every
 * allocation and exposes no allocator, or a latency-critical serving loop
 * whose memory is sized once at start-up and which must not reach
 * cudaMalloc (an implicit synchronisation) while it runs.
 *   Arguments: as attn_decode_paged, without window_left, softcap, num_splits
 *   and workspace (no sliding window, no softcap).
 *   Limits: requests whose split-KV partials need more than 8 MiB (about
 *   (SMs + B) * Hq * (head_dim + 1) * 4 bytes) return ATTN_ERR_SCRATCH_LIMIT;
 *   shapes outside the page-stream decode (more than 8 KV heads, more than 16
 *   query heads per KV head) return ATTN_ERR_UNSUPPORTED.
 *   Set-up: the first call on each device looks up the scratch's device
 *   address (cudaGetSymbolAddress) with that device current; make that first
 *   call before any stream capture.  The address is kept for the life of the
 *   process, so this entry point must not be used on a device after
 *   cudaDeviceReset (or any other teardown of its primary context).
 *   dtype: ATTN_BF16; ATTN_FP8_E4M3 returns ATTN_ERR_UNSUPPORTED (this call
 *   takes no descales).
 *   Errors: bad arguments get the same status as from attn_decode_paged
 *   (for bf16).
 *   Sharing: every call on a device uses the same scratch and leaves its
 *   contents behind (nothing in it needs to start zeroed).  Calls whose
 *   kernels could overlap on the GPU (different streams without ordering)
 *   race on it; order them on one stream or with events.
 *   Allocation: none -- no cudaMalloc, cudaFree or allocating library call.
 */
attn_status_t attn_decode_paged_noalloc(
    const void *q, const void *k_cache, const void *v_cache, const int32_t *block_table,
    int max_blocks_per_seq, int num_blocks, int block_size, const int32_t *seqused_k,
    int B, int num_heads_q, int num_heads_kv, int head_dim, float softmax_scale, int dtype,
    void *o, float *lse, attn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
