/*
 * wf_attn.h -- C ABI of the B200 (sm_100a) attention-forward library.
 *
 * One operation, the scaled-dot-product attention forward
 *
 *     out = softmax(Q * K^T * qkScale + mask) * V
 *
 * with GQA head grouping, boolean keep-masks, additive float masks, in-kernel
 * causal masks, packed variable-length sequences and the MLA split
 * contraction q*k + qRope*kRope; plus the rolling sink+window BlockKVCache
 * that feeds it.
 *
 * Sources the calls follow:
 *   [P1]  "Core 注意力", WorldFoundry docs (openenvision.github.io/WorldFoundry),
 *         sections "选择最窄的入口" (SDPA contract, GQA expansion),
 *         "一个可以在 CPU 或 GPU 上运行的例子" (layouts [B,H,L,D], bool mask =
 *         keep, float mask added) and "Block KV cache 的调用顺序" (cache calls,
 *         their order, sink and window sizes).
 *   [P2]  "MLA Prefill", CANN ATB docs (hiascend.com), "定义" (a C interface
 *         that returns a status) and the parameter table (Q/QRope/K/kRope/V,
 *         qSeqLen/kvSeqLen, mask, headNum, qkScale, kvHeadNum, maskType,
 *         attenOut).
 *
 * Conventions for every call:
 *   - All tensor data pointers are DEVICE pointers of the current CUDA device
 *     unless a parameter says "host".  The library never frees caller memory.
 *   - Tensors are described by wf_tensor_t: dims and strides are in ELEMENTS;
 *     the last dimension must have stride 1.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Launches are asynchronous on that stream.
 *   - Argument errors are reported synchronously, before anything is
 *     launched; wf_last_error_message() then holds a description.
 *   - Device-side conditions that can only be seen while running (bad
 *     sequence lengths, a bounded wait that ran out) are recorded in a device
 *     status word read by wf_get_device_status().
 *   - Not thread-safe per wf_kvcache_t handle; the attention call is
 *     reentrant across host threads.
 */
#ifndef WF_ATTN_H
#define WF_ATTN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define WF_ATTN_VERSION 1

/* Status codes (the [P2] "定义" section returns a status from every call). */
typedef enum wf_status {
    WF_OK = 0,
    WF_ERR_INVALID_ARG = 1,   /* shape / stride / dtype / pointer is not valid */
    WF_ERR_UNSUPPORTED = 2,   /* valid request outside what the kernels implement */
    WF_ERR_ORDER = 3,         /* BlockKVCache call out of the documented order */
    WF_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
    WF_ERR_NO_MEMORY = 5,     /* host or device allocation failed */
    WF_ERR_TIMEOUT = 6,       /* a bounded device wait ran out (device status) */
    WF_ERR_NO_DEVICE = 7      /* no usable sm_100 device for this call */
} wf_status_t;

/* Element types.  WF_U8 is the boolean keep-mask type (nonzero = keep). */
typedef enum wf_dtype {
    WF_F32 = 0,
    WF_BF16 = 1,
    WF_F16 = 2,
    WF_U8 = 3,
    WF_I32 = 4
} wf_dtype_t;

/* maskType.  [P2] table row "maskType" (UNDEFINED / SPEC / MASK_FREE) and row
 * "Mask" (CAUSAL_MASK may pass nullptr); [P1] example section for the two
 * explicit mask kinds.  ATB names map as: UNDEFINED -> NONE; CAUSAL_MASK,
 * MASK_FREE, SPEC -> CAUSAL (generated in the kernel; no mask tensor read).
 * Both causal kinds are bottom-right or top-left alignments of the same
 * predicate; rows that see no key give 0 (and LSE -inf). */
typedef enum wf_mask_type {
    WF_MASK_NONE = 0,
    WF_MASK_CAUSAL = 1,     /* key j visible to query i iff j <= i + (Lk - Lq) */
    WF_MASK_BOOL_KEEP = 2,  /* mask dtype WF_U8, nonzero = keep               */
    WF_MASK_ADDITIVE = 3,   /* mask dtype = q dtype or WF_F32, added to scores */
    WF_MASK_CAUSAL_TOP_LEFT = 4  /* key j visible to query i iff j <= i: the
                                  * alignment of PyTorch SDPA's is_causal ([P1]
                                  * "选择最窄的入口"); the same as WF_MASK_CAUSAL
                                  * when Lq == Lk.  Generated in the kernel. */
} wf_mask_type_t;

/* Tensor descriptor: up to 4 dims, strides in elements, caller-owned data. */
typedef struct wf_tensor {
    void *data;
    int32_t dtype;          /* wf_dtype_t */
    int32_t ndim;
    int64_t shape[4];
    int64_t stride[4];
} wf_tensor_t;

/*
 * wf_attn_fwd -- attention forward.  [P2] "定义" + parameter table (argument
 * set; headNum/kvHeadNum/qkScale), [P1] "选择最窄的入口" (SDPA contract, GQA).
 *
 * Two layouts, chosen by whether qSeqLen is given:
 *
 *   dense  (qSeqLen == kvSeqLen == NULL), the [P1] example layout:
 *     q   [B, headNum,   Lq, Dqk]     out [B, headNum, Lq, Dv]
 *     k   [B, kvHeadNum, Lk, Dqk]     v   [B, kvHeadNum, Lk, Dv]
 *   packed (qSeqLen, kvSeqLen given), the [P2] table layout:
 *     q   [nTokens,   headNum,   Dqk]  out [nTokens, headNum, Dv]
 *     k   [nKvTokens, kvHeadNum, Dqk]  v   [nKvTokens, kvHeadNum, Dv]
 *     qSeqLen, kvSeqLen: WF_I32 [batch] DEVICE arrays; sequence b occupies
 *     rows [sum_{c<b} len_c, sum_{c<=b} len_c).  The lengths are read on the
 *     device; if they sum past nTokens / nKvTokens (or are negative) the
 *     call computes nothing and the device status becomes
 *     WF_ERR_INVALID_ARG.
 *   packed q with padded k / v (4-d k, v and kRope), the [P2] table's
 *   [batch, max_seq, kv_head * D] form viewed as 4 dims:
 *     k   [batch, max_seq, kvHeadNum, Dqk]   v [batch, max_seq, kvHeadNum, Dv]
 *     sequence b's keys are rows [0, kvSeqLen[b]) of entry b; q and out stay
 *     packed.  A kvSeqLen[b] above max_seq is rejected on the device like an
 *     over-long sum.
 *   Keys are read in tiles of 128: K / V rows past a sequence's last key up
 *   to the tile's end (the next sequence's rows, padding, or rows past the
 *   last sequence) are loaded and get weight exactly 0.  They must hold
 *   finite values (0 * Inf is NaN in the product); rows past the end of the
 *   tensor are never read.
 *
 *   qRope / kRope (MLA, [P2] rows QRope/kRope): NULL, or [.., headNum, 64] /
 *     [.., kvHeadNum, 64] in the same layout as q / k.  Scores are then
 *     qkScale * (q.k + qRope.kRope).  Both or neither.
 *   mask: used only for WF_MASK_BOOL_KEEP / WF_MASK_ADDITIVE, dense layout
 *     only: logical [B, headNum, Lq, Lk]; a stride of 0 broadcasts a dim
 *     (size-1 dims must be given with stride 0 or size equal to the full
 *     extent).  Must be NULL otherwise.
 *   headNum % kvHeadNum == 0; query head h reads kv head h / (headNum/kvHeadNum).
 *   qkScale multiplies Q*K^T before the mask is added ([P2] row qkScale).
 *   dtypes: q, k, v, qRope, kRope, out all WF_BF16, all WF_F16 (both
 *     [P2] table types; P is rounded to the same type before P*V), or all
 *     WF_F32 (the F32 path multiplies on TF32 tensor cores; dense layout only,
 *     packed F32 returns WF_ERR_UNSUPPORTED).  Dqk, Dv in {64, 96, 128};
 *     with rope: Dqk = 128, Dv = 128, 16-bit types.
 *   Additive mask dtype: WF_F32, or q's dtype when that is 16-bit.
 *   Alignment: every data pointer 16-byte aligned; every stride except the
 *     last a multiple of 16 bytes.
 *   A query row that sees no key (causal with Lq > Lk, or an all-false
 *   keep-mask row) produces zeros.
 *
 * Returns WF_OK once launched (asynchronous), an argument status otherwise.
 * Ownership: all tensors are the caller's.  The library keeps a per-device
 * workspace (schedule tables) that it grows on demand and frees in
 * wf_shutdown().
 */
wf_status_t wf_attn_fwd(const wf_tensor_t *q, const wf_tensor_t *qRope,
                        const wf_tensor_t *k, const wf_tensor_t *kRope,
                        const wf_tensor_t *v,
                        const wf_tensor_t *qSeqLen, const wf_tensor_t *kvSeqLen,
                        const wf_tensor_t *mask,
                        int32_t headNum, int32_t kvHeadNum, float qkScale,
                        int32_t maskType, wf_tensor_t *out, void *stream);

/*
 * wf_attn_fwd_ex -- wf_attn_fwd with the row log-sum-exp as a second output
 * and a choice of split-KV.  The LSE is what lets results computed over
 * disjoint key sets be combined (wf_attn_merge): the pages name such uses --
 * context-parallel attention ([P1] "选择最窄的入口") and calcType RING ([P2]
 * parameter table) -- without writing the step out.
 *
 *   lse: NULL, or WF_F32 with out's shape minus the last dim -- dense
 *     [B, headNum, Lq], packed [nTokens, headNum] -- any element strides (so a
 *     head-major [headNum, nTokens] buffer may be passed transposed), 4-byte
 *     aligned.  lse = ln sum_j exp(x_j) over the row's visible keys, x_j the
 *     scaled score plus the additive mask; -inf for a row that sees no key.
 *   numSplits: 0 = automatic (dense layout only: when the work units cannot
 *     fill the SMs, the keys of every unit are split into as many contiguous
 *     ranges as fill them, each of at least 4 tiles of 128 keys); 1 = no
 *     split; 2..128 = that many ranges (both layouts).  With more than one
 *     range each one writes an fp32 partial result and its LSE to the
 *     library's per-stream workspace, and a merge pass (as wf_attn_merge)
 *     writes out and lse.  Results differ from the unsplit ones only by
 *     rounding.
 * Everything else, including errors and ownership, as wf_attn_fwd;
 * wf_attn_fwd is this call with lse = NULL and numSplits = 0.
 */
wf_status_t wf_attn_fwd_ex(const wf_tensor_t *q, const wf_tensor_t *qRope,
                           const wf_tensor_t *k, const wf_tensor_t *kRope,
                           const wf_tensor_t *v,
                           const wf_tensor_t *qSeqLen, const wf_tensor_t *kvSeqLen,
                           const wf_tensor_t *mask,
                           int32_t headNum, int32_t kvHeadNum, float qkScale,
                           int32_t maskType, wf_tensor_t *out, wf_tensor_t *lse,
                           int32_t numSplits, void *stream);

/*
 * wf_attn_merge -- combine S attention results of the same query rows, each
 * computed over a different, disjoint set of keys, into the result over all
 * of them (the step behind the uses named at wf_attn_fwd_ex; it follows from
 * the softmax definition):
 *     lse = ln sum_s exp(lseParts[s]),   out = sum_s exp(lseParts[s] - lse) * outParts[s].
 * A part whose LSE is -inf has weight 0 (its row is not read); a row whose
 * parts are all -inf gives 0 and -inf.
 *
 *   outParts: [S, R, Dv] WF_F32, WF_BF16 or WF_F16, normalised partial results (as
 *     wf_attn_fwd_ex writes them), last dim contiguous, 16-byte aligned
 *     pointer and strides.  Dv a multiple of 4.
 *   lseParts: [S, R] WF_F32, natural log, any strides.
 *   out: [R, Dv] WF_F32, WF_BF16 or WF_F16, same layout rules as outParts.
 *   lse: NULL or [R] WF_F32.
 * Rows of a [B, H, L, Dv] or [T, H, Dv] result are passed flattened to R.
 * Returns WF_OK once launched (asynchronous); argument errors launch nothing.
 * All tensors are the caller's.
 */
wf_status_t wf_attn_merge(const wf_tensor_t *outParts, const wf_tensor_t *lseParts,
                          wf_tensor_t *out, wf_tensor_t *lse, void *stream);

/*
 * wf_attn_dca -- dual chunk attention ("Dual Chunk Attention" article: a long
 * sequence cut into chunks, attended within a chunk, to the neighbouring
 * chunk and across chunks with remapped relative positions).  The article
 * gives no formulas; the reading here: every query comes in three forms, the
 * caller having rotated each for its position map, and query i of chunk
 * c = i / chunkSize attends causally to keys j <= i with
 *     qIntra (j in chunk c), qSucc (j in chunk c - 1), qInter (earlier chunks),
 * all scores times qkScale in one softmax.
 *   qIntra, qSucc, qInter: [B, headNum, L, D];  k: [B, kvHeadNum, L, D];
 *   v: [B, kvHeadNum, L, Dv];  out: [B, headNum, L, Dv];  lse: NULL or
 *   [B, headNum, L] WF_F32 (natural log).  WF_BF16 or WF_F16; D, Dv as for
 *   wf_attn_fwd; strides as for its dense layout.
 * Runs as three attention calls over disjoint key sets (causal within the
 * chunks, chunk c against chunk c - 1, chunk c >= 2 against keys before
 * chunk c - 1) and the merge pass; a library-owned per-stream scratch holds
 * the three parts (3 L headNum (Dv x element size + 4) bytes).  Errors as
 * wf_attn_fwd; asynchronous.
 */
wf_status_t wf_attn_dca(const wf_tensor_t *qIntra, const wf_tensor_t *qSucc,
                        const wf_tensor_t *qInter, const wf_tensor_t *k,
                        const wf_tensor_t *v, int64_t chunkSize, int32_t headNum,
                        int32_t kvHeadNum, float qkScale, wf_tensor_t *out,
                        wf_tensor_t *lse, void *stream);

/*
 * wf_attn_fwd_debug -- wf_attn_fwd with test switches for the bounded waits
 * (no counterpart on the pages; a diagnostic aid).
 *   debug_flags bit 0: the kernel's copy engine never loads the first K tile,
 *     so the matrix-multiply stage's bounded wait runs out.  The call still
 *     returns WF_OK; wf_get_device_status() then reports WF_ERR_TIMEOUT and
 *     the device stays usable.  `out` is undefined after a timeout.
 *   timeout_cycles: bound of every device wait in SM clock cycles; 0 selects
 *     the production bound (2^31 cycles, about one second).
 * With debug_flags = 0 and timeout_cycles = 0 this is exactly wf_attn_fwd.
 */
wf_status_t wf_attn_fwd_debug(const wf_tensor_t *q, const wf_tensor_t *qRope,
                              const wf_tensor_t *k, const wf_tensor_t *kRope,
                              const wf_tensor_t *v,
                              const wf_tensor_t *qSeqLen, const wf_tensor_t *kvSeqLen,
                              const wf_tensor_t *mask,
                              int32_t headNum, int32_t kvHeadNum, float qkScale,
                              int32_t maskType, wf_tensor_t *out, void *stream,
                              uint32_t debug_flags, int64_t timeout_cycles);

/*
 * wf_attn_fwd_varlen_noalloc -- the packed-sequence (varlen) bf16 form of
 * wf_attn_fwd that never allocates memory.  The pages have no counterpart;
 * it exists for callers that cannot call cudaMalloc once they run (work
 * captured into CUDA graphs that must leave the allocator alone, runtimes
 * that give the whole device to a pool at start-up, fixed memory budgets).
 *
 * Arguments as in wf_attn_fwd's packed layout (no mask; maskType NONE,
 * CAUSAL or CAUSAL_TOP_LEFT; all tensors WF_BF16).  Instead of an allocated
 * workspace, the schedule tables live in a fixed array inside the library:
 * 65536 int32 words (256 KiB) on every GPU that loads the library, held until
 * the process exits; the work-item counters live in a fixed 4-word array.  A
 * call needs 4 * batch + 5 words (batch <= 16382); larger calls return
 * WF_ERR_INVALID_ARG and launch nothing.  The first call on a device looks
 * the arrays' addresses up (cudaGetSymbolAddress); make that first call
 * before any stream capture.  The addresses are kept for the life of the
 * process: after a cudaDeviceReset, call wf_shutdown (which forgets them)
 * before calling again.  All calls share the arrays: calls whose work
 * overlaps on the GPU (e.g. on different streams) race; calls in order on
 * one stream do not, as each rewrites every word it reads.  Other dtypes and
 * the explicit mask kinds return WF_ERR_UNSUPPORTED, tensors that are not
 * 3-d (the dense layout) WF_ERR_INVALID_ARG; split-KV and the LSE output are
 * not offered here.  wf_attn_fwd itself is
 * no substitute for such callers in any layout: its first call on each
 * (device, stream) allocates a workspace of at least 1 MiB with cudaMalloc.
 */
wf_status_t wf_attn_fwd_varlen_noalloc(const wf_tensor_t *q, const wf_tensor_t *qRope,
                                       const wf_tensor_t *k, const wf_tensor_t *kRope,
                                       const wf_tensor_t *v,
                                       const wf_tensor_t *qSeqLen, const wf_tensor_t *kvSeqLen,
                                       int32_t headNum, int32_t kvHeadNum, float qkScale,
                                       int32_t maskType, wf_tensor_t *out, void *stream);

/* ---------------------------------------------------------------------------
 * BlockKVCache ([P1] "Block KV cache 的调用顺序").
 *
 * The caller owns two buffers k_buf / v_buf of logical shape
 * [B, H, L, Dk] / [B, H, L, Dv] (seq_dim = 2), or [B, L, H, D] (seq_dim = 1);
 * L = sink_size + window_size, a multiple of chunk_size; sink_size is also a
 * multiple of chunk_size and window_size >= chunk_size.  The handle only
 * records the rolling state; the buffers are written by wf_kvcache_update.
 *
 * Every chunk index c runs  before_update(c) -> update -> cached -> after_update(c).
 * before_update(c) is legal when no chunk is in progress and c == 0 (first
 * chunk), c == last committed (overwrite the same logical chunk) or
 * c == last committed + 1 (append, or roll the window).  Anything else returns
 * WF_ERR_ORDER and leaves the state as it was.
 *
 * Chunk c lives in slot c while c < sink/chunk, afterwards in
 * sink/chunk + (c - sink/chunk) mod (window/chunk); slot s covers sequence
 * positions [s*chunk, (s+1)*chunk) of the buffers.  After chunk c the visible
 * tokens are the physical prefix of chunk * min(c+1, L/chunk) positions.
 * ------------------------------------------------------------------------- */
typedef struct wf_kvcache wf_kvcache_t;

/* Create a handle over caller-owned buffers (4-d, same dtype and shape apart
 * from the last dim, last dim contiguous).  No device memory is touched.
 * *out receives the handle, owned by the caller until wf_kvcache_destroy; the
 * buffers must outlive it.  WF_ERR_INVALID_ARG for NULL or malformed buffers,
 * seq_dim other than 1 or 2, sink_size + window_size different from the
 * buffers' length L, L or sink_size not a multiple of chunk_size, or
 * window_size < chunk_size; WF_ERR_NO_MEMORY if the host allocation fails. */
wf_status_t wf_kvcache_create(const wf_tensor_t *k_buf, const wf_tensor_t *v_buf,
                              int32_t seq_dim, int64_t chunk_size,
                              int64_t sink_size, int64_t window_size,
                              wf_kvcache_t **out);

/* Start chunk `chunk_idx` (host only, no device work).  WF_ERR_ORDER while a
 * chunk is in progress or for an index the order rule above does not allow;
 * the state is then unchanged. */
wf_status_t wf_kvcache_before_update(wf_kvcache_t *cache, int64_t chunk_idx);

/* Write the current chunk: k / v have the buffers' shape with exactly
 * chunk_size positions along seq_dim (same dtype, last dim contiguous);
 * copied on `stream` into the chunk's slot (asynchronous; k / v must stay
 * valid until the copy has run).  WF_ERR_ORDER unless before_update was the
 * last call, WF_ERR_INVALID_ARG for a shape or dtype mismatch: nothing is
 * written and the state is unchanged.  WF_ERR_CUDA if a copy cannot be
 * launched (the K copy may have been issued when the V copy fails). */
wf_status_t wf_kvcache_update(wf_kvcache_t *cache, const wf_tensor_t *k,
                              const wf_tensor_t *v, void *stream);

/* Views of the visible prefix, returned in the logical [B, H, vis, D] form
 * (strides of the buffers; the data pointers point into the caller's
 * buffers), ready to pass to wf_attn_fwd as k / v.  Physical ring order:
 * attention without a causal mask does not depend on key order.  Host only.
 * WF_ERR_ORDER before the chunk's update; either view pointer may be NULL. */
wf_status_t wf_kvcache_cached(wf_kvcache_t *cache, wf_tensor_t *k_view,
                              wf_tensor_t *v_view, int64_t *visible_len);

/* wf_kvcache_update_attend -- one chunk's update, cached view and attention
 * in a single kernel ("Core 注意力", section "Block KV cache 的调用顺序": the
 * chunk's update -> cached_k / cached_v -> attention over the cached keys).
 * Call after wf_kvcache_before_update, in place of wf_kvcache_update +
 * wf_kvcache_cached + wf_attn_fwd; follow with wf_kvcache_after_update.
 *   k, v: the chunk, as for wf_kvcache_update.
 *   q, out: [B, headNum, Lq, Dqk / Dv] (dense layout of wf_attn_fwd); the
 *     cache's head count is kvHeadNum.  Attention without a mask over the
 *     visible keys in physical ring order, as wf_attn_fwd over the
 *     wf_kvcache_cached views.
 * The attention kernel reads the chunk's keys and values from k / v directly
 * and stores them into the ring slot as it goes, so no separate copy runs.
 * That needs 16-bit buffers, head sizes 64 or 128 and a chunk size that is a
 * multiple of 128; otherwise the call runs the copy and then wf_attn_fwd
 * (same results).
 * Results and cache contents are bit-identical to the unfused calls.
 * WF_ERR_ORDER out of phase; argument errors as wf_kvcache_update /
 * wf_attn_fwd, with nothing written.  On success the cache is in the state
 * wf_kvcache_cached leaves it in. */
wf_status_t wf_kvcache_update_attend(wf_kvcache_t *cache, const wf_tensor_t *k,
                                     const wf_tensor_t *v, const wf_tensor_t *q,
                                     int32_t headNum, float qkScale, wf_tensor_t *out,
                                     void *stream);

/* Commit chunk `chunk_idx` (must equal the one in progress). Host only.
 * WF_ERR_ORDER before the cached views were taken (or the fused call ran) or
 * for another index; the state is then unchanged. */
wf_status_t wf_kvcache_after_update(wf_kvcache_t *cache, int64_t chunk_idx);

/* Read the state: index in progress (-1 before the first), last committed
 * index (-1 before the first commit), slot of the index in progress (-1 if
 * none), visible length, phase (0 idle, 1 before_update done, 2 update done,
 * 3 cached done).  Any output pointer may be NULL. */
wf_status_t wf_kvcache_get_state(const wf_kvcache_t *cache, int64_t *cur_idx,
                                 int64_t *committed_idx, int64_t *write_slot,
                                 int64_t *visible_len, int32_t *phase);

/* Restore the rolling state: chunk `committed_idx` (-1: none) becomes the
 * last committed chunk, with no chunk in progress, as if the calls up to
 * after_update(committed_idx) had run on this handle.  For resuming a cache
 * whose buffers the caller has restored (e.g. from a checkpoint); the buffers
 * are not touched, and holding the matching contents is the caller's part.
 * Host only.  WF_ERR_ORDER while a chunk is in progress (state unchanged),
 * WF_ERR_INVALID_ARG for committed_idx < -1.  The pages have no counterpart
 * (their cache lives in one process from chunk 0 on). */
wf_status_t wf_kvcache_set_state(wf_kvcache_t *cache, int64_t committed_idx);

/* Copy the visible tokens in LOGICAL chunk order (sink chunks, then the
 * window's chunks oldest first) into k_out / v_out, [B, H, vis, D] (or the
 * seq_dim = 1 form).  Allowed in the same phases as wf_kvcache_cached. */
wf_status_t wf_kvcache_gather_logical(wf_kvcache_t *cache, wf_tensor_t *k_out,
                                      wf_tensor_t *v_out, void *stream);

/* Free the handle (host memory only; the buffers stay the caller's).
 * NULL is ignored. */
void wf_kvcache_destroy(wf_kvcache_t *cache);

/* ---------------------------------------------------------------------------
 * Diagnostics and lifetime.
 * ------------------------------------------------------------------------- */

/* Synchronize `stream`, then read and clear the current device's status
 * word: WF_OK, WF_ERR_TIMEOUT (a bounded wait inside a kernel ran out; the
 * kernel abandoned its work and the affected output is undefined) or
 * WF_ERR_INVALID_ARG (device-side length check failed).  On WF_ERR_TIMEOUT
 * the call also synchronizes the device and resets the library's device-side
 * work-item counters, so that later calls start clean. */
wf_status_t wf_get_device_status(void *stream);

/* Description of the last error on the calling host thread ("" if none). */
const char *wf_last_error_message(void);

/* Library version (WF_ATTN_VERSION). */
int32_t wf_version(void);

/* Free the per-device workspaces and forget the cached device addresses (the
 * status word, the fixed arrays of wf_attn_fwd_varlen_noalloc); the next call
 * sets them up again.  Call with no work in flight, and after a
 * cudaDeviceReset before any other call of the library. */
void wf_shutdown(void);

#ifdef __cplusplus
}
#endif

#endif /* WF_ATTN_H */
