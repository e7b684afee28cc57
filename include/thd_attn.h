/*
 * thd_attn.h -- C ABI of the B200 (sm_100a) packed-THD sliding-window GQA
 * attention forward.
 *
 * The operation (restated from the NeMo AutoModel API pages):
 *
 *   Inputs are packed THD tensors as in MuseMagiPlan.attention and
 *   FlintMagiPlan.attention ("muse_spark.magi_cp" and "flint.magi" pages,
 *   query/key/value parameters): q [T, Hq, D], k and v [T, Hkv, D], with the
 *   documents of the pack delimited by cu_seqlens, "CPU int32 padded document
 *   boundaries [documents + 1]" (_build_magi_plan, cu_seqlens parameter).
 *
 *   For a query token i in document [s, e) and query head h, the visible keys
 *   are V(i) = { j : s <= j <= i and (window == 0 or j > i - window) }: the
 *   window counts the current token and zero means full causal
 *   (FlintMagiPlan.attention, window parameter).  Query head h reads key/value
 *   head g = h / (Hq / Hkv), the repeat_kv mapping ("muse_glimmer.model" page).
 *
 *   s_ij = scale * <q[i,h,:], k[j,g,:]>                       (scale parameter)
 *   Z    = sum_{j in V(i)} exp(s_ij) + exp(sink[h])           (sink parameter;
 *          the sink term is present only when sinks are given and has no
 *          value row)
 *   out[i,h,:] = sum_{j in V(i)} exp(s_ij) v[j,g,:] / Z       (bf16)
 *   lse[i,h]   = ln Z                                          (fp32)
 *
 *   The output is written in the input token order ("Attention output
 *   [tokens, query_heads, head_dim] in the local token order").
 *
 * Conventions shared by every entry point:
 *   - Device pointers are CUDA global-memory pointers on the current device;
 *     q, k, v, out must be 16-byte aligned and dense (row-major, no strides).
 *   - cu_seqlens is a HOST array; it is read during the call only.
 *   - The caller owns every buffer.  The library keeps, per device, a small
 *     cache of tile schedules, one status word and nothing else.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t passed as
 *     void*; NULL = the legacy default stream).  Argument errors are detected
 *     on the host before anything is enqueued and return a negative code.
 *   - A kernel that stops making progress (a bounded wait on the GPU ran out)
 *     records THD_ERR_TIMEOUT in the device status word and exits cleanly;
 *     thd_attn_get_error() reports it.
 */
#ifndef THD_ATTN_H
#define THD_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum thd_status {
    THD_OK = 0,
    THD_ERR_INVALID_ARG = -1,  /* bad pointer, alignment, shape, cu_seqlens, window or scale */
    THD_ERR_UNSUPPORTED = -2,  /* head_dim not in {64,128,256}, or device is not sm_100 */
    THD_ERR_CUDA = -3,         /* a CUDA runtime/driver call failed */
    THD_ERR_TIMEOUT = -4,      /* a bounded wait inside the kernel ran out */
    THD_ERR_NO_MEMORY = -5,    /* the schedule cache could not be allocated */
    THD_ERR_TOO_LARGE = -6,    /* thd_attn_fwd_noalloc: the schedule exceeds its fixed scratch */
    THD_ERR_STALE_SCRATCH = -7, /* thd_attn_fwd_noalloc: a launch found another call's schedule
                                   in the shared scratch and did nothing */
    THD_ERR_BAD_ITEM = -8       /* debug builds (THD_DEBUG=1) only: a forward CTA found a work
                                   item that breaks the schedule's invariants and did nothing */
};

/*
 * Forward pass.
 *
 *   q          bf16 device [T, Hq, D]        (T = cu_seqlens[n_docs])
 *   k, v       bf16 device [T, Hkv, D]
 *   cu_seqlens int32 HOST [n_docs + 1]: cu_seqlens[0] == 0, non-decreasing;
 *              zero-length documents are allowed; T == 0 or n_docs == 0 is a
 *              no-op that returns THD_OK.
 *   Hq, Hkv    query / key-value heads, Hq % Hkv == 0
 *   D          head dim, one of 64, 128, 256
 *   window     >= 0; 0 = full causal, W > 0 = the W most recent keys of the
 *              document including the query's own token
 *   scale      finite and > 0 (score scale, e.g. D^-0.5)
 *   sinks_or_null  fp32 device [Hq] learned sink logits, or NULL for none.
 *              A value of -inf (or very negative) behaves as no sink.
 *   out        bf16 device [T, Hq, D]; every element is written
 *   lse        fp32 device [T, Hq] natural-log log-sum-exp (sink included),
 *              or NULL to skip it
 *   stream     cudaStream_t as void*
 *
 * Returns THD_OK once the kernel is enqueued, or a negative thd_status
 * (nothing is enqueued on error).
 */
int thd_attn_fwd(const void* q, const void* k, const void* v,
                 const int32_t* cu_seqlens, int n_docs,
                 int Hq, int Hkv, int D, int window, float scale,
                 const float* sinks_or_null,
                 void* out, float* lse,
                 void* stream);

/*
 * Synchronises `stream`, returns the status recorded by kernels of this
 * library on the current device since the last call (THD_OK if none) and
 * clears it.  Returns THD_ERR_CUDA if the synchronisation itself fails.
 */
int thd_attn_get_error(void* stream);

/* Static English description of a thd_status value. */
const char* thd_attn_status_string(int status);

/*
 * One unit of work of the tile schedule: a tile of up to 128 query rows of
 * one document for `n_heads` consecutive query heads that share one kv head,
 * against the key tiles [kv_start, kv_start + n_kv * block_n).
 *   q0         first row of the 128-row query tile (may lie before doc_start;
 *              rows before doc_start are computed but never written)
 *   q1         one past the last row (<= the document end)
 *   doc_start  first token of the document
 *   head0      first query head of the item
 *   kv_start   first key of the first key tile (may lie before doc_start;
 *              such keys are masked)
 *   n_kv       number of key tiles (>= 1)
 *   n_heads    query heads in the item
 *   block_n    keys per key tile
 */
typedef struct thd_work_item {
    int32_t q0, q1, doc_start, head0;
    int32_t kv_start, n_kv, n_heads, block_n;
} thd_work_item;

/*
 * Host-only: build the tile schedule thd_attn_fwd uses for these arguments,
 * ordered by chunks of consecutive kv heads whose K/V (T x D bf16 each)
 * fits in 48 MB (so the CTAs in flight share those heads' K/V in L2) and,
 * within a chunk, longest first (non-increasing n_kv), the heads of one
 * (query tile, kv head) adjacent.
 * No CUDA call is made.  `items` may be NULL to query the count.  Writes
 * min(count, capacity) items and sets *n_items = count.  Returns THD_OK or
 * THD_ERR_INVALID_ARG / THD_ERR_UNSUPPORTED for the same argument errors as
 * thd_attn_fwd.
 */
int thd_attn_plan(const int32_t* cu_seqlens, int n_docs, int Hq, int Hkv, int D, int window,
                  thd_work_item* items, int64_t capacity, int64_t* n_items);

/*
 * Local step of a context-parallel forward: the query rows [q_begin, q_end)
 * of the pack against keys and values of the WHOLE pack.  The Magi plans
 * shard the packed tokens over the context-parallel ranks and gather K/V
 * ("muse_spark.magi_cp" page: one plan per microbatch over the rank's local
 * tokens, keys exchanged by the attention engine); a rank that owns rows
 * [q_begin, q_end) and holds the gathered K/V computes exactly those rows of
 * thd_attn_fwd's result.
 *   q          bf16 device [q_end - q_begin, Hq, D]: the rows it owns
 *   k, v       bf16 device [T, Hkv, D]: the whole pack (e.g. all-gathered)
 *   out, lse   [q_end - q_begin, Hq, D] bf16 and [q_end - q_begin, Hq] fp32
 *   other arguments as thd_attn_fwd (cu_seqlens covers the whole pack)
 * 0 <= q_begin <= q_end <= T, else THD_ERR_INVALID_ARG.  thd_attn_fwd is
 * the range [0, T).
 */
int thd_attn_fwd_range(const void* q, const void* k, const void* v,
                       const int32_t* cu_seqlens, int n_docs,
                       int64_t q_begin, int64_t q_end,
                       int Hq, int Hkv, int D, int window, float scale,
                       const float* sinks_or_null,
                       void* out, float* lse,
                       void* stream);

/*
 * thd_attn_fwd_range with the keys restricted to j < k_end: each row sees the
 * keys its causal / document / window rule allows AND below k_end.  This is
 * the part of a context-parallel row that lies on earlier ranks (the Magi
 * plans of the "muse_spark.magi_cp" page exchange keys between the ranks of
 * MuseMagiPlan.attention; a rank owning rows [b, e) can compute the keys at
 * or after b from its own slice and add the keys before b once they have
 * arrived, merging the two with thd_attn_merge).
 *   k, v       bf16 device [T, Hkv, D]; only rows j < k_end are read (rows
 *              below a document start may be read and are masked)
 *   k_end      0 <= k_end <= T, else THD_ERR_INVALID_ARG; k_end = T is
 *              thd_attn_fwd_range
 *   other arguments as thd_attn_fwd_range.  A row with no key below k_end
 *   gets out = 0 and lse = -inf (or, with sinks, lse = the sink logit).
 */
int thd_attn_fwd_range_keys(const void* q, const void* k, const void* v,
                            const int32_t* cu_seqlens, int n_docs,
                            int64_t q_begin, int64_t q_end, int64_t k_end,
                            int Hq, int Hkv, int D, int window, float scale,
                            const float* sinks_or_null,
                            void* out, float* lse,
                            void* stream);

/*
 * Merges two partial results of the same rows computed over disjoint key
 * sets (for example thd_attn_fwd on a rank's own slice of the pack and
 * thd_attn_fwd_range_keys on the keys before it).  The pages print no such
 * step: it is the log-sum-exp combination of two softmax parts, with
 * m = max(lse_a, lse_b), w = exp(lse - m):
 *   lse = m + log(w_a + w_b),  out = (w_a out_a + w_b out_b) / (w_a + w_b);
 * a part with lse = -inf has weight 0 (both -inf: out = 0, lse = -inf).
 * Sinks belong to exactly one of the parts.
 *   out_a, out_b   bf16 device [rows, Hq, D], 16-byte aligned
 *   lse_a, lse_b   fp32 device [rows, Hq] (natural log, as thd_attn_fwd)
 *   out, lse       results, same shapes; may be out_a / lse_a (in place)
 * D in {64, 128, 256} else THD_ERR_UNSUPPORTED; a NULL or misaligned buffer
 * (rows > 0) THD_ERR_INVALID_ARG; rows = 0 is a no-op.  Asynchronous on
 * `stream`.
 */
int thd_attn_merge(const void* out_a, const float* lse_a, const void* out_b, const float* lse_b,
                   int64_t rows, int Hq, int D, void* out, float* lse, void* stream);

/*
 * The forward from HOST buffers, with the copies overlapped with the
 * attention.  The pages have no counterpart of this entry point: it computes
 * the same packed-THD forward as thd_attn_fwd (MuseMagiPlan.attention,
 * "muse_spark.magi_cp" page) for callers whose tensors live in host memory.
 * The pack is split into n_chunks
 * token ranges of equal length; range c's q / k / v rows are copied to the
 * device on a copy stream, its query rows are computed as thd_attn_fwd_range
 * does on `stream` once they have landed (they read only key rows of their
 * own document at or before them, all copied by then), and its out / lse
 * rows are copied back on a second copy stream; copies of later ranges run
 * while earlier ranges compute.  The result equals thd_attn_fwd on the same
 * rows.
 *   q_host, k_host, v_host   bf16 host [T, Hq, D] / [T, Hkv, D] (page-locked
 *                            for the copies to overlap; pageable memory
 *                            works but serialises them)
 *   sinks_host_or_null       fp32 host [Hq] or NULL
 *   out_host, lse_host       bf16 host [T, Hq, D], fp32 host [T, Hq]: written
 *   q_dev .. lse_dev         device buffers of the same shapes (sinks_dev
 *                            [Hq], NULL exactly when sinks_host is), owned by
 *                            the caller, used as staging; 16-byte aligned as
 *                            thd_attn_fwd requires
 *   n_chunks                 1 .. 64 (each range has its own cached schedule;
 *                            the cache keeps 40, so up to about 32 ranges
 *                            stay cached between calls)
 * Asynchronous: returns once everything is queued; `stream` completes after
 * the last device-to-host copy, so synchronising it makes out_host and
 * lse_host valid.  The host buffers must stay untouched until then.  Calls
 * are serialised inside the library (one set of copy streams per device).
 * Errors: THD_ERR_INVALID_ARG for a NULL buffer, a sinks pair with one NULL,
 * n_chunks out of range or an invalid cu_seqlens (checked before any CUDA
 * call); otherwise thd_attn_fwd_range's errors, or THD_ERR_CUDA for a failed
 * copy.  T = 0 is a no-op.
 */
int thd_attn_fwd_host(const void* q_host, const void* k_host, const void* v_host,
                      const int32_t* cu_seqlens, int n_docs,
                      int Hq, int Hkv, int D, int window, float scale,
                      const float* sinks_host_or_null,
                      void* out_host, float* lse_host,
                      void* q_dev, void* k_dev, void* v_dev, float* sinks_dev_or_null,
                      void* out_dev, float* lse_dev,
                      int n_chunks, void* stream);

/* Host-only: the schedule thd_attn_fwd_range uses (q0 of a tile that would
 * reach before q_begin > 0 is raised to q_begin).  Same conventions as
 * thd_attn_plan. */
int thd_attn_plan_range(const int32_t* cu_seqlens, int n_docs, int64_t q_begin, int64_t q_end,
                        int Hq, int Hkv, int D, int window,
                        thd_work_item* items, int64_t capacity, int64_t* n_items);

/* Host-only: the schedule thd_attn_fwd_range_keys uses (key tiles end at
 * min(tile end, k_end); a tile whose rows see no key below k_end keeps one
 * wholly masked key tile).  Same conventions as thd_attn_plan. */
int thd_attn_plan_range_keys(const int32_t* cu_seqlens, int n_docs, int64_t q_begin,
                             int64_t q_end, int64_t k_end, int Hq, int Hkv, int D, int window,
                             thd_work_item* items, int64_t capacity, int64_t* n_items);

/*
 * Allocation-free variant of thd_attn_fwd.  The pages have no counterpart of
 * this entry point: it exists for callers that may not allocate device
 * memory -- runtimes that reserve all device memory up front and hand out
 * only pre-planned buffers, and latency-critical loops that cannot take the
 * device-wide synchronisation cudaMalloc/cudaFree may cause.
 *
 * Arguments and results are those of thd_attn_fwd, plus
 *   device_status_or_null  optional caller-owned device int.  If given, a
 *              kernel stall (THD_ERR_TIMEOUT) or a stale schedule
 *              (THD_ERR_STALE_SCRATCH) is recorded there; the caller zeroes
 *              it, and while it is non-zero, launches skip their work.  If
 *              NULL, the scratch's own status word is used: it keeps the
 *              first error until thd_attn_noalloc_get_error reads and clears
 *              it, and while it is non-zero, launches skip their work.
 *
 * Scratch: a fixed array inside the library's device image (one per GPU that
 * loads the library, kept until the process exits) holds a 256-byte header
 * (status word and schedule tag) and up to 65,536 work items (2 MiB + 256 B).
 * A schedule needs ceil(len/128) items per document per query-head pair (per
 * query head when Hq/Hkv is odd or D == 256); larger schedules return
 * THD_ERR_TOO_LARGE before anything is enqueued.  No call allocates device
 * or host heap memory (no cudaMalloc, cudaFree or allocating library
 * routine).
 *
 * The first call on a device does the set-up (looks up the scratch's device
 * address and clears its header, synchronously): make that first call
 * before any stream capture.  Every call shares the scratch and it keeps the
 * last call's contents: the schedule is re-uploaded, with a new tag, only
 * when the arguments differ from the previous call's on this device.  Each
 * launch checks on the GPU that the scratch still holds the schedule it was
 * enqueued for; if another call's schedule is there, it records
 * THD_ERR_STALE_SCRATCH and writes nothing.  Calls that overlap on the GPU
 * (for example on two streams of one device) race on the scratch; serialise
 * them.
 */
int thd_attn_fwd_noalloc(const void* q, const void* k, const void* v,
                         const int32_t* cu_seqlens, int n_docs,
                         int Hq, int Hkv, int D, int window, float scale,
                         const float* sinks_or_null,
                         void* out, float* lse,
                         int* device_status_or_null,
                         void* stream);

/*
 * Status of thd_attn_fwd_noalloc calls that used the scratch's own status
 * word (device_status_or_null == NULL): synchronises `stream`, returns the
 * first error recorded since the last read (THD_OK if none, or if no call
 * has run on this device yet) and clears it.  Allocates nothing.  Returns
 * THD_ERR_CUDA if the synchronisation or the read fails.
 */
int thd_attn_noalloc_get_error(void* stream);

/*
 * ------------------------------------------------------------------ backward
 * The pages run this attention inside training: the Magi plans are selected
 * "before entering checkpointed layers" and retained by the forward's
 * activation-checkpointing graph ("muse_spark.magi_cp" page,
 * _MuseMagiBatchPlans.select), so the gradient is taken through it.  The
 * backward is the exact derivative of thd_attn_fwd: with P_ij =
 * exp(s_ij - lse_i) from the forward's saved log-sum-exp and dO = dL/d out,
 *   D_i = sum_c dO_ic out_ic,  dS_ij = P_ij (dO_i . v_j - D_i),
 *   dq_i = scale sum_j dS_ij k_j,
 *   dk_j = scale sum over the query heads h of j's kv head and queries i of dS_ij q_i,
 *   dv_j = sum over the same (h, i) of P_ij dO_i,
 *   dsink_h = -sum_i exp(sink_h - lse_i) D_i.
 */

/*
 * One unit of work of the backward's key-side kernel (dk, dv): the 128 keys
 * [k0, k0 + 128) of the document [doc_start, doc_end) for kv head g, against
 * n_q query tiles [k0 + 128 t, k0 + 128 t + 128) of every query head of the
 * group.  Keys or queries at or past doc_end are masked.
 */
typedef struct thd_bwd_kv_item {
    int32_t k0, doc_start, doc_end, g;
    int32_t n_q, pad0, pad1, pad2;
} thd_bwd_kv_item;

/* Bytes of device workspace thd_attn_bwd needs for a pack of total_tokens
 * tokens and Hq query heads (two fp32 values per (token, query head)). */
size_t thd_attn_bwd_workspace_bytes(int64_t total_tokens, int Hq);

/*
 * Backward of thd_attn_fwd for head dim 64, 128 or 256.
 *   q, k, v, cu_seqlens, n_docs, Hq, Hkv, D, window, scale, sinks_or_null
 *              exactly as passed to thd_attn_fwd
 *   out        bf16 device [T, Hq, D]: the forward's output
 *   lse        fp32 device [T, Hq]: the forward's log-sum-exp (required)
 *   dout       bf16 device [T, Hq, D]: gradient of the loss w.r.t. out
 *   dq         bf16 device [T, Hq, D]    (written; caller-owned)
 *   dk, dv     bf16 device [T, Hkv, D]   (written; caller-owned)
 *   dsinks_or_null  fp32 device [Hq]: written with dL/dsink when given
 *              (zeros when sinks_or_null is NULL)
 *   workspace  device scratch of at least thd_attn_bwd_workspace_bytes(T, Hq)
 *              bytes, 16-byte aligned, caller-owned; its contents on entry do
 *              not matter and are garbage on return
 *   stream     cudaStream_t to enqueue on
 * Row-major contiguous tensors, 16-byte aligned bf16 pointers, 4-byte
 * aligned fp32 pointers.  The result is deterministic (no atomics).  Argument
 * errors return a negative code before anything is enqueued; kernel stalls
 * are reported by thd_attn_get_error like the forward's.
 */
int thd_attn_bwd(const void* q, const void* k, const void* v,
                 const void* out, const float* lse, const void* dout,
                 const int32_t* cu_seqlens, int n_docs,
                 int Hq, int Hkv, int D, int window, float scale,
                 const float* sinks_or_null,
                 void* dq, void* dk, void* dv, float* dsinks_or_null,
                 void* workspace, size_t workspace_bytes,
                 void* stream);

/*
 * ------------------------------------------------------------------ prologue
 * Q/K prologue of the attention, in place: every query and key head vector
 * is normalised by the parameter-free RMSNorm ("muse_glimmer.model" page,
 * MuseGlimmerScalelessRMSNorm: y = x / sqrt(mean(x^2) + eps), eps default
 * 1e-5) and then, when apply_rope != 0, turned by the split-half rotary
 * embedding (MuseGlimmerRotaryEmbedding, theta default 500000, and
 * apply_rotary_emb): for k < D/2 with a = position * theta^(-2k/D),
 *   out[k] = y[k] cos a - y[k + D/2] sin a,  out[k + D/2] = y[k + D/2] cos a + y[k] sin a.
 *   q          bf16 device [T, Hq, D], overwritten
 *   k          bf16 device [T, Hkv, D], overwritten (may be NULL if Hkv == 0)
 *   cu_seqlens, n_docs  HOST int32 document boundaries as for thd_attn_fwd
 *   positions_or_null   device int32 [T] positions; NULL = each token's
 *              offset inside its document (the position resets at every
 *              document start of the pack)
 *   D          64, 128 or 256;  eps > 0;  theta > 1 (ignored without RoPE)
 * 16-byte aligned tensors.  fp32 arithmetic with the angle reduced in double
 * precision, one bf16 rounding.  With default positions the library keeps a
 * device copy of the last cu_seqlens per device (updated synchronously when
 * it changes).  Returns THD_OK or a negative code before anything is enqueued.
 */
int thd_qk_norm_rope(void* q, void* k, const int32_t* cu_seqlens, int n_docs,
                     const int32_t* positions_or_null, int Hq, int Hkv, int D,
                     float eps, float theta, int apply_rope, void* stream);

/*
 * ---------------------------------------------------------------- sparse MLA
 * Sparse MLA forward ("mistral_large4.attention" page, sparse_mla): for
 * token t and head h, with the valid slots j (0 <= indices[t, j] < Tg; -1 or
 * anything out of range is an invalid slot, ignored),
 *   s_j = scale * <q[t, h, :], kv[indices[t, j], :]>   (576-wide),
 *   latent = sum_j softmax(s)_j kv[indices[t, j], :512],
 *   out[t, h, :] = value_weight[h] @ latent;  a row with no valid slot is zero.
 *   q             bf16 device [T, H, 576] (absorbed queries, last 64 rotary)
 *   kv            bf16 device [Tg, 576] (latent 512 + rotary 64 per key)
 *   indices       int32 device [T, K] (the caller applies document / causal
 *                 boundaries; each valid slot counts once, as given)
 *   value_weight  bf16 device [H, value_dim, 512]
 *   out           bf16 device [T, H, value_dim], written
 *   workspace     device scratch >= thd_sparse_mla_workspace_bytes(T, H, K)
 *                 (the bf16 latent [T, H, 512], the token's valid slots moved
 *                 to the front, their counts), 16-byte aligned
 * Supported: H a multiple of 128, K a multiple of 64 (pad with -1),
 * value_dim 64, 128 or 256 (else THD_ERR_UNSUPPORTED).  Argument errors
 * return before anything is enqueued; kernel stalls are reported by
 * thd_sparse_mla_get_error.
 */
size_t thd_sparse_mla_workspace_bytes(int64_t T, int H, int K);
int thd_sparse_mla_fwd(const void* q, const void* kv, const int32_t* indices,
                       const void* value_weight, int64_t T, int64_t Tg, int H, int K,
                       int value_dim, float scale, void* out,
                       void* workspace, size_t workspace_bytes, void* stream);
/* Synchronises the stream; returns and clears the sparse-MLA status word. */
int thd_sparse_mla_get_error(void* stream);

/* ABI version of this header: (major << 16) | minor. */
int thd_attn_abi_version(void);

/*
 * Self-test of the stall detector that guards every wait in the kernels (no
 * fault, trap or unbounded wait is involved).  Launches two 32-thread blocks
 * on a private stream and waits for them (about 2.5 s): block 0 waits on a
 * barrier that nothing signals, with the kernels' own bounded wait, which
 * gives up after its 2 s limit and records THD_ERR_TIMEOUT in the device
 * status word; block 1 starts waiting 0.5 s later and gives up as soon as it
 * sees that status.  waited_ns (host, [2]) receives how long each block
 * waited (-1 if a wait was satisfied, which never happens).  Afterwards
 * thd_attn_get_error returns THD_ERR_TIMEOUT once.  Returns
 * THD_ERR_INVALID_ARG for a NULL waited_ns (before any CUDA call), an
 * earlier unread status unchanged without launching, THD_ERR_CUDA if the
 * launch fails.
 */
int thd_attn_selftest_stall(int64_t* waited_ns);

#ifdef __cplusplus
}
#endif

#endif /* THD_ATTN_H */
