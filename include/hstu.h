/*
 * hstu.h -- C ABI of the B200 (sm_100a) HSTU attention library.
 *
 * The operation (per user b, head h, query position i, key position j of the user's sequence):
 *
 *   Hist_b      = L_b - num_targets[b]           history length; the last num_targets[b]
 *                                                tokens are the ranking candidates
 *   allowed     = (j <= i and j < Hist_b) or (j == i)
 *                 causal over the history; a candidate sees the whole history and itself,
 *                 never another candidate
 *   s           = sum_c q[i,h,c] * k[j,h,c] + rab[h][bucket(i - j)]
 *   w           = allowed ? s * sigmoid(s) / n_max : 0          (SiLU weighting, no softmax)
 *   o[i,h,:]    = sum_j w * v[j,h,:]
 *   out[i,h,c]  = (o[i,h,c] - mean_i) / sqrt(var_i + ln_eps) * u[i,h,c]
 *                 mean_i, var_i (biased) over all H*D values of token i
 *
 *   bucket(0) = 0;  bucket(d) = min(NB-1, 1 + floor((NB-1) * ln(d) / ln(n_max))) for d >= 1
 *
 * Sources: HSTU swaps softmax for SiLU-based weighting, adds a relative attention bias and
 * gates elementwise before the output projection (aitrends.kr summary of the NVIDIA
 * recsys post, section "HSTU의 순차 모델링"; news.bpdata.com, section "HSTU").  Inputs are
 * jagged per-user sequences; in serving the HSTU attention kernel reads the user's history
 * K/V from a paged GPU KV table and only the new tokens are computed and appended (NVIDIA
 * blog "Deploying an HSTU Generative Recommender with NVIDIA Dynamo-Triton", sections
 * "Why serving large sequential recommenders is hard" and "Benefits").  The pages leave the
 * bias bucketing, the 1/n_max scale, the LayerNorm axis and eps open; the readings above
 * are this library's definition.
 *
 * Conventions for every call
 *   - All tensor arguments are DEVICE pointers, caller-owned, 16-byte aligned, row-major.
 *     Token tensors are [tokens][H][D] (D contiguous).  Pages are [num_pages][H][P][D].
 *   - Element type: params->dtype (HSTU_DTYPE_BF16 or HSTU_DTYPE_FP32) for q, k, v, u,
 *     pages and out.  rab is always fp32 [H][NB].  Index arrays are int32.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL = legacy
 *     default stream).  They do not synchronise and allocate no device memory.
 *   - Scratch lives in a caller-provided workspace of at least hstu_workspace_size()
 *     bytes, 256-byte aligned, zeroed once with hstu_workspace_init() before first use
 *     (hstu_attn_paged_fwd_noalloc uses a built-in scratch instead).
 *     One workspace must not be used by two calls that may run concurrently.
 *   - Host-detectable argument errors return a negative hstu_status_code and launch
 *     nothing.  Errors only the device can see (a page id out of range, lengths that do
 *     not fit, offsets that decrease, a kernel wait that timed out) set bits of a status
 *     word inside the workspace; the offending user's output rows are written as zeros
 *     and no kernel traps.  Read (and clear) that word with hstu_read_status().
 */
#ifndef HSTU_B200_H
#define HSTU_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HSTU_OK = 0,
    HSTU_ERR_INVALID_ARG = -1,  /* null pointer, bad size, misaligned pointer */
    HSTU_ERR_UNSUPPORTED = -2,  /* a shape this build does not implement */
    HSTU_ERR_WORKSPACE = -3,    /* workspace too small or misaligned */
    HSTU_ERR_CUDA = -4,         /* a CUDA runtime/driver call failed */
    HSTU_ERR_SCRATCH_LIMIT = -5, /* hstu_attn_paged_fwd_noalloc: the request does not fit the
                                    library's built-in 8 MiB scratch */
    HSTU_ERR_CACHE_FULL = -6,    /* hstu_cache_prepare: the batch does not fit in the GPU tier
                                    even with every other user evicted */
    HSTU_ERR_OUTPUT_CAPACITY = -7 /* a caller-sized output array of a cache call is too small */
} hstu_status_code;

typedef enum { HSTU_DTYPE_BF16 = 0, HSTU_DTYPE_FP32 = 1 } hstu_dtype;

/* Bits of the device status word (hstu_read_status). */
enum {
    HSTU_DEV_BAD_PAGE = 1u << 0,     /* page_table entry outside [0, num_pages) */
    HSTU_DEV_BAD_LENGTH = 1u << 1,   /* negative length, num_targets > length, a cached or
                                        appended position beyond max_pages_per_user * P,
                                        or a length above the bound passed on the host */
    HSTU_DEV_BAD_NMAX = 1u << 2,     /* a user's total length exceeds n_max */
    HSTU_DEV_TIMEOUT = 1u << 3       /* an in-kernel wait gave up (kernel returned early) */
};

typedef struct {
    int32_t num_heads;            /* H >= 1 */
    int32_t head_dim;             /* D in {32, 64, 128} */
    int32_t dtype;                /* hstu_dtype */
    int32_t num_buckets;          /* NB in [1, 4096] */
    int32_t n_max;                /* >= 1: the 1/n_max weight scale and the bucket range;
                                     every user's total length must be <= n_max */
    int32_t page_size;            /* P (paged calls): 8, 16, 32, 64 or 128 */
    int32_t num_pages;            /* physical pages in the pool (paged calls) */
    int32_t max_pages_per_user;   /* row stride of page_table (paged calls) */
    float ln_eps;                 /* LayerNorm epsilon, e.g. 1e-5 */
    uint32_t flags;               /* HSTU_FLAG_* bits, 0 for none */
    const float* ln_weight;       /* NULL, or a DEVICE fp32 [H*D] LayerNorm scale gamma */
    const float* ln_bias;         /* NULL, or a DEVICE fp32 [H*D] LayerNorm shift beta */
    const float* rab_time;        /* NULL, or a DEVICE fp32 [H][num_time_buckets] second bias */
    const int32_t* timestamps;    /* DEVICE int32, one per token: all tokens (jagged) or the new
                                     tokens (paged, kv_append); used with rab_time / ts_pages */
    int32_t num_time_buckets;     /* with rab_time: 1 .. 64 */
    int32_t* ts_pages;            /* paged calls: NULL, or DEVICE int32 [num_pages][P] timestamps of
                                     the cached tokens, slot for slot beside the K/V pages */
} hstu_attn_params;

/*
 * Bits of hstu_attn_params.flags.
 *
 * HSTU_FLAG_OVERLAP_PREVIOUS (attention calls on the tensor-core path): the attention kernel is
 * launched with programmatic dependent launch, so its set-up -- the work plan from the length
 * arrays, the page-table reads, barrier and tensor-memory set-up -- may run while the kernel
 * enqueued before it on the same stream is still finishing.  It waits for that kernel before it
 * reads q/k/v/u, the pages or rab and before it writes anything, the status word included.  Set the
 * bit only when the kernel enqueued right before the call does not write seq_offsets,
 * page_table, cached_lens, new_lens or num_targets (for example when consecutive layers run back
 * to back, or when the metadata was copied from the host).  Without the bit the call starts
 * after everything before it on the stream has finished.  This is a scheduling choice of this
 * library; the pages describe no such thing.
 */
enum { HSTU_FLAG_OVERLAP_PREVIOUS = 1u << 0, HSTU_FLAG_LN_PER_HEAD = 1u << 1 };

/*
 * Second (time) bias, on the tensor-core path (bf16, D = 128) of the jagged and paged forward
 * calls (hstu_attn_paged_fwd and _noalloc read the cached tokens' timestamps from ts_pages);
 * the backward, the layer call and the CUDA-core paths return HSTU_ERR_UNSUPPORTED when rab_time
 * is set.  hstu_kv_append writes the appended tokens' timestamps into ts_pages when ts_pages and
 * timestamps are set.  HSTU's input is a timestamp-sorted stream
 * of items and actions (aitrends.kr summary, section "HSTU의 순차 모델링"); the pages name a
 * relative attention bias but not its form.  This library's reading of a time-based bias:
 *     s_ij += rab_time[h][tbucket(ts_i - ts_j)],
 *     tbucket(d) = 0 for d <= 0, else min(num_time_buckets - 1, bit length of d)
 * (1 for d = 1, 2 for d in 2..3, 3 for 4..7, ...: log2-spaced, exact in integers).
 */

/*
 * LayerNorm-gate variants of the epilogue (forward calls; the backward pass returns
 * HSTU_ERR_UNSUPPORTED when any is set).  The pages say only that HSTU gates elementwise before
 * the output projection (aitrends.kr summary, section "HSTU의 순차 모델링"); these are options of
 * this library:
 *   HSTU_FLAG_LN_PER_HEAD : mean and variance over each head's D values of a token instead of
 *                           its whole H*D vector;
 *   ln_weight, ln_bias    : out = (xhat * gamma + beta) * u, gamma and beta indexed by h*D + c
 *                           (NULL: gamma = 1, beta = 0).  4-byte aligned device arrays.
 */

/* Library version string. */
const char* hstu_version(void);

/* Human-readable text for an hstu_status_code. */
const char* hstu_error_string(int code);

/*
 * Workspace bytes needed by one call with at most `max_batch` users, `max_tokens` query
 * tokens in total (jagged: all tokens; paged: all new tokens) and at most `max_new`
 * query tokens per user.  The same workspace serves jagged, paged and append calls whose
 * sizes stay within those bounds.  Returns 0 for invalid params.
 */
size_t hstu_workspace_size(const hstu_attn_params* params, int32_t max_batch, int64_t max_tokens,
                           int32_t max_new);

/* Zero the workspace's status word (and nothing else needs zeroing).  Async on stream. */
int hstu_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/*
 * Synchronise `stream`, copy the workspace's device status word to *flags_out (a bitwise
 * OR of HSTU_DEV_* since the last clear) and, when `clear` is nonzero, reset it to 0.
 */
int hstu_read_status(void* workspace, void* stream, uint32_t* flags_out, int clear);

/*
 * Jagged prefill (no cache): every token of every user is a query.
 *   q, k, v, u, out : [total_tokens][H][D]
 *   seq_offsets     : [B+1] int32, seq_offsets[0] = 0, nondecreasing, seq_offsets[B] =
 *                     total_tokens; user b owns rows seq_offsets[b] .. seq_offsets[b+1]-1
 *   num_targets     : [B] int32 candidates at the end of each user's sequence, or NULL (0)
 *   rab             : [H][NB] fp32
 *   max_seqlen      : host-side upper bound on every user's length (sizes the grid; a user
 *                     longer than it sets HSTU_DEV_BAD_LENGTH)
 * Sections cited above: the HSTU attention formula; jagged inputs.
 */
int hstu_attn_jagged_fwd(const hstu_attn_params* params, const void* q, const void* k,
                         const void* v, const void* u, const int32_t* seq_offsets,
                         const int32_t* num_targets, const float* rab, void* out, int32_t B,
                         int64_t total_tokens, int32_t max_seqlen, void* workspace,
                         size_t workspace_bytes, void* stream);

/*
 * Workspace bytes for hstu_attn_jagged_bwd with at most max_tokens tokens: the status block and
 * two fp32 [tokens][H][D] planes (the recomputed o and its gradient).  0 for invalid params.
 */
size_t hstu_workspace_size_bwd(const hstu_attn_params* params, int64_t max_tokens);

/*
 * Backward pass of hstu_attn_jagged_fwd: the gradients of sum(dout * out) with respect to the
 * inputs, for the same arguments and an upstream gradient dout [total_tokens][H][D] (params
 * dtype).  Outputs are fp32 and overwritten:
 *   dq, dk, dv, du : [total_tokens][H][D]
 *   drab           : [H][NB] (zeroed, then accumulated over every allowed pair)
 * With o recomputed by the forward attention kernels, xhat = (o - mean) * rstd per token:
 *   du = xhat * dout;  do = rstd * (dy - mean(dy) - xhat * mean(dy * xhat)),  dy = dout * u
 *   per allowed pair (i, j), s = q_i . k_j + rab[h][bucket(i - j)], sig = sigmoid(s):
 *   ds = (do_i . v_j) * sig * (1 + s * (1 - sig)) / n_max
 *   dq_i += ds k_j,  dk_j += ds q_i,  dv_j += (s * sig / n_max) do_i,  drab[h][bucket] += ds
 * The workspace must hold hstu_workspace_size_bwd(params, total_tokens) bytes (256-byte aligned,
 * zeroed once with hstu_workspace_init); device-detected errors go to its status word as in the
 * forward.  The pages train HSTU but print no backward pass; this is the chain rule applied to
 * the forward definition above (sources as for hstu_attn_jagged_fwd).
 */
int hstu_attn_jagged_bwd(const hstu_attn_params* params, const void* q, const void* k,
                         const void* v, const void* u, const int32_t* seq_offsets,
                         const int32_t* num_targets, const float* rab, const void* dout,
                         float* dq, float* dk, float* dv, float* du, float* drab, int32_t B,
                         int64_t total_tokens, int32_t max_seqlen, void* workspace,
                         size_t workspace_bytes, void* stream);

/*
 * Paged cache hit: only the new tokens of each user are queries.  User b's keys are its
 * cached_lens[b] history tokens, read through page_table[b] (logical position p lives in
 * page page_table[b][p / P], slot p % P), followed by its new_lens[b] new tokens.  New
 * tokens of user b are rows off_b .. off_b + new_lens[b] - 1 of q_new/k_new/v_new/u_new/out,
 * where off_b = new_lens[0] + ... + new_lens[b-1].  The last num_targets[b] new tokens are
 * candidates.  New token t of user b sits at absolute position cached_lens[b] + t.
 *   k_pages, v_pages : [num_pages][H][P][D]
 *   page_table       : [B][max_pages_per_user] int32 (entries past the user's cached length
 *                      are not read)
 *   cached_lens, new_lens : [B] int32;  num_targets : [B] int32 or NULL (0)
 *   total_new        : sum of new_lens (host value; sizes the epilogue)
 *   max_new          : host-side upper bound on new_lens[b]
 * The result does not depend on whether hstu_kv_append of these new tokens ran before.
 * Sources: the paged GPU KV table and "compute only the new tokens" (NVIDIA blog, sections
 * "Why serving large sequential recommenders is hard" and "Benefits").
 */
int hstu_attn_paged_fwd(const hstu_attn_params* params, const void* q_new, const void* k_new,
                        const void* v_new, const void* u_new, const void* k_pages,
                        const void* v_pages, const int32_t* page_table,
                        const int32_t* cached_lens, const int32_t* new_lens,
                        const int32_t* num_targets, const float* rab, void* out, int32_t B,
                        int64_t total_new, int32_t max_new, void* workspace,
                        size_t workspace_bytes, void* stream);

/*
 * hstu_attn_paged_fwd without a workspace argument.  The pages describe no such call: it is
 * a convenience of this library for callers that cannot allocate device memory or keep a
 * buffer of their own across calls -- for example an operator plugin inside a host runtime
 * that owns all device allocations, or code on a path where allocating would stall or
 * fragment a memory pool.
 *
 * Arguments are those of hstu_attn_paged_fwd, with the workspace pair replaced by
 *   flags_out : optional DEVICE pointer (4-byte aligned) that receives, in stream order, the
 *               HSTU_DEV_* bits this call raised (0 = clean); NULL skips the copy.
 *
 * Scratch: a fixed 8 MiB array (8,388,608 bytes) compiled into the library, one per device,
 * laid out like a workspace.  Nothing is allocated: no cudaMalloc, cudaFree or allocating
 * library routine is called.  A request needs 256 + 4*total_new (rounded up to 256) +
 * 4*total_new*H*D bytes for one fp32 partial plane; if that exceeds 8 MiB the call returns
 * HSTU_ERR_SCRATCH_LIMIT and launches nothing (at H*D = 512 that is total_new > 4087).  Spare
 * room holds further partial planes, so the key range may be split over fewer CTAs than
 * with a full workspace; results agree with hstu_attn_paged_fwd up to fp32 summation order.
 *
 * Of the scratch, only the status word must start at zero; each call clears it on `stream`
 * before its kernels run.  All calls on one device share the array, so two calls that may
 * run concurrently (different streams, different host threads) race and corrupt each
 * other's results: order them on one stream, or use hstu_attn_paged_fwd with separate
 * workspaces.
 *
 * The first call on each device and CUDA context does a one-time set-up: it looks up the
 * array's device address (cudaGetSymbolAddress), which may load the library's device code onto
 * that device; after a device reset or under another context the address is looked up again.
 * Make the first call before any stream capture begins.
 */
int hstu_attn_paged_fwd_noalloc(const hstu_attn_params* params, const void* q_new,
                                const void* k_new, const void* v_new, const void* u_new,
                                const void* k_pages, const void* v_pages,
                                const int32_t* page_table, const int32_t* cached_lens,
                                const int32_t* new_lens, const int32_t* num_targets,
                                const float* rab, void* out, int32_t B, int64_t total_new,
                                int32_t max_new, uint32_t* flags_out, void* stream);

/*
 * Append new history tokens into the pages (the KV cache's "append"; NVIDIA blog, section
 * "Why serving large sequential recommenders is hard").  For user b the first
 * new_lens[b] - num_targets[b] rows of its new tokens (rows off_b.. of k_new/v_new, off_b
 * as in hstu_attn_paged_fwd) are copied to logical positions cached_lens[b] + t; candidates
 * are never appended.  A raw, bit-exact copy of K and V rows.  cached_lens is not modified:
 * the caller advances it afterwards.
 *   k_pages, v_pages : [num_pages][H][P][D], written
 *   k_new, v_new     : [total_new][H][D]; a user whose rows would pass total_new is skipped
 *                      and flagged (HSTU_DEV_BAD_LENGTH)
 *   max_new          : host-side upper bound on new_lens[b]
 * Tokens whose page id is invalid or whose position is beyond max_pages_per_user * P are
 * skipped and flagged (HSTU_DEV_BAD_PAGE / HSTU_DEV_BAD_LENGTH).  The workspace is used
 * only for that status word.
 */
int hstu_kv_append(const hstu_attn_params* params, void* k_pages, void* v_pages,
                   const int32_t* page_table, const void* k_new, const void* v_new,
                   const int32_t* cached_lens, const int32_t* new_lens,
                   const int32_t* num_targets, int32_t B, int64_t total_new, int32_t max_new,
                   void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------------------
 * The HSTU layer around the attention.  The pages say that HSTU replaces softmax attention with
 * SiLU weighting, adds a relative attention bias and gates elementwise before the output
 * projection (aitrends.kr summary, section "HSTU의 순차 모델링"; news.bpdata.com, section
 * "HSTU"); they do not write the projections out.  This library's reading, with no bias vectors,
 * no residual and no input normalisation:
 *
 *   q, k, v, u = the four H*D-column blocks, in that order, of SiLU(x W_qkvu^T), rounded to bf16
 *   g          = LayerNorm(attention(q, k, v)) * u      (hstu_attn_paged_fwd, bf16 out)
 *   y          = g W_out^T
 * ------------------------------------------------------------------------------------------ */

/*
 * y = act(x w^T) on tensor cores: x [M][K], w [N][K] (one output feature per row), y [M][N],
 * all bf16 DEVICE arrays, 16-byte aligned; fp32 accumulation; act = 0 (none) or 1 (SiLU, applied
 * before rounding).  N a multiple of 128, K a multiple of 64.  The workspace (>= 256 bytes,
 * 256-byte aligned) receives HSTU_DEV_TIMEOUT if an in-kernel wait gave up.  Async on stream.
 */
int hstu_linear_fwd(const void* x, const void* w, void* y, int64_t M, int32_t N, int32_t K, int32_t activation,
                    void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes of hstu_layer_paged_fwd: the paged call's workspace plus five bf16
 * [max_tokens][H*D] arrays (q, k, v, u and the gated attention output).  0 if unsupported. */
size_t hstu_workspace_size_layer(const hstu_attn_params* params, int32_t d_model, int32_t max_batch,
                                 int64_t max_tokens, int32_t max_new);

/*
 * One HSTU layer on the paged cache hit, for the new tokens of each user:
 *   x_new  [total_new][d_model]   the layer input of the new tokens (rows as in
 *                                 hstu_attn_paged_fwd: user b's rows start at off_b)
 *   w_qkvu [4*H*D][d_model], w_out [d_model][H*D]   bf16 weights, one output feature per row
 *   y      [total_new][d_model]   the layer output
 * The call computes q, k, v, u, appends the new history tokens' k and v to the user's pages
 * (as hstu_kv_append; the caller advances cached_lens afterwards), runs the paged attention
 * with its LayerNorm gate and the output projection.  Supported: bf16, D = 128, H*D and d_model
 * multiples of 128.  The workspace holds hstu_workspace_size_layer() bytes.
 */
int hstu_layer_paged_fwd(const hstu_attn_params* params, int32_t d_model, const void* x_new, const void* w_qkvu,
                         const void* w_out, void* k_pages, void* v_pages, const int32_t* page_table,
                         const int32_t* cached_lens, const int32_t* new_lens, const int32_t* num_targets,
                         const float* rab, void* y, int32_t B, int64_t total_new, int32_t max_new, void* workspace,
                         size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------------------
 * KV cache management around append: a two-tier paged cache (GPU pages and pinned host pages)
 * with LRU eviction, onboard and offload, and compaction.
 *
 * The pages describe the serving path's cache manager (NVIDIA blog "Deploying an HSTU
 * Generative Recommender with NVIDIA Dynamo-Triton", section "Why serving large sequential
 * recommenders is hard"): the GPU cache is a paged KV table supporting lookup, allocate, append
 * and evict; when GPU space runs short, old users are evicted by an LRU-like policy; host
 * storage is a further tier; the exported path has cache-aware operations for lookup,
 * allocate, onboard, append and offload.  The pages give no algorithm; this library's
 * definition is:
 *
 *   - A user (int64 id) is resident in at most one tier, with a stored length n (tokens),
 *     ceil(n / P) pages of that tier in logical order, and a stamp: the number of the last
 *     hstu_cache_prepare call that had the user in its batch.
 *   - Free pages are handed out lowest id first.
 *   - hstu_cache_prepare(ids, append) serves one batch (distinct ids).  With n_b the stored
 *     length (0 on a miss), user b needs ceil((n_b + append_b) / P) GPU pages (at most
 *     max_pages_per_user).  If the free GPU pages do not cover the batch's extra pages, GPU
 *     residents outside the batch are evicted oldest first -- ordered by (stamp, user id) --
 *     until they do (if even evicting all of them would not, the call fails with
 *     HSTU_ERR_CACHE_FULL).  Evicted users are offloaded to the host tier newest first; a
 *     victim that does not fit in the free host pages takes the pages of host residents
 *     outside the batch that are older than itself, oldest first; if even all of those would
 *     not make room, the victim is dropped.  Then, in batch order: GPU residents get their
 *     extra pages, host residents of the batch are onboarded into fresh GPU pages (their
 *     host pages are freed at the end of the call), misses get fresh pages.  Each batch
 *     user's stamp becomes the call's number and its stored length n_b + append_b: the caller
 *     appends those tokens (hstu_kv_append, or the prefill's append on a miss) after the copies.
 *   - hstu_cache_compact moves GPU pages so that the residents occupy pages [0, live): the
 *     live pages at ids >= live, ascending, go to the free ids < live, ascending.
 *
 * The manager is host code: it owns no device memory and launches nothing.  It returns page
 * rows and lists of (from, to) page pairs; hstu_kv_page_copy moves the pages.  For one
 * prepare call the caller runs, on one stream and in this order: the offload copy (GPU pool ->
 * host pool), the onboard copy (host pool -> GPU pool), then anything that writes the batch's
 * pages or reads them (appends, attention).  Evicted and dropped users' GPU pages may be
 * reused by the same batch, so the offload copy must run first.
 *
 * All cache calls take host pointers, are synchronous, and are safe to call from several
 * threads (each cache has its own lock).  A failed call changes nothing.
 * ------------------------------------------------------------------------------------------ */

typedef struct hstu_kv_cache hstu_kv_cache;

enum { HSTU_TIER_MISS = 0, HSTU_TIER_GPU = 1, HSTU_TIER_HOST = 2 };

/*
 * Create a cache of gpu_pages GPU pages and host_pages host pages (host_pages may be 0: no host
 * tier, evicted users are dropped), page_size P >= 1 tokens per page, at most
 * max_pages_per_user pages per user (the row length of the page rows it returns).
 * *out receives the handle; free it with hstu_cache_destroy.
 */
int hstu_cache_create(int32_t gpu_pages, int32_t host_pages, int32_t page_size,
                      int32_t max_pages_per_user, hstu_kv_cache** out);
void hstu_cache_destroy(hstu_kv_cache* cache);

/* Lookup: for n ids, tier_out[i] = HSTU_TIER_* and len_out[i] = stored length (0 on a miss).
 * Changes nothing (stamps included). */
int hstu_cache_lookup(hstu_kv_cache* cache, const int64_t* user_ids, int32_t n, int32_t* tier_out,
                      int32_t* len_out);

/*
 * Allocate for one batch of B distinct users that will append append_lens[b] >= 0 tokens each
 * (see the definition above).  Outputs (host arrays):
 *   tier_before_out [B]       tier of each user before the call (MISS, GPU or HOST)
 *   cached_lens_out [B]       stored length before the call (0 on a miss): the paged
 *                             attention's cached_lens, and where the append starts
 *   page_table_out  [B][max_pages_per_user]  the user's GPU pages, -1 past them: the page
 *                             table of hstu_attn_paged_fwd and hstu_kv_append
 *   offload_pairs_out [capacity][2]  (GPU page, host page) pairs, *n_offload of them
 *   onboard_pairs_out [capacity][2]  (host page, GPU page) pairs, *n_onboard of them
 *   dropped_out [capacity]    users that left the cache in this call (victims that did not
 *                             fit in the host tier, host residents that made room), in
 *                             the order they were dropped
 * Errors: HSTU_ERR_INVALID_ARG (null pointer, B < 0, repeated id, negative append, a user
 * needing more than max_pages_per_user pages), HSTU_ERR_CACHE_FULL, HSTU_ERR_OUTPUT_CAPACITY
 * (an output list longer than its capacity; the counts hold the lengths needed).
 */
int hstu_cache_prepare(hstu_kv_cache* cache, const int64_t* user_ids, const int32_t* append_lens,
                       int32_t B, int32_t* tier_before_out, int32_t* cached_lens_out,
                       int32_t* page_table_out, int32_t* offload_pairs_out,
                       int32_t offload_capacity, int32_t* n_offload, int32_t* onboard_pairs_out,
                       int32_t onboard_capacity, int32_t* n_onboard, int64_t* dropped_out,
                       int32_t dropped_capacity, int32_t* n_dropped);

/* Evict one user from whichever tier holds it; *tier_out = that tier (MISS if none). */
int hstu_cache_evict(hstu_kv_cache* cache, int64_t user_id, int32_t* tier_out);

/* Compaction of the GPU tier: *n_moves (from, to) pairs into move_pairs_out [capacity][2]
 * (at most gpu_pages are ever needed); sources and destinations are disjoint, so one
 * hstu_kv_page_copy within the GPU pool performs them.  Fetch page rows again afterwards. */
int hstu_cache_compact(hstu_kv_cache* cache, int32_t* move_pairs_out, int32_t capacity,
                       int32_t* n_moves);

/* Current GPU page rows of n users, [n][max_pages_per_user]; all -1 for a user not on the GPU. */
int hstu_cache_page_rows(hstu_kv_cache* cache, const int64_t* user_ids, int32_t n, int32_t* rows_out);

/* stats_out[5] = free GPU pages, free host pages, users on the GPU, users on the host,
 * number of successful prepare calls. */
int hstu_cache_stats(hstu_kv_cache* cache, int64_t* stats_out);

/*
 * Copy whole pages: for i < n_pairs, page pairs[2i] of (src_k, src_v) to page pairs[2i+1] of
 * (dst_k, dst_v), K and V alike; a page is H * P * D elements of params->dtype.  This is the
 * onboard (host pool -> GPU pool), offload (GPU pool -> host pool) and compaction (within the
 * GPU pool) copy of the cache above.
 *   src_k, src_v : [src_pages][H][P][D];  dst_k, dst_v : [dst_pages][H][P][D]
 *   pairs        : [n_pairs][2] int32
 * Every pointer must be device memory of the current device or pinned host memory that the
 * device can address (allocated with cudaHostAlloc/cudaMallocHost, or registered), 16-byte
 * aligned; the call checks both ends of each pool and of the pair array and returns
 * HSTU_ERR_INVALID_ARG otherwise.  Destination pages must be distinct, and within one pool no
 * page may be both a source and a destination (the pairs run in any order).  A pair with a
 * page id out of range is skipped and sets HSTU_DEV_BAD_PAGE in the workspace's status word
 * (the workspace is used for nothing else).  Asynchronous on stream.
 */
int hstu_kv_page_copy(const hstu_attn_params* params, const void* src_k, const void* src_v,
                      int32_t src_pages, void* dst_k, void* dst_v, int32_t dst_pages,
                      const int32_t* pairs, int32_t n_pairs, void* workspace,
                      size_t workspace_bytes, void* stream);

/*
 * Test-only fault injection for the time-out path of the tensor-core attention kernels (bf16,
 * D = 128, jagged and paged).  Every wait of one role of a CTA for another (a copy landing, a
 * product completing, a buffer being released) gives up after a limit, sets HSTU_DEV_TIMEOUT
 * in the status word and makes the CTA's other roles give up too; each role then waits for its
 * own copies and products still in flight (with the full 2 s limit), tensor memory is released
 * and the kernel returns.  The rows of that call are not valid; the next call is unaffected.
 *   kind = HSTU_INJECT_STALL_V : from now on the V-tile producer issues no load, so the first
 *          wait on a V tile runs out after wait_limit_ns (1 ms .. 2 s) instead of 2 s;
 *   kind = 0                   : back to normal calls (wait_limit_ns ignored).
 * Process-wide; calls already enqueued keep the setting they were launched with.  Nothing
 * faults, traps or waits without a limit.  Not for production use.
 */
enum { HSTU_INJECT_STALL_V = 1 };
int hstu_test_inject(uint32_t kind, uint64_t wait_limit_ns);

/*
 * Copy whole timestamp pages ([pages][page_size] int32) for i < n_pairs: page pairs[2i] of src to
 * page pairs[2i+1] of dst -- the timestamp side of an onboard, offload or compaction move made by
 * hstu_kv_page_copy.  Pools may be device memory or pinned host memory, as there; page_size a
 * multiple of 4; bad page ids are skipped and set HSTU_DEV_BAD_PAGE in the workspace.
 */
int hstu_ts_page_copy(const int32_t* src, int32_t src_pages, int32_t* dst, int32_t dst_pages, int32_t page_size,
                      const int32_t* pairs, int32_t n_pairs, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Copy `bytes` bytes from src to dst with the GPU's SMs, as one kernel on `stream`: the upload of
 * a call's inputs from pinned host memory (or the download of its outputs) done by the device
 * reading and writing host memory over the host link, instead of a DMA copy.  Either pointer
 * may be device memory of the current device or pinned host memory the device addresses
 * (cudaHostAlloc/cudaMallocHost or registered); both 16-byte aligned; the ranges must not
 * overlap.  Both ends of both ranges are checked before the launch (HSTU_ERR_INVALID_ARG
 * otherwise).  Asynchronous; the caller keeps the host buffer alive and unchanged until the
 * stream has passed the copy.  A transport choice of this library (the pages describe none).
 */
int hstu_host_copy(void* dst, const void* src, size_t bytes, void* stream);

/*
 * The library's own bucket table: table_out[d] = bucket(d) for d in [0, n), computed on the
 * device in double precision (the function that the attention kernels use).  table_out is
 * a device int32 array of n entries.  Exposed so that tests can compare it with an
 * independent implementation.
 */
int hstu_bucket_table(const hstu_attn_params* params, int32_t n, int32_t* table_out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* HSTU_B200_H */
