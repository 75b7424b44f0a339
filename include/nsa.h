/*
 * nsa.h - C ABI of the B200 (sm_100a) Native Sparse Attention forward pass.
 *
 * What is computed (for every query token t of every sequence, every query
 * head h of KV group g = h / G, G = Hq / Hkv; positions restart at 0 in each
 * sequence; s = softmax_scale):
 *   1. compression ("DeepSeek NSA config.toml" page, section 3,
 *      compress_block_size; "DeepSeek NSA in manufacturing" page, section on
 *      what dynamic sparsity sparsifies: one learned linear map over each
 *      flattened key block), blocks of l tokens at a stride of d:
 *        Kc[i,g,:] = W_K[g] . vec(K[i*d .. i*d+l-1, g, :]),  Vc likewise,
 *      vec index p*D + c (token p of the block, channel c), stored in bf16;
 *   2. compressed branch (config page, section 1): softmax over the complete
 *      blocks i (i*d + l - 1 <= t) of s * q_h . Kc[i,g]; O_cmp = sum p Vc;
 *   3. block scores (manufacturing page, same section: coarse attention of
 *      the query to every compressed block ranks the blocks): selection
 *      block j covers tokens [j*l', j*l' + l' - 1] and
 *        S[t,g,j] = sum over the G heads of group g of the probabilities
 *                   p_h[i] of every complete compressed block i that
 *                   overlaps it
 *      (with l == d == l' that is the sum over heads of p_h[j]);
 *   4. selection (config page, section 3, select_top_k): the top_n blocks
 *      among j*l' <= t by (score descending, index ascending); the block
 *      holding t competes with whatever score step 3 gives it (0 when no
 *      complete compressed block overlaps it);
 *   5. selected branch (config page, section 3, select_block_size): softmax
 *      attention over the tokens u <= t of the chosen blocks;
 *   6. window branch (config page, section 3, sliding_window): softmax
 *      attention over u in [max(0, t-w+1), t];
 *   7. gate (config page, sections 1 and 3, gate_type learned):
 *        out = g_cmp * O_cmp + g_slc * O_slc + g_win * O_win,
 *      with the gate values given per token and head (post-sigmoid).
 * An empty branch contributes 0.  This version supports compression blocks
 * l in {32, 64} with a stride d in {16, 32, 64} that divides l, selection
 * blocks l' in {32, 64}, head_dim in {64, 128}, G in {1, 2, 4, 8, 16},
 * 1 <= top_n <= min(32, 1024 / l') (a token's selected keys fit in 8 chunks
 * of 128), window >= 1; other valid geometries return NSA_ERR_UNSUPPORTED.
 *
 * Memory: every pointer except the plan is caller-owned device memory (bf16
 * is passed as raw 16-bit storage).  The library never allocates device
 * memory in nsa_prefill / nsa_decode; scratch lives in the caller's workspace
 * (nsa_workspace_size).  Device pointers must be 16-byte aligned; row strides
 * are the dense strides implied by the shapes.
 *
 * Errors: every call returns an nsa_status.  Arguments are validated on the
 * host before anything is launched; on error nothing is launched.  Launches
 * are asynchronous on `stream` (a cudaStream_t; NULL is the legacy default
 * stream) and never synchronise the host.  Faults found on the device (a
 * bounded wait that gave up, inconsistent sequence lengths) are recorded in a
 * status word inside the workspace, read back with nsa_read_device_status.
 * There is no fallback path: an unsupported geometry is an error.
 */
#ifndef NSA_B200_H
#define NSA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NSA_OK = 0,
  NSA_ERR_INVALID_ARG = 1,    /* null pointer, negative size, inconsistent shape */
  NSA_ERR_UNSUPPORTED = 2,    /* valid NSA geometry this build does not implement */
  NSA_ERR_MISALIGNED = 3,     /* a device pointer is not 16-byte aligned */
  NSA_ERR_WORKSPACE = 4,      /* workspace missing or smaller than nsa_workspace_size */
  NSA_ERR_CUDA = 5,           /* a CUDA runtime call or launch failed */
  NSA_ERR_DEVICE_TIMEOUT = 6, /* device status: a bounded wait gave up */
  NSA_ERR_DEVICE_BAD_INPUT = 7 /* device status: sequence lengths out of range */
} nsa_status;

typedef enum { NSA_OUT_BF16 = 0, NSA_OUT_F32 = 1 } nsa_out_dtype;
typedef enum {
  NSA_MODE_PREFILL = 0,      /* nsa_prefill, nsa_prefill_noalloc */
  NSA_MODE_DECODE = 1,       /* nsa_decode */
  NSA_MODE_BLOCK_SELECT = 2,        /* nsa_block_select_prefill */
  NSA_MODE_BLOCK_SELECT_DECODE = 3  /* nsa_block_select_decode */
} nsa_mode;

typedef struct {
  int head_dim;          /* D = d_k = d_v: 64 or 128 */
  int num_q_heads;       /* Hq */
  int num_kv_heads;      /* Hkv; Hq / Hkv must be 1, 2, 4, 8 or 16 */
  int cmp_block;         /* l  (compress_block_size) */
  int cmp_stride;        /* d  (compression stride: 16, 32 or 64, dividing l) */
  int sel_block;         /* l' (select_block_size: 32 or 64) */
  int top_n;             /* n  (select_top_k) */
  int window;            /* w  (sliding_window) */
  float softmax_scale;   /* s; 0 selects 1/sqrt(D) */
  int max_batch;         /* upper bound on sequences per call */
  int max_seqlen;        /* upper bound on one sequence's length (prefill) or
                            on the cache capacity (decode) */
  int max_total_tokens;  /* upper bound on packed tokens per prefill call */
  int out_dtype;         /* nsa_out_dtype of `out` */
} nsa_params;

typedef struct nsa_plan_s* nsa_plan_t;

/* Validates `params` and creates a plan (host memory only, no GPU work).
 * Returns NSA_ERR_INVALID_ARG / NSA_ERR_UNSUPPORTED without creating one.
 * A plan is immutable; it may be shared by calls on several streams as long
 * as each concurrent call has its own workspace. */
int nsa_plan_create(const nsa_params* params, nsa_plan_t* plan_out);
/* The same call under its short name. */
int nsa_plan(const nsa_params* params, nsa_plan_t* plan_out);
void nsa_plan_destroy(nsa_plan_t plan);

/* Bytes of device workspace a call of `mode` needs under the plan's bounds
 * (0 for an invalid plan or mode). */
size_t nsa_workspace_size(nsa_plan_t plan, int mode);

/* Named regions of the prefill workspace, for inspection by tests and
 * debugging.  Valid after a completed nsa_prefill on that workspace (or, for
 * mode NSA_MODE_BLOCK_SELECT, nsa_block_select_prefill: STATUS, SCORES, SEL). */
typedef enum {
  NSA_WS_STATUS = 0,  /* int32 status word */
  NSA_WS_O_CMP = 1,   /* fp32 [T_total, Hq, D] compressed-branch output */
  NSA_WS_LSE = 2,     /* fp32 [T_total, Hq] compressed-branch log-sum-exp (natural log) */
  NSA_WS_SCORES = 3,  /* fp32 [T_total, Hkv, (max_seqlen - l) / d + 1] compressed-block
                         scores (sum over the group's heads of the compressed softmax
                         probabilities); entry i of row t is defined for i < the
                         number of complete compressed blocks */
  NSA_WS_SEL = 4,     /* int32 [T_total, Hkv, top_n] selection (when sel_idx is NULL) */
  NSA_WS_WIN = 5,     /* fp32 [T_total, Hq, D] window-branch output times its gate */
  NSA_WS_SEL_SCORES = 6 /* fp32 [T_total, Hkv, max_seqlen / l' + 1] selection-block scores
                           (entry j of row t defined for j <= t / l'); empty (0 bytes)
                           when l == d == l', where NSA_WS_SCORES already holds them */
} nsa_ws_region;
int nsa_workspace_region(nsa_plan_t plan, int mode, int region, size_t* offset, size_t* bytes);

/* Rows of the packed compressed-KV output of a prefill over `total_tokens`
 * tokens: floor(total_tokens / d), an upper bound on the sum over the
 * sequences of their complete compressed blocks, (T_b - l) / d + 1. */
int nsa_cmp_rows(nsa_plan_t plan, int total_tokens);

/*
 * Causal prefill over a packed batch (steps 1-7 for every token).
 *   q          [T_total, Hq, D]  bf16
 *   k, v       [T_total, Hkv, D] bf16
 *   gates      [T_total, Hq, 3]  fp32, order (cmp, slc, win)
 *   w_k, w_v   [Hkv, D, l*D]     fp32 compressor weights
 *   cu_seqlens [batch + 1]       int32 device, cu_seqlens[0] = 0, non-decreasing,
 *                                cu_seqlens[batch] = total_tokens, each length <= max_seqlen
 *   out        [T_total, Hq, D]  bf16 or fp32 (plan out_dtype)
 *   k_cmp, v_cmp [nsa_cmp_rows, Hkv, D] bf16, written: the compressed keys and
 *              values of sequence b occupy rows sum_{b'<b} C(T_b') onward,
 *              C(T) = (T - l) / d + 1 complete blocks (0 when T < l)
 *   sel_idx    [T_total, Hkv, top_n] int32 or NULL: selected block indices of
 *              each token, ascending, -1 padded
 *   workspace  >= nsa_workspace_size(plan, NSA_MODE_PREFILL) bytes, 256-byte aligned
 */
int nsa_prefill(nsa_plan_t plan, const void* q, const void* k, const void* v,
                const float* gates, const float* w_k, const float* w_v,
                const int* cu_seqlens, int batch, int total_tokens, void* out, void* k_cmp,
                void* v_cmp, int* sel_idx, void* workspace, size_t workspace_bytes,
                void* stream);

/*
 * nsa_prefill without a caller workspace, for callers that cannot allocate
 * device memory (code running under a memory pool it does not own, code that
 * must avoid the device synchronisation an allocation can cause, plugins that
 * only receive tensor pointers).  The web pages on NSA have no counterpart of
 * this entry point: it is a deployment convenience of this library.
 * Arguments and results are those of nsa_prefill minus the workspace; the
 * scratch is one file-scope device array of 32 MiB per GPU, held by every GPU
 * that loads the library until the process exits.  Returns
 * NSA_ERR_WORKSPACE when nsa_workspace_size(plan, NSA_MODE_PREFILL) exceeds
 * 32 MiB.  It calls no allocator.  The first call on each device looks up the
 * array's device address (cudaGetSymbolAddress) with that device current:
 * make that first call before any stream capture.  All calls share the array
 * and it keeps the last call's contents (the status word is cleared by every
 * call); calls that overlap on the GPU race on it and must not be issued.
 * The cached address belongs to the device's current context: after a
 * cudaDeviceReset (or any reset of the primary context) this entry point
 * must not be used again in the same process.  Device-side faults of a call
 * land in the array's status word: read them with
 * nsa_noalloc_read_device_status.
 */
int nsa_prefill_noalloc(nsa_plan_t plan, const void* q, const void* k, const void* v,
                        const float* gates, const float* w_k, const float* w_v,
                        const int* cu_seqlens, int batch, int total_tokens, void* out,
                        void* k_cmp, void* v_cmp, int* sel_idx, void* stream);

/* nsa_read_device_status for the static array of nsa_prefill_noalloc:
 * synchronises `stream`, returns the status word of the last no-allocation
 * call on the current device (NSA_OK or NSA_ERR_DEVICE_*) and clears it.
 * Allocates nothing.  Returns NSA_ERR_CUDA if the stream failed or the
 * array's address cannot be found. */
int nsa_noalloc_read_device_status(void* stream);

/*
 * One decode step for a batch of sequences (steps 1-7 for the newest token of
 * each sequence, which the caller has already written into the caches).
 *   q           [batch, Hq, D]             bf16, query of the newest token
 *   k_cache, v_cache [batch, cache_capacity, Hkv, D] bf16
 *   k_cmp_cache, v_cmp_cache [batch, cache_capacity / d, Hkv, D] bf16: the
 *               compressed blocks of every complete block before the newest
 *               token; when the newest token completes a block (len >= l and
 *               (len - l) % d == 0) that block, number (len - l) / d, is
 *               compressed here from the cache and written back
 *   seqlens     [batch] int32 device, tokens in the cache including the newest,
 *               1 <= len <= cache_capacity; cache rows at or past len are never
 *               read
 *   cache_capacity  multiple of l and of l', <= plan max_seqlen, holding at
 *               most 4096 compressed blocks (all of a query's compressed
 *               scores are kept on chip: 262144 tokens at l = d = 64); the
 *               window must be at most 1024 tokens
 *   gates       [batch, Hq, 3] fp32
 *   w_k, w_v    [Hkv, D, l*D] fp32
 *   out         [batch, Hq, D] bf16 or fp32
 *   sel_idx     [batch, Hkv, top_n] int32 or NULL
 *   workspace   >= nsa_workspace_size(plan, NSA_MODE_DECODE) bytes (per
 *               (sequence, KV group): the selection, the compressed branch's
 *               probabilities and the fp32 partial results the last kernel
 *               merges; about 6 MB for 32 sequences of 64k tokens)
 * Three launches: the compression of a block the newest token completed,
 * then two kernels that split every (sequence, group) into units of about
 * 128-256 KB of cache reads; the last unit of each pair merges the branches.
 */
int nsa_decode(nsa_plan_t plan, const void* q, const void* k_cache, const void* v_cache,
               void* k_cmp_cache, void* v_cmp_cache, const int* seqlens, int batch,
               int cache_capacity, const float* gates, const float* w_k, const float* w_v,
               void* out, int* sel_idx, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Select-only block attention (MoBA style) over a packed batch: causal, each
 * query attends to its own block of l' tokens and to the n - 1 best-routed
 * complete blocks before it, with one softmax per head and no other branch.
 * "NSA vs MoBA" page (gtnt.cn/news/122266), section 1: the sequence is cut
 * into blocks and a gate routes every query to a few of them, like a mixture
 * of experts.  Readings of that description (the page gives no formula):
 *   - the routing key of block j of a sequence is the mean of its l' keys,
 *     rounded once to bf16 (nearest even);
 *   - the routing score of block j for token t and KV group g is the sum over
 *     the group's query heads of q_t,h . key_j (shared by the group);
 *   - the n - 1 highest scores among the blocks j < t / l' are taken (ties to
 *     the lower index; all of them when there are at most n - 1), plus t's own
 *     block t / l', whose keys u <= t are attended;
 *   - scale as in nsa_prefill (plan softmax_scale, else 1/sqrt(D)).
 * The plan's sel_block (l'), top_n (n, the own block included), head
 * geometry, scale and out_dtype are used; cmp_block, cmp_stride and window
 * are not.
 *   q          [T_total, Hq, D]  bf16
 *   k, v       [T_total, Hkv, D] bf16
 *   cu_seqlens [batch + 1]       int32 device, as in nsa_prefill
 *   out        [T_total, Hq, D]  bf16 or fp32 (plan out_dtype)
 *   k_mean     [nsa_block_rows, Hkv, D] bf16, written: the routing keys of
 *              sequence b's floor(T_b / l') complete blocks follow those of the
 *              sequences before it; remaining rows are zero-filled
 *   sel_idx    [T_total, Hkv, top_n] int32 or NULL: attended blocks of each
 *              token, ascending (the own block last), -1 padded
 *   workspace  >= nsa_workspace_size(plan, NSA_MODE_BLOCK_SELECT) bytes,
 *              256-byte aligned (regions NSA_WS_STATUS, NSA_WS_SCORES = fp32
 *              [T_total, Hkv, max_seqlen / l'] routing scores, entry j of row t
 *              defined for j < t / l', and NSA_WS_SEL)
 * Returns the same codes as nsa_prefill; device-side faults land in the
 * workspace status word (nsa_read_device_status).  Five launches.
 */
int nsa_block_select_prefill(nsa_plan_t plan, const void* q, const void* k, const void* v,
                             const int* cu_seqlens, int batch, int total_tokens, void* out,
                             void* k_mean, int* sel_idx, void* workspace, size_t workspace_bytes,
                             void* stream);

/*
 * One decode step of select-only block attention for a batch of sequences:
 * the newest token of each sequence (already written into the caches)
 * attends to its own block and to the n - 1 best-routed complete blocks
 * before it, with the readings of nsa_block_select_prefill.
 *   q            [batch, Hq, D]             bf16, query of the newest token
 *   k_cache, v_cache [batch, cache_capacity, Hkv, D] bf16
 *   k_mean_cache [batch, cache_capacity / l', Hkv, D] bf16: the routing keys
 *                of every complete block before the newest token; when the
 *                newest token completes its block (len % l' == 0) that
 *                block's routing key is computed here and written back (it is
 *                routed from the next step on)
 *   seqlens      [batch] int32 device, 1 <= len <= cache_capacity
 *   cache_capacity  multiple of l', <= plan max_seqlen, at most 4096 blocks
 *   out          [batch, Hq, D] bf16 or fp32 (plan out_dtype)
 *   sel_idx      [batch, Hkv, top_n] int32 or NULL (ascending, own block last)
 *   workspace    >= nsa_workspace_size(plan, NSA_MODE_BLOCK_SELECT_DECODE)
 * Three launches: the routing key of a completed block, the routing and
 * top-n kernel, and the selected-block kernel with the merge.
 */
int nsa_block_select_decode(nsa_plan_t plan, const void* q, const void* k_cache,
                            const void* v_cache, void* k_mean_cache, const int* seqlens, int batch,
                            int cache_capacity, void* out, int* sel_idx, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * Token-level top-k attention (DSA style) over a packed batch.  "DeepSeek
 * V3.2-Exp sparse attention" page (bjdmk.com.cn/news/5181035), sections 1 and
 * 3: a light indexer with a ReLU scores every earlier token of a query and
 * the top_k of them take part in the main attention.  Readings (the page
 * gives no formula): the index score of token s <= t for query t is
 * sum_j w_index[t, j] * ReLU(q_index[t, j] . k_index[s]); the top_k tokens
 * by that score (ties to the lower index; all of them when t + 1 <= top_k)
 * are shared by every query head; each head attends (one softmax, the plan's
 * scale) to the keys and values of its KV group at those tokens.  The page's
 * fp8 indexer is a precision choice not made here: the indexer runs on bf16
 * inputs with fp32 accumulation.
 *   q, k, v     as in nsa_prefill (the plan's heads and head dim; Hq <= 64,
 *               Hkv <= 4 at D = 128, Hkv <= 8 at D = 64)
 *   q_index     [T_total, index_heads, index_dim] bf16 (index_heads 1, 2, 4,
 *               8 or 16; index_dim 64 or 128)
 *   w_index     [T_total, index_heads] fp32 per-token head weights
 *   k_index     [T_total, index_dim] bf16
 *   top_k       1 <= top_k <= plan max_seqlen
 *   out         [T_total, Hq, D] bf16 or fp32 (plan out_dtype)
 *   sel_idx     [T_total, top_k] int32 or NULL: chosen tokens (positions in
 *               the sequence), ascending, -1 padded
 *   workspace   >= nsa_token_select_workspace_size(plan, top_k) bytes,
 *               256-byte aligned: the index scores fp32 [T_total, S] with
 *               S = max_seqlen rounded up to a multiple of 4 (entry s of row
 *               t defined for s <= t) and the selection
 * Four launches: metadata, index scores (tcgen05), top-k (a radix select,
 * one CTA per row), attention over the chosen tokens (mma.sync tensor
 * cores).  Plan cmp_block, cmp_stride, sel_block, top_n
 * and window are not used.
 */
int nsa_token_select_prefill(nsa_plan_t plan, const void* q, const void* k, const void* v,
                             const void* q_index, const float* w_index, const void* k_index,
                             int index_heads, int index_dim, int top_k, const int* cu_seqlens,
                             int batch, int total_tokens, void* out, int* sel_idx,
                             void* workspace, size_t workspace_bytes, void* stream);
/* Workspace bytes of nsa_token_select_prefill for `top_k` (0 when invalid). */
size_t nsa_token_select_workspace_size(nsa_plan_t plan, int top_k);

/* Rows of the packed routing-key output of nsa_block_select_prefill over
 * `total_tokens` tokens: floor(total_tokens / l'). */
int nsa_block_rows(nsa_plan_t plan, int total_tokens);

/* Synchronises `stream`, returns the device status word of the last call that
 * used `workspace` (NSA_OK or NSA_ERR_DEVICE_*), and clears it.  Meant for
 * tests and debugging; returns NSA_ERR_CUDA if the stream itself failed. */
int nsa_read_device_status(const void* workspace, void* stream);

/* Launches one CTA whose bounded wait on an mbarrier that nothing signals
 * gives up after about `cycles` SM cycles and records NSA_ERR_DEVICE_TIMEOUT
 * in the workspace status word.  Exercises the timeout path without faulting
 * or hanging the GPU (tests only). */
int nsa_selftest_timeout(void* workspace, size_t workspace_bytes, long long cycles,
                         void* stream);

/* Per-launch timing for benchmarks.  While enabled on the calling thread,
 * nsa_prefill / nsa_block_select_prefill / nsa_decode record a CUDA event on the call's stream before
 * each kernel launch and after the last one (the library owns the events).
 * nsa_profile_stage_ms synchronises the last profiled call's events and
 * writes up to `max_stages` per-launch durations in milliseconds, in launch
 * order; it returns the number of launches of that call, or -1 if no
 * profiled call has been made or a CUDA call failed. */
int nsa_profile_enable(int enable);
int nsa_profile_stage_ms(float* ms, int max_stages);

/* Static description of a status code. */
const char* nsa_strerror(int status);

/* Number of kernel launches made by the last successful nsa_prefill /
 * nsa_block_select_prefill / nsa_decode call on this thread (for launch accounting in benchmarks). */
int nsa_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* NSA_B200_H */
