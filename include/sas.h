/*
 * sas.h -- C ABI of libsas: SAS gated block-sparse causal attention on B200.
 *
 * SAS ("Simple Attention Sparsification via End-to-End Optimization of Context
 * Ranking", arXiv 2609.13141) splits the context into contiguous blocks of
 * `block_size` tokens. For a query at position p, the block holding p is the
 * always-retained current block and the C = floor(p / block_size) blocks
 * before it are the historical candidates. A selector gives one score per
 * historical block; the gate is the softmax of those scores
 * (log g_i = s_i - log sum_j exp s_j) and the current block keeps g_0 = 1.
 * A hard top-K keeps K historical blocks, and log g of each kept block is added
 * to every logit q.k/sqrt(d) of its tokens inside the attention softmax:
 *   o = softmax(q K_S^T / sqrt(d) + log g_S) V_S.
 * Sources: dimensionstp.github.io SAS study note, 1-1 (block-sparse attention
 * eq.), 1-2 (TopK eq.), 2-1 (gate eq.), 2-2 (gated attention eq. and the
 * multiplicative identity), 3-1 (per-query-group selection), 3-7 (decode path);
 * papers.paperslantern.ai arXiv text, 3 (preliminaries: blocks, selected
 * token set), 4 (gate position, normalised gate, training scope, ablation
 * discussion).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Notation: B batch, T query rows per (b, head), Hq query heads, Hkv KV
 *    heads, G = Hq / Hkv query heads per KV group, d head_dim, b block_size,
 *    K top_k, NB = ceil((q_offset + T) / b), p = q_offset + t, C = floor(p / b).
 *  - One block selection per (batch, KV head, query row), shared by the G
 *    query heads of the group; query head h belongs to KV head h / G.
 *  - K counts historical blocks only: a row attends to at most (K + 1) * b
 *    tokens (K kept blocks plus the causal part of the current block).
 *  - Ties between equal scores go to the lower block index; -0.0 ties +0.0;
 *    -inf is a valid score (gate 0, ranked last). NaN and +inf scores are
 *    outside the contract. The kept indices are stored in ascending order.
 *  - All tensors are dense, row-major, in the layouts given per argument, and
 *    live in DEVICE memory unless stated. Every pointer must be 16-byte
 *    aligned. The caller owns and allocates every buffer, including the
 *    workspace; libsas allocates and frees nothing and keeps no state.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *    default stream) and does not synchronise the host.
 *  - Errors: argument, shape, alignment and workspace checks run first and
 *    return a status without launching anything and without touching any
 *    buffer. A failed launch returns SAS_ERR_CUDA (from cudaGetLastError).
 *    Faults inside a running kernel are reported by the CUDA runtime on a
 *    later synchronisation, not by these calls.
 *  - Supported: d in {64, 128}; b in {32, 64}; Hq % Hkv == 0; G <= 8;
 *    1 <= K <= 64. Training calls (fwd/bwd) need q_offset == 0 and T % b == 0.
 *    dtype BF16 or FP32 for q/k/v/o/dO/dq/dk/dv; scores and all statistics are
 *    always float32.
 */
#ifndef SAS_H_
#define SAS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SAS_OK = 0,
    SAS_ERR_INVALID_ARG = 1,   /* null pointer, bad shape, inconsistent sizes */
    SAS_ERR_UNSUPPORTED = 2,   /* valid but outside the supported ranges above */
    SAS_ERR_MISALIGNED = 3,    /* a pointer is not 16-byte aligned */
    SAS_ERR_WORKSPACE = 4,     /* workspace missing or smaller than required */
    SAS_ERR_CUDA = 5           /* a CUDA launch or runtime call failed */
} sas_status;

typedef enum { SAS_DT_BF16 = 0, SAS_DT_FP32 = 1 } sas_dtype;

/* Gate activation: how the selector's scores become the log-gates added to
 * the kept blocks' logits (the current block always keeps g_0 = 1), and the
 * matching score gradient. SOFTMAX is the method's normalised gate; the others
 * are the alternatives the method is compared against (arXiv text 4, design
 * elements "gate activation" and "ranking preservation"; study note 3-3, 3-4).
 *   SOFTMAX: log g_i = s_i - log sum_{j<C} exp s_j.
 *   NONE: every log-gate is 0 and the score gradient is 0 (plain block-sparse).
 *   SIGMOID: independent gates, log g_i = log sigmoid(s_i); kept blocks only
 *     get a score gradient.
 *   RAW: the unnormalised score as the logit bias, log g_i = s_i.
 *   SOFTMAX_SELECTED: softmax over the kept blocks only,
 *     log g_i = s_i - log sum_{j kept} exp s_j (undefined when every kept
 *     score is -inf).
 *   STE: hard gate, g = 1 on every kept block in the forward; the score
 *     gradient is that of the SOFTMAX gate evaluated at g = 1
 *     (straight-through): dL/ds_k = sum_{i kept} Gsum_i g_i ([i=k] - g_k). */
typedef enum {
    SAS_GATE_SOFTMAX = 0,
    SAS_GATE_NONE = 1,
    SAS_GATE_SIGMOID = 2,
    SAS_GATE_RAW = 3,
    SAS_GATE_SOFTMAX_SELECTED = 4,
    SAS_GATE_STE = 5
} sas_gate;

typedef enum { SAS_OP_TOPK = 0, SAS_OP_FWD = 1, SAS_OP_BWD = 2, SAS_OP_DECODE = 3 } sas_op;

typedef struct {
    int32_t batch;         /* B */
    int32_t seq_len;       /* T (training); 1 for decode */
    int32_t q_offset;      /* position of row 0: 0 for training, N - 1 for decode */
    int32_t n_q_heads;     /* Hq */
    int32_t n_kv_heads;    /* Hkv */
    int32_t head_dim;      /* d */
    int32_t block_size;    /* b */
    int32_t top_k;         /* K, historical blocks kept per row */
    float softmax_scale;   /* scale on q.k; <= 0 selects 1/sqrt(d). The log-gate is added unscaled. */
    int32_t dtype;         /* sas_dtype of q/k/v/o/dO/dq/dk/dv */
    int32_t gate;          /* sas_gate */
    /* Selection granularity. 0: one selection per (b, KV head, t), shared by
     * the group's G = Hq / Hkv query heads (study note 3-1: per query group).
     * 1: one selection per (b, query head, t): every query head keeps its own
     * top-K from its own score row and reads the K/V of its KV head h / G;
     * the K/V gradients sum over the G heads. The selection arrays (scores,
     * idx, gate_logit, score_lse, n_sel, dscores) then have Hq rows where the
     * calls below say Hkv, and the workspace sizes follow. */
    int32_t select_heads;
} sas_desc;

/* Bytes of device workspace `op` needs for this shape (0 if none). The caller
 * allocates it and passes it to the call; its contents need not be
 * initialised and are not meaningful afterwards. */
sas_status sas_workspace_size(int32_t op, const sas_desc* desc, size_t* bytes);

/* Gate normaliser and hard top-K (study note 1-2 TopK eq., 2-1 gate eq.;
 * arXiv text 4, normalised gate).
 *   scores     [B, Hkv, T, NB] float32, in: block scores; row t reads [0, C).
 *   idx        [B, Hkv, T, K] int32, out: kept blocks ascending, -1 padded.
 *   gate_logit [B, Hkv, T, K] float32, out: log g of each kept block under
 *              desc.gate (s_i - score_lse under SOFTMAX), 0 in padding.
 *   score_lse  [B, Hkv, T] float32, out: log sum_{i<C} exp s_i (-inf if C = 0).
 *   n_sel      [B, Hkv, T] int32, out: min(K, C).
 * Any q_offset >= 0 is allowed (decode rows use T = 1, q_offset = N - 1). */
sas_status sas_block_topk(const sas_desc* desc, const float* scores, int32_t* idx,
                          float* gate_logit, float* score_lse, int32_t* n_sel, void* stream);

/* Gated block-sparse causal attention forward (study note 2-2 gated attention
 * eq.; arXiv text 4, inner log-space gate, sparse training scope).
 *   q [B, Hq, T, d], k and v [B, Hkv, T, d] (dtype), in.
 *   idx, gate_logit, n_sel: as written by sas_block_topk for this desc, in.
 *   o [B, Hq, T, d] (dtype), out; attn_lse [B, Hq, T] float32, out: the
 *   natural-log log-sum-exp of each row's gated logits (kept for backward).
 *   ws: device workspace of at least sas_workspace_size(SAS_OP_FWD) bytes. */
sas_status sas_gated_attn_fwd(const sas_desc* desc, const void* q, const void* k, const void* v,
                              const int32_t* idx, const float* gate_logit, const int32_t* n_sel,
                              void* o, float* attn_lse, void* ws, size_t ws_bytes, void* stream);

/* Backward of sas_gated_attn_fwd, including the score gradient through the
 * gate (study note 2-2, 3-6 "keeps the selector gradient"; arXiv text 4,
 * gradient of the normalised gate: d log g_i / d s_k = [i = k] - g_k).
 *   q, k, v, o, attn_lse: the forward's inputs and outputs, in.
 *   dO [B, Hq, T, d] (dtype), in: upstream gradient of o.
 *   scores, score_lse, idx, gate_logit, n_sel: the top-K inputs/outputs, in.
 *   dq [B, Hq, T, d], dk and dv [B, Hkv, T, d] (dtype), out (overwritten).
 *   dscores [B, Hkv, T, NB] float32, out (overwritten): dL/ds; 0 for i >= C
 *   and everywhere under SAS_GATE_NONE. With Gsum_i the sum of dL/dlogit over
 *   block i's tokens and the group's G heads, for i < C: under SOFTMAX
 *   dscores_i = [i kept] * Gsum_i - g_i * sum_{k kept} Gsum_k; the other gate
 *   activations apply their own derivative (see sas_gate).
 *   ws: at least sas_workspace_size(SAS_OP_BWD) bytes. */
sas_status sas_gated_attn_bwd(const sas_desc* desc, const void* q, const void* k, const void* v,
                              const void* o, const void* dO, const float* attn_lse,
                              const float* scores, const float* score_lse, const int32_t* idx,
                              const float* gate_logit, const int32_t* n_sel, void* dq, void* dk,
                              void* dv, float* dscores, void* ws, size_t ws_bytes, void* stream);

/* Budgeted sparse decode of one new token per (batch, query head) over a KV
 * cache (study note 3-7 inference path, steps 2-4; 5-6 efficiency).
 * desc: seq_len = 1, q_offset = N - 1 where N is the cache length including
 * the new token; the current block is floor((N - 1) / b) and is causal.
 *   q [B, Hq, d] (dtype), in.
 *   k_cache, v_cache [B, Hkv, cache_stride_tokens, d] (dtype), in; tokens
 *   [0, N) are valid; cache_stride_tokens >= N.
 *   idx, gate_logit, n_sel [B, Hkv, 1, K] / [B, Hkv, 1]: from sas_block_topk
 *   with the same desc; idx == NULL selects dense decode over every token
 *   [0, N) with no gate (gate_logit and n_sel are then ignored).
 *   o [B, Hq, d] (dtype), out.
 *   ws: at least sas_workspace_size(SAS_OP_DECODE) bytes. */
sas_status sas_sparse_decode(const sas_desc* desc, const void* q, const void* k_cache,
                             const void* v_cache, int64_t cache_stride_tokens, const int32_t* idx,
                             const float* gate_logit, const int32_t* n_sel, void* o, void* ws,
                             size_t ws_bytes, void* stream);

/* Paged KV cache with a cache length per sequence (study note 3-7 inference
 * path, step 3: the kept blocks are read from the paged KV cache; 3-1 method
 * table: paged-cache serving backend). A page holds one block (block_size
 * tokens) of every KV head, so a kept block is one page per KV head.
 *   q [B, Hq, d] (dtype), in.
 *   k_pages, v_pages [num_pages, Hkv, b, d] (dtype), in: the page pools.
 *   block_table [B, max_blocks] int32, in: page of block j of sequence i at
 *   [i * max_blocks + j]; entries for blocks [0, ceil(N_i / b)) must be valid
 *   pages (an entry outside [0, num_pages) makes that block be skipped).
 *   max_blocks >= NB = ceil((q_offset + 1) / b).
 *   seq_lens [B] int32, in: N_i, the cache length of sequence i with the new
 *   token, in [1, q_offset + 1] (values outside are clamped); the current
 *   block of sequence i is floor((N_i - 1) / b), causal.
 *   desc: seq_len = 1, q_offset = max_i N_i - 1.
 *   idx, gate_logit, n_sel: from sas_block_topk_varlen with the same desc and
 *   seq_lens; idx == NULL selects dense decode over each sequence's [0, N_i).
 *   o [B, Hq, d] (dtype), out.
 *   ws: at least sas_workspace_size(SAS_OP_DECODE, desc) bytes.
 * bf16, head_dim 128, block 64 only (SAS_ERR_UNSUPPORTED otherwise). */
sas_status sas_sparse_decode_paged(const sas_desc* desc, const void* q, const void* k_pages,
                                   const void* v_pages, int32_t num_pages, const int32_t* block_table,
                                   int32_t max_blocks, const int32_t* seq_lens, const int32_t* idx,
                                   const float* gate_logit, const int32_t* n_sel, void* o, void* ws,
                                   size_t ws_bytes, void* stream);

/* sas_block_topk for decode rows (seq_len = 1) of sequences of different
 * lengths: row (i, g) has C_i = floor((N_i - 1) / b) candidates, N_i =
 * seq_lens[i] (device int32 [B], clamped to [1, q_offset + 1]); desc.q_offset
 * = max_i N_i - 1 sets NB. Outputs as sas_block_topk. */
sas_status sas_block_topk_varlen(const sas_desc* desc, const float* scores, const int32_t* seq_lens,
                                 int32_t* idx, float* gate_logit, float* score_lse, int32_t* n_sel,
                                 void* stream);

/* Block scores of the decode rows from pooled keys: the selector's scan over
 * every cached block of the new token's KV group (study note 3-7 inference
 * path, step 1; 5-6: at long context this scan, not the attention, dominates
 * the decode step). The pages' selector is a trained network; this fixed
 * scorer stands in for it:
 *   scores[b, g, 0, j] = qbar . kbar[b, g, j] for j < C = floor(q_offset / b),
 *   0 for C <= j < NB, with qbar the mean of the group's G query heads.
 *   With desc.select_heads = 1 every query head h scores with its own q_h
 *   against the pooled keys of its KV head h / G, into scores[b, h, 0, :].
 * desc: seq_len = 1, q_offset = N - 1 (as sas_sparse_decode); bf16, d 128.
 *   q [B, Hq, d] bf16, in.
 *   kbar [B, Hkv, kbar_stride_blocks, d] bf16, in: the mean key of each cached
 *   block (kept by the caller beside the cache); kbar_stride_blocks >= C.
 *   scores [B, Hkv, 1, NB] float32, out. */
sas_status sas_block_scores_pooled(const sas_desc* desc, const void* q, const void* kbar,
                                   int64_t kbar_stride_blocks, float* scores, void* stream);

/* The serving step in one call: sas_block_scores_pooled, then sas_block_topk
 * on those scores, then sas_sparse_decode with that selection, enqueued back
 * to back on `stream`. Arguments as in those three calls; scores, idx,
 * gate_logit, score_lse and n_sel are outputs the caller may inspect.
 * ws: at least sas_workspace_size(SAS_OP_DECODE, desc) bytes. */
sas_status sas_sparse_decode_pooled(const sas_desc* desc, const void* q, const void* k_cache,
                                    const void* v_cache, int64_t cache_stride_tokens, const void* kbar,
                                    int64_t kbar_stride_blocks, float* scores, int32_t* idx,
                                    float* gate_logit, float* score_lse, int32_t* n_sel, void* o,
                                    void* ws, size_t ws_bytes, void* stream);

/* Sparse decode that allocates nothing (the paper has no counterpart: this is
 * an interface convenience, not part of the method).
 *
 * For callers that cannot call cudaMalloc: a serving loop with a fixed device
 * memory budget set aside at start-up, a plug-in whose host framework owns all
 * device allocations, or a path where an allocation and its implicit
 * synchronisation are not allowed. Same arguments, results and checks as
 * sas_sparse_decode, minus the workspace: the split partials live in a static
 * device array of SAS_NOALLOC_SCRATCH_BYTES inside libsas, which every GPU
 * that loads the library holds until the process exits.
 *  - Returns SAS_ERR_WORKSPACE, launching nothing, when the shape needs more
 *    scratch than the array holds: exactly when sas_workspace_size(
 *    SAS_OP_DECODE, desc) reports more than SAS_NOALLOC_SCRATCH_BYTES (so a
 *    caller can test a shape in advance).
 *  - The first call on each device looks up the array's device address (a
 *    runtime call that allocates nothing) and keeps it for the life of the
 *    process; make that first call before any stream capture, and do not use
 *    the library across cudaDeviceReset (the kept address would be stale).
 *  - All calls share the one array and it keeps the last call's contents.
 *    Each call writes every partial it reads and zeroes the per-group
 *    counters it uses (with an asynchronous memset on `stream`), but calls
 *    that overlap on the GPU (different streams, or different host threads
 *    on one device, with no ordering between them) race on it.
 *  - No cudaMalloc, cudaFree or allocating library routine is called. */
#define SAS_NOALLOC_SCRATCH_BYTES (8u << 20)
sas_status sas_sparse_decode_noalloc(const sas_desc* desc, const void* q, const void* k_cache,
                                     const void* v_cache, int64_t cache_stride_tokens,
                                     const int32_t* idx, const float* gate_logit,
                                     const int32_t* n_sel, void* o, void* stream);

/* Diagnostics (no counterpart on the pages): number of device-side waits
 * that gave up at the wait limit (sas_set_wait_limit, default 1 s) since the
 * library was loaded; 0 in normal operation. A kernel whose wait gave up
 * leaves NaN in the call's outputs instead of hanging. Synchronises the
 * current device. */
sas_status sas_device_timeouts(uint32_t* count);

/* Diagnostics (no counterpart on the pages): bound, in nanoseconds, on every
 * device-side wait of a kernel for another agent's work (a copy, an MMA, the
 * warps of another role); 0 restores the default of 1 s. A kernel whose wait
 * gives up stops its work, lets the copies and MMAs it started finish, counts
 * the event (sas_device_timeouts) and leaves NaN in the call's outputs
 * instead of hanging. A tiny bound makes waits give up on purpose, to test
 * that path. Process-wide; synchronises the current device. */
sas_status sas_set_wait_limit(uint64_t ns);

/* Diagnostics (no counterpart on the pages): number of CUDA kernels this
 * library has launched since it was loaded, counted on the host after each
 * successful launch. Memsets issued through the runtime are not counted. */
uint64_t sas_kernel_launches(void);

/* Diagnostics (no counterpart on the pages): per-kernel device time.
 * sas_kernel_timing(names) clears earlier records and makes every later
 * entry-point call record a pair of CUDA events on its stream around each
 * kernel it launches whose name is in `names`, a comma-separated list of
 * kernel names ("bwd_tc", "fwd_rows", "block_topk", "decode_partial", ... --
 * the kernel names without the "_kernel" suffix), or around every kernel when
 * `names` is "*". sas_kernel_timing(NULL) stops recording and keeps the
 * records. Each recorded pair costs a few microseconds of device time between
 * kernels, so time only what is needed. Not for use while a stream is being
 * captured into a CUDA graph.
 * sas_kernel_time(name, &ms, &n) waits for the recorded events of that kernel
 * and returns their summed duration (ms) and count (n; 0 and 0.0 if none).
 * Returns SAS_ERR_INVALID_ARG for a NULL argument, SAS_ERR_CUDA if an event
 * could not be created, recorded or read. Records are process-wide. */
sas_status sas_kernel_timing(const char* names);
sas_status sas_kernel_time(const char* kernel, double* total_ms, uint32_t* launches);

/* Static, NUL-terminated description of a status code (never NULL). */
const char* sas_status_string(sas_status status);

#ifdef __cplusplus
}
#endif

#endif /* SAS_H_ */
