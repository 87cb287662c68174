/*
 * misa.h -- C ABI of the B200 (sm_100a) MISA / DSA token-selection indexer.
 *
 * The operations follow "MISA: Mixture of Indexer Sparse Attention for
 * Long-Context LLM Inference" (Hugging Face paper-page abstract, and the
 * gist.science technical summary, sections "Problem statement",
 * "Methodology: MISA" and "Hierarchical variant (MISA-dagger)").
 *
 * The indexer score of token t for a query with head queries q_j, head
 * weights w_j and the token's single index key k_t (shared by all heads) is
 *
 *     I_t = s_t * sum_{j in S} w_j * ReLU(q_j . k_t)
 *
 * with S the set of scoring heads (all H_I heads for the dense DSA indexer,
 * the h routed heads for MISA) and s_t the per-token fp8 scale (1 for bf16).
 * A query at position p sees the causal prefix t = 0..p (L_i = p + 1 tokens).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer inside misa_cache / misa_queries and every buffer argument
 *    is DEVICE memory owned by the caller.  The library never allocates or
 *    frees memory; scratch space is the caller's workspace `ws`, sized by
 *    misa_workspace_bytes() and 16-byte aligned.  The top-k calls need a
 *    workspace even when scores_out is given (per-row score histograms and,
 *    for few long rows, a compact candidate list).
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *    default stream).  Outputs are valid in stream order.  Nothing blocks the
 *    host.  Between calls the library keeps only cached device attributes,
 *    the thread-local error text, and three process-wide test hooks that are
 *    off unless a caller sets them: misa_debug_fail_next (a count of calls
 *    to fail), misa_debug_time_scoring (two events recorded around the
 *    scoring kernels) and misa_debug_select_in_kernel (a kernel choice).  misa_rerank_topk_noalloc's fixed scratch array also
 *    keeps the last call's contents (see there).
 *  - The library's kernels are launched with programmatic stream
 *    serialisation.  No kernel touches memory before the caller's work ahead
 *    of the call has completed.  Inside misa_dagger_decode the append kernel
 *    lets the routed pass start at once (it reads only what the append does
 *    not write until it waits for it); no call's last kernel releases its
 *    dependents early.
 *    A caller's kernel launched without that attribute is ordered as usual.
 *    A caller's kernel that opts into programmatic dependent launch itself,
 *    right after a call, must wait on its grid dependency (griddepcontrol.wait
 *    / cudaGridDependencySynchronize) before it reads the call's outputs, as
 *    after any kernel.
 *  - Arguments are validated on the host before any launch.  A bad argument
 *    returns MISA_ERR_INVALID (MISA_ERR_UNSUPPORTED for shapes outside the
 *    supported range, MISA_ERR_WORKSPACE for a short workspace) and launches
 *    nothing.  A CUDA launch failure returns MISA_ERR_CUDA.  In every non-OK
 *    case misa_last_error() holds a message.  No C++ exception crosses the ABI.
 *  - Conditions that only the device can see (a query position beyond its
 *    sequence, an append past the capacity, a bounded wait that ran out) are
 *    handled without faulting: the affected rows are clamped or skipped and a
 *    MISA_DEV_* bit is OR-ed into cache->status when it is non-NULL.
 *  - Top-k outputs list the selected token indices in ascending order,
 *    followed by -1 padding when the prefix holds fewer than k tokens.
 *    Selection orders by score, ties to the lower token index.
 *  - Supported shapes: d = 128, 1 <= H <= 128, L_cap <= MISA_MAX_L.
 */
#ifndef MISA_H
#define MISA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *misa_stream; /* same type as cudaStream_t */

#if defined(__GNUC__)
#define MISA_API __attribute__((visibility("default")))
#else
#define MISA_API
#endif

#define MISA_MAX_L (1 << 18)   /* longest supported cache: 262144 keys */
#define MISA_MAX_H 128         /* most index heads per query */
#define MISA_D 128             /* index-key width d_I */

typedef enum {
  MISA_OK = 0,
  MISA_ERR_INVALID = 1,
  MISA_ERR_UNSUPPORTED = 2,
  MISA_ERR_WORKSPACE = 3,
  MISA_ERR_CUDA = 4
} misa_status;

typedef enum { MISA_KEY_BF16 = 0, MISA_KEY_FP8_E4M3 = 1 } misa_key_dtype;

typedef enum {
  MISA_OP_ROUTE = 0,        /* misa_route_heads */
  MISA_OP_SCORE_TOPK = 1,   /* misa_score_topk */
  MISA_OP_DENSE_TOPK = 2,   /* dsa_dense_score_topk */
  MISA_OP_RERANK_TOPK = 3,  /* misa_rerank_topk */
  MISA_OP_DAGGER_TOPK = 4,  /* misa_dagger_topk */
  MISA_OP_DAGGER_DECODE = 5 /* misa_dagger_decode */
} misa_op;

/* Bits OR-ed into misa_cache.status by the device. */
#define MISA_DEV_BAD_POSITION 1u  /* q_pos/q_seq outside the cache: row clamped or emptied */
#define MISA_DEV_APPEND_RANGE 2u  /* append beyond L_cap: that sequence was skipped */
#define MISA_DEV_WAIT_TIMEOUT 4u  /* an on-chip pipeline wait ran out of time: outputs invalid */
#define MISA_DEV_BAD_HEAD 8u      /* a head index outside [0, H): head 0 was used instead */
#define MISA_DEV_SMEM_LAYOUT 16u  /* a kernel's shared-memory layout did not fit its allocation: it wrote nothing */

/*
 * Index-key cache of n_seq sequences (one shared index key per token,
 * abstract: "the heads share the same selected token set").
 *   keys    [n_seq][L_cap][d]  bf16 bit patterns (uint16) or e4m3 codes (uint8),
 *                              16-byte aligned
 *   scale   [n_seq][L_cap]     fp32 per-token dequantisation scale s_t > 0;
 *                              must be NULL for bf16 and non-NULL for fp8
 *   seq_len [n_seq]            int32 valid keys per sequence (<= L_cap)
 *   pool    [n_seq][ceil(L_cap/B)][d] fp32 block means (written by
 *                              misa_pool_keys, read by misa_route_heads)
 *   status  [1] uint32 or NULL device error bits (MISA_DEV_*)
 */
typedef struct {
  void *keys;
  float *scale;
  int32_t *seq_len;
  float *pool;
  uint32_t *status;
  int32_t n_seq;
  int32_t L_cap;
  int32_t d;
  int32_t B;
  int32_t dtype; /* misa_key_dtype */
} misa_cache;

/*
 * Index queries (technical summary, "Problem statement": H_I index heads per
 * query; the head weights w are query-dependent).
 *   q     [n_q][H][d] bf16 bit patterns
 *   w     [n_q][H]    fp32 head weights
 *   q_seq [n_q]       int32 sequence of each query
 *   q_pos [n_q]       int32 position of each query; its prefix is 0..q_pos
 * Queries of one sequence should be adjacent (prefill chunks): the batched
 * tensor-core path forms groups of consecutive queries.
 */
typedef struct {
  const uint16_t *q;
  const float *w;
  const int32_t *q_seq;
  const int32_t *q_pos;
  int32_t n_q;
  int32_t H;
} misa_queries;

/*
 * Block mean-pool of the index keys ("Methodology: MISA", step 1: the prefix
 * is cut into M = ceil(L/B) blocks summarised by the mean of their keys).
 *
 * count == 0: rebuild.  For every sequence s, pool[s][m] = mean of the
 *   dequantised keys of block m over the tokens t < seq_len[s] it holds
 *   (a trailing partial block is averaged over its count).  new_keys,
 *   new_scale and new_pos are ignored and may be NULL.
 * count > 0: append (the key-write path).  For every s with new_pos[s] >= 0,
 *   new_keys[s][0..count) (layout [n_seq][count][d], the cache's dtype) and
 *   new_scale[s][0..count) (fp8 only) are written at positions
 *   new_pos[s] .. new_pos[s]+count-1, seq_len[s] becomes new_pos[s]+count,
 *   and the mean of every block holding a written position is recomputed in
 *   the same kernel.  new_pos[s] < 0 leaves sequence s untouched; an append
 *   past L_cap skips the sequence and sets MISA_DEV_APPEND_RANGE.
 *   Appending at the same positions again is idempotent.
 * Errors: MISA_ERR_INVALID for a NULL cache/keys/pool/seq_len, B < 1,
 *   count < 0, or (count > 0) NULL new_keys/new_pos or a scale mismatch.
 */
MISA_API misa_status misa_pool_keys(const misa_cache *cache, const void *new_keys, const float *new_scale,
                           const int32_t *new_pos, int32_t count, misa_stream stream);

/*
 * The key-write path of an e4m3 cache fed bf16 index keys: quantise and
 * append in one pass.  The pages keep the index keys in the model's cache and
 * say nothing of their number format; this call has no counterpart there.
 * For every s with new_pos[s] >= 0, each new key row x = new_keys[s][j]
 * (bf16 bit patterns, layout [n_seq][count][d], 16-byte aligned) becomes
 *     scale = amax_e |x_e| / 448   (1 for a row of zeros),
 *     code_e = e4m3(x_e / scale)   rounded to nearest even, saturated to +-448,
 * with amax, the scale and the quotient in fp32 (IEEE division); codes and
 * scale are written at position new_pos[s] + j, seq_len[s] becomes
 * new_pos[s] + count, and every block holding a written position gets its
 * mean recomputed in the same kernel (from the quantised keys, as
 * misa_pool_keys would).  new_pos[s] < 0 leaves sequence s untouched; an
 * append past L_cap skips the sequence and sets MISA_DEV_APPEND_RANGE.
 * Errors: MISA_ERR_INVALID for a cache that does not hold e4m3 keys, count
 * outside [1, 64], NULL or misaligned new_keys, NULL new_pos (and the
 * checks of misa_pool_keys on the cache).
 */
MISA_API misa_status misa_append_keys_e4m3(const misa_cache *cache, const uint16_t *new_keys,
                                           const int32_t *new_pos, int32_t count, misa_stream stream);

/*
 * Block-pooled head router ("Methodology: MISA", step 1): per-head affinities
 * against the pooled keys, aggregated into a head importance, then the top-h
 * heads of each query.  Importance of head j for query i with prefix L_i:
 *     r_j = |w_j| * sum_{m < ceil(L_i/B)} ReLU(q_j . kbar_m)
 * where blocks wholly inside the prefix use cache->pool and a block cut by the
 * prefix end uses the mean of its keys 0..q_pos (recomputed per query, so
 * the routing stays causal).  Ties go to the lower head index.
 *   heads         [n_q][h]  int32 out, ascending head indices
 *   router_scores [n_q][H]  fp32 out, r_j (may be NULL)
 * Requires a pool built by misa_pool_keys for the current keys.
 * Errors: MISA_ERR_INVALID for h outside [1, H] or NULL q/w/q_seq/q_pos/heads.
 */
MISA_API misa_status misa_route_heads(const misa_cache *cache, const misa_queries *qs, int32_t h,
                             int32_t *heads, float *router_scores,
                             void *ws, size_t ws_bytes, misa_stream stream);

/*
 * The same router with the aggregation chosen.  The pages say only that the
 * per-block affinities a_jm = q_j . kbar_m are aggregated into a head
 * importance; misa_route_heads takes the first reading below, the others are
 * the plain alternatives the wording allows:
 *   MISA_AGG_ABS_SUM     r_j = |w_j| * sum_m ReLU(a_jm)
 *   MISA_AGG_SIGNED_SUM  r_j =  w_j  * sum_m ReLU(a_jm)
 *   MISA_AGG_SUM         r_j =         sum_m ReLU(a_jm)
 *   MISA_AGG_ABS_MAX     r_j = |w_j| * max_m ReLU(a_jm)
 * (the causal tail block counts like any other block).  Same arguments,
 * outputs and errors as misa_route_heads, plus MISA_ERR_INVALID for an
 * unknown agg.
 */
#define MISA_AGG_ABS_SUM 0
#define MISA_AGG_SIGNED_SUM 1
#define MISA_AGG_SUM 2
#define MISA_AGG_ABS_MAX 3
MISA_API misa_status misa_route_heads_agg(const misa_cache *cache, const misa_queries *qs, int32_t h, int32_t agg,
                                          int32_t *heads, float *router_scores, void *ws, size_t ws_bytes,
                                          misa_stream stream);

/*
 * Routed sparse token scoring and top-k ("Methodology: MISA", step 2: only
 * the h selected heads score every prefix token; the top-k tokens are taken
 * on these reduced scores).
 *   heads      [n_q][h] int32 in [0, H) (from misa_route_heads)
 *   topk       [n_q][k] int32 out (ascending token indices, -1 padded)
 *   scores_out [n_q][L_cap] fp32 out or NULL: I_t for t < L_i (other
 *              entries unspecified)
 * With k = k' this is the coarse stage of MISA-dagger.
 * Errors: MISA_ERR_INVALID for h outside [1, H], k < 1 or NULL pointers.
 */
MISA_API misa_status misa_score_topk(const misa_cache *cache, const misa_queries *qs,
                            const int32_t *heads, int32_t h, int32_t k,
                            int32_t *topk, float *scores_out,
                            void *ws, size_t ws_bytes, misa_stream stream);

/*
 * Dense DSA lightning indexer ("Problem statement" and abstract: every prefix
 * token is scored with all H_I heads and the top-k go to the main attention;
 * cost O(H_I L) per query).  Same outputs as misa_score_topk with S = all
 * heads.
 */
MISA_API misa_status dsa_dense_score_topk(const misa_cache *cache, const misa_queries *qs, int32_t k,
                                 int32_t *topk, float *scores_out,
                                 void *ws, size_t ws_bytes, misa_stream stream);

/*
 * Fine stage of MISA-dagger ("Hierarchical variant": the original DSA indexer
 * with all H_I heads re-scores only the k' candidates from the routed pass
 * and recovers the final top-k).
 *   cand       [n_q][k_prime] int32 distinct token indices in any order (-1
 *              entries and indices outside the query's prefix are ignored;
 *              a repeated token is returned at most once)
 *   topk       [n_q][k] int32 out (ascending token indices, -1 padded)
 *   scores_out [n_q][k_prime] fp32 out or NULL: dense score of cand[i][j]
 *              (unspecified where the candidate is ignored)
 * Errors: MISA_ERR_INVALID for k < 1, k_prime < k or NULL pointers.
 */
MISA_API misa_status misa_rerank_topk(const misa_cache *cache, const misa_queries *qs,
                             const int32_t *cand, int32_t k_prime, int32_t k,
                             int32_t *topk, float *scores_out,
                             void *ws, size_t ws_bytes, misa_stream stream);

/*
 * MISA-dagger in one call ("Hierarchical variant": the routed pass keeps the
 * top-k' candidates, the original DSA indexer with all H_I heads re-scores
 * only those and keeps the final top-k).  Same result as misa_score_topk
 * with k = k_prime followed by misa_rerank_topk on its output, without the
 * intermediate ascending ordering of the k' candidates.
 *   heads [n_q][h] int32 in [0, H) (from misa_route_heads)
 *   topk  [n_q][k] int32 out (ascending token indices, -1 padded)
 * Workspace: misa_workspace_bytes(MISA_OP_DAGGER_TOPK, ..., h, k, k_prime).
 * Errors: MISA_ERR_INVALID for h outside [1, H], 1 <= k <= k_prime violated
 * or NULL pointers; MISA_ERR_UNSUPPORTED for k_prime above MISA_MAX_L.
 */
MISA_API misa_status misa_dagger_topk(const misa_cache *cache, const misa_queries *qs,
                                      const int32_t *heads, int32_t h, int32_t k_prime, int32_t k,
                                      int32_t *topk, void *ws, size_t ws_bytes, misa_stream stream);

/*
 * One MISA-dagger decode step in one call: the composition of misa_pool_keys
 * in append mode ("Methodology: MISA", step 1: the block means stay current
 * as keys are written), misa_route_heads (step 1: the top-h heads of every
 * query) and misa_dagger_topk ("Hierarchical variant": the routed top-k'
 * candidates re-ranked with all heads to the final top-k).
 *   new_keys, new_scale, new_pos, count: the keys appended, as in
 *              misa_pool_keys (count >= 1); the queries' prefixes may
 *              include them
 *   heads      [n_q][h] int32 out, each query's routed heads ascending, or
 *              NULL
 *   topk       [n_q][k] int32 out (ascending token indices, -1 padded)
 * Decode batches (few queries per sequence) whose scoring grid fits on the
 * device at once route inside the routed scoring kernel: the C CTAs that
 * score a query each sum the router over a slice of its blocks and then add
 * the C partial sums in a fixed order.  misa_route_heads sums the same terms
 * in another grouping, so a head whose importance equals another's to within
 * rounding can be chosen differently; otherwise the results are those of the
 * three calls in sequence (which is what runs for other shapes).
 * Workspace: misa_workspace_bytes(MISA_OP_DAGGER_DECODE, cache, qs, h, k,
 * k_prime).  Errors: those of the three calls; count outside [1, L_cap] is
 * MISA_ERR_INVALID.
 */
MISA_API misa_status misa_dagger_decode(const misa_cache *cache, const misa_queries *qs, const void *new_keys,
                                        const float *new_scale, const int32_t *new_pos, int32_t count, int32_t h,
                                        int32_t k_prime, int32_t k, int32_t *heads, int32_t *topk, void *ws,
                                        size_t ws_bytes, misa_stream stream);

/*
 * misa_rerank_topk without a caller workspace and without any allocation.
 * The paper has no counterpart of this call: it changes where the scratch
 * lives, not what is computed.  Outputs, ordering and errors are those of
 * misa_rerank_topk.
 *
 * Who needs it: a caller that cannot hand the library device memory, such as
 * a plain C host program with no device allocator of its own, or an engine
 * that has reserved all free device memory for its key cache up front, where
 * a cudaMalloc would fail or stall the device.  The scratch (the per-row score
 * histograms and, when scores_out is NULL, the candidate scores) lives in a
 * fixed array of MISA_NOALLOC_SCRATCH_BYTES inside the library's device
 * image: one per CUDA context that loads the library (normally one per
 * device, the runtime's primary context), held until that context ends.
 * The call allocates and frees nothing; it zeroes the histogram part of the
 * array on `stream` before use.
 *
 * Scratch needed: 8200 bytes per query for the histograms (2048 bins and two
 * counters), plus 4 * k_prime bytes per query when scores_out is NULL, each
 * part rounded up to 256 bytes
 * (8 queries with k_prime = 8192: about 320 KiB).  A larger need returns
 * MISA_ERR_WORKSPACE and launches nothing; use misa_rerank_topk then.
 *
 * Limits of a shared array: calls that may overlap in one context (different
 * streams, or host threads without ordering between them) race on it and
 * give wrong results; calls in stream order on one stream are safe.  The
 * first call in each context looks up the array's device address there (it
 * may load the library's device code), so make it once before any stream
 * capture; the address is then cached per context.  A failed lookup returns
 * MISA_ERR_CUDA.
 */
#define MISA_NOALLOC_SCRATCH_BYTES (4u << 20) /* 4 MiB per context */

MISA_API misa_status misa_rerank_topk_noalloc(const misa_cache *cache, const misa_queries *qs,
                                              const int32_t *cand, int32_t k_prime, int32_t k,
                                              int32_t *topk, float *scores_out, misa_stream stream);

/*
 * Workspace bytes the call `op` (misa_op) needs for these shapes (k is the
 * call's k: k' for the coarse MISA-dagger stage); 0 on invalid arguments.
 * This is the need without scores_out; with scores_out it is smaller.
 * Host-only, launches nothing.
 */
MISA_API size_t misa_workspace_bytes(int32_t op, const misa_cache *cache, const misa_queries *qs,
                            int32_t h, int32_t k, int32_t k_prime);

/* Thread-local text of the last non-OK status ("" if none). */
MISA_API const char *misa_last_error(void);

/* Name of a misa_status value. */
MISA_API const char *misa_status_name(int32_t status);

/* ABI version (incremented on incompatible changes). */
MISA_API int32_t misa_version(void);

/*
 * Fault injection for tests: the next n calls of the entry points above fail
 * with MISA_ERR_CUDA after argument validation and before any launch, as a
 * failing launch would.  n <= 0 switches injection off.
 */
MISA_API void misa_debug_fail_next(int32_t n);

/*
 * Kernel-choice switch for tests and measurements: with on != 0, every call
 * whose shapes allow it selects its top k inside the scoring kernel (the
 * CTAs that scored a row meet at counters in the workspace and select from
 * their on-chip scores), instead of the separate top-k kernels.  The results
 * are the same either way.  Off by default, because on B200 the separate
 * kernels are as fast or faster for these calls; misa_dagger_decode's routed
 * pass selects in-kernel whatever the switch says.  Process-wide.
 */
MISA_API void misa_debug_select_in_kernel(int32_t on);

/*
 * Profiling aid: while both are non-NULL, every misa_score_topk,
 * dsa_dense_score_topk, misa_rerank_topk and misa_rerank_topk_noalloc call
 * records the caller's cudaEvent_t `start` just before and `stop` just after
 * its token-scoring kernel, and misa_dagger_topk around its routed scoring
 * kernel (not the re-rank), on the call's stream, so the kernel's own
 * duration can be read with cudaEventElapsedTime.  Inside a stream capture
 * the records become event nodes of the graph.
 * misa_debug_time_scoring(NULL, NULL) switches it off.
 */
MISA_API void misa_debug_time_scoring(void *start, void *stop);

/*
 * Failure-path check: launch one kernel that waits, with the same bounded
 * wait every on-chip pipeline of the library uses, on an mbarrier that never
 * completes.  After limit_ns (at most 10 s) the wait gives up, ORs
 * MISA_DEV_WAIT_TIMEOUT into *status (device memory) and the kernel returns
 * normally: no fault, no trap, the context stays usable.  Errors:
 * MISA_ERR_INVALID for a NULL status or a limit above 10 s.
 */
MISA_API misa_status misa_debug_wait_timeout(uint32_t *status, uint64_t limit_ns, misa_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* MISA_H */
