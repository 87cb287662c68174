// Host-side launchers shared between the translation units of libmisa.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace misa {

// Bins of the per-row score histogram the scoring kernels build for the top-k
// selection: the top 11 bits of the order-preserving key of each score.
constexpr int TOPK_HIST_BINS = 2048;

// pool.cu
cudaError_t launch_pool_rebuild(const CacheView &c, cudaStream_t s);
// zero != nullptr: the kernel also sets zero[0..zero_n) to 0.  early: the
// next kernel may start before this one completes (it must read nothing this
// one writes before its grid_dep_sync(); the decode step's routed pass)
cudaError_t launch_pool_append(const CacheView &c, const void *new_keys, const float *new_scale,
                               const int32_t *new_pos, int count, cudaStream_t s, uint32_t *zero = nullptr,
                               size_t zero_n = 0, bool early = false);
// The keys an append kernel still running ahead of a routed scoring launch
// writes (launch_pool_append's arguments, with its n_seq CTAs).
struct PendingAppend {
  const void *keys = nullptr;
  const float *scale = nullptr;
  const int32_t *pos = nullptr;  // nullptr: no append pending
  int count = 0;
};
// e4m3 caches: bf16 keys quantised (one scale per token) while appended;
// count <= pool_append_quant_max()
int pool_append_quant_max();
cudaError_t launch_pool_append_quant(const CacheView &c, const uint16_t *new_keys, const int32_t *new_pos, int count,
                                     cudaStream_t s);

// route.cu.  agg: the aggregation of the block affinities into a head's
// importance (MISA_AGG_* of misa.h): weight factor |w|, w or 1, and a sum or
// a maximum over the blocks.
__host__ __device__ inline bool agg_is_max(int agg) { return agg == 3; }
__device__ inline float agg_weight(int agg, float w) { return agg == 1 ? w : agg == 2 ? 1.f : fabsf(w); }
int route_chunks(int M_cap);
size_t route_ws_bytes(int n_q, int H, int M_cap);
cudaError_t launch_route(const CacheView &c, const QueryView &q, int h, int32_t *heads, float *router_scores,
                         void *ws, cudaStream_t s, int agg = 0);
// route_umma.cu: the same routing for many queries per sequence (prefill) on
// tcgen05 tensor cores; launch_route dispatches to it when it applies.
bool route_umma_applies(const CacheView &c, const QueryView &q);
size_t route_umma_ws_bytes(int n_q, int H, int M_cap, int n_seq);
cudaError_t launch_route_umma(const CacheView &c, const QueryView &q, int h, int32_t *heads, float *router_scores,
                              void *ws, cudaStream_t s, int agg = 0);

// Selection inside the scoring kernel (rowsel.cuh): the CTAs that scored a
// row select its top k from their on-chip scores, meeting at counters in
// global memory.  Applies to decode rows on the streaming scorer and to
// re-rank rows, when the launch's CTAs are all resident at once.
constexpr int FUSED_CTR = 8;                                 // counters per row
constexpr int FUSED_ZERO_WORDS = 2 * TOPK_HIST_BINS + FUSED_CTR;  // zeroed per row before the launch
constexpr int FUSED_BCAP = 2048;                             // boundary-bucket entries per row
struct FusedTopk {
  uint32_t *zeroed;   // [n_q][FUSED_ZERO_WORDS], zero before the launch
  uint2 *bucket;      // [n_q][FUSED_BCAP]
  int32_t *winners;   // [n_q][k] scratch of an ascending output (ordered only)
  int32_t *out;       // [n_q][k] the selected tokens
  int k;
  int ordered;        // 1: ascending token order; 0: any order
  // 1 (unordered outputs only): the next kernel finishes the row.  The
  // selecting kernel writes the sure winners to out[0, n) (n = the row's
  // winner counter) and lists a split boundary bucket that fits FUSED_BCAP
  // with the number still to take from it (counters FUSED_CTR_EMIT,
  // FUSED_CTR_BUCKET, FUSED_CTR_NEED of the row's zeroed words); rows whose
  // bucket is larger are finished as usual.  Nothing pads out[n, k).
  int defer;
};
// counters among a row's zeroed words (after its two histograms)
constexpr int FUSED_CTR_EMIT = 3, FUSED_CTR_BUCKET = 4, FUSED_CTR_NEED = 6;
// Whether launch_score_mma can select in the scoring kernel for these shapes
// (fused != nullptr there); otherwise the caller runs launch_topk.
bool score_fusable(const CacheView &c, const QueryView &q, const int32_t *heads, int h, const int32_t *gather,
                   int n_cols);

// score_dispatch.cu: scores[i][t] (row stride ld) for t < L_i, heads given per query
// (heads == nullptr: all H heads, dense).  `gather` != nullptr: row i scores the
// tokens gather[i][0..n_cols) instead of the prefix (re-rank).
// Every launch also adds each written score to row_hist[i][key >> 21] (the
// caller zeroes row_hist, [n_q][TOPK_HIST_BINS] uint32, beforehand).
cudaError_t launch_score_mma(const CacheView &c, const QueryView &q, const int32_t *heads, int h,
                             const int32_t *gather, int n_cols, float *scores, long long ld, uint32_t *row_hist,
                             cudaStream_t s, const FusedTopk *fused = nullptr);

// rerank_umma.cu: the gathered (re-rank) case of launch_score_mma on tcgen05
// tensor cores, for up to 128 scoring heads, and (gather == nullptr, n_cols =
// L_cap) prefix scoring of e4m3 caches with 32 or more heads;
// launch_score_mma dispatches to it when it applies.  Same outputs,
// histogram included.
bool rerank_umma_applies(const QueryView &q, const int32_t *heads, int h);
cudaError_t launch_rerank_umma(const CacheView &c, const QueryView &q, const int32_t *heads, int h,
                               const int32_t *gather, int n_cols, float *scores, long long ld, uint32_t *row_hist,
                               cudaStream_t s, const FusedTopk *fused = nullptr);
bool rerank_fusable(const CacheView &c, const QueryView &q, const int32_t *heads, int h, int n_cols);
// The whole fine stage (all heads on the n_cols candidates of each query,
// then its top k in ascending token order, -1 padded) in one launch: one
// thread-block cluster per query (rerank_cluster.cu).  Applies when a
// cluster holds the candidates (k' <= 8192 for e4m3 keys and up to 64 heads)
// and the device can run one; scores (optional, row pitch ld) receives every
// valid candidate's score.
bool rerank_cluster_applies(const CacheView &c, const QueryView &q, int n_cols, int k);
// pend != nullptr: the candidates come from a top-k' selected with
// FusedTopk::defer (pend = its zeroed words, pend_bucket = its bucket lists).
cudaError_t launch_rerank_cluster(const CacheView &c, const QueryView &q, const int32_t *gather, int n_cols, int k,
                                  int32_t *out, float *scores, long long ld, cudaStream_t s,
                                  const uint32_t *pend = nullptr, const uint2 *pend_bucket = nullptr);
// the same for prefix rows of e4m3 caches with 32 or more scoring heads
bool dense_fusable(const CacheView &c, const QueryView &q, const int32_t *heads, int h);

// score_stream.cu: prefix scoring through the bulk-copy pipeline (used by
// launch_score_mma when gather == nullptr).
// route_part != nullptr (with fused): the h scoring heads are routed inside
// the kernel first (heads ignored), with route_part_slots() x H floats of
// partial sums at route_part; heads_out ([n_q][h]) receives them if not null.
// pending (with route_part): launched right after launch_pool_append(...,
// early = true) with these arguments; the kernel routes while the append
// runs and leaves one CTA slot per appended sequence to its blocks.
cudaError_t launch_score_stream(const CacheView &c, const QueryView &q, const int32_t *heads, int h, float *scores,
                                long long ld, uint32_t *row_hist, cudaStream_t s, const FusedTopk *fused = nullptr,
                                float *route_part = nullptr, int32_t *heads_out = nullptr,
                                const PendingAppend *pending = nullptr);
bool score_stream_fusable(const CacheView &c, const QueryView &q, const int32_t *heads, int h, bool route = false);
// CTA slots (queries x CTAs per query) of the in-kernel router's partial sums
inline int route_part_slots() { return 8 * device_sms(); }

// score_umma.cu: prefix scoring of query batches with many queries per
// sequence (prefill chunks) on tcgen05 tensor cores; writes no histogram.
bool umma_applies(const CacheView &c, const QueryView &q, const int32_t *heads, int h);
cudaError_t launch_score_umma(const CacheView &c, const QueryView &q, const int32_t *heads, int h, float *scores,
                              long long ld, cudaStream_t s);

// topk.cu: per row, the k largest scores, ties to the lower token index;
// outputs are token indices in ascending order, -1 padded.  Row length comes
// from the query prefix (gather == nullptr), or the row holds n_cols
// candidates whose tokens are gather[i][p] (entries < 0 or beyond the prefix
// excluded).  row_hist ([n_q][TOPK_HIST_BINS], zeroed beforehand) holds the
// scoring kernel's histogram over exactly the valid scores when hist_ready;
// otherwise it is filled here first.  Prefix rows of caches longer than
// TOPK_LIST_MIN_L go through a compact list of the elements at or above the
// histogram's boundary bin: list_ws holds topk_list_entries() entries of 8
// bytes and list_cnt 2 * n_q counters, zeroed beforehand (both may be null:
// no list; the selection then reads the rows itself).  ordered == false allows
// the selected tokens of a row in any order (followed by -1 padding).
constexpr int TOPK_LIST_MIN_L = 16384;   // shorter caches never use the list
constexpr int TOPK_LIST_EXTRA = 8192;    // boundary-bin elements listed per row beyond k
size_t topk_list_entries(int n_q, int L_cap, int k);
// n words set to zero on stream s (a small kernel)
cudaError_t launch_zero(uint32_t *p, size_t n, cudaStream_t s);
cudaError_t launch_topk(const CacheView &c, const QueryView &q, const float *scores, long long ld, int n_cols,
                        const int32_t *gather, uint32_t *row_hist, bool hist_ready, void *list_ws,
                        uint32_t *list_cnt, int k, int32_t *out, cudaStream_t s, bool ordered = true);

}  // namespace misa
