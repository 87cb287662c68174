// Dispatch of token scoring to its kernels.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference",
// technical summary, "Methodology: MISA" step 2 (routed heads score the
// prefix), "Problem statement" (the dense indexer) and "Hierarchical
// variant" (all heads re-score the candidate set):
//     I_t = s_t * sum_n w_{i,S_n} * ReLU(q_{i,S_n} . k_t).
//   - gathered candidates (re-rank): rerank_umma_kernel, tcgen05 tensor cores
//     (every head count the library accepts, MISA_MAX_H = 128);
//   - prefix rows of e4m3 caches with 32 or more scoring heads (dense
//     decode): dense_umma_kernel (rerank_umma.cu), persistent over the prefix;
//   - other prefix rows (routed decode, bf16 dense decode): the streaming
//     kernel on mma.sync, which builds the row histograms on the way, or
//     selects the top k itself (score_fusable).
// Prefill chunks (many queries per sequence) are scored by score_umma.cu,
// dispatched by the callers.
#include "internal.h"

namespace misa {

// The kernel launch_score_mma takes for these shapes.
enum class ScoreKernel { rerank, dense, stream };
static ScoreKernel pick(const CacheView &c, const QueryView &q, const int32_t *heads, int h, const int32_t *gather) {
  if (gather) return ScoreKernel::rerank;
  // e4m3 keys with 32 or more scoring heads (dense decode): the dense product
  // on tcgen05 (45 against 139.3 us on mma.sync for 8 x 128K keys and 64
  // heads); fewer heads (routed decode), and bf16 keys (whose 32 KB tiles
  // leave one CTA per SM there: 125 against 77 us for 32 x 32K and 64 heads,
  // measured with the earlier non-persistent tcgen05 form), stream the keys
  // on mma.sync
  const int he = heads ? h : q.H;
  return c.fp8 && he >= 32 ? ScoreKernel::dense : ScoreKernel::stream;
}

cudaError_t launch_score_mma(const CacheView &c, const QueryView &q, const int32_t *heads, int h,
                             const int32_t *gather, int n_cols, float *scores, long long ld, uint32_t *row_hist,
                             cudaStream_t s, const FusedTopk *fused) {
  if (q.n_q == 0) return cudaSuccess;
  if (!rerank_umma_applies(q, heads, h)) return cudaErrorInvalidValue;  // more heads than the library accepts
  switch (pick(c, q, heads, h, gather)) {
    case ScoreKernel::rerank:
      return launch_rerank_umma(c, q, heads, h, gather, n_cols, scores, ld, row_hist, s, fused);
    case ScoreKernel::dense:
      return launch_rerank_umma(c, q, heads, h, nullptr, c.L_cap, scores, ld, row_hist, s, fused);
    default:
      return launch_score_stream(c, q, heads, h, scores, ld, row_hist, s, fused);
  }
}

bool score_fusable(const CacheView &c, const QueryView &q, const int32_t *heads, int h, const int32_t *gather,
                   int n_cols) {
  if (q.n_q == 0 || !rerank_umma_applies(q, heads, h)) return false;
  switch (pick(c, q, heads, h, gather)) {
    case ScoreKernel::rerank:
      return rerank_fusable(c, q, heads, h, n_cols);
    case ScoreKernel::dense:
      return dense_fusable(c, q, heads, h);
    default:
      return score_stream_fusable(c, q, heads, h);
  }
}

}  // namespace misa
