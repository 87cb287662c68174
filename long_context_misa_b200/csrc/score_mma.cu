// Token scoring of gathered candidates (the MISA-dagger fine stage), and the
// dispatch of prefix scoring to the bulk-copy streaming kernel.
//
// Row i scores the tokens gather[i][0..n_cols) of its sequence with the
// given heads ("MISA: Mixture of Indexer Sparse Attention for Long-Context
// LLM Inference", technical summary, "Hierarchical variant": the original
// DSA indexer -- all H_I heads -- re-scores only the candidate set):
//     I_t = s_t * sum_n w_{i,S_n} * ReLU(q_{i,S_n} . k_t).
// The candidate rows are scattered, so each warp loads its 16 key rows
// straight into registers with 16-byte loads (one row per 8-lane group pair)
// and prefetches the next tile's rows while the current one is on the tensor
// cores; fragments, MMA and the fused ReLU / w / head-reduction epilogue are
// shared with the streaming kernel (frag.cuh).  Invalid candidates (negative,
// or outside the query's prefix) are skipped and leave their score unwritten.
#include "frag.cuh"
#include "internal.h"

namespace misa {
namespace {

constexpr int SC_THREADS = 256;
constexpr int SC_WARPS = SC_THREADS / 32;

template <int NT, bool FP8>
__global__ void __launch_bounds__(SC_THREADS) score_gather_kernel(CacheView c, QueryView qv, const int32_t *heads,
                                                                  int h, const int32_t *gather, int n_cols,
                                                                  float *scores, long long ld, int chunk,
                                                                  uint32_t *row_hist) {
  using F = FragCfg<FP8>;
  constexpr int NV = F::NV, ROW = F::ROW;
  __shared__ uint2 bfrag[F::KT * F::TERMS * NT * 32];
  __shared__ float w_s[NT * 8], scale_s[NT * 8];
  __shared__ uint32_t shist[TOPK_HIST_BINS];  // this CTA's share of the row histogram
  const int i = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, cq = lane & 3;
  int s;
  const int Li = query_prefix(c, qv, i, &s);
  const int col0 = blockIdx.x * chunk;
  if (col0 >= n_cols) return;  // uniform over the CTA
  const int col1 = min(col0 + chunk, n_cols);

  for (int b = tid; b < TOPK_HIST_BINS; b += SC_THREADS) shist[b] = 0;
  build_query_frags<NT, FP8, SC_THREADS>(c, qv, i, heads, h, bfrag, w_s, scale_s, tid, [] { __syncthreads(); });
  __syncthreads();
  float wr[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    wr[nt][0] = w_s[nt * 8 + 2 * cq];
    wr[nt][1] = w_s[nt * 8 + 2 * cq + 1];
  }
  const uint8_t *kbase = static_cast<const uint8_t *>(c.keys) + (size_t)s * c.L_cap * ROW;
  const float *sbase = FP8 ? c.scale + (size_t)s * c.L_cap : nullptr;
  const int32_t *grow = gather + (size_t)i * n_cols;

  // candidate tokens of rows g, g+8 of the tile at position r0 (-1: skip)
  auto tokens = [&](int r0, int (&tok)[2]) {
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int p = r0 + g + 8 * hr;
      const int t = p < col1 ? __ldg(grow + p) : -1;
      tok[hr] = (t >= 0 && t < Li) ? t : -1;
    }
  };
  auto load = [&](const int (&tok)[2], uint4 (&kv)[2][NV]) {
#pragma unroll
    for (int hr = 0; hr < 2; ++hr)
#pragma unroll
      for (int ch = 0; ch < NV; ++ch)
        kv[hr][ch] = ldg_stream(kbase + (size_t)max(tok[hr], 0) * ROW + 64 * ch + 16 * cq);
  };

  int r0 = col0 + warp * 16;
  int tok[2] = {-1, -1};
  uint4 kv[2][NV];
  if (r0 < col1) {
    tokens(r0, tok);
    load(tok, kv);
  }
  while (r0 < col1) {
    const int rn = r0 + SC_WARPS * 16;
    int tok_n[2] = {-1, -1};
    uint4 kv_n[2][NV];
    if (rn < col1) {  // prefetch the next tile of this warp
      tokens(rn, tok_n);
      load(tok_n, kv_n);
    }
    const int me = cq & 1;  // lanes cq = 0 / 1 write rows g / g + 8
    float sc = 1.f;
    if (FP8 && cq < 2 && tok[me] >= 0) sc = __ldg(sbase + tok[me]);
    float acc[NT][4];
    tile_mma<NT, FP8>(kv, bfrag, lane, acc);
    const float2 sums = tile_reduce<NT>(acc, wr);
    if (cq < 2 && tok[me] >= 0) {
      const float v = (me ? sums.y : sums.x) * sc;
      scores[(size_t)i * ld + r0 + g + 8 * me] = v;
      atomicAdd(&shist[ordered_key(v) >> 21], 1u);
    }
    if (rn >= col1) break;
    r0 = rn;
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      tok[hr] = tok_n[hr];
#pragma unroll
      for (int ch = 0; ch < NV; ++ch) kv[hr][ch] = kv_n[hr][ch];
    }
  }
  __syncthreads();
  uint32_t *rh = row_hist + (size_t)i * TOPK_HIST_BINS;
  for (int b = tid; b < TOPK_HIST_BINS; b += SC_THREADS) {
    const uint32_t v = shist[b];
    if (v) atomicAdd(rh + b, v);
  }
}

template <int NT, bool FP8>
cudaError_t launch_gather(dim3 grid, const CacheView &c, const QueryView &q, const int32_t *heads, int h,
                          const int32_t *gather, int n_cols, float *scores, long long ld, int chunk,
                          uint32_t *row_hist, cudaStream_t s) {
  score_gather_kernel<NT, FP8><<<grid, SC_THREADS, 0, s>>>(c, q, heads, h, gather, n_cols, scores, ld, chunk,
                                                           row_hist);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_score_mma(const CacheView &c, const QueryView &q, const int32_t *heads, int h,
                             const int32_t *gather, int n_cols, float *scores, long long ld, uint32_t *row_hist,
                             cudaStream_t s) {
  if (q.n_q == 0) return cudaSuccess;
  if (!gather) return launch_score_stream(c, q, heads, h, scores, ld, row_hist, s);
  const int h_eff = heads ? h : q.H;
  int NT = 1;
  while (NT * 8 < h_eff) NT *= 2;
  const int sms = device_sms();
  // about 2 CTAs per SM, each warp with at least 4 tiles of 16 candidates
  const int quantum = SC_WARPS * 16;
  int splits = max(1, 2 * sms / q.n_q);  // one wave of ~2 CTAs per SM
  splits = min(splits, max(1, cdiv(n_cols, 4 * quantum)));
  const int chunk = cdiv(cdiv(n_cols, splits), quantum) * quantum;
  splits = cdiv(n_cols, chunk);
  const dim3 grid(splits, q.n_q);
#define MISA_GATHER_CASE(N)                                                                          \
  case N:                                                                                            \
    return c.fp8 ? launch_gather<N, true>(grid, c, q, heads, h, gather, n_cols, scores, ld, chunk, row_hist, s) \
                 : launch_gather<N, false>(grid, c, q, heads, h, gather, n_cols, scores, ld, chunk, row_hist, s);
  switch (NT) {
    MISA_GATHER_CASE(1)
    MISA_GATHER_CASE(2)
    MISA_GATHER_CASE(4)
    MISA_GATHER_CASE(8)
    MISA_GATHER_CASE(16)
    default:
      return cudaErrorInvalidValue;
  }
#undef MISA_GATHER_CASE
}

}  // namespace misa
