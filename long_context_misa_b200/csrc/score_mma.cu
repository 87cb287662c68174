// Token scoring of gathered candidates (the MISA-dagger fine stage), and the
// dispatch of prefix scoring to the bulk-copy streaming kernel.
//
// Row i scores the tokens gather[i][0..n_cols) of its sequence with the
// given heads ("MISA: Mixture of Indexer Sparse Attention for Long-Context
// LLM Inference", technical summary, "Hierarchical variant": the original
// DSA indexer -- all H_I heads -- re-scores only the candidate set):
//     I_t = s_t * sum_n w_{i,S_n} * ReLU(q_{i,S_n} . k_t).
// The candidate rows are scattered: each warp requests all of its rows at
// once with cp.async into a warp-private shared region (its candidate
// indices first), builds the query fragments meanwhile, then runs the tiles
// from shared memory.  Fragments, MMA and the fused ReLU / w / head-reduction
// epilogue are
// shared with the streaming kernel (frag.cuh).  Invalid candidates (negative,
// or outside the query's prefix) are skipped and leave their score unwritten.
#include "frag.cuh"
#include "internal.h"

namespace misa {
namespace {

constexpr int SC_THREADS = 256;
constexpr int SC_WARPS = SC_THREADS / 32;
constexpr int GT_MAX = 4;  // 16-candidate tiles per warp

template <bool FP8>
struct GatherCfg {
  static constexpr int ROW = FragCfg<FP8>::ROW;       // key bytes per token
  static constexpr int TILE = 16 * ROW;               // one tile of keys
  static constexpr int STAGE = TILE + (FP8 ? 64 : 0); // keys + 16 scales
  static constexpr int WARP_BYTES = GT_MAX * STAGE;
  static constexpr int UNITS = ROW / 16;              // 16-byte units per row
  static constexpr int RPC = 32 / UNITS;              // rows per warp-wide copy
  static constexpr int COPIES = 16 / RPC;             // copies per lane and tile
};

// Warp w of a CTA scores tiles j = 0..GT_MAX-1 of 16 candidates, positions
// col0 + (j * SC_WARPS + w) * 16 + r.  All of a warp's candidate rows are
// requested at once (cp.async into a warp-private region, rows XOR-swizzled
// by parity as in the streaming kernel) before the query fragments are
// built, so the whole gather costs two dependent round trips (indices, then
// rows) that overlap the fragment set-up.
template <int NT, bool FP8>
__global__ void __launch_bounds__(SC_THREADS) score_gather_kernel(CacheView c, QueryView qv, const int32_t *heads,
                                                                  int h, const int32_t *gather, int n_cols,
                                                                  float *scores, long long ld, int chunk,
                                                                  uint32_t *row_hist) {
  using F = FragCfg<FP8>;
  using G = GatherCfg<FP8>;
  constexpr int NV = F::NV, ROW = G::ROW;
  extern __shared__ __align__(128) uint8_t g_smem[];
  __shared__ uint2 bfrag[F::KT * F::TERMS * NT * 32];
  __shared__ float w_s[NT * 8], scale_s[NT * 8];
  __shared__ uint32_t shist[TOPK_HIST_BINS];  // this CTA's share of the row histogram
  __shared__ int32_t tok_s[SC_WARPS][GT_MAX * 16];
  const int i = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, cq = lane & 3;
  int s;
  const int Li = query_prefix(c, qv, i, &s);
  const int col0 = blockIdx.x * chunk;
  const int col1 = min(col0 + chunk, n_cols);
  const uint8_t *kbase = static_cast<const uint8_t *>(c.keys) + (size_t)s * c.L_cap * ROW;
  const float *sbase = FP8 ? c.scale + (size_t)s * c.L_cap : nullptr;
  const int32_t *grow = gather + (size_t)i * n_cols;

  // 1. this warp's candidate tokens (-1: skip), two per lane
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    const int e = lane + 32 * x;                          // entry: tile e / 16, row e % 16
    const int p = col0 + ((e >> 4) * SC_WARPS + warp) * 16 + (e & 15);
    int t = p < col1 ? __ldg(grow + p) : -1;
    tok_s[warp][e] = (t >= 0 && t < Li) ? t : -1;
  }
  __syncwarp();
  // 2. every row of every tile requested at once, one commit group
  const uint32_t ring = smem_addr(g_smem) + warp * G::WARP_BYTES;
  const int c_row = lane / G::UNITS, c_unit = lane % G::UNITS;
#pragma unroll
  for (int j = 0; j < GT_MAX; ++j) {
    const uint32_t st = ring + j * G::STAGE;
#pragma unroll
    for (int k = 0; k < G::COPIES; ++k) {
      const int r = G::RPC * k + c_row;
      const int t = tok_s[warp][j * 16 + r];
      const uint32_t dst = st + r * ROW + 16 * (c_unit ^ ((r & 1) << 2));
      cp_async16(dst, kbase + (size_t)max(t, 0) * ROW + 16 * c_unit, t >= 0);
    }
    if (FP8 && lane < 16) {
      const int t = tok_s[warp][j * 16 + lane];
      cp_async4(st + G::TILE + 4 * lane, sbase + max(t, 0), t >= 0);
    }
  }
  cp_async_commit();

  // 3. query fragments (overlapping the copies)
  for (int b = tid; b < TOPK_HIST_BINS; b += SC_THREADS) shist[b] = 0;
  build_query_frags<NT, FP8, SC_THREADS>(c, qv, i, heads, h, bfrag, w_s, scale_s, tid, [] { __syncthreads(); });
  __syncthreads();
  float wr[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    wr[nt][0] = w_s[nt * 8 + 2 * cq];
    wr[nt][1] = w_s[nt * 8 + 2 * cq + 1];
  }
  cp_async_wait<0>();
  __syncwarp();

  // 4. the tiles, from shared memory
  const int swz = (g & 1) << 2;  // rows g and g + 8 share the parity of g
  const int me = cq & 1;         // lanes cq = 0 / 1 write rows g / g + 8
  const uint8_t *wring = g_smem + warp * G::WARP_BYTES;
#pragma unroll 1
  for (int j = 0; j < GT_MAX; ++j) {
    const int p0 = col0 + (j * SC_WARPS + warp) * 16;
    if (p0 >= col1) break;  // uniform over the warp
    const uint8_t *st = wring + j * G::STAGE;
    uint4 kv[2][NV];
    const uint8_t *rowA = st + g * ROW, *rowB = rowA + 8 * ROW;
#pragma unroll
    for (int ch = 0; ch < NV; ++ch) {
      const int u = (cq + 4 * ch) ^ swz;
      kv[0][ch] = *reinterpret_cast<const uint4 *>(rowA + 16 * u);
      kv[1][ch] = *reinterpret_cast<const uint4 *>(rowB + 16 * u);
    }
    const int rme = g + 8 * me;
    const int t = tok_s[warp][j * 16 + rme];
    const float sc = FP8 ? reinterpret_cast<const float *>(st + G::TILE)[rme] : 1.f;
    float acc[NT][4];
    tile_mma<NT, FP8>(kv, bfrag, lane, acc);
    const float2 sums = tile_reduce<NT>(acc, wr);
    if (cq < 2 && t >= 0) {
      const float v = (me ? sums.y : sums.x) * sc;
      scores[(size_t)i * ld + p0 + rme] = v;
      atomicAdd(&shist[ordered_key(v) >> 21], 1u);
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
  constexpr int SMEM = SC_WARPS * GatherCfg<FP8>::WARP_BYTES;
  struct Tag {};
  const int st = cached_per_device<Tag>([] {
    return 1 + (int)cudaFuncSetAttribute(score_gather_kernel<NT, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         SMEM);
  });
  if (st != 1) return (cudaError_t)(st - 1);
  return launch_kernel(score_gather_kernel<NT, FP8>, grid, dim3(SC_THREADS), SMEM, s, c, q, heads, h, gather, n_cols,
                    scores, ld, chunk, row_hist);
}

}  // namespace

cudaError_t launch_score_mma(const CacheView &c, const QueryView &q, const int32_t *heads, int h,
                             const int32_t *gather, int n_cols, float *scores, long long ld, uint32_t *row_hist,
                             cudaStream_t s) {
  if (q.n_q == 0) return cudaSuccess;
  if (!gather) {
    // e4m3 keys with 32 or more scoring heads (dense decode): the dense
    // product on tcgen05 (74.8 against 139.3 us for 8 x 128K keys and 64
    // heads); fewer heads (routed decode), and bf16 keys (whose 32 KB tiles
    // leave one CTA per SM there: 125 against 77 us for 32 x 32K and 64
    // heads), stream the keys on mma.sync
    const int he = heads ? h : q.H;
    if (c.fp8 && he >= 32 && rerank_umma_applies(q, heads, h))
      return launch_rerank_umma(c, q, heads, h, nullptr, c.L_cap, scores, ld, row_hist, s);
    return launch_score_stream(c, q, heads, h, scores, ld, row_hist, s);
  }
  if (rerank_umma_applies(q, heads, h))
    return launch_rerank_umma(c, q, heads, h, gather, n_cols, scores, ld, row_hist, s);
  const int h_eff = heads ? h : q.H;
  int NT = 1;
  while (NT * 8 < h_eff) NT *= 2;
  // CTAs of up to GT_MAX tiles of 16 candidates per warp; fewer tiles per
  // warp when that still leaves at most about one CTA per SM
  const int sms = device_sms();
  const int quantum = SC_WARPS * 16;
  int tpw = GT_MAX;
  while (tpw > 1 && (long long)q.n_q * cdiv(n_cols, (tpw / 2) * quantum) <= sms) tpw /= 2;
  const int chunk = tpw * quantum;
  const int splits = cdiv(n_cols, chunk);
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
