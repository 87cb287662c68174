// Top-k token selection: radix select over a thread-block cluster.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference":
// the indexer keeps the k highest-scoring prefix tokens for the main sparse
// attention (abstract; technical summary "Methodology: MISA", step 2), and
// MISA-dagger keeps k' candidates from the routed pass ("Hierarchical
// variant").  Order: larger score first, equal scores to the lower position
// (the lower token index, since positions are ascending token indices).
//
// One cluster of CS CTAs (CS in {1,2,4,8}) owns one row; each CTA holds a
// slice of up to 512*E scores in registers as order-preserving 32-bit keys.
// Every element has a unique 64-bit composite key (score key, ~position).
// Radix passes over 8-bit digits of that composite narrow down the k-th
// largest composite: each pass builds a 256-bin histogram of the still
// undecided elements in shared memory (warp-aggregated with match.any), the
// CTAs of the cluster add each other's histograms through distributed shared
// memory, and every CTA takes the same decision.  A pass stops the search as
// soon as the undecided elements of the chosen bin are exactly the ones still
// needed.  The selected positions are then written in ascending order
// (ballots within a warp, a scan over warps, a prefix over cluster ranks), so
// the output is deterministic and sorted.  Scores are read once from memory.
#include <cooperative_groups.h>

#include "internal.h"

namespace cg = cooperative_groups;

namespace misa {
namespace {

constexpr int TK_THREADS = 512;
constexpr int TK_WARPS = TK_THREADS / 32;

struct TopkShared {
  uint32_t hist[2][256];
  uint32_t warp_tot[TK_WARPS];
  uint32_t cta_valid;   // valid elements of this CTA
  uint32_t cta_sel;     // selected elements of this CTA
  uint32_t digit, above, in_bin;
};

__device__ __forceinline__ uint32_t block_sum_u32(uint32_t v, uint32_t *scratch /*[TK_WARPS]*/) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  uint32_t t = 0;
#pragma unroll
  for (int w = 0; w < TK_WARPS; ++w) t += scratch[w];
  __syncthreads();
  return t;
}

template <int E>
__global__ void __launch_bounds__(TK_THREADS, 1) topk_kernel(CacheView c, QueryView qv, const float *scores,
                                                             long long ld, int n_cols, const int32_t *gather, int k,
                                                             int32_t *out) {
  __shared__ TopkShared sh;
  cg::cluster_group cluster = cg::this_cluster();
  const int CS = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int row = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int s;
  const int Li = query_prefix(c, qv, row, &s);
  const int ncols = gather ? n_cols : Li;
  const int base = rank * (TK_THREADS * E) + warp * (32 * E) + lane;  // position of element e: base + 32e

  uint32_t key[E];
  uint64_t valid = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int p = base + 32 * e;
    bool v = p < ncols;
    if (gather && v) {
      const int t = gather[(size_t)row * n_cols + p];
      v = t >= 0 && t < Li;
    }
    key[e] = v ? ordered_key(scores[(size_t)row * ld + p]) : 0u;
    valid |= (uint64_t)v << e;
  }

  // number of valid elements in the row
  uint32_t nv = block_sum_u32((uint32_t)__popcll(valid), sh.warp_tot);
  if (tid == 0) sh.cta_valid = nv;
  cluster.sync();
  uint32_t n_valid = 0;
  for (int r = 0; r < CS; ++r) n_valid += cluster.map_shared_rank(&sh, r)->cta_valid;
  const uint32_t kk = min((uint32_t)k, n_valid);

  // Composite key K = (key, ~pos); find the kk-th largest by 8-bit digits.
  uint32_t P_hi = 0, M_hi = 0, P_lo = 0, M_lo = 0;
  uint32_t need = kk;
  bool done = (kk == n_valid);  // everything valid is selected
  for (int pass = 0; pass < 8 && !done; ++pass) {
    uint32_t *hist = sh.hist[pass & 1];
    for (int b = tid; b < 256; b += TK_THREADS) hist[b] = 0;
    __syncthreads();
    const int shift = 24 - 8 * (pass & 3);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const uint32_t lo = ~(uint32_t)(base + 32 * e);
      const bool cand = ((valid >> e) & 1) && (key[e] & M_hi) == P_hi && (lo & M_lo) == P_lo;
      const uint32_t dig = ((pass < 4 ? key[e] : lo) >> shift) & 255u;
      const uint32_t tag = cand ? dig : 256u;
      const unsigned peers = __match_any_sync(0xffffffffu, tag);
      if (cand && lane == __ffs(peers) - 1) atomicAdd(&hist[dig], (uint32_t)__popc(peers));
    }
    cluster.sync();
    // totals per bin over the cluster; threads 0..255 own one bin each
    uint32_t tot = 0;
    if (tid < 256)
      for (int r = 0; r < CS; ++r) tot += cluster.map_shared_rank(hist, r)[tid];
    // suffix sums over bins (bin 255 is the largest digit)
    uint32_t suf = tot;  // inclusive suffix within the warp (lanes above)
    if (tid < 256) {
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += v;
      }
      if (lane == 0) sh.warp_tot[warp] = suf;  // warp total
    }
    __syncthreads();
    if (tid < 256) {
      uint32_t after = 0;  // bins in higher warps
      for (int w = warp + 1; w < 8; ++w) after += sh.warp_tot[w];
      const uint32_t incl = suf + after;       // sum of bins >= tid
      const uint32_t excl = incl - tot;        // sum of bins > tid
      if (incl >= need && excl < need) {
        sh.digit = tid;
        sh.above = excl;
        sh.in_bin = tot;
      }
    }
    __syncthreads();
    const uint32_t dsel = sh.digit;
    need -= sh.above;
    if (pass < 4) {
      P_hi |= dsel << shift;
      M_hi |= 255u << shift;
    } else {
      P_lo |= dsel << shift;
      M_lo |= 255u << shift;
    }
    done = (sh.in_bin == need);
    __syncthreads();
  }

  // selection predicate: composite >= (P_hi, P_lo) on the decided bits
  auto selected = [&](int e) -> bool {
    const uint32_t lo = ~(uint32_t)(base + 32 * e);
    const uint32_t kh = key[e] & M_hi, kl = lo & M_lo;
    return ((valid >> e) & 1) && (kh > P_hi || (kh == P_hi && kl >= P_lo));
  };
  uint32_t warp_sel = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) warp_sel += __popc(__ballot_sync(0xffffffffu, selected(e)));
  if (lane == 0) sh.warp_tot[warp] = warp_sel;
  __syncthreads();
  uint32_t off = 0, cta_sel = 0;
  for (int w = 0; w < TK_WARPS; ++w) {
    const uint32_t v = sh.warp_tot[w];
    off += (w < warp) ? v : 0;
    cta_sel += v;
  }
  if (tid == 0) sh.cta_sel = cta_sel;
  cluster.sync();
  for (int r = 0; r < rank; ++r) off += cluster.map_shared_rank(&sh, r)->cta_sel;
  int32_t *orow = out + (size_t)row * k;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const uint32_t m = __ballot_sync(0xffffffffu, selected(e));
    if ((m >> lane) & 1) {
      const int p = base + 32 * e;
      const int t = gather ? gather[(size_t)row * n_cols + p] : p;
      const uint32_t o = off + __popc(m & ((1u << lane) - 1u));
      if (o < (uint32_t)k) orow[o] = t;
    }
    off += __popc(m);
  }
  if (rank == CS - 1)
    for (int p = (int)kk + tid; p < k; p += TK_THREADS) orow[p] = -1;
  cluster.sync();  // no CTA leaves while others may still read its shared memory
}

template <int E>
cudaError_t launch_e(int CS, int rows, const CacheView &c, const QueryView &q, const float *scores, long long ld,
                     int n_cols, const int32_t *gather, int k, int32_t *out, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CS, rows);
  cfg.blockDim = dim3(TK_THREADS);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, topk_kernel<E>, c, q, scores, ld, n_cols, gather, k, out);
}

}  // namespace

cudaError_t launch_topk(const CacheView &c, const QueryView &q, const float *scores, long long ld, int n_cols,
                        const int32_t *gather, int k, int32_t *out, cudaStream_t s) {
  if (q.n_q == 0) return cudaSuccess;
  const int cols = gather ? n_cols : c.L_cap;
  // smallest register slice E (elements per thread) with at most 8 CTAs per row,
  // then as many CTAs as the row needs
  int E = 4;
  while (E < 64 && (long long)8 * TK_THREADS * E < cols) E *= 2;
  if (E < 16 && cols > TK_THREADS * E) E = 16;  // rows longer than one CTA: 16 per thread
  int CS = 1;
  while ((long long)CS * TK_THREADS * E < cols) CS *= 2;
  if (CS > 8) return cudaErrorInvalidValue;
  switch (E) {
    case 4: return launch_e<4>(CS, q.n_q, c, q, scores, ld, n_cols, gather, k, out, s);
    case 8: return launch_e<8>(CS, q.n_q, c, q, scores, ld, n_cols, gather, k, out, s);
    case 16: return launch_e<16>(CS, q.n_q, c, q, scores, ld, n_cols, gather, k, out, s);
    case 32: return launch_e<32>(CS, q.n_q, c, q, scores, ld, n_cols, gather, k, out, s);
    case 64: return launch_e<64>(CS, q.n_q, c, q, scores, ld, n_cols, gather, k, out, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace misa
