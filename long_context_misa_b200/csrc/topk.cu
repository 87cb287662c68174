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
// slice of T*E scores in registers as order-preserving 32-bit keys.  Every
// element has a unique composite key (score key, 2^18-1-position).  Radix
// passes over digits of that composite (12, 12, 8 bits of the score key, then
// 12 and 6 bits of the position, the latter only when scores tie) narrow down
// the k-th largest composite: each pass builds a 4096-bin histogram of the
// still undecided elements in shared memory plus a 256-bin coarse summary;
// after one cluster barrier every CTA adds the cluster's coarse bins through
// distributed shared memory, picks the coarse bin, then adds only the 16 fine
// bins inside it (272 remote words per rank instead of 4096), so every CTA
// takes the same decision at a small exchange cost.  The search stops as soon as the undecided
// elements of the chosen bin are exactly the ones still needed.  The selected
// positions are written in ascending order (ballots within a warp, a scan
// over warps, a prefix over cluster ranks): deterministic and sorted.  Scores
// are read from memory once; pass 0 also counts the valid elements.
#include <cooperative_groups.h>

#include "internal.h"

namespace cg = cooperative_groups;

namespace misa {
namespace {

constexpr int NB = 4096;              // bins per pass (12-bit digits)
constexpr int POS_BITS = 18;          // positions < 2^18 = MISA_MAX_L
constexpr uint32_t POS_MAX = (1u << POS_BITS) - 1u;

// digit layout of pass p: value (0 = score key, 1 = position key), shift, width
__device__ __forceinline__ void pass_digit(int p, int &which, int &shift, int &bits) {
  switch (p) {
    case 0: which = 0; shift = 20; bits = 12; break;
    case 1: which = 0; shift = 8; bits = 12; break;
    case 2: which = 0; shift = 0; bits = 8; break;
    case 3: which = 1; shift = 6; bits = 12; break;
    default: which = 1; shift = 0; bits = 6; break;
  }
}
constexpr int N_PASSES = 5;

constexpr int NC = NB / 16;           // coarse bins (256)
constexpr int MAX_CS = 8;

// Sum of word `idx` of `arr` over the first `n` cluster ranks; the remote
// loads are issued together (fixed trip count) and the own rank reads its
// shared memory directly.
__device__ __forceinline__ uint32_t cluster_sum(cg::cluster_group &cl, const uint32_t *arr, int idx, int n, int self) {
  uint32_t v[MAX_CS];
#pragma unroll
  for (int r = 0; r < MAX_CS; ++r)
    v[r] = (r < n) ? (r == self ? arr[idx] : cl.map_shared_rank(arr, r)[idx]) : 0u;
  uint32_t t = 0;
#pragma unroll
  for (int r = 0; r < MAX_CS; ++r) t += v[r];
  return t;
}

template <int T>
struct TopkShared {
  uint32_t hist[2][NB];                // fine histograms (double-buffered across passes)
  uint32_t coarse[2][NC];              // sums of 16 fine bins
  uint32_t warp_tot[T / 32];
  uint32_t cta_sel;
  uint32_t digit, above, in_bin, cdigit, cabove;
};

template <int T, int E, bool GATHER>
__global__ void __launch_bounds__(T, 1) topk_kernel(CacheView c, QueryView qv, const float *scores, long long ld,
                                                    int n_cols, const int32_t *gather, int k, int32_t *out) {
  constexpr int W = T / 32;
  __shared__ TopkShared<T> sh;
  cg::cluster_group cluster = cg::this_cluster();
  const int CS = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int row = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int s;
  const int Li = query_prefix(c, qv, row, &s);
  const int ncols = GATHER ? n_cols : Li;
  const int base = rank * (T * E) + warp * (32 * E) + lane;  // position of element e: base + 32e

  uint32_t key[E];
  int tokid[GATHER ? E : 1];
  uint64_t valid = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int p = base + 32 * e;
    bool v = p < ncols;
    if (GATHER) {
      const int t = v ? __ldg(gather + (size_t)row * n_cols + p) : -1;
      tokid[GATHER ? e : 0] = t;
      v = v && t >= 0 && t < Li;
    }
    key[e] = v ? ordered_key(__ldg(scores + (size_t)row * ld + p)) : 0u;
    valid |= (uint64_t)v << e;
  }

  uint32_t P_hi = 0, M_hi = 0, P_lo = 0, M_lo = 0;
  uint32_t need = 0, kk = 0;
  bool done = false;
  for (int pass = 0; pass < N_PASSES && !done; ++pass) {
    int which, shift, bits;
    pass_digit(pass, which, shift, bits);
    const uint32_t dmask = (1u << bits) - 1u;
    uint32_t *hist = sh.hist[pass & 1];
    for (int b = tid; b < NB; b += T) hist[b] = 0;
    __syncthreads();
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const uint32_t lo = POS_MAX - (uint32_t)(base + 32 * e);
      const bool cand = ((valid >> e) & 1) && (key[e] & M_hi) == P_hi && (lo & M_lo) == P_lo;
      if (cand) atomicAdd(&hist[((which ? lo : key[e]) >> shift) & dmask], 1u);
    }
    __syncthreads();
    // coarse histogram: 256 bins of 16 fine bins each (local)
    uint32_t *coarse = sh.coarse[pass & 1];
    if (tid < NC) {
      const uint4 *f4 = reinterpret_cast<const uint4 *>(hist + 16 * tid);
      uint32_t t = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 x = f4[j];
        t += x.x + x.y + x.z + x.w;
      }
      coarse[tid] = t;
    }
    cluster.sync();
    // coarse digit from the cluster-wide coarse totals (threads 0..255, one bin each)
    uint32_t ctot = 0;
    if (tid < NC) ctot = cluster_sum(cluster, coarse, tid, CS, rank);
    uint32_t suf = ctot;
    if (tid < NC) {
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += v;
      }
      if (lane == 0) sh.warp_tot[warp] = suf;
    }
    __syncthreads();
    if (pass == 0) {
      uint32_t all = 0;
      for (int w = 0; w < NC / 32; ++w) all += sh.warp_tot[w];
      kk = min((uint32_t)k, all);
      need = kk;
      if (kk == all) {  // every valid element is selected (uniform decision)
        done = true;
        __syncthreads();  // warp_tot is reused below
        break;
      }
    }
    if (tid < NC) {
      uint32_t after = 0;
      for (int w = warp + 1; w < NC / 32; ++w) after += sh.warp_tot[w];
      const uint32_t incl = suf + after, excl = incl - ctot;
      if (excl < need && incl >= need) {
        sh.cdigit = tid;
        sh.cabove = excl;
      }
    }
    __syncthreads();
    // fine digit inside the chosen coarse bin (warp 0, lanes 0..15)
    if (warp == 0) {
      const uint32_t cd = sh.cdigit, need2 = need - sh.cabove;
      uint32_t f = 0;
      if (lane < 16) f = cluster_sum(cluster, hist, 16 * cd + lane, CS, rank);
      uint32_t fs = f;
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, fs, o);
        if (lane + o < 16) fs += v;
      }
      const uint32_t fex = fs - f;
      if (lane < 16 && fex < need2 && fs >= need2) {
        sh.digit = 16 * cd + lane;
        sh.above = sh.cabove + fex;
        sh.in_bin = f;
      }
    }
    __syncthreads();
    const uint32_t dsel = sh.digit;
    need -= sh.above;
    if (which == 0) {
      P_hi |= dsel << shift;
      M_hi |= dmask << shift;
    } else {
      P_lo |= dsel << shift;
      M_lo |= dmask << shift;
    }
    done = (sh.in_bin == need);
    __syncthreads();
  }

  // selection predicate: composite >= (P_hi, P_lo) on the decided bits
  auto selected = [&](int e) -> bool {
    const uint32_t lo = POS_MAX - (uint32_t)(base + 32 * e);
    const uint32_t kh = key[e] & M_hi, kl = lo & M_lo;
    return ((valid >> e) & 1) && (kh > P_hi || (kh == P_hi && kl >= P_lo));
  };
  uint32_t warp_sel = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) warp_sel += __popc(__ballot_sync(0xffffffffu, selected(e)));
  if (lane == 0) sh.warp_tot[warp] = warp_sel;
  __syncthreads();
  uint32_t off = 0, cta_sel = 0;
  for (int w = 0; w < W; ++w) {
    const uint32_t v = sh.warp_tot[w];
    off += (w < warp) ? v : 0;
    cta_sel += v;
  }
  if (tid == 0) sh.cta_sel = cta_sel;
  cluster.sync();
  off += cluster_sum(cluster, &sh.cta_sel, 0, rank, rank);
  int32_t *orow = out + (size_t)row * k;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const uint32_t m = __ballot_sync(0xffffffffu, selected(e));
    if ((m >> lane) & 1) {
      const int p = base + 32 * e;
      const int t = GATHER ? tokid[GATHER ? e : 0] : p;
      const uint32_t o = off + __popc(m & ((1u << lane) - 1u));
      if (o < (uint32_t)k) orow[o] = t;
    }
    off += __popc(m);
  }
  if (rank == CS - 1)
    for (int p = (int)kk + tid; p < k; p += T) orow[p] = -1;
  cluster.sync();  // no CTA leaves while others may still read its shared memory
}

template <int T, int E, bool GATHER>
cudaError_t launch_te(int CS, int rows, const CacheView &c, const QueryView &q, const float *scores, long long ld,
                      int n_cols, const int32_t *gather, int k, int32_t *out, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CS, rows);
  cfg.blockDim = dim3(T);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, topk_kernel<T, E, GATHER>, c, q, scores, ld, n_cols, gather, k, out);
}

}  // namespace

cudaError_t launch_topk(const CacheView &c, const QueryView &q, const float *scores, long long ld, int n_cols,
                        const int32_t *gather, int k, int32_t *out, cudaStream_t s) {
  if (q.n_q == 0) return cudaSuccess;
  const long long cols = gather ? n_cols : c.L_cap;
  // 1024 threads x E in {4, 8, 16} per CTA and up to 8 CTAs per row; the
  // longest rows (above 131072) use 512 threads x 64.
  auto go = [&](int T, int E) -> cudaError_t {
    int CS = 1;
    while ((long long)CS * T * E < cols) CS *= 2;
    if (CS > 8) return cudaErrorInvalidValue;
    if (gather) {
      if (T == 1024 && E == 4) return launch_te<1024, 4, true>(CS, q.n_q, c, q, scores, ld, n_cols, gather, k, out, s);
      if (T == 1024 && E == 8) return launch_te<1024, 8, true>(CS, q.n_q, c, q, scores, ld, n_cols, gather, k, out, s);
      if (T == 1024 && E == 16) return launch_te<1024, 16, true>(CS, q.n_q, c, q, scores, ld, n_cols, gather, k, out, s);
      return launch_te<512, 64, true>(CS, q.n_q, c, q, scores, ld, n_cols, gather, k, out, s);
    }
    if (T == 1024 && E == 4) return launch_te<1024, 4, false>(CS, q.n_q, c, q, scores, ld, n_cols, gather, k, out, s);
    if (T == 1024 && E == 8) return launch_te<1024, 8, false>(CS, q.n_q, c, q, scores, ld, n_cols, gather, k, out, s);
    if (T == 1024 && E == 16) return launch_te<1024, 16, false>(CS, q.n_q, c, q, scores, ld, n_cols, gather, k, out, s);
    return launch_te<512, 64, false>(CS, q.n_q, c, q, scores, ld, n_cols, gather, k, out, s);
  };
  if (cols <= 1024 * 4) return go(1024, 4);
  if (cols <= 1024 * 8) return go(1024, 8);
  if (cols <= 8LL * 1024 * 16) return go(1024, 16);
  return go(512, 64);
}

}  // namespace misa
