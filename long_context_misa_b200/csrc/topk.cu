// Top-k token selection: radix select over a thread-block cluster, starting
// from a histogram the scoring kernel built while writing the scores.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference":
// the indexer keeps the k highest-scoring prefix tokens for the main sparse
// attention (abstract; technical summary "Methodology: MISA", step 2), and
// MISA-dagger keeps k' candidates from the routed pass ("Hierarchical
// variant").  Order: larger score first, equal scores to the lower position
// (the lower token index, since positions are ascending token indices).
//
// Keys: the order-preserving 32-bit image of each score; each element's
// composite key is (score key, 2^18-1-position), unique in a row.  The result
// is every element whose composite is at least the kk-th largest one
// (kk = min(k, valid elements)), written in ascending position order.
//
// The scoring kernel has already counted the row's keys by their top 11 bits
// (row_hist, 2048 bins).  One cluster of CS CTAs (CS in {1,2,4,8}) owns a row;
// each CTA keeps its slice of T*E keys in shared memory.
//   1. Every CTA reads row_hist and finds the same boundary bin d0 (block
//      scan, no exchange); it counts its keys above and in d0 and, unless the
//      whole bin is needed, appends its keys in d0 to a shared list.  (barrier 1)
//   2. Rank 0 gathers the lists through distributed shared memory, finishes
//      the radix select on the remaining 21 key bits and the position in its
//      shared memory (2048-bin passes with early exit), and turns the
//      per-rank counts into output offsets.                       (barrier 2)
//   3. Every CTA reads the threshold and its offset and writes its selected
//      positions in order (warp ballots, a scan over warps).      (barrier 3)
// A boundary bin too large to gather falls back to cluster-wide passes.
#include <cooperative_groups.h>

#include "internal.h"

namespace cg = cooperative_groups;

namespace misa {
namespace {

constexpr int POS_BITS = 18;                 // positions < 2^18 = MISA_MAX_L
constexpr uint32_t POS_MAX = (1u << POS_BITS) - 1u;
constexpr int MAX_CS = 8;
constexpr int CAP = 8192;                    // boundary-bin elements rank 0 can gather
constexpr int RB = TOPK_HIST_BINS;           // bins per pass (11-bit digits)
constexpr uint32_t TOP_MASK = 0xFFE00000u;   // the histogram's 11 bits
// passes after the histogram: key bits 20..10, 9..0, then position bits 17..9, 8..0
__device__ constexpr int kShift[4] = {10, 0, 9, 0};
__device__ constexpr int kWidth[4] = {11, 10, 9, 9};

template <int T>
struct SelShared {
  uint32_t lhist[RB];
  uint32_t wtot[T / 32];                     // per-warp totals
  uint32_t wscan[T / 32];                    // scans of wtot
  uint32_t n_cand, n_hi, n_in;               // this CTA: listed, above d0, in d0
  uint32_t res[3];                           // digit, above, in_bin of the last search
  uint32_t dec[4];                           // rank 0's threshold: P_hi, M_hi, P_lo, M_lo
  uint32_t offs[MAX_CS];                     // rank 0's output offset per rank
  uint32_t sel_cnt[MAX_CS];                  // rank 0: selected listed elements per rank
  uint32_t cand_key[CAP];
  uint32_t cand_lo[CAP];
  uint8_t cand_rank[CAP];
};

template <int T, int E>
constexpr int sel_smem_bytes() {
  return (int)sizeof(SelShared<T>) + T * E * 4;
}

// Exclusive scan of the warps' values `mine` (warp w's at wscan[w]) by warp 0;
// returns the block total.  Two barriers.
template <int T>
__device__ __forceinline__ uint32_t warp_totals_scan(uint32_t mine, uint32_t *wtot, uint32_t *wscan) {
  constexpr int W = T / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) wtot[warp] = mine;
  __syncthreads();
  if (warp == 0) {
    const uint32_t v = lane < W ? wtot[lane] : 0u;
    uint32_t inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += u;
    }
    if (lane < W) wscan[lane] = inc - v;
    if (lane == 31) wtot[0] = inc;  // block total (wtot is not read again)
  }
  __syncthreads();
  return wtot[0];
}

// Bin holding the need-th largest element of a 2048-bin histogram whose bins
// [2*tid, 2*tid+1] are c0, c1 (bins grow with the key): res[0..2] = digit,
// count above it, its count.  Three barriers; everyone reads res afterwards.
template <int T>
__device__ __forceinline__ void hist_search(uint32_t c0, uint32_t c1, uint32_t need, SelShared<T> &sh) {
  static_assert(RB == 2 * T, "two bins per thread");
  constexpr int W = T / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t mine = c0 + c1;
  uint32_t suf = mine;  // inclusive suffix over the lanes of this warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t u = __shfl_down_sync(0xffffffffu, suf, o);
    if (lane + o < 32) suf += u;
  }
  if (lane == 0) sh.wtot[warp] = suf;
  __syncthreads();
  if (warp == 0) {  // wscan[w] = elements in warps above w
    const uint32_t v = lane < W ? sh.wtot[lane] : 0u;
    uint32_t sfx = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_down_sync(0xffffffffu, sfx, o);
      if (lane + o < 32) sfx += u;
    }
    if (lane < W) sh.wscan[lane] = sfx - v;
  }
  __syncthreads();
  const uint32_t above1 = (suf - mine) + sh.wscan[warp];  // elements in bins above 2*tid+1
  if (above1 < need && above1 + c1 >= need) {
    sh.res[0] = 2 * threadIdx.x + 1;
    sh.res[1] = above1;
    sh.res[2] = c1;
  } else if (above1 + c1 < need && above1 + c1 + c0 >= need) {
    sh.res[0] = 2 * threadIdx.x;
    sh.res[1] = above1 + c1;
    sh.res[2] = c0;
  }
  __syncthreads();
}

template <int T, int E, bool GATHER>
__global__ void __launch_bounds__(T, 1) select_kernel(CacheView c, QueryView qv, const float *scores, long long ld,
                                                      int n_cols, const int32_t *gather,
                                                      const uint32_t *row_hist, int k, int32_t *out) {
  extern __shared__ __align__(16) uint8_t sel_smem[];
  SelShared<T> &sh = *reinterpret_cast<SelShared<T> *>(sel_smem);
  uint32_t *skey = reinterpret_cast<uint32_t *>(sel_smem + sizeof(SelShared<T>));  // [E][T]
#define KEY(e) skey[(e) * T + tid]
  cg::cluster_group cluster = cg::this_cluster();
  const int CS = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int row = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int s;
  const int Li = query_prefix(c, qv, row, &s);
  const int ncols = GATHER ? n_cols : Li;
  const int base = rank * (T * E) + warp * (32 * E) + lane;  // position of element e: base + 32e

  // ---- load: this thread's keys and two bins of the row histogram ----
  const uint32_t *rh = row_hist + (size_t)row * RB;
  const uint32_t h0 = rh[2 * tid], h1 = rh[2 * tid + 1];
  uint32_t valid = 0;
  {
    int tk[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int p = base + 32 * e;
      tk[e] = (GATHER && p < ncols) ? __ldg(gather + (size_t)row * n_cols + p) : p;
    }
    float sv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int p = base + 32 * e;
      const bool v = p < ncols && (!GATHER || (tk[e] >= 0 && tk[e] < Li));
      sv[e] = v ? scores[(size_t)row * ld + p] : 0.f;
      valid |= (uint32_t)v << e;
    }
#pragma unroll
    for (int e = 0; e < E; ++e) KEY(e) = ((valid >> e) & 1) ? ordered_key(sv[e]) : 0u;
  }
  if (tid == 0) {
    sh.n_cand = 0;
    sh.n_hi = 0;
    sh.n_in = 0;
  }
  if (tid < MAX_CS) sh.sel_cnt[tid] = 0;

  // ---- 1. boundary bin from the histogram (same result in every CTA) ----
  const uint32_t all = warp_totals_scan<T>(__reduce_add_sync(0xffffffffu, h0 + h1), sh.wtot, sh.wscan);
  const uint32_t kk = min((uint32_t)k, all);
  uint32_t need = kk;
  uint32_t P_hi = 0, M_hi = 0, P_lo = 0, M_lo = 0;
  const bool all_in = kk == all;  // uniform: every valid element is selected
  uint32_t d0 = 0, in0 = 0;
  if (!all_in) {
    hist_search<T>(h0, h1, need, sh);
    d0 = sh.res[0];
    need -= sh.res[1];
    in0 = sh.res[2];
    P_hi = d0 << 21;
    M_hi = TOP_MASK;
  }
  const bool listed = !all_in && in0 != need && in0 <= CAP;   // uniform
  const bool fallback = !all_in && in0 != need && in0 > CAP;  // uniform
  uint32_t n_hi = 0, n_in = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const uint32_t kx = KEY(e);
    const bool v = (valid >> e) & 1;
    n_hi += (v && (all_in || (kx >> 21) > d0)) ? 1u : 0u;
    const bool cd = v && !all_in && (kx >> 21) == d0;
    n_in += cd ? 1u : 0u;
    if (listed) {
      const unsigned m = __ballot_sync(0xffffffffu, cd);
      if (m) {
        uint32_t slot = 0;
        if (lane == 0) slot = atomicAdd(&sh.n_cand, (uint32_t)__popc(m));
        slot = __shfl_sync(0xffffffffu, slot, 0);
        if (cd) {
          const uint32_t o = slot + __popc(m & ((1u << lane) - 1u));
          sh.cand_key[o] = kx;
          sh.cand_lo[o] = POS_MAX - (uint32_t)(base + 32 * e);
          sh.cand_rank[o] = (uint8_t)rank;
        }
      }
    }
  }
  n_hi = __reduce_add_sync(0xffffffffu, n_hi);
  n_in = __reduce_add_sync(0xffffffffu, n_in);
  if (lane == 0) {
    atomicAdd(&sh.n_hi, n_hi);
    atomicAdd(&sh.n_in, n_in);
  }
  cluster.sync();  // barrier 1

  // ---- 2. rank 0: exact threshold and output offsets ----
  if (rank == 0 && !fallback) {
    uint32_t cnt_hi[MAX_CS], cnt_in[MAX_CS], cbase[MAX_CS + 1];
    cbase[0] = 0;
#pragma unroll
    for (int r = 0; r < MAX_CS; ++r) {
      const SelShared<T> *o = cluster.map_shared_rank(&sh, r < CS ? r : 0);
      cnt_hi[r] = r < CS ? o->n_hi : 0u;
      cnt_in[r] = r < CS ? o->n_in : 0u;
      cbase[r + 1] = cbase[r] + (r < CS && listed ? o->n_cand : 0u);
    }
    if (listed) {
      const uint32_t C = cbase[MAX_CS];
      // the other ranks' lists go behind this CTA's own
#pragma unroll 4
      for (uint32_t x = cbase[1] + tid; x < C; x += T) {
        int r = 1;
#pragma unroll
        for (int q = 2; q < MAX_CS; ++q) r = (x >= cbase[q]) ? q : r;
        const SelShared<T> *o = cluster.map_shared_rank(&sh, r);
        const uint32_t idx = x - cbase[r];
        sh.cand_key[x] = o->cand_key[idx];
        sh.cand_lo[x] = o->cand_lo[idx];
        sh.cand_rank[x] = o->cand_rank[idx];
      }
      __syncthreads();
      bool done = false;
      for (int p = 0; p < 4 && !done; ++p) {
        const bool lo_word = p >= 2;
        const int sft = kShift[p];
        const uint32_t dm = (1u << kWidth[p]) - 1u;
        for (int b = tid; b < RB; b += T) sh.lhist[b] = 0;
        __syncthreads();
        for (uint32_t x = tid; x < C; x += T) {
          const uint32_t kx = sh.cand_key[x], lx = sh.cand_lo[x];
          if ((kx & M_hi) == P_hi && (lx & M_lo) == P_lo) atomicAdd(&sh.lhist[((lo_word ? lx : kx) >> sft) & dm], 1u);
        }
        __syncthreads();
        hist_search<T>(sh.lhist[2 * tid], sh.lhist[2 * tid + 1], need, sh);
        const uint32_t dg = sh.res[0];
        need -= sh.res[1];
        if (!lo_word) {
          P_hi |= dg << sft;
          M_hi |= dm << sft;
        } else {
          P_lo |= dg << sft;
          M_lo |= dm << sft;
        }
        done = sh.res[2] == need;
      }
      // selected listed elements, per source rank
      for (uint32_t x = tid; x < C; x += T) {
        const uint32_t kh = sh.cand_key[x] & M_hi, kl = sh.cand_lo[x] & M_lo;
        if (kh > P_hi || (kh == P_hi && kl >= P_lo)) atomicAdd(&sh.sel_cnt[sh.cand_rank[x]], 1u);
      }
      __syncthreads();
    }
    if (tid == 0) {
      uint32_t off = 0;
      for (int r = 0; r < MAX_CS; ++r) {
        sh.offs[r] = off;
        off += cnt_hi[r] + (listed ? sh.sel_cnt[r] : cnt_in[r]);  // unlisted: the whole bin d0 is in
      }
      sh.dec[0] = P_hi;
      sh.dec[1] = M_hi;
      sh.dec[2] = P_lo;
      sh.dec[3] = M_lo;
    }
  }
  cluster.sync();  // barrier 2
  uint32_t off = 0;
  if (!fallback) {
    const SelShared<T> *r0 = cluster.map_shared_rank(&sh, 0);
    off = r0->offs[rank];
    P_hi = r0->dec[0];
    M_hi = r0->dec[1];
    P_lo = r0->dec[2];
    M_lo = r0->dec[3];
  } else {
    // Boundary bin beyond the gather capacity: cluster-wide passes over the
    // slices (the histograms meet through distributed shared memory).
    bool done = false;
    for (int p = 0; p < 4 && !done; ++p) {
      const bool lo_word = p >= 2;
      const int sft = kShift[p];
      const uint32_t dm = (1u << kWidth[p]) - 1u;
      for (int b = tid; b < RB; b += T) sh.lhist[b] = 0;
      __syncthreads();
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const uint32_t lo = POS_MAX - (uint32_t)(base + 32 * e), kx = KEY(e);
        if (((valid >> e) & 1) && (kx & M_hi) == P_hi && (lo & M_lo) == P_lo)
          atomicAdd(&sh.lhist[((lo_word ? lo : kx) >> sft) & dm], 1u);
      }
      cluster.sync();
      uint32_t c0 = 0, c1 = 0;
      for (int r = 0; r < CS; ++r) {
        const uint32_t *hr = cluster.map_shared_rank(sh.lhist, r);
        c0 += hr[2 * tid];
        c1 += hr[2 * tid + 1];
      }
      cluster.sync();  // every rank has read every histogram before any clears its own
      hist_search<T>(c0, c1, need, sh);
      const uint32_t dg = sh.res[0];
      need -= sh.res[1];
      if (!lo_word) {
        P_hi |= dg << sft;
        M_hi |= dm << sft;
      } else {
        P_lo |= dg << sft;
        M_lo |= dm << sft;
      }
      done = sh.res[2] == need;
    }
  }

  // ---- 3. ordered output: composite >= (P_hi, P_lo) on the decided bits ----
  uint32_t selm = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const uint32_t lo = POS_MAX - (uint32_t)(base + 32 * e);
    const uint32_t kh = KEY(e) & M_hi, kl = lo & M_lo;
    selm |= (uint32_t)(((valid >> e) & 1) && (kh > P_hi || (kh == P_hi && kl >= P_lo))) << e;
  }
  uint32_t wsel = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) wsel += __popc(__ballot_sync(0xffffffffu, (selm >> e) & 1));
  const uint32_t cta_sel = warp_totals_scan<T>(wsel, sh.wtot, sh.wscan);
  if (fallback) {  // offsets from a prefix over the ranks' selected counts
    if (tid == 0) sh.n_hi = cta_sel;
    cluster.sync();
    for (int r = 0; r < rank; ++r) off += cluster.map_shared_rank(&sh, r)->n_hi;
  }
  off += sh.wscan[warp];
  int32_t *orow = out + (size_t)row * k;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const uint32_t m = __ballot_sync(0xffffffffu, (selm >> e) & 1);
    if ((m >> lane) & 1) {
      const int p = base + 32 * e;
      const int t = GATHER ? __ldg(gather + (size_t)row * n_cols + p) : p;
      const uint32_t o = off + __popc(m & ((1u << lane) - 1u));
      if (o < (uint32_t)k) orow[o] = t;
    }
    off += __popc(m);
  }
  if (rank == CS - 1)
    for (int p = (int)kk + tid; p < k; p += T) orow[p] = -1;
  cluster.sync();  // barrier 3: no CTA leaves while others may still read its shared memory
#undef KEY
}

template <int T, int E, bool GATHER>
cudaError_t launch_te(int CS, int rows, const CacheView &c, const QueryView &q, const float *scores, long long ld,
                      int n_cols, const int32_t *gather, const uint32_t *row_hist, int k, int32_t *out,
                      cudaStream_t s) {
  constexpr int SMEM = sel_smem_bytes<T, E>();
  struct Tag {};
  const int ok = cached_per_device<Tag>([] {
    return cudaFuncSetAttribute(select_kernel<T, E, GATHER>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) ==
                   cudaSuccess
               ? 1
               : -1;
  });
  if (ok < 0) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CS, rows);
  cfg.blockDim = dim3(T);
  cfg.dynamicSmemBytes = SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, select_kernel<T, E, GATHER>, c, q, scores, ld, n_cols, gather, row_hist, k, out);
}

}  // namespace

cudaError_t launch_topk(const CacheView &c, const QueryView &q, const float *scores, long long ld, int n_cols,
                        const int32_t *gather, const uint32_t *row_hist, int k, int32_t *out, cudaStream_t s) {
  if (q.n_q == 0) return cudaSuccess;
  const long long cols = gather ? n_cols : c.L_cap;
  // 1024 threads x E keys per CTA (E in {4, 8, 16, 32}), up to 8 CTAs per row
  int E = 4;
  while (E < 32 && (long long)MAX_CS * 1024 * E < cols) E *= 2;
  if (E < 8 && cols > 1024LL * E) E = 8;
  int CS = 1;
  while ((long long)CS * 1024 * E < cols) CS *= 2;
  if (CS > MAX_CS) return cudaErrorInvalidValue;
#define MISA_TOPK_CASE(EE)                                                                                     \
  case EE:                                                                                                     \
    return gather ? launch_te<1024, EE, true>(CS, q.n_q, c, q, scores, ld, n_cols, gather, row_hist, k, out, s) \
                  : launch_te<1024, EE, false>(CS, q.n_q, c, q, scores, ld, n_cols, gather, row_hist, k, out, s);
  switch (E) {
    MISA_TOPK_CASE(4)
    MISA_TOPK_CASE(8)
    MISA_TOPK_CASE(16)
    MISA_TOPK_CASE(32)
    default:
      return cudaErrorInvalidValue;
  }
#undef MISA_TOPK_CASE
}

}  // namespace misa
