// Top-k token selection from the scores and the per-row histogram the
// scoring kernel built while writing them.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference":
// the indexer keeps the k highest-scoring prefix tokens for the main sparse
// attention (abstract; technical summary "Methodology: MISA", step 2), and
// MISA-dagger keeps k' candidates from the routed pass ("Hierarchical
// variant").  Order: larger score first, equal scores to the lower token
// index.  Every element's composite key (order-preserving image of the score,
// 2^18-1-token) is unique in a row; the result is every element whose
// composite is at least the kk-th largest (kk = min(k, valid elements)),
// written as token indices in ascending order.
//
// The scoring kernel counted the row's keys by their top 11 bits (row_hist,
// 2048 bins).  From it every kernel here finds the same boundary bin d0:
// elements above d0 are selected outright, elements below are not, and only
// the elements inside d0 need the remaining 21 key bits and the token.
//
// select_kernel, one CTA per row:
//   1. boundary bin from the histogram (one warp);
//   2. one pass over the row -- or over the compact list the filter kernel
//      wrote -- marks every element above d0 in a token bitmap in shared
//      memory and lists the elements of d0 (key, token) in shared memory;
//   3. radix passes over the listed d0 elements only (11 key bits; then,
//      once at most 512 elements remain in the boundary bin, their exact
//      ranks by counting) fix the threshold; the winners are marked;
//   4. a popcount scan of the bitmap writes the tokens in ascending order,
//      the outputs split evenly over the threads.
//   A d0 too large to list (degenerate score distributions) falls back to
//   the same radix passes over the whole row, read from global memory.
// filter_kernel (few long rows: decode): many CTAs per row copy the elements
//   at or above d0 into a per-row list, so that the one CTA per row above
//   reads about k + |d0| entries instead of the whole row.
// Tensor-core prefill rows come without a histogram.  sample_thr_kernel
//   reads a sample of each row and writes a bound below its k-th largest key
//   (with high probability); filter_thr_kernel lists the elements at or above
//   the bound; the staged selection counts the list itself (OWN).  A row whose
//   list came out short or overfull is counted and selected from its whole
//   score row instead, so the result never depends on the sample.
#include <algorithm>

#include "selcore.cuh"

namespace misa {
namespace {

constexpr int CAP = TOPK_LIST_EXTRA;         // d0 elements refined in shared memory
constexpr int SEL_T = 512;                   // select_kernel threads
constexpr int SEL_W = SEL_T / 32;
constexpr int FILT_T = 256;                  // filter_kernel threads

struct SelShared {
  Boundary bd;
  uint4 res;                       // a warp search result
  uint32_t thr[2];                 // threshold composite from the counting step
  uint32_t n_small;
  uint32_t wa[SEL_W], wb[SEL_W + 1];
  uint32_t hist[HPAD];
  uint32_t small_key[SEL_T], small_tie[SEL_T];
  uint32_t cand_key[CAP];
  uint32_t cand_tie[CAP];
};

// Visit the filter kernel's list of n entries (key, token), all valid.
template <int T, class F>
__device__ __forceinline__ void sweep_list(const uint2 *lrow, int n, F &&fn) {
  for (int base = 0; base < n; base += T * U) {
    uint32_t key[U];
    int tk[U];
    bool ok[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int p = base + u * T + threadIdx.x;
      uint2 e = make_uint2(0u, 0u);
      if (p < n) e = __ldg(lrow + p);
      ok[u] = p < n;
      key[u] = e.x;
      tk[u] = (int)e.y;
    }
    fn(key, tk, ok, base);
  }
}

// Software-pipelined sweeps for the select kernel: the caller issues the
// first sweep's loads (load_row / load_list) before the row's length and
// boundary are known, and every sweep requests the next one before visiting
// its own elements.  Loads stay below n_load, the row's allocation.
template <bool GATHER>
__device__ __forceinline__ void load_row(const float *srow, const int32_t *grow, int n_load, int base, int (&tk)[U],
                                         float (&sv)[U]) {
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int p = base + u * SEL_T + threadIdx.x;
    const bool in = p < n_load;
    tk[u] = in ? (GATHER ? __ldg(grow + p) : p) : -1;
    sv[u] = in ? __ldg(srow + p) : 0.f;
  }
}

template <bool GATHER, class F>
__device__ __forceinline__ void sweep_row_pf(const float *srow, const int32_t *grow, int n_load, int n, int Li,
                                             int (&tk)[U], float (&sv)[U], F &&fn) {
  for (int base = 0; base < n; base += SEL_T * U) {
    int ct[U];
    uint32_t key[U];
    bool ok[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int p = base + u * SEL_T + threadIdx.x;
      ct[u] = tk[u];
      ok[u] = p < n && tk[u] >= 0 && tk[u] < Li;
      key[u] = ordered_key(sv[u]);
    }
    if (base + SEL_T * U < n) load_row<GATHER>(srow, grow, n_load, base + SEL_T * U, tk, sv);
    fn(key, ct, ok, base);
  }
}

__device__ __forceinline__ void load_list(const uint2 *lrow, int n_load, int base, uint2 (&e)[U]) {
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int p = base + u * SEL_T + threadIdx.x;
    e[u] = p < n_load ? __ldg(lrow + p) : make_uint2(0u, 0u);
  }
}

template <class F>
__device__ __forceinline__ void sweep_list_pf(const uint2 *lrow, int n_load, int n, uint2 (&e)[U], F &&fn) {
  for (int base = 0; base < n; base += SEL_T * U) {
    int ct[U];
    uint32_t key[U];
    bool ok[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      ok[u] = base + u * SEL_T + (int)threadIdx.x < n;
      key[u] = e[u].x;
      ct[u] = (int)e[u].y;
    }
    if (base + SEL_T * U < n) load_list(lrow, n_load, base + SEL_T * U, e);
    fn(key, ct, ok, base);
  }
}

template <bool GATHER, bool FROM_LIST, bool OWN_HIST>
__global__ void __launch_bounds__(SEL_T) select_kernel(CacheView c, QueryView qv, const float *scores, long long ld,
                                                       int n_cols, const int32_t *gather, const uint32_t *row_hist,
                                                       const uint2 *list, const uint32_t *list_cnt, int list_cap,
                                                       int k, int32_t *out) {
  grid_dep_sync();
  extern __shared__ __align__(16) uint8_t sel_smem[];
  SelShared &sh = *reinterpret_cast<SelShared *>(sel_smem);
  uint32_t *bm = reinterpret_cast<uint32_t *>(sel_smem + sizeof(SelShared));  // token bitmap
  const int row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float *srow = scores + (size_t)row * ld;
  const int32_t *grow = GATHER ? gather + (size_t)row * n_cols : nullptr;
  const uint2 *lrow = FROM_LIST ? list + (size_t)row * list_cap : nullptr;
  const int n_load = GATHER ? n_cols : c.L_cap;  // the row's allocation
  int32_t *orow = out + (size_t)row * k;

  // 1. requested together: the first sweep (row or list), the list length,
  //    the query's prefix and the row histogram; every warp then finds the
  //    boundary bin by itself
  int tk[U];
  float sv[U];
  uint2 le[U];
  if (FROM_LIST)
    load_list(lrow, list_cap, 0, le);
  else
    load_row<GATHER>(srow, grow, n_load, 0, tk, sv);
  const int lcnt = FROM_LIST ? min((int)list_cnt[row], list_cap) : 0;
  int s;
  const int Li = query_prefix(c, qv, row, &s);
  const int n = GATHER ? n_cols : Li;
  const int words = cdiv(Li, 32);
  Boundary bd;
  if (!OWN_HIST && warp == 0) {  // one warp: every warp reading 8 KB would cost 16x the wavefronts
    const Boundary b = warp_boundary(row_hist + (size_t)row * RB, k);
    if (lane == 0) sh.bd = b;
  }
  if (tid == 0) sh.n_small = 0;
  for (int w = tid; w < words; w += SEL_T) bm[w] = 0;
  if (OWN_HIST) {
    // no histogram from the scoring kernel: count the row's top 11 key bits
    for (int b = tid; b < HPAD; b += SEL_T) sh.hist[b] = 0;
    __syncthreads();
    sweep_row_pf<GATHER>(srow, grow, n_load, n, Li, tk, sv,
                         [&](const uint32_t(&key)[U], const int(&)[U], const bool(&ok)[U], int) {
#pragma unroll
                           for (int u = 0; u < U; ++u)
                             if (ok[u]) atomicAdd(&sh.hist[hpos(key[u] >> HIST_SHIFT)], 1u);
                         });
    __syncthreads();
    if (warp == 0) {
      const Boundary b = warp_boundary_smem(sh.hist, k);
      if (lane == 0) sh.bd = b;
    }
  }
  __syncthreads();
  bd = sh.bd;

  if (bd.kk > 0) {
    const uint32_t d0 = bd.d0;
    const uint32_t need = bd.need();
    const bool whole = bd.all_in || need == bd.in0;  // no refinement needed
    const bool listed = !whole && bd.in0 <= (uint32_t)CAP;
    uint32_t P_hi = d0 << HIST_SHIFT, M_hi = TOP_MASK, P_lo = 0, M_lo = 0;
    const bool via_list = FROM_LIST && bd.listable((uint32_t)CAP);
    // tokens of a warp's 32 consecutive row positions are consecutive: their
    // bitmap word is the warp's ballot
    const bool word_marks = !GATHER && !via_list;
    auto mark_sweep = [&](const bool(&sel)[U], const int(&tk)[U], int base) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (word_marks) {
          const uint32_t m = __ballot_sync(0xffffffffu, sel[u]);
          const int p0 = base + u * SEL_T + warp * 32;
          if (lane == 0 && p0 < n) bm[p0 >> 5] = m;
        } else if (sel[u]) {
          mark(bm, tk[u]);
        }
      }
    };
    if (whole || listed) {
      // 2. mark everything above the boundary (and d0 too when whole); list
      //    d0 with ballots and one scan over the warps per sweep
      uint32_t n_listed = 0;
      auto visit = [&](const uint32_t(&key)[U], const int(&tk)[U], const bool(&ok)[U], int base) {
        bool sel[U];
        uint32_t lm[U], cnt = 0;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const uint32_t bin = key[u] >> HIST_SHIFT;
          sel[u] = ok[u] && (bd.all_in || bin > d0 || (whole && bin == d0));
          lm[u] = __ballot_sync(0xffffffffu, listed && ok[u] && bin == d0);
          cnt += __popc(lm[u]);
        }
        mark_sweep(sel, tk, base);
        if (listed) {
          if (lane == 0) sh.wa[warp] = cnt;
          __syncthreads();
          const uint32_t x = lane < SEL_W ? sh.wa[lane] : 0u;
          const uint32_t before = __reduce_add_sync(0xffffffffu, lane < warp ? x : 0u);
          const uint32_t tot = __reduce_add_sync(0xffffffffu, x);
          __syncthreads();
          uint32_t slot = n_listed + before;
          const uint32_t lt = lanemask_lt();
#pragma unroll
          for (int u = 0; u < U; ++u) {
            if ((lm[u] >> lane) & 1) {
              const uint32_t o = slot + __popc(lm[u] & lt);
              if (o < (uint32_t)CAP) {
                sh.cand_key[o] = key[u];
                sh.cand_tie[o] = POS_MAX - (uint32_t)tk[u];
              }
            }
            slot += __popc(lm[u]);
          }
          n_listed += tot;
        }
      };
      if (via_list)
        sweep_list_pf(lrow, list_cap, lcnt, le, visit);
      else if (!FROM_LIST && !OWN_HIST)
        sweep_row_pf<GATHER>(srow, grow, n_load, n, Li, tk, sv, visit);
      else
        sweep_row<SEL_T, GATHER>(srow, grow, n, Li, visit);
      __syncthreads();
      if (listed) {
        // 3. exact threshold among the listed elements of d0, then their winners
        const int nc = min((int)n_listed, CAP);
        refine<true, SEL_T>(sh, P_hi, M_hi, P_lo, M_lo, need, bd.in0, [&](auto &&fn) {
          for (int x = tid; x < nc; x += SEL_T) fn(sh.cand_key[x], sh.cand_tie[x], true);
        });
        for (int x = tid; x < nc; x += SEL_T)
          if (at_least(sh.cand_key[x], sh.cand_tie[x], P_hi, M_hi, P_lo, M_lo))
            mark(bm, (int)(POS_MAX - sh.cand_tie[x]));
        __syncthreads();
      }
    } else {
      // d0 too large to list: radix passes over the whole row, then one
      // marking pass (composite at or above the threshold on the decided bits)
      refine<false, SEL_T>(sh, P_hi, M_hi, P_lo, M_lo, need, bd.in0, [&](auto &&fn) {
        sweep_row<SEL_T, GATHER>(srow, grow, n, Li,
                                 [&](const uint32_t(&key)[U], const int(&tk)[U], const bool(&ok)[U], int) {
#pragma unroll
                                   for (int u = 0; u < U; ++u) fn(key[u], POS_MAX - (uint32_t)tk[u], ok[u]);
                                 });
      });
      sweep_row<SEL_T, GATHER>(srow, grow, n, Li,
                               [&](const uint32_t(&key)[U], const int(&tk)[U], const bool(&ok)[U], int base) {
                                 bool sel[U];
#pragma unroll
                                 for (int u = 0; u < U; ++u)
                                   sel[u] = ok[u] && at_least(key[u], POS_MAX - (uint32_t)tk[u], P_hi, M_hi, P_lo,
                                                              M_lo);
                                 mark_sweep(sel, tk, base);
                               });
      __syncthreads();
    }
  }

  // 4. ascending output, staged in the candidate list's space
  write_ascending<SEL_T>(bm, words, k, orow, sh.wa, sh.wb);
}

// Few long prefix rows: every CTA takes a chunk of one row and appends the
// elements at or above the boundary bin, (key, token), to the row's list
// (list_cnt zeroed beforehand).  Rows the list cannot serve are skipped; the
// select kernel reads those rows itself.  EMIT (unordered output): the
// elements above the boundary bin are selected whatever the refinement
// decides, so their tokens go straight to out[row][0..above) (slots from
// emit_cnt, zeroed beforehand) and only the boundary bin is listed.
template <bool EMIT>
__global__ void __launch_bounds__(FILT_T) filter_kernel(CacheView c, QueryView qv, const float *scores, long long ld,
                                                        const uint32_t *row_hist, uint2 *list, uint32_t *list_cnt,
                                                        int list_cap, int k, int chunk, int32_t *out,
                                                        uint32_t *emit_cnt) {
  grid_dep_sync();
  constexpr int FU = 16;
  const int row = blockIdx.y;
  const int lane = threadIdx.x & 31;
  const int p0 = blockIdx.x * chunk;
  const int pl = min(c.L_cap, p0 + chunk);  // loads stay inside the row's allocation
  const float *srow = scores + (size_t)row * ld;
  // the first sweep's scores are requested with the prefix and the histogram
  float sv[FU];
#pragma unroll
  for (int u = 0; u < FU; ++u) {
    const int p = p0 + u * FILT_T + threadIdx.x;
    sv[u] = p < pl ? __ldg(srow + p) : 0.f;
  }
  int s;
  const int Li = query_prefix(c, qv, row, &s);
  if (p0 >= Li) return;  // uniform over the CTA
  const int p1 = min(Li, pl);
  // one warp finds the boundary (every warp reading the 8 KB histogram would
  // multiply the L2 traffic by the warps of all CTAs)
  __shared__ Boundary sbd;
  if (threadIdx.x < 32) {
    const Boundary b = warp_boundary(row_hist + (size_t)row * RB, k);
    if (threadIdx.x == 0) sbd = b;
  }
  __syncthreads();
  const Boundary bd = sbd;
  if (!bd.listable((uint32_t)CAP)) return;  // uniform
  const uint32_t d0 = bd.d0;
  uint2 *lrow = list + (size_t)row * list_cap;
  for (int base = p0; base < p1; base += FILT_T * FU) {
    if (base != p0) {
#pragma unroll
      for (int u = 0; u < FU; ++u) {
        const int p = base + u * FILT_T + threadIdx.x;
        sv[u] = p < p1 ? __ldg(srow + p) : 0.f;
      }
    }
    // per thread: elements to list (low 16 bits) and, EMIT, to emit (high 16)
    uint32_t key[FU], n = 0;
#pragma unroll
    for (int u = 0; u < FU; ++u) {
      const int p = base + u * FILT_T + threadIdx.x;
      key[u] = ordered_key(sv[u]);
      const uint32_t bin = key[u] >> HIST_SHIFT;
      if (p < p1) n += EMIT ? (bin == d0 ? 1u : bin > d0 ? 0x10000u : 0u) : (bin >= d0 ? 1u : 0u);
    }
    uint32_t inc = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += u;
    }
    const uint32_t tot = __shfl_sync(0xffffffffu, inc, 31);
    if (tot == 0) continue;  // warp-uniform
    uint32_t slot = 0, eslot = 0;
    if (lane == 31) {
      if (tot & 0xFFFFu) slot = atomicAdd(list_cnt + row, tot & 0xFFFFu);
      if (EMIT && (tot >> 16)) eslot = atomicAdd(emit_cnt + row, tot >> 16);
    }
    slot = __shfl_sync(0xffffffffu, slot, 31) + (inc & 0xFFFFu) - (n & 0xFFFFu);
    if (EMIT) eslot = __shfl_sync(0xffffffffu, eslot, 31) + (inc >> 16) - (n >> 16);
    int32_t *orow = EMIT ? out + (size_t)row * k : nullptr;
#pragma unroll
    for (int u = 0; u < FU; ++u) {
      const int p = base + u * FILT_T + threadIdx.x;
      const uint32_t bin = key[u] >> HIST_SHIFT;
      if (p < p1 && (EMIT ? bin == d0 : bin >= d0)) {
        if (slot < (uint32_t)list_cap) lrow[slot] = make_uint2(key[u], (uint32_t)p);
        ++slot;
      }
      if (EMIT && p < p1 && bin > d0) {
        if (eslot < (uint32_t)k) orow[eslot] = p;
        ++eslot;
      }
    }
  }
}

// Tensor-core prefill rows (16-byte aligned rows): every CTA streams a chunk
// of one row with 16-byte loads, eight per thread in flight, and appends the
// elements whose key is at least thr[row] (the sampled bound) to the row's
// list (list_cnt zeroed beforehand; it counts past list_cap).
constexpr int FT_T = 256;
constexpr int FT_V = 8;  // float4 loads per thread and sweep
constexpr int FT_PAD = 4 * FT_V + 4;  // floats per thread in the stash (16-byte rows, staggered banks)
__global__ void __launch_bounds__(FT_T) filter_thr_kernel(CacheView c, QueryView qv, const float *scores, long long ld,
                                                          const uint32_t *thr, uint2 *list, uint32_t *list_cnt,
                                                          int list_cap, int chunk) {
  grid_dep_sync();
  __shared__ __align__(16) float stash[FT_T * FT_PAD];
  const int row = blockIdx.y;
  const int lane = threadIdx.x & 31;
  const int p0 = blockIdx.x * chunk;
  const int pl = min(c.L_cap, p0 + chunk);  // 16-byte loads below pl stay inside the row (ld % 4 == 0)
  const float *srow = scores + (size_t)row * ld;
  float4 v[FT_V];
#pragma unroll
  for (int u = 0; u < FT_V; ++u) {
    const int p = p0 + (u * FT_T + (int)threadIdx.x) * 4;
    v[u] = p < pl ? __ldg(reinterpret_cast<const float4 *>(srow + p)) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  int s;
  const int Li = query_prefix(c, qv, row, &s);
  if (p0 >= Li) return;  // uniform over the CTA
  const int p1 = min(Li, pl);
  // key >= bound as a float compare (the key map is monotonic; at worst -0
  // passes a +0 bound, an extra entry the selection sorts out); bound 0 takes all
  const uint32_t bound = __ldg(thr + row);
  const bool all = bound == 0u;
  const float tau = __uint_as_float((bound & 0x80000000u) ? (bound & 0x7FFFFFFFu) : ~bound);
  uint2 *lrow = list + (size_t)row * list_cap;
  for (int base = p0; base < p1; base += FT_T * 4 * FT_V) {
    if (base != p0) {
#pragma unroll
      for (int u = 0; u < FT_V; ++u) {
        const int p = base + (u * FT_T + (int)threadIdx.x) * 4;
        v[u] = p < p1 ? __ldg(reinterpret_cast<const float4 *>(srow + p)) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    // bit 4u + e: element e of this thread's u-th float4 is listed; the
    // values wait in shared memory so that the write pass visits only the
    // set bits (about 6 % of the elements)
    const bool full = base + FT_T * 4 * FT_V <= p1;  // uniform: no element of this sweep past the prefix
    uint32_t mask = 0;
#pragma unroll
    for (int u = 0; u < FT_V; ++u) {
      const int p = base + (u * FT_T + (int)threadIdx.x) * 4;
      const bool in0 = full || p < p1, in1 = full || p + 1 < p1, in2 = full || p + 2 < p1, in3 = full || p + 3 < p1;
      mask |= ((uint32_t)(in0 && (all || v[u].x >= tau)) | (uint32_t)(in1 && (all || v[u].y >= tau)) << 1 |
               (uint32_t)(in2 && (all || v[u].z >= tau)) << 2 | (uint32_t)(in3 && (all || v[u].w >= tau)) << 3)
              << (4 * u);
      *reinterpret_cast<float4 *>(&stash[threadIdx.x * FT_PAD + 4 * u]) = v[u];
    }
    const uint32_t n = __popc(mask);
    uint32_t inc = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t x = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += x;
    }
    const uint32_t tot = __shfl_sync(0xffffffffu, inc, 31);
    if (tot == 0) continue;  // warp-uniform
    uint32_t slot = 0;
    if (lane == 31) slot = atomicAdd(list_cnt + row, tot);
    slot = __shfl_sync(0xffffffffu, slot, 31) + inc - n;
    while (mask) {
      const int bit = __ffs(mask) - 1;
      mask &= mask - 1u;
      const float f = stash[threadIdx.x * FT_PAD + bit];
      if (slot < (uint32_t)list_cap)
        lrow[slot] = make_uint2(ordered_key(f), (uint32_t)(base + ((bit >> 2) * FT_T + (int)threadIdx.x) * 4 + (bit & 3)));
      ++slot;
    }
  }
}

// Row histograms when the scoring kernel built none (tensor-core prefill):
// every CTA counts the top 11 key bits of a chunk of one row in shared memory
// and adds its non-zero bins to row_hist (zeroed beforehand).
constexpr int HIST_T = 256;
__global__ void __launch_bounds__(HIST_T) hist_kernel(CacheView c, QueryView qv, const float *scores, long long ld,
                                                      uint32_t *row_hist, int chunk) {
  grid_dep_sync();
  constexpr int HU = 16;
  __shared__ uint32_t hs[RB];
  const int row = blockIdx.y;
  const int p0 = blockIdx.x * chunk;
  const int pl = min(c.L_cap, p0 + chunk);
  const float *srow = scores + (size_t)row * ld;
  float v[HU];
#pragma unroll
  for (int u = 0; u < HU; ++u) {
    const int p = p0 + u * HIST_T + threadIdx.x;
    v[u] = p < pl ? __ldg(srow + p) : 0.f;
  }
  int s;
  const int Li = query_prefix(c, qv, row, &s);
  if (p0 >= Li) return;  // uniform over the CTA
  const int p1 = min(Li, pl);
  for (int b = threadIdx.x; b < RB; b += HIST_T) hs[b] = 0;
  __syncthreads();
  for (int base = p0; base < p1; base += HIST_T * HU) {
    if (base != p0) {
#pragma unroll
      for (int u = 0; u < HU; ++u) {
        const int p = base + u * HIST_T + threadIdx.x;
        v[u] = p < p1 ? __ldg(srow + p) : 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < HU; ++u)
      if (base + u * HIST_T + (int)threadIdx.x < p1) atomicAdd(&hs[ordered_key(v[u]) >> HIST_SHIFT], 1u);
  }
  __syncthreads();
  uint32_t *rh = row_hist + (size_t)row * RB;
  for (int b = threadIdx.x; b < RB; b += HIST_T)
    if (hs[b]) atomicAdd(rh + b, hs[b]);
}

// ---------------------------------------------------------------------------
// One-round-trip selection for rows whose data fits in shared memory: the
// re-rank rows (scores and candidate tokens) and the filter kernel's lists.
// One thread brings the row's histogram and data into shared memory with
// bulk copies on one mbarrier; every later phase works on shared memory only.
// A list row the filter could not serve falls back to sweeps of the global
// row.
// ---------------------------------------------------------------------------
constexpr int FAST_T = 1024;              // threads of the staged selection
constexpr int FAST_W = FAST_T / 32;
constexpr int FAST_DATA_MAX = 128 * 1024;  // bytes of row data staged in shared memory

struct FastShared {
  alignas(16) uint32_t rhist[RB];  // the row histogram (bulk copy)
  Boundary bd;
  uint64_t bar;
  uint4 res;
  uint32_t thr[2];
  uint32_t n_small;
  int ok;
  uint32_t wa[FAST_W], wb[FAST_W + 1];
  uint32_t hist[HPAD];
  uint32_t small_key[FAST_T], small_tie[FAST_T];
  uint32_t n_d0;
  uint32_t n_out;
};
constexpr int D0CAP = 6144;  // boundary-bin elements compacted in shared memory
// bitmap words, rounded so that the arrays after it stay 16-byte aligned
__host__ __device__ __forceinline__ int bm_words(int L_cap) { return (L_cap + 127) / 128 * 4; }

// One whole warp: boundary from the unpadded histogram in shared memory.
__device__ __forceinline__ Boundary warp_boundary_plain_smem(const uint32_t *h, int k) {
  const int lane = threadIdx.x & 31;
  uint32_t s = 0;
  // lane l sums bins [64 l, 64 l + 64) starting at a rotated offset, so the
  // lanes of each load hit 32 distinct banks
#pragma unroll 16
  for (int j = 0; j < 64; ++j) s += h[lane * 64 + ((j + lane) & 63)];
  uint32_t suf = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_down_sync(0xffffffffu, suf, o);
    if (lane + o < 32) suf += v;
  }
  Boundary b;
  b.total = __shfl_sync(0xffffffffu, suf, 0);
  b.kk = min((uint32_t)k, b.total);
  b.all_in = (uint32_t)k >= b.total;
  b.d0 = 0;
  b.above = 0;
  b.in0 = 0;
  if (b.all_in) return b;
  const uint32_t want = b.kk;
  const uint32_t above_l = suf - s;
  const int owner = __ffs(__ballot_sync(0xffffffffu, above_l < want && suf >= want)) - 1;
  const uint32_t base_above = __shfl_sync(0xffffffffu, above_l, owner);
  const int b0 = owner * 64 + 2 * lane;
  const uint2 cc = *reinterpret_cast<const uint2 *>(h + b0);
  const uint32_t pair = cc.x + cc.y;
  uint32_t psuf = pair;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_down_sync(0xffffffffu, psuf, o);
    if (lane + o < 32) psuf += v;
  }
  const uint32_t a1 = base_above + psuf - pair;
  const bool hit1 = a1 < want && a1 + cc.y >= want;
  const bool hit0 = a1 + cc.y < want && a1 + pair >= want;
  const int src = __ffs(__ballot_sync(0xffffffffu, hit1 || hit0)) - 1;
  b.d0 = __shfl_sync(0xffffffffu, hit1 ? b0 + 1 : b0, src);
  b.above = __shfl_sync(0xffffffffu, hit1 ? a1 : a1 + cc.y, src);
  b.in0 = __shfl_sync(0xffffffffu, hit1 ? cc.y : cc.x, src);
  return b;
}

// Sampled boundary bound (tensor-core prefill, where the scoring kernel
// builds no histogram): for every row, count the top 11 key bits of a
// sample of the row -- the whole row up to SMP_N elements, else SMP_BLOCKS
// blocks of 32 consecutive tokens (one 128-byte line each; scattered single
// sectors read slowly from HBM) spread evenly over the prefix -- and write
// thr[row] from the want-th largest sampled element.  want is the sample's
// expected share of the top k, plus SMP_Z standard deviations of a count
// whose 32-token blocks move together, plus 8: the elements at or above
// thr[row] then number at least k with high probability (a row where they do
// not is still selected exactly, from its whole score row).  A whole-row
// sample takes want = min(k, L_i), which is exact.  thr[row] is a key bound:
// the want-th largest sampled key cut to its top 22 bits (boundary bin, then
// the next 11 bits inside it); 0 takes every element.
// Persistent: CTA b takes rows b, b + gridDim.x, ...; the next row's samples
// are requested before the current row is counted, so their latency hides
// behind the counting.
constexpr int SMP_T = 512;
constexpr int SMP_BL = 32;  // tokens per sample block
constexpr int SMP_BLOCKS = 256;
constexpr int SMP_N = SMP_BLOCKS * SMP_BL;
constexpr int SMP_PER = SMP_N / SMP_T;  // samples per thread
constexpr double SMP_Z = 1.5;           // margin, in standard deviations of the sampled count

// Request row `row`'s samples (all of this thread's before any is used).
__device__ __forceinline__ void sample_load(const CacheView &c, const QueryView &qv, const float *scores,
                                            long long ld, int row, float (&v)[SMP_PER], int &Li, int &n) {
  int s;
  Li = query_prefix(c, qv, row, &s);
  const bool whole = Li <= SMP_N;
  n = whole ? max(Li, 0) : SMP_N;
  const float *srow = scores + (size_t)row * ld;
#pragma unroll
  for (int u = 0; u < SMP_PER; ++u) {
    const int i = u * SMP_T + (int)threadIdx.x;
    int p = i;
    if (!whole) p = (int)((long long)(i / SMP_BL) * (Li - SMP_BL) / (SMP_BLOCKS - 1)) + (i % SMP_BL);
    v[u] = i < n ? __ldg(srow + p) : 0.f;
  }
}

__global__ void __launch_bounds__(SMP_T) sample_thr_kernel(CacheView c, QueryView qv, const float *scores, long long ld,
                                                           int k, uint32_t *thr) {
  grid_dep_sync();
  __shared__ uint32_t hs[RB];
  __shared__ Boundary sb;
  int row = blockIdx.x;
  if (row >= qv.n_q) return;  // uniform
  float v[SMP_PER];
  int Li, n;
  sample_load(c, qv, scores, ld, row, v, Li, n);
  while (true) {
    const int next = row + (int)gridDim.x;
    float vn[SMP_PER];
    int Ln = 0, nn = 0;
    if (next < qv.n_q) sample_load(c, qv, scores, ld, next, vn, Ln, nn);
    for (int b = threadIdx.x; b < RB; b += SMP_T) hs[b] = 0;
    __syncthreads();
#pragma unroll
    for (int u = 0; u < SMP_PER; ++u)
      if (u * SMP_T + (int)threadIdx.x < n) atomicAdd(&hs[ordered_key(v[u]) >> HIST_SHIFT], 1u);
    __syncthreads();
    uint32_t want = (uint32_t)min(k, max(Li, 0));
    if (Li > SMP_N) {
      const double r = (double)k * SMP_N / Li;
      want = (uint32_t)min(2.0 * SMP_N, ceil(r + SMP_Z * sqrt((double)SMP_BL * r) + 8.0));
    }
    if (threadIdx.x < 32) {
      const Boundary b = warp_boundary_plain_smem(hs, (int)want);
      if (threadIdx.x == 0) sb = b;
    }
    __syncthreads();
    const Boundary b = sb;
    if (b.all_in) {
      if (threadIdx.x == 0) thr[row] = 0u;
    } else {
      // second level: the next 11 key bits of the samples inside the boundary bin
      for (int x = threadIdx.x; x < RB; x += SMP_T) hs[x] = 0;
      __syncthreads();
#pragma unroll
      for (int u = 0; u < SMP_PER; ++u) {
        const int i = u * SMP_T + (int)threadIdx.x;
        const uint32_t key = ordered_key(v[u]);
        if (i < n && (key >> HIST_SHIFT) == b.d0) atomicAdd(&hs[(key >> 10) & (RB - 1)], 1u);
      }
      __syncthreads();
      if (threadIdx.x < 32) {
        const Boundary b2 = warp_boundary_plain_smem(hs, (int)(want - b.above));
        if (threadIdx.x == 0) thr[row] = (b.d0 << HIST_SHIFT) | ((b2.all_in ? 0u : b2.d0) << 10);
      }
    }
    __syncthreads();  // hs and sb free for the next row
    if (next >= qv.n_q) break;
    row = next;
    Li = Ln;
    n = nn;
#pragma unroll
    for (int u = 0; u < SMP_PER; ++u) v[u] = vn[u];
  }
}

// LIST: the filter kernel's list (key, token) of the row; else GATHER rows
// (scores and candidate tokens, n_cols of each).  OWN (with LIST): there is
// no row histogram; the list holds the elements at or above a sampled bound,
// and the kernel counts the listed keys itself -- or, when the list missed
// (fewer than min(k, L_i) entries, or more than it holds), the whole row.
// stage_cap: list entries staged in shared memory (<= list_cap, even);
// d0cap: boundary-bin elements compacted there.
// EMITTED (LIST, unordered): the filter already wrote the row's elements
// above the boundary bin to out[row][0..above) and listed only the bin.
template <bool LIST, bool ORDERED, bool OWN = false, bool EMITTED = false>
__global__ void __launch_bounds__(FAST_T) select_smem_kernel(CacheView c, QueryView qv, const float *scores,
                                                            long long ld, int n_cols, const int32_t *gather,
                                                            const uint32_t *row_hist, const uint2 *list,
                                                            const uint32_t *list_cnt, int list_cap, int stage_cap,
                                                            int d0cap, int k, int32_t *out) {
  grid_dep_sync();
  extern __shared__ __align__(16) uint8_t fs_smem[];
  FastShared &sh = *reinterpret_cast<FastShared *>(fs_smem);
  uint8_t *data = fs_smem + sizeof(FastShared);  // 16-byte aligned (sizeof is a multiple of 16)
  const int data_bytes = LIST ? stage_cap * 8 : n_cols * 8;
  uint32_t *bm = reinterpret_cast<uint32_t *>(data + data_bytes);
  uint32_t *d0_key = bm + bm_words(c.L_cap);                              // [d0cap]
  uint32_t *d0_tie = d0_key + d0cap;                                       // [d0cap]
  const uint2 *ent = reinterpret_cast<const uint2 *>(data);                // LIST
  const float *sc = reinterpret_cast<const float *>(data);                 // GATHER
  const int32_t *tk = reinterpret_cast<const int32_t *>(data + n_cols * 4);  // GATHER
  const int row = blockIdx.x;
  const int tid = threadIdx.x;

  int s;
  const int Li = query_prefix(c, qv, row, &s);
  const float *srow = scores + (size_t)row * ld;
  if (tid == 0) {
    mbar_init(&sh.bar, 1);
    fence_mbar_init();
    if (LIST) {
      // the listed entries only, rounded up to an even count (16-byte copies;
      // stage_cap is even)
      const uint32_t n_copy = min(list_cnt[row], (uint32_t)stage_cap);
      const uint32_t ent_bytes = ((n_copy + 1u) & ~1u) * 8u;
      mbar_arrive_expect_tx(&sh.bar, (OWN ? 0u : (uint32_t)RB * 4u) + ent_bytes);
      if (!OWN) bulk_g2s(sh.rhist, row_hist + (size_t)row * RB, RB * 4, &sh.bar);
      if (ent_bytes) bulk_g2s(data, list + (size_t)row * list_cap, ent_bytes, &sh.bar);
    } else {
      mbar_arrive_expect_tx(&sh.bar, RB * 4 + n_cols * 8);
      bulk_g2s(sh.rhist, row_hist + (size_t)row * RB, RB * 4, &sh.bar);
      bulk_g2s(data, scores + (size_t)row * ld, n_cols * 4, &sh.bar);
      bulk_g2s(data + n_cols * 4, gather + (size_t)row * n_cols, n_cols * 4, &sh.bar);
    }
    sh.n_small = 0;
    sh.n_d0 = 0;
    sh.n_out = 0;
  }
  const int lcnt = LIST ? min((int)list_cnt[row], stage_cap) : 0;
  const int words = cdiv(Li, 32);
  for (int w = tid; w < words; w += FAST_T) bm[w] = 0;
  __syncthreads();  // barrier initialised, bitmap clear
  {
    const bool got = mbar_wait(&sh.bar, 0);
    if (!got) flag(c, MISA_DEV_WAIT_TIMEOUT);
    if (tid == 0) sh.ok = got;
  }
  __syncthreads();
  int32_t *orow = out + (size_t)row * k;
  // a winner: marked in the token bitmap (ascending output), or appended to
  // the output at once (any order; one shared atomic per group of lanes)
  auto emit = [&](int tok) {
    if (ORDERED) {
      mark(bm, tok);
    } else {
      const unsigned m = __activemask();
      const int lane = tid & 31, leader = __ffs(m) - 1;
      uint32_t base = 0;
      if (lane == leader) base = atomicAdd(&sh.n_out, (uint32_t)__popc(m));
      base = __shfl_sync(m, base, leader) + __popc(m & lanemask_lt());
      if (base < (uint32_t)k) orow[base] = tok;
    }
  };
  if (!sh.ok) {  // uniform: give up on this row (flagged above)
    for (int p = tid; p < k; p += FAST_T) orow[p] = -1;
    return;
  }
  bool list_ok = false;
  if (OWN) {
    const uint32_t cnt = list_cnt[row];
    list_ok = cnt <= (uint32_t)stage_cap && cnt >= (uint32_t)min(k, max(Li, 0));
    for (int b = tid; b < RB; b += FAST_T) sh.rhist[b] = 0;
    __syncthreads();
    const int n = list_ok ? lcnt : max(Li, 0);
    for (int i = tid; i < n; i += FAST_T)
      atomicAdd(&sh.rhist[(list_ok ? ent[i].x : ordered_key(__ldg(srow + i))) >> HIST_SHIFT], 1u);
    __syncthreads();
  }
  {
    // the boundary bin of the row, searched by the whole block
    const uint4 r = block_select_bin<FAST_T, false>(sh.rhist, (uint32_t)k, sh.wa, sh.wb, &sh.res);
    Boundary b;
    b.total = r.w;
    b.kk = min((uint32_t)k, r.w);
    b.all_in = (uint32_t)k >= r.w;
    b.d0 = b.all_in ? 0u : r.x;
    b.above = b.all_in ? 0u : r.y;
    b.in0 = b.all_in ? 0u : r.z;
    if (tid == 0) {
      sh.bd = b;
      if (EMITTED && b.listable((uint32_t)CAP)) sh.n_out = b.above;  // the filter's tokens come first
    }
  }
  __syncthreads();
  const Boundary bd = sh.bd;

  if (bd.kk > 0) {
    const uint32_t d0 = bd.d0;
    const uint32_t need = bd.need();
    const bool whole = bd.all_in || need == bd.in0;
    // staged elements: (key, token, valid); a list row the filter skipped is
    // read from the global row instead (prefix rows: token = position)
    const bool staged = OWN ? list_ok : (!LIST || bd.listable((uint32_t)CAP));
    auto each = [&](auto &&fn) {
      if (staged) {
        const int n = LIST ? lcnt : n_cols;
        for (int i = tid; i < n; i += FAST_T) {
          if (LIST) {
            const uint2 e = ent[i];
            fn(e.x, (int)e.y, true);
          } else {
            const int t = tk[i];
            fn(ordered_key(sc[i]), t, t >= 0 && t < Li);
          }
        }
      } else {
        for (int i = tid; i < Li; i += FAST_T) fn(ordered_key(__ldg(srow + i)), i, true);
      }
    };
    const bool compact = staged && !whole && bd.in0 <= (uint32_t)d0cap;
    if (compact) {
      // 2. one pass, four elements per thread and step: mark everything above
      //    the boundary; compact the boundary bin's elements (key, tie) with
      //    one shared atomic per warp and step
      const int n = LIST ? lcnt : n_cols;
      const int lane = tid & 31;
      const uint32_t lt = lanemask_lt();
      for (int base = 0; base < n; base += FAST_T * 4) {
        const int i0 = base + tid * 4;
        uint32_t key[4];
        int t[4];
        bool v[4];
        if (LIST) {
          const uint4 *e4 = reinterpret_cast<const uint4 *>(ent + i0);
          const uint4 a = i0 < n ? e4[0] : make_uint4(0u, 0u, 0u, 0u);
          const uint4 b = i0 + 2 < n ? e4[1] : make_uint4(0u, 0u, 0u, 0u);
          key[0] = a.x; t[0] = (int)a.y; key[1] = a.z; t[1] = (int)a.w;
          key[2] = b.x; t[2] = (int)b.y; key[3] = b.z; t[3] = (int)b.w;
#pragma unroll
          for (int e = 0; e < 4; ++e) v[e] = i0 + e < n;
        } else {
          const float4 f = i0 < n ? reinterpret_cast<const float4 *>(sc)[i0 >> 2] : make_float4(0.f, 0.f, 0.f, 0.f);
          const int4 q = i0 < n ? reinterpret_cast<const int4 *>(tk)[i0 >> 2] : make_int4(-1, -1, -1, -1);
          key[0] = ordered_key(f.x); key[1] = ordered_key(f.y); key[2] = ordered_key(f.z); key[3] = ordered_key(f.w);
          t[0] = q.x; t[1] = q.y; t[2] = q.z; t[3] = q.w;
#pragma unroll
          for (int e = 0; e < 4; ++e) v[e] = t[e] >= 0 && t[e] < Li;
        }
        uint32_t flags = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t bin = key[e] >> HIST_SHIFT;
          if (v[e] && bin > d0) emit(t[e]);
          flags |= (uint32_t)(v[e] && bin == d0) << e;
        }
        const uint32_t cnt = __popc(flags);
        uint32_t inc = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t u = __shfl_up_sync(0xffffffffu, inc, o);
          if (lane >= o) inc += u;
        }
        const uint32_t tot = __shfl_sync(0xffffffffu, inc, 31);
        if (tot) {
          uint32_t slot = 0;
          if (lane == 31) slot = atomicAdd(&sh.n_d0, tot);
          slot = __shfl_sync(0xffffffffu, slot, 31) + inc - cnt;
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if ((flags >> e) & 1) {
              if (slot < (uint32_t)d0cap) {
                d0_key[slot] = key[e];
                d0_tie[slot] = POS_MAX - (uint32_t)t[e];
              }
              ++slot;
            }
        }
        (void)lt;
      }
      __syncthreads();
      // 3. threshold among the boundary bin's elements only, then their winners
      const int nd = min((int)sh.n_d0, d0cap);
      uint32_t P_hi = d0 << HIST_SHIFT, M_hi = TOP_MASK, P_lo = 0, M_lo = 0;
      refine<true, FAST_T>(sh, P_hi, M_hi, P_lo, M_lo, need, bd.in0, [&](auto &&fn) {
        for (int x = tid; x < nd; x += FAST_T) fn(d0_key[x], d0_tie[x], true);
      });
      for (int x = tid; x < nd; x += FAST_T)
        if (at_least(d0_key[x], d0_tie[x], P_hi, M_hi, P_lo, M_lo)) emit((int)(POS_MAX - d0_tie[x]));
      __syncthreads();
    } else {
    // 2. everything above the boundary (and the boundary bin when whole)
    each([&](uint32_t kx, int t, bool v) {
      const uint32_t bin = kx >> HIST_SHIFT;
      if (v && (bd.all_in || bin > d0 || (whole && bin == d0))) emit(t);
    });
    __syncthreads();
    if (!whole) {
      // 3. threshold inside d0, then its winners
      uint32_t P_hi = d0 << HIST_SHIFT, M_hi = TOP_MASK, P_lo = 0, M_lo = 0;
      refine<true, FAST_T>(sh, P_hi, M_hi, P_lo, M_lo, need, bd.in0, [&](auto &&fn) {
        each([&](uint32_t kx, int t, bool v) { fn(kx, POS_MAX - (uint32_t)t, v); });
      });
      each([&](uint32_t kx, int t, bool v) {
        if (v && (kx >> HIST_SHIFT) == d0 && at_least(kx, POS_MAX - (uint32_t)t, P_hi, M_hi, P_lo, M_lo)) emit(t);
      });
      __syncthreads();
    }
    }
  }
  // 4. output
  if (ORDERED) {
    write_ascending<FAST_T>(bm, words, k, orow, sh.wa, sh.wb);
  } else {
    __syncthreads();
    for (int p = (int)min(sh.n_out, (uint32_t)k) + tid; p < k; p += FAST_T) orow[p] = -1;
  }
}

constexpr int SMEM_OPTIN_MAX = 227 * 1024;  // largest dynamic shared memory a CTA may opt into

int fast_smem_bytes(bool list, int n_cols, int stage_cap, int L_cap, int d0cap = D0CAP) {
  return (int)sizeof(FastShared) + (list ? stage_cap * 8 : n_cols * 8) + 4 * bm_words(L_cap) + 8 * d0cap;
}

template <bool LIST, bool ORDERED = true, bool OWN = false, bool EMITTED = false>
cudaError_t launch_select_smem(const CacheView &c, const QueryView &q, const float *scores, long long ld, int n_cols,
                               const int32_t *gather, const uint32_t *row_hist, const uint2 *list,
                               const uint32_t *list_cnt, int list_cap, int k, int32_t *out, cudaStream_t s,
                               int stage_cap = -1, int d0cap = D0CAP) {
  constexpr int SMEM_MAX = SMEM_OPTIN_MAX;
  if (stage_cap < 0) stage_cap = list_cap;
  struct Tag {};
  const int st = cached_per_device<Tag>([] {
    return 1 + (int)cudaFuncSetAttribute(select_smem_kernel<LIST, ORDERED, OWN, EMITTED>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_MAX);
  });
  if (st != 1) return (cudaError_t)(st - 1);
  const int smem = fast_smem_bytes(LIST, n_cols, stage_cap, c.L_cap, d0cap);
  return launch_kernel(select_smem_kernel<LIST, ORDERED, OWN, EMITTED>, dim3(q.n_q), dim3(FAST_T), smem, s, c, q, scores, ld,
                       n_cols, gather, row_hist, list, list_cnt, list_cap, stage_cap, d0cap, k, out);
}

// Zero n words (the histograms and list counters before a scoring pass); a
// kernel measured as fast as a memset node in the decode step's graph.
__global__ void __launch_bounds__(256) zero_kernel(uint32_t *p, size_t n) {
  grid_dep_sync();
  for (size_t x = blockIdx.x * 256 + threadIdx.x; x < n; x += (size_t)gridDim.x * 256) p[x] = 0u;
}

int sel_smem_bytes(int L_cap) { return (int)sizeof(SelShared) + 4 * cdiv(L_cap, 32); }
constexpr int SEL_SMEM_MAX = (int)sizeof(SelShared) + 4 * (MISA_MAX_L / 32);

template <bool GATHER, bool FROM_LIST, bool OWN_HIST = false>
cudaError_t launch_select(const CacheView &c, const QueryView &q, const float *scores, long long ld, int n_cols,
                          const int32_t *gather, const uint32_t *row_hist, const uint2 *list,
                          const uint32_t *list_cnt, int list_cap, int k, int32_t *out, cudaStream_t s) {
  struct Tag {};
  const int ok = cached_per_device<Tag>([] {
    return cudaFuncSetAttribute(select_kernel<GATHER, FROM_LIST, OWN_HIST>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                SEL_SMEM_MAX) == cudaSuccess
               ? 1
               : -1;
  });
  if (ok < 0) return cudaErrorInvalidConfiguration;
  return launch_kernel(select_kernel<GATHER, FROM_LIST, OWN_HIST>, dim3(q.n_q), dim3(SEL_T), sel_smem_bytes(c.L_cap), s, c,
                    q, scores, ld, n_cols, gather, row_hist, list, list_cnt, list_cap, k, out);
}

}  // namespace

cudaError_t launch_zero(uint32_t *p, size_t n, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const int blocks = (int)std::min<size_t>((n + 255) / 256, (size_t)2 * device_sms());
  return launch_kernel(zero_kernel, dim3(blocks), dim3(256), 0, s, p, n);
}

size_t topk_list_entries(int n_q, int L_cap, int k) {
  if (n_q < 1 || L_cap <= TOPK_LIST_MIN_L || k < 1) return 0;
  return (size_t)n_q * ((size_t)k + TOPK_LIST_EXTRA);
}

cudaError_t launch_topk(const CacheView &c, const QueryView &q, const float *scores, long long ld, int n_cols,
                        const int32_t *gather, uint32_t *row_hist, bool hist_ready, void *list_ws,
                        uint32_t *list_cnt, int k, int32_t *out, cudaStream_t s, bool ordered) {
  if (q.n_q == 0) return cudaSuccess;
  auto aligned16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (gather) {
    // rows staged whole in shared memory when they fit and the copies stay
    // 16-byte aligned; otherwise swept from global memory
    if (hist_ready && n_cols % 4 == 0 && ld % 4 == 0 && 8LL * n_cols <= FAST_DATA_MAX && aligned16(scores) &&
        aligned16(gather) && aligned16(row_hist) && fast_smem_bytes(false, n_cols, 0, c.L_cap) <= SMEM_OPTIN_MAX)
      return launch_select_smem<false>(c, q, scores, ld, n_cols, gather, row_hist, nullptr, nullptr, 0, k, out, s);
    return launch_select<true, false>(c, q, scores, ld, n_cols, gather, row_hist, nullptr, nullptr, 0, k, out, s);
  }
  const bool list_mode = topk_list_entries(q.n_q, c.L_cap, k) != 0 && list_ws && list_cnt && row_hist;
  if (!hist_ready && !list_mode)
    return launch_select<false, false, true>(c, q, scores, ld, 0, nullptr, nullptr, nullptr, nullptr, 0, k, out, s);
  const int sms = device_sms();
  cudaError_t e = cudaSuccess;
  const int list_cap = k + TOPK_LIST_EXTRA;
  uint2 *list = static_cast<uint2 *>(list_ws);
  const bool smem_list = 8LL * list_cap <= FAST_DATA_MAX && list_cap % 2 == 0 && aligned16(list) &&
                         aligned16(row_hist) && fast_smem_bytes(true, 0, list_cap, c.L_cap) <= SMEM_OPTIN_MAX;
  // about two CTAs per SM over all rows (few rows) or at most 16K elements
  // per CTA (many rows), at least 4096 elements each
  const int per_row = max(1, min(cdiv(c.L_cap, 4096), max(2 * sms / q.n_q, cdiv(c.L_cap, 16384))));
  const int chunk = cdiv(cdiv(c.L_cap, per_row), FILT_T) * FILT_T;
  const dim3 fgrid(cdiv(c.L_cap, chunk), q.n_q);
  if (!hist_ready && smem_list && ld % 4 == 0 && aligned16(scores)) {
    // no histogram: a sampled lower bound of each row's top-k keys (in the
    // histogram's place), the elements at or above it listed, the list
    // counted and selected in shared memory
    uint32_t *thr = row_hist;
    // persistent: the resident CTAs (two per SM at 512 threads) walk the rows
    e = launch_kernel(sample_thr_kernel, dim3(std::min(q.n_q, 2 * sms)), dim3(SMP_T), 0, s, c, q, scores, ld, k, thr);
    if (e != cudaSuccess) return e;
    const int tchunk = 4 * FT_T * FT_V * 2;  // two sweeps per CTA
    e = launch_kernel(filter_thr_kernel, dim3(cdiv(c.L_cap, tchunk), q.n_q), dim3(FT_T), 0, s, c, q, scores, ld, thr,
                      list, list_cnt, list_cap, tchunk);
    if (e != cudaSuccess) return e;
    // lists of up to 7168 entries and 1024 boundary-bin elements: two CTAs
    // per SM (rows beyond take the whole-row path); larger k stages it all
    const bool two = k <= 4096 && fast_smem_bytes(true, 0, 7168, c.L_cap, 1024) <= SMEM_OPTIN_MAX / 2 - 1024;
    const int stage_cap = two ? 7168 : list_cap, d0cap = two ? 1024 : D0CAP;
    return ordered ? launch_select_smem<true, true, true>(c, q, scores, ld, 0, nullptr, thr, list, list_cnt, list_cap,
                                                          k, out, s, stage_cap, d0cap)
                   : launch_select_smem<true, false, true>(c, q, scores, ld, 0, nullptr, thr, list, list_cnt,
                                                           list_cap, k, out, s, stage_cap, d0cap);
  }
  if (!hist_ready) {
    // wide pass over the scores: about 16K elements per CTA
    const int hper_row = cdiv(c.L_cap, 16384);
    const int hchunk = cdiv(cdiv(c.L_cap, hper_row), HIST_T) * HIST_T;
    e = launch_kernel(hist_kernel, dim3(cdiv(c.L_cap, hchunk), q.n_q), dim3(HIST_T), 0, s, c, q, scores, ld, row_hist,
                      hchunk);
    if (e != cudaSuccess) return e;
  }
  if (!list_mode)
    return launch_select<false, false>(c, q, scores, ld, 0, nullptr, row_hist, nullptr, nullptr, 0, k, out, s);
  // unordered output with the staged selection: the filter emits the tokens
  // above the boundary bin itself and lists only the bin
  const bool emit = !ordered && smem_list;
  uint32_t *emit_cnt = list_cnt + q.n_q;
  e = emit ? launch_kernel(filter_kernel<true>, fgrid, dim3(FILT_T), 0, s, c, q, scores, ld, row_hist, list,
                           list_cnt, list_cap, k, chunk, out, emit_cnt)
           : launch_kernel(filter_kernel<false>, fgrid, dim3(FILT_T), 0, s, c, q, scores, ld, row_hist, list,
                           list_cnt, list_cap, k, chunk, out, emit_cnt);
  if (e != cudaSuccess) return e;
  if (smem_list)
    return ordered
               ? launch_select_smem<true, true>(c, q, scores, ld, 0, nullptr, row_hist, list, list_cnt, list_cap, k,
                                                out, s)
               : launch_select_smem<true, false, false, true>(c, q, scores, ld, 0, nullptr, row_hist, list,
                                                              list_cnt, list_cap, k, out, s);
  return launch_select<false, true>(c, q, scores, ld, 0, nullptr, row_hist, list, list_cnt, list_cap, k, out, s);
}

}  // namespace misa
