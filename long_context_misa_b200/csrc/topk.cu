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
#include "internal.h"

namespace misa {
namespace {

constexpr int POS_BITS = 18;                 // token indices < 2^18 = MISA_MAX_L
constexpr uint32_t POS_MAX = (1u << POS_BITS) - 1u;
constexpr int RB = TOPK_HIST_BINS;           // bins of the histogram and of each refinement pass
constexpr int HIST_SHIFT = 21;               // the histogram holds key bits 31..21
constexpr uint32_t TOP_MASK = 0xFFE00000u;
constexpr int CAP = TOPK_LIST_EXTRA;         // d0 elements refined in shared memory
constexpr int SEL_T = 512;                   // select_kernel threads
constexpr int SEL_W = SEL_T / 32;
constexpr int FILT_T = 256;                  // filter_kernel threads
constexpr int U = 16;                        // elements per thread per sweep iteration
constexpr int HPAD = RB + RB / 64;           // shared histogram: one pad word per 64 bins
// refinement passes: key bits 20..10, 9..0, then the token's tie bits 17..9, 8..0
__device__ constexpr int kShift[4] = {10, 0, 9, 0};
__device__ constexpr int kWidth[4] = {11, 10, 9, 9};

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Bin b of a shared refinement histogram: lane l's 64 bins start at word
// 65 l, so the lanes of a warp read distinct banks.
__device__ __forceinline__ int hpos(int b) { return b + (b >> 6); }

// One whole warp: the bin of a RB-bin histogram (larger bin = larger key)
// holding the want-th largest element.  Lane l sums bins [64 l, 64 l + 64);
// the range that holds it is then searched two bins per lane.  Returns to every lane
// {bin, elements in higher bins, its count, total}; bin = ~0 when want is 0
// or above the total.  PAD: shared histogram in the hpos layout, else a
// plain array in global memory.
template <bool PAD>
__device__ __forceinline__ uint4 warp_select_bin(const uint32_t *h, uint32_t want) {
  const int lane = threadIdx.x & 31;
  uint32_t s = 0;
  if (PAD) {
#pragma unroll 16
    for (int j = 0; j < 64; ++j) s += h[lane * 65 + j];
  } else {
    const uint4 *p = reinterpret_cast<const uint4 *>(h + lane * 64);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint4 v = __ldg(p + j);
      s += v.x + v.y + v.z + v.w;
    }
  }
  uint32_t suf = s;  // elements in lanes >= this one
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_down_sync(0xffffffffu, suf, o);
    if (lane + o < 32) suf += v;
  }
  const uint32_t total = __shfl_sync(0xffffffffu, suf, 0);
  if (want == 0 || want > total) return make_uint4(~0u, 0u, 0u, total);
  const uint32_t above_l = suf - s;
  const int owner = __ffs(__ballot_sync(0xffffffffu, above_l < want && suf >= want)) - 1;
  // the owner's 64 bins, two per lane, searched by the whole warp
  const uint32_t base_above = __shfl_sync(0xffffffffu, above_l, owner);
  const int b0 = owner * 64 + 2 * lane;
  uint32_t c0, c1;
  if (PAD) {
    c0 = h[hpos(b0)];
    c1 = h[hpos(b0 + 1)];
  } else {
    const uint2 v = __ldg(reinterpret_cast<const uint2 *>(h + b0));
    c0 = v.x;
    c1 = v.y;
  }
  const uint32_t pair = c0 + c1;
  uint32_t psuf = pair;  // elements in the owner's bins >= b0
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_down_sync(0xffffffffu, psuf, o);
    if (lane + o < 32) psuf += v;
  }
  const uint32_t a1 = base_above + psuf - pair;  // elements above bin b0 + 1
  const bool hit1 = a1 < want && a1 + c1 >= want;
  const bool hit0 = a1 + c1 < want && a1 + pair >= want;
  const int src = __ffs(__ballot_sync(0xffffffffu, hit1 || hit0)) - 1;
  const uint32_t bin = hit1 ? b0 + 1 : b0;
  const uint32_t above = hit1 ? a1 : a1 + c1;
  const uint32_t cnt = hit1 ? c1 : c0;
  return make_uint4(__shfl_sync(0xffffffffu, bin, src), __shfl_sync(0xffffffffu, above, src),
                    __shfl_sync(0xffffffffu, cnt, src), total);
}
// Boundary of a row from its histogram: kk, total, and (unless every valid
// element is selected) the bin d0 with the counts above it and in it.
struct Boundary {
  uint32_t total, kk, d0, above, in0, all_in;
  // elements still to take from d0
  __device__ uint32_t need() const { return kk - above; }
  // a compact list of the elements at or above d0 serves this row: it holds
  // kk (whole bin taken) or fewer than kk + CAP (d0 listed) entries
  __device__ bool listable() const { return kk > 0 && !all_in && (need() == in0 || in0 <= (uint32_t)CAP); }
};

// One whole warp: the row's boundary (valid in every lane).
__device__ __forceinline__ Boundary warp_boundary(const uint32_t *rh, int k) {
  const uint4 r = warp_select_bin<false>(rh, (uint32_t)k);
  Boundary b;
  b.total = r.w;
  b.kk = min((uint32_t)k, r.w);
  b.all_in = (uint32_t)k >= r.w;
  b.d0 = b.all_in ? 0u : r.x;
  b.above = b.all_in ? 0u : r.y;
  b.in0 = b.all_in ? 0u : r.z;
  return b;
}

// The same from a histogram in shared memory (hpos layout).
__device__ __forceinline__ Boundary warp_boundary_smem(const uint32_t *hs, int k) {
  const uint4 r = warp_select_bin<true>(hs, (uint32_t)k);
  Boundary b;
  b.total = r.w;
  b.kk = min((uint32_t)k, r.w);
  b.all_in = (uint32_t)k >= r.w;
  b.d0 = b.all_in ? 0u : r.x;
  b.above = b.all_in ? 0u : r.y;
  b.in0 = b.all_in ? 0u : r.z;
  return b;
}

// Exclusive prefix of `v` over the threads in thread order; *total = block sum.
template <int T>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t *total, uint32_t *wa, uint32_t *wb) {
  constexpr int W = T / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t u = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += u;
  }
  if (lane == 31) wa[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const uint32_t x = lane < W ? wa[lane] : 0u;
    uint32_t s = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += u;
    }
    if (lane < W) wb[lane] = s - x;
    if (lane == W - 1) wb[W] = s;
  }
  __syncthreads();
  *total = wb[W];
  const uint32_t r = wb[warp] + inc - v;
  __syncthreads();  // wa, wb free again on return
  return r;
}

struct SelShared {
  Boundary bd;
  uint4 res;                       // a warp search result
  uint32_t thr[2];                 // threshold composite from the counting step
  uint32_t n_small;
  uint32_t wa[SEL_W], wb[SEL_W + 1];
  uint32_t toff[SEL_T];            // output offset of each thread's bitmap words
  uint32_t hist[HPAD];
  uint32_t small_key[SEL_T], small_tie[SEL_T];
  uint32_t cand_key[CAP];
  uint32_t cand_tie[CAP];
};

// Visit every element of the row in warp- and block-uniform sweeps:
// fn(key, token, ok, base) gets U elements per thread; element u of thread t
// is position base + u*T + t.  Prefix rows: position p is token p with score
// srow[p], p < Li.  Gathered rows: position p is token grow[p] (ok when
// 0 <= token < Li) with score srow[p], p < n.
template <int T, bool GATHER, class F>
__device__ __forceinline__ void sweep_row(const float *srow, const int32_t *grow, int n, int Li, F &&fn) {
  for (int base = 0; base < n; base += T * U) {
    int tk[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int p = base + u * T + threadIdx.x;
      tk[u] = p < n ? (GATHER ? __ldg(grow + p) : p) : -1;
    }
    float sv[U];
    bool ok[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int p = base + u * T + threadIdx.x;
      ok[u] = tk[u] >= 0 && tk[u] < Li;
      sv[u] = ok[u] ? __ldg(srow + p) : 0.f;
    }
    uint32_t key[U];
#pragma unroll
    for (int u = 0; u < U; ++u) key[u] = ordered_key(sv[u]);
    fn(key, tk, ok, base);
  }
}

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

__device__ __forceinline__ void mark(uint32_t *bm, int tok) { atomicOr(bm + (tok >> 5), 1u << (tok & 31)); }

__device__ __forceinline__ bool at_least(uint32_t kx, uint32_t lx, uint32_t P_hi, uint32_t M_hi, uint32_t P_lo,
                                         uint32_t M_lo) {
  const uint32_t kh = kx & M_hi, kl = lx & M_lo;
  return kh > P_hi || (kh == P_hi && kl >= P_lo);
}

// Radix refinement of the threshold among the elements the visitor presents
// (visit(fn) calls fn(key, tie, active) for each, block-uniformly).  P/M:
// prefix and mask decided so far on the key and on the tie; need: elements
// still to take among the in_bin that match the prefix.  With `small`, once
// at most SEL_T elements match, their exact ranks finish the job.
template <bool SMALL, class Visit>
__device__ __forceinline__ void refine(SelShared &sh, uint32_t &P_hi, uint32_t &M_hi, uint32_t &P_lo,
                                       uint32_t &M_lo, uint32_t need, uint32_t in_bin, Visit &&visit) {
  const int tid = threadIdx.x;
  bool done = in_bin == need;
  for (int p = 0; p < 4 && !done; ++p) {
    if (SMALL && p > 0 && in_bin <= (uint32_t)SEL_T) {
      // the in_bin elements matching the prefix: rank each by counting
      visit([&](uint32_t kx, uint32_t lx, bool act) {
        if (act && (kx & M_hi) == P_hi && (lx & M_lo) == P_lo) {
          const uint32_t slot = atomicAdd(&sh.n_small, 1u);
          if (slot < (uint32_t)SEL_T) {
            sh.small_key[slot] = kx;
            sh.small_tie[slot] = lx;
          }
        }
      });
      __syncthreads();
      const int ns = min((int)sh.n_small, SEL_T);
      if (tid < ns) {
        const uint32_t ki = sh.small_key[tid], li = sh.small_tie[tid];
        uint32_t rank = 0;
        for (int j = 0; j < ns; ++j) {
          const uint32_t kj = sh.small_key[j], lj = sh.small_tie[j];
          rank += (kj > ki || (kj == ki && lj > li)) ? 1u : 0u;
        }
        if (rank == need - 1) {
          sh.thr[0] = ki;
          sh.thr[1] = li;
        }
      }
      __syncthreads();
      P_hi = sh.thr[0];
      M_hi = ~0u;
      P_lo = sh.thr[1];
      M_lo = POS_MAX;
      return;
    }
    const bool lo_word = p >= 2;
    const int sft = kShift[p];
    const uint32_t dm = (1u << kWidth[p]) - 1u;
    for (int b = tid; b < HPAD; b += SEL_T) sh.hist[b] = 0;
    __syncthreads();
    visit([&](uint32_t kx, uint32_t lx, bool act) {
      if (act && (kx & M_hi) == P_hi && (lx & M_lo) == P_lo)
        atomicAdd(&sh.hist[hpos(((lo_word ? lx : kx) >> sft) & dm)], 1u);
    });
    __syncthreads();
    if (tid < 32) {
      const uint4 r = warp_select_bin<true>(sh.hist, need);
      if (tid == 0) sh.res = r;
    }
    __syncthreads();
    const uint4 r = sh.res;
    need -= r.y;
    in_bin = r.z;
    if (!lo_word) {
      P_hi |= r.x << sft;
      M_hi |= dm << sft;
    } else {
      P_lo |= r.x << sft;
      M_lo |= dm << sft;
    }
    done = in_bin == need;
  }
}

template <bool GATHER, bool FROM_LIST, bool OWN_HIST>
__global__ void __launch_bounds__(SEL_T) select_kernel(CacheView c, QueryView qv, const float *scores, long long ld,
                                                       int n_cols, const int32_t *gather, const uint32_t *row_hist,
                                                       const uint2 *list, const uint32_t *list_cnt, int list_cap,
                                                       int k, int32_t *out) {
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
  if (!OWN_HIST) bd = warp_boundary(row_hist + (size_t)row * RB, k);
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
    bd = warp_boundary_smem(sh.hist, k);
  }
  __syncthreads();

  if (bd.kk > 0) {
    const uint32_t d0 = bd.d0;
    const uint32_t need = bd.need();
    const bool whole = bd.all_in || need == bd.in0;  // no refinement needed
    const bool listed = !whole && bd.in0 <= (uint32_t)CAP;
    uint32_t P_hi = d0 << HIST_SHIFT, M_hi = TOP_MASK, P_lo = 0, M_lo = 0;
    const bool via_list = FROM_LIST && bd.listable();
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
        refine<true>(sh, P_hi, M_hi, P_lo, M_lo, need, bd.in0, [&](auto &&fn) {
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
      refine<false>(sh, P_hi, M_hi, P_lo, M_lo, need, bd.in0, [&](auto &&fn) {
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

  // 4. ascending output.  Thread t owns bitmap words [t*per, t*per + per);
  //    the outputs are split evenly over the threads (each finds the word
  //    holding its first output by a search over the owners' offsets).
  const int per = cdiv(words, SEL_T);
  {
    const int w0 = min(tid * per, words), w1 = min(w0 + per, words);
    uint32_t cnt = 0;
    for (int w = w0; w < w1; ++w) cnt += __popc(bm[w]);
    uint32_t n_sel;
    sh.toff[tid] = block_excl_scan<SEL_T>(cnt, &n_sel, sh.wa, sh.wb);
    __syncthreads();
    const uint32_t j0 = n_sel * (uint32_t)tid / SEL_T, j1 = n_sel * (uint32_t)(tid + 1) / SEL_T;
    if (j0 < j1) {
      int lo = 0, hi = SEL_T - 1;  // last owner whose offset is <= j0
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (sh.toff[mid] <= j0) lo = mid;
        else hi = mid - 1;
      }
      uint32_t r = j0 - sh.toff[lo];
      int w = lo * per;
      uint32_t m = bm[w];
      while ((uint32_t)__popc(m) <= r) {
        r -= __popc(m);
        m = bm[++w];
      }
      for (; r > 0; --r) m &= m - 1;
      for (uint32_t j = j0; j < j1; ++j) {
        while (m == 0) m = bm[++w];
        const int b = __ffs(m) - 1;
        m &= m - 1;
        if (j < (uint32_t)k) orow[j] = w * 32 + b;
      }
    }
    for (int p = (int)n_sel + tid; p < k; p += SEL_T) orow[p] = -1;
  }
}

// Few long prefix rows: every CTA takes a chunk of one row and appends the
// elements at or above the boundary bin, (key, token), to the row's list
// (list_cnt zeroed beforehand).  Rows the list cannot serve are skipped; the
// select kernel reads those rows itself.
__global__ void __launch_bounds__(FILT_T) filter_kernel(CacheView c, QueryView qv, const float *scores, long long ld,
                                                        const uint32_t *row_hist, uint2 *list, uint32_t *list_cnt,
                                                        int list_cap, int k, int chunk) {
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
  const Boundary bd = warp_boundary(row_hist + (size_t)row * RB, k);  // every warp
  if (!bd.listable()) return;  // uniform
  uint2 *lrow = list + (size_t)row * list_cap;
  for (int base = p0; base < p1; base += FILT_T * FU) {
    if (base != p0) {
#pragma unroll
      for (int u = 0; u < FU; ++u) {
        const int p = base + u * FILT_T + threadIdx.x;
        sv[u] = p < p1 ? __ldg(srow + p) : 0.f;
      }
    }
    uint32_t key[FU], n = 0;
#pragma unroll
    for (int u = 0; u < FU; ++u) {
      const int p = base + u * FILT_T + threadIdx.x;
      key[u] = ordered_key(sv[u]);
      n += (p < p1 && (key[u] >> HIST_SHIFT) >= bd.d0) ? 1u : 0u;
    }
    uint32_t inc = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += u;
    }
    const uint32_t tot = __shfl_sync(0xffffffffu, inc, 31);
    if (tot == 0) continue;  // warp-uniform
    uint32_t slot = 0;
    if (lane == 31) slot = atomicAdd(list_cnt + row, tot);
    slot = __shfl_sync(0xffffffffu, slot, 31) + inc - n;
#pragma unroll
    for (int u = 0; u < FU; ++u) {
      const int p = base + u * FILT_T + threadIdx.x;
      if (p < p1 && (key[u] >> HIST_SHIFT) >= bd.d0) {
        if (slot < (uint32_t)list_cap) lrow[slot] = make_uint2(key[u], (uint32_t)p);
        ++slot;
      }
    }
  }
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
  select_kernel<GATHER, FROM_LIST, OWN_HIST><<<q.n_q, SEL_T, sel_smem_bytes(c.L_cap), s>>>(
      c, q, scores, ld, n_cols, gather, row_hist, list, list_cnt, list_cap, k, out);
  return cudaGetLastError();
}

}  // namespace

size_t topk_list_entries(int n_q, int L_cap, int k) {
  if (n_q < 1 || n_q > TOPK_LIST_MAX_ROWS || L_cap <= TOPK_LIST_MIN_L || k < 1) return 0;
  return (size_t)n_q * ((size_t)k + TOPK_LIST_EXTRA);
}

cudaError_t launch_topk(const CacheView &c, const QueryView &q, const float *scores, long long ld, int n_cols,
                        const int32_t *gather, const uint32_t *row_hist, void *list_ws, uint32_t *list_cnt, int k,
                        int32_t *out, cudaStream_t s) {
  if (q.n_q == 0) return cudaSuccess;
  if (gather)
    return launch_select<true, false>(c, q, scores, ld, n_cols, gather, row_hist, nullptr, nullptr, 0, k, out, s);
  if (!row_hist)
    return launch_select<false, false, true>(c, q, scores, ld, 0, nullptr, nullptr, nullptr, nullptr, 0, k, out, s);
  if (topk_list_entries(q.n_q, c.L_cap, k) == 0 || !list_ws || !list_cnt)
    return launch_select<false, false>(c, q, scores, ld, 0, nullptr, row_hist, nullptr, nullptr, 0, k, out, s);
  const int list_cap = k + TOPK_LIST_EXTRA;
  uint2 *list = static_cast<uint2 *>(list_ws);
  // about two CTAs per SM over all rows, at least 4096 elements each
  const int sms = device_sms();
  const int per_row = max(1, min(cdiv(c.L_cap, 4096), 2 * sms / q.n_q));
  const int chunk = cdiv(cdiv(c.L_cap, per_row), FILT_T) * FILT_T;
  filter_kernel<<<dim3(cdiv(c.L_cap, chunk), q.n_q), FILT_T, 0, s>>>(c, q, scores, ld, row_hist, list, list_cnt,
                                                                     list_cap, k, chunk);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_select<false, true>(c, q, scores, ld, 0, nullptr, row_hist, list, list_cnt, list_cap, k, out, s);
}

}  // namespace misa
