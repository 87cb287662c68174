// Building blocks of the top-k selections (topk.cu and the fused selections
// of the scoring kernels): order-preserving score keys counted in 11-bit
// histograms, block- and warp-wide searches of a histogram's boundary bin,
// radix refinement of a threshold inside that bin, and the ascending output
// of a token bitmap.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM
// Inference": the indexer keeps the k highest-scoring prefix tokens (abstract;
// technical summary "Methodology: MISA", step 2).  Order: larger score first,
// equal scores to the lower token index.  An element's composite key is the
// order-preserving image of its score followed by the tie word
// POS_MAX - token, unique in a row.
#pragma once

#include "internal.h"

namespace misa {
namespace {

constexpr int POS_BITS = 18;                 // token indices < 2^18 = MISA_MAX_L
constexpr uint32_t POS_MAX = (1u << POS_BITS) - 1u;
constexpr int RB = TOPK_HIST_BINS;           // bins of the histogram and of each refinement pass
constexpr int HIST_SHIFT = 21;               // the histogram holds key bits 31..21
constexpr uint32_t TOP_MASK = 0xFFE00000u;
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
// the range that holds it is then searched (shared: two bins per lane; global:
// by its owner, from registers).  Returns to every lane
// {bin, elements in higher bins, its count, total}; bin = ~0 when want is 0
// or above the total.  PAD: shared histogram in the hpos layout, else a
// plain array in global memory, read through the read-only path, or with CG
// through L2 only (a histogram other CTAs of the same kernel wrote).
// A histogram in global memory: every lane keeps its 64 bins in registers
// and the owner walks them itself, so the search costs one round of loads.
template <bool CG>
__device__ __forceinline__ uint4 warp_select_bin_global(const uint32_t *h, uint32_t want) {
  const int lane = threadIdx.x & 31;
  const uint4 *p = reinterpret_cast<const uint4 *>(h + lane * 64);
  uint4 v[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = CG ? __ldcg(p + j) : __ldg(p + j);
  uint32_t s = 0;
#pragma unroll
  for (int j = 0; j < 16; ++j) s += v[j].x + v[j].y + v[j].z + v[j].w;
  uint32_t suf = s;  // elements in lanes >= this one
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t u = __shfl_down_sync(0xffffffffu, suf, o);
    if (lane + o < 32) suf += u;
  }
  const uint32_t total = __shfl_sync(0xffffffffu, suf, 0);
  if (want == 0 || want > total) return make_uint4(~0u, 0u, 0u, total);
  const uint32_t above_l = suf - s;
  const int owner = __ffs(__ballot_sync(0xffffffffu, above_l < want && suf >= want)) - 1;
  // the owner's bins from the highest down: the first that reaches `want`
  uint32_t bin = 0, above = 0, cnt = 0, a = above_l;
  bool found = false;
#pragma unroll
  for (int j = 15; j >= 0; --j) {
    const uint32_t c4[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
    for (int e = 3; e >= 0; --e) {
      const bool hit = !found && a + c4[e] >= want;
      if (hit) {
        bin = (uint32_t)(lane * 64 + 4 * j + e);
        above = a;
        cnt = c4[e];
      }
      found = found || hit;
      a += found ? 0u : c4[e];
    }
  }
  return make_uint4(__shfl_sync(0xffffffffu, bin, owner), __shfl_sync(0xffffffffu, above, owner),
                    __shfl_sync(0xffffffffu, cnt, owner), total);
}

template <bool PAD, bool CG = false>
__device__ __forceinline__ uint4 warp_select_bin(const uint32_t *h, uint32_t want);

// A histogram other CTAs wrote to global memory (read through L2), copied
// by one warp into shared memory (hpos layout, HPAD words of `stage`) in
// one round of loads and searched there; light on registers.
__device__ __forceinline__ uint4 warp_select_bin_staged(const uint32_t *h, uint32_t want, uint32_t *stage) {
  const int lane = threadIdx.x & 31;
  const uint4 *p = reinterpret_cast<const uint4 *>(h + lane * 64);
  uint4 v[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = __ldcg(p + j);
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    uint32_t *d = stage + lane * 65 + 4 * j;  // hpos(64 lane + 4 j)
    d[0] = v[j].x;
    d[1] = v[j].y;
    d[2] = v[j].z;
    d[3] = v[j].w;
  }
  __syncwarp();
  return warp_select_bin<true>(stage, want);
}

template <bool PAD, bool CG>
__device__ __forceinline__ uint4 warp_select_bin(const uint32_t *h, uint32_t want) {
  if constexpr (!PAD) return warp_select_bin_global<CG>(h, want);
  const int lane = threadIdx.x & 31;
  uint32_t s = 0;
#pragma unroll 16
  for (int j = 0; j < 64; ++j) s += h[lane * 65 + j];
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
  const uint32_t c0 = h[hpos(b0)], c1 = h[hpos(b0 + 1)];
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
  // kk (whole bin taken) or fewer than kk + cap (d0 listed) entries
  __device__ bool listable(uint32_t cap) const { return kk > 0 && !all_in && (need() == in0 || in0 <= cap); }
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

// warp_select_bin with every thread of a block of T = RB / 2 threads: thread
// t holds the pair of bins 2p, 2p + 1 with p = T - 1 - t (the highest bins
// go to the first threads), so an exclusive scan in thread order counts the
// elements above each pair, and the thread whose pair holds the want-th
// element publishes the result through *res.  A shared histogram in the hpos
// layout (PAD) or plain.  Called by every thread; returns the same result
// everywhere.
template <int T, bool PAD>
__device__ __forceinline__ uint4 block_select_bin(const uint32_t *h, uint32_t want, uint32_t *wa, uint32_t *wb,
                                                  uint4 *res) {
  static_assert(2 * T == RB, "two bins per thread");
  const int b0 = 2 * (T - 1 - (int)threadIdx.x);
  uint32_t c0, c1;
  if (PAD) {
    c0 = h[hpos(b0)];
    c1 = h[hpos(b0 + 1)];
  } else {
    const uint2 v = *reinterpret_cast<const uint2 *>(h + b0);
    c0 = v.x;
    c1 = v.y;
  }
  uint32_t total;
  const uint32_t above = block_excl_scan<T>(c0 + c1, &total, wa, wb);  // elements in the higher pairs
  if (want == 0 || want > total) return make_uint4(~0u, 0u, 0u, total);  // uniform
  if (above < want && above + c1 >= want) *res = make_uint4(b0 + 1, above, c1, total);
  if (above + c1 < want && above + c1 + c0 >= want) *res = make_uint4(b0, above + c1, c0, total);
  __syncthreads();
  const uint4 r = *res;
  __syncthreads();  // *res free again on return
  return r;
}

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
// at most T elements match, their exact ranks finish the job.
template <bool SMALL, int T, class Sh, class Visit>
__device__ __forceinline__ void refine(Sh &sh, uint32_t &P_hi, uint32_t &M_hi, uint32_t &P_lo,
                                       uint32_t &M_lo, uint32_t need, uint32_t in_bin, Visit &&visit) {
  const int tid = threadIdx.x;
  bool done = in_bin == need;
  for (int p = 0; p < 4 && !done; ++p) {
    if (SMALL && p > 0 && in_bin <= (uint32_t)T) {
      // the in_bin elements matching the prefix: rank each by counting
      visit([&](uint32_t kx, uint32_t lx, bool act) {
        if (act && (kx & M_hi) == P_hi && (lx & M_lo) == P_lo) {
          const uint32_t slot = atomicAdd(&sh.n_small, 1u);
          if (slot < (uint32_t)T) {
            sh.small_key[slot] = kx;
            sh.small_tie[slot] = lx;
          }
        }
      });
      __syncthreads();
      const int ns = min((int)sh.n_small, T);
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
    for (int b = tid; b < HPAD; b += T) sh.hist[b] = 0;
    __syncthreads();
    visit([&](uint32_t kx, uint32_t lx, bool act) {
      if (act && (kx & M_hi) == P_hi && (lx & M_lo) == P_lo)
        atomicAdd(&sh.hist[hpos(((lo_word ? lx : kx) >> sft) & dm)], 1u);
    });
    __syncthreads();
    uint4 r;
    if constexpr (2 * T == RB) {
      r = block_select_bin<T, true>(sh.hist, need, sh.wa, sh.wb, &sh.res);
    } else {
      if (tid < 32) {
        const uint4 x = warp_select_bin<true>(sh.hist, need);
        if (tid == 0) sh.res = x;
      }
      __syncthreads();
      r = sh.res;
    }
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

// Ascending output of the marked tokens: thread t owns bitmap words
// [t*per, t*per + per), counts their bits, takes the slot of its first
// output from a block-wide exclusive scan and writes its own tokens in order
// (the threads of a warp write neighbouring output ranges); then -1 padding
// up to k.  A thread whose words hold many winners writes them all (at most
// 32 per word), which costs less than spreading the outputs evenly over the
// threads by searching the owners' offsets.
template <int T>
__device__ __forceinline__ void write_ascending(const uint32_t *bm, int words, int k, int32_t *orow, uint32_t *wa,
                                                uint32_t *wb) {
  const int tid = threadIdx.x;
  const int per = cdiv(words, T);
  const int w0 = min(tid * per, words), w1 = min(w0 + per, words);
  uint32_t cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(bm[w]);
  uint32_t n_sel;
  uint32_t j = block_excl_scan<T>(cnt, &n_sel, wa, wb);
  const uint32_t n_out = min(n_sel, (uint32_t)k);
  for (int w = w0; w < w1 && j < n_out; ++w) {
    uint32_t m = bm[w];
    while (m && j < n_out) {
      orow[j++] = w * 32 + (__ffs(m) - 1);
      m &= m - 1;
    }
  }
  for (int p = (int)n_out + tid; p < k; p += T) orow[p] = -1;
}

}  // namespace
}  // namespace misa
