// Top-k of one row selected by the CTAs that scored it, with the scores still
// on chip (the fused selection of the decode scoring kernels).
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference":
// the indexer keeps the k highest-scoring tokens (abstract; technical summary
// "Methodology: MISA", step 2), MISA-dagger keeps k' candidates from the
// routed pass and re-ranks them ("Hierarchical variant").  Order: larger
// score first, equal scores to the lower token index (composite key: the
// order-preserving image of the score, then POS_MAX - token).
//
// The C CTAs of a row each hold some of the row's elements (key, token) in
// shared memory or registers and have counted them by their top 11 key bits.
// They meet at counters in global memory (zeroed before the launch):
//   1. every CTA adds its 11-bit counts to the row histogram and waits for
//      the others; every CTA then finds the same boundary bin d0 of the
//      row's kk-th largest key;
//   2. unless d0 is taken whole, every CTA counts the next 11 key bits of
//      its elements inside d0 into a second row histogram and waits again;
//      the 22-bit boundary bucket (d0, d1) follows;
//   3. every CTA writes its elements above the bucket as winners and lists
//      the bucket's elements (a handful for continuous scores);
//   4. the last CTA to arrive ranks the bucket exactly (radix passes and
//      ranks by counting, ties to the lower token), adds its winners and
//      writes the output: unordered (winners in the order they came, then
//      -1 padding) or ascending (a token bitmap in shared memory).
// A bucket too large to list (massively tied scores) is ranked by the last
// CTA from the row's scores in global memory, which every CTA also writes.
//
// The CTAs of a row wait for one another, so the kernel's grid must fit on
// the device at once (the callers size it to one wave of resident CTAs).
// Every wait is bounded: one that runs out sets MISA_DEV_WAIT_TIMEOUT and the
// CTA gives up on the row (its output is then invalid).
#pragma once

#include "selcore.cuh"

namespace misa {
namespace {

constexpr int RS_BCAP = FUSED_BCAP;  // bucket entries listed per row
// words per row zeroed before each launch: the row histogram, the boundary
// bin's histogram and the counters
constexpr int RS_ZERO_WORDS = FUSED_ZERO_WORDS;
static_assert(RS_ZERO_WORDS == 2 * RB + FUSED_CTR, "layout of the zeroed words");
// counters: the two histogram barriers, the last-CTA count, winners and
// bucket entries written, and the barrier of a router fused in front
enum { RS_BAR0 = 0, RS_BAR1 = 1, RS_DONE = 2, RS_EMIT = 3, RS_BUCKET = 4, RS_ROUTE = 5, RS_NEED = 6 };
static_assert(RS_EMIT == FUSED_CTR_EMIT && RS_BUCKET == FUSED_CTR_BUCKET && RS_NEED == FUSED_CTR_NEED &&
                  RS_NEED < FUSED_CTR,
              "counter slots");

constexpr int RS_BSTAGE = 512;  // bucket entries a CTA stages before reserving their slots

// Shared scratch beyond RsShared, used in turn for: a CTA's winners and
// bucket entries before they are written out (elems: the most elements a
// CTA of T threads holds; every warp stages its winners in a private part
// of cdiv(elems, T) * 32 words, which holds the elements a warp visits when
// `each` deals them per warp or in block-wide sweeps); the last CTA's staged
// bucket; the token bitmap of an ascending output.
__host__ __device__ constexpr int rs_max3(int a, int b, int c) { return a > b ? (a > c ? a : c) : (b > c ? b : c); }
__host__ __device__ constexpr int rs_warp_cap(int elems, int T) { return (elems + T - 1) / T * 32; }
__host__ __device__ constexpr int rs_scratch_bytes(int L_cap, int elems, int T) {
  return rs_max3(8 * RS_BCAP, 4 * ((L_cap + 31) / 32 + 4), 4 * (T / 32) * rs_warp_cap(elems, T) + 8 * RS_BSTAGE);
}

template <int T>
struct RsShared {
  Boundary bd;
  uint4 res;
  uint32_t thr[2];
  uint32_t n_small;
  int ok;
  uint32_t n_win, n_bk, base_win, base_bk;  // this CTA's staged winners and bucket entries, their slots
  uint32_t wa[T / 32], wb[T / 32 + 1];
  uint32_t wcnt[T / 32];  // winners staged by each warp
  uint32_t hist[HPAD];
  uint32_t small_key[T], small_tie[T];
};

// Per-row arguments of the fused selection.
struct RsRow {
  uint32_t *zeroed;   // [RS_ZERO_WORDS]: row histogram, bin histogram, counters
  uint2 *bucket;      // [RS_BCAP] (key, token)
  int32_t *winners;   // [k] winners of an ascending output; unused otherwise
  int32_t *out;       // [k] the row's output
  bool defer;         // FusedTopk::defer
};

__device__ __forceinline__ RsRow rs_row(const FusedTopk &f, int i) {
  RsRow r;
  r.zeroed = f.zeroed + (size_t)i * RS_ZERO_WORDS;
  r.bucket = f.bucket + (size_t)i * RS_BCAP;
  r.winners = f.winners ? f.winners + (size_t)i * f.k : nullptr;
  r.out = f.out + (size_t)i * f.k;
  r.defer = f.defer != 0 && f.ordered == 0;
  return r;
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Every thread of the CTA: arrive at *ctr and wait until `target` arrivals
// (bounded).  The same answer in every thread; false when the wait ran out.
template <class Sh>
__device__ __forceinline__ bool row_barrier(Sh &sh, uint32_t *ctr, uint32_t target, const CacheView &c) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();  // this CTA's writes before the arrival
    atomicAdd(ctr, 1u);
    bool ok = ld_acquire_gpu(ctr) >= target;
    if (!ok) {
      const uint64_t t0 = globaltimer_ns();
      while (!(ok = ld_acquire_gpu(ctr) >= target))
        if (globaltimer_ns() - t0 > WAIT_LIMIT_NS) break;
      if (!ok) flag(c, MISA_DEV_WAIT_TIMEOUT);
    }
    sh.ok = ok;
  }
  __syncthreads();
  return sh.ok != 0;
}

// Warp-aggregated append of the lanes with `take` set: one atomic on *cnt
// per warp; returns this lane's slot.  All 32 lanes must call.
__device__ __forceinline__ uint32_t warp_append(uint32_t *cnt, bool take) {
  const uint32_t m = __ballot_sync(0xffffffffu, take);
  if (!m) return 0;
  const int lane = threadIdx.x & 31;
  uint32_t base = 0;
  if (lane == 0) base = atomicAdd(cnt, (uint32_t)__popc(m));
  return __shfl_sync(0xffffffffu, base, 0) + __popc(m & lanemask_lt());
}

// The fused selection of one row (k outputs), called by every thread of each
// of the row's C CTAs after scoring.  shist: the CTA's 11-bit counts of its
// elements (RB words in shared memory, overwritten).  scratch: shared memory
// of rs_scratch_bytes(L_cap, elems, T) bytes (free after scoring), elems the
// most elements `each` presents in this CTA.
//   each(fn):  fn(key, token, valid) for every element of this CTA, called
//              by all 32 lanes of a warp together (warp-uniform trips).
//   sweep(fn): fn(key, tie, valid) for every element of the whole row, read
//              from global memory through L2 (the overflow path), called by
//              every thread in block-uniform sweeps.
template <int T, class Each, class Sweep>
__device__ void row_select(const CacheView &c, RsShared<T> &sh, uint32_t *shist, uint8_t *scratch, const RsRow &rw,
                           int C, int k, int Li, bool ordered, int elems, Each &&each, Sweep &&sweep) {
  const int tid = threadIdx.x;
  uint32_t *hist1 = rw.zeroed, *hist2 = rw.zeroed + RB, *ctr = rw.zeroed + 2 * RB;
  // 1. the row histogram
  for (int b = tid; b < RB; b += T) {
    const uint32_t v = shist[b];
    if (v) atomicAdd(hist1 + b, v);
  }
  if (!row_barrier(sh, ctr + RS_BAR0, (uint32_t)C, c)) return;
  if (tid < 32) {
    const uint4 r = warp_select_bin_staged(hist1, (uint32_t)k, sh.hist);
    Boundary b;
    b.total = r.w;
    b.kk = min((uint32_t)k, r.w);
    b.all_in = (uint32_t)k >= r.w;
    b.d0 = b.all_in ? 0u : r.x;
    b.above = b.all_in ? 0u : r.y;
    b.in0 = b.all_in ? 0u : r.z;
    if (tid == 0) sh.bd = b;
  }
  __syncthreads();
  const Boundary bd = sh.bd;
  const uint32_t need0 = bd.need();
  const bool lvl2 = bd.kk > 0 && !bd.all_in && need0 != bd.in0;
  // 2. the boundary bin's next 11 bits
  uint32_t p22 = 0, need1 = 0, in1 = 0;
  if (lvl2) {
    for (int b = tid; b < RB; b += T) shist[b] = 0;
    __syncthreads();
    each([&](uint32_t key, int, bool valid) {
      if (valid && (key >> HIST_SHIFT) == bd.d0) atomicAdd(&shist[(key >> 10) & (RB - 1)], 1u);
    });
    __syncthreads();
    for (int b = tid; b < RB; b += T) {
      const uint32_t v = shist[b];
      if (v) atomicAdd(hist2 + b, v);
    }
    if (!row_barrier(sh, ctr + RS_BAR1, (uint32_t)C, c)) return;
    if (tid < 32) {
      const uint4 r = warp_select_bin_staged(hist2, need0, sh.hist);
      if (tid == 0) sh.res = r;
    }
    __syncthreads();
    const uint4 r = sh.res;
    p22 = (bd.d0 << 11) | r.x;
    need1 = need0 - r.y;
    in1 = r.z;
  }
  const bool bucket = lvl2 && need1 != in1;  // the 22-bit bucket is split
  // the next kernel finishes the row (rw.defer) unless the split bucket
  // overflows its list: no last CTA then, and the bucket's entries (in1 of
  // them in all, within the list's capacity) go to the list like the winners
  const bool handoff = rw.defer && (!bucket || in1 <= (uint32_t)RS_BCAP);
  int32_t *dst = ordered ? rw.winners : rw.out;
  // 3. this CTA's sure winners, and the bucket's elements: staged in shared
  //    memory (winners in each warp's own part, no atomics; bucket entries,
  //    rare, through a shared counter), then one global atomic per CTA
  //    reserves their slots (the winners of a row's CTAs all count on one
  //    word: per-warp atomics there serialise)
  if (bd.kk > 0) {
    const int lane = tid & 31, warp = tid >> 5;
    const uint32_t pw = (uint32_t)rs_warp_cap(elems, T);
    uint32_t *st_w = reinterpret_cast<uint32_t *>(scratch);
    uint2 *st_b = reinterpret_cast<uint2 *>(scratch + 4 * (T / 32) * pw);
    uint32_t *my_w = st_w + warp * pw;
    if (tid == 0) sh.n_bk = 0;
    __syncthreads();
    uint32_t n_mine = 0;  // warp-uniform
    each([&](uint32_t key, int tok, bool valid) {
      const uint32_t k22 = key >> 10;
      bool sel;
      if (bd.all_in)
        sel = true;
      else if (!lvl2)
        sel = (key >> HIST_SHIFT) >= bd.d0;
      else
        sel = k22 > p22 || (!bucket && k22 == p22);
      const bool win = valid && sel;
      const uint32_t m = __ballot_sync(0xffffffffu, win);
      const uint32_t slot = n_mine + __popc(m & lanemask_lt());
      if (win && slot < pw) my_w[slot] = (uint32_t)tok;
      n_mine += __popc(m);
      const bool in_b = valid && bucket && k22 == p22;
      const uint32_t s2 = warp_append(&sh.n_bk, in_b);
      if (in_b) {
        if (s2 < (uint32_t)RS_BSTAGE) {
          st_b[s2] = make_uint2(key, (uint32_t)tok);
        } else if (handoff) {  // past the staging: straight to the list (it holds all in1)
          const uint32_t g = atomicAdd(ctr + RS_BUCKET, 1u);
          if (g < (uint32_t)RS_BCAP) rw.bucket[g] = make_uint2(key, (uint32_t)tok);
        }
      }
    });
    n_mine = min(n_mine, pw);  // (never clipped: a warp visits at most pw elements)
    if (lane == 0) sh.wcnt[warp] = n_mine;
    __syncthreads();
    const uint32_t nbk = sh.n_bk;
    if (tid == 0) {
      uint32_t nw = 0;
      for (int w = 0; w < T / 32; ++w) nw += sh.wcnt[w];
      sh.base_win = nw ? atomicAdd(ctr + RS_EMIT, nw) : 0u;
      // more bucket entries than staged: count the row past the list's
      // capacity, so that the last CTA ranks it from the scores instead (a
      // handed-over row's list holds them all: the rest went straight there)
      if (handoff)
        sh.base_bk = nbk ? atomicAdd(ctr + RS_BUCKET, min(nbk, (uint32_t)RS_BSTAGE)) : 0u;
      else
        sh.base_bk = nbk ? atomicAdd(ctr + RS_BUCKET, nbk <= (uint32_t)RS_BSTAGE ? nbk : (uint32_t)RS_BCAP + 1u) : 0u;
    }
    __syncthreads();
    uint32_t off = sh.base_win;
    for (int w = 0; w < warp; ++w) off += sh.wcnt[w];
    for (uint32_t x = lane; x < n_mine; x += 32) {
      const uint32_t slot = off + x;
      if (slot < (uint32_t)k) dst[slot] = (int32_t)my_w[x];
    }
    if (handoff || nbk <= (uint32_t)RS_BSTAGE)
      for (uint32_t x = tid; x < min(nbk, (uint32_t)RS_BSTAGE); x += T) {
        const uint32_t slot = sh.base_bk + x;
        if (slot < (uint32_t)RS_BCAP) rw.bucket[slot] = st_b[x];
      }
  }
  if (handoff) {
    if (bucket && blockIdx.x == 0 && tid == 0) ctr[RS_NEED] = need1;
    return;
  }
  // 4. the last CTA of the row finishes it
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const bool last = atomicAdd(ctr + RS_DONE, 1u) == (uint32_t)C - 1u;
    if (last) __threadfence();
    sh.ok = last;
  }
  __syncthreads();
  if (!sh.ok) return;
  if (bucket) {
    const uint32_t nb = __ldcg(ctr + RS_BUCKET);
    uint32_t P_hi = p22 << 10, M_hi = 0xFFFFFC00u, P_lo = 0, M_lo = 0;
    if (nb <= (uint32_t)RS_BCAP) {
      uint32_t *bk = reinterpret_cast<uint32_t *>(scratch), *bt = bk + RS_BCAP;
      for (uint32_t x = tid; x < nb; x += T) {
        const uint2 e = __ldcg(rw.bucket + x);
        bk[x] = e.x;
        bt[x] = POS_MAX - e.y;
      }
      if (tid == 0) sh.n_small = 0;
      __syncthreads();
      const uint32_t nb_r = (nb + T - 1) / T * T;  // warp-uniform trips
      if (nb <= (uint32_t)T) {
        // few elements (the continuous case): each one's rank by counting
        // the bucket's elements above it (composites are unique)
        const uint32_t x = tid;
        bool v = false;
        if (x < nb) {
          const uint32_t kx = bk[x], lx = bt[x];
          uint32_t rank = 0;
          for (uint32_t y = 0; y < nb; ++y) rank += (bk[y] > kx || (bk[y] == kx && bt[y] > lx)) ? 1u : 0u;
          v = rank < need1;
        }
        const uint32_t slot = warp_append(ctr + RS_EMIT, v);
        if (v && slot < (uint32_t)k) dst[slot] = (int32_t)(POS_MAX - bt[x]);
      } else {
        refine<true, T>(sh, P_hi, M_hi, P_lo, M_lo, need1, nb, [&](auto &&fn) {
          for (uint32_t x = tid; x < nb; x += T) fn(bk[x], bt[x], true);
        });
        for (uint32_t x = tid; x < nb_r; x += T) {
          const bool v = x < nb && at_least(bk[x], bt[x], P_hi, M_hi, P_lo, M_lo);
          const uint32_t slot = warp_append(ctr + RS_EMIT, v);
          if (v && slot < (uint32_t)k) dst[slot] = (int32_t)(POS_MAX - bt[x]);
        }
      }
    } else {
      // more tied elements than the bucket lists: rank from the row's scores
      if (tid == 0) sh.n_small = 0;
      __syncthreads();
      refine<false, T>(sh, P_hi, M_hi, P_lo, M_lo, need1, in1, [&](auto &&fn) { sweep(fn); });
      sweep([&](uint32_t key, uint32_t tie, bool valid) {
        const bool v = valid && (key >> 10) == p22 && at_least(key, tie, P_hi, M_hi, P_lo, M_lo);
        const uint32_t slot = warp_append(ctr + RS_EMIT, v);
        if (v && slot < (uint32_t)k) dst[slot] = (int32_t)(POS_MAX - tie);
      });
    }
  }
  __threadfence();  // this CTA's own winners reach L2 before they are read back through it
  __syncthreads();
  const uint32_t n_emit = min(__ldcg(ctr + RS_EMIT), (uint32_t)k);
  if (ordered) {
    uint32_t *bm = reinterpret_cast<uint32_t *>(scratch);
    const int words = cdiv(max(Li, 0), 32);
    for (int w = tid; w < words; w += T) bm[w] = 0;
    __syncthreads();
    for (uint32_t x = tid; x < n_emit; x += T) {
      const int tok = __ldcg(rw.winners + x);
      if (tok >= 0 && tok < Li) mark(bm, tok);
    }
    __syncthreads();
    write_ascending<T>(bm, words, k, rw.out, sh.wa, sh.wb);
  } else {
    for (int p = (int)n_emit + tid; p < k; p += T) rw.out[p] = -1;
  }
}

}  // namespace
}  // namespace misa
