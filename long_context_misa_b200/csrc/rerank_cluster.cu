// The MISA-dagger fine stage in one kernel: every head re-scores a query's
// k' candidates and the k best come out in ascending token order.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference",
// technical summary, "Hierarchical variant": the full DSA indexer (all H_I
// heads) scores only the candidate set kept by the routed pass and keeps the
// top k of it:
//     I_t = s_t * sum_n w_{i,n} * ReLU(q_{i,n} . k_t),   t in cand[i],
// ties to the lower token index (abstract; "Methodology: MISA", step 2).
//
// One thread-block cluster of RC_CL CTAs per query, each CTA one SM.  CTA r
// takes candidates [r * S, (r + 1) * S) (S = TPC tiles of 128): it requests
// their key rows at once with 16-byte cp.async into the 128-byte-swizzled
// K-major layout, builds the query's head matrix Q' meanwhile (bf16, or the
// exact two-term e4m3 split of the bf16 query), and one thread issues every
// tile's tcgen05 MMA (M = 128 candidates, N = the heads rounded up to a power
// of two) into tensor memory.  Eight warps drain it (two per tensor-memory
// lane quarter): ReLU, weights, head sum and the e4m3 token scale give each
// candidate's score, kept in shared memory as an order-preserving key.
//
// The selection runs over the cluster's distributed shared memory with no
// global memory in between: per radix level (the key's bits 31-21, 20-10,
// 9-0, then the tie word POS_MAX - token) every CTA counts its candidates
// that match the prefix decided so far, CTA r sums bins [256 r, 256 r + 256)
// over the cluster, and every CTA reads all the sums and finds the same
// boundary bin.  Once the boundary bin holds few candidates, they are listed
// and each CTA ranks its own against the whole list.  Winners are marked in a
// token bitmap split over the cluster (CTA r owns an eighth of the prefix);
// each CTA counts its part, learns the counts of the CTAs before it, and
// writes its tokens in ascending order; -1 pads the row to k.
//
// Every CTA passes every cluster barrier (a CTA that has to give up carries
// on with no candidates), so no barrier waits on a CTA that left.  The one
// other wait, on the MMAs, is bounded: when it runs out the CTA sets
// MISA_DEV_WAIT_TIMEOUT, waits (bounded) for the MMAs before releasing the
// tensor memory, and takes no candidates.
#include <algorithm>

#include "internal.h"
#include "qprime.cuh"
#include "selcore.cuh"
#include "umma.cuh"

namespace misa {
namespace {

constexpr int RC_CL = 8;          // CTAs per cluster: one query
constexpr int RC_M = 128;         // candidates per tile
constexpr int RC_THREADS = 256;   // 8 warps: two per tensor-memory lane quarter
constexpr int RC_SMALL = 256;     // boundary candidates ranked by counting
constexpr int RC_BIN_SLICE = RB / RC_CL;  // histogram bins summed by each CTA
static_assert(FUSED_BCAP >= RC_THREADS, "one bucket entry per thread inside the list");

template <bool FP8, int HN, int TPC>
struct RcCfg {
  static constexpr int ROW = FP8 ? 128 : 256;  // key bytes per token
  static constexpr int CH = ROW / 16;          // 16-byte chunks per row
  static constexpr int A_BYTES = RC_M * ROW;   // one tile of key rows
  static constexpr int B_BYTES = HN * 256;     // Q': bf16 (two K blocks) or two e4m3 terms
  static constexpr int SLOTS = TPC * RC_M;     // candidates per CTA
  static constexpr int TMEM_COLS = TPC * HN;
  static_assert(TMEM_COLS >= 32 && TMEM_COLS <= 512 && (TMEM_COLS & (TMEM_COLS - 1)) == 0, "tensor-memory columns");
  // after the MMAs the key tiles hold the selection's scratch: the boundary
  // list (key, tie) of SLOTS entries, then this CTA's part of the bitmap
  static constexpr int LIST_OFF = 0;
  static constexpr int BM_OFF = SLOTS * 8;
  static constexpr int BM_WORDS = MISA_MAX_L / 32 / RC_CL;
  static_assert(BM_OFF + 4 * BM_WORDS <= TPC * A_BYTES, "selection scratch inside the key tiles");
  static constexpr int SMEM = 1024 + TPC * A_BYTES + B_BYTES;  // dynamic, with the alignment slack
};

template <int SLOTS>
struct RcShared {
  uint2 bk[FUSED_BCAP];            // a handed-over row's boundary bucket (key, token)
  uint64_t done;
  uint32_t tmem_base;
  int abort;
  alignas(16) float w[128];        // weight per column (0: padding); read as float4
  int32_t tok[SLOTS];              // candidate token per slot (-1: none)
  float scale[SLOTS];              // e4m3 token scale per slot
  uint32_t key[SLOTS];             // order-preserving score key per slot
  uint32_t hist[HPAD];             // this CTA's counts, then the cluster's
  uint32_t tot[RC_BIN_SLICE];      // the cluster's counts of this CTA's bins
  uint32_t small_key[RC_SMALL], small_tie[RC_SMALL];
  uint4 res;
  uint32_t n_list, cnt;            // boundary entries listed here; tokens this CTA outputs
  uint32_t wa[RC_THREADS / 32], wb[RC_THREADS / 32 + 1];
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// every thread of every CTA of the cluster; orders shared-memory writes before it
// with the reads after it, across the cluster
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// the address of `p` (this CTA's shared memory) in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t peer_addr(const void *p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ uint32_t ld_peer(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ void or_peer(uint32_t a, uint32_t v) {
  asm volatile("red.shared::cluster.or.b32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}

// Radix levels of the composite (key, tie): bits of the key, then of the tie.
__device__ __forceinline__ void rc_level(int lvl, bool &lo_word, int &sft, uint32_t &dm) {
  lo_word = lvl >= 3;
  sft = lvl == 0 ? 21 : lvl == 1 ? 10 : lvl == 2 ? 0 : lvl == 3 ? 9 : 0;
  const int width = lvl <= 1 ? 11 : lvl == 2 ? 10 : 9;
  dm = (1u << width) - 1u;
}

template <bool FP8, int HN, int TPC>
__global__ void __cluster_dims__(RC_CL, 1, 1) __launch_bounds__(RC_THREADS, 1)
    rerank_cluster_kernel(CacheView c, QueryView qv, const int32_t *gather, int n_cols, int k, int32_t *out,
                          float *scores, long long ld, const uint32_t *pend, const uint2 *pend_bucket) {
  grid_dep_sync();
  using Cfg = RcCfg<FP8, HN, TPC>;
  constexpr int SLOTS = Cfg::SLOTS;
  extern __shared__ uint8_t rc_raw[];
  // the same dynamic size in every CTA of the cluster: all of them leave here together
  uint8_t *base = aligned_smem_base(rc_raw, Cfg::SMEM - 1024, c);  // 1024-aligned (swizzle atoms)
  if (!base) return;
  uint8_t *a_smem = base;                      // TPC x A_BYTES
  uint8_t *b_smem = base + TPC * Cfg::A_BYTES;  // B_BYTES
  __shared__ RcShared<SLOTS> sh;
  volatile int *abort = &sh.abort;
  const int i = blockIdx.y;
  const uint32_t rank = cluster_rank();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int s;
  const int Li = query_prefix(c, qv, i, &s);
  const int col0 = (int)rank * SLOTS;
  const int ntile = max(0, min(TPC, cdiv(n_cols - col0, RC_M)));
  const uint8_t *kbase = static_cast<const uint8_t *>(c.keys) + (size_t)max(s, 0) * c.L_cap * Cfg::ROW;
  const float *sbase = FP8 ? c.scale + (size_t)max(s, 0) * c.L_cap : nullptr;

  // 1. this CTA's candidates (-1: none, negative, or beyond the prefix).
  //    With a handed-over row (pend != nullptr) only slots below its winner
  //    count hold candidates; the `need` best entries of its boundary bucket
  //    (larger key first, equal keys to the lower token) fill the next ones.
  // (the slots' tokens are requested together with the counters, then masked)
  constexpr int EPT = (SLOTS + RC_THREADS - 1) / RC_THREADS;
  int tk[EPT];
#pragma unroll
  for (int u = 0; u < EPT; ++u) {
    const int e = tid + u * RC_THREADS, p = col0 + e;
    tk[u] = (e < SLOTS && p < n_cols) ? __ldg(gather + (size_t)i * n_cols + p) : -1;
  }
  int n_sure = n_cols, pneed = 0, nb = 0;
  const uint32_t *pctr = nullptr;
  uint2 bk0 = make_uint2(0u, 0u);  // the bucket's first entries, requested with the counters
  if (pend) {
    bk0 = __ldcg(pend_bucket + (size_t)i * FUSED_BCAP + tid);
    pctr = pend + (size_t)i * FUSED_ZERO_WORDS + 2 * RB;
    n_sure = (int)min(__ldcg(pctr + FUSED_CTR_EMIT), (uint32_t)n_cols);
    nb = (int)min(__ldcg(pctr + FUSED_CTR_BUCKET), (uint32_t)FUSED_BCAP);
    pneed = (int)min(__ldcg(pctr + FUSED_CTR_NEED), (uint32_t)(n_cols - n_sure));
  }
#pragma unroll
  for (int u = 0; u < EPT; ++u) {
    const int e = tid + u * RC_THREADS, t = tk[u];
    if (e < SLOTS) sh.tok[e] = (col0 + e < n_sure && t >= 0 && t < Li) ? t : -1;
  }
  if (tid == 0) {
    mbar_init(&sh.done, 1);
    sh.abort = 0;
    fence_mbar_init();
  }
  if (pneed > 0 && n_sure + pneed > col0 && n_sure < col0 + SLOTS) {  // uniform: this CTA holds some of them
    const uint2 *brow = pend_bucket + (size_t)i * FUSED_BCAP;
    if (tid < nb) sh.bk[tid] = bk0;
    for (int x = tid + RC_THREADS; x < nb; x += RC_THREADS) sh.bk[x] = __ldcg(brow + x);
    __syncthreads();
    for (int x = tid; x < nb; x += RC_THREADS) {
      const uint2 ex = sh.bk[x];
      int rank = 0;
      for (int y = 0; y < nb; ++y) {
        const uint2 ey = sh.bk[y];
        rank += (ey.x > ex.x || (ey.x == ex.x && ey.y < ex.y)) ? 1 : 0;
      }
      const int e = n_sure + rank - col0;
      const int t = (int)ex.y;
      if (rank < pneed && e >= 0 && e < SLOTS) sh.tok[e] = (t >= 0 && t < Li) ? t : -1;
    }
  }
  __syncthreads();

  // 2. every key row (and e4m3 scale) requested at once:
  //    row r, 16-byte chunk u at block (u / 8), row r, chunk (u % 8) ^ (r % 8)
  for (int x = tid; x < ntile * RC_M * Cfg::CH; x += RC_THREADS) {
    const int j = x / (RC_M * Cfg::CH), rem = x % (RC_M * Cfg::CH);
    const int r = rem / Cfg::CH, u = rem % Cfg::CH;
    const int t = sh.tok[j * RC_M + r];
    const uint32_t dst = smem_addr(a_smem + j * Cfg::A_BYTES + (u >> 3) * (RC_M * 128) + r * 128 +
                                   (((u & 7) ^ (r & 7)) << 4));
    cp_async16(dst, kbase + (size_t)max(t, 0) * Cfg::ROW + 16 * u, t >= 0);
  }
  if (FP8)
    for (int e = tid; e < ntile * RC_M; e += RC_THREADS) {
      const int t = sh.tok[e];
      cp_async4(smem_addr(&sh.scale[e]), sbase + max(t, 0), t >= 0);
    }
  cp_async_commit();

  // 3. meanwhile: Q', the histogram, tensor memory
  if (tid < 128) build_qprime<FP8, HN>(c, qv, nullptr, qv.H, i, b_smem, sh.w);
  for (int b = tid; b < HPAD; b += RC_THREADS) sh.hist[b] = 0;
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&sh.tmem_base)),
                 "n"(Cfg::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  cp_async_wait<0>();
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // rows and Q' visible to the tensor cores
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = sh.tmem_base;

  // 4. one thread issues every tile's MMAs; one commit for all of them
  if (tid == 0 && ntile > 0) {
    const uint32_t idesc = umma::instr_desc<FP8, RC_M, HN>();
    const uint32_t b_base = smem_addr(b_smem);
    for (int j = 0; j < ntile; ++j) {
      const uint32_t a_base = smem_addr(a_smem + j * Cfg::A_BYTES);
#pragma unroll
      for (int term = 0; term < (FP8 ? 2 : 1); ++term) {
#pragma unroll
        for (int kk = 0; kk < (FP8 ? 4 : 8); ++kk) {
          uint32_t aoff, boff;
          if (FP8) {
            aoff = kk * 32;
            boff = term * (HN * 128) + kk * 32;
          } else {
            aoff = (kk >> 2) * (RC_M * 128) + (kk & 3) * 32;
            boff = (kk >> 2) * (HN * 128) + (kk & 3) * 32;
          }
          umma::mma<FP8>(tmem + j * HN, umma::smem_desc_sw128(a_base + aoff), umma::smem_desc_sw128(b_base + boff),
                         idesc, (term | kk) ? 1u : 0u);
        }
      }
    }
    umma::commit(&sh.done);
  }

  // 5. epilogue: warp w drains lane quarter w % 4 of tiles w / 4, w / 4 + 2, ...
  // every thread waits (bounded); the CTA goes on only if none gave up
  const bool got = __syncthreads_and(ntile == 0 || umma::wait_bar(&sh.done, 0, abort, c)) != 0;
  umma::fence_after();
  if (got) {
    const int q4 = warp & 3, r = 32 * q4 + lane;
    const uint32_t tl = tmem + ((uint32_t)(32 * q4) << 16);
    const float4 *w4 = reinterpret_cast<const float4 *>(sh.w);
    for (int j = warp >> 2; j < ntile; j += 2) {
      float a4[4] = {0.f, 0.f, 0.f, 0.f};  // independent partial sums
#pragma unroll
      for (int cb = 0; cb < HN; cb += 32) {
        uint32_t v[32];
        umma::ld32(tl + j * HN + cb, v);
        umma::ld_wait();
#pragma unroll
        for (int x = 0; x < 32; x += 4) {
          const float4 w = w4[(cb + x) >> 2];
          a4[0] = fmaf(w.x, fmaxf(__uint_as_float(v[x]), 0.f), a4[0]);
          a4[1] = fmaf(w.y, fmaxf(__uint_as_float(v[x + 1]), 0.f), a4[1]);
          a4[2] = fmaf(w.z, fmaxf(__uint_as_float(v[x + 2]), 0.f), a4[2]);
          a4[3] = fmaf(w.w, fmaxf(__uint_as_float(v[x + 3]), 0.f), a4[3]);
        }
      }
      const float acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
      const int e = j * RC_M + r;
      if (sh.tok[e] >= 0) {
        const float val = FP8 ? acc * sh.scale[e] : acc;
        if (scores) scores[(size_t)i * ld + col0 + e] = val;
        const uint32_t key = ordered_key(val);
        sh.key[e] = key;
        atomicAdd(&sh.hist[hpos(key >> 21)], 1u);
      }
    }
  } else if (tid == 0) {
    mbar_wait(&sh.done, 0);  // bounded: the MMAs finish before the tensor memory is released
  }
  umma::fence_before();
  __syncthreads();
  if (warp == 0) {
    umma::fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(Cfg::TMEM_COLS));
  }
  if (!got)  // no candidates from a CTA whose MMAs gave up (its keys were never written)
    for (int e = tid; e < SLOTS; e += RC_THREADS) sh.tok[e] = -1;
  // the key tiles are free: clear this CTA's part of the token bitmap
  const int bm_words = cdiv(cdiv(max(Li, 0), 32), RC_CL);  // words per CTA (<= BM_WORDS)
  uint32_t *bm = reinterpret_cast<uint32_t *>(a_smem + Cfg::BM_OFF);
  uint2 *list = reinterpret_cast<uint2 *>(a_smem + Cfg::LIST_OFF);
  for (int w = tid; w < bm_words; w += RC_THREADS) bm[w] = 0;
  __syncthreads();

  // 6. the cluster's selection
  uint32_t P_hi = 0, M_hi = 0, P_lo = 0, M_lo = 0;
  uint32_t need = (uint32_t)k;
  int mode = 0;  // 1: every valid candidate; 2: the prefix's whole bin; 3: rank the boundary bin's list
  for (int lvl = 0; lvl < 5 && mode == 0; ++lvl) {
    bool lo_word;
    int sft;
    uint32_t dm;
    rc_level(lvl, lo_word, sft, dm);
    if (lvl > 0) {  // level 0 was counted by the epilogue
      for (int b = tid; b < HPAD; b += RC_THREADS) sh.hist[b] = 0;
      __syncthreads();
      for (int e = tid; e < SLOTS; e += RC_THREADS) {
        const int t = sh.tok[e];
        if (t < 0) continue;
        const uint32_t kx = sh.key[e], lx = POS_MAX - (uint32_t)t;
        if ((kx & M_hi) == P_hi && (lx & M_lo) == P_lo) atomicAdd(&sh.hist[hpos(((lo_word ? lx : kx) >> sft) & dm)], 1u);
      }
    }
    __syncthreads();
    cluster_sync();  // every CTA's counts are final
    {
      const int b = (int)rank * RC_BIN_SLICE + tid;  // one bin per thread
      uint32_t a[RC_CL];
#pragma unroll
      for (int r2 = 0; r2 < RC_CL; ++r2) a[r2] = ld_peer(peer_addr(&sh.hist[hpos(b)], (uint32_t)r2));
      uint32_t v = 0;
#pragma unroll
      for (int r2 = 0; r2 < RC_CL; ++r2) v += a[r2];
      sh.tot[tid] = v;
    }
    cluster_sync();  // every slice summed
    {
      uint32_t a[RB / RC_THREADS];
#pragma unroll
      for (int u = 0; u < RB / RC_THREADS; ++u) {
        const int x = tid + u * RC_THREADS;
        a[u] = ld_peer(peer_addr(&sh.tot[x % RC_BIN_SLICE], (uint32_t)(x / RC_BIN_SLICE)));
      }
#pragma unroll
      for (int u = 0; u < RB / RC_THREADS; ++u) sh.hist[hpos(tid + u * RC_THREADS)] = a[u];
    }
    __syncthreads();
    if (warp == 0) {
      const uint4 x = warp_select_bin<true>(sh.hist, need);
      if (lane == 0) sh.res = x;
    }
    __syncthreads();
    const uint4 r = sh.res;
    if (lvl == 0 && (uint32_t)k >= r.w) {
      mode = 1;  // k covers every valid candidate (r.w of them)
      break;
    }
    need -= r.y;  // taken above the bin
    if (!lo_word) {
      P_hi |= r.x << sft;
      M_hi |= dm << sft;
    } else {
      P_lo |= r.x << sft;
      M_lo |= dm << sft;
    }
    if (r.z == need || lvl == 4)
      mode = 2;  // the bin goes whole (after the last level only repeated candidates share it)
    else if (r.z <= (uint32_t)RC_SMALL)
      mode = 3;
  }
  // the prefix through the boundary bin is (P, M); winners lie above it, and
  // in mode 3 the `need` best of the bin's own candidates
  if (mode == 3) {
    if (tid == 0) sh.n_list = 0;
    __syncthreads();
    for (int e = tid; e < SLOTS; e += RC_THREADS) {
      const int t = sh.tok[e];
      if (t < 0) continue;
      const uint32_t kx = sh.key[e], lx = POS_MAX - (uint32_t)t;
      if ((kx & M_hi) == P_hi && (lx & M_lo) == P_lo) list[atomicAdd(&sh.n_list, 1u)] = make_uint2(kx, lx);
    }
    __syncthreads();
  }
  cluster_sync();  // the lists are complete (uniform: every CTA has the same mode)
  uint32_t n_small = 0;
  if (mode == 3) {
    // every CTA copies the whole boundary list (at most RC_SMALL entries)
    uint32_t cnt[RC_CL];
#pragma unroll
    for (int r2 = 0; r2 < RC_CL; ++r2) cnt[r2] = ld_peer(peer_addr(&sh.n_list, (uint32_t)r2));
    uint32_t off = 0;
#pragma unroll
    for (int r2 = 0; r2 < RC_CL; ++r2) {
      for (uint32_t x = tid; x < cnt[r2]; x += RC_THREADS) {
        if (off + x < (uint32_t)RC_SMALL) {
          const uint32_t a = peer_addr(&list[x], (uint32_t)r2);
          sh.small_key[off + x] = ld_peer(a);
          sh.small_tie[off + x] = ld_peer(a + 4);
        }
      }
      off += cnt[r2];
    }
    n_small = min(off, (uint32_t)RC_SMALL);
    __syncthreads();
  }
  // mark the winners in their owners' bitmaps
  const uint32_t per_tok = (uint32_t)bm_words * 32u;
  for (int e = tid; e < SLOTS; e += RC_THREADS) {
    const int t = sh.tok[e];
    if (t < 0) continue;
    const uint32_t kx = sh.key[e], lx = POS_MAX - (uint32_t)t;
    bool win;
    if (mode == 1) {
      win = true;
    } else {
      const uint32_t kh = kx & M_hi, kl = lx & M_lo;
      const bool above = kh > P_hi || (kh == P_hi && kl > P_lo);
      const bool in_bin = kh == P_hi && kl == P_lo;
      if (mode == 2) {
        win = above || in_bin;
      } else {
        uint32_t beat = 0;  // boundary candidates ahead of this one
        if (in_bin)
          for (uint32_t y = 0; y < n_small; ++y) {
            const uint32_t ky = sh.small_key[y], ly = sh.small_tie[y];
            beat += (ky > kx || (ky == kx && ly > lx)) ? 1u : 0u;
          }
        win = above || (in_bin && beat < need);
      }
    }
    if (win) {
      const uint32_t owner = (uint32_t)t / per_tok, off = (uint32_t)t - owner * per_tok;
      or_peer(peer_addr(&bm[off >> 5], owner), 1u << (off & 31));
    }
  }
  cluster_sync();  // every bitmap is complete
  // this CTA's tokens in ascending order, after those of the CTAs before it
  const int per = cdiv(bm_words, RC_THREADS);
  const int w0 = min(tid * per, bm_words), w1 = min(w0 + per, bm_words);
  uint32_t c_own = 0;
  for (int w = w0; w < w1; ++w) c_own += __popc(bm[w]);
  uint32_t n_cta;
  uint32_t j = block_excl_scan<RC_THREADS>(c_own, &n_cta, sh.wa, sh.wb);
  if (tid == 0) sh.cnt = n_cta;
  cluster_sync();  // every CTA's count is published
  uint32_t before = 0, total = 0;
#pragma unroll
  for (int r2 = 0; r2 < RC_CL; ++r2) {
    const uint32_t v = ld_peer(peer_addr(&sh.cnt, (uint32_t)r2));
    before += (uint32_t)r2 < rank ? v : 0u;
    total += v;
  }
  int32_t *orow = out + (size_t)i * k;
  const uint32_t tok0 = rank * per_tok;
  j += before;
  for (int w = w0; w < w1 && j < (uint32_t)k; ++w) {
    uint32_t m = bm[w];
    while (m && j < (uint32_t)k) {
      orow[j++] = (int32_t)(tok0 + 32u * w + (uint32_t)(__ffs(m) - 1));
      m &= m - 1;
    }
  }
  for (int p = (int)min(total, (uint32_t)k) + (int)rank * RC_THREADS + tid; p < k; p += RC_CL * RC_THREADS) orow[p] = -1;
  cluster_sync();  // no CTA leaves while another may still read its shared memory
}

template <bool FP8, int HN, int TPC>
bool rc_fits() {
  struct Tag {};
  return cached_per_device<Tag>([] {
           auto *kern = rerank_cluster_kernel<FP8, HN, TPC>;
           if (opt_in_max_dyn_smem(kern) < RcCfg<FP8, HN, TPC>::SMEM) return -1;
           cudaLaunchConfig_t cfg = {};
           cfg.gridDim = dim3(RC_CL, 1);
           cfg.blockDim = dim3(RC_THREADS);
           cfg.dynamicSmemBytes = RcCfg<FP8, HN, TPC>::SMEM;
           int n = 0;
           if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
             cudaGetLastError();
             return -1;
           }
           return n >= 1 ? 1 : -1;
         }) > 0;
}

// Tiles per CTA for n_cols candidates: the smallest power of two whose
// cluster holds them, 0 when none fits the tensor memory or shared memory.
template <bool FP8, int HN>
int rc_tpc(int n_cols) {
  for (int tpc = 1; tpc <= 8; tpc *= 2) {
    if (tpc * HN > 512 || RcCfg<FP8, HN, 1>::A_BYTES * tpc + HN * 256 + 1024 > 200 * 1024) return 0;
    if (RC_CL * RC_M * tpc >= n_cols) return tpc;
  }
  return 0;
}

template <bool FP8, int HN>
cudaError_t rc_launch_hn(const CacheView &c, const QueryView &q, const int32_t *gather, int n_cols, int k,
                         int32_t *out, float *scores, long long ld, const uint32_t *pend, const uint2 *pend_bucket,
                         cudaStream_t s, bool dry) {
  const int tpc = rc_tpc<FP8, HN>(n_cols);
#define MISA_RC_CASE(T)                                                                                     \
  if (tpc == T) {                                                                                           \
    if constexpr (T * HN <= 512 && (FP8 ? 128 : 256) * RC_M * T + HN * 256 + 1024 <= 200 * 1024) {         \
      if (!rc_fits<FP8, HN, T>()) return cudaErrorNotSupported;                                            \
      if (dry) return cudaSuccess;                                                                          \
      return launch_kernel(rerank_cluster_kernel<FP8, HN, T>, dim3(RC_CL, q.n_q), dim3(RC_THREADS),        \
                           RcCfg<FP8, HN, T>::SMEM, s, c, q, gather, n_cols, k, out, scores, ld, pend,     \
                           pend_bucket);                                                                   \
    }                                                                                                       \
  }
  MISA_RC_CASE(1)
  MISA_RC_CASE(2)
  MISA_RC_CASE(4)
  MISA_RC_CASE(8)
#undef MISA_RC_CASE
  return cudaErrorNotSupported;
}

cudaError_t rc_dispatch(const CacheView &c, const QueryView &q, const int32_t *gather, int n_cols, int k, int32_t *out,
                        float *scores, long long ld, const uint32_t *pend, const uint2 *pend_bucket, cudaStream_t s,
                        bool dry) {
  if (q.n_q < 1 || n_cols < 1 || k < 1 || k > n_cols || q.H > 128) return cudaErrorNotSupported;
  const int hn = q.H <= 32 ? 32 : q.H <= 64 ? 64 : 128;
  if (c.fp8) {
    if (hn == 32) return rc_launch_hn<true, 32>(c, q, gather, n_cols, k, out, scores, ld, pend, pend_bucket, s, dry);
    if (hn == 64) return rc_launch_hn<true, 64>(c, q, gather, n_cols, k, out, scores, ld, pend, pend_bucket, s, dry);
    return rc_launch_hn<true, 128>(c, q, gather, n_cols, k, out, scores, ld, pend, pend_bucket, s, dry);
  }
  if (hn == 32) return rc_launch_hn<false, 32>(c, q, gather, n_cols, k, out, scores, ld, pend, pend_bucket, s, dry);
  if (hn == 64) return rc_launch_hn<false, 64>(c, q, gather, n_cols, k, out, scores, ld, pend, pend_bucket, s, dry);
  return rc_launch_hn<false, 128>(c, q, gather, n_cols, k, out, scores, ld, pend, pend_bucket, s, dry);
}

}  // namespace

bool rerank_cluster_applies(const CacheView &c, const QueryView &q, int n_cols, int k) {
  return rc_dispatch(c, q, nullptr, n_cols, k, nullptr, nullptr, 0, nullptr, nullptr, nullptr, true) == cudaSuccess;
}

cudaError_t launch_rerank_cluster(const CacheView &c, const QueryView &q, const int32_t *gather, int n_cols, int k,
                                  int32_t *out, float *scores, long long ld, cudaStream_t s, const uint32_t *pend,
                                  const uint2 *pend_bucket) {
  return rc_dispatch(c, q, gather, n_cols, k, out, scores, ld, pend, pend_bucket, s, false);
}

}  // namespace misa
