// Re-rank scoring of gathered candidates (the MISA-dagger fine stage) on the
// fifth-generation tensor cores.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference",
// technical summary, "Hierarchical variant": the original DSA indexer -- all
// H_I heads -- re-scores only the candidate set kept by the routed pass:
//     I_t = s_t * sum_n w_{i,n} * ReLU(q_{i,n} . k_t),   t in gather[i].
// For one query the candidates' keys against its heads are a dense product:
// 128 gathered key rows on the MMA M side, the query's scoring heads on N
// (HN columns, zero-weight padding up to a power of two >= 32), d = 128 on K.
//
// gather == nullptr: the candidates are the prefix itself (dense scoring of
// decode queries with many heads, where the same dense product on mma.sync
// would be compute-bound): dense_umma_kernel below, a persistent form that
// builds the query's head matrix once per CTA and streams the prefix.
//
// One CTA of 4 warps takes up to T = 2 tiles of 128 candidates of one query.  It
// requests every key row of its tiles at once with 16-byte cp.async into the
// 128-byte-swizzled K-major layout the MMA reads (invalid candidates are
// zero-filled and never written), builds the query's head matrix Q' (bf16,
// or the exact two-term e4m3 split of a bf16 query with a power-of-two scale
// folded into the weight) while the rows are in flight, then one thread
// issues all the tiles' MMAs into tensor memory and commits them to one
// mbarrier.  The four warps read one candidate row per thread with
// tcgen05.ld, apply ReLU, the weights, the head sum and the e4m3 token scale,
// write the score and count it in the row histogram (shared memory, added to
// row_hist once per CTA).  The wait on the MMAs is bounded: one that runs out
// sets MISA_DEV_WAIT_TIMEOUT and the CTA returns without scores.
#include <cuda.h>

#include <algorithm>

#include "frag.cuh"
#include "internal.h"
#include "qprime.cuh"
#include "rowsel.cuh"
#include "umma.cuh"

namespace misa {
namespace {

constexpr int RR_M = 128;       // candidates per tile
constexpr int RR_THREADS = 128;  // 4 warps: loaders, then one tensor-memory lane quarter each

template <bool FP8, int HN, int TT>
struct RCfg {
  static constexpr int ROW = FP8 ? 128 : 256;       // key bytes per token
  static constexpr int CH = ROW / 16;               // 16-byte chunks per row
  static constexpr int A_BYTES = RR_M * ROW;        // one tile of key rows
  static constexpr int B_BYTES = HN * 256;          // Q': bf16 (two K blocks) or two e4m3 terms
  static constexpr int T = TT;                      // tiles per CTA (T * HN <= 256 tensor-memory columns)
  static_assert(T * HN <= 256 && T <= 4, "tensor-memory columns per CTA");
  static constexpr int TMEM_COLS = T * HN;
  static constexpr int SMEM = 1024 + T * A_BYTES + B_BYTES;
};

struct RerankShared {
  uint64_t done;
  uint32_t tmem_base;
  int abort;
  alignas(16) float w[128];        // weight per column (0: padding); read as float4
  int32_t tok[4 * RR_M];           // candidate token per slot (-1: skip)
  float scale[4 * RR_M];           // e4m3 token scale per slot
  uint32_t hist[TOPK_HIST_BINS];   // this CTA's share of the row histogram
};

// fz.zeroed != nullptr: the row's top fz.k are selected here (rowsel.cuh),
// with each thread's scores kept in registers, instead of the histogram going
// to row_hist.
template <bool FP8, int HN, int TT>
__global__ void __launch_bounds__(RR_THREADS) rerank_umma_kernel(CacheView c, QueryView qv, const int32_t *heads,
                                                                  int h, const int32_t *gather, int n_cols,
                                                                  float *scores, long long ld,
                                                                  uint32_t *row_hist, FusedTopk fz) {
  grid_dep_sync();
  using Cfg = RCfg<FP8, HN, TT>;
  constexpr int T = Cfg::T;
  extern __shared__ uint8_t rr_raw[];
  // the tiles and Q', or (a fused selection, afterwards) its state and scratch
  const uint32_t sel_bytes =
      (uint32_t)((sizeof(RsShared<RR_THREADS>) + 15) / 16 * 16) + rs_scratch_bytes(c.L_cap, T * RR_M, RR_THREADS);
  const uint32_t need = max((uint32_t)(Cfg::SMEM - 1024), fz.zeroed ? sel_bytes : 0u);
  uint8_t *base = aligned_smem_base(rr_raw, need, c);  // 1024-aligned (swizzle atoms)
  if (!base) return;
  uint8_t *a_smem = base;                       // T x A_BYTES
  uint8_t *b_smem = base + T * Cfg::A_BYTES;    // B_BYTES
  __shared__ RerankShared sh;
  volatile int *abort = &sh.abort;
  const int i = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int s;
  const int Li = query_prefix(c, qv, i, &s);
  const int col0 = blockIdx.x * T * RR_M;
  if (!gather && col0 >= Li) return;  // uniform: a prefix row with nothing here (no barrier or allocation yet)
  const int ntile = min(T, cdiv(n_cols - col0, RR_M));
  const uint8_t *kbase = static_cast<const uint8_t *>(c.keys) + (size_t)max(s, 0) * c.L_cap * Cfg::ROW;
  const float *sbase = FP8 ? c.scale + (size_t)max(s, 0) * c.L_cap : nullptr;

  // 1. candidate tokens of this CTA's slots (-1: none, negative, or beyond the prefix)
  for (int e = tid; e < T * RR_M; e += RR_THREADS) {
    const int p = col0 + e;
    const int t = (e < ntile * RR_M && p < n_cols) ? (gather ? __ldg(gather + (size_t)i * n_cols + p) : p) : -1;
    sh.tok[e] = (t >= 0 && t < Li) ? t : -1;
  }
  if (tid == 0) {
    mbar_init(&sh.done, 1);
    sh.abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  // 2. every key row (and e4m3 scale) of every tile requested at once:
  //    row r, 16-byte chunk u at block (u / 8), row r, chunk (u % 8) ^ (r % 8)
  for (int x = tid; x < ntile * RR_M * Cfg::CH; x += RR_THREADS) {
    const int j = x / (RR_M * Cfg::CH), rem = x % (RR_M * Cfg::CH);
    const int r = rem / Cfg::CH, u = rem % Cfg::CH;
    const int t = sh.tok[j * RR_M + r];
    const uint32_t dst = smem_addr(a_smem + j * Cfg::A_BYTES + (u >> 3) * (RR_M * 128) + r * 128 +
                                   (((u & 7) ^ (r & 7)) << 4));
    cp_async16(dst, kbase + (size_t)max(t, 0) * Cfg::ROW + 16 * u, t >= 0);
  }
  if (FP8)
    for (int e = tid; e < ntile * RR_M; e += RR_THREADS) {
      const int t = sh.tok[e];
      cp_async4(smem_addr(&sh.scale[e]), sbase + max(t, 0), t >= 0);
    }
  cp_async_commit();

  // 3. meanwhile: Q', weights, histogram, tensor memory
  build_qprime<FP8, HN>(c, qv, heads, h, i, b_smem, sh.w);
  for (int b = tid; b < TOPK_HIST_BINS; b += RR_THREADS) sh.hist[b] = 0;
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
  if (tid == 0) {
    const uint32_t idesc = umma::instr_desc<FP8, RR_M, HN>();
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
            aoff = (kk >> 2) * (RR_M * 128) + (kk & 3) * 32;
            boff = (kk >> 2) * (HN * 128) + (kk & 3) * 32;
          }
          umma::mma<FP8>(tmem + j * HN, umma::smem_desc_sw128(a_base + aoff), umma::smem_desc_sw128(b_base + boff),
                         idesc, (term | kk) ? 1u : 0u);
        }
      }
    }
    umma::commit(&sh.done);
  }

  // 5. epilogue: candidate row r = 32 * warp + lane of every tile
  const bool got = umma::wait_bar(&sh.done, 0, abort, c);
  umma::fence_after();
  float kept[T];  // fused selection: this thread's scores
#pragma unroll
  for (int j = 0; j < T; ++j) kept[j] = 0.f;
  if (got) {
    const int r = warp * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll
    for (int j = 0; j < T; ++j) {
      if (j >= ntile) break;
      float a4[4] = {0.f, 0.f, 0.f, 0.f};  // independent partial sums
      const float4 *w4 = reinterpret_cast<const float4 *>(sh.w);
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
      const int e = j * RR_M + r;
      const int t = sh.tok[e];
      if (t >= 0) {
        const float val = FP8 ? acc * sh.scale[e] : acc;
        scores[(size_t)i * ld + col0 + e] = val;
        kept[j] = val;
        atomicAdd(&sh.hist[ordered_key(val) >> 21], 1u);
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
  if (fz.zeroed) {
    // the tensor memory is released before any wait on the row's other CTAs
    // (one of them may still be waiting to allocate); a CTA whose MMAs gave
    // up never arrives, and the row's waits run out
    if (!got) return;
    // the key tiles are free: the selection's shared state and scratch go there
    RsShared<RR_THREADS> &rs = *reinterpret_cast<RsShared<RR_THREADS> *>(a_smem);
    uint8_t *scratch = a_smem + (sizeof(RsShared<RR_THREADS>) + 15) / 16 * 16;
    const int r = warp * 32 + lane;
    auto each = [&](auto &&fn) {
#pragma unroll
      for (int j = 0; j < T; ++j) {
        const int t = sh.tok[j * RR_M + r];
        const bool valid = j < ntile && t >= 0;
        fn(valid ? ordered_key(kept[j]) : 0u, t, valid);
      }
    };
    const float *srow = scores + (size_t)i * ld;
    const int32_t *grow = gather + (size_t)i * n_cols;
    auto sweep = [&](auto &&fn) {
      constexpr int SU = 8;
      for (int base = 0; base < n_cols; base += RR_THREADS * SU) {
        int tk[SU];
        float v[SU];
#pragma unroll
        for (int u = 0; u < SU; ++u) {
          const int p = base + u * RR_THREADS + tid;
          tk[u] = p < n_cols ? __ldg(grow + p) : -1;
          v[u] = (tk[u] >= 0 && tk[u] < Li) ? __ldcg(srow + p) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < SU; ++u) {
          const bool ok = tk[u] >= 0 && tk[u] < Li;
          fn(ordered_key(v[u]), POS_MAX - (uint32_t)(ok ? tk[u] : 0), ok);
        }
      }
    };
    row_select<RR_THREADS>(c, rs, sh.hist, scratch, rs_row(fz, i), gridDim.x, fz.k, Li, fz.ordered != 0, T * RR_M,
                           each, sweep);
    return;
  }
  if (got) {
    uint32_t *rh = row_hist + (size_t)i * TOPK_HIST_BINS;
    for (int b = tid; b < TOPK_HIST_BINS; b += RR_THREADS) {
      const uint32_t v = sh.hist[b];
      if (v) atomicAdd(rh + b, v);
    }
  }
}

// ---- dense prefix scoring of e4m3 caches (gather == nullptr) --------------
// A query's whole prefix against all its scoring heads: per 128-token tile
// the dense product D[t][n] = K[t] . Q'[n] (M = 128 tokens, N = HN columns,
// kind::f8f6f4 on the keys as stored against the two-term e4m3 split of the
// query).  Persistent and warp-specialised: CTA `part` of a query walks the
// tiles part, part + nparts, ... of its prefix (two CTAs per SM over all
// queries, so the CTAs read neighbouring tiles at the same time).
//   warps 0-1  producers: each key tile (16 KB, 128 consecutive tokens) is
//              copied with 16-byte cp.async into a ring of DS_STAGES stages
//              in the 128-byte-swizzled K-major layout (every warp
//              instruction one contiguous 512-byte span); a producer thread
//              keeps DS_LAG tiles in flight and marks a tile full once its
//              own copies of it have landed;
//   warp 2     owns the tensor memory; one thread issues each tile's MMAs into
//              one of two accumulator buffers and commits the stage back to
//              the producers and the buffer to the epilogue;
//   warps 3-6  the epilogue, one tensor-memory lane quarter per warp, one
//              token row per thread, draining the tiles in turn: ReLU, the
//              weights, the head sum (four independent partial sums) and the
//              e4m3 token scale (requested DS_SD tiles ahead), the score
//              written and counted.
// The two accumulator buffers let tile j + 1's MMAs run while tile j is
// drained.  Two such CTAs per SM stream the prefix faster than one CTA with
// twice the ring, more producers or a second epilogue set (measured).
// With a fused selection every score also stays in shared memory and the
// query's CTAs select its top k afterwards (rowsel.cuh).  Every wait is
// bounded: one that runs out sets MISA_DEV_WAIT_TIMEOUT and the CTA winds
// down without selecting.
constexpr int DS_STAGES = 4;
constexpr int DS_PROD = 2;                  // producer warps
constexpr int DS_LAG = DS_STAGES - 2;       // tiles a producer thread has in flight before marking one full
constexpr int DS_MMA_WARP = DS_PROD;
constexpr int DS_EPI0 = DS_PROD + 1;        // first epilogue warp
constexpr int DS_EPI = 4;  // sets of four warps, one per tensor-memory lane quarter
constexpr int DS_SETS = DS_EPI / 4;  // 1: one set drains every tile; 2: set b drains buffer b (tiles j % 2 == b)
static_assert(DS_SETS == 1 || DS_SETS == 2, "epilogue sets");
constexpr int DS_THREADS = 32 * (DS_EPI0 + DS_EPI);
constexpr int DS_CTAS = 2;  // CTAs per SM (two pipelines stream more than one with twice the ring)
constexpr int DS_SD = 6;  // set iterations a drain's token scales are requested ahead
constexpr int DS_SQ = 8;  // their slots per epilogue thread (> DS_SD: a slot is read before it is refilled)

template <int HN>
struct DSCfg {
  static constexpr int A_BYTES = RR_M * 128;  // one e4m3 key tile
  static constexpr int B_BYTES = HN * 256;    // Q': two e4m3 terms
  static constexpr int TMEM_COLS = 2 * HN;    // two accumulator buffers
  static constexpr int RING = DS_STAGES * A_BYTES + B_BYTES;  // from the 1024-byte-aligned base
  static_assert(TMEM_COLS >= 32 && TMEM_COLS <= 512, "tensor-memory columns");
};

struct DsShared {
  uint64_t full[DS_STAGES], empty[DS_STAGES];  // key stages: loaded / consumed
  uint64_t tfull[2], tempty[2];                // accumulators: written / drained
  uint32_t tmem_base;
  int abort;
  alignas(16) float w[128];                    // weight per column (0: padding)
  uint32_t hist[TOPK_HIST_BINS];               // this CTA's share of the row histogram
  float escl[DS_SQ][32 * DS_EPI];              // epilogue threads' token scales in flight
};

// Dynamic shared memory of a dense launch: alignment slack, the ring and Q',
// then (fused) the scores of max_tiles tiles.
template <int HN>
__host__ __device__ int dense_smem(int max_tiles, bool fused) {
  return 1024 + DSCfg<HN>::RING + (fused ? max_tiles * RR_M * 4 : 0);
}

template <int HN>
__global__ void __launch_bounds__(DS_THREADS, DS_CTAS)
    dense_umma_kernel(CacheView c, QueryView qv, const int32_t *heads, int h, float *scores, long long ld,
                      uint32_t *row_hist, int nparts, FusedTopk fz, int max_tiles) {
  grid_dep_sync();
  using Cfg = DSCfg<HN>;
  extern __shared__ uint8_t ds_raw[];
  const bool fused = fz.zeroed != nullptr;
  uint8_t *base = aligned_smem_base(ds_raw, dense_smem<HN>(max_tiles, fused) - 1024, c);  // 1024-aligned
  if (!base) return;
  uint8_t *a_smem = base;                             // DS_STAGES x A_BYTES
  uint8_t *b_smem = base + DS_STAGES * Cfg::A_BYTES;  // B_BYTES
  float *sc_s = reinterpret_cast<float *>(base + Cfg::RING);  // fused: [max_tiles][128]
  __shared__ DsShared sh;
  volatile int *abort = &sh.abort;
  const int i = blockIdx.y, part = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int s;
  const int Li = query_prefix(c, qv, i, &s);
  const int n_tiles = cdiv(max(Li, 0), RR_M);
  const int n_my = part < n_tiles ? cdiv(n_tiles - part, nparts) : 0;
  // a CTA without tiles leaves at once, unless the row's selection needs it
  if (n_my == 0 && !fused) return;  // uniform; nothing initialised yet

  if (tid == 0) {
    for (int st = 0; st < DS_STAGES; ++st) {
      mbar_init(&sh.full[st], 32 * DS_PROD);  // every producer thread
      mbar_init(&sh.empty[st], 1);            // the MMAs' commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh.tfull[b], 1);
      mbar_init(&sh.tempty[b], 4);  // the four warps of the set that drains it
    }
    sh.abort = 0;
    fence_mbar_init();
  }
  for (int b = tid; b < TOPK_HIST_BINS; b += DS_THREADS) sh.hist[b] = 0;
  if (warp >= DS_EPI0 && warp < DS_EPI0 + 4)  // the first four epilogue warps
    build_qprime<true, HN>(c, qv, heads, h, i, b_smem, sh.w, tid - 32 * DS_EPI0);
  if (warp == DS_MMA_WARP) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&sh.tmem_base)),
                 "n"(Cfg::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // Q' visible to the tensor cores
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = sh.tmem_base;
  uint32_t committed = 0;   // MMA thread: tiles whose MMAs it committed

  if (warp < DS_PROD) {
    // ---- producers: thread pt copies chunk pt % 8 of rows pt / 8 + 16 m ----
    const int pt = tid;
    const uint8_t *kbase = static_cast<const uint8_t *>(c.keys) + (size_t)s * c.L_cap * 128;
    int marked = 0;  // tiles this thread has marked full
    int j = 0;
    for (; j < n_my; ++j) {
      const int st = j % DS_STAGES;
      if (!umma::wait_bar(&sh.empty[st], ((j / DS_STAGES) & 1) ^ 1, abort, c)) break;
      const int t0 = (part + j * nparts) * RR_M;
      const uint32_t dst = smem_addr(a_smem + st * Cfg::A_BYTES);
#pragma unroll
      for (int m = 0; m < RR_M * 8 / (32 * DS_PROD); ++m) {
        const int x = pt + 32 * DS_PROD * m, r = x >> 3, u = x & 7;
        const bool ok = t0 + r < Li;
        cp_async16(dst + r * 128 + ((u ^ (r & 7)) << 4), ok ? kbase + (size_t)(t0 + r) * 128 + 16 * u : kbase, ok);
      }
      cp_async_commit();
      if (j >= DS_LAG) {  // the tile issued DS_LAG tiles ago has landed (this thread's part)
        cp_async_wait<DS_LAG>();
        mbar_arrive(&sh.full[(j - DS_LAG) % DS_STAGES]);
        marked = j - DS_LAG + 1;
      }
    }
    cp_async_wait<0>();  // no copy in flight past here
    if (j == n_my)
      for (int jj = marked; jj < n_my; ++jj) mbar_arrive(&sh.full[jj % DS_STAGES]);
  } else if (warp == DS_MMA_WARP) {
    // ---- MMA issuer ----
    if (lane == 0) {
      const uint32_t idesc = umma::instr_desc<true, RR_M, HN>();
      const uint32_t b_base = smem_addr(b_smem);
      for (int j = 0; j < n_my; ++j) {
        const int st = j % DS_STAGES, buf = j & 1;
        if (!umma::wait_bar(&sh.tempty[buf], ((j >> 1) & 1) ^ 1, abort, c)) break;
        umma::fence_after();
        if (!umma::wait_bar(&sh.full[st], (j / DS_STAGES) & 1, abort, c)) break;
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the copied rows, to the tensor cores
        umma::fence_after();
        const uint32_t a_base = smem_addr(a_smem + st * Cfg::A_BYTES);
#pragma unroll
        for (int term = 0; term < 2; ++term)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma::mma<true>(tmem + buf * HN, umma::smem_desc_sw128(a_base + kk * 32),
                            umma::smem_desc_sw128(b_base + term * (HN * 128) + kk * 32), idesc, (term | kk) ? 1u : 0u);
        umma::commit(&sh.empty[st]);
        umma::commit(&sh.tfull[buf]);
        committed = j + 1;
      }
    }
  } else {
    // ---- epilogue: set `set` drains the tiles j = set, set + DS_SETS, ...
    //      (accumulator buffer j % 2); token row r ----
    const int set = (warp - DS_EPI0) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t tl0 = tmem + ((uint32_t)(quarter * 32) << 16);
    const float4 *w4 = reinterpret_cast<const float4 *>(sh.w);
    const float *srow_scale = c.scale + (size_t)s * c.L_cap;
    // the token scales of this thread's rows travel DS_SD tiles of its set
    // ahead, by cp.async into its own slots (a load consumed two tiles later
    // left every drain waiting on memory latency)
    const int et = tid - 32 * DS_EPI0;
    auto fetch = [&](int n) {  // the scale of row r of the set's n-th tile; one group per call
      const int jn = set + DS_SETS * n, t = (part + jn * nparts) * RR_M + r;
      const bool ok = jn < n_my && t < Li;
      cp_async4(smem_addr(&sh.escl[n % DS_SQ][et]), ok ? srow_scale + t : srow_scale, ok);
      cp_async_commit();
    };
#pragma unroll
    for (int n = 0; n < DS_SD; ++n) fetch(n);
    for (int j = set, n = 0; j < n_my; j += DS_SETS, ++n) {
      const int t = (part + j * nparts) * RR_M + r, buf = j & 1;
      const uint32_t tl = tl0 + buf * HN;
      fetch(n + DS_SD);
      if (!umma::wait_bar(&sh.tfull[buf], (j >> 1) & 1, abort, c)) break;
      umma::fence_after();
      float a4[4] = {0.f, 0.f, 0.f, 0.f};  // independent partial sums
#pragma unroll
      for (int cb = 0; cb < HN; cb += 32) {
        uint32_t v[32];
        umma::ld32(tl + cb, v);
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
      umma::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.tempty[buf]);
      cp_async_wait<DS_SD>();  // this tile's scale (older groups) has landed
      const float scl = sh.escl[n % DS_SQ][et];
      if (t < Li) {
        const float val = acc * scl;
        scores[(size_t)i * ld + t] = val;
        if (fused) sc_s[j * RR_M + r] = val;
        atomicAdd(&sh.hist[ordered_key(val) >> 21], 1u);
      }
    }
    cp_async_wait<0>();
  }

  // ---- wind-down: no copy (every role waited for its own) and no MMA in
  //      flight when the memory is released ----
  __syncthreads();
  if (warp == DS_MMA_WARP && lane == 0 && committed > 0) {
    const uint32_t jl = committed - 1;  // the last committed accumulator buffer
    mbar_wait(&sh.tfull[jl & 1], (jl >> 1) & 1);  // bounded
  }
  umma::fence_before();
  __syncthreads();
  if (warp == DS_MMA_WARP) {
    umma::fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(Cfg::TMEM_COLS));
  }
  if (*abort) return;  // uniform (read after the barrier)
  if (fused) {
    // the ring is free: the selection's shared state and scratch go there
    RsShared<DS_THREADS> &rs = *reinterpret_cast<RsShared<DS_THREADS> *>(a_smem);
    uint8_t *scratch = a_smem + (sizeof(RsShared<DS_THREADS>) + 15) / 16 * 16;
    const int total = max_tiles * RR_M;
    auto each = [&](auto &&fn) {
      for (int x = tid; x < (total + DS_THREADS - 1) / DS_THREADS * DS_THREADS; x += DS_THREADS) {
        const int j = x / RR_M, rr = x % RR_M;
        const int tok = (part + j * nparts) * RR_M + rr;
        const bool valid = x < total && j < n_my && tok < Li;
        fn(valid ? ordered_key(sc_s[x]) : 0u, tok, valid);
      }
    };
    const float *srow = scores + (size_t)i * ld;
    auto sweep = [&](auto &&fn) {
      constexpr int SU = 8;
      for (int b0 = 0; b0 < Li; b0 += DS_THREADS * SU) {
        float v[SU];
#pragma unroll
        for (int u = 0; u < SU; ++u) {
          const int p = b0 + u * DS_THREADS + tid;
          v[u] = p < Li ? __ldcg(srow + p) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < SU; ++u) {
          const int p = b0 + u * DS_THREADS + tid;
          fn(ordered_key(v[u]), POS_MAX - (uint32_t)p, p < Li);
        }
      }
    };
    row_select<DS_THREADS>(c, rs, sh.hist, scratch, rs_row(fz, i), nparts, fz.k, Li, fz.ordered != 0, total, each,
                           sweep);
    return;
  }
  uint32_t *rh = row_hist + (size_t)i * TOPK_HIST_BINS;
  for (int b = tid; b < TOPK_HIST_BINS; b += DS_THREADS) {
    const uint32_t v = sh.hist[b];
    if (v) atomicAdd(rh + b, v);
  }
}

// Launch shape of a dense e4m3 call: one CTA per SM over all queries.
struct DensePlan {
  int nparts = 0, max_tiles = 0, smem = 0;
  bool ok = false;
};

template <int HN>
DensePlan plan_dense(const CacheView &c, const QueryView &q, bool fused) {
  DensePlan p;
  struct Tag {};
  const int max_dyn = cached_per_device<Tag>([] { return opt_in_max_dyn_smem(dense_umma_kernel<HN>); });
  const int sms = device_sms();
  const int n_tiles = cdiv(c.L_cap, RR_M);
  // DS_CTAS per SM (more CTAs than fit only queue); a fused selection needs
  // its whole grid resident, so it takes what the occupancy query confirms
  int per_sm = DS_CTAS;
  if (fused) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, dense_umma_kernel<HN>, DS_THREADS,
                                                      dense_smem<HN>(cdiv(n_tiles, sms), true)) != cudaSuccess) {
      cudaGetLastError();
      n = 1;
    }
    per_sm = std::max(1, std::min(n, DS_CTAS));
  }
  p.nparts = std::max(1, std::min(n_tiles, per_sm * sms / std::max(q.n_q, 1)));
  p.max_tiles = cdiv(n_tiles, p.nparts);
  p.smem = dense_smem<HN>(p.max_tiles, fused);
  // a fused selection's state and scratch reuse the ring
  const int sel = (int)((sizeof(RsShared<DS_THREADS>) + 15) / 16 * 16) + rs_scratch_bytes(c.L_cap, p.max_tiles * RR_M, DS_THREADS);
  p.ok = p.smem <= max_dyn && (!fused || ((long long)p.nparts * q.n_q <= (long long)per_sm * sms && sel <= DSCfg<HN>::RING)) && c.fp8 &&
         (reinterpret_cast<uintptr_t>(c.keys) & 15u) == 0;
  return p;
}

template <int HN>
cudaError_t launch_dense(const CacheView &c, const QueryView &q, const int32_t *heads, int h, float *scores,
                         long long ld, uint32_t *row_hist, cudaStream_t s, const FusedTopk *fz) {
  const DensePlan p = plan_dense<HN>(c, q, fz != nullptr);
  if (!p.ok) return cudaErrorInvalidConfiguration;
  FusedTopk none = {};
  return launch_kernel(dense_umma_kernel<HN>, dim3(p.nparts, q.n_q), dim3(DS_THREADS), p.smem, s, c, q, heads, h,
                       scores, ld, row_hist, p.nparts, fz ? *fz : none, p.max_tiles);
}

// Dynamic shared memory of a re-rank launch: the key tiles and Q', at least
// the fused selection's state and scratch (which reuse the tiles' space).
template <bool FP8, int HN, int TT>
int rerank_smem(const CacheView &c, bool fused) {
  using Cfg = RCfg<FP8, HN, TT>;
  const int sel = 1024 + (int)((sizeof(RsShared<RR_THREADS>) + 15) / 16 * 16) + rs_scratch_bytes(c.L_cap, TT * RR_M, RR_THREADS);
  return fused ? std::max(Cfg::SMEM, sel) : Cfg::SMEM;
}

// the kernel's dynamic shared-memory limit, raised once per device (-1: failed)
template <bool FP8, int HN, int TT>
int rerank_max_dyn() {
  struct Tag {};
  return cached_per_device<Tag>([] { return opt_in_max_dyn_smem(rerank_umma_kernel<FP8, HN, TT>); });
}

// A fused selection needs every CTA of the grid resident at once.
template <bool FP8, int HN, int TT>
bool rerank_fits(const CacheView &c, const QueryView &q, int n_cols) {
  using Cfg = RCfg<FP8, HN, TT>;
  const int smem = rerank_smem<FP8, HN, TT>(c, true);
  if (smem > rerank_max_dyn<FP8, HN, TT>()) return false;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rerank_umma_kernel<FP8, HN, TT>, RR_THREADS, smem) !=
      cudaSuccess)
    return false;
  const long long grid = (long long)cdiv(n_cols, Cfg::T * RR_M) * q.n_q;
  return grid <= (long long)per_sm * device_sms();
}

template <bool FP8, int HN, int TT>
cudaError_t launch_tt(const CacheView &c, const QueryView &q, const int32_t *heads, int h, const int32_t *gather,
                      int n_cols, float *scores, long long ld, uint32_t *row_hist, cudaStream_t s,
                      const FusedTopk *fz) {
  using Cfg = RCfg<FP8, HN, TT>;
  if (rerank_smem<FP8, HN, TT>(c, fz != nullptr) > rerank_max_dyn<FP8, HN, TT>()) return cudaErrorInvalidConfiguration;
  if (fz && !rerank_fits<FP8, HN, TT>(c, q, n_cols)) return cudaErrorInvalidConfiguration;
  const dim3 grid(cdiv(n_cols, Cfg::T * RR_M), q.n_q);
  FusedTopk none = {};
  return launch_kernel(rerank_umma_kernel<FP8, HN, TT>, grid, dim3(RR_THREADS), rerank_smem<FP8, HN, TT>(c, fz != nullptr),
                       s, c, q, heads, h, gather, n_cols, scores, ld, row_hist, fz ? *fz : none);
}

// Gathered candidates: 2 tiles per CTA (more CTAs shorten each gather chain);
// a prefix row: the persistent dense kernel.
// Tiles per CTA of a fused re-rank: two when that grid is resident at once,
// else four (half the CTAs; at most 64 heads), else 0 (no fused selection).
// The occupancy query answers one CTA per SM for this kernel, so the
// four-tile form is what a batch of 8 x 8192 candidates takes.
template <bool FP8, int HN>
int rerank_fused_tiles(const CacheView &c, const QueryView &q, int n_cols) {
  if (rerank_fits<FP8, HN, 2>(c, q, n_cols)) return 2;
  if constexpr (HN <= 64) {
    if (rerank_fits<FP8, HN, 4>(c, q, n_cols)) return 4;
  }
  return 0;
}

template <bool FP8, int HN>
cudaError_t launch_hn(const CacheView &c, const QueryView &q, const int32_t *heads, int h, const int32_t *gather,
                      int n_cols, float *scores, long long ld, uint32_t *row_hist, cudaStream_t s,
                      const FusedTopk *fz) {
  if (gather && fz) {
    const int tt = rerank_fused_tiles<FP8, HN>(c, q, n_cols);
    if constexpr (HN <= 64) {
      if (tt == 4) return launch_tt<FP8, HN, 4>(c, q, heads, h, gather, n_cols, scores, ld, row_hist, s, fz);
    }
    if (tt != 2) return cudaErrorInvalidConfiguration;
  }
  if (gather) return launch_tt<FP8, HN, 2>(c, q, heads, h, gather, n_cols, scores, ld, row_hist, s, fz);
  if (!FP8) return cudaErrorInvalidValue;  // dense decode of bf16 keys streams on mma.sync
  return launch_dense<HN>(c, q, heads, h, scores, ld, row_hist, s, fz);
}

int rerank_hn(const QueryView &q, const int32_t *heads, int h) {
  const int h_eff = heads ? h : q.H;
  return h_eff <= 32 ? 32 : h_eff <= 64 ? 64 : 128;
}

}  // namespace

bool rerank_umma_applies(const QueryView &q, const int32_t *heads, int h) {
  const int h_eff = heads ? h : q.H;
  return h_eff >= 1 && h_eff <= 128;
}

cudaError_t launch_rerank_umma(const CacheView &c, const QueryView &q, const int32_t *heads, int h,
                               const int32_t *gather, int n_cols, float *scores, long long ld, uint32_t *row_hist,
                               cudaStream_t s, const FusedTopk *fused) {
  if (q.n_q == 0 || n_cols == 0) return cudaSuccess;
#define MISA_RERANK_CASE(N)                                                                           \
  case N:                                                                                             \
    return c.fp8 ? launch_hn<true, N>(c, q, heads, h, gather, n_cols, scores, ld, row_hist, s, fused) \
                 : launch_hn<false, N>(c, q, heads, h, gather, n_cols, scores, ld, row_hist, s, fused);
  switch (rerank_hn(q, heads, h)) {
    MISA_RERANK_CASE(32)
    MISA_RERANK_CASE(64)
    MISA_RERANK_CASE(128)
    default:
      return cudaErrorInvalidValue;
  }
#undef MISA_RERANK_CASE
}

bool dense_fusable(const CacheView &c, const QueryView &q, const int32_t *heads, int h) {
  if (q.n_q == 0 || !c.fp8) return false;
  switch (rerank_hn(q, heads, h)) {
    case 32:
      return plan_dense<32>(c, q, true).ok;
    case 64:
      return plan_dense<64>(c, q, true).ok;
    case 128:
      return plan_dense<128>(c, q, true).ok;
    default:
      return false;
  }
}

bool rerank_fusable(const CacheView &c, const QueryView &q, const int32_t *heads, int h, int n_cols) {
  if (q.n_q == 0 || n_cols == 0) return false;
  switch (rerank_hn(q, heads, h)) {
    case 32:
      return (c.fp8 ? rerank_fused_tiles<true, 32>(c, q, n_cols) : rerank_fused_tiles<false, 32>(c, q, n_cols)) > 0;
    case 64:
      return (c.fp8 ? rerank_fused_tiles<true, 64>(c, q, n_cols) : rerank_fused_tiles<false, 64>(c, q, n_cols)) > 0;
    case 128:
      return (c.fp8 ? rerank_fused_tiles<true, 128>(c, q, n_cols) : rerank_fused_tiles<false, 128>(c, q, n_cols)) > 0;
    default:
      return false;
  }
}

}  // namespace misa
