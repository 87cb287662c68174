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

// Q' of query i in shared memory: row n = the n-th scoring head (zero rows
// past h_eff), two threads per row (half of its 16-byte chunks each, the pair
// agreeing on the e4m3 scale through a shuffle), in the 128-byte-swizzled
// K-major layout the MMA reads; bf16 as is, or the exact two-term e4m3 split
// with the power-of-two scale folded into the weight w_s[n].
template <bool FP8, int HN>
__device__ __forceinline__ void build_qprime(const CacheView &c, const QueryView &qv, const int32_t *heads, int h,
                                             int i, uint8_t *b_smem, float *w_s) {
  const int tid = threadIdx.x;
  const int H = qv.H;
  const int h_eff = heads ? h : H;
  for (int x = tid; x < 2 * HN; x += RR_THREADS) {  // whole warps: HN >= 32
    const int n = x >> 1, half = x & 1;
    int hd = -1;
    if (n < h_eff) {
      hd = heads ? __ldg(heads + (size_t)i * h + n) : n;
      if (hd < 0 || hd >= H) {
        if (half == 0) flag(c, MISA_DEV_BAD_HEAD);
        hd = -1;
      }
    }
    const uint4 *row = reinterpret_cast<const uint4 *>(qv.q + ((size_t)i * H + max(hd, 0)) * D) + half * 8;
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = hd >= 0 ? __ldg(row + u) : make_uint4(0u, 0u, 0u, 0u);
    float wv = hd >= 0 ? __ldg(qv.w + (size_t)i * H + hd) : 0.f;
    if (!FP8) {
#pragma unroll
      for (int u8 = 0; u8 < 8; ++u8) {
        const int u = half * 8 + u8;
        *reinterpret_cast<uint4 *>(b_smem + (u >> 3) * (HN * 128) + n * 128 + (((u & 7) ^ (n & 7)) << 4)) = v[u8];
      }
    } else {
      float m = 0.f;
#pragma unroll
      for (int u8 = 0; u8 < 8; ++u8) {
        const uint32_t ww[4] = {v[u8].x, v[u8].y, v[u8].z, v[u8].w};
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const float2 f = bf16x2_to_float2(ww[p]);
          m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
      }
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      const float sc = e4m3_head_scale(m);
      wv = wv / sc;  // exact: sc is a power of two
      // input chunk u (8 elements) -> 8 bytes of each term at byte 8u of the row
#pragma unroll
      for (int u8 = 0; u8 < 8; ++u8) {
        const int u = half * 8 + u8;
        uint2 t1, t2;
        split_e4m3(v[u8], sc, t1, t2);
        const int off = n * 128 + (((u >> 1) ^ (n & 7)) << 4) + (u & 1) * 8;
        *reinterpret_cast<uint2 *>(b_smem + off) = t1;
        *reinterpret_cast<uint2 *>(b_smem + HN * 128 + off) = t2;
      }
    }
    if (half == 0) w_s[n] = wv;
  }
}

template <bool FP8, int HN, int TT>
__global__ void __launch_bounds__(RR_THREADS) rerank_umma_kernel(CacheView c, QueryView qv, const int32_t *heads,
                                                                  int h, const int32_t *gather, int n_cols,
                                                                  float *scores, long long ld,
                                                                  uint32_t *row_hist) {
  grid_dep_sync();
  using Cfg = RCfg<FP8, HN, TT>;
  constexpr int T = Cfg::T;
  extern __shared__ uint8_t rr_raw[];
  uint8_t *base = rr_raw + ((1024u - (smem_addr(rr_raw) & 1023u)) & 1023u);  // 1024-aligned (swizzle atoms)
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
  if (got) {
    const int r = warp * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    for (int j = 0; j < ntile; ++j) {
      float acc = 0.f;
      const float4 *w4 = reinterpret_cast<const float4 *>(sh.w);
#pragma unroll
      for (int cb = 0; cb < HN; cb += 32) {
        uint32_t v[32];
        umma::ld32(tl + j * HN + cb, v);
        umma::ld_wait();
#pragma unroll
        for (int x = 0; x < 32; x += 4) {
          const float4 w = w4[(cb + x) >> 2];
          acc = fmaf(w.x, fmaxf(__uint_as_float(v[x]), 0.f), acc);
          acc = fmaf(w.y, fmaxf(__uint_as_float(v[x + 1]), 0.f), acc);
          acc = fmaf(w.z, fmaxf(__uint_as_float(v[x + 2]), 0.f), acc);
          acc = fmaf(w.w, fmaxf(__uint_as_float(v[x + 3]), 0.f), acc);
        }
      }
      const int e = j * RR_M + r;
      const int t = sh.tok[e];
      if (t >= 0) {
        const float val = FP8 ? acc * sh.scale[e] : acc;
        scores[(size_t)i * ld + col0 + e] = val;
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
  if (got) {
    uint32_t *rh = row_hist + (size_t)i * TOPK_HIST_BINS;
    for (int b = tid; b < TOPK_HIST_BINS; b += RR_THREADS) {
      const uint32_t v = sh.hist[b];
      if (v) atomicAdd(rh + b, v);
    }
  }
}

// ---- dense prefix scoring (gather == nullptr) ------------------------------
// A query's whole prefix against all its scoring heads, the same dense
// product over contiguous tokens.  Persistent: a CTA builds Q' once, then
// walks chunks part, part + nparts, ... of its query's prefix (DT tiles of
// 128 tokens each), with chunks j + 1 .. j + NBUF - 1's key rows and scales
// in flight (coalesced 16-byte cp.async into a ring of NBUF shared-memory
// buffers) while chunk j is multiplied and drained; the grid holds the
// resident CTAs (two per SM for e4m3 keys).  Measured for 8 x 128K
// e4m3 keys and 64 heads: 45 us with two-tile chunks and two buffers, 63 us
// with one-tile chunks and three buffers (three CTAs per SM: the per-chunk
// barriers and MMA round trip weigh more).  One mbarrier
// phase per chunk; every wait is bounded, and after each wait the CTA agrees
// through a barrier whether to go on, so that a wait that ran out ends every
// thread's loop at the same chunk.
template <bool FP8, int HN>
struct DCfg {
  static constexpr int ROW = FP8 ? 128 : 256;
  static constexpr int CH = ROW / 16;                    // 16-byte chunks per key row
  static constexpr int DT = HN >= 128 ? 1 : 2;           // tiles per chunk
  static constexpr int NBUF = 2;                         // chunks staged (the current one + 1 ahead)
  static constexpr int CT = DT * RR_M;                   // tokens per chunk
  static constexpr int A_BYTES = RR_M * ROW;             // one tile of key rows
  static constexpr int CHUNK_BYTES = DT * A_BYTES;
  static constexpr int B_BYTES = HN * 256;
  static constexpr int TMEM_COLS = DT * HN < 32 ? 32 : DT * HN;
  static constexpr int SMEM = 1024 + NBUF * CHUNK_BYTES + B_BYTES;
  static_assert(DT * HN <= 256, "tensor-memory columns per CTA");
};

struct DenseShared {
  uint64_t done;
  uint32_t tmem_base;
  int abort;
  alignas(16) float w[128];        // weight per column (0: padding); read as float4
  float scale[2 * 2 * RR_M];       // the chunks' e4m3 token scales, CT per buffer
  uint32_t hist[TOPK_HIST_BINS];   // this CTA's share of the row histogram
};

template <bool FP8, int HN>
__global__ void __launch_bounds__(RR_THREADS) dense_umma_kernel(CacheView c, QueryView qv, const int32_t *heads, int h,
                                                                 float *scores, long long ld, uint32_t *row_hist,
                                                                 int nparts) {
  grid_dep_sync();
  using Cfg = DCfg<FP8, HN>;
  extern __shared__ uint8_t dn_raw[];
  uint8_t *base = dn_raw + ((1024u - (smem_addr(dn_raw) & 1023u)) & 1023u);  // 1024-aligned (swizzle atoms)
  static_assert(Cfg::NBUF * Cfg::CT <= 2 * 2 * RR_M, "the scale ring");
  uint8_t *a_smem = base;                             // NBUF x CHUNK_BYTES
  uint8_t *b_smem = base + Cfg::NBUF * Cfg::CHUNK_BYTES;  // B_BYTES
  __shared__ DenseShared sh;
  volatile int *abort = &sh.abort;
  const int i = blockIdx.y, part = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int s;
  const int Li = query_prefix(c, qv, i, &s);
  const int n_chunks = cdiv(max(Li, 0), Cfg::CT);
  const int n_my = part < n_chunks ? cdiv(n_chunks - part, nparts) : 0;
  if (n_my == 0) return;  // uniform: nothing allocated yet
  const uint8_t *kbase = static_cast<const uint8_t *>(c.keys) + (size_t)s * c.L_cap * Cfg::ROW;
  const float *sbase = FP8 ? c.scale + (size_t)s * c.L_cap : nullptr;

  // chunk j's key rows (zero-filled past the prefix) and scales into buffer
  // j % NBUF: consecutive threads take consecutive 16-byte pieces of the
  // chunk's contiguous rows.  Always one commit group per call.
  auto issue = [&](int j) {
    if (j < n_my) {
      const int t0 = (part + j * nparts) * Cfg::CT;
      uint8_t *a = a_smem + (j % Cfg::NBUF) * Cfg::CHUNK_BYTES;
      for (int x = tid; x < Cfg::CT * Cfg::CH; x += RR_THREADS) {
        const int rr = x / Cfg::CH, u = x % Cfg::CH;
        const int tile = rr / RR_M, r = rr % RR_M, t = t0 + rr;
        const uint32_t dst =
            smem_addr(a + tile * Cfg::A_BYTES + (u >> 3) * (RR_M * 128) + r * 128 + (((u & 7) ^ (r & 7)) << 4));
        cp_async16(dst, kbase + (size_t)min(t, Li - 1) * Cfg::ROW + 16 * u, t < Li);
      }
      if (FP8)
        for (int e = tid; e < Cfg::CT; e += RR_THREADS) {
          const int t = t0 + e;
          cp_async4(smem_addr(&sh.scale[(j % Cfg::NBUF) * Cfg::CT + e]), sbase + min(t, Li - 1), t < Li);
        }
    }
    cp_async_commit();
  };

#pragma unroll
  for (int j = 0; j < Cfg::NBUF - 1; ++j) issue(j);
  build_qprime<FP8, HN>(c, qv, heads, h, i, b_smem, sh.w);
  for (int b = tid; b < TOPK_HIST_BINS; b += RR_THREADS) sh.hist[b] = 0;
  if (tid == 0) {
    mbar_init(&sh.done, 1);
    sh.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&sh.tmem_base)),
                 "n"(Cfg::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  umma::fence_before();
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = sh.tmem_base;
  const uint32_t idesc = umma::instr_desc<FP8, RR_M, HN>();
  uint32_t committed = 0, waited = 0;  // thread 0: chunks whose MMAs it committed / saw complete

  for (int j = 0; j < n_my; ++j) {
    issue(j + Cfg::NBUF - 1);                                       // into chunk j - 1's buffer
    cp_async_wait<Cfg::NBUF - 1>();                                 // chunk j: this thread's copies landed
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // ... and Q': visible to the tensor cores
    umma::fence_before();
    __syncthreads();
    umma::fence_after();
    const int t0 = (part + j * nparts) * Cfg::CT;
    const int ntile = min(Cfg::DT, cdiv(Li - t0, RR_M));
    // this thread's token scales of the chunk, read before the barrier after
    // which a thread may refill this buffer with chunk j + NBUF
    const int r = warp * 32 + lane;
    float scl[Cfg::DT];
#pragma unroll
    for (int tt = 0; tt < Cfg::DT; ++tt) scl[tt] = FP8 ? sh.scale[(j % Cfg::NBUF) * Cfg::CT + tt * RR_M + r] : 1.f;
    if (tid == 0) {
      const uint32_t a0 = smem_addr(a_smem + (j % Cfg::NBUF) * Cfg::CHUNK_BYTES), b_base = smem_addr(b_smem);
      for (int tt = 0; tt < ntile; ++tt) {
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
            umma::mma<FP8>(tmem + tt * HN, umma::smem_desc_sw128(a0 + tt * Cfg::A_BYTES + aoff),
                           umma::smem_desc_sw128(b_base + boff), idesc, (term | kk) ? 1u : 0u);
          }
        }
      }
      umma::commit(&sh.done);
      ++committed;
    }
    if (umma::wait_bar(&sh.done, (uint32_t)(j & 1), abort, c) && tid == 0) ++waited;
    __syncthreads();  // one view of *abort in every thread
    if (*abort) break;
    umma::fence_after();
    // epilogue: row r = 32 * warp + lane of every tile of the chunk
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    const float4 *w4 = reinterpret_cast<const float4 *>(sh.w);
#pragma unroll
    for (int tt = 0; tt < Cfg::DT; ++tt) {
      if (tt >= ntile) break;
      float acc = 0.f;
#pragma unroll
      for (int cb = 0; cb < HN; cb += 32) {
        uint32_t v[32];
        umma::ld32(tl + tt * HN + cb, v);
        umma::ld_wait();
#pragma unroll
        for (int x = 0; x < 32; x += 4) {
          const float4 w = w4[(cb + x) >> 2];
          acc = fmaf(w.x, fmaxf(__uint_as_float(v[x]), 0.f), acc);
          acc = fmaf(w.y, fmaxf(__uint_as_float(v[x + 1]), 0.f), acc);
          acc = fmaf(w.z, fmaxf(__uint_as_float(v[x + 2]), 0.f), acc);
          acc = fmaf(w.w, fmaxf(__uint_as_float(v[x + 3]), 0.f), acc);
        }
      }
      const int e = tt * RR_M + r, t = t0 + e;
      if (t < Li) {
        const float val = acc * scl[tt];
        scores[(size_t)i * ld + t] = val;
        atomicAdd(&sh.hist[ordered_key(val) >> 21], 1u);
      }
    }
  }

  // wind-down: no copy and no MMA in flight when the memory is released
  cp_async_wait<0>();
  if (tid == 0 && committed > waited) mbar_wait(&sh.done, (committed - 1) & 1);  // bounded
  umma::fence_before();
  __syncthreads();
  if (warp == 0) {
    umma::fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(Cfg::TMEM_COLS));
  }
  if (!*abort) {
    uint32_t *rh = row_hist + (size_t)i * TOPK_HIST_BINS;
    for (int b = tid; b < TOPK_HIST_BINS; b += RR_THREADS) {
      const uint32_t v = sh.hist[b];
      if (v) atomicAdd(rh + b, v);
    }
  }
}

template <bool FP8, int HN>
cudaError_t launch_dense(const CacheView &c, const QueryView &q, const int32_t *heads, int h, float *scores,
                         long long ld, uint32_t *row_hist, cudaStream_t s) {
  using Cfg = DCfg<FP8, HN>;
  struct Tag {};
  const int st = cached_per_device<Tag>([] {
    cudaError_t e = cudaFuncSetAttribute(dense_umma_kernel<FP8, HN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg::SMEM);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(dense_umma_kernel<FP8, HN>, cudaFuncAttributePreferredSharedMemoryCarveout,
                               (int)cudaSharedmemCarveoutMaxShared);
    return 1 + (int)e;
  });
  if (st != 1) return (cudaError_t)(st - 1);
  // the resident CTAs over all rows, each walking several chunks: two per SM
  // when two fit in the SM's 228 KB of shared memory (e4m3 keys: at most
  // 94 KB each at every head count), else one.  (The runtime's occupancy
  // query answered one per SM for e4m3 at 64 heads, and a grid sized from it
  // took 54 us instead of 45.)
  constexpr int per_sm = 2 * (Cfg::SMEM + (int)sizeof(DenseShared) + 1024) <= 228 * 1024 ? 2 : 1;
  const int nparts = std::max(1, std::min(cdiv(c.L_cap, Cfg::CT), per_sm * device_sms() / q.n_q));
  return launch_kernel(dense_umma_kernel<FP8, HN>, dim3(nparts, q.n_q), dim3(RR_THREADS), Cfg::SMEM, s, c, q, heads,
                       h, scores, ld, row_hist, nparts);
}

template <bool FP8, int HN, int TT>
cudaError_t launch_tt(const CacheView &c, const QueryView &q, const int32_t *heads, int h, const int32_t *gather,
                      int n_cols, float *scores, long long ld, uint32_t *row_hist, cudaStream_t s) {
  using Cfg = RCfg<FP8, HN, TT>;
  struct Tag {};
  const int st = cached_per_device<Tag>([] {
    return 1 + (int)cudaFuncSetAttribute(rerank_umma_kernel<FP8, HN, TT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
  });
  if (st != 1) return (cudaError_t)(st - 1);
  const dim3 grid(cdiv(n_cols, Cfg::T * RR_M), q.n_q);
  return launch_kernel(rerank_umma_kernel<FP8, HN, TT>, grid, dim3(RR_THREADS), Cfg::SMEM, s, c, q, heads, h, gather,
                       n_cols, scores, ld, row_hist);
}

// Gathered candidates: 2 tiles per CTA (more CTAs shorten each gather chain);
// a prefix row: the persistent dense kernel.
template <bool FP8, int HN>
cudaError_t launch_hn(const CacheView &c, const QueryView &q, const int32_t *heads, int h, const int32_t *gather,
                      int n_cols, float *scores, long long ld, uint32_t *row_hist, cudaStream_t s) {
  return gather ? launch_tt<FP8, HN, 2>(c, q, heads, h, gather, n_cols, scores, ld, row_hist, s)
                : launch_dense<FP8, HN>(c, q, heads, h, scores, ld, row_hist, s);
}

}  // namespace

bool rerank_umma_applies(const QueryView &q, const int32_t *heads, int h) {
  const int h_eff = heads ? h : q.H;
  return h_eff >= 1 && h_eff <= 128;
}

cudaError_t launch_rerank_umma(const CacheView &c, const QueryView &q, const int32_t *heads, int h,
                               const int32_t *gather, int n_cols, float *scores, long long ld, uint32_t *row_hist,
                               cudaStream_t s) {
  if (q.n_q == 0 || n_cols == 0) return cudaSuccess;
  const int h_eff = heads ? h : q.H;
  const int hn = h_eff <= 32 ? 32 : h_eff <= 64 ? 64 : 128;
#define MISA_RERANK_CASE(N)                                                                        \
  case N:                                                                                          \
    return c.fp8 ? launch_hn<true, N>(c, q, heads, h, gather, n_cols, scores, ld, row_hist, s)     \
                 : launch_hn<false, N>(c, q, heads, h, gather, n_cols, scores, ld, row_hist, s);
  switch (hn) {
    MISA_RERANK_CASE(32)
    MISA_RERANK_CASE(64)
    MISA_RERANK_CASE(128)
    default:
      return cudaErrorInvalidValue;
  }
#undef MISA_RERANK_CASE
}

}  // namespace misa
