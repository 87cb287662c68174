// Token scoring of one query's causal prefix (decode shape: one key stream
// per query, bound by the key read).
//
// Computes I_t = s_t * sum_{n < h} w_{i,S_n} * ReLU(q_{i,S_n} . k_t) for every
// prefix token t of query i ("MISA: Mixture of Indexer Sparse Attention for
// Long-Context LLM Inference", technical summary, "Methodology: MISA" step 2
// with the routed heads S; "Problem statement" with S = all H_I heads).
//
// Streaming: every warp owns a private 2-3 stage ring of key tiles (4 KB: 32
// e4m3 or 16 bf16 tokens) in shared memory, filled with cp.async (16 bytes per lane, each warp
// instruction one contiguous 512-byte span, so every request is whole L2
// lines) and drained with cp.async.wait_group -- no cross-warp barrier in the
// main loop.  Tiles are dealt round-robin over all warps of all CTAs working
// on a query, so the requests in flight at any moment cover adjacent
// addresses.  Within a tile, 16-byte unit u of row r is stored at unit
// u ^ 4*(r & 1), which lets the fragment loads below hit 32 distinct banks.
// (On this part a one-thread cp.async.bulk ring peaked near 4.4 TB/s for
// this stream and plain 16-byte loads near 5.2 TB/s, hence this design.)
//
// Compute: lane (g, c) reads units c and c+4 (e4m3) or c, c+4, c+8, c+12
// (bf16) of rows g and g+8 of each 16-token half, which feed mma.sync A
// fragments directly
// (frag.cuh: bf16 keys on the bf16 MMA; e4m3 keys on the e4m3 MMA against an
// exact two-term e4m3 split of the query, so keys are never widened).  ReLU,
// the w-weighting and the reduction over heads run on the accumulators; the
// per-head products never leave the SM.  s_t > 0 multiplies the reduced score.
// Up to 16 scoring heads keep their query fragments in registers.
#include "frag.cuh"
#include "internal.h"

namespace misa {
namespace {

constexpr int WARPS = 8;
constexpr int THREADS = 32 * WARPS;

template <int NT, bool FP8>
struct StreamCfg {
  static constexpr int ROW = FragCfg<FP8>::ROW;        // bytes per key row
  static constexpr int TT = (FP8 && NT <= 2) ? 32 : 16; // tokens per tile (1 or 2 MMA M sides)
  static constexpr int TILE = TT * ROW;                 // 4 KB, or 2 KB for e4m3 with many heads
  static constexpr int NS = FP8 ? 2 : 3;                // stages per warp (2 measured fastest for e4m3)
  static constexpr int SCALE = FP8 ? TT * 4 : 0;        // the tile's scales
  static constexpr int STAGE = TILE + SCALE;
  static constexpr int WARP_BYTES = NS * STAGE;
  static constexpr int COPIES = TILE / 512;             // 16-byte cp.async per lane per tile
};


// scale_vec: the per-token scales may be copied 4 at a time (16-byte aligned
// groups inside the cache); otherwise they are read one by one.
template <int NT, bool FP8>
__global__ void __launch_bounds__(THREADS) score_stream_kernel(CacheView c, QueryView qv, const int32_t *heads,
                                                               int h, float *scores, long long ld, int scale_vec,
                                                               uint32_t *row_hist) {
  grid_dep_sync();
  using Cfg = StreamCfg<NT, FP8>;
  using F = FragCfg<FP8>;
  constexpr int NS = Cfg::NS, ROW = Cfg::ROW, NV = F::NV, TT = Cfg::TT;
  constexpr int UNITS = ROW / 16;         // 16-byte units per row
  constexpr int RPC = 32 / UNITS;         // rows covered by one warp-wide copy
  constexpr bool BREG = NT <= 2;          // query fragments held in registers
  constexpr int NB = F::KT * F::TERMS * NT;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint2 bfrag[NB * 32];
  __shared__ float w_s[NT * 8], scale_s[NT * 8];
  __shared__ uint32_t shist[TOPK_HIST_BINS];  // this CTA's share of the row histogram

  const int i = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, cq = lane & 3;
  int s;
  const int Li = query_prefix(c, qv, i, &s);
  const int ntile_all = cdiv(Li, TT);
  const int nwarps = gridDim.x * WARPS;
  const int wg = blockIdx.x * WARPS + warp;  // this warp takes tiles wg, wg + nwarps, ...
  const int my_tiles = wg < ntile_all ? cdiv(ntile_all - wg, nwarps) : 0;
  const uint32_t ring = smem_addr(smem) + warp * Cfg::WARP_BYTES;
  const uint8_t *gkeys = static_cast<const uint8_t *>(c.keys) + (size_t)s * c.L_cap * ROW;
  const float *gscale = FP8 ? c.scale + (size_t)s * c.L_cap : nullptr;

  // Copy k of a tile moves rows RPC*k + lane/UNITS, unit lane%UNITS; the
  // destination unit is XOR-swizzled by the row parity (which only depends
  // on the lane, RPC being even).
  const int c_row = lane / UNITS, c_unit = lane % UNITS;
  const uint32_t c_dst = c_row * ROW + 16 * (c_unit ^ ((c_row & 1) << 2));
  const uint8_t *c_src = gkeys + c_row * ROW + 16 * c_unit;

  auto issue = [&](int j) {  // always one commit group per call
    if (j < my_tiles) {
      const int t0 = (wg + j * nwarps) * TT;
      const uint32_t st = ring + (j % NS) * Cfg::STAGE;
      const uint8_t *src = c_src + (size_t)t0 * ROW;
      if (t0 + TT <= Li) {
#pragma unroll
        for (int k = 0; k < Cfg::COPIES; ++k) cp_async16(st + c_dst + 512 * k, src + 512 * k);
      } else {
#pragma unroll
        for (int k = 0; k < Cfg::COPIES; ++k) {
          const bool ok = t0 + RPC * k + c_row < Li;
          cp_async16(st + c_dst + 512 * k, ok ? src + 512 * k : gkeys, ok);
        }
      }
      if (FP8 && lane < TT / 4) {
        const int tg = t0 + 4 * lane;
        const bool ok = scale_vec && tg + 4 <= c.L_cap;
        cp_async16(st + Cfg::TILE + 16 * lane, ok ? gscale + tg : gscale, ok);
      }
    }
    cp_async_commit();
  };
#pragma unroll
  for (int j = 0; j < NS - 1; ++j) issue(j);  // start streaming before the query set-up
  for (int b = tid; b < TOPK_HIST_BINS; b += THREADS) shist[b] = 0;

  build_query_frags<NT, FP8, THREADS>(c, qv, i, heads, h, bfrag, w_s, scale_s, tid, [] { __syncthreads(); });
  __syncthreads();
  float wr[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    wr[nt][0] = w_s[nt * 8 + 2 * cq];
    wr[nt][1] = w_s[nt * 8 + 2 * cq + 1];
  }
  uint2 breg[BREG ? NB : 1];
  if constexpr (BREG) {
#pragma unroll
    for (int e = 0; e < NB; ++e) breg[e] = bfrag[e * 32 + lane];
  }

  const int swz = (g & 1) << 2;  // rows g and g + 8 share the parity of g
  const int me = cq & 1;         // lanes cq = 0 / 1 write rows g / g + 8 of a sub-tile
  for (int j = 0; j < my_tiles; ++j) {
    issue(j + NS - 1);
    cp_async_wait<NS - 1>();  // tile j has landed (this lane's copies)
    __syncwarp();             // ... and every other lane's
    const int t0 = (wg + j * nwarps) * TT;
    const uint8_t *st = smem + (ring - smem_addr(smem)) + (j % NS) * Cfg::STAGE;
    uint4 kv[TT / 16][2][NV];
    float sc[TT / 16];
#pragma unroll
    for (int m = 0; m < TT / 16; ++m) {
      const uint8_t *rowA = st + (16 * m + g) * ROW, *rowB = rowA + 8 * ROW;
#pragma unroll
      for (int ch = 0; ch < NV; ++ch) {
        const int u = (cq + 4 * ch) ^ swz;
        kv[m][0][ch] = *reinterpret_cast<const uint4 *>(rowA + 16 * u);
        kv[m][1][ch] = *reinterpret_cast<const uint4 *>(rowB + 16 * u);
      }
      sc[m] = 1.f;
      if (FP8) {
        const int row = 16 * m + g + 8 * me, trow = t0 + row;
        const bool in_smem = scale_vec && t0 + (row & ~3) + 4 <= c.L_cap;
        if (in_smem)
          sc[m] = reinterpret_cast<const float *>(st + Cfg::TILE)[row];
        else if (cq < 2 && trow < Li)
          sc[m] = __ldg(gscale + trow);
      }
    }
    __syncwarp();  // every lane has read the stage before it is refilled
#pragma unroll
    for (int m = 0; m < TT / 16; ++m) {
      float acc[NT][4];
      if constexpr (BREG)
        tile_mma_reg<NT, FP8>(kv[m], breg, acc);
      else
        tile_mma<NT, FP8>(kv[m], bfrag, lane, acc);
      const float2 sums = tile_reduce<NT>(acc, wr);
      const int trow = t0 + 16 * m + g + 8 * me;
      if (cq < 2 && trow < Li) {
        const float v = (me ? sums.y : sums.x) * sc[m];
        scores[(size_t)i * ld + trow] = v;
        atomicAdd(&shist[ordered_key(v) >> 21], 1u);
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();
  uint32_t *rh = row_hist + (size_t)i * TOPK_HIST_BINS;
  for (int b = tid; b < TOPK_HIST_BINS; b += THREADS) {
    const uint32_t v = shist[b];
    if (v) atomicAdd(rh + b, v);
  }
}

template <int NT, bool FP8>
cudaError_t launch_nt(const CacheView &c, const QueryView &q, const int32_t *heads, int h, float *scores,
                      long long ld, uint32_t *row_hist, cudaStream_t s) {
  constexpr int SMEM = WARPS * StreamCfg<NT, FP8>::WARP_BYTES;
  const int sms = device_sms();
  // resident CTAs per SM (also sets the shared-memory opt-in), once per device
  struct Tag {};
  const int per_sm = cached_per_device<Tag>([] {
    if (cudaFuncSetAttribute(score_stream_kernel<NT, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) !=
        cudaSuccess)
      return -1;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, score_stream_kernel<NT, FP8>, THREADS, SMEM) !=
        cudaSuccess)
      return -1;
    return max(n, 1);
  });
  if (per_sm < 0) return cudaErrorInvalidConfiguration;
  // one wave: a CTA beyond the resident slots would double the kernel time
  int splits = max(1, per_sm * sms / q.n_q);
  splits = min(splits, max(1, cdiv(cdiv(c.L_cap, StreamCfg<NT, FP8>::TT), 2 * WARPS)));  // >= 2 tiles per warp
  const int scale_vec = FP8 && (reinterpret_cast<uintptr_t>(c.scale) & 15) == 0 && c.L_cap % 4 == 0;
  return launch_kernel(score_stream_kernel<NT, FP8>, dim3(splits, q.n_q), dim3(THREADS), SMEM, s, c, q, heads, h, scores,
                    ld, scale_vec, row_hist);
}

}  // namespace

cudaError_t launch_score_stream(const CacheView &c, const QueryView &q, const int32_t *heads, int h, float *scores,
                                long long ld, uint32_t *row_hist, cudaStream_t s) {
  if (q.n_q == 0) return cudaSuccess;
  const int h_eff = heads ? h : q.H;
  int NT = 1;
  while (NT * 8 < h_eff) NT *= 2;
#define MISA_STREAM_CASE(N)                                                   \
  case N:                                                                     \
    return c.fp8 ? launch_nt<N, true>(c, q, heads, h, scores, ld, row_hist, s) \
                 : launch_nt<N, false>(c, q, heads, h, scores, ld, row_hist, s);
  switch (NT) {
    MISA_STREAM_CASE(1)
    MISA_STREAM_CASE(2)
    MISA_STREAM_CASE(4)
    MISA_STREAM_CASE(8)
    MISA_STREAM_CASE(16)
    default:
      return cudaErrorInvalidValue;
  }
#undef MISA_STREAM_CASE
}

}  // namespace misa
