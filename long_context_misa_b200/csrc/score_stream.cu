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
#include <algorithm>

#include "frag.cuh"
#include "internal.h"
#include "route_slice.cuh"
#include "rowsel.cuh"

namespace misa {
namespace {

constexpr int WARPS = 8;
constexpr int THREADS = 32 * WARPS;
static_assert(MISA_MAX_H <= THREADS, "one thread per head in the router");

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
// fz.zeroed != nullptr: the row's top fz.k are selected here (rowsel.cuh)
// instead of the histogram going to row_hist; every scored element also stays
// in shared memory, [warp][max_tiles][TT] after the ring.
// route_part != nullptr (with fz): the query's h scoring heads are routed
// here first (route_slice.cuh; heads is ignored): this CTA's partial router
// sums go to route_part[i][blockIdx.x][H], the row's CTAs meet, and every one
// ranks the heads from all the partials; CTA 0 of the row writes them to
// heads_out[i][h] when it is not null.
template <int NT, bool FP8>
__global__ void __launch_bounds__(THREADS) score_stream_kernel(CacheView c, QueryView qv, const int32_t *heads,
                                                               int h, float *scores, long long ld, int scale_vec,
                                                               uint32_t *row_hist, FusedTopk fz, int max_tiles,
                                                               int region, float *route_part, int32_t *heads_out,
                                                               PendingAppend pa) {
  // an append kernel still running ahead (pa.pos): the router runs before
  // the wait on it (below); otherwise the wait comes first
  grid_dep_sync_unless(route_part != nullptr && pa.pos != nullptr);
  const bool early = route_part != nullptr && pa.pos != nullptr;
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
  const int Li = early ? query_prefix_appended(c, qv, i, &s, pa.pos, pa.count) : query_prefix(c, qv, i, &s);
  const int ntile_all = cdiv(Li, TT);
  const int nwarps = gridDim.x * WARPS;
  const int wg = blockIdx.x * WARPS + warp;  // this warp takes tiles wg, wg + nwarps, ...
  const int my_tiles = wg < ntile_all ? cdiv(ntile_all - wg, nwarps) : 0;
  const uint32_t ring = smem_addr(smem) + warp * Cfg::WARP_BYTES;
  const bool fused = fz.zeroed != nullptr;
  float *sc_s = reinterpret_cast<float *>(smem + region);  // fused: this CTA's scores
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
  // routing in front of the scan
  __shared__ float r_tail[D];                   // the causal tail block's mean
  __shared__ float r_wsum[WARPS * MISA_MAX_H];  // per-warp partial sums
  __shared__ float r_out[MISA_MAX_H];           // this CTA's partials, then the importances
  __shared__ float r_w[MISA_MAX_H];             // the query's head weights
  __shared__ int r_keep[MISA_MAX_H];
  __shared__ int32_t r_heads[NT * 8];
  __shared__ struct { int ok; } r_bar;
  const bool route = route_part != nullptr;
  // with routing, the query's H rows wait in the ring's last stage (unused
  // until the scan starts), RPW rows per warp; the host checks H <= WARPS * RPW
  constexpr int RPW = Cfg::STAGE / (2 * D);
  const uint32_t q_stage = smem_addr(smem) + (NS - 1) * Cfg::STAGE;
  auto qrow_s = [&](int j) -> const uint16_t * {
    return reinterpret_cast<const uint16_t *>(smem + (j / RPW) * Cfg::WARP_BYTES + (NS - 1) * Cfg::STAGE +
                                              (j % RPW) * 2 * D);
  };
  if (!route) {
#pragma unroll
    for (int j = 0; j < NS - 1; ++j) issue(j);  // start streaming before the query set-up
  } else {
    // the router's loads go first: the query rows and weights here, this
    // CTA's pool blocks inside route_slice; the ring's first tiles follow
    for (int x = tid; x < qv.H * 16; x += THREADS) {
      const int j = x >> 4, u = x & 15;
      cp_async16(q_stage + (j / RPW) * Cfg::WARP_BYTES + (j % RPW) * 2 * D + 16 * u,
                 qv.q + ((size_t)i * qv.H + j) * D + 8 * u);
    }
    cp_async_commit();
    // the weights land in registers meanwhile (H <= MISA_MAX_H <= THREADS)
    const float w_mine = tid < qv.H ? __ldg(qv.w + (size_t)i * qv.H + tid) : 0.f;
    const int Mi = cdiv(Li, c.B), full = Li / c.B, C = gridDim.x;
    const int m0 = (int)((long long)blockIdx.x * Mi / C), m1 = (int)((long long)(blockIdx.x + 1) * Mi / C);
    // Early: nothing the append writes is read before the wait.  Its tokens
    // in the cut block come from its input rows (the same bytes), and a CTA
    // whose pool blocks it rewrites waits first; the ring and every counter
    // wait too.  All of it uniform over the CTA.
    KeySource ks;
    bool waited = !early;
    if (early) {
      const int ap = pa.pos[s];
      if (ap >= 0 && (long long)ap + pa.count <= c.L_cap) {  // the append takes this sequence
        ks.ovr_keys = static_cast<const uint8_t *>(pa.keys) + (size_t)s * pa.count * ROW;
        ks.ovr_scale = FP8 ? pa.scale + (size_t)s * pa.count : nullptr;
        ks.ovr_t0 = ap;
        ks.ovr_n = pa.count;
        if (ap / c.B < min(m1, full) && (ap + pa.count - 1) / c.B >= m0) {
          grid_dep_sync();
          waited = true;
        }
      }
    }
    if (full < Mi && full >= m0 && full < m1) {  // uniform: this CTA holds the block cut by the prefix end
      block_key_sum<128>(c, s, full * c.B, Li, reinterpret_cast<float *>(shist), r_tail, ks);
      if (tid < D) r_tail[tid] *= 1.f / (float)(Li - full * c.B);
      __syncthreads();
    }
    route_slice<WARPS>(c, s, qv.H, m0, m1, full, r_tail, r_wsum, r_out, qrow_s, [&] {
      if (waited) {
#pragma unroll
        for (int j = 0; j < NS - 1; ++j) issue(j);
      }
      if (tid < qv.H) r_w[tid] = w_mine;
      if (waited)
        cp_async_wait<NS - 1>();  // the query rows (the group before the ring's)
      else
        cp_async_wait<0>();  // the query rows (the only group yet)
      __syncthreads();
    });
    if (!waited) {
      grid_dep_sync();  // the append is complete: its keys, block means and cleared words are visible
#pragma unroll
      for (int j = 0; j < NS - 1; ++j) issue(j);
    }
    float *prow = route_part + (size_t)i * C * qv.H;
    for (int j = tid; j < qv.H; j += THREADS) prow[(size_t)blockIdx.x * qv.H + j] = r_out[j];
    if (!row_barrier(r_bar, fz.zeroed + (size_t)i * RS_ZERO_WORDS + 2 * RB + RS_ROUTE, (uint32_t)C, c)) {
      cp_async_wait<0>();  // no copy in flight when the CTA leaves
      return;
    }
    // the partials are staged in the scores' region (not yet in use), when it holds them
    route_rank(qv.H, r_w, prow, C, h, r_out, r_keep, r_heads, sc_s, fused ? WARPS * max_tiles * TT : 0);
    if (blockIdx.x == 0 && heads_out)
      for (int n = tid; n < h; n += THREADS) heads_out[(size_t)i * h + n] = r_heads[n];
  }
  for (int b = tid; b < TOPK_HIST_BINS; b += THREADS) shist[b] = 0;

  if (route)
    build_query_frags<NT, FP8, THREADS>(c, qv, i, heads, h, bfrag, w_s, scale_s, tid, [] { __syncthreads(); },
                                        r_heads, QSmem<decltype(qrow_s)>{qrow_s, r_w});
  else
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
        if (fused) sc_s[(warp * max_tiles + j) * TT + 16 * m + g + 8 * me] = v;
        atomicAdd(&shist[ordered_key(v) >> 21], 1u);
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();
  if (fused) {
    // the ring is free: the selection's shared state and scratch go there
    RsShared<THREADS> &rs = *reinterpret_cast<RsShared<THREADS> *>(smem);
    uint8_t *scratch = smem + (sizeof(RsShared<THREADS>) + 15) / 16 * 16;
    // every warp visits the elements of its own tiles (token t0 + r of its
    // j-th tile at [warp][j][r]); trip counts are uniform within the warp
    const float *sc_w = sc_s + warp * max_tiles * TT;
    const int n_el = my_tiles * TT;
    auto each = [&](auto &&fn) {
      for (int x = lane; x < (n_el + 31) / 32 * 32; x += 32) {
        const int j = x / TT, r = x % TT;
        const int tok = (wg + j * nwarps) * TT + r;
        const bool valid = x < n_el && tok < Li;
        fn(valid ? ordered_key(sc_w[x]) : 0u, tok, valid);
      }
    };
    const float *srow = scores + (size_t)i * ld;
    auto sweep = [&](auto &&fn) {
      constexpr int SU = 8;
      for (int base = 0; base < Li; base += THREADS * SU) {
        float v[SU];
#pragma unroll
        for (int u = 0; u < SU; ++u) {
          const int p = base + u * THREADS + tid;
          v[u] = p < Li ? __ldcg(srow + p) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < SU; ++u) {
          const int p = base + u * THREADS + tid;
          fn(ordered_key(v[u]), POS_MAX - (uint32_t)p, p < Li);
        }
      }
    };
    row_select<THREADS>(c, rs, shist, scratch, rs_row(fz, i), gridDim.x, fz.k, Li, fz.ordered != 0,
                        WARPS * max_tiles * TT, each, sweep);
    return;
  }
  uint32_t *rh = row_hist + (size_t)i * TOPK_HIST_BINS;
  for (int b = tid; b < TOPK_HIST_BINS; b += THREADS) {
    const uint32_t v = shist[b];
    if (v) atomicAdd(rh + b, v);
  }
}

// Launch shape of one scoring call: splits CTAs per query (one wave of the
// resident CTAs), dynamic shared memory, and -- for a fused selection -- the
// tiles a warp scores at most and where its scores start.
struct StreamPlan {
  int splits = 0, smem = 0, max_tiles = 0, region = 0;
  bool ok = false;
};

// reserve: CTA slots left to the blocks of a kernel running alongside (an
// append kernel that triggered this launch early: one slot per block).
template <int NT, bool FP8>
StreamPlan plan_nt(const CacheView &c, const QueryView &q, bool fused, int reserve = 0) {
  using Cfg = StreamCfg<NT, FP8>;
  constexpr int RING = WARPS * Cfg::WARP_BYTES;
  StreamPlan p;
  const int sms = device_sms();
  // the largest dynamic shared memory any launch may ask for (also the opt-in)
  struct Tag {};
  const int max_dyn = cached_per_device<Tag>([] { return opt_in_max_dyn_smem(score_stream_kernel<NT, FP8>); });
  if (max_dyn < RING) return p;
  auto per_sm_for = [&](int smem) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, score_stream_kernel<NT, FP8>, THREADS, smem) != cudaSuccess)
      return 0;
    return n;
  };
  const int ntile = cdiv(c.L_cap, Cfg::TT);
  auto splits_for = [&](int per_sm) {
    // one wave: a CTA beyond the resident slots would double the kernel time
    int sp = std::max(1, (per_sm * sms - reserve) / std::max(q.n_q, 1));
    return std::min(sp, std::max(1, cdiv(ntile, 2 * WARPS)));  // >= 2 tiles per warp
  };
  if (!fused) {
    struct TagR {};
    const int per_sm = cached_per_device<TagR>([&] { return std::max(per_sm_for(RING), 1); });
    p.splits = splits_for(per_sm);
    p.smem = RING;
    p.ok = true;
    return p;
  }
  // fused: the ring (reused for the selection afterwards) and the scores
  int per_sm = per_sm_for(RING);
  for (int it = 0; it < 3 && per_sm > 0; ++it) {
    const int sp = splits_for(per_sm);
    const int mt = cdiv(ntile, sp * WARPS);
    const int sel = (int)((sizeof(RsShared<THREADS>) + 15) / 16 * 16) + rs_scratch_bytes(c.L_cap, WARPS * mt * Cfg::TT, THREADS);
    const int region = (std::max(RING, sel) + 127) / 128 * 128;
    const int smem = region + WARPS * mt * Cfg::TT * 4;
    const int fit = smem <= max_dyn ? per_sm_for(smem) : 0;
    if (fit >= per_sm) {  // the grid is resident at once
      if ((long long)sp * q.n_q > (long long)fit * sms) return p;
      p.splits = sp;
      p.smem = smem;
      p.max_tiles = mt;
      p.region = region;
      p.ok = true;
      return p;
    }
    per_sm = fit;  // fewer CTAs per SM: fewer splits, more tiles each
  }
  return p;
}

// With routing in the kernel the query's rows are staged in the ring's last
// stage: RPW rows of 2 * D bytes per warp.
template <int NT, bool FP8>
constexpr int route_q_rows() {
  return WARPS * (StreamCfg<NT, FP8>::STAGE / (2 * D));
}

template <int NT, bool FP8>
cudaError_t launch_nt(const CacheView &c, const QueryView &q, const int32_t *heads, int h, float *scores,
                      long long ld, uint32_t *row_hist, cudaStream_t s, const FusedTopk *fz, float *route_part,
                      int32_t *heads_out, const PendingAppend *pending) {
  const PendingAppend pa = route_part && pending ? *pending : PendingAppend();
  const StreamPlan p = plan_nt<NT, FP8>(c, q, fz != nullptr, pa.pos ? c.n_seq : 0);
  if (!p.ok) return cudaErrorInvalidConfiguration;
  if (route_part && (!fz || (long long)p.splits * q.n_q > route_part_slots() || q.H > route_q_rows<NT, FP8>()))
    return cudaErrorInvalidValue;
  const int scale_vec = FP8 && (reinterpret_cast<uintptr_t>(c.scale) & 15) == 0 && c.L_cap % 4 == 0;
  FusedTopk none = {};
  return launch_kernel(score_stream_kernel<NT, FP8>, dim3(p.splits, q.n_q), dim3(THREADS), p.smem, s, c, q, heads, h,
                       scores, ld, scale_vec, row_hist, fz ? *fz : none, p.max_tiles, p.region, route_part,
                       heads_out, pa);
}

int stream_nt_h(int h_eff) {
  int NT = 1;
  while (NT * 8 < h_eff) NT *= 2;
  return NT;
}

int stream_nt(const QueryView &q, const int32_t *heads, int h) { return stream_nt_h(heads ? h : q.H); }

}  // namespace

cudaError_t launch_score_stream(const CacheView &c, const QueryView &q, const int32_t *heads, int h, float *scores,
                                long long ld, uint32_t *row_hist, cudaStream_t s, const FusedTopk *fused,
                                float *route_part, int32_t *heads_out, const PendingAppend *pending) {
  if (q.n_q == 0) return cudaSuccess;
#define MISA_STREAM_CASE(N)                                                                                      \
  case N:                                                                                                        \
    return c.fp8 ? launch_nt<N, true>(c, q, heads, h, scores, ld, row_hist, s, fused, route_part, heads_out,     \
                                      pending)                                                                   \
                 : launch_nt<N, false>(c, q, heads, h, scores, ld, row_hist, s, fused, route_part, heads_out,    \
                                       pending);
  switch (route_part ? stream_nt_h(h) : stream_nt(q, heads, h)) {
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

bool score_stream_fusable(const CacheView &c, const QueryView &q, const int32_t *heads, int h, bool route) {
  if (q.n_q == 0) return false;
#define MISA_STREAM_CASE(N)                                                                     \
  case N: {                                                                                     \
    const StreamPlan p = c.fp8 ? plan_nt<N, true>(c, q, true) : plan_nt<N, false>(c, q, true); \
    const int rows = c.fp8 ? route_q_rows<N, true>() : route_q_rows<N, false>();                \
    return p.ok && (!route || ((long long)p.splits * q.n_q <= route_part_slots() && q.H <= rows)); \
  }
  switch (route ? stream_nt_h(h) : stream_nt(q, heads, h)) {
    MISA_STREAM_CASE(1)
    MISA_STREAM_CASE(2)
    MISA_STREAM_CASE(4)
    MISA_STREAM_CASE(8)
    MISA_STREAM_CASE(16)
    default:
      return false;
  }
#undef MISA_STREAM_CASE
}

}  // namespace misa
