// The block-pooled router computed by the CTAs that then score the query's
// prefix (decode, routing fused into the scoring kernel).
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference",
// technical summary, "Methodology: MISA", step 1: per-head affinities against
// the mean-pooled index keys, aggregated into an importance per head, top-h
// heads kept:
//     r_j = |w_j| * sum_{m < M_i} ReLU(q_j . kbar_m),   M_i = ceil(L_i / B),
// the block cut by the prefix end averaged over its tokens up to the query.
//
// Each of the C CTAs of a query takes a contiguous slice of its M_i blocks
// and sums ReLU(q_j . kbar_m) over the slice for every head j (route_slice);
// the C partial sums meet in global memory, and after a row barrier every CTA
// adds them in the same order and ranks the heads (route_rank), so all CTAs of
// the query agree on its heads.
//
// route_slice runs on mma.sync m16n8k16 with the query heads on the M side
// (16 heads per m-tile, bf16 as stored) and 8 pooled blocks on the N side:
// each fp32 pooled key is split into bf16 hi = RN(k) and lo = RN(k - hi), both
// multiplied by the query, so the product keeps about 16 significant bits of
// the pooled key, with exact products and fp32 accumulation (the numerics of
// the separate decode router).  The K dimension is permuted the same way on
// both operands so that every lane's 16-byte loads feed whole fragments: lane
// (g, c) reads elements 32ch + 8c .. + 7 of its rows.
#pragma once

#include "keysum.cuh"

namespace misa {
namespace {

__device__ __forceinline__ uint32_t rsl_pack_bf16(float lo_elem, float hi_elem) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo_elem, hi_elem);
  return *reinterpret_cast<uint32_t *>(&v);
}

// hi and lo bf16 terms of two fp32 elements
__device__ __forceinline__ void rsl_split(float x, float y, uint32_t &hi, uint32_t &lo) {
  hi = rsl_pack_bf16(x, y);
  const float2 h = bf16x2_to_float2(hi);
  lo = rsl_pack_bf16(x - h.x, y - h.y);
}

// Partial router sums of query i (sequence s) over its blocks [m0, m1):
// out[j] = sum_m ReLU(q_j . kbar_m) for j < H, in shared memory.  Blocks
// below `full` come from the pool; block `full` (the one cut by the prefix
// end) from tail[128] (shared, its mean over the present tokens).  wsum:
// shared [NW][MISA_MAX_H].  qrow(j): head j's query row (128 bf16) in shared
// memory, readable once `ready` has run.  Every thread of the CTA (NW warps)
// calls; `ready` is called once by every thread, after this warp's first
// pool loads are in flight and before the first query read (it may hold a
// barrier).
template <int NW, class QRow, class Ready>
__device__ void route_slice(const CacheView &c, int s, int H, int m0, int m1, int full, const float *tail,
                            float *wsum, float *out, QRow &&qrow, Ready &&ready) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, cq = lane & 3;
  const int MT = cdiv(H, 16);
  const int M_cap = cdiv(c.L_cap, c.B);
  // warp w keeps one m-tile of 16 heads (w % MT) and takes every
  // (NW / MT)-th n-tile of 8 blocks, two n-tiles per round: the loads of a
  // round are all issued before its first product
  const int wpm = NW / MT;  // warps per m-tile (MT divides NW: MT in {1, 2, 4, 8})
  const int mt = warp % MT;
  const int ha = 16 * mt + g, hb = ha + 8;
  float racc0 = 0.f, racc1 = 0.f;  // heads ha, hb
  bool first = true;
  auto load = [&](int nt, float4 (&x)[4][2]) {
    const int m = m0 + 8 * nt + g;  // this lane's block (B column g)
    const float *prow = m >= m1 ? nullptr : m < full ? c.pool + ((size_t)s * M_cap + m) * D : m == full ? tail : nullptr;
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
      x[ch][0] = prow ? *reinterpret_cast<const float4 *>(prow + 32 * ch + 8 * cq) : make_float4(0.f, 0.f, 0.f, 0.f);
      x[ch][1] = prow ? *reinterpret_cast<const float4 *>(prow + 32 * ch + 8 * cq + 4) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  auto product = [&](const float4 (&x)[4][2]) {
    const uint16_t *qa_row = qrow(ha < H ? ha : 0), *qb_row = qrow(hb < H ? hb : 0);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
      const uint4 qa = ha < H ? *reinterpret_cast<const uint4 *>(qa_row + 32 * ch + 8 * cq) : make_uint4(0u, 0u, 0u, 0u);
      const uint4 qb = hb < H ? *reinterpret_cast<const uint4 *>(qb_row + 32 * ch + 8 * cq) : make_uint4(0u, 0u, 0u, 0u);
      uint32_t bh0, bl0, bh1, bl1;
      const uint32_t a0[4] = {qa.x, qb.x, qa.y, qb.y};  // k-tile 2ch
      const uint32_t a1[4] = {qa.z, qb.z, qa.w, qb.w};  // k-tile 2ch + 1
      rsl_split(x[ch][0].x, x[ch][0].y, bh0, bl0);
      rsl_split(x[ch][0].z, x[ch][0].w, bh1, bl1);
      mma_bf16_16816(acc, a0, bh0, bh1);
      mma_bf16_16816(acc, a0, bl0, bl1);
      rsl_split(x[ch][1].x, x[ch][1].y, bh0, bl0);
      rsl_split(x[ch][1].z, x[ch][1].w, bh1, bl1);
      mma_bf16_16816(acc, a1, bh0, bh1);
      mma_bf16_16816(acc, a1, bl0, bl1);
    }
    // ReLU of every (head, block) product, summed over this tile's blocks;
    // absent blocks multiplied zero keys and add nothing
    racc0 += fmaxf(acc[0], 0.f) + fmaxf(acc[1], 0.f);
    racc1 += fmaxf(acc[2], 0.f) + fmaxf(acc[3], 0.f);
  };
  const int rounds = cdiv(max(m1 - m0, 0), 8 * 2 * wpm);  // the same in every warp
  for (int r = 0; r < rounds || first; ++r) {
    const int nt0 = warp / MT + 2 * wpm * r, nt1 = nt0 + wpm;
    float4 x0[4][2], x1[4][2];
    load(nt0, x0);
    load(nt1, x1);
    if (first) {
      ready();
      first = false;
    }
    if (r < rounds) {
      product(x0);
      product(x1);
    }
  }
  // the four lanes of a row group hold the same heads' sums over different blocks
  racc0 += __shfl_xor_sync(0xffffffffu, racc0, 1);
  racc0 += __shfl_xor_sync(0xffffffffu, racc0, 2);
  racc1 += __shfl_xor_sync(0xffffffffu, racc1, 1);
  racc1 += __shfl_xor_sync(0xffffffffu, racc1, 2);
  if (cq == 0) {
    wsum[warp * MISA_MAX_H + ha] = racc0;
    wsum[warp * MISA_MAX_H + hb] = racc1;
  }
  __syncthreads();
  // head j's sum: the warps holding its m-tile, in warp order
  for (int j = tid; j < H; j += 32 * NW) {
    float v = 0.f;
    for (int w = (j >> 4) % MT; w < NW; w += MT) v += wsum[w * MISA_MAX_H + j];
    out[j] = v;
  }
  __syncthreads();
}

// After the row barrier: the query's importances from the C partial sums
// (part[cc * H + j], written by the C CTAs), r_j = |w_j| * sum (w_s: the
// query's H head weights in shared memory), and its h
// best heads in ascending order into sheads (head j is kept iff fewer than h
// heads beat it: larger r, or equal r and a lower index).  Four threads per
// head: each adds a quarter of the partials in order, the quarters are
// combined in a fixed order, so every CTA of the query gets the same sums.
// r_s, keep_s: shared [MISA_MAX_H]; stage: shared scratch of stage_cap floats
// for the partials; every thread calls (blockDim.x a multiple of 32, at
// least H).
__device__ void route_rank(int H, const float *w_s, const float *part, int C, int h, float *r_s, int *keep_s,
                           int32_t *sheads, float *stage, int stage_cap) {
  const int tid = threadIdx.x, lane = tid & 31;
  const bool staged = C * H <= stage_cap;
  if (staged) {  // every partial requested at once, eight loads in flight per thread
    constexpr int UL = 8;
    for (int x0 = tid; x0 < C * H; x0 += UL * (int)blockDim.x) {
      float v[UL];
#pragma unroll
      for (int u = 0; u < UL; ++u) {
        const int x = x0 + u * (int)blockDim.x;
        v[u] = x < C * H ? __ldcg(part + x) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < UL; ++u) {
        const int x = x0 + u * (int)blockDim.x;
        if (x < C * H) stage[x] = v[u];
      }
    }
    __syncthreads();
  }
  const int qq = tid & 3;  // quarter
  const int c0 = C * qq / 4, c1 = C * (qq + 1) / 4;
  const int per = blockDim.x >> 2;  // heads per sweep
  for (int jb = 0; jb < H; jb += per) {
    const int j = jb + (tid >> 2);
    float acc = 0.f;
    if (j < H)
#pragma unroll 8
      for (int cc = c0; cc < c1; ++cc) acc += staged ? stage[cc * H + j] : __ldcg(part + (size_t)cc * H + j);
    // quarters of a head sit in four consecutive lanes: (q0 + q1) + (q2 + q3)
    const float o1 = __shfl_xor_sync(0xffffffffu, acc, 1);
    const float pair = (qq & 1) ? o1 + acc : acc + o1;
    const float o2 = __shfl_xor_sync(0xffffffffu, pair, 2);
    const float tot = (qq & 2) ? o2 + pair : pair + o2;
    if (j < H && qq == 0) r_s[j] = fabsf(w_s[j]) * tot;
  }
  __syncthreads();
  // rank: each of the four threads counts the heads of a quarter that beat j
  for (int jb = 0; jb < H; jb += per) {
    const int j = jb + (tid >> 2);
    int beaten = 0;
    if (j < H) {
      const float r = r_s[j];
      for (int o = qq; o < H; o += 4) {
        const float ro = r_s[o];
        beaten += (ro > r) || (ro == r && o < j);
      }
    }
    beaten += __shfl_xor_sync(0xffffffffu, beaten, 1);
    beaten += __shfl_xor_sync(0xffffffffu, beaten, 2);
    if (j < H && qq == 0) keep_s[j] = beaten < h;
  }
  __syncthreads();
  // kept heads in ascending order: a head's position counts the kept heads below it
  if (tid < 32 * cdiv(H, 32)) {
    const bool kept = tid < H && keep_s[tid];
    const uint32_t m = __ballot_sync(0xffffffffu, kept);
    uint32_t lt = 0;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(lt));
    int pos = __popc(m & lt);
    for (int w = 0; w < (tid >> 5); ++w)
      for (int x = 32 * w; x < 32 * w + 32 && x < H; ++x) pos += keep_s[x];
    if (kept && pos < h) sheads[pos] = tid;  // a NaN importance can break the strict order
  }
  (void)lane;
  __syncthreads();
}

}  // namespace
}  // namespace misa
