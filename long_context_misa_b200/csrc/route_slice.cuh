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
// shared [NW][MISA_MAX_H].  Every thread of the CTA (NW warps) calls.
template <int NW>
__device__ void route_slice(const CacheView &c, const QueryView &qv, int i, int s, int m0, int m1, int full,
                            const float *tail, float *wsum, float *out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, cq = lane & 3;
  const int H = qv.H, MT = cdiv(H, 16);
  const int M_cap = cdiv(c.L_cap, c.B);
  const uint16_t *qrow = qv.q + (size_t)i * H * D;
  // one m-tile of 16 heads at a time (few live registers); the pooled keys
  // are read again for every m-tile, from L2
  for (int mt = 0; mt < MT; ++mt) {
    const int ha = 16 * mt + g, hb = ha + 8;
    float racc0 = 0.f, racc1 = 0.f;  // heads ha, hb
    for (int nt = warp; m0 + 8 * nt < m1; nt += NW) {
      const int m = m0 + 8 * nt + g;  // this lane's block (B column g)
      const float *prow =
          m >= m1 ? nullptr : m < full ? c.pool + ((size_t)s * M_cap + m) * D : m == full ? tail : nullptr;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        float4 x0 = make_float4(0.f, 0.f, 0.f, 0.f), x1 = x0;
        if (prow) {
          x0 = *reinterpret_cast<const float4 *>(prow + 32 * ch + 8 * cq);
          x1 = *reinterpret_cast<const float4 *>(prow + 32 * ch + 8 * cq + 4);
        }
        const uint4 qa = ha < H ? __ldg(reinterpret_cast<const uint4 *>(qrow + (size_t)ha * D + 32 * ch + 8 * cq))
                                : make_uint4(0u, 0u, 0u, 0u);
        const uint4 qb = hb < H ? __ldg(reinterpret_cast<const uint4 *>(qrow + (size_t)hb * D + 32 * ch + 8 * cq))
                                : make_uint4(0u, 0u, 0u, 0u);
        uint32_t bh0, bl0, bh1, bl1;
        const uint32_t a0[4] = {qa.x, qb.x, qa.y, qb.y};  // k-tile 2ch
        const uint32_t a1[4] = {qa.z, qb.z, qa.w, qb.w};  // k-tile 2ch + 1
        rsl_split(x0.x, x0.y, bh0, bl0);
        rsl_split(x0.z, x0.w, bh1, bl1);
        mma_bf16_16816(acc, a0, bh0, bh1);
        mma_bf16_16816(acc, a0, bl0, bl1);
        rsl_split(x1.x, x1.y, bh0, bl0);
        rsl_split(x1.z, x1.w, bh1, bl1);
        mma_bf16_16816(acc, a1, bh0, bh1);
        mma_bf16_16816(acc, a1, bl0, bl1);
      }
      // ReLU of every (head, block) product, summed over this tile's blocks;
      // absent blocks multiplied zero keys and add nothing
      racc0 += fmaxf(acc[0], 0.f) + fmaxf(acc[1], 0.f);
      racc1 += fmaxf(acc[2], 0.f) + fmaxf(acc[3], 0.f);
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
  }
  __syncthreads();
  for (int j = tid; j < H; j += 32 * NW) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) v += wsum[w * MISA_MAX_H + j];
    out[j] = v;
  }
  __syncthreads();
}

// After the row barrier: the query's importances from the C partial sums
// (part[cc * H + j], written by the C CTAs, added in the order cc = 0..C-1),
// r_j = |w_j| * sum, and its h best heads in ascending order into sheads
// (head j is kept iff fewer than h heads beat it: larger r, or equal r and a
// lower index).  r_s, keep_s: shared [MISA_MAX_H].  Every thread calls.
__device__ void route_rank(const QueryView &qv, int i, const float *part, int C, int h, float *r_s, int *keep_s,
                           int32_t *sheads) {
  const int tid = threadIdx.x, H = qv.H;
  for (int j = tid; j < H; j += blockDim.x) {
    float acc = 0.f;
    for (int cc = 0; cc < C; ++cc) acc += __ldcg(part + (size_t)cc * H + j);
    r_s[j] = fabsf(__ldg(qv.w + (size_t)i * H + j)) * acc;
  }
  __syncthreads();
  for (int j = tid; j < H; j += blockDim.x) {
    const float r = r_s[j];
    int beaten = 0;
    for (int o = 0; o < H; ++o) {
      const float ro = r_s[o];
      beaten += (ro > r) || (ro == r && o < j);
    }
    keep_s[j] = beaten < h;
  }
  __syncthreads();
  for (int j = tid; j < H; j += blockDim.x) {
    if (!keep_s[j]) continue;
    int pos = 0;
    for (int o = 0; o < j; ++o) pos += keep_s[o];
    if (pos < h) sheads[pos] = j;  // a NaN importance can break the strict order
  }
  __syncthreads();
}

}  // namespace
}  // namespace misa
