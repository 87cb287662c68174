// Block-pooled head router.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference",
// technical summary, "Methodology: MISA", step 1: per-head affinities are
// computed against block-level statistics (the mean-pooled index keys) rather
// than individual tokens, aggregated into an importance per head, and the
// top-h heads are kept; cost O(H_I * M).  Aggregation read here:
//     r_j = |w_j| * sum_{m < M_i} ReLU(q_j . kbar_m),   M_i = ceil(L_i / B),
// where the block cut by the query's prefix end is recomputed from its keys
// (tokens floor(L_i/B)*B .. q_pos), so routing never sees a future token.
//
// route_partial_kernel: grid (chunks of 64 pooled keys, queries), 4 warps.
//   The affinities q_j . kbar_m are a [64 blocks x 128] x [128 x H] product
//   on mma.sync m16n8k16: each fp32 pooled key is split into bf16 hi + lo
//   (hi = RN(k), lo = RN(k - hi)) and both halves are multiplied by the bf16
//   query, so the product keeps ~16 significant bits of the pooled key with
//   exact products and fp32 accumulation.  Warp w owns blocks 16w..16w+15 of
//   the chunk; ReLU and the sum over blocks happen on the accumulator
//   registers, and the four warps' column sums meet in shared memory.
// route_finish_kernel: one CTA per query sums the chunk partials in a fixed
//   order, applies |w_j| and keeps the h best heads: head j is kept iff fewer
//   than h heads beat it (larger r, or equal r and lower index); the kept
//   heads are written in ascending order.
#include "internal.h"
#include "keysum.cuh"

namespace misa {
namespace {

constexpr int RB = 64;               // pooled keys per CTA
constexpr int ROUTE_THREADS = 128;   // 4 warps x 16 pooled keys
constexpr int PSTRIDE = D + 16;      // floats per staged pooled row: conflict-free 16-byte loads
constexpr int KT = 8;                // k-tiles of 16 over d = 128
constexpr int MAX_NT = MISA_MAX_H / 8;

size_t route_smem_bytes(int H) {
  const int NT = (H + 7) / 8;
  return sizeof(float) * ((size_t)RB * PSTRIDE + 16 * D + D + 4 * MAX_NT * 8) + sizeof(uint2) * KT * NT * 32;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo_elem, float hi_elem) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo_elem, hi_elem);
  return *reinterpret_cast<uint32_t *>(&v);
}

__global__ void __launch_bounds__(ROUTE_THREADS) route_partial_kernel(CacheView c, QueryView qv, float *partial,
                                                                      int n_chunks, int agg) {
  grid_dep_sync();
  extern __shared__ __align__(16) float smem[];
  float *p_s = smem;                          // [RB][PSTRIDE] pooled keys (fp32)
  float *part = p_s + RB * PSTRIDE;           // [16][128] key-sum scratch
  float *tail = part + 16 * D;                // [128]
  float *colsum = tail + D;                   // [4 warps][H]
  uint2 *bfrag = reinterpret_cast<uint2 *>(colsum + 4 * MAX_NT * 8);  // [kt][nt][lane]
  const int i = blockIdx.y, chunk = blockIdx.x;
  int s;
  const int Li = query_prefix(c, qv, i, &s);
  const int Mi = cdiv(Li, c.B);
  const int m0 = chunk * RB;
  if (m0 >= Mi) return;              // uniform over the CTA
  const int full = Li / c.B;         // blocks wholly inside the prefix
  const int M_cap = cdiv(c.L_cap, c.B);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, cq = lane & 3;
  const int H = qv.H, NT = (H + 7) / 8;

  // query heads as B fragments: k-tile kt, lane (g, cq) holds head n = 8nt + g,
  // physical elements 16kt + 4cq + {0,1} (b0) and + {2,3} (b1)
  // (fixed trip counts, loads first: one memory round trip, not one per element)
  {
    constexpr int PER = KT * MAX_NT * 32 / ROUTE_THREADS;
    uint2 v[PER];
#pragma unroll
    for (int it = 0; it < PER; ++it) {
      const int e = tid + it * ROUTE_THREADS;
      const int l = e & 31, nt = (e >> 5) % NT, kt = (e >> 5) / NT;
      const int n = nt * 8 + (l >> 2);
      v[it] = make_uint2(0u, 0u);
      if (e < KT * NT * 32 && n < H)
        v[it] = __ldg(reinterpret_cast<const uint2 *>(qv.q + ((size_t)i * H + n) * D + 16 * kt + 4 * (l & 3)));
    }
#pragma unroll
    for (int it = 0; it < PER; ++it) {
      const int e = tid + it * ROUTE_THREADS;
      if (e < KT * NT * 32) bfrag[e] = v[it];
    }
  }
  // pooled keys of whole blocks; the rest of the chunk is zero (ReLU(0) = 0)
  const int nb = min(RB, Mi - m0);
  {
    constexpr int PER = RB * (D / 4) / ROUTE_THREADS;
    float4 x[PER];
#pragma unroll
    for (int it = 0; it < PER; ++it) {
      const int v = tid + it * ROUTE_THREADS;
      const int r = v / (D / 4), e4 = v % (D / 4), m = m0 + r;
      x[it] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < nb && m < full) x[it] = __ldg(reinterpret_cast<const float4 *>(c.pool + ((size_t)s * M_cap + m) * D + 4 * e4));
    }
#pragma unroll
    for (int it = 0; it < PER; ++it) {
      const int v = tid + it * ROUTE_THREADS;
      *reinterpret_cast<float4 *>(p_s + (v / (D / 4)) * PSTRIDE + 4 * (v % (D / 4))) = x[it];
    }
  }
  const bool has_tail = full < Mi && full >= m0 && full < m0 + RB;  // uniform
  if (has_tail) {
    block_key_sum<128>(c, s, full * c.B, Li, part, tail);
    const float inv = 1.f / (float)(Li - full * c.B);
    p_s[(full - m0) * PSTRIDE + tid] = tail[tid] * inv;
  }
  __syncthreads();

  // warp w: pooled keys 16w + g and 16w + g + 8
  float racc[MAX_NT][2];
#pragma unroll
  for (int nt = 0; nt < MAX_NT; ++nt) racc[nt][0] = racc[nt][1] = 0.f;
  const float *rowA = p_s + (16 * warp + g) * PSTRIDE;
  const float *rowB = rowA + 8 * PSTRIDE;
  float acc[MAX_NT][4];
#pragma unroll
  for (int nt = 0; nt < MAX_NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
  for (int kt = 0; kt < KT; ++kt) {
    const float4 xa = *reinterpret_cast<const float4 *>(rowA + 16 * kt + 4 * cq);
    const float4 xb = *reinterpret_cast<const float4 *>(rowB + 16 * kt + 4 * cq);
    uint32_t hi[4], lo[4];
    hi[0] = pack_bf16(xa.x, xa.y);
    hi[1] = pack_bf16(xb.x, xb.y);
    hi[2] = pack_bf16(xa.z, xa.w);
    hi[3] = pack_bf16(xb.z, xb.w);
    {
      const float2 h0 = bf16x2_to_float2(hi[0]), h1 = bf16x2_to_float2(hi[1]);
      const float2 h2 = bf16x2_to_float2(hi[2]), h3 = bf16x2_to_float2(hi[3]);
      lo[0] = pack_bf16(xa.x - h0.x, xa.y - h0.y);
      lo[1] = pack_bf16(xb.x - h1.x, xb.y - h1.y);
      lo[2] = pack_bf16(xa.z - h2.x, xa.w - h2.y);
      lo[3] = pack_bf16(xb.z - h3.x, xb.w - h3.y);
    }
#pragma unroll
    for (int nt = 0; nt < MAX_NT; ++nt) {
      if (nt < NT) {
        const uint2 b = bfrag[(kt * NT + nt) * 32 + lane];
        mma_bf16_16816(acc[nt], hi, b.x, b.y);
        mma_bf16_16816(acc[nt], lo, b.x, b.y);
      }
    }
  }
#pragma unroll
  for (int nt = 0; nt < MAX_NT; ++nt) {
    if (agg_is_max(agg)) {
      racc[nt][0] = fmaxf(fmaxf(acc[nt][0], 0.f), fmaxf(acc[nt][2], 0.f));
      racc[nt][1] = fmaxf(fmaxf(acc[nt][1], 0.f), fmaxf(acc[nt][3], 0.f));
    } else {
      racc[nt][0] = fmaxf(acc[nt][0], 0.f) + fmaxf(acc[nt][2], 0.f);  // head 8nt + 2cq
      racc[nt][1] = fmaxf(acc[nt][1], 0.f) + fmaxf(acc[nt][3], 0.f);  // head 8nt + 2cq + 1
    }
  }
  // sum over the 8 row groups of the warp (lanes with equal cq)
#pragma unroll
  for (int nt = 0; nt < MAX_NT; ++nt)
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        const float x = __shfl_xor_sync(0xffffffffu, racc[nt][u], o);
        racc[nt][u] = agg_is_max(agg) ? fmaxf(racc[nt][u], x) : racc[nt][u] + x;
      }
  if (g == 0) {
#pragma unroll
    for (int nt = 0; nt < MAX_NT; ++nt)
      if (nt < NT) {
        colsum[warp * (MAX_NT * 8) + 8 * nt + 2 * cq] = racc[nt][0];
        colsum[warp * (MAX_NT * 8) + 8 * nt + 2 * cq + 1] = racc[nt][1];
      }
  }
  __syncthreads();
  if (tid < H) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float x = colsum[w * (MAX_NT * 8) + tid];
      v = agg_is_max(agg) ? fmaxf(v, x) : v + x;
    }
    partial[((size_t)i * n_chunks + chunk) * H + tid] = v;
  }
}

__global__ void __launch_bounds__(MISA_MAX_H) route_finish_kernel(CacheView c, QueryView qv, const float *partial,
                                                                  int n_chunks, int h, int32_t *heads,
                                                                  float *router_scores, int agg) {
  grid_dep_sync();
  __shared__ float r_s[MISA_MAX_H];
  __shared__ int warp_cnt[MISA_MAX_H / 32];
  const int i = blockIdx.x, j = threadIdx.x, H = qv.H;
  int s;
  const int Li = query_prefix(c, qv, i, &s);
  const int nc = cdiv(cdiv(Li, c.B), RB);
  float r = 0.f;
  if (j < H) {
    float acc = 0.f;
#pragma unroll 16
    for (int ch = 0; ch < nc; ++ch) {
      const float x = __ldg(partial + ((size_t)i * n_chunks + ch) * H + j);
      acc = agg_is_max(agg) ? fmaxf(acc, x) : acc + x;
    }
    r = agg_weight(agg, qv.w[(size_t)i * H + j]) * acc;
    r_s[j] = r;
    if (router_scores) router_scores[(size_t)i * H + j] = r;
  }
  __syncthreads();
  bool keep = false;
  if (j < H) {
    int beaten = 0;
    for (int o = 0; o < H; ++o) {
      const float ro = r_s[o];
      beaten += (ro > r) || (ro == r && o < j);
    }
    keep = beaten < h;
  }
  const unsigned b = __ballot_sync(0xffffffffu, keep);
  if ((j & 31) == 0) warp_cnt[j >> 5] = __popc(b);
  __syncthreads();
  if (keep) {
    int pos = __popc(b & ((1u << (j & 31)) - 1u));
    for (int w = 0; w < (j >> 5); ++w) pos += warp_cnt[w];
    if (pos < h) heads[(size_t)i * h + pos] = j;  // a NaN score can break the strict order
  }
}

}  // namespace

int route_chunks(int M_cap) { return cdiv(M_cap, RB); }

size_t route_ws_bytes(int n_q, int H, int M_cap) {
  return sizeof(float) * (size_t)n_q * route_chunks(M_cap) * H;
}

cudaError_t launch_route(const CacheView &c, const QueryView &q, int h, int32_t *heads, float *router_scores,
                         void *ws, cudaStream_t s, int agg) {
  if (q.n_q == 0) return cudaSuccess;
  if (route_umma_applies(c, q)) return launch_route_umma(c, q, h, heads, router_scores, ws, s, agg);
  const int M_cap = cdiv(c.L_cap, c.B);
  const int n_chunks = route_chunks(M_cap);
  const size_t smem = route_smem_bytes(q.H);
  struct Tag {};
  const int opt_in = cached_per_device<Tag>([] {
    return cudaFuncSetAttribute(route_partial_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)route_smem_bytes(MISA_MAX_H)) == cudaSuccess ? 1 : -1;
  });
  if (opt_in < 0) return cudaErrorInvalidConfiguration;
  cudaError_t e;
  float *partial = static_cast<float *>(ws);
  e = launch_kernel(route_partial_kernel, dim3(n_chunks, q.n_q), dim3(ROUTE_THREADS), smem, s, c, q, partial, n_chunks,
                    agg);
  if (e != cudaSuccess) return e;
  return launch_kernel(route_finish_kernel, dim3(q.n_q), dim3(MISA_MAX_H), 0, s, c, q, partial, n_chunks, h, heads,
                    router_scores, agg);
}

}  // namespace misa
