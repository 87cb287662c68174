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
// route_partial_kernel: grid (chunks of 32 pooled keys, queries), 8 warps.
//   Lane l of every warp owns pooled key m = chunk*32 + l; warp w owns heads
//   w, w+8, ...; the query heads and the 32 pooled keys sit in shared memory
//   as fp32 (pooled rows padded to 129 floats so the 32 lanes hit 32 banks).
//   Each warp writes sum_m ReLU(q_j . kbar_m) over its lanes for its heads.
// route_finish_kernel: one CTA per query sums the chunk partials in a fixed
//   order, applies |w_j| and keeps the h best heads: head j is kept iff fewer
//   than h heads beat it (larger r, or equal r and lower index); the kept
//   heads are written in ascending order.
#include "internal.h"
#include "keysum.cuh"

namespace misa {
namespace {

constexpr int RB = 32;             // pooled keys per CTA
constexpr int ROUTE_THREADS = 256; // 8 warps
constexpr int ROUTE_WARPS = ROUTE_THREADS / 32;
constexpr int PROW = D + 1;        // padded pooled-row stride (floats)
constexpr int HG = 8;              // heads accumulated together by one warp

size_t route_smem_bytes(int H) { return sizeof(float) * ((size_t)H * D + RB * PROW + 16 * D + D); }

__global__ void __launch_bounds__(ROUTE_THREADS) route_partial_kernel(CacheView c, QueryView qv, float *partial,
                                                                      int n_chunks) {
  extern __shared__ float smem[];
  float *q_s = smem;                 // [H][128]
  float *p_s = q_s + qv.H * D;       // [RB][PROW]
  float *part = p_s + RB * PROW;     // [16][128] key-sum scratch
  float *tail = part + 16 * D;       // [128]
  const int i = blockIdx.y, chunk = blockIdx.x;
  int s;
  const int Li = query_prefix(c, qv, i, &s);
  const int Mi = cdiv(Li, c.B);
  const int m0 = chunk * RB;
  if (m0 >= Mi) return;              // uniform over the CTA
  const int full = Li / c.B;         // blocks wholly inside the prefix
  const int M_cap = cdiv(c.L_cap, c.B);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = qv.H;

  const uint32_t *qsrc = reinterpret_cast<const uint32_t *>(qv.q + (size_t)i * H * D);
  for (int v = tid; v < H * D / 2; v += blockDim.x) {
    float2 f = bf16x2_to_float2(__ldg(qsrc + v));
    q_s[2 * v] = f.x;
    q_s[2 * v + 1] = f.y;
  }
  const int nb = min(RB, Mi - m0);
  for (int v = tid; v < RB * D; v += blockDim.x) {
    const int r = v / D, e = v % D, m = m0 + r;
    p_s[r * PROW + e] = (r < nb && m < full) ? c.pool[((size_t)s * M_cap + m) * D + e] : 0.f;
  }
  const bool has_tail = full < Mi && full >= m0 && full < m0 + RB;  // uniform
  if (has_tail) {
    block_key_sum<false>(c, s, full * c.B, Li, part, tail);
    const float inv = 1.f / (float)(Li - full * c.B);
    if (tid < D) p_s[(full - m0) * PROW + tid] = tail[tid] * inv;
  }
  __syncthreads();

  const bool valid = lane < nb;
  const float *prow = p_s + lane * PROW;
  for (int j0 = warp * HG; j0 < H; j0 += ROUTE_WARPS * HG) {
    float acc[HG];
#pragma unroll
    for (int g = 0; g < HG; ++g) acc[g] = 0.f;
    for (int d0 = 0; d0 < D; d0 += 32) {
      float kr[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) kr[e] = prow[d0 + e];
#pragma unroll
      for (int g = 0; g < HG; ++g) {
        const int j = min(j0 + g, H - 1);
        const float4 *qq = reinterpret_cast<const float4 *>(q_s + j * D + d0);
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 qv4 = qq[e4];
          acc[g] = fmaf(qv4.x, kr[4 * e4 + 0], acc[g]);
          acc[g] = fmaf(qv4.y, kr[4 * e4 + 1], acc[g]);
          acc[g] = fmaf(qv4.z, kr[4 * e4 + 2], acc[g]);
          acc[g] = fmaf(qv4.w, kr[4 * e4 + 3], acc[g]);
        }
      }
    }
#pragma unroll
    for (int g = 0; g < HG; ++g) {
      float v = valid ? fmaxf(acc[g], 0.f) : 0.f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0 && j0 + g < H) partial[((size_t)i * n_chunks + chunk) * H + j0 + g] = v;
    }
  }
}

__global__ void __launch_bounds__(MISA_MAX_H) route_finish_kernel(CacheView c, QueryView qv, const float *partial,
                                                                  int n_chunks, int h, int32_t *heads,
                                                                  float *router_scores) {
  __shared__ float r_s[MISA_MAX_H];
  __shared__ int warp_cnt[MISA_MAX_H / 32];
  const int i = blockIdx.x, j = threadIdx.x, H = qv.H;
  int s;
  const int Li = query_prefix(c, qv, i, &s);
  const int nc = cdiv(cdiv(Li, c.B), RB);
  float r = 0.f;
  if (j < H) {
    float acc = 0.f;
    for (int ch = 0; ch < nc; ++ch) acc += partial[((size_t)i * n_chunks + ch) * H + j];
    r = fabsf(qv.w[(size_t)i * H + j]) * acc;
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
                         void *ws, cudaStream_t s) {
  if (q.n_q == 0) return cudaSuccess;
  const int M_cap = cdiv(c.L_cap, c.B);
  const int n_chunks = route_chunks(M_cap);
  const size_t smem = route_smem_bytes(q.H);
  cudaError_t e = cudaFuncSetAttribute(route_partial_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  float *partial = static_cast<float *>(ws);
  route_partial_kernel<<<dim3(n_chunks, q.n_q), ROUTE_THREADS, smem, s>>>(c, q, partial, n_chunks);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  route_finish_kernel<<<q.n_q, MISA_MAX_H, 0, s>>>(c, q, partial, n_chunks, h, heads, router_scores);
  return cudaGetLastError();
}

}  // namespace misa
