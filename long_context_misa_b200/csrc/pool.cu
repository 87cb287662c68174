// Block mean-pool of the index keys, and the fused key-append + pool update.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference",
// technical summary, "Methodology: MISA", step 1: the prefix is cut into
// M = ceil(L/B) blocks, each summarised by the mean of its index keys.
//
// Layout: keys [n_seq][L_cap][128] (bf16: 256 B/token, e4m3: 128 B/token plus
// an fp32 scale), pool [n_seq][ceil(L_cap/B)][128] fp32.
// Rebuild: one CTA of 128 threads per block streams 16-byte vectors of fixed
// coordinates over a strided subset of the block's tokens; partial sums meet
// in shared memory.  Append (the key-write path): one CTA of 512 threads per
// sequence writes the new keys and recomputes every touched block in the
// same kernel, taking the new tokens from the input rather than re-reading
// the cache, so the whole update costs one round trip of loads.
// Quantising append (e4m3 caches fed bf16 keys): each warp quantises rows
// of the new keys -- amax over the row by shuffles, s = amax / 448 (1 for a
// zero row), codes = e4m3(x / s) rounded to nearest even and saturated --
// into shared memory, from where they are written to the cache and read by
// the same block-mean update.
#include "frag.cuh"
#include "internal.h"
#include "keysum.cuh"

namespace misa {
namespace {

constexpr int REBUILD_THREADS = 128;
constexpr int APPEND_THREADS = 512;

__global__ void __launch_bounds__(REBUILD_THREADS) pool_rebuild_kernel(CacheView c) {
  grid_dep_sync();
  __shared__ float sm_part[(REBUILD_THREADS / 8) * D];
  __shared__ float sm_out[D];
  const int s = blockIdx.y, m = blockIdx.x;
  const int len = min(c.seq_len[s], c.L_cap);
  const int t0 = m * c.B;
  if (t0 >= len) return;
  const int t1 = min(t0 + c.B, len);
  block_key_sum<REBUILD_THREADS>(c, s, t0, t1, sm_part, sm_out);
  const int M_cap = cdiv(c.L_cap, c.B);
  c.pool[((size_t)s * M_cap + m) * D + threadIdx.x] = sm_out[threadIdx.x] / (float)(t1 - t0);
}

// zero / zero_n: words the next kernels count into, cleared here too (so that
// a decode step needs no separate zeroing launch).
__global__ void __launch_bounds__(APPEND_THREADS) pool_append_kernel(CacheView c, const void *new_keys,
                                                                     const float *new_scale,
                                                                     const int32_t *new_pos, int count,
                                                                     uint32_t *zero, size_t zero_n, int early) {
  grid_dep_sync();
  if (early) grid_dep_launch();  // the routed pass routes meanwhile
  for (size_t x = (size_t)blockIdx.x * APPEND_THREADS + threadIdx.x; x < zero_n; x += (size_t)gridDim.x * APPEND_THREADS)
    zero[x] = 0u;
  __shared__ float sm_part[(APPEND_THREADS / 8) * D];
  __shared__ float sm_out[D];
  const int s = blockIdx.x;
  const int pos = new_pos[s];
  if (pos < 0) return;
  if ((long long)pos + count > c.L_cap) {
    if (threadIdx.x == 0) flag(c, MISA_DEV_APPEND_RANGE);
    return;
  }
  const int row_bytes = c.fp8 ? D : 2 * D;
  const uint8_t *src = static_cast<const uint8_t *>(new_keys) + (size_t)s * count * row_bytes;
  const float *src_scale = c.fp8 ? new_scale + (size_t)s * count : nullptr;
  uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint8_t *>(const_cast<void *>(c.keys)) +
                                         ((size_t)s * c.L_cap + pos) * row_bytes);
  const uint4 *src4 = reinterpret_cast<const uint4 *>(src);
  for (int v = threadIdx.x; v < count * (row_bytes / 16); v += blockDim.x) dst[v] = src4[v];
  if (c.fp8) {
    float *sc = const_cast<float *>(c.scale) + (size_t)s * c.L_cap + pos;
    for (int t = threadIdx.x; t < count; t += blockDim.x) sc[t] = src_scale[t];
  }
  KeySource ks;
  ks.ovr_keys = src;
  ks.ovr_scale = src_scale;
  ks.ovr_t0 = pos;
  ks.ovr_n = count;
  const int len = pos + count;
  const int M_cap = cdiv(c.L_cap, c.B);
  for (int m = pos / c.B; m <= (len - 1) / c.B; ++m) {
    const int t0 = m * c.B, t1 = min(t0 + c.B, len);
    block_key_sum<APPEND_THREADS>(c, s, t0, t1, sm_part, sm_out, ks);
    if (threadIdx.x < D) c.pool[((size_t)s * M_cap + m) * D + threadIdx.x] = sm_out[threadIdx.x] / (float)(t1 - t0);
  }
  if (threadIdx.x == 0) c.seq_len[s] = len;
}

constexpr int QAPPEND_MAX = 64;  // new tokens per sequence in one quantising append

__global__ void __launch_bounds__(APPEND_THREADS) pool_append_quant_kernel(CacheView c, const uint16_t *new_keys,
                                                                           const int32_t *new_pos, int count) {
  grid_dep_sync();
  __shared__ float sm_part[(APPEND_THREADS / 8) * D];
  __shared__ float sm_out[D];
  __shared__ __align__(16) uint8_t codes[QAPPEND_MAX * D];
  __shared__ float scales[QAPPEND_MAX];
  const int s = blockIdx.x;
  const int pos = new_pos[s];
  if (pos < 0) return;
  if ((long long)pos + count > c.L_cap) {
    if (threadIdx.x == 0) flag(c, MISA_DEV_APPEND_RANGE);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint16_t *src = new_keys + (size_t)s * count * D;
  for (int j = warp; j < count; j += APPEND_THREADS / 32) {
    // lane: elements 4 lane .. 4 lane + 3 of row j
    const uint2 v = *reinterpret_cast<const uint2 *>(src + (size_t)j * D + 4 * lane);
    const float2 a = bf16x2_to_float2(v.x), b = bf16x2_to_float2(v.y);
    float m = fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(b.x), fabsf(b.y)));
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float sc = m > 0.f ? __fdiv_rn(m, 448.f) : 1.f;
    const uint32_t c01 = f32x2_to_e4m3x2(__fdiv_rn(a.x, sc), __fdiv_rn(a.y, sc));
    const uint32_t c23 = f32x2_to_e4m3x2(__fdiv_rn(b.x, sc), __fdiv_rn(b.y, sc));
    *reinterpret_cast<uint32_t *>(codes + j * D + 4 * lane) = (c01 & 0xFFFFu) | (c23 << 16);
    if (lane == 0) scales[j] = sc;
  }
  __syncthreads();
  uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint8_t *>(const_cast<void *>(c.keys)) +
                                         ((size_t)s * c.L_cap + pos) * D);
  for (int v = threadIdx.x; v < count * (D / 16); v += blockDim.x) dst[v] = reinterpret_cast<const uint4 *>(codes)[v];
  float *sc_dst = const_cast<float *>(c.scale) + (size_t)s * c.L_cap + pos;
  for (int t = threadIdx.x; t < count; t += blockDim.x) sc_dst[t] = scales[t];
  KeySource ks;
  ks.ovr_keys = codes;
  ks.ovr_scale = scales;
  ks.ovr_t0 = pos;
  ks.ovr_n = count;
  const int len = pos + count;
  const int M_cap = cdiv(c.L_cap, c.B);
  for (int m = pos / c.B; m <= (len - 1) / c.B; ++m) {
    const int t0 = m * c.B, t1 = min(t0 + c.B, len);
    block_key_sum<APPEND_THREADS>(c, s, t0, t1, sm_part, sm_out, ks);
    if (threadIdx.x < D) c.pool[((size_t)s * M_cap + m) * D + threadIdx.x] = sm_out[threadIdx.x] / (float)(t1 - t0);
  }
  if (threadIdx.x == 0) c.seq_len[s] = len;
}

}  // namespace

int pool_append_quant_max() { return QAPPEND_MAX; }

cudaError_t launch_pool_append_quant(const CacheView &c, const uint16_t *new_keys, const int32_t *new_pos, int count,
                                     cudaStream_t s) {
  return launch_kernel(pool_append_quant_kernel, dim3(c.n_seq), dim3(APPEND_THREADS), 0, s, c, new_keys, new_pos,
                       count);
}

cudaError_t launch_pool_rebuild(const CacheView &c, cudaStream_t s) {
  dim3 grid(cdiv(c.L_cap, c.B), c.n_seq);
  return launch_kernel(pool_rebuild_kernel, grid, dim3(REBUILD_THREADS), 0, s, c);
}

cudaError_t launch_pool_append(const CacheView &c, const void *new_keys, const float *new_scale,
                               const int32_t *new_pos, int count, cudaStream_t s, uint32_t *zero, size_t zero_n,
                               bool early) {
  return launch_kernel(pool_append_kernel, dim3(c.n_seq), dim3(APPEND_THREADS), 0, s, c, new_keys, new_scale, new_pos,
                       count, zero, zero_n, early ? 1 : 0);
}

}  // namespace misa
