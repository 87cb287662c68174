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
#include "internal.h"
#include "keysum.cuh"

namespace misa {
namespace {

constexpr int REBUILD_THREADS = 128;
constexpr int APPEND_THREADS = 512;

__global__ void __launch_bounds__(REBUILD_THREADS) pool_rebuild_kernel(CacheView c) {
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

__global__ void __launch_bounds__(APPEND_THREADS) pool_append_kernel(CacheView c, const void *new_keys,
                                                                     const float *new_scale,
                                                                     const int32_t *new_pos, int count) {
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

}  // namespace

cudaError_t launch_pool_rebuild(const CacheView &c, cudaStream_t s) {
  dim3 grid(cdiv(c.L_cap, c.B), c.n_seq);
  return launch_kernel(pool_rebuild_kernel, grid, dim3(REBUILD_THREADS), 0, s, c);
}

cudaError_t launch_pool_append(const CacheView &c, const void *new_keys, const float *new_scale,
                               const int32_t *new_pos, int count, cudaStream_t s) {
  return launch_kernel(pool_append_kernel, dim3(c.n_seq), dim3(APPEND_THREADS), 0, s, c, new_keys, new_scale, new_pos, count);
}

}  // namespace misa
