// The query's head matrix Q' for the tensor-core re-rank and dense kernels.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference",
// technical summary, "Hierarchical variant" and "Problem statement": the
// scoring heads' query rows q_{i,n} (bf16) and weights w_{i,n} are the N side
// of the tcgen05 products K . Q'^T.
#pragma once

#include "frag.cuh"

namespace misa {
namespace {

// Q' of query i in shared memory: row n = the n-th scoring head (zero rows
// past h_eff), two threads per row (half of its 16-byte chunks each, the pair
// agreeing on the e4m3 scale through a shuffle), in the 128-byte-swizzled
// K-major layout the MMA reads; bf16 as is, or the exact two-term e4m3 split
// with the power-of-two scale folded into the weight w_s[n].  128 threads
// call, numbered `tid` = 0 .. 127 (whole warps).
template <bool FP8, int HN>
__device__ __forceinline__ void build_qprime(const CacheView &c, const QueryView &qv, const int32_t *heads, int h,
                                             int i, uint8_t *b_smem, float *w_s, int tid = threadIdx.x) {
  const int H = qv.H;
  const int h_eff = heads ? h : H;
  for (int x = tid; x < 2 * HN; x += 128) {  // whole warps: HN >= 32
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

}  // namespace
}  // namespace misa
