// Block-wide sum of a range of dequantised index keys (shared by the pool and
// router kernels).
#pragma once

#include "common.cuh"

namespace misa {

// Where a token's key comes from: the cache, except tokens [ovr_t0, ovr_t0 +
// ovr_n) which are read from `ovr_keys` / `ovr_scale` (rows in the cache's
// layout) -- the keys an append writes in the same kernel.
struct KeySource {
  const void *ovr_keys = nullptr;
  const float *ovr_scale = nullptr;
  int ovr_t0 = 0, ovr_n = 0;
};

// Sum of keys [t0, t1) of sequence s into sm_out[128] (fp32).  Every thread of
// the block must call this (it holds two barriers); NT threads take part
// (NT = 128 or 512, and a multiple of the row's 16-byte chunk count).
// sm_part must hold NT / 8 rows of 128 floats.
template <int NT>
__device__ void block_key_sum(const CacheView &c, int s, int t0, int t1, float *sm_part, float *sm_out,
                              const KeySource &src = KeySource()) {
  const int tid = threadIdx.x;
  const bool worker = tid < NT;
  const int chunks = c.fp8 ? 8 : 16;      // 16-byte chunks per row
  const int rows = NT / chunks;           // rows per sweep
  if (worker) {
    const int chunk = tid % chunks, r = tid / chunks;
    const size_t row_bytes = c.fp8 ? D : 2 * D;
    const uint8_t *base = static_cast<const uint8_t *>(c.keys) + (size_t)s * c.L_cap * row_bytes + 16 * chunk;
    const uint8_t *obase = static_cast<const uint8_t *>(src.ovr_keys) + 16 * chunk;
    if (!c.fp8) {
      float acc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll 4
      for (int t = t0 + r; t < t1; t += rows) {
        const bool o = (unsigned)(t - src.ovr_t0) < (unsigned)src.ovr_n;
        const uint4 v = o ? *reinterpret_cast<const uint4 *>(obase + (size_t)(t - src.ovr_t0) * row_bytes)
                          : ldg_stream(base + (size_t)t * row_bytes);
        float2 f;
        f = bf16x2_to_float2(v.x); acc[0] += f.x; acc[1] += f.y;
        f = bf16x2_to_float2(v.y); acc[2] += f.x; acc[3] += f.y;
        f = bf16x2_to_float2(v.z); acc[4] += f.x; acc[5] += f.y;
        f = bf16x2_to_float2(v.w); acc[6] += f.x; acc[7] += f.y;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) sm_part[r * D + chunk * 8 + e] = acc[e];
    } else {
      float acc[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) acc[e] = 0.f;
      const float *sc = c.scale + (size_t)s * c.L_cap;
#pragma unroll 2
      for (int t = t0 + r; t < t1; t += rows) {
        const bool o = (unsigned)(t - src.ovr_t0) < (unsigned)src.ovr_n;
        const uint4 v = o ? *reinterpret_cast<const uint4 *>(obase + (size_t)(t - src.ovr_t0) * row_bytes)
                          : ldg_stream(base + (size_t)t * row_bytes);
        const float st = o ? src.ovr_scale[t - src.ovr_t0] : __ldg(sc + t);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 lo = f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)(w4[q] & 0xFFFF)));
          const float2 hi = f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)(w4[q] >> 16)));
          acc[4 * q + 0] = fmaf(st, lo.x, acc[4 * q + 0]);
          acc[4 * q + 1] = fmaf(st, lo.y, acc[4 * q + 1]);
          acc[4 * q + 2] = fmaf(st, hi.x, acc[4 * q + 2]);
          acc[4 * q + 3] = fmaf(st, hi.y, acc[4 * q + 3]);
        }
      }
#pragma unroll
      for (int e = 0; e < 16; ++e) sm_part[r * D + chunk * 16 + e] = acc[e];
    }
  }
  __syncthreads();
  if (tid < D) {
    float tot = 0.f;
    for (int rr = 0; rr < rows; ++rr) tot += sm_part[rr * D + tid];
    sm_out[tid] = tot;
  }
  __syncthreads();
}

}  // namespace misa
