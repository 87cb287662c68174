// Block-wide sum of a range of dequantised index keys (shared by the pool and
// router kernels).  Launch shape: 128 threads.
#pragma once

#include "common.cuh"

namespace misa {

constexpr int KEYSUM_THREADS = 128;

// Plain (coherent) 16-byte load: used where the same kernel wrote the data.
__device__ __forceinline__ uint4 ld_coherent(const void *p) { return *reinterpret_cast<const uint4 *>(p); }

// Sum of keys [t0, t1) of sequence s into sm_out[128] (fp32), block-wide.
// FRESH: the keys may have been written earlier in this kernel, so the
// non-coherent read-only path must not be used.
template <bool FRESH>
__device__ void block_key_sum(const CacheView &c, int s, int t0, int t1, float *sm_part /*[16][128]*/,
                              float *sm_out /*[128]*/) {
  // Every thread of the block must call this (it holds two barriers); the
  // first 128 threads do the work.
  const int tid = threadIdx.x;
  const bool worker = tid < KEYSUM_THREADS;
  const int rows = c.fp8 ? 16 : 8;
  if (worker) {
    if (!c.fp8) {
      // 16 lanes cover one 256-byte row; 8 rows per sweep.
      const int chunk = tid & 15, r = tid >> 4;
      float acc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = 0.f;
      const uint16_t *base = static_cast<const uint16_t *>(c.keys) + ((size_t)s * c.L_cap) * D + chunk * 8;
#pragma unroll 4
      for (int t = t0 + r; t < t1; t += 8) {
        uint4 v = FRESH ? ld_coherent(base + (size_t)t * D) : ldg_stream(base + (size_t)t * D);
        float2 f;
        f = bf16x2_to_float2(v.x); acc[0] += f.x; acc[1] += f.y;
        f = bf16x2_to_float2(v.y); acc[2] += f.x; acc[3] += f.y;
        f = bf16x2_to_float2(v.z); acc[4] += f.x; acc[5] += f.y;
        f = bf16x2_to_float2(v.w); acc[6] += f.x; acc[7] += f.y;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) sm_part[r * D + chunk * 8 + e] = acc[e];
    } else {
      // 8 lanes cover one 128-byte row; 16 rows per sweep.
      const int chunk = tid & 7, r = tid >> 3;
      float acc[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) acc[e] = 0.f;
      const uint8_t *base = static_cast<const uint8_t *>(c.keys) + ((size_t)s * c.L_cap) * D + chunk * 16;
      const float *sc = c.scale + (size_t)s * c.L_cap;
#pragma unroll 2
      for (int t = t0 + r; t < t1; t += 16) {
        uint4 v = FRESH ? ld_coherent(base + (size_t)t * D) : ldg_stream(base + (size_t)t * D);
        const float st = FRESH ? sc[t] : __ldg(sc + t);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float2 lo = f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)(w4[q] & 0xFFFF)));
          float2 hi = f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)(w4[q] >> 16)));
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
  if (worker) {
    float tot = 0.f;
    for (int rr = 0; rr < rows; ++rr) tot += sm_part[rr * D + tid];
    sm_out[tid] = tot;
  }
  __syncthreads();
}

}  // namespace misa
