// Warp-level tensor-core fragments shared by the token-scoring kernels.
//
// A 16-token tile of keys is the M side of mma.sync, the scoring heads (8 per
// n-tile) the N side, d = 128 the K side; fp32 accumulation.  The k dimension
// is permuted so that each lane's 16-byte loads of a key row feed whole A
// fragments: lane (g = lane/4, c = lane%4) reads bytes 64*ch + 16*c of rows g
// and g+8 (ch = 0..3 for bf16 rows of 256 B, 0..1 for e4m3 rows of 128 B).
// The query fragments use the same permutation, so the dot products are
// unchanged.
//
// bf16 keys: m16n8k16 bf16 MMA, keys used as stored.
// e4m3 keys: m16n8k32 e4m3 MMA, keys used as stored (no widening).  Each bf16
//   query head q_n is scaled by 2^e_n (exact; max|q_n| * 2^e_n in [64, 128))
//   and split into two e4m3 terms, q1 = RN(q) and q2 = RN(q - q1).  A bf16
//   value has 8 significant bits and q1 keeps 4, so the residual has at most
//   4 and q1 + q2 == q exactly unless the residual falls below the e4m3
//   subnormal step (elements under 2^-9 of the head's largest one; their
//   error is below 2^-10 of the scaled value).  Both terms accumulate into
//   the same fp32 accumulator; 2^-e_n is folded into the head weight.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace misa {

template <bool FP8>
struct FragCfg {
  static constexpr int KT = FP8 ? 4 : 8;      // k-tiles over d = 128
  static constexpr int TERMS = FP8 ? 2 : 1;   // query terms per k-tile
  static constexpr int NV = FP8 ? 2 : 4;      // 16-byte chunks per row and lane
  static constexpr int ROW = FP8 ? D : 2 * D; // bytes per key row
};

__device__ __forceinline__ void mma_e4m3_16832(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two fp32 -> two e4m3 codes (low byte = first), round to nearest, saturating.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float a, float b) {
  return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint32_t v) {
  return f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)v));
}

// 8 consecutive bf16 query elements scaled by `scale` -> two e4m3 terms (8 codes each).
__device__ __forceinline__ void split_e4m3(uint4 q8, float scale, uint2 &t1, uint2 &t2) {
  const uint32_t w[4] = {q8.x, q8.y, q8.z, q8.w};
  uint32_t c1[4], c2[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const float2 f = bf16x2_to_float2(w[p]);
    const float a = f.x * scale, b = f.y * scale;
    c1[p] = f32x2_to_e4m3x2(a, b);
    const float2 back = e4m3x2_to_f32x2(c1[p]);
    c2[p] = f32x2_to_e4m3x2(a - back.x, b - back.y);
  }
  t1 = make_uint2(c1[0] | (c1[1] << 16), c1[2] | (c1[3] << 16));
  t2 = make_uint2(c2[0] | (c2[1] << 16), c2[2] | (c2[3] << 16));
}

// 2^(7 - E) for max = m * 2^E, m in [0.5, 1): max * scale in [64, 128).
__device__ __forceinline__ float e4m3_head_scale(float amax) {
  if (!(amax > 0.f) || !isfinite(amax)) return 1.f;
  const int E = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 126;
  const int e = min(max(7 - E, -100), 100);
  return ldexpf(1.f, e);
}

// Scoring-head query fragments and weights in shared memory.
//   bfrag [KT][TERMS][NT][32] uint2, w_s [NT*8] (head weight / query scale),
//   scale_s [NT*8] scratch.
// heads == nullptr: all H heads; slots >= h_eff are zero.  sheads != nullptr:
// the h heads of this query in shared memory (heads is then ignored).
// Threads [0, NTHR) must all call; `sync` is a barrier over exactly those
// threads, and one more is needed before the fragments are read.  Loops have
// fixed trip counts so every load is issued before it is used.
// QSmem: the query already sits in shared memory (qrow(j): head j's row,
// w_in: its H weights); QGlobal: it is read from qv.
struct QGlobal {};
template <class QRow>
struct QSmem {
  QRow qrow;
  const float *w_in;
};

template <int NT, bool FP8, int NTHR, class Sync, class QSrc = QGlobal>
__device__ __forceinline__ void build_query_frags(const CacheView &c, const QueryView &qv, int i,
                                                  const int32_t *heads, int h, uint2 *bfrag, float *w_s,
                                                  float *scale_s, int tid, Sync sync,
                                                  const int32_t *sheads = nullptr, QSrc qsrc = QSrc()) {
  using F = FragCfg<FP8>;
  constexpr bool GQ = std::is_same<QSrc, QGlobal>::value;
  const int H = qv.H;
  auto row_of = [&](int j) -> const uint16_t * {
    if constexpr (GQ)
      return qv.q + ((size_t)i * H + j) * D;
    else
      return qsrc.qrow(j);
  };
  auto ld16 = [&](const void *p) -> uint4 {
    if constexpr (GQ)
      return __ldg(reinterpret_cast<const uint4 *>(p));
    else
      return *reinterpret_cast<const uint4 *>(p);
  };
  auto ld8 = [&](const void *p) -> uint2 {
    if constexpr (GQ)
      return __ldg(reinterpret_cast<const uint2 *>(p));
    else
      return *reinterpret_cast<const uint2 *>(p);
  };
  const int h_eff = (heads || sheads) ? h : H;
  auto head_of = [&](int n) -> int {
    int j = sheads ? sheads[n] : heads ? __ldg(heads + (size_t)i * h + n) : n;
    if (j < 0 || j >= H) {
      flag(c, MISA_DEV_BAD_HEAD);
      j = 0;
    }
    return j;
  };
  static_assert(NT * 8 <= NTHR, "one thread per head slot");
  const int n_me = tid;  // head slot owned by this thread (if < NT*8)
  if (FP8) {
    float sc = 1.f;
    if (n_me < NT * 8 && n_me < h_eff) {
      const uint4 *row = reinterpret_cast<const uint4 *>(row_of(head_of(n_me)));
      uint4 v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) v[u] = ld16(row + u);
      float m = 0.f;
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const uint32_t ww[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const float2 f = bf16x2_to_float2(ww[p]);
          m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
      }
      sc = e4m3_head_scale(m);
    }
    if (n_me < NT * 8) scale_s[n_me] = sc;
    sync();
  }
  // fragments: entry e = (kt*NT + nt)*32 + lane of term t is stored at
  // ((kt*TERMS + t)*NT + nt)*32 + lane
  constexpr int ENTRIES = F::KT * NT * 32;
  constexpr int PER = (ENTRIES + NTHR - 1) / NTHR;
  int hd[PER];
#pragma unroll
  for (int it = 0; it < PER; ++it) {
    const int e = tid + it * NTHR;
    const int n = ((e >> 5) % NT) * 8 + ((e & 31) >> 2);
    hd[it] = (e < ENTRIES && n < h_eff) ? head_of(n) : -1;
  }
  uint4 raw[PER];
#pragma unroll
  for (int it = 0; it < PER; ++it) {
    const int e = tid + it * NTHR;
    const int kt = (e >> 5) / NT, c4 = e & 3;
    raw[it] = make_uint4(0u, 0u, 0u, 0u);
    if (hd[it] >= 0) {
      const uint16_t *qrow = row_of(hd[it]);
      if (FP8) {
        // k-tile kt = 2ch + u: a0/b0 <- elements 64ch + 16c + 8u + 0..3, a2/b1 <- + 4..7
        raw[it] = ld16(qrow + 64 * (kt >> 1) + 16 * c4 + 8 * (kt & 1));
      } else {
        // k-tile kt = 2ch + u: a0/b0 <- elements 32ch + 8c + 4u + 0..1, a2/b1 <- + 2..3
        const uint2 v = ld8(qrow + 32 * (kt >> 1) + 8 * c4 + 4 * (kt & 1));
        raw[it].x = v.x;
        raw[it].y = v.y;
      }
    }
  }
#pragma unroll
  for (int it = 0; it < PER; ++it) {
    const int e = tid + it * NTHR;
    if (e >= ENTRIES) continue;
    const int l = e & 31, nt = (e >> 5) % NT, kt = (e >> 5) / NT;
    const int n = nt * 8 + (l >> 2);
    uint2 t1 = make_uint2(raw[it].x, raw[it].y), t2 = make_uint2(0u, 0u);
    if (FP8 && hd[it] >= 0) split_e4m3(raw[it], scale_s[n], t1, t2);
    bfrag[((kt * F::TERMS + 0) * NT + nt) * 32 + l] = t1;
    if (FP8) bfrag[((kt * F::TERMS + 1) * NT + nt) * 32 + l] = t2;
  }
  if (n_me < NT * 8) {
    float wv = 0.f;
    if (n_me < h_eff) {
      if constexpr (GQ)
        wv = __ldg(qv.w + (size_t)i * H + head_of(n_me));
      else
        wv = qsrc.w_in[head_of(n_me)];
      if (FP8) wv /= scale_s[n_me];  // exact: power of two
    }
    w_s[n_me] = wv;
  }
}

// Accumulate one 16-token tile: kv[0] holds row g's chunks, kv[1] row g+8's.
template <int NT, bool FP8>
__device__ __forceinline__ void tile_mma(const uint4 (&kv)[2][FragCfg<FP8>::NV], const uint2 *bfrag, int lane,
                                         float (&acc)[NT][4]) {
  using F = FragCfg<FP8>;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
  for (int kt = 0; kt < F::KT; ++kt) {
    const int ch = kt >> 1, u = kt & 1;
    const uint4 A = kv[0][ch], Bv = kv[1][ch];
    uint32_t a[4];
    a[0] = u ? A.z : A.x;
    a[1] = u ? Bv.z : Bv.x;
    a[2] = u ? A.w : A.y;
    a[3] = u ? Bv.w : Bv.y;
#pragma unroll
    for (int t = 0; t < F::TERMS; ++t)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint2 b = bfrag[((kt * F::TERMS + t) * NT + nt) * 32 + lane];
        if (FP8)
          mma_e4m3_16832(acc[nt], a, b.x, b.y);
        else
          mma_bf16_16816(acc[nt], a, b.x, b.y);
      }
  }
}

// As tile_mma, with the query fragments already in registers
// (b[(kt*TERMS + t)*NT + nt], used when NT is small).
template <int NT, bool FP8>
__device__ __forceinline__ void tile_mma_reg(const uint4 (&kv)[2][FragCfg<FP8>::NV],
                                             const uint2 (&b)[FragCfg<FP8>::KT * FragCfg<FP8>::TERMS * NT],
                                             float (&acc)[NT][4]) {
  using F = FragCfg<FP8>;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
  for (int kt = 0; kt < F::KT; ++kt) {
    const int ch = kt >> 1, u = kt & 1;
    const uint4 A = kv[0][ch], Bv = kv[1][ch];
    uint32_t a[4];
    a[0] = u ? A.z : A.x;
    a[1] = u ? Bv.z : Bv.x;
    a[2] = u ? A.w : A.y;
    a[3] = u ? Bv.w : Bv.y;
#pragma unroll
    for (int t = 0; t < F::TERMS; ++t)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint2 bb = b[(kt * F::TERMS + t) * NT + nt];
        if (FP8)
          mma_e4m3_16832(acc[nt], a, bb.x, bb.y);
        else
          mma_bf16_16816(acc[nt], a, bb.x, bb.y);
      }
  }
}

// ReLU, head weights and the reduction over heads: returns (row g, row g+8)
// totals, identical in the 4 lanes of a row group.
template <int NT>
__device__ __forceinline__ float2 tile_reduce(const float (&acc)[NT][4], const float (&wr)[NT][2]) {
  float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    sum0 = fmaf(wr[nt][0], fmaxf(acc[nt][0], 0.f), sum0);
    sum0 = fmaf(wr[nt][1], fmaxf(acc[nt][1], 0.f), sum0);
    sum1 = fmaf(wr[nt][0], fmaxf(acc[nt][2], 0.f), sum1);
    sum1 = fmaf(wr[nt][1], fmaxf(acc[nt][3], 0.f), sum1);
  }
  sum0 += __shfl_xor_sync(0xffffffffu, sum0, 1);
  sum0 += __shfl_xor_sync(0xffffffffu, sum0, 2);
  sum1 += __shfl_xor_sync(0xffffffffu, sum1, 1);
  sum1 += __shfl_xor_sync(0xffffffffu, sum1, 2);
  return make_float2(sum0, sum1);
}

}  // namespace misa
