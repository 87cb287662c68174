// Token scoring on the warp-level tensor path (decode and re-rank).
//
// Computes, for each query row i and each scored token t,
//     I_t = s_t * sum_{n < h} w_{i,S_n} * ReLU(q_{i,S_n} . k_t)
// ("MISA: Mixture of Indexer Sparse Attention for Long-Context LLM
// Inference", technical summary: "Methodology: MISA" step 2 with the routed
// heads S; "Problem statement" (dense DSA) with S = all H_I heads).
//
// One query per CTA row of the grid and a contiguous token range per CTA:
// this is the shape of single-query decode, where a query has one key stream
// and no other query shares it, so the kernel is bound by the key read.  The
// per-token work (h x 128 MACs on 128..256 key bytes) is done by mma.sync
// m16n8k16 with 16 tokens as the M side and 8 routed heads per n-tile as the
// N side; fp32 accumulation.  Keys go straight from HBM to registers (16-byte
// loads, one token row per 8 lanes group) -- no shared-memory staging -- and
// the k dimension is permuted so that each 16-byte load feeds whole A
// fragments; the routed query heads are packed in shared memory with the same
// permutation.  e4m3 keys are widened to f16 (exact); their queries are
// rounded to f16 (exact for the query magnitudes that occur) and s_t is
// applied once per token after the head reduction (s_t > 0 commutes with
// ReLU).  The ReLU, w-weighting and head reduction happen in registers: the
// per-head products never leave the SM.
#include "internal.h"

namespace misa {
namespace {

constexpr int SC_THREADS = 256;
constexpr int SC_WARPS = SC_THREADS / 32;
constexpr int KT = 8;  // k-tiles of 16 over d = 128

template <int NT, bool FP8, bool GATHER>
__global__ void __launch_bounds__(SC_THREADS) score_mma_kernel(CacheView c, QueryView qv, const int32_t *heads,
                                                               int h, const int32_t *gather, int n_cols,
                                                               float *scores, long long ld, int chunk) {
  __shared__ uint2 bfrag[KT * NT * 32];  // B fragments, [kt][nt][lane]
  __shared__ float w_s[NT * 8];
  const int i = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, cq = lane & 3;
  int s;
  const int Li = query_prefix(c, qv, i, &s);
  const int ncols = GATHER ? n_cols : Li;
  const int col0 = blockIdx.x * chunk;
  if (col0 >= ncols) return;
  const int col1 = min(col0 + chunk, ncols);
  const int H = qv.H;
  const int h_eff = heads ? h : H;

  // Pack the scoring heads' queries as B fragments (k permuted to match the
  // key loads below).  bf16 k-tile kt = 2*ch + u covers physical elements
  // 32ch + 8cq + 4u + {0,1} (fragment b0) and +{2,3} (b1); the f16 (fp8 key)
  // k-tile kt = 4*ch + u covers 64ch + 16cq + 4u + {0,1} and +{2,3}.
  for (int e = tid; e < KT * NT * 32; e += SC_THREADS) {
    const int l = e & 31, nt = (e >> 5) % NT, kt = (e >> 5) / NT;
    const int n = nt * 8 + (l >> 2), c4 = l & 3;
    uint2 v = make_uint2(0u, 0u);
    if (n < h_eff) {
      int j = heads ? heads[(size_t)i * h + n] : n;
      if (j < 0 || j >= H) {
        flag(c, MISA_DEV_BAD_HEAD);
        j = 0;
      }
      const uint16_t *qrow = qv.q + ((size_t)i * H + j) * D;
      int off;
      if (FP8) {
        const int ch = kt >> 2, u = kt & 3;
        off = 64 * ch + 16 * c4 + 4 * u;
      } else {
        const int ch = kt >> 1, u = kt & 1;
        off = 32 * ch + 8 * c4 + 4 * u;
      }
      uint32_t p0 = *reinterpret_cast<const uint32_t *>(qrow + off);
      uint32_t p1 = *reinterpret_cast<const uint32_t *>(qrow + off + 2);
      if (FP8) {
        p0 = bf16x2_to_f16x2(p0);
        p1 = bf16x2_to_f16x2(p1);
      }
      v = make_uint2(p0, p1);
    }
    bfrag[e] = v;
  }
  if (tid < NT * 8) {
    float wv = 0.f;
    if (tid < h_eff) {
      const int j = heads ? heads[(size_t)i * h + tid] : tid;
      wv = (j >= 0 && j < H) ? qv.w[(size_t)i * H + j] : 0.f;
    }
    w_s[tid] = wv;
  }
  __syncthreads();
  float wr[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    wr[nt][0] = w_s[nt * 8 + 2 * cq];
    wr[nt][1] = w_s[nt * 8 + 2 * cq + 1];
  }

  const size_t row_bytes = FP8 ? D : 2 * D;
  const uint8_t *kbase = static_cast<const uint8_t *>(c.keys) + (size_t)s * c.L_cap * row_bytes;
  const float *sbase = FP8 ? c.scale + (size_t)s * c.L_cap : nullptr;
  constexpr int NV = FP8 ? 2 : 4;  // 16-byte loads per row per thread

  for (int r0 = col0 + warp * 16; r0 < col1; r0 += SC_WARPS * 16) {
    // token rows of this lane: r0 + g and r0 + g + 8
    int tok[2];
    bool ok[2];
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int p = r0 + g + 8 * hr;
      int t = p;
      bool v = p < col1;
      if (GATHER) {
        t = v ? gather[(size_t)i * n_cols + p] : -1;
        v = v && t >= 0 && t < Li;
      }
      ok[hr] = v;
      tok[hr] = v ? t : 0;
    }
    uint4 kv[2][NV];
#pragma unroll
    for (int hr = 0; hr < 2; ++hr)
#pragma unroll
      for (int ch = 0; ch < NV; ++ch)
        kv[hr][ch] = ldg_stream(kbase + (size_t)tok[hr] * row_bytes + 64 * ch + 16 * cq);

    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
    for (int kt = 0; kt < KT; ++kt) {
      uint32_t a[4];
      if (FP8) {
        const int ch = kt >> 2, u = kt & 3;
        const uint32_t wA = (&kv[0][ch].x)[u], wB = (&kv[1][ch].x)[u];
        a[0] = e4m3x2_to_f16x2((uint16_t)(wA & 0xFFFF));
        a[1] = e4m3x2_to_f16x2((uint16_t)(wB & 0xFFFF));
        a[2] = e4m3x2_to_f16x2((uint16_t)(wA >> 16));
        a[3] = e4m3x2_to_f16x2((uint16_t)(wB >> 16));
      } else {
        const int ch = kt >> 1, u = kt & 1;
        const uint4 A = kv[0][ch], Bv = kv[1][ch];
        a[0] = u ? A.z : A.x;
        a[1] = u ? Bv.z : Bv.x;
        a[2] = u ? A.w : A.y;
        a[3] = u ? Bv.w : Bv.y;
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint2 b = bfrag[(kt * NT + nt) * 32 + lane];
        if (FP8)
          mma_f16_16816(acc[nt], a, b.x, b.y);
        else
          mma_bf16_16816(acc[nt], a, b.x, b.y);
      }
    }
    float sum0 = 0.f, sum1 = 0.f;  // rows g and g + 8
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
    if (cq < 2) {
      const int hr = cq;
      const float v = hr ? sum1 : sum0;
      if (ok[hr]) {
        const float st = FP8 ? __ldg(sbase + tok[hr]) : 1.f;
        scores[(size_t)i * ld + (r0 + g + 8 * hr)] = v * st;
      }
    }
  }
}

template <int NT, bool FP8, bool GATHER>
cudaError_t launch_nt(dim3 grid, const CacheView &c, const QueryView &q, const int32_t *heads, int h,
                      const int32_t *gather, int n_cols, float *scores, long long ld, int chunk, cudaStream_t s) {
  score_mma_kernel<NT, FP8, GATHER><<<grid, SC_THREADS, 0, s>>>(c, q, heads, h, gather, n_cols, scores, ld, chunk);
  return cudaGetLastError();
}

template <bool FP8, bool GATHER>
cudaError_t launch_dt(int NT, dim3 grid, const CacheView &c, const QueryView &q, const int32_t *heads, int h,
                      const int32_t *gather, int n_cols, float *scores, long long ld, int chunk, cudaStream_t s) {
  switch (NT) {
    case 1: return launch_nt<1, FP8, GATHER>(grid, c, q, heads, h, gather, n_cols, scores, ld, chunk, s);
    case 2: return launch_nt<2, FP8, GATHER>(grid, c, q, heads, h, gather, n_cols, scores, ld, chunk, s);
    case 4: return launch_nt<4, FP8, GATHER>(grid, c, q, heads, h, gather, n_cols, scores, ld, chunk, s);
    case 8: return launch_nt<8, FP8, GATHER>(grid, c, q, heads, h, gather, n_cols, scores, ld, chunk, s);
    case 16: return launch_nt<16, FP8, GATHER>(grid, c, q, heads, h, gather, n_cols, scores, ld, chunk, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_score_mma(const CacheView &c, const QueryView &q, const int32_t *heads, int h,
                             const int32_t *gather, int n_cols, float *scores, long long ld, cudaStream_t s) {
  if (q.n_q == 0) return cudaSuccess;
  const int h_eff = heads ? h : q.H;
  int NT = 1;
  while (NT * 8 < h_eff) NT *= 2;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int cols = gather ? n_cols : c.L_cap;
  // enough CTAs for ~4 per SM, each a multiple of 16 tokens per warp
  const int quantum = SC_WARPS * 16;
  int splits = max(1, cdiv(4 * sms, q.n_q));
  splits = min(splits, cdiv(cols, quantum));
  const int chunk = cdiv(cdiv(cols, splits), quantum) * quantum;
  splits = cdiv(cols, chunk);
  dim3 grid(splits, q.n_q);
  if (c.fp8)
    return gather ? launch_dt<true, true>(NT, grid, c, q, heads, h, gather, n_cols, scores, ld, chunk, s)
                  : launch_dt<true, false>(NT, grid, c, q, heads, h, gather, n_cols, scores, ld, chunk, s);
  return gather ? launch_dt<false, true>(NT, grid, c, q, heads, h, gather, n_cols, scores, ld, chunk, s)
                : launch_dt<false, false>(NT, grid, c, q, heads, h, gather, n_cols, scores, ld, chunk, s);
}

}  // namespace misa
