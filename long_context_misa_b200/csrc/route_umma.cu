// Block-pooled head router for prefill chunks on the tcgen05 tensor cores.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference",
// technical summary, "Methodology: MISA", step 1: per-head affinities against
// the mean-pooled index keys, aggregated into a head importance, then the
// top-h heads:
//     r_j = |w_j| * sum_{m < M_i} ReLU(q_j . kbar_m),   M_i = ceil(L_i / B),
// the block cut by the query's prefix end being the mean of its keys up to
// the query (routing never sees a future token).
//
// For many queries per sequence the affinities of all whole blocks form one
// dense product: 128 query-head rows (the query matrix [n_q * H][128] read
// as is) on the MMA M side, 128 pooled blocks on N, d = 128 on K.  The fp32
// pool is split into bf16 hi + lo (hi = RN(k), lo = RN(k - hi)) once per
// call and both terms accumulate into the same tensor-memory columns, which
// keeps ~16 significant bits of the pooled key with exact products and fp32
// sums -- the precision of the mma.sync router.  The epilogue sums ReLU of a
// row over the blocks wholly inside its query's prefix; a second kernel adds
// the causal tail block in fp32 and keeps the top-h heads.
//
// route_umma_kernel: one CTA per group of 128 rows, two CTAs per SM (their
// set-up latencies overlap); warp 0 issues TMA loads (the group's query rows,
// then hi/lo pool tiles of 64 blocks into a 2-stage ring), warp 1 owns the
// tensor memory and issues the MMAs, warps 2..5 drain two accumulator
// buffers of 64 columns.  When the group holds whole queries (H divides 128,
// 16 <= H) the same CTA finishes them: the tail block's mean, its affinity
// with each head (query rows still in shared memory), r and the top-h heads;
// otherwise route_tail_finish_kernel does that from the row sums.
#include <algorithm>

#include "internal.h"
#include "keysum.cuh"
#include "umma.cuh"

namespace misa {
namespace {

constexpr int RU_M = 128;              // query-head rows per group
constexpr int RU_N = 64;               // pooled blocks per tile
constexpr int RU_STAGES = 2;
constexpr int RU_THREADS = 192;        // TMA warp, MMA warp, 4 epilogue warps
constexpr int RU_A_BYTES = RU_M * 256; // the group's rows: bf16, two 128-byte K blocks
constexpr int RU_B_TERM = RU_N * 256;  // one pool term of a tile
constexpr int RU_B_STAGE = 2 * RU_B_TERM;

struct RouteShared {
  uint64_t afull, full[RU_STAGES], empty[RU_STAGES], tfull[2], tempty[2];
  uint32_t tmem_base;
  int abort;
  int n_pass;
  int first_seq, multi, max_full;  // one-sequence fast path of the pass set-up
  int pass_seq[RU_M];   // distinct sequences of the group's rows
  int pass_full[RU_M];  // most whole blocks among their queries
  int row_full[RU_M];   // per row: whole blocks inside its query's prefix
  int row_seq[RU_M];    // per row: its sequence (-1: no query)
  // fused finish (128 / H queries per group, at most 8); its key-sum scratch
  // and tail sums use the pool stages, idle once the group's MMAs are done
  int q_li[8], q_t0[8];
  float rsc[RU_M];      // r of every row
  int keep[RU_M];
};

constexpr int ru_smem_bytes() { return 1024 + RU_A_BYTES + RU_STAGES * RU_B_STAGE + (int)sizeof(RouteShared); }

__device__ __forceinline__ uint32_t bf2_bits(__nv_bfloat162 v) { return *reinterpret_cast<uint32_t *>(&v); }

// pool (fp32) -> hi, lo (bf16), four elements per step
__global__ void __launch_bounds__(256) pool_split_kernel(const float4 *pool, size_t n4, uint2 *hi, uint2 *lo) {
  grid_dep_sync();
  for (size_t x = blockIdx.x * (size_t)256 + threadIdx.x; x < n4; x += (size_t)gridDim.x * 256) {
    const float4 v = __ldg(pool + x);
    const __nv_bfloat162 h01 = __floats2bfloat162_rn(v.x, v.y), h23 = __floats2bfloat162_rn(v.z, v.w);
    const float2 f01 = __bfloat1622float2(h01), f23 = __bfloat1622float2(h23);
    const __nv_bfloat162 l01 = __floats2bfloat162_rn(v.x - f01.x, v.y - f01.y);
    const __nv_bfloat162 l23 = __floats2bfloat162_rn(v.z - f23.x, v.w - f23.y);
    hi[x] = make_uint2(bf2_bits(h01), bf2_bits(h23));
    lo[x] = make_uint2(bf2_bits(l01), bf2_bits(l23));
  }
}

__global__ void __launch_bounds__(RU_THREADS, 2)
    route_umma_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap hmap,
                      const __grid_constant__ CUtensorMap lmap, CacheView c, QueryView qv, float *rsum,
                      int n_groups, int fuse, int h, int32_t *heads, float *router_scores, int agg) {
  grid_dep_sync();
  extern __shared__ uint8_t ru_raw[];
  uint8_t *base = aligned_smem_base(ru_raw, ru_smem_bytes() - 1024, c);  // 1024-aligned (swizzle atoms)
  if (!base) return;
  uint8_t *a_smem = base;
  uint8_t *b_smem = base + RU_A_BYTES;
  RouteShared &sh = *reinterpret_cast<RouteShared *>(b_smem + RU_STAGES * RU_B_STAGE);
  volatile int *abort = &sh.abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = qv.H;
  const int M_cap = cdiv(c.L_cap, c.B);

  const int per = cdiv(n_groups, (int)gridDim.x);
  const int g0 = min(n_groups, (int)blockIdx.x * per), g1 = min(n_groups, g0 + per);
  if (g0 >= g1) return;  // uniform; nothing allocated yet

  if (tid == 0) {
    mbar_init(&sh.afull, 1);
    for (int s = 0; s < RU_STAGES; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh.tfull[b], 1);
      mbar_init(&sh.tempty[b], 4);
    }
    sh.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&sh.tmem_base)),
                 "n"(2 * RU_N));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    umma::fence_before();
  }
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = sh.tmem_base;

  uint32_t it_load = 0, it_mma = 0, j_mma = 0, j_epi = 0, a_phase = 0;
  int last_fill[RU_STAGES];
#pragma unroll
  for (int s = 0; s < RU_STAGES; ++s) last_fill[s] = -1;
  bool a_loaded = false, mma_issued = false;

  for (int g = g0; g < g1 && !*abort; ++g) {
    // ---- the group's rows: query, sequence, whole blocks ----
    if (tid == 0) {
      sh.first_seq = -1;
      sh.multi = 0;
      sh.max_full = 0;
    }
    for (int r = tid; r < RU_M; r += RU_THREADS) {
      const int row = g * RU_M + r, qi = row / H;
      int s = -1, Li = 0;
      if (qi < qv.n_q) Li = query_prefix(c, qv, qi, &s);
      sh.row_full[r] = Li / c.B;
      sh.row_seq[r] = (Li / c.B) > 0 ? s : -1;
    }
    if (warp == 0 && lane == 0) {  // the group's query rows (rows beyond n_q * H read as zeros)
      mbar_arrive_expect_tx(&sh.afull, RU_A_BYTES);
      const uint32_t dst = smem_addr(a_smem);
      umma::tma_load_2d(dst, &qmap, 0, g * RU_M, &sh.afull);
      umma::tma_load_2d(dst + RU_M * 128, &qmap, 64, g * RU_M, &sh.afull);
      a_loaded = true;
    }
    __syncthreads();
    // the rows' sequences: one (the usual case) is settled with shared atomics
    if (tid < RU_M && sh.row_seq[tid] >= 0) atomicCAS(&sh.first_seq, -1, sh.row_seq[tid]);
    __syncthreads();
    if (tid < RU_M && sh.row_seq[tid] >= 0) {
      if (sh.row_seq[tid] != sh.first_seq) sh.multi = 1;
      atomicMax(&sh.max_full, sh.row_full[tid]);
    }
    __syncthreads();
    if (tid == 0 && !sh.multi) {
      sh.n_pass = sh.first_seq >= 0 ? 1 : 0;
      sh.pass_seq[0] = sh.first_seq;
      sh.pass_full[0] = sh.max_full;
    } else if (tid == 0) {
      int np = 0;
      for (int r = 0; r < RU_M; ++r) {
        const int s = sh.row_seq[r];
        if (s < 0) continue;
        int p = 0;
        while (p < np && sh.pass_seq[p] != s) ++p;
        if (p == np) {
          sh.pass_seq[np] = s;
          sh.pass_full[np] = 0;
          ++np;
        }
        sh.pass_full[p] = max(sh.pass_full[p], sh.row_full[r]);
      }
      sh.n_pass = np;
    }
    __syncthreads();
    const int n_pass = sh.n_pass;
    float acc = 0.f;  // epilogue: this row's sum over whole blocks
    bool a_waited = false;

    for (int pass = 0; pass < n_pass; ++pass) {
      const int seq = sh.pass_seq[pass];
      const int n_tiles = cdiv(sh.pass_full[pass], RU_N);
      if (warp == 0) {
        if (lane == 0) {
          for (int t = 0; t < n_tiles; ++t, ++it_load) {
            const int st = it_load % RU_STAGES;
            if (!umma::wait_bar(&sh.empty[st], ((it_load / RU_STAGES) & 1) ^ 1, abort, c)) break;
            mbar_arrive_expect_tx(&sh.full[st], RU_B_STAGE);
            const uint32_t dst = smem_addr(b_smem + st * RU_B_STAGE);
            const int y = seq * M_cap + t * RU_N;
            umma::tma_load_2d(dst, &hmap, 0, y, &sh.full[st]);
            umma::tma_load_2d(dst + RU_N * 128, &hmap, 64, y, &sh.full[st]);
            umma::tma_load_2d(dst + RU_B_TERM, &lmap, 0, y, &sh.full[st]);
            umma::tma_load_2d(dst + RU_B_TERM + RU_N * 128, &lmap, 64, y, &sh.full[st]);
            last_fill[st] = (int)((it_load / RU_STAGES) & 1);
          }
        }
      } else if (warp == 1) {
        if (lane == 0) {
          const uint32_t idesc = umma::instr_desc<false, RU_M, RU_N>();
          const uint32_t a_base = smem_addr(a_smem);
          if (n_tiles > 0 && !a_waited) {
            if (umma::wait_bar(&sh.afull, a_phase, abort, c)) a_waited = true;
            umma::fence_after();
          }
          for (int t = 0; t < n_tiles && a_waited; ++t, ++it_mma, ++j_mma) {
            const int st = it_mma % RU_STAGES, buf = j_mma & 1;
            if (!umma::wait_bar(&sh.tempty[buf], ((j_mma >> 1) & 1) ^ 1, abort, c)) break;
            umma::fence_after();
            if (!umma::wait_bar(&sh.full[st], (it_mma / RU_STAGES) & 1, abort, c)) break;
            umma::fence_after();
            const uint32_t b_base = smem_addr(b_smem + st * RU_B_STAGE);
            const uint32_t d = tmem + buf * RU_N;
#pragma unroll
            for (int term = 0; term < 2; ++term) {
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {
                const uint32_t aoff = (kk >> 2) * (RU_M * 128) + (kk & 3) * 32;
                const uint32_t boff = (kk >> 2) * (RU_N * 128) + (kk & 3) * 32;
                umma::mma<false>(d, umma::smem_desc_sw128(a_base + aoff),
                                 umma::smem_desc_sw128(b_base + term * RU_B_TERM + boff), idesc,
                                 (term | kk) ? 1u : 0u);
              }
            }
            umma::commit(&sh.empty[st]);
            umma::commit(&sh.tfull[buf]);
            mma_issued = true;
          }
        }
      } else {
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const bool mine = sh.row_seq[r] == seq;
        const int full = sh.row_full[r];
        for (int t = 0; t < n_tiles; ++t, ++j_epi) {
          const int buf = j_epi & 1;
          if (!umma::wait_bar(&sh.tfull[buf], (j_epi >> 1) & 1, abort, c)) break;
          umma::fence_after();
          const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + buf * RU_N;
#pragma unroll
          for (int ch = 0; ch < RU_N / 32; ch += 2) {
            uint32_t v0[32], v1[32];
            umma::ld32(taddr + ch * 32, v0);
            umma::ld32(taddr + ch * 32 + 32, v1);
            umma::ld_wait();
            const int m0 = t * RU_N + ch * 32;
#pragma unroll
            for (int x = 0; x < 32; ++x) {
              const float r0 = fmaxf(__uint_as_float(v0[x]), 0.f), r1 = fmaxf(__uint_as_float(v1[x]), 0.f);
              if (mine && m0 + x < full) acc = agg_is_max(agg) ? fmaxf(acc, r0) : acc + r0;
              if (mine && m0 + 32 + x < full) acc = agg_is_max(agg) ? fmaxf(acc, r1) : acc + r1;
            }
          }
          umma::fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh.tempty[buf]);
        }
      }
      __syncthreads();  // every role is done with this pass
      if (*abort) break;
    }
    if (!fuse) {
      if (warp >= 2) {
        const int r = (warp & 3) * 32 + lane, row = g * RU_M + r;
        if (row / H < qv.n_q) rsum[row] = acc;
      }
    } else if (!*abort) {
      // ---- fused finish: the group's RU_M / H whole queries ----
      // (every pool load was consumed and every MMA committed before the
      // last pass ended, so the stages are free)
      const int QG = RU_M / H;
      float *part = reinterpret_cast<float *>(b_smem);  // [16][D] key-sum scratch
      float *tailm = part + 16 * D;                      // [QG][D] tail-block key sums
      int prev_li = 0, prev_t0 = -1, prev_s = -1;
      for (int qg = 0; qg < QG; ++qg) {  // uniform: every thread takes part in the key sums
        const int qi = g * QG + qg;
        int s = -1, Li = 0;
        if (qi < qv.n_q) Li = query_prefix(c, qv, qi, &s);
        const int t0 = (Li / c.B) * c.B;
        if (tid == 0) {
          sh.q_li[qg] = Li;
          sh.q_t0[qg] = t0;
        }
        if (Li > t0 && s == prev_s && t0 == prev_t0 && prev_li > t0 && Li >= prev_li && Li - prev_li <= 8) {
          // the previous query's tail block plus the few keys between them
          if (tid < D) {
            float a = tailm[(qg - 1) * D + tid];
            for (int t = prev_li; t < Li; ++t) {
              const size_t e = ((size_t)s * c.L_cap + t) * D + tid;
              if (c.fp8) {
                const uint8_t b = __ldg(static_cast<const uint8_t *>(c.keys) + e);
                a = fmaf(__ldg(c.scale + (size_t)s * c.L_cap + t), f16x2_to_float2(e4m3x2_to_f16x2(b)).x, a);
              } else {
                a += bf16_bits_to_float(__ldg(static_cast<const uint16_t *>(c.keys) + e));
              }
            }
            tailm[qg * D + tid] = a;
          }
        } else if (Li > t0) {
          block_key_sum<128>(c, s, t0, Li, part, tailm + qg * D);
        }
        __syncthreads();
        prev_li = Li;
        prev_t0 = t0;
        prev_s = s;
      }
      __syncthreads();
      if (warp >= 2) {
        const int r = (warp & 3) * 32 + lane, qg = r / H, hd = r % H, qi = g * QG + qg;
        float rr = 0.f;
        if (qi < qv.n_q) {
          const int Li = sh.q_li[qg], t0 = sh.q_t0[qg];
          float a = acc;
          if (Li > t0 && umma::wait_bar(&sh.afull, a_phase, abort, c)) {  // the query rows in shared memory
            float dot = 0.f;
#pragma unroll 4
            for (int u = 0; u < 16; ++u) {
              const uint4 v = *reinterpret_cast<const uint4 *>(a_smem + (u >> 3) * (RU_M * 128) + r * 128 +
                                                               (((u & 7) ^ (r & 7)) << 4));
              const uint32_t ww[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int p = 0; p < 4; ++p) {
                const float2 f = bf16x2_to_float2(ww[p]);
                dot = fmaf(f.x, tailm[qg * D + 8 * u + 2 * p], dot);
                dot = fmaf(f.y, tailm[qg * D + 8 * u + 2 * p + 1], dot);
              }
            }
            const float rt = fmaxf(dot * (1.f / (float)(Li - t0)), 0.f);
            a = agg_is_max(agg) ? fmaxf(a, rt) : a + rt;
          }
          rr = agg_weight(agg, __ldg(qv.w + (size_t)qi * H + hd)) * a;
          if (router_scores) router_scores[(size_t)qi * H + hd] = rr;
        }
        sh.rsc[r] = rr;
      }
      __syncthreads();
      if (warp >= 2) {  // head hd is kept iff fewer than h heads beat it (larger r, or equal r and lower index)
        const int r = (warp & 3) * 32 + lane, qg = r / H, hd = r % H;
        const float rr = sh.rsc[r];
        int beaten = 0;
        for (int o = 0; o < H; ++o) {
          const float ro = sh.rsc[qg * H + o];
          beaten += (ro > rr) || (ro == rr && o < hd);
        }
        sh.keep[r] = beaten < h;
      }
      __syncthreads();
      if (warp >= 2) {  // kept heads in ascending order
        const int r = (warp & 3) * 32 + lane, qg = r / H, hd = r % H, qi = g * QG + qg;
        if (qi < qv.n_q && sh.keep[r]) {
          int pos = 0;
          for (int o = 0; o < hd; ++o) pos += sh.keep[qg * H + o];
          if (pos < h) heads[(size_t)qi * h + pos] = hd;  // a NaN score can break the strict order
        }
      }
    }
    a_phase ^= 1;
    __syncthreads();  // the group's rows and tables are free again
  }

  // ---- wind-down: nothing in flight when the tensor memory is released ----
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < RU_STAGES; ++s)
      if (last_fill[s] >= 0) umma::wait_bar(&sh.full[s], (uint32_t)last_fill[s], abort, c);
    if (a_loaded) umma::wait_bar(&sh.afull, a_phase ^ 1, abort, c);
  }
  if (warp == 1 && lane == 0 && mma_issued) {
    const uint32_t jl = j_mma - 1;
    umma::wait_bar(&sh.tfull[jl & 1], (jl >> 1) & 1, abort, c);
  }
  umma::fence_before();
  __syncthreads();
  if (warp == 1) {
    umma::fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(2 * RU_N));
  }
}

// One CTA per query: the causal tail block (mean of the keys from the last
// whole block to the query) in fp32, r_j = |w_j| * (whole-block sum + ReLU of
// the tail affinity), then the h best heads (fewer than h heads beat a kept
// one: larger r, or equal r and lower index), written in ascending order.
__global__ void __launch_bounds__(MISA_MAX_H) route_tail_finish_kernel(CacheView c, QueryView qv, const float *rsum,
                                                                       int h, int32_t *heads, float *router_scores,
                                                                       int agg) {
  grid_dep_sync();
  __shared__ float part[16 * D];
  __shared__ float tail[D];
  __shared__ float r_s[MISA_MAX_H];
  __shared__ int warp_cnt[MISA_MAX_H / 32];
  const int i = blockIdx.x, j = threadIdx.x, H = qv.H;
  int s;
  const int Li = query_prefix(c, qv, i, &s);
  const int t0 = (Li / c.B) * c.B;
  const bool has_tail = Li > t0;  // uniform
  if (has_tail) block_key_sum<MISA_MAX_H>(c, s, t0, Li, part, tail);
  __syncthreads();
  float r = 0.f;
  if (j < H) {
    float acc = rsum[(size_t)i * H + j];
    if (has_tail) {
      const float inv = 1.f / (float)(Li - t0);
      const uint4 *row = reinterpret_cast<const uint4 *>(qv.q + ((size_t)i * H + j) * D);
      float dot = 0.f;
#pragma unroll 4
      for (int u = 0; u < 16; ++u) {
        const uint4 v = __ldg(row + u);
        const uint32_t ww[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const float2 f = bf16x2_to_float2(ww[p]);
          dot = fmaf(f.x, tail[8 * u + 2 * p], dot);
          dot = fmaf(f.y, tail[8 * u + 2 * p + 1], dot);
        }
      }
      const float rt = fmaxf(dot * inv, 0.f);
      acc = agg_is_max(agg) ? fmaxf(acc, rt) : acc + rt;
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
    if (pos < h) heads[(size_t)i * h + pos] = j;
  }
}

}  // namespace

size_t route_umma_ws_bytes(int n_q, int H, int M_cap, int n_seq) {
  const size_t split = (size_t)n_seq * M_cap * D * 2;  // one bf16 term
  return 2 * ((split + 255) & ~size_t(255)) + sizeof(float) * (size_t)n_q * H;
}

bool route_umma_applies(const CacheView &c, const QueryView &q) { return umma_applies(c, q, nullptr, q.H); }

cudaError_t launch_route_umma(const CacheView &c, const QueryView &q, int h, int32_t *heads, float *router_scores,
                              void *ws, cudaStream_t s, int agg) {
  if (q.n_q == 0) return cudaSuccess;
  const int M_cap = cdiv(c.L_cap, c.B);
  const size_t split = (((size_t)c.n_seq * M_cap * D * 2) + 255) & ~size_t(255);
  uint8_t *w8 = static_cast<uint8_t *>(ws);
  uint2 *hi = reinterpret_cast<uint2 *>(w8), *lo = reinterpret_cast<uint2 *>(w8 + split);
  float *rsum = reinterpret_cast<float *>(w8 + 2 * split);
  const size_t n4 = (size_t)c.n_seq * M_cap * D / 4;
  const int sms = device_sms();
  cudaError_t e = launch_kernel(pool_split_kernel, dim3((unsigned)std::min<size_t>((n4 + 255) / 256, 4 * sms)),
                                dim3(256), 0, s, reinterpret_cast<const float4 *>(c.pool), n4, hi, lo);
  if (e != cudaSuccess) return e;
  CUtensorMap qmap, hmap, lmap;
  const unsigned long long pool_rows = (unsigned long long)c.n_seq * M_cap;
  if (!umma::make_map_2d(&qmap, q.q, false, (unsigned long long)q.n_q * q.H, 64, RU_M) ||
      !umma::make_map_2d(&hmap, hi, false, pool_rows, 64, RU_N) || !umma::make_map_2d(&lmap, lo, false, pool_rows, 64, RU_N))
    return cudaErrorNotSupported;
  constexpr int SMEM = ru_smem_bytes();
  struct Tag {};
  const int st = cached_per_device<Tag>([] {
    return 1 + (int)cudaFuncSetAttribute(route_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  });
  if (st != 1) return (cudaError_t)(st - 1);
  const int n_groups = cdiv(q.n_q * q.H, RU_M);
  const int fuse = q.H >= 16 && q.H <= RU_M && RU_M % q.H == 0;  // groups of whole queries: finish in the kernel
  e = launch_kernel(route_umma_kernel, dim3(n_groups), dim3(RU_THREADS), SMEM, s, qmap, hmap, lmap, c, q, rsum,
                    n_groups, fuse, h, heads, router_scores, agg);
  if (e != cudaSuccess || fuse) return e;
  return launch_kernel(route_tail_finish_kernel, dim3(q.n_q), dim3(MISA_MAX_H), 0, s, c, q, rsum, h, heads,
                       router_scores, agg);
}

}  // namespace misa
