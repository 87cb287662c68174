// Token scoring of prefill chunks on the fifth-generation tensor cores
// (tcgen05.mma, accumulators in tensor memory, key tiles staged by TMA).
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference",
// technical summary, "Methodology: MISA" step 2 (the routed heads S_i score
// every prefix token) and "Problem statement" (the dense indexer, S_i = all
// H_I heads):
//     I_{i,t} = s_t * sum_{j in S_i} w_{i,j} * ReLU(q_{i,j} . k_t),  t < L_i.
// The key k_t is shared by all heads, so the scoring heads of a group of
// queries stack into one matrix Q' [256 x 128] (query-major, HPQ columns per
// query, HPQ = the number of scoring heads rounded up to a power of two, at
// least 4) and
// every 128-token tile of keys is one dense MMA  D[t][n] = K[t] . Q'[n]:
// tokens on the M side, query-heads on the N side, fp32 accumulators in
// tensor memory.  The epilogue reads a token row per thread, applies ReLU and
// the weights, sums each query's HPQ columns, multiplies by s_t and writes
// the causal part of the query's score row; per-head products never reach
// global memory.
//
// bf16 keys: kind::f16 MMA on bf16 keys and the bf16 query heads.
// e4m3 keys: kind::f8f6f4 MMA on the keys as stored and an exact two-term
//   e4m3 split of each query head (scaled by a power of two folded into its
//   weight), both terms accumulating into the same tensor-memory columns.
//
// One persistent CTA per SM walks a contiguous range of (query group, token
// tile) items.  Warp 0 issues the TMA loads of key tiles into a ring of
// shared-memory stages, warp 1 (which also owns the tensor memory) issues the
// MMAs from one thread, warps 2..9 drain the accumulators (two warps per
// lane quarter, half of the columns each); two accumulator
// buffers of 256 columns let the MMAs of one tile overlap the epilogue of the
// previous.  Every wait is bounded: a wait that runs out sets
// MISA_DEV_WAIT_TIMEOUT and the CTA winds down.
#include <cuda.h>

#include <algorithm>
#include <cstring>

#include "frag.cuh"
#include "internal.h"
#include "umma.cuh"

namespace misa {
namespace {

constexpr int UM_M = 128;                 // tokens per tile
constexpr int UM_N = 256;                 // query-head columns per tile
constexpr int B_BYTES = 65536;            // Q' tile: 256 x 128 bf16, or two e4m3 terms

struct UmmaShared {
  alignas(16) float wcol[UM_N];     // weight of every column (0 for padding); read as float4
  uint64_t full[8], empty[8];       // key stages: loaded / consumed
  uint64_t tfull[2], tempty[2];     // accumulator buffers: written / drained
  uint32_t tmem_base;
  int abort;
  int n_pass;
  int pass_seq[UM_N];               // distinct sequences of the group's queries
  int pass_len[UM_N];               // longest prefix among them
  int q_len[UM_N];                  // per query of the group: prefix length (0: none)
  int q_seq[UM_N];
  int q_lenp[UM_N];                 // prefix length if the query belongs to the current pass, else 0
};

constexpr int SMEM_OPTIN = 232448;  // 227 KB of shared memory per CTA (opt-in maximum)

template <bool FP8, int HPQ>
struct UCfg {
  static constexpr int ROW = FP8 ? 128 : 256;           // key bytes per token
  static constexpr int A_BYTES = UM_M * ROW;            // one key tile
  static constexpr int KSTEPS = FP8 ? 4 : 8;            // MMAs per term and tile (K = 32 / 16)
  static constexpr int TERMS = FP8 ? 2 : 1;
  // Epilogue warps: four per tensor-memory lane quarter (a quarter of the
  // columns each) when a query spans at most 8 columns (the routed case:
  // more warps hide the latency of the ReLU / weight chains), else two (half
  // of the columns; a query never straddles two warps).
  static constexpr int SPLIT = HPQ <= 8 ? 4 : 2;
  static constexpr int EPI_WARPS = 4 * SPLIT;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int SPAN = UM_N / SPLIT;  // columns per epilogue warp
  // With 8 or 16 queries per warp's columns score tiles leave through TMA
  // stores: every epilogue warp stages its 32 tokens x QH queries in two
  // private buffers.  With fewer queries a warp writes at most 4 scores per
  // tile and plain stores are cheaper than small TMA boxes; with 32 the
  // staging would not fit.
  static constexpr int QH = SPAN / HPQ;
  static constexpr bool TMA_OUT = QH >= 8 && QH <= 16;
  static constexpr int OUT_BUF = TMA_OUT ? 32 * QH * 4 : 0;  // bytes of one staging buffer
  static constexpr int FIXED = 1024 /* alignment slack */ + B_BYTES + 2 * EPI_WARPS * OUT_BUF + (int)sizeof(UmmaShared);
  static constexpr int STAGES_MAX = FP8 ? 8 : 4;
  static constexpr int STAGES =
      (SMEM_OPTIN - FIXED) / A_BYTES < STAGES_MAX ? (SMEM_OPTIN - FIXED) / A_BYTES : STAGES_MAX;
  static constexpr int SMEM = FIXED + STAGES * A_BYTES;
  static_assert(STAGES >= 2 && SMEM <= SMEM_OPTIN, "shared memory layout");
};

// ---- the kernel -----------------------------------------------------------

// Items: (group g, tile tau) flattened as g * n_tiles + tau; this CTA takes
// [item0, item1).  A group holds QPT = 256 / HPQ consecutive queries.
template <bool FP8, int HPQ>
__global__ void __launch_bounds__(UCfg<FP8, HPQ>::THREADS, 1)
    score_umma_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap omap,
                      int out_tma, CacheView c, QueryView qv, const int32_t *heads, int h, float *scores,
                      long long ld, int n_tiles, long long n_items) {
  grid_dep_sync();
  using Cfg = UCfg<FP8, HPQ>;
  constexpr int QPT = UM_N / HPQ;
  extern __shared__ uint8_t um_raw[];
  uint8_t *base = aligned_smem_base(um_raw, Cfg::SMEM - 1024, c);  // 1024-aligned (swizzle atoms)
  if (!base) return;
  uint8_t *a_smem = base;                                    // STAGES x A_BYTES (1024-aligned each)
  uint8_t *b_smem = base + Cfg::STAGES * Cfg::A_BYTES;       // B_BYTES
  constexpr int EPI_WARPS = Cfg::EPI_WARPS, UM_THREADS = Cfg::THREADS;
  float *out_smem = reinterpret_cast<float *>(b_smem + B_BYTES);  // 2 x EPI_WARPS staging buffers
  UmmaShared &sh = *reinterpret_cast<UmmaShared *>(b_smem + B_BYTES + 2 * EPI_WARPS * Cfg::OUT_BUF);
  volatile int *abort = &sh.abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = qv.H;
  const int h_eff = heads ? h : H;

  const long long per = (n_items + gridDim.x - 1) / gridDim.x;
  const long long item0 = min(n_items, (long long)blockIdx.x * per);
  const long long item1 = min(n_items, item0 + per);
  if (item0 >= item1) return;  // uniform; nothing allocated yet

  if (tid == 0) {
    for (int s = 0; s < Cfg::STAGES; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh.tfull[b], 1);
      mbar_init(&sh.tempty[b], EPI_WARPS);
    }
    sh.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_addr(&sh.tmem_base)));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    umma::fence_before();
  }
  __syncthreads();
  umma::fence_after();
  const uint32_t tmem = sh.tmem_base;

  // pipeline counters (same sequence of tiles in every role)
  uint32_t it_load = 0, it_mma = 0, j_mma = 0, j_epi = 0;
  uint32_t ob = 0;  // epilogue: staging buffer of the next TMA store
  uint32_t last_fill_parity[8];
#pragma unroll
  for (int s = 0; s < 8; ++s) last_fill_parity[s] = 2;  // 2: never filled
  bool mma_issued = false;

  for (long long item = item0; item < item1 && !*abort;) {
    const int g = (int)(item / n_tiles);
    const int tau0 = (int)(item % n_tiles);
    const int tau1 = (int)min((long long)n_tiles, item1 - (long long)g * n_tiles);  // exclusive
    item = (long long)g * n_tiles + tau1;

    // ---- segment set-up: the group's queries, weights and Q' tile ----
    for (int ql = tid; ql < QPT; ql += UM_THREADS) {
      const int qi = g * QPT + ql;
      int s = -1, Li = 0;
      if (qi < qv.n_q) Li = query_prefix(c, qv, qi, &s);
      sh.q_len[ql] = Li;
      sh.q_seq[ql] = Li > 0 ? s : -1;
    }
    // rows n = ql * HPQ + j of Q': query g*QPT + ql, its j-th scoring head
    for (int n = tid; n < UM_N; n += UM_THREADS) {
      const int ql = n / HPQ, j = n % HPQ, qi = g * QPT + ql;
      int hd = -1;
      if (qi < qv.n_q && j < h_eff) {
        hd = heads ? __ldg(heads + (size_t)qi * h + j) : j;
        if (hd < 0 || hd >= H) {
          flag(c, MISA_DEV_BAD_HEAD);
          hd = 0;
        }
      }
      float wv = 0.f;
      const uint4 *row = reinterpret_cast<const uint4 *>(qv.q + ((size_t)(hd >= 0 ? qi : 0) * H + max(hd, 0)) * D);
      if (hd >= 0) wv = __ldg(qv.w + (size_t)qi * H + hd);
      if (!FP8) {
        // 16-byte chunk u of the row: K-block u / 8, chunk u % 8 of the 128-byte swizzled row
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint4 v[8];
#pragma unroll
          for (int x = 0; x < 8; ++x) v[x] = hd >= 0 ? __ldg(row + half * 8 + x) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
          for (int x = 0; x < 8; ++x)
            *reinterpret_cast<uint4 *>(b_smem + half * (UM_N * 128) + n * 128 + ((x ^ (n & 7)) << 4)) = v[x];
        }
      } else {
        float m = 0.f;
        if (hd >= 0) {
#pragma unroll 4
          for (int u = 0; u < 16; ++u) {
            const uint4 v = __ldg(row + u);
            const uint32_t ww[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              const float2 f = bf16x2_to_float2(ww[p]);
              m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
            }
          }
        }
        const float sc = e4m3_head_scale(m);
        wv = wv / sc;  // exact: sc is a power of two
        // input chunk u (8 elements) -> 8 bytes of each term at byte 8u of the row
#pragma unroll 2
        for (int u = 0; u < 16; ++u) {
          const uint4 v = hd >= 0 ? __ldg(row + u) : make_uint4(0u, 0u, 0u, 0u);
          uint2 t1, t2;
          split_e4m3(v, sc, t1, t2);
          const int ch = u >> 1, half = u & 1;
          const int off = n * 128 + ((ch ^ (n & 7)) << 4) + half * 8;
          *reinterpret_cast<uint2 *>(b_smem + off) = t1;
          *reinterpret_cast<uint2 *>(b_smem + UM_N * 128 + off) = t2;
        }
      }
      sh.wcol[n] = wv;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    if (tid == 0) {  // distinct sequences of the group, with their longest prefix
      int np = 0;
      for (int ql = 0; ql < QPT; ++ql) {
        const int s = sh.q_seq[ql];
        if (s < 0) continue;
        int p = 0;
        while (p < np && sh.pass_seq[p] != s) ++p;
        if (p == np) {
          sh.pass_seq[np] = s;
          sh.pass_len[np] = 0;
          ++np;
        }
        sh.pass_len[p] = max(sh.pass_len[p], sh.q_len[ql]);
      }
      sh.n_pass = np;
    }
    __syncthreads();
    const int n_pass = sh.n_pass;

    for (int pass = 0; pass < n_pass; ++pass) {
      const int seq = sh.pass_seq[pass];
      for (int ql = tid; ql < QPT; ql += UM_THREADS) sh.q_lenp[ql] = sh.q_seq[ql] == seq ? sh.q_len[ql] : 0;
      __syncthreads();
      const int t_end = min(tau1, cdiv(sh.pass_len[pass], UM_M));  // tiles [tau0, t_end) hold prefix tokens
      if (warp == 0) {
        // ---- TMA producer ----
        if (lane == 0) {
          for (int tau = tau0; tau < t_end; ++tau, ++it_load) {
            const int st = it_load % Cfg::STAGES;
            if (!umma::wait_bar(&sh.empty[st], ((it_load / Cfg::STAGES) & 1) ^ 1, abort, c)) break;
            mbar_arrive_expect_tx(&sh.full[st], Cfg::A_BYTES);
            const uint32_t dst = smem_addr(a_smem + st * Cfg::A_BYTES);
            const int y = seq * c.L_cap + tau * UM_M;
            if (FP8) {
              umma::tma_load_2d(dst, &kmap, 0, y, &sh.full[st]);
            } else {
              umma::tma_load_2d(dst, &kmap, 0, y, &sh.full[st]);
              umma::tma_load_2d(dst + UM_M * 128, &kmap, 64, y, &sh.full[st]);
            }
            last_fill_parity[st] = (it_load / Cfg::STAGES) & 1;
          }
        }
      } else if (warp == 1) {
        // ---- MMA issuer ----
        if (lane == 0) {
          const uint32_t idesc = umma::instr_desc<FP8, UM_M, UM_N>();
          const uint32_t b_base = smem_addr(b_smem);
          for (int tau = tau0; tau < t_end; ++tau, ++it_mma, ++j_mma) {
            const int st = it_mma % Cfg::STAGES, buf = j_mma & 1;
            if (!umma::wait_bar(&sh.tempty[buf], ((j_mma >> 1) & 1) ^ 1, abort, c)) break;
            umma::fence_after();
            if (!umma::wait_bar(&sh.full[st], (it_mma / Cfg::STAGES) & 1, abort, c)) break;
            umma::fence_after();
            const uint32_t a_base = smem_addr(a_smem + st * Cfg::A_BYTES);
            const uint32_t d = tmem + buf * UM_N;
#pragma unroll
            for (int t = 0; t < Cfg::TERMS; ++t) {
#pragma unroll
              for (int kk = 0; kk < Cfg::KSTEPS; ++kk) {
                uint32_t aoff, boff;
                if (FP8) {
                  aoff = kk * 32;
                  boff = t * (UM_N * 128) + kk * 32;
                } else {
                  aoff = (kk >> 2) * (UM_M * 128) + (kk & 3) * 32;
                  boff = (kk >> 2) * (UM_N * 128) + (kk & 3) * 32;
                }
                umma::mma<FP8>(d, umma::smem_desc_sw128(a_base + aoff), umma::smem_desc_sw128(b_base + boff), idesc,
                          (t | kk) ? 1u : 0u);
              }
            }
            umma::commit(&sh.empty[st]);
            umma::commit(&sh.tfull[buf]);
            mma_issued = true;
          }
        }
      } else {
        // ---- epilogue: one token row per thread, SPAN columns per warp ----
        const int e = warp - 2;
        const int quarter = warp & 3;              // tensor-memory lanes this warp may read
        const int col0 = (e / 4) * Cfg::SPAN;      // its columns
        const int r = quarter * 32 + lane;
        const float4 *wv = reinterpret_cast<const float4 *>(sh.wcol + col0);
        // TMA stores of whole [QH queries x 32 tokens] boxes, when every
        // query of this warp's half belongs to this pass (tokens past a
        // query's prefix are written too; they are unspecified)
        const int qa = col0 / HPQ;  // first query of the warp's columns
        bool tma_ok = false;
        if constexpr (Cfg::TMA_OUT) {
          if (out_tma) {
            tma_ok = true;
            for (int x = 0; x < Cfg::QH; ++x) {
              const int s2 = sh.q_seq[qa + x];
              tma_ok &= (s2 == seq || s2 < 0);
            }
          }
        }
        // e4m3 token scales are loaded one tile ahead, so that their latency
        // hides behind a tile of epilogue work instead of stalling the stores
        // (addresses are recomputed where used rather than held across the
        // tile: the routed form has 96 registers a thread)
        const size_t srow0 = (size_t)seq * c.L_cap;
        float st_next = (FP8 && tau0 < t_end && tau0 * UM_M + r < c.L_cap) ? __ldg(c.scale + srow0 + tau0 * UM_M + r)
                                                                          : 1.f;
        for (int tau = tau0; tau < t_end; ++tau, ++j_epi) {
          const int buf = j_epi & 1;
          const int t = tau * UM_M + r;
          const float st_scale = st_next;
          if (FP8 && tau + 1 < t_end) st_next = t + UM_M < c.L_cap ? __ldg(c.scale + srow0 + t + UM_M) : 1.f;
          float *stg = out_smem + (e * 2 + (int)ob) * (Cfg::OUT_BUF / 4);  // [QH][32]
          if (tma_ok) {  // the store that last read this buffer is done reading it
            if (lane == 0) umma::bulk_wait_read<1>();
            __syncwarp();
          }
          auto emit = [&](int ql, float x) {
            if (tma_ok)
              stg[(ql - qa) * 32 + lane] = x;
            else if (t < sh.q_lenp[ql])
              scores[((size_t)g * QPT + ql) * ld + t] = x;
          };
          if (!umma::wait_bar(&sh.tfull[buf], (j_epi >> 1) & 1, abort, c)) break;
          umma::fence_after();
          const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + buf * UM_N + col0;
          float acc = 0.f;  // running sum of a query wider than one chunk
          // CH chunks of 32 columns per tensor-memory round trip: two, or one
          // where the CTA's 18 warps leave 96 registers a thread (routed)
          constexpr int CH = Cfg::SPLIT == 4 ? 1 : 2;
#pragma unroll 1
          for (int ch = 0; ch < Cfg::SPAN / 32; ch += CH) {
            uint32_t vv[CH][32];
#pragma unroll
            for (int hc = 0; hc < CH; ++hc) umma::ld32(taddr + (ch + hc) * 32, vv[hc]);
            umma::ld_wait();
#pragma unroll
            for (int hc = 0; hc < CH; ++hc) {
              const uint32_t(&v)[32] = vv[hc];
              const int cb = (ch + hc) * 32;  // first column of this chunk (within the half)
              float part[32 / 4];
#pragma unroll
              for (int x4 = 0; x4 < 8; ++x4) {
                const float4 w4 = wv[(cb >> 2) + x4];
                float p = w4.x * fmaxf(__uint_as_float(v[4 * x4]), 0.f);
                p = fmaf(w4.y, fmaxf(__uint_as_float(v[4 * x4 + 1]), 0.f), p);
                p = fmaf(w4.z, fmaxf(__uint_as_float(v[4 * x4 + 2]), 0.f), p);
                part[x4] = fmaf(w4.w, fmaxf(__uint_as_float(v[4 * x4 + 3]), 0.f), p);
              }
              // queries of this chunk: HPQ / 4 partial sums each (HPQ <= 32),
              // or the chunk is part of one query (HPQ > 32)
              if constexpr (HPQ <= 32) {
                constexpr int QPC = 32 / HPQ;  // queries per chunk
                constexpr int PPQ = 8 / QPC;                   // partial sums per query
#pragma unroll
                for (int qc = 0; qc < QPC; ++qc) {
                  float sum = 0.f;
#pragma unroll
                  for (int x = 0; x < PPQ; ++x) sum += part[qc * PPQ + x];
                  emit((col0 + cb) / HPQ + qc, sum * st_scale);
                }
              } else {
#pragma unroll
                for (int x = 0; x < 8; ++x) acc += part[x];
                if (((col0 + cb + 32) % HPQ) == 0) {
                  emit((col0 + cb) / HPQ, acc * st_scale);
                  acc = 0.f;
                }
              }
            }
          }
          umma::fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh.tempty[buf]);
          if (tma_ok) {
            umma::fence_proxy_async();
            __syncwarp();
            if (lane == 0) {
              umma::tma_store_2d(&omap, smem_addr(stg), tau * UM_M + quarter * 32, g * QPT + qa);
              umma::bulk_commit();
            }
            ob ^= 1u;
          }
        }
      }
      __syncthreads();  // every role is done with this pass
      if (*abort) break;
    }
    __syncthreads();  // Q' and the group's tables are free again
  }

  // ---- wind-down: nothing in flight when the tensor memory is released ----
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < Cfg::STAGES; ++s)
      if (last_fill_parity[s] < 2) umma::wait_bar(&sh.full[s], last_fill_parity[s], abort, c);
  }
  if (warp == 1 && lane == 0 && mma_issued) {
    const uint32_t jl = j_mma - 1;  // the last committed accumulator buffer
    umma::wait_bar(&sh.tfull[jl & 1], (jl >> 1) & 1, abort, c);
  }
  if (warp >= 2 && lane == 0) umma::bulk_wait_all();  // score stores complete, staging free
  umma::fence_before();
  __syncthreads();
  if (warp == 1) {
    umma::fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
  }
}

// ---- host side ----------------------------------------------------------

template <bool FP8, int HPQ>
cudaError_t launch_hpq(const CUtensorMap &map, const CacheView &c, const QueryView &q, const int32_t *heads, int h,
                       float *scores, long long ld, cudaStream_t s) {
  using Cfg = UCfg<FP8, HPQ>;
  constexpr int SMEM = Cfg::SMEM;
  struct Tag {};
  // the attribute call's status, cached per device (+1 so that 0 means unset)
  const int st = cached_per_device<Tag>([] {
    return 1 + (int)cudaFuncSetAttribute(score_umma_kernel<FP8, HPQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         SMEM);
  });
  if (st != 1) return (cudaError_t)(st - 1);
  constexpr int QPT = UM_N / HPQ;
  const int n_groups = cdiv(q.n_q, QPT);
  const int n_tiles = cdiv(c.L_cap, UM_M);
  const long long n_items = (long long)n_groups * n_tiles;
  const int grid = (int)std::min<long long>(device_sms(), n_items);
  CUtensorMap omap;
  memset(&omap, 0, sizeof(omap));
  const int out_tma =
      Cfg::TMA_OUT && umma::make_map_f32_rows(&omap, scores, (unsigned long long)c.L_cap, (unsigned long long)q.n_q,
                                              (unsigned long long)ld, 32, Cfg::TMA_OUT ? Cfg::QH : 1);
  return launch_kernel(score_umma_kernel<FP8, HPQ>, dim3(grid), dim3(Cfg::THREADS), SMEM, s, map, omap, out_tma, c, q,
                       heads, h, scores, ld, n_tiles, n_items);
}

}  // namespace

bool umma_applies(const CacheView &c, const QueryView &q, const int32_t *heads, int h) {
  const int h_eff = heads ? h : q.H;
  return q.n_q >= 64 && q.n_q >= 8 * c.n_seq && h_eff <= UM_N && umma::encoder_available();
}

cudaError_t launch_score_umma(const CacheView &c, const QueryView &q, const int32_t *heads, int h, float *scores,
                              long long ld, cudaStream_t s) {
  if (q.n_q == 0) return cudaSuccess;
  CUtensorMap map;
  if (!umma::make_map_2d(&map, c.keys, c.fp8, (unsigned long long)c.n_seq * c.L_cap, c.fp8 ? 128 : 64, UM_M))
    return cudaErrorNotSupported;
  const int h_eff = heads ? h : q.H;
  int hpq = 4;  // at least 4 columns per query (zero-weight padding)
  while (hpq < h_eff) hpq *= 2;
#define MISA_UMMA_CASE(N)                                                                                  \
  case N:                                                                                                  \
    return c.fp8 ? launch_hpq<true, N>(map, c, q, heads, h, scores, ld, s)                                 \
                 : launch_hpq<false, N>(map, c, q, heads, h, scores, ld, s);
  switch (hpq) {
    MISA_UMMA_CASE(4)
    MISA_UMMA_CASE(8)
    MISA_UMMA_CASE(16)
    MISA_UMMA_CASE(32)
    MISA_UMMA_CASE(64)
    MISA_UMMA_CASE(128)
    default:
      return cudaErrorInvalidValue;
  }
#undef MISA_UMMA_CASE
}

namespace umma {

using EncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                 const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiled encode_fn() {
  static EncodeTiled fn = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (EncodeTiled) nullptr;
    return reinterpret_cast<EncodeTiled>(p);
  }();
  return fn;
}

bool encoder_available() { return encode_fn() != nullptr; }

bool make_map_2d(CUtensorMap *map, const void *base, bool u8, unsigned long long rows, int box_x, int box_rows) {
  EncodeTiled enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(u8 ? D : 2 * D)};
  const cuuint32_t box[2] = {(cuuint32_t)box_x, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, u8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base),
             dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_f32_rows(CUtensorMap *map, const float *base, unsigned long long cols, unsigned long long rows,
                       unsigned long long ld, int box_x, int box_rows) {
  EncodeTiled enc = encode_fn();
  if (!enc || (reinterpret_cast<uintptr_t>(base) & 15u) || (ld * sizeof(float)) % 16 != 0) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(ld * sizeof(float))};
  const cuuint32_t box[2] = {(cuuint32_t)box_x, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace umma
}  // namespace misa
