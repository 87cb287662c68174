// C ABI of the MISA / DSA indexer: argument validation, workspace layout and
// dispatch to the kernels.  Declarations and semantics: include/misa.h.
#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cuda.h>

#include <nvtx3/nvToolsExt.h>

#include "internal.h"

namespace {

// One NVTX range per library call that launches work, named after the entry
// point, so that a profiler's timeline shows each call around its kernels.
// Without a profiler attached the calls are no-ops.
struct NvtxRange {
  explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange &) = delete;
  NvtxRange &operator=(const NvtxRange &) = delete;
};

thread_local char g_err[512] = "";
std::atomic<int> g_fail_next{0};
// Selection inside the scoring kernels for the calls other than the decode
// step's routed pass (misa_debug_select_in_kernel).  Off by default: there
// the separate top-k kernels are as fast or faster on B200 -- the fused
// selection's cross-CTA phases (two row barriers, two histogram searches in
// L2, the last CTA's bucket) take about 21 us, as long as the filter and
// select kernels they replace, and a fused re-rank of 8 x 8192 candidates
// needs four-tile CTAs to be resident at once (38.6 us against 15.5 + 12.5).
// The decode step's routed pass selects in-kernel always: its in-kernel
// router needs the same resident CTAs and hides behind the key prefetch.
std::atomic<int> g_select_in_kernel{0};
std::atomic<void *> g_ev_start{nullptr}, g_ev_stop{nullptr};

// Launch the scoring kernel, bracketed by the profiling events when set.
template <class F>
cudaError_t timed_scoring(cudaStream_t stream, F &&launch) {
  void *a = g_ev_start.load(), *b = g_ev_stop.load();
  // External records: inside a stream capture they become event-record nodes
  // that stamp the time on every graph launch.
  unsigned flags = 0;
  if (a && b) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
      flags = cudaEventRecordExternal;
    cudaError_t e = cudaEventRecordWithFlags(static_cast<cudaEvent_t>(a), stream, flags);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = launch();
  if (e == cudaSuccess && a && b) e = cudaEventRecordWithFlags(static_cast<cudaEvent_t>(b), stream, flags);
  return e;
}

misa_status fail(misa_status st, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

misa_status cuda_fail(cudaError_t e, const char *where) {
  return fail(MISA_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Consume one injected failure, if any (after validation, before any launch).
bool injected_failure(const char *where, misa_status *st) {
  int n = g_fail_next.load();
  while (n > 0) {
    if (g_fail_next.compare_exchange_weak(n, n - 1)) {
      *st = fail(MISA_ERR_CUDA, "%s: injected failure (misa_debug_fail_next)", where);
      return true;
    }
  }
  return false;
}

misa_status check_cache(const misa_cache *c, bool need_pool) {
  if (!c) return fail(MISA_ERR_INVALID, "cache is NULL");
  if (!c->keys || !c->seq_len) return fail(MISA_ERR_INVALID, "cache keys/seq_len is NULL");
  if (need_pool && !c->pool) return fail(MISA_ERR_INVALID, "cache pool is NULL");
  if (c->dtype != MISA_KEY_BF16 && c->dtype != MISA_KEY_FP8_E4M3)
    return fail(MISA_ERR_INVALID, "unknown key dtype %d", c->dtype);
  if ((c->dtype == MISA_KEY_FP8_E4M3) != (c->scale != nullptr))
    return fail(MISA_ERR_INVALID, "scale must be non-NULL exactly for fp8 keys");
  if (c->d != MISA_D) return fail(MISA_ERR_UNSUPPORTED, "d=%d unsupported (only %d)", c->d, MISA_D);
  if (c->n_seq < 1 || c->L_cap < 1 || c->B < 1)
    return fail(MISA_ERR_INVALID, "n_seq=%d L_cap=%d B=%d must be >= 1", c->n_seq, c->L_cap, c->B);
  if (c->L_cap > MISA_MAX_L) return fail(MISA_ERR_UNSUPPORTED, "L_cap=%d above %d", c->L_cap, MISA_MAX_L);
  if (!aligned16(c->keys)) return fail(MISA_ERR_INVALID, "keys must be 16-byte aligned");
  if (c->pool && !aligned16(c->pool)) return fail(MISA_ERR_INVALID, "pool must be 16-byte aligned");
  return MISA_OK;
}

misa_status check_queries(const misa_queries *q) {
  if (!q) return fail(MISA_ERR_INVALID, "queries is NULL");
  if (q->n_q < 0 || q->n_q > 65535) return fail(MISA_ERR_INVALID, "n_q=%d outside [0, 65535]", q->n_q);
  if (q->H < 1 || q->H > MISA_MAX_H) return fail(MISA_ERR_UNSUPPORTED, "H=%d outside [1, %d]", q->H, MISA_MAX_H);
  if (q->n_q > 0 && (!q->q || !q->w || !q->q_seq || !q->q_pos))
    return fail(MISA_ERR_INVALID, "queries q/w/q_seq/q_pos is NULL");
  if (q->q && !aligned16(q->q)) return fail(MISA_ERR_INVALID, "q must be 16-byte aligned");
  return MISA_OK;
}

misa::CacheView view(const misa_cache *c) {
  misa::CacheView v;
  v.keys = c->keys;
  v.scale = c->scale;
  v.seq_len = c->seq_len;
  v.pool = c->pool;
  v.status = c->status;
  v.n_seq = c->n_seq;
  v.L_cap = c->L_cap;
  v.B = c->B;
  v.fp8 = c->dtype == MISA_KEY_FP8_E4M3;
  return v;
}

misa::QueryView view(const misa_queries *q) {
  misa::QueryView v;
  v.q = q->q;
  v.w = q->w;
  v.q_seq = q->q_seq;
  v.q_pos = q->q_pos;
  v.n_q = q->n_q;
  v.H = q->H;
  return v;
}

size_t round_up(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace of the score + top-k calls: [row histograms + top-k list
// counters (zeroed together)][scores, unless the caller passes scores_out]
// [top-k list, prefix rows that use one].
// row histograms, then two counters per row (list entries, emitted tokens)
size_t hist_words(const misa_queries *q) { return (size_t)q->n_q * (misa::TOPK_HIST_BINS + 2); }
size_t ws_hist(const misa_queries *q) { return round_up(sizeof(uint32_t) * hist_words(q)); }
size_t ws_list(const misa_cache *c, const misa_queries *q, int k) {
  return round_up(8 * misa::topk_list_entries(q->n_q, c->L_cap, k));
}

size_t ws_score(const misa_cache *c, const misa_queries *q) {
  return round_up(sizeof(float) * (size_t)q->n_q * c->L_cap);
}

// Workspace of misa_dagger_topk: [histograms + list counters][re-rank
// histograms] (one zeroing launch for both) [routed scores][top-k' list]
// [candidates n_q x k'][re-rank scores n_q x k'].
// (the re-rank histograms start on a 256-byte boundary: rows are read with
// 16-byte loads and bulk copies)
size_t rerank_hist_words(const misa_queries *q) { return (size_t)q->n_q * misa::TOPK_HIST_BINS; }
size_t ws_dagger_hist(const misa_queries *q) {
  return ws_hist(q) + round_up(sizeof(uint32_t) * rerank_hist_words(q));
}
size_t ws_fz_zero(const misa_queries *q);
size_t ws_fz_bucket(const misa_queries *q);
size_t ws_fz_win(const misa_queries *q, int k);
// [hist + counters][re-rank hist][fused zeroed: routed pass][fused zeroed:
// re-rank] (zeroed by one launch) [routed scores][top-k' list][bucket]
// [winners][candidates][re-rank scores]
size_t ws_dagger(const misa_cache *c, const misa_queries *q, int k_prime, int k) {
  const size_t cand = round_up(sizeof(int32_t) * (size_t)q->n_q * k_prime);
  return ws_dagger_hist(q) + 2 * ws_fz_zero(q) + ws_score(c, q) + ws_list(c, q, k_prime) + ws_fz_bucket(q) +
         ws_fz_win(q, k) + 2 * cand;
}

// Regions of a selection done inside the scoring kernel (misa::FusedTopk):
// words zeroed before the launch, the boundary bucket, the winners of an
// ascending output.  Every workspace reserves them beside the regions of the
// separate top-k kernels; which set a call uses is decided per call
// (misa::score_fusable).
size_t ws_fz_zero(const misa_queries *q) { return round_up(sizeof(uint32_t) * (size_t)q->n_q * misa::FUSED_ZERO_WORDS); }
size_t ws_fz_bucket(const misa_queries *q) { return round_up(sizeof(uint2) * (size_t)q->n_q * misa::FUSED_BCAP); }
size_t ws_fz_win(const misa_queries *q, int k) { return round_up(sizeof(int32_t) * (size_t)q->n_q * k); }

// score + top-k: [hist + counters][fused zeroed][scores, unless scores_out]
// [top-k list][bucket][winners]
size_t ws_score_topk(const misa_cache *c, const misa_queries *q, int k, bool scores_out) {
  return ws_hist(q) + ws_fz_zero(q) + (scores_out ? 0 : ws_score(c, q)) + ws_list(c, q, k) + ws_fz_bucket(q) +
         ws_fz_win(q, k);
}
// re-rank: [hist][fused zeroed][scores, unless scores_out][bucket][winners]
size_t ws_rerank(const misa_queries *q, int k_prime, int k, bool scores_out) {
  return ws_hist(q) + ws_fz_zero(q) + (scores_out ? 0 : round_up(sizeof(float) * (size_t)q->n_q * k_prime)) +
         ws_fz_bucket(q) + ws_fz_win(q, k);
}

misa::FusedTopk fused_args(uint32_t *zeroed, void *bucket, void *winners, int32_t *out, int k, bool ordered) {
  misa::FusedTopk f;
  f.zeroed = zeroed;
  f.bucket = static_cast<uint2 *>(bucket);
  f.winners = static_cast<int32_t *>(winners);
  f.out = out;
  f.k = k;
  f.ordered = ordered ? 1 : 0;
  f.defer = 0;
  return f;
}

// misa_dagger_decode: [misa_dagger_topk's workspace][router: the separate
// router's workspace, or the in-kernel router's partial sums][heads]
size_t ws_route(const misa_cache *c, const misa_queries *q) {
  const int M_cap = misa::cdiv(c->L_cap, c->B);
  return round_up(std::max(misa::route_ws_bytes(q->n_q, q->H, M_cap),
                           misa::route_umma_ws_bytes(q->n_q, q->H, M_cap, c->n_seq)));
}
size_t ws_decode_router(const misa_cache *c, const misa_queries *q) {
  return std::max(ws_route(c, q), round_up(sizeof(float) * (size_t)misa::route_part_slots() * q->H));
}
size_t ws_decode(const misa_cache *c, const misa_queries *q, int h, int k_prime, int k) {
  return ws_dagger(c, q, k_prime, k) + ws_decode_router(c, q) + round_up(sizeof(int32_t) * (size_t)q->n_q * h);
}

misa_status check_ws(void *ws, size_t have, size_t need) {
  if (have < need) return fail(MISA_ERR_WORKSPACE, "workspace %zu bytes, need %zu", have, need);
  if (need > 0 && (!ws || !aligned16(ws))) return fail(MISA_ERR_INVALID, "workspace NULL or not 16-byte aligned");
  return MISA_OK;
}

// Scores then top-k, shared by the routed and dense entry points.
misa_status score_then_topk(const char *who, const misa_cache *cache, const misa_queries *qs,
                            const int32_t *heads, int h, int k, int32_t *topk, float *scores_out, void *ws,
                            cudaStream_t stream) {
  misa::CacheView c = view(cache);
  misa::QueryView q = view(qs);
  uint8_t *w8 = static_cast<uint8_t *>(ws);
  uint32_t *hist = reinterpret_cast<uint32_t *>(w8);
  uint32_t *list_cnt = hist + (size_t)qs->n_q * misa::TOPK_HIST_BINS;
  uint32_t *fz_zero = reinterpret_cast<uint32_t *>(w8 + ws_hist(qs));
  uint8_t *after = w8 + ws_hist(qs) + ws_fz_zero(qs);
  float *scores = scores_out ? scores_out : reinterpret_cast<float *>(after);
  uint8_t *list = after + (scores_out ? 0 : ws_score(cache, qs));
  uint8_t *bucket = list + ws_list(cache, qs, k);
  uint8_t *winners = bucket + ws_fz_bucket(qs);
  // many queries per sequence (prefill chunks): tensor-core scoring, and the
  // selection counts each row itself; otherwise the streaming scorer selects
  // in-kernel when its grid is resident at once, or builds the row
  // histograms on the way for the top-k kernels
  const bool umma = misa::umma_applies(c, q, heads, h);
  const bool fused = g_select_in_kernel.load() && !umma && misa::score_fusable(c, q, heads, h, nullptr, 0);
  cudaError_t e = fused ? misa::launch_zero(fz_zero, (size_t)qs->n_q * misa::FUSED_ZERO_WORDS, stream)
                        : misa::launch_zero(hist, hist_words(qs), stream);
  if (e != cudaSuccess) return cuda_fail(e, who);
  const misa::FusedTopk fz = fused_args(fz_zero, bucket, winners, topk, k, true);
  e = timed_scoring(stream, [&] {
    return umma ? misa::launch_score_umma(c, q, heads, h, scores, cache->L_cap, stream)
                : misa::launch_score_mma(c, q, heads, h, nullptr, 0, scores, cache->L_cap, hist, stream,
                                         fused ? &fz : nullptr);
  });
  if (e != cudaSuccess) return cuda_fail(e, who);
  if (fused) return MISA_OK;
  e = misa::launch_topk(c, q, scores, cache->L_cap, 0, nullptr, hist, !umma, list, list_cnt, k, topk, stream);
  if (e != cudaSuccess) return cuda_fail(e, who);
  return MISA_OK;
}

// The bounded wait every pipeline of the library uses, on an mbarrier that
// never completes: after limit_ns it records MISA_DEV_WAIT_TIMEOUT and the
// kernel returns normally (the failure path, exercised without a fault).
__global__ void wait_timeout_kernel(uint32_t *status, unsigned long long limit_ns) {
  misa::grid_dep_sync();
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    misa::mbar_init(&bar, 1);
    misa::fence_mbar_init();
  }
  __syncthreads();
  if (!misa::mbar_wait(&bar, 0, limit_ns) && threadIdx.x == 0) atomicOr(status, MISA_DEV_WAIT_TIMEOUT);
}

// Scratch of misa_rerank_topk_noalloc: part of the library's device image, so
// the caller never supplies memory and the call never allocates any.
static __device__ __align__(256) uint8_t g_noalloc_scratch[MISA_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch in the current context.  Every context
// that loads the library's device code holds its own copy of the array, so
// the address belongs to a context, not to a device: after cudaDeviceReset,
// or when a driver-API caller makes another context current on the same
// device, the earlier address is dead.  Addresses are therefore cached per
// context, keyed by the driver's context ID (unique for the life of the
// process, where a context handle can be reused), and looked up with
// cudaGetSymbolAddress on the first call in each context.
using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// Current context's ID; false when there is no current context or the
// driver entry points are unavailable (the caller then looks the address up
// without caching it).
bool current_context_id(unsigned long long *id) {
  static CtxGetCurrentFn get_current = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    return cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
                   q == cudaDriverEntryPointSuccess
               ? reinterpret_cast<CtxGetCurrentFn>(p)
               : nullptr;
  }();
  static CtxGetIdFn get_id = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    return cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
                   q == cudaDriverEntryPointSuccess
               ? reinterpret_cast<CtxGetIdFn>(p)
               : nullptr;
  }();
  CUcontext ctx = nullptr;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

misa_status noalloc_scratch(const char *who, void **out) {
  constexpr int SLOTS = 64;
  static std::mutex mu;
  static unsigned long long ids[SLOTS];  // 0: empty (driver context IDs start at 1)
  static void *addrs[SLOTS];
  static int next_slot = 0;
  unsigned long long id = 0;
  const bool keyed = current_context_id(&id) && id != 0;
  if (keyed) {
    std::lock_guard<std::mutex> lock(mu);
    for (int j = 0; j < SLOTS; ++j)
      if (ids[j] == id) {
        *out = addrs[j];
        return MISA_OK;
      }
  }
  void *p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return cuda_fail(e, "misa_rerank_topk_noalloc: cudaGetSymbolAddress");
  if (!p) return fail(MISA_ERR_CUDA, "%s: cudaGetSymbolAddress returned NULL", who);
  // the lookup may have made the primary context current: key it now
  if (keyed || (current_context_id(&id) && id != 0)) {
    std::lock_guard<std::mutex> lock(mu);
    ids[next_slot] = id;
    addrs[next_slot] = p;
    next_slot = (next_slot + 1) % SLOTS;
  }
  *out = p;
  return MISA_OK;
}

// MISA-dagger on validated arguments (misa_dagger_topk): routed scores and
// their k' candidates, then every head on the candidates and the final k.
// With route_part (misa_dagger_decode, fused routed pass only) the scoring
// kernel routes the queries itself and writes their heads to heads_out.
// dagger_zero_words(): the words from the workspace's start that a call
// counts into when both passes select in-kernel or neither does, or
// everything up to the end of the fused words when the passes differ;
// zero_done: a kernel before (the decode step's append) cleared them.
size_t dagger_zero_words(const misa_queries *qs, bool f1, bool f2) {
  const size_t fz_end = (ws_dagger_hist(qs) + ws_fz_zero(qs)) / sizeof(uint32_t) + (size_t)qs->n_q * misa::FUSED_ZERO_WORDS;
  return (f1 || f2) ? fz_end : ws_hist(qs) / sizeof(uint32_t) + rerank_hist_words(qs);
}

misa_status dagger_body(const char *who, const misa_cache *cache, const misa_queries *qs, const int32_t *heads,
                        int h, int k_prime, int k, int32_t *topk, void *ws, cudaStream_t stream,
                        float *route_part = nullptr, int32_t *heads_out = nullptr, bool zero_done = false,
                        const misa::PendingAppend *pending = nullptr) {
  misa::CacheView c = view(cache);
  misa::QueryView q = view(qs);
  uint8_t *w8 = static_cast<uint8_t *>(ws);
  uint32_t *hist = reinterpret_cast<uint32_t *>(w8);
  uint32_t *list_cnt = hist + (size_t)qs->n_q * misa::TOPK_HIST_BINS;
  uint32_t *rhist = reinterpret_cast<uint32_t *>(w8 + ws_hist(qs));
  uint32_t *fz1 = reinterpret_cast<uint32_t *>(w8 + ws_dagger_hist(qs));
  uint32_t *fz2 = reinterpret_cast<uint32_t *>(w8 + ws_dagger_hist(qs) + ws_fz_zero(qs));
  uint8_t *p = w8 + ws_dagger_hist(qs) + 2 * ws_fz_zero(qs);
  float *scores = reinterpret_cast<float *>(p);
  p += ws_score(cache, qs);
  void *list = p;
  p += ws_list(cache, qs, k_prime);
  uint8_t *bucket = p;
  p += ws_fz_bucket(qs);
  uint8_t *winners = p;
  p += ws_fz_win(qs, k);
  int32_t *cand = reinterpret_cast<int32_t *>(p);
  float *rscores = reinterpret_cast<float *>(p + round_up(sizeof(int32_t) * (size_t)qs->n_q * k_prime));
  // routed pass: scores, then the k' candidates in any order; selected in the
  // scoring kernels when their grids are resident at once
  const bool umma = !route_part && misa::umma_applies(c, q, heads, h);
  const bool f1 = route_part || (g_select_in_kernel.load() && !umma && misa::score_fusable(c, q, heads, h, nullptr, 0));
  const bool f2 = g_select_in_kernel.load() && misa::score_fusable(c, q, nullptr, q.H, cand, k_prime);
  // both passes' counting words, zeroed by one launch: the histograms and
  // counters of the top-k kernels, the fused selections' words, or both
  uint32_t *z0 = (f1 && f2) ? fz1 : hist;
  uint32_t *z1 = hist + dagger_zero_words(qs, f1, f2);
  cudaError_t e = zero_done ? cudaSuccess : misa::launch_zero(z0, (size_t)(z1 - z0), stream);
  if (e != cudaSuccess) return cuda_fail(e, who);
  // the fine pass in one cluster kernel: a top-k' selected in the routed
  // scoring kernel leaves its boundary bucket for that kernel to finish
  const bool cluster = !f2 && misa::rerank_cluster_applies(c, q, k_prime, k);
  misa::FusedTopk fzc = fused_args(fz1, bucket, nullptr, cand, k_prime, false);
  fzc.defer = f1 && cluster ? 1 : 0;
  e = timed_scoring(stream, [&] {
    if (route_part)
      return misa::launch_score_stream(c, q, nullptr, h, scores, cache->L_cap, hist, stream, &fzc, route_part,
                                       heads_out, pending);
    return umma ? misa::launch_score_umma(c, q, heads, h, scores, cache->L_cap, stream)
                : misa::launch_score_mma(c, q, heads, h, nullptr, 0, scores, cache->L_cap, hist, stream,
                                         f1 ? &fzc : nullptr);
  });
  if (e != cudaSuccess) return cuda_fail(e, who);
  if (!f1) {
    e = misa::launch_topk(c, q, scores, cache->L_cap, 0, nullptr, hist, !umma, list, list_cnt, k_prime, cand, stream,
                          false);
    if (e != cudaSuccess) return cuda_fail(e, who);
  }
  // fine pass: every head on the candidates, ascending final top-k; one
  // cluster kernel when a cluster holds a query's candidates
  if (cluster) {
    e = misa::launch_rerank_cluster(c, q, cand, k_prime, k, topk, nullptr, 0, stream, fzc.defer ? fz1 : nullptr,
                                    fzc.defer ? reinterpret_cast<const uint2 *>(bucket) : nullptr);
    if (e != cudaSuccess) return cuda_fail(e, who);
    return MISA_OK;
  }
  const misa::FusedTopk fzr = fused_args(fz2, bucket, winners, topk, k, true);
  e = misa::launch_score_mma(c, q, nullptr, q.H, cand, k_prime, rscores, k_prime, rhist, stream, f2 ? &fzr : nullptr);
  if (e != cudaSuccess) return cuda_fail(e, who);
  if (f2) return MISA_OK;
  e = misa::launch_topk(c, q, rscores, k_prime, k_prime, cand, rhist, true, nullptr, nullptr, k, topk, stream);
  if (e != cudaSuccess) return cuda_fail(e, who);
  return MISA_OK;
}

}  // namespace

extern "C" {

misa_status misa_pool_keys(const misa_cache *cache, const void *new_keys, const float *new_scale,
                           const int32_t *new_pos, int32_t count, misa_stream stream) {
  NvtxRange nvtx("misa_pool_keys");
  misa_status st = check_cache(cache, true);
  if (st != MISA_OK) return st;
  if (count < 0) return fail(MISA_ERR_INVALID, "count=%d < 0", count);
  if (count > 0) {
    if (!new_keys || !new_pos) return fail(MISA_ERR_INVALID, "append needs new_keys and new_pos");
    if ((cache->dtype == MISA_KEY_FP8_E4M3) != (new_scale != nullptr))
      return fail(MISA_ERR_INVALID, "new_scale must be non-NULL exactly for fp8 keys");
    if (!aligned16(new_keys)) return fail(MISA_ERR_INVALID, "new_keys must be 16-byte aligned");
    if (count > cache->L_cap) return fail(MISA_ERR_INVALID, "count=%d above L_cap=%d", count, cache->L_cap);
  }
  if (injected_failure("misa_pool_keys", &st)) return st;
  misa::CacheView c = view(cache);
  cudaError_t e = count == 0 ? misa::launch_pool_rebuild(c, stream)
                             : misa::launch_pool_append(c, new_keys, new_scale, new_pos, count, stream);
  if (e != cudaSuccess) return cuda_fail(e, "misa_pool_keys");
  return MISA_OK;
}

misa_status misa_append_keys_e4m3(const misa_cache *cache, const uint16_t *new_keys, const int32_t *new_pos,
                                  int32_t count, misa_stream stream) {
  NvtxRange nvtx("misa_append_keys_e4m3");
  misa_status st = check_cache(cache, true);
  if (st != MISA_OK) return st;
  if (cache->dtype != MISA_KEY_FP8_E4M3) return fail(MISA_ERR_INVALID, "the cache does not hold e4m3 keys");
  if (count < 1 || count > misa::pool_append_quant_max())
    return fail(MISA_ERR_INVALID, "count=%d outside [1, %d]", count, misa::pool_append_quant_max());
  if (count > cache->L_cap) return fail(MISA_ERR_INVALID, "count=%d above L_cap=%d", count, cache->L_cap);
  if (!new_keys || !new_pos) return fail(MISA_ERR_INVALID, "new_keys and new_pos must be non-NULL");
  if (!aligned16(new_keys)) return fail(MISA_ERR_INVALID, "new_keys must be 16-byte aligned");
  if (injected_failure("misa_append_keys_e4m3", &st)) return st;
  cudaError_t e = misa::launch_pool_append_quant(view(cache), new_keys, new_pos, count, stream);
  if (e != cudaSuccess) return cuda_fail(e, "misa_append_keys_e4m3");
  return MISA_OK;
}

size_t misa_workspace_bytes(int32_t op, const misa_cache *cache, const misa_queries *qs, int32_t h, int32_t k,
                            int32_t k_prime) {
  if (!cache || !qs || cache->B < 1 || cache->L_cap < 1 || qs->n_q < 0 || qs->H < 1) return 0;
  switch (op) {
    case MISA_OP_ROUTE:
      return ws_route(cache, qs);
    case MISA_OP_SCORE_TOPK:
    case MISA_OP_DENSE_TOPK:
      return k > 0 ? ws_score_topk(cache, qs, k, false) : 0;
    case MISA_OP_RERANK_TOPK:
      return k_prime > 0 && k > 0 ? ws_rerank(qs, k_prime, k, false) : 0;
    case MISA_OP_DAGGER_TOPK:
      return k_prime > 0 && k > 0 ? ws_dagger(cache, qs, k_prime, k) : 0;
    case MISA_OP_DAGGER_DECODE:
      return k_prime > 0 && k > 0 && h > 0 ? ws_decode(cache, qs, h, k_prime, k) : 0;
    default:
      return 0;
  }
}

misa_status misa_route_heads_agg(const misa_cache *cache, const misa_queries *qs, int32_t h, int32_t agg,
                                 int32_t *heads, float *router_scores, void *ws, size_t ws_bytes,
                                 misa_stream stream) {
  NvtxRange nvtx("misa_route_heads_agg");
  misa_status st = check_cache(cache, true);
  if (st != MISA_OK) return st;
  if ((st = check_queries(qs)) != MISA_OK) return st;
  if (h < 1 || h > qs->H) return fail(MISA_ERR_INVALID, "h=%d outside [1, H=%d]", h, qs->H);
  if (agg < MISA_AGG_ABS_SUM || agg > MISA_AGG_ABS_MAX) return fail(MISA_ERR_INVALID, "agg=%d unknown", agg);
  if (qs->n_q > 0 && !heads) return fail(MISA_ERR_INVALID, "heads is NULL");
  if ((st = check_ws(ws, ws_bytes, misa_workspace_bytes(MISA_OP_ROUTE, cache, qs, h, 0, 0))) != MISA_OK) return st;
  if (injected_failure("misa_route_heads", &st)) return st;
  cudaError_t e = misa::launch_route(view(cache), view(qs), h, heads, router_scores, ws, stream, agg);
  if (e != cudaSuccess) return cuda_fail(e, "misa_route_heads");
  return MISA_OK;
}

misa_status misa_route_heads(const misa_cache *cache, const misa_queries *qs, int32_t h, int32_t *heads,
                             float *router_scores, void *ws, size_t ws_bytes, misa_stream stream) {
  return misa_route_heads_agg(cache, qs, h, MISA_AGG_ABS_SUM, heads, router_scores, ws, ws_bytes, stream);
}

misa_status misa_score_topk(const misa_cache *cache, const misa_queries *qs, const int32_t *heads, int32_t h,
                            int32_t k, int32_t *topk, float *scores_out, void *ws, size_t ws_bytes,
                            misa_stream stream) {
  NvtxRange nvtx("misa_score_topk");
  misa_status st = check_cache(cache, false);
  if (st != MISA_OK) return st;
  if ((st = check_queries(qs)) != MISA_OK) return st;
  if (h < 1 || h > qs->H) return fail(MISA_ERR_INVALID, "h=%d outside [1, H=%d]", h, qs->H);
  if (k < 1) return fail(MISA_ERR_INVALID, "k=%d < 1", k);
  if (qs->n_q > 0 && (!heads || !topk)) return fail(MISA_ERR_INVALID, "heads/topk is NULL");
  if ((st = check_ws(ws, ws_bytes, ws_score_topk(cache, qs, k, scores_out != nullptr))) != MISA_OK) return st;
  if (injected_failure("misa_score_topk", &st)) return st;
  if (qs->n_q == 0) return MISA_OK;
  return score_then_topk("misa_score_topk", cache, qs, heads, h, k, topk, scores_out, ws, stream);
}

misa_status dsa_dense_score_topk(const misa_cache *cache, const misa_queries *qs, int32_t k, int32_t *topk,
                                 float *scores_out, void *ws, size_t ws_bytes, misa_stream stream) {
  NvtxRange nvtx("dsa_dense_score_topk");
  misa_status st = check_cache(cache, false);
  if (st != MISA_OK) return st;
  if ((st = check_queries(qs)) != MISA_OK) return st;
  if (k < 1) return fail(MISA_ERR_INVALID, "k=%d < 1", k);
  if (qs->n_q > 0 && !topk) return fail(MISA_ERR_INVALID, "topk is NULL");
  if ((st = check_ws(ws, ws_bytes, ws_score_topk(cache, qs, k, scores_out != nullptr))) != MISA_OK) return st;
  if (injected_failure("dsa_dense_score_topk", &st)) return st;
  if (qs->n_q == 0) return MISA_OK;
  return score_then_topk("dsa_dense_score_topk", cache, qs, nullptr, qs->H, k, topk, scores_out, ws, stream);
}

misa_status misa_rerank_topk(const misa_cache *cache, const misa_queries *qs, const int32_t *cand,
                             int32_t k_prime, int32_t k, int32_t *topk, float *scores_out, void *ws,
                             size_t ws_bytes, misa_stream stream) {
  NvtxRange nvtx("misa_rerank_topk");
  misa_status st = check_cache(cache, false);
  if (st != MISA_OK) return st;
  if ((st = check_queries(qs)) != MISA_OK) return st;
  if (k < 1 || k_prime < k) return fail(MISA_ERR_INVALID, "need 1 <= k=%d <= k_prime=%d", k, k_prime);
  if (k_prime > MISA_MAX_L) return fail(MISA_ERR_UNSUPPORTED, "k_prime=%d above %d", k_prime, MISA_MAX_L);
  if (qs->n_q > 0 && (!cand || !topk)) return fail(MISA_ERR_INVALID, "cand/topk is NULL");
  if ((st = check_ws(ws, ws_bytes, ws_rerank(qs, k_prime, k, scores_out != nullptr))) != MISA_OK) return st;
  if (injected_failure("misa_rerank_topk", &st)) return st;
  if (qs->n_q == 0) return MISA_OK;
  misa::CacheView c = view(cache);
  misa::QueryView q = view(qs);
  uint8_t *w8 = static_cast<uint8_t *>(ws);
  uint32_t *hist = reinterpret_cast<uint32_t *>(w8);
  uint32_t *fz_zero = reinterpret_cast<uint32_t *>(w8 + ws_hist(qs));
  uint8_t *after = w8 + ws_hist(qs) + ws_fz_zero(qs);
  float *scores = scores_out ? scores_out : reinterpret_cast<float *>(after);
  uint8_t *bucket = after + (scores_out ? 0 : round_up(sizeof(float) * (size_t)qs->n_q * k_prime));
  uint8_t *winners = bucket + ws_fz_bucket(qs);
  const bool fused = g_select_in_kernel.load() && misa::score_fusable(c, q, nullptr, q.H, cand, k_prime);
  if (!fused && misa::rerank_cluster_applies(c, q, k_prime, k)) {
    cudaError_t e = timed_scoring(stream, [&] {
      return misa::launch_rerank_cluster(c, q, cand, k_prime, k, topk, scores_out, k_prime, stream);
    });
    if (e != cudaSuccess) return cuda_fail(e, "misa_rerank_topk");
    return MISA_OK;
  }
  cudaError_t e = fused ? misa::launch_zero(fz_zero, (size_t)qs->n_q * misa::FUSED_ZERO_WORDS, stream)
                        : misa::launch_zero(hist, (size_t)qs->n_q * misa::TOPK_HIST_BINS, stream);
  if (e != cudaSuccess) return cuda_fail(e, "misa_rerank_topk");
  const misa::FusedTopk fz = fused_args(fz_zero, bucket, winners, topk, k, true);
  e = timed_scoring(stream, [&] {
    return misa::launch_score_mma(c, q, nullptr, q.H, cand, k_prime, scores, k_prime, hist, stream,
                                  fused ? &fz : nullptr);
  });
  if (e != cudaSuccess) return cuda_fail(e, "misa_rerank_topk");
  if (fused) return MISA_OK;
  e = misa::launch_topk(c, q, scores, k_prime, k_prime, cand, hist, true, nullptr, nullptr, k, topk, stream);
  if (e != cudaSuccess) return cuda_fail(e, "misa_rerank_topk");
  return MISA_OK;
}

misa_status misa_rerank_topk_noalloc(const misa_cache *cache, const misa_queries *qs, const int32_t *cand,
                                     int32_t k_prime, int32_t k, int32_t *topk, float *scores_out,
                                     misa_stream stream) {
  NvtxRange nvtx("misa_rerank_topk_noalloc");
  const char *who = "misa_rerank_topk_noalloc";
  misa_status st = check_cache(cache, false);
  if (st != MISA_OK) return st;
  if ((st = check_queries(qs)) != MISA_OK) return st;
  if (k < 1 || k_prime < k) return fail(MISA_ERR_INVALID, "need 1 <= k=%d <= k_prime=%d", k, k_prime);
  if (k_prime > MISA_MAX_L) return fail(MISA_ERR_UNSUPPORTED, "k_prime=%d above %d", k_prime, MISA_MAX_L);
  if (qs->n_q > 0 && (!cand || !topk)) return fail(MISA_ERR_INVALID, "cand/topk is NULL");
  const size_t need = ws_hist(qs) + (scores_out ? 0 : round_up(sizeof(float) * (size_t)qs->n_q * k_prime));
  if (need > MISA_NOALLOC_SCRATCH_BYTES)
    return fail(MISA_ERR_WORKSPACE,
                "%s: n_q=%d, k_prime=%d need %zu bytes of scratch, the fixed array holds %u; pass scores_out, "
                "split the batch, or call misa_rerank_topk with a workspace",
                who, qs->n_q, k_prime, need, MISA_NOALLOC_SCRATCH_BYTES);
  if (injected_failure(who, &st)) return st;
  void *ws = nullptr;
  if ((st = noalloc_scratch(who, &ws)) != MISA_OK) return st;
  if (qs->n_q == 0) return MISA_OK;
  misa::CacheView c = view(cache);
  misa::QueryView q = view(qs);
  uint32_t *hist = static_cast<uint32_t *>(ws);
  float *scores = scores_out ? scores_out : reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + ws_hist(qs));
  cudaError_t e = misa::launch_zero(hist, (size_t)qs->n_q * misa::TOPK_HIST_BINS, stream);
  if (e != cudaSuccess) return cuda_fail(e, who);
  e = timed_scoring(stream, [&] {
    return misa::launch_score_mma(c, q, nullptr, q.H, cand, k_prime, scores, k_prime, hist, stream);
  });
  if (e != cudaSuccess) return cuda_fail(e, who);
  e = misa::launch_topk(c, q, scores, k_prime, k_prime, cand, hist, true, nullptr, nullptr, k, topk, stream);
  if (e != cudaSuccess) return cuda_fail(e, who);
  return MISA_OK;
}

misa_status misa_dagger_topk(const misa_cache *cache, const misa_queries *qs, const int32_t *heads, int32_t h,
                             int32_t k_prime, int32_t k, int32_t *topk, void *ws, size_t ws_bytes,
                             misa_stream stream) {
  NvtxRange nvtx("misa_dagger_topk");
  const char *who = "misa_dagger_topk";
  misa_status st = check_cache(cache, false);
  if (st != MISA_OK) return st;
  if ((st = check_queries(qs)) != MISA_OK) return st;
  if (h < 1 || h > qs->H) return fail(MISA_ERR_INVALID, "h=%d outside [1, H=%d]", h, qs->H);
  if (k < 1 || k_prime < k) return fail(MISA_ERR_INVALID, "need 1 <= k=%d <= k_prime=%d", k, k_prime);
  if (k_prime > MISA_MAX_L) return fail(MISA_ERR_UNSUPPORTED, "k_prime=%d above %d", k_prime, MISA_MAX_L);
  if (qs->n_q > 0 && (!heads || !topk)) return fail(MISA_ERR_INVALID, "heads/topk is NULL");
  if ((st = check_ws(ws, ws_bytes, ws_dagger(cache, qs, k_prime, k))) != MISA_OK) return st;
  if (injected_failure(who, &st)) return st;
  if (qs->n_q == 0) return MISA_OK;
  return dagger_body(who, cache, qs, heads, h, k_prime, k, topk, ws, stream);
}

misa_status misa_dagger_decode(const misa_cache *cache, const misa_queries *qs, const void *new_keys,
                               const float *new_scale, const int32_t *new_pos, int32_t count, int32_t h,
                               int32_t k_prime, int32_t k, int32_t *heads, int32_t *topk, void *ws, size_t ws_bytes,
                               misa_stream stream) {
  NvtxRange nvtx("misa_dagger_decode");
  const char *who = "misa_dagger_decode";
  misa_status st = check_cache(cache, true);
  if (st != MISA_OK) return st;
  if ((st = check_queries(qs)) != MISA_OK) return st;
  if (count < 1 || count > cache->L_cap)
    return fail(MISA_ERR_INVALID, "count=%d outside [1, L_cap=%d]", count, cache->L_cap);
  if (!new_keys || !new_pos) return fail(MISA_ERR_INVALID, "new_keys and new_pos must be non-NULL");
  if ((cache->dtype == MISA_KEY_FP8_E4M3) != (new_scale != nullptr))
    return fail(MISA_ERR_INVALID, "new_scale must be non-NULL exactly for fp8 keys");
  if (!aligned16(new_keys)) return fail(MISA_ERR_INVALID, "new_keys must be 16-byte aligned");
  if (h < 1 || h > qs->H) return fail(MISA_ERR_INVALID, "h=%d outside [1, H=%d]", h, qs->H);
  if (k < 1 || k_prime < k) return fail(MISA_ERR_INVALID, "need 1 <= k=%d <= k_prime=%d", k, k_prime);
  if (k_prime > MISA_MAX_L) return fail(MISA_ERR_UNSUPPORTED, "k_prime=%d above %d", k_prime, MISA_MAX_L);
  if (qs->n_q > 0 && !topk) return fail(MISA_ERR_INVALID, "topk is NULL");
  if ((st = check_ws(ws, ws_bytes, ws_decode(cache, qs, h, k_prime, k))) != MISA_OK) return st;
  if (injected_failure(who, &st)) return st;
  misa::CacheView c = view(cache);
  misa::QueryView q = view(qs);
  uint8_t *w8 = static_cast<uint8_t *>(ws);
  uint8_t *rws = w8 + ws_dagger(cache, qs, k_prime, k);
  int32_t *hbuf = heads ? heads : reinterpret_cast<int32_t *>(rws + ws_decode_router(cache, qs));
  // decode batches whose scoring grid is resident at once: routing inside the
  // routed scoring kernel, both selections inside their scoring kernels, and
  // their counting words cleared by the append kernel
  const bool fused = qs->n_q > 0 && !misa::umma_applies(c, q, nullptr, h) &&
                     misa::score_stream_fusable(c, q, nullptr, h, true);
  uint32_t *z0 = nullptr;
  size_t zn = 0;
  if (fused) {
    // the re-rank's fusion does not depend on the candidates' values
    const bool f2 =
        g_select_in_kernel.load() && misa::score_fusable(c, q, nullptr, q.H, reinterpret_cast<const int32_t *>(w8), k_prime);
    const bool cluster = !f2 && misa::rerank_cluster_applies(c, q, k_prime, k);
    // words the step counts into: the routed pass's selection words, then
    // the re-rank's (in-kernel selection), or its histograms just before them
    // (separate top-k kernels); the cluster re-rank counts in shared memory
    const size_t fz1 = ws_dagger_hist(qs) / sizeof(uint32_t), fzw = (size_t)qs->n_q * misa::FUSED_ZERO_WORDS;
    const size_t first = cluster || f2 ? fz1 : ws_hist(qs) / sizeof(uint32_t);
    const size_t last = f2 ? fz1 + round_up(sizeof(uint32_t) * fzw) / sizeof(uint32_t) + fzw : fz1 + fzw;
    z0 = reinterpret_cast<uint32_t *>(w8) + first;
    zn = last - first;
  }
  // fused: the routed pass routes while the append runs (it reads nothing
  // the append writes before waiting for it)
  cudaError_t e = misa::launch_pool_append(c, new_keys, new_scale, new_pos, count, stream, z0, zn, fused);
  if (e != cudaSuccess) return cuda_fail(e, who);
  if (qs->n_q == 0) return MISA_OK;
  if (fused) {
    misa::PendingAppend pa;
    pa.keys = new_keys;
    pa.scale = new_scale;
    pa.pos = new_pos;
    pa.count = count;
    return dagger_body(who, cache, qs, nullptr, h, k_prime, k, topk, ws, stream, reinterpret_cast<float *>(rws),
                       heads, true, &pa);
  }
  e = misa::launch_route(c, q, h, hbuf, nullptr, rws, stream, MISA_AGG_ABS_SUM);
  if (e != cudaSuccess) return cuda_fail(e, who);
  return dagger_body(who, cache, qs, hbuf, h, k_prime, k, topk, ws, stream);
}

misa_status misa_debug_wait_timeout(uint32_t *status, uint64_t limit_ns, misa_stream stream) {
  NvtxRange nvtx("misa_debug_wait_timeout");
  if (!status) return fail(MISA_ERR_INVALID, "status is NULL");
  if (limit_ns > 10000000000ull) return fail(MISA_ERR_INVALID, "limit_ns=%llu above 10 s", (unsigned long long)limit_ns);
  cudaError_t e = misa::launch_kernel(wait_timeout_kernel, dim3(1), dim3(32), 0, stream, status,
                                      (unsigned long long)limit_ns);
  if (e != cudaSuccess) return cuda_fail(e, "misa_debug_wait_timeout");
  return MISA_OK;
}

const char *misa_last_error(void) { return g_err; }

const char *misa_status_name(int32_t status) {
  switch (status) {
    case MISA_OK: return "MISA_OK";
    case MISA_ERR_INVALID: return "MISA_ERR_INVALID";
    case MISA_ERR_UNSUPPORTED: return "MISA_ERR_UNSUPPORTED";
    case MISA_ERR_WORKSPACE: return "MISA_ERR_WORKSPACE";
    case MISA_ERR_CUDA: return "MISA_ERR_CUDA";
    default: return "MISA_STATUS_UNKNOWN";
  }
}

int32_t misa_version(void) { return 1; }

void misa_debug_fail_next(int32_t n) { g_fail_next.store(n > 0 ? n : 0); }

void misa_debug_select_in_kernel(int32_t on) { g_select_in_kernel.store(on ? 1 : 0); }

void misa_debug_time_scoring(void *start, void *stop) {
  g_ev_start.store(start);
  g_ev_stop.store(stop);
}

}  // extern "C"
