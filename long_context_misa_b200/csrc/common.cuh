// Shared device helpers of the MISA / DSA indexer library (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include <atomic>
#include <utility>

#include "misa.h"  // include/ (on the -I path)

namespace misa {

constexpr int D = MISA_D;  // index-key width

// Device view of the caller's cache and queries (plain pointers, by value).
struct CacheView {
  const void *keys;
  const float *scale;
  int32_t *seq_len;
  float *pool;
  uint32_t *status;
  int n_seq, L_cap, B, fp8;
};

struct QueryView {
  const uint16_t *q;
  const float *w;
  const int32_t *q_seq;
  const int32_t *q_pos;
  int n_q, H;
};

__device__ __forceinline__ void flag(const CacheView &c, uint32_t bit) {
  if (c.status) atomicOr(c.status, bit);
}

// Prefix length L_i = q_pos + 1 of query i, clamped to its sequence.
__device__ __forceinline__ int query_prefix(const CacheView &c, const QueryView &qv, int i, int *seq) {
  int s = qv.q_seq[i], p = qv.q_pos[i];
  if (s < 0 || s >= c.n_seq || p < 0) {
    flag(c, MISA_DEV_BAD_POSITION);
    *seq = 0;
    return 0;
  }
  int len = min(c.seq_len[s], c.L_cap);
  int L = p + 1;
  if (L > len) {
    flag(c, MISA_DEV_BAD_POSITION);
    L = max(len, 0);
  }
  *seq = s;
  return L;
}

// query_prefix as it reads once an append kernel (launch_pool_append with
// new_pos, count) has set the sequences' lengths: for a caller that may run
// while that append still does.
__device__ __forceinline__ int query_prefix_appended(const CacheView &c, const QueryView &qv, int i, int *seq,
                                                     const int32_t *new_pos, int count) {
  int s = qv.q_seq[i], p = qv.q_pos[i];
  if (s < 0 || s >= c.n_seq || p < 0) {
    flag(c, MISA_DEV_BAD_POSITION);
    *seq = 0;
    return 0;
  }
  const int ap = new_pos[s];
  const bool appended = ap >= 0 && (long long)ap + count <= c.L_cap;  // else the append leaves the sequence alone
  int len = min(appended ? ap + count : c.seq_len[s], c.L_cap);
  int L = p + 1;
  if (L > len) {
    flag(c, MISA_DEV_BAD_POSITION);
    L = max(len, 0);
  }
  *seq = s;
  return L;
}

// Order-preserving map of fp32 onto uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t ordered_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b16) { return __uint_as_float(b16 << 16); }

// Two packed bf16 (low half first) -> float2.
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t v) {
  return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xFFFF0000u));
}

// Two e4m3 codes (low byte first) -> two exact f16 values packed in one register.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t v) {
  __half2_raw r = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)v, __NV_E4M3);
  return (uint32_t)r.x | ((uint32_t)r.y << 16);
}

__device__ __forceinline__ float2 f16x2_to_float2(uint32_t v) {
  __half2 h = *reinterpret_cast<__half2 *>(&v);
  return __half22float2(h);
}

// bf16 bits -> f16 bits (round to nearest; exact for |x| in [2^-14, 65504]
// and for bf16 values whose 8 significant bits fit f16 subnormals).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) {
  float2 f = bf16x2_to_float2(v);
  __half2 h = __floats2half2_rn(f.x, f.y);
  return *reinterpret_cast<uint32_t *>(&h);
}

// Warp-level tensor-core MMA m16n8k16, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ldg_stream(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__host__ __device__ constexpr int cdiv(int a, int b) { return (a + b - 1) / b; }

// Programmatic dependent launch.  Every kernel of the library is launched
// with programmatic stream serialisation and calls grid_dep_sync() as its
// first statement: the kernel's launch and block scheduling may then overlap
// the previous kernel's last blocks and its completion, and the wait holds
// every thread until the previous grid has completed with its writes
// visible.  Kernels do not trigger their dependents early, so a successor's
// blocks are scheduled only as this kernel's blocks exit (waiting successor
// blocks that sat beside a running prefill kernel cost 45 us of a 0.7 ms
// call).  One pair is the exception: the decode step's append kernel
// triggers at once, and the routed scoring kernel after it routes before its
// wait, reading only inputs the append does not write (score_stream.cu).
// Because the wait comes before any global access, tensor memory allocation
// or early return in every kernel, every earlier kernel is complete
// (transitively) before a kernel reads anything, and no kernel requests
// tensor memory while its predecessor still holds some.
__device__ __forceinline__ void grid_dep_sync() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// The first statement of a kernel that may be launched early on purpose:
// the wait, unless `early`; the kernel then calls grid_dep_sync() itself
// before it reads anything its predecessor writes.
__device__ __forceinline__ void grid_dep_sync_unless(bool early) {
  if (!early) grid_dep_sync();
}
// Let the dependent grid be scheduled now (it still waits for this grid's
// completion at its own grid_dep_sync()).
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Kernel launch through cudaLaunchKernelEx, with the programmatic
// serialisation attribute above.
template <class... KArgs, class... Args>
inline cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                 Args &&...args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Per-device cached integer (device attributes, occupancy results): computed
// once per device by `f` on first use, then read without driver calls.
constexpr int MAX_DEVICES = 64;
template <class Tag, class F>
inline int cached_per_device(F &&f) {
  static std::atomic<int> cache[MAX_DEVICES];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= MAX_DEVICES) return f();
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    v = f();
    cache[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

// Raise a kernel's dynamic shared-memory limit to the most the device allows
// next to the kernel's own static shared memory.  Returns that limit (bytes)
// or -1 on failure.
template <class K>
inline int opt_in_max_dyn_smem(K *kernel) {
  int dev = 0, optin = 0;
  cudaFuncAttributes fa;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
      cudaFuncGetAttributes(&fa, kernel) != cudaSuccess)
    return -1;
  const int mx = optin - (int)fa.sharedSizeBytes;
  if (mx <= 0 || cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, mx) != cudaSuccess)
    return -1;
  // all of the SM's configurable memory as shared memory: the occupancy
  // query (and the co-residency a fused selection relies on) then counts
  // the CTAs that really fit
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared) != cudaSuccess)
    return -1;
  return mx;
}

struct SmCountTag {};
inline int device_sms() {
  return cached_per_device<SmCountTag>([] {
    int dev = 0, v = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    return v;
  });
}

}  // namespace misa

namespace misa {

// ---------------------------------------------------------------------------
// mbarrier / bulk-copy helpers (sm_90+ PTX), with time-bounded waits.
// ---------------------------------------------------------------------------

// Longest time any on-chip pipeline wait may take before the kernel gives up,
// records MISA_DEV_WAIT_TIMEOUT and returns (nanoseconds of %globaltimer).
constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of `bar` to complete; false once `limit_ns`
// (default WAIT_LIMIT_NS) has passed.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns = WAIT_LIMIT_NS) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > limit_ns) return false;
  return true;
}

// cp.async (LDGSTS) copies global -> shared; `valid` false copies nothing
// and zero-fills the destination (the source address must still be valid).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(valid ? 4 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// The tensor-core kernels lay out their shared memory from the first
// 1024-byte boundary of the dynamic allocation (the 128-byte-swizzle atoms of
// TMA destinations and MMA operands need it), and every launch allocates
// 1024 bytes of slack for that.  Returns the aligned base, or nullptr when
// `need` bytes from it do not fit in the dynamic shared memory the kernel was
// launched with (a layout and an allocation that disagree): thread 0 then
// flags MISA_DEV_SMEM_LAYOUT and the caller returns before any shared-memory
// access.  The answer is the same in every thread.
__device__ __forceinline__ uint8_t *aligned_smem_base(uint8_t *raw, uint32_t need, const CacheView &c) {
  const uint32_t pad = (1024u - (smem_addr(raw) & 1023u)) & 1023u;
  uint32_t dyn;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
  if (pad + need > dyn) {
    if (threadIdx.x == 0) flag(c, MISA_DEV_SMEM_LAYOUT);
    return nullptr;
  }
  return raw + pad;
}

// Bulk (non-tensor) copy global -> this CTA's shared memory, completing on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

}  // namespace misa
