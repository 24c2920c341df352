// Shared device helpers of the QSA kernels (sm_100a): the per-device error
// word, bounded mbarrier waits, bulk (TMA-engine) copies and cp.async.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace qsa {

// Error bits of the per-device error word (read by qsa_get_device_error).
enum : uint32_t {
  kErrBounds = 1u,    // block-table entry / logical page / position out of range
  kErrTimeout = 2u,   // a bounded wait ran out
  kErrBadInput = 4u,  // malformed lengths, counts or selection rows
};

// One word per device: every kernel ORs its findings in; the host reads and
// clears it after synchronising.
__device__ uint32_t g_error_flags;

__device__ __forceinline__ void record_error(uint32_t bits) { atomicOr(&g_error_flags, bits); }

// Programmatic dependent launch.  The library launches its kernels (all
// but compress_append, see qsa_api.cu) with programmatic stream
// serialisation: such a kernel may be
// scheduled once every CTA of the kernel before it has started, so its
// CTAs are resident, past their launch, when that kernel ends.  Every kernel
// opens with pdl_open() before anything else: it lets the next kernel
// launch, then waits until the work before it on the stream has completed
// and its memory is visible.  Without a programmatic dependency (a kernel
// from elsewhere, a copy) the wait returns at once.
__device__ __forceinline__ void pdl_open() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// A bounded wait gives up after about this many SM cycles (~1 s at 1.9 GHz).
constexpr long long kWaitCycles = 2000000000LL;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier --
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

// Makes mbarrier initialisation visible to the async (bulk copy) proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete.  Gives up after
// kWaitCycles, records kErrTimeout and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) {
      record_error(kErrTimeout);
      return false;
    }
  }
  return true;
}

// Same, but shares a CTA-wide abort flag: once any thread of the CTA has
// given up, every later wait returns false at once (so a stalled pipeline
// costs one timeout, not one per stage).
__device__ __forceinline__ bool mbar_wait_abortable(uint64_t *bar, uint32_t parity,
                                                    volatile int *abort_flag) {
  if (*abort_flag) return false;
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitCycles) {
      record_error(kErrTimeout);
      *abort_flag = 1;
      return false;
    }
  }
  return true;
}

// -------------------------------------------------------------- bulk copy --
// L2 policy: streamed data that is read once.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// Global -> shared bulk copy completed on `bar` (complete_tx).  dst, src and
// bytes must be multiples of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// --------------------------------------------------------------- cp.async --
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
// Same, zero-filling the 16 bytes instead of reading when `valid` is false
// (the source address is then not accessed).
__device__ __forceinline__ void cp_async16_zfill(void *dst, const void *src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------------- named barriers --
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ------------------------------------------------------------ utilities --
__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ long long ceil_div_ll(long long a, long long b) {
  return (a + b - 1) / b;
}

__device__ __forceinline__ int ld_cg_s32(const int32_t *p) {
  int v;
  asm volatile("ld.global.cg.s32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ int4 ld_cg_v4(const int32_t *p) {
  int4 v;
  asm volatile("ld.global.cg.v4.s32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ float4 ld_cg_f4(const float *p) {
  float4 v;
  asm volatile("ld.global.cg.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ float ld_cg_f32(const float *p) {
  float v;
  asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
}

// Cache description passed to kernels by value.
struct CacheDev {
  int num_pages, page_size, num_kv_heads, head_dim, idx_dim, kv_dtype;
  const void *k_cache, *v_cache;
  const float *k_scale, *v_scale;
  int16_t *kc;
  int8_t *ring;
  int ring_rows;
  const int32_t *block_table;
  int max_pages_per_req;
};

// Physical page of logical page `lp` of request r, or -1 (and an error bit)
// when the logical page lies outside the block table or the entry is not a
// valid page.
__device__ __forceinline__ int physical_page(const CacheDev &c, int r, long long lp) {
  if (lp < 0 || lp >= c.max_pages_per_req) {
    record_error(kErrBounds);
    return -1;
  }
  const int p = c.block_table[(long long)r * c.max_pages_per_req + lp];
  if (p < 0 || p >= c.num_pages) {
    record_error(kErrBounds);
    return -1;
  }
  return p;
}

}  // namespace qsa
