// Shared device helpers of the QSA kernels (sm_100a): the per-device error
// word, programmatic launch, cp.async, named barriers and L2 policies.
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
  kErrTimeout = 2u,   // a bounded wait ran out (kept for the ABI; no kernel of this version waits)
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

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------- L2 policy --
// Streamed data that is read once.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
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

// Packed compressed-key page (P tokens, R = P/4 micro-block rows, indexer
// dim d): a key value v (a sum of 4 int8 keys, -512 <= v <= 508) is stored
// as its low byte v & 255 and a 2-bit high field (v >> 8) + 2 in [0, 3], so
// v = 256 * (field - 2) + low byte.  A page holds the R rows of d low bytes,
// then the high fields as 32-bit words, then padding to 16 bytes.  Word
// (w, row) holds the fields of dims 16w .. 16w+15 of a row and sits at word
// index w * R + row of the high part (dim-group major, so four consecutive
// rows of one dim group are 16 contiguous bytes); dim 16w + 4s + k is at bits
// 8k + 2s, so (word >> 2s) & 0x03030303 holds the fields of dims
// 16w + 4s .. 16w + 4s + 3 in its four bytes.
__host__ __device__ __forceinline__ long long kc_lo_bytes(int page_size, int d) {
  return (long long)(page_size / 4) * d;
}
__host__ __device__ __forceinline__ long long kc_page_bytes(int page_size, int d) {
  return kc_lo_bytes(page_size, d) + (((long long)(page_size / 4) * (d / 4) + 15) / 16) * 16;
}

// Cache description passed to kernels by value.
struct CacheDev {
  int num_pages, page_size, num_kv_heads, head_dim, idx_dim, kv_dtype;
  const void *k_cache, *v_cache;
  const float *k_scale, *v_scale;
  uint8_t *kc;  // packed compressed keys, kc_page_bytes per page
  int8_t *ring;
  int ring_rows;
  const int32_t *block_table;
  int max_pages_per_req;
  // row of block_table of each request, or NULL for row r: the queries of
  // a prefill share their request's row
  const int32_t *table_row;
};

// Physical page of logical page `lp` of request r, or -1 (and an error bit)
// when the logical page lies outside the block table or the entry is not a
// valid page.
__device__ __forceinline__ int physical_page(const CacheDev &c, int r, long long lp) {
  if (lp < 0 || lp >= c.max_pages_per_req) {
    record_error(kErrBounds);
    return -1;
  }
  const long long row = c.table_row ? (long long)c.table_row[r] : (long long)r;
  const int p = c.block_table[row * c.max_pages_per_req + lp];
  if (p < 0 || p >= c.num_pages) {
    record_error(kErrBounds);
    return -1;
  }
  return p;
}

}  // namespace qsa
