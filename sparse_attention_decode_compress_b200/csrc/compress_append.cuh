// qsa_compress_append: raw indexer keys -> ring + compressed-key cache.
//
// Method: micro-block compression at ratio 4 (blog "Qwen 4 QSA 迎来解码上下文
// 并行…", section 拉取请求实际改变了什么); the raw keys of positions not yet
// pooled live in a circular cache and the pooled keys in a compressed-key
// cache, both updated before selection (PR #53896 完整报告, QSAIndexer.forward
// excerpt).  Pooling = plain int sum; a partial block holds the sum of the
// tokens present so far.
//
// Launch: grid (chunks, B).  Each CTA refreshes up to kBlocksPerCta
// micro-blocks of one request; a group of d/16 threads owns one block row,
// each thread 16 dimensions (16 bytes per token in; 16 low bytes and one
// 32-bit word of high fields out, in the packed page layout of
// qsa_common.cuh).  Only the first micro-block of a call can hold positions
// older than pos0; it belongs to chunk 0, which reads those raw keys from
// the ring and only then (after a barrier) overwrites the ring with the
// newest positions.
#pragma once
#include "qsa_common.cuh"

namespace qsa {

constexpr int kAppendThreads = 256;
constexpr int kAppendBlocksPerCta = 64;

template <int DI>
__global__ void __launch_bounds__(kAppendThreads) compress_append_kernel(
    CacheDev c, int B, const int32_t *__restrict__ pos0, const int32_t *__restrict__ cu_new,
    const int8_t *__restrict__ k_new, int max_new) {
  pdl_open();
  constexpr int kThreadsPerRow = DI / 16;
  constexpr int kRowsPerIter = kAppendThreads / kThreadsPerRow;
  const int r = blockIdx.y;
  const int a = cu_new[r];
  const int n_new = cu_new[r + 1] - a;
  const int p0 = pos0[r];
  if (n_new < 0 || n_new > max_new || p0 < 0) {
    if (blockIdx.x == 0 && threadIdx.x == 0) record_error(kErrBadInput);
    return;
  }
  if (n_new == 0) return;
  const long long pend = (long long)p0 + n_new;
  const long long b_first = p0 / 4;
  const long long b_last = (pend - 1) / 4;
  const long long nb = b_last - b_first + 1;
  const int bpp = c.page_size / 4;  // micro-blocks per page
  const long long page_bytes = kc_page_bytes(c.page_size, DI);
  const long long lo_bytes = kc_lo_bytes(c.page_size, DI);
  const int lane_row = threadIdx.x / kThreadsPerRow;
  const int dw = threadIdx.x % kThreadsPerRow;  // this thread's dims: 16*dw .. 16*dw+15
  const int8_t *ring_r = c.ring + (long long)r * 4 * DI;

  const long long blk0 = (long long)blockIdx.x * kAppendBlocksPerCta;
  for (int it = lane_row; it < kAppendBlocksPerCta; it += kRowsPerIter) {
    const long long bi = blk0 + it;
    if (bi >= nb) break;
    const long long b = b_first + bi;
    int s[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) s[j] = 0;
    const long long t_end = min(4 * b + 4, pend);
    for (long long t = 4 * b; t < t_end; ++t) {
      const int8_t *src = (t >= p0) ? k_new + (a + (t - p0)) * (long long)DI + 16 * dw
                                    : ring_r + (t & 3) * DI + 16 * dw;
#pragma unroll
      for (int j4 = 0; j4 < 4; ++j4) {
        const char4 v = *reinterpret_cast<const char4 *>(src + 4 * j4);
        s[4 * j4] += v.x;
        s[4 * j4 + 1] += v.y;
        s[4 * j4 + 2] += v.z;
        s[4 * j4 + 3] += v.w;
      }
    }
    const int page = physical_page(c, r, b / bpp);
    if (page < 0) continue;
    // low bytes of dims 4u .. 4u+3 in word u; high field of dim 4s' + k at
    // bits 8k + 2s'
    uint32_t lo[4] = {0u, 0u, 0u, 0u}, hi = 0u;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      lo[j / 4] |= (uint32_t)(s[j] & 255) << (8 * (j % 4));
      hi |= ((uint32_t)((s[j] >> 8) + 2) & 3u) << (8 * (j % 4) + 2 * (j / 4));
    }
    uint8_t *pg = c.kc + (long long)page * page_bytes;
    const int row = (int)(b % bpp);
    *reinterpret_cast<uint4 *>(pg + (long long)row * DI + 16 * dw) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    *reinterpret_cast<uint32_t *>(pg + lo_bytes + 4 * ((long long)dw * bpp + row)) = hi;
  }

  if (blockIdx.x != 0) return;
  __syncthreads();  // the ring reads of block b_first are done
  // Ring: slot p % 4 <- key of the newest position p (the last <= 4 of them).
  const long long q0 = max((long long)p0, pend - 4);
  constexpr int kChar4PerRow = DI / 4;
  for (int i = threadIdx.x; i < 4 * kChar4PerRow; i += kAppendThreads) {
    const long long p = q0 + i / kChar4PerRow;
    if (p >= pend) continue;
    const int d4 = (i % kChar4PerRow) * 4;
    *reinterpret_cast<char4 *>(c.ring + ((long long)r * 4 + (p & 3)) * DI + d4) =
        *reinterpret_cast<const char4 *>(k_new + (a + (p - p0)) * (long long)DI + d4);
  }
}

}  // namespace qsa
