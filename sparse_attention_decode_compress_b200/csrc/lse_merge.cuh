// qsa_lse_merge: log-sum-exp combine of KV-partition partial attention.
//
// Method: partial attention results of the context slices are merged at the
// end (blog "Qwen 4 QSA 迎来解码上下文并行…", section 拉取请求实际改变了什么):
//   lse = log sum_s exp(lse_s),  o = sum_s exp(lse_s - lse) * o_s.
// One warp per output row; each lane handles float4 slices of the row, so
// every partial row is read once with 16-byte coalesced loads.
#pragma once
#include "qsa_common.cuh"

namespace qsa {

constexpr int kMergeThreads = 256;
constexpr int kMergeMaxSplits = 64;

// Merges output row `row` of S split partials (o_part [S, rows, D], lse_part
// [S, rows]) into o[row], lse[row]; one warp.  Lane s < S holds lse_s; the
// maximum and the sum of weights come from shuffles; each lane accumulates
// float4 slices in split order with explicit fused multiply-adds, so every
// caller (the merge kernel, the decode kernels' fused merge) gets the same
// bits.
__device__ __forceinline__ void merge_row(int S, long long rows, int D, const float *o_part,
                                          const float *lse_part, long long row, float *o,
                                          float *lse, int lane) {
  float mx = -INFINITY;
  for (int s = lane; s < S; s += 32) mx = fmaxf(mx, __ldcg(lse_part + (long long)s * rows + row));
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  float z = 0.f;
  for (int s = lane; s < S; s += 32) {
    const float l = __ldcg(lse_part + (long long)s * rows + row);
    z += (l == -INFINITY) ? 0.f : __expf(l - mx);
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
  const bool empty = (mx == -INFINITY) || !(z > 0.f);
  const float lse_row = empty ? -INFINITY : mx + __logf(z);
  if (lane == 0) lse[row] = lse_row;
  for (int d = lane * 4; d < D; d += 128) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (!empty) {
      for (int s = 0; s < S; ++s) {
        const float l = __ldcg(lse_part + (long long)s * rows + row);
        if (l == -INFINITY) continue;
        const float w = __expf(l - lse_row);
        const float4 v = __ldcg(reinterpret_cast<const float4 *>(o_part + ((long long)s * rows + row) * D + d));
        acc.x = __fmaf_rn(w, v.x, acc.x);
        acc.y = __fmaf_rn(w, v.y, acc.y);
        acc.z = __fmaf_rn(w, v.z, acc.z);
        acc.w = __fmaf_rn(w, v.w, acc.w);
      }
    }
    *reinterpret_cast<float4 *>(o + row * D + d) = acc;
  }
}

__global__ void __launch_bounds__(kMergeThreads) lse_merge_kernel(
    int S, long long rows, int D, const float *__restrict__ o_part,
    const float *__restrict__ lse_part, float *__restrict__ o, float *__restrict__ lse) {
  pdl_open();
  const long long row = (long long)blockIdx.x * (kMergeThreads / 32) + (threadIdx.x >> 5);
  if (row >= rows) return;
  merge_row(S, rows, D, o_part, lse_part, row, o, lse, threadIdx.x & 31);
}

}  // namespace qsa
