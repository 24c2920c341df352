// Normalised-pooling indexer: float compressed keys and float block scores.
//
// Method: the indexer pools each 4-token micro-block's raw keys by the
// compress ratio and normalises the result before it enters the
// compressed-key cache (PR #53896 完整报告, QSAIndexer.forward excerpt under
// 关键源码片段; the module list under 实现拆解 names an RMS norm for the
// indexer, apply_qsa_rmsnorm).  Pooling is read as the mean of the tokens
// present in the block, the normalisation as RMS normalisation
//   k_c = m / sqrt(mean_j m_j^2 + eps) * (1 + w_j),   m = block mean,
// and the score as the float dot product with the indexer query; the
// selection is that of the integer indexer (index_topk.cuh) on float keys.
//
// Storage: raw keys (and the ring of the newest 4 positions) are bf16; the
// compressed keys are stored as fp16 (|k_c| <= sqrt(d) * max|1 + w|, within
// fp16 range, 11 significant bits) in pages of [P/4 rows][d] that share the
// block table of the K/V cache.
//
// Kernels:
//   compress_append_norm_kernel<d>  grid (chunks, B): a group of d/8 threads
//     owns one block row (8 dims each: 16 bytes of bf16 in, 16 bytes of fp16
//     out); the mean square is reduced across the group with shuffles.
//   index_scan_norm_kernel<d>  persistent warps over items of 16 * (256/d)
//     rows: 16-byte streaming loads of fp16 keys, fp32 dot products, a
//     butterfly reduce-scatter across the d/8 lanes of a row, float score
//     bits written to the L2-resident score buffer, which select_kernel
//     <FloatKeys> then reads.
#pragma once
#include "index_topk.cuh"

namespace qsa {
namespace norm {

constexpr int kAppendThreads = 256;
constexpr int kAppendBlocksPerCta = 64;

struct AppendParams {
  CacheDev c;           // geometry and block table (kc / ring of the integer indexer unused)
  __half *kcn;          // [num_pages, P/4, d] fp16 normalised compressed keys
  __nv_bfloat16 *ring;  // [ring_rows, 4, d] bf16 raw keys of the newest positions
  const float *weight;  // [d] or NULL: the norm's per-dim weight w, applied as (1 + w)
  float eps;
  int B;
  const int32_t *pos0, *cu_new;
  const __nv_bfloat16 *k_new;  // [N, d]
  int max_new;
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4 v, float (&f)[8]) {
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x = __bfloat1622float2(h[i]);
    f[2 * i] = x.x;
    f[2 * i + 1] = x.y;
  }
}

template <int DI>
__global__ void __launch_bounds__(kAppendThreads) compress_append_norm_kernel(AppendParams a) {
  pdl_open();
  constexpr int kG = DI / 8;  // threads per block row
  constexpr int kRowsPerIter = kAppendThreads / kG;
  const CacheDev &c = a.c;
  const int r = blockIdx.y;
  const int base = a.cu_new[r];
  const int n_new = a.cu_new[r + 1] - base;
  const int p0 = a.pos0[r];
  if (n_new < 0 || n_new > a.max_new || p0 < 0) {
    if (blockIdx.x == 0 && threadIdx.x == 0) record_error(kErrBadInput);
    return;
  }
  if (n_new == 0) return;
  const long long pend = (long long)p0 + n_new;
  const long long b_first = p0 / 4;
  const long long nb = (pend - 1) / 4 - b_first + 1;
  const int bpp = c.page_size / 4;
  const int lane = threadIdx.x & 31;
  const int lane_row = threadIdx.x / kG;
  const int dw = threadIdx.x % kG;  // dims 8*dw .. 8*dw+7
  const unsigned gmask = ((kG == 32) ? 0xffffffffu : ((1u << kG) - 1u)) << (lane & ~(kG - 1));
  const __nv_bfloat16 *ring_r = a.ring + (long long)r * 4 * DI;
  float w1[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) w1[j] = 1.f + (a.weight ? a.weight[8 * dw + j] : 0.f);

  const long long blk0 = (long long)blockIdx.x * kAppendBlocksPerCta;
  for (int it = lane_row; it < kAppendBlocksPerCta; it += kRowsPerIter) {
    const long long bi = blk0 + it;
    if (bi >= nb) break;  // uniform across the row's group
    const long long b = b_first + bi;
    float s[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) s[j] = 0.f;
    const long long t_end = min(4 * b + 4, pend);
    for (long long t = 4 * b; t < t_end; ++t) {
      const __nv_bfloat16 *src = (t >= p0) ? a.k_new + (base + (t - p0)) * (long long)DI + 8 * dw
                                           : ring_r + (t & 3) * DI + 8 * dw;
      float f[8];
      bf16x8_to_f32(*reinterpret_cast<const uint4 *>(src), f);
#pragma unroll
      for (int j = 0; j < 8; ++j) s[j] += f[j];
    }
    const float cnt = (float)(t_end - 4 * b);
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) ss = fmaf(s[j], s[j], ss);
#pragma unroll
    for (int o = kG / 2; o >= 1; o >>= 1) ss += __shfl_xor_sync(gmask, ss, o);
    // mean m = s / cnt; mean_j m_j^2 = ss / (d cnt^2)
    const float ms = ss / ((float)DI * cnt * cnt);
    const float inv = 1.f / (cnt * sqrtf(ms + a.eps));
    const int page = physical_page(c, r, b / bpp);
    if (page < 0) continue;
    __align__(16) __half h[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) h[j] = __float2half_rn(s[j] * inv * w1[j]);
    __half *dst = a.kcn + ((long long)page * bpp + (b % bpp)) * DI + 8 * dw;
    *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<const uint4 *>(h);
  }

  if (blockIdx.x != 0) return;
  __syncthreads();  // the ring reads of block b_first are done
  const long long q0 = max((long long)p0, pend - 4);
  constexpr int kVecPerRow = DI / 8;  // 16-byte vectors per bf16 row
  for (int i = threadIdx.x; i < 4 * kVecPerRow; i += kAppendThreads) {
    const long long p = q0 + i / kVecPerRow;
    if (p >= pend) continue;
    const int d8 = (i % kVecPerRow) * 8;
    *reinterpret_cast<uint4 *>(a.ring + ((long long)r * 4 + (p & 3)) * DI + d8) =
        *reinterpret_cast<const uint4 *>(a.k_new + (base + (p - p0)) * (long long)DI + d8);
  }
}

// ------------------------------------------------------------- the scan --
struct ScanParams {
  topk::Params p;        // request lengths, scores buffer (float bits), selection
  const __half *kcn;     // [num_pages, P/4, d]
  const __nv_bfloat16 *q;  // [B, d]
};

constexpr int kScanThreads = 128;
constexpr int kItemLoads = 16;

// Float reduce-scatter of 16 per-lane partial sums over groups of LPR lanes
// (as topk::reduce_scatter16): afterwards lane l holds 16/LPR sums, value k
// being load index ((l % LPR) << (4 - log2 LPR)) | k.
template <int LPR>
__device__ __forceinline__ void reduce_scatter16f(float (&v)[16], int lane) {
  int n = 16;
#pragma unroll
  for (int o = LPR / 2; o >= 1; o >>= 1) {
    const bool upper = (lane & o) != 0;
    const int h = n / 2;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i < h) {
        const float send = upper ? v[i] : v[i + h];
        const float keepv = upper ? v[i + h] : v[i];
        v[i] = keepv + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
    n = h;
  }
}

template <int DI>
__global__ void __launch_bounds__(kScanThreads) index_scan_norm_kernel(ScanParams sp) {
  pdl_open();
  static_assert(DI == 32 || DI == 64 || DI == 128, "indexer dim");
  const topk::Params &p = sp.p;
  constexpr int kLPR = DI / 8;                     // lanes per row (8 dims, 16 bytes each)
  constexpr int kRPI = 32 / kLPR;                  // rows per load instruction
  constexpr int kRowsPerItem = kItemLoads * kRPI;
  constexpr int kR = (kLPR == 16) ? 4 : (kLPR == 8) ? 3 : 2;  // log2(kLPR)
  constexpr int kVals = 16 >> kR;
  const int lane = threadIdx.x & 31;
  const long long warp_id = ((long long)blockIdx.x * kScanThreads + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * kScanThreads) >> 5;
  const int bpp = p.c.page_size / 4;
  const int sub = lane % kLPR;
  const int grp = lane / kLPR;
  const uint64_t pol_stream = l2_policy_evict_first();
  const uint64_t pol_keep = topk::l2_policy_evict_last();
  topk::ItemWalker wk;
  wk.start(p, kRowsPerItem, warp_id == 0 && lane == 0);
  int cur_r = -1;
  float q[8];

  auto fetch_pages = [&](int r, int row0, int &lp0_out) -> int {
    const int lp0 = row0 / bpp;
    lp0_out = lp0;
    const int lp = lp0 + lane;
    int v = -1;
    if (lp < p.c.max_pages_per_req) {
      v = p.c.block_table[(long long)r * p.c.max_pages_per_req + lp];
      if (v >= p.c.num_pages) v = -1;
    }
    return v;
  };

  long long it = warp_id;
  if (!wk.seek(p, it)) return;
  int nr = wk.r;
  int nrow0 = (int)(it - wk.cum) * kRowsPerItem;
  int nlp0 = 0;
  int npg = fetch_pages(nr, nrow0, nlp0);
  while (true) {
    const int r = nr, row0 = nrow0, lp0 = nlp0, pg_lane = npg;
    const int n = wk.n;
    if (r != cur_r) {
      cur_r = r;
      float f[8];
      bf16x8_to_f32(*reinterpret_cast<const uint4 *>(sp.q + (long long)r * DI + 8 * sub), f);
#pragma unroll
      for (int j = 0; j < 8; ++j) q[j] = f[j];
    }
    uint4 v[kItemLoads];
#pragma unroll
    for (int i = 0; i < kItemLoads; ++i) {
      const int row = row0 + i * kRPI + grp;
      const int lp = row / bpp;
      const int rin = row - lp * bpp;
      const int j = lp - lp0;
      int pg = __shfl_sync(0xffffffffu, pg_lane, j & 31);
      if (j >= 32) {
        pg = (lp < p.c.max_pages_per_req) ? p.c.block_table[(long long)r * p.c.max_pages_per_req + lp] : -1;
        if (pg >= p.c.num_pages) pg = -1;
      }
      v[i] = make_uint4(0, 0, 0, 0);
      if (row < n) {
        if (pg >= 0) {
          v[i] = topk::scan_load(reinterpret_cast<const uint4 *>(
                                     sp.kcn + ((long long)pg * bpp + rin) * DI + 8 * sub),
                                 pol_stream);
        } else if (sub == 0) {
          record_error(kErrBounds);
        }
      }
    }
    it += nwarps;
    const bool more = wk.seek(p, it);
    if (more) {
      nr = wk.r;
      nrow0 = (int)(it - wk.cum) * kRowsPerItem;
      npg = fetch_pages(nr, nrow0, nlp0);
    }
    float acc[16];
#pragma unroll
    for (int i = 0; i < kItemLoads; ++i) {
      const __half2 *h = reinterpret_cast<const __half2 *>(&v[i]);
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 x = __half22float2(h[k]);
        a0 = fmaf(x.x, q[2 * k], a0);
        a1 = fmaf(x.y, q[2 * k + 1], a1);
      }
      acc[i] = a0 + a1;
    }
    reduce_scatter16f<kLPR>(acc, lane);
    int32_t *sc = p.scores + (long long)r * p.max_blocks;
#pragma unroll
    for (int k = 0; k < kVals; ++k) {
      const int i = ((lane % kLPR) << (4 - kR)) | k;
      const int row = row0 + i * kRPI + grp;
      if (row < n) topk::score_store(sc + row, __float_as_int(acc[k]), pol_keep);
    }
    if (!more) break;
  }
}

}  // namespace norm
}  // namespace qsa
