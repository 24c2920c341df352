// qsa_index_topk: weight-free block scoring + exact top-k selection.
//
// Method: the indexer scores every compressed micro-block against the query
// and keeps the best 512 (blog "Qwen 4 QSA 迎来解码上下文并行…", section
// 拉取请求实际改变了什么; PR #53896 完整报告, 执行摘要: weight-free top-k over
// the compressed-key cache; QSAIndexer.forward excerpt: fixed-width output
// padded with -1).  score = exact int32 dot(q_idx, kc); ties -> lower block
// index; kept blocks listed in ascending order.
//
// Design (B200): the scan is an HBM stream of int16 compressed keys
// (256 B per block at d = 128).  A persistent grid (2 CTAs per SM) walks
// fixed-size work units (request, run of blocks).  In each CTA one producer
// thread streams 4 KiB stages of compressed-key rows from their pages into a
// 16-stage shared-memory ring with cp.async.bulk (completion on mbarriers,
// L2 evict-first); eight consumer warps turn each stage into 16..64 scores
// with dp2a (int16 x int8 pairs) and a butterfly reduce-scatter, and write the
// scores to an L2-resident buffer.  The CTA that finishes the last unit of a
// request (atomic ticket) runs that request's selection while the other CTAs
// keep streaming: a 4096-bin histogram of the high score bits finds the
// threshold bin, the blocks above it are kept outright, the threshold bin's
// blocks are gathered in shared memory and bitonic-sorted by (score desc,
// index asc), and the kept indices are bitonic-sorted ascending.  A request
// whose threshold bin overflows shared memory falls back to exact radix
// passes over the score buffer.
#pragma once
#include "qsa_common.cuh"

namespace qsa {
namespace topk {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;  // + one producer warp
constexpr int kStageBytes = 4096;
constexpr int kStages = 16;
constexpr int kHistBins = 4096;  // first digit: bits [25:14] of score + 2^25
constexpr int kCandCap = 2048;   // threshold-bin candidates kept in shared memory
constexpr int kMaxTopk = 4096;
constexpr int kScoreBias = 1 << 25;  // |score| <= 2^23 for d <= 128 and int8 inputs
constexpr int kBarSelect = 1;        // named barrier of the consumer warps

struct Smem {
  alignas(128) uint8_t stage[kStages][kStageBytes];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  int hist[kHistBins];  // also the kept-index list (kMaxTopk ints) after pass A
  unsigned long long cand[kCandCap];
  int warp_tot[kConsumerWarps];
  int sel_req;     // request to select after this unit, or -1
  int bin, above;  // threshold bin and count strictly above it
  int nkeep, ncand;
  int fb_key, fb_above, fb_idx;  // fallback path results
  int abort_flag;                // a wait of this CTA gave up
};

struct Params {
  CacheDev c;
  int B;
  const int8_t *q_idx;
  const int32_t *ctx_lens;
  const int32_t *n_sel;
  int max_blocks;
  int topk;
  int32_t *sel;
  int32_t *scores;   // [B, max_blocks]
  int32_t *tickets;  // [B], zero between calls
  int unit_rows;     // multiple of the rows of one stage
};

// Competing blocks of request r, validated the same way in every thread:
// n = n_sel[r] (or ceil(L/4)), clipped to [0, min(ceil(L/4), max_blocks)].
// Only a caller with `report` set records a malformed request.
__device__ __forceinline__ int request_blocks(const Params &p, int r, bool report = false) {
  const int L = p.ctx_lens[r];
  const long long nb = ((long long)max(L, 0) + 3) / 4;
  long long n = p.n_sel ? (long long)p.n_sel[r] : nb;
  const long long lim = min(nb, (long long)p.max_blocks);
  if (L < 1 || n < 0 || n > lim) {
    if (report) record_error(kErrBadInput);
    n = (L < 1 || n < 0) ? 0 : lim;
  }
  return (int)n;
}

__device__ __forceinline__ int request_units(const Params &p, int n) {
  return n > 0 ? ceil_div(n, p.unit_rows) : 1;
}

// Walks the persistent unit sequence u = blockIdx.x, += gridDim.x, mapping
// each unit to (request, first row, rows).
struct UnitWalker {
  int r = 0, cum = 0, n = 0, units = 0;
  bool report = false;
  __device__ __forceinline__ void start(const Params &p, bool rep) {
    report = rep;
    r = 0;
    cum = 0;
    n = request_blocks(p, 0, report);
    units = request_units(p, n);
  }
  // Advances to the request holding unit u; returns false past the end.
  __device__ __forceinline__ bool seek(const Params &p, long long u) {
    while (r < p.B && u >= (long long)cum + units) {
      cum += units;
      ++r;
      if (r < p.B) {
        n = request_blocks(p, r, report);
        units = request_units(p, n);
      }
    }
    return r < p.B;
  }
};

// Order-preserving unsigned key of a score in [0, 2^26).  Valid inputs give
// |score| <= 2^23; the clamp only keeps corrupt cache contents from indexing
// outside the histogram.
__device__ __forceinline__ uint32_t score_key(int s) {
  s = max(min(s, kScoreBias - 1), -kScoreBias);
  return (uint32_t)(s + kScoreBias);
}

// ------------------------------------------------------------ selection --

__device__ __forceinline__ void bitonic_sort_u64(unsigned long long *a, int n_pow2, int tid) {
  for (int k = 2; k <= n_pow2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < n_pow2; i += kConsumers) {
        const int l = i ^ j;
        if (l > i) {
          const unsigned long long x = a[i], y = a[l];
          const bool up = (i & k) == 0;
          if ((x > y) == up) {
            a[i] = y;
            a[l] = x;
          }
        }
      }
      named_bar_sync(kBarSelect, kConsumers);
    }
  }
}

__device__ __forceinline__ void bitonic_sort_i32(int *a, int n_pow2, int tid) {
  for (int k = 2; k <= n_pow2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < n_pow2; i += kConsumers) {
        const int l = i ^ j;
        if (l > i) {
          const int x = a[i], y = a[l];
          const bool up = (i & k) == 0;
          if ((x > y) == up) {
            a[i] = y;
            a[l] = x;
          }
        }
      }
      named_bar_sync(kBarSelect, kConsumers);
    }
  }
}

__device__ __forceinline__ int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

// Finds, in hist[0..nbins), the bin where the running count taken from the
// top bin down (desc = true) or from bin 0 up first reaches `rank` (>= 1).
// Writes the bin and the count strictly before it (in that order) to *bin and
// *before.  Executed by all consumer threads; ends with a barrier.
__device__ void find_rank_bin(const int *hist, int nbins, int rank, bool desc, int *bin,
                              int *before, Smem &sm, int tid) {
  const int per = nbins / kConsumers;  // nbins is a multiple of kConsumers
  // thread t owns the t-th group of bins in the scan order
  int local = 0;
  for (int k = 0; k < per; ++k) {
    const int b = desc ? (nbins - 1 - (tid * per + k)) : (tid * per + k);
    local += hist[b];
  }
  // exclusive scan over threads in scan order
  int incl = local;
  const int lane = tid & 31, w = tid >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) sm.warp_tot[w] = incl;
  named_bar_sync(kBarSelect, kConsumers);
  int base = 0;
  for (int i = 0; i < w; ++i) base += sm.warp_tot[i];
  const int excl = base + incl - local;
  if (excl < rank && rank <= excl + local) {
    int cum = excl;
    for (int k = 0; k < per; ++k) {
      const int b = desc ? (nbins - 1 - (tid * per + k)) : (tid * per + k);
      if (cum + hist[b] >= rank) {
        *bin = b;
        *before = cum;
        break;
      }
      cum += hist[b];
    }
  }
  named_bar_sync(kBarSelect, kConsumers);
}

// Exact fallback when the threshold bin does not fit in shared memory:
// radix passes over the score buffer.  Establishes the exact threshold key,
// then (on a tie at the threshold) the largest kept index among the tied
// blocks, then gathers the kept set.
__device__ void select_fallback(const int32_t *sc, int n, int K, Smem &sm, int tid) {
  int *hist = sm.hist;
  const uint32_t b1 = (uint32_t)sm.bin;
  // pass: bits [13:7] among keys with digit1 == b1; then bits [6:0]
  uint32_t prefix = b1;  // key >> shift
  int above = sm.above;
  int shift = 14;
  const int widths[2] = {7, 7};
  for (int pass = 0; pass < 2; ++pass) {
    const int nb = 1 << widths[pass];
    const int nshift = shift - widths[pass];
    for (int i = tid; i < kHistBins; i += kConsumers) hist[i] = 0;
    named_bar_sync(kBarSelect, kConsumers);
    for (int i = tid; i < n; i += kConsumers) {
      const uint32_t k = score_key(ld_cg_s32(sc + i));
      if ((k >> shift) == prefix) atomicAdd(&hist[(k >> nshift) & (nb - 1)], 1);
    }
    named_bar_sync(kBarSelect, kConsumers);
    if (tid == 0) {
      int cum = above;
      for (int b = nb - 1; b >= 0; --b) {
        if (cum + hist[b] >= K) {
          sm.fb_key = b;
          sm.fb_above = cum;
          break;
        }
        cum += hist[b];
      }
    }
    named_bar_sync(kBarSelect, kConsumers);
    prefix = (prefix << widths[pass]) | (uint32_t)sm.fb_key;
    above = sm.fb_above;
    shift = nshift;
  }
  const uint32_t tkey = prefix;  // exact threshold key
  const int need = K - above;    // tied blocks to keep, lowest indices first
  // count ties; if some must be dropped, find the need-th smallest tied index
  if (tid == 0) sm.ncand = 0;
  named_bar_sync(kBarSelect, kConsumers);
  int myties = 0;
  for (int i = tid; i < n; i += kConsumers) myties += (score_key(ld_cg_s32(sc + i)) == tkey);
  atomicAdd(&sm.ncand, myties);
  named_bar_sync(kBarSelect, kConsumers);
  int idx_limit = 0x7fffffff;
  if (sm.ncand > need) {
    // radix select on the index (ascending), 3 passes of 8 bits over 24 bits
    uint32_t ipre = 0;
    int before = 0;
    for (int pass = 0; pass < 3; ++pass) {
      const int sh = 16 - 8 * pass;
      for (int i = tid; i < kHistBins; i += kConsumers) hist[i] = 0;
      named_bar_sync(kBarSelect, kConsumers);
      for (int i = tid; i < n; i += kConsumers) {
        if (score_key(ld_cg_s32(sc + i)) != tkey) continue;
        if (((uint32_t)i >> (sh + 8)) != ipre) continue;
        atomicAdd(&hist[((uint32_t)i >> sh) & 255], 1);
      }
      named_bar_sync(kBarSelect, kConsumers);
      if (tid == 0) {
        int cum = before;
        for (int b = 0; b < 256; ++b) {
          if (cum + hist[b] >= need) {
            sm.fb_idx = b;
            sm.fb_above = cum;
            break;
          }
          cum += hist[b];
        }
      }
      named_bar_sync(kBarSelect, kConsumers);
      ipre = (ipre << 8) | (uint32_t)sm.fb_idx;
      before = sm.fb_above;
    }
    idx_limit = (int)ipre;
  }
  // gather the kept set
  int *keep = sm.hist;
  if (tid == 0) sm.nkeep = 0;
  named_bar_sync(kBarSelect, kConsumers);
  for (int i = tid; i < n; i += kConsumers) {
    const uint32_t k = score_key(ld_cg_s32(sc + i));
    if (k > tkey || (k == tkey && i <= idx_limit)) {
      const int slot = atomicAdd(&sm.nkeep, 1);
      if (slot < kMaxTopk) keep[slot] = i;
    }
  }
  named_bar_sync(kBarSelect, kConsumers);
}

// Selection of request r by the kConsumers consumer threads.
__device__ void select_request(const Params &p, int r, Smem &sm, int tid) {
  const int n = request_blocks(p, r);
  const int K = p.topk;
  int32_t *out = p.sel + (long long)r * K;
  const int32_t *sc = p.scores + (long long)r * p.max_blocks;
  if (n <= K) {
    for (int i = tid; i < K; i += kConsumers) out[i] = i < n ? i : -1;
    return;
  }
  int *hist = sm.hist;
  // pass A: histogram of the first digit
  for (int i = tid; i < kHistBins; i += kConsumers) hist[i] = 0;
  named_bar_sync(kBarSelect, kConsumers);
  const int n4 = n & ~3;
  for (int i = tid * 4; i < n4; i += kConsumers * 4) {
    const int4 v = ld_cg_v4(sc + i);
    atomicAdd(&hist[score_key(v.x) >> 14], 1);
    atomicAdd(&hist[score_key(v.y) >> 14], 1);
    atomicAdd(&hist[score_key(v.z) >> 14], 1);
    atomicAdd(&hist[score_key(v.w) >> 14], 1);
  }
  for (int i = n4 + tid; i < n; i += kConsumers) atomicAdd(&hist[score_key(ld_cg_s32(sc + i)) >> 14], 1);
  named_bar_sync(kBarSelect, kConsumers);
  find_rank_bin(hist, kHistBins, K, true, &sm.bin, &sm.above, sm, tid);
  const uint32_t b1 = (uint32_t)sm.bin;
  // pass B: keep blocks above the bin; gather the bin's blocks
  int *keep = sm.hist;  // histogram no longer needed
  if (tid == 0) {
    sm.nkeep = 0;
    sm.ncand = 0;
  }
  named_bar_sync(kBarSelect, kConsumers);
  for (int i = tid; i < n; i += kConsumers) {
    const uint32_t k = score_key(ld_cg_s32(sc + i));
    const uint32_t d1 = k >> 14;
    if (d1 > b1) {
      const int slot = atomicAdd(&sm.nkeep, 1);
      if (slot < kMaxTopk) keep[slot] = i;
    } else if (d1 == b1) {
      const int slot = atomicAdd(&sm.ncand, 1);
      if (slot < kCandCap)
        sm.cand[slot] = ((unsigned long long)(0xffffffffu - k) << 32) | (uint32_t)i;
    }
  }
  named_bar_sync(kBarSelect, kConsumers);
  const int above = sm.above;
  const int ncand = sm.ncand;
  if (ncand <= kCandCap) {
    const int np2 = next_pow2(ncand);
    for (int i = ncand + tid; i < np2; i += kConsumers) sm.cand[i] = ~0ull;
    named_bar_sync(kBarSelect, kConsumers);
    bitonic_sort_u64(sm.cand, np2, tid);
    for (int j = tid; j < K - above; j += kConsumers)
      keep[above + j] = (int)(uint32_t)(sm.cand[j] & 0xffffffffu);
    named_bar_sync(kBarSelect, kConsumers);
  } else {
    select_fallback(sc, n, K, sm, tid);
  }
  // kept indices ascending
  const int kp2 = next_pow2(K);
  for (int i = K + tid; i < kp2; i += kConsumers) keep[i] = 0x7fffffff;
  named_bar_sync(kBarSelect, kConsumers);
  bitonic_sort_i32(keep, kp2, tid);
  for (int i = tid; i < K; i += kConsumers) out[i] = keep[i];
}

// ------------------------------------------------------------- the scan --

// Butterfly reduce-scatter of 16 per-lane partial sums over groups of LPR
// lanes (LPR = lanes that share one compressed-key row).
template <int LPR>
__device__ __forceinline__ void reduce_scatter16(int (&v)[16], int lane) {
  int n = 16;
#pragma unroll
  for (int o = LPR / 2; o >= 1; o >>= 1) {
    if (n > 1) {
      const bool upper = (lane & o) != 0;
      const int h = n / 2;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (i < h) {
          const int send = upper ? v[i] : v[i + h];
          const int keepv = upper ? v[i + h] : v[i];
          v[i] = keepv + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      n = h;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    }
  }
}

template <int DI>
__global__ void __launch_bounds__(kThreads, 2) index_topk_kernel(Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  constexpr int kRowBytes = DI * 2;
  constexpr int kStageRows = kStageBytes / kRowBytes;  // 16 / 32 / 64
  constexpr int kLPR = DI / 4;                         // lanes per row (8 B each)
  constexpr int kRPI = 32 / kLPR;                      // rows per warp load
  static_assert(kStageRows / kRPI == 16, "16 loads per lane per stage");
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int bpp = p.c.page_size / 4;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    sm.sel_req = -1;
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  const long long total_stride = gridDim.x;

  if (warp == kConsumerWarps) {
    // ------------------------------------------------ producer warp --
    if (lane != 0) return;
    const uint64_t pol = l2_policy_evict_first();
    UnitWalker wk;
    wk.start(p, blockIdx.x == 0);
    long long g = 0;  // stage sequence number of this CTA
    bool alive = true;
    for (long long u = blockIdx.x; alive && wk.seek(p, u); u += total_stride) {
      const int r = wk.r;
      const long long row_begin = (u - wk.cum) * (long long)p.unit_rows;
      const int rows = (int)max(0LL, min((long long)p.unit_rows, (long long)wk.n - row_begin));
      const int nst = ceil_div(rows, kStageRows);
      for (int st = 0; st < nst; ++st, ++g) {
        const int slot = (int)(g % kStages);
        const uint32_t par = (uint32_t)((g / kStages) & 1) ^ 1u;
        if (!mbar_wait_abortable(&sm.empty[slot], par, &sm.abort_flag)) {
          alive = false;
          break;
        }
        const long long b0 = row_begin + (long long)st * kStageRows;
        const int nrows = min(kStageRows, rows - st * kStageRows);
        // bytes of the valid page segments of this stage
        uint32_t bytes = 0;
        for (int k = 0; k < nrows;) {
          const long long b = b0 + k;
          const int seg = min(nrows - k, bpp - (int)(b % bpp));
          const long long lp = b / bpp;
          if (lp < p.c.max_pages_per_req) {
            const int pg = p.c.block_table[(long long)r * p.c.max_pages_per_req + lp];
            if (pg >= 0 && pg < p.c.num_pages) bytes += seg * kRowBytes;
          }
          k += seg;
        }
        mbar_arrive_expect_tx(&sm.full[slot], bytes);
        for (int k = 0; k < nrows;) {
          const long long b = b0 + k;
          const int seg = min(nrows - k, bpp - (int)(b % bpp));
          const int pg = physical_page(p.c, r, b / bpp);
          if (pg >= 0) {
            const int16_t *src = p.c.kc + ((long long)pg * bpp + (b % bpp)) * DI;
            bulk_g2s(&sm.stage[slot][k * kRowBytes], src, seg * kRowBytes, &sm.full[slot], pol);
          }
          k += seg;
        }
      }
    }
    // Drain: every copy issued must land before the CTA may exit.
    for (long long k = max(0LL, g - kStages); k < g; ++k)
      if (!mbar_wait(&sm.full[k % kStages], (uint32_t)((k / kStages) & 1))) break;
    return;
  }

  // ---------------------------------------------------- consumer warps --
  UnitWalker wk;
  wk.start(p, false);
  long long g = 0;
  int cur_r = -1;
  uint32_t qword = 0;
  for (long long u = blockIdx.x; wk.seek(p, u); u += total_stride) {
    const int r = wk.r;
    const long long row_begin = (u - wk.cum) * (long long)p.unit_rows;
    const int rows = (int)max(0LL, min((long long)p.unit_rows, (long long)wk.n - row_begin));
    const int nst = ceil_div(rows, kStageRows);
    if (r != cur_r) {
      cur_r = r;
      qword = *reinterpret_cast<const uint32_t *>(p.q_idx + (long long)r * DI + (lane % kLPR) * 4);
    }
    int32_t *sc = p.scores + (long long)r * p.max_blocks;
    for (int st = 0; st < nst; ++st, ++g) {
      if ((int)(g % kConsumerWarps) != warp) continue;
      const int slot = (int)(g % kStages);
      const uint32_t par = (uint32_t)((g / kStages) & 1);
      mbar_wait_abortable(&sm.full[slot], par, &sm.abort_flag);
      const uint8_t *base = sm.stage[slot];
      int acc[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int row = i * kRPI + lane / kLPR;
        const uint2 w = *reinterpret_cast<const uint2 *>(base + row * kRowBytes + (lane % kLPR) * 8);
        int a = __dp2a_lo((int)w.x, (int)qword, 0);
        acc[i] = __dp2a_hi((int)w.y, (int)qword, a);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[slot]);
      reduce_scatter16<kLPR>(acc, lane);
      const long long b0 = row_begin + (long long)st * kStageRows;
      const int nrows = min(kStageRows, rows - st * kStageRows);
      if constexpr (kLPR == 32) {
        // lane pairs hold row (lane >> 1)
        const int row = lane >> 1;
        if ((lane & 1) == 0 && row < nrows) sc[b0 + row] = acc[0];
      } else if constexpr (kLPR == 16) {
        // lane holds i = lane & 15 of row group lane >> 4: row = i * 2 + (lane >> 4)
        const int row = (lane & 15) * kRPI + (lane >> 4);
        if (row < nrows) sc[b0 + row] = acc[0];
      } else {
        // kLPR == 8: lane holds i = ((lane & 7) << 1) | k, k = 0, 1
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int i = ((lane & 7) << 1) | k;
          const int row = i * kRPI + (lane >> 3);
          if (row < nrows) sc[b0 + row] = acc[k];
        }
      }
    }
    // unit done: publish the scores, take a ticket
    __threadfence();
    named_bar_sync(kBarSelect, kConsumers);
    if (tid == 0) {
      const int t = atomicAdd(&p.tickets[r], 1);
      sm.sel_req = (t == wk.units - 1) ? r : -1;
      if (sm.sel_req >= 0) {
        p.tickets[r] = 0;  // every unit of r has reported; reset for the next call
        __threadfence();
      }
    }
    named_bar_sync(kBarSelect, kConsumers);
    const int sr = sm.sel_req;
    if (sr >= 0) {
      __threadfence();  // see every other CTA's published scores
      select_request(p, sr, sm, tid);
      named_bar_sync(kBarSelect, kConsumers);
    }
  }
}

}  // namespace topk
}  // namespace qsa
