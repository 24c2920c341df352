// qsa_sparse_prefill: QSA over many query tokens per request (a prefill
// chunk), each token with its own selection.
//
// Method: a prefill token p is a causal query over its prefix [0, p] and is
// computed like a decode query at that position: the compressed keys of the
// blocks 0 .. floor(p/4) as p sees them (the block holding p sums only its
// tokens <= p), scored against p's indexer query, top-k kept, exact softmax
// attention over the kept tokens up to p.  The blog page ("Qwen 4 QSA 迎来解码
// 上下文并行…", section 为什么一篇关于未发布架构的 serving PR 仍然值得你花时间)
// names a native sparse-prefill kernel for the QSA path and nothing more;
// this reading follows the decode path of the same pages.
//
// Scoring many tokens against the same prefix keys is a dense contraction,
// S[token][block] = q_idx[token] . kc[block], so it runs on the tensor cores:
// tcgen05.mma kind::i8 with int32 accumulators in tensor memory.  The packed
// key value v = 256 (f - 2) + lo (low byte lo, 2-bit field f) splits the
// contraction in two exact integer MMAs,
//     S = Q . LO  (s8 x u8)  +  256 * Q . (F - 2)  (s8 x s8),
// whose two accumulators the epilogue combines (|S| < 2^23).  The block
// holding p enters the MMA with all its cached tokens; a per-token fix-up
// subtracts the dot products of the tokens after p (all in the chunk).  The
// per-token selection and attention then reuse select_kernel and the decode
// kernels, each token being a request of length p + 1 whose block-table row
// is its request's.
#pragma once
#include "index_topk.cuh"

namespace qsa {
namespace pre {

constexpr int kTokTile = 128;     // query tokens per tile (MMA M)
constexpr int kBlkTile = 128;     // micro-blocks per MMA (N)
constexpr int kBlkPerCta = 1024;  // blocks one CTA walks, in sub-tiles of kBlkTile
constexpr int kThreads = 128;     // 4 warps: each owns 32 TMEM lanes (tokens) in the epilogue
constexpr int kTmemCols = 256;    // two int32 accumulators of kBlkTile columns
constexpr unsigned long long kWaitNs = 2000000000ull;  // bound of an MMA-completion wait

struct ScanParams {
  CacheDev c;
  const int32_t *cu_q;      // [B+1] query tokens of request r: rows cu_q[r] .. cu_q[r+1]-1
  const int32_t *ctx_lens;  // [B] cached tokens of request r (its query tokens are the last ones)
  const int8_t *q_idx;      // [Nq, d] indexer queries
  int max_blocks;           // row stride of scores
  int n_tok;                // Nq = cu_q[B]
  int32_t *scores;          // [Nq, max_blocks]
};

template <int DI>
struct Smem {
  uint8_t qa[kTokTile * DI];        // A: query tile, K-major, swizzled
  uint8_t lo[2][kBlkTile * DI];     // B of the first MMA: low key bytes (u8)
  uint8_t f2[2][kBlkTile * DI];     // B of the second MMA: high fields minus 2 (s8)
  alignas(8) uint64_t mbar;
  uint32_t tmem_base;
  int timed_out;
};
template <int DI>
constexpr size_t smem_bytes() { return sizeof(Smem<DI>) + 1024; }

// Byte offset of 16-byte chunk `ch` of row `row` in a K-major tile of
// RB-byte rows with the matching RB-byte swizzle (the layout the tensor
// core reads through a descriptor of that swizzle mode; tiles are
// 1024-byte aligned): the chunk index is XORed with the row bits above it.
template <int RB>
__device__ __forceinline__ int swz_off(int row, int ch) {
  constexpr int kB = RB == 128 ? 3 : RB == 64 ? 2 : 1;
  const int lin = row * RB + ch * 16;
  return lin ^ (((lin >> 7) & ((1 << kB) - 1)) << 4);
}

// Shared-memory matrix descriptor of a K-major swizzled tile of RB-byte
// rows: start address, leading offset 1 (unused by swizzled K-major
// layouts), stride of 8 rows between core-matrix groups, version 1,
// swizzle mode (128 B: 2, 64 B: 4, 32 B: 6).
template <int RB>
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr) {
  constexpr uint64_t kLayout = RB == 128 ? 2 : RB == 64 ? 4 : 6;
  uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)((8 * RB) >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= kLayout << 61;
  return d;
}

// Instruction descriptor of kind::i8: int32 accumulator, A signed, B
// signed or unsigned, both K-major, N = kBlkTile, M = kTokTile.
__host__ __device__ constexpr uint32_t idesc_i8(bool b_signed) {
  return (2u << 4) | (1u << 7) | ((b_signed ? 1u : 0u) << 10) |
         ((uint32_t)(kBlkTile >> 3) << 17) | ((uint32_t)(kTokTile >> 4) << 24);
}

__device__ __forceinline__ void mma_i8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n"
      :
      : "r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u),
        "r"(0u), "r"(0u));
}

__device__ __forceinline__ void umma_commit(uint64_t *mbar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(mbar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Waits for phase `parity` of the mbarrier to complete, for at most
// kWaitNs; false when the wait ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t *mbar, uint32_t parity) {
  const uint32_t a = smem_u32(mbar);
  const unsigned long long t0 = globaltimer();
  while (true) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred P;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, P;\n\t}\n"
        : "=r"(ok)
        : "r"(a), "r"(parity)
        : "memory");
    if (ok) return true;
    if (globaltimer() - t0 > kWaitNs) return false;
  }
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, "
      "[%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Grid (ceil(max_blocks / kBlkPerCta), ceil(max_q / kTokTile), B).  A CTA
// scores the query tokens of one tile of one request against blocks
// [x * kBlkPerCta, ...) up to the last block its last token competes over.
template <int DI>
__global__ void __launch_bounds__(kThreads) prefill_scan_kernel(ScanParams sp) {
  pdl_open();
  static_assert(DI == 32 || DI == 64 || DI == 128, "indexer dim");
  constexpr int RB = DI;  // bytes per int8 row
  constexpr int kChunks = RB / 16;
  constexpr int kKSteps = DI / 32;  // kind::i8 consumes 32 bytes of K per MMA
  extern __shared__ uint8_t smem_raw[];
  Smem<DI> &sm =
      *reinterpret_cast<Smem<DI> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = blockIdx.z;
  const int q0 = sp.cu_q[r];
  const int nq = sp.cu_q[r + 1] - q0;
  const int L = sp.ctx_lens[r];
  const int t0 = blockIdx.y * kTokTile;
  if (nq < 0 || L < nq || q0 < 0 || q0 + nq > sp.n_tok) {
    if (tid == 0 && blockIdx.x == 0 && blockIdx.y == 0) record_error(kErrBadInput);
    return;
  }
  if (t0 >= nq) return;
  const int ntok = min(kTokTile, nq - t0);
  const int p_hi = L - nq + t0 + ntok - 1;  // position of the tile's last token
  const int nb_need = min(p_hi / 4 + 1, sp.max_blocks);
  const int b_begin = blockIdx.x * kBlkPerCta;
  if (b_begin >= nb_need) return;
  const int b_end = min(b_begin + kBlkPerCta, nb_need);
  const int nsub = (b_end - b_begin + kBlkTile - 1) / kBlkTile;
  const int bpp = sp.c.page_size / 4;
  const long long page_bytes = kc_page_bytes(sp.c.page_size, DI);
  const long long lo_bytes = kc_lo_bytes(sp.c.page_size, DI);

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&sm.tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&sm.mbar)) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    sm.timed_out = 0;
  }
  // query tile: thread i writes token row t0 + i (zero rows past the tile)
  {
    uint4 v[kChunks];
#pragma unroll
    for (int c = 0; c < kChunks; ++c) v[c] = make_uint4(0, 0, 0, 0);
    if (tid < ntok) {
      const uint4 *src = reinterpret_cast<const uint4 *>(sp.q_idx + (long long)(q0 + t0 + tid) * DI);
#pragma unroll
      for (int c = 0; c < kChunks; ++c) v[c] = src[c];
    }
#pragma unroll
    for (int c = 0; c < kChunks; ++c) *reinterpret_cast<uint4 *>(sm.qa + swz_off<RB>(tid, c)) = v[c];
  }
  // key sub-tile j into buffer s: thread i owns block row b_begin + j*kBlkTile + i
  auto load_keys = [&](int j, int s) {
    const int b = b_begin + j * kBlkTile + tid;
    uint4 lo[kChunks];
    uint32_t hw[kChunks];
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
      lo[c] = make_uint4(0, 0, 0, 0);
      hw[c] = 0xAAAAAAAAu;  // every field 2: f - 2 = 0
    }
    if (b < b_end) {
      const int lp = b / bpp, rin = b - lp * bpp;
      const int pg = physical_page(sp.c, r, lp);
      if (pg >= 0) {
        const uint8_t *pb = sp.c.kc + (long long)pg * page_bytes;
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
          lo[c] = *reinterpret_cast<const uint4 *>(pb + (long long)rin * DI + 16 * c);
          hw[c] = *reinterpret_cast<const uint32_t *>(pb + lo_bytes + 4LL * ((long long)c * bpp + rin));
        }
      }
    }
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
      *reinterpret_cast<uint4 *>(sm.lo[s] + swz_off<RB>(tid, c)) = lo[c];
      // dim 16c + 4u + k sits at bits 8k + 2u of the field word: byte 4u + k
      // of chunk c gets its field minus 2
      uint4 f;
      f.x = __vsub4((hw[c] >> 0) & 0x03030303u, 0x02020202u);
      f.y = __vsub4((hw[c] >> 2) & 0x03030303u, 0x02020202u);
      f.z = __vsub4((hw[c] >> 4) & 0x03030303u, 0x02020202u);
      f.w = __vsub4((hw[c] >> 6) & 0x03030303u, 0x02020202u);
      *reinterpret_cast<uint4 *>(sm.f2[s] + swz_off<RB>(tid, c)) = f;
    }
  };
  load_keys(0, 0);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t a_addr = smem_u32(sm.qa);
  int32_t *const out_rows = sp.scores + (long long)(q0 + t0) * sp.max_blocks;
  const int row = warp * 32 + lane;  // this thread's token in the tile (TMEM lane)

  for (int j = 0; j < nsub; ++j) {
    const int s = j & 1;
    if (tid == 0) {
      tc_fence_after();
      const uint64_t ad = smem_desc<RB>(a_addr);
      const uint64_t bl = smem_desc<RB>(smem_u32(sm.lo[s]));
      const uint64_t bf = smem_desc<RB>(smem_u32(sm.f2[s]));
#pragma unroll
      for (int kk = 0; kk < kKSteps; ++kk) {
        // K advances 32 bytes along the swizzled rows: +2 in 16-byte units
        mma_i8(tmem, ad + 2 * kk, bl + 2 * kk, idesc_i8(false), kk > 0);
        mma_i8(tmem + kBlkTile, ad + 2 * kk, bf + 2 * kk, idesc_i8(true), kk > 0);
      }
      umma_commit(&sm.mbar);
    }
    __syncwarp();
    if (j + 1 < nsub) {
      load_keys(j + 1, s ^ 1);  // buffer s^1 was read by MMA j-1, which completed
      fence_async_smem();
    }
    const bool ok = mbar_wait(&sm.mbar, (uint32_t)(j & 1));
    tc_fence_after();
    if (!ok) sm.timed_out = 1;
    if (__syncthreads_or(!ok)) break;
    // epilogue: this thread's token row, 16 columns at a time
    const int bcol0 = b_begin + j * kBlkTile;
    const int ncol = min(kBlkTile, b_end - bcol0);
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll 1
    for (int c0 = 0; c0 < kBlkTile; c0 += 16) {
      uint32_t a1[16], a2[16];
      tmem_ld16(lane_addr + c0, a1);
      tmem_ld16(lane_addr + kBlkTile + c0, a2);
      tmem_ld_wait();
      if (row < ntok) {
        int32_t *dst = out_rows + (long long)row * sp.max_blocks + bcol0 + c0;
        int32_t v[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = (int32_t)a1[e] + 256 * (int32_t)a2[e];
        if (c0 + 16 <= ncol && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
#pragma unroll
          for (int e = 0; e < 16; e += 4)
            *reinterpret_cast<int4 *>(dst + e) = make_int4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e)
            if (c0 + e < ncol) dst[e] = v[e];
        }
      }
    }
    tc_fence_before();
    __syncthreads();  // TMEM read before the next MMA; next keys written
  }
  if (sm.timed_out && tid == 0) record_error(kErrTimeout);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

// Per query token (one warp each): its length p + 1 and block-table row for
// the selection and the decode, and the fix-up of its own block's score:
// the MMA scored the block holding p with every cached token of it, so the
// dot products of the tokens after p (at most 3, all in the chunk) are
// subtracted.
struct PrepParams {
  int B, n_tok;
  const int32_t *cu_q, *ctx_lens;
  const int8_t *q_idx, *k_chunk;  // [Nq, d]: indexer queries and raw keys of the chunk
  int d, max_blocks;
  int32_t *scores;                // [Nq, max_blocks]
  int32_t *tok_len, *tok_row;     // [Nq] outputs
};

__global__ void __launch_bounds__(256) prefill_prep_kernel(PrepParams pp) {
  pdl_open();
  const int tok = (int)((blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (tok >= pp.n_tok) return;
  int lo = 0, hi = pp.B;  // request r with cu_q[r] <= tok < cu_q[r+1]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (pp.cu_q[mid] <= tok) lo = mid;
    else hi = mid;
  }
  const int r = lo;
  const int q0 = pp.cu_q[r], nq = pp.cu_q[r + 1] - q0;
  const int L = pp.ctx_lens[r];
  if (nq < 0 || L < nq || tok < q0 || tok - q0 >= nq) {
    if (lane == 0) {
      record_error(kErrBadInput);
      pp.tok_len[tok] = 0;
      pp.tok_row[tok] = r;
    }
    return;
  }
  const int p = L - nq + (tok - q0);
  const int b = p >> 2;
  const int e = min(4 * b + 3, L - 1);
  int corr = 0;
  for (int t = p + 1; t <= e; ++t) {
    const int8_t *k = pp.k_chunk + (long long)(q0 + (t - (L - nq))) * pp.d;
    const int8_t *q = pp.q_idx + (long long)tok * pp.d;
    for (int j = lane; j < pp.d; j += 32) corr += (int)q[j] * (int)k[j];
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) corr += __shfl_xor_sync(0xffffffffu, corr, o);
  if (lane == 0) {
    pp.tok_len[tok] = p + 1;
    pp.tok_row[tok] = r;
    if (corr != 0 && b < pp.max_blocks) pp.scores[(long long)tok * pp.max_blocks + b] -= corr;
  }
}

}  // namespace pre
}  // namespace qsa
