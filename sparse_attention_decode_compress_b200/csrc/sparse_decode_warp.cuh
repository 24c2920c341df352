// qsa_sparse_decode, BF16 / FP8 caches: persistent warp-level split-KV
// flash-decoding on mma.sync bf16 tiles.
//
// Chunks of the extended selection inside each split (sparse_decode.cuh),
// online softmax in fp32, P fed to the PV product as a bf16 hi + lo pair
// (two MMAs, ~16 significant bits), LSE merge of a split's chunks by the
// last chunk to finish.  FP8 E4M3 tiles go from shared memory straight into
// f16 fragments and both products run in f16 (fp8_frag.cuh); the
// per-(page, head) K scale multiplies the logits and the V scale multiplies
// P.  Organised for memory-level parallelism on
// B200: one CTA of NW warps per SM, each warp an independent worker that
// takes (request, kv head, chunk) items from an atomic counter and streams
// its chunk through its own ring of NS 16-token K/V stages with cp.async
// (NS - 1 stages in flight while one is computed).  No CTA
// barriers: warps never wait for each other, results go straight from the
// MMA accumulators to global memory.
#pragma once
#include "fp8_frag.cuh"

namespace qsa {
namespace dec {

constexpr int kTokW = 16;         // tokens per stage
constexpr int kCounterInts = 64;  // workspace header: [0] next item (then the split tickets)

// Shared-memory layout of one worker warp: a ring of NS 16-token K/V stages
// and the chunk's token metadata.
template <int D, bool FP8, int NS, int CAP = kChunkBlocks>
struct WarpState {
  static constexpr int kRowBytes = D * (FP8 ? 1 : 2);
  static constexpr int kCap = CAP;  // micro-blocks a chunk may hold
  alignas(128) uint8_t ring[NS][2][kTokW * kRowBytes];
  int boff[CAP];  // cache row (token, head g) of each micro-block's first token
  // byte j of word b: visibility bits of token j of micro-block b (bit t:
  // visible to query token t); a token visible to none is not loaded
  uint32_t vmask4[CAP];
  float ks[FP8 ? CAP : 1];  // fp8 scales of each micro-block's page
  float vs[FP8 ? CAP : 1];
  Plan pl;
  __device__ __forceinline__ unsigned vmask(int tok) const {
    return reinterpret_cast<const unsigned char *>(vmask4)[tok];
  }
};

// Micro-blocks of token metadata a worker warp holds at a time: a work item
// longer than that streams in pieces of this many.
template <bool FP8>
__host__ __device__ constexpr int warp_piece_blocks() { return FP8 ? 2 * kChunkBlocks : kChunkBlocks; }

template <int D, bool FP8, int NW, int NS>
struct WarpSmem {
  WarpState<D, FP8, NS, warp_piece_blocks<FP8>()> w[NW];
};

__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// P^T B fragments of one 8-column tile from this lane's values (token gq:
// v0, v1; token gq + 8: v2, v3) as a hi + lo pair, bf16 or (F16) f16: the
// accumulator layout transposed to the B layout with movmatrix.
template <bool F16>
__device__ __forceinline__ void p_frags(float v0, float v1, float v2, float v3, uint32_t (&hi)[2],
                                        uint32_t (&lo)[2]) {
  if constexpr (F16) {
    const __half2 h01 = __floats2half2_rn(v0, v1), h23 = __floats2half2_rn(v2, v3);
    const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
    hi[0] = movmatrix_t(*reinterpret_cast<const uint32_t *>(&h01));
    hi[1] = movmatrix_t(*reinterpret_cast<const uint32_t *>(&h23));
    lo[0] = movmatrix_t(pack_f16(v0 - f01.x, v1 - f01.y));
    lo[1] = movmatrix_t(pack_f16(v2 - f23.x, v3 - f23.y));
  } else {
    const __nv_bfloat162 h01 = __floats2bfloat162_rn(v0, v1), h23 = __floats2bfloat162_rn(v2, v3);
    const float2 f01 = __bfloat1622float2(h01), f23 = __bfloat1622float2(h23);
    hi[0] = movmatrix_t(*reinterpret_cast<const uint32_t *>(&h01));
    hi[1] = movmatrix_t(*reinterpret_cast<const uint32_t *>(&h23));
    lo[0] = movmatrix_t(pack_bf16(v0 - f01.x, v1 - f01.y));
    lo[1] = movmatrix_t(pack_bf16(v2 - f23.x, v3 - f23.y));
  }
}

// Warp-level: empty splits of (r, g) get o = 0, lse = -inf.
template <int D>
__device__ void write_empty_splits_warp(const Params &p, const Plan &pl, int r, int g, int lane) {
  for (int s = 0; s < p.S; ++s) {
    if (pl.ch_count[s] != 0) continue;
    for (int i = lane; i < p.M * D; i += 32) {
      const int m = i / D, d = i % D;
      p.o_part[out_row(p, s, r, g, m) * D + d] = 0.f;
      if (d == 0) p.lse_part[out_row(p, s, r, g, m)] = -INFINITY;
    }
  }
}

// Micro-block metadata of entries [eb, ee) of the extended selection (at
// most WS::kCap): cache row of the first token, the tokens' visibility bits
// and fp8 scales.  Token i is visible to query token
// t (position p_t = p0 + t) when i <= p_t and (its block is selected or
// i > p0).  A micro-block never straddles a page (P % 4 == 0), so token j of
// block b sits j * Hkv rows after its first token.
template <typename WS, bool FP8>
__device__ void fill_meta_warp(const Params &p, const Plan &pl, int r, int g, WS &W, int lane,
                               const int *stash, int eb, int ee) {
  const int32_t *sel_r = stash ? stash : p.sel + (long long)r * p.topk;
  const int P = p.c.page_size, Hkv = p.c.num_kv_heads;
  const bool pow2 = (P & (P - 1)) == 0;
  const int lgP = 31 - __clz(P);
  // one lane per micro-block (kCap / 32 each), one page lookup per block;
  // every block slot is written (slots past the piece: nothing visible)
  constexpr int kPer = WS::kCap / 32;
  int bl[kPer], pg[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = eb + lane + 32 * i;
    bl[i] = (e < ee) ? ext_block(sel_r, pl, e) : -1;
  }
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    pg[i] = -1;
    if (bl[i] >= 0) {
      const long long t0 = 4LL * bl[i];
      if (t0 < pl.L) {
        pg[i] = physical_page(p.c, r, pow2 ? (t0 >> lgP) : t0 / P);
      } else {
        record_error(kErrBadInput);  // selected block beyond the context
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int kb = lane + 32 * i;  // block index in the piece
    const int e = eb + kb;
    const long long t0 = 4LL * bl[i];
    const bool ins = e < pl.nvalid;
    int boff = -1;
    uint32_t vm4 = 0;
    float ks = 1.f, vs = 1.f;
    if (pg[i] >= 0) {
      const long long tin = pow2 ? (t0 & (P - 1)) : t0 % P;
      boff = (int)(((long long)pg[i] * P + tin) * Hkv + g);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const long long t = t0 + j;
        unsigned vm = 0;
        if (t < pl.L)
          for (int q = 0; q < p.T; ++q)
            if (t <= (long long)pl.p0 + q && (ins || t > pl.p0)) vm |= 1u << q;
        vm4 |= vm << (8 * j);
      }
      if (FP8) {
        ks = p.c.k_scale[(long long)pg[i] * Hkv + g];
        vs = p.c.v_scale[(long long)pg[i] * Hkv + g];
      }
    }
    W.boff[kb] = boff;
    W.vmask4[kb] = vm4;
    if (FP8) {
      W.ks[kb] = ks;
      W.vs[kb] = vs;
    }
  }
}

// cp.async of stage st of the chunk into ring slot `slot` (rows swizzled for
// bf16; fp8 rows land raw and are converted before use).  A lane copies the
// same 16-byte column of kTokW / kRowsPerPass rows of K and of V; their
// metadata is read into registers before the first copy is issued.
template <int D, bool FP8, typename WS>
__device__ __forceinline__ void issue_stage_warp(const Params &p, WS &W, int slot, int st,
                                                 int lane) {
  constexpr int kRowBytes = WS::kRowBytes;
  constexpr int kCh = kRowBytes / 16;           // 16-byte chunks per row
  constexpr int kRowsPerPass = 32 / kCh;        // rows one warp-wide pass covers
  constexpr int kPasses = kTokW / kRowsPerPass;
  const uint8_t *kbase = static_cast<const uint8_t *>(p.c.k_cache);
  const uint8_t *vbase = static_cast<const uint8_t *>(p.c.v_cache);
  const int Hkv = p.c.num_kv_heads;
  const int ch = lane % kCh, r0 = lane / kCh;
  int off[kPasses];
  bool load[kPasses];
#pragma unroll
  for (int j = 0; j < kPasses; ++j) {
    const int tok = st * kTokW + r0 + j * kRowsPerPass;
    load[j] = W.vmask(tok) != 0u;
    off[j] = load[j] ? W.boff[tok >> 2] + (tok & 3) * Hkv : 0;
  }
#pragma unroll
  for (int kv = 0; kv < 2; ++kv) {
#pragma unroll
    for (int j = 0; j < kPasses; ++j) {
      const int row = r0 + j * kRowsPerPass;
      uint8_t *dst = W.ring[slot][kv] + (FP8 ? fp8_swz<D>(row, ch) : swz<D>(row, ch));
      const uint8_t *src = (kv ? vbase : kbase) + (long long)off[j] * kRowBytes + ch * 16;
      cp_async16_zfill(dst, src, load[j]);
    }
  }
}

// Power-of-two reference of the chunk's V scales (fp8): the binade of the
// largest |vs| over its nblk micro-blocks; all lanes of the warp get it.
template <typename WS>
__device__ __forceinline__ float chunk_vsref(const WS &W, int nblk, int lane) {
  float mx = 0.f;
  for (int kb = lane; kb < nblk; kb += 32) mx = fmaxf(mx, fabsf(W.vs[kb]));
#pragma unroll
  for (int o2 = 16; o2 >= 1; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
  return vs_binade(mx);
}

// Tensor-core decode, tokens on M: per 16-token stage
//   S^T[16 tokens x 8*NT rows] = K[16 x D] . Q^T          (mma m16n8k16, A = K
//                                                          from smem, B = Q in
//                                                          registers)
//   P^T = exp2(S^T * scale - m) per query row (a column here); transposed to
//         the B layout of the next product with movmatrix, as bf16 hi + lo
//   O^T[D x 8*NT] += V^T[D x 16 tokens] . P^T              (A = V rows loaded
//                                                          with ldmatrix.trans)
// Query rows m = t*G + j (head g*G + j of query token t) sit on the N side in
// tiles of 8, so G*T = 8 uses every MMA lane.
template <int D, int NT, bool FP8, int NW, int NS>
__global__ void __launch_bounds__(NW * 32, 1) sparse_decode_warp_kernel(Params p) {
  pdl_open();
  extern __shared__ uint8_t smem_raw[];
  using SM = WarpSmem<D, FP8, NW, NS>;
  using WS = WarpState<D, FP8, NS, warp_piece_blocks<FP8>()>;
  SM &sm = *reinterpret_cast<SM *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  WS &W = sm.w[warp];
  Plan &pl = W.pl;
  const int Hkv = p.c.num_kv_heads;
  const int total_items = p.B * Hkv * p.nch;
  const int gq = lane >> 2, cq = lane & 3;
  constexpr int MD = D / 16;  // m-tiles of O^T (16 dims each)

  // first item: the warp's own index, numbered across CTAs first so that a
  // batch with fewer items than warps still loads every SM evenly; later
  // items: from the work counter, which hands out indices from the number
  // of warps on
  const int nwarps = gridDim.x * NW;
  bool first = true;
  while (true) {
    int it = warp * gridDim.x + blockIdx.x;
    if (!first) {
      if (lane == 0) it = nwarps + atomicAdd(&p.counters[0], 1);
      it = __shfl_sync(0xffffffffu, it, 0);
    }
    first = false;
    if (it >= total_items) break;
    const int c = it % p.nch;
    const int g = (it / p.nch) % Hkv;
    const int r = it / (p.nch * Hkv);

    // Q as B fragments: n-tile j, k-step kk: b0 = Q[row 8j+gq][16kk+2cq, +1],
    // b1 = Q[row 8j+gq][16kk+2cq+8, +9]; rows >= M are zero.  Issued first so
    // the loads overlap the plan.  fp8: f16 fragments in the permuted k order
    // of fp8_frag.cuh, and csc = the logit factor of each of this lane's
    // columns (scale_log2 times the inverse Q scale of its row).
    uint32_t qb[NT][MD][2];
    float csc[NT][2];
    {
      const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(p.q);
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        const int m = 8 * j + gq;
        const bool ok = m < p.M;
        const __nv_bfloat16 *qrow =
            qg + (((long long)r * p.T + (ok ? m / p.G : 0)) * p.Hq + g * p.G + (ok ? m % p.G : 0)) * D;
        if constexpr (FP8) {
          const float qinv = q_frags_f16<D>(ok ? qrow : nullptr, cq, qb[j]);
#pragma unroll
          for (int e = 0; e < 2; ++e)
            csc[j][e] = p.scale_log2 * __shfl_sync(0xffffffffu, qinv, (2 * cq + e) * 4);
        } else {
#pragma unroll
          for (int kk = 0; kk < MD; ++kk) {
            qb[j][kk][0] = ok ? *reinterpret_cast<const uint32_t *>(qrow + 16 * kk + 2 * cq) : 0u;
            qb[j][kk][1] = ok ? *reinterpret_cast<const uint32_t *>(qrow + 16 * kk + 2 * cq + 8) : 0u;
          }
          csc[j][0] = csc[j][1] = p.scale_log2;
        }
      }
    }
    // the selection row goes to the last ring slot (idle until stage NS-1)
    constexpr int kStashInts = (int)(sizeof(W.ring[0]) / sizeof(int));
    int *stash = p.topk <= kStashInts ? reinterpret_cast<int *>(&W.ring[NS - 1][0][0]) : nullptr;
    make_plan(p, r, c, pl, stash);
    __syncwarp();
    if (c == 0) write_empty_splits_warp<D>(p, pl, r, g, lane);
    if (!pl.active) continue;
    const int e_begin = pl.e_begin, e_end = pl.e_end;

    // query token of each of this lane's columns (rows 8j + 2cq + e); -1 = padding
    int tcol[NT][2];
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int m = 8 * j + 2 * cq + e;
        tcol[j][e] = m < p.M ? m / p.G : -1;
      }

    float o[MD][NT][4];
    float mcol[NT][2], lcol[NT][2];
#pragma unroll
    for (int i = 0; i < MD; ++i)
#pragma unroll
      for (int j = 0; j < NT; ++j) o[i][j][0] = o[i][j][1] = o[i][j][2] = o[i][j][3] = 0.f;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      mcol[j][0] = mcol[j][1] = -INFINITY;
      lcol[j][0] = lcol[j][1] = 0.f;
    }
    // fp8: P carries vs / vsref, vsref a power of two that only grows from
    // piece to piece (the partial sums are rescaled when it does); the
    // output is multiplied by it
    float vsref = 1.f, vsinv = 1.f;

    // the item streams in pieces of at most kCap micro-blocks (the ring is
    // drained between pieces); the first piece reads the stashed selection
    for (int pb = e_begin; pb < e_end; pb += WS::kCap) {
      const int pe = min(pb + WS::kCap, e_end);
      fill_meta_warp<WS, FP8>(p, pl, r, g, W, lane, pb == e_begin ? stash : nullptr, pb, pe);
      __syncwarp();
      if constexpr (FP8) {
        const float vr = chunk_vsref(W, pe - pb, lane);
        const float vn = (pb == e_begin) ? vr : fmaxf(vsref, vr);
        if (vn != vsref && pb != e_begin) {
          const float f = vsref / vn;
#pragma unroll
          for (int i = 0; i < MD; ++i)
#pragma unroll
            for (int j = 0; j < NT; ++j)
#pragma unroll
              for (int k = 0; k < 4; ++k) o[i][j][k] *= f;
        }
        vsref = vn;
        vsinv = 1.f / vn;
      }
      const int nst = (pe - pb + 3) / 4;  // 4 micro-blocks per stage
#pragma unroll
      for (int s0 = 0; s0 < NS - 1; ++s0) {
        if (s0 < nst) issue_stage_warp<D, FP8>(p, W, s0, s0, lane);
        cp_async_commit();
      }
      for (int st = 0; st < nst; ++st) {
        {
          const int sn = st + NS - 1;
          if (sn < nst) issue_stage_warp<D, FP8>(p, W, sn % NS, sn, lane);
          cp_async_commit();
        }
        cp_async_wait<NS - 1>();
        __syncwarp();
        const int slot = st % NS;
        const uint8_t *ks_t = W.ring[slot][0];
        const uint8_t *vs_t = W.ring[slot][1];
        const int tb = st * kTokW;  // piece index of the stage's first token

        // ---- S^T = K Q^T (even and odd k-steps in two accumulators: shorter chains)
        float sacc[NT][4], sac2[NT][4];
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) sacc[j][e] = sac2[j][e] = 0.f;
        if constexpr (FP8) {
#pragma unroll
          for (int j = 0; j < NT; ++j) qk_fp8<D>(ks_t, gq, cq, qb[j], sacc[j], sac2[j]);
        } else {
#pragma unroll
          for (int kk = 0; kk < MD; ++kk) {
            uint32_t a0, a1, a2, a3;
            {
              const int row = (lane & 7) + 8 * ((lane >> 3) & 1);
              const int ch = 2 * kk + (lane >> 4);
              ldsm_x4(a0, a1, a2, a3, ks_t + swz<D>(row, ch));
            }
#pragma unroll
            for (int j = 0; j < NT; ++j) {
              if (kk & 1) mma_bf16(sac2[j], a0, a1, a2, a3, qb[j][kk][0], qb[j][kk][1]);
              else mma_bf16(sacc[j], a0, a1, a2, a3, qb[j][kk][0], qb[j][kk][1]);
            }
          }
        }
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) sacc[j][e] += sac2[j][e];

        // ---- mask, online softmax per column, P^T as bf16 hi + lo B fragments
        const unsigned vm0 = W.vmask(tb + gq), vm1 = W.vmask(tb + gq + 8);
        float ksc0 = 1.f, ksc1 = 1.f, vsc0 = 1.f, vsc1 = 1.f;
        if constexpr (FP8) {
          ksc0 = W.ks[(tb + gq) >> 2];
          ksc1 = W.ks[(tb + gq + 8) >> 2];
          vsc0 = W.vs[(tb + gq) >> 2] * vsinv;
          vsc1 = W.vs[(tb + gq + 8) >> 2] * vsinv;
        }
        uint32_t bhi[NT][2], blo[NT][2];
        bool rescale = false;
        float alpha[NT][2];
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          float x[4];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int t = tcol[j][e];
            const bool ok0 = t >= 0 && ((vm0 >> t) & 1u);
            const bool ok1 = t >= 0 && ((vm1 >> t) & 1u);
            x[e] = ok0 ? sacc[j][e] * csc[j][e] * ksc0 : -INFINITY;      // token gq
            x[2 + e] = ok1 ? sacc[j][2 + e] * csc[j][e] * ksc1 : -INFINITY;  // token gq+8
          }
          float pj[4];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            float mx = fmaxf(x[e], x[2 + e]);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float m_old = mcol[j][e];
            const float m_new = fmaxf(m_old, mx);
            const float base = (m_new == -INFINITY) ? 0.f : m_new;
            const float a = (m_new == -INFINITY) ? 1.f : ex2(m_old - base);  // empty column: keep
            alpha[j][e] = a;
            rescale |= (a != 1.f);
            mcol[j][e] = m_new;
            pj[e] = ex2(x[e] - base);
            pj[2 + e] = ex2(x[2 + e] - base);
            lcol[j][e] = lcol[j][e] * a + pj[e] + pj[2 + e];  // this lane's two tokens
          }
          const float v0 = pj[0] * vsc0, v1 = pj[1] * vsc0, v2 = pj[2] * vsc1, v3 = pj[3] * vsc1;
          // tile of tokens 0-7 (lane holds token gq, cols 2cq..) -> b0; tokens 8-15 -> b1
          p_frags<FP8>(v0, v1, v2, v3, bhi[j], blo[j]);
        }
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int i = 0; i < MD; ++i)
#pragma unroll
            for (int j = 0; j < NT; ++j) {
              o[i][j][0] *= alpha[j][0];
              o[i][j][1] *= alpha[j][1];
              o[i][j][2] *= alpha[j][0];
              o[i][j][3] *= alpha[j][1];
            }
        }

        // ---- O^T += V^T P^T
        if constexpr (FP8) {
          VRaw<D> vr;
          v_raw_fp8<D>(vs_t, gq, cq, vr);
#pragma unroll
          for (int i = 0; i < MD; ++i) {
            uint32_t a0, a1, a2, a3;
            v_frag_fp8<D>(vr, i, a0, a1, a2, a3);
#pragma unroll
            for (int j = 0; j < NT; ++j) {
              mma_f16(o[i][j], a0, a1, a2, a3, bhi[j][0], bhi[j][1]);
              mma_f16(o[i][j], a0, a1, a2, a3, blo[j][0], blo[j][1]);
            }
          }
        } else {
#pragma unroll
          for (int i = 0; i < MD; ++i) {
            uint32_t a0, a1, a2, a3;
            {
              const int row = (lane & 7) + 8 * (lane >> 4);
              const int ch = 2 * i + ((lane >> 3) & 1);
              ldsm_x4_t(a0, a1, a2, a3, vs_t + swz<D>(row, ch));
            }
#pragma unroll
            for (int j = 0; j < NT; ++j) {
              mma_bf16(o[i][j], a0, a1, a2, a3, bhi[j][0], bhi[j][1]);
              mma_bf16(o[i][j], a0, a1, a2, a3, blo[j][0], blo[j][1]);
            }
          }
        }
        __syncwarp();  // the slot may be refilled by the next issue
      }
      cp_async_wait<0>();
      __syncwarp();
    }  // pieces

    // ---- chunk result: column sums over the 8 token lanes, then o and lse
    const int s_idx = pl.split;
    const bool direct = pl.nchunks_split == 1;
    const long long wslot = ((long long)r * Hkv + g) * p.nch + c;
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float l = lcol[j][e];
        l += __shfl_xor_sync(0xffffffffu, l, 4);
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        const int m = 8 * j + 2 * cq + e;
        if (m >= p.M) continue;
        const float inv = l > 0.f ? vsref / l : 0.f;
        float *orow = direct ? p.o_part + out_row(p, s_idx, r, g, m) * D : p.ws_o + (wslot * p.M + m) * D;
        if constexpr (FP8) {
          store_col_fp8<D>(orow, [&](int i, int k) { return o[i][j][k]; }, e, gq, inv);
        } else {
#pragma unroll
          for (int i = 0; i < MD; ++i) {
            orow[16 * i + gq] = o[i][j][e] * inv;
            orow[16 * i + gq + 8] = o[i][j][2 + e] * inv;
          }
        }
        if (gq == 0) {
          const float lse = l > 0.f ? (mcol[j][e] + __log2f(l)) * kLn2 : -INFINITY;
          if (direct) p.lse_part[out_row(p, s_idx, r, g, m)] = lse;
          else p.ws_lse[wslot * p.M + m] = lse;
        }
      }
    if (direct) continue;

    // ---- several chunks in this split: the last to finish merges them
    __threadfence();
    __syncwarp();
    int last = 0;
    if (lane == 0) {
      int32_t *ticket = p.tickets + ((long long)r * Hkv + g) * p.S + s_idx;
      const int t = atomicAdd(ticket, 1);
      last = (t == pl.nchunks_split - 1);
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (!last) continue;
    __threadfence();
    const long long slot0 = ((long long)r * Hkv + g) * p.nch + pl.first_chunk_of_split;
    const int nc = pl.nchunks_split;
    float *lse_c = reinterpret_cast<float *>(&W.ring[0][0][0]);  // [nc][M], ring is idle now
    for (int i = lane; i < nc * p.M; i += 32) lse_c[i] = __ldcg(p.ws_lse + slot0 * p.M + i);
    __syncwarp();
    for (int e4 = lane; e4 < p.M * D / 4; e4 += 32) {
      const int m = (e4 * 4) / D, d = (e4 * 4) % D;
      float mx = -INFINITY;
      for (int cc = 0; cc < nc; ++cc) mx = fmaxf(mx, lse_c[cc * p.M + m]);
      float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
      float den = 0.f;
      if (mx != -INFINITY) {
        for (int cc = 0; cc < nc; cc += 4) {
          float4 ov[4];
#pragma unroll
          for (int u = 0; u < 4; ++u)
            ov[u] = (cc + u < nc) ? __ldcg(reinterpret_cast<const float4 *>(
                                        p.ws_o + ((slot0 + cc + u) * p.M + m) * D + d))
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            if (cc + u >= nc) break;
            const float l = lse_c[(cc + u) * p.M + m];
            const float w = (l == -INFINITY) ? 0.f : __expf(l - mx);
            den += w;
            num.x += w * ov[u].x;
            num.y += w * ov[u].y;
            num.z += w * ov[u].z;
            num.w += w * ov[u].w;
          }
        }
      }
      const float inv = den > 0.f ? 1.f / den : 0.f;
      *reinterpret_cast<float4 *>(p.o_part + out_row(p, s_idx, r, g, m) * D + d) =
          make_float4(num.x * inv, num.y * inv, num.z * inv, num.w * inv);
      if (d == 0) p.lse_part[out_row(p, s_idx, r, g, m)] = den > 0.f ? mx + __logf(den) : -INFINITY;
    }
    __syncwarp();
  }
}

}  // namespace dec
}  // namespace qsa
