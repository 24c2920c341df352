// qsa_sparse_decode with bf16 caches and more than 8 query rows per kv head
// (MTP verify, wide GQA groups): the stream-K partition of
// sparse_decode_streamk.cuh run by the warp groups of
// sparse_decode_group.cuh.
//
// Group i of W takes the entries [floor(i X / W), floor((i + 1) X / W)) of
// the batch's padded extended selections laid end to end, cut into segments
// at pair and split boundaries.  A group is GW warps, one per 8-row tile of
// the M = G * T query rows; they share one K/V ring, the plan and the token
// metadata, and meet at a named barrier every stage (the stage arithmetic
// of sparse_decode_group_kernel).  Each segment's normalised partial goes to
// slot k = i - (first group of the segment's (pair, split)), and
// streamk_merge_kernel merges the slots as for the one-warp kernel.
//
// With chunks inside splits (the work-counter kernel), the MTP verify batch
// (128 pairs x 2 splits) made 512 items for 592 groups: 80 groups idle and
// ~64 stages per busy group.  Equal ranges give every group ~28 stages.
#pragma once
#include "sparse_decode_group.cuh"
#include "sparse_decode_streamk.cuh"

namespace qsa {
namespace dec {

template <int D, int NW, int NS, int GW>
struct SKGroupSmem {
  WarpState<D, false, NS, kGroupChunkBlocks> g[NW / GW];
};

// Token metadata of entries [eb, ee) (at most WS::kCap) of pair (r, g)'s
// extended selection, written by the GW * 32 threads of a group (thread tig
// of nthr); the contents of fill_meta_group for bf16 caches.
template <typename WS>
__device__ void fill_meta_group_range(const Params &p, const Plan &pl, int r, int g, WS &W, int tig,
                                      int nthr, const int *stash, int eb, int ee) {
  const int32_t *sel_r = stash ? stash : p.sel + (long long)r * p.topk;
  const int P = p.c.page_size, Hkv = p.c.num_kv_heads;
  const bool pow2 = (P & (P - 1)) == 0;
  const int lgP = 31 - __clz(P);
  for (int kb = tig; kb < WS::kCap; kb += nthr) {
    const int e = eb + kb;
    const int b = (e < ee) ? ext_block(sel_r, pl, e) : -1;
    int pg = -1;
    if (b >= 0) {
      const long long t0 = 4LL * b;
      if (t0 < pl.L) pg = physical_page(p.c, r, pow2 ? (t0 >> lgP) : t0 / P);
      else record_error(kErrBadInput);  // selected block beyond the context
    }
    const long long t0 = 4LL * b;
    const bool ins = e < pl.nvalid;
    int boff = -1;
    uint32_t vm4 = 0;
    if (pg >= 0) {
      const long long tin = pow2 ? (t0 & (P - 1)) : t0 % P;
      boff = (int)(((long long)pg * P + tin) * Hkv + g);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const long long t = t0 + j;
        unsigned vm = 0;
        if (t < pl.L)
          for (int q = 0; q < p.T; ++q)
            if (t <= (long long)pl.p0 + q && (ins || t > pl.p0)) vm |= 1u << q;
        vm4 |= vm << (8 * j);
      }
    }
    W.boff[kb] = boff;
    W.vmask4[kb] = vm4;
  }
}

template <int D, int NW, int NS, int GW>
__global__ void __launch_bounds__(NW * 32, 1) sparse_decode_streamk_group_kernel(SKParams sk) {
  pdl_open();
  static_assert(NW % GW == 0, "warps per CTA must be a multiple of the group size");
  static_assert(NS >= 2, "ring depth");
  constexpr int NG = NW / GW;
  const Params &p = sk.p;
  extern __shared__ uint8_t smem_raw[];
  using SM = SKGroupSmem<D, NW, NS, GW>;
  using WS = WarpState<D, false, NS, kGroupChunkBlocks>;
  SM &sm = *reinterpret_cast<SM *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = warp / GW, wig = warp % GW;  // group, and this warp's 8-row tile
  const int tig = wig * 32 + lane;
  WS &W = sm.g[grp];
  Plan &pl = W.pl;
  const int bar = 1 + grp;
  auto gsync = [&]() { named_bar_sync(bar, GW * 32); };
  const int Hkv = p.c.num_kv_heads;
  const int gq = lane >> 2, cq = lane & 3;
  constexpr int MD = D / 16;
  const int gi = blockIdx.x * NG + grp;  // this group's range of the entries
  if (gi >= sk.W) return;                // the whole group
  const long long x_end = sk_range_begin(gi + 1, sk.X, sk.W);
  long long x = sk_range_begin(gi, sk.X, sk.W);
  constexpr int kStashInts = (int)(sizeof(W.ring[0]) / sizeof(int));
  int *stash = p.topk <= kStashInts ? reinterpret_cast<int *>(&W.ring[NS - 1][0][0]) : nullptr;
  int planned_r = -1;
  long long q_pair = -1;
  bool stash_ok = false;  // the stash holds planned_r's row (until a stage refills its slot)
  uint32_t qb[MD][2];
  int tcol[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int m = 8 * wig + 2 * cq + e;
    tcol[e] = m < p.M ? m / p.G : -1;
  }

  while (x < x_end) {
    const long long P = x / sk.E;
    const int r = (int)(P / Hkv), g = (int)(P % Hkv);
    const int e_lo = (int)(x - P * sk.E);
    const int e_hi = (int)(min(x_end, (P + 1) * sk.E) - P * sk.E);
    x = P * sk.E + e_hi;
    if (r != planned_r) {
      // the ring is idle once every warp has drained it; the selection row
      // goes to its last slot, read only by the metadata fill right after
      cp_async_wait<0>();
      gsync();
      if (wig == 0) {
        make_plan(p, r, -1, pl, stash);
        __syncwarp();
        if (lane <= p.S) sk.sk_ebound[(long long)r * (p.S + 1) + lane] = pl.e_bound[lane];
      }
      gsync();
      stash_ok = stash != nullptr;
      planned_r = r;
    }
    const int nE = pl.nE;
    for (int s = p.s_lo; s < p.s_hi; ++s) {
      const int eb = max(e_lo, pl.e_bound[s]);
      const int ee = min(min(e_hi, nE), pl.e_bound[s + 1]);
      if (eb >= ee) continue;
      float o[MD][4];
      float mcol[2] = {-INFINITY, -INFINITY}, lcol[2] = {0.f, 0.f};
#pragma unroll
      for (int i = 0; i < MD; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
      // the segment streams in metadata pieces of at most kCap entries
      for (int pb = eb; pb < ee; pb += WS::kCap) {
        const int pe = min(pb + WS::kCap, ee);
        cp_async_wait<0>();
        gsync();  // no warp still reads the ring or the metadata
        fill_meta_group_range<WS>(p, pl, r, g, W, tig, GW * 32, stash_ok ? stash : nullptr, pb, pe);
        gsync();
        stash_ok = false;  // the stages below may refill the stash's ring slot
        const int nst = (pe - pb + 3) / 4;
#pragma unroll
        for (int s0 = 0; s0 < NS - 1; ++s0) {
          if (s0 < nst) issue_stage_group<D, false, GW>(p, W, s0, s0, tig);
          cp_async_commit();
        }
        if (P != q_pair) {
          // Q B-fragments of this warp's tile (rows m = 8 * wig + gq),
          // loaded behind the first stages (the barriers of the plan and the
          // metadata fill wait for the loads in flight)
          const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(p.q);
          const int m = 8 * wig + gq;
          const bool ok = m < p.M;
          const __nv_bfloat16 *qrow =
              qg + (((long long)r * p.T + (ok ? m / p.G : 0)) * p.Hq + g * p.G + (ok ? m % p.G : 0)) * D;
#pragma unroll
          for (int kk = 0; kk < MD; ++kk) {
            qb[kk][0] = ok ? *reinterpret_cast<const uint32_t *>(qrow + 16 * kk + 2 * cq) : 0u;
            qb[kk][1] = ok ? *reinterpret_cast<const uint32_t *>(qrow + 16 * kk + 2 * cq + 8) : 0u;
          }
          q_pair = P;
        }
        for (int st = 0; st < nst; ++st) {
          cp_async_wait<NS - 2>();  // this thread's share of stage st has landed
          gsync();                  // ... everyone's; and slot (st - 1) % NS is free
          {
            const int sn = st + NS - 1;
            if (sn < nst) issue_stage_group<D, false, GW>(p, W, sn % NS, sn, tig);
            cp_async_commit();
          }
          const int slot = st % NS;
          const uint8_t *ks_t = W.ring[slot][0];
          const uint8_t *vs_t = W.ring[slot][1];
          const int tb = st * kTokW;
          // ---- S^T = K Q^T for this warp's tile
          float sacc[4] = {0.f, 0.f, 0.f, 0.f}, sac2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int kk = 0; kk < MD; ++kk) {
            uint32_t a0, a1, a2, a3;
            const int row = (lane & 7) + 8 * ((lane >> 3) & 1);
            const int ch = 2 * kk + (lane >> 4);
            ldsm_x4(a0, a1, a2, a3, ks_t + swz<D>(row, ch));
            if (kk & 1) mma_bf16(sac2, a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
            else mma_bf16(sacc, a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) sacc[e] += sac2[e];
          // ---- mask, online softmax per column, P^T as bf16 hi + lo fragments
          const unsigned vm0 = W.vmask(tb + gq), vm1 = W.vmask(tb + gq + 8);
          float xx[4];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int t = tcol[e];
            const bool ok0 = t >= 0 && ((vm0 >> t) & 1u);
            const bool ok1 = t >= 0 && ((vm1 >> t) & 1u);
            xx[e] = ok0 ? sacc[e] * p.scale_log2 : -INFINITY;
            xx[2 + e] = ok1 ? sacc[2 + e] * p.scale_log2 : -INFINITY;
          }
          float pj[4], alpha[2];
          bool rescale = false;
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            float mx = fmaxf(xx[e], xx[2 + e]);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float m_old = mcol[e];
            const float m_new = fmaxf(m_old, mx);
            const float base = (m_new == -INFINITY) ? 0.f : m_new;
            const float a = (m_new == -INFINITY) ? 1.f : ex2(m_old - base);
            alpha[e] = a;
            rescale |= (a != 1.f);
            mcol[e] = m_new;
            pj[e] = ex2(xx[e] - base);
            pj[2 + e] = ex2(xx[2 + e] - base);
            lcol[e] = lcol[e] * a + pj[e] + pj[2 + e];
          }
          uint32_t bhi[2], blo[2];
          p_frags<false>(pj[0], pj[1], pj[2], pj[3], bhi, blo);
          if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
            for (int i = 0; i < MD; ++i) {
              o[i][0] *= alpha[0];
              o[i][1] *= alpha[1];
              o[i][2] *= alpha[0];
              o[i][3] *= alpha[1];
            }
          }
          // ---- O^T += V^T P^T
#pragma unroll
          for (int i = 0; i < MD; ++i) {
            uint32_t a0, a1, a2, a3;
            const int row = (lane & 7) + 8 * (lane >> 4);
            const int ch = 2 * i + ((lane >> 3) & 1);
            ldsm_x4_t(a0, a1, a2, a3, vs_t + swz<D>(row, ch));
            mma_bf16(o[i], a0, a1, a2, a3, bhi[0], bhi[1]);
            mma_bf16(o[i], a0, a1, a2, a3, blo[0], blo[1]);
          }
        }
        cp_async_wait<0>();
      }  // pieces

      // ---- the segment's partial, this warp's rows: slot k of (pair, split s)
      const int k = gi - sk_warp_of(P * sk.E + pl.e_bound[s], sk.X, sk.W);
      if (k < 0 || k >= sk.K) {
        if (tig == 0) record_error(kErrBadInput);
        continue;
      }
      const long long slot = ((P * p.S + s) * sk.K + k);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float l = lcol[e];
        l += __shfl_xor_sync(0xffffffffu, l, 4);
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        const int m = 8 * wig + 2 * cq + e;
        if (m >= p.M) continue;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        float *orow = sk.sk_o + (slot * p.M + m) * D;
#pragma unroll
        for (int i = 0; i < MD; ++i) {
          orow[16 * i + gq] = o[i][e] * inv;
          orow[16 * i + gq + 8] = o[i][2 + e] * inv;
        }
        if (gq == 0) sk.sk_lse[slot * p.M + m] = l > 0.f ? (mcol[e] + __log2f(l)) * kLn2 : -INFINITY;
      }
    }
  }
}

}  // namespace dec
}  // namespace qsa
