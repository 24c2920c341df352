// qsa_sparse_decode with more than 8 query rows per kv head (MTP verify,
// wide GQA groups): warp groups instead of single warps.
//
// A work item is the same (request, kv head, chunk) as in
// sparse_decode_warp.cuh, but it belongs to a group of GW warps, one per
// 8-row tile of the M = G * T query rows.  The group shares one K/V ring,
// the chunk's plan and its token metadata: the K/V of a stage cross HBM
// once and every warp runs the one-tile arithmetic (S^T = K Q^T for its 8
// rows, online softmax, O^T += V^T P^T).  One warp carrying all M rows held
// 4x the accumulators, spilled, and spent ~4x the cycles per stage.
//
// Synchronisation inside a group uses one named barrier (id 1 + group):
// every stage waits for the warp's own cp.async share of the stage, then
// for the group, which also tells every warp that the ring slot read in
// the previous stage is free to refill.  All control decisions are read
// from the group's shared memory, so the warps of a group take the same
// path and meet at every barrier.
#pragma once
#include "sparse_decode_warp.cuh"

namespace qsa {
namespace dec {

// Chunk capacity of a group: a group streams GW times faster than a warp
// of the same rows, so it takes whole splits when the batch is small.
constexpr int kGroupChunkBlocks = 512;

template <int D, bool FP8, int NW, int NS, int GW>
struct GroupSmem {
  WarpState<D, FP8, NS, kGroupChunkBlocks> g[NW / GW];
  int item[NW / GW];
  int last[NW / GW];
};

// Token metadata of the chunk, written by the GW * 32 threads of a group
// (thread tig of nthr); same contents as fill_meta_warp.
template <typename WS, bool FP8>
__device__ void fill_meta_group(const Params &p, const Plan &pl, int r, int g, WS &W, int tig,
                                int nthr, const int *stash) {
  const int32_t *sel_r = stash ? stash : p.sel + (long long)r * p.topk;
  const int P = p.c.page_size, Hkv = p.c.num_kv_heads;
  const bool pow2 = (P & (P - 1)) == 0;
  const int lgP = 31 - __clz(P);
  for (int kb = tig; kb < WS::kCap; kb += nthr) {
    const int e = pl.e_begin + kb;
    const int b = (e < pl.e_end) ? ext_block(sel_r, pl, e) : -1;
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
    float ks = 1.f, vs = 1.f;
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
      if (FP8) {
        ks = p.c.k_scale[(long long)pg * Hkv + g];
        vs = p.c.v_scale[(long long)pg * Hkv + g];
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

// This thread's share (thread tig of GW * 32) of the cp.async copies of
// stage st into ring slot `slot`; layout as issue_stage_warp.
template <int D, bool FP8, int GW, typename WS>
__device__ __forceinline__ void issue_stage_group(const Params &p, WS &W, int slot, int st, int tig) {
  constexpr int kRowBytes = WS::kRowBytes;
  constexpr int kCh = kRowBytes / 16;             // 16-byte chunks per row
  constexpr int kItems = 2 * kTokW * kCh;          // copies per stage (K and V)
  constexpr int kPer = (kItems + GW * 32 - 1) / (GW * 32);
  const uint8_t *kbase = static_cast<const uint8_t *>(p.c.k_cache);
  const uint8_t *vbase = static_cast<const uint8_t *>(p.c.v_cache);
  const int Hkv = p.c.num_kv_heads;
  int off[kPer];
  bool load[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int it = tig + GW * 32 * i;
    const int rem = it % (kTokW * kCh);
    const int tok = st * kTokW + rem / kCh;
    load[i] = it < kItems && W.vmask(tok) != 0u;
    off[i] = load[i] ? W.boff[tok >> 2] + (tok & 3) * Hkv : 0;
  }
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int it = tig + GW * 32 * i;
    if (it >= kItems) break;
    const int kv = it / (kTokW * kCh);
    const int rem = it % (kTokW * kCh);
    const int row = rem / kCh, ch = rem % kCh;
    uint8_t *dst = W.ring[slot][kv] + (FP8 ? fp8_swz<D>(row, ch) : swz<D>(row, ch));
    const uint8_t *src = (kv ? vbase : kbase) + (long long)off[i] * kRowBytes + ch * 16;
    cp_async16_zfill(dst, src, load[i]);
  }
}

template <int D, bool FP8, int NW, int NS, int GW>
__global__ void __launch_bounds__(NW * 32, 1) sparse_decode_group_kernel(Params p) {
  pdl_open();
  static_assert(NW % GW == 0, "warps per CTA must be a multiple of the group size");
  static_assert(NS >= 2, "ring depth");
  constexpr int NG = NW / GW;
  extern __shared__ uint8_t smem_raw[];
  using SM = GroupSmem<D, FP8, NW, NS, GW>;
  using WS = WarpState<D, FP8, NS, kGroupChunkBlocks>;
  SM &sm = *reinterpret_cast<SM *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = warp / GW, wig = warp % GW;  // group, and this warp's 8-row tile
  const int tig = wig * 32 + lane;
  WS &W = sm.g[grp];
  Plan &pl = W.pl;
  const int bar = 1 + grp;
  auto gsync = [&]() { named_bar_sync(bar, GW * 32); };
  const int Hkv = p.c.num_kv_heads;
  const int total_items = p.B * Hkv * p.nch;
  const int gq = lane >> 2, cq = lane & 3;
  constexpr int MD = D / 16;
  const int ngroups = gridDim.x * NG;

  bool first = true;
  while (true) {
    if (tig == 0) {
      // first item: the group's own index, numbered across CTAs first;
      // later items: from the work counter, from the number of groups on
      int it = grp * gridDim.x + blockIdx.x;
      if (!first) it = ngroups + atomicAdd(&p.counters[0], 1);
      sm.item[grp] = it;
    }
    first = false;
    gsync();
    const int it = sm.item[grp];
    if (it >= total_items) break;
    const int c = it % p.nch;
    const int g = (it / p.nch) % Hkv;
    const int r = it / (p.nch * Hkv);

    // Q B-fragments of this warp's tile: rows m = 8 * wig + gq (fp8: f16
    // in the order of fp8_frag.cuh); csc = the logit factor of each column
    uint32_t qb[MD][2];
    float csc[2];
    {
      const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(p.q);
      const int m = 8 * wig + gq;
      const bool ok = m < p.M;
      const __nv_bfloat16 *qrow =
          qg + (((long long)r * p.T + (ok ? m / p.G : 0)) * p.Hq + g * p.G + (ok ? m % p.G : 0)) * D;
      if constexpr (FP8) {
        const float qinv = q_frags_f16<D>(ok ? qrow : nullptr, cq, qb);
#pragma unroll
        for (int e = 0; e < 2; ++e)
          csc[e] = p.scale_log2 * __shfl_sync(0xffffffffu, qinv, (2 * cq + e) * 4);
      } else {
#pragma unroll
        for (int kk = 0; kk < MD; ++kk) {
          qb[kk][0] = ok ? *reinterpret_cast<const uint32_t *>(qrow + 16 * kk + 2 * cq) : 0u;
          qb[kk][1] = ok ? *reinterpret_cast<const uint32_t *>(qrow + 16 * kk + 2 * cq + 8) : 0u;
        }
        csc[0] = csc[1] = p.scale_log2;
      }
    }
    constexpr int kStashInts = (int)(sizeof(W.ring[0]) / sizeof(int));
    int *stash = p.topk <= kStashInts ? reinterpret_cast<int *>(&W.ring[NS - 1][0][0]) : nullptr;
    if (wig == 0) {
      make_plan(p, r, c, pl, stash);
      __syncwarp();
      if (c == 0) write_empty_splits_warp<D>(p, pl, r, g, lane);
    }
    gsync();
    if (!pl.active) continue;
    fill_meta_group<WS, FP8>(p, pl, r, g, W, tig, GW * 32, stash);
    gsync();
    const float vsref = FP8 ? chunk_vsref(W, pl.e_end - pl.e_begin, lane) : 1.f;
    const float vsinv = 1.f / vsref;

    int tcol[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int m = 8 * wig + 2 * cq + e;
      tcol[e] = m < p.M ? m / p.G : -1;
    }
    const int nst = (pl.e_end - pl.e_begin + 3) / 4;
    float o[MD][4];
    float mcol[2] = {-INFINITY, -INFINITY}, lcol[2] = {0.f, 0.f};
#pragma unroll
    for (int i = 0; i < MD; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
#pragma unroll
    for (int s0 = 0; s0 < NS - 1; ++s0) {
      if (s0 < nst) issue_stage_group<D, FP8, GW>(p, W, s0, s0, tig);
      cp_async_commit();
    }
    for (int st = 0; st < nst; ++st) {
      cp_async_wait<NS - 2>();  // this thread's share of stage st has landed
      gsync();                  // ... everyone's; and slot (st - 1) % NS is free
      {
        const int sn = st + NS - 1;
        if (sn < nst) issue_stage_group<D, FP8, GW>(p, W, sn % NS, sn, tig);
        cp_async_commit();
      }
      const int slot = st % NS;
      const uint8_t *ks_t = W.ring[slot][0];
      const uint8_t *vs_t = W.ring[slot][1];
      const int tb = st * kTokW;

      // ---- S^T = K Q^T for this warp's tile
      float sacc[4] = {0.f, 0.f, 0.f, 0.f}, sac2[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (FP8) {
        qk_fp8<D>(ks_t, gq, cq, qb, sacc, sac2);
      } else {
#pragma unroll
        for (int kk = 0; kk < MD; ++kk) {
          uint32_t a0, a1, a2, a3;
          const int row = (lane & 7) + 8 * ((lane >> 3) & 1);
          const int ch = 2 * kk + (lane >> 4);
          ldsm_x4(a0, a1, a2, a3, ks_t + swz<D>(row, ch));
          if (kk & 1) mma_bf16(sac2, a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
          else mma_bf16(sacc, a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
        }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[e] += sac2[e];

      // ---- mask, online softmax per column, P^T as bf16 hi + lo fragments
      const unsigned vm0 = W.vmask(tb + gq), vm1 = W.vmask(tb + gq + 8);
      float ksc0 = 1.f, ksc1 = 1.f, vsc0 = 1.f, vsc1 = 1.f;
      if constexpr (FP8) {
        ksc0 = W.ks[(tb + gq) >> 2];
        ksc1 = W.ks[(tb + gq + 8) >> 2];
        vsc0 = W.vs[(tb + gq) >> 2] * vsinv;
        vsc1 = W.vs[(tb + gq + 8) >> 2] * vsinv;
      }
      float x[4];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int t = tcol[e];
        const bool ok0 = t >= 0 && ((vm0 >> t) & 1u);
        const bool ok1 = t >= 0 && ((vm1 >> t) & 1u);
        x[e] = ok0 ? sacc[e] * csc[e] * ksc0 : -INFINITY;
        x[2 + e] = ok1 ? sacc[2 + e] * csc[e] * ksc1 : -INFINITY;
      }
      float pj[4], alpha[2];
      bool rescale = false;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float mx = fmaxf(x[e], x[2 + e]);
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
        pj[e] = ex2(x[e] - base);
        pj[2 + e] = ex2(x[2 + e] - base);
        lcol[e] = lcol[e] * a + pj[e] + pj[2 + e];
      }
      const float v0 = pj[0] * vsc0, v1 = pj[1] * vsc0, v2 = pj[2] * vsc1, v3 = pj[3] * vsc1;
      uint32_t bhi[2], blo[2];
      p_frags<FP8>(v0, v1, v2, v3, bhi, blo);
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
      if constexpr (FP8) {
        VRaw<D> vr;
        v_raw_fp8<D>(vs_t, gq, cq, vr);
#pragma unroll
        for (int i = 0; i < MD; ++i) {
          uint32_t a0, a1, a2, a3;
          v_frag_fp8<D>(vr, i, a0, a1, a2, a3);
          mma_f16(o[i], a0, a1, a2, a3, bhi[0], bhi[1]);
          mma_f16(o[i], a0, a1, a2, a3, blo[0], blo[1]);
        }
      } else {
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
    }
    cp_async_wait<0>();

    // ---- chunk result of this warp's rows
    const int s_idx = pl.split;
    const bool direct = pl.nchunks_split == 1;
    const long long wslot = ((long long)r * Hkv + g) * p.nch + c;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float l = lcol[e];
      l += __shfl_xor_sync(0xffffffffu, l, 4);
      l += __shfl_xor_sync(0xffffffffu, l, 8);
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      const int m = 8 * wig + 2 * cq + e;
      if (m >= p.M) continue;
      const float inv = l > 0.f ? vsref / l : 0.f;
      float *orow = direct ? p.o_part + out_row(p, s_idx, r, g, m) * D : p.ws_o + (wslot * p.M + m) * D;
      if constexpr (FP8) {
        store_col_fp8<D>(orow, [&](int i, int k) { return o[i][k]; }, e, gq, inv);
      } else {
#pragma unroll
        for (int i = 0; i < MD; ++i) {
          orow[16 * i + gq] = o[i][e] * inv;
          orow[16 * i + gq + 8] = o[i][2 + e] * inv;
        }
      }
      if (gq == 0) {
        const float lse = l > 0.f ? (mcol[e] + __log2f(l)) * kLn2 : -INFINITY;
        if (direct) p.lse_part[out_row(p, s_idx, r, g, m)] = lse;
        else p.ws_lse[wslot * p.M + m] = lse;
      }
    }
    if (direct) continue;  // the next item's first barrier orders the group

    // ---- several chunks in this split: the last to finish merges them
    __threadfence();
    gsync();
    if (tig == 0) {
      int32_t *ticket = p.tickets + ((long long)r * Hkv + g) * p.S + s_idx;
      const int t = atomicAdd(ticket, 1);
      const int is_last = (t == pl.nchunks_split - 1);
      sm.last[grp] = is_last;
    }
    gsync();
    if (!sm.last[grp]) continue;
    __threadfence();
    const long long slot0 = ((long long)r * Hkv + g) * p.nch + pl.first_chunk_of_split;
    const int nc = pl.nchunks_split;
    // each warp merges its own 8 rows; their lse staged in its part of the
    // (idle) ring
    float *lse_c = reinterpret_cast<float *>(&W.ring[0][0][0]) + wig * (nc * 8);
    for (int i = lane; i < nc * 8; i += 32) {
      const int cc = i / 8, m = 8 * wig + i % 8;
      lse_c[i] = m < p.M ? __ldcg(p.ws_lse + (slot0 + cc) * p.M + m) : -INFINITY;
    }
    __syncwarp();
    for (int e4 = lane; e4 < 8 * D / 4; e4 += 32) {
      const int mi = (e4 * 4) / D, d = (e4 * 4) % D;
      const int m = 8 * wig + mi;
      if (m >= p.M) continue;
      float mx = -INFINITY;
      for (int cc = 0; cc < nc; ++cc) mx = fmaxf(mx, lse_c[cc * 8 + mi]);
      float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
      float den = 0.f;
      if (mx != -INFINITY) {
        for (int cc = 0; cc < nc; ++cc) {
          const float l = lse_c[cc * 8 + mi];
          if (l == -INFINITY) continue;
          const float4 ov = __ldcg(reinterpret_cast<const float4 *>(p.ws_o + ((slot0 + cc) * p.M + m) * D + d));
          const float w = __expf(l - mx);
          den += w;
          num.x += w * ov.x;
          num.y += w * ov.y;
          num.z += w * ov.z;
          num.w += w * ov.w;
        }
      }
      const float inv = den > 0.f ? 1.f / den : 0.f;
      *reinterpret_cast<float4 *>(p.o_part + out_row(p, s_idx, r, g, m) * D + d) =
          make_float4(num.x * inv, num.y * inv, num.z * inv, num.w * inv);
      if (d == 0) p.lse_part[out_row(p, s_idx, r, g, m)] = den > 0.f ? mx + __logf(den) : -INFINITY;
    }
  }
}

}  // namespace dec
}  // namespace qsa
