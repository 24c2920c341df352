// qsa_sparse_decode with bf16 caches and at most 8 query rows per kv head
// (the T = 1 GQA decode): stream-K over the selected entries of the batch.
//
// The extended selection of every (request r, kv head g) pair is padded to
// E = topk (+2 for the speculative tail when T > 1) entries, and the pairs'
// lists are laid end to end: X = B * Hkv * E entries.  Warp w of W takes the
// fixed range [floor(w X / W), floor((w + 1) X / W)), so every warp streams
// the same number of entries whatever the splits, requests and heads (only
// padding past a pair's real entries and entries of splits outside the
// computed range are skipped).  A range is cut into segments at pair and
// split boundaries; each segment is streamed with a fresh online softmax
// through the warp's cp.async ring (the stage arithmetic of
// sparse_decode_warp.cuh) and its normalised partial (o, lse) goes to slot
// k = w - (first warp of the segment's (pair, split)) of that (pair, split).
// A second kernel (streamk_merge_kernel) merges the slots of every (pair,
// split) into o_part and, for the merged call, the splits into o.
//
// Compared with chunks inside splits (work counter, tickets, the last chunk
// merging): no idle warps, no chunk-size spread between splits, no atomics,
// no workspace state that must start at zero, and the merge runs on the
// whole GPU after the decode instead of in the decode's last warps.  Measured
// at 256k (ncu, per launch): 55 us of decode + 8.5 us of merge against
// 63 + 5.4 us (+ the header reset) for the chunked kernel.  The fp8 decode
// keeps the chunked kernel: its warps would meet 3-4 split boundaries each,
// and the restarts and the larger merge cost more than the balance gains.
// A warp whose range crosses a split or pair boundary restarts its ring
// there (~3 us).  Streaming a warp's segments back to back instead (one
// metadata piece per request, segments padded to whole stages, the partial
// written between stages) measured slower: 64.9 against 57.5 us per launch
// at batch 128 x 16k, with 3.5x the instruction-fetch stalls.
#pragma once
#include "sparse_decode_warp.cuh"

namespace qsa {
namespace dec {

struct SKParams {
  Params p;            // shapes, caches, selection, outputs (o_part, lse_part)
  int E;               // entries per pair in the global list
  long long X;         // B * Hkv * E
  int W;               // warps of the launch
  int K;               // partial slots per (pair, split)
  float *sk_o;         // [B * Hkv, S, K, M, D] normalised partials
  float *sk_lse;       // [B * Hkv, S, K, M]
  int32_t *sk_ebound;  // [B, S + 1] split boundaries in the extended selection
  float *o;            // merged output [B, T, Hq, D] or NULL
  float *lse;          // merged lse [B, T, Hq] or NULL
};

// The warp whose range holds global entry x: the largest w with
// floor(w X / W) <= x.
__host__ __device__ __forceinline__ int sk_warp_of(long long x, long long X, int W) {
  return (int)(((x + 1) * (long long)W - 1) / X);
}
__host__ __device__ __forceinline__ long long sk_range_begin(int w, long long X, int W) {
  return (long long)w * X / W;
}

template <int D, int NW, int NS>
__global__ void __launch_bounds__(NW * 32, 1) sparse_decode_streamk_kernel(SKParams sk) {
  pdl_open();
  const Params &p = sk.p;
  extern __shared__ uint8_t smem_raw[];
  using SM = WarpSmem<D, false, NW, NS>;
  using WS = WarpState<D, false, NS, warp_piece_blocks<false>()>;
  constexpr int NT = 1;
  SM &sm = *reinterpret_cast<SM *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  WS &W = sm.w[warp];
  Plan &pl = W.pl;
  const int Hkv = p.c.num_kv_heads;
  const int gq = lane >> 2, cq = lane & 3;
  constexpr int MD = D / 16;
  const int w = blockIdx.x * NW + warp;
  if (w >= sk.W) return;
  const long long x_end = sk_range_begin(w + 1, sk.X, sk.W);
  long long x = sk_range_begin(w, sk.X, sk.W);
  constexpr int kStashInts = (int)(sizeof(W.ring[0]) / sizeof(int));
  int *stash = p.topk <= kStashInts ? reinterpret_cast<int *>(&W.ring[NS - 1][0][0]) : nullptr;
  int planned_r = -1, q_pair = -1;
  bool stash_ok = false;  // the stash holds planned_r's row (until a stage refills its slot)
  uint32_t qb[NT][MD][2];
  float csc[NT][2];
  int tcol[NT][2];

  while (x < x_end) {
    const long long P = x / sk.E;
    const int r = (int)(P / Hkv), g = (int)(P % Hkv);
    const int e_lo = (int)(x - P * sk.E);
    const int e_hi = (int)(min(x_end, (P + 1) * sk.E) - P * sk.E);
    x = P * sk.E + e_hi;
    if (r != planned_r) {
      // the selection row is stashed in the ring's last slot (idle until
      // its stage): only the metadata fill right after the plan reads it,
      // before any stage refills that slot
      cp_async_wait<0>();
      __syncwarp();
      make_plan(p, r, -1, pl, stash);
      __syncwarp();
      stash_ok = stash != nullptr;
      if (lane <= p.S) sk.sk_ebound[(long long)r * (p.S + 1) + lane] = pl.e_bound[lane];
      planned_r = r;
    }
    // this pair's entries of each computed split within the warp's range:
    // one segment per split, streamed with a fresh online softmax
    const int nE = pl.nE;
    for (int s = p.s_lo; s < p.s_hi; ++s) {
      const int eb = max(e_lo, pl.e_bound[s]);
      const int ee = min(min(e_hi, nE), pl.e_bound[s + 1]);
      if (eb >= ee) continue;
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
      // the segment streams in metadata pieces of at most kCap entries
      for (int pb = eb; pb < ee; pb += WS::kCap) {
        const int pe = min(pb + WS::kCap, ee);
        cp_async_wait<0>();  // no stage in flight into the stash's slot
        __syncwarp();
        fill_meta_warp<WS, false>(p, pl, r, g, W, lane, stash_ok ? stash : nullptr, pb, pe);
        __syncwarp();
        stash_ok = false;  // the stages below may refill the stash's ring slot
        const int nst = (pe - pb + 3) / 4;
#pragma unroll
        for (int s0 = 0; s0 < NS - 1; ++s0) {
          if (s0 < nst) issue_stage_warp<D, false>(p, W, s0, s0, lane);
          cp_async_commit();
        }
        if ((int)P != q_pair) {
          // Q as B fragments (as sparse_decode_warp_kernel), rows >= M zero,
          // loaded behind the first stages: the warp barriers of the plan
          // and the metadata fill wait for the warp's loads in flight, so Q
          // issued before them held the prologue up by its own latency
          const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(p.q);
#pragma unroll
          for (int j = 0; j < NT; ++j) {
            const int m = 8 * j + gq;
            const bool ok = m < p.M;
            const __nv_bfloat16 *qrow =
                qg + (((long long)r * p.T + (ok ? m / p.G : 0)) * p.Hq + g * p.G + (ok ? m % p.G : 0)) * D;
#pragma unroll
            for (int kk = 0; kk < MD; ++kk) {
              qb[j][kk][0] = ok ? *reinterpret_cast<const uint32_t *>(qrow + 16 * kk + 2 * cq) : 0u;
              qb[j][kk][1] = ok ? *reinterpret_cast<const uint32_t *>(qrow + 16 * kk + 2 * cq + 8) : 0u;
            }
            csc[j][0] = csc[j][1] = p.scale_log2;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int mm = 8 * j + 2 * cq + e;
              tcol[j][e] = mm < p.M ? mm / p.G : -1;
            }
          }
          q_pair = (int)P;
        }
        for (int st = 0; st < nst; ++st) {
          {
            const int sn = st + NS - 1;
            if (sn < nst) issue_stage_warp<D, false>(p, W, sn % NS, sn, lane);
            cp_async_commit();
          }
          cp_async_wait<NS - 1>();
          __syncwarp();
          const int slot = st % NS;
          const uint8_t *ks_t = W.ring[slot][0];
          const uint8_t *vs_t = W.ring[slot][1];
          const int tb = st * kTokW;
          float sacc[NT][4], sac2[NT][4];
#pragma unroll
          for (int j = 0; j < NT; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) sacc[j][e] = sac2[j][e] = 0.f;
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
#pragma unroll
          for (int j = 0; j < NT; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) sacc[j][e] += sac2[j][e];
          const unsigned vm0 = W.vmask(tb + gq), vm1 = W.vmask(tb + gq + 8);
          uint32_t bhi[NT][2], blo[NT][2];
          bool rescale = false;
          float alpha[NT][2];
#pragma unroll
          for (int j = 0; j < NT; ++j) {
            float xx[4];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int t = tcol[j][e];
              const bool ok0 = t >= 0 && ((vm0 >> t) & 1u);
              const bool ok1 = t >= 0 && ((vm1 >> t) & 1u);
              xx[e] = ok0 ? sacc[j][e] * csc[j][e] : -INFINITY;
              xx[2 + e] = ok1 ? sacc[j][2 + e] * csc[j][e] : -INFINITY;
            }
            float pj[4];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              float mx = fmaxf(xx[e], xx[2 + e]);
              mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
              mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
              mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
              const float m_old = mcol[j][e];
              const float m_new = fmaxf(m_old, mx);
              const float base = (m_new == -INFINITY) ? 0.f : m_new;
              const float al = (m_new == -INFINITY) ? 1.f : ex2(m_old - base);
              alpha[j][e] = al;
              rescale |= (al != 1.f);
              mcol[j][e] = m_new;
              pj[e] = ex2(xx[e] - base);
              pj[2 + e] = ex2(xx[2 + e] - base);
              lcol[j][e] = lcol[j][e] * al + pj[e] + pj[2 + e];
            }
            p_frags<false>(pj[0], pj[1], pj[2], pj[3], bhi[j], blo[j]);
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
          __syncwarp();  // the slot may be refilled by the next issue
        }
        cp_async_wait<0>();
        __syncwarp();
      }  // pieces

      // ---- the segment's partial: slot k of (pair, split s)
      const int k = w - sk_warp_of(P * sk.E + pl.e_bound[s], sk.X, sk.W);
      if (k < 0 || k >= sk.K) {
        if (lane == 0) record_error(kErrBadInput);
        continue;
      }
      const long long slot = ((P * p.S + s) * sk.K + k);
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
          const float inv = l > 0.f ? 1.f / l : 0.f;
          float *orow = sk.sk_o + (slot * p.M + m) * D;
#pragma unroll
          for (int i = 0; i < MD; ++i) {
            orow[16 * i + gq] = o[i][j][e] * inv;
            orow[16 * i + gq + 8] = o[i][j][2 + e] * inv;
          }
          if (gq == 0) sk.sk_lse[slot * p.M + m] = l > 0.f ? (mcol[j][e] + __log2f(l)) * kLn2 : -INFINITY;
        }
    }
  }
}

// Merge of the stream-K partials: one warp per (pair, query row m).  For
// each computed split s the slots of the warps that streamed part of it
// are combined by log-sum-exp into o_part[s - s_lo] (an empty split gives
// o = 0, lse = -inf).  With `o` set, the row's splits are then merged into
// o / lse with the operations of merge_row (qsa_lse_merge), on the values
// just computed, so the result has the same bits as qsa_lse_merge of o_part.
// The (split, slot) pairs of the row are flattened across the lanes: each
// split's maximum lse is taken first, then every slot is weighed by
// exp(lse - maximum) (lane-parallel) and the weights and the weighted rows
// (a float4 slice per lane, 16 slot rows loaded together) are summed in
// slot order, so a split's bits do not depend on the lanes its slots land
// on (which depend on the splits a call computes).  Up to 16 slots per row
// take one round of loads (lse and rows together); more take a pass over
// the lse for the maxima and a second over lse and rows.  (A running maximum with a rescale per
// slot, serial over the slots, cost ~60 instructions per slot: 15 us per
// launch at batch 16 with ~32 slots per split, 8.6 us at batch 128.)
constexpr int kSKMergeThreads = 128;
constexpr int kSKMergeSlots = 16;  // slot rows loaded together

template <int D, int NSMAX>
__global__ void __launch_bounds__(kSKMergeThreads) streamk_merge_kernel(SKParams sk) {
  pdl_open();
  static_assert(D % 4 == 0 && D <= 128, "float4 slices of one warp");
  const Params &p = sk.p;
  const int Hkv = p.c.num_kv_heads;
  const long long wid = ((long long)blockIdx.x * kSKMergeThreads + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long pairs = (long long)p.B * Hkv;
  if (wid >= pairs * p.M) return;
  const long long P = wid / p.M;
  const int m = (int)(wid % p.M);
  const int r = (int)(P / Hkv), g = (int)(P % Hkv);
  const int ns = p.s_hi - p.s_lo;  // <= NSMAX
  const int d = 4 * lane;          // this lane's float4 slice (d < D)
  // lane i < ns: split s_lo + i, its first slot and slot count
  int nk = 0;
  if (lane < ns) {
    const int s = p.s_lo + lane;
    const int e0 = sk.sk_ebound[(long long)r * (p.S + 1) + s];
    const int e1 = sk.sk_ebound[(long long)r * (p.S + 1) + s + 1];
    if (e1 > e0) {
      const int wf = sk_warp_of(P * sk.E + e0, sk.X, sk.W);
      const int wl = sk_warp_of(P * sk.E + e1 - 1, sk.X, sk.W);
      nk = min(wl - wf + 1, sk.K);
    }
  }
  // first flattened index of each split (exclusive scan over lanes)
  int first = nk;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, first, o);
    if (lane >= o) first += y;
  }
  first -= nk;
  const int total = __shfl_sync(0xffffffffu, first + nk, 31);
  // flattened index f -> (split i, slot) and that slot's lse
  auto locate = [&](int f, int &si, long long &slot) {
    si = -1;
    int kk = 0;
#pragma unroll
    for (int i = 0; i < NSMAX; ++i) {
      const int fi = __shfl_sync(0xffffffffu, first, i);
      const int ni = __shfl_sync(0xffffffffu, nk, i);
      if (i < ns && f >= fi && f < fi + ni) {
        si = i;
        kk = f - fi;
      }
    }
    slot = (P * p.S + p.s_lo + max(si, 0)) * sk.K + kk;
  };
  float mxs[NSMAX];
  float4 os[NSMAX];
  float dens[NSMAX];
#pragma unroll
  for (int i = 0; i < NSMAX; ++i) {
    mxs[i] = -INFINITY;
    os[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    dens[i] = 0.f;
  }
  // the running maximum of each split over the lanes' slots
  auto split_max = [&](int si, float lv) {
#pragma unroll
    for (int i = 0; i < NSMAX; ++i) {
      if (i >= ns) break;
      float x = (si == i) ? lv : -INFINITY;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, off));
      mxs[i] = fmaxf(mxs[i], x);
    }
  };
  // exp(lse - its split's maximum), 0 for an empty segment
  auto weight = [&](int si, float lv) {
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < NSMAX; ++i)
      if (i == si) mx = mxs[i];
    return (lv == -INFINITY) ? 0.f : __expf(lv - mx);
  };
  // the rows of slots sub .. sub + nround - 1 (held by those lanes), loaded together
  auto load_rows = [&](float4 (&v)[kSKMergeSlots], long long slot, int sub, int nround) {
#pragma unroll
    for (int j = 0; j < kSKMergeSlots; ++j) {
      const long long sj = __shfl_sync(0xffffffffu, slot, sub + j);
      v[j] = (j < nround && d < D)
                 ? __ldcg(reinterpret_cast<const float4 *>(sk.sk_o + (sj * p.M + m) * D + d))
                 : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  // weights and weighted rows added in slot order
  auto accumulate = [&](const float4 (&v)[kSKMergeSlots], int si, float wgt, int sub, int nround) {
#pragma unroll
    for (int j = 0; j < kSKMergeSlots; ++j) {
      if (j >= nround) break;
      const int i = __shfl_sync(0xffffffffu, si, sub + j);
      const float w = __shfl_sync(0xffffffffu, wgt, sub + j);
      if (w == 0.f) continue;  // an empty segment (or an unwritten slot) adds nothing
#pragma unroll
      for (int q = 0; q < NSMAX; ++q) {
        if (q != i) continue;
        dens[q] += w;
        os[q].x = __fmaf_rn(w, v[j].x, os[q].x);
        os[q].y = __fmaf_rn(w, v[j].y, os[q].y);
        os[q].z = __fmaf_rn(w, v[j].z, os[q].z);
        os[q].w = __fmaf_rn(w, v[j].w, os[q].w);
      }
    }
  };
  if (total <= kSKMergeSlots) {
    // one round: the slots' lse and rows loaded together
    int si;
    long long slot;
    locate(lane, si, slot);
    const float lv = (si >= 0) ? __ldcg(sk.sk_lse + slot * p.M + m) : -INFINITY;
    float4 v[kSKMergeSlots];
    load_rows(v, slot, 0, total);
    split_max(si, lv);
    accumulate(v, si, weight(si, lv), 0, total);
  } else {
    // pass 1: each split's maximum lse
    for (int base = 0; base < total; base += 32) {
      int si;
      long long slot;
      locate(base + lane, si, slot);
      split_max(si, (si >= 0) ? __ldcg(sk.sk_lse + slot * p.M + m) : -INFINITY);
    }
    // pass 2: the weights and the weighted rows
    for (int base = 0; base < total; base += 32) {
      int si;
      long long slot;
      locate(base + lane, si, slot);
      const float lv = (si >= 0) ? __ldcg(sk.sk_lse + slot * p.M + m) : -INFINITY;
      const float wgt = weight(si, lv);
      const int nb = min(32, total - base);
      for (int sub = 0; sub < nb; sub += kSKMergeSlots) {
        float4 v[kSKMergeSlots];
        const int nround = min(kSKMergeSlots, nb - sub);
        load_rows(v, slot, sub, nround);
        accumulate(v, si, wgt, sub, nround);
      }
    }
  }
  // the splits' results: o_part / lse_part
  float lse_mine = -INFINITY;  // lane i: lse of split i
#pragma unroll
  for (int i = 0; i < NSMAX; ++i) {
    if (i >= ns) break;
    const bool ok = mxs[i] != -INFINITY && dens[i] > 0.f;
    const float inv = ok ? 1.f / dens[i] : 0.f;
    os[i].x *= inv;
    os[i].y *= inv;
    os[i].z *= inv;
    os[i].w *= inv;
    const float lse_i = ok ? mxs[i] + __logf(dens[i]) : -INFINITY;
    if (lane == i) lse_mine = lse_i;
    const long long orow_idx = out_row(p, p.s_lo + i, r, g, m);
    if (d < D) *reinterpret_cast<float4 *>(p.o_part + orow_idx * D + d) = os[i];
    if (lane == 0) p.lse_part[orow_idx] = lse_i;
  }
  if (!sk.o) return;
  // merge_row's operations: maximum and sum of weights by shuffles, then
  // the splits in order with fused multiply-adds
  float fm = lane < ns ? lse_mine : -INFINITY;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) fm = fmaxf(fm, __shfl_xor_sync(0xffffffffu, fm, off));
  float z = (lane < ns && lse_mine != -INFINITY) ? __expf(lse_mine - fm) : 0.f;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
  const bool empty = (fm == -INFINITY) || !(z > 0.f);
  const float lse_row = empty ? -INFINITY : fm + __logf(z);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (!empty) {
#pragma unroll
    for (int i = 0; i < NSMAX; ++i) {
      if (i >= ns) break;
      const float l = __shfl_sync(0xffffffffu, lse_mine, i);
      if (l == -INFINITY) continue;
      const float wgt = __expf(l - lse_row);
      acc.x = __fmaf_rn(wgt, os[i].x, acc.x);
      acc.y = __fmaf_rn(wgt, os[i].y, acc.y);
      acc.z = __fmaf_rn(wgt, os[i].z, acc.z);
      acc.w = __fmaf_rn(wgt, os[i].w, acc.w);
    }
  }
  const int t = m / p.G, h = g * p.G + m % p.G;
  const long long row = ((long long)r * p.T + t) * p.Hq + h;
  if (d < D) *reinterpret_cast<float4 *>(sk.o + row * D + d) = acc;
  if (lane == 0) sk.lse[row] = lse_row;
}

}  // namespace dec
}  // namespace qsa
