// qsa_sparse_decode: exact softmax attention over the selected tokens of the
// uncompressed paged K/V, split into KV partitions.
//
// Method: final softmax and value aggregation run on the uncompressed K and V
// of the ~2,048 selected token positions; each decode-context-parallel rank
// reads only its own slice of the cache and the partial results are merged
// afterwards (blog "Qwen 4 QSA 迎来解码上下文并行…", section 拉取请求实际改变了
// 什么).  MTP: the selection of query token 0 is reused by the speculative
// tokens (PR #53896 完整报告, 实现拆解), which also see the speculative tail.
//
// Work decomposition (shared by both kernels): work items are (request r,
// kv head g, chunk).  The "extended selection" of r is the sorted selection
// row followed by the speculative-tail blocks that are not selected; split s
// owns the entries whose block lies in its page slice (a contiguous range,
// since the list is sorted), cut into ceil(n / chunk) chunks of equal size
// (to one entry), `chunk` <= kChunkBlocks micro-blocks being chosen by the
// host for the batch shape.
// A split with one chunk writes o_part/lse_part directly; a split with
// several chunks stages them in the workspace and the chunk that finishes
// last (atomic ticket) merges them by log-sum-exp.
//
// This file holds the split/chunk plan, the output helpers and the plain
// CUDA-core kernel for fp32 caches (one CTA per item, online softmax per
// query row); the tensor-core kernel for bf16 / fp8 caches is in
// sparse_decode_warp.cuh.
#pragma once
#include "qsa_common.cuh"

namespace qsa {
namespace dec {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kChunkBlocks = 128;  // largest chunk the host picks (bf16 metadata piece), micro-blocks
constexpr int kChunkTokens = kChunkBlocks * 4;
constexpr int kMinChunkBlocks = 32;  // smallest chunk the host picks
constexpr int kMaxSplits = 16;
constexpr int kMaxT = 4;
constexpr int kMaxRows = 32;  // G * T
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct Params {
  CacheDev c;
  int B, T, Hq, G, M;
  const void *q;
  const int32_t *ctx_lens;
  const int32_t *sel;
  int topk;
  float scale_log2;  // sm_scale * log2(e)
  int S;
  float *o_part;    // [S, B, T, Hq, D]
  float *lse_part;  // [S, B, T, Hq]
  float *ws_o;      // [B, Hkv, nch, M, D]
  float *ws_lse;    // [B, Hkv, nch, M]
  int32_t *tickets;  // [B, Hkv, S], zeroed by the call's reset kernel
  int32_t *counters; // work counters of the persistent kernels, zeroed likewise
  int nch;           // chunk slots per (r, g)
  int chunk;         // target micro-blocks per chunk, kMinChunkBlocks..kChunkBlocks
  // splits computed: [s_lo, s_hi) of S (a decode-context-parallel rank
  // computes its own); o_part / lse_part hold them from index 0
  int s_lo = 0, s_hi = 0;
};

// First kernel of every decode call: zeroes the workspace header (the work
// counters and the split tickets), so the caller's workspace may hold
// anything.  It goes on the stream right before the decode kernel, both with
// programmatic launch: the decode's CTAs become resident while this runs.
__global__ void __launch_bounds__(1024) decode_header_reset_kernel(int32_t *hdr, int n) {
  pdl_open();
  for (int i = threadIdx.x; i < n; i += blockDim.x) hdr[i] = 0;
}

// Per-CTA plan, computed by warp 0.
struct Plan {
  int L, p0, nvalid, nE, n_extra;
  int extra[2];
  int split, nchunks_split, chunk_in_split, first_chunk_of_split;
  int e_begin, e_end;
  int active;  // this CTA owns a chunk
  int e_bound[kMaxSplits + 1];
  int ch_count[kMaxSplits];
  long long tb[kMaxSplits + 1];  // token boundary of each split
};

// Entry k of the extended selection of request r.
__device__ __forceinline__ int ext_block(const int32_t *sel_r, const Plan &pl, int k) {
  return k < pl.nvalid ? sel_r[k] : pl.extra[k - pl.nvalid];
}

// One warp reads the selection row once, coalesced, and derives the split
// boundaries in the extended list: the split index of a selected block
// (binary search of its first token in the split boundaries) never
// decreases along the ascending row, so the lane holding entry k writes
// e_bound[s] = k for every split s it starts.  If `stash` is not NULL the row
// is also copied there (entries [0, topk)).
__device__ void make_plan(const Params &p, int r, int chunk, Plan &pl, int *stash = nullptr) {
  const int lane = threadIdx.x & 31;
  const int32_t *sel_r = p.sel + (long long)r * p.topk;
  constexpr int kBatch = 16;  // entries per lane loaded before any is used
  // the first batch of the selection row is loaded together with the
  // context length (the row is always readable; an empty context ignores it)
  int v[kBatch];
#pragma unroll
  for (int j = 0; j < kBatch; ++j) {
    const int k = j * 32 + lane;
    v[j] = (k < p.topk) ? sel_r[k] : -1;
  }
  int L = p.ctx_lens[r];
  if (L < p.T) {
    if (lane == 0) record_error(kErrBadInput);
    L = 0;
  }
  const int p0 = L - p.T;
  const long long NP = ((long long)L + p.c.page_size - 1) / p.c.page_size;
  if (lane <= p.S) pl.tb[lane] = min(((long long)lane * NP / p.S) * p.c.page_size, (long long)L);
  __syncwarp();
  // below[s] (kept in e_bound[s] by lane 0): selected blocks starting
  // before the token boundary of split s
  if (lane < p.S) pl.e_bound[lane] = 0;
  __syncwarp();
  int nvalid = 0, last = -1;
  const int n_entries = (L > 0) ? p.topk : 0;
  for (int base = 0; base < n_entries; base += 32 * kBatch) {
    if (base > 0) {
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int k = base + j * 32 + lane;
        v[j] = (k < n_entries) ? sel_r[k] : -1;
      }
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int k = base + j * 32 + lane;
      if (stash && k < n_entries) stash[k] = v[j];
      nvalid += v[j] >= 0;
      last = max(last, v[j]);
    }
#pragma unroll 1
    for (int sb = 1; sb < p.S; ++sb) {
      const long long tbs = pl.tb[sb];
      int cnt = 0;
#pragma unroll
      for (int j = 0; j < kBatch; ++j) cnt += __popc(__ballot_sync(0xffffffffu, v[j] >= 0 && 4LL * v[j] < tbs));
      if (lane == 0) pl.e_bound[sb] += cnt;
    }
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
    nvalid += __shfl_xor_sync(0xffffffffu, nvalid, o);
  }
  __syncwarp();
  if (lane == 0) {
    pl.L = L;
    pl.p0 = p0;
    pl.nvalid = nvalid;
    if (last >= 0 && 4LL * last > (long long)p0) record_error(kErrBadInput);
    int ne = 0;
    if (L > 0 && p.T > 1) {
      const int bs = (p0 + 1) >> 2, be = (L - 1) >> 2;
      for (int b = bs; b <= be && ne < 2; ++b)
        if (b > last) pl.extra[ne++] = b;
    }
    pl.n_extra = ne;
    pl.nE = nvalid + ne;
    // speculative-tail blocks follow every selected block: they move the
    // boundaries of the splits after theirs
    pl.e_bound[0] = 0;
    for (int s = 1; s < p.S; ++s) {
      int add = 0;
      for (int x = 0; x < ne; ++x) add += (4LL * pl.extra[x] < pl.tb[s]);
      pl.e_bound[s] = min(pl.e_bound[s], nvalid) + add;
    }
    pl.e_bound[p.S] = pl.nE;
    int cum = 0;
    pl.active = 0;
    for (int s = 0; s < p.S; ++s) {
      const int n = pl.e_bound[s + 1] - pl.e_bound[s];
      // chunks of n / ch <= p.chunk entries; -1 marks a split not computed here
      const int ch = (s < p.s_lo || s >= p.s_hi) ? -1 : (n + p.chunk - 1) / p.chunk;
      pl.ch_count[s] = ch;
      if (!pl.active && chunk >= cum && chunk < cum + ch) {
        const int k = chunk - cum;
        pl.active = 1;
        pl.split = s;
        pl.nchunks_split = ch;
        pl.chunk_in_split = k;
        pl.first_chunk_of_split = cum;
        pl.e_begin = pl.e_bound[s] + (int)((long long)k * n / ch);
        pl.e_end = pl.e_bound[s] + (int)((long long)(k + 1) * n / ch);
      }
      cum += max(ch, 0);
    }
  }
  __syncwarp();
}

// Output row m of (r, g) in split s: query token t = m / G, head
// h = g*G + m % G; splits are stored from s_lo on.
__device__ __forceinline__ long long out_row(const Params &p, int s, int r, int g, int m) {
  const int t = m / p.G, h = g * p.G + m % p.G;
  return (((long long)(s - p.s_lo) * p.B + r) * p.T + t) * p.Hq + h;
}

// Empty splits of (r, g) get o = 0, lse = -inf (written by chunk 0's CTA).
template <int D>
__device__ void write_empty_splits(const Params &p, const Plan &pl, int r, int g) {
  for (int s = 0; s < p.S; ++s) {
    if (pl.ch_count[s] != 0) continue;
    for (int i = threadIdx.x; i < p.M * D; i += blockDim.x) {
      const int m = i / D, d = i % D;
      p.o_part[out_row(p, s, r, g, m) * D + d] = 0.f;
      if (d == 0) p.lse_part[out_row(p, s, r, g, m)] = -INFINITY;
    }
  }
}

// Writes this chunk's result (o_s [M][D] normalised, lse [M] natural log, in
// shared memory) to the split outputs, merging the split's chunks when it is
// the last of them to finish.
// `wsm` is shared scratch of at least nch * M floats that the caller no
// longer needs (it may alias o_s only beyond its first M * D floats).
template <int D>
__device__ void finish_chunk(const Params &p, const Plan &pl, int r, int g, const float *o_s,
                             const float *lse_s, int *flag, float *wsm) {
  const int s = pl.split;
  if (pl.nchunks_split == 1) {
    for (int i = threadIdx.x; i < p.M * D; i += blockDim.x) {
      const int m = i / D, d = i % D;
      p.o_part[out_row(p, s, r, g, m) * D + d] = o_s[m * D + d];
      if (d == 0) p.lse_part[out_row(p, s, r, g, m)] = lse_s[m];
    }
    return;
  }
  const int Hkv = p.c.num_kv_heads;
  const long long slot = ((long long)r * Hkv + g) * p.nch + (blockIdx.x);
  float *wo = p.ws_o + slot * p.M * D;
  float *wl = p.ws_lse + slot * p.M;
  for (int i = threadIdx.x; i < p.M * D; i += blockDim.x) wo[i] = o_s[i];
  for (int i = threadIdx.x; i < p.M; i += blockDim.x) wl[i] = lse_s[i];
  __threadfence();
  __syncthreads();
  int32_t *ticket = p.tickets + ((long long)r * Hkv + g) * p.S + s;
  if (threadIdx.x == 0) {
    const int t = atomicAdd(ticket, 1);
    *flag = (t == pl.nchunks_split - 1);  // all chunks of the split have reported
  }
  __syncthreads();
  if (!*flag) return;
  __threadfence();
  // merge the split's chunks: their lse into shared memory first (one batch
  // of loads), then each output element reads its chunk partials with
  // independent loads
  const long long slot0 = ((long long)r * Hkv + g) * p.nch + pl.first_chunk_of_split;
  const int nc = pl.nchunks_split;
  float *lse_c = wsm;  // [nc][M]
  for (int i = threadIdx.x; i < nc * p.M; i += blockDim.x)
    lse_c[i] = __ldcg(p.ws_lse + slot0 * p.M + i);
  __syncthreads();
  for (int i = threadIdx.x; i < p.M * D; i += blockDim.x) {
    const int m = i / D, d = i % D;
    float mx = -INFINITY;
    for (int c = 0; c < nc; ++c) mx = fmaxf(mx, lse_c[c * p.M + m]);
    float num = 0.f, den = 0.f;
    if (mx != -INFINITY) {
      int c = 0;
      for (; c + 4 <= nc; c += 4) {
        float ov[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) ov[u] = __ldcg(p.ws_o + ((slot0 + c + u) * p.M + m) * D + d);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float l = lse_c[(c + u) * p.M + m];
          const float w = (l == -INFINITY) ? 0.f : __expf(l - mx);
          den += w;
          num += w * ov[u];
        }
      }
      for (; c < nc; ++c) {
        const float l = lse_c[c * p.M + m];
        const float w = (l == -INFINITY) ? 0.f : __expf(l - mx);
        den += w;
        num += w * __ldcg(p.ws_o + ((slot0 + c) * p.M + m) * D + d);
      }
    }
    p.o_part[out_row(p, s, r, g, m) * D + d] = den > 0.f ? num / den : 0.f;
    if (d == 0) p.lse_part[out_row(p, s, r, g, m)] = den > 0.f ? mx + __logf(den) : -INFINITY;
  }
}

// Per-token metadata of a chunk (256 token slots).
struct TokMeta {
  long long off[kChunkTokens];  // element offset of the (token, head g) row, -1 = not loaded
  int pos[kChunkTokens];        // logical position, -1 = no token
  unsigned char insel[kChunkTokens];
  float ks[kChunkTokens];       // fp8 scales (1 otherwise)
  float vs[kChunkTokens];
};

template <int D>
__device__ void fill_meta(const Params &p, const Plan &pl, int r, int g, TokMeta &tm) {
  const int32_t *sel_r = p.sel + (long long)r * p.topk;
  const int P = p.c.page_size, Hkv = p.c.num_kv_heads;
  const bool fp8 = p.c.kv_dtype == 2;
  for (int k = threadIdx.x; k < kChunkTokens; k += blockDim.x) {
    const int e = pl.e_begin + k / 4;
    long long off = -1;
    int pos = -1;
    float ks = 1.f, vs = 1.f;
    unsigned char ins = 0;
    if (e < pl.e_end) {
      const int b = ext_block(sel_r, pl, e);
      const long long i = 4LL * b + (k & 3);
      if (b >= 0 && i < pl.L) {
        const int page = physical_page(p.c, r, i / P);
        if (page >= 0) {
          off = (((long long)page * P + (i % P)) * Hkv + g) * D;
          pos = (int)i;
          ins = e < pl.nvalid;
          if (fp8) {
            ks = p.c.k_scale[(long long)page * Hkv + g];
            vs = p.c.v_scale[(long long)page * Hkv + g];
          }
        }
      } else if (b >= 0 && (k & 3) == 0 && 4LL * b >= pl.L) {
        record_error(kErrBadInput);  // selected block beyond the context
      }
    }
    tm.off[k] = off;
    tm.pos[k] = pos;
    tm.insel[k] = ins;
    tm.ks[k] = ks;
    tm.vs[k] = vs;
  }
}

// ------------------------------------------------------------ MMA helpers --
__device__ __forceinline__ void ldsm_x4(uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3,
                                        const void *addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(addr)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3,
                                          const void *addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(addr)));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// 2^x with the SFU approximation (relative error about 2^-22); -inf -> 0.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// Byte offset of 16-byte chunk `ch` of row `row` in a swizzled tile whose
// rows are D bf16 (D*2 bytes).
template <int D>
__device__ __forceinline__ int swz(int row, int ch) {
  return row * (D * 2) + ((ch ^ (row & 7)) << 4);
}

// ------------------------------------------------------- fp32 K/V path --
// Plain CUDA-core path for fp32 caches.  The CTA stages the chunk's K and V
// rows 32 tokens at a time in shared memory; warp w holds query rows w,
// w + 4, ... .  For each tile a lane scores one token against the warp's
// rows (dot products from shared memory, no shuffles), the online softmax
// runs across the warp (one max and one sum per row and tile), and a lane
// accumulates D / 32 output dims over the tile's tokens.
constexpr int kF32Tile = 32;

template <int D>
struct F32Smem {
  TokMeta tm;
  Plan pl;
  float o[kMaxRows * D];
  float lse[kMaxRows];
  float scratch[kMaxRows * (4096 / kMinChunkBlocks + 2 + kMaxSplits)];  // nch * M floats
  alignas(16) float q[kMaxRows][D];
  alignas(16) float kt[kF32Tile][D + 4];  // padded rows: the per-lane row reads miss no bank
  alignas(16) float vt[kF32Tile][D];
  float pt[kWarps][kMaxRows / kWarps][kF32Tile];
  int flag;
};

template <int D>
__global__ void __launch_bounds__(kThreads) sparse_decode_f32_kernel(Params p) {
  pdl_open();
  extern __shared__ uint8_t smem_raw[];
  using SM = F32Smem<D>;
  SM &sm = *reinterpret_cast<SM *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const int chunk = blockIdx.x, g = blockIdx.y, r = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  Plan &pl = sm.pl;
  if (warp == 0) make_plan(p, r, chunk, pl);
  __syncthreads();
  if (chunk == 0) write_empty_splits<D>(p, pl, r, g);
  if (!pl.active) return;
  fill_meta<D>(p, pl, r, g, sm.tm);
  constexpr int kPer = D / 32;
  constexpr int kR = kMaxRows / kWarps;  // rows per warp
  const float *kc = static_cast<const float *>(p.c.k_cache);
  const float *vc = static_cast<const float *>(p.c.v_cache);
  const float *qg = static_cast<const float *>(p.q);
  for (int i = tid; i < p.M * D; i += kThreads) {
    const int m = i / D, d = i % D;
    sm.q[m][d] = qg[(((long long)r * p.T + m / p.G) * p.Hq + g * p.G + m % p.G) * D + d];
  }
  const int ntok = (pl.e_end - pl.e_begin) * 4;
  const int p0 = pl.p0;
  float acc[kR][kPer], mx[kR], l[kR];
  int tq[kR];  // query token of each row, -1: no row
#pragma unroll
  for (int i = 0; i < kR; ++i) {
    const int m = warp + kWarps * i;
    tq[i] = m < p.M ? m / p.G : -1;
#pragma unroll
    for (int j = 0; j < kPer; ++j) acc[i][j] = 0.f;
    mx[i] = -INFINITY;
    l[i] = 0.f;
  }
  for (int k0 = 0; k0 < ntok; k0 += kF32Tile) {
    __syncthreads();  // metadata and q written; the previous tile consumed
    for (int i = tid; i < kF32Tile * D / 4; i += kThreads) {
      const int t = i / (D / 4), d = 4 * (i % (D / 4));
      const long long off = sm.tm.off[k0 + t];  // -1: no token (slots past the chunk too)
      float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), vv = kv;
      if (off >= 0) {
        kv = *reinterpret_cast<const float4 *>(kc + off + d);
        vv = *reinterpret_cast<const float4 *>(vc + off + d);
      }
      *reinterpret_cast<float4 *>(&sm.kt[t][d]) = kv;
      *reinterpret_cast<float4 *>(&sm.vt[t][d]) = vv;
    }
    __syncthreads();
    // scores of token k0 + lane against the warp's rows
    float sc[kR];
#pragma unroll
    for (int i = 0; i < kR; ++i) sc[i] = 0.f;
#pragma unroll 4
    for (int d = 0; d < D; d += 4) {
      const float4 kv = *reinterpret_cast<const float4 *>(&sm.kt[lane][d]);
#pragma unroll
      for (int i = 0; i < kR; ++i) {
        if (tq[i] < 0) continue;
        const float4 qv = *reinterpret_cast<const float4 *>(&sm.q[warp + kWarps * i][d]);
        sc[i] += kv.x * qv.x + kv.y * qv.y + kv.z * qv.z + kv.w * qv.w;
      }
    }
    const int pos = sm.tm.pos[k0 + lane];
    const bool ins = sm.tm.insel[k0 + lane];
#pragma unroll
    for (int i = 0; i < kR; ++i) {
      if (tq[i] < 0) continue;
      const bool vis = pos >= 0 && pos <= p0 + tq[i] && (ins || pos > p0);
      const float x = vis ? sc[i] * p.scale_log2 : -INFINITY;
      float mt = x;
#pragma unroll
      for (int o2 = 16; o2 >= 1; o2 >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o2));
      const float mn = fmaxf(mx[i], mt);
      const float base = (mn == -INFINITY) ? 0.f : mn;
      const float a = (mn == -INFINITY) ? 1.f : exp2f(mx[i] - base);
      const float pv = exp2f(x - base);  // 0 for an invisible token
      float ps = pv;
#pragma unroll
      for (int o2 = 16; o2 >= 1; o2 >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o2);
      l[i] = l[i] * a + ps;
      mx[i] = mn;
      sm.pt[warp][i][lane] = pv;
#pragma unroll
      for (int j = 0; j < kPer; ++j) acc[i][j] *= a;
    }
    __syncwarp();
#pragma unroll 4
    for (int t = 0; t < kF32Tile; ++t) {
      float vv[kPer];
#pragma unroll
      for (int j = 0; j < kPer; ++j) vv[j] = sm.vt[t][lane + 32 * j];
#pragma unroll
      for (int i = 0; i < kR; ++i) {
        if (tq[i] < 0) continue;
        const float pw = sm.pt[warp][i][t];
#pragma unroll
        for (int j = 0; j < kPer; ++j) acc[i][j] += pw * vv[j];
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kR; ++i) {
    const int m = warp + kWarps * i;
    if (m >= p.M) continue;
#pragma unroll
    for (int j = 0; j < kPer; ++j) sm.o[m * D + lane + 32 * j] = l[i] > 0.f ? acc[i][j] / l[i] : 0.f;
    if (lane == 0) sm.lse[m] = l[i] > 0.f ? (mx[i] + __log2f(l[i])) * kLn2 : -INFINITY;
  }
  __syncthreads();
  finish_chunk<D>(p, pl, r, g, sm.o, sm.lse, &sm.flag, sm.scratch);
}

}  // namespace dec
}  // namespace qsa
