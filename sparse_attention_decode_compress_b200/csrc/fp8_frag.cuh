// FP8 E4M3 K/V tiles read straight into f16 tensor-core fragments.
//
// Every E4M3 value is exact in f16, and one cvt.rn.f16x2.e4m3x2 converts two
// of them, so the fp8 decode runs both products in f16 (mma m16n8k16 f16 ->
// f32) with its K and V fragments built in registers from the raw fp8 tile:
// no converted copy of the stage in shared memory, ~4x fewer conversion
// instructions than fp8 -> f32 -> bf16, and the shared memory saved holds
// more stages in flight.
//
// The other operands are brought into f16's range:
//   - Q is scaled per query row by a power of two 2^e with
//     2^14 <= max|q| * 2^e < 2^15.  bf16 has 8 significant bits and f16 11,
//     so every element at least 2^-28 of the row maximum converts exactly;
//     the logits are multiplied by 2^-e.
//   - P (<= 1) carries the per-(page, head) V scale relative to a power of
//     two `vsref` of the chunk (the largest scale's binade), so P * vs /
//     vsref < 2; the chunk's output is multiplied by vsref.
//   - P is fed as an f16 hi + lo pair: ~22 significant bits down to 2^-14,
//     an absolute error below 2^-25 under it.
//
// The contractions leave two orderings free, used to make each lane's bytes
// contiguous:
//   - S^T = K Q^T sums over the head dimension: a k-step may take any 16 dims
//     as long as K and Q take the same ones.  Lane (gq, cq) of k-step
//     kk = 4i + u holds dims 16(cq + 4i) + 4u + {0, 1} in fragment registers
//     a0 / a1 (tokens gq / gq + 8) and b0, and dims + {2, 3} in a2 / a3 and
//     b1, so one 16-byte load of a token row feeds four k-steps.
//   - O^T = V^T P^T has the head dimension on M: m-tile i, row gq is dim
//     (D/8) gq + 2i and row gq + 8 is dim (D/8) gq + 2i + 1.  A lane's V bytes
//     of one token are then D/8 contiguous bytes, and its output columns D/8
//     contiguous floats.
#pragma once
#include "sparse_decode.cuh"

namespace qsa {
namespace dec {

// Byte offset of 16-byte chunk ch of row `row` in a raw fp8 tile of D-byte
// rows.  The XOR pattern keeps both fragment reads below free of bank
// conflicts at D = 128 (the K read of rows gq, gq + 1 and the V read of rows
// 2cq, 2cq + 1 in one 8-lane phase); at D = 64 the V read is 2-way.
template <int D>
__device__ __forceinline__ int fp8_swz(int row, int ch) {
  static_assert(D == 64 || D == 128, "fp8 tile layout");
  const int x = (D == 128) ? ((row & 6) ^ ((row & 1) << 2)) : ((row >> 1) & 3);
  return row * D + ((ch ^ x) << 4);
}

// Two E4M3 values -> f16x2 (the lower byte to the lower half): the low
// (bytes 0, 1) or the high (bytes 2, 3) half of a word.
__device__ __forceinline__ uint32_t e4m3x2_f16x2(uint32_t w) {
  uint32_t d;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, l;\n\t}"
      : "=r"(d) : "r"(w));
  return d;
}
__device__ __forceinline__ uint32_t e4m3x2_f16x2_hi(uint32_t w) {
  uint32_t d;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, h;\n\t}"
      : "=r"(d) : "r"(w));
  return d;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// 2^e as a float, e in [-126, 127].
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((e + 127) << 23); }

// Q B-fragments of one 8-row tile in f16, in the k order above, for query row
// `qrow` (nullptr: a padding row, all zero).  Returns 2^-e, the factor that
// takes this row's logits back to Q's scale (lanes of one row agree).
template <int D>
__device__ __forceinline__ float q_frags_f16(const __nv_bfloat16 *qrow, int cq,
                                             uint32_t (&qb)[D / 16][2]) {
  constexpr int MD = D / 16;
  uint2 raw[MD];
  uint32_t mx = 0;
#pragma unroll
  for (int kk = 0; kk < MD; ++kk) {
    const int i = kk >> 2, u = kk & 3;
    raw[kk] = qrow ? *reinterpret_cast<const uint2 *>(qrow + 16 * (cq + 4 * i) + 4 * u)
                   : make_uint2(0u, 0u);
    mx = max(mx, max(max(raw[kk].x & 0x7fffu, (raw[kk].x >> 16) & 0x7fffu),
                     max(raw[kk].y & 0x7fffu, (raw[kk].y >> 16) & 0x7fffu)));
  }
  mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
  mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  // bf16 magnitude bits order like the values; biased exponent E:
  // 2^(E-127) <= max < 2^(E-126), so e = 141 - E puts max in [2^14, 2^15)
  const int E = (int)(mx >> 7);
  const int e = (mx == 0u) ? 0 : min(141 - E, 126);
  const float sc = pow2f(e);
#pragma unroll
  for (int kk = 0; kk < MD; ++kk) {
    const uint32_t w[2] = {raw[kk].x, raw[kk].y};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float lo = __uint_as_float(w[h] << 16) * sc;
      const float hi = __uint_as_float(w[h] & 0xffff0000u) * sc;
      qb[kk][h] = pack_f16(lo, hi);
    }
  }
  return pow2f(-e);
}

// S^T[16 tokens x 8] += K[16 x D] . Q^T for one 8-row tile, K read from the
// raw fp8 tile; even and odd k-steps go to two accumulators.
template <int D>
__device__ __forceinline__ void qk_fp8(const uint8_t *kt, int gq, int cq,
                                       const uint32_t (&qb)[D / 16][2], float (&s0)[4],
                                       float (&s1)[4]) {
#pragma unroll
  for (int i = 0; i < D / 64; ++i) {
    const uint4 r0 = *reinterpret_cast<const uint4 *>(kt + fp8_swz<D>(gq, cq + 4 * i));
    const uint4 r1 = *reinterpret_cast<const uint4 *>(kt + fp8_swz<D>(gq + 8, cq + 4 * i));
    const uint32_t w0[4] = {r0.x, r0.y, r0.z, r0.w};
    const uint32_t w1[4] = {r1.x, r1.y, r1.z, r1.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int kk = 4 * i + u;
      const uint32_t a0 = e4m3x2_f16x2(w0[u]), a1 = e4m3x2_f16x2(w1[u]);
      const uint32_t a2 = e4m3x2_f16x2_hi(w0[u]), a3 = e4m3x2_f16x2_hi(w1[u]);
      if (kk & 1) mma_f16(s1, a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
      else mma_f16(s0, a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
    }
  }
}

// This lane's V bytes of the stage: tokens 2cq, 2cq + 1, 2cq + 8, 2cq + 9,
// dims (D/8) gq .. + D/8, as D/32 words per token.
template <int D>
struct VRaw {
  uint32_t t[4][D / 32];
};

template <int D>
__device__ __forceinline__ void v_raw_fp8(const uint8_t *vt, int gq, int cq, VRaw<D> &v) {
  const int tok[4] = {2 * cq, 2 * cq + 1, 2 * cq + 8, 2 * cq + 9};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if constexpr (D == 128) {
      const uint4 x = *reinterpret_cast<const uint4 *>(vt + fp8_swz<D>(tok[k], gq));
      v.t[k][0] = x.x;
      v.t[k][1] = x.y;
      v.t[k][2] = x.z;
      v.t[k][3] = x.w;
    } else {
      const uint2 x =
          *reinterpret_cast<const uint2 *>(vt + fp8_swz<D>(tok[k], gq >> 1) + 8 * (gq & 1));
      v.t[k][0] = x.x;
      v.t[k][1] = x.y;
    }
  }
}

// A fragments of m-tile i of V^T (dims (D/8) gq + 2i and + 1; tokens 2cq,
// 2cq + 1 in a0 / a1 and 2cq + 8, 2cq + 9 in a2 / a3).
template <int D>
__device__ __forceinline__ void v_frag_fp8(const VRaw<D> &v, int i, uint32_t &a0, uint32_t &a1,
                                           uint32_t &a2, uint32_t &a3) {
  const int w = i >> 1;
  const uint32_t sel = (i & 1) ? 0x7362u : 0x5140u;  // bytes (2i, 2i+1) of the two tokens, interleaved
  const uint32_t lo = prmt(v.t[0][w], v.t[1][w], sel);
  const uint32_t hi = prmt(v.t[2][w], v.t[3][w], sel);
  a0 = e4m3x2_f16x2(lo);
  a1 = e4m3x2_f16x2_hi(lo);
  a2 = e4m3x2_f16x2(hi);
  a3 = e4m3x2_f16x2_hi(hi);
}

// Power-of-two reference of a chunk's V scales: the binade of the largest
// |vs| (1 when all are zero).
__device__ __forceinline__ float vs_binade(float mx_abs) {
  const int E = (__float_as_int(mx_abs) >> 23) & 0xff;
  return (mx_abs > 0.f) ? pow2f(min(max(E, 1), 254) - 127) : 1.f;
}

// Stores this lane's column of an O^T tile in the fp8 dim order: m-tile i
// holds dims (D/8) gq + 2i (c0 / c1) and + 1 (c2 / c3).
template <int D, typename Acc>
__device__ __forceinline__ void store_col_fp8(float *orow, const Acc &o, int e, int gq, float inv) {
#pragma unroll
  for (int w = 0; w < D / 32; ++w) {
    const float4 v = make_float4(o(2 * w, e) * inv, o(2 * w, 2 + e) * inv, o(2 * w + 1, e) * inv,
                                 o(2 * w + 1, 2 + e) * inv);
    *reinterpret_cast<float4 *>(orow + (D / 8) * gq + 4 * w) = v;
  }
}

}  // namespace dec
}  // namespace qsa
