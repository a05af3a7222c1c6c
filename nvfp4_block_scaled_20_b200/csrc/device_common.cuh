// Device helpers shared by the sm_100a NVFP4 kernels: hardware conversions,
// packed fp32x2 arithmetic, 256-bit loads, the 16-point Hadamard butterfly
// and the per-block encoder.  Every floating-point step is an explicit
// round-to-nearest-even instruction (no contraction into fused multiply-add)
// so that results are reproducible bit for bit.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace nvfp4 {

// ----------------------------------------------------------------- errors
// Device error word values (same numbering as nvfp4_status).
constexpr uint32_t kDevErrTimeout = 6u;

// ----------------------------------------------------------------- packing
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpack2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

// Packed fp32x2 arithmetic (sm_100+), each lane-half one IEEE RN operation.
// Only used where no multiply feeds an add: the assembler may contract a
// packed multiply and a dependent packed add into a fused multiply-add.
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
// Packed subtract and fused multiply-add: only in approx_err16 below, whose
// result is used with an error bound (contraction there is harmless).
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// ----------------------------------------------------------------- loads
// 16 consecutive elements -> fp32.  bf16: one 256-bit load; fp32: two.
__device__ __forceinline__ void load16(const __nv_bfloat16* p, float v[16]) {
  uint32_t w[8];
  asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]),
                 "=r"(w[6]), "=r"(w[7])
               : "l"(p));
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
// 16 consecutive bf16 as 8 raw words (element 2i in the low half of word i).
__device__ __forceinline__ void load16_raw(const __nv_bfloat16* p, uint32_t w[8]) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]),
                 "=r"(w[6]), "=r"(w[7])
               : "l"(p));
}

// max(|a|, |b|) per bf16 half (sign bits cleared; an exact selection).
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a & 0x7FFF7FFFu), "r"(b & 0x7FFF7FFFu));
  return r;
}

__device__ __forceinline__ void load16(const float* p, float v[16]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    asm volatile("ld.global.nc.L1::no_allocate.v8.f32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=f"(v[8 * h + 0]), "=f"(v[8 * h + 1]), "=f"(v[8 * h + 2]), "=f"(v[8 * h + 3]),
                   "=f"(v[8 * h + 4]), "=f"(v[8 * h + 5]), "=f"(v[8 * h + 6]), "=f"(v[8 * h + 7])
                 : "l"(p + 8 * h));
  }
}

// One element (scalar path for strided access).
__device__ __forceinline__ float load1(const __nv_bfloat16* p) {
  unsigned short u;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(u) : "l"(p));
  return __uint_as_float(uint32_t(u) << 16);
}
__device__ __forceinline__ float load1(const float* p) { return __ldg(p); }

// Two adjacent elements (column pair of a row-major matrix).
__device__ __forceinline__ void load2(const __nv_bfloat16* p, float& a, float& b) {
  uint32_t u;
  asm volatile("ld.global.nc.b32 %0, [%1];" : "=r"(u) : "l"(p));
  a = __uint_as_float(u << 16);
  b = __uint_as_float(u & 0xFFFF0000u);
}
__device__ __forceinline__ void load2(const float* p, float& a, float& b) {
  float2 f = __ldg(reinterpret_cast<const float2*>(p));
  a = f.x;
  b = f.y;
}

// ----------------------------------------------------------------- convert
// fp32 -> E4M3 (round to nearest even, saturate to 448), low byte of result.
__device__ __forceinline__ uint32_t f32_to_e4m3(float t) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(t));
  return r & 0xFFu;
}
// E4M3 code (low byte) -> fp32, exact.
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  uint32_t h2;
  uint16_t c = (uint16_t)code;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}
// Two fp32 -> one byte of two E2M1 codes (lo in bits 0-3), RN, saturating.
__device__ __forceinline__ uint32_t f32x2_to_e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{ .reg .b8 b; cvt.rn.satfinite.e2m1x2.f32 b, %1, %2; cvt.u32.u8 %0, b; }"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}
// Byte of two E2M1 codes -> the two values as packed fp32x2 (exact).
__device__ __forceinline__ uint64_t e2m1x2_to_f32x2(uint32_t byte) {
  uint32_t h2;
  asm("{ .reg .b8 b; cvt.u8.u32 b, %1; cvt.rn.f16x2.e2m1x2 %0, b; }" : "=r"(h2) : "r"(byte));
  float lo = __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
  float hi = __half2float(__ushort_as_half((unsigned short)(h2 >> 16)));
  return pack2(lo, hi);
}

// ----------------------------------------------------------------- RHT
// y = 1/4 * H16 * diag(s) * x, s_j = -1 where bit j of mask is set.  Sign
// flip, butterflies with strides 1, 2, 4, 8 ((a, b) -> (a + b, a - b), fp32
// RN), then the exact scaling by 1/4.  Strides 2, 4 and 8 pair elements of
// equal parity, so they run on packed pairs (v[2k], v[2k+1]): each lane of a
// packed add is the same IEEE operation as the scalar one.
__device__ __forceinline__ void rht16_butterflies(float v[16]) {
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    const float a = v[i], b = v[i + 1];
    v[i] = __fadd_rn(a, b);
    v[i + 1] = __fsub_rn(a, b);
  }
  uint64_t P[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) P[k] = pack2(v[2 * k], v[2 * k + 1]);
#pragma unroll
  for (int hp = 1; hp < 8; hp <<= 1) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (k & hp) continue;
      const uint64_t a = P[k], b = P[k + hp];
      P[k] = add2(a, b);
      P[k + hp] = sub2(a, b);
    }
  }
  const uint64_t quarter = pack2(0.25f, 0.25f);
#pragma unroll
  for (int k = 0; k < 8; ++k) unpack2(mul2(P[k], quarter), v[2 * k], v[2 * k + 1]);
}
__device__ __forceinline__ void rht16(float v[16], uint32_t mask) {
#pragma unroll
  for (int j = 0; j < 16; ++j)
    v[j] = __uint_as_float(__float_as_uint(v[j]) ^ (((mask >> j) & 1u) << 31));
  rht16_butterflies(v);
}

// ----------------------------------------------------------------- encoder
// Global scale from the tensor amax: amax / (6 * 448); 1 for amax == 0.
__device__ __forceinline__ float alpha_from_amax(float amax) {
  return amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
}

__device__ __forceinline__ float absmax16(const float v[16]) {
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(v[i]));
  return m;
}

// Squared-error sum of 16 values in the fixed order (i, i+8), (i, i+4),
// (i, i+2), (i, i+1); e[] holds the 16 squares as 8 fp32x2 pairs
// (e[k] = {sq[2k], sq[2k+1]}).
__device__ __forceinline__ float tree16(const uint64_t e[8]) {
  uint64_t a0 = add2(e[0], e[4]), a1 = add2(e[1], e[5]);
  uint64_t a2 = add2(e[2], e[6]), a3 = add2(e[3], e[7]);
  uint64_t b0 = add2(a0, a2), b1 = add2(a1, a3);
  uint64_t c = add2(b0, b1);
  float lo, hi;
  unpack2(c, lo, hi);
  return __fadd_rn(lo, hi);
}

// Codes of correctly rounded quotients without dividing every element.
//
// q = RN(x * r), with r the hardware reciprocal of the divisor (at most one
// ulp off), is within 2^-22 (relative) of the correctly rounded quotient Q.
// The E2M1 and E4M3 conversions are monotone, so if the conversions of
// q*(1 - 2^-20) and q*(1 + 2^-20) -- an interval that contains Q -- give the
// same code, that is the code of Q.  Only when the two differ (Q within about
// 2^-20 of a rounding boundary of the target format, ~0.1% of elements) is
// the quotient computed with an IEEE division.
constexpr float kUp = 1.0f + 0x1p-20f, kDn = 1.0f - 0x1p-20f;

__device__ __forceinline__ float rcp_approx(float s) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s));
  return r;
}

// Range where the reciprocal bound above is established (no flush to zero).
__device__ __forceinline__ bool rcp_ok(float s) { return s >= 0x1p-125f && s <= 0x1p+125f; }

// Eight fp32 -> four bytes of E2M1 code pairs in one word (element 2j in the
// low nibble of byte j), round to nearest even, saturating.
__device__ __forceinline__ uint32_t cvt8_e2m1(const float a[8]) {
  uint32_t r;
  asm("{ .reg .b8 b0, b1, b2, b3;\n"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n"
      "mov.b32 %0, {b0, b1, b2, b3}; }"
      : "=r"(r)
      : "f"(a[0]), "f"(a[1]), "f"(a[2]), "f"(a[3]), "f"(a[4]), "f"(a[5]), "f"(a[6]), "f"(a[7]));
  return r;
}

// Word of four E2M1 code pairs -> eight exact fp32 values.
__device__ __forceinline__ void dec8_e2m1(uint32_t w, float v[8]) {
  uint32_t h[4];
  asm("{ .reg .b8 b0, b1, b2, b3;\n"
      "mov.b32 {b0, b1, b2, b3}, %4;\n"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n"
      "cvt.rn.f16x2.e2m1x2 %3, b3; }"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(w));
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    v[2 * k] = __half2float(__ushort_as_half((unsigned short)(h[k] & 0xFFFFu)));
    v[2 * k + 1] = __half2float(__ushort_as_half((unsigned short)(h[k] >> 16)));
  }
}

// E2M1 codes of RN(y/s) for 8 elements (s > 0) as one word.
__device__ __forceinline__ uint32_t codes8_exact(const float* y, float s) {
  float q[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) q[i] = __fdiv_rn(y[i], s);
  return cvt8_e2m1(q);
}

// Redo, with IEEE divisions, the code pairs of one 8-element word whose two
// bracket conversions disagree (diff = ca ^ cb, nonzero bytes mark them).
// Out of line: a call cannot be if-converted, so the rare exact path costs
// nothing when it is not taken.
static __device__ __noinline__ uint32_t fix_word_call(uint32_t ca, uint32_t diff, float y0, float y1,
                                               float y2, float y3, float y4, float y5, float y6,
                                               float y7, float s) {
  const float y[8] = {y0, y1, y2, y3, y4, y5, y6, y7};
  uint32_t w = ca;
#pragma unroll 1
  for (int k = 0; k < 4; ++k) {
    if ((diff >> (8 * k)) & 0xFFu) {
      const uint32_t b = f32x2_to_e2m1x2(__fdiv_rn(y[2 * k], s), __fdiv_rn(y[2 * k + 1], s));
      w = (w & ~(0xFFu << (8 * k))) | (b << (8 * k));
    }
  }
  return w;
}

// E2M1 codes of RN(y/s) for 16 elements (s > 0) as two words.  Pairs whose
// bracket conversions disagree (about 1% of pairs on activations) are redone
// exactly by fix_word_call.
__device__ __forceinline__ void codes16(const float y[16], float s, uint32_t w[2]) {
  if (rcp_ok(s)) {
    const float r = rcp_approx(s);
    const uint64_t rr = pack2(r, r), up = pack2(kUp, kUp), dn = pack2(kDn, kDn);
    uint32_t diff[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float a[8], b[8];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint64_t q = mul2(pack2(y[8 * h + 2 * k], y[8 * h + 2 * k + 1]), rr);
        unpack2(mul2(q, up), a[2 * k], a[2 * k + 1]);
        unpack2(mul2(q, dn), b[2 * k], b[2 * k + 1]);
      }
      w[h] = cvt8_e2m1(a);
      diff[h] = w[h] ^ cvt8_e2m1(b);
    }
    if (diff[0] | diff[1]) {
#pragma unroll
      for (int h = 0; h < 2; ++h)
        if (diff[h])
          w[h] = fix_word_call(w[h], diff[h], y[8 * h], y[8 * h + 1], y[8 * h + 2], y[8 * h + 3],
                               y[8 * h + 4], y[8 * h + 5], y[8 * h + 6], y[8 * h + 7], s);
    }
    return;
  }
  w[0] = codes8_exact(y, s);
  w[1] = codes8_exact(y + 8, s);
}

// Two fp32 -> two E4M3 codes (a in bits 8-15, b in bits 0-7), RN, saturating.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float a, float b) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(a), "f"(b));
  return r;
}

// Per-tensor constants for the candidate scale codes.
struct ScaleCtx {
  float alpha;
  float c6, c4;  // ~ 1/(6 alpha), 1/(4 alpha)
  bool fast;
};

__device__ __forceinline__ ScaleCtx make_scale_ctx(float alpha) {
  ScaleCtx c;
  c.alpha = alpha;
  c.fast = rcp_ok(alpha);
  const float ia = c.fast ? rcp_approx(alpha) : 0.0f;
  c.c6 = __fmul_rn(ia, 1.0f / 6.0f);
  c.c4 = __fmul_rn(ia, 0.25f);
  return c;
}

// Exact E4M3 codes of the two candidate scales (out of line; see codes16).
static __device__ __noinline__ uint2 scale_codes_exact_call(float bmax, float alpha) {
  const float u = __fdiv_rn(bmax, alpha);
  return make_uint2(f32_to_e4m3(__fdiv_rn(u, 6.0f)), f32_to_e4m3(__fmul_rn(u, 0.25f)));
}

// E4M3 codes of t6 = RN(RN(bmax / alpha) / 6) and t4 = RN(bmax / alpha) / 4.
__device__ __forceinline__ void scale_codes(float bmax, const ScaleCtx& c, uint32_t& e6,
                                            uint32_t& e4) {
  bool exact = !c.fast;
  if (!exact) {
    const float t6 = __fmul_rn(bmax, c.c6), t4 = __fmul_rn(bmax, c.c4);
    const uint32_t p6 = f32x2_to_e4m3x2(__fmul_rn(t6, kUp), __fmul_rn(t6, kDn));
    const uint32_t p4 = f32x2_to_e4m3x2(__fmul_rn(t4, kUp), __fmul_rn(t4, kDn));
    e6 = p6 & 0xFFu;
    e4 = p4 & 0xFFu;
    exact = ((p6 >> 8) != e6) || ((p4 >> 8) != e4);
  }
  if (exact) {  // out of line, as in codes16
    const uint2 e = scale_codes_exact_call(bmax, c.alpha);
    e6 = e.x;
    e4 = e.y;
  }
}

// One candidate encoding of a 16-element row segment under scale s:
// codes (8 bytes) and the row's squared error sum (y - val(q) * s)^2.
// s == 0 encodes all +0 with error sum(y^2).
struct Cand {
  uint32_t lo, hi;  // packed codes
  float err;
};

__device__ __forceinline__ Cand encode16(const float y[16], float s) {
  Cand c;
  uint64_t sq[8];
  if (s == 0.0f) {
    c.lo = c.hi = 0u;
#pragma unroll
    for (int k = 0; k < 8; ++k)
      sq[k] = pack2(__fmul_rn(y[2 * k], y[2 * k]), __fmul_rn(y[2 * k + 1], y[2 * k + 1]));
  } else {
    uint32_t w[2];
    codes16(y, s, w);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float v[8];
      dec8_e2m1(w[h], v);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        // Scalar intrinsics: documented never to be merged into a fused
        // multiply-add (the packed f32x2 forms are contracted by the
        // assembler, which would change y - v*s in its last bit).
        const float r0 = __fsub_rn(y[8 * h + 2 * k], __fmul_rn(v[2 * k], s));
        const float r1 = __fsub_rn(y[8 * h + 2 * k + 1], __fmul_rn(v[2 * k + 1], s));
        sq[4 * h + k] = pack2(__fmul_rn(r0, r0), __fmul_rn(r1, r1));
      }
    }
    c.lo = w[0];
    c.hi = w[1];
  }
  c.err = tree16(sq);
  return c;
}

// Candidate scale s = dec(e) * alpha.
__device__ __forceinline__ float cand_scale(uint32_t e, float alpha) {
  return __fmul_rn(e4m3_to_f32(e), alpha);
}

// Full 1D block encoding with the optional 4-vs-6 pick (ties keep 6).
__device__ __forceinline__ void quantize_block16(const float y[16], const ScaleCtx& ctx,
                                                 bool four_over_six, uint32_t& lo, uint32_t& hi,
                                                 uint32_t& scale) {
  uint32_t e6, e4;
  scale_codes(absmax16(y), ctx, e6, e4);
  Cand c6 = encode16(y, cand_scale(e6, ctx.alpha));
  lo = c6.lo;
  hi = c6.hi;
  scale = e6;
  if (four_over_six) {
    Cand c4 = encode16(y, cand_scale(e4, ctx.alpha));
    if (c4.err < c6.err) {
      lo = c4.lo;
      hi = c4.hi;
      scale = e4;
    }
  }
}

// ----------------------------------------------------------------- fast pick
// The 4-vs-6 pick without the exact error sums in the common case.
//
// For a candidate with scale s > 0 (a normal E4M3 code, so that every
// quotient Q = y/s is at most 6.4 and every residual |Q - v| at most 1):
//  * the exact error E (fp32 products, differences, squares and the tree,
//    as the encoding defines it) is within 304 * 2^-24 * s^2 of
//    s^2 * sum (Q - v)^2 -- each of the 16 terms is off by at most
//    15 * 2^-24 * s^2 and the four tree levels add 4 * 2^-24 of the sum;
//  * approx_err16 (quotients through the hardware reciprocal, within 2^-18
//    of Q; fused multiply-adds) is within 2^-12 of sum (Q - v)^2 -- each
//    square is off by at most 2^-16, a boundary element that rounds the
//    other way included, since both neighbours are then equally far.
// So |E - s^2 * approx| < 2^-11.8 * s^2, and with the margin B = 2^-10 * s^2
// the pick is certain when the two intervals [A - B, A + B] do not overlap.
// Otherwise (and for zero or subnormal scale codes, or scales outside the
// reciprocal's range) the block takes the exact path.
constexpr float kPickMargin = 0x1p-10f;

// q - v(q) for a packed pair of quotients, v the E2M1 value: the code pair's
// half-precision values enter through mixed-precision fused multiply-adds
// (-1 * v + q, rounded once to fp32), the same fp32 numbers as widening v
// and subtracting.
__device__ __forceinline__ uint64_t e2m1_diff_pair(uint64_t q) {
  float lo, hi;
  unpack2(q, lo, hi);
  float dlo, dhi;
  asm("{ .reg .b8 c;\n"
      ".reg .b32 h2;\n"
      ".reg .b16 vl, vh;\n"
      "cvt.rn.satfinite.e2m1x2.f32 c, %3, %2;\n"
      "cvt.rn.f16x2.e2m1x2 h2, c;\n"
      "mov.b32 {vl, vh}, h2;\n"
      "fma.rn.f32.f16 %0, vl, %4, %2;\n"
      "fma.rn.f32.f16 %1, vh, %4, %3; }"
      : "=f"(dlo), "=f"(dhi)
      : "f"(lo), "f"(hi), "h"((unsigned short)0xBC00u));
  return pack2(dlo, dhi);
}

// sum_i (q_i - v_i)^2 over 16 elements, q = y * r, v = the E2M1 value of q.
__device__ __forceinline__ float approx_err16(const float y[16], float r) {
  const uint64_t rr = pack2(r, r);
  uint64_t acc[2] = {0ull, 0ull};
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint64_t d = e2m1_diff_pair(mul2(pack2(y[2 * k], y[2 * k + 1]), rr));
    acc[k & 1] = fma2(d, d, acc[k & 1]);
  }
  float a0, a1, b0, b1;
  unpack2(acc[0], a0, a1);
  unpack2(acc[1], b0, b1);
  return (a0 + a1) + (b0 + b1);
}

// 0: keep the 6-candidate, 1: take the 4-candidate, 2: too close to call.
__device__ __forceinline__ int certified_pick(float a6, float s6, float a4, float s4,
                                              float margin) {
  const float q6 = s6 * s6, q4 = s4 * s4;
  const float A6 = a6 * q6, A4 = a4 * q4;
  const float B = margin * (q6 + q4);
  if (A4 + B < A6) return 1;
  if (A4 > A6 + B) return 0;
  return 2;
}

// Whether the fast pick applies to this pair of candidate scale codes.
__device__ __forceinline__ bool fast_pick_ok(uint32_t e6, float s6, float s4) {
  return e6 >= 8u && rcp_ok(s6) && rcp_ok(s4);  // e4 >= e6
}

// E2M1 codes of RN(y/s) for 16 elements from r = rcp_approx(s) (s in the
// reciprocal's range), bracketed as in codes16: q*(1 +- 2^-20) becomes
// y * (r*(1 +- 2^-20)), which still lies on the same side of the correctly
// rounded quotient (the reciprocal is off by at most 2^-22, each product
// rounds by 2^-24).  Returns false when a pair is ambiguous (the codes are
// then to be redone exactly).
__device__ __forceinline__ bool codes16_try(const float y[16], float r, uint32_t w[2]) {
  const float ru = r * kUp, rd = r * kDn;
  const uint64_t up = pack2(ru, ru), dn = pack2(rd, rd);
  uint32_t diff = 0u;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float a[8], b[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint64_t yy = pack2(y[8 * h + 2 * k], y[8 * h + 2 * k + 1]);
      unpack2(mul2(yy, up), a[2 * k], a[2 * k + 1]);
      unpack2(mul2(yy, dn), b[2 * k], b[2 * k + 1]);
    }
    w[h] = cvt8_e2m1(a);
    diff |= w[h] ^ cvt8_e2m1(b);
  }
  return diff == 0u;
}

// Scale codes by the bracket only; false when either is ambiguous.
__device__ __forceinline__ bool scale_codes_try(float bmax, const ScaleCtx& c, uint32_t& e6,
                                                uint32_t& e4) {
  if (!c.fast) return false;
  const float t6 = __fmul_rn(bmax, c.c6), t4 = __fmul_rn(bmax, c.c4);
  const uint32_t p6 = f32x2_to_e4m3x2(__fmul_rn(t6, kUp), __fmul_rn(t6, kDn));
  const uint32_t p4 = f32x2_to_e4m3x2(__fmul_rn(t4, kUp), __fmul_rn(t4, kDn));
  e6 = p6 & 0xFFu;
  e4 = p4 & 0xFFu;
  return (p6 >> 8) == e6 && (p4 >> 8) == e4;
}

// Outcome of the fast block encoder.
enum : uint32_t {
  kBlockDone = 0,   // codes and scale final
  kBlockCodes = 1,  // scale final; codes to be redone exactly with it
  kBlockExact = 2,  // the whole block to be redone by quantize_block16
};

// One 16-element block through the fast path: bracketed scale codes, the
// certified 4-vs-6 pick, bracketed codes of the winner.  Every result it
// reports as final equals quantize_block16's; the rest it hands back.
__device__ __forceinline__ uint32_t quantize_block16_try(const float y[16], const ScaleCtx& ctx,
                                                         bool four_over_six, uint32_t& lo,
                                                         uint32_t& hi, uint32_t& scale) {
  uint32_t e6, e4;
  if (!scale_codes_try(absmax16(y), ctx, e6, e4)) return kBlockExact;
  const float s6 = cand_scale(e6, ctx.alpha);
  uint32_t ew = e6;
  float sw = s6;
  if (four_over_six && e4 != e6) {  // equal codes: identical candidates, 6 wins the tie
    const float s4 = cand_scale(e4, ctx.alpha);
    if (!fast_pick_ok(e6, s6, s4)) return kBlockExact;
    const int pick = certified_pick(approx_err16(y, rcp_approx(s6)), s6,
                                    approx_err16(y, rcp_approx(s4)), s4, kPickMargin);
    if (pick == 2) return kBlockExact;
    if (pick == 1) {
      ew = e4;
      sw = s4;
    }
  }
  scale = ew;
  if (sw == 0.0f) {
    lo = hi = 0u;
    return kBlockDone;
  }
  if (!rcp_ok(sw)) return kBlockCodes;
  uint32_t w[2];
  const bool ok = codes16_try(y, rcp_approx(sw), w);
  lo = w[0];
  hi = w[1];
  return ok ? kBlockDone : kBlockCodes;
}

// ----------------------------------------------------------------- packed encoder
// The block encoder above, on a block held as 8 packed fp32 pairs (element 2k
// in the low half of yy[k]) from its first step to its last, so no pair is
// ever re-packed; both candidate scale codes are bracketed and decoded as one
// pair.  Every result it reports as final equals quantize_block16's (same
// arithmetic, same certified bounds); the rest it hands back.

// Raw bf16 words of a block -> packed fp32 pairs (exact).
__device__ __forceinline__ void widen_pairs(const uint32_t w[8], uint64_t yy[8]) {
#pragma unroll
  for (int k = 0; k < 8; ++k)
    yy[k] = pack2(__uint_as_float(w[k] << 16), __uint_as_float(w[k] & 0xFFFF0000u));
}
__device__ __forceinline__ void pairs_of(const float v[16], uint64_t yy[8]) {
#pragma unroll
  for (int k = 0; k < 8; ++k) yy[k] = pack2(v[2 * k], v[2 * k + 1]);
}

// max |y| over the 16 bf16 values of a raw block (an exact selection): per
// half, max.xorsign.abs keeps max(|a|, |b|) as the magnitude.
__device__ __forceinline__ uint32_t maxabs_bf16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ float absmax16_raw(const uint32_t w[8]) {
  const uint32_t a = maxabs_bf16x2(maxabs_bf16x2(w[0], w[1]), maxabs_bf16x2(w[2], w[3]));
  const uint32_t b = maxabs_bf16x2(maxabs_bf16x2(w[4], w[5]), maxabs_bf16x2(w[6], w[7]));
  const uint32_t m = maxabs_bf16x2(a, b) & 0x7FFF7FFFu;
  return fmaxf(__uint_as_float(m << 16), __uint_as_float(m & 0xFFFF0000u));
}
__device__ __forceinline__ float absmax16_pairs(const uint64_t yy[8]) {
  float m = 0.0f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float a, b;
    unpack2(yy[k], a, b);
    m = fmaxf(m, fmaxf(fabsf(a), fabsf(b)));
  }
  return m;
}

// Both candidate scale codes from one bracket pair: t = (t6, t4) =
// bmax * (c6, c4) (the same products as scale_codes_try), bracketed by
// (1 +- 2^-20); false when either code is ambiguous.  *pair: the 6-code in
// bits 0-7, the 4-code in bits 8-15.
__device__ __forceinline__ bool scale_pair_try(float bmax, const ScaleCtx& c, uint32_t& pair) {
  if (!c.fast) return false;
  const uint64_t t = mul2(pack2(bmax, bmax), pack2(c.c6, c.c4));
  float t6u, t4u, t6d, t4d;
  unpack2(mul2(t, pack2(kUp, kUp)), t6u, t4u);
  unpack2(mul2(t, pack2(kDn, kDn)), t6d, t4d);
  const uint32_t pu = f32x2_to_e4m3x2(t4u, t6u), pd = f32x2_to_e4m3x2(t4d, t6d);
  pair = pu & 0xFFFFu;
  return (pu & 0xFFFFu) == (pd & 0xFFFFu);
}

// (s6, s4) = (dec(e6) * alpha, dec(e4) * alpha) for a code pair as above.
__device__ __forceinline__ uint64_t scale_pair_values(uint32_t pair, float alpha) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)pair));
  const float d6 = __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
  const float d4 = __half2float(__ushort_as_half((unsigned short)(h2 >> 16)));
  return mul2(pack2(d6, d4), pack2(alpha, alpha));
}

// approx_err16 on packed pairs.
__device__ __forceinline__ float approx_err16_pairs(const uint64_t yy[8], float r) {
  const uint64_t rr = pack2(r, r);
  uint64_t acc[2] = {0ull, 0ull};
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint64_t d = e2m1_diff_pair(mul2(yy[k], rr));
    acc[k & 1] = fma2(d, d, acc[k & 1]);
  }
  float a0, a1;
  unpack2(add2(acc[0], acc[1]), a0, a1);
  return a0 + a1;
}

// codes16_try on packed pairs.
__device__ __forceinline__ bool codes16_try_pairs(const uint64_t yy[8], float r, uint32_t w[2]) {
  const float ru = r * kUp, rd = r * kDn;
  const uint64_t up = pack2(ru, ru), dn = pack2(rd, rd);
  uint32_t diff = 0u;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float a[8], b[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      unpack2(mul2(yy[4 * h + k], up), a[2 * k], a[2 * k + 1]);
      unpack2(mul2(yy[4 * h + k], dn), b[2 * k], b[2 * k + 1]);
    }
    w[h] = cvt8_e2m1(a);
    diff |= w[h] ^ cvt8_e2m1(b);
  }
  return diff == 0u;
}

// quantize_block16_try on packed pairs with the block max given.
__device__ __forceinline__ uint32_t quantize_block16_pairs(const uint64_t yy[8], float bmax,
                                                           const ScaleCtx& ctx, bool four_over_six,
                                                           uint32_t& lo, uint32_t& hi,
                                                           uint32_t& scale) {
  uint32_t pair;
  if (!scale_pair_try(bmax, ctx, pair)) return kBlockExact;
  const uint32_t e6 = pair & 0xFFu, e4 = pair >> 8;
  float s6, s4;
  unpack2(scale_pair_values(pair, ctx.alpha), s6, s4);
  uint32_t ew = e6;
  float sw = s6;
  if (four_over_six && e4 != e6) {  // equal codes: identical candidates, 6 wins the tie
    if (!fast_pick_ok(e6, s6, s4)) return kBlockExact;
    const int pick = certified_pick(approx_err16_pairs(yy, rcp_approx(s6)), s6,
                                    approx_err16_pairs(yy, rcp_approx(s4)), s4, kPickMargin);
    if (pick == 2) return kBlockExact;
    if (pick == 1) {
      ew = e4;
      sw = s4;
    }
  }
  scale = ew;
  if (sw == 0.0f) {
    lo = hi = 0u;
    return kBlockDone;
  }
  if (!rcp_ok(sw)) return kBlockCodes;
  uint32_t w[2];
  const bool ok = codes16_try_pairs(yy, rcp_approx(sw), w);
  lo = w[0];
  hi = w[1];
  return ok ? kBlockDone : kBlockCodes;
}

// Byte offset of scale (r, kb) in the chosen layout.
// Every tensor the library encodes has fewer than 2^32 blocks (the entry
// points check), so rows, block columns and the 512-byte atom index all fit in
// 32 bits; only the final byte offset is widened.
__device__ __forceinline__ int64_t sf_offset(int64_t r, int64_t kb, int64_t kb_total, int layout) {
  const uint32_t r32 = (uint32_t)r, kb32 = (uint32_t)kb, kt = (uint32_t)kb_total;
  if (layout == 0) return (int64_t)((uint64_t)r32 * kt + kb32);
  const uint32_t groups = (kt + 3) >> 2;
  return (int64_t)(((uint64_t)((r32 >> 7) * groups + (kb32 >> 2)) << 9) +
                   (((r32 & 31) << 4) | (((r32 >> 5) & 3) << 2) | (kb32 & 3)));
}

// Atomic max of a non-negative float stored as its bit pattern.
__device__ __forceinline__ void atomic_max_nonneg(uint32_t* slot, float v) {
  atomicMax(slot, __float_as_uint(v));
}

}  // namespace nvfp4
