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
// RN), then the exact scaling by 1/4.
__device__ __forceinline__ void rht16(float v[16], uint32_t mask) {
#pragma unroll
  for (int j = 0; j < 16; ++j)
    v[j] = __uint_as_float(__float_as_uint(v[j]) ^ (((mask >> j) & 1u) << 31));
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (i & h) continue;
      float a = v[i], b = v[i + h];
      v[i] = __fadd_rn(a, b);
      v[i + h] = __fsub_rn(a, b);
    }
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = __fmul_rn(v[j], 0.25f);
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

// One candidate encoding of a 16-element row segment under scale s > 0:
// codes (8 bytes, element 2j in the low nibble of byte j) and the row's
// squared error.  s == 0 encodes all +0 with error sum(y^2).
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
    for (int k = 0; k < 8; ++k) sq[k] = pack2(__fmul_rn(y[2 * k], y[2 * k]), __fmul_rn(y[2 * k + 1], y[2 * k + 1]));
  } else {
    uint32_t bytes[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float q0 = __fdiv_rn(y[2 * k], s);
      float q1 = __fdiv_rn(y[2 * k + 1], s);
      bytes[k] = f32x2_to_e2m1x2(q0, q1);
      float v0, v1;
      unpack2(e2m1x2_to_f32x2(bytes[k]), v0, v1);
      // Scalar intrinsics: documented never to be merged into a fused
      // multiply-add (the packed f32x2 forms are contracted by the
      // assembler, which would change y - v*s in its last bit).
      const float r0 = __fsub_rn(y[2 * k], __fmul_rn(v0, s));
      const float r1 = __fsub_rn(y[2 * k + 1], __fmul_rn(v1, s));
      sq[k] = pack2(__fmul_rn(r0, r0), __fmul_rn(r1, r1));
    }
    c.lo = bytes[0] | (bytes[1] << 8) | (bytes[2] << 16) | (bytes[3] << 24);
    c.hi = bytes[4] | (bytes[5] << 8) | (bytes[6] << 16) | (bytes[7] << 24);
  }
  c.err = tree16(sq);
  return c;
}

// Scale of one candidate: t = (bmax / alpha) / M, e = E4M3(t), s = dec(e) * alpha.
__device__ __forceinline__ float cand_scale(float u, float M, float alpha, uint32_t& e) {
  float t = __fdiv_rn(u, M);
  e = f32_to_e4m3(t);
  return __fmul_rn(e4m3_to_f32(e), alpha);
}

// Full 1D block encoding with the optional 4-vs-6 pick (ties keep 6).
__device__ __forceinline__ void quantize_block16(const float y[16], float alpha, bool four_over_six,
                                                 uint32_t& lo, uint32_t& hi, uint32_t& scale) {
  const float u = __fdiv_rn(absmax16(y), alpha);
  uint32_t e6;
  const float s6 = cand_scale(u, 6.0f, alpha, e6);
  Cand c6 = encode16(y, s6);
  lo = c6.lo;
  hi = c6.hi;
  scale = e6;
  if (four_over_six) {
    uint32_t e4;
    const float s4 = cand_scale(u, 4.0f, alpha, e4);
    Cand c4 = encode16(y, s4);
    if (c4.err < c6.err) {
      lo = c4.lo;
      hi = c4.hi;
      scale = e4;
    }
  }
}

// Byte offset of scale (r, kb) in the chosen layout.
__device__ __forceinline__ int64_t sf_offset(int64_t r, int64_t kb, int64_t kb_total, int layout) {
  if (layout == 0) return r * kb_total + kb;
  const int64_t kb_groups = (kb_total + 3) >> 2;
  return (((r >> 7) * kb_groups + (kb >> 2)) << 9) + ((r & 31) << 4) + (((r >> 5) & 3) << 2) +
         (kb & 3);
}

// Atomic max of a non-negative float stored as its bit pattern.
__device__ __forceinline__ void atomic_max_nonneg(uint32_t* slot, float v) {
  atomicMax(slot, __float_as_uint(v));
}

}  // namespace nvfp4
