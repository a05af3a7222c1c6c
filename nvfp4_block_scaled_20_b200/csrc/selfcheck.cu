// Conformance sweep of the hardware conversions the encoders rely on.
//
// The quantizers take every rounding decision with the sm_100a conversion
// instructions cvt.rn.satfinite.e2m1x2.f32 (element codes) and
// cvt.rn.satfinite.e4m3x2.f32 (scale codes); their bracketing arguments
// (codes of q (1 +- 2^-20) that agree are the code of the exact quotient)
// assume both are round-to-nearest-even, saturating conversions everywhere.
// This kernel converts a range of fp32 bit patterns with exactly the
// helpers the encoders call, so a test can compare every input of a range
// with the format's definition.
#include "device_common.cuh"
#include "kernels.h"

namespace nvfp4 {

namespace {

constexpr int kSweepThreads = 256;

// Thread step: 16 consecutive bit patterns, one 16-byte store.
__global__ void __launch_bounds__(kSweepThreads)
    convert_sweep_kernel(int target, uint32_t first, uint64_t count, uint8_t* out) {
  const uint64_t groups = count / 16;
  for (uint64_t g = (uint64_t)blockIdx.x * kSweepThreads + threadIdx.x; g < groups;
       g += (uint64_t)gridDim.x * kSweepThreads) {
    const uint32_t b0 = first + (uint32_t)(g * 16);
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t word = 0u;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float lo = __uint_as_float(b0 + 4 * k + 2 * j);
        const float hi = __uint_as_float(b0 + 4 * k + 2 * j + 1);
        uint32_t pair;  // byte of lo | byte of hi << 8
        if (target == 0) {
          const uint32_t c = f32x2_to_e2m1x2(lo, hi);  // lo code in bits 0-3
          pair = (c & 0xFu) | ((c >> 4) & 0xFu) << 8;
        } else {
          const uint32_t c = f32x2_to_e4m3x2(hi, lo);  // first operand in bits 8-15
          pair = c & 0xFFFFu;
        }
        word |= pair << (16 * j);
      }
      w[k] = word;
    }
    *reinterpret_cast<uint4*>(out + g * 16) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  // the ragged tail (count % 16 patterns), one thread
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    for (uint64_t i = groups * 16; i < count; ++i) {
      const float v = __uint_as_float(first + (uint32_t)i);
      out[i] = (uint8_t)(target == 0 ? (f32x2_to_e2m1x2(v, 0.0f) & 0xFu)
                                     : (f32x2_to_e4m3x2(0.0f, v) & 0xFFu));
    }
  }
}

}  // namespace

cudaError_t launch_convert_sweep(int target, uint32_t first, uint64_t count, uint8_t* out,
                                 cudaStream_t s) {
  const uint64_t groups = (count + 15) / 16;
  uint64_t grid = (groups + kSweepThreads - 1) / kSweepThreads;
  const uint64_t cap = (uint64_t)num_sms() * 8;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  convert_sweep_kernel<<<(unsigned)grid, kSweepThreads, 0, s>>>(target, first, count, out);
  return cudaGetLastError();
}

}  // namespace nvfp4
