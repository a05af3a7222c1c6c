// sm_100a NVFP4 quantizers, dequantizer and standalone RHT16.
//
// Current scaling needs the whole-tensor amax before the first element can be
// encoded, so a quantization is two HBM passes: an amax pass (1) and an
// encode pass (2).  Both passes are grid-stride, one 16-element block per
// thread per step, 256-bit coalesced loads; the encode pass writes 8 bytes
// of codes per block and one scale byte in the requested layout.  Batched
// calls (KV cache) carry up to kMaxBatch tensors in the kernel parameters,
// one tensor per blockIdx.y, so one launch covers a whole cache per pass.
#include "device_common.cuh"
#include "kernels.h"

namespace nvfp4 {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float block_reduce_max(float v) {
  __shared__ float red[kThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) red[w] = v;
  __syncthreads();
  if (w == 0) {
    v = (l < kThreads / 32) ? red[l] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  }
  return v;
}

__device__ __forceinline__ float tensor_alpha(const QBatch& p, int t) {
  return p.gs_in ? *p.gs_in : alpha_from_amax(__uint_as_float(p.amax_slots[t]));
}

// ------------------------------------------------------------------------
// Pass 1: amax.  Blocks along the contiguous dim (block_axis 0).
template <typename T, bool RHT>
__global__ void __launch_bounds__(kThreads) amax_rows_kernel(const __grid_constant__ QBatch p) {
  const QTensor& q = p.t[blockIdx.y];
  const T* x = static_cast<const T*>(q.x);
  const uint32_t kbpr = (uint32_t)(q.cols >> 4);
  const uint64_t nblk = (uint64_t)q.rows * kbpr;
  float m = 0.0f;
  for (uint64_t u = (uint64_t)blockIdx.x * kThreads + threadIdx.x; u < nblk;
       u += (uint64_t)gridDim.x * kThreads) {
    const uint32_t r = (uint32_t)u / kbpr, kb = (uint32_t)u - r * kbpr;
    float v[16];
    load16(x + (int64_t)r * q.ld + (int64_t)kb * 16, v);
    if (RHT) rht16(v, p.mask);
    m = fmaxf(m, absmax16(v));
  }
  m = block_reduce_max(m);
  if (threadIdx.x == 0) atomic_max_nonneg(&p.amax_slots[blockIdx.y], m);
}

// Pass 1 for blocks along rows (block_axis 1): unit = (column pair, 64 rows).
template <typename T, bool RHT>
__global__ void __launch_bounds__(kThreads) amax_cols_kernel(const __grid_constant__ QBatch p) {
  const QTensor& q = p.t[blockIdx.y];
  const T* x = static_cast<const T*>(q.x);
  const uint32_t ncp = (uint32_t)((q.cols + 1) >> 1);
  const uint32_t nrc = (uint32_t)((q.rows + 63) >> 6);
  const uint64_t nunits = (uint64_t)ncp * nrc;
  float m = 0.0f;
  for (uint64_t u = (uint64_t)blockIdx.x * kThreads + threadIdx.x; u < nunits;
       u += (uint64_t)gridDim.x * kThreads) {
    const uint32_t rc = (uint32_t)u / ncp, cp = (uint32_t)u - rc * ncp;
    const int64_t c0 = 2 * (int64_t)cp;
#pragma unroll 1
    for (int g = 0; g < 4; ++g) {
      const int64_t rg = 64 * (int64_t)rc + 16 * g;
      if (rg >= q.rows) break;
      float a[16], b[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) load2(x + (rg + j) * q.ld + c0, a[j], b[j]);
      if (RHT) {
        rht16(a, p.mask);
        rht16(b, p.mask);
      }
      m = fmaxf(m, absmax16(a));
      m = fmaxf(m, absmax16(b));
    }
  }
  m = block_reduce_max(m);
  if (threadIdx.x == 0) atomic_max_nonneg(&p.amax_slots[blockIdx.y], m);
}

// Zero the padding entries of a tcgen05-layout scale buffer.
__device__ void zero_sf_padding(uint8_t* sf, int64_t rows, int64_t kbpr) {
  const int64_t rows_pad = (rows + 127) & ~int64_t(127);
  const int64_t kb_pad = (kbpr + 3) & ~int64_t(3);
  const int64_t tid = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  const int64_t step = (int64_t)gridDim.x * kThreads;
  const int64_t n1 = (rows_pad - rows) * kb_pad;  // whole padding rows
  for (int64_t i = tid; i < n1; i += step) {
    const int64_t r = rows + i / kb_pad, kb = i % kb_pad;
    sf[sf_offset(r, kb, kbpr, 1)] = 0;
  }
  const int64_t extra = kb_pad - kbpr;  // padding blocks of real rows
  const int64_t n2 = rows * extra;
  for (int64_t i = tid; i < n2; i += step) {
    const int64_t r = i / extra, kb = kbpr + i % extra;
    sf[sf_offset(r, kb, kbpr, 1)] = 0;
  }
}

// ------------------------------------------------------------------------
// Pass 2: encode, blocks along the contiguous dim.
template <typename T, bool RHT>
__global__ void __launch_bounds__(kThreads) quant_rows_kernel(const __grid_constant__ QBatch p) {
  const int t = blockIdx.y;
  const QTensor& q = p.t[t];
  const T* x = static_cast<const T*>(q.x);
  const float alpha = tensor_alpha(p, t);
  if (blockIdx.x == 0 && threadIdx.x == 0 && q.gs_out) *q.gs_out = alpha;
  const uint32_t kbpr = (uint32_t)(q.cols >> 4);
  const uint64_t nblk = (uint64_t)q.rows * kbpr;
  const bool fos = p.four_over_six != 0;
  for (uint64_t u = (uint64_t)blockIdx.x * kThreads + threadIdx.x; u < nblk;
       u += (uint64_t)gridDim.x * kThreads) {
    const uint32_t r = (uint32_t)u / kbpr, kb = (uint32_t)u - r * kbpr;
    float v[16];
    load16(x + (int64_t)r * q.ld + (int64_t)kb * 16, v);
    if (RHT) rht16(v, p.mask);
    uint32_t lo, hi, sc;
    quantize_block16(v, alpha, fos, lo, hi, sc);
    *reinterpret_cast<uint2*>(q.codes + (int64_t)r * (q.cols >> 1) + (int64_t)kb * 8) =
        make_uint2(lo, hi);
    q.scales[sf_offset(r, kb, kbpr, p.sf_layout)] = (uint8_t)sc;
  }
  if (p.sf_layout == 1) zero_sf_padding(q.scales, q.rows, kbpr);
}

// Pass 2, blocks along rows; output transposed: codes [cols, rows/2],
// scales for cols rows x rows/16 blocks.
template <typename T, bool RHT>
__global__ void __launch_bounds__(kThreads) quant_cols_kernel(const __grid_constant__ QBatch p) {
  const int t = blockIdx.y;
  const QTensor& q = p.t[t];
  const T* x = static_cast<const T*>(q.x);
  const float alpha = tensor_alpha(p, t);
  if (blockIdx.x == 0 && threadIdx.x == 0 && q.gs_out) *q.gs_out = alpha;
  const uint32_t ncp = (uint32_t)((q.cols + 1) >> 1);
  const uint32_t nrc = (uint32_t)((q.rows + 63) >> 6);
  const uint64_t nunits = (uint64_t)ncp * nrc;
  const int64_t out_row_bytes = q.rows >> 1;
  const int64_t kb_total = q.rows >> 4;
  const bool fos = p.four_over_six != 0;
  for (uint64_t u = (uint64_t)blockIdx.x * kThreads + threadIdx.x; u < nunits;
       u += (uint64_t)gridDim.x * kThreads) {
    const uint32_t rc = (uint32_t)u / ncp, cp = (uint32_t)u - rc * ncp;
    const int64_t c0 = 2 * (int64_t)cp;
#pragma unroll 1
    for (int g = 0; g < 4; ++g) {
      const int64_t rg = 64 * (int64_t)rc + 16 * g;
      if (rg >= q.rows) break;
      float a[16], b[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) load2(x + (rg + j) * q.ld + c0, a[j], b[j]);
      if (RHT) {
        rht16(a, p.mask);
        rht16(b, p.mask);
      }
      uint32_t lo, hi, sc;
      quantize_block16(a, alpha, fos, lo, hi, sc);
      *reinterpret_cast<uint2*>(q.codes + c0 * out_row_bytes + (rg >> 1)) = make_uint2(lo, hi);
      q.scales[sf_offset(c0, rg >> 4, kb_total, p.sf_layout)] = (uint8_t)sc;
      quantize_block16(b, alpha, fos, lo, hi, sc);
      *reinterpret_cast<uint2*>(q.codes + (c0 + 1) * out_row_bytes + (rg >> 1)) =
          make_uint2(lo, hi);
      q.scales[sf_offset(c0 + 1, rg >> 4, kb_total, p.sf_layout)] = (uint8_t)sc;
    }
  }
  if (p.sf_layout == 1) zero_sf_padding(q.scales, q.cols, kb_total);
}

// ------------------------------------------------------------------------
// 2D 16x16 tiles.  A warp holds two adjacent tiles of one 16-row band: lane l
// owns row (l & 15) of tile (l >> 4).  Tile max and tile error reduce across
// the 16 lanes of a half-warp with xor shuffles 8, 4, 2, 1 -- the same
// pairwise order as the per-row sum.
template <typename T>
__global__ void __launch_bounds__(kThreads) quant_2d_kernel(const __grid_constant__ QBatch p) {
  const QTensor& q = p.t[0];
  const T* x = static_cast<const T*>(q.x);
  const float alpha = tensor_alpha(p, 0);
  if (blockIdx.x == 0 && threadIdx.x == 0 && q.gs_out) *q.gs_out = alpha;
  const uint32_t kbpr = (uint32_t)(q.cols >> 4);
  const uint32_t npair = (kbpr + 1) >> 1;
  const uint32_t nunits = (uint32_t)(q.rows >> 4) * npair;
  const int lane = threadIdx.x & 31;
  const uint32_t warps = kThreads / 32;
  const bool fos = p.four_over_six != 0;
  for (uint32_t u = blockIdx.x * warps + (threadIdx.x >> 5); u < nunits; u += gridDim.x * warps) {
    const uint32_t tr = u / npair, tp = u - tr * npair;
    const int64_t r = (int64_t)tr * 16 + (lane & 15);
    const uint32_t kb = tp * 2 + (lane >> 4);
    const bool valid = kb < kbpr;
    float v[16];
    if (valid) {
      load16(x + r * q.ld + (int64_t)kb * 16, v);
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = 0.0f;
    }
    float tmax = absmax16(v);
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xFFFFFFFFu, tmax, o));
    const float uu = __fdiv_rn(tmax, alpha);
    uint32_t e6;
    const float s6 = cand_scale(uu, 6.0f, alpha, e6);
    Cand c6 = encode16(v, s6);
    float err6 = c6.err;
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) err6 = __fadd_rn(err6, __shfl_xor_sync(0xFFFFFFFFu, err6, o));
    uint32_t lo = c6.lo, hi = c6.hi, sc = e6;
    if (fos) {
      uint32_t e4;
      const float s4 = cand_scale(uu, 4.0f, alpha, e4);
      Cand c4 = encode16(v, s4);
      float err4 = c4.err;
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) err4 = __fadd_rn(err4, __shfl_xor_sync(0xFFFFFFFFu, err4, o));
      if (err4 < err6) {
        lo = c4.lo;
        hi = c4.hi;
        sc = e4;
      }
    }
    if (valid) {
      *reinterpret_cast<uint2*>(q.codes + r * (q.cols >> 1) + (int64_t)kb * 8) = make_uint2(lo, hi);
      q.scales[sf_offset(r, kb, kbpr, p.sf_layout)] = (uint8_t)sc;
    }
  }
  if (p.sf_layout == 1) zero_sf_padding(q.scales, q.rows, kbpr);
}

// ------------------------------------------------------------------------
// Dequantization, one 16-block per thread step, all tensors of a batch in
// one launch (tensor = blockIdx.y).
template <bool BF16>
__global__ void __launch_bounds__(kThreads) dequant_kernel(const __grid_constant__ DQBatch p) {
  const DQTensor& q = p.t[blockIdx.y];
  const float alpha = *q.gs;
  const uint64_t aa = pack2(alpha, alpha);
  const uint32_t kbpr = (uint32_t)(q.cols >> 4);
  const uint64_t nblk = (uint64_t)q.rows * kbpr;
  for (uint64_t u = (uint64_t)blockIdx.x * kThreads + threadIdx.x; u < nblk;
       u += (uint64_t)gridDim.x * kThreads) {
    const uint32_t r = (uint32_t)u / kbpr, kb = (uint32_t)u - r * kbpr;
    const uint2 c = __ldg(reinterpret_cast<const uint2*>(q.codes + (int64_t)r * (q.cols >> 1) +
                                                         (int64_t)kb * 8));
    const float d = e4m3_to_f32(__ldg(q.scales + sf_offset(r, kb, kbpr, p.sf_layout)));
    const uint64_t dd = pack2(d, d);
    float o[16];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint32_t byte = ((k < 4 ? c.x : c.y) >> (8 * (k & 3))) & 0xFFu;
      const uint64_t vd = mul2(e2m1x2_to_f32x2(byte), dd);  // exact
      unpack2(mul2(vd, aa), o[2 * k], o[2 * k + 1]);
    }
    if (BF16) {
      uint32_t w[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        __nv_bfloat162 h = __floats2bfloat162_rn(o[2 * k], o[2 * k + 1]);
        w[k] = *reinterpret_cast<uint32_t*>(&h);
      }
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(q.out) + (int64_t)r * q.ldo + (int64_t)kb * 16;
      asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(dst), "r"(w[0]),
                   "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                   : "memory");
    } else {
      float* dst = static_cast<float*>(q.out) + (int64_t)r * q.ldo + (int64_t)kb * 16;
#pragma unroll
      for (int h = 0; h < 2; ++h)
        asm volatile("st.global.v8.f32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(dst + 8 * h),
                     "f"(o[8 * h]), "f"(o[8 * h + 1]), "f"(o[8 * h + 2]), "f"(o[8 * h + 3]),
                     "f"(o[8 * h + 4]), "f"(o[8 * h + 5]), "f"(o[8 * h + 6]), "f"(o[8 * h + 7])
                     : "memory");
    }
  }
}

// ------------------------------------------------------------------------
// Standalone RHT16 (parity tool for the fused transform): fp32 output.
template <typename T>
__global__ void __launch_bounds__(kThreads)
    rht_kernel(const T* x, int64_t rows, int64_t cols, int64_t ld, int block_axis, uint32_t mask,
               float* out) {
  const uint64_t n = block_axis == 0 ? (uint64_t)rows * (cols >> 4) : (uint64_t)(rows >> 4) * cols;
  for (uint64_t u = (uint64_t)blockIdx.x * kThreads + threadIdx.x; u < n;
       u += (uint64_t)gridDim.x * kThreads) {
    float v[16];
    if (block_axis == 0) {
      const int64_t r = (int64_t)(u / (uint64_t)(cols >> 4)), c = (int64_t)(u % (uint64_t)(cols >> 4)) * 16;
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = load1(x + r * ld + c + j);
      rht16(v, mask);
#pragma unroll
      for (int j = 0; j < 16; ++j) out[r * cols + c + j] = v[j];
    } else {
      const int64_t rg = (int64_t)(u / (uint64_t)cols) * 16, c = (int64_t)(u % (uint64_t)cols);
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = load1(x + (rg + j) * ld + c);
      rht16(v, mask);
#pragma unroll
      for (int j = 0; j < 16; ++j) out[(rg + j) * cols + c] = v[j];
    }
  }
}

__global__ void finalize_alpha_kernel(const uint32_t* slot, float* gs_out) {
  *gs_out = alpha_from_amax(__uint_as_float(*slot));
}

int grid_for(uint64_t work_items, int n_tensors) {
  const uint64_t want = (work_items + kThreads - 1) / kThreads;
  const uint64_t cap = (uint64_t)num_sms() * 8 / (uint64_t)(n_tensors > 0 ? n_tensors : 1);
  uint64_t g = want < cap ? want : cap;
  return (int)(g < 1 ? 1 : g);
}

uint64_t max_units(const QBatch& b, bool cols_units) {
  uint64_t m = 0;
  for (int i = 0; i < b.n; ++i) {
    const QTensor& q = b.t[i];
    const uint64_t u = cols_units ? (uint64_t)((q.cols + 1) / 2) * (uint64_t)((q.rows + 63) / 64)
                                  : (uint64_t)q.rows * (uint64_t)(q.cols / 16);
    m = u > m ? u : m;
  }
  return m;
}

}  // namespace

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
  }
  return n;
}

cudaError_t launch_amax(const QBatch& b, cudaStream_t s) {
  const bool cols = b.block_axis == 1;
  dim3 grid(grid_for(max_units(b, cols), b.n), b.n);
#define NVFP4_AMAX(T, R)                                                            \
  (cols ? amax_cols_kernel<T, R><<<grid, kThreads, 0, s>>>(b)                        \
        : amax_rows_kernel<T, R><<<grid, kThreads, 0, s>>>(b))
  if (b.bf16) {
    if (b.rht) NVFP4_AMAX(__nv_bfloat16, true); else NVFP4_AMAX(__nv_bfloat16, false);
  } else {
    if (b.rht) NVFP4_AMAX(float, true); else NVFP4_AMAX(float, false);
  }
#undef NVFP4_AMAX
  return cudaGetLastError();
}

cudaError_t launch_quantize_1d(const QBatch& b, cudaStream_t s) {
  const bool cols = b.block_axis == 1;
  dim3 grid(grid_for(max_units(b, cols), b.n), b.n);
#define NVFP4_Q1(T, R)                                                              \
  (cols ? quant_cols_kernel<T, R><<<grid, kThreads, 0, s>>>(b)                       \
        : quant_rows_kernel<T, R><<<grid, kThreads, 0, s>>>(b))
  if (b.bf16) {
    if (b.rht) NVFP4_Q1(__nv_bfloat16, true); else NVFP4_Q1(__nv_bfloat16, false);
  } else {
    if (b.rht) NVFP4_Q1(float, true); else NVFP4_Q1(float, false);
  }
#undef NVFP4_Q1
  return cudaGetLastError();
}

cudaError_t launch_quantize_2d(const QBatch& b, cudaStream_t s) {
  const QTensor& q = b.t[0];
  const uint64_t units = (uint64_t)(q.rows / 16) * (uint64_t)((q.cols / 16 + 1) / 2);
  // one warp per unit: 8 units per CTA
  uint64_t want = (units + 7) / 8, cap = (uint64_t)num_sms() * 8;
  int grid = (int)(want < cap ? (want < 1 ? 1 : want) : cap);
  if (b.bf16)
    quant_2d_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(b);
  else
    quant_2d_kernel<float><<<grid, kThreads, 0, s>>>(b);
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const DQBatch& b, cudaStream_t s) {
  uint64_t m = 0;
  for (int i = 0; i < b.n; ++i) {
    const uint64_t u = (uint64_t)b.t[i].rows * (uint64_t)(b.t[i].cols / 16);
    m = u > m ? u : m;
  }
  dim3 grid(grid_for(m, b.n), b.n);
  if (b.out_bf16)
    dequant_kernel<true><<<grid, kThreads, 0, s>>>(b);
  else
    dequant_kernel<false><<<grid, kThreads, 0, s>>>(b);
  return cudaGetLastError();
}

cudaError_t launch_rht16(const void* x, int bf16, int64_t rows, int64_t cols, int64_t ld,
                         int block_axis, uint32_t mask, float* out, cudaStream_t s) {
  const uint64_t n = (uint64_t)rows * (uint64_t)cols / 16;
  const int grid = grid_for(n, 1);
  if (bf16)
    rht_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(static_cast<const __nv_bfloat16*>(x), rows,
                                                        cols, ld, block_axis, mask, out);
  else
    rht_kernel<float><<<grid, kThreads, 0, s>>>(static_cast<const float*>(x), rows, cols, ld,
                                                block_axis, mask, out);
  return cudaGetLastError();
}

cudaError_t launch_finalize_alpha(const uint32_t* amax_slot, float* gs_out, cudaStream_t s) {
  finalize_alpha_kernel<<<1, 1, 0, s>>>(amax_slot, gs_out);
  return cudaGetLastError();
}

}  // namespace nvfp4
