// sm_100a NVFP4 quantizers, dequantizer and standalone RHT16.
//
// Current scaling needs the whole-tensor amax before the first element can be
// encoded, so a quantization is two passes, two kernels on one stream:
//   amax:   grid-stride over the tensor (256-bit coalesced loads, several in
//           flight per thread), one partial maximum per CTA written to its own
//           workspace slot -- no atomics, nothing to clear between calls;
//   encode: launched as a programmatic dependent of the amax kernel, so its
//           launch overlaps the amax pass; it waits for the amax grid,
//           reduces the partials into the global scale and encodes one
//           16-element block per thread step (both 4-vs-6 candidates, 8 bytes
//           of codes and one scale byte in the requested layout).
// A tensor that fits in L2 is read from HBM once: the encode pass finds it in
// L2.  Batched calls (KV cache) carry up to kMaxBatch tensors in the kernel
// parameters, one tensor per blockIdx.y.
#include <cuda.h>

#include <type_traits>

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
  __syncthreads();  // red[] may be reused by the next call
  return v;
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// n / d for 32-bit n by a multiply-high (d fixed per tensor; d >= 1): with
// l = ceil(log2 d) and m = floor(2^32 (2^l - d) / d) + 1, n / d equals
// (mulhi(n, m) + n) >> l for every 32-bit n.
struct FastDiv {
  uint32_t m, l;
};
__device__ __forceinline__ FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  f.l = d > 1u ? 32u - __clz(d - 1u) : 0u;
  f.m = (uint32_t)(((((uint64_t)1 << f.l) - d) << 32) / d + 1u);
  return f;
}
__device__ __forceinline__ uint32_t fastdiv(uint32_t n, FastDiv f) {
  return (uint32_t)(((uint64_t)__umulhi(n, f.m) + n) >> f.l);
}

// Global scale of tensor t from the amax kernel's partials (ga of them);
// call after pdl_wait().  Every thread of the CTA gets the value.
__device__ float reduce_partials(const float* part, int ga) {
  float m = 0.0f;
  for (int i = threadIdx.x; i < ga; i += kThreads) m = fmaxf(m, part[i]);
  m = block_reduce_max(m);
  __shared__ float s_m;
  if (threadIdx.x == 0) s_m = m;
  __syncthreads();
  return s_m;
}

// The CTAs of a launch that work on one tensor: cta-th of ncta.  A launch
// over one tensor (or one tensor per blockIdx.y) uses (blockIdx.x,
// gridDim.x); a mixed launch gives each tensor a range of blockIdx.x.
struct Slice {
  uint32_t cta, ncta;
};

// ------------------------------------------------------------------------
// Amax pass.

// bf16 without the transform: the max stays on packed raw words; kAmaxDepth
// 32-byte loads in flight per thread (enough bytes in flight per SM to cover
// the HBM latency at three CTAs per SM; the load form itself was measured not
// to matter: non-coherent, plain, evict-first and bulk copies stream alike).
constexpr int kAmaxDepth = 8;
// Address of 16-block u of a row-major tensor: contiguous rows (ld == cols)
// need no division; otherwise the row comes from a multiply-high division.
template <typename T>
__device__ __forceinline__ const T* block_ptr(const T* x, uint64_t u, bool contig, uint32_t kbpr,
                                              FastDiv div, int64_t ld) {
  if (contig) return x + u * 16;
  const uint32_t r = fastdiv((uint32_t)u, div);
  return x + (int64_t)r * ld + (int64_t)((uint32_t)u - r * kbpr) * 16;
}

__device__ float amax_rows_bf16_raw(const QTensor& q, const Slice sl) {
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(q.x);
  const uint32_t kbpr = (uint32_t)(q.cols >> 4);
  const uint64_t nblk = (uint64_t)q.rows * kbpr;
  const bool contig = q.ld == q.cols;
  const FastDiv div = make_fastdiv(kbpr);
  const uint64_t stride = (uint64_t)sl.ncta * kThreads;
  uint32_t m2 = 0u;
  for (uint64_t u = (uint64_t)sl.cta * kThreads + threadIdx.x; u < nblk; u += kAmaxDepth * stride) {
    uint32_t w[kAmaxDepth][8];
#pragma unroll
    for (int j = 0; j < kAmaxDepth; ++j) {
      const uint64_t uj = u + j * stride;
      if (uj < nblk) {
        load16_raw(block_ptr(x, uj, contig, kbpr, div, q.ld), w[j]);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) w[j][i] = 0u;
      }
    }
#pragma unroll
    for (int j = 0; j < kAmaxDepth; ++j)
#pragma unroll
      for (int i = 0; i < 8; ++i) m2 = absmax_bf16x2(m2, w[j][i]);
  }
  return fmaxf(__uint_as_float(m2 << 16), __uint_as_float(m2 & 0xFFFF0000u));
}

template <typename T, bool RHT>
__device__ float amax_rows(const QTensor& q, uint32_t mask, const Slice sl) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value && !RHT) return amax_rows_bf16_raw(q, sl);
  const T* x = static_cast<const T*>(q.x);
  const uint32_t kbpr = (uint32_t)(q.cols >> 4);
  const uint64_t nblk = (uint64_t)q.rows * kbpr;
  const bool contig = q.ld == q.cols;
  const FastDiv div = make_fastdiv(kbpr);
  const uint64_t stride = (uint64_t)sl.ncta * kThreads;
  float m = 0.0f;
  // two blocks per thread per trip, both loads issued before any use
  for (uint64_t u = (uint64_t)sl.cta * kThreads + threadIdx.x; u < nblk; u += 2 * stride) {
    float v[2][16];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint64_t uj = u + j * stride;
      if (uj < nblk) {
        load16(block_ptr(x, uj, contig, kbpr, div, q.ld), v[j]);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[j][i] = 0.0f;
      }
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      if (RHT) rht16(v[j], mask);
      m = fmaxf(m, absmax16(v[j]));
    }
  }
  return m;
}

// 16 rows x one column pair (element pairs: the row-axis mode needs no more
// than 4-byte row alignment), as loaded; widened to two fp32 columns.
template <typename T> struct RawPair;
template <> struct RawPair<__nv_bfloat16> {
  uint32_t w[16];
  __device__ __forceinline__ void load(const __nv_bfloat16* p, int64_t ld) {
#pragma unroll
    for (int j = 0; j < 16; ++j)
      asm volatile("ld.global.nc.b32 %0, [%1];" : "=r"(w[j]) : "l"(p + j * ld));
  }
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int j = 0; j < 16; ++j) w[j] = 0u;
  }
  __device__ __forceinline__ void widen(float a[16], float b[16]) const {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      a[j] = __uint_as_float(w[j] << 16);
      b[j] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
  }
};
template <> struct RawPair<float> {
  float2 f[16];
  __device__ __forceinline__ void load(const float* p, int64_t ld) {
#pragma unroll
    for (int j = 0; j < 16; ++j) f[j] = __ldg(reinterpret_cast<const float2*>(p + j * ld));
  }
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int j = 0; j < 16; ++j) f[j] = make_float2(0.0f, 0.0f);
  }
  __device__ __forceinline__ void widen(float a[16], float b[16]) const {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      a[j] = f[j].x;
      b[j] = f[j].y;
    }
  }
};

// Per-thread amax over the row-axis units (column pair x 16 rows; rows % 16
// == 0 and cols even for this mode), with the RHT applied along rows when
// enabled; two units' loads in flight per thread.
template <typename T, bool RHT>
__device__ float amax_cols(const QTensor& q, uint32_t mask, const Slice sl) {
  const T* x = static_cast<const T*>(q.x);
  const uint32_t ncp = (uint32_t)(q.cols >> 1);
  const uint32_t nunits = ncp * (uint32_t)(q.rows >> 4);
  const FastDiv div = make_fastdiv(ncp);
  const uint32_t stride = sl.ncta * kThreads;
  float m = 0.0f;
  for (uint32_t u = sl.cta * kThreads + threadIdx.x; u < nunits; u += 2 * stride) {
    RawPair<T> raw[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint32_t uj = u + j * stride;
      if (uj < nunits) {
        const uint32_t rg = fastdiv(uj, div), cp = uj - rg * ncp;
        raw[j].load(x + (int64_t)rg * 16 * q.ld + 2 * (int64_t)cp, q.ld);
      } else {
        raw[j].zero();
      }
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float a[16], b[16];
      raw[j].widen(a, b);
      if (RHT) {
        rht16(a, mask);
        rht16(b, mask);
      }
      m = fmaxf(m, fmaxf(absmax16(a), absmax16(b)));
    }
  }
  return m;
}

// Zero the padding entries of a tcgen05-layout scale buffer.
__device__ void zero_sf_padding(uint8_t* sf, int64_t rows, int64_t kbpr, const Slice sl) {
  const int64_t rows_pad = (rows + 127) & ~int64_t(127);
  const int64_t kb_pad = (kbpr + 3) & ~int64_t(3);
  const int64_t tid = (int64_t)sl.cta * kThreads + threadIdx.x;
  const int64_t step = (int64_t)sl.ncta * kThreads;
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

// Raw 16-element block as loaded: bf16 keeps its 8 packed words, fp32 its 16
// values; widened to fp32 when used.
template <typename T> struct RawBlock;
template <> struct RawBlock<__nv_bfloat16> {
  uint32_t w[8];
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { load16_raw(p, w); }
  __device__ __forceinline__ void widen(float v[16]) const {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
  // the block as packed fp32 pairs (after the transform when RHT) and its max |y|
  template <bool RHT>
  __device__ __forceinline__ float prepare(uint64_t yy[8], uint32_t mask) const {
    if constexpr (RHT) {
      float v[16];
      widen(v);
      rht16(v, mask);
      pairs_of(v, yy);
      return absmax16(v);
    } else {
      widen_pairs(w, yy);
      return absmax16_raw(w);
    }
  }
};
template <> struct RawBlock<float> {
  float f[16];
  __device__ __forceinline__ void load(const float* p) { load16(p, f); }
  __device__ __forceinline__ void widen(float v[16]) const {
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = f[i];
  }
  template <bool RHT>
  __device__ __forceinline__ float prepare(uint64_t yy[8], uint32_t mask) const {
    float v[16];
    widen(v);
    if (RHT) rht16(v, mask);
    pairs_of(v, yy);
    return absmax16(v);
  }
};

// Blocks the fast encoder hands back are queued per warp (block index and
// the final scale code, or kRedoAll) and redone exactly by the whole warp
// when the queue fills and at the end, so a rare block does not stall the
// other 31 lanes at every step.
constexpr int kQueueCap = 128;            // entries per warp
constexpr uint32_t kRedoAll = 0xFFFFFFFFu;  // redo the pick as well

struct WarpQueue {
  uint2* item;  // shared memory, kQueueCap entries
  uint32_t n;   // same value on every lane
  uint4* data;  // shared memory, 2 x 16 bytes per entry (the block's raw input), or nullptr
  __device__ __forceinline__ void push(bool need, uint32_t idx, uint32_t code,
                                       const uint32_t* raw8 = nullptr) {
    const uint32_t m = __ballot_sync(0xFFFFFFFFu, need);
    if (need) {
      const uint32_t slot = n + __popc(m & ((1u << (threadIdx.x & 31)) - 1u));
      item[slot] = make_uint2(idx, code);
      if (raw8) {
        data[2 * slot] = make_uint4(raw8[0], raw8[1], raw8[2], raw8[3]);
        data[2 * slot + 1] = make_uint4(raw8[4], raw8[5], raw8[6], raw8[7]);
      }
    }
    n += __popc(m);
  }
  // redo(entry, its 32 raw bytes or garbage when pushed without them)
  template <typename F>
  __device__ __forceinline__ void drain(F&& redo) {
    __syncwarp();
    for (uint32_t i = threadIdx.x & 31; i < n; i += 32) redo(item[i], data + 2 * i);
    __syncwarp();
    n = 0;
  }
};

__device__ __forceinline__ void store_codes(uint8_t* dst, uint32_t lo, uint32_t hi) {
  *reinterpret_cast<uint2*>(dst) = make_uint2(lo, hi);
}

// The exact encoding of one block for a queued entry: the whole block
// (kRedoAll) or its codes under the given final scale code.
__device__ __forceinline__ void redo_block(const float v[16], uint32_t code, const ScaleCtx& ctx,
                                           bool fos, uint8_t* codes_dst, uint8_t* scale_dst) {
  uint32_t lo, hi, sc;
  if (code == kRedoAll) {
    quantize_block16(v, ctx, fos, lo, hi, sc);
    *scale_dst = (uint8_t)sc;
  } else {
    uint32_t w[2];
    codes16(v, cand_scale(code, ctx.alpha), w);
    lo = w[0];
    hi = w[1];
  }
  store_codes(codes_dst, lo, hi);
}

// Encode pass, 16-blocks along the contiguous dim.  CTA-uniform grid-stride
// over blocks, the next block's load issued before the current one is
// encoded.
template <typename T, bool RHT>
__device__ void encode_rows(const QTensor& q, float alpha, const QBatch& p, uint2* qbuf,
                            uint4* qdata, const Slice sl) {
  const T* x = static_cast<const T*>(q.x);
  const uint32_t kbpr = (uint32_t)(q.cols >> 4);
  const uint32_t nblk = (uint32_t)q.rows * kbpr;  // < 2^32, checked on the host
  const FastDiv div = make_fastdiv(kbpr);
  const bool fos = p.four_over_six != 0;
  const ScaleCtx ctx = make_scale_ctx(alpha);
  const uint32_t stride = sl.ncta * kThreads;
  // codes rows are cols / 2 bytes, so block b's codes start at 8 b; a
  // contiguous input (ld == cols) and row-major scales need no division
  const bool contig = q.ld == q.cols;
  auto src = [&](uint32_t b) { return block_ptr(x, b, contig, kbpr, div, q.ld); };
  auto codes_at = [&](uint32_t b) { return q.codes + (int64_t)b * 8; };
  auto scale_at = [&](uint32_t b) {
    if (p.sf_layout == 0) return q.scales + b;
    const uint32_t r = fastdiv(b, div);
    return q.scales + sf_offset(r, b - r * kbpr, kbpr, 1);
  };
  // bf16 blocks are queued with their raw input, fp32 blocks are reloaded
  constexpr bool kCarry = std::is_same<T, __nv_bfloat16>::value;
  auto redo = [&](uint2 it, const uint4* d) {
    float v[16];
    if constexpr (kCarry) {
      const uint4 d0 = d[0], d1 = d[1];
      const uint32_t w[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
    } else {
      RawBlock<T> blk;
      blk.load(src(it.x));
      blk.widen(v);
    }
    if (RHT) rht16(v, p.mask);
    redo_block(v, it.y, ctx, fos, codes_at(it.x), scale_at(it.x));
  };
  WarpQueue wq{qbuf, 0u, qdata};
  uint32_t u = sl.cta * kThreads + threadIdx.x;
  RawBlock<T> next;
  if (u < nblk) next.load(src(u));
  for (uint32_t base = sl.cta * kThreads; base < nblk; base += stride, u += stride) {
    const RawBlock<T> cur = next;
    if (u + stride < nblk) next.load(src(u + stride));
    uint32_t st = kBlockDone, sc = 0u;
    if (u < nblk) {
      uint32_t lo, hi;
#if NVFP4_ROWS_PACKED
      uint64_t yy[8];
      const float bmax = cur.template prepare<RHT>(yy, p.mask);
      st = quantize_block16_pairs(yy, bmax, ctx, fos, lo, hi, sc);
#else
      float v[16];
      cur.widen(v);
      if (RHT) rht16(v, p.mask);
      st = quantize_block16_try(v, ctx, fos, lo, hi, sc);
#endif
      if (st == kBlockDone) store_codes(codes_at(u), lo, hi);
      if (st != kBlockExact) *scale_at(u) = (uint8_t)sc;
    }
    if constexpr (kCarry)
      wq.push(st != kBlockDone, u, st == kBlockExact ? kRedoAll : sc, cur.w);
    else
      wq.push(st != kBlockDone, u, st == kBlockExact ? kRedoAll : sc);
    if (wq.n > kQueueCap - 32) wq.drain(redo);
  }
  wq.drain(redo);
  if (p.sf_layout == 1) zero_sf_padding(q.scales, q.rows, kbpr, sl);
}

// Encode pass, blocks along rows; output transposed: codes [cols, rows/2],
// scales for cols rows x rows/16 blocks.  Unit = column pair x 16 rows (two
// blocks), the next unit's loads issued before the current one is encoded.
template <typename T, bool RHT>
__device__ void encode_cols(const QTensor& q, float alpha, const QBatch& p, uint2* qbuf,
                            const Slice sl) {
  const T* x = static_cast<const T*>(q.x);
  const uint32_t ncp = (uint32_t)(q.cols >> 1);
  const uint32_t kb_total = (uint32_t)(q.rows >> 4);
  const uint32_t nunits = ncp * kb_total;
  const int64_t out_row_bytes = q.rows >> 1;
  const FastDiv div = make_fastdiv(ncp), div_out = make_fastdiv(kb_total);
  const bool fos = p.four_over_six != 0;
  const ScaleCtx ctx = make_scale_ctx(alpha);
  const uint32_t stride = sl.ncta * kThreads;
  auto src = [&](uint32_t unit) {
    const uint32_t rg = fastdiv(unit, div);
    return x + (int64_t)rg * 16 * q.ld + 2 * (int64_t)(unit - rg * ncp);
  };
  // queued entries hold the output block index c * kb_total + kb
  auto redo = [&](uint2 it, const uint4*) {
    const uint32_t c = fastdiv(it.x, div_out), kb = it.x - c * kb_total;
    float v[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = load1(x + ((int64_t)kb * 16 + j) * q.ld + c);
    if (RHT) rht16(v, p.mask);
    redo_block(v, it.y, ctx, fos, q.codes + (int64_t)c * out_row_bytes + (int64_t)kb * 8,
               q.scales + sf_offset(c, kb, kb_total, p.sf_layout));
  };
  WarpQueue wq{qbuf, 0u, nullptr};
  uint32_t u = sl.cta * kThreads + threadIdx.x;
  RawPair<T> next;
  if (u < nunits) next.load(src(u), q.ld);
  for (uint32_t base = sl.cta * kThreads; base < nunits; base += stride, u += stride) {
    const RawPair<T> cur = next;
    if (u + stride < nunits) next.load(src(u + stride), q.ld);
    uint32_t st[2] = {kBlockDone, kBlockDone}, sc[2] = {0u, 0u}, ob[2] = {0u, 0u};
    if (u < nunits) {
      const uint32_t kb = fastdiv(u, div), c0 = 2 * (u - kb * ncp);
      float col[2][16];
      cur.widen(col[0], col[1]);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (RHT) rht16(col[h], p.mask);
        uint32_t lo, hi;
        st[h] = quantize_block16_try(col[h], ctx, fos, lo, hi, sc[h]);
        const uint32_t c = c0 + h;
        ob[h] = c * kb_total + kb;
        if (st[h] == kBlockDone)
          store_codes(q.codes + (int64_t)c * out_row_bytes + (int64_t)kb * 8, lo, hi);
        if (st[h] != kBlockExact) q.scales[sf_offset(c, kb, kb_total, p.sf_layout)] = (uint8_t)sc[h];
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h)
      wq.push(st[h] != kBlockDone, ob[h], st[h] == kBlockExact ? kRedoAll : sc[h]);
    if (wq.n > kQueueCap - 64) wq.drain(redo);
  }
  wq.drain(redo);
  if (p.sf_layout == 1) zero_sf_padding(q.scales, q.cols, kb_total, sl);
}

// ------------------------------------------------------------------------
// Row-axis (transposing) mode for bf16 inputs, staged through shared memory
// by TMA.  The input is walked in tiles of 64 rows x 128 columns (16 KB, one
// cp.async.bulk.tensor each, zero-filled past the tensor's edges), kTmaStages
// tiles in flight per CTA.  In a tile, thread t owns the column pair
// 2 (t % 64), 2 (t % 64) + 1 and the 16-row group t / 64: it reads its 16
// words (one bf16 pair per row) from shared memory -- a warp reads 32
// consecutive words of a row, conflict-free -- and handles the two
// 16-element blocks along rows; the four row groups of a tile fill one
// 32-byte run of each output row's codes.  A bounded wait that runs out
// records NVFP4_ERR_TIMEOUT; the CTA then waits for its loads in flight
// (bounded) and stops.
constexpr int kTmaRows = 64, kTmaCols = 128;
constexpr int kTmaTileBytes = kTmaRows * kTmaCols * 2;
// tiles in flight per CTA: the amax pass, the encode pass (which also holds
// its queue of handed-back blocks in shared memory, kColsQueueCap entries per
// warp) and the CTAs per SM the encode pass is compiled for
constexpr int kTmaStages = 4;
#ifndef NVFP4_COLS_ENC_STAGES
#define NVFP4_COLS_ENC_STAGES 4
#endif
#ifndef NVFP4_COLS_QCAP
#define NVFP4_COLS_QCAP 128
#endif
#ifndef NVFP4_COLS_MINB
#define NVFP4_COLS_MINB 2
#endif
constexpr int kColsEncStages = NVFP4_COLS_ENC_STAGES;
constexpr int kColsQueueCap = NVFP4_COLS_QCAP;
constexpr int tma_smem_bytes(int stages) { return stages * kTmaTileBytes + 128; }
constexpr uint64_t kTmaWaitNs = 2000000000ull, kTmaDrainNs = 200000000ull;

struct ColsMaps {
  CUtensorMap m[kMaxBatch];
};

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ bool bar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  if (bar_try(bar, parity)) return true;
  uint64_t t0;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  for (uint32_t i = 1;; ++i) {
    if (bar_try(bar, parity)) return true;
    if ((i & 63) == 0) {
      uint64_t t;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
      if (t - t0 > limit_ns) return false;
    }
  }
}

// The tile ring of one CTA over its share of a tensor's tiles (tile i of the
// CTA = sl.cta + i * sl.ncta): thread 0 keeps the next kTmaStages - 1 tiles
// loading; fn(tile, smem of the tile) runs on every thread.  Returns false
// after a wait ran out (error recorded, loads in flight drained).
template <int kTmaStages, typename F>
__device__ bool tma_tile_loop(const CUtensorMap* map, const QTensor& q, const Slice sl,
                              uint8_t* smem, uint32_t* err, F&& fn) {
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kTmaStages * kTmaTileBytes);
  __shared__ int abort_flag;
  const uint32_t ntc = (uint32_t)((q.cols + kTmaCols - 1) / kTmaCols);
  const uint32_t ntiles = (uint32_t)((q.rows + kTmaRows - 1) / kTmaRows) * ntc;
  const uint32_t mine = sl.cta < ntiles ? (ntiles - sl.cta + sl.ncta - 1) / sl.ncta : 0u;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kTmaStages; ++i)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(&full[i])) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    abort_flag = 0;
  }
  __syncthreads();
  auto issue = [&](uint32_t i) {  // thread 0: tile i of this CTA into slot i % kTmaStages
    const uint32_t t = sl.cta + i * sl.ncta;
    const uint32_t bar = smem_addr(&full[i % kTmaStages]);
    const int32_t c0 = (int32_t)((t % ntc) * kTmaCols), r0 = (int32_t)((t / ntc) * kTmaRows);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
                 "r"(kTmaTileBytes)
                 : "memory");
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(smem + (i % kTmaStages) * kTmaTileBytes)),
        "l"((uint64_t)map), "r"(c0), "r"(r0), "r"(bar)
        : "memory");
  };
  uint32_t issued = 0;
  if (threadIdx.x == 0)
    for (; issued < mine && issued < (uint32_t)kTmaStages - 1; ++issued) issue(issued);
  bool ok = true;
  for (uint32_t i = 0; i < mine; ++i) {
    if (threadIdx.x == 0 && issued < mine) issue(issued++);  // the slot freed by tile i - 1
    if (!bar_wait(smem_addr(&full[i % kTmaStages]), (i / kTmaStages) & 1u, kTmaWaitNs)) {
      abort_flag = 1;
    } else {
      fn(sl.cta + i * sl.ncta, smem + (i % kTmaStages) * kTmaTileBytes);
    }
    __syncthreads();  // every thread is done with slot i before it is refilled
    if (abort_flag) {
      ok = false;
      break;
    }
  }
  if (!ok && threadIdx.x == 0) {
    atomicOr(err, kDevErrTimeout);
    // loads still in flight: the unconsumed tiles are among the last
    // kTmaStages issued (tiles before those were waited for)
    for (uint32_t j = issued > (uint32_t)kTmaStages ? issued - kTmaStages : 0u; j < issued; ++j)
      bar_wait(smem_addr(&full[j % kTmaStages]), (j / kTmaStages) & 1u, kTmaDrainNs);
  }
  return ok;
}

// This thread's 16 words of a tile: rows 16 g .. 16 g + 15 of column pair cp
// (word j = row j, both columns).  With the transform, the signs s_j are
// applied here, to both columns of a row at once.
template <bool RHT>
__device__ __forceinline__ void tile_words(const uint8_t* tile, uint32_t mask, uint32_t w[16]) {
  const uint32_t cp = threadIdx.x & 63, g = threadIdx.x >> 6;
  const uint32_t* tw = reinterpret_cast<const uint32_t*>(tile) + (16 * g) * (kTmaCols / 2) + cp;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    w[j] = tw[j * (kTmaCols / 2)];
    if (RHT) w[j] ^= ((mask >> j) & 1u) * 0x80008000u;
  }
}
// The column block h (0: even column, 1: odd column) of those words, widened,
// with the butterflies of the transform along rows when RHT.
template <bool RHT>
__device__ __forceinline__ void column_block(const uint32_t w[16], int h, float v[16]) {
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(h ? (w[j] & 0xFFFF0000u) : (w[j] << 16));
  if (RHT) rht16_butterflies(v);
}

template <bool RHT>
__global__ void __launch_bounds__(kThreads, 3)
    amax_cols_tma_kernel(const __grid_constant__ QBatch p, const __grid_constant__ ColsMaps maps) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int t = blockIdx.y;
  const QTensor& q = p.t[t];
  const Slice sl{blockIdx.x, gridDim.x};
  float m = 0.0f;
  tma_tile_loop<kTmaStages>(&maps.m[t], q, sl, smem, p.err, [&](uint32_t, const uint8_t* tile) {
    uint32_t w[16];
    tile_words<RHT>(tile, p.mask, w);  // zero past the tensor's edges: no effect on the max
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float v[16];
      column_block<RHT>(w, h, v);
      m = fmaxf(m, absmax16(v));
    }
  });
  m = block_reduce_max(m);
  if (threadIdx.x == 0) p.partials[t * kMaxAmaxCtas + sl.cta] = m;
  pdl_trigger();
}

// The amax pass of a contiguous tensor (row blocks, no RHT) through shared
// memory: the tensor's bytes as 16 KB chunks, each one cp.async.bulk into a
// 4-deep ring per CTA (chunk i of this CTA into slot i % 4), the same bounded
// waits and drain as the tiled loop.  The last chunk may be shorter (a
// multiple of 32 bytes).  fn(slot, bytes) reads the chunk.
template <int kStages, typename F>
__device__ bool bulk_chunk_loop(const uint8_t* src, uint64_t n_bytes, const Slice sl,
                                uint8_t* smem, uint32_t* err, F&& fn) {
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kTmaTileBytes);
  __shared__ int abort_flag;
  const uint64_t nchunks = (n_bytes + kTmaTileBytes - 1) / kTmaTileBytes;
  const uint32_t mine =
      sl.cta < nchunks ? (uint32_t)((nchunks - sl.cta + sl.ncta - 1) / sl.ncta) : 0u;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(&full[i])) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    abort_flag = 0;
  }
  __syncthreads();
  auto bytes_of = [&](uint32_t i) {
    const uint64_t off = (uint64_t)(sl.cta + (uint64_t)i * sl.ncta) * kTmaTileBytes;
    const uint64_t left = n_bytes - off;
    return (uint32_t)(left < (uint64_t)kTmaTileBytes ? left : (uint64_t)kTmaTileBytes);
  };
  auto issue = [&](uint32_t i) {  // thread 0
    const uint64_t off = (uint64_t)(sl.cta + (uint64_t)i * sl.ncta) * kTmaTileBytes;
    const uint32_t bar = smem_addr(&full[i % kStages]), nb = bytes_of(i);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(nb)
                 : "memory");
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(smem + (i % kStages) * kTmaTileBytes)),
        "l"(src + off), "r"(nb), "r"(bar)
        : "memory");
  };
  uint32_t issued = 0;
  if (threadIdx.x == 0)
    for (; issued < mine && issued < (uint32_t)kStages - 1; ++issued) issue(issued);
  bool ok = true;
  for (uint32_t i = 0; i < mine; ++i) {
    if (threadIdx.x == 0 && issued < mine) issue(issued++);  // the slot freed by chunk i - 1
    if (!bar_wait(smem_addr(&full[i % kStages]), (i / kStages) & 1u, kTmaWaitNs)) {
      abort_flag = 1;
    } else {
      fn(smem + (i % kStages) * kTmaTileBytes, bytes_of(i));
    }
    __syncthreads();  // every thread is done with slot i before it is refilled
    if (abort_flag) {
      ok = false;
      break;
    }
  }
  if (!ok && threadIdx.x == 0) {
    atomicOr(err, kDevErrTimeout);
    for (uint32_t j = issued > (uint32_t)kStages ? issued - kStages : 0u; j < issued; ++j)
      bar_wait(smem_addr(&full[j % kStages]), (j / kStages) & 1u, kTmaDrainNs);
  }
  return ok;
}

// Thread t reads 16-byte words t, t + 256, ... of a chunk (a warp reads 512
// contiguous bytes per load: no bank conflicts).
template <typename T>
__global__ void __launch_bounds__(kThreads, 3) amax_flat_bulk_kernel(const __grid_constant__ QBatch p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int t = blockIdx.y;
  const QTensor& q = p.t[t];
  const Slice sl{blockIdx.x, gridDim.x};
  const uint64_t n_bytes = (uint64_t)q.rows * (uint64_t)q.cols * sizeof(T);
  uint32_t m2 = 0u;  // bf16: max |x| per half, as bits
  float mf = 0.0f;
  bulk_chunk_loop<kTmaStages>(static_cast<const uint8_t*>(q.x), n_bytes, sl, smem, p.err,
                              [&](const uint8_t* chunk, uint32_t bytes) {
    const uint4* c4 = reinterpret_cast<const uint4*>(chunk);
    const uint32_t nw = bytes >> 4;
#pragma unroll
    for (uint32_t k = 0; k < (uint32_t)kTmaTileBytes / 16 / kThreads; ++k) {
      const uint32_t i = threadIdx.x + k * kThreads;
      if (i < nw) {
        const uint4 v = c4[i];
        if constexpr (std::is_same<T, __nv_bfloat16>::value) {
          m2 = absmax_bf16x2(m2, v.x);
          m2 = absmax_bf16x2(m2, v.y);
          m2 = absmax_bf16x2(m2, v.z);
          m2 = absmax_bf16x2(m2, v.w);
        } else {
          mf = fmaxf(mf, fmaxf(fmaxf(fabsf(__uint_as_float(v.x)), fabsf(__uint_as_float(v.y))),
                               fmaxf(fabsf(__uint_as_float(v.z)), fabsf(__uint_as_float(v.w)))));
        }
      }
    }
  });
  float m = std::is_same<T, __nv_bfloat16>::value
                ? fmaxf(__uint_as_float(m2 << 16), __uint_as_float(m2 & 0xFFFF0000u))
                : mf;
  m = block_reduce_max(m);
  if (threadIdx.x == 0) p.partials[t * kMaxAmaxCtas + sl.cta] = m;
  pdl_trigger();
}

template <bool RHT>
__global__ void __launch_bounds__(kThreads, NVFP4_COLS_MINB)
    encode_cols_tma_kernel(const __grid_constant__ QBatch p, const __grid_constant__ ColsMaps maps,
                           int ga) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int t = blockIdx.y;
  const QTensor& q = p.t[t];
  const Slice sl{blockIdx.x, gridDim.x};
  float alpha;
  if (p.gs_in) {
    alpha = *p.gs_in;
  } else {
    pdl_wait();
    alpha = alpha_from_amax(reduce_partials(p.partials + t * kMaxAmaxCtas, ga));
  }
  if (sl.cta == 0 && threadIdx.x == 0 && q.gs_out) *q.gs_out = alpha;
  // per-warp queue of handed-back blocks; each entry carries the block's 16
  // input values (bf16, element j in half j % 2 of word j / 2), so the redo
  // reads shared memory, not the tile's rows in global memory again
  __shared__ uint2 queue[kThreads / 32][kColsQueueCap];
  __shared__ uint4 qdata[kThreads / 32][kColsQueueCap][2];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t qn = 0;  // same value on every lane
  const uint32_t kb_total = (uint32_t)(q.rows >> 4);
  const int64_t out_row_bytes = q.rows >> 1;
  const FastDiv div_out = make_fastdiv(kb_total);
  const bool fos = p.four_over_six != 0;
  const ScaleCtx ctx = make_scale_ctx(alpha);
  const uint32_t ntc = (uint32_t)((q.cols + kTmaCols - 1) / kTmaCols);
  // queued entries hold the output block index c * kb_total + kb
  auto drain = [&]() {
    __syncwarp();
    for (uint32_t i = lane; i < qn; i += 32) {
      const uint2 it = queue[warp][i];
      const uint4 d0 = qdata[warp][i][0], d1 = qdata[warp][i][1];
      const uint32_t dw[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
      float v[16];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        v[2 * k] = __uint_as_float(dw[k] << 16);
        v[2 * k + 1] = __uint_as_float(dw[k] & 0xFFFF0000u);
      }
      if (RHT) rht16_butterflies(v);  // signs already applied to the queued words
      const uint32_t c = fastdiv(it.x, div_out), kb = it.x - c * kb_total;
      redo_block(v, it.y, ctx, fos, q.codes + (int64_t)c * out_row_bytes + (int64_t)kb * 8,
                 q.scales + sf_offset(c, kb, kb_total, p.sf_layout));
    }
    __syncwarp();
    qn = 0;
  };
  tma_tile_loop<kColsEncStages>(&maps.m[t], q, sl, smem, p.err,
                                [&](uint32_t tile_id, const uint8_t* tile) {
    uint32_t w[16];
    tile_words<RHT>(tile, p.mask, w);
    const uint32_t kb = (tile_id / ntc) * (kTmaRows / 16) + (threadIdx.x >> 6);
    const int64_t c0 = (int64_t)(tile_id % ntc) * kTmaCols + 2 * (threadIdx.x & 63);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t c = c0 + h;
      const bool valid = kb < kb_total && c < q.cols;
      uint32_t st = kBlockDone, sc = 0u;
      if (valid) {
        float v[16];
        column_block<RHT>(w, h, v);
        uint64_t yy[8];
        pairs_of(v, yy);
        uint32_t lo, hi;
        st = quantize_block16_pairs(yy, absmax16(v), ctx, fos, lo, hi, sc);
        if (st == kBlockDone) store_codes(q.codes + c * out_row_bytes + (int64_t)kb * 8, lo, hi);
        if (st != kBlockExact) q.scales[sf_offset(c, kb, kb_total, p.sf_layout)] = (uint8_t)sc;
      }
      const bool need = st != kBlockDone;
      const uint32_t m = __ballot_sync(0xFFFFFFFFu, need);
      if (need) {
        const uint32_t slot = qn + __popc(m & ((1u << lane) - 1u));
        queue[warp][slot] = make_uint2((uint32_t)c * kb_total + kb,
                                       st == kBlockExact ? kRedoAll : sc);
        uint32_t dw[8];  // column h's 16 values, two rows per word
#pragma unroll
        for (int k = 0; k < 8; ++k)
          dw[k] = h ? ((w[2 * k] >> 16) | (w[2 * k + 1] & 0xFFFF0000u))
                    : ((w[2 * k] & 0xFFFFu) | (w[2 * k + 1] << 16));
        qdata[warp][slot][0] = make_uint4(dw[0], dw[1], dw[2], dw[3]);
        qdata[warp][slot][1] = make_uint4(dw[4], dw[5], dw[6], dw[7]);
      }
      qn += __popc(m);
    }
    if (qn > kColsQueueCap - 64) drain();
  });
  drain();
  if (p.sf_layout == 1) zero_sf_padding(q.scales, q.cols, kb_total, sl);
}

// Encode pass, 16x16 tiles.  A warp holds two adjacent tiles of one 16-row
// band: lane l owns row (l & 15) of tile (l >> 4).  Tile max and tile error
// reduce across the 16 lanes of a half-warp with xor shuffles 8, 4, 2, 1 --
// the same pairwise order as the per-row sum, and the same result on every
// lane of the half-warp, so each tile's decisions are uniform over its lanes.
// The pick is certified from approximate row errors as in the 1D path (the
// tile margin is the sum of its 16 rows' margins); a tile too close to call
// is redone exactly by its half-warp, and rows whose codes are ambiguous are
// queued for an exact redo under the tile's scale.
template <typename T>
__device__ void encode_2d(const QTensor& q, float alpha, const QBatch& p, uint2* qbuf,
                          const Slice sl) {
  const T* x = static_cast<const T*>(q.x);
  const uint32_t kbpr = (uint32_t)(q.cols >> 4);
  const uint32_t npair = (kbpr + 1) >> 1;
  const uint32_t nunits = (uint32_t)(q.rows >> 4) * npair;
  const int lane = threadIdx.x & 31;
  const unsigned hmask = 0xFFFFu << (lane & 16);
  const uint32_t warps = kThreads / 32;
  const bool fos = p.four_over_six != 0;
  const ScaleCtx ctx = make_scale_ctx(alpha);
  const FastDiv div = make_fastdiv(npair), div_blk = make_fastdiv(kbpr);
  // queued entries hold the block index r * kbpr + kb and the tile's scale
  auto redo = [&](uint2 it, const uint4*) {
    const uint32_t r = fastdiv(it.x, div_blk), kb = it.x - r * kbpr;
    float v[16];
    load16(x + (int64_t)r * q.ld + (int64_t)kb * 16, v);
    redo_block(v, it.y, ctx, fos, q.codes + (int64_t)r * (q.cols >> 1) + (int64_t)kb * 8, nullptr);
  };
  // this lane's block of unit u: row r, block column kb (false past the last column)
  auto block_of = [&](uint32_t u, int64_t& r, uint32_t& kb) {
    const uint32_t tr = fastdiv(u, div), tp = u - tr * npair;
    r = (int64_t)tr * 16 + (lane & 15);
    kb = tp * 2 + (lane >> 4);
    return kb < kbpr;
  };
  WarpQueue wq{qbuf, 0u, nullptr};
  const uint32_t ustride = sl.ncta * warps;
  uint32_t u = sl.cta * warps + (threadIdx.x >> 5);
  // the next unit's block is loaded before the current one is encoded
  RawBlock<T> next;
  if (u < nunits) {
    int64_t r;
    uint32_t kb;
    if (block_of(u, r, kb)) next.load(x + r * q.ld + (int64_t)kb * 16);
  }
  for (; u < nunits; u += ustride) {
    int64_t r;
    uint32_t kb;
    const bool valid = block_of(u, r, kb);
    const RawBlock<T> cur = next;
    if (u + ustride < nunits) {
      int64_t rn;
      uint32_t kbn;
      if (block_of(u + ustride, rn, kbn)) next.load(x + rn * q.ld + (int64_t)kbn * 16);
    }
    float v[16];
    if (valid) {
      cur.widen(v);
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = 0.0f;
    }
    float tmax = absmax16(v);
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xFFFFFFFFu, tmax, o));
    uint32_t e6, e4;
    scale_codes(tmax, ctx, e6, e4);
    const float s6 = cand_scale(e6, alpha);
    uint32_t ew = e6, lo = 0u, hi = 0u, st = kBlockDone;
    float sw = s6;
    bool exact_tile = false;
    if (fos && e4 != e6) {
      const float s4 = cand_scale(e4, alpha);
      int pick = 2;
      if (fast_pick_ok(e6, s6, s4)) {
        float a6 = approx_err16(v, rcp_approx(s6)), a4 = approx_err16(v, rcp_approx(s4));
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) {
          a6 += __shfl_xor_sync(hmask, a6, o);
          a4 += __shfl_xor_sync(hmask, a4, o);
        }
        pick = certified_pick(a6, s6, a4, s4, 16.0f * kPickMargin);
      }
      if (pick == 1) {
        ew = e4;
        sw = s4;
      } else if (pick == 2) {  // exact tile errors
        exact_tile = true;
        Cand c6 = encode16(v, s6);
        Cand c4 = encode16(v, s4);
        float err6 = c6.err, err4 = c4.err;
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) {
          err6 = __fadd_rn(err6, __shfl_xor_sync(hmask, err6, o));
          err4 = __fadd_rn(err4, __shfl_xor_sync(hmask, err4, o));
        }
        const bool four = err4 < err6;
        lo = four ? c4.lo : c6.lo;
        hi = four ? c4.hi : c6.hi;
        ew = four ? e4 : e6;
      }
    }
    if (!exact_tile && sw != 0.0f) {
      uint32_t w[2];
      st = rcp_ok(sw) && codes16_try(v, rcp_approx(sw), w) ? kBlockDone : kBlockCodes;
      lo = w[0];
      hi = w[1];
    }
    const uint32_t blk = (uint32_t)r * kbpr + kb;
    if (valid) {
      if (st == kBlockDone) store_codes(q.codes + r * (q.cols >> 1) + (int64_t)kb * 8, lo, hi);
      q.scales[sf_offset(r, kb, kbpr, p.sf_layout)] = (uint8_t)ew;
    }
    wq.push(valid && st != kBlockDone, blk, ew);
    if (wq.n > kQueueCap - 32) wq.drain(redo);
  }
  wq.drain(redo);
  if (p.sf_layout == 1) zero_sf_padding(q.scales, q.rows, kbpr, sl);
}

// kModeMixed: 1D row-block and 2D tensors in one launch (no RHT).
enum { kModeRows = 0, kModeCols = 1, kMode2D = 2, kModeMixed = 3 };

// Tensor of CTA b in a mixed launch (end[] = ends of the tensors' CTA
// ranges) and the CTA's place in that tensor's range.
__device__ __forceinline__ int tensor_of(const int32_t* end, int n, uint32_t b, Slice& sl) {
  int t = 0;
  while (t < n - 1 && (int32_t)b >= end[t]) ++t;
  const int32_t begin = t ? end[t - 1] : 0;
  sl.cta = b - (uint32_t)begin;
  sl.ncta = (uint32_t)(end[t] - begin);
  return t;
}

// One CTA of the amax pass over tensor blockIdx.y (mixed: over the tensor
// whose range holds blockIdx.x): its partial maximum goes to
// partials[t * kMaxAmaxCtas + (its index within the tensor's CTAs)].
template <typename T, int MODE, bool RHT>
__global__ void __launch_bounds__(kThreads, 3) amax_kernel(const __grid_constant__ QBatch p) {
  Slice sl{blockIdx.x, gridDim.x};
  int t = blockIdx.y;
  if constexpr (MODE == kModeMixed) t = tensor_of(p.amax_end, p.n, blockIdx.x, sl);
  // the row-axis mode reads its input as element pairs in both passes: its
  // rows need not satisfy the contiguous path's 32-byte alignment
  float m = MODE == kModeCols ? amax_cols<T, RHT>(p.t[t], p.mask, sl)
                              : amax_rows<T, RHT>(p.t[t], p.mask, sl);
  m = block_reduce_max(m);
  if (threadIdx.x == 0) p.partials[t * kMaxAmaxCtas + sl.cta] = m;
  pdl_trigger();
}

// Global scale only: one CTA per tensor reduces the partials.
__global__ void __launch_bounds__(kThreads) finalize_kernel(const __grid_constant__ QBatch p, int ga) {
  pdl_wait();
  const int t = blockIdx.x;
  const float a = alpha_from_amax(reduce_partials(p.partials + t * kMaxAmaxCtas, ga));
  if (threadIdx.x == 0 && p.t[t].gs_out) *p.t[t].gs_out = a;
}

// Encode pass over tensor blockIdx.y.  ga = number of amax partials (0 when
// the global scale is given).
// Resident CTAs per SM the encode kernels are compiled for: the row-axis mode
// holds two 16-element columns per thread and needs the larger register file.
#ifndef NVFP4_ROWS_PACKED
#define NVFP4_ROWS_PACKED 1
#endif
#ifndef NVFP4_ROWS_MIN_BLOCKS
#define NVFP4_ROWS_MIN_BLOCKS 3
#endif
template <typename T, int MODE>
constexpr int encode_min_blocks() {
  return MODE == kModeCols ? 2
         : (MODE == kModeRows && std::is_same<T, float>::value) ? 2
         : (MODE == kModeRows || MODE == kModeMixed) ? NVFP4_ROWS_MIN_BLOCKS
                                                     : 3;
}

template <typename T, int MODE, bool RHT>
__global__ void __launch_bounds__(kThreads, encode_min_blocks<T, MODE>()) encode_kernel(const __grid_constant__ QBatch p, int ga) {
  Slice sl{blockIdx.x, gridDim.x};
  int t = blockIdx.y;
  if constexpr (MODE == kModeMixed) {
    t = tensor_of(p.enc_end, p.n, blockIdx.x, sl);
    ga = p.amax_end[t] - (t ? p.amax_end[t - 1] : 0);
  }
  float alpha;
  if (p.gs_in) {
    alpha = *p.gs_in;
  } else {
    pdl_wait();
    alpha = alpha_from_amax(reduce_partials(p.partials + t * kMaxAmaxCtas, ga));
  }
  if (sl.cta == 0 && threadIdx.x == 0 && p.t[t].gs_out) *p.t[t].gs_out = alpha;
  __shared__ uint2 queue[kThreads / 32][kQueueCap];
  __shared__ uint4 qraw[kThreads / 32][2 * kQueueCap];
  uint2* qbuf = queue[threadIdx.x >> 5];
  uint4* qdata = qraw[threadIdx.x >> 5];
  if constexpr (MODE == kModeRows) {
    encode_rows<T, RHT>(p.t[t], alpha, p, qbuf, qdata, sl);
  } else if constexpr (MODE == kModeCols) {
    encode_cols<T, RHT>(p.t[t], alpha, p, qbuf, sl);
  } else if constexpr (MODE == kMode2D) {
    encode_2d<T>(p.t[t], alpha, p, qbuf, sl);
  } else {
    if (p.two_d_of[t]) encode_2d<T>(p.t[t], alpha, p, qbuf, sl);
    else encode_rows<T, false>(p.t[t], alpha, p, qbuf, qdata, sl);
  }
}

uint64_t max_units(const QBatch& b, int mode) {
  uint64_t units = 0;
  for (int i = 0; i < b.n; ++i) {
    const QTensor& q = b.t[i];
    // 16-blocks (rows), column pairs x 16 rows (cols), threads of 2-tile warps (2D)
    uint64_t u = mode == kModeRows ? (uint64_t)q.rows * (uint64_t)(q.cols / 16)
               : mode == kModeCols ? (uint64_t)(q.cols / 2) * (uint64_t)(q.rows / 16)
                                   : (uint64_t)(q.rows / 16) * (uint64_t)((q.cols / 16 + 1) / 2) * 32;
    units = u > units ? u : units;
  }
  return units;
}

// ------------------------------------------------------------------------
// Dequantization, one 16-block per thread step, all tensors of a batch in
// one launch (tensor = blockIdx.y).
template <bool BF16>
__device__ __forceinline__ void dequant_block(const DQTensor& q, int64_t r, uint32_t kb,
                                              uint32_t kbpr, int sf_layout, uint64_t aa,
                                              int64_t out_row) {
  const uint2 c = __ldg(reinterpret_cast<const uint2*>(q.codes + r * (q.cols >> 1) + (int64_t)kb * 8));
  const float d = e4m3_to_f32(__ldg(q.scales + sf_offset(r, kb, kbpr, sf_layout)));
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
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(q.out) + out_row * q.ldo + (int64_t)kb * 16;
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(dst), "r"(w[0]),
                 "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                 : "memory");
  } else {
    float* dst = static_cast<float*>(q.out) + out_row * q.ldo + (int64_t)kb * 16;
#pragma unroll
    for (int h = 0; h < 2; ++h)
      asm volatile("st.global.v8.f32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(dst + 8 * h),
                   "f"(o[8 * h]), "f"(o[8 * h + 1]), "f"(o[8 * h + 2]), "f"(o[8 * h + 3]),
                   "f"(o[8 * h + 4]), "f"(o[8 * h + 5]), "f"(o[8 * h + 6]), "f"(o[8 * h + 7])
                   : "memory");
  }
}

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
    dequant_block<BF16>(q, r, kb, kbpr, p.sf_layout, aa, r);
  }
}

// Row-gather dequantization: output row o of every tensor is source row
// begin[i] + (o - prefix[i]) for the range i holding o (binary search over
// the merged ranges).
template <bool BF16>
__global__ void __launch_bounds__(kThreads) dequant_rows_kernel(const __grid_constant__ DQGather g) {
  const DQTensor& q = g.b.t[blockIdx.y];
  const float alpha = *q.gs;
  const uint64_t aa = pack2(alpha, alpha);
  const uint32_t kbpr = (uint32_t)(q.cols >> 4);
  const int64_t rows_out = g.prefix[g.n_ranges];
  const uint64_t nblk = (uint64_t)rows_out * kbpr;
  for (uint64_t u = (uint64_t)blockIdx.x * kThreads + threadIdx.x; u < nblk;
       u += (uint64_t)gridDim.x * kThreads) {
    const int64_t o = (int64_t)(u / kbpr);
    const uint32_t kb = (uint32_t)(u - (uint64_t)o * kbpr);
    int lo = 0, hi = g.n_ranges - 1;  // last range with prefix <= o
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (g.prefix[mid] <= o) lo = mid;
      else hi = mid - 1;
    }
    dequant_block<BF16>(q, g.begin[lo] + (o - g.prefix[lo]), kb, kbpr, g.b.sf_layout, aa, o);
  }
}

// ------------------------------------------------------------------------
// Transpose of a 2D (16x16-tile) encoding: the data-gradient GEMM's weight
// operand.  A CTA takes 64 input rows x 256 input columns of codes, and loads
// the next tile's codes and scale bytes while it writes the current one.  Thread
// (i, j) = (t / 32, t % 32) loads the 8 x 8 block of codes at rows
// 8 i .. 8 i + 7, columns 8 j .. 8 j + 7 as eight 32-bit words (a warp reads
// 128 contiguous bytes of one row per load) and transposes it in registers:
// three stages swap 4x4, 2x2 and 1x1 blocks of 4-bit codes with masks and
// shifts, after which word k holds input column 8 j + k with the code of
// input row 8 i + r in nibble r.  The words go through shared memory, and
// four threads write each output row (input column) of the tile: thread q of
// the four writes the 8 bytes of input rows 16 q .. 16 q + 15 and the scale
// byte of that 16 x 16 tile (output block (c, b) takes the tile scale of
// input (16 b, c / 16)), so a warp store covers whole 32-byte sectors of
// eight output rows.  The shared-memory word of (staging row k, output row o)
// sits at column tr_slot(o, k), which keeps both sides free of bank
// conflicts.  rows and cols are multiples of 16.
constexpr int kTrRows = 64, kTrCols = 256;
__device__ __forceinline__ void nib_swap(uint32_t& a, uint32_t& b, int s, uint32_t m) {
  const uint32_t t = ((a >> s) ^ b) & m;
  a ^= t << s;
  b ^= t;
}
__device__ __forceinline__ int tr_slot(int o, int k) {
  const int j = o >> 3;
  return 8 * j + (((o & 7) + j + (j >> 3) + k) & 7);
}
__global__ void __launch_bounds__(kThreads)
    transpose_2d_kernel(const uint8_t* codes, const uint8_t* scales, int sf_in, int64_t rows,
                        int64_t cols, uint8_t* out_codes, uint8_t* out_scales, int sf_out) {
  __shared__ uint32_t t[8][kTrCols];  // [input row block][output row, swizzled]
  const uint32_t tiles_c = (uint32_t)((cols + kTrCols - 1) / kTrCols);
  const uint32_t ntiles = (uint32_t)((rows + kTrRows - 1) / kTrRows) * tiles_c;
  const int i = threadIdx.x >> 5, j = threadIdx.x & 31;
  // write side: per pass of 64 output rows, warp i takes two rows from each
  // of four row groups of eight, so that its 32 reads hit 32 banks
  const int q = j & 3, e = j >> 2;
  const int o_lo = 8 * (4 * (i & 1) + (e & 3)) + 2 * (i >> 1) + (e >> 2);
  const int64_t in_row_bytes = cols >> 1, out_row_bytes = rows >> 1;
  const uint32_t kb_out = (uint32_t)(rows >> 4), kb_in = (uint32_t)(cols >> 4);
  constexpr int kPasses = kTrCols / 64;
  // A tile's global reads, issued one tile ahead: the thread's 8 x 8 block of
  // codes and the scale bytes of the output blocks it writes.
  uint32_t w[8], sc[kPasses];
  auto fetch = [&](uint32_t tile) {
    const uint32_t tr = tile / tiles_c;
    const int64_t r0 = (int64_t)tr * kTrRows, c0 = (int64_t)(tile - tr * tiles_c) * kTrCols;
    const int64_t r = r0 + 8 * i, c = c0 + 8 * j;
    const uint8_t* src = codes + r * in_row_bytes + (c >> 1);
#pragma unroll
    for (int k = 0; k < 8; ++k)
      w[k] = (r + k < rows && c < cols)
                 ? __ldg(reinterpret_cast<const uint32_t*>(src + (int64_t)k * in_row_bytes))
                 : 0u;
    const bool rows_in = 16 * q < rows - r0;
    const uint32_t rb16 = (uint32_t)(r0 + 16 * q);
#pragma unroll
    for (int pass = 0; pass < kPasses; ++pass) {
      const int64_t cc = c0 + 64 * pass + o_lo;
      sc[pass] = (rows_in && cc < cols)
                     ? (uint32_t)__ldg(scales + sf_offset(rb16, (uint32_t)(cc >> 4), kb_in, sf_in))
                     : 0u;
    }
  };
  if (blockIdx.x < ntiles) fetch(blockIdx.x);
  for (uint32_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const uint32_t tr = tile / tiles_c;
    const int64_t r0 = (int64_t)tr * kTrRows, c0 = (int64_t)(tile - tr * tiles_c) * kTrCols;
#pragma unroll
    for (int k = 0; k < 4; ++k) nib_swap(w[k], w[k + 4], 16, 0x0000FFFFu);
    nib_swap(w[0], w[2], 8, 0x00FF00FFu);
    nib_swap(w[1], w[3], 8, 0x00FF00FFu);
    nib_swap(w[4], w[6], 8, 0x00FF00FFu);
    nib_swap(w[5], w[7], 8, 0x00FF00FFu);
#pragma unroll
    for (int k = 0; k < 8; k += 2) nib_swap(w[k], w[k + 1], 4, 0x0F0F0F0Fu);
#pragma unroll
    for (int k = 0; k < 8; ++k) t[i][tr_slot(8 * j + k, i)] = w[k];
    uint32_t s_cur[kPasses];
#pragma unroll
    for (int pass = 0; pass < kPasses; ++pass) s_cur[pass] = sc[pass];
    __syncthreads();
    if (tile + gridDim.x < ntiles) fetch(tile + gridDim.x);  // in flight during the writes
    // 16 input rows = 8 bytes = 2 words; rows - r0 is a multiple of 16
    if (16 * q < rows - r0) {
      const uint32_t rb = (uint32_t)(r0 >> 4) + (uint32_t)q;
      uint8_t* dst = out_codes + (r0 >> 1) + 8 * q;
#pragma unroll
      for (int pass = 0; pass < kPasses; ++pass) {
        const int o = 64 * pass + o_lo;
        const int64_t c = c0 + o;
        if (c < cols) {
          *reinterpret_cast<uint2*>(dst + c * out_row_bytes) =
              make_uint2(t[2 * q][tr_slot(o, 2 * q)], t[2 * q + 1][tr_slot(o, 2 * q + 1)]);
          out_scales[sf_offset((uint32_t)c, rb, kb_out, sf_out)] = (uint8_t)s_cur[pass];
        }
      }
    }
    __syncthreads();
  }
  if (sf_out == 1) zero_sf_padding(out_scales, cols, rows >> 4, Slice{blockIdx.x, gridDim.x});
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

int grid_for(uint64_t work_items, int n_tensors) {
  const uint64_t want = (work_items + kThreads - 1) / kThreads;
  const uint64_t cap = (uint64_t)num_sms() * 8 / (uint64_t)(n_tensors > 0 ? n_tensors : 1);
  uint64_t g = want < cap ? want : cap;
  return (int)(g < 1 ? 1 : g);
}

}  // namespace

int num_sms() {
  static const int n = [] {
    int dev = 0, c = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0)
      c = 148;
    return c;
  }();
  return n;
}

namespace {

template <typename K, typename... Args>
cudaError_t launch_ex(K kern, dim3 grid, cudaStream_t s, bool pdl, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Every tensor of the batch contiguous (ld == cols), 16-byte aligned and with
// whole 32-byte rows of blocks: the bulk-copy amax pass applies.
inline bool flat_bulk_ok(const QBatch& b) {
  for (int i = 0; i < b.n; ++i) {
    const QTensor& q = b.t[i];
    if (q.ld != q.cols || ((uintptr_t)q.x & 15u) || q.rows < 1 || q.cols < 1) return false;
  }
  return true;
}

// The bulk-copy amax pass for element type T (its shared-memory attribute is
// set once per instantiation).
template <typename T>
cudaError_t launch_amax_flat(dim3 grid, cudaStream_t s, const QBatch& b) {
  const int smem_bytes = tma_smem_bytes(kTmaStages);
  static const bool attr_ok =
      cudaFuncSetAttribute(amax_flat_bulk_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem_bytes) == cudaSuccess;
  if (!attr_ok) return cudaErrorNotSupported;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem_bytes;
  cfg.stream = s;
  cfg.attrs = nullptr;
  cfg.numAttrs = 0;
  return cudaLaunchKernelEx(&cfg, amax_flat_bulk_kernel<T>, b);
}

template <typename T, int MODE, bool RHT>
cudaError_t launch_mode(const QBatch& b, cudaStream_t s) {
  const uint64_t units = max_units(b, MODE);
  const uint64_t per_cta = (uint64_t)kThreads;
  int ga = 0;
  if (!b.gs_in && b.amax_ready && !b.amax_only) {
    // the producer of x left per-CTA maxima in every slot of the workspace
    ga = kMaxAmaxCtas;
  } else if (!b.gs_in) {
    // amax pass: three CTAs per SM (eight 32-byte loads in flight per thread)
    uint64_t want = (units + 4 * per_cta - 1) / (4 * per_cta);
    uint64_t cap = (uint64_t)num_sms() * 3;
    if (cap > (uint64_t)kMaxAmaxCtas) cap = kMaxAmaxCtas;
    ga = (int)(want < 1 ? 1 : (want < cap ? want : cap));
    cudaError_t e;
    if (MODE == kModeRows && !RHT && flat_bulk_ok(b)) {
      // contiguous tensors: 16 KB chunks staged by bulk copies
      uint64_t chunks = 0;
      for (int i = 0; i < b.n; ++i) {
        const uint64_t c = ((uint64_t)b.t[i].rows * (uint64_t)b.t[i].cols * sizeof(T) +
                            kTmaTileBytes - 1) / kTmaTileBytes;
        chunks = c > chunks ? c : chunks;
      }
      uint64_t cap_b = (uint64_t)num_sms() * 3 / (uint64_t)b.n;
      if (cap_b > (uint64_t)kMaxAmaxCtas) cap_b = kMaxAmaxCtas;
      if (cap_b < 1) cap_b = 1;
      ga = (int)(chunks < cap_b ? (chunks < 1 ? 1 : chunks) : cap_b);
      e = launch_amax_flat<T>(dim3(ga, b.n), s, b);
    } else {
      e = launch_ex(amax_kernel<T, MODE, RHT>, dim3(ga, b.n), s, false, b);
    }
    if (e != cudaSuccess) return e;
    if (b.amax_only) return launch_ex(finalize_kernel, dim3(b.n), s, true, b, ga);
  }
  // one full wave of resident CTAs across all tensors
  static const int occ = [] {
    int o = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, encode_kernel<T, MODE, RHT>, kThreads,
                                                      0) != cudaSuccess ||
        o < 1)
      o = encode_min_blocks<T, MODE>();
    return o;
  }();
  uint64_t cap = (uint64_t)num_sms() * (uint64_t)occ / (uint64_t)b.n;
  if (cap < 1) cap = 1;
  uint64_t want = (units + per_cta - 1) / per_cta;
  const unsigned gx = (unsigned)(want < 1 ? 1 : (want < cap ? want : cap));
  return launch_ex(encode_kernel<T, MODE, RHT>, dim3(gx, b.n), s, !b.gs_in, b, ga);
}

typedef CUresult (*TensorMapEncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                      const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                      const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                      CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// One 64 x 128 tile map per bf16 tensor of the batch (zero fill past the
// edges); false if the driver refuses one.
bool make_cols_maps(const QBatch& b, ColsMaps& maps) {
  TensorMapEncodeFn fn = (TensorMapEncodeFn)tensor_map_encoder();
  if (!fn) return false;
  for (int i = 0; i < b.n; ++i) {
    const QTensor& q = b.t[i];
    if (q.rows == 0 || q.cols == 0) return false;
    cuuint64_t dims[2] = {(cuuint64_t)q.cols, (cuuint64_t)q.rows};
    cuuint64_t strides[1] = {(cuuint64_t)q.ld * 2};
    cuuint32_t box[2] = {(cuuint32_t)kTmaCols, (cuuint32_t)kTmaRows};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&maps.m[i], CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(q.x), dims, strides,
           box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  return true;
}

template <typename K>
cudaError_t launch_maps(K kern, dim3 grid, cudaStream_t s, bool pdl, const QBatch& b,
                        const ColsMaps& maps, int ga, bool with_ga, int smem_bytes) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem_bytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (with_ga) return cudaLaunchKernelEx(&cfg, (void (*)(QBatch, ColsMaps, int))kern, b, maps, ga);
  return cudaLaunchKernelEx(&cfg, (void (*)(QBatch, ColsMaps))kern, b, maps);
}

// Row-axis quantization of bf16 tensors through the TMA-staged kernels;
// returns cudaErrorNotSupported (nothing launched) when a map cannot be made.
template <bool RHT>
cudaError_t launch_cols_tma(const QBatch& b, cudaStream_t s) {
  ColsMaps maps;  // copied into the launch parameters
  if (!make_cols_maps(b, maps)) return cudaErrorNotSupported;
  static const bool attrs_ok = [] {
    return cudaFuncSetAttribute(amax_cols_tma_kernel<RHT>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                tma_smem_bytes(kTmaStages)) == cudaSuccess &&
           cudaFuncSetAttribute(encode_cols_tma_kernel<RHT>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                tma_smem_bytes(kColsEncStages)) == cudaSuccess;
  }();
  if (!attrs_ok) return cudaErrorNotSupported;
  uint64_t tiles = 0;
  for (int i = 0; i < b.n; ++i) {
    const QTensor& q = b.t[i];
    const uint64_t t = (uint64_t)((q.rows + kTmaRows - 1) / kTmaRows) *
                       (uint64_t)((q.cols + kTmaCols - 1) / kTmaCols);
    tiles = t > tiles ? t : tiles;
  }
  int ga = 0;
  if (!b.gs_in) {
    uint64_t cap = (uint64_t)num_sms() * 3 / (uint64_t)b.n;
    if (cap > (uint64_t)kMaxAmaxCtas) cap = kMaxAmaxCtas;
    if (cap < 1) cap = 1;
    ga = (int)(tiles < cap ? (tiles < 1 ? 1 : tiles) : cap);
    cudaError_t e = launch_maps(amax_cols_tma_kernel<RHT>, dim3(ga, b.n), s, false, b, maps, 0,
                                false, tma_smem_bytes(kTmaStages));
    if (e != cudaSuccess) return e;
    if (b.amax_only) return launch_ex(finalize_kernel, dim3(b.n), s, true, b, ga);
  }
  uint64_t cap = (uint64_t)num_sms() * NVFP4_COLS_MINB / (uint64_t)b.n;
  if (cap < 1) cap = 1;
  const unsigned gx = (unsigned)(tiles < cap ? (tiles < 1 ? 1 : tiles) : cap);
  return launch_maps(encode_cols_tma_kernel<RHT>, dim3(gx, b.n), s, !b.gs_in, b, maps, ga, true,
                     tma_smem_bytes(kColsEncStages));
}

template <typename T>
cudaError_t launch_typed(const QBatch& b, cudaStream_t s) {
  if (b.two_d) return launch_mode<T, kMode2D, false>(b, s);
  if (b.block_axis == 1) {
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
      const cudaError_t e = b.rht ? launch_cols_tma<true>(b, s) : launch_cols_tma<false>(b, s);
      if (e != cudaErrorNotSupported) return e;
    }
    return b.rht ? launch_mode<T, kModeCols, true>(b, s) : launch_mode<T, kModeCols, false>(b, s);
  }
  return b.rht ? launch_mode<T, kModeRows, true>(b, s) : launch_mode<T, kModeRows, false>(b, s);
}

}  // namespace

cudaError_t launch_quantize(const QBatch& b, cudaStream_t s) {
  return b.bf16 ? launch_typed<__nv_bfloat16>(b, s) : launch_typed<float>(b, s);
}

namespace {

// Splits `total` CTAs between the tensors in proportion to weight[i], each
// at least 1 and at most cap[i]; writes the ranges' ends, returns the sum.
int32_t split_ctas(const double* weight, const uint64_t* cap, int n, uint64_t total,
                   int32_t* end) {
  double w = 0.0;
  for (int i = 0; i < n; ++i) w += weight[i];
  int32_t acc = 0;
  for (int i = 0; i < n; ++i) {
    uint64_t g = (uint64_t)((double)total * weight[i] / (w > 0.0 ? w : 1.0));
    if (g > cap[i]) g = cap[i];
    if (g < 1) g = 1;
    acc += (int32_t)g;
    end[i] = acc;
  }
  return acc;
}

template <typename T>
cudaError_t launch_mixed_typed(QBatch& b, cudaStream_t s) {
  double wa[kMaxBatch], we[kMaxBatch];
  uint64_t ca[kMaxBatch], ce[kMaxBatch];
  for (int i = 0; i < b.n; ++i) {
    const QTensor& q = b.t[i];
    const uint64_t blocks = (uint64_t)q.rows * (uint64_t)(q.cols / 16);
    const uint64_t units = b.two_d_of[i] ? (uint64_t)(q.rows / 16) * (uint64_t)((q.cols / 16 + 1) / 2) * 32
                                          : blocks;
    wa[i] = (double)blocks;
    // the tile encoder spends about 1.2x the row encoder's instructions per element
    we[i] = (double)blocks * (b.two_d_of[i] ? 1.2 : 1.0);
    ca[i] = (blocks + 4 * kThreads - 1) / (4 * kThreads);
    if (ca[i] > (uint64_t)kMaxAmaxCtas) ca[i] = kMaxAmaxCtas;
    ce[i] = (units + kThreads - 1) / kThreads;
  }
  static const int occ = [] {
    int o = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, encode_kernel<T, kModeMixed, false>,
                                                      kThreads, 0) != cudaSuccess ||
        o < 1)
      o = encode_min_blocks<T, kModeMixed>();
    return o;
  }();
  const int32_t ga = split_ctas(wa, ca, b.n, (uint64_t)num_sms() * 3, b.amax_end);
  const int32_t ge = split_ctas(we, ce, b.n, (uint64_t)num_sms() * (uint64_t)occ, b.enc_end);
  cudaError_t e = launch_ex(amax_kernel<T, kModeMixed, false>, dim3(ga), s, false, b);
  if (e != cudaSuccess) return e;
  return launch_ex(encode_kernel<T, kModeMixed, false>, dim3(ge), s, true, b, 0);
}

}  // namespace

cudaError_t launch_quantize_mixed(QBatch& b, cudaStream_t s) {
  return b.bf16 ? launch_mixed_typed<__nv_bfloat16>(b, s) : launch_mixed_typed<float>(b, s);
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

cudaError_t launch_dequantize_rows(const DQGather& g, cudaStream_t s) {
  const uint64_t m = (uint64_t)g.prefix[g.n_ranges] * (uint64_t)(g.b.t[0].cols / 16);
  uint64_t mx = m;
  for (int i = 1; i < g.b.n; ++i) {
    const uint64_t u = (uint64_t)g.prefix[g.n_ranges] * (uint64_t)(g.b.t[i].cols / 16);
    mx = u > mx ? u : mx;
  }
  dim3 grid(grid_for(mx, g.b.n), g.b.n);
  if (g.b.out_bf16)
    dequant_rows_kernel<true><<<grid, kThreads, 0, s>>>(g);
  else
    dequant_rows_kernel<false><<<grid, kThreads, 0, s>>>(g);
  return cudaGetLastError();
}

cudaError_t launch_transpose_2d(const uint8_t* codes, const uint8_t* scales, int sf_in,
                                int64_t rows, int64_t cols, uint8_t* out_codes,
                                uint8_t* out_scales, int sf_out, cudaStream_t s) {
  const uint64_t tiles = (uint64_t)((rows + kTrRows - 1) / kTrRows) *
                         (uint64_t)((cols + kTrCols - 1) / kTrCols);
  // one wave of resident CTAs, each looping over tiles (its next tile's loads
  // overlap its current tile's stores)
  static const int per_sm = [] {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, transpose_2d_kernel, kThreads, 0) !=
            cudaSuccess ||
        n < 1)
      n = 4;
    return n;
  }();
  const uint64_t cap = (uint64_t)num_sms() * (uint64_t)per_sm;
  const int grid = (int)(tiles < cap ? (tiles < 1 ? 1 : tiles) : cap);
  transpose_2d_kernel<<<grid, kThreads, 0, s>>>(codes, scales, sf_in, rows, cols, out_codes,
                                               out_scales, sf_out);
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


}  // namespace nvfp4
