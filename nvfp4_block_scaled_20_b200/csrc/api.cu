// C ABI of the NVFP4 library (declared in include/nvfp4.h): argument
// validation on the host, workspace carve-up, kernel launches.  Nothing here
// allocates device memory or synchronizes (except nvfp4_get_device_error).
#include <algorithm>
#include <atomic>
#include <cstring>
#include <memory>
#include <vector>

#include "../../include/nvfp4.h"
#include "kernels.h"

using namespace nvfp4;

namespace {

constexpr size_t kErrWordBytes = 256;  // error word, padded
inline bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }
inline int64_t elem_bytes(int32_t dt) { return dt == NVFP4_BF16 ? 2 : 4; }
inline bool dtype_ok(int32_t dt) { return dt == NVFP4_F32 || dt == NVFP4_BF16; }
inline cudaStream_t S(void* s) { return static_cast<cudaStream_t>(s); }

// Workspace layout: [0, 4) device error word, then kMaxAmaxCtas fp32
// partial maxima per tensor from 256 on.  Nothing in it needs clearing.
uint32_t* err_word(void* ws) { return static_cast<uint32_t*>(ws); }
// nvfp4_gemm's partial-sum slabs (the split last round) follow the error word
// and one tensor's amax partials, 1 KB aligned; one slab is an fp32 256 x 256
// tile.
constexpr size_t kSlabOffset = (kErrWordBytes + kMaxAmaxCtas * sizeof(float) + 1023) / 1024 * 1024;
constexpr size_t kSlabBytes = 256 * 256 * sizeof(float);
float* partials(void* ws) {
  return reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kErrWordBytes);
}

// Shape / alignment rules of one quantizer input.
nvfp4_status check_input(const void* x, int32_t dtype, int64_t rows, int64_t cols, int64_t ld,
                         int block_axis, bool two_d) {
  if (!dtype_ok(dtype)) return NVFP4_ERR_INVALID_ARG;
  if (rows < 0 || cols < 0 || ld < cols) return NVFP4_ERR_SHAPE;
  if (!x && rows > 0 && cols > 0) return NVFP4_ERR_INVALID_ARG;
  if (block_axis == 0 && cols % 16) return NVFP4_ERR_SHAPE;
  if ((block_axis == 1 || two_d) && rows % 16) return NVFP4_ERR_SHAPE;
  if (two_d && cols % 16) return NVFP4_ERR_SHAPE;
  if (block_axis == 1 && cols % 8) return NVFP4_ERR_SHAPE;
  // the kernels index blocks with 32-bit integers
  if ((double)rows * (double)cols / 16.0 >= 4.0e9) return NVFP4_ERR_SHAPE;
  // contiguous 16-blocks are read with 256-bit loads: 32-byte aligned rows;
  // the row-axis path reads element pairs: 16-byte aligned rows suffice
  const size_t need = (block_axis == 0 || two_d) ? 32 : 16;
  if (!aligned(x, need) || (ld * elem_bytes(dtype)) % (int64_t)need) return NVFP4_ERR_ALIGN;
  return NVFP4_OK;
}

nvfp4_status check_qparams(const nvfp4_qparams* qp, bool two_d) {
  if (!qp) return NVFP4_ERR_INVALID_ARG;
  if (qp->block_axis != 0 && qp->block_axis != 1) return NVFP4_ERR_INVALID_ARG;
  if (qp->sf_layout != NVFP4_SF_ROWMAJOR && qp->sf_layout != NVFP4_SF_TCGEN05)
    return NVFP4_ERR_INVALID_ARG;
  if (two_d && (qp->rht_enable || qp->block_axis != 0)) return NVFP4_ERR_INVALID_ARG;
  // a producer's amax is of the untransformed values
  if (qp->amax_from_workspace != 0 && qp->amax_from_workspace != 1) return NVFP4_ERR_INVALID_ARG;
  if (qp->amax_from_workspace && qp->rht_enable) return NVFP4_ERR_INVALID_ARG;
  if (qp->global_scale_in && !aligned(qp->global_scale_in, 4)) return NVFP4_ERR_ALIGN;
  return NVFP4_OK;
}

void fill_batch_common(QBatch& b, int32_t dtype, const nvfp4_qparams* qp, void* ws) {
  std::memset(&b, 0, sizeof(b));
  b.bf16 = dtype == NVFP4_BF16;
  b.four_over_six = qp->four_over_six != 0;
  b.rht = qp->rht_enable != 0;
  b.mask = qp->rht_sign_mask;
  b.block_axis = qp->block_axis;
  b.sf_layout = qp->sf_layout;
  b.gs_in = qp->global_scale_in;
  b.amax_ready = qp->amax_from_workspace != 0;
  b.partials = ws ? partials(ws) : nullptr;
  b.err = ws ? err_word(ws) : nullptr;
}

nvfp4_status cuda_status(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

std::atomic<uint64_t> g_wait_limit_ns{0};  // 0: kDefaultWaitLimitNs
std::atomic<int32_t> g_test_stall{0};

}  // namespace

uint64_t nvfp4::gemm_wait_limit_ns() {
  const uint64_t v = g_wait_limit_ns.load();
  return v ? v : kDefaultWaitLimitNs;
}

int32_t nvfp4::gemm_test_stall() { return g_test_stall.load(); }

namespace {

nvfp4_status quantize_common(const void* x, int32_t dtype, int64_t rows, int64_t cols, int64_t ld,
                             const nvfp4_qparams* qp, uint8_t* codes, uint8_t* scales,
                             float* gs_out, void* ws, size_t ws_bytes, void* stream, bool two_d) {
  nvfp4_status st = check_qparams(qp, two_d);
  if (st != NVFP4_OK) return st;
  st = check_input(x, dtype, rows, cols, ld, qp->block_axis, two_d);
  if (st != NVFP4_OK) return st;
  if (rows == 0 || cols == 0) return NVFP4_OK;  // empty: nothing to read or write
  if (!codes || !scales || !gs_out) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(codes, 16) || !aligned(scales, 4) || !aligned(gs_out, 4)) return NVFP4_ERR_ALIGN;
  if (!ws || ws_bytes < nvfp4_workspace_bytes(1)) return NVFP4_ERR_WORKSPACE;
  QBatch b;
  fill_batch_common(b, dtype, qp, ws);
  b.two_d = two_d ? 1 : 0;
  b.n = 1;
  b.t[0] = QTensor{x, codes, scales, gs_out, rows, cols, ld};
  return cuda_status(launch_quantize(b, S(stream)));
}

}  // namespace

extern "C" {

size_t nvfp4_workspace_bytes(int32_t n_tensors) {
  if (n_tensors < 0) n_tensors = 0;
  return kErrWordBytes + (size_t)n_tensors * kMaxAmaxCtas * sizeof(float);
}

int64_t nvfp4_codes_bytes(int64_t rows, int64_t cols) { return rows * cols / 2; }

int64_t nvfp4_scales_bytes(int64_t rows, int64_t cols, int32_t sf_layout) {
  const int64_t kb = cols / 16;
  if (sf_layout == NVFP4_SF_TCGEN05) return (rows + 127) / 128 * 128 * ((kb + 3) / 4) * 4;
  return rows * kb;
}

nvfp4_status nvfp4_global_scale(const void* x, int32_t dtype, int64_t rows, int64_t cols,
                                int64_t ld, const nvfp4_qparams* qp, float* global_scale_out,
                                void* ws, size_t ws_bytes, void* stream) {
  nvfp4_status st = check_qparams(qp, false);
  if (st != NVFP4_OK) return st;
  st = check_input(x, dtype, rows, cols, ld, qp->block_axis, false);
  if (st != NVFP4_OK) return st;
  if (!global_scale_out) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(global_scale_out, 4)) return NVFP4_ERR_ALIGN;
  if (!ws || ws_bytes < nvfp4_workspace_bytes(1)) return NVFP4_ERR_WORKSPACE;
  QBatch b;
  fill_batch_common(b, dtype, qp, ws);
  b.gs_in = nullptr;
  b.amax_ready = 0;  // this call is the amax pass
  b.amax_only = 1;
  b.n = 1;
  b.t[0] = QTensor{x, nullptr, nullptr, global_scale_out, rows, cols, ld};
  // an empty tensor runs the same two kernels: amax 0, global scale 1
  return cuda_status(launch_quantize(b, S(stream)));
}

nvfp4_status nvfp4_quantize_1d(const void* x, int32_t dtype, int64_t rows, int64_t cols,
                               int64_t ld, const nvfp4_qparams* qp, uint8_t* codes,
                               uint8_t* scales, float* global_scale_out, void* ws,
                               size_t ws_bytes, void* stream) {
  return quantize_common(x, dtype, rows, cols, ld, qp, codes, scales, global_scale_out, ws,
                         ws_bytes, stream, false);
}

nvfp4_status nvfp4_quantize_2d(const void* x, int32_t dtype, int64_t rows, int64_t cols,
                               int64_t ld, const nvfp4_qparams* qp, uint8_t* codes,
                               uint8_t* scales, float* global_scale_out, void* ws,
                               size_t ws_bytes, void* stream) {
  return quantize_common(x, dtype, rows, cols, ld, qp, codes, scales, global_scale_out, ws,
                         ws_bytes, stream, true);
}

nvfp4_status nvfp4_quantize_1d_batched(const nvfp4_tensor_desc* descs, int32_t n, int32_t dtype,
                                       const nvfp4_qparams* qp, void* ws, size_t ws_bytes,
                                       void* stream) {
  if (!descs || n < 0) return NVFP4_ERR_INVALID_ARG;
  nvfp4_status st = check_qparams(qp, false);
  if (st != NVFP4_OK) return st;
  if (qp->global_scale_in || qp->amax_from_workspace) return NVFP4_ERR_INVALID_ARG;
  if (!dtype_ok(dtype)) return NVFP4_ERR_INVALID_ARG;
  for (int32_t i = 0; i < n; ++i) {
    const nvfp4_tensor_desc& d = descs[i];
    st = check_input(d.x, dtype, d.rows, d.cols, d.ld, qp->block_axis, false);
    if (st != NVFP4_OK) return st;
    if (!d.codes || !d.scales || !d.global_scale) return NVFP4_ERR_INVALID_ARG;
    if (!aligned(d.codes, 16) || !aligned(d.scales, 4) || !aligned(d.global_scale, 4))
      return NVFP4_ERR_ALIGN;
  }
  if (!ws || ws_bytes < nvfp4_workspace_bytes(n)) return NVFP4_ERR_WORKSPACE;
  if (n == 0) return NVFP4_OK;
  for (int32_t base = 0; base < n; base += kMaxBatch) {
    QBatch b;
    fill_batch_common(b, dtype, qp, ws);
    b.partials = partials(ws) + (size_t)base * kMaxAmaxCtas;
    b.n = (n - base) < kMaxBatch ? (n - base) : kMaxBatch;
    for (int32_t i = 0; i < b.n; ++i) {
      const nvfp4_tensor_desc& d = descs[base + i];
      b.t[i] = QTensor{d.x, d.codes, d.scales, d.global_scale, d.rows, d.cols, d.ld};
    }
    if (launch_quantize(b, S(stream)) != cudaSuccess) return NVFP4_ERR_CUDA;
  }
  return NVFP4_OK;
}

nvfp4_status nvfp4_quantize_mixed(const nvfp4_tensor_desc* descs, const int32_t* two_d,
                                  int32_t n, int32_t dtype, const nvfp4_qparams* qp, void* ws,
                                  size_t ws_bytes, void* stream) {
  if (!descs || !two_d || n < 0) return NVFP4_ERR_INVALID_ARG;
  if (n > kMaxBatch) return NVFP4_ERR_SHAPE;
  nvfp4_status st = check_qparams(qp, true);  // block_axis 0, no RHT
  if (st != NVFP4_OK) return st;
  if (qp->global_scale_in || qp->amax_from_workspace) return NVFP4_ERR_INVALID_ARG;
  if (!dtype_ok(dtype)) return NVFP4_ERR_INVALID_ARG;
  for (int32_t i = 0; i < n; ++i) {
    const nvfp4_tensor_desc& d = descs[i];
    if (two_d[i] != 0 && two_d[i] != 1) return NVFP4_ERR_INVALID_ARG;
    st = check_input(d.x, dtype, d.rows, d.cols, d.ld, 0, two_d[i] != 0);
    if (st != NVFP4_OK) return st;
    // an empty tensor only receives its global scale (1.0)
    const bool empty = d.rows == 0 || d.cols == 0;
    if ((!empty && (!d.codes || !d.scales)) || !d.global_scale) return NVFP4_ERR_INVALID_ARG;
    if (!aligned(d.codes, 16) || !aligned(d.scales, 4) || !aligned(d.global_scale, 4))
      return NVFP4_ERR_ALIGN;
  }
  if (!ws || ws_bytes < nvfp4_workspace_bytes(n)) return NVFP4_ERR_WORKSPACE;
  if (n == 0) return NVFP4_OK;
  QBatch b;
  fill_batch_common(b, dtype, qp, ws);
  b.n = n;
  for (int32_t i = 0; i < n; ++i) {
    const nvfp4_tensor_desc& d = descs[i];
    b.t[i] = QTensor{d.x, d.codes, d.scales, d.global_scale, d.rows, d.cols, d.ld};
    b.two_d_of[i] = (int8_t)two_d[i];
  }
  return cuda_status(launch_quantize_mixed(b, S(stream)));
}

nvfp4_status nvfp4_dequantize(const nvfp4_tensor_desc* descs, int32_t n, int32_t out_dtype,
                              int32_t sf_layout, void* stream) {
  if (!descs || n < 0 || !dtype_ok(out_dtype)) return NVFP4_ERR_INVALID_ARG;
  if (sf_layout != NVFP4_SF_ROWMAJOR && sf_layout != NVFP4_SF_TCGEN05) return NVFP4_ERR_INVALID_ARG;
  for (int32_t i = 0; i < n; ++i) {
    const nvfp4_tensor_desc& d = descs[i];
    if (!d.codes || !d.scales || !d.global_scale || !d.out) return NVFP4_ERR_INVALID_ARG;
    if (d.rows < 0 || d.cols < 0 || d.cols % 16 || d.ld < d.cols) return NVFP4_ERR_SHAPE;
    if ((double)d.rows * (double)d.cols / 16.0 >= 4.0e9) return NVFP4_ERR_SHAPE;
    if (!aligned(d.codes, 8) || !aligned(d.out, 32) || (d.ld * elem_bytes(out_dtype)) % 32)
      return NVFP4_ERR_ALIGN;
  }
  for (int32_t base = 0; base < n; base += kMaxBatch) {
    DQBatch b;
    std::memset(&b, 0, sizeof(b));
    b.out_bf16 = out_dtype == NVFP4_BF16;
    b.sf_layout = sf_layout;
    b.n = 0;
    for (int32_t i = base; i < n && i < base + kMaxBatch; ++i) {
      const nvfp4_tensor_desc& d = descs[i];
      if (d.rows == 0 || d.cols == 0) continue;
      b.t[b.n++] = DQTensor{d.codes, d.scales, d.global_scale, d.out, d.rows, d.cols, d.ld};
    }
    if (b.n == 0) continue;
    cudaError_t e = launch_dequantize(b, S(stream));
    if (e != cudaSuccess) return NVFP4_ERR_CUDA;
  }
  return NVFP4_OK;
}

nvfp4_status nvfp4_dequantize_rows(const nvfp4_tensor_desc* descs, int32_t n,
                                   const int64_t* row_ranges, int32_t n_ranges,
                                   int32_t out_dtype, int32_t sf_layout, void* stream) {
  if (!descs || n < 0 || n_ranges < 0 || (n_ranges > 0 && !row_ranges) || !dtype_ok(out_dtype))
    return NVFP4_ERR_INVALID_ARG;
  if (sf_layout != NVFP4_SF_ROWMAJOR && sf_layout != NVFP4_SF_TCGEN05) return NVFP4_ERR_INVALID_ARG;
  if (n_ranges > kMaxRowRanges) return NVFP4_ERR_SHAPE;
  // merge: sort by begin, join overlapping and touching ranges, drop empty ones
  std::vector<std::pair<int64_t, int64_t>> r;
  for (int32_t i = 0; i < n_ranges; ++i) {
    const int64_t b = row_ranges[2 * i], e = row_ranges[2 * i + 1];
    if (b < 0 || e < b) return NVFP4_ERR_SHAPE;
    if (e > b) r.emplace_back(b, e);
  }
  std::sort(r.begin(), r.end());
  std::vector<std::pair<int64_t, int64_t>> m;
  for (const auto& x : r) {
    if (!m.empty() && x.first <= m.back().second) m.back().second = std::max(m.back().second, x.second);
    else m.push_back(x);
  }
  const int64_t last = m.empty() ? 0 : m.back().second;
  for (int32_t i = 0; i < n; ++i) {
    const nvfp4_tensor_desc& d = descs[i];
    if (!d.codes || !d.scales || !d.global_scale || !d.out) return NVFP4_ERR_INVALID_ARG;
    if (d.rows < 0 || d.cols < 0 || d.cols % 16 || d.ld < d.cols || last > d.rows)
      return NVFP4_ERR_SHAPE;
    if ((double)d.rows * (double)d.cols / 16.0 >= 4.0e9) return NVFP4_ERR_SHAPE;
    if (!aligned(d.codes, 8) || !aligned(d.out, 32) || (d.ld * elem_bytes(out_dtype)) % 32)
      return NVFP4_ERR_ALIGN;
  }
  if (m.empty() || n == 0) return NVFP4_OK;
  // large (about 24 KB): kept off the host stack
  std::unique_ptr<DQGather> g(new DQGather);
  std::memset(g.get(), 0, sizeof(DQGather));
  g->n_ranges = (int32_t)m.size();
  g->prefix[0] = 0;
  for (size_t i = 0; i < m.size(); ++i) {
    g->begin[i] = m[i].first;
    g->prefix[i + 1] = g->prefix[i] + (m[i].second - m[i].first);
  }
  g->b.out_bf16 = out_dtype == NVFP4_BF16;
  g->b.sf_layout = sf_layout;
  for (int32_t base = 0; base < n; base += kMaxBatch) {
    g->b.n = 0;
    for (int32_t i = base; i < n && i < base + kMaxBatch; ++i) {
      const nvfp4_tensor_desc& d = descs[i];
      if (d.cols == 0) continue;
      g->b.t[g->b.n++] = DQTensor{d.codes, d.scales, d.global_scale, d.out, d.rows, d.cols, d.ld};
    }
    if (g->b.n == 0) continue;
    cudaError_t e = launch_dequantize_rows(*g, S(stream));
    if (e != cudaSuccess) return NVFP4_ERR_CUDA;
  }
  return NVFP4_OK;
}

nvfp4_status nvfp4_transpose_2d(const uint8_t* codes, const uint8_t* scales,
                                int32_t sf_layout_in, int64_t rows, int64_t cols,
                                uint8_t* out_codes, uint8_t* out_scales, int32_t sf_layout_out,
                                void* stream) {
  auto layout_ok = [](int32_t l) { return l == NVFP4_SF_ROWMAJOR || l == NVFP4_SF_TCGEN05; };
  if (!layout_ok(sf_layout_in) || !layout_ok(sf_layout_out)) return NVFP4_ERR_INVALID_ARG;
  if (rows < 0 || cols < 0 || rows % 16 || cols % 16) return NVFP4_ERR_SHAPE;
  if ((double)rows * (double)cols / 16.0 >= 4.0e9) return NVFP4_ERR_SHAPE;
  if (rows == 0 || cols == 0) return NVFP4_OK;
  if (!codes || !scales || !out_codes || !out_scales) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(codes, 8) || !aligned(out_codes, 8)) return NVFP4_ERR_ALIGN;
  return cuda_status(launch_transpose_2d(codes, scales, sf_layout_in, rows, cols, out_codes,
                                         out_scales, sf_layout_out, S(stream)));
}

namespace {
nvfp4_status gemm_common(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_alpha,
                         const uint8_t* b_codes, const uint8_t* b_sf, const float* b_alpha,
                         int64_t M, int64_t N, int64_t K, void* out, int32_t out_dtype,
                         int64_t ldo, int32_t epilogue, void* ws, size_t ws_bytes, void* stream,
                         const GemmArgs* lora);
}  // namespace

nvfp4_status nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_alpha,
                        const uint8_t* b_codes, const uint8_t* b_sf, const float* b_alpha,
                        int64_t M, int64_t N, int64_t K, void* out, int32_t out_dtype, int64_t ldo,
                        int32_t epilogue, void* ws, size_t ws_bytes, void* stream) {
  return gemm_common(a_codes, a_sf, a_alpha, b_codes, b_sf, b_alpha, M, N, K, out, out_dtype, ldo,
                     epilogue, ws, ws_bytes, stream, nullptr);
}

size_t nvfp4_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t epilogue) {
  const size_t base = nvfp4_workspace_bytes((epilogue & NVFP4_EPI_AMAX) ? 1 : 0);
  const int64_t slabs = gemm_split_slabs(M, N, K, epilogue);
  return slabs > 0 ? kSlabOffset + (size_t)slabs * kSlabBytes : base;
}

size_t nvfp4_lora_scratch_bytes(int64_t M, int64_t rank) {
  return (M > 0 && rank > 0) ? (size_t)M * (size_t)rank * 4u : 0u;
}

nvfp4_status nvfp4_gemm_lora(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_alpha,
                             const uint8_t* b_codes, const uint8_t* b_sf, const float* b_alpha,
                             int64_t M, int64_t N, int64_t K, const void* lora_u, int64_t ldu,
                             const void* lora_b, int64_t ldl, int64_t rank, float lora_scale,
                             void* scratch, size_t scratch_bytes, void* out, int32_t out_dtype,
                             int64_t ldo, int32_t epilogue, void* ws, size_t ws_bytes,
                             void* stream) {
  if (!lora_u || !lora_b || !scratch) return NVFP4_ERR_INVALID_ARG;
  if (rank < 64 || rank > 1024 || rank % 64 || ldu < rank || ldl < rank) return NVFP4_ERR_SHAPE;
  if (!(lora_scale == lora_scale) || lora_scale > 3.0e38f || lora_scale < -3.0e38f)
    return NVFP4_ERR_INVALID_ARG;  // finite scale
  if (!aligned(lora_u, 16) || !aligned(lora_b, 16) || !aligned(scratch, 16) || (ldu * 2) % 16 ||
      (ldl * 2) % 16)
    return NVFP4_ERR_ALIGN;
  if (scratch_bytes < nvfp4_lora_scratch_bytes(M, rank)) return NVFP4_ERR_WORKSPACE;
  GemmArgs l{};
  l.lora_u = lora_u;
  l.lora_b = lora_b;
  l.ldu = ldu;
  l.ldl = ldl;
  l.rank = rank;
  l.lora_scale = lora_scale;
  l.u_scaled = scratch;
  return gemm_common(a_codes, a_sf, a_alpha, b_codes, b_sf, b_alpha, M, N, K, out, out_dtype, ldo,
                     epilogue, ws, ws_bytes, stream, &l);
}

}  // extern "C"

namespace {
nvfp4_status gemm_common(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_alpha,
                         const uint8_t* b_codes, const uint8_t* b_sf, const float* b_alpha,
                         int64_t M, int64_t N, int64_t K, void* out, int32_t out_dtype,
                         int64_t ldo, int32_t epilogue, void* ws, size_t ws_bytes, void* stream,
                         const GemmArgs* lora) {
  if (!a_codes || !a_sf || !a_alpha || !b_codes || !b_sf || !b_alpha || !out)
    return NVFP4_ERR_INVALID_ARG;
  if (!dtype_ok(out_dtype)) return NVFP4_ERR_INVALID_ARG;
  const int32_t act = epilogue & ~NVFP4_EPI_AMAX;
  if (act != NVFP4_EPI_NONE && act != NVFP4_EPI_GELU_TANH) return NVFP4_ERR_INVALID_ARG;
  if (M < 1 || N < 16 || K < 64 || N % 16 || K % 64 || ldo < N) return NVFP4_ERR_SHAPE;
  if (!aligned(a_codes, 16) || !aligned(b_codes, 16) || !aligned(a_sf, 16) || !aligned(b_sf, 16) ||
      !aligned(out, 16) || (ldo * elem_bytes(out_dtype)) % 16 || !aligned(a_alpha, 4) ||
      !aligned(b_alpha, 4))
    return NVFP4_ERR_ALIGN;
  const bool want_amax = (epilogue & NVFP4_EPI_AMAX) != 0;
  if (!ws || ws_bytes < nvfp4_workspace_bytes(want_amax ? 1 : 0)) return NVFP4_ERR_WORKSPACE;
  GemmArgs g;
  g.a_codes = a_codes;
  g.a_sf = a_sf;
  g.a_alpha = a_alpha;
  g.b_codes = b_codes;
  g.b_sf = b_sf;
  g.b_alpha = b_alpha;
  g.M = M;
  g.N = N;
  g.K = K;
  g.out = out;
  g.out_bf16 = out_dtype == NVFP4_BF16;
  g.ldo = ldo;
  g.epilogue = epilogue;
  g.err = err_word(ws);
  g.amax_partials = want_amax ? partials(ws) : nullptr;
  g.wait_limit_ns = gemm_wait_limit_ns();
  g.stall = gemm_test_stall();
  g.lora_u = nullptr;
  g.lora_b = nullptr;
  g.rank = 0;
  g.u_scaled = nullptr;
  g.slabs = nullptr;
  g.slab_cap = 0;
  if (!lora && ws_bytes >= kSlabOffset + kSlabBytes && aligned(ws, 16)) {
    g.slabs = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kSlabOffset);
    g.slab_cap = (int64_t)((ws_bytes - kSlabOffset) / kSlabBytes);
  }
  if (lora) {
    g.lora_u = lora->lora_u;
    g.lora_b = lora->lora_b;
    g.ldu = lora->ldu;
    g.ldl = lora->ldl;
    g.rank = lora->rank;
    g.lora_scale = lora->lora_scale;
    g.u_scaled = lora->u_scaled;
  }
  bool unsupported = false;
  int e = launch_gemm(g, S(stream), &unsupported);
  if (unsupported) return NVFP4_ERR_UNSUPPORTED;
  return e == 0 ? NVFP4_OK : NVFP4_ERR_CUDA;
}
}  // namespace

extern "C" {

nvfp4_status nvfp4_rht16(const void* x, int32_t dtype, int64_t rows, int64_t cols, int64_t ld,
                         int32_t block_axis, uint32_t sign_mask, float* out, void* stream) {
  if (!x || !out || !dtype_ok(dtype)) return NVFP4_ERR_INVALID_ARG;
  if (block_axis != 0 && block_axis != 1) return NVFP4_ERR_INVALID_ARG;
  if (rows < 0 || cols < 0 || ld < cols) return NVFP4_ERR_SHAPE;
  if ((block_axis == 0 && cols % 16) || (block_axis == 1 && rows % 16)) return NVFP4_ERR_SHAPE;
  if (!aligned(x, (size_t)elem_bytes(dtype)) || !aligned(out, 4)) return NVFP4_ERR_ALIGN;
  if (rows == 0 || cols == 0) return NVFP4_OK;
  return cuda_status(launch_rht16(x, dtype == NVFP4_BF16, rows, cols, ld, block_axis, sign_mask,
                                  out, S(stream)));
}

nvfp4_status nvfp4_set_wait_limit(uint64_t ns) {
  g_wait_limit_ns.store(ns);
  return NVFP4_OK;
}

nvfp4_status nvfp4_set_test_stall(int32_t on) {
  if (on != 0 && on != 1) return NVFP4_ERR_INVALID_ARG;
  g_test_stall.store(on);
  return NVFP4_OK;
}

nvfp4_status nvfp4_convert_sweep(int32_t target, uint32_t first_bits, int64_t count,
                                 uint8_t* out, void* stream) {
  if (target != 0 && target != 1) return NVFP4_ERR_INVALID_ARG;
  if (count < 0 || (uint64_t)first_bits + (uint64_t)count > (1ull << 32)) return NVFP4_ERR_SHAPE;
  if (count == 0) return NVFP4_OK;
  if (!out) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(out, 16)) return NVFP4_ERR_ALIGN;
  return cuda_status(launch_convert_sweep(target, first_bits, (uint64_t)count, out, S(stream)));
}

nvfp4_status nvfp4_get_device_error(void* ws, int32_t* error_out, void* stream) {
  if (!ws || !error_out) return NVFP4_ERR_INVALID_ARG;
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, S(stream)) != cudaSuccess)
    return NVFP4_ERR_CUDA;
  if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return NVFP4_ERR_CUDA;
  *error_out = (int32_t)v;
  if (v != 0 && cudaMemsetAsync(ws, 0, sizeof(v), S(stream)) != cudaSuccess) return NVFP4_ERR_CUDA;
  return NVFP4_OK;
}

const char* nvfp4_status_string(int32_t s) {
  switch (s) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_SHAPE: return "shape violates the call's rules";
    case NVFP4_ERR_ALIGN: return "pointer or leading dimension misaligned";
    case NVFP4_ERR_WORKSPACE: return "workspace missing or too small";
    case NVFP4_ERR_CUDA: return "CUDA call failed";
    case NVFP4_ERR_TIMEOUT: return "bounded device wait timed out";
    case NVFP4_ERR_UNSUPPORTED: return "not supported by this library";
    default: return "unknown status";
  }
}

}  // extern "C"
