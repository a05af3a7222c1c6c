// Batched 1D quantization that needs no workspace from the caller.
//
// Some callers cannot hand the library any device memory beyond the tensors
// themselves: a plugin running inside another framework whose allocator owns
// every device byte and forbids side allocations, code that must not call
// cudaMalloc because it would synchronize the device in the middle of a
// latency-critical loop, or a C caller that only holds the raw pointers of its
// tensors.  For them the per-tensor scratch of the amax pass (one partial
// maximum per amax CTA) lives in the fixed array below, which is part of the
// library's device image: every GPU that loads the library holds its
// 4 * (64 + kNoAllocMaxTensors * kMaxAmaxCtas) = 114,944 bytes (~115 KB) until
// exit.
#include <cstring>
#include <mutex>

#include "../../include/nvfp4.h"
#include "kernels.h"

namespace {

constexpr int kNoAllocMaxTensors = 64;
constexpr int kMaxDevices = 64;

// [0] device error word; from [64] on, kMaxAmaxCtas partial maxima (fp32
// bits) per tensor of a call.  Every slot a call reads it has written in the
// same call, so nothing needs clearing.
static __device__ __align__(256) uint32_t g_noalloc_amax[64 + kNoAllocMaxTensors * nvfp4::kMaxAmaxCtas];
static_assert(sizeof(g_noalloc_amax) == 114944, "scratch size stated in the header");

std::mutex g_mu;
uint32_t* g_addr[kMaxDevices] = {};

// Device address of g_noalloc_amax on the current device, looked up once per
// device (host code only sees a stand-in for the array, never its address).
nvfp4_status scratch_address(uint32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_amax) != cudaSuccess || !p) return NVFP4_ERR_CUDA;
    g_addr[dev] = static_cast<uint32_t*>(p);
  }
  *out = g_addr[dev];
  return NVFP4_OK;
}

inline bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

}  // namespace

extern "C" nvfp4_status nvfp4_quantize_1d_batched_noalloc(const nvfp4_tensor_desc* descs,
                                                          int32_t n, int32_t dtype,
                                                          const nvfp4_qparams* qp, void* stream) {
  using namespace nvfp4;
  if (!descs || !qp || n < 0) return NVFP4_ERR_INVALID_ARG;
  if (n > kNoAllocMaxTensors) return NVFP4_ERR_SHAPE;  // more tensors than scratch slots
  if (qp->global_scale_in || qp->block_axis != 0 || qp->amax_from_workspace)
    return NVFP4_ERR_INVALID_ARG;
  if (qp->sf_layout != NVFP4_SF_ROWMAJOR && qp->sf_layout != NVFP4_SF_TCGEN05)
    return NVFP4_ERR_INVALID_ARG;
  if (dtype != NVFP4_F32 && dtype != NVFP4_BF16) return NVFP4_ERR_INVALID_ARG;
  const int64_t esz = dtype == NVFP4_BF16 ? 2 : 4;
  // the same per-descriptor rules as nvfp4_quantize_1d_batched, empty tensors
  // included: an empty tensor is still launched (it receives its global
  // scale, 1.0), so its output pointers must be valid and aligned
  for (int32_t i = 0; i < n; ++i) {
    const nvfp4_tensor_desc& d = descs[i];
    if (d.rows < 0 || d.cols < 0 || d.ld < d.cols || d.cols % 16) return NVFP4_ERR_SHAPE;
    if ((double)d.rows * (double)d.cols / 16.0 >= 4.0e9) return NVFP4_ERR_SHAPE;
    if (!d.x && d.rows > 0 && d.cols > 0) return NVFP4_ERR_INVALID_ARG;
    if (!d.codes || !d.scales || !d.global_scale) return NVFP4_ERR_INVALID_ARG;
    if (!aligned(d.x, 32) || (d.ld * esz) % 32 || !aligned(d.codes, 16) || !aligned(d.scales, 4) ||
        !aligned(d.global_scale, 4))
      return NVFP4_ERR_ALIGN;
  }
  if (n == 0) return NVFP4_OK;
  uint32_t* slots = nullptr;
  nvfp4_status st = scratch_address(&slots);
  if (st != NVFP4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int32_t base = 0; base < n; base += kMaxBatch) {
    QBatch b;
    memset(&b, 0, sizeof(b));
    b.bf16 = dtype == NVFP4_BF16;
    b.four_over_six = qp->four_over_six != 0;
    b.rht = qp->rht_enable != 0;
    b.mask = qp->rht_sign_mask;
    b.block_axis = 0;
    b.sf_layout = qp->sf_layout;
    b.gs_in = nullptr;
    b.err = slots;
    b.partials = reinterpret_cast<float*>(slots + 64) + (size_t)base * kMaxAmaxCtas;
    b.n = 0;
    for (int32_t i = base; i < n && i < base + kMaxBatch; ++i) {
      const nvfp4_tensor_desc& d = descs[i];
      b.t[b.n++] = QTensor{d.x, d.codes, d.scales, d.global_scale, d.rows, d.cols, d.ld};
    }
    if (launch_quantize(b, s) != cudaSuccess) return NVFP4_ERR_CUDA;
  }
  return NVFP4_OK;
}
