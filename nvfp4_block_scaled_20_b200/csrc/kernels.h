// Internal launcher interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace nvfp4 {

constexpr int kMaxBatch = 64;  // tensors per batched launch (kernel parameter space)
// Per-CTA partial maxima of the amax pass: at most this many CTAs per tensor,
// one fp32 slot each in the workspace.
constexpr int kMaxAmaxCtas = 448;

struct QTensor {
  const void* x;
  uint8_t* codes;
  uint8_t* scales;
  float* gs_out;
  int64_t rows;  // input rows
  int64_t cols;  // input cols
  int64_t ld;    // input leading dimension (elements)
};

struct QBatch {
  QTensor t[kMaxBatch];
  int32_t n;
  int32_t bf16;  // 1: bf16 input, 0: fp32
  int32_t four_over_six;
  int32_t rht;
  uint32_t mask;
  int32_t block_axis;
  int32_t sf_layout;
  int32_t two_d;        // 1: 16x16 tiles (block_axis 0, no RHT)
  int32_t amax_only;    // 1: only the amax pass; writes the global scale
  int32_t amax_ready;   // 1: the partials are already in the workspace (no amax pass)
  const float* gs_in;   // device; nullptr => from the amax pass
  float* partials;      // device, kMaxAmaxCtas slots per tensor (amax pass output)
  uint32_t* err;        // device error word
  // Mixed launch (launch_quantize_mixed): 1D row-block and 2D tensors in one
  // 1D grid per pass; tensor i owns blockIdx.x in [end[i-1], end[i]).
  int32_t amax_end[kMaxBatch];
  int32_t enc_end[kMaxBatch];
  int8_t two_d_of[kMaxBatch];  // 1: tensor i is quantized in 16x16 tiles
};

struct DQTensor {
  const uint8_t* codes;
  const uint8_t* scales;
  const float* gs;
  void* out;
  int64_t rows, cols, ldo;
};

struct DQBatch {
  DQTensor t[kMaxBatch];
  int32_t n;
  int32_t out_bf16;
  int32_t sf_layout;
};

// Row-gather dequantization: the same source rows of every tensor, given as
// disjoint sorted ranges [begin[i], begin[i] + len_i); output row o comes
// from range i where prefix[i] <= o < prefix[i + 1].
constexpr int kMaxRowRanges = 1024;
struct DQGather {
  DQBatch b;
  int32_t n_ranges;
  int64_t begin[kMaxRowRanges];
  int64_t prefix[kMaxRowRanges + 1];
};

struct GemmArgs {
  const uint8_t* a_codes;
  const uint8_t* a_sf;
  const float* a_alpha;
  const uint8_t* b_codes;
  const uint8_t* b_sf;
  const float* b_alpha;
  int64_t M, N, K;
  void* out;
  int32_t out_bf16;
  int64_t ldo;
  int32_t epilogue;  // activation (low 4 bits); NVFP4_EPI_AMAX bit
  uint32_t* err;  // device error word
  float* amax_partials;  // non-null: per-CTA output amax (kMaxAmaxCtas slots)
  uint64_t wait_limit_ns;  // bound of each pipeline wait before the kernel gives up
  int32_t stall;           // test hook (nvfp4_set_test_stall)
  // LoRA branch (rank 0: none): u [M, rank] bf16 (row stride ldu), bl [N, rank]
  // bf16 (row stride ldl), out += scale * u bl^T; u_scaled: bf16 [M, 2 rank]
  // scratch for the scaled adapter input
  const void* lora_u;
  const void* lora_b;
  int64_t ldu, ldl, rank;
  float lora_scale;
  void* u_scaled;
  // Partial-sum slabs for splitting the last round's tiles along K (null or
  // slab_cap 0: no split): slab_cap fp32 [256, 256] slabs, 16-byte aligned.
  float* slabs;
  int64_t slab_cap;
};
// Partial-sum slabs the launch of this GEMM would use with room for all of
// them (0: it runs unsplit).
int64_t gemm_split_slabs(int64_t M, int64_t N, int64_t K, int32_t epilogue);

// Default bound of a GEMM pipeline wait, and the process-wide settings
// (nvfp4_set_wait_limit, 0 restores the default; nvfp4_set_test_stall).
constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;
uint64_t gemm_wait_limit_ns();
int32_t gemm_test_stall();

int num_sms();
// The driver's cuTensorMapEncodeTiled (looked up once), or nullptr.
void* tensor_map_encoder();

// Each returns a cudaError_t from the launch.
// Quantization: an amax kernel writing per-CTA partial maxima, then the
// encode kernel (programmatic dependent launch) that reduces them into the
// global scale; only the encode kernel when gs_in is given, only the amax
// kernel and a finalize kernel when amax_only is set.
cudaError_t launch_quantize(const QBatch& b, cudaStream_t s);
// 1D (block_axis 0, no RHT) and 2D tensors of one dtype, each with its own
// global scale from its amax: one amax launch and one encode launch for all,
// CTAs split between the tensors in proportion to their work.  Results equal
// the per-tensor launches'.  Fills the CTA ranges of b.
cudaError_t launch_quantize_mixed(QBatch& b, cudaStream_t s);
cudaError_t launch_dequantize(const DQBatch& b, cudaStream_t s);
cudaError_t launch_dequantize_rows(const DQGather& g, cudaStream_t s);
cudaError_t launch_transpose_2d(const uint8_t* codes, const uint8_t* scales, int sf_in,
                                int64_t rows, int64_t cols, uint8_t* out_codes,
                                uint8_t* out_scales, int sf_out, cudaStream_t s);
// Hardware conversions of the fp32 bit patterns first .. first + count - 1
// (target 0: E2M1 code per byte, 1: E4M3 byte).
cudaError_t launch_convert_sweep(int target, uint32_t first, uint64_t count, uint8_t* out,
                                 cudaStream_t s);
cudaError_t launch_rht16(const void* x, int bf16, int64_t rows, int64_t cols, int64_t ld,
                         int block_axis, uint32_t mask, float* out, cudaStream_t s);
// Returns 0 on success, a cudaError_t value otherwise; sets *unsupported for
// shapes the library does not handle.
int launch_gemm(const GemmArgs& a, cudaStream_t s, bool* unsupported);

}  // namespace nvfp4
