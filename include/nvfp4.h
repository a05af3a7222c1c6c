/*
 * nvfp4.h -- C ABI of the B200 (sm_100a) NVFP4 W4A4 linear-layer library.
 *
 * NVFP4 as defined on the LongLive-2.0 pages ("LongLive-2.0: An NVFP4
 * Parallel Infrastructure for Long Video Generation"; "explainer" below is
 * the paper-graph-ui architecture page, section 3.4 "Detailed, Sentence-Based
 * Technical Breakdown"):
 *   X^ = X^_FP4 * a_FP8 * a_FP32  -- E2M1 4-bit elements, one FP8 E4M3 scale
 *   per 16 elements, one FP32 scale per tensor ("NVFP4 numeric format",
 *   "Hierarchical scaling").
 *
 * Conventions for every entry point
 *   - Ownership: the caller allocates and frees every buffer (device memory
 *     unless a parameter says "host").  The library never allocates, frees or
 *     keeps a pointer after the call returns.
 *   - Asynchrony: work is enqueued on `stream` (a cudaStream_t passed as
 *     void*; NULL = the legacy default stream).  No call synchronizes, except
 *     nvfp4_get_device_error.
 *   - Errors: arguments are validated on the host before anything is
 *     enqueued; a failed check returns a status and enqueues nothing.  A
 *     CUDA launch failure returns NVFP4_ERR_CUDA.  Faults detected on the
 *     device (a bounded wait that ran out) are recorded in the workspace
 *     error word and read back with nvfp4_get_device_error.
 *   - Element packing: two E2M1 codes per byte, element 2j in the low
 *     nibble, element 2j+1 in the high nibble; code bit 3 is the sign.
 *   - Scale bytes are UE4M3 (sign bit 0).  Two layouts:
 *       NVFP4_SF_ROWMAJOR: byte (r, kb) at r * (cols/16) + kb.
 *       NVFP4_SF_TCGEN05:  the tcgen05 block-scaled layout: 512-byte atoms of
 *         128 rows x 4 blocks, byte (r, kb) at
 *         ((r/128) * ceil(kb_total/4) + kb/4) * 512
 *           + (r%32)*16 + ((r%128)/32)*4 + kb%4,
 *         rows padded to a multiple of 128 and blocks to a multiple of 4;
 *         the quantizers write zeros into the padding.
 *   - Alignment (leading dimensions are in elements; a violation returns
 *     NVFP4_ERR_ALIGN): a quantizer input read along its contiguous rows
 *     (block_axis 0, and the 2D quantizer) starts on a 32-byte boundary and
 *     every row does too (ld * element size a multiple of 32); an input read
 *     across rows (block_axis 1) needs 16 bytes for both.  Codes buffers are
 *     16-byte aligned (8 for nvfp4_dequantize), scale buffers and global
 *     scales 4-byte aligned, dequantized outputs 32-byte aligned with 32-byte
 *     rows, GEMM operands (codes and scales) and outputs 16-byte aligned with
 *     16-byte output rows; nvfp4_rht16 takes an element-aligned input and a
 *     4-byte aligned output.
 */
#ifndef NVFP4_H_
#define NVFP4_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum nvfp4_status {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1, /* NULL pointer, unknown enum value            */
  NVFP4_ERR_SHAPE = 2,       /* a dimension violates the call's shape rule  */
  NVFP4_ERR_ALIGN = 3,       /* pointer or leading dimension misaligned     */
  NVFP4_ERR_WORKSPACE = 4,   /* workspace NULL or smaller than required     */
  NVFP4_ERR_CUDA = 5,        /* a CUDA runtime/driver call failed           */
  NVFP4_ERR_TIMEOUT = 6,     /* a bounded device wait ran out (device side) */
  NVFP4_ERR_UNSUPPORTED = 7  /* valid request the library does not implement */
} nvfp4_status;

typedef enum nvfp4_dtype { NVFP4_F32 = 0, NVFP4_BF16 = 1 } nvfp4_dtype;

typedef enum nvfp4_sf_layout {
  NVFP4_SF_ROWMAJOR = 0,
  NVFP4_SF_TCGEN05 = 1
} nvfp4_sf_layout;

typedef enum nvfp4_epilogue {
  NVFP4_EPI_NONE = 0,
  NVFP4_EPI_GELU_TANH = 1, /* 0.5 y (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3))) */
  /* Or-ed into an activation: the GEMM also records the output's amax for
   * its next quantization (see nvfp4_gemm). */
  NVFP4_EPI_AMAX = 16
} nvfp4_epilogue;

/* Quantizer options.
 *   four_over_six  1: per block, encode with the scale that maps the block
 *                  max to 6 and with the one that maps it to 4, keep the one
 *                  with the lower squared error (ties keep 6) -- explainer,
 *                  NVFP4 Inference, "Scale-search mechanism".  0: 6-rule only
 *                  ("Quantization rule for a tensor block").
 *   rht_enable     1: 16-point random Hadamard transform of every 16-block
 *                  (along the block axis) before amax and encoding --
 *                  explainer, "Random Hadamard Transform (RHT) for gradient
 *                  stabilization".  1D quantizers only.
 *   rht_sign_mask  bit j set => sign s_j = -1 in y = 1/4 H16 diag(s) x
 *                  (Sylvester-ordered H16).
 *   block_axis     0: 16-blocks along the contiguous dim: codes [rows,
 *                  cols/2], scales for rows x cols/16.  1 (1D only): blocks
 *                  along rows, output transposed: codes [cols, rows/2],
 *                  scales for cols x rows/16 (WGRAD operands, K = tokens).
 *   sf_layout      nvfp4_sf_layout of the scale output.
 *   global_scale_in  device pointer to a_FP32; NULL => computed as
 *                  amax / (6 * 448) over the (transformed) tensor, 1.0 for an
 *                  all-zero tensor.
 *   amax_from_workspace  1: the tensor's amax is already in the workspace,
 *                  left there by the nvfp4_gemm that produced the tensor
 *                  (epilogue with NVFP4_EPI_AMAX, same workspace): the amax
 *                  pass is skipped, only the encode pass runs (the fused
 *                  "amax from the up-GEMM's epilogue" variant).  Needs
 *                  rht_enable 0 (NVFP4_ERR_INVALID_ARG otherwise) and
 *                  global_scale_in NULL (a given scale wins); single-tensor
 *                  quantize calls only (the batched and mixed calls return
 *                  NVFP4_ERR_INVALID_ARG); ignored by nvfp4_global_scale.
 *                  0: the usual amax pass. */
typedef struct nvfp4_qparams {
  int32_t four_over_six;
  int32_t rht_enable;
  uint32_t rht_sign_mask;
  int32_t block_axis;
  int32_t sf_layout;
  int32_t amax_from_workspace;
  const float* global_scale_in;
} nvfp4_qparams;

/* One tensor of a batched call (KV cache: one per layer and K/V).
 *   quantize:   x [rows, ld] input (dtype of the call), codes/scales outputs,
 *               global_scale = device float written with a_FP32.
 *   dequantize: codes/scales inputs, global_scale = device float a_FP32 read,
 *               out [rows, ld] output (dtype of the call); x unused. */
typedef struct nvfp4_tensor_desc {
  const void* x;
  void* out;
  uint8_t* codes;
  uint8_t* scales;
  float* global_scale;
  int64_t rows;
  int64_t cols;
  int64_t ld;
} nvfp4_tensor_desc;

/* ------------------------------------------------------------ sizes ---- */

/* Bytes of device workspace a call needs: a device error word plus the amax
 * pass's per-CTA partial maxima for each tensor (n_tensors = 1 for the
 * single-tensor calls, 0 for nvfp4_gemm).  Its contents need no
 * initialization except the error word, which must start at zero (it is
 * cleared by nvfp4_get_device_error). */
NVFP4_API size_t nvfp4_workspace_bytes(int32_t n_tensors);

/* Bytes of the packed codes of a [rows, cols] block-axis-0 encoding. */
NVFP4_API int64_t nvfp4_codes_bytes(int64_t rows, int64_t cols);

/* Bytes of the scale buffer for `rows` rows of `cols` elements. */
NVFP4_API int64_t nvfp4_scales_bytes(int64_t rows, int64_t cols, int32_t sf_layout);

/* ------------------------------------------------------------ quantize -- */

/* Global scale only (the amax pass): *global_scale_out = a_FP32 of x under
 * qp (RHT and block_axis honoured; qp->global_scale_in ignored).
 * explainer, "Hierarchical scaling" (tensor-wise FP32 scale).
 * x: device [rows, ld] of dtype.  Shape rules as nvfp4_quantize_1d. */
NVFP4_API nvfp4_status nvfp4_global_scale(const void* x, int32_t dtype, int64_t rows,
                                int64_t cols, int64_t ld,
                                const nvfp4_qparams* qp,
                                float* global_scale_out, void* workspace,
                                size_t workspace_bytes, void* stream);

/* 1D NVFP4 quantization -- explainer, "NVFP4 training recipe for AR
 * training" (1D blocks of 16 along the reduction dimension) and
 * "Quantization rule for a tensor block".
 *   x        device [rows, ld] of dtype (NVFP4_F32 or NVFP4_BF16).
 *   codes    device, nvfp4_codes_bytes of the output shape.
 *   scales   device, nvfp4_scales_bytes of the output shape and layout.
 *   global_scale_out  device float; receives a_FP32 (may equal
 *            qp->global_scale_in).
 * Shape: cols % 16 == 0; block_axis 1 also needs rows % 16 == 0.
 * Runs the amax pass then the quantize pass (one pass with
 * global_scale_in).  Workspace: nvfp4_workspace_bytes(1). */
NVFP4_API nvfp4_status nvfp4_quantize_1d(const void* x, int32_t dtype, int64_t rows,
                               int64_t cols, int64_t ld,
                               const nvfp4_qparams* qp, uint8_t* codes,
                               uint8_t* scales, float* global_scale_out,
                               void* workspace, size_t workspace_bytes,
                               void* stream);

/* 2D NVFP4 quantization of a weight [rows, cols] in 16x16 tiles, one scale
 * per tile (written to the scale entries of the tile's 16 rows), the 4-vs-6
 * pick on the tile's 256 values -- explainer, "NVFP4 training recipe for AR
 * training" (2D block scaling, "e.g., 16x16").  rows % 16 == 0,
 * cols % 16 == 0; rht_enable and block_axis must be 0.  Arguments as
 * nvfp4_quantize_1d. */
NVFP4_API nvfp4_status nvfp4_quantize_2d(const void* x, int32_t dtype, int64_t rows,
                               int64_t cols, int64_t ld,
                               const nvfp4_qparams* qp, uint8_t* codes,
                               uint8_t* scales, float* global_scale_out,
                               void* workspace, size_t workspace_bytes,
                               void* stream);

/* Batched 1D quantization (KV cache): n tensors, each with its own a_FP32
 * (one per layer and K/V), all of one dtype, one launch per pass --
 * explainer, "KV cache quantization" / "Chunkwise quantization procedure"
 * ([T*H, d] rows, 16-blocks along d).  qp applies to every tensor
 * (global_scale_in must be NULL: each tensor gets its own scale).
 * descs: HOST array of n descriptors.  Workspace: nvfp4_workspace_bytes(n). */
NVFP4_API nvfp4_status nvfp4_quantize_1d_batched(const nvfp4_tensor_desc* descs,
                                       int32_t n, int32_t dtype,
                                       const nvfp4_qparams* qp,
                                       void* workspace,
                                       size_t workspace_bytes, void* stream);

/* Mixed quantization: the operands of W4A4 linear layers -- 1D activations
 * and 2D weights (explainer, "NVFP4 training recipe for AR training": 1D
 * blocks for activations and gradients, 16x16 blocks for weights) -- in one
 * amax launch and one encode launch for all tensors, the GPU's CTAs split
 * between them in proportion to their work.  Codes, scales and global
 * scales are identical to nvfp4_quantize_1d / nvfp4_quantize_2d on each
 * tensor (the split changes only which CTA does what).
 *   descs[i]   x, codes, scales, global_scale, rows, cols, ld as in the
 *              single-tensor calls (HOST array of n).
 *   two_d[i]   HOST array of n: 0 = 1D blocks along cols, 1 = 16x16 tiles.
 *   dtype      one input dtype for all tensors.
 *   qp         four_over_six and sf_layout apply to all; rht_enable and
 *              block_axis must be 0 and global_scale_in NULL (each tensor
 *              gets the global scale of its own amax).
 * n <= 64 (else NVFP4_ERR_SHAPE); shape and alignment rules per tensor as
 * in the single-tensor calls; an empty tensor (rows or cols 0) only gets
 * its global scale, 1.0 (its codes and scales may be NULL).
 * Workspace: nvfp4_workspace_bytes(n). */
NVFP4_API nvfp4_status nvfp4_quantize_mixed(const nvfp4_tensor_desc* descs,
                                  const int32_t* two_d, int32_t n,
                                  int32_t dtype, const nvfp4_qparams* qp,
                                  void* workspace, size_t workspace_bytes,
                                  void* stream);

/* Batched 1D quantization that takes no workspace (the paper has no
 * counterpart; this is a library convenience).  For callers that cannot
 * allocate device memory or pass a workspace: code running inside another
 * framework's allocator that forbids side allocations, loops that must not
 * call cudaMalloc because it synchronizes the device, or C callers holding
 * only their tensors' raw pointers.  The per-tensor amax scratch is a fixed
 * array inside the library (about 115 KB on every GPU that loads it, kept
 * until the process exits); the call allocates and frees nothing.
 *   descs, n, dtype, qp: as nvfp4_quantize_1d_batched; block_axis must be 0
 *   and global_scale_in NULL.  n <= 64, else NVFP4_ERR_SHAPE.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  Calls share the array: it keeps the last call's contents (each
 * call overwrites every slot it reads before reading it), and calls that
 * overlap on the GPU (other streams, other threads) race on it -- serialize
 * them. */
NVFP4_API nvfp4_status nvfp4_quantize_1d_batched_noalloc(const nvfp4_tensor_desc* descs,
                                                         int32_t n, int32_t dtype,
                                                         const nvfp4_qparams* qp, void* stream);

/* ------------------------------------------------------------ dequant --- */

/* Parallel dequantization of n tensors in one launch: out = val(q) * d *
 * a_FP32 (fp32 product, then round-to-nearest-even to bf16 for NVFP4_BF16)
 * -- explainer, "Hierarchical scaling" and "Parallel CUDA dequantization
 * kernel" (every CTA independent, all tensors in a single launch).
 * descs: HOST array; per tensor codes/scales/global_scale are read and out
 * [rows, ld] of out_dtype is written.  cols % 16 == 0. */
NVFP4_API nvfp4_status nvfp4_dequantize(const nvfp4_tensor_desc* descs, int32_t n,
                              int32_t out_dtype, int32_t sf_layout,
                              void* stream);

/* Transpose of a 2D (16x16-tile) encoding (explainer, section 3.4, "The
 * three GEMMs of backpropagation in NVFP4": the data-gradient GEMM
 * dA = dO . W takes the weight in NVFP4, contracted along W's rows; with one
 * scale per 16x16 tile the encoding of W holds W^T's blocks, so the codes are
 * transposed and no element is re-quantized).
 *   codes [rows, cols/2], scales (sf_layout_in): an encoding written by
 *     nvfp4_quantize_2d of a [rows, cols] matrix (every row of a tile holds
 *     the tile's scale; the output takes each tile's first row).
 *   out_codes [cols, rows/2], out_scales (sf_layout_out, cols rows x
 *     rows/16 blocks; nvfp4_scales_bytes(cols, rows, layout) bytes): the
 *     encoding of the transpose, ready as the B operand of nvfp4_gemm.  The
 *     global scale is unchanged (the caller reuses it).
 *   rows, cols multiples of 16 (NVFP4_ERR_SHAPE); codes buffers 8-byte
 *   aligned.  Bit-exact with the transposed oracle encoding. */
NVFP4_API nvfp4_status nvfp4_transpose_2d(const uint8_t* codes, const uint8_t* scales,
                                          int32_t sf_layout_in, int64_t rows, int64_t cols,
                                          uint8_t* out_codes, uint8_t* out_scales,
                                          int32_t sf_layout_out, void* stream);

/* Gathering dequantization for a sliding-window KV cache with attention
 * sinks (explainer, section 3.4, "Multi-shot attention sink": the effective
 * key/value set is the global sink, the shot-level sink given by START and
 * LEN, and the window KV[t-W, t), overlapping entries deduplicated;
 * "Parallel CUDA dequantization kernel").  The same source rows of every
 * tensor are dequantized, in increasing row order, into contiguous output
 * rows: one launch for all tensors.
 *   descs[i]: codes, scales (sf_layout), global_scale, out, rows, cols as in
 *     nvfp4_dequantize; out has room for the gathered rows (ld = row
 *     stride in elements).
 *   row_ranges: HOST array of n_ranges pairs {begin, end}, half-open source
 *     row ranges (for a [heads * tokens, d] cache: head h's tokens [a, b)
 *     are rows [h*tokens + a, h*tokens + b)).  The ranges are sorted and
 *     merged on the host (overlapping or touching ranges joined, empty ones
 *     dropped); output row o is the o-th row of the union.
 *   n_ranges <= 1024 (NVFP4_ERR_SHAPE beyond); begin < 0, end < begin or a
 *   union reaching past any tensor's rows: NVFP4_ERR_SHAPE.  Alignment as
 *   nvfp4_dequantize.  Bit-exact with nvfp4_dequantize on the same rows. */
NVFP4_API nvfp4_status nvfp4_dequantize_rows(const nvfp4_tensor_desc* descs, int32_t n,
                                             const int64_t* row_ranges, int32_t n_ranges,
                                             int32_t out_dtype, int32_t sf_layout,
                                             void* stream);

/* ------------------------------------------------------------ GEMM ------ */

/* Block-scaled FP4 GEMM on the 5th-generation tensor cores
 * (tcgen05.mma kind::mxf4nvf4, UE4M3 scales per 16 elements, fp32
 * accumulation in tensor memory):
 *   out[m, n] = epi( a_alpha * b_alpha *
 *                    sum_k val(a_mk) sA[m, k/16] * val(b_nk) sB[n, k/16] )
 * -- explainer, "The three GEMMs of backpropagation in NVFP4" (Y = X W^T
 * forward, WGRAD with both operands quantized along the tokens).
 *   a_codes  device [M, K/2] (K-major),  a_sf device, NVFP4_SF_TCGEN05
 *            layout for M rows, K/16 blocks;  a_alpha device float.
 *   b_codes  device [N, K/2] (K-major),  b_sf, b_alpha likewise for N rows.
 *   out      device [M, ldo] of out_dtype (NVFP4_BF16: RNE; NVFP4_F32).
 *   epilogue nvfp4_epilogue, applied in fp32 before the conversion;
 *            with NVFP4_EPI_AMAX or-ed in, every CTA also writes the largest
 *            |stored value| (after the activation and the rounding to
 *            out_dtype; rows past M excluded) into the amax partials of ws,
 *            which must then be nvfp4_workspace_bytes(1) bytes: a following
 *            nvfp4_quantize_1d / _2d of out with that workspace and
 *            qp->amax_from_workspace = 1 skips its amax pass and gives the
 *            same codes, scales and global scale as without it.
 * Shape: M >= 1, N % 16 == 0, K % 64 == 0, ldo >= N, ldo * elem % 16 == 0.
 * Workspace: nvfp4_workspace_bytes(0) (the device error word) at least.
 * With nvfp4_gemm_workspace_bytes(M, N, K, epilogue) bytes, 16-byte aligned,
 * the tiles of the persistent schedule's last, partial round are each split
 * along K among otherwise idle SM pairs (long K, plain epilogue only): their
 * fp32 partial sums go to the workspace and a second kernel on the same
 * stream adds them in a fixed order, scales and stores them.  The result is
 * deterministic; against the unsplit kernel it differs only by the order of
 * the fp32 additions over K. */
NVFP4_API nvfp4_status nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_sf,
                        const float* a_alpha, const uint8_t* b_codes,
                        const uint8_t* b_sf, const float* b_alpha, int64_t M,
                        int64_t N, int64_t K, void* out, int32_t out_dtype,
                        int64_t ldo, int32_t epilogue, void* workspace,
                        size_t workspace_bytes, void* stream);

/* Workspace bytes with which nvfp4_gemm splits its last partial round for
 * this shape and epilogue (room for the error word, the amax partials and
 * one fp32 256 x 256 slab per split unit); nvfp4_workspace_bytes of the call
 * when the launch would not split.  Depends on the current device's SM
 * count; without a usable device, nvfp4_workspace_bytes of the call.  Like
 * every workspace it serves one call in flight at a time (the split tiles'
 * partial sums live in it until the call's reduction kernel has run). */
NVFP4_API size_t nvfp4_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t epilogue);

/* Bytes of the scratch nvfp4_gemm_lora needs for an M-row activation and a
 * rank-`rank` adapter (the scaled adapter input, bf16 [M, 2 rank]). */
NVFP4_API size_t nvfp4_lora_scratch_bytes(int64_t M, int64_t rank);

/* W4A4 linear layer with its low-rank adapter in one GEMM -- notes, section
 * 3.4 "NVFP4 training and DMD LoRA" (the quantized LoRA linear: frozen NVFP4
 * backbone, bf16 adapter, delta = (x A^T) B^T * scale, rank 128 and alpha 128
 * in the released adapter) and explainer, section 3.4 (W ~ Dequant(Q(W0)) +
 * (alpha/r) B A; the deployed layer keeps the branch separate):
 *   out[m, n] = epi( a_alpha b_alpha sum_k a_mk sA b_nk sB
 *                    + lora_scale * sum_j lora_u[m, j] lora_b[n, j] ).
 * The adapter's product runs on the tensor cores in the same kernel, into the
 * same fp32 accumulator as the FP4 product, after each tile's FP4 stages
 * (tcgen05.mma kind::f16, bf16 x bf16): lora_u * lora_scale / (a_alpha
 * b_alpha) is first written to scratch as the bf16 pair hi + lo (within 2^-17
 * of the fp32 value), so one epilogue scaling by a_alpha b_alpha serves both
 * terms.
 *   FP4 operands, out, epilogue, workspace: as nvfp4_gemm.
 *   lora_u   device bf16 [M, rank], row stride ldu: x A^T, the adapter's
 *            first product (16-byte aligned, ldu * 2 a multiple of 16).
 *   lora_b   device bf16 [N, rank], row stride ldl: B (same alignment).
 *   rank     a multiple of 64, 64..1024; lora_scale finite (alpha / rank).
 *   scratch  device, nvfp4_lora_scratch_bytes(M, rank) bytes, 16-byte
 *            aligned; overwritten.
 * lora_scale / (a_alpha b_alpha) must be finite. */
NVFP4_API nvfp4_status nvfp4_gemm_lora(const uint8_t* a_codes, const uint8_t* a_sf,
                                       const float* a_alpha, const uint8_t* b_codes,
                                       const uint8_t* b_sf, const float* b_alpha, int64_t M,
                                       int64_t N, int64_t K, const void* lora_u, int64_t ldu,
                                       const void* lora_b, int64_t ldl, int64_t rank,
                                       float lora_scale, void* scratch, size_t scratch_bytes,
                                       void* out, int32_t out_dtype, int64_t ldo,
                                       int32_t epilogue, void* workspace, size_t workspace_bytes,
                                       void* stream);

/* ------------------------------------------------------------ RHT ------- */

/* Standalone 16-point RHT, y = 1/4 H16 diag(s) x on every 16-group along
 * block_axis (0: contiguous dim, cols % 16 == 0; 1: rows, rows % 16 == 0),
 * the same transform the quantizers fuse -- explainer, "Random Hadamard
 * Transform (RHT) for gradient stabilization".
 *   x device [rows, ld] of dtype; out device fp32 [rows, cols]. */
NVFP4_API nvfp4_status nvfp4_rht16(const void* x, int32_t dtype, int64_t rows,
                         int64_t cols, int64_t ld, int32_t block_axis,
                         uint32_t sign_mask, float* out, void* stream);

/* ------------------------------------------------------------ checks ---- */

/* Conformance sweep of the hardware conversions every encoder takes its
 * rounding decisions with: the element cast to E2M1 ("rounded to the nearest
 * E2M1 value", explainer, "Quantization rule for a tensor block") and the
 * block-scale cast to E4M3 ("cast_E4M3 ... rounding to the nearest
 * representable E4M3 value", same paragraph), both round-to-nearest-even and
 * saturating (to 6 and to 448).  The encoders' bracketed decisions are exact
 * only if both conversions are, for every fp32 input; this call lets a test
 * compare a whole range of inputs with the formats' definitions.
 *   target  0: out[i] = E2M1 code (sign in bit 3, low nibble) of v_i;
 *           1: out[i] = E4M3 byte of v_i.
 *   v_i     the fp32 value whose bit pattern is first_bits + i, 0 <= i < count;
 *           first_bits + count <= 2^32 (NVFP4_ERR_SHAPE otherwise).
 *   out     device, count bytes, 16-byte aligned. */
NVFP4_API nvfp4_status nvfp4_convert_sweep(int32_t target, uint32_t first_bits, int64_t count,
                                           uint8_t* out, void* stream);

/* Bound, in nanoseconds, of every wait in nvfp4_gemm's pipeline (0 restores
 * the default, 2 s), for the whole process, read at each nvfp4_gemm call.
 * A wait that runs out records NVFP4_ERR_TIMEOUT in the workspace error
 * word; the kernel then waits (with bounds of its own, independent of this
 * one) for the copies and MMAs it issued, frees its tensor memory and
 * returns, leaving the device usable.  The pages' system-level failure
 * handling is outside this library; the bound is the device-side guard every
 * kernel wait carries. */
NVFP4_API nvfp4_status nvfp4_set_wait_limit(uint64_t ns);

/* Test hook of the timeout path, for the whole process, read at each
 * nvfp4_gemm call: with on = 1 every GEMM's MMA issuer first waits on a
 * barrier that nothing ever completes, while the producers' first stages are
 * in flight; the wait runs out after the nvfp4_set_wait_limit bound and the
 * kernel takes its abort path (NVFP4_ERR_TIMEOUT in the error word, output
 * not written).  on = 0 (the default) turns it off; other values return
 * NVFP4_ERR_INVALID_ARG. */
NVFP4_API nvfp4_status nvfp4_set_test_stall(int32_t on);

/* ------------------------------------------------------------ status ---- */

/* Synchronizes `stream`, copies the workspace's device error word to the
 * HOST int32 *error_out (0 = none, else an nvfp4_status value) and clears
 * it.  Returns NVFP4_ERR_CUDA if the copy fails. */
NVFP4_API nvfp4_status nvfp4_get_device_error(void* workspace, int32_t* error_out,
                                    void* stream);

/* Static, NUL-terminated description of a status value. */
NVFP4_API const char* nvfp4_status_string(int32_t status);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H_ */
