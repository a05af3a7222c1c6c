/*
 * NVFP4 reference oracle -- plain, slow, single-threaded C.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call this file:
 * only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline leg load
 * the shared library built from it.  It shares no source, header, table or
 * helper with the CUDA library.
 *
 * What it follows (LongLive-2.0: An NVFP4 Parallel Infrastructure for Long
 * Video Generation; "explainer" = the paper-graph-ui architecture page,
 * "notes" = the paper-notes-site page):
 *   - E2M1 element grid and the maxima 6 / 448:      explainer §3.4, NVFP4
 *     Training, "NVFP4 numeric format" and "Hierarchical scaling".
 *   - X^ = X^_FP4 * a_FP8 * a_FP32:                  explainer §3.4, same
 *     paragraph ("Hierarchical scaling"), the reconstruction equation.
 *   - block scale = cast_E4M3(max|U_B| / 6), then each value divided by the
 *     scale and rounded to the nearest E2M1 value:   explainer §3.4,
 *     "Quantization rule for a tensor block".
 *   - 1D blocks (16 along the reduction dim) for activations / gradients,
 *     2D 16x16 tiles for weights:                    explainer §3.4, "NVFP4
 *     training recipe for AR training".
 *   - the 4-vs-6 pick (two candidate scales, keep the one with the lower
 *     squared reconstruction error):                 explainer §3.4, NVFP4
 *     Inference, "Scale-search mechanism".
 *   - random Hadamard transform before quantizing the WGRAD operands:
 *     explainer §3.4, "Random Hadamard Transform (RHT) for gradient
 *     stabilization".
 *   - KV cache: [T*H, d] rows quantized in 16-blocks along d with a global
 *     FP32 scale:                                    explainer §3.4, "KV cache
 *     quantization" / "Chunkwise quantization procedure".
 *   - the three GEMMs Y = X W^T etc. on NVFP4 operands: explainer §3.4, "The
 *     three GEMMs of backpropagation in NVFP4".
 *   - the LoRA branch scale * (x A^T) B^T added to a W4A4 output: notes §3.4,
 *     "NVFP4 training and DMD LoRA" (quantized LoRA linear).
 *
 * Where the pages leave a step open the reading taken is written next to the
 * code (global-scale formula, rounding ties, saturation, the error sum's
 * precision and order, RHT size/order/normalisation).
 *
 * Floating point: every fp32 operation is one IEEE round-to-nearest-even
 * operation; build with -ffp-contract=off (no fused multiply-add).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_SF_ROWMAJOR 0
#define ORC_SF_TCGEN05 1

/* ------------------------------------------------------------------------ */
/* E2M1 element codec                                                        */
/* ------------------------------------------------------------------------ */

/* Magnitudes of the 3-bit E2M1 code (1 sign, 2 exponent, 1 mantissa bit):
 * the set {0, 0.5, 1, 1.5, 2, 3, 4, 6} printed in "NVFP4 numeric format". */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double orc_e2m1_value(int code) {
  double m = E2M1_MAG[code & 7];
  return (code & 8) ? -m : m;
}

/* Nearest E2M1 value to v.  Reading of "rounded to the nearest E2M1 value":
 * distance ties go to the code whose mantissa bit is 0 (even), magnitudes
 * above 6 saturate to 6, the sign bit is the sign bit of v (so small
 * negatives give -0, code 0x8).  Inputs are finite or +-inf. */
int orc_e2m1_encode(float v) {
  int sign = signbit(v) ? 8 : 0;
  double a = fabs((double)v);
  if (isinf(a)) return sign | 7;
  int best = 0;
  double best_d = a; /* distance to magnitude 0 */
  for (int m = 1; m < 8; ++m) {
    double d = fabs(a - E2M1_MAG[m]); /* exact in double */
    if (d < best_d || (d == best_d && (m & 1) == 0 && (best & 1) == 1)) {
      best = m;
      best_d = d;
    }
  }
  return sign | best;
}

/* ------------------------------------------------------------------------ */
/* E4M3 block-scale codec (unsigned use: scales are positive)                */
/* ------------------------------------------------------------------------ */

/* E4M3: exponent bias 7, 3 mantissa bits, exponent field 0 = subnormal
 * (m * 2^-9), largest finite 1.75 * 2^8 = 448 (code 0x7E); 0x7F is NaN. */
double orc_e4m3_decode(int code) {
  int e = (code >> 3) & 15;
  int m = code & 7;
  if (e == 0) return ldexp((double)m, -9);
  return ldexp(1.0 + m / 8.0, e - 7);
}

/* cast_E4M3 of "Quantization rule for a tensor block": nearest E4M3 value,
 * ties to the even mantissa, saturating at 448 (reading: the pages say only
 * "rounding to the nearest representable E4M3 value"; a candidate scale can
 * exceed 448, see the 4-candidate below).  t >= 0 finite (or +inf). */
int orc_e4m3_encode(float t) {
  if (!(t > 0.0f)) return 0;
  if (t >= 448.0f) return 0x7E;
  int ex;
  (void)frexp((double)t, &ex); /* t = f * 2^ex, f in [0.5, 1) */
  int E = ex - 1;               /* t in [2^E, 2^(E+1)) */
  if (E < -6) {                 /* subnormal range: units of 2^-9 */
    double q = rint(ldexp((double)t, 9)); /* exact scaling, RNE */
    return (int)q;                        /* 8 becomes 2^-6: code 0x08 */
  }
  double q = rint(ldexp((double)t, 3 - E)); /* in [8, 16] */
  if (q >= 16.0) {
    E += 1;
    q = 8.0;
  }
  int code = ((E + 7) << 3) | ((int)q - 8);
  if (code > 0x7E) code = 0x7E;
  return code;
}

/* The two element/scale casts above over a contiguous range of fp32 bit
 * patterns (first_bits + i, i < n), one code per output byte -- the oracle's
 * side of the exhaustive conversion sweeps (no arithmetic of its own). */
void orc_e2m1_encode_bits(uint32_t first_bits, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) {
    uint32_t u = first_bits + (uint32_t)i;
    float v;
    memcpy(&v, &u, 4);
    out[i] = (uint8_t)orc_e2m1_encode(v);
  }
}

void orc_e4m3_encode_bits(uint32_t first_bits, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) {
    uint32_t u = first_bits + (uint32_t)i;
    float v;
    memcpy(&v, &u, 4);
    out[i] = (uint8_t)orc_e4m3_encode(v);
  }
}

/* ------------------------------------------------------------------------ */
/* bf16 round-to-nearest-even of an fp32 value (finite inputs)               */
/* ------------------------------------------------------------------------ */
uint16_t orc_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------------ */
/* 16-point random Hadamard transform                                        */
/* ------------------------------------------------------------------------ */

/* y = (1/4) * H16 * diag(s) * x with the Sylvester-ordered H16
 * (H[i][j] = (-1)^popcount(i & j)), s_j = -1 where bit j of mask is set.
 * Reading of "Random Hadamard Transform" (entries +-1/sqrt(d), d = 16 here):
 * sign flip, then the in-place butterfly with strides 1, 2, 4, 8, each
 * (a, b) -> (a + b, a - b) in fp32, then the exact scaling by 1/4. */
void orc_rht16_block(float v[16], uint32_t mask) {
  for (int j = 0; j < 16; ++j)
    if ((mask >> j) & 1u) v[j] = -v[j];
  for (int h = 1; h < 16; h <<= 1) {
    for (int i = 0; i < 16; ++i) {
      if (i & h) continue;
      float a = v[i], b = v[i + h];
      v[i] = a + b;
      v[i + h] = a - b;
    }
  }
  for (int j = 0; j < 16; ++j) v[j] = v[j] * 0.25f;
}

/* Transform of a [rows, cols] matrix (leading dimension ld) in 16-groups
 * along the contiguous dim (block_axis 0) or along rows (block_axis 1).
 * out is [rows, cols] contiguous.  Returns 0, or -1 on a bad shape. */
int orc_rht16(const float* x, int64_t rows, int64_t cols, int64_t ld,
              int block_axis, uint32_t mask, float* out) {
  float v[16];
  if (block_axis == 0) {
    if (cols % 16) return -1;
    for (int64_t r = 0; r < rows; ++r)
      for (int64_t c = 0; c < cols; c += 16) {
        for (int j = 0; j < 16; ++j) v[j] = x[r * ld + c + j];
        orc_rht16_block(v, mask);
        for (int j = 0; j < 16; ++j) out[r * cols + c + j] = v[j];
      }
  } else {
    if (rows % 16) return -1;
    for (int64_t c = 0; c < cols; ++c)
      for (int64_t r = 0; r < rows; r += 16) {
        for (int j = 0; j < 16; ++j) v[j] = x[(r + j) * ld + c];
        orc_rht16_block(v, mask);
        for (int j = 0; j < 16; ++j) out[(r + j) * cols + c] = v[j];
      }
  }
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Global scale                                                              */
/* ------------------------------------------------------------------------ */

/* alpha_FP32 from the tensor amax.  The pages give no formula (only that it
 * is a per-tensor FP32 scale, "Hierarchical scaling").  Reading: alpha =
 * amax / (M_FP4 * M_FP8) = amax / 2688 in fp32, so that the block holding
 * the tensor maximum gets the largest E4M3 scale (448) under the 6-rule;
 * alpha = 1 for an all-zero tensor. */
float orc_alpha_from_amax(float amax) {
  if (!(amax > 0.0f)) return 1.0f;
  return amax / 2688.0f;
}

/* ------------------------------------------------------------------------ */
/* Scale-factor layouts                                                      */
/* ------------------------------------------------------------------------ */

/* Byte offset of scale (row r, 16-block kb) in a buffer for kb_total blocks
 * per row.  Row-major: r * kb_total + kb.  tcgen05 block-scaled layout
 * (public PTX / cuBLAS block-scaling documentation): 512-byte atoms of 128
 * rows x 4 blocks, offset (r%32)*16 + ((r%128)/32)*4 + kb%4 inside an atom,
 * atoms ordered by 128-row band, then by 4-block group along K. */
int64_t orc_sf_offset(int64_t r, int64_t kb, int64_t kb_total, int layout) {
  if (layout == ORC_SF_ROWMAJOR) return r * kb_total + kb;
  int64_t kb_groups = (kb_total + 3) / 4;
  return ((r / 128) * kb_groups + kb / 4) * 512 + (r % 32) * 16 +
         ((r % 128) / 32) * 4 + (kb % 4);
}

int64_t orc_sf_bytes(int64_t rows, int64_t kb_total, int layout) {
  if (layout == ORC_SF_ROWMAJOR) return rows * kb_total;
  return ((rows + 127) / 128) * 128 * ((kb_total + 3) / 4) * 4;
}

/* ------------------------------------------------------------------------ */
/* Block quantization with the 4-vs-6 pick                                   */
/* ------------------------------------------------------------------------ */

/* Sum of 16 fp32 values in the fixed pairwise order (i, i+8), (i, i+4),
 * (i, i+2), (i, i+1).  Reading: the pages say "mean-squared reconstruction
 * error" without a precision or order; this fixes both. */
static float tree_sum16(const float e[16]) {
  float a[8], b[4], c[2];
  for (int i = 0; i < 8; ++i) a[i] = e[i] + e[i + 8];
  for (int i = 0; i < 4; ++i) b[i] = a[i] + a[i + 4];
  for (int i = 0; i < 2; ++i) c[i] = b[i] + b[i + 2];
  return c[0] + c[1];
}

/* One candidate encoding of a block of nrows x 16 values y (nrows = 1 for a
 * 1D block, 16 for a 2D tile) whose max magnitude is bmax:
 *   t = (bmax / alpha) / M          (two fp32 divisions, in that order)
 *   e = cast_E4M3(t), d = decode(e), s = d * alpha   (fp32)
 *   q_i = nearest E2M1 of (y_i / s)                  (fp32 division)
 *   err = sum_i (y_i - val(q_i) * s)^2               (fp32, fixed tree; rows
 *         first, then the same tree across the 16 row sums of a tile)
 * A scale that rounds to zero encodes the block as all +0 codes with error
 * sum(y_i^2). */
static void candidate(const float* y, int nrows, float bmax, float alpha,
                      float M, uint8_t* q, int* ecode, float* err) {
  float t = (bmax / alpha) / M;
  int e = orc_e4m3_encode(t);
  float d = (float)orc_e4m3_decode(e);
  float s = d * alpha;
  float rowsum[16];
  float sq[16];
  for (int r = 0; r < nrows; ++r) {
    for (int i = 0; i < 16; ++i) {
      float yi = y[r * 16 + i];
      float res;
      if (s == 0.0f) {
        q[r * 16 + i] = 0;
        res = yi;
      } else {
        int code = orc_e2m1_encode(yi / s);
        q[r * 16 + i] = (uint8_t)code;
        float v = (float)orc_e2m1_value(code);
        float rec = v * s;
        res = yi - rec;
      }
      sq[i] = res * res;
    }
    rowsum[r] = tree_sum16(sq);
  }
  *ecode = e;
  *err = (nrows == 1) ? rowsum[0] : tree_sum16(rowsum);
}

/* Encode one block: 6-rule, and with four_over_six the 4-candidate too,
 * keeping the 4-encoding only when its error is strictly lower (ties keep
 * the standard 6-rule) -- "Scale-search mechanism". */
static int quantize_block(const float* y, int nrows, float alpha,
                          int four_over_six, uint8_t* q_out) {
  float bmax = 0.0f;
  for (int i = 0; i < nrows * 16; ++i) {
    float a = fabsf(y[i]);
    if (a > bmax) bmax = a;
  }
  uint8_t q6[256], q4[256];
  int e6, e4;
  float err6, err4;
  candidate(y, nrows, bmax, alpha, 6.0f, q6, &e6, &err6);
  if (four_over_six) {
    candidate(y, nrows, bmax, alpha, 4.0f, q4, &e4, &err4);
    if (err4 < err6) {
      memcpy(q_out, q4, (size_t)nrows * 16);
      return e4;
    }
  }
  memcpy(q_out, q6, (size_t)nrows * 16);
  return e6;
}

static void put_code(uint8_t* codes, int64_t row_bytes, int64_t r, int64_t c,
                     uint8_t q) {
  uint8_t* p = codes + r * row_bytes + c / 2;
  if (c & 1)
    *p = (uint8_t)((*p & 0x0F) | (q << 4));
  else
    *p = (uint8_t)((*p & 0xF0) | q);
}

/* Global amax of a [rows, cols] matrix, after the 16-point RHT when rht is
 * set (along block_axis). */
float orc_amax(const float* x, int64_t rows, int64_t cols, int64_t ld,
               int rht, uint32_t mask, int block_axis) {
  float amax = 0.0f;
  if (!rht) {
    for (int64_t r = 0; r < rows; ++r)
      for (int64_t c = 0; c < cols; ++c) {
        float a = fabsf(x[r * ld + c]);
        if (a > amax) amax = a;
      }
    return amax;
  }
  float* t = (float*)malloc((size_t)(rows * cols) * sizeof(float));
  if (!t) return -1.0f;
  if (orc_rht16(x, rows, cols, ld, block_axis, mask, t) != 0) {
    free(t);
    return -1.0f;
  }
  for (int64_t i = 0; i < rows * cols; ++i) {
    float a = fabsf(t[i]);
    if (a > amax) amax = a;
  }
  free(t);
  return amax;
}

/* 1D quantization.  block_axis 0: rows x cols, 16-blocks along the
 * contiguous dim; outputs codes [rows, cols/2] and scales for rows rows and
 * cols/16 blocks.  block_axis 1: 16-blocks along rows; the oracle takes the
 * plain route -- transpose first, then the block_axis-0 path -- so outputs
 * are codes [cols, rows/2] and scales for cols rows and rows/16 blocks.
 * rht: 16-point RHT on each block before amax and encoding.
 * alpha_in: NULL to compute alpha from the amax, else used as is.
 * Returns 0, or -1 on a bad shape / allocation failure. */
int orc_quantize_1d(const float* x, int64_t rows, int64_t cols, int64_t ld,
                    int four_over_six, int rht, uint32_t mask, int block_axis,
                    int sf_layout, const float* alpha_in, uint8_t* codes,
                    uint8_t* scales, float* alpha_out) {
  const float* src = x;
  float* tmp = NULL;
  int64_t R = rows, C = cols, L = ld;
  if (block_axis == 1) {
    if (rows % 16) return -1;
    tmp = (float*)malloc((size_t)(rows * cols) * sizeof(float));
    if (!tmp) return -1;
    for (int64_t r = 0; r < rows; ++r)
      for (int64_t c = 0; c < cols; ++c) tmp[c * rows + r] = x[r * ld + c];
    src = tmp;
    R = cols;
    C = rows;
    L = rows;
  }
  if (C % 16) {
    free(tmp);
    return -1;
  }
  float alpha;
  if (alpha_in) {
    alpha = *alpha_in;
  } else {
    float amax = orc_amax(src, R, C, L, rht, mask, 0);
    if (amax < 0.0f) {
      free(tmp);
      return -1;
    }
    alpha = orc_alpha_from_amax(amax);
  }
  int64_t kb_total = C / 16;
  memset(scales, 0, (size_t)orc_sf_bytes(R, kb_total, sf_layout));
  memset(codes, 0, (size_t)(R * C / 2));
  float y[16];
  uint8_t q[16];
  for (int64_t r = 0; r < R; ++r) {
    for (int64_t kb = 0; kb < kb_total; ++kb) {
      for (int i = 0; i < 16; ++i) y[i] = src[r * L + kb * 16 + i];
      if (rht) orc_rht16_block(y, mask);
      int e = quantize_block(y, 1, alpha, four_over_six, q);
      for (int i = 0; i < 16; ++i) put_code(codes, C / 2, r, kb * 16 + i, q[i]);
      scales[orc_sf_offset(r, kb, kb_total, sf_layout)] = (uint8_t)e;
    }
  }
  if (alpha_out) *alpha_out = alpha;
  free(tmp);
  return 0;
}

/* 2D quantization of a weight matrix [rows, cols] in 16x16 tiles (rows and
 * cols multiples of 16): one scale per tile, chosen on the tile's 256
 * values, written to the scale entries of all 16 rows of the tile. */
int orc_quantize_2d(const float* x, int64_t rows, int64_t cols, int64_t ld,
                    int four_over_six, int sf_layout, const float* alpha_in,
                    uint8_t* codes, uint8_t* scales, float* alpha_out) {
  if (rows % 16 || cols % 16) return -1;
  float alpha = alpha_in ? *alpha_in
                         : orc_alpha_from_amax(orc_amax(x, rows, cols, ld, 0, 0, 0));
  int64_t kb_total = cols / 16;
  memset(scales, 0, (size_t)orc_sf_bytes(rows, kb_total, sf_layout));
  memset(codes, 0, (size_t)(rows * cols / 2));
  float y[256];
  uint8_t q[256];
  for (int64_t tr = 0; tr < rows; tr += 16) {
    for (int64_t kb = 0; kb < kb_total; ++kb) {
      for (int r = 0; r < 16; ++r)
        for (int i = 0; i < 16; ++i) y[r * 16 + i] = x[(tr + r) * ld + kb * 16 + i];
      int e = quantize_block(y, 16, alpha, four_over_six, q);
      for (int r = 0; r < 16; ++r) {
        for (int i = 0; i < 16; ++i)
          put_code(codes, cols / 2, tr + r, kb * 16 + i, q[r * 16 + i]);
        scales[orc_sf_offset(tr + r, kb, kb_total, sf_layout)] = (uint8_t)e;
      }
    }
  }
  if (alpha_out) *alpha_out = alpha;
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Dequantization: x^ = val(q) * d * alpha ("Hierarchical scaling")          */
/* ------------------------------------------------------------------------ */

/* (val(q) * d) is exact in fp32; one fp32 multiply by alpha; then, for the
 * bf16 output, one round-to-nearest-even to bf16.  out_f32 and/or out_bf16
 * may be NULL. */
void orc_dequantize(const uint8_t* codes, const uint8_t* scales, float alpha,
                    int64_t rows, int64_t cols, int sf_layout, float* out_f32,
                    uint16_t* out_bf16) {
  int64_t kb_total = cols / 16;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t c = 0; c < cols; ++c) {
      uint8_t byte = codes[r * (cols / 2) + c / 2];
      int q = (c & 1) ? (byte >> 4) : (byte & 15);
      int e = scales[orc_sf_offset(r, c / 16, kb_total, sf_layout)];
      float vd = (float)(orc_e2m1_value(q) * orc_e4m3_decode(e));
      float xh = vd * alpha;
      if (out_f32) out_f32[r * cols + c] = xh;
      if (out_bf16) out_bf16[r * cols + c] = orc_bf16_rne(xh);
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Transpose of a 2D (16x16-tile) encoding, for the data-gradient GEMM        */
/* ------------------------------------------------------------------------ */

/* The data-gradient GEMM dA = dO . W contracts W along its output dimension
 * ("The three GEMMs of backpropagation in NVFP4": DGRAD takes W in NVFP4),
 * so it needs W^T blocked along W's rows.  With one scale per 16x16 tile
 * ("Quantization rule for a tensor block", 2D blocks for weights) the
 * encoding of W already holds W^T's blocks: element (c, r) of the output is
 * element (r, c) of the input, and output block (c, b) -- 16 elements along
 * W's rows 16b .. 16b+15 -- has the scale of the tile (b, c/16), read from
 * input row 16b.  rows and cols are multiples of 16.  Returns 0, or -1 on a
 * bad shape. */
int orc_transpose_2d(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols,
                     int sf_layout_in, uint8_t* out_codes, uint8_t* out_scales,
                     int sf_layout_out) {
  if (rows < 0 || cols < 0 || rows % 16 || cols % 16) return -1;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t c = 0; c < cols; ++c) {
      uint8_t byte = codes[r * (cols / 2) + c / 2];
      uint8_t q = (uint8_t)((c & 1) ? (byte >> 4) : (byte & 15));
      put_code(out_codes, rows / 2, c, r, q);
    }
  }
  int64_t out_kb = rows / 16, in_kb = cols / 16;
  for (int64_t c = 0; c < cols; ++c)
    for (int64_t b = 0; b < out_kb; ++b)
      out_scales[orc_sf_offset(c, b, out_kb, sf_layout_out)] =
          scales[orc_sf_offset(16 * b, c / 16, in_kb, sf_layout_in)];
  return 0;
}

/* ------------------------------------------------------------------------ */
/* GEMM reference on the encodings: Y[m,n] = sum_k a^_mk * b^_nk (fp64)       */
/* ------------------------------------------------------------------------ */

static double deq64(const uint8_t* codes, const uint8_t* sf, double alpha,
                    int64_t r, int64_t k, int64_t K, int layout) {
  uint8_t byte = codes[r * (K / 2) + k / 2];
  int q = (k & 1) ? (byte >> 4) : (byte & 15);
  int e = sf[orc_sf_offset(r, k / 16, K / 16, layout)];
  return orc_e2m1_value(q) * orc_e4m3_decode(e) * alpha; /* exact in fp64 */
}

/* A = [M, K] codes (K-major) with scales, B = [N, K] likewise; Y = A B^T.
 * For each of the n pairs (mi[i], ni[i]) writes y[i] = the exact dot product
 * of the dequantized rows, accumulated in fp64 in increasing k, and
 * s[i] = sum_k |a^ b^| (the tolerance scale). */
void orc_gemm_pairs(const uint8_t* a_codes, const uint8_t* a_sf, float a_alpha,
                    int a_layout, const uint8_t* b_codes, const uint8_t* b_sf,
                    float b_alpha, int b_layout, int64_t K, int64_t n,
                    const int64_t* mi, const int64_t* ni, double* y, double* s) {
  for (int64_t i = 0; i < n; ++i) {
    double acc = 0.0, sabs = 0.0;
    for (int64_t k = 0; k < K; ++k) {
      double p = deq64(a_codes, a_sf, a_alpha, mi[i], k, K, a_layout) *
                 deq64(b_codes, b_sf, b_alpha, ni[i], k, K, b_layout);
      acc += p;
      sabs += fabs(p);
    }
    y[i] = acc;
    s[i] = sabs;
  }
}

/* Full [M, N] output (row-major) -- small shapes only. */
void orc_gemm(const uint8_t* a_codes, const uint8_t* a_sf, float a_alpha,
              int a_layout, const uint8_t* b_codes, const uint8_t* b_sf,
              float b_alpha, int b_layout, int64_t M, int64_t N, int64_t K,
              double* y, double* s) {
  double* ad = (double*)malloc((size_t)(M * K) * sizeof(double));
  double* bd = (double*)malloc((size_t)(N * K) * sizeof(double));
  if (!ad || !bd) {
    free(ad);
    free(bd);
    return;
  }
  for (int64_t m = 0; m < M; ++m)
    for (int64_t k = 0; k < K; ++k)
      ad[m * K + k] = deq64(a_codes, a_sf, a_alpha, m, k, K, a_layout);
  for (int64_t nn = 0; nn < N; ++nn)
    for (int64_t k = 0; k < K; ++k)
      bd[nn * K + k] = deq64(b_codes, b_sf, b_alpha, nn, k, K, b_layout);
  for (int64_t m = 0; m < M; ++m)
    for (int64_t nn = 0; nn < N; ++nn) {
      double acc = 0.0, sabs = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        double p = ad[m * K + k] * bd[nn * K + k];
        acc += p;
        sabs += fabs(p);
      }
      y[m * N + nn] = acc;
      s[m * N + nn] = sabs;
    }
  free(ad);
  free(bd);
}

/* Low-rank branch of a quantized LoRA linear layer (notes, §3.4 "NVFP4
 * training and DMD LoRA": the frozen backbone's weight stays quantized and a
 * bf16 rank-r adapter adds scale * B (A x); overview: W ~ Dequant(Q(W0)) +
 * delta W).  Reading: the adapter's first product u = x A^T [M, r] is
 * given (bf16 widened to fp32), the branch adds scale * u B^T to the base
 * output.  y[m, n] += scale * sum_j u[m, j] bl[n, j] and
 * s[m, n] += |scale| * sum_j |u[m, j] bl[n, j]| (the tolerance scale), the
 * sum in fp64 in increasing j; y, s row-major [M, N]. */
void orc_lora_add(const float* u, const float* bl, int64_t M, int64_t N, int64_t r,
                  double scale, double* y, double* s) {
  for (int64_t m = 0; m < M; ++m)
    for (int64_t nn = 0; nn < N; ++nn) {
      double acc = 0.0, sabs = 0.0;
      for (int64_t j = 0; j < r; ++j) {
        const double p = (double)u[m * r + j] * (double)bl[nn * r + j];
        acc += p;
        sabs += fabs(p);
      }
      y[m * N + nn] += scale * acc;
      s[m * N + nn] += fabs(scale) * sabs;
    }
}

/* GELU, tanh approximation (Hendrycks & Gimpel, 2016), in double. */
double orc_gelu_tanh(double x) {
  const double k0 = 0.7978845608028654; /* sqrt(2/pi) */
  return 0.5 * x * (1.0 + tanh(k0 * (x + 0.044715 * x * x * x)));
}
