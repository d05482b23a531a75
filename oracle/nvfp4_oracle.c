/*
 * nvfp4_oracle.c -- plain, slow CPU oracle of the NVFP4 W4A4 path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check and
 * the bench harness's CPU-baseline / reference legs may load this library.  It
 * shares no code, header, table or constant generator with the CUDA library;
 * neither side includes or links the other.
 *
 * What it computes (sources: the LongLive-2.0 pages):
 *  - neurohive.io, "LongLive-2.0: NVIDIA научила модель генерировать длинное
 *    видео ... с квантованием NVFP4", section "Ключевые компоненты LongLive-2.0",
 *    NVFP4 paragraph: each element is E2M1 (2 exponent bits, 1 mantissa bit),
 *    with a block scale per 16 elements and a per-tensor scale; applied to the
 *    weights and activations of the DiT linear layers.
 *  - tailorednewshub.com, "LongLive-2.0: Infraestructura paralela NVFP4 para
 *    video largo", section "Entrenamiento NVFP4": the block scale is FP8 and the
 *    tensor scale FP32; section "Inferencia W4A4 NVFP4": BF16 GEMMs become FP4
 *    GEMMs and the KV cache is stored as NVFP4.
 *  - hyper.ai, LongLive-2.0 paper summary, section "方法" (Method), second
 *    paragraph: the KV cache is quantized in frame blocks of eight frames and
 *    rebuilt by a dequantization kernel for windowed attention.
 *  - 171host.com, "LongLive 2.0 技术拆解", section 2.2: a local window of 9
 *    latent frames plus 3 permanent sink frames.
 *
 * The pages fix the format but not the scale recipe; the recipe below is the
 * one this project adopts (amax / (6*448) tensor scale, RNE everywhere), and
 * every open reading is listed with the design notes.
 *
 * Arithmetic: every float operation is a single IEEE-754 binary32 operation
 * rounded to nearest-even (compile with -ffp-contract=off, no fast-math), in
 * the order written.  Nearest-value searches are brute force over the format's
 * value set in binary64.  GEMM references are binary64 sums of exactly
 * dequantized operands.
 *
 * KV scale rule "Four Over Six" (tailorednewshub.com article, section
 * "Inferencia W4A4 NVFP4": the KV cache uses micro-block scaling with an
 * adaptive scale choice named Four Over Six; the pages give no formula).  The
 * reading taken here: per 16-element block, scale the block maximum onto 6
 * (the standard rule) or onto 4, quantize with each, and keep the one whose
 * squared error against the exactly decoded values is smaller (ties keep 6).
 *
 * FFN activation (GEMM epilogue option): GELU in its tanh form,
 * 0.5 y (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3))), in binary64 with the C
 * library's tanh.  The DiT's blocks are attention and FFN (171host.com
 * teardown, usage section "训练管线": LoRA on Attn/FFN); the pages name no
 * activation, and the tanh form is the reading taken.
 *
 * Windowed attention over the cache (the consumer of the window rebuild:
 * hyper.ai summary, section "方法"; 3 sinks + 9 window frames, 171host.com
 * section 2.2): out = softmax(scale * q k^T) v over the window's tokens in
 * slot-list order, every query seeing every window token, in binary64 on the
 * bf16 K and V the window rebuild produces.
 *
 * Parity pins (tests/test_oracle_*.py): exhaustive decode of all 16 E2M1 codes
 * and 256 E4M3 bytes against ml_dtypes / torch, encode against the same
 * libraries on tie and random values, exact round trips of representable
 * tensors, the per-block error bound, the 16 / 4.5-bit size ratio printed on
 * the pages (~3.6x), and tiny GEMMs against numpy and closed forms.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_ARG 1        /* bad shape / argument */
#define ORC_ERR_NONFINITE 2  /* an input element is NaN or Inf */
#define ORC_ERR_DOMAIN 3     /* tensor scale outside {0} U [2^-108, 2^100] */

/* ------------------------------------------------------------------ */
/* threads                                                             */
/* ------------------------------------------------------------------ */
int orc_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
  return omp_get_max_threads();
#else
  (void)n;
  return 1;
#endif
}

/* ------------------------------------------------------------------ */
/* Format definitions                                                  */
/* ------------------------------------------------------------------ */

/* E2M1 value of a 4-bit code: sign bit 3, exponent bits 2..1 (bias 1),
 * mantissa bit 0; exponent 0 is subnormal (m * 0.5).  No Inf, no NaN. */
double orc_e2m1_value(int code) {
  int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return s ? -v : v;
}

/* OCP FP8 E4M3 ("fn") value of a byte: sign bit 7, exponent bits 6..3
 * (bias 7), mantissa bits 2..0; exponent 0 is subnormal (m/8 * 2^-6);
 * exponent 15 with mantissa 7 is NaN; there is no Inf. */
double orc_e4m3_value(int byte) {
  int s = (byte >> 7) & 1, e = (byte >> 3) & 15, m = byte & 7;
  if (e == 15 && m == 7) return NAN;
  double v = (e == 0) ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
  return s ? -v : v;
}

/* E4M3 round-to-nearest-even with saturation: the nearest of the 127
 * non-negative finite values (codes 0x00..0x7E) to |r|; on a tie the code
 * with an even last bit; sign bit copied from r.  Values at or above 448
 * saturate to 448 (taken first: for huge |r| the binary64 distances would
 * no longer separate the candidates).  Below 448 every distance to the two
 * neighbours of |r| is exact in binary64. */
int orc_e4m3_encode(float r) {
  double x = fabs((double)r);
  if (x >= 448.0) return 0x7E | (signbit(r) ? 0x80 : 0); /* saturation */
  int best = 0;
  double bd = x; /* distance to code 0 (value 0) */
  for (int c = 1; c <= 0x7E; ++c) {
    double d = fabs(x - orc_e4m3_value(c));
    if (d < bd || (d == bd && (c & 1) == 0)) { best = c; bd = d; }
  }
  return best | (signbit(r) ? 0x80 : 0);
}

/* E2M1 round-to-nearest-even with saturation: the nearest of the 8
 * magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6} to |y|, ties to the even code,
 * sign bit copied from y (so a negative value that rounds to zero is -0).
 * |y| >= 6 saturates to 6. */
int orc_e2m1_encode(float y) {
  double x = fabs((double)y);
  if (x >= 6.0) return 7 | (signbit(y) ? 0x8 : 0); /* saturation */
  int best = 0;
  double bd = x;
  for (int c = 1; c <= 7; ++c) {
    double d = fabs(x - orc_e2m1_value(c));
    if (d < bd || (d == bd && (c & 1) == 0)) { best = c; bd = d; }
  }
  return best | (signbit(y) ? 0x8 : 0);
}

static float f32_from_bits(uint32_t b) { float f; memcpy(&f, &b, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t b; memcpy(&b, &f, 4); return b; }

/* binary32 -> bfloat16, round to nearest even.  bfloat16 values are the
 * binary32 values whose low 16 bits are zero; pick the nearer of the two
 * neighbours of f (toward zero, away from zero), ties to the even one.  The
 * neighbour past the largest finite bfloat16 is Inf, placed at 2^128 for the
 * distance, as IEEE overflow rounding does. */
uint16_t orc_bf16_from_f32(float f) {
  uint32_t b = bits_from_f32(f);
  if (isnan(f)) return (uint16_t)((b >> 16) | 0x40);
  uint32_t t = b & 0xFFFF0000u;          /* toward zero */
  uint32_t u = t + 0x10000u;             /* away from zero (same sign) */
  double ft = (double)f32_from_bits(t);
  double fu = ((u & 0x7F800000u) == 0x7F800000u)
                  ? copysign(ldexp(1.0, 128), (double)f)
                  : (double)f32_from_bits(u);
  double dt = fabs((double)f - ft), du = fabs(fu - (double)f);
  if (dt < du) return (uint16_t)(t >> 16);
  if (du < dt) return (uint16_t)(u >> 16);
  return (uint16_t)((((t >> 16) & 1u) == 0) ? (t >> 16) : (u >> 16));
}

float orc_f32_from_bf16(uint16_t h) { return f32_from_bits((uint32_t)h << 16); }

/* ------------------------------------------------------------------ */
/* Scale-factor layouts                                                */
/* ------------------------------------------------------------------ */

/* Byte offset of block scale (row, kb) in the tensor-core layout: 128-row x
 * 4-block tiles of 512 bytes, tiles ordered row-tile major then block-tile;
 * inside a tile, row r and block c sit at (r%32)*16 + ((r/32)%4)*4 + c%4.
 * nkb = number of 16-element blocks per row. */
int64_t orc_sf_mma_offset(int64_t row, int64_t kb, int64_t nkb) {
  int64_t ktiles = (nkb + 3) / 4;
  int64_t tile = (row / 128) * ktiles + kb / 4;
  return tile * 512 + (row % 32) * 16 + ((row / 32) % 4) * 4 + (kb % 4);
}

int64_t orc_sf_mma_bytes(int64_t rows, int64_t cols) {
  return ((rows + 127) / 128) * 128 * (((cols / 16) + 3) / 4) * 4;
}

/* Permute row-major block scales [rows][nkb] into the tensor-core layout
 * (padding bytes zero). */
int orc_sf_to_mma(const uint8_t* sf, int64_t rows, int64_t cols, uint8_t* out) {
  if (cols % 16) return ORC_ERR_ARG;
  int64_t nkb = cols / 16;
  memset(out, 0, (size_t)orc_sf_mma_bytes(rows, cols));
  for (int64_t i = 0; i < rows; ++i)
    for (int64_t kb = 0; kb < nkb; ++kb)
      out[orc_sf_mma_offset(i, kb, nkb)] = sf[i * nkb + kb];
  return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Quantize (steps: tensor amax -> s_t; block amax -> s_b; codes)      */
/* ------------------------------------------------------------------ */

/* dtype: 0 = bfloat16 bits (uint16), 1 = float32 */
static float load_elem(const void* x, int dtype, int64_t idx) {
  if (dtype == 0) return orc_f32_from_bf16(((const uint16_t*)x)[idx]);
  return ((const float*)x)[idx];
}

static int s_t_in_domain(float s_t) {
  return s_t == 0.0f || (s_t >= ldexpf(1.0f, -108) && s_t <= ldexpf(1.0f, 100));
}

/* Tensor scale: s_t = amax / (6 * 448) with amax = max |x| over the
 * tensor (one binary32 division).  Returns ORC_ERR_NONFINITE if any element
 * is NaN/Inf. */
int orc_tensor_scale(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                     float* amax_out, float* s_t_out) {
  if (rows < 0 || cols < 0 || ld < cols) return ORC_ERR_ARG;
  float amax = 0.0f;
  int bad = 0;
#pragma omp parallel for reduction(max : amax) reduction(| : bad) schedule(static)
  for (int64_t i = 0; i < rows; ++i)
    for (int64_t j = 0; j < cols; ++j) {
      float v = load_elem(x, dtype, i * ld + j);
      if (!isfinite(v)) bad = 1;
      else amax = fmaxf(amax, fabsf(v));
    }
  if (bad) return ORC_ERR_NONFINITE;
  if (amax_out) *amax_out = amax;
  *s_t_out = amax / 2688.0f; /* 2688 = 6 * 448 */
  return ORC_OK;
}

/* Block scale of one 16-element block: r = amax_b / (6 * s_t) (the product
 * rounded first, then one division), s_b = E4M3_RNE_sat(r).  s_t == 0 gives
 * s_b = 0. */
int orc_block_scale(float amax_b, float s_t) {
  if (s_t == 0.0f) return 0;
  float six_st = 6.0f * s_t;
  float r = amax_b / six_st;
  return orc_e4m3_encode(r);
}

/* Code of one element: 0 when the block scale is 0; otherwise
 * d = s_b * s_t, y = x / d, q = E2M1_RNE_sat(y). */
int orc_element_code(float x, int s_b_byte, float s_t) {
  if (s_b_byte == 0) return 0;
  float s_b = (float)orc_e4m3_value(s_b_byte);
  float d = s_b * s_t;
  float y = x / d;
  return orc_e2m1_encode(y);
}

/* Block scale with the block maximum mapped onto `top` (6: the standard
 * rule; 4: the Four Over Six alternative): E4M3_RNE_sat(amax_b / (top * s_t)),
 * the product rounded first. */
static int block_scale_onto(float amax_b, float s_t, float top) {
  if (s_t == 0.0f) return 0;
  float t_st = top * s_t;
  float r = amax_b / t_st;
  return orc_e4m3_encode(r);
}

/* Squared error of a 16-element block coded with scale byte s_b, against the
 * exactly decoded values v(q) * s_b * s_t (exact in binary64): the sum, in
 * element order, of (|x_i| - v(|q_i|) * s_b * s_t)^2, each operation one
 * binary64 rounding. */
static double block_sq_error(const float* xs, int s_b, float s_t) {
  double e = 0.0;
  for (int t = 0; t < 16; ++t) {
    int q = orc_element_code(xs[t], s_b, s_t);
    double recon = orc_e2m1_value(q & 7) * orc_e4m3_value(s_b);
    recon = recon * (double)s_t;
    double diff = (double)fabsf(xs[t]) - recon;
    e = e + diff * diff;
  }
  return e;
}

/* Scale byte of a block under `rule` (0: onto 6; 1: Four Over Six). */
int orc_block_scale_rule(const float* xs, float s_t, int rule) {
  float amax_b = 0.0f;
  for (int t = 0; t < 16; ++t) amax_b = fmaxf(amax_b, fabsf(xs[t]));
  int s6 = block_scale_onto(amax_b, s_t, 6.0f);
  if (rule == 0) return s6;
  int s4 = block_scale_onto(amax_b, s_t, 4.0f);
  return block_sq_error(xs, s4, s_t) < block_sq_error(xs, s6, s_t) ? s4 : s6;
}

/* Quantize a rows x cols tensor (row stride ld elements) to NVFP4.
 *   codes: [rows][cols/2] bytes, element 2j in the low nibble of byte j
 *   sf:    [rows][cols/16] E4M3 bytes (row-major)
 *   s_t:   tensor scale (computed, or taken from *s_t_in when non-NULL)
 */
static int quantize_rule(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                         uint8_t* codes, uint8_t* sf, float* s_t_out, const float* s_t_in,
                         int rule) {
  if (cols % 16 != 0 || rows < 0 || ld < cols || (dtype != 0 && dtype != 1)) return ORC_ERR_ARG;
  float s_t;
  if (s_t_in) {
    s_t = *s_t_in;
  } else {
    int st = orc_tensor_scale(x, dtype, rows, cols, ld, NULL, &s_t);
    if (st) return st;
  }
  if (!s_t_in_domain(s_t)) return ORC_ERR_DOMAIN;
  int64_t nkb = cols / 16;
  int bad = 0;
#pragma omp parallel for reduction(| : bad) schedule(static)
  for (int64_t i = 0; i < rows; ++i) {
    for (int64_t kb = 0; kb < nkb; ++kb) {
      float xs[16];
      float amax_b = 0.0f;
      for (int t = 0; t < 16; ++t) {
        xs[t] = load_elem(x, dtype, i * ld + kb * 16 + t);
        if (!isfinite(xs[t])) bad = 1;
        amax_b = fmaxf(amax_b, fabsf(xs[t]));
      }
      int s_b = rule == 0 ? orc_block_scale(amax_b, s_t) : orc_block_scale_rule(xs, s_t, rule);
      sf[i * nkb + kb] = (uint8_t)s_b;
      for (int t = 0; t < 16; t += 2) {
        int q0 = orc_element_code(xs[t], s_b, s_t);
        int q1 = orc_element_code(xs[t + 1], s_b, s_t);
        codes[i * (cols / 2) + kb * 8 + t / 2] = (uint8_t)(q0 | (q1 << 4));
      }
    }
  }
  if (bad) return ORC_ERR_NONFINITE;
  *s_t_out = s_t;
  return ORC_OK;
}

int orc_quantize(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                 uint8_t* codes, uint8_t* sf, float* s_t_out, const float* s_t_in) {
  return quantize_rule(x, dtype, rows, cols, ld, codes, sf, s_t_out, s_t_in, 0);
}

/* ------------------------------------------------------------------ */
/* Dequantize                                                          */
/* ------------------------------------------------------------------ */

/* One element: bf16_RNE( (v(q) * s_b) * s_t ); v(q)*s_b is exact in
 * binary32, the product with s_t is one binary32 rounding. */
uint16_t orc_dequant_elem(int code, int s_b_byte, float s_t) {
  float v = (float)orc_e2m1_value(code);
  float s_b = (float)orc_e4m3_value(s_b_byte);
  float vs = v * s_b;
  float f = vs * s_t;
  return orc_bf16_from_f32(f);
}

/* codes/sf as produced by orc_quantize (row-major sf) -> bf16 [rows][cols] */
int orc_dequantize(const uint8_t* codes, const uint8_t* sf, float s_t, int64_t rows,
                   int64_t cols, uint16_t* out) {
  if (cols % 16 != 0 || rows < 0) return ORC_ERR_ARG;
  int64_t nkb = cols / 16;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < rows; ++i)
    for (int64_t j = 0; j < cols; ++j) {
      int byte = codes[i * (cols / 2) + j / 2];
      int q = (j % 2 == 0) ? (byte & 0xF) : (byte >> 4);
      out[i * cols + j] = orc_dequant_elem(q, sf[i * nkb + j / 16], s_t);
    }
  return ORC_OK;
}

/* Exact dequantized value v(q) * s_b * s_t in binary64 (exact: at most
 * 2 + 4 + 24 significant bits). */
int orc_dequantize_exact(const uint8_t* codes, const uint8_t* sf, float s_t, int64_t rows,
                         int64_t cols, double* out) {
  if (cols % 16 != 0 || rows < 0) return ORC_ERR_ARG;
  int64_t nkb = cols / 16;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < rows; ++i)
    for (int64_t j = 0; j < cols; ++j) {
      int byte = codes[i * (cols / 2) + j / 2];
      int q = (j % 2 == 0) ? (byte & 0xF) : (byte >> 4);
      out[i * cols + j] = orc_e2m1_value(q) * orc_e4m3_value(sf[i * nkb + j / 16]) * (double)s_t;
    }
  return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* GEMM reference                                                      */
/* ------------------------------------------------------------------ */

/* y[m][n] = sum_k a[m][k] * w[n][k] and S[m][n] = sum_k |a[m][k] * w[n][k]|
 * in binary64, where a and w are the exactly dequantized NVFP4 operands
 * (A: M x K, W: N x K, both with row-major block scales).  Only the rows
 * listed in row_ids (n_rows of them) are computed; y and S are
 * [n_rows][N].  row_ids == NULL means all M rows. */
int orc_gemm(const uint8_t* a_codes, const uint8_t* a_sf, float a_st, const uint8_t* w_codes,
             const uint8_t* w_sf, float w_st, int64_t M, int64_t N, int64_t K,
             const int64_t* row_ids, int64_t n_rows, double* y, double* S) {
  if (K % 16 != 0 || M < 0 || N < 0) return ORC_ERR_ARG;
  if (!row_ids) n_rows = M;
  for (int64_t r = 0; r < n_rows; ++r) {
    int64_t m = row_ids ? row_ids[r] : r;
    if (m < 0 || m >= M) return ORC_ERR_ARG;
  }
  double* a = (double*)malloc(sizeof(double) * (size_t)(n_rows > 0 ? n_rows : 1) * (size_t)(K > 0 ? K : 1));
  if (!a) return ORC_ERR_ARG;
  for (int64_t r = 0; r < n_rows; ++r) {
    int64_t m = row_ids ? row_ids[r] : r;
    orc_dequantize_exact(a_codes + m * (K / 2), a_sf + m * (K / 16), a_st, 1, K, a + r * K);
  }
#pragma omp parallel
  {
    double* w = (double*)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
#pragma omp for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
      for (int64_t k = 0; k < K; ++k) {
        int byte = w_codes[n * (K / 2) + k / 2];
        int q = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
        w[k] = orc_e2m1_value(q) * orc_e4m3_value(w_sf[n * (K / 16) + k / 16]) * (double)w_st;
      }
      for (int64_t r = 0; r < n_rows; ++r) {
        double acc = 0.0, mag = 0.0;
        for (int64_t k = 0; k < K; ++k) {
          double p = a[r * K + k] * w[k];
          acc += p;
          mag += fabs(p);
        }
        y[r * N + n] = acc;
        S[r * N + n] = mag;
      }
    }
    free(w);
  }
  free(a);
  return ORC_OK;
}


/* GELU, tanh form, on n binary64 values: out[i] = 0.5 y (1 + tanh(c (y + 0.044715 y^3)))
 * with c = sqrt(2 / pi), each operation one binary64 rounding. */
int orc_gelu_tanh(const double* y, double* out, int64_t n) {
  if (n < 0) return ORC_ERR_ARG;
  const double c = sqrt(2.0 / 3.14159265358979323846);
  for (int64_t i = 0; i < n; ++i) {
    const double v = y[i];
    if (!isfinite(v)) return ORC_ERR_NONFINITE;
    const double inner = c * (v + 0.044715 * (v * v * v));
    out[i] = 0.5 * v * (1.0 + tanh(inner));
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* KV cache chunk codec                                                */
/* ------------------------------------------------------------------ */

/* Quantize one chunk of n_frames latent frames of K (or V), bf16
 * [n_frames*tpf tokens][heads][head_dim] with a token stride of
 * token_stride elements (head_dim contiguous, heads packed).  The tensor
 * scale is one per chunk (the chunk is the unit the pages quantize: blocks of
 * up to eight frames); blocks of 16 run along head_dim.  Frame f is written
 * to codes + f*frame_code_bytes and sf + f*frame_sf_bytes (row-major
 * [tpf][heads][head_dim/16]); its tensor scale to s_t[f]. */
int orc_kv_quant_chunk(const uint16_t* kv, int64_t token_stride, int n_frames, int tpf, int heads,
                       int head_dim, uint8_t* codes, uint8_t* sf, float* s_t, int rule) {
  if (head_dim % 16 != 0 || n_frames < 0 || tpf < 0 || heads < 0 ||
      token_stride < (int64_t)heads * head_dim || (rule != 0 && rule != 1))
    return ORC_ERR_ARG;
  int64_t tokens = (int64_t)n_frames * tpf;
  int64_t row_elems = (int64_t)heads * head_dim;
  /* gather the chunk into a dense [tokens][heads*head_dim] matrix, then the
   * chunk is one NVFP4 tensor of tokens*heads rows by head_dim columns */
  uint16_t* dense = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(tokens * row_elems + 1));
  if (!dense) return ORC_ERR_ARG;
  for (int64_t t = 0; t < tokens; ++t)
    memcpy(dense + t * row_elems, kv + t * token_stride, sizeof(uint16_t) * (size_t)row_elems);
  float st;
  int rc = quantize_rule(dense, 0, tokens * heads, head_dim, head_dim, codes, sf, &st, NULL, rule);
  free(dense);
  if (rc) return rc;
  for (int f = 0; f < n_frames; ++f) s_t[f] = st;
  return ORC_OK;
}

/* Rebuild bf16 K (or V) for a list of frame slots: out is
 * [n_slots*tpf][heads][head_dim], slot i taken from codes/sf/s_t of pool
 * slot slot_ids[i] (pool layout as written by orc_kv_quant_chunk, one frame
 * per slot). */
int orc_kv_dequant_window(const uint8_t* pool_codes, const uint8_t* pool_sf, const float* pool_st,
                          int n_pool, const int32_t* slot_ids, int n_slots, int tpf, int heads,
                          int head_dim, uint16_t* out) {
  if (head_dim % 16 != 0) return ORC_ERR_ARG;
  int64_t rows = (int64_t)tpf * heads;
  int64_t frame_codes = rows * head_dim / 2, frame_sf = rows * head_dim / 16;
  for (int i = 0; i < n_slots; ++i) {
    int s = slot_ids[i];
    if (s < 0 || s >= n_pool) return ORC_ERR_ARG;
    int rc = orc_dequantize(pool_codes + s * frame_codes, pool_sf + s * frame_sf, pool_st[s], rows,
                            head_dim, out + (int64_t)i * rows * head_dim);
    if (rc) return rc;
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* windowed attention                                                  */
/* ------------------------------------------------------------------ */

static double bf16_value(uint16_t b) { return (double)f32_from_bits((uint32_t)b << 16); }

/* q: bf16 bits, token t at q + t*q_stride, head h at +h*head_dim; k, v: bf16
 * bits [n_kv][heads][head_dim].  For each requested query token rows[r] (all
 * 0..n_rows-1 when rows is NULL) and head h:
 *   p_j = exp(scale * sum_d q[d] k_j[d] - max_j(...)) / sum_j exp(...),
 *   out[r][h][d] = sum_j p_j v_j[d],   E[r][h][d] = sum_j p_j |v_j[d]|,
 * each sum in index order, binary64. */
int orc_window_attention(const uint16_t* q, int64_t q_stride, const int64_t* rows, int64_t n_rows,
                         const uint16_t* k, const uint16_t* v, int64_t n_kv, int heads,
                         int head_dim, double scale, double* out, double* E) {
  if (n_rows < 0 || n_kv < 1 || heads < 1 || head_dim < 1 || !(scale > 0.0)) return ORC_ERR_ARG;
  int err = ORC_OK;
#pragma omp parallel for schedule(dynamic)
  for (int64_t r = 0; r < n_rows; ++r) {
    const int64_t t = rows ? rows[r] : r;
    double* logit = (double*)malloc((size_t)n_kv * sizeof(double));
    if (!logit) { err = ORC_ERR_ARG; continue; }
    for (int h = 0; h < heads; ++h) {
      const uint16_t* qh = q + t * q_stride + (int64_t)h * head_dim;
      double mx = -INFINITY;
      for (int64_t j = 0; j < n_kv; ++j) {
        const uint16_t* kj = k + (j * heads + h) * (int64_t)head_dim;
        double dot = 0.0;
        for (int d = 0; d < head_dim; ++d) dot += bf16_value(qh[d]) * bf16_value(kj[d]);
        logit[j] = scale * dot;
        if (logit[j] > mx) mx = logit[j];
      }
      double sum = 0.0;
      for (int64_t j = 0; j < n_kv; ++j) {
        logit[j] = exp(logit[j] - mx);
        sum += logit[j];
      }
      double* o = out + (r * heads + h) * (int64_t)head_dim;
      double* e = E + (r * heads + h) * (int64_t)head_dim;
      for (int d = 0; d < head_dim; ++d) o[d] = e[d] = 0.0;
      for (int64_t j = 0; j < n_kv; ++j) {
        const double p = logit[j] / sum;
        const uint16_t* vj = v + (j * heads + h) * (int64_t)head_dim;
        for (int d = 0; d < head_dim; ++d) {
          const double x = bf16_value(vj[d]);
          o[d] += p * x;
          e[d] += p * fabs(x);
        }
      }
    }
    free(logit);
  }
  return err;
}
