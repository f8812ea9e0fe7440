/*
 * fp8_oracle.c -- CPU oracle for the FP8 linear layer with delayed scaling.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file: only tests/, the smoke check and the benchmark's CPU-baseline leg
 * do.  It shares no header, table or helper with the CUDA library.
 *
 * It is written to be read against the source pages (the AstrAI commit logs),
 * not to be fast:
 *   - fp8 values come from a 256-entry table built from the format definitions
 *     (E4M3 "fn": bias 7, no infinities, S.1111.111 = NaN; E5M2: bias 15,
 *     IEEE-style inf/NaN);
 *   - the saturating round-to-nearest-even cast scans every finite code;
 *   - amax is the max of |x| over the RAW input values in fp32 (the pages fixed
 *     a bug where the quantized max was used: astrai/extension/fp8.py @3e57cc8,
 *     amax bullet; "fp32-domain amax references", astrai/extension/ops @057c0d3);
 *   - the scale ring step folds the new amax into hist[step % H], reduces the
 *     whole window with max and publishes fp8_max / max as the next scale
 *     (tests/extension @2eeac02, ring-finalize bullets);
 *   - GEMMs accumulate products in fp32 with k ascending, divide by the product
 *     of the two operand scales, add the bias in fp32 and round once to bf16
 *     (astrai @4019dda, fused-bias bullet; csrc @2eeac02, FP8Params bias
 *     bullet).  An exact integer dot (__int128) and sum |a_k b_k| are computed
 *     alongside for tolerance checks.
 * Parallelism: OpenMP over independent output rows only; every output element
 * is computed by the same sequential loop it would have single-threaded.
 * Build flags keep IEEE single precision exactly as written: no fast-math, no
 * FMA contraction (-ffp-contract=off); x86-64 evaluates float in float.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_E4M3 = 0, ORC_E5M2 = 1 };
enum { ORC_BF16 = 0, ORC_FP16 = 1, ORC_FP32 = 2, ORC_DT_E4M3 = 3, ORC_DT_E5M2 = 4 };

/* ---------------------------------------------------------------- formats */

/* Value of one fp8 code, straight from the bit-field definition. */
static double fp8_value(int fmt, int code) {
  int sign = (code >> 7) & 1;
  int e, m, ebits_max, bias, mbits;
  if (fmt == ORC_E4M3) { e = (code >> 3) & 0xF; m = code & 0x7; ebits_max = 15; bias = 7;  mbits = 3; }
  else                 { e = (code >> 2) & 0x1F; m = code & 0x3; ebits_max = 31; bias = 15; mbits = 2; }
  double v;
  if (fmt == ORC_E4M3) {
    if (e == ebits_max && m == 7) return NAN;          /* only NaN pattern: S.1111.111 */
  } else {
    if (e == ebits_max) return m == 0 ? (sign ? -INFINITY : INFINITY) : NAN;
  }
  if (e == 0) v = ldexp((double)m, 1 - bias - mbits);               /* subnormal */
  else        v = ldexp(1.0 + ldexp((double)m, -mbits), e - bias);  /* normal */
  return sign ? -v : v;
}

void orc_decode_table(int fmt, double* out256) {
  for (int c = 0; c < 256; ++c) out256[c] = fp8_value(fmt, c);
}

double orc_fp8_max(int fmt) { return fmt == ORC_E4M3 ? 448.0 : 57344.0; }

/* Largest finite positive code of each format. */
static int max_code(int fmt) { return fmt == ORC_E4M3 ? 0x7E : 0x7B; }

/* Value tables, filled once from fp8_value (call before any parallel region). */
static double g_tab[2][256];
static uint8_t g_enc_ready = 0;
static void ensure_tables(void) {
  if (g_enc_ready) return;
  orc_decode_table(ORC_E4M3, g_tab[0]);
  orc_decode_table(ORC_E5M2, g_tab[1]);
  g_enc_ready = 1;
}

/* Saturating, round-to-nearest-even cast of one fp32 value.  NaN -> 0x7F;
 * |v| >= fp8_max (inf included) -> +-max code; otherwise the nearest finite
 * grid value, found by scanning all non-negative finite codes, ties going to
 * the code whose mantissa LSB (= code LSB) is 0.  The sign is kept, so -0 and
 * negative values that round to zero give 0x80. */
uint8_t orc_encode(int fmt, float v) {
  ensure_tables();
  const double* tab = g_tab[fmt == ORC_E4M3 ? 0 : 1];
  if (isnan(v)) return 0x7F;
  uint8_t sign = signbit(v) ? 0x80 : 0x00;
  double a = fabs((double)v);
  int top = max_code(fmt);
  if (a >= tab[top]) return (uint8_t)(sign | top);
  int best = 0;
  double bestd = a;  /* distance to +0 (code 0) */
  for (int c = 1; c <= top; ++c) {
    double d = fabs(tab[c] - a);
    if (d < bestd || (d == bestd && (c & 1) == 0)) { best = c; bestd = d; }
  }
  return (uint8_t)(sign | best);
}

/* ------------------------------------------------------------ bf16 / fp16 */

static float bits_to_f32(uint32_t b) { float f; memcpy(&f, &b, 4); return f; }
static uint32_t f32_to_bits(float f) { uint32_t b; memcpy(&b, &f, 4); return b; }

float orc_bf16_to_f32(uint16_t h) { return bits_to_f32((uint32_t)h << 16); }

/* IEEE binary16 -> fp32 from the definition (exact). */
float orc_fp16_to_f32(uint16_t h) {
  int s = (h >> 15) & 1, e = (h >> 10) & 0x1F, m = h & 0x3FF;
  double v;
  if (e == 0x1F) v = m ? NAN : INFINITY;
  else if (e == 0) v = ldexp((double)m, -24);
  else v = ldexp(1.0 + ldexp((double)m, -10), e - 15);
  return (float)(s ? -v : v);
}

/* fp32 -> bf16, round to nearest, ties to even.  The two candidates are the
 * bf16 values just below and just above |v| (bf16 = fp32 with the low 16 bits
 * zero); past the largest finite bf16 the upper candidate is 2^128 (= inf). */
uint16_t orc_bf16_rne(float v) {
  if (isnan(v)) return 0x7FC0;
  uint32_t b = f32_to_bits(v);
  uint32_t lo = b & 0xFFFF0000u;
  if (lo == b) return (uint16_t)(lo >> 16);
  uint32_t hi = lo + 0x10000u;
  double dv = fabs((double)v);
  double vlo = fabs((double)bits_to_f32(lo));
  double vhi = ((hi & 0x7FFFFFFFu) == 0x7F800000u) ? ldexp(1.0, 128) : fabs((double)bits_to_f32(hi));
  double dlo = dv - vlo, dhi = vhi - dv;
  if (dlo < dhi) return (uint16_t)(lo >> 16);
  if (dhi < dlo) return (uint16_t)(hi >> 16);
  return (uint16_t)((((lo >> 16) & 1u) == 0) ? (lo >> 16) : (hi >> 16));
}

static float load_in(const void* p, int dtype, int64_t idx) {
  switch (dtype) {
    case ORC_BF16: return orc_bf16_to_f32(((const uint16_t*)p)[idx]);
    case ORC_FP16: return orc_fp16_to_f32(((const uint16_t*)p)[idx]);
    case ORC_FP32: return ((const float*)p)[idx];
    default: return NAN;
  }
}

/* ------------------------------------------------------------ quantize */

/* amax = max |x| over all non-NaN elements, taken on the raw input values
 * (a max is independent of evaluation order, so rows may run in parallel). */
float orc_amax(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld) {
  float m = 0.0f;
#pragma omp parallel for reduction(max : m) schedule(static)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) {
      float v = load_in(x, dtype, r * ld + c);
      if (isnan(v)) continue;
      float a = fabsf(v);
      if (a > m) m = a;
    }
  return m;
}

/* q = encode(fp32(x) * s): the product is one IEEE fp32 multiply (rounded to
 * nearest even), then the saturating RNE cast.  Bytes between cols and ld_out
 * are written as zero. */
void orc_quantize(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld_in,
                  int fmt, float s, uint8_t* out, int64_t ld_out) {
  ensure_tables();
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t c = 0; c < cols; ++c) {
      float p = load_in(x, dtype, r * ld_in + c) * s;
      out[r * ld_out + c] = orc_encode(fmt, p);
    }
    for (int64_t c = cols; c < ld_out; ++c) out[r * ld_out + c] = 0;
  }
}

/* ------------------------------------------------------------ scale ring */

/* One delayed-scaling ring step.  hist has H slots (slots never written hold
 * 0).  The new amax goes to hist[step % H]; the window max m is taken over all
 * H slots, the current amax included; the next scale is fp8_max / m (one IEEE
 * fp32 division) when m is positive and finite and the quotient is finite,
 * otherwise the previous scale stays.  Returns the new scale; *step advances. */
float orc_ring_step(float* hist, int H, uint32_t* step, float scale, float amax, int fmt) {
  hist[*step % (uint32_t)H] = amax;
  float m = 0.0f;
  for (int i = 0; i < H; ++i) if (hist[i] > m) m = hist[i];
  *step += 1;
  float fmax = (float)orc_fp8_max(fmt);
  if (!(m > 0.0f) || isinf(m)) return scale;
  float s2 = fmax / m;
  if (isinf(s2)) return scale;
  return s2;
}

/* ------------------------------------------------------------ GEMM */

/* Integer image of an fp8 value: E4M3 = i * 2^-9, E5M2 = i * 2^-16. */
static int fmt_shift(int fmt) { return fmt == ORC_E4M3 ? 9 : 16; }

/* C[i,j] = sum_k A(i,k) * B(j,k) with A(i,k) = a[i*a_si + k*a_sk] and
 * B(j,k) = b[j*b_sj + k*b_sk] (strides in elements), so one routine serves the
 * forward (X W^T), dX (G W) and dW (G^T X) layouts.
 *   acc_f32[i*J+j]: products accumulated in fp32, k = 0,1,...,Kc-1;
 *   exact[i*J+j]  : the exact dot (int128), rounded once to double (optional);
 *   sumabs[i*J+j] : sum_k |A(i,k) B(j,k)| in double (optional).
 * Non-finite operands follow IEEE fp32 arithmetic (the pages state fp32
 * accumulation and nothing on special values): a NaN operand, an inf x 0
 * product or products of both infinite signs make the output NaN, other
 * infinite products make it +-inf; then all three outputs hold that value. */
void orc_gemm(int64_t I, int64_t J, int64_t Kc,
              const uint8_t* a, int fmt_a, int64_t a_si, int64_t a_sk,
              const uint8_t* b, int fmt_b, int64_t b_sj, int64_t b_sk,
              float* acc_f32, double* exact, double* sumabs) {
  ensure_tables();
  const double* ta = g_tab[fmt_a];
  const double* tb = g_tab[fmt_b];
  const double ua = ldexp(1.0, fmt_shift(fmt_a)), ub = ldexp(1.0, fmt_shift(fmt_b));
  const int sh = fmt_shift(fmt_a) + fmt_shift(fmt_b);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < I; ++i) {
    for (int64_t j = 0; j < J; ++j) {
      float acc = 0.0f;
      __int128 ex = 0;
      double sa = 0.0;
      int finite = 1;
      for (int64_t k = 0; k < Kc; ++k) {
        double va = ta[a[i * a_si + k * a_sk]];
        double vb = tb[b[j * b_sj + k * b_sk]];
        float p = (float)(va * vb);  /* exact for finite operands (at most 8 significant bits) */
        acc = acc + p;               /* IEEE fp32: inf and NaN propagate as fp32 arithmetic does */
        if (!isfinite(va) || !isfinite(vb)) { finite = 0; continue; }
        if (exact) ex += (__int128)(int64_t)(va * ua) * (__int128)(int64_t)(vb * ub);
        if (sumabs) sa += fabs(va * vb);
      }
      if (!finite) {  /* acc is +-inf or NaN: the exact sum is that value too */
        acc_f32[i * J + j] = acc;
        if (exact) exact[i * J + j] = acc;
        if (sumabs) sumabs[i * J + j] = fabs(acc);
        continue;
      }
      acc_f32[i * J + j] = acc;
      if (exact) exact[i * J + j] = ldexp((double)ex, -sh);
      if (sumabs) sumabs[i * J + j] = sa;
    }
  }
}

/* The same dot products for a list of n (i, j) output coordinates only, for
 * sampled checks of shapes whose full product is too slow on the CPU.  Each
 * point is the loop of orc_gemm for that (i, j): fp32 accumulation with k
 * ascending, sum |a_k b_k| in double; with a NaN or infinite operand the
 * accumulator is whatever IEEE fp32 arithmetic makes of it (NaN, or +-inf)
 * and so is the sum of magnitudes. */
void orc_gemm_points(int64_t n, const int64_t* ii, const int64_t* jj, int64_t Kc,
                     const uint8_t* a, int fmt_a, int64_t a_si, int64_t a_sk,
                     const uint8_t* b, int fmt_b, int64_t b_sj, int64_t b_sk,
                     float* acc_f32, double* sumabs) {
  ensure_tables();
  const double* ta = g_tab[fmt_a];
  const double* tb = g_tab[fmt_b];
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < n; ++t) {
    int64_t i = ii[t], j = jj[t];
    float acc = 0.0f;
    double sa = 0.0;
    int finite = 1;
    for (int64_t k = 0; k < Kc; ++k) {
      double va = ta[a[i * a_si + k * a_sk]];
      double vb = tb[b[j * b_sj + k * b_sk]];
      float p = (float)(va * vb);
      acc = acc + p;
      if (!isfinite(va) || !isfinite(vb)) { finite = 0; continue; }
      sa += fabs(va * vb);
    }
    acc_f32[t] = acc;
    sumabs[t] = finite ? sa : fabs(acc);
  }
}

/* Epilogue for n accumulator values laid out [rows, cols] (row stride cols):
 * v = acc / (sa * sb) in fp32, plus the bias of column j in fp32, then one
 * RNE rounding to bf16.  bias_dtype ORC_BF16 reads bf16 bias; ORC_DT_E4M3 /
 * ORC_DT_E5M2 read an fp8 bias whose value is decode(b8) / bias_scale.  A NULL
 * bias adds nothing.  col_idx (optional) gives the column of each value when
 * the values are scattered samples rather than a dense [rows, cols] block. */
void orc_epilogue(int64_t rows, int64_t cols, const float* acc, float sa, float sb,
                  const void* bias, int bias_dtype, float bias_scale,
                  const int64_t* col_idx, uint16_t* out_bf16, float* out_f32) {
  ensure_tables();
  float den = sa * sb;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) {
      int64_t t = r * cols + c;
      int64_t j = col_idx ? col_idx[t] : c;
      float v = acc[t] / den;
      if (bias) {
        float bv;
        if (bias_dtype == ORC_BF16) bv = orc_bf16_to_f32(((const uint16_t*)bias)[j]);
        else {
          float d = (float)g_tab[bias_dtype == ORC_DT_E4M3 ? 0 : 1][((const uint8_t*)bias)[j]];
          bv = d / bias_scale;
        }
        v = v + bv;
      }
      if (out_f32) out_f32[t] = v;
      out_bf16[t] = orc_bf16_rne(v);
    }
}

/* ------------------------------------------------------------ dbias */

/* dbias[n] = bf16( sum_m g[m,n] ), the sum in fp32 with m ascending.  A bf16 /
 * fp16 / fp32 g is read as is; an fp8 g (dtype ORC_DT_E4M3 / ORC_DT_E5M2) is
 * dequantized element by element first, decode(g8) / sg, as the pages require
 * before the bias sum (astrai/extension/ops @057c0d3, grad dtype bullet). */
void orc_dbias(const void* g, int dtype, int64_t M, int64_t N, int64_t ld, float sg,
               uint16_t* out_bf16, float* out_f32, double* out_sumabs) {
  ensure_tables();
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    float s = 0.0f;
    double sa = 0.0;
    for (int64_t m = 0; m < M; ++m) {
      float v;
      if (dtype == ORC_DT_E4M3 || dtype == ORC_DT_E5M2) {
        float d = (float)g_tab[dtype == ORC_DT_E4M3 ? 0 : 1][((const uint8_t*)g)[m * ld + n]];
        v = d / sg;
      } else {
        v = load_in(g, dtype, m * ld + n);
      }
      s = s + v;
      sa += fabs((double)v);
    }
    out_bf16[n] = orc_bf16_rne(s);
    if (out_f32) out_f32[n] = s;
    if (out_sumabs) out_sumabs[n] = sa;
  }
}

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ------------------------------------------------------------ array helpers */

void orc_encode_array(int fmt, const float* v, int64_t n, uint8_t* out) {
  ensure_tables();
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = orc_encode(fmt, v[i]);
}

void orc_bf16_rne_array(const float* v, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_rne(v[i]);
}
