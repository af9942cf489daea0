/*
 * oracle.c -- plain scalar CPU oracle for the quantized decoder projection
 *             Y = (s_x (x) s_w) . (Q(X) . W_q^T)
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link or
 * call this file: only the tests, the smoke check and the benchmark's CPU
 * baseline use it.  It shares no code, header, table or constant with the CUDA
 * library; the two meet only through the seeded inputs.
 *
 * It is deliberately slow and obvious: one scalar loop per definition, exact
 * integer accumulation, and IEEE single precision exactly where the method
 * computes a scale or a quotient.  Build with -O2 -ffp-contract=off and no
 * fast-math so that every float expression is one IEEE operation.
 *
 * Sources (cited by page title and section):
 *  [W8A8]  "Llama 3.1 8B Instruct W8A8" model page, intro paragraph: int8
 *          weights, a bf16 scale for each output row, activations quantized to
 *          int8 per token; "Loading": int8 products accumulated in int32.
 *  [FP8R]  "Meta-Llama-3.1-8B-Instruct-FP8-dynamic" README, "Model
 *          Optimizations" and the "Creation" recipe: FP8 weights, per-channel
 *          static symmetric; FP8 activations, per-token dynamic symmetric.
 *  [FP8B]  "Qwen3 8B FP8" model page, intro paragraph: E4M3 weights with one
 *          scale per 128x128 block, the scale a multiplier; widths multiples
 *          of 128; "Loading": activations quantized to FP8 in groups of 128.
 *  [OCP]   OCP 8-bit Floating Point Specification (E4M3: bias 7, three
 *          mantissa bits, no infinities, S.1111.111 is NaN, max 448).
 *
 * Readings where the pages are silent (each restated in the design notes):
 *  - symmetric scale = absmax / 127 (int8) or absmax / 448 (E4M3), one IEEE
 *    f32 division; quantize by the IEEE f32 quotient x / s, then round half
 *    to even; int8 clamps to [-127, 127], E4M3 saturates to +-448.
 *  - an all-zero row / token / group gets scale 0 and codes 0.
 *  - the W8A8 weight scale is rounded to bf16 first and the weights are
 *    quantized with that rounded scale; FP8 scales stay f32.
 *  - row-scheme epilogue: y = bf16( ((float)acc * s_x[m]) * s_w[n] ), f32
 *    left to right; block scheme: y = bf16( sum_kb P_kb * s_x[m,kb] *
 *    s_w[n/128,kb] ) with P_kb exact and the sum in f64, rounded once.
 *  - weight-only ("equivalent") product: the activations are not rounded at
 *    all; each weight is dequantized (code x its row or block scale, exact in
 *    f64), multiplied by the bf16 activation (exact in f64), summed in f64 and
 *    rounded once to bf16.  Only that f64 sum rounds: its error is at most
 *    (K-1) 2^-53 sum_k |x w|.
 */
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

/* Planted mistakes for the mutation test (tests/test_oracle_mutants.py):
 * the default build has ORACLE_MUTANT 0 and none of them. */
#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif
#define MUTANT(n) (ORACLE_MUTANT == (n))

#define ORACLE_INT8_ROW 0
#define ORACLE_FP8_ROW 1
#define ORACLE_FP8_BLOCK 2

/* ------------------------------------------------------------------------ */
/* Codecs                                                                   */
/* ------------------------------------------------------------------------ */

/* bf16 -> f32: a bf16 is the top half of an f32 (exact). */
float oracle_bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* f32 -> bf16, round half to even on the dropped 16 bits (finite inputs;
 * NaN is kept quiet). */
uint16_t oracle_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40u);
  uint32_t lsb = (u >> 16) & 1u;
  if (!MUTANT(1)) u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

/* f64 -> bf16 with a single rounding (half to even).  bf16 keeps 8
 * significant bits over the f32 exponent range; below 2^-126 its spacing is
 * the fixed 2^-133. */
uint16_t oracle_f64_to_bf16(double v) {
  double a = fabs(v);
  double r;
  if (a == 0.0) {
    r = 0.0;
  } else if (a < ldexp(1.0, -126)) {
    r = ldexp(nearbyint(ldexp(a, 133)), -133);
  } else {
    int e;
    double fr = frexp(a, &e); /* a = fr * 2^e, fr in [0.5, 1) */
    r = ldexp(nearbyint(ldexp(fr, 8)), e - 8);
  }
  uint16_t sign = signbit(v) ? 0x8000u : 0u;
  if (r > 3.3895313892515355e38) return sign | 0x7F80u; /* beyond the largest bf16: inf */
  float f = (float)r; /* exact: r has at most 8 significant bits */
  uint32_t u;
  memcpy(&u, &f, 4);
  return sign | (uint16_t)(u >> 16);
}

/* E4M3 code -> value [OCP]: sign, 4-bit exponent (bias 7), 3-bit mantissa;
 * exponent field 0 is subnormal (m * 2^-9); 0x7F / 0xFF are NaN. */
double oracle_e4m3_decode(uint8_t c) {
  int s = (c >> 7) & 1, e = (c >> 3) & 15, m = c & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m, -9);
  else
    v = ldexp(1.0 + m / 8.0, e - 7);
  return s ? -v : v;
}

/* f32 -> E4M3 [OCP], round to nearest, ties to the even code, saturating to
 * +-448 (code 0x7E / 0xFE); the sign of zero is kept. */
uint8_t oracle_e4m3_encode(float v) {
  if (isnan(v)) return 0x7F;
  uint8_t sign = signbit(v) ? 0x80 : 0x00;
  double a = fabs((double)v);
  if (a >= 448.0) return sign | 0x7E;
  if (a < ldexp(1.0, -6)) {
    /* subnormal range: multiples of 2^-9; a result of 8 is 2^-6, the
     * smallest normal, whose code is also 8 (exponent field 1, mantissa 0) */
    double q = nearbyint(a * 512.0);
    if (MUTANT(3) && q < 8.0) q = 0.0;
    return sign | (uint8_t)q;
  }
  int e;
  double fr = frexp(a, &e); /* a = (2 fr) * 2^(e-1), 2 fr in [1, 2) */
  e -= 1;
  double mant = MUTANT(2) ? round((2.0 * fr - 1.0) * 8.0) : nearbyint((2.0 * fr - 1.0) * 8.0);
  if (mant == 8.0) {
    mant = 0.0;
    e += 1;
  }
  int field = e + 7;
  if (field > 15 || (field == 15 && mant > 6.0)) return sign | 0x7E;
  return sign | (uint8_t)((field << 3) | (int)mant);
}

/* f32 quotient -> int8 code: round half to even, clamp to [-127, 127]. */
int32_t oracle_int8_round(float t) {
  float r = MUTANT(4) ? truncf(t) : nearbyintf(t);
  if (r > 127.0f) r = 127.0f;
  if (r < -127.0f) r = -127.0f;
  return (int32_t)r;
}

/* E4M3 code -> exact integer in units of 2^-9 (every finite E4M3 value is an
 * integer multiple of 2^-9 of magnitude at most 448 * 2^9 = 229376). */
static int64_t e4m3_units_table[256];
static int e4m3_units_ready = 0;

static int64_t e4m3_units(uint8_t c) {
  if (!e4m3_units_ready) { /* filled once from the decoder above */
    for (int i = 0; i < 256; ++i) {
      double v = oracle_e4m3_decode((uint8_t)i);
      e4m3_units_table[i] = isnan(v) ? 0 : (int64_t)ldexp(v, 9);
    }
    e4m3_units_ready = 1;
  }
  return e4m3_units_table[c];
}

/* ------------------------------------------------------------------------ */
/* Quantizers                                                               */
/* ------------------------------------------------------------------------ */

static uint8_t quantize_one(int scheme, float x, float s) {
  float t = (s > 0.0f) ? (MUTANT(16) ? x * (1.0f / s) : x / s) : 0.0f;
  if (scheme == ORACLE_INT8_ROW) return (uint8_t)(int8_t)oracle_int8_round(t);
  return oracle_e4m3_encode(t);
}

/* Weight quantization (offline, checkpoint side).
 *  int8 row  [W8A8]: s_w[n] = bf16(max_k |w[n,k]| / 127), q = clamp(rne(w / s_w))
 *  fp8 row   [FP8R]: s_w[n] = max_k |w[n,k]| / 448,      q = e4m3(w / s_w)
 *  fp8 block [FP8B]: s_w[nb,kb] = max over the 128x128 block / 448, q = e4m3(w / s_w)
 * w: bf16 [N,K] row-major; wq: [N,K] bytes; sw: [N] or [N/128, K/128].
 * Returns 0, or -1 on a shape the scheme does not allow. */
int oracle_quantize_weight(int scheme, const uint16_t* w, int64_t N, int64_t K, uint8_t* wq,
                           float* sw) {
  if (N <= 0 || K <= 0) return -1;
  if (scheme == ORACLE_FP8_BLOCK) {
    if (N % 128 || K % 128) return -1;
    int64_t KB = K / 128;
    for (int64_t nb = 0; nb < N / 128; ++nb)
      for (int64_t kb = 0; kb < KB; ++kb) {
        float a = 0.0f;
        for (int64_t n = nb * 128; n < nb * 128 + 128; ++n)
          for (int64_t k = kb * 128; k < kb * 128 + 128; ++k)
            a = fmaxf(a, fabsf(oracle_bf16_to_f32(w[n * K + k])));
        if (MUTANT(11)) a = fabsf(oracle_bf16_to_f32(w[nb * 128 * K + kb * 128]));
        float s = MUTANT(18) ? a * (1.0f / 448.0f) : a / 448.0f;
        sw[nb * KB + kb] = s;
        for (int64_t n = nb * 128; n < nb * 128 + 128; ++n)
          for (int64_t k = kb * 128; k < kb * 128 + 128; ++k)
            wq[n * K + k] = quantize_one(scheme, oracle_bf16_to_f32(w[n * K + k]), s);
      }
    return 0;
  }
  if (scheme != ORACLE_INT8_ROW && scheme != ORACLE_FP8_ROW) return -1;
  for (int64_t n = 0; n < N; ++n) {
    float a = 0.0f;
    for (int64_t k = 0; k < K; ++k) a = fmaxf(a, fabsf(oracle_bf16_to_f32(w[n * K + k])));
    float s;
    if (scheme == ORACLE_INT8_ROW)
      s = MUTANT(5) ? a / 127.0f : oracle_bf16_to_f32(oracle_f32_to_bf16(a / 127.0f));
    else
      s = MUTANT(18) ? a * (1.0f / 448.0f) : a / 448.0f;
    sw[n] = s;
    for (int64_t k = 0; k < K; ++k)
      wq[n * K + k] = quantize_one(scheme, oracle_bf16_to_f32(w[n * K + k]), s);
  }
  return 0;
}

/* Activation quantization (dynamic, per call).
 *  int8 row  [W8A8]: per token m: s = max_k |x| / 127, q = clamp(rne(x / s))
 *  fp8 row   [FP8R]: per token m: s = max_k |x| / 448, q = e4m3(x / s)
 *  fp8 block [FP8B]: per token m and 128-input group g: s = max_{k in g} |x| / 448
 * x: bf16 [M,K]; qx: [M,K] bytes; sx: [M] or [M, K/128]. */
int oracle_quantize_act(int scheme, const uint16_t* x, int64_t M, int64_t K, uint8_t* qx,
                        float* sx) {
  if (M < 0 || K <= 0) return -1;
  if (scheme == ORACLE_FP8_BLOCK && K % 128) return -1;
  if (scheme < 0 || scheme > 2) return -1;
  int64_t G = (scheme == ORACLE_FP8_BLOCK) ? K / 128 : 1;
  int64_t width = K / G;
  float qmax = (scheme == ORACLE_INT8_ROW) ? (MUTANT(6) ? 128.0f : 127.0f) : 448.0f;
  for (int64_t m = 0; m < M; ++m)
    for (int64_t g = 0; g < G; ++g) {
      const uint16_t* xs = x + m * K + g * width;
      float a = 0.0f;
      for (int64_t k = 0; k < width; ++k) a = fmaxf(a, fabsf(oracle_bf16_to_f32(xs[k])));
      if (MUTANT(7)) /* per-token absmax where a per-group one is due */
        for (int64_t k = 0; k < K; ++k) a = fmaxf(a, fabsf(oracle_bf16_to_f32(x[m * K + k])));
      float s = MUTANT(17) ? a * (1.0f / qmax) : a / qmax;
      sx[m * G + g] = s;
      for (int64_t k = 0; k < width; ++k)
        qx[m * K + g * width + k] = quantize_one(scheme, oracle_bf16_to_f32(xs[k]), s);
    }
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Products                                                                 */
/* ------------------------------------------------------------------------ */

/* Exact int8 dot product summed in int32 [W8A8 "Loading"].  |acc| <= K * 127^2,
 * which fits in int32 for K <= 133144 (checked by the caller). */
static int32_t dot_i8(const uint8_t* a, const uint8_t* b, int64_t K) {
  int32_t acc = 0;
  for (int64_t k = 0; k < K; ++k)
    acc += MUTANT(8) ? (int32_t)a[k] * (int32_t)(int8_t)b[k]
                     : (int32_t)(int8_t)a[k] * (int32_t)(int8_t)b[k];
  return acc;
}

/* Exact E4M3 dot product in units of 2^-18 (each product is an integer
 * multiple of 2^-18 below 2^36; a sum of fewer than 2^17 of them stays below
 * 2^53, so it is also exact once converted to f64). */
static int64_t dot_e4m3_units(const uint8_t* a, const uint8_t* b, int64_t K) {
  int64_t acc = 0;
  for (int64_t k = 0; k < K; ++k) acc += e4m3_units(a[k]) * e4m3_units(b[k]);
  return acc;
}

/* One output element y[m,n] (bf16 bits).  acc_i32 receives the int32
 * accumulator (int8 scheme), acc_f64 the exact pre-scale accumulator (row
 * schemes) or the exact f64 value before the final rounding (block scheme). */
static uint16_t linear_one(int scheme, const uint8_t* qx, const float* sx, const uint8_t* wq,
                           const float* sw, int64_t N, int64_t K, int64_t m, int64_t n,
                           int32_t* acc_i32, double* acc_f64) {
  const uint8_t* a = qx + m * K;
  const uint8_t* b = wq + n * K;
  if (scheme == ORACLE_INT8_ROW) {
    int32_t acc = dot_i8(a, b, K);
    if (acc_i32) *acc_i32 = acc;
    if (acc_f64) *acc_f64 = (double)acc;
    float y = ((float)acc * sx[m]) * (MUTANT(9) ? 1.0f : sw[n]);
    return oracle_f32_to_bf16(y);
  }
  if (scheme == ORACLE_FP8_ROW) {
    double acc = ldexp((double)dot_e4m3_units(a, b, MUTANT(12) ? K - 1 : K), -18); /* exact */
    if (acc_f64) *acc_f64 = acc;
    float y = ((float)acc * sx[m]) * sw[n];
    return oracle_f32_to_bf16(y);
  }
  /* block scheme: partial sum per 128-wide K block, scaled, summed in f64 */
  int64_t KB = K / 128;
  double y = 0.0;
  for (int64_t kb = 0; kb < KB; ++kb) {
    double p = ldexp((double)dot_e4m3_units(a + kb * 128, b + kb * 128, 128), -18);
    int64_t wi = MUTANT(10) ? kb * (N / 128) + (n / 128) : (n / 128) * KB + kb;
    y += p * (double)sx[m * KB + kb] * (double)sw[wi];
  }
  if (acc_f64) *acc_f64 = y;
  return oracle_f64_to_bf16(y);
}

static int check_linear_shape(int scheme, int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N <= 0 || K <= 0) return -1;
  if (scheme < 0 || scheme > 2) return -1;
  if (scheme == ORACLE_FP8_BLOCK && (N % 128 || K % 128)) return -1;
  if (scheme == ORACLE_INT8_ROW && K > 133144) return -1; /* int32 range */
  if (scheme != ORACLE_INT8_ROW && K >= 131072) return -1; /* int64 / f64 exactness */
  return 0;
}

/* Full product: y[M,N] bf16 bits from quantized operands.  acc_i32 [M,N]
 * (int8 scheme) and acc_f64 [M,N] may be NULL. */
int oracle_linear(int scheme, const uint8_t* qx, const float* sx, const uint8_t* wq,
                  const float* sw, int64_t M, int64_t N, int64_t K, uint16_t* y,
                  int32_t* acc_i32, double* acc_f64) {
  if (check_linear_shape(scheme, M, N, K)) return -1;
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n)
      y[m * N + n] = linear_one(scheme, qx, sx, wq, sw, N, K, m, n,
                                acc_i32 ? acc_i32 + m * N + n : 0, acc_f64 ? acc_f64 + m * N + n : 0);
  return 0;
}

/* Sampled product: the P outputs (pm[i], pn[i]) only, for full-size shapes. */
int oracle_linear_sampled(int scheme, const uint8_t* qx, const float* sx, const uint8_t* wq,
                          const float* sw, int64_t M, int64_t N, int64_t K, const int64_t* pm,
                          const int64_t* pn, int64_t P, uint16_t* y, int32_t* acc_i32,
                          double* acc_f64) {
  if (check_linear_shape(scheme, M, N, K)) return -1;
  for (int64_t i = 0; i < P; ++i) {
    if (pm[i] < 0 || pm[i] >= M || pn[i] < 0 || pn[i] >= N) return -1;
    y[i] = linear_one(scheme, qx, sx, wq, sw, N, K, pm[i], pn[i], acc_i32 ? acc_i32 + i : 0,
                      acc_f64 ? acc_f64 + i : 0);
  }
  return 0;
}

/* Rows [n0, n1) of a full product, for splitting a large case across
 * processes: y, acc_i32 and acc_f64 are [M, n1-n0]. */
int oracle_linear_rows(int scheme, const uint8_t* qx, const float* sx, const uint8_t* wq,
                       const float* sw, int64_t M, int64_t N, int64_t K, int64_t n0, int64_t n1,
                       uint16_t* y, int32_t* acc_i32, double* acc_f64) {
  if (check_linear_shape(scheme, M, N, K) || n0 < 0 || n1 > N || n0 > n1) return -1;
  int64_t W = n1 - n0;
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = n0; n < n1; ++n) {
      int64_t o = m * W + (n - n0);
      y[o] = linear_one(scheme, qx, sx, wq, sw, N, K, m, n, acc_i32 ? acc_i32 + o : 0,
                        acc_f64 ? acc_f64 + o : 0);
    }
  return 0;
}

/* The whole method on bf16 inputs: quantize X (per call) and run the
 * product against already-quantized weights.  qx/sx are caller scratch of
 * the quantize_act sizes. */
int oracle_forward(int scheme, const uint16_t* x, const uint8_t* wq, const float* sw, int64_t M,
                   int64_t N, int64_t K, uint8_t* qx, float* sx, uint16_t* y) {
  if (oracle_quantize_act(scheme, x, M, K, qx, sx)) return -1;
  return oracle_linear(scheme, qx, sx, wq, sw, M, N, K, y, 0, 0);
}

/* ------------------------------------------------------------------------ */
/* Weight-only products ("equivalent" numerics)                             */
/* ------------------------------------------------------------------------ */

/* The pages' loader option numerics="equivalent" never rounds the input
 * ("Llama 3.1 8B Instruct W8A8", "Against bf16"; "Qwen3 8B FP8", "Against
 * bf16"), and the W8A8 model page's "Context" contrasts W8A8 with W8A16,
 * which quantizes only the weights and keeps computing in bf16.  So here X
 * stays bf16 and only W is quantized:
 *   y[m,n] = bf16( sum_k x[m,k] * (q_w[n,k] * s_w) ),
 * s_w = s_w[n] (row schemes) or s_w[n/128, k/128] (block scheme).
 * The dequantized weight needs at most 24 + 4 significant bits (int8 codes
 * have 7, E4M3 4, scales 24) and its product with a bf16 (8 bits) is exact in
 * f64; the sum over k is the one f64 rounding, then one rounding to bf16. */
static double weight_value(int scheme, const uint8_t* wq, const float* sw, int64_t N, int64_t K,
                           int64_t n, int64_t k) {
  uint8_t c = wq[n * K + k];
  double code = (scheme == ORACLE_INT8_ROW) ? (double)(int8_t)c : oracle_e4m3_decode(c);
  double s;
  if (scheme == ORACLE_FP8_BLOCK)
    s = MUTANT(14) ? (double)sw[(k / 128) * (N / 128) + n / 128] : (double)sw[(n / 128) * (K / 128) + k / 128];
  else
    s = (double)sw[n];
  return MUTANT(13) ? code : code * s;
}

static uint16_t linear_wo_one(int scheme, const uint16_t* x, const uint8_t* wq, const float* sw,
                              int64_t N, int64_t K, int64_t m, int64_t n, double* acc_f64) {
  double y = 0.0;
  for (int64_t k = MUTANT(15) ? 1 : 0; k < K; ++k)
    y += (double)oracle_bf16_to_f32(x[m * K + k]) * weight_value(scheme, wq, sw, N, K, n, k);
  if (acc_f64) *acc_f64 = y;
  return oracle_f64_to_bf16(y);
}

/* Output columns [n0, n1) of the weight-only product: x bf16 [M,K], wq [N,K],
 * sw as for the quantized product; y and acc_f64 (the f64 value before the
 * final rounding, may be NULL) are [M, n1-n0]. */
int oracle_linear_wo_rows(int scheme, const uint16_t* x, const uint8_t* wq, const float* sw,
                          int64_t M, int64_t N, int64_t K, int64_t n0, int64_t n1, uint16_t* y,
                          double* acc_f64) {
  if (M < 0 || N <= 0 || K <= 0 || scheme < 0 || scheme > 2) return -1;
  if (scheme == ORACLE_FP8_BLOCK && (N % 128 || K % 128)) return -1;
  if (n0 < 0 || n1 > N || n0 > n1) return -1;
  int64_t W = n1 - n0;
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = n0; n < n1; ++n) {
      int64_t o = m * W + (n - n0);
      y[o] = linear_wo_one(scheme, x, wq, sw, N, K, m, n, acc_f64 ? acc_f64 + o : 0);
    }
  return 0;
}

/* Bulk forms of the codecs, for sweeps over many values. */
void oracle_e4m3_encode_n(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(v[i]);
}
void oracle_f32_to_bf16_n(const float* v, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_bf16(v[i]);
}
void oracle_int8_round_n(const float* v, int64_t n, int32_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_int8_round(v[i]);
}
void oracle_f64_to_bf16_n(const double* v, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_f64_to_bf16(v[i]);
}

/* Sanity hook for the harness: 1 when the FPU rounds to nearest. */
int oracle_rounding_is_nearest(void) { return fegetround() == FE_TONEAREST; }
