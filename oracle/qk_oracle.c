/*
 * qk_oracle.c -- plain, slow, obviously-correct CPU oracle for the W8A8
 * INT8 quantized linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg do.  It shares no code, header, helper,
 * constant or table with the CUDA path: every formula below is written out
 * again from the pages' definitions.
 *
 * Sources (page title, section):
 *  - "write-int8-quantized-kernel" (agentmods skill), "Inputs the agent
 *    should gather first": per-token and per-output-channel granularity,
 *    symmetric range [-127, 127] with zero-point 0, mandatory INT32
 *    accumulation, FP32 output after dequantisation.
 *  - "KV-cache kernels" (day 26), section 02 "Scales and dequantization":
 *    int8 products accumulate in int32, output = acc * a_scale * b_scale;
 *    section 03: per-group scales every 64-128 channels.
 *  - vLLM PR "fused silu_and_mul + dynamic per-token FP8 quantization",
 *    Purpose / Algorithm: per-token scale = max(absmax, 1e-12) / qmax from the
 *    token's own absmax, quantisation with the per-token inverse scale,
 *    activation silu(gate) * up computed in fp32.
 *  - "16. Deploying Custom Kernels", C++ Kernel Interface: GemmConfig fields
 *    m, n, k, int8 a and b, int32 c, fp32 scale_a / scale_b, output_scale.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - qmax = 127 (INT8 symmetric); epsilon is the fp32 literal 1e-12f and is
 *    applied before the divide; scale = max(amax, 1e-12f) / 127 (fp32 RN).
 *  - quantisation multiplies by inv = 1 / scale (fp32 RN), rounds half to
 *    even and clamps to [-127, 127].
 *  - silu(g) = g / (1 + exp(-g)) in fp32 with a fixed exp (qko_exp below),
 *    h = silu(g) * u in fp32, quantised without rounding h to bf16.
 *  - per-channel epilogue: o = (((float)acc * sa[m]) * sw[n]) * alpha,
 *    left to right, every step fp32 RN, no FMA contraction.
 *  - per-group epilogue (group 128 along K): f = 0; for g ascending:
 *    f = fmaf((float)P_g, sw[n][g], f); o = (f * sa[m]) * alpha.
 *  - bf16 output = round-to-nearest-even of o.
 *
 * FP8 variant (same vLLM PR, Purpose / Algorithm: the pages' own kernel
 * quantises to float8_e4m3fn, scale = max(absmax, 1e-12) / fp8_max,
 * "optionally clamped by scale_ub"; "The Quantization Ladder" page (day 11)
 * on e4m3 spending its bits on mantissa):
 *  - e4m3 is the OCP E4M3FN format: 1 sign, 4 exponent bits (bias 7), 3
 *    mantissa bits, no infinities, S.1111.111 NaN; largest finite 448,
 *    smallest normal 2^-6, smallest subnormal 2^-9.
 *  - scale = max(amax, 1e-12f) / 448 (fp32 RN); with an upper bound ub the
 *    written scale is min(that, ub) (the scale itself is clamped, as the
 *    page's sentence reads); inv = 1 / scale (fp32 RN).
 *  - q = e4m3(clamp(x * inv, -448, 448)), converted round-to-nearest-even.
 *  - the FP8 GEMM's accumulator is the exact dot product of the decoded
 *    values (every e4m3 value is an integer multiple of 2^-9, so products
 *    are integer multiples of 2^-18 and the sum is exact in int64), rounded
 *    once to fp32; the epilogue is the per-channel one above.
 *
 * Asymmetric per-token INT8 ("write-int8-quantized-kernel", Inputs the agent
 * should gather first: asymmetric quantisation maps [-128, 127] to an
 * arbitrary range with a non-zero zero-point):
 *  - the row's range [lo, hi] is widened to hold 0 (so the zero-point is
 *    representable); scale = max(hi - lo, 1e-12f) / 255, inv = 1 / scale;
 *  - zp = clamp(rne(-128 - lo * inv), -128, 127);
 *    q = clamp(rne(x * inv) + zp, -128, 127), x ~ (q - zp) * scale;
 *  - the GEMM's accumulator is sum_k (q - zp) * w = acc - zp * wsum[n],
 *    wsum[n] = sum_k w[n][k]; the epilogue is the per-channel one.
 *
 * Static per-tensor INT8 (same page: per-tensor granularity, scales computed
 * offline): inv = 1 / scale, q = clamp(rne(x * inv), -127, 127).
 *
 * Build: gcc -O2 -ffp-contract=off -fPIC -shared -pthread (no fast-math),
 * so every float operation below is a single IEEE binary32 RN operation.
 *
 * Parity pins: every function here is pinned by tests that do not call back
 * into this file's arithmetic (closed forms, brute force with numpy int64,
 * exact tie cases, error bounds against float64 math, torch's bf16 cast).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define QKO_OK 0
#define QKO_ERR_ARG 1
#define QKO_ERR_OVERFLOW 4

#define QKO_F32 0
#define QKO_BF16 1

/* ----------------------------------------------------------------------- */
/* bf16 <-> fp32                                                           */
/* ----------------------------------------------------------------------- */

/* bf16 is the top half of a binary32: widening is a 16-bit shift (exact). */
static float qko_bf16_bits_to_f32(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* Round a binary32 to bf16, nearest-even on the 16 dropped bits.  NaN is
 * returned as the canonical quiet NaN (never produced by the method). */
uint16_t qko_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0u)
    return (uint16_t)0x7fc0u;
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

void qko_f32_to_bf16_array(const float* in, uint16_t* out, int64_t count) {
  for (int64_t i = 0; i < count; ++i) out[i] = qko_f32_to_bf16(in[i]);
}

static float qko_load(const void* base, int dtype, int64_t idx) {
  if (dtype == QKO_BF16) return qko_bf16_bits_to_f32(((const uint16_t*)base)[idx]);
  return ((const float*)base)[idx];
}

/* ----------------------------------------------------------------------- */
/* exp and SiLU                                                            */
/* ----------------------------------------------------------------------- */

/*
 * qko_exp -- fixed binary32 exponential, so that the fused SiLU is one
 * well-defined function on every machine.  Method: Cody & Waite argument
 * reduction t = n*ln2 + r with n = rint(t*log2 e) and ln2 split into a
 * binary32 head and tail; e^r by its Taylor series to degree 7 (|r| <= ln2/2
 * gives a truncation error below 6e-9 relative); e^t = e^r * 2^n with 2^n
 * assembled from exponent bits.  t is clamped to [-87, 88] so that 2^n and
 * the result stay normal and finite.
 */
float qko_exp(float t) {
  const float log2e = (float)1.4426950408889634074;
  const float ln2_hi = (float)0.69314718055994530942;
  const float ln2_lo = (float)(0.69314718055994530942 - (double)(float)0.69314718055994530942);
  if (t < -87.0f) t = -87.0f;
  if (t > 88.0f) t = 88.0f;
  float n = rintf(t * log2e);
  float r = fmaf(-n, ln2_hi, t);
  r = fmaf(-n, ln2_lo, r);
  /* Taylor coefficients 1/j!, j = 7 .. 0, each rounded once to binary32. */
  float p = (float)(1.0 / 5040.0);
  p = fmaf(p, r, (float)(1.0 / 720.0));
  p = fmaf(p, r, (float)(1.0 / 120.0));
  p = fmaf(p, r, (float)(1.0 / 24.0));
  p = fmaf(p, r, (float)(1.0 / 6.0));
  p = fmaf(p, r, 0.5f);
  p = fmaf(p, r, 1.0f);
  p = fmaf(p, r, 1.0f);
  int32_t e = (int32_t)n + 127; /* in [1, 254] after the clamp */
  uint32_t bits = ((uint32_t)e) << 23;
  float two_n;
  memcpy(&two_n, &bits, sizeof two_n);
  return p * two_n;
}

/* silu(g) = g * sigmoid(g) = g / (1 + exp(-g)), binary32 RN throughout. */
float qko_silu(float g) {
  float e = qko_exp(-g);
  float d = 1.0f + e;
  return g / d;
}

/* ----------------------------------------------------------------------- */
/* Dynamic per-token symmetric quantisation                                */
/* ----------------------------------------------------------------------- */

/* One row: amax = max|x| (exact), scale = max(amax, 1e-12f) / 127,
 * inv = 1 / scale, q = clamp(round_half_even(x * inv), -127, 127). */
void qko_quantize_row(const float* x, int k, int8_t* q, float* scale) {
  float amax = 0.0f;
  for (int i = 0; i < k; ++i) {
    float a = fabsf(x[i]);
    if (a > amax) amax = a;
  }
  float s = fmaxf(amax, 1e-12f) / 127.0f;
  float inv = 1.0f / s;
  for (int i = 0; i < k; ++i) {
    float y = x[i] * inv;
    float r = nearbyintf(y); /* default rounding mode: nearest, ties to even */
    if (r > 127.0f) r = 127.0f;
    if (r < -127.0f) r = -127.0f;
    q[i] = (int8_t)(int)r;
  }
  *scale = s;
}

/* x: [m, k] row-major, fp32 or bf16 bits.  q: [m, k] int8.  scale: [m]. */
int qko_quantize_per_token(int m, int k, const void* x, int dtype, int8_t* q, float* scale) {
  if (m < 0 || k <= 0 || (dtype != QKO_F32 && dtype != QKO_BF16)) return QKO_ERR_ARG;
  float* row = (float*)malloc(sizeof(float) * (size_t)k);
  if (!row) return QKO_ERR_ARG;
  for (int r = 0; r < m; ++r) {
    for (int i = 0; i < k; ++i) row[i] = qko_load(x, dtype, (int64_t)r * k + i);
    qko_quantize_row(row, k, q + (int64_t)r * k, scale + r);
  }
  free(row);
  return QKO_OK;
}

/* h[r, i] = silu(gate[r, i]) * up[r, i] (fp32, not rounded to bf16), then the
 * per-token quantisation of h.  gate and up rows are ld elements apart, so a
 * concatenated [T, 2d] buffer (gate = base, up = base + d, ld = 2d) and two
 * separate [T, d] tensors (ld = d) are both accepted. */
int qko_silu_mul_quant_per_token(int m, int k, const void* gate, const void* up, int64_t ld,
                                 int dtype, int8_t* q, float* scale) {
  if (m < 0 || k <= 0 || ld < k || (dtype != QKO_F32 && dtype != QKO_BF16)) return QKO_ERR_ARG;
  float* h = (float*)malloc(sizeof(float) * (size_t)k);
  if (!h) return QKO_ERR_ARG;
  for (int r = 0; r < m; ++r) {
    for (int i = 0; i < k; ++i) {
      float g = qko_load(gate, dtype, (int64_t)r * ld + i);
      float u = qko_load(up, dtype, (int64_t)r * ld + i);
      h[i] = qko_silu(g) * u;
    }
    qko_quantize_row(h, k, q + (int64_t)r * k, scale + r);
  }
  free(h);
  return QKO_OK;
}

/* ----------------------------------------------------------------------- */
/* INT8 x INT8 -> INT32 GEMM and the dequantisation epilogues               */
/* ----------------------------------------------------------------------- */

/* acc[m][n] = sum_k a[m][k] * w[n][k], summed in int64 and checked against
 * the int32 range (a result outside it is an error, never a wrap). */
typedef struct {
  int m0, m1, n, k, group, mode;
  const int8_t* a;
  const int8_t* w;
  const float* sa;
  const float* sw;
  float alpha;
  int32_t* acc;
  float* out;
  int overflow;
} qko_job;

#define QKO_MODE_ACC 0
#define QKO_MODE_GROUP 1

static void* qko_rows_worker(void* p) {
  qko_job* j = (qko_job*)p;
  const int n = j->n, k = j->k;
  for (int r = j->m0; r < j->m1; ++r) {
    const int8_t* ar = j->a + (int64_t)r * k;
    for (int c = 0; c < n; ++c) {
      const int8_t* wr = j->w + (int64_t)c * k;
      if (j->mode == QKO_MODE_ACC) {
        int64_t s = 0;
        for (int i = 0; i < k; ++i) s += (int64_t)ar[i] * (int64_t)wr[i];
        if (s > INT32_MAX || s < INT32_MIN) j->overflow = 1;
        j->acc[(int64_t)r * n + c] = (int32_t)s;
      } else {
        /* per-group: an int32 partial per group of `group` K-columns, then
         * fp32 accumulation across groups in ascending group order. */
        const int ng = k / j->group;
        float f = 0.0f;
        int64_t total = 0;
        for (int g = 0; g < ng; ++g) {
          int64_t p = 0;
          for (int i = g * j->group; i < (g + 1) * j->group; ++i)
            p += (int64_t)ar[i] * (int64_t)wr[i];
          if (p > INT32_MAX || p < INT32_MIN) j->overflow = 1;
          total += p;
          f = fmaf((float)(int32_t)p, j->sw[(int64_t)c * ng + g], f);
        }
        if (total > INT32_MAX || total < INT32_MIN) j->overflow = 1;
        if (j->acc) j->acc[(int64_t)r * n + c] = (int32_t)total;
        float o = f * j->sa[r];
        o = o * j->alpha;
        j->out[(int64_t)r * n + c] = o;
      }
    }
  }
  return NULL;
}

static int qko_run_rows(qko_job* base, int m, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > m) nthreads = m > 0 ? m : 1;
  qko_job* jobs = (qko_job*)calloc((size_t)nthreads, sizeof(qko_job));
  pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
  if (!jobs || !th) {
    free(jobs);
    free(th);
    return QKO_ERR_ARG;
  }
  for (int t = 0; t < nthreads; ++t) {
    jobs[t] = *base;
    jobs[t].m0 = (int)((int64_t)m * t / nthreads);
    jobs[t].m1 = (int)((int64_t)m * (t + 1) / nthreads);
    jobs[t].overflow = 0;
  }
  for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], NULL, qko_rows_worker, &jobs[t]);
  qko_rows_worker(&jobs[0]);
  int overflow = jobs[0].overflow;
  for (int t = 1; t < nthreads; ++t) {
    pthread_join(th[t], NULL);
    overflow |= jobs[t].overflow;
  }
  free(jobs);
  free(th);
  return overflow ? QKO_ERR_OVERFLOW : QKO_OK;
}

/* a: [m, k] int8, w: [n, k] int8 (one output channel per row), acc: [m, n]. */
int qko_gemm_s32(int m, int n, int k, const int8_t* a, const int8_t* w, int32_t* acc, int nthreads) {
  if (m < 0 || n < 0 || k <= 0) return QKO_ERR_ARG;
  qko_job j;
  memset(&j, 0, sizeof j);
  j.n = n;
  j.k = k;
  j.mode = QKO_MODE_ACC;
  j.a = a;
  j.w = w;
  j.acc = acc;
  return qko_run_rows(&j, m, nthreads);
}

/* Per-token x per-channel dequantisation, written left to right:
 * o = (((float)acc * sa[m]) * sw[n]) * alpha. */
int qko_epilogue_per_channel(int m, int n, const int32_t* acc, const float* sa, const float* sw,
                             float alpha, float* out) {
  if (m < 0 || n < 0) return QKO_ERR_ARG;
  for (int r = 0; r < m; ++r) {
    for (int c = 0; c < n; ++c) {
      float o = (float)acc[(int64_t)r * n + c];
      o = o * sa[r];
      o = o * sw[c];
      o = o * alpha;
      out[(int64_t)r * n + c] = o;
    }
  }
  return QKO_OK;
}

/* Per-group (group along K) GEMM + epilogue.  sw: [n, k / group] row-major.
 * acc (nullable) receives the full-K int32 sum (= the sum of the partials). */
int qko_gemm_group(int m, int n, int k, int group, const int8_t* a, const int8_t* w,
                   const float* sa, const float* sw, float alpha, float* out, int32_t* acc,
                   int nthreads) {
  if (m < 0 || n < 0 || k <= 0 || group <= 0 || k % group != 0) return QKO_ERR_ARG;
  qko_job j;
  memset(&j, 0, sizeof j);
  j.n = n;
  j.k = k;
  j.group = group;
  j.mode = QKO_MODE_GROUP;
  j.a = a;
  j.w = w;
  j.sa = sa;
  j.sw = sw;
  j.alpha = alpha;
  j.acc = acc;
  j.out = out;
  return qko_run_rows(&j, m, nthreads);
}

/* ----------------------------------------------------------------------- */
/* FP8 e4m3 (E4M3FN) encode / decode                                       */
/* ----------------------------------------------------------------------- */

/* value of an e4m3 code: subnormal (exponent field 0) m * 2^-9, normal
 * (8 + m) * 2^(e - 10) = (1 + m / 8) * 2^(e - 7); S.1111.111 is NaN. */
float qko_e4m3_to_f32(uint8_t b) {
  const int e = (b >> 3) & 15, m = b & 7;
  if (e == 15 && m == 7) return NAN;
  const float v = e == 0 ? ldexpf((float)m, -9) : ldexpf((float)(8 + m), e - 10);
  return (b & 0x80) ? -v : v;
}

/* The code's value in units of 2^-9 (an integer for every finite code). */
static int64_t qko_e4m3_units(uint8_t b) {
  const int e = (b >> 3) & 15, m = b & 7;
  const int64_t u = e == 0 ? (int64_t)m : (int64_t)(8 + m) << (e - 1);
  return (b & 0x80) ? -u : u;
}

/* Nearest e4m3 value to a finite x, ties to the even code; |x| >= 448 gives
 * +-448 (the quantiser clamps to [-448, 448] before converting).  The
 * spacing in [2^E, 2^(E+1)) is 2^(E-3) for E >= -6, and 2^-9 below 2^-6;
 * dividing by a power of two is exact, so nearbyintf does the rounding. */
uint8_t qko_f32_to_e4m3(float x) {
  const uint8_t sign = signbit(x) ? 0x80 : 0x00;
  const float a = fabsf(x);
  if (a >= 448.0f) return sign | 0x7E;
  if (a == 0.0f) return sign;
  int ex;
  frexpf(a, &ex);  /* a = f * 2^ex, f in [0.5, 1) */
  int E = ex - 1;  /* a in [2^E, 2^(E+1)) */
  if (E < -6) E = -6;
  const float spacing = ldexpf(1.0f, E - 3);
  const float steps = nearbyintf(a / spacing); /* ties to even */
  const float v = steps * spacing;             /* exact */
  if (v == 0.0f) return sign;
  frexpf(v, &ex);
  const int E2 = ex - 1;
  if (E2 < -6) return sign | (uint8_t)(int)(v / ldexpf(1.0f, -9));
  const int m = (int)(v / ldexpf(1.0f, E2 - 3)) - 8; /* 0..7 */
  return sign | (uint8_t)(((E2 + 7) << 3) | m);
}

void qko_f32_to_e4m3_array(const float* in, uint8_t* out, int64_t count) {
  for (int64_t i = 0; i < count; ++i) out[i] = qko_f32_to_e4m3(in[i]);
}

/* ----------------------------------------------------------------------- */
/* Dynamic per-token FP8 quantisation                                      */
/* ----------------------------------------------------------------------- */

/* One row: amax = max|x|, scale = max(amax, 1e-12f) / 448, clamped above by
 * *ub when ub is given; inv = 1 / scale; q = e4m3(clamp(x * inv, +-448)). */
void qko_quantize_row_fp8(const float* x, int k, const float* ub, uint8_t* q, float* scale) {
  float amax = 0.0f;
  for (int i = 0; i < k; ++i) {
    float ax = fabsf(x[i]);
    if (ax > amax) amax = ax;
  }
  float s = fmaxf(amax, 1e-12f) / 448.0f;
  if (ub && s > *ub) s = *ub;
  float inv = 1.0f / s;
  for (int i = 0; i < k; ++i) {
    float y = x[i] * inv;
    if (y > 448.0f) y = 448.0f;
    if (y < -448.0f) y = -448.0f;
    q[i] = qko_f32_to_e4m3(y);
  }
  *scale = s;
}

int qko_quantize_per_token_fp8(int m, int k, const void* x, int dtype, const float* ub,
                               uint8_t* q, float* scale) {
  if (m < 0 || k <= 0 || (dtype != QKO_F32 && dtype != QKO_BF16)) return QKO_ERR_ARG;
  float* row = (float*)malloc(sizeof(float) * (size_t)k);
  if (!row) return QKO_ERR_ARG;
  for (int r = 0; r < m; ++r) {
    for (int i = 0; i < k; ++i) row[i] = qko_load(x, dtype, (int64_t)r * k + i);
    qko_quantize_row_fp8(row, k, ub, q + (int64_t)r * k, scale + r);
  }
  free(row);
  return QKO_OK;
}

/* silu(gate) * up (fp32, as qko_silu_mul_quant_per_token), then the FP8
 * per-token quantisation of the row. */
int qko_silu_mul_quant_per_token_fp8(int m, int k, const void* gate, const void* up, int64_t ld,
                                     int dtype, const float* ub, uint8_t* q, float* scale) {
  if (m < 0 || k <= 0 || ld < k || (dtype != QKO_F32 && dtype != QKO_BF16)) return QKO_ERR_ARG;
  float* h = (float*)malloc(sizeof(float) * (size_t)k);
  if (!h) return QKO_ERR_ARG;
  for (int r = 0; r < m; ++r) {
    for (int i = 0; i < k; ++i) {
      float gv = qko_load(gate, dtype, (int64_t)r * ld + i);
      float uv = qko_load(up, dtype, (int64_t)r * ld + i);
      h[i] = qko_silu(gv) * uv;
    }
    qko_quantize_row_fp8(h, k, ub, q + (int64_t)r * k, scale + r);
  }
  free(h);
  return QKO_OK;
}

/* ----------------------------------------------------------------------- */
/* FP8 x FP8 GEMM (exact accumulator) and its per-channel epilogue          */
/* ----------------------------------------------------------------------- */

typedef struct {
  int m0, m1, n, k;
  const uint8_t* a;
  const uint8_t* w;
  const float* sa;
  const float* sw;
  float alpha;
  double* acc;
  float* out;
} qko_fp8_job;

static void* qko_fp8_worker(void* p) {
  qko_fp8_job* j = (qko_fp8_job*)p;
  for (int r = j->m0; r < j->m1; ++r) {
    const uint8_t* ar = j->a + (int64_t)r * j->k;
    for (int c = 0; c < j->n; ++c) {
      const uint8_t* wr = j->w + (int64_t)c * j->k;
      int64_t s = 0; /* units of 2^-18 */
      for (int i = 0; i < j->k; ++i) s += qko_e4m3_units(ar[i]) * qko_e4m3_units(wr[i]);
      const double exact = ldexp((double)s, -18);
      if (j->acc) j->acc[(int64_t)r * j->n + c] = exact;
      if (j->out) {
        float o = (float)exact; /* the exact sum rounded once to fp32 */
        o = o * j->sa[r];
        o = o * j->sw[c];
        o = o * j->alpha;
        j->out[(int64_t)r * j->n + c] = o;
      }
    }
  }
  return NULL;
}

/* a: [m, k] e4m3 codes, w: [n, k] e4m3 codes.  acc (nullable): the exact dot
 * products as double (exact while |sum| < 2^35, i.e. k * 448^2 < 2^35 --
 * always so below k = 171,000); out (nullable): the fp32 epilogue. */
int qko_gemm_fp8(int m, int n, int k, const uint8_t* a, const uint8_t* w, const float* sa,
                 const float* sw, float alpha, double* acc, float* out, int nthreads) {
  if (m < 0 || n < 0 || k <= 0 || k > 171000) return QKO_ERR_ARG;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > m) nthreads = m > 0 ? m : 1;
  qko_fp8_job* jobs = (qko_fp8_job*)calloc((size_t)nthreads, sizeof(qko_fp8_job));
  pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
  if (!jobs || !th) {
    free(jobs);
    free(th);
    return QKO_ERR_ARG;
  }
  for (int t = 0; t < nthreads; ++t) {
    jobs[t].m0 = (int)((int64_t)m * t / nthreads);
    jobs[t].m1 = (int)((int64_t)m * (t + 1) / nthreads);
    jobs[t].n = n;
    jobs[t].k = k;
    jobs[t].a = a;
    jobs[t].w = w;
    jobs[t].sa = sa;
    jobs[t].sw = sw;
    jobs[t].alpha = alpha;
    jobs[t].acc = acc;
    jobs[t].out = out;
  }
  for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], NULL, qko_fp8_worker, &jobs[t]);
  qko_fp8_worker(&jobs[0]);
  for (int t = 1; t < nthreads; ++t) pthread_join(th[t], NULL);
  free(jobs);
  free(th);
  return QKO_OK;
}

/* ----------------------------------------------------------------------- */
/* Asymmetric per-token INT8 ("write-int8-quantized-kernel", Inputs:        */
/* asymmetric maps [-128, 127] to an arbitrary range with a non-zero        */
/* zero-point, which adds arithmetic to the hot loop).                      */
/* ----------------------------------------------------------------------- */

/* One row: lo = min(min x, 0), hi = max(max x, 0) (the range holds zero, so
 * the zero-point lies in [-128, 127]); scale = max(hi - lo, 1e-12f) / 255;
 * inv = 1 / scale; zp = clamp(round_half_even(-128 - lo * inv), -128, 127);
 * q = clamp(round_half_even(x * inv) + zp, -128, 127); x ~ (q - zp) * scale. */
void qko_quantize_row_asym(const float* x, int k, int8_t* q, float* scale, int32_t* zp) {
  float lo = 0.0f, hi = 0.0f;
  for (int i = 0; i < k; ++i) {
    if (x[i] < lo) lo = x[i];
    if (x[i] > hi) hi = x[i];
  }
  const float s = fmaxf(hi - lo, 1e-12f) / 255.0f;
  const float inv = 1.0f / s;
  float z = nearbyintf(-128.0f - lo * inv);
  if (z < -128.0f) z = -128.0f;
  if (z > 127.0f) z = 127.0f;
  for (int i = 0; i < k; ++i) {
    float r = nearbyintf(x[i] * inv) + z;
    if (r > 127.0f) r = 127.0f;
    if (r < -128.0f) r = -128.0f;
    q[i] = (int8_t)(int)r;
  }
  *scale = s;
  *zp = (int32_t)z;
}

int qko_quantize_per_token_asym(int m, int k, const void* x, int dtype, int8_t* q, float* scale,
                                int32_t* zp) {
  if (m < 0 || k <= 0 || (dtype != QKO_F32 && dtype != QKO_BF16)) return QKO_ERR_ARG;
  float* row = (float*)malloc(sizeof(float) * (size_t)k);
  if (!row) return QKO_ERR_ARG;
  for (int r = 0; r < m; ++r) {
    for (int i = 0; i < k; ++i) row[i] = qko_load(x, dtype, (int64_t)r * k + i);
    qko_quantize_row_asym(row, k, q + (int64_t)r * k, scale + r, zp + r);
  }
  free(row);
  return QKO_OK;
}

/* wsum[n] = sum_k w[n][k] (int64, checked against the int32 range). */
int qko_weight_row_sums(int n, int k, const int8_t* w, int32_t* wsum) {
  if (n < 0 || k <= 0) return QKO_ERR_ARG;
  for (int c = 0; c < n; ++c) {
    int64_t t = 0;
    for (int i = 0; i < k; ++i) t += w[(int64_t)c * k + i];
    if (t > INT32_MAX || t < INT32_MIN) return QKO_ERR_OVERFLOW;
    wsum[c] = (int32_t)t;
  }
  return QKO_OK;
}

/* acc[m][n] = sum_k (a[m][k] - zp[m]) * w[n][k], in int64, checked against
 * the int32 range; it equals the plain sum minus zp[m] * wsum[n]. */
int qko_gemm_s32_asym(int m, int n, int k, const int8_t* a, const int32_t* zp, const int8_t* w,
                      int32_t* acc) {
  if (m < 0 || n < 0 || k <= 0) return QKO_ERR_ARG;
  int overflow = 0;
  for (int r = 0; r < m; ++r) {
    for (int c = 0; c < n; ++c) {
      int64_t s = 0;
      for (int i = 0; i < k; ++i)
        s += ((int64_t)a[(int64_t)r * k + i] - zp[r]) * (int64_t)w[(int64_t)c * k + i];
      if (s > INT32_MAX || s < INT32_MIN) overflow = 1;
      acc[(int64_t)r * n + c] = (int32_t)s;
    }
  }
  return overflow ? QKO_ERR_OVERFLOW : QKO_OK;
}

/* ----------------------------------------------------------------------- */
/* Static per-tensor INT8 ("write-int8-quantized-kernel", Inputs: per-     */
/* tensor granularity, one scale for the entire tensor, computed offline).  */
/* ----------------------------------------------------------------------- */

/* inv = 1 / scale (fp32 RN); q = clamp(round_half_even(x * inv), -127, 127);
 * values beyond 127 * scale saturate. */
int qko_quantize_static(int m, int k, const void* x, int dtype, float scale, int8_t* q) {
  if (m < 0 || k <= 0 || (dtype != QKO_F32 && dtype != QKO_BF16) || !(scale > 0.0f))
    return QKO_ERR_ARG;
  const float inv = 1.0f / scale;
  for (int64_t i = 0; i < (int64_t)m * k; ++i) {
    float r = nearbyintf(qko_load(x, dtype, i) * inv);
    if (r > 127.0f) r = 127.0f;
    if (r < -127.0f) r = -127.0f;
    q[i] = (int8_t)(int)r;
  }
  return QKO_OK;
}
