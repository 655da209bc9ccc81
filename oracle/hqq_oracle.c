/*
 * hqq_oracle.c - plain, slow, scalar CPU oracle of the calibration-free HQQ weight
 * quantize / dequantize path.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's CPU
 * baseline may load or run this code. The product path (the CUDA library and its Python
 * binding) never calls it, and it shares no code, header, table or helper with that path.
 *
 * Precision: fp32 arithmetic, round to nearest even, no FMA contraction (build with
 * -ffp-contract=off, never -ffast-math), fp64 only for the three sums named below.
 *
 * Sources, by page title and section. The pages give no equation for the solver, so each
 * step below is the plainest reading of the passage cited next to it:
 *   [guide 2.1]  "HQQ calibration-free guide" (lnwmold.com) §2.1: no calibration data;
 *                the non-convex problem is split into two sub-problems solved in turn
 *                through an auxiliary variable with a quadratic penalty.
 *   [guide 2.2]  same page §2.2: nbits 8/4/3/2/1; group_size weights share one
 *                scale/zero; axis picks the grouping direction.
 *   [guide 3.2]  same page §3.2: dequantize() and unpack(dtype=uint8).
 *   [tutorial 2] "HQQ tutorial" (devpress.csdn.net) §2: the loss is lenient on small
 *                errors, strict on large ones, protects outliers; auxiliary variable +
 *                alternating optimisation.
 *   [tutorial 3.3] same page §3.3: per-group scale and zero point; quant_zero /
 *                quant_scale store them with a higher precision such as 8 bits.
 *   [analysis]   "Dropbox HQQ analysis" (ainews.cool), technical deep dive: reconstruction
 *                error of W against scale * quantized levels; auxiliary variable and
 *                alternating minimisation between it and the quantization parameters.
 *   [skill]      "hqq-quantization skill summary" (nav.superapi.store), usage: outputs
 *                W_q, scale, zero; dequantize().
 *
 * Readings taken where the pages are silent (all listed in the design notes):
 *   R1 iters = number of zero updates; iters+1 candidate zeros are evaluated (the RTN
 *      zero first), each scored by the error of its own codes.
 *   R2 the error is the lp "norm" sum_j |r_j|^p with the same p as the shrinkage.
 *   R3 a constant group (max == min) takes s = step = 1.
 *   R4 rint() is round half to even.
 *   R5 strict <: the earliest candidate wins a tie.
 *   R6 sum(Ws) and sum(We) are accumulated in fp64, sum(Q) in fp32 (exact integers), and
 *      z is rounded to fp32 once.
 *   R7 shrinkage: sign(r)*max(|r| - |r|^(p-1)/beta, 0) (one step of the generalised
 *      soft-threshold; the textbook soft-threshold at p = 1).
 *   R8 the stored scale is the step (dequantization multiplies by it).
 *   R10 second level: 8-bit min/max round-to-nearest, no solver, runs of `group` values.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#if defined(__FAST_MATH__)
#error "the oracle must not be built with -ffast-math"
#endif

#define ORACLE_MAX_GROUP 1024

/* a^(p-1) for a > 0, rounded once to fp32 (R7): the power is evaluated in fp64 and then
 * rounded to fp32, which gives the correctly rounded fp32 value except for inputs within a
 * few fp64 ulps of an fp32 rounding boundary (a libm powf may be an ulp off the correctly
 * rounded value, and differently so on each platform). */
static float pow_pm1(float a, float p) {
  return (float)pow((double)a, (double)(p - 1.0f));
}

/* lp generalised soft-threshold of one residual value (R7, after [guide 2.1] and
 * [tutorial 2]). t = |r|^(p-1) is passed in so that the caller can reuse it for the
 * error term; t = +inf for r == 0. */
static float shrink_lp(float r, float t, float inv_beta) {
  float a = fabsf(r);
  float m = a - t * inv_beta;
  m = fmaxf(m, 0.0f);
  return copysignf(m, r);
}

/* Exposed for the pins: a^(p-1) as the solver rounds it. */
float hqq_oracle_pow_pm1(float a, float p) { return pow_pm1(a, p); }

/* Exposed for the special-case pins (p = 1 is the textbook soft-threshold). */
float hqq_oracle_shrink(float r, float beta, float p) {
  float a = fabsf(r);
  float t = a > 0.0f ? pow_pm1(a, p) : INFINITY;
  float inv_beta = 1.0f / beta;
  return shrink_lp(r, t, inv_beta);
}

/*
 * The solver for one group of G weights w[0..G).
 *   Min/max RTN init ([tutorial 3.3]: one scale and one zero per group), then iters+1
 *   evaluations of candidate zeros with best-error tracking, each followed (except the
 *   last) by the auxiliary-variable step and the closed-form zero update
 *   ([guide 2.1], [analysis]).
 * Outputs: codes[G], *scale_out (= step, R8), *zero_out (= best zero, fp32).
 * Optional traces (may be NULL): z_trace[k], e_trace[k] for k = 0..iters.
 * Returns the best error.
 */
float hqq_oracle_quantize_group(const float* w, int G, int nbits, int iters, float p, float beta0,
                                float kappa, uint8_t* codes, float* scale_out, float* zero_out,
                                float* z_trace, float* e_trace) {
  const float qmax = (float)((1 << nbits) - 1);
  float Ws[ORACLE_MAX_GROUP];
  float Q[ORACLE_MAX_GROUP];
  float r[ORACLE_MAX_GROUP];
  float t[ORACLE_MAX_GROUP];

  /* 1. min/max round-to-nearest initialisation. */
  float mn = w[0], mx = w[0];
  for (int j = 1; j < G; ++j) {
    if (w[j] < mn) mn = w[j];
    if (w[j] > mx) mx = w[j];
  }
  float s, step;
  if (mx > mn) {
    float range = mx - mn;
    s = qmax / range;    /* codes per unit of weight */
    step = range / qmax; /* weight per code: the stored scale (R8) */
  } else {
    s = 1.0f; /* R3 */
    step = 1.0f;
  }
  float z = -mn * s; /* RTN zero: maps mn to code 0 (not rounded) */

  double acc = 0.0;
  for (int j = 0; j < G; ++j) {
    Ws[j] = w[j] * s;
    acc += (double)Ws[j];
  }
  const float S_ws = (float)acc; /* R6 */

  float best_e = INFINITY;
  float z_best = z;
  float beta = beta0;

  /* 2./3. evaluations and updates. */
  for (int k = 0; k <= iters; ++k) {
    float e = 0.0f;
    for (int j = 0; j < G; ++j) {
      float v = Ws[j] + z;
      float q = rintf(v); /* R4 */
      q = fmaxf(q, 0.0f);
      q = fminf(q, qmax);
      Q[j] = q;
      float back = q - z;        /* code offset from the zero */
      float wr = back * step;    /* dequantized weight */
      r[j] = w[j] - wr;          /* residual */
      float a = fabsf(r[j]);
      t[j] = a > 0.0f ? pow_pm1(a, p) : INFINITY;
      if (a > 0.0f) e += a * t[j]; /* |r|^p (R2) */
    }
    if (z_trace) z_trace[k] = z;
    if (e_trace) e_trace[k] = e;
    if (e < best_e) { /* R5 */
      best_e = e;
      z_best = z;
    }
    if (k == iters) break;

    float inv_beta = 1.0f / beta;
    float sumQ = 0.0f;
    double sumWe = 0.0;
    for (int j = 0; j < G; ++j) {
      float We = shrink_lp(r[j], t[j], inv_beta); /* auxiliary error variable (R7) */
      sumWe += (double)We;
      sumQ += Q[j];
    }
    /* closed-form zero: the mean over the group of Q - (w - We)*s, written with the
     * pre-scaled Ws = w*s (R6: one rounding to fp32). */
    double num = (double)sumQ - (double)S_ws + (double)s * sumWe;
    z = (float)(num / (double)G);
    beta = beta * kappa;
  }

  /* 4. final codes with the best zero. */
  for (int j = 0; j < G; ++j) {
    float q = rintf(Ws[j] + z_best);
    q = fmaxf(q, 0.0f);
    q = fminf(q, qmax);
    codes[j] = (uint8_t)q;
  }
  *scale_out = step;
  *zero_out = z_best;
  return best_e;
}

/* Step 4 alone for a given zero: the codes clamp(rint(w_j*s + zero), 0, qmax) of one
 * group with its min/max scale s (used to check a candidate zero chosen elsewhere). */
void hqq_oracle_codes_at_zero(const float* w, int G, int nbits, float zero, uint8_t* codes) {
  const float qmax = (float)((1 << nbits) - 1);
  float mn = w[0], mx = w[0];
  for (int j = 1; j < G; ++j) {
    if (w[j] < mn) mn = w[j];
    if (w[j] > mx) mx = w[j];
  }
  float s = 1.0f;
  if (mx > mn) s = qmax / (mx - mn);
  for (int j = 0; j < G; ++j) {
    float q = rintf(w[j] * s + zero);
    q = fmaxf(q, 0.0f);
    q = fminf(q, qmax);
    codes[j] = (uint8_t)q;
  }
}

/* Gather group g of a row-major [rows, cols] matrix ([guide 2.2] axis). */
static void gather_group(const float* W, int64_t rows, int64_t cols, int G, int axis, int64_t g,
                         float* w) {
  (void)rows;
  if (axis == 1) {
    int64_t per_row = cols / G;
    int64_t r = g / per_row, cb = g % per_row;
    const float* src = W + r * cols + cb * G;
    for (int j = 0; j < G; ++j) w[j] = src[j];
  } else {
    int64_t rb = g / cols, c = g % cols;
    for (int j = 0; j < G; ++j) w[j] = W[(rb * G + j) * cols + c];
  }
}

typedef struct {
  const float* W;
  int64_t rows, cols;
  int nbits, G, axis, iters;
  float p, beta0, kappa;
  uint8_t* codes;
  float *scale, *zero, *best_err;
  const int64_t* group_ids; /* NULL: all groups [g_begin, g_end) */
  int64_t g_begin, g_end;
} oracle_job;

static void* run_job(void* arg) {
  oracle_job* jb = (oracle_job*)arg;
  float w[ORACLE_MAX_GROUP];
  for (int64_t i = jb->g_begin; i < jb->g_end; ++i) {
    int64_t g = jb->group_ids ? jb->group_ids[i] : i;
    gather_group(jb->W, jb->rows, jb->cols, jb->G, jb->axis, g, w);
    float s, z;
    float e = hqq_oracle_quantize_group(w, jb->G, jb->nbits, jb->iters, jb->p, jb->beta0,
                                        jb->kappa, jb->codes + i * jb->G, &s, &z, NULL, NULL);
    jb->scale[i] = s;
    jb->zero[i] = z;
    if (jb->best_err) jb->best_err[i] = e;
  }
  return NULL;
}

/*
 * Quantize the groups `group_ids[0..n_sel)` (or, with group_ids == NULL, all
 * rows*cols/G groups in g order) of the fp32 matrix W, using `nthreads` POSIX threads
 * over groups. Outputs are indexed by position i in the selection: codes[i*G + j],
 * scale[i], zero[i], best_err[i] (best_err may be NULL).
 * Returns 0, or -1 on an argument error.
 */
int hqq_oracle_quantize(const float* W, int64_t rows, int64_t cols, int nbits, int G, int axis,
                        int iters, float p, float beta0, float kappa, const int64_t* group_ids,
                        int64_t n_sel, uint8_t* codes, float* scale, float* zero,
                        float* best_err, int nthreads) {
  if (G <= 0 || G > ORACLE_MAX_GROUP || nbits < 1 || nbits > 8) return -1;
  if (axis == 1 && cols % G) return -1;
  if (axis == 0 && rows % G) return -1;
  int64_t n = group_ids ? n_sel : rows * cols / G;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (n < nthreads) nthreads = n > 0 ? (int)n : 1;
  oracle_job jobs[256];
  pthread_t th[256];
  for (int i = 0; i < nthreads; ++i) {
    oracle_job* jb = &jobs[i];
    jb->W = W; jb->rows = rows; jb->cols = cols; jb->nbits = nbits; jb->G = G;
    jb->axis = axis; jb->iters = iters; jb->p = p; jb->beta0 = beta0; jb->kappa = kappa;
    jb->codes = codes; jb->scale = scale; jb->zero = zero; jb->best_err = best_err;
    jb->group_ids = group_ids;
    jb->g_begin = n * i / nthreads;
    jb->g_end = n * (i + 1) / nthreads;
  }
  if (nthreads == 1) {
    run_job(&jobs[0]);
    return 0;
  }
  for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, run_job, &jobs[i]);
  for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
  return 0;
}

/* Packed size in bytes of n codes (layout of the library header, restated here). */
int64_t hqq_oracle_packed_bytes(int64_t n, int nbits) {
  if (nbits == 3) return 4 * ((n + 9) / 10);
  return (n * nbits + 7) / 8;
}

/* Bit-pack n codes in stream order ([guide 3.2] unpack(dtype=uint8) is the inverse):
 * nbits 8/4/2/1 -> 8/nbits codes per byte, least significant first; nbits 3 -> 10 codes
 * per little-endian 32-bit word, 3 bits each from bit 0, bits 30..31 zero. */
void hqq_oracle_pack(const uint8_t* codes, int64_t n, int nbits, uint8_t* out) {
  int64_t nb = hqq_oracle_packed_bytes(n, nbits);
  memset(out, 0, (size_t)nb);
  if (nbits == 3) {
    for (int64_t k = 0; k < n; ++k) {
      int64_t word = k / 10;
      int bit = (int)(k % 10) * 3;
      uint32_t v = (uint32_t)(codes[k] & 7u) << bit;
      for (int b = 0; b < 4; ++b) out[word * 4 + b] |= (uint8_t)(v >> (8 * b));
    }
    return;
  }
  int per = 8 / nbits;
  for (int64_t k = 0; k < n; ++k) {
    int shift = (int)(k % per) * nbits;
    out[k / per] |= (uint8_t)((codes[k] & ((1u << nbits) - 1u)) << shift);
  }
}

void hqq_oracle_unpack(const uint8_t* packed, int64_t n, int nbits, uint8_t* codes) {
  if (nbits == 3) {
    for (int64_t k = 0; k < n; ++k) {
      int64_t word = k / 10;
      uint32_t v = (uint32_t)packed[word * 4] | ((uint32_t)packed[word * 4 + 1] << 8) |
                   ((uint32_t)packed[word * 4 + 2] << 16) | ((uint32_t)packed[word * 4 + 3] << 24);
      codes[k] = (uint8_t)((v >> ((k % 10) * 3)) & 7u);
    }
    return;
  }
  int per = 8 / nbits;
  for (int64_t k = 0; k < n; ++k)
    codes[k] = (uint8_t)((packed[k / per] >> ((k % per) * nbits)) & ((1u << nbits) - 1u));
}

/* Dequantize codes (g order, unpacked) into the fp32 row-major matrix out[rows, cols]:
 * out = (float(Q) - zero)*scale, two separate fp32 operations ([guide 3.2], [skill]). */
void hqq_oracle_dequantize(const uint8_t* codes, const float* scale, const float* zero,
                           int64_t rows, int64_t cols, int G, int axis, float* out) {
  int64_t n_groups = rows * cols / G;
  for (int64_t g = 0; g < n_groups; ++g) {
    for (int j = 0; j < G; ++j) {
      float q = (float)codes[g * G + j];
      float d = q - zero[g];
      float v = d * scale[g];
      int64_t idx;
      if (axis == 1) {
        idx = g * G + j;
      } else {
        int64_t rb = g / cols, c = g % cols;
        idx = (rb * G + j) * cols + c;
      }
      out[idx] = v;
    }
  }
}

/* Second level ([tutorial 3.3], R10): 8-bit min/max round-to-nearest of n values in runs
 * of `group`; mm[2*i] = step2, mm[2*i+1] = zero2 of run i. */
void hqq_oracle_quantize_meta(const float* m, int64_t n, int group, uint8_t* q, float* mm) {
  int64_t runs = (n + group - 1) / group;
  for (int64_t i = 0; i < runs; ++i) {
    int64_t b = i * group, e = b + group < n ? b + group : n;
    float mn = m[b], mx = m[b];
    for (int64_t k = b + 1; k < e; ++k) {
      if (m[k] < mn) mn = m[k];
      if (m[k] > mx) mx = m[k];
    }
    float s2, st2;
    if (mx > mn) {
      float range = mx - mn;
      s2 = 255.0f / range;
      st2 = range / 255.0f;
    } else {
      s2 = 1.0f;
      st2 = 1.0f;
    }
    float z2 = -mn * s2;
    for (int64_t k = b; k < e; ++k) {
      float v = m[k] * s2;
      v = v + z2;
      float c = rintf(v);
      c = fmaxf(c, 0.0f);
      c = fminf(c, 255.0f);
      q[k] = (uint8_t)c;
    }
    mm[2 * i] = st2;
    mm[2 * i + 1] = z2;
  }
}

void hqq_oracle_dequantize_meta(const uint8_t* q, const float* mm, int64_t n, int group,
                                float* out) {
  for (int64_t k = 0; k < n; ++k) {
    int64_t i = k / group;
    float d = (float)q[k] - mm[2 * i + 1];
    out[k] = d * mm[2 * i];
  }
}

/* ------------------------------------------------------------------ MXFP4 weight-only
 * [guide 5.1] "HQQ calibration-free guide" (lnwmold.com) §5.1 lists an mxfp4 weight-only
 * mode among the on-the-fly quantization modes; the pages give no further definition, so
 * the encoding is the plainest reading: the Open Compute Project Microscaling (MX) format
 * MXFP4 - blocks of 32 consecutive elements along a row share one E8M0 scale (a power of
 * two, stored as the biased exponent e + 127), and every element is an FP4 E2M1 number
 * (sign, 2 exponent bits, 1 mantissa bit: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6).
 * Conversion as that specification defines it:
 *   e  = floor(log2(max_i |V_i|)) - 2      (2 = exponent of E2M1's largest normal 6 = 1.5*2^2)
 *        clamped to the E8M0 range [-127, 127]; an all-zero block takes e = -127 (reading R14)
 *   P_i = V_i / 2^e rounded to the nearest E2M1 value, ties to the value with an even
 *        mantissa bit, magnitudes above 6 saturating to 6; the sign is kept (reading R15:
 *        -0 encodes as sign bit set, magnitude 0)
 *   dequantization: V'_i = P_i * 2^e.
 * Codes are packed two per byte, element 2j in the low nibble (as the 4-bit integer codes). */
static const float kE2M1[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

uint8_t hqq_oracle_e2m1_encode(float v) {
  const uint8_t sign = signbit(v) ? 8 : 0;
  const float a = fabsf(v);
  int best = 0;
  for (int m = 1; m < 8; ++m) {  /* nearest grid value; on a tie the even mantissa bit */
    const float db = fabsf(a - kE2M1[best]), dm = fabsf(a - kE2M1[m]);
    if (dm < db || (dm == db && (m & 1) == 0)) best = m;
  }
  if (a > 6.0f) best = 7; /* saturation (also covered by the search above) */
  return (uint8_t)(sign | best);
}

float hqq_oracle_e2m1_decode(uint8_t code) {
  const float m = kE2M1[code & 7];
  return (code & 8) ? -m : m;
}

int hqq_oracle_mx_exponent(const float* v, int n) {
  float amax = 0.0f;
  for (int i = 0; i < n; ++i) amax = fmaxf(amax, fabsf(v[i]));
  if (amax == 0.0f) return -127;
  int ex;
  (void)frexpf(amax, &ex); /* amax = f * 2^ex, f in [0.5, 1): floor(log2 amax) = ex - 1 */
  int e = (ex - 1) - 2;
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return e;
}

void hqq_oracle_mxfp4_quantize(const float* W, int64_t rows, int64_t cols, uint8_t* codes,
                               uint8_t* scales) {
  const int64_t nb = rows * cols / 32;
  for (int64_t b = 0; b < nb; ++b) {
    const float* v = W + b * 32; /* row-major: block b = (r, c/32) */
    const int e = hqq_oracle_mx_exponent(v, 32);
    scales[b] = (uint8_t)(e + 127);
    for (int i = 0; i < 32; ++i) {
      const float x = ldexpf(v[i], -e); /* exact division by the power of two */
      const uint8_t c = hqq_oracle_e2m1_encode(x);
      const int64_t k = b * 32 + i;
      if ((k & 1) == 0)
        codes[k / 2] = c;
      else
        codes[k / 2] |= (uint8_t)(c << 4);
    }
  }
}

void hqq_oracle_mxfp4_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t rows,
                                 int64_t cols, float* out) {
  const int64_t n = rows * cols;
  for (int64_t k = 0; k < n; ++k) {
    const uint8_t c = (k & 1) ? (uint8_t)(codes[k / 2] >> 4) : (uint8_t)(codes[k / 2] & 15);
    out[k] = ldexpf(hqq_oracle_e2m1_decode(c), (int)scales[k / 32] - 127);
  }
}
