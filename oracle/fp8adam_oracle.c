/*
 * fp8adam_oracle.c -- plain, slow, scalar CPU oracle for the AdamW step with
 * FP8-stored moments.  TEST INFRASTRUCTURE ONLY: it is called by the tests,
 * by the smoke check and by the timed CPU baseline, never by the library.  It
 * shares no code, header, table or constant with the CUDA path.
 *
 * Sources (cited by page title and section):
 *   [EXPL]  blog.daoxuan.cc explainer of "Scaling FP8 training to
 *           trillion-token LLMs", section "Adam 为什么给第一矩选 E4M3、第二矩选
 *           E5M2" and its sub-sections "两种 FP8 格式差在指数位和尾数位" (format
 *           table), "Adam 的更新公式决定了两边需求不对称", "一个数值例子"
 *           (worked example) and "实验证据 (Fig. 5)".
 *   [PAPER] "Scaling FP8 training to trillion-token LLMs" (Fishman, Chmiel,
 *           Banner, Soudry), abstract: both Adam moments quantised to FP8.
 *   [ZYXY]  "FP8训练的稳定性挑战：E5M2与E4M3格式在梯度更新与前向传播中的混合精度
 *           策略", sections "FP8格式简介" (bit table), "FP8混合精度训练的稳定性
 *           挑战" (overflow/underflow, rounding error), "应对FP8训练稳定性挑战的
 *           策略" (amax-driven range adjustment, exponent-bias adjustment),
 *           "代码示例" (optim.AdamW) and the transformer_engine example
 *           (DelayedScaling, margin 0).
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes of the repository):
 *   R1 AdamW equations: decoupled decay + bias correction, eps added after the
 *      square root, one fp32 operation per line, no FMA contraction.
 *   R2 The update uses this step's unquantised fp32 m, v; FP8 is the storage
 *      format carried to the next step.
 *   R3 Per-tensor power-of-two scale from the previous step's amax (history
 *      length 1, margin 0); step 1 (or every step in "current" scaling) takes
 *      the amax of the step itself from a pre-pass.
 *   R4 amax == 0 or non-finite keeps the previous scale.
 *   R5 Round to nearest, ties to the even code, saturate to +-max (satfinite);
 *      NaN encodes to 0x7F.
 *
 * Precision: every floating-point line is a single IEEE binary32 operation
 * (the method stores m, v for an fp32 update).  Build with
 * -ffp-contract=off and without -ffast-math; the entry points clear x86
 * FTZ/DAZ while they run so subnormals behave as IEEE requires.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#if defined(__x86_64__)
#include <xmmintrin.h>
#endif

/* Format identifiers of the oracle (kept equal to the library's enum by the
 * tests, not by a shared header). */
enum { ORC_E4M3 = 0, ORC_E5M2 = 1, ORC_FP32 = 2 };

/* ------------------------------------------------------------------------ */
/* FP/rounding environment guard                                              */
/* ------------------------------------------------------------------------ */
typedef struct { unsigned csr; } fpenv_guard;

static fpenv_guard env_enter(void) {
  fpenv_guard g = {0};
#if defined(__x86_64__)
  g.csr = _mm_getcsr();
  /* bit 15 = flush-to-zero, bit 6 = denormals-are-zero; rounding bits 13-14
   * forced to round-to-nearest. */
  _mm_setcsr(g.csr & ~((1u << 15) | (1u << 6) | (3u << 13)));
#endif
  return g;
}
static void env_leave(fpenv_guard g) {
#if defined(__x86_64__)
  _mm_setcsr(g.csr);
#else
  (void)g;
#endif
}

/* ------------------------------------------------------------------------ */
/* Codec ([EXPL] format table; [ZYXY] "FP8格式简介")                          */
/* ------------------------------------------------------------------------ */
/* E4M3 (OCP "fn" variant): 1 sign, 4 exponent (bias 7), 3 mantissa bits; the
 * all-ones pattern S.1111.111 is NaN, there is no infinity, max 0x7E = 448.
 * E5M2: 1 sign, 5 exponent (bias 15), 2 mantissa bits, IEEE-like: exponent 31
 * with mantissa 0 is infinity, mantissa != 0 is NaN, max 0x7B = 57344. */
static int fmt_mbits(int fmt) { return fmt == ORC_E4M3 ? 3 : 2; }
static int fmt_ebits(int fmt) { return fmt == ORC_E4M3 ? 4 : 5; }
static int fmt_bias(int fmt) { return fmt == ORC_E4M3 ? 7 : 15; }
static unsigned fmt_maxcode(int fmt) { return fmt == ORC_E4M3 ? 0x7Eu : 0x7Bu; }
/* exponent of the largest finite value: FMAX = 1.75 * 2^Ef */
static int fmt_emax(int fmt) { return fmt == ORC_E4M3 ? 8 : 15; }

/* Closed-form decode: (-1)^s * 2^(e-bias) * (1 + f/2^M) for e > 0 and
 * (-1)^s * 2^(1-bias) * (f/2^M) for e == 0; special codes as above. */
static float closed_form_decode(int fmt, uint32_t code) {
  const int M = fmt_mbits(fmt), E = fmt_ebits(fmt), bias = fmt_bias(fmt);
  code &= 0xFFu;
  const int s = (int)(code >> 7);
  const int e = (int)((code >> M) & ((1u << E) - 1u));
  const int f = (int)(code & ((1u << M) - 1u));
  double val;
  if (fmt == ORC_E4M3) {
    if (e == 15 && f == 7) return NAN;
  } else {
    if (e == 31) {
      if (f == 0) return s ? -INFINITY : INFINITY;
      return NAN;
    }
  }
  if (e == 0)
    val = ldexp((double)f / (double)(1 << M), 1 - bias);
  else
    val = ldexp(1.0 + (double)f / (double)(1 << M), e - bias);
  return (float)(s ? -val : val);
}

/* The 256 decoded values of each format, filled once from the closed form
 * when the library is loaded (the oracle is otherwise too slow for the
 * exhaustive tests). */
static float g_table[2][256];
__attribute__((constructor)) static void build_tables(void) {
  for (int fmt = 0; fmt < 2; ++fmt)
    for (uint32_t c = 0; c < 256; ++c) g_table[fmt][c] = closed_form_decode(fmt, c);
}

float ref_decode(int fmt, uint32_t code) { return g_table[fmt == ORC_E4M3 ? 0 : 1][code & 0xFFu]; }

float ref_fmax(int fmt) { return ref_decode(fmt, fmt_maxcode(fmt)); }

/* Encode: the finite code whose value is nearest to x, a tie going to the
 * code with a 0 least-significant bit; |x| >= FMAX (and +-inf) saturates to
 * +-FMAX; NaN gives 0x7F; the sign of x is kept, so -0 and negative values
 * that round to zero give 0x80.  The nearest code is found by bisection over
 * the non-negative finite codes, whose values increase with the code. */
uint32_t ref_encode(int fmt, float x) {
  if (isnan(x)) return 0x7Fu;
  const float* tab = g_table[fmt == ORC_E4M3 ? 0 : 1];
  const uint32_t sign = signbit(x) ? 0x80u : 0u;
  const double a = fabs((double)x);
  const uint32_t cmax = fmt_maxcode(fmt);
  if (a >= (double)tab[cmax]) return sign | cmax;
  /* largest code lo with value <= a (value of code 0 is 0 <= a always) */
  uint32_t lo = 0, hi = cmax; /* invariant: tab[lo] <= a < tab[hi] */
  while (hi - lo > 1) {
    const uint32_t mid = (lo + hi) / 2;
    if ((double)tab[mid] <= a) lo = mid; else hi = mid;
  }
  /* exact in double: a and the two neighbours lie within one binade (or in
   * the subnormal range) and carry at most 24 significant bits */
  const double dlo = a - (double)tab[lo];
  const double dhi = (double)tab[hi] - a;
  uint32_t c;
  if (dlo < dhi) c = lo;
  else if (dhi < dlo) c = hi;
  else c = (lo & 1u) ? hi : lo;
  return sign | c;
}

/* Bulk helpers for the exhaustive tests (no arithmetic beyond the above). */
void ref_encode_array(int fmt, const float* x, int64_t n, uint8_t* out) {
  fpenv_guard g = env_enter();
  for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)ref_encode(fmt, x[i]);
  env_leave(g);
}

/* Encodes the floats whose bit patterns are first, first+1, ..., first+n-1. */
void ref_encode_bits_range(int fmt, uint32_t first, int64_t n, uint8_t* out) {
  fpenv_guard g = env_enter();
  for (int64_t i = 0; i < n; ++i) {
    const uint32_t b = first + (uint32_t)i;
    float x;
    memcpy(&x, &b, 4);
    out[i] = (uint8_t)ref_encode(fmt, x);
  }
  env_leave(g);
}

void ref_decode_array(int fmt, const uint8_t* c, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = ref_decode(fmt, c[i]);
}

/* ------------------------------------------------------------------------ */
/* Per-tensor power-of-two scale ([ZYXY] "动态范围调整", "指数偏置调整",       */
/* DelayedScaling margin=0): the largest 2^k with amax * 2^k <= FMAX.          */
/* ------------------------------------------------------------------------ */
float ref_pow2scale(int fmt, float amax, float s_prev, int margin) {
  if (!isfinite(amax) || !(amax > 0.0f)) return s_prev; /* R4 */
  int e2;
  const float fr = frexpf(amax, &e2); /* amax = fr * 2^e2, fr in [0.5, 1) */
  const float f = 2.0f * fr;          /* amax = f * 2^(e2-1), f in [1, 2) */
  const int e = e2 - 1;
  /* f * 2^(Ef-e) <= 1.75 * 2^Ef iff f <= 1.75, otherwise one power less */
  int k = fmt_emax(fmt) - e - (f > 1.75f ? 1 : 0) - margin;
  if (k > 126) k = 126;
  if (k < -126) k = -126;
  return ldexpf(1.0f, k);
}

/* ------------------------------------------------------------------------ */
/* The step ([EXPL] "Adam 的更新公式决定了两边需求不对称"; [ZYXY] "代码示例"      */
/* optim.AdamW; [PAPER] abstract).                                            */
/* ------------------------------------------------------------------------ */
static float bf16_to_f32(uint16_t b) {
  const uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* max that lets a NaN through and keeps it */
static float max_keep_nan(float acc, float x) {
  if (isnan(acc)) return acc;
  if (isnan(x)) return x;
  return x > acc ? x : acc;
}

static float load_moment(int fmt, const void* base, int64_t i, float inv_scale) {
  if (fmt == ORC_FP32) return ((const float*)base)[i];
  const float d = ref_decode(fmt, ((const uint8_t*)base)[i]);
  return d * inv_scale;
}

/* Hyper-parameters of step t, computed in double and rounded once to fp32. */
typedef struct {
  float b1, omb1, b2, omb2, step_size, isbc2, eps, decay;
} ref_consts;

static ref_consts make_consts(float lr, float beta1, float beta2, float eps,
                              float wd, int64_t t) {
  ref_consts c;
  const double bc1 = 1.0 - pow((double)beta1, (double)t);
  const double bc2 = 1.0 - pow((double)beta2, (double)t);
  c.b1 = beta1;
  c.omb1 = (float)(1.0 - (double)beta1);
  c.b2 = beta2;
  c.omb2 = (float)(1.0 - (double)beta2);
  c.step_size = (float)((double)lr / bc1);
  c.isbc2 = (float)(1.0 / sqrt(bc2));
  c.eps = eps;
  c.decay = (float)(1.0 - (double)lr * (double)wd);
  return c;
}

/* Exposes the rounded constants so tests can check them against the
 * library's documented definitions. out: b1, omb1, b2, omb2, step_size,
 * isbc2, eps, decay. */
void ref_step_constants(float lr, float beta1, float beta2, float eps, float wd,
                        int64_t t, float* out8) {
  const ref_consts c = make_consts(lr, beta1, beta2, eps, wd, t);
  out8[0] = c.b1; out8[1] = c.omb1; out8[2] = c.b2; out8[3] = c.omb2;
  out8[4] = c.step_size; out8[5] = c.isbc2; out8[6] = c.eps; out8[7] = c.decay;
}

/* Flags of the step. */
#define ORC_FLAG_JIT_EVERY_STEP 2u

/* One AdamW step on one tensor.
 *   p[n]       fp32 master params, updated in place
 *   g[n]       bf16 gradient bits
 *   m[n], v[n] moment storage: uint8 codes (E4M3/E5M2) or fp32 (FP32)
 *   *scale_m, *scale_v   per-tensor scales (code = enc(x * scale))
 *   *amax_m,  *amax_v    max |m|, max |v| of the unquantised moments of the
 *                        last step (input: previous step; output: this step)
 *   stats[2]   (optional) += flushed v count, += saturated count
 * An empty tensor (n == 0) is left untouched.  Returns 0, or -1 on a bad
 * argument. */
int ref_fp8adam_step_tensor(int64_t n, float* p, const uint16_t* g, void* m,
                            void* v, float* scale_m, float* scale_v,
                            float* amax_m, float* amax_v, int m_fmt, int v_fmt,
                            float lr, float beta1, float beta2, float eps,
                            float wd, int64_t t, uint32_t flags,
                            uint64_t* stats) {
  if (n < 0 || t < 1) return -1;
  if (m_fmt < 0 || m_fmt > 2 || v_fmt < 0 || v_fmt > 2) return -1;
  if (n == 0) return 0;
  fpenv_guard guard = env_enter();
  const ref_consts c = make_consts(lr, beta1, beta2, eps, wd, t);
  const float s_m = *scale_m, s_v = *scale_v;
  const float inv_s_m = 1.0f / s_m; /* exact: a power of two */
  const float inv_s_v = 1.0f / s_v;

  /* amax that sets this step's encode scale: previous step's, or (step 1,
   * "current" scaling) this step's own from a pre-pass of the same math */
  float amax_in_m = *amax_m, amax_in_v = *amax_v;
  const int jit = (t == 1) || (flags & ORC_FLAG_JIT_EVERY_STEP);
  if (jit) {
    float am = 0.0f, av = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
      const float gi = bf16_to_f32(g[i]);
      const float mo = load_moment(m_fmt, m, i, inv_s_m);
      const float vo = load_moment(v_fmt, v, i, inv_s_v);
      const float t1 = c.b1 * mo;
      const float t2 = c.omb1 * gi;
      const float mn = t1 + t2;
      const float gg = gi * gi;
      const float t3 = c.b2 * vo;
      const float t4 = c.omb2 * gg;
      const float vn = t3 + t4;
      am = max_keep_nan(am, fabsf(mn));
      av = max_keep_nan(av, fabsf(vn));
    }
    amax_in_m = am;
    amax_in_v = av;
  }
  const float s_m_new =
      m_fmt == ORC_FP32 ? s_m : ref_pow2scale(m_fmt, amax_in_m, s_m, 0);
  const float s_v_new =
      v_fmt == ORC_FP32 ? s_v : ref_pow2scale(v_fmt, amax_in_v, s_v, 0);
  const float fmax_m = m_fmt == ORC_FP32 ? INFINITY : ref_fmax(m_fmt);
  const float fmax_v = v_fmt == ORC_FP32 ? INFINITY : ref_fmax(v_fmt);

  float am = 0.0f, av = 0.0f;
  uint64_t flushed = 0, saturated = 0;
  for (int64_t i = 0; i < n; ++i) {
    const float gi = bf16_to_f32(g[i]);
    const float mo = load_moment(m_fmt, m, i, inv_s_m);
    const float vo = load_moment(v_fmt, v, i, inv_s_v);
    /* exponential moving averages of g and g^2 */
    const float t1 = c.b1 * mo;
    const float t2 = c.omb1 * gi;
    const float mn = t1 + t2;
    const float gg = gi * gi;
    const float t3 = c.b2 * vo;
    const float t4 = c.omb2 * gg;
    const float vn = t3 + t4;
    am = max_keep_nan(am, fabsf(mn));
    av = max_keep_nan(av, fabsf(vn));
    /* storage for the next step */
    if (m_fmt == ORC_FP32) {
      ((float*)m)[i] = mn;
    } else {
      const float xm = mn * s_m_new;
      ((uint8_t*)m)[i] = (uint8_t)ref_encode(m_fmt, xm);
      if (fabsf(xm) > fmax_m) ++saturated;
    }
    if (v_fmt == ORC_FP32) {
      ((float*)v)[i] = vn;
    } else {
      const float xv = vn * s_v_new;
      const uint32_t q = ref_encode(v_fmt, xv);
      ((uint8_t*)v)[i] = (uint8_t)q;
      if (vn > 0.0f && (q & 0x7Fu) == 0u) ++flushed;
      if (fabsf(xv) > fmax_v) ++saturated;
    }
    /* decoupled-decay, bias-corrected AdamW update from the fp32 m, v */
    const float sq = sqrtf(vn);
    const float den0 = sq * c.isbc2;
    const float den = den0 + c.eps;
    const float u = mn / den;
    const float pd = p[i] * c.decay;
    const float w = c.step_size * u;
    p[i] = pd - w;
  }
  *scale_m = s_m_new;
  *scale_v = s_v_new;
  *amax_m = am;
  *amax_v = av;
  if (stats) {
    stats[0] += flushed;
    stats[1] += saturated;
  }
  env_leave(guard);
  return 0;
}
