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
 *   R6 Stochastic rounding (an option): Philox4x32-10 draws keyed by seed,
 *      counter (element, tensor, step); either 32-bit draws with the exact
 *      probability quantised to 2^-32 (ref_encode_sr), or 16-bit draws in the
 *      lane order of the B200's stochastic-rounding conversion
 *      (ref_encode_sr16).
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

/* ======================================================================== */
/* Extensions (next rows of the build): scaling and read-back variants,      */
/* stochastic rounding, fused loss-scale/clip multiplier, bf16 param copy.   */
/* The default path above is untouched; ref_fp8adam_step_tensor_ex with all  */
/* options off computes exactly what ref_fp8adam_step_tensor computes.       */
/* ======================================================================== */

/* Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
 * easy as 1, 2, 3", SC 2011): ten rounds of two 32x32->64 multiplies, the key
 * bumped by the Weyl constants between rounds. */
void ref_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4]) {
  uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
  uint32_t k0 = key_in[0], k1 = key_in[1];
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint64_t p0 = (uint64_t)0xD2511F53u * (uint64_t)c0;
    const uint64_t p1 = (uint64_t)0xCD9E8D57u * (uint64_t)c2;
    const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    const uint32_t n0 = hi1 ^ c1 ^ k0, n1 = lo1, n2 = hi0 ^ c3 ^ k1, n3 = lo0;
    c0 = n0; c1 = n1; c2 = n2; c3 = n3;
  }
  out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* The 32 random bits of element j of tensor `tensor` at step t for moment
 * `which` (0 = m, 1 = v): counter (j/2 low, j/2 high, tensor, t low), key
 * (seed low, seed high); element j takes outputs 2*(j&1) + which. */
uint32_t ref_sr_bits(uint64_t seed, int32_t tensor, int64_t t, int64_t j, int which) {
  const uint64_t q = (uint64_t)j >> 1;
  const uint32_t ctr[4] = {(uint32_t)q, (uint32_t)(q >> 32), (uint32_t)tensor, (uint32_t)t};
  const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  uint32_t out[4];
  ref_philox4x32_10(ctr, key, out);
  return out[2 * (int)(j & 1) + which];
}

/* Stochastic rounding of x to the format: NaN -> 0x7F; |x| >= FMAX -> +-FMAX;
 * otherwise, with lo <= |x| < hi the two neighbouring finite values, round up
 * to hi iff r * (hi - lo) < (|x| - lo) * 2^32 (probability (|x|-lo)/(hi-lo)
 * quantised to 2^-32); evaluated exactly in double. */
uint32_t ref_encode_sr(int fmt, float x, uint32_t r) {
  if (isnan(x)) return 0x7Fu;
  const float* tab = g_table[fmt == ORC_E4M3 ? 0 : 1];
  const uint32_t sign = signbit(x) ? 0x80u : 0u;
  const double a = fabs((double)x);
  const uint32_t cmax = fmt_maxcode(fmt);
  if (a >= (double)tab[cmax]) return sign | cmax;
  uint32_t lo = 0, hi = cmax;
  while (hi - lo > 1) {
    const uint32_t mid = (lo + hi) / 2;
    if ((double)tab[mid] <= a) lo = mid; else hi = mid;
  }
  const double below = a - (double)tab[lo];                  /* exact */
  const double gap = (double)tab[hi] - (double)tab[lo];      /* a power of two */
  const int up = (double)r * gap < below * 4294967296.0;     /* both sides exact */
  return sign | (up ? hi : lo);
}

void ref_encode_sr_array(int fmt, const float* x, const uint32_t* r, uint8_t* out, int64_t n) {
  fpenv_guard g = env_enter();
  for (int64_t j = 0; j < n; ++j) out[j] = (uint8_t)ref_encode_sr(fmt, x[j], r[j]);
  env_leave(g);
}

/* ---- stochastic rounding with 16-bit draws ---------------------------------
 * A second reading of "随机舍入" ([ZYXY], "应对FP8训练稳定性挑战的策略"; the
 * page fixes neither the generator nor the resolution of the draw).  Each
 * code takes a 16-bit draw r, and x rounds up to hi iff
 *     floor((|x| - lo) / (hi - lo) * 2^16) + r >= 2^16,
 * i.e. with probability (|x|-lo)/(hi-lo) rounded down to a multiple of
 * 2^-16.  The draws of four consecutive codes come from one 32-bit word: the
 * first code takes the word's low half, the second the low half with its 16
 * bits in reverse order, the third the high half, the fourth the high half
 * reversed.  That is the rounding rule and the lane assignment of the
 * B200's f32 -> fp8 x4 stochastic-rounding conversion (measured on the
 * device over every lane and every field value on a sample of inputs);
 * saturation and NaN as in ref_encode_sr. */

/* the low 16 bits of x in reverse order */
uint32_t ref_rev16(uint32_t x) {
  uint32_t r = 0;
  for (int b = 0; b < 16; ++b)
    if (x & (1u << b)) r |= 1u << (15 - b);
  return r;
}

/* the draw of code k (0..3) among the four codes a word serves */
uint32_t ref_sr16_draw(uint32_t w, int k) {
  const uint32_t half = k < 2 ? (w & 0xFFFFu) : (w >> 16);
  return (k & 1) ? ref_rev16(half) : half;
}

uint32_t ref_encode_sr16(int fmt, float x, uint32_t r16) {
  if (isnan(x)) return 0x7Fu;
  const float* tab = g_table[fmt == ORC_E4M3 ? 0 : 1];
  const uint32_t sign = signbit(x) ? 0x80u : 0u;
  const double a = fabs((double)x);
  const uint32_t cmax = fmt_maxcode(fmt);
  if (a >= (double)tab[cmax]) return sign | cmax;
  uint32_t lo = 0, hi = cmax;
  while (hi - lo > 1) {
    const uint32_t mid = (lo + hi) / 2;
    if ((double)tab[mid] <= a) lo = mid; else hi = mid;
  }
  const double below = a - (double)tab[lo];              /* exact */
  const double gap = (double)tab[hi] - (double)tab[lo];  /* a power of two */
  const double f16 = floor(below / gap * 65536.0);       /* exact: scaling by powers of two */
  const int up = f16 + (double)(r16 & 0xFFFFu) >= 65536.0;
  return sign | (up ? hi : lo);
}

/* out[j] = the code of x[j] with draw r16[j] */
void ref_encode_sr16_array(int fmt, const float* x, const uint32_t* r16, uint8_t* out, int64_t n) {
  fpenv_guard g = env_enter();
  for (int64_t j = 0; j < n; ++j) out[j] = (uint8_t)ref_encode_sr16(fmt, x[j], r16[j]);
  env_leave(g);
}

/* out[j] = the code of x[j] with the draw of code j % 4 of word w[j / 4] */
void ref_encode_sr16_words(int fmt, const float* x, const uint32_t* w, uint8_t* out, int64_t n) {
  fpenv_guard g = env_enter();
  for (int64_t j = 0; j < n; ++j)
    out[j] = (uint8_t)ref_encode_sr16(fmt, x[j], ref_sr16_draw(w[j >> 2], (int)(j & 3)));
  env_leave(g);
}

/* The 16-bit draw of element j of tensor `tensor` at step t for moment
 * `which` (0 = m, 1 = v): one Philox4x32-10 call per eight elements, counter
 * (j/8 low, j/8 high, tensor, t low), key (seed low, seed high); elements
 * 8q .. 8q+3 take outputs 0 (m) and 1 (v), elements 8q+4 .. 8q+7 outputs 2
 * and 3; within its word, element j is code j % 4. */
uint32_t ref_sr16_bits(uint64_t seed, int32_t tensor, int64_t t, int64_t j, int which) {
  const uint64_t q = (uint64_t)j >> 3;
  const uint32_t ctr[4] = {(uint32_t)q, (uint32_t)(q >> 32), (uint32_t)tensor, (uint32_t)t};
  const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  uint32_t out[4];
  ref_philox4x32_10(ctr, key, out);
  return ref_sr16_draw(out[2 * (int)((j >> 2) & 1) + which], (int)(j & 3));
}

/* bf16 nearest-even rounding of an fp32 value written from the definition:
 * 8 significant bits, rint() (round half to even) on the scaled significand. */
uint16_t ref_f32_to_bf16(float x) {
  uint32_t u;
  memcpy(&u, &x, 4);
  if (isnan(x)) return (uint16_t)((u >> 16) | 0x0040u);  /* quiet NaN, sign kept */
  if (isinf(x) || x == 0.0f) return (uint16_t)(u >> 16);
  int e;
  (void)frexp((double)x, &e);               /* x = fr * 2^e, |fr| in [0.5, 1) */
  /* bf16 keeps 8 significant bits for normals; below 2^-126 the quantum is
   * fixed at 2^-133 (subnormals) */
  int q = e - 8;
  if (q < -133) q = -133;
  const double n = rint(ldexp((double)x, -q));             /* ties to even */
  const double y = ldexp(n, q);
  float yf = (float)y;                                      /* exact or overflow to inf */
  uint32_t v;
  memcpy(&v, &yf, 4);
  return (uint16_t)(v >> 16);
}

/* Global gradient statistics of the fused unscale / clip pre-pass:
 * *sumsq = the exact sum of g^2 over all tensors, rounded once to double
 * (each bf16 g^2 is an integer times a power of two; they are summed in a
 * fixed-point accumulator wide enough to be exact), *nonfinite = count of
 * non-finite gradients. */
#define ACC_LIMBS 12  /* 768 bits: g^2 spans 2^-266 .. 2^256, plus carry room */
void ref_grad_sumsq(int32_t T, const int64_t* numel, const uint16_t* const* grads, double* sumsq,
                    uint64_t* nonfinite) {
  uint64_t acc[ACC_LIMBS] = {0};
  uint64_t bad = 0;
  for (int32_t i = 0; i < T; ++i) {
    for (int64_t j = 0; j < numel[i]; ++j) {
      const uint16_t b = grads[i][j];
      const uint32_t ex = (b >> 7) & 0xFFu, man = b & 0x7Fu;
      if (ex == 0xFFu) { ++bad; continue; }
      /* |g| = sig * 2^(e2) with sig the integer significand (8 bits) */
      const uint32_t sig = ex ? (man | 0x80u) : man;
      const int e2 = ex ? (int)ex - 127 - 7 : -126 - 7;
      if (!sig) continue;
      /* g^2 = sig^2 * 2^(2*e2); bit position relative to 2^-280 */
      const uint64_t sq = (uint64_t)sig * sig;
      const int pos = 2 * e2 + 280;
      const int limb = pos / 64, sh = pos % 64;
      unsigned __int128 add = (unsigned __int128)sq << sh;
      for (int k = limb; k < ACC_LIMBS && add; ++k) {
        const unsigned __int128 s = (unsigned __int128)acc[k] + (uint64_t)add;
        acc[k] = (uint64_t)s;
        add = (add >> 64) + (s >> 64);
      }
    }
  }
  /* round the exact value once to double: sum the limbs from the most
   * significant, using long double only to collect 64 bits at a time is not
   * exact, so take the top 128 bits of the number and a sticky bit */
  int top = ACC_LIMBS - 1;
  while (top >= 0 && acc[top] == 0) --top;
  if (top < 0) { *sumsq = 0.0; *nonfinite = bad; return; }
  const int lead = 63 - __builtin_clzll(acc[top]);   /* leading bit inside limb */
  const int msb = top * 64 + lead;                    /* absolute bit index */
  /* 54 bits starting at msb (53 + guard) plus sticky */
  uint64_t mant = 0;
  int sticky = 0;
  for (int b = 0; b < 54; ++b) {
    const int bit = msb - b;
    mant <<= 1;
    if (bit >= 0) mant |= (acc[bit / 64] >> (bit % 64)) & 1u;
  }
  for (int bit = msb - 54; bit >= 0 && !sticky; --bit)
    if ((acc[bit / 64] >> (bit % 64)) & 1u) sticky = 1;
  /* mant has 54 bits: 53 kept + 1 guard */
  uint64_t kept = mant >> 1;
  const int guard = (int)(mant & 1u);
  if (guard && (sticky || (kept & 1u))) ++kept;       /* round half to even */
  *sumsq = ldexp((double)kept, msb - 52 - 280);
  *nonfinite = bad;
}

/* The fused gradient multiplier of a step: c = (1/loss_scale) * min(1,
 * max_norm / (norm + 1e-6)) with norm = sqrt(sumsq) / loss_scale (the L2 norm
 * of the unscaled gradients, as clip_grad_norm_ defines it); max_norm <= 0
 * disables clipping.  Computed in double, rounded once to fp32. */
float ref_grad_multiplier(double sumsq, float loss_scale, float max_norm) {
  const double inv = 1.0 / (double)loss_scale;
  double coef = 1.0;
  if (max_norm > 0.0f) {
    const double norm = sqrt(sumsq) * inv;
    coef = (double)max_norm / (norm + 1e-6);
    if (coef > 1.0) coef = 1.0;
  }
  return (float)(inv * coef);
}

/* Extension flags. */
#define ORC_FLAG_UPDATE_FROM_STORED 4u
#define ORC_FLAG_STOCHASTIC 8u
#define ORC_FLAG_SR_DRAW16 32u  /* with ORC_FLAG_STOCHASTIC: 16-bit draws (ref_encode_sr16) */

typedef struct {
  uint32_t flags;         /* ORC_FLAG_* */
  int32_t margin_m, margin_v;
  int32_t hist_len;       /* > 1: scale from the max of the last hist_len amax */
  float* hist_m;          /* [hist_len] this tensor's ring, slot (t-1) % hist_len */
  float* hist_v;
  uint64_t seed;          /* stochastic rounding */
  int32_t tensor_index;   /* stochastic rounding counter */
  float grad_mult;        /* g is multiplied by this first (1.0f: off) */
  int32_t skip;           /* non-zero: leave everything untouched */
  uint16_t* p_bf16;       /* optional: bf16 copy of the updated params */
} ref_step_opts;

static float hist_max(const float* h, int n) {
  float a = 0.0f;
  for (int k = 0; k < n; ++k) a = max_keep_nan(a, h[k]);
  return a;
}

static uint32_t encode_opt(int fmt, float x, const ref_step_opts* o, int64_t t, int64_t j, int which) {
  if ((o->flags & ORC_FLAG_STOCHASTIC) && (o->flags & ORC_FLAG_SR_DRAW16))
    return ref_encode_sr16(fmt, x, ref_sr16_bits(o->seed, o->tensor_index, t, j, which));
  if (o->flags & ORC_FLAG_STOCHASTIC)
    return ref_encode_sr(fmt, x, ref_sr_bits(o->seed, o->tensor_index, t, j, which));
  return ref_encode(fmt, x);
}

int ref_fp8adam_step_tensor_ex(int64_t n, float* p, const uint16_t* g, void* m, void* v,
                               float* scale_m, float* scale_v, float* amax_m, float* amax_v,
                               int m_fmt, int v_fmt, float lr, float beta1, float beta2,
                               float eps, float wd, int64_t t, uint32_t flags,
                               const ref_step_opts* o, uint64_t* stats) {
  if (n < 0 || t < 1 || !o) return -1;
  if (m_fmt < 0 || m_fmt > 2 || v_fmt < 0 || v_fmt > 2) return -1;
  if (o->hist_len > 1 && (!o->hist_m || !o->hist_v)) return -1;
  if (n == 0 || o->skip) return 0;
  fpenv_guard guard = env_enter();
  const ref_consts c = make_consts(lr, beta1, beta2, eps, wd, t);
  const float s_m = *scale_m, s_v = *scale_v;
  const float inv_s_m = 1.0f / s_m;
  const float inv_s_v = 1.0f / s_v;
  const float gm = o->grad_mult;

  float amax_in_m = *amax_m, amax_in_v = *amax_v;
  if (o->hist_len > 1) {
    amax_in_m = hist_max(o->hist_m, o->hist_len);
    amax_in_v = hist_max(o->hist_v, o->hist_len);
  }
  const int jit = (t == 1) || (flags & ORC_FLAG_JIT_EVERY_STEP);
  if (jit) {
    float am = 0.0f, av = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
      const float g0 = bf16_to_f32(g[i]);
      const float gi = g0 * gm;
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
  const float s_m_new = m_fmt == ORC_FP32 ? s_m : ref_pow2scale(m_fmt, amax_in_m, s_m, o->margin_m);
  const float s_v_new = v_fmt == ORC_FP32 ? s_v : ref_pow2scale(v_fmt, amax_in_v, s_v, o->margin_v);
  const float inv_s_m_new = 1.0f / s_m_new;
  const float inv_s_v_new = 1.0f / s_v_new;
  const float fmax_m = m_fmt == ORC_FP32 ? INFINITY : ref_fmax(m_fmt);
  const float fmax_v = v_fmt == ORC_FP32 ? INFINITY : ref_fmax(v_fmt);

  float am = 0.0f, av = 0.0f;
  uint64_t flushed = 0, saturated = 0;
  for (int64_t i = 0; i < n; ++i) {
    const float g0 = bf16_to_f32(g[i]);
    const float gi = g0 * gm;
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
    float mu = mn, vu = vn; /* the moments the update reads */
    if (m_fmt == ORC_FP32) {
      ((float*)m)[i] = mn;
    } else {
      const float xm = mn * s_m_new;
      const uint32_t q = encode_opt(m_fmt, xm, o, t, i, 0);
      ((uint8_t*)m)[i] = (uint8_t)q;
      if (fabsf(xm) > fmax_m) ++saturated;
      if (o->flags & ORC_FLAG_UPDATE_FROM_STORED) mu = ref_decode(m_fmt, q) * inv_s_m_new;
    }
    if (v_fmt == ORC_FP32) {
      ((float*)v)[i] = vn;
    } else {
      const float xv = vn * s_v_new;
      const uint32_t q = encode_opt(v_fmt, xv, o, t, i, 1);
      ((uint8_t*)v)[i] = (uint8_t)q;
      if (vn > 0.0f && (q & 0x7Fu) == 0u) ++flushed;
      if (fabsf(xv) > fmax_v) ++saturated;
      if (o->flags & ORC_FLAG_UPDATE_FROM_STORED) vu = ref_decode(v_fmt, q) * inv_s_v_new;
    }
    const float sq = sqrtf(vu);
    const float den0 = sq * c.isbc2;
    const float den = den0 + c.eps;
    const float u = mu / den;
    const float pd = p[i] * c.decay;
    const float w = c.step_size * u;
    p[i] = pd - w;
    if (o->p_bf16) o->p_bf16[i] = ref_f32_to_bf16(p[i]);
  }
  *scale_m = s_m_new;
  *scale_v = s_v_new;
  *amax_m = am;
  *amax_v = av;
  if (o->hist_len > 1) {
    o->hist_m[(t - 1) % o->hist_len] = am;
    o->hist_v[(t - 1) % o->hist_len] = av;
  }
  if (stats) {
    stats[0] += flushed;
    stats[1] += saturated;
  }
  env_leave(guard);
  return 0;
}

void ref_f32_to_bf16_array(const float* x, int64_t n, uint16_t* out) {
  fpenv_guard g = env_enter();
  for (int64_t i = 0; i < n; ++i) out[i] = ref_f32_to_bf16(x[i]);
  env_leave(g);
}
