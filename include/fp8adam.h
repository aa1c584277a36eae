/*
 * fp8adam.h -- C ABI of the B200 (sm_100a) AdamW step with FP8-stored
 * moments.
 *
 * What the library computes (sources cited by page title and section):
 *   - "Scaling FP8 training to trillion-token LLMs" (abstract): both Adam
 *     moments are quantised to FP8.
 *   - blog.daoxuan.cc explainer of that paper, section "Adam 为什么给第一矩选
 *     E4M3、第二矩选 E5M2": the first moment m is stored in E4M3 (precision),
 *     the second moment v in E5M2 (range); sub-section "两种 FP8 格式差在指数位
 *     和尾数位" gives the two bit layouts.
 *   - "FP8训练的稳定性挑战：E5M2与E4M3格式在梯度更新与前向传播中的混合精度策略",
 *     section "代码示例" (optim.AdamW) for the update, section
 *     "应对FP8训练稳定性挑战的策略" (amax-tracked range and exponent-bias
 *     adjustment) and its transformer_engine example (DelayedScaling,
 *     margin 0) for the per-tensor scale.
 *
 * One step, per tensor i and element j (all fp32, no FMA contraction):
 *   g      = bf16 gradient widened to fp32
 *   m_old  = dec(qm) / scale_m[i]          v_old = dec(qv) / scale_v[i]
 *   m      = b1*m_old + (1-b1)*g            v     = b2*v_old + (1-b2)*g*g
 *   amax_m[i] = max|m|, amax_v[i] = max|v| over the tensor (unquantised)
 *   s'     = largest 2^k, |k| <= 126, with amax_prev * 2^k <= max of the
 *            format (448 for E4M3, 57344 for E5M2); amax_prev is the previous
 *            step's amax, or this step's own at step 1 (a pre-pass); an amax
 *            of 0, inf or NaN keeps the previous scale
 *   qm     = enc(m * s'_m)                  qv    = enc(v * s'_v)
 *            (round to nearest, ties to even code, saturate to +-max, NaN
 *            -> NaN code)
 *   p      = p*(1 - lr*wd) - (lr/(1-b1^t)) * m / (sqrt(v)/sqrt(1-b2^t) + eps)
 *            evaluated as den = sqrtf(v)*isbc2; den = den + eps; u = m/den;
 *            p = p*decay; p = p - step_size*u, with isbc2, step_size and
 *            decay computed in double on the host and rounded once to fp32.
 *   scale_m[i] = s'_m, scale_v[i] = s'_v after the step.
 * The update uses this step's unquantised m and v; the FP8 codes carry them
 * to the next step.
 *
 * Memory and ownership.  The caller owns every tensor buffer: params (fp32),
 * grads (bf16 bit patterns), m and v (uint8 codes, or fp32 in FP8ADAM_FP32
 * mode), and the per-tensor arrays scale_m/scale_v/amax_m/amax_v (fp32,
 * num_tensors each).  All are device pointers, fixed from create to destroy.
 * Initial state: codes 0, scales 1.0, amax 0.0.  The context owns its
 * device-side tables and accumulators.
 *
 * Threading.  A context is used from one host thread and one stream at a
 * time.  fp8adam_step is asynchronous on the given stream and never
 * synchronises the host.  The CUDA device current at create must be current
 * at every call.
 *
 * Errors.  Every function returns FP8ADAM_OK (0) or a negative code; argument
 * errors are detected on the host before any GPU work is queued.
 */
#ifndef FP8ADAM_H
#define FP8ADAM_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FP8ADAM_OK 0
#define FP8ADAM_ERR_INVALID_ARG (-1)     /* null pointer, bad size or hyper-parameter */
#define FP8ADAM_ERR_UNSUPPORTED_FMT (-2) /* format id not in fp8adam_fmt */
#define FP8ADAM_ERR_CUDA (-3)            /* a CUDA runtime call failed */
#define FP8ADAM_ERR_OOM (-4)             /* device allocation failed in create */
#define FP8ADAM_ERR_WRONG_DEVICE (-5)    /* current device differs from create's */
#define FP8ADAM_ERR_NOALLOC_LIMIT (-6)   /* more tensors than fp8adam_step_noalloc holds */
#define FP8ADAM_ERR_DEVICE_TIMEOUT (-7)  /* a kernel's bounded wait ran out (see fp8adam_check) */
#define FP8ADAM_ERR_DEBUG_BOUNDS (-8)    /* debug build: an access outside its tensor was skipped */
#define FP8ADAM_ERR_OVERLAP (-9)         /* create, step_noalloc: a written buffer overlaps another */
#define FP8ADAM_ERR_SCHEDULE_END (-10)   /* a scheduled step ran past its schedule (see fp8adam_check) */

/* Storage format of a moment. */
typedef enum {
  FP8ADAM_E4M3 = 0, /* OCP E4M3 ("fn"): bias 7, max 448, S.1111.111 = NaN, no inf */
  FP8ADAM_E5M2 = 1, /* E5M2: bias 15, max 57344, IEEE-style inf/NaN */
  FP8ADAM_FP32 = 2  /* unquantised fp32 moment (reference mode, 4 B/element) */
} fp8adam_fmt;

/* Flags of fp8adam_create. */
#define FP8ADAM_FLAG_STATS 1u            /* count flushed v and saturated codes */
#define FP8ADAM_FLAG_JIT_EVERY_STEP 2u   /* "current" scaling: pre-pass every step */
#define FP8ADAM_FLAG_NO_TMA 16u          /* load through per-thread vector loads only
                                            (for comparison; same results).  By
                                            default, FP8 m and v on 16-byte
                                            aligned tensors are staged through
                                            shared memory with TMA bulk copies. */

/* One tensor.  param: fp32[numel]; grad: bf16[numel] (raw bits); m, v:
 * uint8[numel] codes or fp32[numel] in FP8ADAM_FP32 mode.  Any numel in [0, 2^48]
 * (an empty tensor is skipped and its state left as is).  Buffers that are
 * 16-byte aligned take the vectorised path; others are processed element by
 * element, with the same results. */
typedef struct {
  float* param;
  const uint16_t* grad;
  void* m;
  void* v;
  int64_t numel;
} fp8adam_tensor;

typedef struct fp8adam_ctx fp8adam_ctx; /* opaque */

/* Builds the device tensor table and chunk table of a whole parameter list
 * (one step = one kernel launch over all tensors).  Copies `tensors`
 * (host array) to the device, allocates the context's accumulators and
 * synchronises once.  scale_m/scale_v/amax_m/amax_v: device fp32
 * [num_tensors].  m_fmt/v_fmt: fp8adam_fmt.  Returns INVALID_ARG for null
 * pointers, num_tensors < 1, numel < 0 or > 2^48; UNSUPPORTED_FMT; OVERLAP if a
 * buffer the step writes (param, m, v, and with fp8adam_create_ex the bf16
 * copies) overlaps any other buffer of the list (gradients, which are only
 * read, may overlap one another); OOM; CUDA.  Checked on the host before
 * any CUDA call. */
int fp8adam_create(const fp8adam_tensor* tensors, int32_t num_tensors,
                   float* scale_m, float* scale_v, float* amax_m,
                   float* amax_v, int32_t m_fmt, int32_t v_fmt,
                   uint32_t flags, fp8adam_ctx** out);

/* One AdamW step (t = step, 1-based) on every tensor of the context, queued
 * on `cuda_stream` (a cudaStream_t; NULL = legacy default stream).  Requires
 * 0 <= beta1, beta2 < 1, eps >= 0, finite lr and weight_decay, step >= 1;
 * otherwise INVALID_ARG with nothing queued.  At step 1 (or every step with
 * FP8ADAM_FLAG_JIT_EVERY_STEP) an amax pre-pass runs first.  The staged step
 * kernel is launched with programmatic dependent launch: it may start while
 * the previous kernel on the stream finishes, and reads nothing that kernel
 * can write before that kernel has completed (results are unchanged).
 * Returns CUDA if a launch fails. */
int fp8adam_step(fp8adam_ctx* ctx, float lr, float beta1, float beta2,
                 float eps, float weight_decay, int64_t step,
                 void* cuda_stream);

/* Reads the counters accumulated since create or the last reset (only with
 * FP8ADAM_FLAG_STATS; zeros otherwise): out[0] = v elements with v > 0 whose
 * code is +-0 ("flushed"), out[1] = elements whose scaled m or v exceeded the
 * format's max (saturated; one count per moment).  `out` is host memory;
 * waits for `cuda_stream`. */
int fp8adam_get_stats(fp8adam_ctx* ctx, uint64_t* out, void* cuda_stream);

/* Zeroes the counters (queued on cuda_stream). */
int fp8adam_reset_stats(fp8adam_ctx* ctx, void* cuda_stream);

/* Checks the context's device error word (waits for cuda_stream): returns
 * FP8ADAM_OK; FP8ADAM_ERR_DEVICE_TIMEOUT if a step kernel's bounded wait for
 * its shared-memory copies ran out (each wait gives up after about 1 s; the
 * CTA waits, bounded, for its copies in flight and leaves its chunk
 * unfinished, and CTAs that start later return at once); in the debug build,
 * FP8ADAM_ERR_DEBUG_BOUNDS if a bounds check skipped an access.  On an error
 * it also clears the error word and the per-step device state (amax
 * accumulators, chunk counters), so the context can run the next step; the
 * params and moments of the failed step are partly updated and should be
 * restored from a checkpoint. */
int fp8adam_check(fp8adam_ctx* ctx, void* cuda_stream);

/* Debug build only (libfp8adam_debug.so, compiled with FP8ADAM_DEBUG; the
 * release build returns FP8ADAM_ERR_INVALID_ARG and checks nothing).
 * fp8adam_debug_inject_wait: from the next launch on, CTA `cta` of a staged
 * step kernel arms the barrier of its sub-tile `subtile` but issues no copies
 * for it, so that wait runs out and the kernel takes its timeout path (for
 * testing the bounded waits without a GPU fault); -1, -1 switches it off.
 * fp8adam_debug_set_numel: lowers tensor `tensor`'s element count in the
 * device tensor table (not below 0, not above its real size), so the chunk
 * table runs past it and the bounds checks fire (every access stays inside
 * the real buffers). */
int fp8adam_debug_inject_wait(int32_t cta, int32_t subtile);
int fp8adam_debug_set_numel(fp8adam_ctx* ctx, int32_t tensor, int64_t numel);

/* Frees the context (synchronises the device first).  NULL is accepted. */
int fp8adam_destroy(fp8adam_ctx* ctx);

/* Static description of an error code. */
const char* fp8adam_strerror(int code);

/* ---- options: scaling and read-back variants, stochastic rounding, fused
 * loss-scale removal / clipping / skip-on-non-finite, bf16 param copy -----
 * Sources: "FP8训练的稳定性挑战…", section "应对FP8训练稳定性挑战的策略"
 * (stochastic rounding, gradient clipping, adaptive gradient scaling), its
 * GradScaler / clip_grad_norm_ examples and the transformer_engine
 * DelayedScaling example (margin, amax_history_len, amax algo MAX); the
 * daoxuan.cc explainer's numeric example (v cut to 0 -> 1/(0+eps)) for the
 * update from stored moments. */
#define FP8ADAM_FLAG_UPDATE_FROM_STORED 4u   /* the update reads dec(code)/scale */
#define FP8ADAM_FLAG_STOCHASTIC_ROUNDING 8u  /* codes rounded stochastically */
/* With FP8ADAM_FLAG_STOCHASTIC_ROUNDING (INVALID_ARG without it): 16-bit
 * draws instead of 32-bit ones, rounded by the B200's stochastic-rounding
 * conversion (cvt.rs, four codes per instruction, one Philox4x32-10 call per
 * eight elements).  The code of element j of tensor i rounds up iff
 * floor((|x|-lo)/(hi-lo) * 2^16) + r >= 2^16, with r the draw of code j % 4
 * of word 2*((j/4) % 2) + (0 for m, 1 for v) of the Philox4x32-10 call with
 * counter (j/8 low, j/8 high, id(i), step low 32 bits) and key (seed low,
 * seed high), draws as fp8adam_encode_sr16 takes them; id(i) and the seed
 * are fp8adam_options' (sr_counter_ids, seed).  The probability of rounding
 * up is the exact one rounded down to a multiple of 2^-16. */
#define FP8ADAM_FLAG_SR_DRAW16 32u

typedef struct {
  float* scale_m;            /* as fp8adam_create: device fp32 [num_tensors] */
  float* scale_v;
  float* amax_m;
  float* amax_v;
  int32_t m_fmt;             /* fp8adam_fmt */
  int32_t v_fmt;
  uint32_t flags;            /* FP8ADAM_FLAG_* */
  int32_t margin_m;          /* scale = 2^(k - margin), k as above; 0..64 */
  int32_t margin_v;
  int32_t amax_history_len;  /* <= 1: the previous step's amax; > 1 (<= 1024): the
                                max over the last amax_history_len steps */
  float* amax_history_m;     /* device fp32 [amax_history_len][num_tensors], zero
                                at the start of training, caller-owned (part of the
                                checkpointed state); slot (step-1) % len holds the
                                amax of that step.  NULL when len <= 1. */
  float* amax_history_v;
  uint64_t seed;             /* stochastic rounding: random bits of element j of
                                tensor i at step t for moment w (0 = m, 1 = v) are
                                word 2*(j&1) + w of Philox4x32-10 with counter
                                (j/2 low, j/2 high, id(i), t low 32 bits) and key
                                (seed low, seed high); a code rounds up to the
                                next grid value iff r*(hi-lo) < (|x|-lo)*2^32
                                (16-bit draws: FP8ADAM_FLAG_SR_DRAW16).  id(i)
                                is sr_counter_ids[i], or i. */
  uint16_t* const* param_bf16; /* host array [num_tensors] of device bf16 buffers
                                  [numel] receiving the updated params rounded to
                                  nearest even (entries may be NULL), or NULL */
  int32_t chunk_elems;       /* elements per CTA: 0 = guided by the work left
                                (each chunk, in launch order, takes the
                                elements still to come / resident CTAs,
                                rounded down to a multiple of 4096 within
                                [8192, 131072], or [4096, 131072] for a list
                                too small to fill one wave of 8192-element
                                chunks); otherwise a multiple of 4096
                                in [4096, 131072].  A tensor's last chunk, and
                                one that would cross a multiple of 2^33
                                elements of its tensor, is cut shorter.
                                Results do not depend on it. */
  const uint32_t* sr_counter_ids; /* host array [num_tensors], read by create:
                                tensor i's word in the stochastic-rounding
                                counter (id(i) above), e.g. its index in a model
                                whose tensors are split over several contexts
                                (ZeRO-1 shards), so that every tensor draws the
                                same bits as in one context over the whole
                                model; NULL: i.  Any values; tensors sharing an
                                id and a seed share their draws. */
} fp8adam_options;

/* fp8adam_create with options (fp8adam_create is this call with the options
 * all off).  Returns INVALID_ARG for bad options. */
int fp8adam_create_ex(const fp8adam_tensor* tensors, int32_t num_tensors,
                      const fp8adam_options* opts, fp8adam_ctx** out);

typedef struct {
  float lr, beta1, beta2, eps, weight_decay;
  int64_t step;              /* 1-based */
  float loss_scale;          /* gradients are divided by it (1: none; > 0) */
  float max_norm;            /* <= 0: no clipping; else the global L2 norm of the
                                unscaled gradients over all tensors is clipped to it */
  int32_t skip_nonfinite;    /* non-zero: if any gradient is inf/NaN the whole step
                                leaves every buffer untouched */
} fp8adam_step_params;

/* One step with per-step gradient handling.  When max_norm > 0 or
 * skip_nonfinite is set, a pre-pass over all gradients computes (in a fixed
 * reduction order) sumsq = sum of g^2, the multiplier c = (1/loss_scale) *
 * min(1, max_norm / (sqrt(sumsq)/loss_scale + 1e-6)) (double, rounded once to
 * fp32; clip_grad_norm_'s formula) and the non-finite count; the step then
 * uses g*c in place of g.  With only loss_scale != 1 there is no pre-pass: c =
 * 1/loss_scale (double, rounded once to fp32; the same value) is a kernel
 * argument.  Asynchronous on cuda_stream. */
int fp8adam_step_ex(fp8adam_ctx* ctx, const fp8adam_step_params* params,
                    void* cuda_stream);

/* One step (as fp8adam_step_ex) whose gradients come from host memory.
 * host_grads: host array [num_tensors] of host pointers; host_grads[i] holds
 * tensor i's numel bf16 gradients (may be NULL for an empty tensor).  Pinned
 * (page-locked) buffers let the copies run asynchronously and overlap the
 * step.  Each is copied into the tensor's device gradient buffer (the grad
 * pointer given at create) on a copy stream owned by the context, which first
 * waits for the work already queued on cuda_stream.  The tensors are taken in
 * up to 8 groups of about equal size, cut at tensor boundaries; the step of a
 * group is queued on cuda_stream behind that group's copies only, so the
 * copies of later groups overlap it.  With max_norm > 0 or skip_nonfinite
 * the step waits for all copies (the global norm needs every gradient).  amax_host (optional, host float [2 * num_tensors], pinned for
 * an asynchronous copy): receives amax_m then amax_v of this step.
 * Asynchronous: host buffers must stay valid, and amax_host is written, only
 * once the work queued on cuda_stream has completed.  The results equal
 * fp8adam_step_ex after copying the gradients.  Returns INVALID_ARG for a
 * NULL host pointer of a non-empty tensor or bad parameters, WRONG_DEVICE,
 * CUDA on a failed copy or launch.
 * Source of the step: as fp8adam_step_ex; the host-to-device gradient copy
 * is this library's end-to-end entry point (no passage on the pages). */
int fp8adam_step_host(fp8adam_ctx* ctx, const fp8adam_step_params* params,
                      const uint16_t* const* host_grads, float* amax_host,
                      void* cuda_stream);

/* ---- steps that can be captured in a CUDA graph ------------------------
 * fp8adam_step and fp8adam_step_ex pass the step's constants (t, lr, ...) as
 * kernel arguments, so a captured launch would replay the same step.  A
 * scheduled step instead takes them from device memory:
 *
 * fp8adam_set_schedule: steps[k] (host array, count >= 1) are the parameters
 * of steps first .. first + count - 1 (steps[k].step = steps[0].step + k,
 * each valid as for fp8adam_step_ex; lr and the other values may change from
 * step to step, e.g. a learning-rate schedule).  Their constants are computed
 * on the host exactly as fp8adam_step_ex computes them and copied to the
 * device, and the context's device step counter is set to steps[0].step.
 * Waits for cuda_stream (steps already queued may read the old schedule).
 * Without FP8ADAM_FLAG_JIT_EVERY_STEP the schedule starts at step 2 or later:
 * step 1 takes the amax pre-pass, which the host decides (run it with
 * fp8adam_step).  If any entry needs the grad-norm pre-pass (loss_scale != 1,
 * max_norm > 0 or skip_nonfinite), every scheduled step runs it (an entry
 * without those options gets multiplier 1 and the same results).
 *
 * fp8adam_step_scheduled: queues one step on cuda_stream: a one-thread kernel
 * copies the entry of the device step counter and advances the counter, then
 * the step's kernels read that entry.  It keeps no per-step state on the host,
 * so it can be captured once into a CUDA graph and the graph replayed, each
 * replay the next step.  A step past the end of the schedule updates nothing
 * and sets the context's error word: fp8adam_check then returns
 * FP8ADAM_ERR_SCHEDULE_END (and clears it).  The results of each step equal
 * fp8adam_step_ex with that entry's parameters.  INVALID_ARG without a
 * schedule.
 *
 * fp8adam_get_schedule_step: *next_step = the step the next scheduled step
 * will run (waits for cuda_stream). */
int fp8adam_set_schedule(fp8adam_ctx* ctx, const fp8adam_step_params* steps,
                         int32_t count, void* cuda_stream);
int fp8adam_step_scheduled(fp8adam_ctx* ctx, void* cuda_stream);
int fp8adam_get_schedule_step(fp8adam_ctx* ctx, int64_t* next_step,
                              void* cuda_stream);

/* Results of the last fp8adam_step_ex pre-pass: *grad_norm = the global L2
 * norm of the unscaled gradients, *skipped = 1 if that step was skipped.
 * Host outputs; waits for cuda_stream.  Zeros if no pre-pass ran. */
int fp8adam_get_grad_info(fp8adam_ctx* ctx, double* grad_norm,
                          uint32_t* skipped, void* cuda_stream);

/* ---- device codec (verification entry points) -------------------------
 * impl 0 = hardware conversion (cvt.rn.satfinite.{e4m3x2,e5m2x2}.f32 /
 * cvt.rn.f16x2.{e4m3x2,e5m2x2}), impl 1 = integer/bit-manipulation path.
 * Both implement the codec described above. */

/* out[j] = enc(fmt, x[j]) for j < n; x, out device pointers. */
int fp8adam_encode(int32_t fmt, const float* x, uint8_t* out, int64_t n,
                   int32_t impl, void* cuda_stream);

/* out[j] = enc(fmt, float with bit pattern first + j), j < n <= 2^32 - first:
 * encodes a range of the fp32 bit-pattern space without an input buffer. */
int fp8adam_encode_bits_range(int32_t fmt, uint32_t first, int64_t n,
                              uint8_t* out, int32_t impl, void* cuda_stream);

/* Stochastic rounding with caller-given random words: out[j] = the code of
 * x[j] rounded to the grid value below |x[j]| (lo) or above it (hi), up iff
 * r[j]*(hi-lo) < (|x[j]|-lo)*2^32; saturating to the largest finite code;
 * NaN -> 0x7F.  The encoder of FP8ADAM_FLAG_STOCHASTIC_ROUNDING.  x, r, out
 * device pointers of n elements; returns INVALID_ARG for n < 0 or a NULL
 * pointer with n > 0, UNSUPPORTED_FMT for fmt other than E4M3/E5M2.
 * Source: "随机舍入" in section "应对FP8训练稳定性挑战的策略" of
 * "FP8训练的稳定性挑战…". */
int fp8adam_encode_sr(int32_t fmt, const float* x, const uint32_t* r,
                      uint8_t* out, int64_t n, void* cuda_stream);

/* Stochastic rounding with 16-bit draws and caller-given words: out[j] = the
 * code of x[j], rounded up to hi iff floor((|x[j]|-lo)/(hi-lo) * 2^16) + r >=
 * 2^16, with r the draw of code j % 4 from word w[j / 4]: code 0 takes the
 * word's low 16 bits, code 1 the low 16 bits in reverse bit order, code 2 the
 * high 16 bits, code 3 the high 16 bits reversed; saturating to the largest
 * finite code; NaN -> 0x7F.  The encoder of FP8ADAM_FLAG_SR_DRAW16, one
 * hardware conversion per word.  x, out: device arrays of n elements; w:
 * device array of (n + 3) / 4 words.  Returns INVALID_ARG for n < 0 or a NULL
 * pointer with n > 0, UNSUPPORTED_FMT for fmt other than E4M3/E5M2.
 * Source: "随机舍入" in section "应对FP8训练稳定性挑战的策略" of
 * "FP8训练的稳定性挑战…" (which fixes no resolution for the draws). */
int fp8adam_encode_sr16(int32_t fmt, const float* x, const uint32_t* w,
                        uint8_t* out, int64_t n, void* cuda_stream);

/* out[j] = dec(fmt, codes[j]) as fp32. */
int fp8adam_decode(int32_t fmt, const uint8_t* codes, float* out, int64_t n,
                   int32_t impl, void* cuda_stream);

/* Number of kernels launched by fp8adam_step and the codec entry points in
 * this process since load (for accounting launches inside a timed region). */
uint64_t fp8adam_launch_count(void);

/* ---- allocation-free step ------------------------------------------------
 * No counterpart in the paper or the pages: this is a service for callers
 * that cannot allocate device memory -- a custom allocator or memory-pool
 * callback, a framework hook that must not grow the footprint, a process
 * whose memory is reserved up front, or a runtime that forbids cudaMalloc
 * after start-up.  fp8adam_create allocates tables and accumulators; this
 * call allocates nothing (no cudaMalloc, no cudaFree, no allocating library
 * routine).
 *
 * It performs one step exactly as fp8adam_create(...) + fp8adam_step(...)
 * with the same arguments would (same kernels' arithmetic, same results),
 * using as scratch one fixed device array inside the library: the tensor
 * table, per-tensor chunk offsets, amax accumulators and completion
 * counters for at most FP8ADAM_NOALLOC_MAX_TENSORS tensors (about 288 KiB,
 * held by every GPU that loads the library until the process exits).
 * The caller passes all inputs and outputs as for fp8adam_create; flags may
 * be 0 or FP8ADAM_FLAG_JIT_EVERY_STEP (no statistics).
 *
 * - num_tensors > FP8ADAM_NOALLOC_MAX_TENSORS returns FP8ADAM_ERR_NOALLOC_LIMIT
 *   with nothing queued; other argument errors as fp8adam_create/step,
 *   overlapping written buffers (FP8ADAM_ERR_OVERLAP) included.
 * - A NaN moment gives the canonical NaN amax (bits 0x7FFFFFFF), as the
 *   regular step does.
 * - The first call on a device looks up the scratch array's device address
 *   (cudaGetSymbolAddress) with that device current.
 * - Each call copies the tensor table from host memory into the scratch
 *   (the copy waits for work already queued on cuda_stream) and clears the
 *   accumulators, so no state carries over between calls.
 * - Every call shares the one scratch array: calls that overlap on the GPU
 *   (different streams, or different host threads) race and must not be
 *   issued; serialise them on one stream from one thread.
 * - Its kernel launches are not counted by fp8adam_launch_count. */
#define FP8ADAM_NOALLOC_MAX_TENSORS 4096
int fp8adam_step_noalloc(const fp8adam_tensor* tensors, int32_t num_tensors,
                         float* scale_m, float* scale_v, float* amax_m,
                         float* amax_v, int32_t m_fmt, int32_t v_fmt,
                         uint32_t flags, float lr, float beta1, float beta2,
                         float eps, float weight_decay, int64_t step,
                         void* cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* FP8ADAM_H */
