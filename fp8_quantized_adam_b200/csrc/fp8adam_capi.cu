// fp8adam_capi.cu -- the C ABI declared in include/fp8adam.h.
//
// Host side of the FP8-moment AdamW step: argument validation, the device
// tensor and chunk tables, per-step constants (computed in double, rounded
// once to fp32) and kernel dispatch over the (m format, v format, stats)
// variants, the option kernels and the gradient pre-pass.
// The kernels are in fp8adam_step.cuh; the codec in fp8_codec.cuh.

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <atomic>
#include <cstddef>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <new>
#include <vector>

#include "../../include/fp8adam.h"
#include "fp8_codec.cuh"
#include "fp8adam_ext.cuh"
#include "fp8adam_ext_tma.cuh"
#include "fp8adam_step.cuh"
#include "fp8adam_step_tma.cuh"

using namespace fp8adam;

namespace {

std::atomic<uint64_t> g_launches{0};

// ------------------------------------------------------------ codec kernels
template <int FMT, int IMPL>
__device__ __forceinline__ uint32_t enc1(float x) {
  if constexpr (IMPL == 0) return enc1_hw<FMT>(x);
  else return enc1_sw<FMT>(x);
}

// 4 consecutive inputs per thread so the hardware path uses both lanes of
// the x2 conversions.
template <int FMT, int IMPL>
__global__ void encode_kernel(const float* __restrict__ x, uint8_t* __restrict__ out, int64_t n) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x * 4;
  for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4; i < n; i += stride) {
    if (i + 4 <= n) {
      if constexpr (IMPL == 0) {
        const uint32_t lo = enc2_hw<FMT>(x[i], x[i + 1]);
        const uint32_t hi = enc2_hw<FMT>(x[i + 2], x[i + 3]);
        out[i] = (uint8_t)lo; out[i + 1] = (uint8_t)(lo >> 8);
        out[i + 2] = (uint8_t)hi; out[i + 3] = (uint8_t)(hi >> 8);
      } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) out[i + k] = (uint8_t)enc1<FMT, IMPL>(x[i + k]);
      }
    } else {
      for (int64_t k = i; k < n; ++k) out[k] = (uint8_t)enc1<FMT, IMPL>(x[k]);
    }
  }
}

// codes of the floats with bit patterns first .. first + n - 1; 4 per thread,
// written as one 32-bit word when aligned
template <int FMT, int IMPL>
__global__ void encode_bits_kernel(uint32_t first, uint8_t* __restrict__ out, int64_t n) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x * 4;
  for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4; i < n; i += stride) {
    float x[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) x[k] = __uint_as_float(first + (uint32_t)(i + k));
    if (i + 4 <= n) {
      uint32_t w;
      if constexpr (IMPL == 0) {
        w = enc2_hw<FMT>(x[0], x[1]) | (enc2_hw<FMT>(x[2], x[3]) << 16);
      } else {
        w = enc1_sw<FMT>(x[0]) | (enc1_sw<FMT>(x[1]) << 8) | (enc1_sw<FMT>(x[2]) << 16) |
            (enc1_sw<FMT>(x[3]) << 24);
      }
      *reinterpret_cast<uint32_t*>(out + i) = w;
    } else {
      for (int64_t k = i; k < n; ++k) out[k] = (uint8_t)enc1<FMT, IMPL>(x[k - i]);
    }
  }
}

template <int FMT, int IMPL>
__global__ void decode_kernel(const uint8_t* __restrict__ c, float* __restrict__ out, int64_t n) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x * 2;
  for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 2; i < n; i += stride) {
    if constexpr (IMPL == 0) {
      const uint32_t pair = (uint32_t)c[i] | (i + 1 < n ? (uint32_t)c[i + 1] << 8 : 0u);
      const float2 f = dec2_hw<FMT>(pair);
      out[i] = f.x;
      if (i + 1 < n) out[i + 1] = f.y;
    } else {
      out[i] = dec1_sw<FMT>(c[i]);
      if (i + 1 < n) out[i + 1] = dec1_sw<FMT>(c[i + 1]);
    }
  }
}

template <int FMT>
__global__ void encode_sr_kernel(const float* __restrict__ x, const uint32_t* __restrict__ r,
                                 uint8_t* __restrict__ out, int64_t n) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    out[i] = (uint8_t)enc1_sr<FMT>(x[i], r[i]);
}

// four codes per word: out[4q + k] = code k of x[4q .. 4q+3] rounded with
// word w[q] (inputs past n are 0 and their codes are not written)
template <int FMT>
__global__ void encode_sr16_kernel(const float* __restrict__ x, const uint32_t* __restrict__ w,
                                   uint8_t* __restrict__ out, int64_t n) {
  const int64_t nw = (n + 3) >> 2;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < nw; q += stride) {
    const int64_t i = q << 2;
    const float x0 = x[i];
    const float x1 = i + 1 < n ? x[i + 1] : 0.0f;
    const float x2 = i + 2 < n ? x[i + 2] : 0.0f;
    const float x3 = i + 3 < n ? x[i + 3] : 0.0f;
    const uint32_t d = cvt_rs4<FMT>(x0, x1, x2, x3, w[q]);
    out[i] = (uint8_t)d;
    if (i + 1 < n) out[i + 1] = (uint8_t)(d >> 8);
    if (i + 2 < n) out[i + 2] = (uint8_t)(d >> 16);
    if (i + 3 < n) out[i + 3] = (uint8_t)(d >> 24);
  }
}

int grid_for(int64_t n, int per_thread) {
  const int64_t want = (n + (int64_t)256 * per_thread - 1) / ((int64_t)256 * per_thread);
  const int64_t cap = 148 * 16;
  return (int)(want < 1 ? 1 : (want > cap ? cap : want));
}

int last_error() {
  return cudaGetLastError() == cudaSuccess ? FP8ADAM_OK : FP8ADAM_ERR_CUDA;
}

// ------------------------------------------------------------ dispatch tables
using StepFn = void (*)(const StepArgs);
template <int MF, int VF, bool S> StepFn step_fn() { return &fp8adam_step_kernel<MF, VF, S>; }
template <int MF, int VF> StepFn amax_fn() { return &fp8adam_amax_kernel<MF, VF>; }

StepFn pick_step(int mf, int vf, bool stats) {
  static const StepFn t[3][3][2] = {
      {{step_fn<0, 0, false>(), step_fn<0, 0, true>()}, {step_fn<0, 1, false>(), step_fn<0, 1, true>()},
       {step_fn<0, 2, false>(), step_fn<0, 2, true>()}},
      {{step_fn<1, 0, false>(), step_fn<1, 0, true>()}, {step_fn<1, 1, false>(), step_fn<1, 1, true>()},
       {step_fn<1, 2, false>(), step_fn<1, 2, true>()}},
      {{step_fn<2, 0, false>(), step_fn<2, 0, true>()}, {step_fn<2, 1, false>(), step_fn<2, 1, true>()},
       {step_fn<2, 2, false>(), step_fn<2, 2, true>()}}};
  return t[mf][vf][stats ? 1 : 0];
}
StepFn pick_amax(int mf, int vf) {
  static const StepFn t[3][3] = {{amax_fn<0, 0>(), amax_fn<0, 1>(), amax_fn<0, 2>()},
                                 {amax_fn<1, 0>(), amax_fn<1, 1>(), amax_fn<1, 2>()},
                                 {amax_fn<2, 0>(), amax_fn<2, 1>(), amax_fn<2, 2>()}};
  return t[mf][vf];
}

using TmaFn = void (*)(const StepArgs, uint32_t*);
template <int MF, int VF, bool S> TmaFn tma_fn() { return &fp8adam_step_tma_kernel<MF, VF, S>; }
TmaFn pick_tma(int mf, int vf, bool stats) {  // FP8 formats only
  static const TmaFn t[2][2][2] = {
      {{tma_fn<0, 0, false>(), tma_fn<0, 0, true>()}, {tma_fn<0, 1, false>(), tma_fn<0, 1, true>()}},
      {{tma_fn<1, 0, false>(), tma_fn<1, 0, true>()}, {tma_fn<1, 1, false>(), tma_fn<1, 1, true>()}}};
  return t[mf][vf][stats ? 1 : 0];
}

using ExtFn = void (*)(const ExtArgs);
template <int MF, int VF, bool S> ExtFn ext_fn() { return &fp8adam_step_ext_kernel<MF, VF, S>; }
template <int MF, int VF> ExtFn aext_fn() { return &fp8adam_amax_ext_kernel<MF, VF>; }

ExtFn pick_ext(int mf, int vf, bool stats) {
  static const ExtFn t[3][3][2] = {
      {{ext_fn<0, 0, false>(), ext_fn<0, 0, true>()}, {ext_fn<0, 1, false>(), ext_fn<0, 1, true>()},
       {ext_fn<0, 2, false>(), ext_fn<0, 2, true>()}},
      {{ext_fn<1, 0, false>(), ext_fn<1, 0, true>()}, {ext_fn<1, 1, false>(), ext_fn<1, 1, true>()},
       {ext_fn<1, 2, false>(), ext_fn<1, 2, true>()}},
      {{ext_fn<2, 0, false>(), ext_fn<2, 0, true>()}, {ext_fn<2, 1, false>(), ext_fn<2, 1, true>()},
       {ext_fn<2, 2, false>(), ext_fn<2, 2, true>()}}};
  return t[mf][vf][stats ? 1 : 0];
}
using ExtTmaFn = void (*)(const ExtArgs, uint32_t*);
// srk: the rounding kind (0 nearest, 1 stochastic with 32-bit draws, 2 with
// 16-bit draws)
template <int MF, int VF, bool S, int K> ExtTmaFn ext_tma_fn() { return &fp8adam_step_ext_tma_kernel<MF, VF, S, K>; }
template <int MF, int VF, bool S, int K> ExtTmaFn ext_tma_lean_fn() {
  return &fp8adam_step_ext_tma_kernel<MF, VF, S, K, false>;
}
template <int MF, int VF, bool S> struct ExtTmaRow {
  ExtTmaFn k[3] = {ext_tma_fn<MF, VF, S, 0>(), ext_tma_fn<MF, VF, S, 1>(), ext_tma_fn<MF, VF, S, 2>()};
  ExtTmaFn lean[2] = {ext_tma_lean_fn<MF, VF, S, 1>(), ext_tma_lean_fn<MF, VF, S, 2>()};
};
template <bool S> const ExtTmaFn* ext_tma_row(int mf, int vf, bool lean) {  // FP8 formats only
  static const ExtTmaRow<0, 0, S> r00;
  static const ExtTmaRow<0, 1, S> r01;
  static const ExtTmaRow<1, 0, S> r10;
  static const ExtTmaRow<1, 1, S> r11;
  if (mf == 0) return vf == 0 ? (lean ? r00.lean : r00.k) : (lean ? r01.lean : r01.k);
  return vf == 0 ? (lean ? r10.lean : r10.k) : (lean ? r11.lean : r11.k);
}
// the lean stochastic-rounding kernels (no update-from-stored, no bf16 copy,
// gradient multiplier 1); srk 1 or 2
ExtTmaFn pick_ext_tma_sr_lean(int mf, int vf, bool stats, int srk) {
  return (stats ? ext_tma_row<true>(mf, vf, true) : ext_tma_row<false>(mf, vf, true))[srk - 1];
}
ExtTmaFn pick_ext_tma(int mf, int vf, bool stats, int srk) {
  return (stats ? ext_tma_row<true>(mf, vf, false) : ext_tma_row<false>(mf, vf, false))[srk];
}
ExtFn pick_amax_ext(int mf, int vf) {
  static const ExtFn t[3][3] = {{aext_fn<0, 0>(), aext_fn<0, 1>(), aext_fn<0, 2>()},
                                {aext_fn<1, 0>(), aext_fn<1, 1>(), aext_fn<1, 2>()},
                                {aext_fn<2, 0>(), aext_fn<2, 1>(), aext_fn<2, 2>()}};
  return t[mf][vf];
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// A staged step kernel launched with programmatic dependent launch: it may
// start while the previous kernel on the stream finishes (it waits for that
// kernel's writes with griddepcontrol.wait).
template <typename Args>
cudaError_t launch_staged_pdl(void (*fn)(const Args, uint32_t*), dim3 grid, dim3 block, cudaStream_t st,
                              const Args& args, uint32_t* err) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = kTmaSmemBytes;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fn, args, err);
}

static_assert(FP8ADAM_FLAG_UPDATE_FROM_STORED == kExtFromStored && FP8ADAM_FLAG_STOCHASTIC_ROUNDING == kExtStochastic &&
                  FP8ADAM_FLAG_SR_DRAW16 == kExtSrDraw16,
              "the step passes these flag bits to the kernels unchanged");

// the rounding kind of a flag set (0 nearest, 1 SR with 32-bit draws, 2 SR with 16-bit draws)
int sr_kind_of(uint32_t flags) {
  if (!(flags & FP8ADAM_FLAG_STOCHASTIC_ROUNDING)) return 0;
  return (flags & FP8ADAM_FLAG_SR_DRAW16) ? 2 : 1;
}

// Guided chunk lengths (fp8adam_create_ex with chunk_elems 0): see there.
constexpr int64_t kGuidedRounds = 1;
constexpr int64_t kGuidedMin = 8192;
constexpr int64_t kCounterSpan = 1ll << 33;  // a chunk stays within one span of 2^33 elements

// Constants of step t: computed in double, rounded once to fp32.
StepConsts make_consts(const fp8adam_step_params& p) {
  const double bc1 = 1.0 - std::pow((double)p.beta1, (double)p.step);
  const double bc2 = 1.0 - std::pow((double)p.beta2, (double)p.step);
  StepConsts c;
  c.b1 = p.beta1;
  c.omb1 = (float)(1.0 - (double)p.beta1);
  c.b2 = p.beta2;
  c.omb2 = (float)(1.0 - (double)p.beta2);
  c.step_size = (float)((double)p.lr / bc1);
  c.isbc2 = (float)(1.0 / std::sqrt(bc2));
  c.eps = p.eps;
  c.decay = (float)(1.0 - (double)p.lr * (double)p.weight_decay);
  return c;
}

// A scheduled step's first kernel (one thread): copy the entry of the
// device step counter to `cur` and advance the counter; past the end of the
// schedule, mark `cur` invalid (the step's kernels then do nothing) and set
// bit 1 of the error word.
__global__ void sched_select_kernel(const SchedEntry* sched, int64_t first, int32_t count, int64_t* next_step,
                                    SchedEntry* cur, uint32_t* err) {
  const int64_t k = *next_step - first;
  if (k < 0 || k >= count) {
    cur->valid = 0;
    atomicOr(err, 2u);
    return;
  }
  *cur = sched[k];
  cur->valid = 1;
  *next_step += 1;
}

// True if two of the byte ranges overlap and at least one of them is
// written.  Sorted by start, a range overlaps an earlier one iff it starts
// before the furthest end seen so far (of any range if it is written, of
// the written ranges if it is only read).
struct ByteRange {
  uintptr_t begin, end;
  bool written;
};
bool written_range_overlaps(std::vector<ByteRange>& r) {
  std::sort(r.begin(), r.end(), [](const ByteRange& a, const ByteRange& b) { return a.begin < b.begin; });
  uintptr_t end_all = 0, end_written = 0;
  for (const ByteRange& x : r) {
    if (x.begin < (x.written ? end_all : end_written)) return true;
    end_all = end_all > x.end ? end_all : x.end;
    if (x.written) end_written = end_written > x.end ? end_written : x.end;
  }
  return false;
}

// NVTX range over a host call (visible to Nsight tools; a no-op without one)
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

}  // namespace

// ------------------------------------------------------------ the context
struct fp8adam_ctx {
  int device = -1;
  int32_t T = 0;
  int32_t m_fmt = 0, v_fmt = 0;
  uint32_t flags = 0;
  int32_t total_units = 0;  // chunks of the whole list = grid of every per-step kernel
  int32_t chunk_elems = 0;  // elements per chunk
  float *scale_m = nullptr, *scale_v = nullptr, *amax_m = nullptr, *amax_v = nullptr;
  TensorDesc* d_tensors = nullptr;
  Chunk* d_chunks = nullptr;
  ChunkDesc* d_cdesc = nullptr;  // the chunk table with each chunk's tensor buffers (staged step)
  // options of fp8adam_create_ex
  int32_t margin_m = 0, margin_v = 0, hist_len = 0;
  float *hist_m = nullptr, *hist_v = nullptr;
  uint64_t seed = 0;
  uint16_t** d_bf16 = nullptr;  // device [T] bf16 outputs, or null
  uint32_t* d_sr_ids = nullptr; // device [T] SR counter words of the tensors, or null (their indices)
  bool ext = false;             // any option on: the variant kernels run
  bool tma = false;             // default step through the TMA-staged kernel
  uint32_t* d_error = nullptr;  // device error word (bounded waits that ran out)
  // gradient pre-pass of fp8adam_step_ex: [chunks] partials, non-finite
  // count, multiplier, skip flag, norm
  double* d_partial = nullptr;
  unsigned long long* d_nonfinite = nullptr;
  float* d_grad_mult = nullptr;
  uint32_t* d_skip = nullptr;
  double* d_norm = nullptr;
  uint32_t* d_state = nullptr;  // [5T]: acc_m, acc_v, jit_m, jit_v, done
  unsigned long long* d_stats = nullptr;
  // fp8adam_step_host: each tensor's device gradient buffer and size, and
  // the tensor groups (cut at tensor boundaries, about equal in elements)
  // whose steps overlap the copies of the groups after them
  std::vector<uint16_t*> grad_dev;    // [T]
  std::vector<int64_t> numel;         // [T]
  std::vector<int32_t> grp_tensor;    // [G+1] first tensor of each group
  std::vector<int32_t> grp_chunk;     // [G+1] first chunk of each group
  cudaStream_t copy_stream = nullptr; // created on first use
  // fp8adam_set_schedule / fp8adam_step_scheduled: the entries of steps
  // sched_first .. sched_first + sched_count - 1, the device step counter and
  // the entry of the step in flight
  SchedEntry* d_sched = nullptr;
  int32_t sched_cap = 0, sched_count = 0;
  int64_t sched_first = 0;
  bool sched_prepass = false;         // some entry needs the grad-norm pre-pass
  int64_t* d_next_step = nullptr;
  SchedEntry* d_cur = nullptr;
  cudaEvent_t start_event = nullptr;
  std::vector<cudaEvent_t> grp_event; // [G] the group's copies are done
};

static void free_ctx(fp8adam_ctx* c) {
  if (!c) return;
  cudaFree(c->d_tensors);
  cudaFree(c->d_chunks);
  cudaFree(c->d_cdesc);
  cudaFree(c->d_error);
  cudaFree(c->d_bf16);
  cudaFree(c->d_sr_ids);
  cudaFree(c->d_partial);
  cudaFree(c->d_nonfinite);
  cudaFree(c->d_grad_mult);
  cudaFree(c->d_skip);
  cudaFree(c->d_norm);
  cudaFree(c->d_state);
  cudaFree(c->d_stats);
  cudaFree(c->d_sched);
  cudaFree(c->d_next_step);
  cudaFree(c->d_cur);
  for (cudaEvent_t e : c->grp_event)
    if (e) cudaEventDestroy(e);
  if (c->start_event) cudaEventDestroy(c->start_event);
  if (c->copy_stream) cudaStreamDestroy(c->copy_stream);
  delete c;
}

extern "C" int fp8adam_create(const fp8adam_tensor* tensors, int32_t num_tensors, float* scale_m,
                              float* scale_v, float* amax_m, float* amax_v, int32_t m_fmt,
                              int32_t v_fmt, uint32_t flags, fp8adam_ctx** out) {
  if (!out) return FP8ADAM_ERR_INVALID_ARG;
  *out = nullptr;
  if (flags & ~(FP8ADAM_FLAG_STATS | FP8ADAM_FLAG_JIT_EVERY_STEP | FP8ADAM_FLAG_NO_TMA))
    return FP8ADAM_ERR_INVALID_ARG;
  fp8adam_options o;
  std::memset(&o, 0, sizeof(o));
  o.scale_m = scale_m;
  o.scale_v = scale_v;
  o.amax_m = amax_m;
  o.amax_v = amax_v;
  o.m_fmt = m_fmt;
  o.v_fmt = v_fmt;
  o.flags = flags;
  return fp8adam_create_ex(tensors, num_tensors, &o, out);
}

extern "C" int fp8adam_create_ex(const fp8adam_tensor* tensors, int32_t num_tensors, const fp8adam_options* opts,
                                 fp8adam_ctx** out) {
  if (!out) return FP8ADAM_ERR_INVALID_ARG;
  *out = nullptr;
  if (!opts) return FP8ADAM_ERR_INVALID_ARG;
  float *scale_m = opts->scale_m, *scale_v = opts->scale_v, *amax_m = opts->amax_m, *amax_v = opts->amax_v;
  const int32_t m_fmt = opts->m_fmt, v_fmt = opts->v_fmt;
  const uint32_t flags = opts->flags;
  if (!tensors || num_tensors < 1 || !scale_m || !scale_v || !amax_m || !amax_v)
    return FP8ADAM_ERR_INVALID_ARG;
  if (m_fmt < 0 || m_fmt > 2 || v_fmt < 0 || v_fmt > 2) return FP8ADAM_ERR_UNSUPPORTED_FMT;
  if (flags & ~(FP8ADAM_FLAG_STATS | FP8ADAM_FLAG_JIT_EVERY_STEP | FP8ADAM_FLAG_UPDATE_FROM_STORED |
                FP8ADAM_FLAG_STOCHASTIC_ROUNDING | FP8ADAM_FLAG_NO_TMA | FP8ADAM_FLAG_SR_DRAW16))
    return FP8ADAM_ERR_INVALID_ARG;
  if ((flags & FP8ADAM_FLAG_SR_DRAW16) && !(flags & FP8ADAM_FLAG_STOCHASTIC_ROUNDING))
    return FP8ADAM_ERR_INVALID_ARG;
  if (opts->chunk_elems < 0 || opts->chunk_elems > kChunk || opts->chunk_elems % kTile != 0)
    return FP8ADAM_ERR_INVALID_ARG;
  if (opts->margin_m < 0 || opts->margin_m > 64 || opts->margin_v < 0 || opts->margin_v > 64 ||
      opts->amax_history_len < 0 || opts->amax_history_len > 1024 ||
      (opts->amax_history_len > 1 && (!opts->amax_history_m || !opts->amax_history_v)))
    return FP8ADAM_ERR_INVALID_ARG;

  for (int32_t i = 0; i < num_tensors; ++i) {
    const fp8adam_tensor& t = tensors[i];
    // 2^48 elements bounds every size and byte offset computed below far from overflow
    if (t.numel < 0 || t.numel > ((int64_t)1 << 48)) return FP8ADAM_ERR_INVALID_ARG;
    if (t.numel > 0 && (!t.param || !t.grad || !t.m || !t.v)) return FP8ADAM_ERR_INVALID_ARG;
  }
  // no written buffer (p, m, v, the bf16 copy) may overlap any other buffer
  try {
    std::vector<ByteRange> ranges;
    ranges.reserve((size_t)num_tensors * 5);
    const size_t mb = m_fmt == FP8ADAM_FP32 ? 4 : 1, vb = v_fmt == FP8ADAM_FP32 ? 4 : 1;
    for (int32_t i = 0; i < num_tensors; ++i) {
      const fp8adam_tensor& t = tensors[i];
      if (t.numel == 0) continue;
      const size_t n = (size_t)t.numel;
      auto add = [&](const void* p, size_t bytes, bool w) {
        ranges.push_back(ByteRange{(uintptr_t)p, (uintptr_t)p + bytes, w});
      };
      add(t.param, 4 * n, true);
      add(t.grad, 2 * n, false);
      add(t.m, mb * n, true);
      add(t.v, vb * n, true);
      if (opts->param_bf16 && opts->param_bf16[i]) add(opts->param_bf16[i], 2 * n, true);
    }
    if (written_range_overlaps(ranges)) return FP8ADAM_ERR_OVERLAP;
  } catch (...) {
    return FP8ADAM_ERR_OOM;
  }
  int dev = -1, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return FP8ADAM_ERR_CUDA;
  }
  // The chunk table: one CTA per chunk, chunks in launch order.  With
  // chunk_elems set, every chunk has that length (a tensor's last may be
  // shorter).  Otherwise the lengths are guided by the work still to come:
  // each chunk takes the remaining elements / (kGuidedRounds x resident
  // CTAs), rounded down to a whole tile, within [kGuidedMin, kChunk]
  // (kGuidedRounds 1, 2, 4 and kGuidedMin 4096, 8192 were timed: 1 and 8192
  // are best on the 100M, 7B and 20K-tensor layouts).  Long
  // chunks early keep the per-CTA set-up and amax flush rare; the shrinking
  // chunks at the end of the table leave only a short last wave.  A chunk
  // never crosses a multiple of 2^33 elements of its tensor (the stochastic-
  // rounding counter's high word is then constant within a chunk).
  int64_t total_elems_all = 0;
  for (int32_t i = 0; i < num_tensors; ++i) total_elems_all += tensors[i].numel;
  const int64_t slots = (int64_t)sms * 4;  // resident CTAs of the step kernels
  // a list that does not fill one wave of kGuidedMin chunks (a latency case)
  // gets one-tile chunks, for the most CTAs
  const int64_t guided_min = total_elems_all < slots * kGuidedMin ? kTile : kGuidedMin;
  std::vector<TensorDesc> desc;
  std::vector<Chunk> chunks;
  try {
    desc.resize((size_t)num_tensors);
    int64_t remaining = total_elems_all;
    for (int32_t i = 0; i < num_tensors; ++i) {
      const fp8adam_tensor& t = tensors[i];
      TensorDesc& d = desc[(size_t)i];
      d.p = t.param;
      d.g = t.grad;
      d.m = t.m;
      d.v = t.v;
      d.numel = t.numel;
      d.aligned = aligned16(t.param) && aligned16(t.grad) && aligned16(t.m) && aligned16(t.v);
      int32_t units = 0;
      for (int64_t st = 0; st < t.numel;) {
        int64_t len = opts->chunk_elems;
        if (len == 0) {
          len = remaining / (kGuidedRounds * slots) / kTile * kTile;
          len = len < guided_min ? guided_min : (len > kChunk ? kChunk : len);
        }
        const int64_t to_end = t.numel - st;
        const int64_t to_boundary = (st / kCounterSpan + 1) * kCounterSpan - st;
        len = std::min(len, std::min(to_end, to_boundary));
        chunks.push_back(Chunk{i, (int32_t)len, st});
        st += len;
        remaining -= len;
        ++units;
        if (chunks.size() > (size_t)INT32_MAX / 2) return FP8ADAM_ERR_INVALID_ARG;
      }
      d.nunits = units;
    }
  } catch (...) {
    return FP8ADAM_ERR_OOM;
  }
  const int64_t total_units = (int64_t)chunks.size();
  const int64_t chunk = opts->chunk_elems;  // 0: guided lengths

  fp8adam_ctx* c = new (std::nothrow) fp8adam_ctx();
  if (!c) return FP8ADAM_ERR_OOM;
  try {
    c->grad_dev.resize((size_t)num_tensors);
    c->numel.resize((size_t)num_tensors);
    int64_t total_elems = 0;
    for (int32_t i = 0; i < num_tensors; ++i) {
      c->grad_dev[(size_t)i] = const_cast<uint16_t*>(tensors[i].grad);
      c->numel[(size_t)i] = tensors[i].numel;
      total_elems += tensors[i].numel;
    }
    // groups for fp8adam_step_host: up to kHostGroups, cut after the tensor
    // that reaches the next equal share of the elements
    constexpr int kHostGroups = 8;
    c->grp_tensor.push_back(0);
    c->grp_chunk.push_back(0);
    int64_t cum = 0, cum_chunks = 0;
    for (int32_t i = 0; i < num_tensors; ++i) {
      cum += tensors[i].numel;
      cum_chunks += desc[(size_t)i].nunits;
      const int g = (int)c->grp_tensor.size();  // groups closed so far + 1
      if (i + 1 == num_tensors || (g < kHostGroups && cum * kHostGroups >= total_elems * g)) {
        c->grp_tensor.push_back(i + 1);
        c->grp_chunk.push_back((int32_t)cum_chunks);
      }
    }
  } catch (...) {
    delete c;
    return FP8ADAM_ERR_OOM;
  }
  c->device = dev;
  c->chunk_elems = (int32_t)chunk;
  c->T = num_tensors;
  c->m_fmt = m_fmt;
  c->v_fmt = v_fmt;
  c->flags = flags;
  c->total_units = (int32_t)total_units;
  c->scale_m = scale_m;
  c->scale_v = scale_v;
  c->amax_m = amax_m;
  c->amax_v = amax_v;
  c->margin_m = opts->margin_m;
  c->margin_v = opts->margin_v;
  c->hist_len = opts->amax_history_len > 1 ? opts->amax_history_len : 0;
  c->hist_m = c->hist_len ? opts->amax_history_m : nullptr;
  c->hist_v = c->hist_len ? opts->amax_history_v : nullptr;
  c->seed = opts->seed;
  c->ext = (flags & (FP8ADAM_FLAG_UPDATE_FROM_STORED | FP8ADAM_FLAG_STOCHASTIC_ROUNDING)) || c->margin_m ||
           c->margin_v || c->hist_len || opts->param_bf16;
  const size_t T = (size_t)num_tensors;
  if (cudaMalloc(&c->d_tensors, T * sizeof(TensorDesc)) != cudaSuccess ||
      cudaMalloc(&c->d_chunks, (chunks.empty() ? 1 : chunks.size()) * sizeof(Chunk)) != cudaSuccess ||
      cudaMalloc(&c->d_state, 5 * T * sizeof(uint32_t)) != cudaSuccess ||
      cudaMalloc(&c->d_stats, 2 * sizeof(unsigned long long)) != cudaSuccess) {
    cudaGetLastError();
    free_ctx(c);
    return FP8ADAM_ERR_OOM;
  }
  std::vector<ChunkDesc> cdesc;
  try {
    cdesc.resize(chunks.size());
  } catch (...) {
    free_ctx(c);
    return FP8ADAM_ERR_OOM;
  }
  for (size_t k = 0; k < chunks.size(); ++k) {
    const TensorDesc& d = desc[(size_t)chunks[k].tensor];
    cdesc[k] = ChunkDesc{d.p, d.g, d.m, d.v, chunks[k].start, d.numel, chunks[k].len, chunks[k].tensor,
                         d.nunits, d.aligned};
  }
  if (cudaMalloc(&c->d_cdesc, (cdesc.empty() ? 1 : cdesc.size()) * sizeof(ChunkDesc)) != cudaSuccess) {
    cudaGetLastError();
    free_ctx(c);
    return FP8ADAM_ERR_OOM;
  }
  if ((!cdesc.empty() && cudaMemcpy(c->d_cdesc, cdesc.data(), cdesc.size() * sizeof(ChunkDesc),
                                    cudaMemcpyHostToDevice) != cudaSuccess) ||
      cudaMemcpy(c->d_tensors, desc.data(), T * sizeof(TensorDesc), cudaMemcpyHostToDevice) != cudaSuccess ||
      (!chunks.empty() &&
       cudaMemcpy(c->d_chunks, chunks.data(), chunks.size() * sizeof(Chunk), cudaMemcpyHostToDevice) != cudaSuccess) ||
      cudaMemset(c->d_state, 0, 5 * T * sizeof(uint32_t)) != cudaSuccess ||
      cudaMemset(c->d_stats, 0, 2 * sizeof(unsigned long long)) != cudaSuccess ||
      cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    free_ctx(c);
    return FP8ADAM_ERR_CUDA;
  }
  // gradient pre-pass buffers (partials over the step grid) and options
  if (cudaMalloc(&c->d_partial, (size_t)(c->total_units > 0 ? c->total_units : 1) * sizeof(double)) != cudaSuccess ||
      cudaMalloc(&c->d_nonfinite, sizeof(unsigned long long)) != cudaSuccess ||
      cudaMalloc(&c->d_grad_mult, sizeof(float)) != cudaSuccess ||
      cudaMalloc(&c->d_skip, sizeof(uint32_t)) != cudaSuccess ||
      cudaMalloc(&c->d_norm, sizeof(double)) != cudaSuccess ||
      cudaMalloc(&c->d_error, sizeof(uint32_t)) != cudaSuccess ||
      (opts->param_bf16 && cudaMalloc(&c->d_bf16, T * sizeof(uint16_t*)) != cudaSuccess) ||
      (opts->sr_counter_ids && cudaMalloc(&c->d_sr_ids, T * sizeof(uint32_t)) != cudaSuccess)) {
    cudaGetLastError();
    free_ctx(c);
    return FP8ADAM_ERR_OOM;
  }
  c->tma = m_fmt != FP8ADAM_FP32 && v_fmt != FP8ADAM_FP32 && !(flags & FP8ADAM_FLAG_NO_TMA);
  const bool stats_on = (flags & FP8ADAM_FLAG_STATS) != 0;
  const int srk = sr_kind_of(flags);
  if (c->tma && (cudaFuncSetAttribute((const void*)pick_tma(m_fmt, v_fmt, stats_on),
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, kTmaSmemBytes) != cudaSuccess ||
                 cudaFuncSetAttribute((const void*)pick_ext_tma(m_fmt, v_fmt, stats_on, srk),
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, kTmaSmemBytes) != cudaSuccess ||
                 (srk && cudaFuncSetAttribute((const void*)pick_ext_tma_sr_lean(m_fmt, v_fmt, stats_on, srk),
                                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              kTmaSmemBytes) != cudaSuccess))) {
    cudaGetLastError();
    free_ctx(c);
    return FP8ADAM_ERR_CUDA;
  }
  if (cudaMemset(c->d_skip, 0, sizeof(uint32_t)) != cudaSuccess ||
      cudaMemset(c->d_error, 0, sizeof(uint32_t)) != cudaSuccess ||
      cudaMemset(c->d_norm, 0, sizeof(double)) != cudaSuccess ||
      (opts->param_bf16 &&
       cudaMemcpy(c->d_bf16, opts->param_bf16, T * sizeof(uint16_t*), cudaMemcpyHostToDevice) != cudaSuccess) ||
      (opts->sr_counter_ids &&
       cudaMemcpy(c->d_sr_ids, opts->sr_counter_ids, T * sizeof(uint32_t), cudaMemcpyHostToDevice) != cudaSuccess) ||
      cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    free_ctx(c);
    return FP8ADAM_ERR_CUDA;
  }
  *out = c;
  return FP8ADAM_OK;
}

static bool valid_hparams(float lr, float beta1, float beta2, float eps, float weight_decay, int64_t step) {
  return step >= 1 && std::isfinite(lr) && std::isfinite(weight_decay) && beta1 >= 0.0f && beta1 < 1.0f &&
         beta2 >= 0.0f && beta2 < 1.0f && eps >= 0.0f && std::isfinite(eps);
}

// The grad-norm pre-pass is needed for clipping (the global norm) and for
// skip-on-non-finite (the non-finite count).  A loss scale alone is a
// constant multiplier, 1/loss_scale, computed on the host as the pre-pass's
// finalize kernel computes it without clipping (double, rounded once).
static bool needs_prepass(const fp8adam_step_params& p) {
  return p.max_norm > 0.0f || p.skip_nonfinite != 0;
}
static float host_multiplier(const fp8adam_step_params& p) {
  return (float)(1.0 / (double)p.loss_scale);
}

// The step over chunks [c0, c1) of the chunk table: every chunk of the
// tensors in that range (ranges start and end at tensor boundaries).
// `first`: the range is the step's first, so the JIT accumulators are
// cleared before it.  The grad-norm pre-pass needs all gradients: with it
// the range is the whole table.
// `cur` (a scheduled step): the kernels take the constants and per-step
// options from that device entry instead of `p`; whether the pre-passes run
// is then decided per schedule (grad norm) or per context (JIT amax).
// `pdl`: launch the staged step kernel (default or options) with
// programmatic dependent launch (the steps of fp8adam_step /
// fp8adam_step_ex, back to back on a stream).
static int run_step_range(fp8adam_ctx* ctx, const fp8adam_step_params& p, cudaStream_t st, int32_t c0, int32_t c1,
                          bool first, const SchedEntry* cur = nullptr, bool pdl = false) {
  if (c1 <= c0) return FP8ADAM_OK;  // only empty tensors
  const bool prepass = cur ? ctx->sched_prepass : needs_prepass(p);
  const bool ext = ctx->ext || prepass || (!cur && p.loss_scale != 1.0f);

  StepArgs a;
  a.c = make_consts(p);
  a.cur = cur;

  const size_t T = (size_t)ctx->T;
  uint32_t* acc_m = ctx->d_state;
  uint32_t* acc_v = ctx->d_state + T;
  uint32_t* jit_m = ctx->d_state + 2 * T;
  uint32_t* jit_v = ctx->d_state + 3 * T;
  a.tensors = ctx->d_tensors;
  a.chunks = ctx->d_chunks + c0;
  a.cdesc = ctx->d_cdesc + c0;
  a.num_tensors = ctx->T;
  a.scale_m = ctx->scale_m;
  a.scale_v = ctx->scale_v;
  a.amax_m = ctx->amax_m;
  a.amax_v = ctx->amax_v;
  a.done = ctx->d_state + 4 * T;
  a.stats = ctx->d_stats;
  a.acc_m = acc_m;
  a.acc_v = acc_v;

  const dim3 block(kThreads), grid((unsigned)(c1 - c0));
  const bool jit = (!cur && p.step == 1) || (ctx->flags & FP8ADAM_FLAG_JIT_EVERY_STEP);
  const bool stats = (ctx->flags & FP8ADAM_FLAG_STATS) != 0;
  if (!ext) {
    if (jit) {
      if (first && cudaMemsetAsync(jit_m, 0, 2 * T * sizeof(uint32_t), st) != cudaSuccess) return FP8ADAM_ERR_CUDA;
      StepArgs pre = a;
      pre.acc_m = jit_m;
      pre.acc_v = jit_v;
      pre.amax_in_m = nullptr;
      pre.amax_in_v = nullptr;
      pick_amax(ctx->m_fmt, ctx->v_fmt)<<<grid, block, 0, st>>>(pre);
      g_launches.fetch_add(1, std::memory_order_relaxed);
      a.amax_in_m = jit_m;
      a.amax_in_v = jit_v;
    } else {
      a.amax_in_m = reinterpret_cast<const uint32_t*>(ctx->amax_m);
      a.amax_in_v = reinterpret_cast<const uint32_t*>(ctx->amax_v);
    }
    if (ctx->tma && pdl) {
      if (launch_staged_pdl(pick_tma(ctx->m_fmt, ctx->v_fmt, stats), grid, block, st, a, ctx->d_error) !=
          cudaSuccess) {
        cudaGetLastError();
        return FP8ADAM_ERR_CUDA;
      }
    } else if (ctx->tma)
      pick_tma(ctx->m_fmt, ctx->v_fmt, stats)<<<grid, block, kTmaSmemBytes, st>>>(a, ctx->d_error);
    else
      pick_step(ctx->m_fmt, ctx->v_fmt, stats)<<<grid, block, 0, st>>>(a);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return last_error();
  }

  ExtArgs e;
  e.flags = ctx->flags & (FP8ADAM_FLAG_UPDATE_FROM_STORED | FP8ADAM_FLAG_STOCHASTIC_ROUNDING | FP8ADAM_FLAG_SR_DRAW16);
  e.margin_m = ctx->margin_m;
  e.margin_v = ctx->margin_v;
  e.use_hist = (ctx->hist_len > 1 && !jit) ? 1 : 0;
  e.hist_len = ctx->hist_len;
  e.hist_slot = ctx->hist_len ? (int32_t)((p.step - 1) % ctx->hist_len) : 0;
  e.hist_m = ctx->hist_m;
  e.hist_v = ctx->hist_v;
  for (int r = 0; r < 10; ++r) {  // Philox4x32-10 key schedule (Weyl increments)
    e.sr_key[r][0] = (uint32_t)ctx->seed + (uint32_t)r * 0x9E3779B9u;
    e.sr_key[r][1] = (uint32_t)(ctx->seed >> 32) + (uint32_t)r * 0xBB67AE85u;
  }
  e.t_lo = (uint32_t)p.step;
  e.gm_const = cur ? 1.0f : host_multiplier(p);
  e.grad_mult = nullptr;
  e.skip = nullptr;
  e.p_bf16 = ctx->d_bf16;
  e.sr_ids = (ctx->flags & FP8ADAM_FLAG_STOCHASTIC_ROUNDING) ? ctx->d_sr_ids : nullptr;
  if (prepass) {
    NvtxRange pre("fp8adam grad-norm pre-pass");
    if (cudaMemsetAsync(ctx->d_nonfinite, 0, sizeof(unsigned long long), st) != cudaSuccess)
      return FP8ADAM_ERR_CUDA;
    fp8adam_gradnorm_partial_kernel<<<grid, block, 0, st>>>(a, ctx->d_partial, ctx->d_nonfinite);
    fp8adam_gradnorm_finalize_kernel<<<1, block, 0, st>>>(ctx->d_partial, (int)(c1 - c0), ctx->d_nonfinite,
                                                          p.loss_scale, p.max_norm, p.skip_nonfinite, cur,
                                                          ctx->d_grad_mult, ctx->d_skip, ctx->d_norm);
    g_launches.fetch_add(2, std::memory_order_relaxed);
    e.grad_mult = ctx->d_grad_mult;
    e.skip = ctx->d_skip;
  }
  if (jit) {
    if (first && cudaMemsetAsync(jit_m, 0, 2 * T * sizeof(uint32_t), st) != cudaSuccess) return FP8ADAM_ERR_CUDA;
    ExtArgs pre = e;
    pre.s = a;
    pre.s.acc_m = jit_m;
    pre.s.acc_v = jit_v;
    pre.s.amax_in_m = nullptr;
    pre.s.amax_in_v = nullptr;
    pick_amax_ext(ctx->m_fmt, ctx->v_fmt)<<<grid, block, 0, st>>>(pre);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    a.amax_in_m = jit_m;
    a.amax_in_v = jit_v;
  } else {
    a.amax_in_m = reinterpret_cast<const uint32_t*>(ctx->amax_m);
    a.amax_in_v = reinterpret_cast<const uint32_t*>(ctx->amax_v);
  }
  e.s = a;
  const int srk = sr_kind_of(e.flags);
  if (ctx->tma) {
    const bool lean = srk && !(e.flags & FP8ADAM_FLAG_UPDATE_FROM_STORED) && !ctx->d_bf16 && e.grad_mult == nullptr &&
                      e.gm_const == 1.0f;
    const ExtTmaFn fn = lean ? pick_ext_tma_sr_lean(ctx->m_fmt, ctx->v_fmt, stats, srk)
                             : pick_ext_tma(ctx->m_fmt, ctx->v_fmt, stats, srk);
    if (pdl) {
      if (launch_staged_pdl(fn, grid, block, st, e, ctx->d_error) != cudaSuccess) {
        cudaGetLastError();
        return FP8ADAM_ERR_CUDA;
      }
    } else {
      fn<<<grid, block, kTmaSmemBytes, st>>>(e, ctx->d_error);
    }
  } else
    pick_ext(ctx->m_fmt, ctx->v_fmt, stats)<<<grid, block, 0, st>>>(e);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return last_error();
}

static int run_step(fp8adam_ctx* ctx, const fp8adam_step_params& p, cudaStream_t st) {
  NvtxRange range("fp8adam_step");
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FP8ADAM_ERR_CUDA;
  if (dev != ctx->device) return FP8ADAM_ERR_WRONG_DEVICE;
  return run_step_range(ctx, p, st, 0, ctx->total_units, true, nullptr, true);
}

extern "C" int fp8adam_step(fp8adam_ctx* ctx, float lr, float beta1, float beta2, float eps,
                            float weight_decay, int64_t step, void* cuda_stream) {
  if (!ctx) return FP8ADAM_ERR_INVALID_ARG;
  if (!valid_hparams(lr, beta1, beta2, eps, weight_decay, step)) return FP8ADAM_ERR_INVALID_ARG;
  fp8adam_step_params p;
  p.lr = lr;
  p.beta1 = beta1;
  p.beta2 = beta2;
  p.eps = eps;
  p.weight_decay = weight_decay;
  p.step = step;
  p.loss_scale = 1.0f;
  p.max_norm = 0.0f;
  p.skip_nonfinite = 0;
  return run_step(ctx, p, static_cast<cudaStream_t>(cuda_stream));
}

extern "C" int fp8adam_step_ex(fp8adam_ctx* ctx, const fp8adam_step_params* params, void* cuda_stream) {
  if (!ctx || !params) return FP8ADAM_ERR_INVALID_ARG;
  const fp8adam_step_params& p = *params;
  if (!valid_hparams(p.lr, p.beta1, p.beta2, p.eps, p.weight_decay, p.step)) return FP8ADAM_ERR_INVALID_ARG;
  if (!(p.loss_scale > 0.0f) || !std::isfinite(p.loss_scale) || std::isnan(p.max_norm) ||
      std::isinf(p.max_norm))
    return FP8ADAM_ERR_INVALID_ARG;
  return run_step(ctx, p, static_cast<cudaStream_t>(cuda_stream));
}

static bool valid_step_params(const fp8adam_step_params& p) {
  return valid_hparams(p.lr, p.beta1, p.beta2, p.eps, p.weight_decay, p.step) && p.loss_scale > 0.0f &&
         std::isfinite(p.loss_scale) && !std::isnan(p.max_norm) && !std::isinf(p.max_norm);
}

extern "C" int fp8adam_set_schedule(fp8adam_ctx* ctx, const fp8adam_step_params* steps, int32_t count,
                                    void* cuda_stream) {
  if (!ctx || !steps || count < 1) return FP8ADAM_ERR_INVALID_ARG;
  const int64_t first = steps[0].step;
  // step 1 takes the amax pre-pass decided on the host, so a schedule starts
  // after it unless every step has the pre-pass (current scaling)
  if (first < 2 && !(ctx->flags & FP8ADAM_FLAG_JIT_EVERY_STEP)) return FP8ADAM_ERR_INVALID_ARG;
  std::vector<SchedEntry> host;
  try {
    host.resize((size_t)count);
  } catch (...) {
    return FP8ADAM_ERR_OOM;
  }
  bool prepass = false;
  for (int32_t k = 0; k < count; ++k) {
    const fp8adam_step_params& p = steps[k];
    if (!valid_step_params(p) || p.step != first + k) return FP8ADAM_ERR_INVALID_ARG;
    SchedEntry& e = host[(size_t)k];
    e.c = make_consts(p);
    e.loss_scale = p.loss_scale;
    e.max_norm = p.max_norm;
    e.skip_nonfinite = p.skip_nonfinite ? 1 : 0;
    e.t_lo = (uint32_t)p.step;
    e.hist_slot = ctx->hist_len ? (int32_t)((p.step - 1) % ctx->hist_len) : 0;
    e.valid = 1;
    // a scheduled step reads its loss scale from the entry, so any scale
    // other than 1 takes the pre-pass (whose finalize kernel reads it)
    prepass = prepass || needs_prepass(p) || p.loss_scale != 1.0f;
  }
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FP8ADAM_ERR_CUDA;
  if (dev != ctx->device) return FP8ADAM_ERR_WRONG_DEVICE;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  // the steps already queued may still read the old schedule
  if (cudaStreamSynchronize(st) != cudaSuccess) return FP8ADAM_ERR_CUDA;
  if (count > ctx->sched_cap) {
    cudaFree(ctx->d_sched);
    ctx->d_sched = nullptr;
    ctx->sched_cap = 0;
    if (cudaMalloc(&ctx->d_sched, (size_t)count * sizeof(SchedEntry)) != cudaSuccess) {
      cudaGetLastError();
      return FP8ADAM_ERR_OOM;
    }
    ctx->sched_cap = count;
  }
  if ((!ctx->d_next_step && cudaMalloc(&ctx->d_next_step, sizeof(int64_t)) != cudaSuccess) ||
      (!ctx->d_cur && cudaMalloc(&ctx->d_cur, sizeof(SchedEntry)) != cudaSuccess)) {
    cudaGetLastError();
    return FP8ADAM_ERR_OOM;
  }
  if (cudaMemcpy(ctx->d_sched, host.data(), (size_t)count * sizeof(SchedEntry), cudaMemcpyHostToDevice) !=
          cudaSuccess ||
      cudaMemcpy(ctx->d_next_step, &first, sizeof(first), cudaMemcpyHostToDevice) != cudaSuccess)
    return FP8ADAM_ERR_CUDA;
  ctx->sched_first = first;
  ctx->sched_count = count;
  ctx->sched_prepass = prepass;
  return FP8ADAM_OK;
}

extern "C" int fp8adam_step_scheduled(fp8adam_ctx* ctx, void* cuda_stream) {
  if (!ctx || ctx->sched_count == 0) return FP8ADAM_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FP8ADAM_ERR_CUDA;
  if (dev != ctx->device) return FP8ADAM_ERR_WRONG_DEVICE;
  if (ctx->total_units == 0) return FP8ADAM_OK;
  NvtxRange range("fp8adam_step_scheduled");
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  sched_select_kernel<<<1, 1, 0, st>>>(ctx->d_sched, ctx->sched_first, ctx->sched_count, ctx->d_next_step,
                                       ctx->d_cur, ctx->d_error);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  // the host-side parameters only fill the unused kernel arguments
  fp8adam_step_params p;
  std::memset(&p, 0, sizeof(p));
  p.lr = 0.0f;
  p.beta1 = p.beta2 = 0.5f;
  p.step = 2;
  p.loss_scale = 1.0f;
  return run_step_range(ctx, p, st, 0, ctx->total_units, true, ctx->d_cur);
}

extern "C" int fp8adam_get_schedule_step(fp8adam_ctx* ctx, int64_t* next_step, void* cuda_stream) {
  if (!ctx || !next_step || !ctx->d_next_step) return FP8ADAM_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  if (cudaMemcpyAsync(next_step, ctx->d_next_step, sizeof(int64_t), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return FP8ADAM_ERR_CUDA;
  return FP8ADAM_OK;
}

extern "C" int fp8adam_step_host(fp8adam_ctx* ctx, const fp8adam_step_params* params,
                                 const uint16_t* const* host_grads, float* amax_host, void* cuda_stream) {
  if (!ctx || !params || !host_grads) return FP8ADAM_ERR_INVALID_ARG;
  const fp8adam_step_params& p = *params;
  if (!valid_hparams(p.lr, p.beta1, p.beta2, p.eps, p.weight_decay, p.step)) return FP8ADAM_ERR_INVALID_ARG;
  if (!(p.loss_scale > 0.0f) || !std::isfinite(p.loss_scale) || std::isnan(p.max_norm) ||
      std::isinf(p.max_norm))
    return FP8ADAM_ERR_INVALID_ARG;
  for (int32_t i = 0; i < ctx->T; ++i)
    if (ctx->numel[(size_t)i] > 0 && !host_grads[i]) return FP8ADAM_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FP8ADAM_ERR_CUDA;
  if (dev != ctx->device) return FP8ADAM_ERR_WRONG_DEVICE;
  const int G = (int)ctx->grp_tensor.size() - 1;
  if (!ctx->copy_stream) {  // first use: the copy stream and its events
    if (cudaStreamCreateWithFlags(&ctx->copy_stream, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&ctx->start_event, cudaEventDisableTiming) != cudaSuccess) {
      cudaGetLastError();
      return FP8ADAM_ERR_CUDA;
    }
    try {
      ctx->grp_event.assign((size_t)G, nullptr);
    } catch (...) {
      return FP8ADAM_ERR_OOM;
    }
    for (int g = 0; g < G; ++g)
      if (cudaEventCreateWithFlags(&ctx->grp_event[(size_t)g], cudaEventDisableTiming) != cudaSuccess) {
        cudaGetLastError();
        return FP8ADAM_ERR_CUDA;
      }
  }
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  // the copies wait for the work already queued on the step's stream (the
  // previous step may still read the gradient buffers)
  if (cudaEventRecord(ctx->start_event, st) != cudaSuccess ||
      cudaStreamWaitEvent(ctx->copy_stream, ctx->start_event, 0) != cudaSuccess)
    return FP8ADAM_ERR_CUDA;
  // with the grad-norm pre-pass every gradient is needed before any update:
  // one group; otherwise group g's step waits only for group g's copies
  const bool whole = needs_prepass(p);
  const int ng = whole ? 1 : G;
  NvtxRange range("fp8adam_step_host");
  bool first = true;  // no chunk of this step has been launched yet (clears the JIT accumulators)
  for (int g = 0; g < ng; ++g) {
    const int32_t t0 = whole ? 0 : ctx->grp_tensor[(size_t)g];
    const int32_t t1 = whole ? ctx->T : ctx->grp_tensor[(size_t)g + 1];
    for (int32_t i = t0; i < t1; ++i) {
      const int64_t n = ctx->numel[(size_t)i];
      if (n > 0 && cudaMemcpyAsync(ctx->grad_dev[(size_t)i], host_grads[i], (size_t)n * sizeof(uint16_t),
                                   cudaMemcpyHostToDevice, ctx->copy_stream) != cudaSuccess)
        return FP8ADAM_ERR_CUDA;
    }
    cudaEvent_t ev = ctx->grp_event[(size_t)g];
    if (cudaEventRecord(ev, ctx->copy_stream) != cudaSuccess || cudaStreamWaitEvent(st, ev, 0) != cudaSuccess)
      return FP8ADAM_ERR_CUDA;
    const int32_t c0 = whole ? 0 : ctx->grp_chunk[(size_t)g];
    const int32_t c1 = whole ? ctx->total_units : ctx->grp_chunk[(size_t)g + 1];
    const int rc = run_step_range(ctx, p, st, c0, c1, first);
    if (rc != FP8ADAM_OK) return rc;
    if (c1 > c0) first = false;
  }
  if (amax_host && ctx->T > 0) {
    const size_t bytes = (size_t)ctx->T * sizeof(float);
    if (cudaMemcpyAsync(amax_host, ctx->amax_m, bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaMemcpyAsync(amax_host + ctx->T, ctx->amax_v, bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
      return FP8ADAM_ERR_CUDA;
  }
  return last_error();
}

extern "C" int fp8adam_get_grad_info(fp8adam_ctx* ctx, double* grad_norm, uint32_t* skipped, void* cuda_stream) {
  if (!ctx || !grad_norm || !skipped) return FP8ADAM_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  double n = 0.0;
  uint32_t k = 0;
  if (cudaMemcpyAsync(&n, ctx->d_norm, sizeof(double), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemcpyAsync(&k, ctx->d_skip, sizeof(uint32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return FP8ADAM_ERR_CUDA;
  *grad_norm = n;
  *skipped = k;
  return FP8ADAM_OK;
}

extern "C" int fp8adam_get_stats(fp8adam_ctx* ctx, uint64_t* out, void* cuda_stream) {
  if (!ctx || !out) return FP8ADAM_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  unsigned long long h[2] = {0, 0};
  if (cudaMemcpyAsync(h, ctx->d_stats, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return FP8ADAM_ERR_CUDA;
  out[0] = h[0];
  out[1] = h[1];
  return FP8ADAM_OK;
}

extern "C" int fp8adam_reset_stats(fp8adam_ctx* ctx, void* cuda_stream) {
  if (!ctx) return FP8ADAM_ERR_INVALID_ARG;
  return cudaMemsetAsync(ctx->d_stats, 0, 2 * sizeof(unsigned long long),
                         static_cast<cudaStream_t>(cuda_stream)) == cudaSuccess
             ? FP8ADAM_OK
             : FP8ADAM_ERR_CUDA;
}

extern "C" int fp8adam_check(fp8adam_ctx* ctx, void* cuda_stream) {
  if (!ctx) return FP8ADAM_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  uint32_t e = 0, bounds = 0;
  if (cudaMemcpyAsync(&e, ctx->d_error, sizeof(e), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return FP8ADAM_ERR_CUDA;
#ifdef FP8ADAM_DEBUG
  if (cudaMemcpyFromSymbolAsync(&bounds, g_debug_flags, sizeof(bounds), 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return FP8ADAM_ERR_CUDA;
#endif
  if (cudaStreamSynchronize(st) != cudaSuccess) return FP8ADAM_ERR_CUDA;
  if (!e && !bounds) return FP8ADAM_OK;
  // A step stopped part-way: clear the error word and the per-step device
  // state (amax accumulators, JIT amax, chunk counters) so the next step
  // starts clean.  The elements of the failed step are partly updated.
  if (cudaMemsetAsync(ctx->d_state, 0, 5 * (size_t)ctx->T * sizeof(uint32_t), st) != cudaSuccess ||
      cudaMemsetAsync(ctx->d_error, 0, sizeof(uint32_t), st) != cudaSuccess)
    return FP8ADAM_ERR_CUDA;
#ifdef FP8ADAM_DEBUG
  const uint32_t zero = 0;
  if (cudaMemcpyToSymbolAsync(g_debug_flags, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return FP8ADAM_ERR_CUDA;
#endif
  if (cudaStreamSynchronize(st) != cudaSuccess) return FP8ADAM_ERR_CUDA;
  if (bounds) return FP8ADAM_ERR_DEBUG_BOUNDS;
  return (e & 1u) ? FP8ADAM_ERR_DEVICE_TIMEOUT : FP8ADAM_ERR_SCHEDULE_END;
}

extern "C" int fp8adam_debug_inject_wait(int32_t cta, int32_t subtile) {
#ifdef FP8ADAM_DEBUG
  if (cudaMemcpyToSymbol(g_inject_cta, &cta, sizeof(cta)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_inject_sub, &subtile, sizeof(subtile)) != cudaSuccess)
    return FP8ADAM_ERR_CUDA;
  return FP8ADAM_OK;
#else
  (void)cta;
  (void)subtile;
  return FP8ADAM_ERR_INVALID_ARG;  // the release build has no injection point
#endif
}

extern "C" int fp8adam_debug_set_numel(fp8adam_ctx* ctx, int32_t tensor, int64_t numel) {
#ifdef FP8ADAM_DEBUG
  if (!ctx || tensor < 0 || tensor >= ctx->T || numel < 0 || numel > ctx->numel[(size_t)tensor])
    return FP8ADAM_ERR_INVALID_ARG;
  if (cudaMemcpy(reinterpret_cast<char*>(ctx->d_tensors + tensor) + offsetof(TensorDesc, numel), &numel,
                 sizeof(numel), cudaMemcpyHostToDevice) != cudaSuccess)
    return FP8ADAM_ERR_CUDA;
  return FP8ADAM_OK;
#else
  (void)ctx;
  (void)tensor;
  (void)numel;
  return FP8ADAM_ERR_INVALID_ARG;
#endif
}

extern "C" int fp8adam_destroy(fp8adam_ctx* ctx) {
  if (!ctx) return FP8ADAM_OK;
  const int rc = cudaDeviceSynchronize() == cudaSuccess ? FP8ADAM_OK : FP8ADAM_ERR_CUDA;
  free_ctx(ctx);
  return rc;
}

extern "C" const char* fp8adam_strerror(int code) {
  switch (code) {
    case FP8ADAM_OK: return "ok";
    case FP8ADAM_ERR_INVALID_ARG: return "invalid argument";
    case FP8ADAM_ERR_UNSUPPORTED_FMT: return "unsupported moment format";
    case FP8ADAM_ERR_CUDA: return "CUDA runtime error";
    case FP8ADAM_ERR_DEBUG_BOUNDS: return "a kernel access outside its tensor was skipped (debug build)";
    case FP8ADAM_ERR_OVERLAP: return "a written buffer (param, m, v or bf16 copy) overlaps another buffer";
    case FP8ADAM_ERR_SCHEDULE_END: return "a scheduled step ran past the end of its schedule (nothing was updated)";
    case FP8ADAM_ERR_OOM: return "device allocation failed";
    case FP8ADAM_ERR_WRONG_DEVICE: return "current device differs from the context's";
    case FP8ADAM_ERR_NOALLOC_LIMIT: return "more tensors than the allocation-free step holds (FP8ADAM_NOALLOC_MAX_TENSORS)";
    case FP8ADAM_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait for its copies ran out; the state is not usable";
    default: return "unknown error";
  }
}

// ------------------------------------------------------------ codec API
#define FP8ADAM_CODEC_DISPATCH(KERNEL, GRID, ...)                                  \
  do {                                                                             \
    if (fmt == 0 && impl == 0) KERNEL<0, 0><<<GRID, 256, 0, st>>>(__VA_ARGS__);    \
    else if (fmt == 0) KERNEL<0, 1><<<GRID, 256, 0, st>>>(__VA_ARGS__);            \
    else if (impl == 0) KERNEL<1, 0><<<GRID, 256, 0, st>>>(__VA_ARGS__);           \
    else KERNEL<1, 1><<<GRID, 256, 0, st>>>(__VA_ARGS__);                          \
    g_launches.fetch_add(1, std::memory_order_relaxed);                            \
  } while (0)

extern "C" int fp8adam_encode(int32_t fmt, const float* x, uint8_t* out, int64_t n, int32_t impl,
                              void* cuda_stream) {
  if (fmt < 0 || fmt > 1) return FP8ADAM_ERR_UNSUPPORTED_FMT;
  if (impl < 0 || impl > 1 || n < 0 || (n > 0 && (!x || !out))) return FP8ADAM_ERR_INVALID_ARG;
  if (n == 0) return FP8ADAM_OK;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  FP8ADAM_CODEC_DISPATCH(encode_kernel, grid_for(n, 4), x, out, n);
  return last_error();
}

extern "C" int fp8adam_encode_bits_range(int32_t fmt, uint32_t first, int64_t n, uint8_t* out,
                                         int32_t impl, void* cuda_stream) {
  if (fmt < 0 || fmt > 1) return FP8ADAM_ERR_UNSUPPORTED_FMT;
  if (impl < 0 || impl > 1 || n < 0 || (n > 0 && !out) || n > (int64_t)(1ull << 32) - (int64_t)first ||
      ((uintptr_t)out & 3u))
    return FP8ADAM_ERR_INVALID_ARG;
  if (n == 0) return FP8ADAM_OK;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  FP8ADAM_CODEC_DISPATCH(encode_bits_kernel, grid_for(n, 4), first, out, n);
  return last_error();
}

extern "C" int fp8adam_encode_sr(int32_t fmt, const float* x, const uint32_t* r, uint8_t* out, int64_t n,
                                 void* cuda_stream) {
  if (fmt < 0 || fmt > 1) return FP8ADAM_ERR_UNSUPPORTED_FMT;
  if (n < 0 || (n > 0 && (!x || !r || !out))) return FP8ADAM_ERR_INVALID_ARG;
  if (n == 0) return FP8ADAM_OK;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  if (fmt == 0) encode_sr_kernel<0><<<grid_for(n, 1), 256, 0, st>>>(x, r, out, n);
  else encode_sr_kernel<1><<<grid_for(n, 1), 256, 0, st>>>(x, r, out, n);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return last_error();
}

extern "C" int fp8adam_encode_sr16(int32_t fmt, const float* x, const uint32_t* w, uint8_t* out, int64_t n,
                                   void* cuda_stream) {
  if (fmt < 0 || fmt > 1) return FP8ADAM_ERR_UNSUPPORTED_FMT;
  if (n < 0 || (n > 0 && (!x || !w || !out))) return FP8ADAM_ERR_INVALID_ARG;
  if (n == 0) return FP8ADAM_OK;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  if (fmt == 0) encode_sr16_kernel<0><<<grid_for(n, 4), 256, 0, st>>>(x, w, out, n);
  else encode_sr16_kernel<1><<<grid_for(n, 4), 256, 0, st>>>(x, w, out, n);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return last_error();
}

extern "C" int fp8adam_decode(int32_t fmt, const uint8_t* codes, float* out, int64_t n, int32_t impl,
                              void* cuda_stream) {
  if (fmt < 0 || fmt > 1) return FP8ADAM_ERR_UNSUPPORTED_FMT;
  if (impl < 0 || impl > 1 || n < 0 || (n > 0 && (!codes || !out))) return FP8ADAM_ERR_INVALID_ARG;
  if (n == 0) return FP8ADAM_OK;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  FP8ADAM_CODEC_DISPATCH(decode_kernel, grid_for(n, 2), codes, out, n);
  return last_error();
}

extern "C" uint64_t fp8adam_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }
