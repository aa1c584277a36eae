// fp8adam_capi.cu -- the C ABI declared in include/fp8adam.h.
//
// Host side of the FP8-moment AdamW step: argument validation, the device
// tensor/chunk tables, per-step constants (computed in double, rounded once
// to fp32) and kernel dispatch over the (m format, v format, stats) variants.
// The kernels are in fp8adam_step.cuh; the codec in fp8_codec.cuh.

#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <new>
#include <vector>

#include "../../include/fp8adam.h"
#include "fp8_codec.cuh"
#include "fp8adam_step.cuh"

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

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

// ------------------------------------------------------------ the context
struct fp8adam_ctx {
  int device = -1;
  int32_t T = 0;
  int32_t m_fmt = 0, v_fmt = 0;
  uint32_t flags = 0;
  int32_t nchunks = 0;
  float *scale_m = nullptr, *scale_v = nullptr, *amax_m = nullptr, *amax_v = nullptr;
  TensorDesc* d_tensors = nullptr;
  Chunk* d_chunks = nullptr;
  uint32_t* d_state = nullptr;  // [5T]: acc_m, acc_v, jit_m, jit_v, done
  unsigned long long* d_stats = nullptr;
};

static void free_ctx(fp8adam_ctx* c) {
  if (!c) return;
  cudaFree(c->d_tensors);
  cudaFree(c->d_chunks);
  cudaFree(c->d_state);
  cudaFree(c->d_stats);
  delete c;
}

extern "C" int fp8adam_create(const fp8adam_tensor* tensors, int32_t num_tensors, float* scale_m,
                              float* scale_v, float* amax_m, float* amax_v, int32_t m_fmt,
                              int32_t v_fmt, uint32_t flags, fp8adam_ctx** out) {
  if (!out) return FP8ADAM_ERR_INVALID_ARG;
  *out = nullptr;
  if (!tensors || num_tensors < 1 || !scale_m || !scale_v || !amax_m || !amax_v)
    return FP8ADAM_ERR_INVALID_ARG;
  if (m_fmt < 0 || m_fmt > 2 || v_fmt < 0 || v_fmt > 2) return FP8ADAM_ERR_UNSUPPORTED_FMT;
  if (flags & ~(FP8ADAM_FLAG_STATS | FP8ADAM_FLAG_JIT_EVERY_STEP)) return FP8ADAM_ERR_INVALID_ARG;

  std::vector<TensorDesc> desc((size_t)num_tensors);
  std::vector<Chunk> chunks;
  int64_t total_chunks = 0;
  for (int32_t i = 0; i < num_tensors; ++i) {
    const fp8adam_tensor& t = tensors[i];
    if (t.numel < 0) return FP8ADAM_ERR_INVALID_ARG;
    if (t.numel > 0 && (!t.param || !t.grad || !t.m || !t.v)) return FP8ADAM_ERR_INVALID_ARG;
    const int64_t nc = (t.numel + kChunk - 1) / kChunk;
    if (nc > INT32_MAX) return FP8ADAM_ERR_INVALID_ARG;
    total_chunks += nc;
  }
  if (total_chunks > INT32_MAX) return FP8ADAM_ERR_INVALID_ARG;
  chunks.reserve((size_t)total_chunks);
  for (int32_t i = 0; i < num_tensors; ++i) {
    const fp8adam_tensor& t = tensors[i];
    TensorDesc& d = desc[(size_t)i];
    d.p = t.param;
    d.g = t.grad;
    d.m = t.m;
    d.v = t.v;
    d.numel = t.numel;
    d.nchunks = (int32_t)((t.numel + kChunk - 1) / kChunk);
    d.aligned = aligned16(t.param) && aligned16(t.grad) && aligned16(t.m) && aligned16(t.v);
    for (int64_t s = 0; s < t.numel; s += kChunk) {
      Chunk c;
      c.tensor = i;
      c.start = s;
      c.len = (int32_t)(t.numel - s < kChunk ? t.numel - s : kChunk);
      chunks.push_back(c);
    }
  }

  fp8adam_ctx* c = new (std::nothrow) fp8adam_ctx();
  if (!c) return FP8ADAM_ERR_OOM;
  if (cudaGetDevice(&c->device) != cudaSuccess) {
    delete c;
    return FP8ADAM_ERR_CUDA;
  }
  c->T = num_tensors;
  c->m_fmt = m_fmt;
  c->v_fmt = v_fmt;
  c->flags = flags;
  c->nchunks = (int32_t)chunks.size();
  c->scale_m = scale_m;
  c->scale_v = scale_v;
  c->amax_m = amax_m;
  c->amax_v = amax_v;
  const size_t T = (size_t)num_tensors;
  if (cudaMalloc(&c->d_tensors, T * sizeof(TensorDesc)) != cudaSuccess ||
      cudaMalloc(&c->d_chunks, (chunks.empty() ? 1 : chunks.size()) * sizeof(Chunk)) != cudaSuccess ||
      cudaMalloc(&c->d_state, 5 * T * sizeof(uint32_t)) != cudaSuccess ||
      cudaMalloc(&c->d_stats, 2 * sizeof(unsigned long long)) != cudaSuccess) {
    cudaGetLastError();
    free_ctx(c);
    return FP8ADAM_ERR_OOM;
  }
  if (cudaMemcpy(c->d_tensors, desc.data(), T * sizeof(TensorDesc), cudaMemcpyHostToDevice) != cudaSuccess ||
      (!chunks.empty() &&
       cudaMemcpy(c->d_chunks, chunks.data(), chunks.size() * sizeof(Chunk), cudaMemcpyHostToDevice) !=
           cudaSuccess) ||
      cudaMemset(c->d_state, 0, 5 * T * sizeof(uint32_t)) != cudaSuccess ||
      cudaMemset(c->d_stats, 0, 2 * sizeof(unsigned long long)) != cudaSuccess ||
      cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    free_ctx(c);
    return FP8ADAM_ERR_CUDA;
  }
  *out = c;
  return FP8ADAM_OK;
}

extern "C" int fp8adam_step(fp8adam_ctx* ctx, float lr, float beta1, float beta2, float eps,
                            float weight_decay, int64_t step, void* cuda_stream) {
  if (!ctx) return FP8ADAM_ERR_INVALID_ARG;
  if (step < 1 || !std::isfinite(lr) || !std::isfinite(weight_decay) || !(beta1 >= 0.0f) ||
      !(beta1 < 1.0f) || !(beta2 >= 0.0f) || !(beta2 < 1.0f) || !(eps >= 0.0f) || !std::isfinite(eps))
    return FP8ADAM_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FP8ADAM_ERR_CUDA;
  if (dev != ctx->device) return FP8ADAM_ERR_WRONG_DEVICE;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  if (ctx->nchunks == 0) return FP8ADAM_OK;  // every tensor empty

  // constants of step t: double, rounded once to fp32
  const double bc1 = 1.0 - std::pow((double)beta1, (double)step);
  const double bc2 = 1.0 - std::pow((double)beta2, (double)step);
  StepArgs a;
  a.c.b1 = beta1;
  a.c.omb1 = (float)(1.0 - (double)beta1);
  a.c.b2 = beta2;
  a.c.omb2 = (float)(1.0 - (double)beta2);
  a.c.step_size = (float)((double)lr / bc1);
  a.c.isbc2 = (float)(1.0 / std::sqrt(bc2));
  a.c.eps = eps;
  a.c.decay = (float)(1.0 - (double)lr * (double)weight_decay);

  const size_t T = (size_t)ctx->T;
  uint32_t* acc_m = ctx->d_state;
  uint32_t* acc_v = ctx->d_state + T;
  uint32_t* jit_m = ctx->d_state + 2 * T;
  uint32_t* jit_v = ctx->d_state + 3 * T;
  a.tensors = ctx->d_tensors;
  a.chunks = ctx->d_chunks;
  a.scale_m = ctx->scale_m;
  a.scale_v = ctx->scale_v;
  a.amax_m = ctx->amax_m;
  a.amax_v = ctx->amax_v;
  a.done = ctx->d_state + 4 * T;
  a.stats = ctx->d_stats;

  const dim3 grid((unsigned)ctx->nchunks), block(kThreads);
  const bool jit = step == 1 || (ctx->flags & FP8ADAM_FLAG_JIT_EVERY_STEP);
  if (jit) {
    if (cudaMemsetAsync(jit_m, 0, 2 * T * sizeof(uint32_t), st) != cudaSuccess) return FP8ADAM_ERR_CUDA;
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
  a.acc_m = acc_m;
  a.acc_v = acc_v;
  pick_step(ctx->m_fmt, ctx->v_fmt, (ctx->flags & FP8ADAM_FLAG_STATS) != 0)<<<grid, block, 0, st>>>(a);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return last_error();
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
    case FP8ADAM_ERR_OOM: return "device allocation failed";
    case FP8ADAM_ERR_WRONG_DEVICE: return "current device differs from the context's";
    case FP8ADAM_ERR_NOALLOC_LIMIT: return "more tensors than the allocation-free step holds (FP8ADAM_NOALLOC_MAX_TENSORS)";
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
