// fp8adam_noalloc.cu -- fp8adam_step_noalloc: the same AdamW step as
// fp8adam_create + fp8adam_step, for callers that cannot allocate memory.
//
// Who needs it: code that runs where allocation is not allowed or not
// possible -- inside a custom allocator or memory-pool callback, in a
// framework hook that must not grow the device footprint, in a process whose
// memory is fully reserved up front, or from a runtime that forbids
// cudaMalloc after start-up.  The regular path allocates its tables and
// accumulators in fp8adam_create; this entry point instead uses one
// file-scope device array of fixed size, so it allocates nothing at all.
//
// The scratch array lives in this library's device image: every GPU that
// loads the library holds it (about 288 KiB) until the process exits.  It
// holds the tensor table, the per-tensor chunk offsets, the amax
// accumulators and the per-tensor completion counters, for at most
// FP8ADAM_NOALLOC_MAX_TENSORS tensors.

#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>

#include "../../include/fp8adam.h"
#include "fp8_codec.cuh"
#include "fp8adam_step.cuh"

using namespace fp8adam;

namespace {

constexpr int kMaxT = FP8ADAM_NOALLOC_MAX_TENSORS;

// Byte layout of the scratch array (offsets are multiples of 256).
constexpr size_t round256(size_t x) { return (x + 255) / 256 * 256; }
constexpr size_t kDescOff = 0;
constexpr size_t kBeginOff = round256(kDescOff + sizeof(TensorDesc) * kMaxT);
constexpr size_t kAccOff = round256(kBeginOff + sizeof(int32_t) * (kMaxT + 1));
constexpr size_t kAccWords = 5 * (size_t)kMaxT;  // acc_m, acc_v, jit_m, jit_v, done
constexpr size_t kScratchBytes = round256(kAccOff + sizeof(uint32_t) * kAccWords);

// The scratch.  In host code this name is only a stand-in for the symbol,
// not a device address: host code must use the address obtained from
// cudaGetSymbolAddress (below), never the name itself.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Host-side image of the tensor table and chunk offsets, copied into the
// scratch by every call, and the byte ranges of the overlap check (static
// storage, not an allocation).
struct HostImage {
  TensorDesc desc[kMaxT];
  int32_t begin[kMaxT + 1];
};
static HostImage g_host_image;

struct ByteRange {
  uintptr_t begin, end;
  bool written;
};
static ByteRange g_ranges[4 * kMaxT];

// True if two of the n byte ranges overlap and at least one of them is
// written (param, m and v are written, grad is read).  Sorted by start in
// place (std::sort allocates nothing), a range overlaps an earlier one iff
// it starts before the furthest end seen so far: of any range if it is
// written, of the written ranges if it is only read.
bool written_range_overlaps(ByteRange* r, size_t n) {
  std::sort(r, r + n, [](const ByteRange& a, const ByteRange& b) { return a.begin < b.begin; });
  uintptr_t end_all = 0, end_written = 0;
  for (size_t k = 0; k < n; ++k) {
    const ByteRange& x = r[k];
    if (x.begin < (x.written ? end_all : end_written)) return true;
    end_all = end_all > x.end ? end_all : x.end;
    if (x.written) end_written = end_written > x.end ? end_written : x.end;
  }
  return false;
}

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_ptr[kMaxDevices];

// Device address of the scratch on the current device; looked up once per
// device (by the first call made while that device is current).
int scratch_address(int dev, unsigned char** out) {
  if (dev < 0 || dev >= kMaxDevices) return FP8ADAM_ERR_CUDA;
  void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (!p) {
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return FP8ADAM_ERR_CUDA;
    }
    g_scratch_ptr[dev].store(p, std::memory_order_release);
  }
  *out = static_cast<unsigned char*>(p);
  return FP8ADAM_OK;
}

struct NoAllocArgs {
  const TensorDesc* tensors;
  const int32_t* begin;  // [T+1] first chunk of each tensor
  int32_t num_tensors;
  float* scale_m;
  float* scale_v;
  float* amax_m;
  float* amax_v;
  const uint32_t* amax_in_m;
  const uint32_t* amax_in_v;
  uint32_t* acc_m;
  uint32_t* acc_v;
  uint32_t* done;
  StepConsts c;
};

// tensor owning chunk b: the last t with begin[t] <= b
__device__ __forceinline__ int owner_of(const int32_t* begin, int T, int b) {
  int lo = 0, hi = T;  // begin[lo] <= b < begin[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (begin[mid] <= b) lo = mid; else hi = mid;
  }
  return lo;
}

template <int MF, int VF, bool WRITE>
__global__ void __launch_bounds__(kThreads) noalloc_kernel(const NoAllocArgs a) {
  __shared__ uint32_t red[2][kThreads / 32];
  const int b = (int)blockIdx.x;
  const int ti = owner_of(a.begin, a.num_tensors, b);
  const TensorDesc td = a.tensors[ti];
  const int64_t start = (int64_t)(b - a.begin[ti]) * kChunk;
  const int32_t len = (int32_t)(td.numel - start < kChunk ? td.numel - start : kChunk);
  const StepConsts c = a.c;

  const float s_m = a.scale_m[ti];
  const float s_v = a.scale_v[ti];
  float s_m_new = s_m, s_v_new = s_v;
  if constexpr (WRITE) {
    if constexpr (MF != kFP32) s_m_new = pow2scale<MF>(__uint_as_float(a.amax_in_m[ti]), s_m);
    if constexpr (VF != kFP32) s_v_new = pow2scale<VF>(__uint_as_float(a.amax_in_v[ti]), s_v);
  }
  const float inv_s_m = __fdiv_rn(1.0f, s_m);
  const float inv_s_v = __fdiv_rn(1.0f, s_v);
  float am = 0.0f, av = 0.0f;  // NaN-keeping max, as the regular step kernels reduce it
  uint32_t unused_f = 0, unused_s = 0;
  const int64_t end = start + len;
  int64_t scalar_from = start;

  if (td.aligned) {
    const int64_t vec_end = start + (int64_t)(len / kVec) * kVec;
    for (int64_t i = start + (int64_t)threadIdx.x * kVec; i < vec_end; i += kTile) {
      float4 pv[4];
      if constexpr (WRITE) {
#pragma unroll
        for (int k = 0; k < 4; ++k) pv[k] = ld_stream_f4(td.p + i + 4 * k);
      }
      const uint4 g0 = ld_ro_u4(td.g + i);
      const uint4 g1 = ld_ro_u4(td.g + i + 8);
      Tile16<MF> tm;
      Tile16<VF> tv;
      tm.load(td.m, i);
      tv.load(td.v, i);
      const uint32_t gw[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float mo[4], vo[4], mn[4], vn[4];
        tm.decode4(k, inv_s_m, mo);
        tv.decode4(k, inv_s_v, vo);
        const float g[4] = {bf16_lo(gw[2 * k]), bf16_hi(gw[2 * k]), bf16_lo(gw[2 * k + 1]),
                            bf16_hi(gw[2 * k + 1])};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          moments(c, g[j], mo[j], vo[j], mn[j], vn[j]);
          am = fmax_nan(am, fabsf(mn[j]));
          av = fmax_nan(av, fabsf(vn[j]));
        }
        if constexpr (WRITE) {
          float pk[4] = {pv[k].x, pv[k].y, pv[k].z, pv[k].w};
#pragma unroll
          for (int j = 0; j < 4; ++j) pk[j] = update(c, pk[j], mn[j], vn[j]);
          pv[k] = make_float4(pk[0], pk[1], pk[2], pk[3]);
          tm.template encode4<false, false>(k, s_m_new, mn, unused_f, unused_s);
          tv.template encode4<false, true>(k, s_v_new, vn, unused_f, unused_s);
        }
      }
      if constexpr (WRITE) {
#pragma unroll
        for (int k = 0; k < 4; ++k) st_stream_f4(td.p + i + 4 * k, pv[k]);
        tm.store(td.m, i);
        tv.store(td.v, i);
      }
    }
    scalar_from = vec_end;
  }
  for (int64_t i = scalar_from + threadIdx.x; i < end; i += kThreads) {
    const float g = __uint_as_float((uint32_t)td.g[i] << 16);
    float mn, vn;
    moments(c, g, load1<MF>(td.m, i, inv_s_m), load1<VF>(td.v, i, inv_s_v), mn, vn);
    am = fmax_nan(am, fabsf(mn));
    av = fmax_nan(av, fabsf(vn));
    if constexpr (WRITE) {
      td.p[i] = update(c, td.p[i], mn, vn);
      store1<MF, false, false>(td.m, i, mn, s_m_new, unused_f, unused_s);
      store1<VF, false, true>(td.v, i, vn, s_v_new, unused_f, unused_s);
    }
  }

  const uint32_t bm = block_max(__float_as_uint(am), red[0]);
  const uint32_t bv = block_max(__float_as_uint(av), red[1]);
  if (threadIdx.x == 0) {
    if (bm) atomicMax(a.acc_m + ti, bm);
    if (bv) atomicMax(a.acc_v + ti, bv);
    if constexpr (WRITE) {
      __threadfence();
      const uint32_t prev = atomicAdd(a.done + ti, 1u);
      if (prev == (uint32_t)td.nunits - 1u) {
        __threadfence();
        a.amax_m[ti] = __uint_as_float(atomicExch(a.acc_m + ti, 0u));
        a.amax_v[ti] = __uint_as_float(atomicExch(a.acc_v + ti, 0u));
        a.scale_m[ti] = s_m_new;
        a.scale_v[ti] = s_v_new;
        a.done[ti] = 0u;
      }
    }
  }
}

using NoAllocFn = void (*)(const NoAllocArgs);
template <int MF, int VF, bool W> NoAllocFn fn() { return &noalloc_kernel<MF, VF, W>; }
NoAllocFn pick(int mf, int vf, bool write) {
  static const NoAllocFn t[3][3][2] = {
      {{fn<0, 0, false>(), fn<0, 0, true>()}, {fn<0, 1, false>(), fn<0, 1, true>()}, {fn<0, 2, false>(), fn<0, 2, true>()}},
      {{fn<1, 0, false>(), fn<1, 0, true>()}, {fn<1, 1, false>(), fn<1, 1, true>()}, {fn<1, 2, false>(), fn<1, 2, true>()}},
      {{fn<2, 0, false>(), fn<2, 0, true>()}, {fn<2, 1, false>(), fn<2, 1, true>()}, {fn<2, 2, false>(), fn<2, 2, true>()}}};
  return t[mf][vf][write ? 1 : 0];
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" int fp8adam_step_noalloc(const fp8adam_tensor* tensors, int32_t num_tensors, float* scale_m,
                                    float* scale_v, float* amax_m, float* amax_v, int32_t m_fmt,
                                    int32_t v_fmt, uint32_t flags, float lr, float beta1, float beta2,
                                    float eps, float weight_decay, int64_t step, void* cuda_stream) {
  if (!tensors || num_tensors < 1 || !scale_m || !scale_v || !amax_m || !amax_v)
    return FP8ADAM_ERR_INVALID_ARG;
  if (num_tensors > kMaxT) return FP8ADAM_ERR_NOALLOC_LIMIT;
  if (m_fmt < 0 || m_fmt > 2 || v_fmt < 0 || v_fmt > 2) return FP8ADAM_ERR_UNSUPPORTED_FMT;
  if (flags & ~FP8ADAM_FLAG_JIT_EVERY_STEP) return FP8ADAM_ERR_INVALID_ARG;
  if (step < 1 || !std::isfinite(lr) || !std::isfinite(weight_decay) || !(beta1 >= 0.0f) ||
      !(beta1 < 1.0f) || !(beta2 >= 0.0f) || !(beta2 < 1.0f) || !(eps >= 0.0f) || !std::isfinite(eps))
    return FP8ADAM_ERR_INVALID_ARG;

  // tensor table and chunk offsets, built in static host storage
  int64_t chunks = 0;
  for (int32_t i = 0; i < num_tensors; ++i) {
    const fp8adam_tensor& t = tensors[i];
    if (t.numel < 0 || t.numel > ((int64_t)1 << 48)) return FP8ADAM_ERR_INVALID_ARG;
    if (t.numel > 0 && (!t.param || !t.grad || !t.m || !t.v)) return FP8ADAM_ERR_INVALID_ARG;
    TensorDesc& d = g_host_image.desc[i];
    d.p = t.param;
    d.g = t.grad;
    d.m = t.m;
    d.v = t.v;
    d.numel = t.numel;
    const int64_t nc = (t.numel + kChunk - 1) / kChunk;
    if (nc > INT32_MAX) return FP8ADAM_ERR_INVALID_ARG;
    d.nunits = (int32_t)nc;
    d.aligned = aligned16(t.param) && aligned16(t.grad) && aligned16(t.m) && aligned16(t.v);
    g_host_image.begin[i] = (int32_t)chunks;
    chunks += nc;
    if (chunks > INT32_MAX) return FP8ADAM_ERR_INVALID_ARG;
  }
  g_host_image.begin[num_tensors] = (int32_t)chunks;

  // as fp8adam_create: no written buffer (p, m, v) may overlap another buffer
  {
    const size_t mb = m_fmt == FP8ADAM_FP32 ? 4 : 1, vb = v_fmt == FP8ADAM_FP32 ? 4 : 1;
    size_t nr = 0;
    for (int32_t i = 0; i < num_tensors; ++i) {
      const fp8adam_tensor& t = tensors[i];
      if (t.numel == 0) continue;
      const size_t n = (size_t)t.numel;
      g_ranges[nr++] = ByteRange{(uintptr_t)t.param, (uintptr_t)t.param + 4 * n, true};
      g_ranges[nr++] = ByteRange{(uintptr_t)t.grad, (uintptr_t)t.grad + 2 * n, false};
      g_ranges[nr++] = ByteRange{(uintptr_t)t.m, (uintptr_t)t.m + mb * n, true};
      g_ranges[nr++] = ByteRange{(uintptr_t)t.v, (uintptr_t)t.v + vb * n, true};
    }
    if (written_range_overlaps(g_ranges, nr)) return FP8ADAM_ERR_OVERLAP;
  }

  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FP8ADAM_ERR_CUDA;
  unsigned char* scratch = nullptr;
  if (scratch_address(dev, &scratch) != FP8ADAM_OK) return FP8ADAM_ERR_CUDA;
  if (chunks == 0) return FP8ADAM_OK;  // every tensor empty
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);

  const size_t T = (size_t)num_tensors;
  TensorDesc* d_desc = reinterpret_cast<TensorDesc*>(scratch + kDescOff);
  int32_t* d_begin = reinterpret_cast<int32_t*>(scratch + kBeginOff);
  uint32_t* acc = reinterpret_cast<uint32_t*>(scratch + kAccOff);
  uint32_t* acc_m = acc;
  uint32_t* acc_v = acc + kMaxT;
  uint32_t* jit_m = acc + 2 * kMaxT;
  uint32_t* jit_v = acc + 3 * kMaxT;
  uint32_t* done = acc + 4 * kMaxT;
  // the source is pageable static storage: the copy has consumed it when the
  // call returns
  if (cudaMemcpyAsync(d_desc, g_host_image.desc, T * sizeof(TensorDesc), cudaMemcpyHostToDevice, st) !=
          cudaSuccess ||
      cudaMemcpyAsync(d_begin, g_host_image.begin, (T + 1) * sizeof(int32_t), cudaMemcpyHostToDevice, st) !=
          cudaSuccess ||
      cudaMemsetAsync(acc, 0, kAccWords * sizeof(uint32_t), st) != cudaSuccess) {
    cudaGetLastError();
    return FP8ADAM_ERR_CUDA;
  }

  NoAllocArgs a;
  const double bc1 = 1.0 - std::pow((double)beta1, (double)step);
  const double bc2 = 1.0 - std::pow((double)beta2, (double)step);
  a.c.b1 = beta1;
  a.c.omb1 = (float)(1.0 - (double)beta1);
  a.c.b2 = beta2;
  a.c.omb2 = (float)(1.0 - (double)beta2);
  a.c.step_size = (float)((double)lr / bc1);
  a.c.isbc2 = (float)(1.0 / std::sqrt(bc2));
  a.c.eps = eps;
  a.c.decay = (float)(1.0 - (double)lr * (double)weight_decay);
  a.tensors = d_desc;
  a.begin = d_begin;
  a.num_tensors = num_tensors;
  a.scale_m = scale_m;
  a.scale_v = scale_v;
  a.amax_m = amax_m;
  a.amax_v = amax_v;
  a.done = done;

  const dim3 grid((unsigned)chunks), block(kThreads);
  const bool jit = step == 1 || (flags & FP8ADAM_FLAG_JIT_EVERY_STEP);
  if (jit) {
    NoAllocArgs pre = a;
    pre.acc_m = jit_m;
    pre.acc_v = jit_v;
    pre.amax_in_m = nullptr;
    pre.amax_in_v = nullptr;
    pick(m_fmt, v_fmt, false)<<<grid, block, 0, st>>>(pre);
    a.amax_in_m = jit_m;
    a.amax_in_v = jit_v;
  } else {
    a.amax_in_m = reinterpret_cast<const uint32_t*>(amax_m);
    a.amax_in_v = reinterpret_cast<const uint32_t*>(amax_v);
  }
  a.acc_m = acc_m;
  a.acc_v = acc_v;
  pick(m_fmt, v_fmt, true)<<<grid, block, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? FP8ADAM_OK : FP8ADAM_ERR_CUDA;
}
