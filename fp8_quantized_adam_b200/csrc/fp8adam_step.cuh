// fp8adam_step.cuh -- the fused AdamW step with FP8-stored moments (sm_100a).
//
// Method: "Scaling FP8 training to trillion-token LLMs" (abstract: both Adam
// moments in FP8); blog.daoxuan.cc explainer of that paper, section "Adam
// 为什么给第一矩选 E4M3、第二矩选 E5M2" (m in E4M3, v in E5M2; m and v are
// moving averages of g and g^2); update as optim.AdamW in "FP8训练的稳定性挑战…",
// section "代码示例"; per-tensor scale from the tracked amax ("应对FP8训练稳定性
// 挑战的策略", DelayedScaling with margin 0).
//
// Design for B200: the step is a pure HBM stream (read p 4 B, g 2 B, m 1 B,
// v 1 B; write p 4 B, m 1 B, v 1 B per element).  One launch covers a whole
// parameter list through a chunk table: CTA b handles chunk b, a run of
// elements of one tensor (lengths guided by the work still to come: long
// chunks first, short ones last; up to kChunk), 4 CTAs of 256 threads resident per
// SM (64 registers).  Each thread moves 16 elements per iteration with 16-byte
// loads and stores (4 x p, 2 x g, 1 x m, 1 x v), streaming cache hints, all
// fp32 arithmetic as single IEEE operations (no FMA contraction), hardware
// cvt for the FP8 conversions.  The new amax of the chunk is reduced with a
// NaN-keeping max, a warp redux and one atomicMax per moment; the CTA that
// completes a tensor's last chunk (per-tensor counter) publishes its amax and
// scale, so a step is a single kernel (plus an amax pre-pass at step 1).
// (Measured on the 7B-shaped layout: within 2% of a kernel with the same
// loads and stores and no arithmetic.)
#pragma once

#include <stdint.h>

#include "fp8_codec.cuh"
#include "fp8adam_debug.cuh"

namespace fp8adam {

constexpr int kThreads = 256;
constexpr int kVec = 16;                     // elements per thread per tile
constexpr int kTile = kThreads * kVec;       // 4096 elements per tile
constexpr int64_t kChunk = 32 * (int64_t)kTile;  // 131072: the largest chunk (one CTA's work)

// resident CTAs per SM the step kernel is built for (register budget): FP8
// moments fit 64 registers per thread (4 x 256 threads), fp32 moments 128
template <int MF, int VF>
struct StepOccupancy {
  static constexpr int kMinBlocks = (MF != 2 && VF != 2) ? 4 : 2;
};

struct TensorDesc {
  float* p;
  const uint16_t* g;
  void* m;
  void* v;
  int64_t numel;
  int32_t nunits;   // chunks of the tensor
  int32_t aligned;  // all four buffers 16-byte aligned
};

// One chunk: `len` elements of tensor `tensor` from `start` (one CTA's work).
struct Chunk {
  int32_t tensor;
  int32_t len;
  int64_t start;
};

// A chunk with what the staged step needs to start it, in one 64-byte
// record: its tensor's buffers and sizes next to the chunk's range, so a CTA
// can issue its first copies after a single load.
struct ChunkDesc {
  float* p;
  const uint16_t* g;
  void* m;
  void* v;
  int64_t start;   // first element of the chunk in its tensor
  int64_t numel;   // the tensor's size
  int32_t len;     // elements of the chunk
  int32_t tensor;
  int32_t nunits;  // chunks of the tensor
  int32_t aligned; // the tensor's four buffers are 16-byte aligned
};

struct StepConsts {
  float b1, omb1, b2, omb2, step_size, isbc2, eps, decay;
};

// One step of a device-side schedule (fp8adam_set_schedule): the constants
// and per-step options, computed on the host; the step reads the entry the
// schedule's select kernel copied for it (valid = 0: the schedule ran out,
// and the step does nothing).
struct SchedEntry {
  StepConsts c;
  float loss_scale, max_norm;
  int32_t skip_nonfinite;
  uint32_t t_lo;      // the step (stochastic rounding's counter word)
  int32_t hist_slot;  // (t - 1) % amax history length
  int32_t valid;
};

struct StepArgs {
  const TensorDesc* tensors;     // [T]
  const Chunk* chunks;           // [chunks] tensor and start of each chunk (one per CTA)
  const ChunkDesc* cdesc;        // [chunks] the same chunks with their tensors' buffers (staged step)
  int32_t num_tensors;
  float* scale_m;            // [T] in: decode scale; out: encode scale of this step
  float* scale_v;
  float* amax_m;             // [T] out: max |m| of this step
  float* amax_v;
  const uint32_t* amax_in_m; // [T] amax that sets the encode scale (bits)
  const uint32_t* amax_in_v;
  uint32_t* acc_m;           // [T] amax accumulators (bits), zero between steps
  uint32_t* acc_v;
  uint32_t* done;            // [T] finished-tile counters, zero between steps
  unsigned long long* stats; // [2] flushed, saturated (STATS only)
  StepConsts c;
  const SchedEntry* cur;     // scheduled step: constants from here; else null (use c)
};

// The step's constants: the kernel argument, or the current schedule entry.
// False when the schedule has run out (the kernel then does nothing).
__device__ __forceinline__ bool step_consts(const StepArgs& a, StepConsts& c) {
  if (a.cur == nullptr) {
    c = a.c;
    return true;
  }
  if (!a.cur->valid) return false;
  c = a.cur->c;
  return true;
}

// ------------------------------------------------------------ memory access
__device__ __forceinline__ float4 ld_stream_f4(const float* p) {
  return __ldcs(reinterpret_cast<const float4*>(p));
}
__device__ __forceinline__ void st_stream_f4(float* p, float4 v) {
  __stcs(reinterpret_cast<float4*>(p), v);
}
__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
  return __ldcs(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ void st_stream_u4(void* p, uint4 v) {
  __stcs(reinterpret_cast<uint4*>(p), v);
}
// read-only input, not kept in L1
__device__ __forceinline__ uint4 ld_ro_u4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ------------------------------------------------------------ the math
// One element: EMAs, amax candidates.  Single-rounding fp32 operations in
// the order documented in include/fp8adam.h.
__device__ __forceinline__ void moments(const StepConsts& c, float g, float mo, float vo,
                                        float& m, float& v) {
  const float t1 = __fmul_rn(c.b1, mo);
  const float t2 = __fmul_rn(c.omb1, g);
  m = __fadd_rn(t1, t2);
  const float gg = __fmul_rn(g, g);
  const float t3 = __fmul_rn(c.b2, vo);
  const float t4 = __fmul_rn(c.omb2, gg);
  v = __fadd_rn(t3, t4);
}

__device__ __forceinline__ float update(const StepConsts& c, float p, float m, float v) {
  const float sq = __fsqrt_rn(v);
  const float den0 = __fmul_rn(sq, c.isbc2);
  const float den = __fadd_rn(den0, c.eps);
  const float u = __fdiv_rn(m, den);
  const float pd = __fmul_rn(p, c.decay);
  const float w = __fmul_rn(c.step_size, u);
  return __fsub_rn(pd, w);
}

__device__ __forceinline__ uint32_t umax(uint32_t a, uint32_t b) { return a > b ? a : b; }
// max that returns NaN if either input is NaN (the canonical, positive NaN)
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}
// |x| as ordered bits: integer max over them is a float max that keeps NaN
__device__ __forceinline__ uint32_t abs_bits(float x) { return __float_as_uint(x) & 0x7FFFFFFFu; }

// ------------------------------------------------------------ moment tiles
// 16 consecutive moments of one thread, handled as 4 groups of 4 (one 32-bit
// word of codes per group): load, decode group k, encode group k in place,
// store.
template <int FMT>
struct Tile16 {  // FP8 codes
  uint32_t w[4];
  __device__ __forceinline__ void load(const void* base, int64_t i) {
    const uint4 r = ld_stream_u4(static_cast<const uint8_t*>(base) + i);
    w[0] = r.x; w[1] = r.y; w[2] = r.z; w[3] = r.w;
  }
  __device__ __forceinline__ void decode4(int k, float inv_s, float (&out)[4]) const {
    const float2 a = dec2_hw<FMT>(w[k] & 0xFFFFu);
    const float2 b = dec2_hw<FMT>(w[k] >> 16);
    out[0] = __fmul_rn(a.x, inv_s);
    out[1] = __fmul_rn(a.y, inv_s);
    out[2] = __fmul_rn(b.x, inv_s);
    out[3] = __fmul_rn(b.y, inv_s);
  }
  template <bool STATS, bool IS_V>
  __device__ __forceinline__ void encode4(int k, float s, const float (&x)[4], uint32_t& flushed,
                                          uint32_t& sat) {
    float y[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) y[j] = __fmul_rn(x[j], s);
    w[k] = enc2_hw<FMT>(y[0], y[1]) | (enc2_hw<FMT>(y[2], y[3]) << 16);
    if constexpr (STATS) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        sat += fabsf(y[j]) > FmtTraits<FMT>::kMax ? 1u : 0u;
        if constexpr (IS_V) flushed += (x[j] > 0.0f && ((w[k] >> (8 * j)) & 0x7Fu) == 0u) ? 1u : 0u;
      }
    }
  }
  __device__ __forceinline__ void store(void* base, int64_t i) const {
    st_stream_u4(static_cast<uint8_t*>(base) + i, make_uint4(w[0], w[1], w[2], w[3]));
  }
};

template <>
struct Tile16<kFP32> {  // unquantised fp32 moments
  float4 r[4];
  __device__ __forceinline__ void load(const void* base, int64_t i) {
#pragma unroll
    for (int k = 0; k < 4; ++k) r[k] = ld_stream_f4(static_cast<const float*>(base) + i + 4 * k);
  }
  __device__ __forceinline__ void decode4(int k, float, float (&out)[4]) const {
    out[0] = r[k].x; out[1] = r[k].y; out[2] = r[k].z; out[3] = r[k].w;
  }
  template <bool STATS, bool IS_V>
  __device__ __forceinline__ void encode4(int k, float, const float (&x)[4], uint32_t&, uint32_t&) {
    r[k] = make_float4(x[0], x[1], x[2], x[3]);
  }
  __device__ __forceinline__ void store(void* base, int64_t i) const {
#pragma unroll
    for (int k = 0; k < 4; ++k) st_stream_f4(static_cast<float*>(base) + i + 4 * k, r[k]);
  }
};

// single elements (ragged tails, unaligned tensors)
template <int FMT>
__device__ __forceinline__ float load1(const void* base, int64_t i, float inv_s) {
  if constexpr (FMT == kFP32) {
    return static_cast<const float*>(base)[i];
  } else {
    return __fmul_rn(dec1_hw<FMT>(static_cast<const uint8_t*>(base)[i]), inv_s);
  }
}
template <int FMT, bool STATS, bool IS_V>
__device__ __forceinline__ void store1(void* base, int64_t i, float x, float s, uint32_t& flushed,
                                       uint32_t& sat) {
  if constexpr (FMT == kFP32) {
    static_cast<float*>(base)[i] = x;
  } else {
    const float y = __fmul_rn(x, s);
    const uint32_t q = enc1_hw<FMT>(y);
    static_cast<uint8_t*>(base)[i] = (uint8_t)q;
    if constexpr (STATS) {
      sat += fabsf(y) > FmtTraits<FMT>::kMax ? 1u : 0u;
      if constexpr (IS_V) flushed += (x > 0.0f && (q & 0x7Fu) == 0u) ? 1u : 0u;
    }
  }
}

// ------------------------------------------------------------ reductions
// Block-wide max of ordered bits; result valid in thread 0.
__device__ __forceinline__ uint32_t block_max(uint32_t x, uint32_t* sm) {
  x = __reduce_max_sync(0xFFFFFFFFu, x);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) sm[warp] = x;
  __syncthreads();
  uint32_t r = 0;
  if (threadIdx.x == 0) {
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) r = umax(r, sm[w]);
  }
  return r;
}
__device__ __forceinline__ uint32_t block_sum(uint32_t x, uint32_t* sm) {
  x = __reduce_add_sync(0xFFFFFFFFu, x);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) sm[warp] = x;
  __syncthreads();
  uint32_t r = 0;
  if (threadIdx.x == 0) {
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) r += sm[w];
  }
  return r;
}

// ------------------------------------------------------------ tile bodies
// One full 16-element group per thread of an aligned tensor (vector path).
template <int MF, int VF, bool STATS, bool WRITE>
__device__ __forceinline__ void group16(const TensorDesc& td, int64_t i, const StepConsts& c, float inv_s_m,
                                        float inv_s_v, float s_m_new, float s_v_new, float& am, float& av,
                                        uint32_t& flushed, uint32_t& sat) {
  FP8ADAM_BOUNDS(i >= 0 && i + kVec <= td.numel);
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
    const float g[4] = {bf16_lo(gw[2 * k]), bf16_hi(gw[2 * k]), bf16_lo(gw[2 * k + 1]), bf16_hi(gw[2 * k + 1])};
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
      tm.template encode4<STATS, false>(k, s_m_new, mn, flushed, sat);
      tv.template encode4<STATS, true>(k, s_v_new, vn, flushed, sat);
    }
  }
  if constexpr (WRITE) {
#pragma unroll
    for (int k = 0; k < 4; ++k) st_stream_f4(td.p + i + 4 * k, pv[k]);
    tm.store(td.m, i);
    tv.store(td.v, i);
  }
}

// One element (ragged tails, unaligned tensors).
template <int MF, int VF, bool STATS, bool WRITE>
__device__ __forceinline__ void element1(const TensorDesc& td, int64_t i, const StepConsts& c, float inv_s_m,
                                         float inv_s_v, float s_m_new, float s_v_new, float& am, float& av,
                                         uint32_t& flushed, uint32_t& sat) {
  FP8ADAM_BOUNDS(i >= 0 && i < td.numel);
  const float g = __uint_as_float((uint32_t)td.g[i] << 16);
  float mn, vn;
  moments(c, g, load1<MF>(td.m, i, inv_s_m), load1<VF>(td.v, i, inv_s_v), mn, vn);
  am = fmax_nan(am, fabsf(mn));
  av = fmax_nan(av, fabsf(vn));
  if constexpr (WRITE) {
    td.p[i] = update(c, td.p[i], mn, vn);
    store1<MF, STATS, false>(td.m, i, mn, s_m_new, flushed, sat);
    store1<VF, STATS, true>(td.v, i, vn, s_v_new, flushed, sat);
  }
}

// ------------------------------------------------------------ one segment
// The element range [e0, e1) of tensor ti: moments, update, codes, then the
// amax flush.  `units` is the number of work units the range stands for;
// the flush that brings the tensor's count to td.nunits publishes its amax
// and scale (every CTA that reads them for this step has done so by then).
// WRITE = false is the amax pre-pass (no stores, nothing published).
template <int MF, int VF, bool STATS, bool WRITE>
__device__ __forceinline__ void run_segment(const StepArgs& a, int ti, int64_t e0, int64_t e1, uint32_t units,
                                            uint32_t (*red)[kThreads / 32]) {
  FP8ADAM_BOUNDS(ti >= 0 && ti < a.num_tensors);
  const TensorDesc td = a.tensors[ti];
  FP8ADAM_BOUNDS(e0 >= 0 && e0 <= e1 && e1 <= td.numel);
  StepConsts c;
  if (!step_consts(a, c)) return;
  const float s_m = a.scale_m[ti];
  const float s_v = a.scale_v[ti];
  float s_m_new = s_m, s_v_new = s_v;
  if constexpr (WRITE && MF != kFP32) s_m_new = pow2scale<MF>(__uint_as_float(a.amax_in_m[ti]), s_m);
  if constexpr (WRITE && VF != kFP32) s_v_new = pow2scale<VF>(__uint_as_float(a.amax_in_v[ti]), s_v);
  const float inv_s_m = __fdiv_rn(1.0f, s_m);  // exact: powers of two
  const float inv_s_v = __fdiv_rn(1.0f, s_v);

  float am = 0.0f, av = 0.0f;
  uint32_t flushed = 0, sat = 0;
  int64_t scalar_from = e0;
  if (td.aligned) {
    for (int64_t i = e0 + (int64_t)threadIdx.x * kVec; i + kVec <= e1; i += kTile)
      group16<MF, VF, STATS, WRITE>(td, i, c, inv_s_m, inv_s_v, s_m_new, s_v_new, am, av, flushed, sat);
    scalar_from = e0 + (e1 - e0) / kVec * kVec;
  }
  for (int64_t i = scalar_from + threadIdx.x; i < e1; i += kThreads)
    element1<MF, VF, STATS, WRITE>(td, i, c, inv_s_m, inv_s_v, s_m_new, s_v_new, am, av, flushed, sat);

  const uint32_t bm = block_max(__float_as_uint(am), red[0]);
  const uint32_t bv = block_max(__float_as_uint(av), red[1]);
  uint32_t bf = 0, bs = 0;
  if constexpr (STATS && WRITE) {
    bf = block_sum(flushed, red[2]);
    bs = block_sum(sat, red[3]);
  }
  if (threadIdx.x == 0) {
    if (bm) atomicMax(a.acc_m + ti, bm);
    if (bv) atomicMax(a.acc_v + ti, bv);
    if constexpr (WRITE) {
      if constexpr (STATS) {
        if (bf) atomicAdd(a.stats + 0, (unsigned long long)bf);
        if (bs) atomicAdd(a.stats + 1, (unsigned long long)bs);
      }
      __threadfence();
      const uint32_t prev = atomicAdd(a.done + ti, units);
      if (prev + units == (uint32_t)td.nunits) {
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

// ------------------------------------------------------------ the schedule
// One CTA per chunk (a multiple of kTile elements of one tensor, chosen per
// context; a tensor's last chunk may be short).  f(ti, e0, e1, units) runs
// the chunk as the element range [e0, e1) of tensor ti, one work unit.
template <typename F>
__device__ __forceinline__ void for_each_segment(const StepArgs& a, F&& f) {
  const Chunk ch = a.chunks[blockIdx.x];  // one 16-byte load: tensor, length, start
  f(ch.tensor, ch.start, ch.start + ch.len, 1u);
}

template <int MF, int VF, bool STATS, bool WRITE>
__device__ __forceinline__ void step_body(const StepArgs& a) {
  __shared__ uint32_t red[4][kThreads / 32];
  for_each_segment(a, [&](int ti, int64_t e0, int64_t e1, uint32_t units) {
    run_segment<MF, VF, STATS, WRITE>(a, ti, e0, e1, units, red);
  });
}

template <int MF, int VF, bool STATS>
__global__ void __launch_bounds__(kThreads, StepOccupancy<MF, VF>::kMinBlocks)
fp8adam_step_kernel(const StepArgs a) {
  step_body<MF, VF, STATS, true>(a);
}

template <int MF, int VF>
__global__ void __launch_bounds__(kThreads, StepOccupancy<MF, VF>::kMinBlocks)
fp8adam_amax_kernel(const StepArgs a) {
  step_body<MF, VF, false, false>(a);
}

}  // namespace fp8adam
