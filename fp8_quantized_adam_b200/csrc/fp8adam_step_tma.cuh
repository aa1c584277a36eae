// fp8adam_step_tma.cuh -- the default step with its loads staged through
// shared memory by the Tensor Memory Accelerator (sm_100a).
//
// Same arithmetic, same results as fp8adam_step_kernel (shared device
// functions).  For FP8 m and v: a chunk's p, g, m, v are brought in as
// 1-D bulk copies (cp.async.bulk global -> shared, no multicast) of
// kSub-element sub-tiles through a kStages-deep ring of shared-memory stages
// (3 x 16 KB), each completed on an mbarrier.  One thread issues the copies;
// all threads consume a stage from shared memory (2 x 4 elements each),
// store p and the new codes straight to global, and release the stage.  The
// copies run ahead of the arithmetic, so the bytes in flight no longer depend
// on registers.  4 CTAs of 256 threads per SM (62-64 registers, 48 KB of
// shared memory each).  A chunk's first copies are issued before its
// per-tensor loads and scale arithmetic, which then overlap the fill.
// Measured on the 7B-shaped layout: 14.12 ms per step against 14.85 ms for
// per-thread vector loads and 14.1 ms for a probe with the same copies and no
// arithmetic; a warp-specialised form (separate producer warp, empty/full
// barriers) and 1024-element sub-tiles were slower.
//
// A tensor that is not 16-byte aligned, and the part of a chunk beyond its
// last whole sub-tile, go through the per-thread path of fp8adam_step.cuh.
// Every wait is bounded in time (about 1 s on the global timer, each try
// suspending at most 20 us): on a timeout the CTA sets bit 0 of *err, waits
// (bounded) for its copies in flight and leaves the chunk unfinished; CTAs
// that start later see the flag and return at once (the host reads it
// through fp8adam_check).
#pragma once

#include <stdint.h>

#include "fp8_codec.cuh"
#include "fp8adam_step.cuh"

namespace fp8adam {

constexpr int kSub = 2048;                    // elements per stage (2 x 4 per thread)
constexpr int kStages = 3;
// Bounded waits: each try suspends at most kSuspendNs (the hint); a wait
// gives up after kWaitNs on the global timer, or after kWaitLimit tries.
constexpr uint32_t kSuspendNs = 20000;        // 20 us
constexpr uint32_t kWaitNs = 1000000000u;     // 1 s (the timer's low word wraps after 4.29 s)
constexpr uint32_t kWaitLimit = 1u << 20;

struct __align__(128) TmaStage {              // 16 KB
  float p[kSub];
  uint16_t g[kSub];
  uint8_t m[kSub];
  uint8_t v[kSub];
};
constexpr int kTmaSmemBytes = kStages * (int)sizeof(TmaStage);  // 48 KB: 4 CTAs per SM

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity), "r"(kSuspendNs)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint32_t globaltimer_lo_ns() {
  uint32_t t;
  asm volatile("mov.u32 %0, %%globaltimer_lo;" : "=r"(t));
  return t;
}
// bounded wait; false if the limit ran out.  The first try needs no timer.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint32_t t0 = globaltimer_lo_ns();
  for (uint32_t it = 0; it < kWaitLimit; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_lo_ns() - t0 > kWaitNs) return false;  // modular: exact across a wrap
  }
  return false;
}
// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`
// (16-byte aligned addresses, size a multiple of 16)
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_addr(dst)),
               "l"(src), "r"(bytes), "r"(smem_addr(bar))
               : "memory");
}

// 4 elements of stage `st` from stage offset j (a multiple of 4), global
// element index i of tensor td.  A warp's 32 threads take 128 consecutive
// elements, so every shared-memory read and global store is contiguous.
template <int MF, int VF, bool STATS>
__device__ __forceinline__ void consume4(const TmaStage& st, int j, const TensorDesc& td, int64_t i,
                                         const StepConsts& c, float inv_s_m, float inv_s_v, float s_m_new,
                                         float s_v_new, float& am, float& av, uint32_t& flushed, uint32_t& sat) {
  FP8ADAM_BOUNDS(i >= 0 && i + 4 <= td.numel);
  const float4 pin = *reinterpret_cast<const float4*>(&st.p[j]);
  const uint2 gq = *reinterpret_cast<const uint2*>(&st.g[j]);
  const uint32_t mw = *reinterpret_cast<const uint32_t*>(&st.m[j]);
  const uint32_t vw = *reinterpret_cast<const uint32_t*>(&st.v[j]);
  const float2 ma = dec2_hw<MF>(mw & 0xFFFFu), mb = dec2_hw<MF>(mw >> 16);
  const float2 va = dec2_hw<VF>(vw & 0xFFFFu), vb = dec2_hw<VF>(vw >> 16);
  const float mo[4] = {__fmul_rn(ma.x, inv_s_m), __fmul_rn(ma.y, inv_s_m), __fmul_rn(mb.x, inv_s_m),
                       __fmul_rn(mb.y, inv_s_m)};
  const float vo[4] = {__fmul_rn(va.x, inv_s_v), __fmul_rn(va.y, inv_s_v), __fmul_rn(vb.x, inv_s_v),
                       __fmul_rn(vb.y, inv_s_v)};
  const float g[4] = {bf16_lo(gq.x), bf16_hi(gq.x), bf16_lo(gq.y), bf16_hi(gq.y)};
  const float p4[4] = {pin.x, pin.y, pin.z, pin.w};
  float pout[4], mn[4], vn[4], ym[4], yv[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    moments(c, g[e], mo[e], vo[e], mn[e], vn[e]);
    am = fmax_nan(am, fabsf(mn[e]));
    av = fmax_nan(av, fabsf(vn[e]));
    pout[e] = update(c, p4[e], mn[e], vn[e]);
    ym[e] = __fmul_rn(mn[e], s_m_new);
    yv[e] = __fmul_rn(vn[e], s_v_new);
  }
  const uint32_t mq = enc2_hw<MF>(ym[0], ym[1]) | (enc2_hw<MF>(ym[2], ym[3]) << 16);
  const uint32_t vq = enc2_hw<VF>(yv[0], yv[1]) | (enc2_hw<VF>(yv[2], yv[3]) << 16);
  if constexpr (STATS) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      sat += fabsf(ym[e]) > FmtTraits<MF>::kMax ? 1u : 0u;
      sat += fabsf(yv[e]) > FmtTraits<VF>::kMax ? 1u : 0u;
      flushed += (vn[e] > 0.0f && ((vq >> (8 * e)) & 0x7Fu) == 0u) ? 1u : 0u;
    }
  }
  st_stream_f4(td.p + i, make_float4(pout[0], pout[1], pout[2], pout[3]));
  __stcs(reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(td.m) + i), mq);
  __stcs(reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(td.v) + i), vq);
}

// Sub-tile k of the chunk that starts at element e0 of td into stage
// k % kStages (thread 0 only): arm the stage's barrier with the byte count,
// then issue the four bulk copies.
__device__ __forceinline__ void tma_issue(const TensorDesc& td, int64_t e0, int k, TmaStage* stage, uint64_t* full) {
  TmaStage& st = stage[k % kStages];
  uint64_t* bar = &full[k % kStages];
  const int64_t b = e0 + (int64_t)k * kSub;
  mbar_arrive_expect_tx(bar, (uint32_t)sizeof(TmaStage));
  if (debug_skip_copies(k)) return;  // debug build: this stage's bytes never arrive
  bulk_load(st.p, td.p + b, kSub * 4, bar);
  bulk_load(st.g, td.g + b, kSub * 2, bar);
  bulk_load(st.m, static_cast<const uint8_t*>(td.m) + b, kSub, bar);
  bulk_load(st.v, static_cast<const uint8_t*>(td.v) + b, kSub, bar);
}

// The staged pipeline over the first nsub whole sub-tiles of the chunk that
// starts at element e0 of td, in two parts so that a kernel can do its own
// set-up while the first copies are in flight:
// - tma_begin initialises the stage barriers and has thread 0 issue the
//   first kStages sub-tiles;
// - tma_run then has every thread call body(st, j, i, h) for its 2 groups of
//   4 elements of each sub-tile (stage st, stage offset j, global element i,
//   group h = 0 or 1, a constant once the loop is unrolled), refilling each
//   stage once all threads are done with it.
// `full` and `abort_flag` live in the kernel's shared memory.  tma_run
// returns false if a wait gave up: then bit 0 of *err is set and the copies
// still in flight have been waited for (bounded), so the CTA can return.
__device__ __forceinline__ void tma_begin(const TensorDesc& td, int64_t e0, int nsub, TmaStage* stage,
                                          uint64_t* full, int& abort_flag) {
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int k = 0; k < kStages && k < nsub; ++k) tma_issue(td, e0, k, stage, full);
  }
  __syncthreads();
}

template <typename Body>
__device__ __forceinline__ bool tma_run(const TensorDesc& td, int64_t e0, int nsub, TmaStage* stage,
                                        uint64_t* full, int& abort_flag, uint32_t* err, Body&& body) {
  for (int k = 0; k < nsub; ++k) {
    const int s = k % kStages;
    if (!mbar_wait(&full[s], (uint32_t)((k / kStages) & 1))) abort_flag = 1;
    __syncthreads();
    if (abort_flag) {
      if (threadIdx.x == 0) {
        atomicOr(err, 1u);
        const int last = k + kStages < nsub ? k + kStages : nsub;  // copies issued and not consumed
        for (int q = k; q < last; ++q) (void)mbar_wait(&full[q % kStages], (uint32_t)((q / kStages) & 1));
      }
      __syncthreads();
      return false;  // the chunk stays unfinished; the host sees the flag
    }
#pragma unroll
    for (int h = 0; h < kSub / (4 * kThreads); ++h) {  // 2 groups of 4 elements per thread
      const int j = h * (4 * kThreads) + 4 * (int)threadIdx.x;
      body(stage[s], j, e0 + (int64_t)k * kSub + j, h);
    }
    __syncthreads();  // every thread is done reading stage s
    if (threadIdx.x == 0 && k + kStages < nsub) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic reads before the async refill
      tma_issue(td, e0, k + kStages, stage, full);
    }
  }
  return true;
}

template <int MF, int VF, bool STATS>
__global__ void __launch_bounds__(kThreads, 4)
fp8adam_step_tma_kernel(const StepArgs a, uint32_t* err) {
  static_assert(MF != kFP32 && VF != kFP32, "the staged path carries 1-byte codes");
  extern __shared__ __align__(128) unsigned char tma_smem[];
  TmaStage* stage = reinterpret_cast<TmaStage*>(tma_smem);
  __shared__ __align__(8) uint64_t full[kStages];
  __shared__ uint32_t red[4][kThreads / 32];
  __shared__ int abort_flag;

  // The chunk's record is static (written at create), so it is read before
  // the previous kernel in the stream has finished.  With programmatic
  // dependent launch (the step launched back to back with the previous one),
  // this grid starts while that kernel's last CTAs still run: every CTA lets
  // the next step's grid start once all of this grid's CTAs have started,
  // and waits for the previous grid's writes before it reads anything they
  // may touch (params, moments, scales, amax, counters, the error word).
  // Launched without it, both instructions return at once.
  const ChunkDesc cd = a.cdesc[blockIdx.x];
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const uint32_t err_word = *(volatile const uint32_t*)err;
  if (err_word) return;  // an earlier CTA timed out: stop at once
  const int ti = cd.tensor;
  FP8ADAM_BOUNDS(ti >= 0 && ti < a.num_tensors);
  TensorDesc td;
  td.p = cd.p;
  td.g = cd.g;
  td.m = cd.m;
  td.v = cd.v;
  td.numel = cd.numel;
  td.nunits = cd.nunits;
  td.aligned = cd.aligned;
#ifdef FP8ADAM_DEBUG
  td.numel = a.tensors[ti].numel;  // the debug build checks against the tensor table (set by a debug hook)
#endif
  if (a.cur && !a.cur->valid) return;  // a scheduled step past the end of its schedule
  const int64_t e0 = cd.start, e1 = cd.start + cd.len;
  FP8ADAM_BOUNDS(e0 >= 0 && e0 <= e1 && e1 <= td.numel);
  // whole sub-tiles go through the staged pipeline (aligned tensors only);
  // the first copies are issued before the per-tensor loads below
  const int nsub = td.aligned ? (int)((e1 - e0) / kSub) : 0;
  tma_begin(td, e0, nsub, stage, full, abort_flag);
  StepConsts c;
  (void)step_consts(a, c);
  const float s_m = a.scale_m[ti];
  const float s_v = a.scale_v[ti];
  const float s_m_new = pow2scale<MF>(__uint_as_float(a.amax_in_m[ti]), s_m);
  const float s_v_new = pow2scale<VF>(__uint_as_float(a.amax_in_v[ti]), s_v);
  const float inv_s_m = __fdiv_rn(1.0f, s_m);
  const float inv_s_v = __fdiv_rn(1.0f, s_v);
  float am = 0.0f, av = 0.0f;
  uint32_t flushed = 0, sat = 0;

  if (!tma_run(td, e0, nsub, stage, full, abort_flag, err, [&](const TmaStage& st, int j, int64_t i, int) {
        consume4<MF, VF, STATS>(st, j, td, i, c, inv_s_m, inv_s_v, s_m_new, s_v_new, am, av, flushed, sat);
      }))
    return;

  // the rest of the chunk (a tensor's ragged end, or an unaligned tensor)
  const int64_t r0 = e0 + (int64_t)nsub * kSub;
  int64_t scalar_from = r0;
  if (td.aligned) {
    for (int64_t i = r0 + (int64_t)threadIdx.x * kVec; i + kVec <= e1; i += kTile)
      group16<MF, VF, STATS, true>(td, i, c, inv_s_m, inv_s_v, s_m_new, s_v_new, am, av, flushed, sat);
    scalar_from = r0 + (e1 - r0) / kVec * kVec;
  }
  for (int64_t i = scalar_from + threadIdx.x; i < e1; i += kThreads)
    element1<MF, VF, STATS, true>(td, i, c, inv_s_m, inv_s_v, s_m_new, s_v_new, am, av, flushed, sat);

  // flush and publish, as in run_segment
  const uint32_t bm = block_max(__float_as_uint(am), red[0]);
  const uint32_t bv = block_max(__float_as_uint(av), red[1]);
  uint32_t bf = 0, bs = 0;
  if constexpr (STATS) {
    bf = block_sum(flushed, red[2]);
    bs = block_sum(sat, red[3]);
  }
  if (threadIdx.x == 0) {
    if (bm) atomicMax(a.acc_m + ti, bm);
    if (bv) atomicMax(a.acc_v + ti, bv);
    if constexpr (STATS) {
      if (bf) atomicAdd(a.stats + 0, (unsigned long long)bf);
      if (bs) atomicAdd(a.stats + 1, (unsigned long long)bs);
    }
    __threadfence();
    const uint32_t prev = atomicAdd(a.done + ti, 1u);
    if (prev + 1u == (uint32_t)td.nunits) {
      __threadfence();
      a.amax_m[ti] = __uint_as_float(atomicExch(a.acc_m + ti, 0u));
      a.amax_v[ti] = __uint_as_float(atomicExch(a.acc_v + ti, 0u));
      a.scale_m[ti] = s_m_new;
      a.scale_v[ti] = s_v_new;
      a.done[ti] = 0u;
    }
  }
}

}  // namespace fp8adam
