// fp8adam_ext_tma.cuh -- the variant step (options of fp8adam_create_ex /
// fp8adam_step_ex) with its loads staged through shared memory by bulk
// copies, for FP8 m and v.
//
// The pipeline is the default staged step's (tma_begin / tma_run: 3 x 16 KB stages,
// one issuing thread, bounded waits, 4 CTAs of 256 threads per SM); the
// element work adds the options to the default step's:
//   - the gradient multiplier (loss-scale removal and clipping: from the
//     grad-norm pre-pass, or a host constant 1/loss_scale without one), one
//     multiply;
//   - the encode scales from the amax history and the margin (per chunk);
//   - the rounding (a compile-time kind): round-to-nearest with the hardware
//     conversion; stochastic rounding with 32-bit draws (Philox4x32-10 words
//     for two elements per call, and the integer SR encoder); or stochastic
//     rounding with 16-bit draws (one call per eight elements, four codes per
//     hardware stochastic-rounding conversion);
//   - the update from the stored moments (a uniform branch: decode the new
//     codes again);
//   - the bf16 copy of the new params (a uniform branch: one 8-byte store
//     per 4 elements).
// The ragged end of a chunk and unaligned tensors go through the per-thread
// element paths of fp8adam_ext.cuh with the same rounding mode.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "fp8_codec.cuh"
#include "fp8adam_ext.cuh"
#include "fp8adam_step.cuh"
#include "fp8adam_step_tma.cuh"

namespace fp8adam {

__device__ __forceinline__ uint32_t bf16_pair(float lo, float hi) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
         ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
}

// four codes (each < 256) into one word, byte k = ck
__device__ __forceinline__ uint32_t pack4(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3) {
  return __byte_perm(__byte_perm(c0, c1, 0x7740), __byte_perm(c2, c3, 0x7740), 0x5410);
}

// 4 elements of stage `st` at offset j (global element i, a multiple of 4).
// SRK: 0 round to nearest, 1 stochastic with 32-bit draws (computed here
// from su), 2 stochastic with 16-bit draws (the words wm, wv of the four m
// and the four v codes, from the caller).  OPTS: the update-from-stored and
// bf16-copy options may be on (runtime flags) and the gradient multiplier may
// differ from 1; without them (the lean stochastic-rounding kernels) their
// code is compiled out.
template <int MF, int VF, bool STATS, int SRK, bool OPTS>
__device__ __forceinline__ void ext_consume4(const ExtArgs& a, const TmaStage& st, int j, const TensorDesc& td,
                                             const ExtSeg& sg, const SrChunk& su, uint32_t wm, uint32_t wv,
                                             int64_t i, float& am, float& av, uint32_t& flushed, uint32_t& sat) {
  FP8ADAM_BOUNDS(i >= 0 && i + 4 <= td.numel);
  const StepConsts& c = sg.c;
  const float4 pin = *reinterpret_cast<const float4*>(&st.p[j]);
  const uint2 gq = *reinterpret_cast<const uint2*>(&st.g[j]);
  const uint32_t mw = *reinterpret_cast<const uint32_t*>(&st.m[j]);
  const uint32_t vw = *reinterpret_cast<const uint32_t*>(&st.v[j]);
  const float2 ma = dec2_hw<MF>(mw & 0xFFFFu), mb = dec2_hw<MF>(mw >> 16);
  const float2 va = dec2_hw<VF>(vw & 0xFFFFu), vb = dec2_hw<VF>(vw >> 16);
  const float mo[4] = {__fmul_rn(ma.x, sg.inv_s_m), __fmul_rn(ma.y, sg.inv_s_m), __fmul_rn(mb.x, sg.inv_s_m),
                       __fmul_rn(mb.y, sg.inv_s_m)};
  const float vo[4] = {__fmul_rn(va.x, sg.inv_s_v), __fmul_rn(va.y, sg.inv_s_v), __fmul_rn(vb.x, sg.inv_s_v),
                       __fmul_rn(vb.y, sg.inv_s_v)};
  // the lean instance runs only with the multiplier 1 (no loss scale, no clipping)
  const float g[4] = {OPTS ? __fmul_rn(bf16_lo(gq.x), sg.gm) : bf16_lo(gq.x),
                      OPTS ? __fmul_rn(bf16_hi(gq.x), sg.gm) : bf16_hi(gq.x),
                      OPTS ? __fmul_rn(bf16_lo(gq.y), sg.gm) : bf16_lo(gq.y),
                      OPTS ? __fmul_rn(bf16_hi(gq.y), sg.gm) : bf16_hi(gq.y)};
  const float p4[4] = {pin.x, pin.y, pin.z, pin.w};
  float mn[4], vn[4], ym[4], yv[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    moments(c, g[e], mo[e], vo[e], mn[e], vn[e]);
    am = fmax_nan(am, fabsf(mn[e]));
    av = fmax_nan(av, fabsf(vn[e]));
    ym[e] = __fmul_rn(mn[e], sg.s_m_new);
    yv[e] = __fmul_rn(vn[e], sg.s_v_new);
  }
  uint32_t mq, vq;
  if constexpr (SRK == 1) {
    // words of elements (i, i+1) and (i+2, i+3): .x/.y = m/v of the even
    // element, .z/.w = m/v of the odd one
    const uint4 r0 = sr_words_chunk(a, su, (uint32_t)(i >> 1));
    const uint4 r1 = sr_words_chunk(a, su, (uint32_t)(i >> 1) + 1u);
    mq = pack4(enc1_sr<MF>(ym[0], r0.x), enc1_sr<MF>(ym[1], r0.z), enc1_sr<MF>(ym[2], r1.x),
               enc1_sr<MF>(ym[3], r1.z));
    vq = pack4(enc1_sr<VF>(yv[0], r0.y), enc1_sr<VF>(yv[1], r0.w), enc1_sr<VF>(yv[2], r1.y),
               enc1_sr<VF>(yv[3], r1.w));
  } else if constexpr (SRK == 2) {
    mq = cvt_rs4<MF>(ym[0], ym[1], ym[2], ym[3], wm);
    vq = cvt_rs4<VF>(yv[0], yv[1], yv[2], yv[3], wv);
  } else {
    mq = enc2_hw<MF>(ym[0], ym[1]) | (enc2_hw<MF>(ym[2], ym[3]) << 16);
    vq = enc2_hw<VF>(yv[0], yv[1]) | (enc2_hw<VF>(yv[2], yv[3]) << 16);
  }
  float mu[4] = {mn[0], mn[1], mn[2], mn[3]};
  float vu[4] = {vn[0], vn[1], vn[2], vn[3]};
  if (OPTS && (a.flags & kExtFromStored)) {  // the update reads the stored values
    const float2 qa = dec2_hw<MF>(mq & 0xFFFFu), qb = dec2_hw<MF>(mq >> 16);
    const float2 ra = dec2_hw<VF>(vq & 0xFFFFu), rb = dec2_hw<VF>(vq >> 16);
    mu[0] = __fmul_rn(qa.x, sg.inv_s_m_new);
    mu[1] = __fmul_rn(qa.y, sg.inv_s_m_new);
    mu[2] = __fmul_rn(qb.x, sg.inv_s_m_new);
    mu[3] = __fmul_rn(qb.y, sg.inv_s_m_new);
    vu[0] = __fmul_rn(ra.x, sg.inv_s_v_new);
    vu[1] = __fmul_rn(ra.y, sg.inv_s_v_new);
    vu[2] = __fmul_rn(rb.x, sg.inv_s_v_new);
    vu[3] = __fmul_rn(rb.y, sg.inv_s_v_new);
  }
  float pout[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) pout[e] = update(c, p4[e], mu[e], vu[e]);
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
  if (OPTS && sg.pb)
    __stcs(reinterpret_cast<uint2*>(sg.pb + i), make_uint2(bf16_pair(pout[0], pout[1]), bf16_pair(pout[2], pout[3])));
}

// SRK: the rounding kind of ext_consume4; OPTS as there (the lean SR kernels
// are launched only when update-from-stored and the bf16 copy are off and the
// gradient multiplier is 1).
template <int MF, int VF, bool STATS, int SRK, bool OPTS = true>
__global__ void __launch_bounds__(kThreads, 4)
fp8adam_step_ext_tma_kernel(const ExtArgs a, uint32_t* err) {
  static_assert(MF != kFP32 && VF != kFP32, "the staged path carries 1-byte codes");
  static_assert(SRK != 2 || (kSub == 8 * kThreads && kTile % 8 == 0 && kSub % 8 == 0),
                "16-bit draws: two groups of four per thread and stage, chunks starting at multiples of 8");
  extern __shared__ __align__(128) unsigned char tma_smem[];
  TmaStage* stage = reinterpret_cast<TmaStage*>(tma_smem);
  __shared__ __align__(8) uint64_t full[kStages];
  __shared__ uint32_t red[4][kThreads / 32];
  __shared__ int abort_flag;

  // The chunk and tensor tables are static (written at create), so they are
  // read before the previous kernel in the stream has finished.  With
  // programmatic dependent launch this grid starts while that kernel's last
  // CTAs still run: every CTA lets the next grid start once all of this
  // grid's CTAs have started, then waits for the previous grid's writes
  // before it reads anything a step writes (the error word, the skip flag,
  // the schedule entry, the multiplier, scales, amax, params, moments).
  // Launched without it, both instructions return at once.
  const Chunk ch = a.s.chunks[blockIdx.x];
  const int ti = ch.tensor;
  FP8ADAM_BOUNDS(ti >= 0 && ti < a.s.num_tensors);
  const TensorDesc td = a.s.tensors[ti];
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (*(volatile const uint32_t*)err) return;  // an earlier CTA timed out: stop at once
  if (a.skip && *a.skip) return;              // a non-finite gradient: the step is skipped
  if (a.s.cur && !a.s.cur->valid) return;     // the schedule ran out
  const int64_t e0 = ch.start, e1 = ch.start + ch.len;
  FP8ADAM_BOUNDS(e0 >= 0 && e0 <= e1 && e1 <= td.numel);
  // whole sub-tiles are staged when the tensor and its bf16 output (if any)
  // are 16-byte aligned; the first copies are issued before the set-up below
  // (multiplier, scales from the amax history, constants)
  const uint16_t* pb = a.p_bf16 ? a.p_bf16[ti] : nullptr;
  const bool staged = td.aligned && (pb == nullptr || ((uintptr_t)pb & 15u) == 0);
  const int nsub = staged ? (int)((e1 - e0) / kSub) : 0;
  tma_begin(td, e0, nsub, stage, full, abort_flag);
  const float gm = a.grad_mult ? *a.grad_mult : a.gm_const;
  const ExtSeg sg = ext_setup<MF, VF>(a, ti, gm);
  float am = 0.0f, av = 0.0f;
  uint32_t flushed = 0, sat = 0;

  SrChunk su{0u, 0u, 0u};
  if constexpr (SRK == 1) su = sr_chunk(a, sg.sr_id, sg.t_lo, e0 >> 1);
  if constexpr (SRK == 2) su = sr_chunk(a, sg.sr_id, sg.t_lo, e0 >> 3);
  uint32_t w1m = 0, w1v = 0;  // 16-bit draws: the words of this thread's second group of the stage
  if (!tma_run(td, e0, nsub, stage, full, abort_flag, err, [&](const TmaStage& st, int j, int64_t i, int h) {
        uint32_t wm = 0, wv = 0;
        if constexpr (SRK == 2) {
          if (h == 0) {
            // The stage's first group of thread t is elements i .. i+3 (i = 8q
            // for even t, 8q + 4 for odd t), its second i + 1024 .. i + 1027.
            // One Philox call per thread and stage: even t takes the call of
            // its first group's eight elements (its own four and those of
            // t + 1), odd t that of its second group's (those of t - 1 and its
            // own); each passes the neighbour the two words it needs.
            // the counter's low word: i/8, or (i + 1024)/8 = i/8 + 128 for odd
            // t (i = 8q + 4); modulo 2^32 like the counter word itself
            const bool odd = (threadIdx.x & 1u) != 0;
            const uint4 w = sr_words_chunk(a, su, (uint32_t)(i >> 3) + (odd ? (uint32_t)(4 * kThreads / 8) : 0u));
            const uint32_t g0 = __shfl_xor_sync(0xFFFFFFFFu, odd ? w.x : w.z, 1);
            const uint32_t g1 = __shfl_xor_sync(0xFFFFFFFFu, odd ? w.y : w.w, 1);
            wm = odd ? g0 : w.x;
            wv = odd ? g1 : w.y;
            w1m = odd ? w.z : g0;
            w1v = odd ? w.w : g1;
          } else {
            wm = w1m;
            wv = w1v;
          }
        }
        ext_consume4<MF, VF, STATS, SRK, OPTS>(a, st, j, td, sg, su, wm, wv, i, am, av, flushed, sat);
      }))
    return;
  // the ragged end (under one sub-tile) or an unaligned tensor, element by element
  constexpr int kElemRound = SRK == 1 ? kRoundStochastic : (SRK == 2 ? kRoundStochastic16 : kRoundNearest);
  for (int64_t i = e0 + (int64_t)nsub * kSub + threadIdx.x; i < e1; i += kThreads)
    ext_element<MF, VF, STATS, kElemRound>(a, td, sg, i, am, av, flushed, sat);
  ext_flush<STATS>(a, ti, td.nunits, sg, am, av, flushed, sat, red);
}

}  // namespace fp8adam
