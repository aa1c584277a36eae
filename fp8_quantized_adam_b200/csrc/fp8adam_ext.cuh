// fp8adam_ext.cuh -- optional variants of the FP8-moment AdamW step.
//
// These are the options of fp8adam_create_ex / fp8adam_step_ex; the default
// step kernels (fp8adam_step_tma_kernel, fp8adam_step_kernel) contain none of
// them.  This file has the element code of the options, the per-thread-load
// variant kernel and the pre-passes; fp8adam_ext_tma.cuh the staged kernel.
//   - amax history (DelayedScaling "amax_history_len", algo MAX) and margin
//     ("margin"), from the transformer_engine example of "FP8训练的稳定性挑战…";
//   - update from the stored (requantised) moments instead of this step's
//     fp32 ones (the reading behind the daoxuan.cc explainer's "1/(0+eps)"
//     case, sub-section "一个数值例子");
//   - stochastic rounding of the codes ("随机舍入" in "应对FP8训练稳定性挑战的
//     策略"), with random bits from Philox4x32-10 (Salmon, Moraes, Dror, Shaw,
//     "Parallel random numbers: as easy as 1, 2, 3", SC 2011): 32-bit draws
//     with the integer encoder below, or 16-bit draws rounded by the
//     hardware's stochastic-rounding conversion (four codes per instruction);
//   - a fused gradient multiplier (loss-scale removal and global-norm
//     clipping: "梯度缩放", "梯度裁剪" and the clip_grad_norm_ example) and
//     skip-on-non-finite, fed by a deterministic grad-norm pre-pass;
//   - a bf16 copy of the updated params.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "fp8_codec.cuh"
#include "fp8adam_step.cuh"

namespace fp8adam {

enum ExtFlags : uint32_t {
  kExtFromStored = 4u,  // the update reads dec(code)/scale
  kExtStochastic = 8u,  // stochastic rounding of the codes
  kExtSrDraw16 = 32u,   // with kExtStochastic: 16-bit draws, rounded by the hardware conversion
};

struct ExtArgs {
  StepArgs s;               // tensors, tiles, scales, amax, accumulators, constants
  uint32_t flags;           // kExt* bits
  int32_t margin_m, margin_v;
  int32_t use_hist;         // scale from the max of the amax ring (not at JIT steps)
  int32_t hist_len;         // ring length (>= 1 when hist_m is set)
  int32_t hist_slot;        // this step's slot, (t-1) % hist_len
  float* hist_m;            // [hist_len][T] or null
  float* hist_v;
  uint32_t sr_key[10][2];    // Philox round keys: round r uses seed + r * (0x9E3779B9, 0xBB67AE85)
  uint32_t t_lo;             // the step (counter word 3)
  const float* grad_mult;   // device scalar from the grad-norm pre-pass, or null (then gm_const)
  float gm_const;           // gradient multiplier without a pre-pass: 1/loss_scale (1.0: none)
  const uint32_t* skip;     // device flag, or null
  uint16_t* const* p_bf16;  // device array [T] of bf16 outputs (entries may be null), or null
  const uint32_t* sr_ids;   // device array [T]: each tensor's word in the SR counter, or null (its index)
};

// ------------------------------------------------------------ Philox4x32-10
constexpr uint32_t kPhiloxM0 = 0xD2511F53u, kPhiloxM1 = 0xCD9E8D57u;

// One round: each product as one 32 x 32 -> 64-bit multiply (low and high
// words together).
__device__ __forceinline__ uint4 philox_round(uint4 c, uint32_t k0, uint32_t k1) {
  const uint64_t p0 = (uint64_t)kPhiloxM0 * c.x;
  const uint64_t p1 = (uint64_t)kPhiloxM1 * c.z;
  return make_uint4((uint32_t)(p1 >> 32) ^ c.y ^ k0, (uint32_t)p1, (uint32_t)(p0 >> 32) ^ c.w ^ k1, (uint32_t)p0);
}

// The random words of counter (q, tensor id, step): with 32-bit draws those
// of elements (2q, 2q+1) (.x/.y: m/v of 2q, .z/.w: of 2q+1), with 16-bit
// draws those of elements 8q .. 8q+7.  `id` is the tensor's counter word
// (ExtArgs::sr_ids, by default its index in the table).
__device__ __forceinline__ uint4 sr_words(const ExtArgs& a, uint32_t id, uint32_t t_lo, int64_t q) {
  uint4 c = make_uint4((uint32_t)q, (uint32_t)((uint64_t)q >> 32), id, t_lo);
#pragma unroll
  for (int r = 0; r < 10; ++r) c = philox_round(c, a.sr_key[r][0], a.sr_key[r][1]);
  return c;
}

// The same words within one chunk.  A chunk never crosses a multiple of
// 2^33 elements of its tensor (the chunk table is cut there), so the
// counter's words 1..3 are the same for all its pairs, and so is half of the
// first round's output: computed once per chunk.
struct SrChunk {
  uint32_t x1, y1, w1;
};
__device__ __forceinline__ SrChunk sr_chunk(const ExtArgs& a, uint32_t id, uint32_t t_lo, int64_t q0) {
  const uint64_t p1 = (uint64_t)kPhiloxM1 * id;
  SrChunk u;
  u.x1 = (uint32_t)(p1 >> 32) ^ (uint32_t)((uint64_t)q0 >> 32) ^ a.sr_key[0][0];
  u.y1 = (uint32_t)p1;
  u.w1 = t_lo ^ a.sr_key[0][1];
  return u;
}
__device__ __forceinline__ uint4 sr_words_chunk(const ExtArgs& a, const SrChunk& u, uint32_t q_lo) {
  const uint64_t p0 = (uint64_t)kPhiloxM0 * q_lo;
  uint4 c = make_uint4(u.x1, u.y1, (uint32_t)(p0 >> 32) ^ u.w1, (uint32_t)p0);
#pragma unroll
  for (int r = 1; r < 10; ++r) c = philox_round(c, a.sr_key[r][0], a.sr_key[r][1]);
  return c;
}

// ------------------------------------------------------------ SR encoder
// Round up to the next grid value iff r < (|x| - lo) / (hi - lo) * 2^32 (that
// is r * (hi - lo) < (|x| - lo) * 2^32); saturate; NaN -> 0x7F.
//
// On the normal grid (2^emin <= |x| < max), the common case, one range test
// selects the integer path: the spacing is 2^sh fp32 ulps of |x|, the code
// is |x|'s bits shifted right by sh (rebiased), and the condition is exactly
// "the top 32 - sh bits of r are below the sh dropped bits".  It is computed
// as a carry: adding 2^sh - 1 - (r >> (32 - sh)) to the bits carries into
// the kept part exactly when (r >> (32 - sh)) < the dropped bits, so the
// code is one subtract-add and one shift (rebias folded into the constant).
// Below 2^emin the spacing is fixed: y = |x| / spacing is exact, and the
// threshold is ceil(frac(y) * 2^32).  (Adding 2^emin with round-toward-zero
// instead, to reuse the integer test, was measured slower.)
template <int FMT>
__device__ __forceinline__ uint32_t enc1_sr(float x, uint32_t r) {
  using T = FmtTraits<FMT>;
  constexpr int sh = 23 - T::kMant;
  constexpr uint32_t kMinNormal = (uint32_t)(127 + 1 - T::kBias) << 23;  // bits of 2^emin
  const uint32_t u = __float_as_uint(x);
  const uint32_t a = u & 0x7FFFFFFFu;
  uint32_t code;
  if (a - kMinNormal < T::kMaxBits - kMinNormal) {  // normal grid, below the max
    // (a - kMinNormal) >> sh + 2^M, plus the carry of the draw (modular: a >= kMinNormal here)
    constexpr uint32_t kBias = (1u << sh) - 1u + (1u << (T::kMant + sh)) - kMinNormal;
    code = (a - (r >> (32 - sh)) + kBias) >> sh;
  } else if (a >= T::kMaxBits) {                     // saturate, or NaN
    if (a > 0x7F800000u) return 0x7Fu;
    code = T::kMaxCode;
  } else {                                           // below 2^emin
    // y = |x| / (spacing 2^(1-bias-M)), exact; n = floor(y), f = y - n exact
    const float y = __fmul_rn(__uint_as_float(a), __uint_as_float((uint32_t)(127 + T::kBias - 1 + T::kMant) << 23));
    const float n = floorf(y);
    const float f = __fsub_rn(y, n);
    const uint32_t thr = __float2uint_ru(__fmul_rn(f, 4294967296.0f));  // ceil(f * 2^32); the product is exact
    code = (uint32_t)n + (r < thr ? 1u : 0u);
  }
  return ((u >> 24) & 0x80u) | code;
}

// ------------------------------------------------------------ SR with 16-bit draws
// cvt.rs.satfinite.{e4m3x4,e5m2x4}.f32 (sm_100a): four values to four codes
// in one instruction, each rounded stochastically with 16 random bits: up iff
// floor((|x|-lo)/(hi-lo) * 2^16) + r >= 2^16, saturating to the largest
// finite code, NaN -> 0x7F.  Byte k of the result is the code of xk; x0
// takes the word's low half as r, x1 the low half with its bits in reverse
// order, x2 the high half, x3 the high half reversed.
template <int FMT>
__device__ __forceinline__ uint32_t cvt_rs4(float x0, float x1, float x2, float x3, uint32_t w) {
  uint32_t d;
  if constexpr (FMT == kE4M3)
    asm("cvt.rs.satfinite.e4m3x4.f32 %0, {%1, %2, %3, %4}, %5;" : "=r"(d) : "f"(x3), "f"(x2), "f"(x1), "f"(x0), "r"(w));
  else
    asm("cvt.rs.satfinite.e5m2x4.f32 %0, {%1, %2, %3, %4}, %5;" : "=r"(d) : "f"(x3), "f"(x2), "f"(x1), "f"(x0), "r"(w));
  return d;
}

// One value as code `lane` (0..3) of word w (the other three inputs are 0,
// which every draw leaves at code 0).
template <int FMT>
__device__ __forceinline__ uint32_t enc1_sr16(float x, uint32_t w, int lane) {
  const uint32_t d = cvt_rs4<FMT>(lane == 0 ? x : 0.0f, lane == 1 ? x : 0.0f, lane == 2 ? x : 0.0f,
                                  lane == 3 ? x : 0.0f, w);
  return (d >> (8 * lane)) & 0xFFu;
}

// ------------------------------------------------------------ scale with margin
template <int FMT>
__device__ __forceinline__ float pow2scale_margin(float amax, float s_prev, int margin) {
  const uint32_t b = __float_as_uint(amax);
  if (!(amax > 0.0f) || b >= 0x7F800000u) return s_prev;
  int k;
  if (b < 0x00800000u) {
    // subnormal amax = man * 2^-149: leading bit p gives the exponent p - 149
    const int p = 31 - __clz(b);
    const uint32_t frac = (b << (23 - p)) & 0x7FFFFFu;
    k = FmtTraits<FMT>::kEmax - (p - 149) - (frac > 0x600000u ? 1 : 0);
  } else {
    const int e = (int)(b >> 23) - 127;
    k = FmtTraits<FMT>::kEmax - e - ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0);
  }
  k -= margin;
  k = k > 126 ? 126 : (k < -126 ? -126 : k);
  return __uint_as_float((uint32_t)(k + 127) << 23);
}

// ------------------------------------------------------------ encode/store
// Rounding of the codes: fixed at compile time (the staged kernels, one
// instantiation each) or read from ExtArgs::flags (the per-thread-load kernel).
enum SrMode : int { kRoundNearest = 0, kRoundStochastic = 1, kRoundByFlag = 2, kRoundStochastic16 = 3 };

// 0: round to nearest; 1: SR with 32-bit draws; 2: SR with 16-bit draws
template <int SRM>
__device__ __forceinline__ int sr_kind(const ExtArgs& a) {
  if constexpr (SRM == kRoundByFlag)
    return (a.flags & kExtStochastic) ? ((a.flags & kExtSrDraw16) ? 2 : 1) : 0;
  else if constexpr (SRM == kRoundStochastic) return 1;
  else if constexpr (SRM == kRoundStochastic16) return 2;
  else return 0;
}

// The random words of elements i .. i+3 (i a multiple of 4) for m and v.
// 32-bit draws: one word per code, from the call of pair i/2 and i/2 + 1
// (.x/.y of a call: m/v of its even element, .z/.w: of its odd element).
// 16-bit draws: one word per four codes, from the call of i/8 (.x/.y: m/v of
// elements 8q .. 8q+3, .z/.w: of 8q+4 .. 8q+7).

// Encodes one moment value (x * s) and returns the value the update reads.
// r: the element's 32-bit draw, or (16-bit draws) the word of its four codes,
// of which it is code `lane`.
template <int FMT, bool STATS, bool IS_V, int SRM>
__device__ __forceinline__ float ext_q(const ExtArgs& a, float x, float s, float inv_s, uint32_t r, int lane,
                                       uint32_t& code, uint32_t& flushed, uint32_t& sat) {
  if constexpr (FMT == kFP32) {
    code = 0;
    return x;
  } else {
    const float y = __fmul_rn(x, s);
    const int k = sr_kind<SRM>(a);
    code = k == 1 ? enc1_sr<FMT>(y, r) : (k == 2 ? enc1_sr16<FMT>(y, r, lane) : enc1_hw<FMT>(y));
    if constexpr (STATS) {
      sat += fabsf(y) > FmtTraits<FMT>::kMax ? 1u : 0u;
      if constexpr (IS_V) flushed += (x > 0.0f && (code & 0x7Fu) == 0u) ? 1u : 0u;
    }
    return (a.flags & kExtFromStored) ? __fmul_rn(dec1_hw<FMT>(code), inv_s) : x;
  }
}

struct ExtSeg {  // per tensor segment
  StepConsts c;   // the step's constants (argument or schedule entry)
  float inv_s_m, inv_s_v, s_m_new, s_v_new, inv_s_m_new, inv_s_v_new, gm;
  uint16_t* pb;
  int ti;
  uint32_t sr_id;     // the tensor's word in the SR counter
  uint32_t t_lo;      // the step, for the SR counter
  int32_t hist_slot;  // this step's slot of the amax history ring
};

// One element (tails, unaligned tensors).
template <int MF, int VF, bool STATS, int SRM>
__device__ __forceinline__ void ext_element(const ExtArgs& a, const TensorDesc& td, const ExtSeg& sg, int64_t i,
                                            float& am, float& av, uint32_t& flushed, uint32_t& sat) {
  FP8ADAM_BOUNDS(i >= 0 && i < td.numel);
  const StepConsts& c = sg.c;
  uint32_t rm = 0, rv = 0;
  const int srk = sr_kind<SRM>(a);
  if (srk == 1) {
    const uint4 r = sr_words(a, sg.sr_id, sg.t_lo, i >> 1);
    rm = (i & 1) ? r.z : r.x;
    rv = (i & 1) ? r.w : r.y;
  } else if (srk == 2) {
    const uint4 r = sr_words(a, sg.sr_id, sg.t_lo, i >> 3);
    rm = ((i >> 2) & 1) ? r.z : r.x;
    rv = ((i >> 2) & 1) ? r.w : r.y;
  }
  const float g = __fmul_rn(__uint_as_float((uint32_t)td.g[i] << 16), sg.gm);
  float mn, vn;
  moments(c, g, load1<MF>(td.m, i, sg.inv_s_m), load1<VF>(td.v, i, sg.inv_s_v), mn, vn);
  am = fmax_nan(am, fabsf(mn));
  av = fmax_nan(av, fabsf(vn));
  uint32_t qm, qv;
  const int lane = (int)(i & 3);
  const float mu = ext_q<MF, STATS, false, SRM>(a, mn, sg.s_m_new, sg.inv_s_m_new, rm, lane, qm, flushed, sat);
  const float vu = ext_q<VF, STATS, true, SRM>(a, vn, sg.s_v_new, sg.inv_s_v_new, rv, lane, qv, flushed, sat);
  if constexpr (MF == kFP32) static_cast<float*>(td.m)[i] = mn; else static_cast<uint8_t*>(td.m)[i] = (uint8_t)qm;
  if constexpr (VF == kFP32) static_cast<float*>(td.v)[i] = vn; else static_cast<uint8_t*>(td.v)[i] = (uint8_t)qv;
  const float pn = update(c, td.p[i], mu, vu);
  td.p[i] = pn;
  if (sg.pb) sg.pb[i] = __bfloat16_as_ushort(__float2bfloat16_rn(pn));
}

// 16 elements of an aligned tensor (vector loads/stores, as the default step).
template <int MF, int VF, bool STATS, int SRM>
__device__ __forceinline__ void ext_group16(const ExtArgs& a, const TensorDesc& td, const ExtSeg& sg, int64_t i,
                                            float& am, float& av, uint32_t& flushed, uint32_t& sat) {
  FP8ADAM_BOUNDS(i >= 0 && i + kVec <= td.numel);
  const StepConsts& c = sg.c;
  float4 pv[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) pv[k] = ld_stream_f4(td.p + i + 4 * k);
  const uint4 g0 = ld_ro_u4(td.g + i);
  const uint4 g1 = ld_ro_u4(td.g + i + 8);
  Tile16<MF> tm;
  Tile16<VF> tv;
  tm.load(td.m, i);
  tv.load(td.v, i);
  const uint32_t gw[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
  uint32_t pbw[8];
  uint4 w16 = make_uint4(0, 0, 0, 0);  // 16-bit draws: the words of the current eight elements
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float mo[4], vo[4], mn[4], vn[4], mu[4], vu[4];
    tm.decode4(k, sg.inv_s_m, mo);
    tv.decode4(k, sg.inv_s_v, vo);
    const float g[4] = {__fmul_rn(bf16_lo(gw[2 * k]), sg.gm), __fmul_rn(bf16_hi(gw[2 * k]), sg.gm),
                        __fmul_rn(bf16_lo(gw[2 * k + 1]), sg.gm), __fmul_rn(bf16_hi(gw[2 * k + 1]), sg.gm)};
    uint32_t rmj[4] = {0, 0, 0, 0}, rvj[4] = {0, 0, 0, 0};
    const int srk = sr_kind<SRM>(a);
    if (srk == 1) {
      const uint4 r0 = sr_words(a, sg.sr_id, sg.t_lo, (i + 4 * k) >> 1);
      const uint4 r1 = sr_words(a, sg.sr_id, sg.t_lo, ((i + 4 * k) >> 1) + 1);
      rmj[0] = r0.x; rmj[1] = r0.z; rmj[2] = r1.x; rmj[3] = r1.z;
      rvj[0] = r0.y; rvj[1] = r0.w; rvj[2] = r1.y; rvj[3] = r1.w;
    } else if (srk == 2) {  // i + 4k is a multiple of 4: one word for the four m codes, one for the v codes
      // one call per eight elements: a new one unless this group is the
      // second half of the previous group's eight
      const int64_t e = i + 4 * k;
      if (k % 2 == 0 || (e & 7) == 0) w16 = sr_words(a, sg.sr_id, sg.t_lo, e >> 3);
      const bool second = ((e >> 2) & 1) != 0;
      rmj[0] = rmj[1] = rmj[2] = rmj[3] = second ? w16.z : w16.x;
      rvj[0] = rvj[1] = rvj[2] = rvj[3] = second ? w16.w : w16.y;
    }
    uint32_t qm[4], qv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      moments(c, g[j], mo[j], vo[j], mn[j], vn[j]);
      am = fmax_nan(am, fabsf(mn[j]));
      av = fmax_nan(av, fabsf(vn[j]));
      mu[j] = ext_q<MF, STATS, false, SRM>(a, mn[j], sg.s_m_new, sg.inv_s_m_new, rmj[j], j, qm[j], flushed, sat);
      vu[j] = ext_q<VF, STATS, true, SRM>(a, vn[j], sg.s_v_new, sg.inv_s_v_new, rvj[j], j, qv[j], flushed, sat);
    }
    float pk[4] = {pv[k].x, pv[k].y, pv[k].z, pv[k].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) pk[j] = update(c, pk[j], mu[j], vu[j]);
    pv[k] = make_float4(pk[0], pk[1], pk[2], pk[3]);
    pbw[2 * k] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(pk[0])) |
                 ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(pk[1])) << 16);
    pbw[2 * k + 1] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(pk[2])) |
                     ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(pk[3])) << 16);
    if constexpr (MF != kFP32) tm.w[k] = qm[0] | (qm[1] << 8) | (qm[2] << 16) | (qm[3] << 24);
    else tm.r[k] = make_float4(mn[0], mn[1], mn[2], mn[3]);
    if constexpr (VF != kFP32) tv.w[k] = qv[0] | (qv[1] << 8) | (qv[2] << 16) | (qv[3] << 24);
    else tv.r[k] = make_float4(vn[0], vn[1], vn[2], vn[3]);
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) st_stream_f4(td.p + i + 4 * k, pv[k]);
  tm.store(td.m, i);
  tv.store(td.v, i);
  if (sg.pb) {  // 16 bf16 = 32 bytes; the bf16 buffer is 16-byte aligned when the tensor is
    __stcs(reinterpret_cast<uint4*>(sg.pb + i), make_uint4(pbw[0], pbw[1], pbw[2], pbw[3]));
    __stcs(reinterpret_cast<uint4*>(sg.pb + i + 8), make_uint4(pbw[4], pbw[5], pbw[6], pbw[7]));
  }
}

// ------------------------------------------------------------ the variant step
// Per-chunk constants: this step's decode scales, the encode scales from the
// amax (or the max of the amax history) with the margin, the multiplier and
// the bf16 output of tensor ti.
template <int MF, int VF>
__device__ __forceinline__ ExtSeg ext_setup(const ExtArgs& a, int ti, float gm) {
  const StepArgs& S = a.s;
  ExtSeg sg;
  sg.ti = ti;
  sg.sr_id = a.sr_ids ? a.sr_ids[ti] : (uint32_t)ti;
  sg.gm = gm;
  if (S.cur != nullptr) {  // a scheduled step (the kernel checked that the entry is valid)
    sg.c = S.cur->c;
    sg.t_lo = S.cur->t_lo;
    sg.hist_slot = S.cur->hist_slot;
  } else {
    sg.c = S.c;
    sg.t_lo = a.t_lo;
    sg.hist_slot = a.hist_slot;
  }
  sg.pb = a.p_bf16 ? a.p_bf16[ti] : nullptr;
  const float s_m = S.scale_m[ti], s_v = S.scale_v[ti];
  float am_in = __uint_as_float(S.amax_in_m[ti]);
  float av_in = __uint_as_float(S.amax_in_v[ti]);
  if (a.use_hist) {
    float hm = 0.0f, hv = 0.0f;
    for (int k = 0; k < a.hist_len; ++k) {
      hm = fmax_nan(hm, a.hist_m[(int64_t)k * S.num_tensors + ti]);
      hv = fmax_nan(hv, a.hist_v[(int64_t)k * S.num_tensors + ti]);
    }
    am_in = hm;
    av_in = hv;
  }
  sg.s_m_new = s_m;
  sg.s_v_new = s_v;
  if constexpr (MF != kFP32) sg.s_m_new = pow2scale_margin<MF>(am_in, s_m, a.margin_m);
  if constexpr (VF != kFP32) sg.s_v_new = pow2scale_margin<VF>(av_in, s_v, a.margin_v);
  sg.inv_s_m = __fdiv_rn(1.0f, s_m);
  sg.inv_s_v = __fdiv_rn(1.0f, s_v);
  sg.inv_s_m_new = __fdiv_rn(1.0f, sg.s_m_new);
  sg.inv_s_v_new = __fdiv_rn(1.0f, sg.s_v_new);
  return sg;
}

// The vector path needs the tensor's four buffers and its bf16 output (if
// any) 16-byte aligned.
__device__ __forceinline__ bool ext_vec_ok(const TensorDesc& td, const ExtSeg& sg) {
  return td.aligned && (sg.pb == nullptr || ((uintptr_t)sg.pb & 15u) == 0);
}

// Elements [e0, e1) of the chunk through the per-thread paths.
template <int MF, int VF, bool STATS, int SRM>
__device__ __forceinline__ void ext_range(const ExtArgs& a, const TensorDesc& td, const ExtSeg& sg, int64_t e0,
                                          int64_t e1, float& am, float& av, uint32_t& flushed, uint32_t& sat) {
  int64_t scalar_from = e0;
  if (ext_vec_ok(td, sg)) {
    for (int64_t i = e0 + (int64_t)threadIdx.x * kVec; i + kVec <= e1; i += kTile)
      ext_group16<MF, VF, STATS, SRM>(a, td, sg, i, am, av, flushed, sat);
    scalar_from = e0 + (e1 - e0) / kVec * kVec;
  }
  for (int64_t i = scalar_from + threadIdx.x; i < e1; i += kThreads)
    ext_element<MF, VF, STATS, SRM>(a, td, sg, i, am, av, flushed, sat);
}

// Block reduction of the chunk's amax (and counters), then the publish of
// the tensor's amax, history slot and scales by the CTA that finishes it.
template <bool STATS>
__device__ __forceinline__ void ext_flush(const ExtArgs& a, int ti, int32_t nunits, const ExtSeg& sg, float am,
                                          float av, uint32_t flushed, uint32_t sat, uint32_t (*red)[kThreads / 32]) {
  const StepArgs& S = a.s;
  const uint32_t bm = block_max(__float_as_uint(am), red[0]);
  const uint32_t bv = block_max(__float_as_uint(av), red[1]);
  uint32_t bf = 0, bs = 0;
  if constexpr (STATS) {
    bf = block_sum(flushed, red[2]);
    bs = block_sum(sat, red[3]);
  }
  if (threadIdx.x == 0) {
    if (bm) atomicMax(S.acc_m + ti, bm);
    if (bv) atomicMax(S.acc_v + ti, bv);
    if constexpr (STATS) {
      if (bf) atomicAdd(S.stats + 0, (unsigned long long)bf);
      if (bs) atomicAdd(S.stats + 1, (unsigned long long)bs);
    }
    __threadfence();
    const uint32_t prev = atomicAdd(S.done + ti, 1u);
    if (prev + 1u == (uint32_t)nunits) {
      __threadfence();
      const uint32_t fm = atomicExch(S.acc_m + ti, 0u);
      const uint32_t fv = atomicExch(S.acc_v + ti, 0u);
      S.amax_m[ti] = __uint_as_float(fm);
      S.amax_v[ti] = __uint_as_float(fv);
      if (a.hist_m) {
        a.hist_m[(int64_t)sg.hist_slot * S.num_tensors + ti] = __uint_as_float(fm);
        a.hist_v[(int64_t)sg.hist_slot * S.num_tensors + ti] = __uint_as_float(fv);
      }
      S.scale_m[ti] = sg.s_m_new;
      S.scale_v[ti] = sg.s_v_new;
      S.done[ti] = 0u;
    }
  }
}

// The per-thread-load variant step (fp32 moments, or staging switched off);
// the rounding mode comes from the flags.
template <int MF, int VF, bool STATS>
__global__ void __launch_bounds__(kThreads, 2)
fp8adam_step_ext_kernel(const ExtArgs a) {
  __shared__ uint32_t red[4][kThreads / 32];
  if (a.skip && *a.skip) return;  // a non-finite gradient: the step is skipped
  if (a.s.cur && !a.s.cur->valid) return;  // the schedule ran out
  const float gm = a.grad_mult ? *a.grad_mult : a.gm_const;
  const Chunk ch = a.s.chunks[blockIdx.x];
  const int ti = ch.tensor;
  FP8ADAM_BOUNDS(ti >= 0 && ti < a.s.num_tensors);
  const TensorDesc td = a.s.tensors[ti];
  FP8ADAM_BOUNDS(ch.start >= 0 && ch.len >= 0 && ch.start + ch.len <= td.numel);
  const ExtSeg sg = ext_setup<MF, VF>(a, ti, gm);
  float am = 0.0f, av = 0.0f;
  uint32_t flushed = 0, sat = 0;
  ext_range<MF, VF, STATS, kRoundByFlag>(a, td, sg, ch.start, ch.start + ch.len, am, av, flushed, sat);
  ext_flush<STATS>(a, ti, td.nunits, sg, am, av, flushed, sat, red);
}

// ------------------------------------------------------------ amax pre-pass
// Step-1 / current-scaling pre-pass of the variant step: the same moments
// (with the gradient multiplier), no stores; accumulates into s.acc_m/acc_v.
// 16 elements per thread-iteration with vector loads on aligned tensors.
template <int MF, int VF>
__global__ void __launch_bounds__(kThreads, StepOccupancy<MF, VF>::kMinBlocks)
fp8adam_amax_ext_kernel(const ExtArgs a) {
  __shared__ uint32_t red[2][kThreads / 32];
  if (a.skip && *a.skip) return;
  const StepArgs& S = a.s;
  StepConsts c;
  if (!step_consts(S, c)) return;
  const float gm = a.grad_mult ? *a.grad_mult : a.gm_const;
  const Chunk ch = S.chunks[blockIdx.x];
  const int ti = ch.tensor;
  FP8ADAM_BOUNDS(ti >= 0 && ti < S.num_tensors);
  const TensorDesc td = S.tensors[ti];
  const int64_t e0 = ch.start, e1 = ch.start + ch.len;
  FP8ADAM_BOUNDS(e0 >= 0 && e0 <= e1 && e1 <= td.numel);
  const float inv_s_m = __fdiv_rn(1.0f, S.scale_m[ti]);
  const float inv_s_v = __fdiv_rn(1.0f, S.scale_v[ti]);
  float am = 0.0f, av = 0.0f;
  int64_t scalar_from = e0;
  if (td.aligned) {
    for (int64_t i = e0 + (int64_t)threadIdx.x * kVec; i + kVec <= e1; i += kTile) {
      const uint4 g0 = ld_ro_u4(td.g + i);
      const uint4 g1 = ld_ro_u4(td.g + i + 8);
      Tile16<MF> tm;
      Tile16<VF> tv;
      tm.load(td.m, i);
      tv.load(td.v, i);
      const uint32_t gw[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float mo[4], vo[4];
        tm.decode4(k, inv_s_m, mo);
        tv.decode4(k, inv_s_v, vo);
        const float g[4] = {__fmul_rn(bf16_lo(gw[2 * k]), gm), __fmul_rn(bf16_hi(gw[2 * k]), gm),
                            __fmul_rn(bf16_lo(gw[2 * k + 1]), gm), __fmul_rn(bf16_hi(gw[2 * k + 1]), gm)};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float mn, vn;
          moments(c, g[j], mo[j], vo[j], mn, vn);
          am = fmax_nan(am, fabsf(mn));
          av = fmax_nan(av, fabsf(vn));
        }
      }
    }
    scalar_from = e0 + (e1 - e0) / kVec * kVec;
  }
  for (int64_t i = scalar_from + threadIdx.x; i < e1; i += kThreads) {
    const float g = __fmul_rn(__uint_as_float((uint32_t)td.g[i] << 16), gm);
    float mn, vn;
    moments(c, g, load1<MF>(td.m, i, inv_s_m), load1<VF>(td.v, i, inv_s_v), mn, vn);
    am = fmax_nan(am, fabsf(mn));
    av = fmax_nan(av, fabsf(vn));
  }
  const uint32_t bm = block_max(__float_as_uint(am), red[0]);
  const uint32_t bv = block_max(__float_as_uint(av), red[1]);
  if (threadIdx.x == 0) {
    if (bm) atomicMax(S.acc_m + ti, bm);
    if (bv) atomicMax(S.acc_v + ti, bv);
  }
}

// ------------------------------------------------------------ grad-norm pre-pass
// Per CTA: the sum of g^2 (each term exact in double) over its chunk, in a
// fixed order (each thread's elements in sequence, then a fixed
// shuffle/shared-memory tree), written to partial[blockIdx.x]; non-finite
// gradients are counted (not summed).  The fixed grid makes the result
// reproducible run to run.
__device__ __forceinline__ double block_sum_d(double x, double* sm) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) sm[warp] = x;
  __syncthreads();
  double r = 0.0;
  if (threadIdx.x == 0) {
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) r += sm[w];
  }
  return r;
}

// acc += g^2 for one bf16 gradient (bits b, low 16 bits).  A normal bf16 is
// widened to double by placing its exponent and 7 mantissa bits (no
// conversion instruction); g^2 has at most 16 significant bits, so the fused
// multiply-add rounds once, exactly like adding the exact square.  Zero adds
// nothing; inf and NaN are counted, not summed.
__device__ __forceinline__ void sumsq1(uint32_t b, double& acc, uint32_t& bad) {
  const uint32_t h = b & 0x7FFFu;
  if (h - 0x80u < 0x7F00u) {  // exponent field 1..254
    const double x = __hiloint2double((int)((h << 13) + (896u << 20)), 0);
    acc = __fma_rn(x, x, acc);
  } else if (h >= 0x7F80u) {
    ++bad;
  } else if (h != 0u) {  // subnormal
    const double x = (double)__uint_as_float(h << 16);
    acc = __fma_rn(x, x, acc);
  }
}

__global__ void __launch_bounds__(kThreads)
fp8adam_gradnorm_partial_kernel(const StepArgs a, double* partial, unsigned long long* nonfinite) {
  __shared__ double red[kThreads / 32];
  __shared__ uint32_t redi[kThreads / 32];
  double acc = 0.0;
  uint32_t bad = 0;
  const Chunk ch = a.chunks[blockIdx.x];
  FP8ADAM_BOUNDS(ch.tensor >= 0 && ch.tensor < a.num_tensors);
  const TensorDesc td = a.tensors[ch.tensor];
  const int64_t e0 = ch.start, e1 = ch.start + ch.len;
  FP8ADAM_BOUNDS(e0 >= 0 && e0 <= e1 && e1 <= td.numel);
  const int64_t vec_end = td.aligned ? e0 + (e1 - e0) / kVec * kVec : e0;
  // Fast path: each gradient widened to double (exact) and squared into the
  // sum by one fused multiply-add (exact square, one rounding), with no
  // per-element tests.  Zero adds nothing and a subnormal its exact square,
  // as in sumsq1, and the order is the same, so the sum is the same.  An inf
  // or NaN makes the sum non-finite: the thread then redoes its elements with
  // sumsq1, which counts them instead.
  for (int64_t i = e0 + (int64_t)threadIdx.x * kVec; i < vec_end; i += kTile) {
    const uint4 g0 = ld_ro_u4(td.g + i);
    const uint4 g1 = ld_ro_u4(td.g + i + 8);
    const uint32_t gw[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const double lo = (double)bf16_lo(gw[k]);
      const double hi = (double)bf16_hi(gw[k]);
      acc = __fma_rn(lo, lo, acc);
      acc = __fma_rn(hi, hi, acc);
    }
  }
  for (int64_t i = vec_end + threadIdx.x; i < e1; i += kThreads) {
    const double x = (double)__uint_as_float((uint32_t)td.g[i] << 16);
    acc = __fma_rn(x, x, acc);
  }
  if (!isfinite(acc)) {  // a non-finite gradient in this thread's elements
    acc = 0.0;
    for (int64_t i = e0 + (int64_t)threadIdx.x * kVec; i < vec_end; i += kTile) {
      const uint4 g0 = ld_ro_u4(td.g + i);
      const uint4 g1 = ld_ro_u4(td.g + i + 8);
      const uint32_t gw[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        sumsq1(gw[k] & 0xFFFFu, acc, bad);
        sumsq1(gw[k] >> 16, acc, bad);
      }
    }
    for (int64_t i = vec_end + threadIdx.x; i < e1; i += kThreads) sumsq1(td.g[i], acc, bad);
  }
  const double s = block_sum_d(acc, red);
  const uint32_t nb = block_sum(bad, redi);
  if (threadIdx.x == 0) {
    partial[blockIdx.x] = s;
    if (nb) atomicAdd(nonfinite, (unsigned long long)nb);
  }
}

// One CTA: the fixed-order total, the multiplier and the skip flag (the
// options from `cur` on a scheduled step).
// c = (1/loss_scale) * min(1, max_norm / (norm + 1e-6)), norm = sqrt(sum)/loss_scale
// (clip_grad_norm_'s definition on the unscaled gradients); max_norm <= 0 =
// no clipping; all in double, c rounded once to fp32.
__global__ void __launch_bounds__(kThreads)
fp8adam_gradnorm_finalize_kernel(const double* partial, int n, const unsigned long long* nonfinite,
                                 float loss_scale, float max_norm, int skip_nonfinite, const SchedEntry* cur,
                                 float* grad_mult, uint32_t* skip, double* norm_out) {
  __shared__ double red[kThreads / 32];
  double acc = 0.0;
  for (int k = threadIdx.x; k < n; k += kThreads) acc = __dadd_rn(acc, partial[k]);
  const double sum = block_sum_d(acc, red);
  if (threadIdx.x == 0) {
    if (cur != nullptr) {  // a scheduled step: the options of its entry
      if (!cur->valid) {
        *skip = 1u;  // the schedule ran out: nothing is updated
        return;
      }
      loss_scale = cur->loss_scale;
      max_norm = cur->max_norm;
      skip_nonfinite = cur->skip_nonfinite;
    }
    const double inv = __ddiv_rn(1.0, (double)loss_scale);
    const double norm = __dmul_rn(__dsqrt_rn(sum), inv);
    double coef = 1.0;
    if (max_norm > 0.0f) {
      coef = __ddiv_rn((double)max_norm, __dadd_rn(norm, 1e-6));
      if (coef > 1.0) coef = 1.0;
    }
    *grad_mult = __double2float_rn(__dmul_rn(inv, coef));
    *norm_out = norm;
    *skip = (skip_nonfinite && *nonfinite != 0ull) ? 1u : 0u;
  }
}

}  // namespace fp8adam
