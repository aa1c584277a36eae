// fp8adam_debug.cuh -- checks compiled into the debug build only
// (-DFP8ADAM_DEBUG, libfp8adam_debug.so); the release build has none of them.
//
// - Bounds: every global access of the step kernels is checked against its
//   tensor (and every chunk against the tensor table) before it is made; a
//   violation skips the access and sets bit 0 of g_debug_flags, which
//   fp8adam_check reports as FP8ADAM_ERR_DEBUG_BOUNDS.  Nothing traps.
// - Wait injection: CTA g_inject_cta skips the bulk copies of its sub-tile
//   g_inject_sub (the stage's barrier is armed, the bytes never arrive), so
//   its bounded wait runs out and the kernel takes its timeout path.  Set by
//   fp8adam_debug_inject_wait; off (-1) by default.
#pragma once

#include <stdint.h>

namespace fp8adam {

#ifdef FP8ADAM_DEBUG
static __device__ uint32_t g_debug_flags;
static __device__ int32_t g_inject_cta = -1;
static __device__ int32_t g_inject_sub = -1;

__device__ __forceinline__ bool debug_in_bounds(bool ok) {
  if (!ok) atomicOr(&g_debug_flags, 1u);
  return ok;
}
__device__ __forceinline__ bool debug_skip_copies(int sub) {
  return (int32_t)blockIdx.x == g_inject_cta && sub == g_inject_sub;
}
// leaves the enclosing void function when the condition fails
#define FP8ADAM_BOUNDS(cond) \
  do {                                              \
    if (!::fp8adam::debug_in_bounds(cond)) return;  \
  } while (0)
#else
__device__ __forceinline__ bool debug_skip_copies(int) { return false; }
#define FP8ADAM_BOUNDS(cond) \
  do {                       \
  } while (0)
#endif

}  // namespace fp8adam
