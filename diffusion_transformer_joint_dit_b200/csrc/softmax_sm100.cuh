// Softmax building blocks shared by the attention kernels: one thread owns
// one query row of a 128-key score tile held in registers (4 x 32 words as
// tcgen05.ld returns them).  The packed f32x2 FMA / add and the three-input
// max of sm_100 cut the FP32-pipe instruction count of the row max, the
// scale-and-bias and the row sum; the exponentials run on MUFU (ex2).
#pragma once

#include <cstdint>

#include "sm100_ptx.cuh"

namespace jattn {

// ---------------------------------------------------------- packed fp32 ----

__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  return (static_cast<uint64_t>(__float_as_uint(hi)) << 32) | __float_as_uint(lo);
}
__device__ __forceinline__ float f2_lo(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float f2_hi(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }

__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// --------------------------------------------------------- tile helpers ----

// Row maxima of the two 64-key halves of a score tile.
__device__ __forceinline__ void row_max_halves(const uint32_t (&sv)[4][32], float& m_lo, float& m_hi) {
  float a = -INFINITY, b = -INFINITY, c = -INFINITY, d = -INFINITY;
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    a = fmax3(a, __uint_as_float(sv[0][i]), __uint_as_float(sv[0][i + 1]));
    b = fmax3(b, __uint_as_float(sv[1][i]), __uint_as_float(sv[1][i + 1]));
    c = fmax3(c, __uint_as_float(sv[2][i]), __uint_as_float(sv[2][i + 1]));
    d = fmax3(d, __uint_as_float(sv[3][i]), __uint_as_float(sv[3][i + 1]));
  }
  m_lo = fmaxf(a, b);
  m_hi = fmaxf(c, d);
}

// P = exp2(s * c + b) of a 128-key tile with (c, b) per 64-key half,
// packed in place two per word (keys [0,64) into sv[0], [64,128) into
// sv[2]) as bf16 or fp16, and the fp32 row sum of the unrounded values (two
// packed accumulators, alternating).
template <bool kF16>
__device__ __forceinline__ float exp_pack_sum(uint32_t (&sv)[4][32], float c_lo, float b_lo, float c_hi, float b_hi) {
  uint64_t acc0 = 0, acc1 = 0;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const float cc = c < 2 ? c_lo : c_hi;
    const float bb = c < 2 ? b_lo : b_hi;
    const uint64_t cc2 = f2_pack(cc, cc), bb2 = f2_pack(bb, bb);
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const uint64_t x = f2_fma(f2_pack(__uint_as_float(sv[c][i]), __uint_as_float(sv[c][i + 1])), cc2, bb2);
      const float lo = ex2_approx(f2_lo(x)), hi = ex2_approx(f2_hi(x));
      sv[c & 2][(c & 1) * 16 + (i >> 1)] = kF16 ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi);
      if (i & 2) acc1 = f2_add(acc1, f2_pack(lo, hi)); else acc0 = f2_add(acc0, f2_pack(lo, hi));
    }
  }
  const uint64_t a = f2_add(acc0, acc1);
  return f2_lo(a) + f2_hi(a);
}


}  // namespace jattn
