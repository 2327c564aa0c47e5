// Softmax building blocks shared by the attention kernels: one thread owns
// one query row of a 128-key score tile held in registers (4 x 32 words as
// tcgen05.ld returns them).
//
// At head dim 128 the exponentials of a score tile take as long on the
// SM's MUFU units (16 ex2 per clock) as the two MMAs that produce and
// consume it take on the tensor core, so the softmax offloads a fixed share
// of its exp2 calls to the FMA pipe (a range-reduced polynomial, below),
// and uses the packed f32x2 FMA / add and the three-input max of sm_100 to
// cut its FP32-pipe instruction count.
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

// ------------------------------------------------------- polynomial exp2 ----
// exp2(x) = 2^n * p(f), n = round(x), f = x - n in [-1/2, 1/2] (Cody-Waite
// reduction).  Adding 1.5 * 2^23 rounds x to an integer held in the low
// mantissa bits of t, whose bit pattern shifted left by 23 is n in the
// exponent field.  p is the degree-3 minimax fit of 2^f (relative error
// 7.5e-5) computed by fit_exp2_poly.py in this directory.  Arguments below
// -125 are clamped (the result is then ~2^-125, not 0, and 2^n p(f) stays a
// normal float); callers use it only on unmasked scores, which the lazy-max
// softmax keeps within [-inf, 8].
constexpr float kPolyC0 = 9.999280572e-01f;
constexpr float kPolyC1 = 6.932609677e-01f;
constexpr float kPolyC2 = 2.426111251e-01f;
constexpr float kPolyC3 = 5.517166853e-02f;
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x2) {
  const float xl = fmaxf(f2_lo(x2), -125.f), xh = fmaxf(f2_hi(x2), -125.f);
  const uint64_t x = f2_pack(xl, xh);
  const uint64_t t = f2_add(x, f2_pack(kRoundMagic, kRoundMagic));
  const uint64_t n = f2_add(t, f2_pack(-kRoundMagic, -kRoundMagic));
  const uint64_t f = f2_fma(n, f2_pack(-1.f, -1.f), x);
  uint64_t p = f2_fma(f2_pack(kPolyC3, kPolyC3), f, f2_pack(kPolyC2, kPolyC2));
  p = f2_fma(p, f, f2_pack(kPolyC1, kPolyC1));
  p = f2_fma(p, f, f2_pack(kPolyC0, kPolyC0));
  const uint32_t lo = static_cast<uint32_t>(p) + (static_cast<uint32_t>(t) << 23);
  const uint32_t hi = static_cast<uint32_t>(p >> 32) + (static_cast<uint32_t>(t >> 32) << 23);
  return (static_cast<uint64_t>(hi) << 32) | lo;
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

// P = exp2(s * c + b) with (c, b) per 64-key half, packed in place two per
// word (keys [0,64) into sv[0], [64,128) into sv[2]) as bf16 or fp16, and
// the fp32 row sums of each half: of the packed (rounded) values when
// kRoundedSum, else of the fp32 values.  With `poly`, one pair in every
// kPolyEvery pairs takes the polynomial exp2 instead of MUFU.
template <bool kF16, int kPolyEvery, bool kRoundedSum>
__device__ __forceinline__ void exp_pack_tile(uint32_t (&sv)[4][32], float c_lo, float b_lo, float c_hi,
                                              float b_hi, bool poly, float& sum_lo, float& sum_hi) {
  uint64_t acc_lo = 0, acc_hi = 0;  // packed partial sums (0.0f, 0.0f)
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const float cc = c < 2 ? c_lo : c_hi;
    const float bb = c < 2 ? b_lo : b_hi;
    const uint64_t cc2 = f2_pack(cc, cc), bb2 = f2_pack(bb, bb);
    uint64_t acc = 0;
    float acc_a = 0.f, acc_b = 0.f;  // bf16 rounded-sum path: even / odd keys
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const uint64_t x = f2_fma(f2_pack(__uint_as_float(sv[c][i]), __uint_as_float(sv[c][i + 1])), cc2, bb2);
      uint64_t p;
      if (kPolyEvery > 0 && poly && ((i >> 1) % (kPolyEvery > 0 ? kPolyEvery : 1)) == kPolyEvery - 1) {
        p = exp2_poly2(x);
      } else {
        p = f2_pack(ex2_approx(f2_lo(x)), ex2_approx(f2_hi(x)));
      }
      const uint32_t packed = kF16 ? pack_f16x2(f2_lo(p), f2_hi(p)) : pack_bf16x2(f2_lo(p), f2_hi(p));
      sv[c & 2][(c & 1) * 16 + (i >> 1)] = packed;
      // With kRoundedSum the row sum adds the *rounded* P the MMA multiplies
      // V by, so that O = sum(P V) / sum(P) uses one set of weights.  With
      // the lazy max a dominant key's P lies in (1, 2^8] and is inexact in
      // bf16 (2^-9); summing the rounded value cancels that rounding in the
      // quotient.  bf16 halves are added straight into fp32 with the
      // mixed-precision add; fp16 P rounds 8x finer, where the fp32 sum is
      // kept.
      if (kRoundedSum && !kF16) {
        asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
            "add.rn.f32.bf16 %0, lo, %0;\n\tadd.rn.f32.bf16 %1, hi, %1;\n\t}"
            : "+f"(acc_a), "+f"(acc_b)
            : "r"(packed));
      } else {
        uint64_t pr = p;
        if (kRoundedSum) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&packed));
          pr = f2_pack(f.x, f.y);
        }
        acc = f2_add(acc, pr);
      }
    }
    if (kRoundedSum && !kF16) acc = f2_pack(acc_a, acc_b);
    if (c < 2) acc_lo = f2_add(acc_lo, acc); else acc_hi = f2_add(acc_hi, acc);
  }
  sum_lo = f2_lo(acc_lo) + f2_hi(acc_lo);
  sum_hi = f2_lo(acc_hi) + f2_hi(acc_hi);
}

// P = exp2(s * c + b) of a 128-key tile with (c, b) per 64-key half,
// packed in place two per word (keys [0,64) into sv[0], [64,128) into
// sv[2]) as bf16 or fp16; no row sum (see sum_packed).
template <bool kF16>
__device__ __forceinline__ void exp_pack_only(uint32_t (&sv)[4][32], float c_lo, float b_lo, float c_hi, float b_hi) {
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
    }
  }
}

// fp32 sum of the 64 bf16 (kF16 = false) or fp16 values packed two per
// word in p[0..31]: the P values exactly as the P.V MMA multiplies V by
// them, so that the row sum and the numerator use one set of weights.
template <bool kF16>
__device__ __forceinline__ float sum_packed(const uint32_t (&p)[32]) {
  float a = 0.f, b = 0.f, c = 0.f, d = 0.f;
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    if (kF16) {
      const float2 x = __half22float2(*reinterpret_cast<const __half2*>(&p[i]));
      const float2 y = __half22float2(*reinterpret_cast<const __half2*>(&p[i + 1]));
      a += x.x; b += x.y; c += y.x; d += y.y;
    } else {
      asm("{\n\t.reg .b16 l0, h0, l1, h1;\n\tmov.b32 {l0, h0}, %4;\n\tmov.b32 {l1, h1}, %5;\n\t"
          "add.rn.f32.bf16 %0, l0, %0;\n\tadd.rn.f32.bf16 %1, h0, %1;\n\t"
          "add.rn.f32.bf16 %2, l1, %2;\n\tadd.rn.f32.bf16 %3, h1, %3;\n\t}"
          : "+f"(a), "+f"(b), "+f"(c), "+f"(d)
          : "r"(p[i]), "r"(p[i + 1]));
    }
  }
  return (a + b) + (c + d);
}

}  // namespace jattn
