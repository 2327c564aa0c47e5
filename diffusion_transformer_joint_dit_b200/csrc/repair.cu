// FP8 attention with a repair budget, for sm_100a: the keys whose E4M3
// quantisation lost the most are attended with their exact K' and V rows.
//
// The NVIDIA tutorial on FLUX 3 Image Klein ("Quantized and sparse
// attention" section) runs VC-Attention FP8 with a repair budget rho that
// selects the fraction of tokens with the highest quantisation error for
// residual correction.  Reading implemented here, per (batch, head):
//   error   e_t = |K'_t - Kd_t|^2 + |V_t - Vd_t|^2 (exact bf16 rows against
//           their dequantised E4M3 values, fp32)            repair_error_kernel
//   select  the m = ceil(rho N) largest e_t, ties to the lower token index,
//           listed in token order (radix select)            repair_select_kernel
//   gather  the exact K' (RMSNorm + RoPE recomputed) and V rows of the
//           selected tokens                                 repair_gather_kernel
//   apply   O and LSE of the FP8 attention corrected as if the selected keys
//           had been attended with their exact rows          repair_apply_kernel
// The correction of a query row with FP8 log-sum-exp L and output O:
//   a = sum_T exp(s_x - L) v_x - exp(s_q - L) v_q,  z = sum_T exp(s_x - L) - exp(s_q - L)
//   O' = (O + a) / (1 + z),  L' = L + ln(1 + z)
// with s_x = scale * qd . k'_t and s_q = scale * qd . kd_t.  The products run
// on the tensor cores (mma.sync m16n8k16, FP16 operands: E4M3 codes and the
// bf16 rows are exact in FP16 over the range they take, fp32 accumulate);
// the budget is small (85 keys at N = 16896), so this pass is short.
#include "jattn_internal.h"
#include "sm100_ptx.cuh"

namespace jattn {

namespace repair {

constexpr int kD = 128;

__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
  const __half2_raw r = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two & 0xFFFFu), __NV_E4M3);
  return static_cast<uint32_t>(r.x) | (static_cast<uint32_t>(r.y) << 16);
}

// 8 E4M3 codes (little-endian in a uint2) -> 8 floats.
__device__ __forceinline__ void e4m3x8_to_float(uint2 c, float (&x)[8]) {
  const uint32_t w[2] = {c.x, c.y};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint32_t lo = e4m3x2_to_f16x2(w[i]), hi = e4m3x2_to_f16x2(w[i] >> 16);
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&lo));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&hi));
    x[4 * i] = a.x; x[4 * i + 1] = a.y; x[4 * i + 2] = b.x; x[4 * i + 3] = b.y;
  }
}

__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
  const float2 f = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  const __half2 h = __floats2half2_rn(f.x, f.y);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// ------------------------------------------------------ 1. token errors ----
// One warp per (b, token); a half-warp per (token, head) row (lane: 8
// channels), two heads per pass, as in the BF16 prologue.
constexpr int kErrWarps = 8;

__global__ void __launch_bounds__(kErrWarps * 32)
repair_error_kernel(const __grid_constant__ PrologueArgs a, const uint8_t* __restrict__ k8,
                    const uint8_t* __restrict__ v8, const float* __restrict__ ks, const float* __restrict__ vs,
                    float* __restrict__ err) {
  const int lane = threadIdx.x & 31;
  const long long token = static_cast<long long>(blockIdx.x) * kErrWarps + (threadIdx.x >> 5);
  if (token >= static_cast<long long>(a.B) * a.N) return;  // whole warp
  const int b = static_cast<int>(token / a.N);
  const int t = static_cast<int>(token - static_cast<long long>(b) * a.N);
  const int half = lane >> 4, l16 = lane & 15, axis = l16 >> 3, pair0 = (l16 & 7) * 4;
  const int nblk = (a.N + kQuantBlock - 1) / kQuantBlock;
  int row, col;
  token_pos(a, t, row, col);
  float c[4], s[4];
  lane_rotations(a, axis == 0 ? row : col, pair0, c, s);
  float wk[8];
  load_weights(a.k_w, l16, wk);
  for (int h0 = 0; h0 < a.H; h0 += 2) {
    const int h = min(h0 + half, a.H - 1);     // both halves run the shuffles
    const size_t r = static_cast<size_t>(token) * a.H + h;
    const uint4 kraw = __ldg(reinterpret_cast<const uint4*>(a.k) + r * 16 + l16);
    const uint4 vraw = __ldg(reinterpret_cast<const uint4*>(a.v) + r * 16 + l16);
    const uint2 kc = __ldg(reinterpret_cast<const uint2*>(k8) + r * 16 + l16);
    const uint2 vc = __ldg(reinterpret_cast<const uint2*>(v8) + r * 16 + l16);
    const float ksc = __ldg(ks + (static_cast<size_t>(b) * a.H + h) * nblk + t / kQuantBlock);
    const float vsc = __ldg(vs + (static_cast<size_t>(b) * a.H + h) * nblk + t / kQuantBlock);
    float kx[8], vx[8], kq[8], vq[8];
    unpack8(norm_rope_row(kraw, wk, c, s, a.eps), kx);  // the bf16 K' the prologue quantises
    unpack8(vraw, vx);
    e4m3x8_to_float(kc, kq);
    e4m3x8_to_float(vc, vq);
    float e = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float dk = kx[i] - kq[i] * ksc, dv = vx[i] - vq[i] * vsc;
      e = fmaf(dk, dk, e);
      e = fmaf(dv, dv, e);
    }
    e += __shfl_xor_sync(0xffffffffu, e, 1);
    e += __shfl_xor_sync(0xffffffffu, e, 2);
    e += __shfl_xor_sync(0xffffffffu, e, 4);
    e += __shfl_xor_sync(0xffffffffu, e, 8);
    if (l16 == 0 && h0 + half < a.H) err[(static_cast<size_t>(b) * a.H + h) * a.N + t] = e;
  }
}

// ------------------------------------------------------ 2. top-m select ----
// One CTA per (b, h).  Errors are >= 0, so their bit patterns order like
// unsigned integers: four 8-bit radix passes find the m-th largest value
// theta and how many tokens equal to theta are taken (the first ones in
// token order); a block-wide scan then lists the selected tokens in order.
constexpr int kSelThreads = 512;

__device__ __forceinline__ unsigned block_excl_scan(unsigned flag, unsigned* warp_tot, unsigned& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, flag != 0u);
  const unsigned within = __popc(bal & ((1u << lane) - 1u));
  __syncthreads();
  if (lane == 0) warp_tot[warp] = __popc(bal);
  __syncthreads();
  unsigned before = 0, all = 0;
  for (int w = 0; w < kSelThreads / 32; ++w) {
    const unsigned n = warp_tot[w];
    before += w < warp ? n : 0u;
    all += n;
  }
  total = all;
  return before + within;
}

__global__ void __launch_bounds__(kSelThreads)
repair_select_kernel(const float* __restrict__ err, int N, int m, int* __restrict__ idx) {
  __shared__ unsigned hist[256];
  __shared__ unsigned s_prefix, s_k;
  __shared__ unsigned warp_tot[kSelThreads / 32];
  const int bh = blockIdx.y * gridDim.x + blockIdx.x;  // (b, h) row of err / idx
  const float* e = err + static_cast<size_t>(bh) * N;
  int* out = idx + static_cast<size_t>(bh) * m;
  unsigned prefix = 0, mask = 0, k = static_cast<unsigned>(m);
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    for (int t = threadIdx.x; t < N; t += kSelThreads) {
      const unsigned u = __float_as_uint(__ldg(e + t));
      if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      unsigned cum = 0, dsel = 0, kk = k;
      for (int d = 255; d >= 0; --d) {
        if (cum + hist[d] >= k) {
          dsel = static_cast<unsigned>(d);
          kk = k - cum;
          break;
        }
        cum += hist[d];
      }
      s_prefix = prefix | (dsel << shift);
      s_k = kk;
    }
    __syncthreads();
    prefix = s_prefix;
    k = s_k;
    mask |= 255u << shift;
  }
  const unsigned theta = prefix, take_eq = k;  // m-th largest value; ties of it to take
  unsigned eq_seen = 0, written = 0;
  for (int t0 = 0; t0 < N; t0 += kSelThreads) {
    const int t = t0 + threadIdx.x;
    const unsigned u = t < N ? __float_as_uint(__ldg(e + t)) : 0u;
    const bool gt = t < N && u > theta;
    const bool eq = t < N && u == theta;
    unsigned eq_total;
    const unsigned eq_rank = block_excl_scan(eq ? 1u : 0u, warp_tot, eq_total);
    const bool sel = gt || (eq && eq_seen + eq_rank < take_eq);
    unsigned sel_total;
    const unsigned pos = block_excl_scan(sel ? 1u : 0u, warp_tot, sel_total);
    if (sel) out[written + pos] = t;
    eq_seen += eq_total;
    written += sel_total;
  }
}

// ---------------------------------------------------------- 3. gather ----
// Half-warp per selected (b, h, i) row: exact K' (RMSNorm + RoPE of the raw
// K row, bf16) and the raw V row.
__global__ void __launch_bounds__(256)
repair_gather_kernel(const __grid_constant__ PrologueArgs a, const int* __restrict__ idx, int m,
                     __nv_bfloat16* __restrict__ k_sel, __nv_bfloat16* __restrict__ v_sel) {
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(a.B) * a.H * m;
  const long long r0 = (static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5)) * 2;
  if (r0 >= rows) return;  // whole warp
  const int half = lane >> 4, l16 = lane & 15, axis = l16 >> 3, pair0 = (l16 & 7) * 4;
  const long long r = min(r0 + half, rows - 1);  // both halves run the shuffles
  const int i = static_cast<int>(r % m);
  const long long bh = r / m;
  const int h = static_cast<int>(bh % a.H), b = static_cast<int>(bh / a.H);
  const int t = __ldg(idx + bh * m + i);
  int row, col;
  token_pos(a, t, row, col);
  float c[4], s[4];
  lane_rotations(a, axis == 0 ? row : col, pair0, c, s);
  float wk[8];
  load_weights(a.k_w, l16, wk);
  const size_t src = (static_cast<size_t>(b) * a.N + t) * a.H + h;
  const uint4 kraw = __ldg(reinterpret_cast<const uint4*>(a.k) + src * 16 + l16);
  const uint4 vraw = __ldg(reinterpret_cast<const uint4*>(a.v) + src * 16 + l16);
  const uint4 ky = norm_rope_row(kraw, wk, c, s, a.eps);
  if (r0 + half < rows) {
    reinterpret_cast<uint4*>(k_sel)[r * 16 + l16] = ky;
    reinterpret_cast<uint4*>(v_sel)[r * 16 + l16] = vraw;
  }
}

// ----------------------------------------------------------- 4. apply ----
// CTA = 8 warps x 16 query rows = 128 query rows (two FP8 scale blocks) per
// pass.  The selected keys are staged in shared memory as FP16, up to
// kStageMax at a time: when they all fit, a CTA stages them once and walks a
// run of passes (about one CTA per SM over the grid); otherwise each CTA
// takes one pass and restages per group of kStageMax keys.
constexpr int kApplyWarps = 8;
constexpr int kApplyQ = kApplyWarps * 16;  // query rows per pass
constexpr int kStageMax = 128;             // selected keys staged at a time
constexpr int kKStride = kD + 8;         // fp16 per K row (bank-conflict padding)
constexpr int kVStride = kStageMax + 8;  // fp16 per transposed V row

struct ApplySmem {
  uint8_t q[kApplyQ][kD];                // Q codes of the current query block
  __half kx[kStageMax][kKStride];        // exact K' (fp16)
  __half kq[kStageMax][kKStride];        // K codes (fp16)
  __half vx[kD][kVStride];               // exact V, transposed
  __half vq[kD][kVStride];               // V codes, transposed
  float ks[kStageMax], vs[kStageMax];
};
constexpr int kApplySmemBytes = static_cast<int>(sizeof(ApplySmem)) + 128;

struct ApplyParams {
  const uint8_t* q8;
  const float* q_scale;
  const uint8_t* k8;
  const uint8_t* v8;
  const float* k_scale;
  const float* v_scale;
  const int* idx;
  const __nv_bfloat16* k_sel;
  const __nv_bfloat16* v_sel;
  __nv_bfloat16* o;
  float* lse;
  int H, N, m;
  int passes_per_cta;
  float scale_log2;
};

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Stage selected keys [i0, i0 + n) of (b, h) into shared memory (FP16),
// zero-padding up to a multiple of 32.
__device__ __forceinline__ void stage_keys(const ApplyParams& p, ApplySmem& sm, int b, int h, size_t bh, int nblk,
                                           int i0, int n) {
  const int n32 = (n + 31) & ~31;
  for (int e = threadIdx.x; e < n32 * (kD / 8); e += blockDim.x) {
    const int i = e / (kD / 8), c8 = (e % (kD / 8)) * 8;
    uint4 kx = make_uint4(0, 0, 0, 0), vx = kx;
    uint2 kc = make_uint2(0, 0), vc = kc;
    if (i < n) {
      const size_t sr = (bh * p.m + i0 + i) * kD + c8;
      kx = __ldg(reinterpret_cast<const uint4*>(p.k_sel + sr));
      vx = __ldg(reinterpret_cast<const uint4*>(p.v_sel + sr));
      const int t = __ldg(p.idx + bh * p.m + i0 + i);
      const size_t cr = ((static_cast<size_t>(b) * p.N + t) * p.H + h) * kD + c8;
      kc = __ldg(reinterpret_cast<const uint2*>(p.k8 + cr));
      vc = __ldg(reinterpret_cast<const uint2*>(p.v8 + cr));
      if (c8 == 0) {
        sm.ks[i] = __ldg(p.k_scale + bh * nblk + t / kQuantBlock);
        sm.vs[i] = __ldg(p.v_scale + bh * nblk + t / kQuantBlock);
      }
    } else if (c8 == 0) {
      sm.ks[i] = 0.f;
      sm.vs[i] = 0.f;
    }
    const uint32_t kxw[4] = {kx.x, kx.y, kx.z, kx.w}, vxw[4] = {vx.x, vx.y, vx.z, vx.w};
    const uint32_t kcw[2] = {kc.x, kc.y}, vcw[2] = {vc.x, vc.y};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      *reinterpret_cast<uint32_t*>(&sm.kx[i][c8 + 2 * j]) = bf16x2_to_f16x2(kxw[j]);
      *reinterpret_cast<uint32_t*>(&sm.kq[i][c8 + 2 * j]) = e4m3x2_to_f16x2(kcw[j >> 1] >> (16 * (j & 1)));
      const uint32_t v2 = bf16x2_to_f16x2(vxw[j]);
      const uint32_t vq2 = e4m3x2_to_f16x2(vcw[j >> 1] >> (16 * (j & 1)));
      sm.vx[c8 + 2 * j][i] = *reinterpret_cast<const __half*>(&v2);
      sm.vx[c8 + 2 * j + 1][i] = *(reinterpret_cast<const __half*>(&v2) + 1);
      sm.vq[c8 + 2 * j][i] = *reinterpret_cast<const __half*>(&vq2);
      sm.vq[c8 + 2 * j + 1][i] = *(reinterpret_cast<const __half*>(&vq2) + 1);
    }
  }
}

__global__ void __launch_bounds__(kApplyWarps * 32, 1)
repair_apply_kernel(const __grid_constant__ ApplyParams p) {
  extern __shared__ uint8_t smem_raw[];
  ApplySmem& sm = *reinterpret_cast<ApplySmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tq = lane & 3;
  const int h = blockIdx.y, b = blockIdx.z;
  const int N = p.N, H = p.H, m = p.m;
  const int nblk = (N + kQuantBlock - 1) / kQuantBlock;
  const size_t bh = static_cast<size_t>(b) * H + h;
  const bool staged_once = m <= kStageMax;
  const int npass = (N + kApplyQ - 1) / kApplyQ;
  const int qb0 = blockIdx.x * p.passes_per_cta;
  const int qb1 = min(qb0 + p.passes_per_cta, npass);
  const float log2e = 1.4426950408889634f;

  if (staged_once) {
    stage_keys(p, sm, b, h, bh, nblk, 0, m);
    __syncthreads();
  }
#pragma unroll 1
  for (int qb = qb0; qb < qb1; ++qb) {
    const int q0 = qb * kApplyQ;
    __syncthreads();  // previous block's readers of sm.q are done
    for (int e = threadIdx.x; e < kApplyQ * (kD / 16); e += blockDim.x) {
      const int rr = e / (kD / 16), cc = e % (kD / 16);
      const int q = q0 + rr;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (q < N) v = __ldg(reinterpret_cast<const uint4*>(p.q8 + ((static_cast<size_t>(b) * N + q) * H + h) * kD) + cc);
      *reinterpret_cast<uint4*>(&sm.q[rr][cc * 16]) = v;
    }
    __syncthreads();
    // A fragments (this warp's 16 query rows x 128 channels), FP16 codes.
    uint32_t qa[kD / 16][4];
    {
      const int ra = warp * 16 + g, rb = ra + 8;
#pragma unroll
      for (int ks = 0; ks < kD / 16; ++ks) {
        const int c0 = ks * 16 + 2 * tq;
        qa[ks][0] = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(&sm.q[ra][c0]));
        qa[ks][1] = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(&sm.q[rb][c0]));
        qa[ks][2] = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(&sm.q[ra][c0 + 8]));
        qa[ks][3] = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(&sm.q[rb][c0 + 8]));
      }
    }
    const float qsc = __ldg(p.q_scale + bh * nblk + (q0 + warp * 16) / kQuantBlock);
    const int row_a = q0 + warp * 16 + g, row_b = row_a + 8;
    const float l2a = row_a < N ? p.lse[bh * N + row_a] * log2e : 0.f;
    const float l2b = row_b < N ? p.lse[bh * N + row_b] * log2e : 0.f;
    const float sx = qsc * p.scale_log2;
    float acc[kD / 8][4];
#pragma unroll
    for (int n = 0; n < kD / 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    float za = 0.f, zb = 0.f;  // sum exp(s_x - L) - exp(s_q - L), rows a, b

#pragma unroll 1
    for (int s0 = 0; s0 < m; s0 += kStageMax) {
      const int ns = min(kStageMax, m - s0);
      if (!staged_once) {
        __syncthreads();
        stage_keys(p, sm, b, h, bh, nblk, s0, ns);
        __syncthreads();
      }
#pragma unroll 1
      for (int c0k = 0; c0k < ns; c0k += 32) {
        uint32_t wa[4][4];  // A fragments of [w_x (32 keys) | -w_q (32 keys)]
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
          float cx[4] = {0.f, 0.f, 0.f, 0.f}, cq[4] = {0.f, 0.f, 0.f, 0.f};
          const int key = c0k + nt * 8 + g;  // B column of this lane
#pragma unroll
          for (int ks = 0; ks < kD / 16; ++ks) {
            const int cc = ks * 16 + 2 * tq;
            mma16816(cx, qa[ks], *reinterpret_cast<const uint32_t*>(&sm.kx[key][cc]),
                     *reinterpret_cast<const uint32_t*>(&sm.kx[key][cc + 8]));
            mma16816(cq, qa[ks], *reinterpret_cast<const uint32_t*>(&sm.kq[key][cc]),
                     *reinterpret_cast<const uint32_t*>(&sm.kq[key][cc + 8]));
          }
          float wx[4], wq[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int kk = c0k + nt * 8 + 2 * tq + (j & 1);
            const bool live = kk < ns;
            const float l2 = j < 2 ? l2a : l2b;
            wx[j] = live ? ex2_approx(cx[j] * sx - l2) : 0.f;
            wq[j] = live ? ex2_approx(cq[j] * (sx * sm.ks[kk]) - l2) : 0.f;
            if (j < 2) za += wx[j] - wq[j]; else zb += wx[j] - wq[j];
            wq[j] *= sm.vs[kk];  // V's block scale folded into the weight
          }
          const int kstep = nt >> 1, hi = nt & 1;
          wa[kstep][2 * hi] = pack_h2(wx[0], wx[1]);
          wa[kstep][2 * hi + 1] = pack_h2(wx[2], wx[3]);
          wa[2 + kstep][2 * hi] = pack_h2(-wq[0], -wq[1]);
          wa[2 + kstep][2 * hi + 1] = pack_h2(-wq[2], -wq[3]);
        }
        // acc += [w_x | -w_q] [V_x ; V_q]
#pragma unroll
        for (int n = 0; n < kD / 8; ++n) {
          const int dcol = n * 8 + g;
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const __half(*vt)[kVStride] = k4 < 2 ? sm.vx : sm.vq;
            const int kb = c0k + (k4 & 1) * 16 + 2 * tq;
            mma16816(acc[n], wa[k4], *reinterpret_cast<const uint32_t*>(&vt[dcol][kb]),
                     *reinterpret_cast<const uint32_t*>(&vt[dcol][kb + 8]));
          }
        }
      }
    }

    // Row sums over the quad, then O' = (O + a) / (1 + z), L' = L + ln(1 + z).
    za += __shfl_xor_sync(0xffffffffu, za, 1);
    za += __shfl_xor_sync(0xffffffffu, za, 2);
    zb += __shfl_xor_sync(0xffffffffu, zb, 1);
    zb += __shfl_xor_sync(0xffffffffu, zb, 2);
    const float ia = 1.f / (1.f + za), ib = 1.f / (1.f + zb);
#pragma unroll
    for (int n = 0; n < kD / 8; ++n) {
      const int c = n * 8 + 2 * tq;
      if (row_a < N) {
        __nv_bfloat162* o2 =
            reinterpret_cast<__nv_bfloat162*>(p.o + ((static_cast<size_t>(b) * N + row_a) * H + h) * kD + c);
        const float2 f = __bfloat1622float2(*o2);
        *o2 = __floats2bfloat162_rn((f.x + acc[n][0]) * ia, (f.y + acc[n][1]) * ia);
      }
      if (row_b < N) {
        __nv_bfloat162* o2 =
            reinterpret_cast<__nv_bfloat162*>(p.o + ((static_cast<size_t>(b) * N + row_b) * H + h) * kD + c);
        const float2 f = __bfloat1622float2(*o2);
        *o2 = __floats2bfloat162_rn((f.x + acc[n][2]) * ib, (f.y + acc[n][3]) * ib);
      }
    }
    if (tq == 0) {
      if (row_a < N) p.lse[bh * N + row_a] += __logf(1.f + za);
      if (row_b < N) p.lse[bh * N + row_b] += __logf(1.f + zb);
    }
  }
}

}  // namespace repair

cudaError_t launch_repair_select(const PrologueArgs& a, const RepairProblem& r, cudaStream_t s) {
  using namespace repair;
  const long long tokens = static_cast<long long>(a.B) * a.N;
  repair_error_kernel<<<static_cast<unsigned>((tokens + kErrWarps - 1) / kErrWarps), kErrWarps * 32, 0, s>>>(
      a, static_cast<const uint8_t*>(r.k8), static_cast<const uint8_t*>(r.v8), r.k_scale, r.v_scale, r.err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || r.m == 0) return e;
  repair_select_kernel<<<dim3(a.H, a.B), kSelThreads, 0, s>>>(r.err, a.N, r.m, r.idx);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const long long rows = static_cast<long long>(a.B) * a.H * r.m;
  repair_gather_kernel<<<static_cast<unsigned>((rows + 15) / 16), 256, 0, s>>>(
      a, r.idx, r.m, static_cast<__nv_bfloat16*>(r.k_sel), static_cast<__nv_bfloat16*>(r.v_sel));
  return cudaGetLastError();
}

cudaError_t launch_repair_apply(const RepairProblem& r, int B, int H, int N, float softmax_scale, cudaStream_t s) {
  using namespace repair;
  if (r.m == 0) return cudaSuccess;
  ApplyParams p;
  p.q8 = static_cast<const uint8_t*>(r.q8);
  p.q_scale = r.q_scale;
  p.k8 = static_cast<const uint8_t*>(r.k8);
  p.v8 = static_cast<const uint8_t*>(r.v8);
  p.k_scale = r.k_scale;
  p.v_scale = r.v_scale;
  p.idx = r.idx;
  p.k_sel = static_cast<const __nv_bfloat16*>(r.k_sel);
  p.v_sel = static_cast<const __nv_bfloat16*>(r.v_sel);
  p.o = static_cast<__nv_bfloat16*>(r.o);
  p.lse = r.lse;
  p.H = H;
  p.N = N;
  p.m = r.m;
  // Keys staged once: about one CTA per SM, each walking a run of passes.
  const int npass = (N + kApplyQ - 1) / kApplyQ;
  int per_head = 1;
  if (r.m <= kStageMax) per_head = std::max(1, std::min(npass, device_sm_count() / std::max(1, B * H)));
  p.passes_per_cta = r.m <= kStageMax ? (npass + per_head - 1) / per_head : 1;
  p.scale_log2 = static_cast<float>(static_cast<double>(softmax_scale) * 1.4426950408889634074);
  cudaError_t e = set_smem_attr(reinterpret_cast<const void*>(repair_apply_kernel), kApplySmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((npass + p.passes_per_cta - 1) / p.passes_per_cta, H, B);
  repair_apply_kernel<<<grid, kApplyWarps * 32, kApplySmemBytes, s>>>(p);
  return cudaGetLastError();
}

}  // namespace jattn
