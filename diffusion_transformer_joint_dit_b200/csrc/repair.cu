// FP8 attention with a repair budget, for sm_100a: the keys whose E4M3
// quantisation lost the most are attended with their exact K' and V rows.
//
// The NVIDIA tutorial on FLUX 3 Image Klein ("Quantized and sparse
// attention" section) runs VC-Attention FP8 with a repair budget rho: a
// share rho of the tokens, those that quantisation hurt most, gets a
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
// on the tensor cores (tcgen05, TMEM accumulators; E4M3 codes and the bf16
// rows are exact in FP16 over the range they take); the budget is small (85
// keys at N = 16896), so this pass is short.
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
// token order); the warps then list the selected tokens of their token
// segments in order.
constexpr int kSelThreads = 512;

__global__ void __launch_bounds__(kSelThreads)
repair_select_kernel(const float* __restrict__ err, int N, int m, int* __restrict__ idx) {
  __shared__ unsigned hist[256];
  __shared__ unsigned s_prefix, s_k;
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
    if (threadIdx.x < 32) {
      // The digit d with count(digits > d) < k <= count(digits >= d): lane l
      // holds digits 8 l .. 8 l + 7; suffix sums over the lanes find the
      // lane that holds d, which then walks its eight counts.
      const int lane = threadIdx.x;
      unsigned c[8], tot = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c[i] = hist[lane * 8 + i];
        tot += c[i];
      }
      unsigned incl = tot;  // digits >= 8 lane
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned v = __shfl_down_sync(0xffffffffu, incl, o);
        if (lane + o < 32) incl += v;
      }
      unsigned cum = incl - tot;  // digits > 8 lane + 7
      if (cum < k && k <= incl) {
        unsigned dsel = 0, kk = k;
#pragma unroll
        for (int i = 7; i >= 0; --i) {
          if (cum + c[i] >= k) {
            dsel = static_cast<unsigned>(lane * 8 + i);
            kk = k - cum;
            break;
          }
          cum += c[i];
        }
        s_prefix = prefix | (dsel << shift);
        s_k = kk;
      }
    }
    __syncthreads();
    prefix = s_prefix;
    k = s_k;
    mask |= 255u << shift;
  }
  const unsigned theta = prefix, take_eq = k;  // m-th largest value; ties of it to take
  // Listing: warp w owns the contiguous token segment [w seg, (w + 1) seg).
  // One counting sweep, one barrier for the per-warp counts, then each warp
  // writes its selected tokens in order with ballots.
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int kWarps = kSelThreads / 32;
  __shared__ unsigned s_gt[kWarps], s_eq[kWarps];
  const int seg = (N + kWarps - 1) / kWarps;
  const int s0 = min(N, warp * seg), s1 = min(N, s0 + seg);
  unsigned n_gt = 0, n_eq = 0;
  for (int base = s0; base < s1; base += 32) {
    const int t = base + lane;
    const unsigned u = t < s1 ? __float_as_uint(__ldg(e + t)) : 0u;
    n_gt += __popc(__ballot_sync(0xffffffffu, t < s1 && u > theta));
    n_eq += __popc(__ballot_sync(0xffffffffu, t < s1 && u == theta));
  }
  if (lane == 0) {
    s_gt[warp] = n_gt;
    s_eq[warp] = n_eq;
  }
  __syncthreads();
  unsigned written = 0, eq_seen = 0;  // selected tokens and ties of theta before this warp's segment
  for (int w = 0; w < warp; ++w) {
    const unsigned eq_take = eq_seen < take_eq ? min(s_eq[w], take_eq - eq_seen) : 0u;
    written += s_gt[w] + eq_take;
    eq_seen += s_eq[w];
  }
  const unsigned below = (1u << lane) - 1u;
  for (int base = s0; base < s1; base += 32) {
    const int t = base + lane;
    const unsigned u = t < s1 ? __float_as_uint(__ldg(e + t)) : 0u;
    const bool gt = t < s1 && u > theta;
    const bool eq = t < s1 && u == theta;
    const unsigned eq_bal = __ballot_sync(0xffffffffu, eq);
    const bool sel = gt || (eq && eq_seen + __popc(eq_bal & below) < take_eq);
    const unsigned sel_bal = __ballot_sync(0xffffffffu, sel);
    if (sel) out[written + __popc(sel_bal & below)] = t;
    written += __popc(sel_bal);
    eq_seen += __popc(eq_bal);
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
// tcgen05 correction pass.  CTA = 4 warps; a pass covers 128 query rows, one
// per thread and TMEM lane.  The selected keys of the (b, h) (up to
// kStageMax per group, padded to P, a multiple of 32) sit in shared memory
// in the 128-byte-swizzled layouts the MMAs read:
//   Kx16  exact K' as FP16, K-major (two 64-channel boxes of P rows)
//   Kq8   K codes (E4M3), K-major (one box of P rows)
//   V16   [exact V ; V codes] as FP16, MN-major (two 64-channel boxes of 2P rows)
// Per pass the Q codes land twice, as an E4M3 tile and widened to FP16, and
// one thread issues
//   S_x = Q16 . Kx16^T  (kind::f16)                 -> TMEM [0, P)
//   S_q = Q8  . Kq8^T   (kind::f8f6f4)              -> TMEM [128, 128 + P)
// each thread turns its row into W = [w_x | -w_q s_v] (FP16 pairs, TMEM
// [384, 384 + P)) and z, and then
//   O_c = W . V16       (kind::f16, A from TMEM)    -> TMEM [256, 384)
// after which the thread rewrites its O and L rows.  With more than
// kStageMax selected keys, the groups run one after another inside a pass,
// accumulating O_c and z.  With one group (the keys staged once) the passes
// are pipelined: the next pass's S MMAs follow this pass's P.V in issue
// order and run during its epilogue.  Exact K' and V rows must lie within
// the FP16 range (E4M3 codes and bf16 rows of moderate size are exact in
// FP16).
constexpr int kApplyThreads = 128;
constexpr int kApplyQ = 128;            // query rows per pass (= TMEM lanes)
constexpr int kStageMax = 128;          // selected keys per group
constexpr uint32_t kColSx = 0, kColSq = 128, kColO = 256, kColW = 384;
constexpr uint32_t kApplyTmemCols = 512;

struct ApplyCtrl {
  uint64_t s_full;
  uint64_t o_full;
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

constexpr int kSmQ8 = 0;                              // 128 rows x 128 B
constexpr int kSmQ16 = kSmQ8 + kApplyQ * 128;         // 2 boxes x 128 rows x 128 B
constexpr int kSmKx = kSmQ16 + 2 * kApplyQ * 128;     // 2 boxes x P rows x 128 B
constexpr int kSmKq = kSmKx + 2 * kStageMax * 128;    // P rows x 128 B
constexpr int kSmV = kSmKq + kStageMax * 128;         // 2 boxes x 2P rows x 128 B
constexpr int kSmCtrl = kSmV + 4 * kStageMax * 128;
constexpr int kApplySmemBytes = kSmCtrl + static_cast<int>(sizeof(ApplyCtrl)) + 1024;

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
  uint64_t timeout_ns;
};

// Byte offset of 16-byte chunk `chunk` of row `r` in a 128-byte-swizzled
// tile (rows of 128 B, 1024-byte aligned base).
__device__ __forceinline__ uint32_t sw128(int r, int chunk) {
  return static_cast<uint32_t>(r * 128 + ((chunk ^ (r & 7)) << 4));
}

// 8 bf16 -> 8 FP16 (exact for moderate magnitudes).
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 v) {
  return make_uint4(bf16x2_to_f16x2(v.x), bf16x2_to_f16x2(v.y), bf16x2_to_f16x2(v.z), bf16x2_to_f16x2(v.w));
}

// 16 E4M3 codes -> 16 FP16 values (exact), as two 16-byte chunks.
__device__ __forceinline__ void e4m3x16_to_f16(uint4 c, uint4& lo, uint4& hi) {
  lo = make_uint4(e4m3x2_to_f16x2(c.x), e4m3x2_to_f16x2(c.x >> 16), e4m3x2_to_f16x2(c.y),
                  e4m3x2_to_f16x2(c.y >> 16));
  hi = make_uint4(e4m3x2_to_f16x2(c.z), e4m3x2_to_f16x2(c.z >> 16), e4m3x2_to_f16x2(c.w),
                  e4m3x2_to_f16x2(c.w >> 16));
}

// Stage selected keys [i0, i0 + ns) of (b, h), zero-padded to P rows.
__device__ __forceinline__ void apply_stage_keys(const ApplyParams& p, uint8_t* sm, float* s_ks, float* s_vs, int b,
                                                 int h, size_t bh, int nblk, int i0, int ns, int P) {
#pragma unroll 4
  for (int e = threadIdx.x; e < P * 16; e += kApplyThreads) {  // exact rows: 8 channels per task
    const int i = e >> 4, c8 = e & 15;
    uint4 kx = make_uint4(0, 0, 0, 0), vx = kx;
    if (i < ns) {
      const size_t sr = (bh * p.m + i0 + i) * kD + c8 * 8;
      kx = __ldg(reinterpret_cast<const uint4*>(p.k_sel + sr));
      vx = __ldg(reinterpret_cast<const uint4*>(p.v_sel + sr));
    }
    const int box = c8 >> 3, ch = c8 & 7;
    *reinterpret_cast<uint4*>(sm + kSmKx + box * P * 128 + sw128(i, ch)) = bf16x8_to_f16x8(kx);
    *reinterpret_cast<uint4*>(sm + kSmV + box * 2 * P * 128 + sw128(i, ch)) = bf16x8_to_f16x8(vx);
  }
#pragma unroll 3
  for (int e = threadIdx.x; e < P * 8; e += kApplyThreads) {   // codes: 16 channels per task
    const int i = e >> 3, c16 = e & 7;
    uint4 kc = make_uint4(0, 0, 0, 0), vc = kc;
    float ksc = 0.f, vsc = 0.f;
    if (i < ns) {
      const int t = min(max(__ldg(p.idx + bh * p.m + i0 + i), 0), p.N - 1);  // in range for any list
      const size_t cr = ((static_cast<size_t>(b) * p.N + t) * p.H + h) * kD + c16 * 16;
      kc = __ldg(reinterpret_cast<const uint4*>(p.k8 + cr));
      vc = __ldg(reinterpret_cast<const uint4*>(p.v8 + cr));
      ksc = __ldg(p.k_scale + bh * nblk + t / kQuantBlock);
      vsc = __ldg(p.v_scale + bh * nblk + t / kQuantBlock);
    }
    *reinterpret_cast<uint4*>(sm + kSmKq + sw128(i, c16)) = kc;
    uint4 lo, hi;
    e4m3x16_to_f16(vc, lo, hi);
    uint8_t* vbox = sm + kSmV + (c16 >> 2) * 2 * P * 128;
    const int c8 = (c16 & 3) * 2;
    *reinterpret_cast<uint4*>(vbox + sw128(P + i, c8)) = lo;
    *reinterpret_cast<uint4*>(vbox + sw128(P + i, c8 + 1)) = hi;
    if (c16 == 0) {
      s_ks[i] = ksc;
      s_vs[i] = vsc;
    }
  }
}

// This thread's 8 chunks of the pass's Q codes (zero past N): task e =
// thread + 128 k, row e / 8, chunk e % 8.
__device__ __forceinline__ void apply_load_q(const ApplyParams& p, int b, int h, int q0, uint4 (&qn)[8]) {
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int e = threadIdx.x + k * kApplyThreads;
    const int row = q0 + (e >> 3);
    qn[k] = make_uint4(0, 0, 0, 0);
    if (row < p.N)
      qn[k] = __ldg(reinterpret_cast<const uint4*>(p.q8 + ((static_cast<size_t>(b) * p.N + row) * p.H + h) * kD) +
                    (e & 7));
  }
}

__device__ __forceinline__ void apply_store_q(uint8_t* sm, const uint4 (&qn)[8]) {
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int e = threadIdx.x + k * kApplyThreads;
    const int r = e >> 3, c16 = e & 7;
    *reinterpret_cast<uint4*>(sm + kSmQ8 + sw128(r, c16)) = qn[k];
    uint4 lo, hi;
    e4m3x16_to_f16(qn[k], lo, hi);
    uint8_t* qbox = sm + kSmQ16 + (c16 >> 2) * kApplyQ * 128;
    const int c8 = (c16 & 3) * 2;
    *reinterpret_cast<uint4*>(qbox + sw128(r, c8)) = lo;
    *reinterpret_cast<uint4*>(qbox + sw128(r, c8 + 1)) = hi;
  }
}

__global__ void __launch_bounds__(kApplyThreads, 1)
repair_apply_kernel(const __grid_constant__ ApplyParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ float s_ks[kStageMax], s_vs[kStageMax];  // block scales of the staged keys
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  ApplyCtrl* ctrl = reinterpret_cast<ApplyCtrl*>(sm + kSmCtrl);
  volatile int* abort_flag = &ctrl->abort;
  const int warp = threadIdx.x >> 5;
  const int h = blockIdx.y, b = blockIdx.z;
  const int N = p.N, m = p.m;
  const int nblk = (N + kQuantBlock - 1) / kQuantBlock;
  const size_t bh = static_cast<size_t>(b) * p.H + h;
  const int ngroups = (m + kStageMax - 1) / kStageMax;
  const int npass = (N + kApplyQ - 1) / kApplyQ;
  const int pass0 = blockIdx.x * p.passes_per_cta;
  const int pass1 = min(pass0 + p.passes_per_cta, npass);
  const float log2e = 1.4426950408889634f;

  if (threadIdx.x == 0) {
    mbar_init(&ctrl->s_full, 1);
    mbar_init(&ctrl->o_full, 1);
    mbar_init(&ctrl->mma_done, 1);
    ctrl->abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&ctrl->tmem_base, kApplyTmemCols);
    tmem_relinquish();
  }
  if (ngroups == 1) {
    apply_stage_keys(p, sm, s_ks, s_vs, b, h, bh, nblk, 0, m, (m + 31) & ~31);
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;
  const uint32_t lane_sel = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t idesc_pv = make_idesc(0, 0, true, kApplyQ, kD);  // f16 W (TMEM) x f16 V (MN-major)
  uint32_t s_phase = 0, o_phase = 0;
  bool ok = true;

  // Per-pass inputs of this thread's row, loaded one pass ahead: the Q
  // codes, the row's Q scale and its log-sum-exp.
  uint4 qn[8];
  float qsc_n = 0.f, lse_n = 0.f;
  auto prefetch = [&](int q0) {
    apply_load_q(p, b, h, q0, qn);
    const int r = q0 + static_cast<int>(threadIdx.x);
    qsc_n = r < N ? __ldg(p.q_scale + bh * nblk + r / kQuantBlock) : 0.f;
    lse_n = r < N ? p.lse[bh * N + r] : 0.f;
  };
  if (pass0 < pass1) prefetch(pass0 * kApplyQ);
  if (ngroups == 1) {
    // One key group, staged once: passes are pipelined.  The S MMAs of pass
    // p + 1 are issued right after the P.V MMA of pass p (Q of pass p + 1
    // is staged while W of pass p is formed), so they run during pass p's
    // epilogue; S_x / S_q and W / O_c are separate TMEM regions.
    const int ns = m, P = (m + 31) & ~31;
    auto issue_s = [&]() {
      tc_fence_after();
      const uint32_t idesc_x = make_idesc(0, 0, false, kApplyQ, P);  // f16 x f16, K-major
      const uint32_t idesc_q = make_idesc(0, 0, false, kApplyQ, P);  // e4m3 x e4m3, K-major
      const uint32_t q16 = smem_u32(sm + kSmQ16), kx = smem_u32(sm + kSmKx);
      const uint32_t q8 = smem_u32(sm + kSmQ8), kq = smem_u32(sm + kSmKq);
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk) {
        const uint32_t aoff = (kk >> 2) * (kApplyQ * 128) + (kk & 3) * 32;
        const uint32_t boff = (kk >> 2) * (P * 128) + (kk & 3) * 32;
        mma_f16_ss(tmem + kColSx, smem_desc_sw128(q16 + aoff, 16, 1024), smem_desc_sw128(kx + boff, 16, 1024),
                   idesc_x, kk > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < kD / 32; ++kk)
        mma_f8_ss(tmem + kColSq, smem_desc_sw128(q8 + kk * 32, 16, 1024), smem_desc_sw128(kq + kk * 32, 16, 1024),
                  idesc_q, kk > 0 ? 1u : 0u);
      mma_commit(&ctrl->s_full);
    };
    float cur_qsc = 0.f, cur_lse = 0.f;
    if (pass0 < pass1) {
      apply_store_q(sm, qn);
      fence_proxy_async_smem();
      cur_qsc = qsc_n;
      cur_lse = lse_n;
      if (pass0 + 1 < pass1) prefetch((pass0 + 1) * kApplyQ);
      __syncthreads();
      if (threadIdx.x == 0 && ok) issue_s();
    }
#pragma unroll 1
    for (int pass = pass0; pass < pass1; ++pass) {
      const int q0 = pass * kApplyQ;
      const int row = q0 + threadIdx.x;
      const bool live = row < N;
      const float lse_row = cur_lse;
      const float l2 = lse_row * log2e;
      const float sx = cur_qsc * p.scale_log2;
      float z = 0.f;
      __nv_bfloat16* orow = p.o + ((static_cast<size_t>(b) * N + (live ? row : 0)) * p.H + h) * kD;
      if (ok) ok = mbar_wait(&ctrl->s_full, s_phase & 1u, abort_flag, p.timeout_ns);
      ++s_phase;
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < P; c0 += 32) {
          uint32_t ax[32], aq[32];
          tmem_ld32(tmem + lane_sel + kColSx + c0, ax);
          tmem_ld32(tmem + lane_sel + kColSq + c0, aq);
          tmem_ld_wait(ax);
          tmem_ld_wait(aq);
          uint32_t wx[16], wq[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            float ex[2], eq[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int key = c0 + j + u;
              const bool in = key < ns;
              ex[u] = in ? ex2_approx(__uint_as_float(ax[j + u]) * sx - l2) : 0.f;
              eq[u] = in ? ex2_approx(__uint_as_float(aq[j + u]) * (sx * s_ks[key]) - l2) : 0.f;
              z += ex[u] - eq[u];
              eq[u] *= -s_vs[key];  // V's block scale folded into the weight of the codes
            }
            wx[j >> 1] = pack_f16x2(ex[0], ex[1]);
            wq[j >> 1] = pack_f16x2(eq[0], eq[1]);
          }
          tmem_st16(tmem + lane_sel + kColW + c0 / 2, wx);
          tmem_st16(tmem + lane_sel + kColW + P / 2 + c0 / 2, wq);
        }
        tmem_st_wait();
      }
      // The S MMAs of this pass have completed: the Q buffer takes the next
      // pass's rows.
      float nxt_qsc = 0.f, nxt_lse = 0.f;
      if (pass + 1 < pass1) {
        apply_store_q(sm, qn);
        fence_proxy_async_smem();
        nxt_qsc = qsc_n;
        nxt_lse = lse_n;
      }
      tc_fence_before();
      __syncthreads();  // W of every row in TMEM, S read, next Q staged
      if (threadIdx.x == 0 && ok) {
        tc_fence_after();
        const uint32_t v16 = smem_u32(sm + kSmV);
#pragma unroll 1
        for (int kk = 0; kk < (2 * P) / 16; ++kk)
          mma_f16_ts(tmem + kColO, tmem + kColW + kk * 8, smem_desc_sw128(v16 + kk * 16 * 128, 2 * P * 128, 1024),
                     idesc_pv, kk > 0 ? 1u : 0u);
        mma_commit(&ctrl->o_full);
        if (pass + 1 < pass1) issue_s();  // in issue order after P.V, which read W
      }
      if (pass + 2 < pass1) prefetch((pass + 2) * kApplyQ);  // in flight during the epilogue
      uint4 o_in[kD / 8];
#pragma unroll
      for (int i = 0; i < kD / 8; ++i)
        o_in[i] = live ? *reinterpret_cast<const uint4*>(orow + i * 8) : make_uint4(0, 0, 0, 0);
      if (ok) ok = mbar_wait(&ctrl->o_full, o_phase & 1u, abort_flag, p.timeout_ns);
      ++o_phase;
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        const float inv = 1.f / (1.f + z);
#pragma unroll
        for (int c = 0; c < kD / 32; ++c) {
          uint32_t a[32];
          tmem_ld32(tmem + lane_sel + kColO + c * 32, a);
          tmem_ld_wait(a);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const uint4 ov = o_in[c * 4 + q4];
            const uint32_t w[4] = {ov.x, ov.y, ov.z, ov.w};
            uint32_t r[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float lo = (__uint_as_float(w[i] << 16) + __uint_as_float(a[q4 * 8 + 2 * i])) * inv;
              const float hi = (__uint_as_float(w[i] & 0xFFFF0000u) + __uint_as_float(a[q4 * 8 + 2 * i + 1])) * inv;
              r[i] = pack_bf16x2(lo, hi);
            }
            if (live) *reinterpret_cast<uint4*>(orow + c * 32 + q4 * 8) = make_uint4(r[0], r[1], r[2], r[3]);
          }
        }
        if (live) p.lse[bh * N + row] = lse_row + __logf(1.f + z);
      }
      tc_fence_before();
      __syncthreads();  // O_c read before the next pass's P.V overwrites it
      cur_qsc = nxt_qsc;
      cur_lse = nxt_lse;
    }
  } else
#pragma unroll 1
  for (int pass = pass0; pass < pass1; ++pass) {
    const int q0 = pass * kApplyQ;
    apply_store_q(sm, qn);
    fence_proxy_async_smem();
    const int row = q0 + threadIdx.x;
    const bool live = row < N;
    const float lse_row = lse_n;
    const float l2 = lse_row * log2e;
    const float sx = qsc_n * p.scale_log2;
    float z = 0.f;  // sum over selected keys of exp(s_x - L) - exp(s_q - L)
    __nv_bfloat16* orow = p.o + ((static_cast<size_t>(b) * N + (live ? row : 0)) * p.H + h) * kD;
    uint4 o_in[kD / 8];
#pragma unroll 1
    for (int g = 0; g < ngroups; ++g) {
      const int ns = min(kStageMax, m - g * kStageMax);
      const int P = (ns + 31) & ~31;
      if (ngroups > 1) {
        // The previous group's MMAs have completed (o_full waited below).
        apply_stage_keys(p, sm, s_ks, s_vs, b, h, bh, nblk, g * kStageMax, ns, P);
        fence_proxy_async_smem();
      }
      __syncthreads();  // Q (and keys) written; previous readers of TMEM done
      if (threadIdx.x == 0 && ok) {
        tc_fence_after();
        const uint32_t idesc_x = make_idesc(0, 0, false, kApplyQ, P);  // f16 x f16, K-major
        const uint32_t idesc_q = make_idesc(0, 0, false, kApplyQ, P);  // e4m3 x e4m3, K-major
        const uint32_t q16 = smem_u32(sm + kSmQ16), kx = smem_u32(sm + kSmKx);
        const uint32_t q8 = smem_u32(sm + kSmQ8), kq = smem_u32(sm + kSmKq);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t aoff = (kk >> 2) * (kApplyQ * 128) + (kk & 3) * 32;
          const uint32_t boff = (kk >> 2) * (P * 128) + (kk & 3) * 32;
          mma_f16_ss(tmem + kColSx, smem_desc_sw128(q16 + aoff, 16, 1024), smem_desc_sw128(kx + boff, 16, 1024),
                     idesc_x, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < kD / 32; ++kk)
          mma_f8_ss(tmem + kColSq, smem_desc_sw128(q8 + kk * 32, 16, 1024), smem_desc_sw128(kq + kk * 32, 16, 1024),
                    idesc_q, kk > 0 ? 1u : 0u);
        mma_commit(&ctrl->s_full);
      }
      if (g == 0 && pass + 1 < pass1) prefetch(q0 + kApplyQ);  // next pass, in flight meanwhile
      if (ok) ok = mbar_wait(&ctrl->s_full, s_phase & 1u, abort_flag, p.timeout_ns);
      ++s_phase;
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < P; c0 += 32) {
          uint32_t ax[32], aq[32];
          tmem_ld32(tmem + lane_sel + kColSx + c0, ax);
          tmem_ld32(tmem + lane_sel + kColSq + c0, aq);
          tmem_ld_wait(ax);
          tmem_ld_wait(aq);
          uint32_t wx[16], wq[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            float ex[2], eq[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int key = c0 + j + u;
              const bool in = key < ns;
              ex[u] = in ? ex2_approx(__uint_as_float(ax[j + u]) * sx - l2) : 0.f;
              eq[u] = in ? ex2_approx(__uint_as_float(aq[j + u]) * (sx * s_ks[key]) - l2) : 0.f;
              z += ex[u] - eq[u];
              eq[u] *= -s_vs[key];  // V's block scale folded into the weight of the codes
            }
            wx[j >> 1] = pack_f16x2(ex[0], ex[1]);
            wq[j >> 1] = pack_f16x2(eq[0], eq[1]);
          }
          tmem_st16(tmem + lane_sel + kColW + c0 / 2, wx);
          tmem_st16(tmem + lane_sel + kColW + P / 2 + c0 / 2, wq);
        }
        tmem_st_wait();
      }
      tc_fence_before();
      __syncthreads();  // W of every row is in TMEM
      if (threadIdx.x == 0 && ok) {
        tc_fence_after();
        const uint32_t v16 = smem_u32(sm + kSmV);
#pragma unroll 1
        for (int kk = 0; kk < (2 * P) / 16; ++kk)
          mma_f16_ts(tmem + kColO, tmem + kColW + kk * 8, smem_desc_sw128(v16 + kk * 16 * 128, 2 * P * 128, 1024),
                     idesc_pv, (g > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&ctrl->o_full);
      }
      if (g == ngroups - 1) {
        // This row of O, in flight while the tensor core computes O_c.
#pragma unroll
        for (int i = 0; i < kD / 8; ++i)
          o_in[i] = live ? *reinterpret_cast<const uint4*>(orow + i * 8) : make_uint4(0, 0, 0, 0);
      }
      if (ok) ok = mbar_wait(&ctrl->o_full, o_phase & 1u, abort_flag, p.timeout_ns);
      ++o_phase;
      ok = __all_sync(0xffffffffu, ok);
    }
    // Epilogue: O' = (O + a) / (1 + z), L' = L + ln(1 + z).
    if (ok) {
      tc_fence_after();
      const float inv = 1.f / (1.f + z);
#pragma unroll
      for (int c = 0; c < kD / 32; ++c) {
        uint32_t a[32];
        uint4 ov[4];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) ov[q4] = o_in[c * 4 + q4];
        tmem_ld32(tmem + lane_sel + kColO + c * 32, a);
        tmem_ld_wait(a);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const uint32_t w[4] = {ov[q4].x, ov[q4].y, ov[q4].z, ov[q4].w};
          uint32_t r[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float lo = (__uint_as_float(w[i] << 16) + __uint_as_float(a[q4 * 8 + 2 * i])) * inv;
            const float hi = (__uint_as_float(w[i] & 0xFFFF0000u) + __uint_as_float(a[q4 * 8 + 2 * i + 1])) * inv;
            r[i] = pack_bf16x2(lo, hi);
          }
          if (live) *reinterpret_cast<uint4*>(orow + c * 32 + q4 * 8) = make_uint4(r[0], r[1], r[2], r[3]);
        }
      }
      if (live) p.lse[bh * N + row] = lse_row + __logf(1.f + z);
    }
    tc_fence_before();
    __syncthreads();  // O_c read before the next pass's MMAs overwrite TMEM
  }

  // Teardown: every issued MMA has completed before TMEM is released.
  if (threadIdx.x == 0) {
    mma_commit(&ctrl->mma_done);
    int never = 0;
    mbar_wait(&ctrl->mma_done, 0, &never, p.timeout_ns);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kApplyTmemCols);
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
  p.scale_log2 = static_cast<float>(static_cast<double>(softmax_scale) * 1.4426950408889634074);
  p.timeout_ns = r.timeout_ns;
  // Keys staged once: about one CTA per SM, each walking a run of passes;
  // more keys than one group: one pass per CTA.
  const int npass = (N + kApplyQ - 1) / kApplyQ;
  int per_head = 1;
  if (r.m <= kStageMax) per_head = std::max(1, std::min(npass, device_sm_count() / std::max(1, B * H)));
  p.passes_per_cta = r.m <= kStageMax ? (npass + per_head - 1) / per_head : 1;
  cudaError_t e = set_smem_attr(reinterpret_cast<const void*>(repair_apply_kernel), kApplySmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((npass + p.passes_per_cta - 1) / p.passes_per_cta, H, B);
  repair_apply_kernel<<<grid, kApplyThreads, kApplySmemBytes, s>>>(p);
  return cudaGetLastError();
}

}  // namespace jattn
