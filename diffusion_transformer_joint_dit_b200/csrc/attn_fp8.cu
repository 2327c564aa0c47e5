// Joint attention forward from E4M3 block-quantised Q, K, V, for sm_100a.
//
// FP8 Q/K and FP8 V attention ("Quantized and sparse attention" section of
// the NVIDIA tutorial on FLUX 3 Image Klein: qk_dtype / v_dtype fp8).  The
// inputs are E4M3 codes with one fp32 scale per (batch, head, 64 tokens):
// X = decode(code) * scale.  The kernel computes softmax(scale Qd Kd^T) Vd:
//
//   S_raw = q8 . k8 on the tensor core (tcgen05 kind::f8f6f4, fp32 accum);
//   x     = S_raw * (sq(row) * sk(col block) * softmax_scale * log2 e);
//   P     = exp2(x - m), written to TMEM as FP16;
//   V16   = code * (sv(block) / 2^e), widened and scaled to FP16 in shared
//           memory by the converter warps;
//   O    += P . V16;  l = sum P (fp32; the largest P of each tile counted
//           as the FP16 value the MMA uses);
//   O     = O * 2^e / l.
//
// The per-(b, h) power of two 2^e >= max_block sv / 128 keeps |V16| <=
// 448 * 128 < 65504.  An all-zero V block (scale 1, zero codes) adds
// nothing to O whatever its factor, and blocks whose scales lie 2^12 below
// the largest still land in FP16's normal range.  P is FP16 (not E4M3): an
// E4M3 P costs about 2.5% relative L2, FP16 P about 2e-4 on these
// workloads.  The lazy maximum moves only when a tile's max exceeds it by
// more than 14 (log2 units), so P <= 2^14 stays well inside FP16.
//
// CTA = 256 query rows of one (b, h) as two 128-row Q tiles, as in the BF16
// kernel.  Warps: 0-7 softmax (two warpgroups), 8 TMA producer, 9 MMA issuer
// and TMEM owner, 10-11 V converters (E4M3 smem tile -> FP16 smem tile in the
// 128-byte-swizzled MN-major layout the P.V MMA reads).
#include <cuda_fp8.h>

#include "jattn_internal.h"
#include "sm100_ptx.cuh"
#include "softmax_sm100.cuh"

namespace jattn {

namespace fp8attn {

constexpr int kBM = 128;
constexpr int kTiles = 2;
constexpr int kBN = 128;
constexpr int kD = 128;
constexpr int kKStages = 3;
constexpr int kVStages = 3;
constexpr int kTile8 = kBM * kD;               // 16 KB: 128 rows x 128 e4m3
constexpr int kTile16 = kBN * kD * 2;          // 32 KB: 128 keys x 128 fp16
constexpr int kBox16 = kTile16 / 2;            // 16 KB: 128 keys x 64 channels
constexpr int kSoftmaxWarps = 4 * kTiles;      // 8
constexpr int kLoadWarp = kSoftmaxWarps;       // 8
constexpr int kMmaWarp = kSoftmaxWarps + 1;    // 9
constexpr int kCvtWarp0 = kSoftmaxWarps + 2;   // 10, 11
constexpr int kCvtThreads = 64;
constexpr int kThreads = (kSoftmaxWarps + 4) * 32;  // 384
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 14.0f;

struct Ctrl {
  uint64_t q_full;
  uint64_t k_full[kKStages];
  uint64_t k_empty[kKStages];
  uint64_t v_full[kVStages];
  uint64_t v_empty[kVStages];
  uint64_t vh_full[2];
  uint64_t vh_empty[2];
  uint64_t s_full[kTiles];
  uint64_t p_full[kTiles];
  uint64_t o_full;
  uint64_t mma_done;
  uint64_t norm_ready;
  uint32_t tmem_base;
  int abort;
  float v_norm;        // 2^e >= max sv over the (b, h) / 128
};

constexpr int kSmemQ = 0;
constexpr int kSmemK = kSmemQ + kTiles * kTile8;
constexpr int kSmemV = kSmemK + kKStages * kTile8;
constexpr int kSmemVh = kSmemV + kVStages * kTile8;
constexpr int kSmemCtrl = kSmemVh + 2 * kTile16;
constexpr int kSmemBytes = kSmemCtrl + static_cast<int>(sizeof(Ctrl)) + 1024;

struct Params {
  __nv_bfloat16* o;
  float* lse;
  const float* q_scale;
  const float* k_scale;
  const float* v_scale;
  int H, N, nblk;
  float scale_log2;
  uint64_t timeout_ns;
};

__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  int never = 0;
  return mbar_wait_sleep(bar, parity, &never, timeout_ns);
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 16 E4M3 codes -> 16 FP16 values times the block factor f (an FP16 pair
// (f, f)), as two 16-byte chunks: each code widens exactly, the product
// rounds once.
__device__ __forceinline__ void widen16_scaled(const uint4& src, __half2 f, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {src.x, src.y, src.z, src.w};
  uint32_t out[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2_raw a = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[i] & 0xFFFFu), __NV_E4M3);
    const __half2_raw b = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[i] >> 16), __NV_E4M3);
    const __half2 ha = __hmul2(__half2(a), f), hb = __hmul2(__half2(b), f);
    out[2 * i] = *reinterpret_cast<const uint32_t*>(&ha);
    out[2 * i + 1] = *reinterpret_cast<const uint32_t*>(&hb);
  }
  lo = make_uint4(out[0], out[1], out[2], out[3]);
  hi = make_uint4(out[4], out[5], out[6], out[7]);
}

__global__ void __launch_bounds__(kThreads, 1)
attn_fp8_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ Params prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + kSmemCtrl);
  volatile int* abort_flag = &ctrl->abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int m0 = blockIdx.x * (kBM * kTiles);
  const int N = prm.N;
  const int n_kv = (N + kBN - 1) / kBN;
  const size_t scale_row = (static_cast<size_t>(b) * prm.H + h) * prm.nblk;

  if (threadIdx.x == 0) {
    mbar_init(&ctrl->q_full, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&ctrl->k_full[s], 1);
      mbar_init(&ctrl->k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&ctrl->v_full[s], 1);
      mbar_init(&ctrl->v_empty[s], kCvtThreads);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctrl->vh_full[i], kCvtThreads);
      mbar_init(&ctrl->vh_empty[i], 1);
    }
    for (int t = 0; t < kTiles; ++t) {
      mbar_init(&ctrl->s_full[t], 1);
      mbar_init(&ctrl->p_full[t], 4 * 32);
    }
    mbar_init(&ctrl->o_full, 1);
    mbar_init(&ctrl->mma_done, 1);
    mbar_init(&ctrl->norm_ready, kCvtThreads);
    ctrl->abort = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&ctrl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;

  if (warp == kLoadWarp) {
    // ------------------------------------------------------ TMA producer ----
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      mbar_arrive_expect_tx(&ctrl->q_full, kTiles * kTile8);
      for (int t = 0; t < kTiles; ++t)
        tma_load_4d(smem + kSmemQ + t * kTile8, &tm_q, &ctrl->q_full, 0, h, m0 + t * kBM, b);
      int nk = 0, nv = 0;  // fills issued
      for (int j = 0; j < n_kv; ++j) {
        const int ks = j % kKStages, vs = j % kVStages;
        if (!mbar_wait_sleep(&ctrl->k_empty[ks], ((j / kKStages) & 1) ^ 1, abort_flag, prm.timeout_ns)) break;
        mbar_arrive_expect_tx(&ctrl->k_full[ks], kTile8);
        tma_load_4d(smem + kSmemK + ks * kTile8, &tm_k, &ctrl->k_full[ks], 0, h, j * kBN, b);
        ++nk;
        if (!mbar_wait_sleep(&ctrl->v_empty[vs], ((j / kVStages) & 1) ^ 1, abort_flag, prm.timeout_ns)) break;
        mbar_arrive_expect_tx(&ctrl->v_full[vs], kTile8);
        tma_load_4d(smem + kSmemV + vs * kTile8, &tm_v, &ctrl->v_full[vs], 0, h, j * kBN, b);
        ++nv;
      }
      // Drain: the last fill of every slot has landed before the CTA may exit.
      drain_wait(&ctrl->q_full, 0, prm.timeout_ns);
      for (int i = (nk > kKStages ? nk - kKStages : 0); i < nk; ++i)
        drain_wait(&ctrl->k_full[i % kKStages], (i / kKStages) & 1, prm.timeout_ns);
      for (int i = (nv > kVStages ? nv - kVStages : 0); i < nv; ++i)
        drain_wait(&ctrl->v_full[i % kVStages], (i / kVStages) & 1, prm.timeout_ns);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------- MMA issuer ----
    if (lane == 0) {
      constexpr uint32_t idesc_qk = make_idesc(0, 0, false, kBM, kBN);  // e4m3 x e4m3, K-major both
      constexpr uint32_t idesc_pv = make_idesc(0, 0, true, kBM, kD);    // f16 P (TMEM) x f16 V (MN-major)
      // Descriptors of the first tile of each operand; adding (offset >> 4)
      // to the start-address field moves a descriptor in shared memory.
      const uint64_t dq0 = smem_desc_sw128(smem_u32(smem + kSmemQ), 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(smem_u32(smem + kSmemK), 16, 1024);
      const uint64_t dv0 = smem_desc_sw128(smem_u32(smem + kSmemVh), kBox16, 1024);

      auto issue_qk = [&](int t, int ks) {
        const uint32_t d = tmem + t * kBN;
        const uint64_t qa = dq0 + static_cast<uint64_t>((t * kTile8) >> 4);
        const uint64_t kb = dk0 + static_cast<uint64_t>((ks * kTile8) >> 4);
#pragma unroll
        for (int kk = 0; kk < kD / 32; ++kk) {  // 32 e4m3 channels (32 bytes) per MMA
          mma_f8_ss(d, qa + static_cast<uint64_t>((kk * 32) >> 4), kb + static_cast<uint64_t>((kk * 32) >> 4),
                    idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int t, int vb, bool acc) {
        const uint32_t d = tmem + 2 * kBN + t * kD;
        const uint32_t p = tmem + t * kBN;
        const uint64_t v = dv0 + static_cast<uint64_t>((vb * kTile16) >> 4);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          mma_f16_ts(d, p + kk * 8, v + static_cast<uint64_t>((kk * 16 * 128) >> 4), idesc_pv,
                     (acc || kk > 0) ? 1u : 0u);
      };

      bool ok = mbar_wait_sleep(&ctrl->q_full, 0, abort_flag, prm.timeout_ns);
      if (ok) ok = mbar_wait_sleep(&ctrl->k_full[0], 0, abort_flag, prm.timeout_ns);
      if (ok) {
        tc_fence_after();
        issue_qk(0, 0);
        mma_commit(&ctrl->s_full[0]);
        issue_qk(1, 0);
        mma_commit(&ctrl->s_full[1]);
        mma_commit(&ctrl->k_empty[0]);
      }
      for (int j = 0; j < n_kv && ok; ++j) {
        const int vb = j & 1;
        ok = mbar_wait_sleep(&ctrl->vh_full[vb], (j >> 1) & 1, abort_flag, prm.timeout_ns);
        if (!ok) break;
        const bool has_next = j + 1 < n_kv;
        const int ks = (j + 1) % kKStages;
        ok = mbar_wait_sleep(&ctrl->p_full[0], j & 1, abort_flag, prm.timeout_ns);
        if (!ok) break;
        tc_fence_after();
        issue_pv(0, vb, j > 0);
        if (has_next) {
          ok = mbar_wait_sleep(&ctrl->k_full[ks], ((j + 1) / kKStages) & 1, abort_flag, prm.timeout_ns);
          if (!ok) break;
          tc_fence_after();
          issue_qk(0, ks);
          mma_commit(&ctrl->s_full[0]);
        }
        ok = mbar_wait_sleep(&ctrl->p_full[1], j & 1, abort_flag, prm.timeout_ns);
        if (!ok) break;
        tc_fence_after();
        issue_pv(1, vb, j > 0);
        mma_commit(&ctrl->vh_empty[vb]);
        if (has_next) {
          issue_qk(1, ks);
          mma_commit(&ctrl->s_full[1]);
          mma_commit(&ctrl->k_empty[ks]);
        }
      }
      if (ok) mma_commit(&ctrl->o_full);
      mma_commit(&ctrl->mma_done);
      drain_wait(&ctrl->mma_done, 0, prm.timeout_ns);
    }
    __syncwarp();
  } else if (warp >= kCvtWarp0) {
    // ------------------------------------------------- V converters (x2) ----
    const int ct = threadIdx.x - kCvtWarp0 * 32;  // 0..63
    // Per-head V normaliser 2^e >= max block scale (power of two: exact).
    float mx = 0.f;
    for (int i = ct; i < prm.nblk; i += kCvtThreads) mx = fmaxf(mx, __ldg(prm.v_scale + scale_row + i));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    __shared__ float s_vmax[2];
    if (lane == 0) s_vmax[warp - kCvtWarp0] = mx;
    named_bar_sync(1, kCvtThreads);
    if (ct == 0) {
      const float m = fmaxf(s_vmax[0], s_vmax[1]);
      int e = 0;
      if (m > 0.f) {
        frexpf(m, &e);  // m = f * 2^e, f in [0.5, 1)  ->  2^e > m
      }
      ctrl->v_norm = ldexpf(1.0f, e - 7);  // > max sv / 128
    }
    named_bar_sync(1, kCvtThreads);
    const float inv_norm = 1.0f / ctrl->v_norm;  // a power of two: exact
    mbar_arrive(&ctrl->norm_ready);

    const uint8_t* vsrc_base = smem + kSmemV;
    for (int j = 0; j < n_kv; ++j) {
      const int vs = j % kVStages, vb = j & 1;
      bool ok = mbar_wait_sleep(&ctrl->v_full[vs], (j / kVStages) & 1, abort_flag, prm.timeout_ns);
      ok = ok && mbar_wait_sleep(&ctrl->vh_empty[vb], ((j >> 1) & 1) ^ 1, abort_flag, prm.timeout_ns);
      if (!ok) break;
      const uint8_t* src = vsrc_base + vs * kTile8;
      uint8_t* dst = smem + kSmemVh + vb * kTile16;
      // Block factors sv / 2^e of this tile's two 64-key blocks (a partial
      // last tile reads the last block's scale for its zero-filled rows).
      const __half2 f_lo = __float2half2_rn(__ldg(prm.v_scale + scale_row + 2 * j) * inv_norm);
      const __half2 f_hi = __float2half2_rn(__ldg(prm.v_scale + scale_row + min(2 * j + 1, prm.nblk - 1)) * inv_norm);
#pragma unroll 4
      for (int i = 0; i < (kBN * 8) / kCvtThreads; ++i) {
        // 16-byte source chunk (row r, channel chunk c16).  Consecutive lanes
        // take consecutive rows of one chunk column: each group of 8 lanes
        // then touches 8 distinct swizzled bank groups on load and store.
        const int idx = ct + i * kCvtThreads;
        const int r = idx & (kBN - 1), c16 = idx >> 7;
        const uint4 raw = *reinterpret_cast<const uint4*>(src + r * 128 + ((c16 ^ (r & 7)) << 4));
        uint4 lo, hi;
        widen16_scaled(raw, r < 64 ? f_lo : f_hi, lo, hi);
        const int box = c16 >> 2;             // channels 16*c16.. -> 64-channel box
        const int c8 = (c16 & 3) * 2;         // first 8-channel chunk inside the box
        uint8_t* row = dst + box * kBox16 + r * 128;
        *reinterpret_cast<uint4*>(row + ((c8 ^ (r & 7)) << 4)) = lo;
        *reinterpret_cast<uint4*>(row + (((c8 + 1) ^ (r & 7)) << 4)) = hi;
      }
      fence_async_smem();  // generic-proxy smem writes -> visible to the tensor core
      mbar_arrive(&ctrl->v_empty[vs]);
      mbar_arrive(&ctrl->vh_full[vb]);
    }
  } else {
    // ------------------------------------------- softmax + epilogue (x2) ----
    const int t = warp >> 2;
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_sel = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t s_addr = tmem + lane_sel + t * kBN;
    const uint32_t o_addr = tmem + lane_sel + 2 * kBN + t * kD;
    const int row = m0 + t * kBM + r;
    const float sq = row < N ? __ldg(prm.q_scale + scale_row + row / 64) * prm.scale_log2 : 0.f;

    bool ok = __all_sync(0xffffffffu, mbar_wait(&ctrl->norm_ready, 0, abort_flag, prm.timeout_ns));
    const float v_norm = ctrl->v_norm;

    float m = -INFINITY;
    float l = 0.f;
    for (int j = 0; j < n_kv && ok; ++j) {
      // Block scales of this KV tile's two 64-key halves (block 2j, 2j+1).
      const int kb0 = 2 * j, kb1 = min(2 * j + 1, prm.nblk - 1);
      const float c0 = sq * __ldg(prm.k_scale + scale_row + kb0);
      const float c1 = sq * __ldg(prm.k_scale + scale_row + kb1);
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&ctrl->s_full[t], static_cast<uint32_t>(j) & 1u, abort_flag, prm.timeout_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sv[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + c * 32, sv[c]);
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_wait(sv[c]);  // ties the loaded registers to the wait
      const int nvalid = N - j * kBN;
      if (nvalid < kBN) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c * 32 + i >= nvalid) sv[c][i] = __float_as_uint(-INFINITY);
      }
      float mx_lo, mx_hi;
      row_max_halves(sv, mx_lo, mx_hi);
      // Scaled maxima of the two halves (scales are > 0; a fully masked
      // half has max -inf and stays -inf).
      const float hm0 = mx_lo * c0;
      const float hm1 = mx_hi * c1;
      const float mnew = fmaxf(m, fmaxf(hm0, hm1));
      const bool need = mnew > m + kRescaleThreshold;
      float corr = 1.f;
      if (need) {
        corr = ex2_approx(m - mnew);
        l *= corr;
        m = mnew;
      }
      // Row sum: fp32 sum of the unrounded P plus the fp16 rounding of the
      // tile's largest P (formed as the packing loop forms it), so that a
      // dominant key has the same weight in O = sum fp16(P) V16 and in l.
      const float pm = ex2_approx(fmaxf(fmaf(mx_lo, c0, -m), fmaf(mx_hi, c1, -m)));
      const float fix = __half2float(__float2half_rn(pm)) - pm;
      const float lt = exp_pack_sum<true>(sv, c0, -m, c1, -m) + fix;
      tmem_st32(s_addr, sv[0]);
      tmem_st32(s_addr + 32, sv[2]);
      // O correction after P is out of registers (keeps register pressure
      // down); it only has to land before this tile's P.V is issued.
      if (j > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t ov[16];
          tmem_ld16(o_addr + c * 16, ov);
          tmem_ld_wait16(ov);
#pragma unroll
          for (int i = 0; i < 16; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * corr);
          tmem_st16(o_addr + c * 16, ov);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&ctrl->p_full[t]);
      l += lt;
    }

    if (ok && __all_sync(0xffffffffu, mbar_wait(&ctrl->o_full, 0, abort_flag, prm.timeout_ns))) {
      tc_fence_after();
      const float f = v_norm / l;
      __nv_bfloat16* orow = prm.o + ((static_cast<size_t>(b) * N + row) * prm.H + h) * kD;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t ov[32];
        tmem_ld32(o_addr + c * 32, ov);
        tmem_ld_wait(ov);
        if (row < N) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint4 u;
            u.x = pack_bf16x2(__uint_as_float(ov[8 * q4 + 0]) * f, __uint_as_float(ov[8 * q4 + 1]) * f);
            u.y = pack_bf16x2(__uint_as_float(ov[8 * q4 + 2]) * f, __uint_as_float(ov[8 * q4 + 3]) * f);
            u.z = pack_bf16x2(__uint_as_float(ov[8 * q4 + 4]) * f, __uint_as_float(ov[8 * q4 + 5]) * f);
            u.w = pack_bf16x2(__uint_as_float(ov[8 * q4 + 6]) * f, __uint_as_float(ov[8 * q4 + 7]) * f);
            dst[q4] = u;
          }
        }
      }
      if (prm.lse != nullptr && row < N) {
        // ln sum exp(scale s) = (m + log2(sum P)) ln 2, with sum P = l.
        prm.lse[(static_cast<size_t>(b) * prm.H + h) * N + row] = (m + __log2f(l)) * 0.69314718055994530942f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace fp8attn

cudaError_t launch_attn_fp8(const AttnProblem& p, cudaStream_t s) {
  using namespace fp8attn;
  CUtensorMap tq, tk, tv;
  cudaError_t e;
  if ((e = make_act_map(&tq, p.q, p.B, p.N, p.H, 1)) != cudaSuccess) return e;
  if ((e = make_act_map(&tk, p.k, p.B, p.N, p.H, 1)) != cudaSuccess) return e;
  if ((e = make_act_map(&tv, p.v, p.B, p.N, p.H, 1)) != cudaSuccess) return e;
  if ((e = set_smem_attr(reinterpret_cast<const void*>(attn_fp8_kernel), kSmemBytes)) != cudaSuccess) return e;
  Params prm;
  prm.o = static_cast<__nv_bfloat16*>(p.o);
  prm.lse = p.lse;
  prm.q_scale = p.q_scale;
  prm.k_scale = p.k_scale;
  prm.v_scale = p.v_scale;
  prm.H = p.H;
  prm.N = p.N;
  prm.nblk = (p.N + kQuantBlock - 1) / kQuantBlock;
  prm.scale_log2 = static_cast<float>(static_cast<double>(p.softmax_scale) * 1.4426950408889634074);
  prm.timeout_ns = p.timeout_ns;
  dim3 grid((p.N + kBM * kTiles - 1) / (kBM * kTiles), p.H, p.B);
  attn_fp8_kernel<<<grid, kThreads, kSmemBytes, s>>>(tq, tk, tv, prm);
  return cudaGetLastError();
}

}  // namespace jattn
