// Prologue of the joint attention: per-head RMSNorm of Q and K, 2-D RoPE on
// the tokens' (row, col) latent-grid positions, and (FP8 mode) E4M3 block
// quantisation of Q', K' and V with one scale per (batch, head, 64 tokens).
//
// Source of the operation: the QKV projection epilogue that applies
// query/key normalisation and rotary position embedding ("GEMM kernel
// optimization" section of the NVIDIA tutorial on accelerating FLUX 3 Image
// Klein with TensorRT LLM VisualGen) and FP8 Q/K/V attention inputs
// ("Quantized and sparse attention" section of the same tutorial).
//
// Memory-bound.  Rows of 128 bf16 channels (256 B) are read with 128-bit
// loads, one row per half-warp: lane l16 = lane % 16 owns channels
// [8*l16, 8*l16 + 8).  Lanes 0-7 of a half hold the row-position half of
// the head (channels 0-63), lanes 8-15 the column-position half, so each
// lane rotates 4 self-contained adjacent pairs.  Row sums of squares are
// reduced with 4 xor-shuffles inside the half-warp.
#include <cuda_fp8.h>

#include "jattn_internal.h"
#include "positions.cuh"
#include "sm100_ptx.cuh"
#include "softmax_sm100.cuh"

namespace jattn {

namespace {

// cos / sin of pos * omega for the lane's 4 channel pairs.  The angle is
// formed and reduced to [-pi, pi] in double, then evaluated in float.
__device__ __forceinline__ void lane_rotations(const PrologueArgs& a, int pos, int pair0, float (&c)[4],
                                               float (&s)[4]) {
  constexpr double kTwoPi = 6.283185307179586476925286766559;
  constexpr double kInvTwoPi = 0.15915494309189533576888376337251;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const double phi = static_cast<double>(pos) * a.omega[pair0 + m];
    const double r = phi - rint(phi * kInvTwoPi) * kTwoPi;
    sincosf(static_cast<float>(r), &s[m], &c[m]);
  }
}

__device__ __forceinline__ void unpack8(const uint4& u, float (&x)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 pack8(const float (&y)[8]) {
  uint4 u;
  u.x = pack_bf16x2(y[0], y[1]);
  u.y = pack_bf16x2(y[2], y[3]);
  u.z = pack_bf16x2(y[4], y[5]);
  u.w = pack_bf16x2(y[6], y[7]);
  return u;
}

// RMSNorm over the half-warp's row, weight, then rotate the lane's 4 pairs.
// Returns the bf16-rounded result packed.  `valid` rows contribute zeros to
// nothing: every lane of a half-warp shares the same validity.
__device__ __forceinline__ uint4 norm_rope_row(const uint4& raw, const float (&w)[8], const float (&c)[4],
                                               const float (&s)[4], float eps) {
  float x[8];
  unpack8(raw, x);
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) ss = fmaf(x[i], x[i], ss);
  ss += __shfl_xor_sync(0xffffffffu, ss, 1);
  ss += __shfl_xor_sync(0xffffffffu, ss, 2);
  ss += __shfl_xor_sync(0xffffffffu, ss, 4);
  ss += __shfl_xor_sync(0xffffffffu, ss, 8);
  const float r = rsqrtf(ss * (1.0f / kHeadDim) + eps);
  float y[8];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const float a0 = x[2 * m] * r * w[2 * m];
    const float a1 = x[2 * m + 1] * r * w[2 * m + 1];
    y[2 * m] = fmaf(a0, c[m], -a1 * s[m]);
    y[2 * m + 1] = fmaf(a0, s[m], a1 * c[m]);
  }
  return pack8(y);
}

// As norm_rope_row, also folding max |y| of the unrounded fp32 results into
// `amax` (rounding to bf16 is monotonic, so rounding the final maximum gives
// the maximum of the rounded values).  Sum of squares and the x * r * w
// products use packed f32x2 arithmetic.
__device__ __forceinline__ uint4 norm_rope_row_amax(const uint4& raw, const float (&w)[8], const float (&c)[4],
                                                    const float (&s)[4], float eps, float& amax) {
  float x[8];
  unpack8(raw, x);
  uint64_t x2[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) x2[m] = f2_pack(x[2 * m], x[2 * m + 1]);
  uint64_t s2 = f2_mul(x2[0], x2[0]);
#pragma unroll
  for (int m = 1; m < 4; ++m) s2 = f2_fma(x2[m], x2[m], s2);
  float ss = f2_lo(s2) + f2_hi(s2);
  ss += __shfl_xor_sync(0xffffffffu, ss, 1);
  ss += __shfl_xor_sync(0xffffffffu, ss, 2);
  ss += __shfl_xor_sync(0xffffffffu, ss, 4);
  ss += __shfl_xor_sync(0xffffffffu, ss, 8);
  const float r = rsqrtf(ss * (1.0f / kHeadDim) + eps);
  const uint64_t r2 = f2_pack(r, r);
  float y[8];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const uint64_t a2 = f2_mul(f2_mul(x2[m], r2), f2_pack(w[2 * m], w[2 * m + 1]));
    const float a0 = f2_lo(a2), a1 = f2_hi(a2);
    y[2 * m] = fmaf(a0, c[m], -a1 * s[m]);
    y[2 * m + 1] = fmaf(a0, s[m], a1 * c[m]);
  }
#pragma unroll
  for (int m = 0; m < 4; ++m) amax = fmax3(amax, fabsf(y[2 * m]), fabsf(y[2 * m + 1]));
  return pack8(y);
}

__device__ __forceinline__ void load_weights(const float* w, int l16, float (&out)[8]) {
  if (w == nullptr) {
#pragma unroll
    for (int i = 0; i < 8; ++i) out[i] = 1.f;
  } else {
    const float4 a = __ldg(reinterpret_cast<const float4*>(w + 8 * l16));
    const float4 b = __ldg(reinterpret_cast<const float4*>(w + 8 * l16 + 4));
    out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
    out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
  }
}

// ------------------------------------------------------------ BF16 mode ----
// One warp per (b, token); heads in batches of kRows per half-warp, Q and K
// together, so the lane's 4 rotations are computed once per token.
constexpr int kBf16Warps = 8;
constexpr int kRows = 4;

__global__ void __launch_bounds__(kBf16Warps * 32) prologue_bf16_kernel(const __grid_constant__ PrologueArgs a) {
  const int lane = threadIdx.x & 31;
  const long long token = static_cast<long long>(blockIdx.x) * kBf16Warps + (threadIdx.x >> 5);
  if (token >= static_cast<long long>(a.B) * a.N) return;
  const int t = static_cast<int>(token % a.N);
  const int half = lane >> 4;
  const int l16 = lane & 15;
  const int axis = l16 >> 3;
  const int pair0 = (l16 & 7) * 4;

  int row, col;
  token_pos(a, t, row, col);
  float c[4], s[4];
  lane_rotations(a, axis == 0 ? row : col, pair0, c, s);
  float wq[8], wk[8];
  load_weights(a.q_w, l16, wq);
  load_weights(a.k_w, l16, wk);

  const size_t row_base = static_cast<size_t>(token) * a.H;  // row index of head 0
  const uint4* qin = reinterpret_cast<const uint4*>(a.q);
  const uint4* kin = reinterpret_cast<const uint4*>(a.k);
  uint4* qout = reinterpret_cast<uint4*>(a.q_out);
  uint4* kout = reinterpret_cast<uint4*>(a.k_out);

  for (int h0 = 0; h0 < a.H; h0 += 2 * kRows) {
    uint4 rq[kRows], rk[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int h = h0 + 2 * r + half;
      const size_t idx = (row_base + h) * 16 + l16;
      if (h < a.H) {
        rq[r] = __ldcs(qin + idx);
        rk[r] = __ldcs(kin + idx);
      } else {
        rq[r] = make_uint4(0, 0, 0, 0);
        rk[r] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int h = h0 + 2 * r + half;
      const uint4 yq = norm_rope_row(rq[r], wq, c, s, a.eps);
      const uint4 yk = norm_rope_row(rk[r], wk, c, s, a.eps);
      if (h < a.H) {
        const size_t idx = (row_base + h) * 16 + l16;
        qout[idx] = yq;
        kout[idx] = yk;
      }
    }
  }
}

// ------------------------------------------------------------- FP8 mode ----
// Persistent kernel.  CTA c processes a contiguous run of work items
// (64-token block, batch, pair of heads), block-major, so the rotation
// table of a block (cos, sin of its 64 tokens x 64 channel pairs, 32 KB of
// shared memory) is built once and reused for every head pair of the block.
// An item's Q, K and V rows (64 tokens x 2 heads x 256 B = 32 KB each) come
// in by TMA into one of two shared-memory buffers.  Every warp copies its
// rows of the item into registers first and then arrives on the buffer's
// `empty` barrier; thread 0 refills the buffer with the next-but-one item
// as soon as all have, so two items' copies are in flight while the
// arithmetic of this one runs.
// Warp w handles head w / 8 of the pair and tokens [8 (w mod 8), +8), a
// half-warp per row: each lane keeps 4 rows of 8 channels of Q, K and V in
// registers from normalisation to quantisation.  The block absmax needs
// every processed value of the block: each warp reduces its 8 tokens of Q,
// K and V (one redux.sync each), and the eight warps of a head exchange the
// three partial maxima through shared memory at one named barrier per item.
// The exchange slots alternate between items, so no second barrier is
// needed before they are rewritten.
constexpr int kF8Pair = 2;                                       // heads per item
constexpr int kF8WarpsPerHead = 8;
constexpr int kF8Warps = kF8Pair * kF8WarpsPerHead;              // 16
constexpr int kF8Threads = kF8Warps * 32;                        // 512
constexpr int kF8Rows = kQuantBlock / (2 * kF8WarpsPerHead);     // 4 rows per lane
constexpr int kF8TileBytes = kQuantBlock * kF8Pair * kHeadDim * 2;  // 32 KB
constexpr int kF8SmemRot = 0;                                    // float2 [64][64]
constexpr int kF8SmemBuf = kQuantBlock * 64 * 8;                 // 32 KB
constexpr int kF8SmemBytes = kF8SmemBuf + 2 * 3 * kF8TileBytes + 1024;  // + alignment slack

// max |x| over 8 bf16 as packed 16-bit integers: with the sign bits cleared,
// bf16 magnitudes order like unsigned integers (inf and NaN excepted, which
// finite inputs do not produce).  Returns the two 16-bit lane maxima.
__device__ __forceinline__ uint32_t absmax8_u16x2(const uint4& u, uint32_t m) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) asm("max.u16x2 %0, %0, %1;" : "+r"(m) : "r"(w[i] & 0x7FFF7FFFu));
  return m;
}

// Warp-wide maximum of a non-negative float: non-negative IEEE floats order
// like their bit patterns as unsigned integers.
__device__ __forceinline__ float warp_max_nonneg(float x) {
  uint32_t u;
  asm volatile("redux.sync.max.u32 %0, %1, 0xffffffff;" : "=r"(u) : "r"(__float_as_uint(x)));
  return __uint_as_float(u);
}

__device__ __forceinline__ uint2 quant8(const uint4& u, float inv) {
  float x[8];
  unpack8(u, x);
  const uint64_t inv2 = f2_pack(inv, inv);
  uint32_t out[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint64_t p2 = f2_mul(f2_pack(x[4 * i + 2 * j], x[4 * i + 2 * j + 1]), inv2);  // correctly rounded
      float2 f;
      f.x = f2_lo(p2);
      f.y = f2_hi(p2);
      const __nv_fp8x2_storage_t p = __nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);
      word |= static_cast<uint32_t>(p) << (16 * j);
    }
    out[i] = word;
  }
  return make_uint2(out[0], out[1]);
}

__global__ void __launch_bounds__(kF8Threads, 1)
prologue_fp8_kernel(const __grid_constant__ PrologueArgs a, const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, int n_items) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float2 (*s_rot)[64] = reinterpret_cast<float2 (*)[64]>(smem + kF8SmemRot);  // [token][axis * 32 + pair]
  __shared__ uint64_t s_full[2];   // the buffer's Q, K, V rows have landed
  __shared__ uint64_t s_empty[2];  // every warp has copied the buffer's rows into registers
  // Partial block maxima: [item parity][head of the pair][Q, K, V][warp of the head].
  __shared__ __align__(16) float s_amax[2][kF8Pair][3][kF8WarpsPerHead];
  __shared__ int s_abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int half = lane >> 4;
  const int l16 = lane & 15;
  const int axis = l16 >> 3;
  const int pair0 = (l16 & 7) * 4;
  const int hl = warp / kF8WarpsPerHead;       // head of the pair
  const int tq = warp % kF8WarpsPerHead;       // token group of the block
  const int tok0 = 2 * kF8Rows * tq + half;    // lane's rows: tokens tok0 + 2 i
  const int bar_id = 1 + hl;                   // the warps of head hl
  const int nblk = (a.N + kQuantBlock - 1) / kQuantBlock;
  const int n_pairs = (a.H + kF8Pair - 1) / kF8Pair;
  const int begin = static_cast<int>(static_cast<long long>(blockIdx.x) * n_items / gridDim.x);
  const int end = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * n_items / gridDim.x);
  const CUtensorMap* maps[3] = {&tm_q, &tm_k, &tm_v};

  auto coords = [&](int item, int& blk, int& b, int& hp) {
    hp = item % n_pairs;
    const int rest = item / n_pairs;
    b = rest % a.B;
    blk = rest / a.B;
  };
  auto tile = [&](int buf, int x) { return smem + kF8SmemBuf + (buf * 3 + x) * kF8TileBytes; };
  // Thread 0: TMA of item `item`'s Q, K, V rows into buffer `buf`.
  auto issue = [&](int item, int buf) {
    int blk, b, hp;
    coords(item, blk, b, hp);
    mbar_arrive_expect_tx(&s_full[buf], 3 * kF8TileBytes);
#pragma unroll
    for (int x = 0; x < 3; ++x) tma_load_4d(tile(buf, x), maps[x], &s_full[buf], 0, hp * kF8Pair, blk * kQuantBlock, b);
  };

  float wq[8], wk[8];
  load_weights(a.q_w, l16, wq);
  load_weights(a.k_w, l16, wk);

  int issued_end = begin;  // thread 0: one past the last item whose copies were issued
  if (threadIdx.x == 0) {
    for (int u = 0; u < 2; ++u) {
      mbar_init(&s_full[u], 1);
      mbar_init(&s_empty[u], kF8Warps);
    }
    s_abort = 0;
    fence_barrier_init();
    if (begin < end) {
      for (int x = 0; x < 3; ++x) prefetch_tensormap(maps[x]);
      issue(begin, 0);
      issued_end = begin + 1;
      if (begin + 1 < end) {
        issue(begin + 1, 1);
        issued_end = begin + 2;
      }
    }
  }
  __syncthreads();

  constexpr double kTwoPi = 6.283185307179586476925286766559;
  constexpr double kInvTwoPi = 0.15915494309189533576888376337251;
  int cur_blk = -1;
  for (int item = begin; item < end; ++item) {
    const int i = item - begin;
    const int buf = i & 1;
    int blk, b, hp;
    coords(item, blk, b, hp);
    const int t0 = blk * kQuantBlock;
    const int h = hp * kF8Pair + hl;
    if (blk != cur_blk) {  // same for the whole CTA
      __syncthreads();     // every warp is done with the previous block's table
      for (int e = threadIdx.x; e < kQuantBlock * 64; e += kF8Threads) {
        const int tok = e >> 6, pr = e & 63;
        int row = 0, col = 0;
        if (t0 + tok < a.N) token_pos(a, t0 + tok, row, col);
        const double phi = static_cast<double>(pr < 32 ? row : col) * a.omega[pr & 31];
        const double rr = phi - rint(phi * kInvTwoPi) * kTwoPi;
        float sn, cs;
        sincosf(static_cast<float>(rr), &sn, &cs);
        s_rot[tok][pr] = make_float2(cs, sn);
      }
      __syncthreads();
      cur_blk = blk;
    }

    const bool ok = mbar_wait(&s_full[buf], static_cast<uint32_t>(i >> 1) & 1u, &s_abort, a.timeout_ns);
    uint4 rows[3][kF8Rows];  // [Q, K, V][row]
#pragma unroll
    for (int x = 0; x < 3; ++x) {
      const uint4* src = reinterpret_cast<const uint4*>(tile(buf, x));
#pragma unroll
      for (int r = 0; r < kF8Rows; ++r)
        rows[x][r] = ok ? src[((tok0 + 2 * r) * kF8Pair + hl) * 16 + l16] : make_uint4(0, 0, 0, 0);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s_empty[buf]);
    // Refill this buffer with item i + 2 once every warp has copied item i's
    // rows out of it (the buffer's (i >> 1)-th use).
    if (threadIdx.x == 0 && item + 2 < end && !s_abort &&
        mbar_wait(&s_empty[buf], static_cast<uint32_t>(i >> 1) & 1u, &s_abort, a.timeout_ns)) {
      issue(item + 2, buf);
      issued_end = item + 3;
    }

    // Q and K: RMSNorm, weight, rotation (one table read per row serves
    // both), and the block maxima of the bf16 results over valid tokens.
    float amax[3] = {0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < kF8Rows; ++r) {
      const int tok = tok0 + 2 * r;
      const float4 r0 = *reinterpret_cast<const float4*>(&s_rot[tok][axis * 32 + pair0]);
      const float4 r1 = *reinterpret_cast<const float4*>(&s_rot[tok][axis * 32 + pair0 + 2]);
      const float c[4] = {r0.x, r0.z, r1.x, r1.z};
      const float sn[4] = {r0.y, r0.w, r1.y, r1.w};
      float aq = 0.f, ak = 0.f;
      rows[0][r] = norm_rope_row_amax(rows[0][r], wq, c, sn, a.eps, aq);
      rows[1][r] = norm_rope_row_amax(rows[1][r], wk, c, sn, a.eps, ak);
      if (t0 + tok < a.N) {
        amax[0] = fmaxf(amax[0], aq);
        amax[1] = fmaxf(amax[1], ak);
      }
    }
    amax[0] = __bfloat162float(__float2bfloat16_rn(amax[0]));
    amax[1] = __bfloat162float(__float2bfloat16_rn(amax[1]));
    {
      uint32_t m2 = 0;  // V: max |v| of the bf16 inputs (rows past N are zero-filled)
#pragma unroll
      for (int r = 0; r < kF8Rows; ++r) m2 = absmax8_u16x2(rows[2][r], m2);
      amax[2] = fmaxf(__uint_as_float(m2 << 16), __uint_as_float(m2 & 0xFFFF0000u));
    }
    float(*slot)[kF8WarpsPerHead] = s_amax[i & 1][hl];
#pragma unroll
    for (int x = 0; x < 3; ++x) {
      const float m = warp_max_nonneg(amax[x]);
      if (lane == 0) slot[x][tq] = m;
    }
    named_bar_sync(bar_id, kF8WarpsPerHead * 32);
#pragma unroll
    for (int x = 0; x < 3; ++x) {
      const float4 lo = *reinterpret_cast<const float4*>(&slot[x][0]);
      const float4 hi = *reinterpret_cast<const float4*>(&slot[x][4]);
      amax[x] = fmaxf(fmax3(lo.x, lo.y, fmax3(lo.z, lo.w, hi.x)), fmax3(hi.y, hi.z, hi.w));
    }

    if (ok && h < a.H) {
#pragma unroll
      for (int x = 0; x < 3; ++x) {
        const float inv = amax[x] > 0.f ? __fdiv_rn(448.0f, amax[x]) : 0.f;
        if (tq == 0 && lane == 0) {
          float* sc = x == 0 ? a.q_scale : (x == 1 ? a.k_scale : a.v_scale);
          sc[(static_cast<size_t>(b) * a.H + h) * nblk + blk] = amax[x] > 0.f ? __fdiv_rn(amax[x], 448.0f) : 1.0f;
        }
        uint2* out = reinterpret_cast<uint2*>(x == 0 ? a.q_out : (x == 1 ? a.k_out : a.v_out));
#pragma unroll
        for (int r = 0; r < kF8Rows; ++r) {
          const int t = t0 + tok0 + 2 * r;
          if (t < a.N) __stcs(out + ((static_cast<size_t>(b) * a.N + t) * a.H + h) * 16 + l16, quant8(rows[x][r], inv));
        }
      }
    }
  }
  // Drain: the copies of the last two issued items have landed before the
  // CTA exits (all of them, unless a wait timed out).
  if (threadIdx.x == 0) {
    int never = 0;
    for (int item = (issued_end - 2 > begin ? issued_end - 2 : begin); item < issued_end; ++item) {
      const int i = item - begin;
      mbar_wait(&s_full[i & 1], static_cast<uint32_t>(i >> 1) & 1u, &never, a.timeout_ns);
    }
  }
}

}  // namespace

cudaError_t launch_prologue_bf16(const PrologueArgs& a, cudaStream_t s) {
  const long long tokens = static_cast<long long>(a.B) * a.N;
  const unsigned grid = static_cast<unsigned>((tokens + kBf16Warps - 1) / kBf16Warps);
  prologue_bf16_kernel<<<grid, kBf16Warps * 32, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_prologue_fp8(const PrologueArgs& a, cudaStream_t s) {
  CUtensorMap tq, tk, tv;
  cudaError_t e;
  if ((e = make_rows_map(&tq, a.q, a.B, a.N, a.H, kF8Pair, kQuantBlock)) != cudaSuccess) return e;
  if ((e = make_rows_map(&tk, a.k, a.B, a.N, a.H, kF8Pair, kQuantBlock)) != cudaSuccess) return e;
  if ((e = make_rows_map(&tv, a.v, a.B, a.N, a.H, kF8Pair, kQuantBlock)) != cudaSuccess) return e;
  if ((e = set_smem_attr(reinterpret_cast<const void*>(prologue_fp8_kernel), kF8SmemBytes)) != cudaSuccess) return e;
  const long long n_items = static_cast<long long>((a.N + kQuantBlock - 1) / kQuantBlock) * a.B *
                            ((a.H + kF8Pair - 1) / kF8Pair);
  const int sms = device_sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  const int grid = static_cast<int>(n_items < sms ? n_items : sms);
  prologue_fp8_kernel<<<grid, kF8Threads, kF8SmemBytes, s>>>(a, tq, tk, tv, static_cast<int>(n_items));
  return cudaGetLastError();
}

}  // namespace jattn
