// Fused QKV projection for sm_100a: Q, K, V = x W_s^T per token stream s,
// with query/key RMSNorm and 2-D RoPE applied in the GEMM epilogue, the
// fusion the NVIDIA tutorial on FLUX 3 Image Klein describes in its "GEMM
// kernel optimization" section (there with FP8/NVFP4 weights; here BF16).
//
// Design: persistent clusters of two CTAs (one per SM) sharing
// tcgen05.mma.cta_group::2 M=256 N=256 K=16: a pair computes an output tile
// of 256 tokens x 256 features (two heads); CTA r of the pair holds the
// tile's tokens [128 r, 128 r + 128) as its A operand and features
// [128 r, 128 r + 128) as its half of B, and receives its 128 token rows
// of the accumulator in its own TMEM.  Each SM thus takes 32 KB per
// 64-channel K step from L2 instead of 48 KB (one-SM tiles of the same
// shape measured L2-bound at about 74% of the tensor peak).
//   warp 0     TMA producer (both CTAs): its A rows and B half per K step
//              into a 6-stage ring (128-byte swizzle, K-major); completion
//              is counted on the leader's barrier
//   warp 1     TMEM allocator (both CTAs, paired allocation); the leader's
//              lane 0 issues every MMA of the pair
//   warps 2-5  epilogue (both CTAs): TMEM lane quarter = warp mod 4, one
//              token row per thread
// Two 256-column TMEM accumulators let the epilogue of one tile overlap the
// main loop of the next.  A tile's rows belong to one (batch, stream): the
// tile list enumerates each batch element's text rows, then its image +
// reference rows, in 256-row tiles; rows past the stream's end are computed
// but not stored.  Because a tile holds whole heads, a thread owns all 128
// channels of its row's head: the RMSNorm sum of squares is a thread-local
// loop (first pass over TMEM), the scaling, weights and rotation a second
// pass, 32 channels at a time.
#include "jattn_internal.h"
#include "positions.cuh"
#include "sm100_ptx.cuh"

namespace jattn {

namespace qkvgemm {

constexpr int kBM = 128;                       // tokens per CTA (= TMEM lanes); 256 per pair
constexpr int kBN = 256;                       // output features per tile (two heads)
constexpr int kBNh = kBN / 2;                  // features per CTA (its half of B)
constexpr int kBK = 64;                        // input channels per stage (128 B: one swizzle atom)
constexpr int kStages = 6;
constexpr int kABytes = kBM * kBK * 2;         // 16 KB
constexpr int kBBytes = kBNh * kBK * 2;        // 16 KB
constexpr int kStageBytes = kABytes + kBBytes; // per CTA; the leader's barrier counts both CTAs
constexpr int kD = 128;
constexpr int kLoadWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kThreads = 6 * 32;
constexpr uint32_t kTmemCols = 512;            // two accumulators of kBN columns
constexpr uint16_t kPairMask = 0x3;

struct Ctrl {
  uint64_t full[kStages];  // leader: stage s of both CTAs landed
  uint64_t empty[kStages]; // each CTA: stage s consumed by the pair's MMAs
  uint64_t acc_full[2];    // each CTA: accumulator a holds a finished tile
  uint64_t acc_empty[2];   // leader: accumulator a drained by both CTAs' epilogues
  uint64_t mma_done;       // each CTA: every pair MMA complete
  uint32_t tmem_base;
  int abort;
};

constexpr int kSmemRing = 0;
constexpr int kSmemCtrl = kStages * kStageBytes;
constexpr int kSmemBytes = kSmemCtrl + static_cast<int>(sizeof(Ctrl)) + 1024;  // + alignment slack

struct Params {
  const float* rope;        // [N, 64, 2]
  const float* qw[2];       // per-stream Q norm weights (NULL = 1)
  const float* kw[2];
  __nv_bfloat16* out[3];    // Q, K, V [B, N, H, d]
  int B, N, H, n_txt;
  int k_steps;              // C / 64
  int tiles_txt, tiles_img; // 256-row tiles per batch element and stream
  int n_tiles_n;            // 3 H d / 256
  int group_n;              // feature tiles per raster group
  int n_tiles;
  float eps;
  uint64_t timeout_ns;
};

struct Tile {
  int stream, b, tok0, tok_end, nt;
};

// Tile order: the feature tiles are cut into groups of group_n; group g
// runs over every row tile before group g + 1 starts, row-major inside the
// group.  The pairs working at one time then share a W panel set of group_n
// feature tiles (sized on the host to stay resident in L2 while x streams
// through), instead of needing all of W for every row tile.
__device__ __forceinline__ Tile tile_at(const Params& p, int t) {
  Tile x;
  const int per_b = p.tiles_txt + p.tiles_img;
  const int n_mt = p.B * per_b;
  const int g = t / (n_mt * p.group_n);
  const int width = min(p.group_n, p.n_tiles_n - g * p.group_n);
  const int rg = t - g * n_mt * p.group_n;
  const int mt = rg / width;
  x.nt = g * p.group_n + (rg - mt * width);
  x.b = mt / per_b;
  const int r = mt - x.b * per_b;
  if (r < p.tiles_txt) {
    x.stream = 0;
    x.tok0 = r * 2 * kBM;
    x.tok_end = p.n_txt;
  } else {
    x.stream = 1;
    x.tok0 = p.n_txt + (r - p.tiles_txt) * 2 * kBM;
    x.tok_end = p.N;
  }
  return x;
}

__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  int never = 0;
  return mbar_wait(bar, parity, &never, timeout_ns);
}

__global__ void __launch_bounds__(kThreads, 1)
qkv_fused_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w0,
                 const __grid_constant__ CUtensorMap tm_w1, const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + kSmemCtrl);
  volatile int* abort_flag = &ctrl->abort;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();     // 0 = leader
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctrl->full[s], 1);
      mbar_init(&ctrl->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&ctrl->acc_full[a], 1);
      mbar_init(&ctrl->acc_empty[a], 2 * 4 * 32);
    }
    mbar_init(&ctrl->mma_done, 1);
    ctrl->abort = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(&ctrl->tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers initialised and TMEM allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;

  if (warp == kLoadWarp) {
    // ------------------------------------------------------ TMA producer ----
    if (lane == 0) {
      prefetch_tensormap(&tm_x);
      prefetch_tensormap(&tm_w0);
      prefetch_tensormap(&tm_w1);
      const uint32_t full0 = mapa_shared(smem_u32(&ctrl->full[0]), 0);  // leader's barriers
      int it = 0;
      bool ok = true;
      for (int t = pair; t < p.n_tiles && ok; t += n_pairs) {
        const Tile tl = tile_at(p, t);
        const CUtensorMap* wmap = tl.stream == 0 ? &tm_w0 : &tm_w1;
        const int row0 = tl.b * p.N + tl.tok0 + kBM * static_cast<int>(rank);
        const int f0 = tl.nt * kBN + kBNh * static_cast<int>(rank);
        for (int ks = 0; ks < p.k_steps; ++ks, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&ctrl->empty[s], (static_cast<uint32_t>(it / kStages) & 1u) ^ 1u, abort_flag,
                         p.timeout_ns)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + kSmemRing + s * kStageBytes;
          if (rank == 0) mbar_arrive_expect_tx(&ctrl->full[s], 2 * kStageBytes);
          tma_load_2d_pair(st, &tm_x, full0 + s * 8, ks * kBK, row0);
          tma_load_2d_pair(st + kABytes, wmap, full0 + s * 8, ks * kBK, f0);
        }
      }
      // Drain (leader): every fill of both CTAs has landed on its barriers.
      if (rank == 0) {
        for (int s = 0; s < kStages && s < it; ++s) {
          const int last = s + ((it - 1 - s) / kStages) * kStages;
          drain_wait(&ctrl->full[s], static_cast<uint32_t>(last / kStages) & 1u, p.timeout_ns);
        }
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------- MMA issuer (leader) ----
    if (lane == 0) {
      if (rank == 0) {
        constexpr uint32_t idesc = make_idesc(1, 1, false, 2 * kBM, kBN);  // M=256 over the pair
        const uint32_t ring = smem_u32(smem + kSmemRing);
        int it = 0;
        bool ok = true;
        int lt = 0;
        for (int t = pair; t < p.n_tiles && ok; t += n_pairs, ++lt) {
          const int a = lt & 1;
          ok = mbar_wait(&ctrl->acc_empty[a], (static_cast<uint32_t>(lt >> 1) & 1u) ^ 1u, abort_flag,
                         p.timeout_ns);
          if (!ok) break;
          tc_fence_after();
          const uint32_t d = tmem + a * kBN;
          for (int ks = 0; ks < p.k_steps; ++ks, ++it) {
            const int s = it % kStages;
            // TMA-filled stage: its completion is what the barrier reports,
            // so the MMAs may read it right after the wait.
            ok = mbar_wait(&ctrl->full[s], static_cast<uint32_t>(it / kStages) & 1u, abort_flag, p.timeout_ns);
            if (!ok) break;
            const uint32_t sa = ring + s * kStageBytes;
            const uint32_t sb = sa + kABytes;
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              mma_f16_ss_pair(d, smem_desc_sw128(sa + kk * 32, 16, 1024), smem_desc_sw128(sb + kk * 32, 16, 1024),
                              idesc, (ks > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit_pair(&ctrl->empty[s], kPairMask);
          }
          if (!ok) break;
          mma_commit_pair(&ctrl->acc_full[a], kPairMask);
        }
        mma_commit_pair(&ctrl->mma_done, kPairMask);
      }
      // Both CTAs: no TMEM release before every pair MMA has completed.
      drain_wait(&ctrl->mma_done, 0, p.timeout_ns);
    }
    __syncwarp();
  } else {
    // --------------------------------------------------------- epilogue ----
    const int wq = warp & 3;                   // TMEM lane quarter
    const int r = wq * 32 + lane;              // row within this CTA's half of the tile
    const uint32_t lane_sel = static_cast<uint32_t>(wq * 32) << 16;
    const int HD = p.H * kD;
    const uint32_t acc_empty0 = mapa_shared(smem_u32(&ctrl->acc_empty[0]), 0);  // leader's barriers
    int lt = 0;
    bool ok = true;
    for (int t = pair; t < p.n_tiles && ok; t += n_pairs, ++lt) {
      const int a = lt & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&ctrl->acc_full[a], static_cast<uint32_t>(lt >> 1) & 1u, abort_flag,
                                             p.timeout_ns));
      if (!ok) break;
      tc_fence_after();
      const Tile tl = tile_at(p, t);
      const int f0 = tl.nt * kBN;
      const int part = f0 / HD;                // 0 = Q, 1 = K, 2 = V
      const int h0 = (f0 - part * HD) / kD;
      const int tok = tl.tok0 + kBM * static_cast<int>(rank) + r;
      const bool store = tok < tl.tok_end;
      const float* nw = part == 0 ? p.qw[tl.stream] : (part == 1 ? p.kw[tl.stream] : nullptr);
      const float* rope = p.rope + static_cast<size_t>(store ? tok : 0) * 128;
      __nv_bfloat16* orow = p.out[part] + ((static_cast<size_t>(tl.b) * p.N + tok) * p.H + h0) * kD;
#pragma unroll 1
      for (int j = 0; j < 2; ++j) {            // the tile's two heads
        const uint32_t col = tmem + lane_sel + a * kBN + j * kD;
        float rs = 1.f;
        if (part < 2) {
          // Pass 1: sum of squares of the row's 128 channels.
          float ss0 = 0.f, ss1 = 0.f;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t v[32];
            tmem_ld32(col + c * 32, v);
            tmem_ld_wait(v);
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              ss0 = fmaf(__uint_as_float(v[i]), __uint_as_float(v[i]), ss0);
              ss1 = fmaf(__uint_as_float(v[i + 1]), __uint_as_float(v[i + 1]), ss1);
            }
          }
          rs = rsqrtf((ss0 + ss1) * (1.0f / kD) + p.eps);
        }
        // Pass 2: scale, weight, rotate (Q, K), round to bf16, store.
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld32(col + c * 32, v);
          tmem_ld_wait(v);
          uint32_t packed[16];
          if (part < 2) {
            float w[32];
            if (nw != nullptr) {
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float4 q4 = __ldg(reinterpret_cast<const float4*>(nw + c * 32) + i);
                w[4 * i] = q4.x; w[4 * i + 1] = q4.y; w[4 * i + 2] = q4.z; w[4 * i + 3] = q4.w;
              }
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) w[i] = 1.f;
            }
            // Channels c*32 .. c*32+31 are pairs c*16 .. c*16+15 of the
            // table row (pairs 0-31 row axis, 32-63 column axis).
            const float4* rp = reinterpret_cast<const float4*>(rope + c * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 cs = __ldg(rp + i);  // (cos, sin) of pairs 2i, 2i+1 of this chunk
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const int e = 4 * i + 2 * u;
                const float a0 = __uint_as_float(v[e]) * rs * w[e];
                const float a1 = __uint_as_float(v[e + 1]) * rs * w[e + 1];
                const float cc = u == 0 ? cs.x : cs.z;
                const float sn = u == 0 ? cs.y : cs.w;
                packed[2 * i + u] = pack_bf16x2(fmaf(a0, cc, -a1 * sn), fmaf(a0, sn, a1 * cc));
              }
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i)
              packed[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
          }
          if (store) {
            uint4* dst = reinterpret_cast<uint4*>(orow + j * kD + c * 32);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
              __stcs(dst + q4, make_uint4(packed[4 * q4], packed[4 * q4 + 1], packed[4 * q4 + 2], packed[4 * q4 + 3]));
          }
        }
      }
      tc_fence_before();
      mbar_arrive_cluster(acc_empty0 + a * 8);
    }
  }

  tc_fence_before();
  cluster_sync();  // neither CTA leaves while the pair may still touch its memory
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace qkvgemm

cudaError_t launch_qkv_fused(const QkvProblem& q, cudaStream_t s) {
  using namespace qkvgemm;
  CUtensorMap tx, tw0, tw1;
  cudaError_t e;
  const long long rows = static_cast<long long>(q.B) * q.N;
  if ((e = make_kmajor_map(&tx, q.x, rows, q.C, kBM)) != cudaSuccess) return e;
  const void* w0 = q.w[0] != nullptr ? q.w[0] : q.w[1];
  const void* w1 = q.w[1] != nullptr ? q.w[1] : q.w[0];
  if ((e = make_kmajor_map(&tw0, w0, 3LL * q.H * kD, q.C, kBNh)) != cudaSuccess) return e;
  if ((e = make_kmajor_map(&tw1, w1, 3LL * q.H * kD, q.C, kBNh)) != cudaSuccess) return e;
  if ((e = set_smem_attr(reinterpret_cast<const void*>(qkv_fused_kernel), kSmemBytes)) != cudaSuccess) return e;
  Params p;
  p.rope = q.rope;
  for (int i = 0; i < 2; ++i) {
    p.qw[i] = q.qw[i];
    p.kw[i] = q.kw[i];
  }
  p.out[0] = static_cast<__nv_bfloat16*>(q.q);
  p.out[1] = static_cast<__nv_bfloat16*>(q.k);
  p.out[2] = static_cast<__nv_bfloat16*>(q.v);
  p.B = q.B;
  p.N = q.N;
  p.H = q.H;
  p.n_txt = q.n_txt;
  p.k_steps = q.C / kBK;
  p.tiles_txt = (q.n_txt + 2 * kBM - 1) / (2 * kBM);
  p.tiles_img = (q.N - q.n_txt + 2 * kBM - 1) / (2 * kBM);
  p.n_tiles_n = 3 * q.H * kD / kBN;
  {
    // Raster groups: the W panels of one group (kBN rows x C channels per
    // feature tile, bf16) take at most 32 MiB, so that with the copies both
    // halves of the L2 may hold they stay resident next to the x rows and
    // the output lines in flight.
    const long long panel = static_cast<long long>(kBN) * q.C * 2;
    const long long budget = 32LL << 20;
    const int n_groups = static_cast<int>((p.n_tiles_n * panel + budget - 1) / budget);
    p.group_n = (p.n_tiles_n + n_groups - 1) / n_groups;
  }
  const long long n_tiles = static_cast<long long>(q.B) * (p.tiles_txt + p.tiles_img) * p.n_tiles_n;
  if (n_tiles > 0x7fffffff) return cudaErrorInvalidValue;
  p.n_tiles = static_cast<int>(n_tiles);
  p.eps = q.eps;
  p.timeout_ns = q.timeout_ns;
  const int sms = device_sm_count();
  if (sms < 2) return cudaErrorInvalidDevice;
  const int pairs = p.n_tiles < sms / 2 ? p.n_tiles : sms / 2;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, qkv_fused_kernel, tx, tw0, tw1, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return e;
  }
  return cudaGetLastError();
}

// (cos, sin) of every token's 64 RoPE pairs; one thread per (token, pair).
__global__ void rope_table_kernel(const __grid_constant__ PrologueArgs a, float2* table) {
  const long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= static_cast<long long>(a.N) * 64) return;
  const int t = static_cast<int>(e >> 6), pr = static_cast<int>(e & 63);
  int row, col;
  token_pos(a, t, row, col);
  constexpr double kTwoPi = 6.283185307179586476925286766559;
  constexpr double kInvTwoPi = 0.15915494309189533576888376337251;
  const double phi = static_cast<double>(pr < 32 ? row : col) * a.omega[pr & 31];
  const double red = phi - rint(phi * kInvTwoPi) * kTwoPi;
  float sn, cs;
  sincosf(static_cast<float>(red), &sn, &cs);
  table[e] = make_float2(cs, sn);
}

cudaError_t launch_rope_table(const PrologueArgs& a, float* table, cudaStream_t s) {
  const long long n = static_cast<long long>(a.N) * 64;
  const unsigned grid = static_cast<unsigned>((n + 255) / 256);
  rope_table_kernel<<<grid, 256, 0, s>>>(a, reinterpret_cast<float2*>(table));
  return cudaGetLastError();
}

}  // namespace jattn
