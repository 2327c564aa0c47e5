// Joint attention forward, BF16 operands, for sm_100a.
//
// O = softmax(scale * Q K^T) V over the whole joint [text | image | ref]
// sequence of one (batch, head); the operation the NVIDIA tutorial on
// FLUX 3 Image Klein ("Quantized and sparse attention" section) calls
// VANILLA BF16 attention, the largest share of DiT GPU time at 2048^2.
//
// Design (one CTA = 256 query rows of one (b, h) = two 128-row Q tiles):
//   warps 0-3  softmax for Q tile 0 (TMEM S0 / O0), then its epilogue
//   warps 4-7  softmax for Q tile 1 (TMEM S1 / O1), then its epilogue
//   warp 8     TMA producer: Q tiles once, then K_j, V_j into a ring of
//              32 KB shared-memory slots (128-byte swizzle, two 64-channel
//              boxes per 128-row tile)
//   warp 9     TMEM allocator and the single thread issuing tcgen05.mma
// Tensor memory (512 columns): S0 [0,128) S1 [128,256) O0 [256,384)
// O1 [384,512), all fp32 with TMEM lane = query row.  P_i (bf16, packed two
// per column) overwrites columns [0,64) of S_i and feeds the P.V MMA
// straight from TMEM.
//
// Per KV tile j the MMA thread issues, in order,
//   PV0_j, QK0_{j+1}, PV1_j, QK1_{j+1}
// so that while one softmax warpgroup works on its S tile the tensor core
// runs the other tile's MMAs.  tcgen05.mma ops of one thread execute in
// issue order, so QK_{j+1} writing S_i/P_i after PV_j read P_i is safe, and
// the commit that signals S_i(j+1) also covers PV_i(j): the softmax may then
// rescale O_i and overwrite P_i.
//
// Online softmax in the exp2 domain with a lazy maximum: the reference max
// m of a row only moves when the new tile's max exceeds it by more than 16
// (log2 units); P is then at most 2^16, harmless for bf16 P and fp32 O / l.
// The O rescale (a TMEM read-modify-write) is thus rare after the first
// tiles, keys with outlier logits included.  Tail keys (N not a multiple of
// 128) are masked to -inf; tail query rows read zero-filled Q and are not
// stored.
//
// The row sum is the fp32 sum of the unrounded P plus the bf16 rounding of
// each tile's largest P, so that a dominant key carries the same weight in
// O = sum bf16(P) V and in l; its last step follows the hand-off of P to
// the MMA issuer.  The producer and MMA threads wait with suspending
// mbarrier waits, so that they take no issue slots from the softmax warps
// of their SM sub-partitions while they wait.
//
// Split tail (kSplit): a launch covers whole waves of work items (256
// query rows of one (b, h)), one CTA per SM; the items of a last, partial
// wave are run by a second launch in which a cluster of two CTAs shares an
// item, each over half of the KV tiles.  At the end CTA 1 writes its
// unnormalised O rows, m and l into CTA 0's (then idle) shared memory and
// CTA 0 merges the two halves:
//   m = max(m0, m1),  l = 2^(m0-m) l0 + 2^(m1-m) l1,
//   O = (2^(m0-m) O0 + 2^(m1-m) O1) / l.
// The partial wave then takes half as long.  After a main launch the tail
// uses programmatic dependent launch (its CTAs take SMs as the main
// launch's retire) and completes only after the main launch has.
//
// Block-sparse variant (kSparse): the tutorial's Sol-Attention runs a
// generic block-sparse attention kernel.  A CTA's 256 query rows are one
// query block; it visits only the KV tiles listed for that block (a count
// and increasing tile indices per (b, h, query block)) instead of all of
// them, with the same pipeline.  A block with an empty list writes O = 0
// and LSE = -inf.
#include "jattn_internal.h"
#include "sm100_ptx.cuh"
#include "softmax_sm100.cuh"

namespace jattn {

namespace bf16attn {

constexpr int kBM = 128;           // query rows per Q tile (= TMEM lanes)
constexpr int kTiles = 2;          // Q tiles per CTA
constexpr int kBN = 128;           // keys per KV tile
constexpr int kD = 128;            // head dim
constexpr int kStages = 4;         // K/V ring slots
constexpr int kTileBytes = kBM * kD * 2;       // 32 KB
constexpr int kBoxBytes = kTileBytes / 2;      // 16 KB: 128 rows x 64 channels
constexpr int kSoftmaxWarps = 4 * kTiles;
constexpr int kLoadWarp = kSoftmaxWarps;       // 8
constexpr int kMmaWarp = kSoftmaxWarps + 1;    // 9
constexpr int kThreads = (kSoftmaxWarps + 2) * 32;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 16.0f;

struct Ctrl {
  uint64_t q_full;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[kTiles];
  uint64_t p_full[kTiles];
  uint64_t o_full;
  uint64_t mma_done;
  uint64_t peer_free;     // split, CTA 1: CTA 0's shared memory may take the partial result
  uint64_t partial_full;  // split, CTA 0: CTA 1's partial result has landed
  uint32_t tmem_base;
  int abort;
};

constexpr int kSmemQ = 0;
constexpr int kSmemRing = kTiles * kTileBytes;
constexpr int kSmemCtrl = kSmemRing + kStages * kTileBytes;
constexpr int kSmemBytes = kSmemCtrl + static_cast<int>(sizeof(Ctrl)) + 1024;  // + alignment slack
// Split tail: CTA 1's partial result in CTA 0's Q + ring region, O as
// [32 column quads][256 rows][4] fp32 (each thread's 16-byte stores land in
// consecutive chunks), then m[256] and l[256].
constexpr int kPartO = 0;
constexpr int kPartM = kPartO + kTiles * kBM * kD * 4;  // 128 KB
constexpr int kPartL = kPartM + kTiles * kBM * 4;
static_assert(kPartL + kTiles * kBM * 4 <= kSmemCtrl, "partial result must fit below the barriers");

struct Params {
  __nv_bfloat16* o;
  float* lse;
  const int* kv_idx;  // block-sparse only: [B, H, n_qb, n_kv] tile lists
  const int* kv_cnt;  // block-sparse only: [B, H, n_qb] list lengths
  int H, N;
  int n_qb;           // query blocks (256 rows) per (b, h)
  int item0;          // first work item of this launch; item = (b * H + h) * n_qb + qb
  float scale_log2;
  uint64_t timeout_ns;
};

// Wait that only gives up on time (used while draining at teardown).
__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  int never = 0;
  return mbar_wait_sleep(bar, parity, &never, timeout_ns);
}

template <bool kSparse, bool kSplit>
__global__ void __launch_bounds__(kThreads, 1)
attn_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ Params prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + kSmemCtrl);
  volatile int* abort_flag = &ctrl->abort;

  // The split-tail launch that follows this one may start its CTAs as this
  // grid's CTAs retire (programmatic dependent launch; no-op otherwise).
  if constexpr (!kSplit) asm volatile("griddepcontrol.launch_dependents;");
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Work item of this CTA (split: of its cluster; rank = CTA in the pair).
  const int item = prm.item0 + static_cast<int>(kSplit ? blockIdx.x >> 1 : blockIdx.x);
  const int rank = kSplit ? static_cast<int>(blockIdx.x & 1) : 0;
  const int qb = item % prm.n_qb;
  const int h = (item / prm.n_qb) % prm.H;
  const int b = item / (prm.n_qb * prm.H);
  const int m0 = qb * (kBM * kTiles);
  const int N = prm.N;
  const int n_kv = (N + kBN - 1) / kBN;
  // KV tiles visited: all of them, the query block's list, or (split) one
  // half of them (the host splits only when n_kv >= 2).
  const int* list = nullptr;
  int n_iter = n_kv;
  int kv0 = 0;
  if constexpr (kSparse) {
    list = prm.kv_idx + static_cast<size_t>(item) * n_kv;
    n_iter = min(max(__ldg(prm.kv_cnt + item), 0), n_kv);
  }
  if constexpr (kSplit) {
    const int half = (n_kv + 1) / 2;
    kv0 = rank == 0 ? 0 : half;
    n_iter = rank == 0 ? half : n_kv - half;
  }
  // Tile of the jj-th visit (clamped into range: memory-safe for any list).
  auto tile_of = [&](int jj) -> int {
    if constexpr (kSparse) return min(max(__ldg(list + jj), 0), n_kv - 1);
    return kv0 + jj;
  };

  if (threadIdx.x == 0) {
    mbar_init(&ctrl->q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctrl->kv_full[s], 1);
      mbar_init(&ctrl->kv_empty[s], 1);
    }
    for (int t = 0; t < kTiles; ++t) {
      mbar_init(&ctrl->s_full[t], 1);
      mbar_init(&ctrl->p_full[t], 4 * 32);
    }
    mbar_init(&ctrl->o_full, 1);
    mbar_init(&ctrl->mma_done, 1);
    mbar_init(&ctrl->peer_free, kTiles * kBM);     // every softmax thread of CTA 0
    mbar_init(&ctrl->partial_full, kTiles * kBM);  // every softmax thread of CTA 1
    ctrl->abort = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&ctrl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (kSplit) cluster_sync();  // the peer's barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;

  if (warp == kLoadWarp) {
    // ------------------------------------------------------ TMA producer ----
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      mbar_arrive_expect_tx(&ctrl->q_full, kTiles * kTileBytes);
      for (int t = 0; t < kTiles; ++t) {
        uint8_t* dst = smem + kSmemQ + t * kTileBytes;
        tma_load_4d(dst, &tm_q, &ctrl->q_full, 0, h, m0 + t * kBM, b);
        tma_load_4d(dst + kBoxBytes, &tm_q, &ctrl->q_full, 64, h, m0 + t * kBM, b);
      }
      int it = 0;
      bool ok = true;
      for (int jj = 0; jj < n_iter && ok; ++jj) {
        const int j = tile_of(jj);
        for (int which = 0; which < 2; ++which, ++it) {
          const int slot = it % kStages;
          const uint32_t round = static_cast<uint32_t>(it / kStages);
          if (!mbar_wait_sleep(&ctrl->kv_empty[slot], (round & 1u) ^ 1u, abort_flag, prm.timeout_ns)) {
            ok = false;
            break;
          }
          const CUtensorMap* map = which == 0 ? &tm_k : &tm_v;
          uint8_t* dst = smem + kSmemRing + slot * kTileBytes;
          mbar_arrive_expect_tx(&ctrl->kv_full[slot], kTileBytes);
          tma_load_4d(dst, map, &ctrl->kv_full[slot], 0, h, j * kBN, b);
          tma_load_4d(dst + kBoxBytes, map, &ctrl->kv_full[slot], 64, h, j * kBN, b);
        }
      }
      // Drain: every fill issued has landed before the CTA may exit.
      drain_wait(&ctrl->q_full, 0, prm.timeout_ns);
      for (int s = 0; s < kStages && s < it; ++s) {
        const int last = s + ((it - 1 - s) / kStages) * kStages;  // last fill index of slot s
        drain_wait(&ctrl->kv_full[s], static_cast<uint32_t>(last / kStages) & 1u, prm.timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------- MMA issuer ----
    if (lane == 0) {
      constexpr uint32_t idesc_qk = make_idesc(1, 1, false, kBM, kBN);  // bf16 x bf16, K-major both
      constexpr uint32_t idesc_pv = make_idesc(1, 1, true, kBM, kD);    // P (TMEM) x V (MN-major)
      // Descriptors of the first Q tile and ring slot; the start-address
      // field is bits [0,14) in 16-byte units, so adding (offset >> 4)
      // moves a descriptor within shared memory.
      const uint64_t dq0 = smem_desc_sw128(smem_u32(smem + kSmemQ), 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(smem_u32(smem + kSmemRing), 16, 1024);
      const uint64_t dv0 = smem_desc_sw128(smem_u32(smem + kSmemRing), kBoxBytes, 1024);

      auto issue_qk = [&](int t, int slot) {
        const uint32_t d = tmem + t * kBN;  // S_t
        const uint64_t qa = dq0 + static_cast<uint64_t>((t * kTileBytes) >> 4);
        const uint64_t kb = dk0 + static_cast<uint64_t>((slot * kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kBoxBytes + (kk & 3) * 32) >> 4);
          mma_f16_ss(d, qa + off, kb + off, idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int t, int slot, bool acc) {
        const uint32_t d = tmem + 2 * kBN + t * kD;  // O_t
        const uint32_t p = tmem + t * kBN;           // P_t (packed bf16 in S_t columns)
        const uint64_t vb = dv0 + static_cast<uint64_t>((slot * kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          mma_f16_ts(d, p + kk * 8, vb + static_cast<uint64_t>((kk * 16 * 128) >> 4), idesc_pv,
                     (acc || kk > 0) ? 1u : 0u);
        }
      };

      bool ok = mbar_wait_sleep(&ctrl->q_full, 0, abort_flag, prm.timeout_ns);
      int it = 0;
      if (ok && n_iter > 0) ok = mbar_wait_sleep(&ctrl->kv_full[0], 0, abort_flag, prm.timeout_ns);
      if (ok && n_iter > 0) {
        tc_fence_after();
        issue_qk(0, 0);
        mma_commit(&ctrl->s_full[0]);
        issue_qk(1, 0);
        mma_commit(&ctrl->s_full[1]);
        mma_commit(&ctrl->kv_empty[0]);
        it = 1;
      }
      for (int j = 0; j < n_iter && ok; ++j) {
        const int slot_v = it % kStages;
        ok = mbar_wait_sleep(&ctrl->kv_full[slot_v], static_cast<uint32_t>(it / kStages) & 1u, abort_flag,
                       prm.timeout_ns);
        ++it;
        if (!ok) break;
        const bool has_next = j + 1 < n_iter;
        const int slot_k = it % kStages;
        // Q tile 0
        ok = mbar_wait_sleep(&ctrl->p_full[0], static_cast<uint32_t>(j) & 1u, abort_flag, prm.timeout_ns);
        if (!ok) break;
        tc_fence_after();
        issue_pv(0, slot_v, j > 0);
        if (has_next) {
          ok = mbar_wait_sleep(&ctrl->kv_full[slot_k], static_cast<uint32_t>(it / kStages) & 1u, abort_flag,
                         prm.timeout_ns);
          if (!ok) break;
          tc_fence_after();
          issue_qk(0, slot_k);
          mma_commit(&ctrl->s_full[0]);
        }
        // Q tile 1
        ok = mbar_wait_sleep(&ctrl->p_full[1], static_cast<uint32_t>(j) & 1u, abort_flag, prm.timeout_ns);
        if (!ok) break;
        tc_fence_after();
        issue_pv(1, slot_v, j > 0);
        mma_commit(&ctrl->kv_empty[slot_v]);
        if (has_next) {
          issue_qk(1, slot_k);
          mma_commit(&ctrl->s_full[1]);
          mma_commit(&ctrl->kv_empty[slot_k]);
          ++it;
        }
      }
      if (ok) mma_commit(&ctrl->o_full);
      // Drain: all issued MMAs complete before TMEM is released.
      mma_commit(&ctrl->mma_done);
      drain_wait(&ctrl->mma_done, 0, prm.timeout_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------- softmax + epilogue (x2) ----
    const int t = warp >> 2;                 // Q tile of this warpgroup
    const int wq = warp & 3;                 // TMEM lane quarter
    const int r = wq * 32 + lane;            // row within the tile
    const uint32_t lane_sel = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t s_addr = tmem + lane_sel + t * kBN;
    const uint32_t o_addr = tmem + lane_sel + 2 * kBN + t * kD;
    const float sl2 = prm.scale_log2;

    float m = -INFINITY;  // reference row max (log2 units of scaled logits)
    float l = 0.f;        // row sum of exp2(x - m)
    bool ok = true;
    for (int j = 0; j < n_iter; ++j) {
      const int tile = tile_of(j);  // issued before the wait: its latency hides there
      // Warp-uniform outcome: the tcgen05.ld/st below are warp-collective.
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

      const int nvalid = N - tile * kBN;  // >= 1
      if (nvalid < kBN) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c * 32 + i >= nvalid) sv[c][i] = __float_as_uint(-INFINITY);
      }
      float mx_lo, mx_hi;
      row_max_halves(sv, mx_lo, mx_hi);
      const float mnew = fmaxf(m, fmaxf(mx_lo, mx_hi) * sl2);
      const bool need = mnew > m + kRescaleThreshold;
      float corr = 1.f;
      if (need) {
        corr = ex2_approx(m - mnew);  // 0 on the first tile
        l *= corr;
        m = mnew;
      }
      // Row sum: the fp32 sum of the unrounded P, plus the bf16 rounding of
      // the tile's largest P (formed bit for bit as the packing loop forms
      // it), so that a dominant key has the same weight in the numerator
      // O = sum bf16(P) V and in l.
      const float pm = ex2_approx(fmaf(fmaxf(mx_lo, mx_hi), sl2, -m));
      const float fix = __bfloat162float(__float2bfloat16_rn(pm)) - pm;
      // P = exp2(s * scale * log2e - m), packed two bf16 per 32-bit word in
      // place: keys [0,64) land in sv[0], keys [64,128) in sv[2].
      const float lt = exp_pack_sum<false>(sv, sl2, -m, sl2, -m) + fix;
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

    ok = ok && __all_sync(0xffffffffu, mbar_wait(&ctrl->o_full, 0, abort_flag, prm.timeout_ns));
    if (ok) tc_fence_after();
    const int prow = t * kBM + r;  // row within the CTA's 256
    float a_own = 1.f, a_peer = 0.f;  // split, CTA 0: weights of the two halves
    bool store = ok;
    if constexpr (kSplit) {
      if (rank == 1) {
        // Send the unnormalised O row, m and l to CTA 0 once its shared
        // memory is idle (its MMAs and copies are complete).
        store = false;
        bool free = ok && __all_sync(0xffffffffu, mbar_wait(&ctrl->peer_free, 0, abort_flag, prm.timeout_ns));
        if (free) {
          fence_acq_rel_cluster();
          const uint32_t base = mapa_shared(smem_u32(smem), 0);
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t ov[32];
            tmem_ld32(o_addr + c * 32, ov);
            tmem_ld_wait(ov);
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              st_cluster_v4(base + kPartO + (((c * 8 + q4) * (kTiles * kBM) + prow) << 4), ov[4 * q4], ov[4 * q4 + 1],
                            ov[4 * q4 + 2], ov[4 * q4 + 3]);
          }
          st_cluster_f32(base + kPartM + prow * 4, m);
          st_cluster_f32(base + kPartL + prow * 4, l);
          mbar_arrive_cluster(mapa_shared(smem_u32(&ctrl->partial_full), 0));
        }
      } else {
        // This CTA's Q and ring are idle: let CTA 1 write there, then merge.
        mbar_arrive_cluster(mapa_shared(smem_u32(&ctrl->peer_free), 1));
        store = ok && __all_sync(0xffffffffu, mbar_wait(&ctrl->partial_full, 0, abort_flag, prm.timeout_ns));
        if (store) {
          fence_acq_rel_cluster();
          const float m1 = *reinterpret_cast<const float*>(smem + kPartM + prow * 4);
          const float l1 = *reinterpret_cast<const float*>(smem + kPartL + prow * 4);
          const float mm = fmaxf(m, m1);
          a_own = ex2_approx(m - mm);
          a_peer = ex2_approx(m1 - mm);
          l = a_own * l + a_peer * l1;
          m = mm;
        }
      }
    }

    if (store) {
      const int row = m0 + prow;
      // l > 0 whenever a tile was visited (the row max contributes 1).
      const bool empty = kSparse && !(l > 0.f);
      const float inv_l = empty ? 0.f : 1.0f / l;
      const float f_own = a_own * inv_l, f_peer = a_peer * inv_l;
      __nv_bfloat16* orow = prm.o + ((static_cast<size_t>(b) * N + row) * prm.H + h) * kD;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t ov[32];
        tmem_ld32(o_addr + c * 32, ov);
        tmem_ld_wait(ov);
        if constexpr (kSparse) {
          if (empty) {
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = 0u;  // O's columns were never written
          }
        }
        float o[32];
        if constexpr (kSplit) {
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float4 pv = *reinterpret_cast<const float4*>(smem + kPartO + (((c * 8 + q4) * (kTiles * kBM) + prow) << 4));
            o[4 * q4 + 0] = fmaf(__uint_as_float(ov[4 * q4 + 0]), f_own, pv.x * f_peer);
            o[4 * q4 + 1] = fmaf(__uint_as_float(ov[4 * q4 + 1]), f_own, pv.y * f_peer);
            o[4 * q4 + 2] = fmaf(__uint_as_float(ov[4 * q4 + 2]), f_own, pv.z * f_peer);
            o[4 * q4 + 3] = fmaf(__uint_as_float(ov[4 * q4 + 3]), f_own, pv.w * f_peer);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __uint_as_float(ov[i]) * inv_l;
        }
        if (row < N) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint4 u;
            u.x = pack_bf16x2(o[8 * q4 + 0], o[8 * q4 + 1]);
            u.y = pack_bf16x2(o[8 * q4 + 2], o[8 * q4 + 3]);
            u.z = pack_bf16x2(o[8 * q4 + 4], o[8 * q4 + 5]);
            u.w = pack_bf16x2(o[8 * q4 + 6], o[8 * q4 + 7]);
            dst[q4] = u;
          }
        }
      }
      if (prm.lse != nullptr && row < N) {
        prm.lse[(static_cast<size_t>(b) * prm.H + h) * N + row] =
            empty ? -INFINITY : (m + __log2f(l)) * 0.69314718055994530942f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  // Split: neither CTA of the pair leaves while the other may still touch
  // its shared memory (every wait above is bounded, so both arrive).
  if constexpr (kSplit) cluster_sync();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  // Split tail: this grid may have started before the preceding one (the
  // main launch) finished; it completes only after that one has, so that
  // stream order holds for the work after the call.
  if constexpr (kSplit) asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace bf16attn


namespace {

template <bool kSparse>
cudaError_t launch_bf16(const AttnProblem& p, const int* kv_idx, const int* kv_cnt, cudaStream_t s) {
  using namespace bf16attn;
  CUtensorMap tq, tk, tv;
  cudaError_t e;
  if ((e = make_act_map(&tq, p.q, p.B, p.N, p.H, 2)) != cudaSuccess) return e;
  if ((e = make_act_map(&tk, p.k, p.B, p.N, p.H, 2)) != cudaSuccess) return e;
  if ((e = make_act_map(&tv, p.v, p.B, p.N, p.H, 2)) != cudaSuccess) return e;
  const int n_qb = (p.N + kBM * kTiles - 1) / (kBM * kTiles);
  const int n_kv = (p.N + kBN - 1) / kBN;
  const long long n_items = static_cast<long long>(n_qb) * p.H * p.B;
  if (n_items > 0x3fffffff) return cudaErrorInvalidValue;
  Params prm;
  prm.o = static_cast<__nv_bfloat16*>(p.o);
  prm.lse = p.lse;
  prm.kv_idx = kv_idx;
  prm.kv_cnt = kv_cnt;
  prm.H = p.H;
  prm.N = p.N;
  prm.n_qb = n_qb;
  prm.item0 = 0;
  prm.scale_log2 = static_cast<float>(static_cast<double>(p.softmax_scale) * 1.4426950408889634074);
  prm.timeout_ns = p.timeout_ns;
  // One CTA per SM: the items beyond the last whole wave form a partial
  // wave.  If it fills at most half of the SMs, those items run split over
  // KV halves (two CTAs each, a cluster per item) in a second launch.
  int n_tail = 0;
  if (!kSparse && n_kv >= 2) {
    const int sms = device_sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;
    const int rem = static_cast<int>(n_items % sms);
    if (2 * rem <= sms) n_tail = rem;
  }
  const int n_main = static_cast<int>(n_items) - n_tail;
  if (n_main > 0) {
    if ((e = set_smem_attr(reinterpret_cast<const void*>(attn_bf16_kernel<kSparse, false>), kSmemBytes)) !=
        cudaSuccess)
      return e;
    attn_bf16_kernel<kSparse, false><<<n_main, kThreads, kSmemBytes, s>>>(tq, tk, tv, prm);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if constexpr (!kSparse) {
    if (n_tail > 0) {
      const void* fn = reinterpret_cast<const void*>(attn_bf16_kernel<false, true>);
      if ((e = set_smem_attr(fn, kSmemBytes)) != cudaSuccess) return e;
      prm.item0 = n_main;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * n_tail, 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = kSmemBytes;
      cfg.stream = s;
      cudaLaunchAttribute attr[2];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      // After a main launch, the tail's CTAs may take SMs as the main
      // launch's CTAs retire: the main kernel releases them at its start,
      // and the tail reads nothing the main launch writes (the inputs were
      // complete before the main launch began).  Without a main launch the
      // tail is ordered normally after whatever precedes it, whose results
      // it reads.
      attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[1].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = n_main > 0 ? 2 : 1;
      if ((e = cudaLaunchKernelEx(&cfg, attn_bf16_kernel<false, true>, tq, tk, tv, prm)) != cudaSuccess) return e;
    }
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bf16(const AttnProblem& p, cudaStream_t s) {
  return launch_bf16<false>(p, nullptr, nullptr, s);
}

cudaError_t launch_attn_bf16_sparse(const AttnProblem& p, const int* kv_idx, const int* kv_cnt, cudaStream_t s) {
  return launch_bf16<true>(p, kv_idx, kv_cnt, s);
}

}  // namespace jattn
