// Block selection of the block-sparse attention, for sm_100a.
//
// The NVIDIA tutorial on FLUX 3 Image Klein ("Quantized and sparse
// attention" section) runs Sol-Attention, a generic block-sparse attention
// whose sparsity a parameter tau sets, without defining tau or the block
// rule.  Reading implemented here, per (batch, head):
//   pool    qbar_i = mean of the Q' rows of query block i (256 tokens),
//           kbar_j = mean of the K' rows of key block j (128 tokens), the
//           last block of each kind partial                 sparse_pool_kernel
//   score   p_ij = softmax_j(scale * qbar_i . kbar_j)
//   keep    j iff p_ij >= tau / n_kb, plus the first j of largest p_ij;
//           listed in increasing j with their count         sparse_select_kernel
// The lists drive the block-sparse variant of the BF16 attention kernel,
// whose CTA (256 query rows) is exactly one query block and whose KV tile
// (128 keys) is one key block.
#include "jattn_internal.h"
#include "sm100_ptx.cuh"

namespace jattn {

namespace sparse {

constexpr int kD = 128;
constexpr int kQBlock = 256;
constexpr int kKBlock = 128;
constexpr int kPoolHeads = 8;                      // heads per pool CTA
constexpr int kPoolCols = kPoolHeads * (kD / 8);   // 16-byte columns per token row
constexpr int kPoolThreads = 2 * kPoolCols;        // x 2 token halves = 256

// One CTA per (query block, group of 8 heads, b).  Thread (half, col) sums
// its 8 channels of Q' and K' over the 128 tokens of half `half` of the
// query block, in token order; that half is one key block, and the two
// halves' Q sums add (half 0 + half 1) to the query block's.
__global__ void __launch_bounds__(kPoolThreads)
sparse_pool_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, int H, int N,
                   float* __restrict__ qbar, float* __restrict__ kbar) {
  __shared__ float s_q[kPoolCols][8];
  const int col = threadIdx.x % kPoolCols, half = threadIdx.x / kPoolCols;
  const int h = blockIdx.y * kPoolHeads + col / (kD / 8);
  const int c8 = (col % (kD / 8)) * 8;
  const int b = blockIdx.z;
  const int nqb = (N + kQBlock - 1) / kQBlock, nkb = (N + kKBlock - 1) / kKBlock;
  const int t0 = blockIdx.x * kQBlock + half * kKBlock;
  const int t1 = min(t0 + kKBlock, N);
  const bool live = h < H;
  float sq[8], sk[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) sq[i] = sk[i] = 0.f;
  if (live) {
    const size_t stride = static_cast<size_t>(H) * kD;
    const __nv_bfloat16* qp = q + (static_cast<size_t>(b) * N * H + h) * kD + c8;
    const __nv_bfloat16* kp = k + (static_cast<size_t>(b) * N * H + h) * kD + c8;
#pragma unroll 4
    for (int t = t0; t < t1; ++t) {
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(qp + t * stride));
      const uint4 c = __ldg(reinterpret_cast<const uint4*>(kp + t * stride));
      const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        sq[2 * i] += __uint_as_float(aw[i] << 16);
        sq[2 * i + 1] += __uint_as_float(aw[i] & 0xFFFF0000u);
        sk[2 * i] += __uint_as_float(cw[i] << 16);
        sk[2 * i + 1] += __uint_as_float(cw[i] & 0xFFFF0000u);
      }
    }
  }
  // Key block (one half) mean.
  const int kb = blockIdx.x * 2 + half;
  if (live && t0 < N) {
    const float inv = 1.f / static_cast<float>(t1 - t0);
    float4* dst = reinterpret_cast<float4*>(kbar + ((static_cast<size_t>(b) * H + h) * nkb + kb) * kD + c8);
    dst[0] = make_float4(sk[0] * inv, sk[1] * inv, sk[2] * inv, sk[3] * inv);
    dst[1] = make_float4(sk[4] * inv, sk[5] * inv, sk[6] * inv, sk[7] * inv);
  }
  // Query block mean: half 0 + half 1.
  if (half == 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) s_q[col][i] = sq[i];
  }
  __syncthreads();
  if (half == 0 && live) {
    const int q0 = blockIdx.x * kQBlock;
    const float inv = 1.f / static_cast<float>(min(q0 + kQBlock, N) - q0);
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = (sq[i] + s_q[col][i]) * inv;
    float4* dst =
        reinterpret_cast<float4*>(qbar + ((static_cast<size_t>(b) * H + h) * nqb + blockIdx.x) * kD + c8);
    dst[0] = make_float4(m[0], m[1], m[2], m[3]);
    dst[1] = make_float4(m[4], m[5], m[6], m[7]);
  }
}

constexpr int kSelThreads = 256;

// One CTA per (query block, h, b): scores of all key blocks (a warp per key
// block, lane = 4 channels), softmax, threshold and the ordered list.
__global__ void __launch_bounds__(kSelThreads)
sparse_select_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar, int H, int nqb, int nkb,
                     float scale, float thr, float* __restrict__ probs, int* __restrict__ kv_idx,
                     int* __restrict__ kv_cnt) {
  extern __shared__ float s_p[];  // [nkb]
  __shared__ float s_red[kSelThreads / 32];
  __shared__ int s_top[kSelThreads / 32];
  __shared__ unsigned s_tot[kSelThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const size_t bh = static_cast<size_t>(b) * H + h;
  const float4 qv = __ldg(reinterpret_cast<const float4*>(qbar + (bh * nqb + i) * kD) + lane);
  for (int j = warp; j < nkb; j += kSelThreads / 32) {
    const float4 kv = __ldg(reinterpret_cast<const float4*>(kbar + (bh * nkb + j) * kD) + lane);
    float d = qv.x * kv.x + qv.y * kv.y + qv.z * kv.z + qv.w * kv.w;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
    if (lane == 0) s_p[j] = scale * d;
  }
  __syncthreads();
  // Row max.
  float mx = -INFINITY;
  for (int j = threadIdx.x; j < nkb; j += kSelThreads) mx = fmaxf(mx, s_p[j]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) s_red[warp] = mx;
  __syncthreads();
  mx = s_red[0];
  for (int w = 1; w < kSelThreads / 32; ++w) mx = fmaxf(mx, s_red[w]);
  __syncthreads();
  // Softmax denominator, then the probabilities in place.
  float sum = 0.f;
  for (int j = threadIdx.x; j < nkb; j += kSelThreads) sum += expf(s_p[j] - mx);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) s_red[warp] = sum;
  __syncthreads();
  sum = 0.f;
  for (int w = 0; w < kSelThreads / 32; ++w) sum += s_red[w];
  const float inv = 1.f / sum;
  float* prow = probs != nullptr ? probs + (bh * nqb + i) * nkb : nullptr;
  float pm = -1.f;
  int top = 0x7fffffff;
  for (int j = threadIdx.x; j < nkb; j += kSelThreads) {
    const float p = expf(s_p[j] - mx) * inv;
    s_p[j] = p;
    if (prow != nullptr) prow[j] = p;
    if (p > pm) {  // increasing j: keeps the first index of this thread's maximum
      pm = p;
      top = j;
    }
  }
  // The first index of the largest probability, over the block.
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float op = __shfl_xor_sync(0xffffffffu, pm, o);
    const int ot = __shfl_xor_sync(0xffffffffu, top, o);
    if (op > pm || (op == pm && ot < top)) {
      pm = op;
      top = ot;
    }
  }
  __syncthreads();  // s_red reads of the sum are done
  if (lane == 0) {
    s_red[warp] = pm;
    s_top[warp] = top;
  }
  __syncthreads();
  pm = s_red[0];
  top = s_top[0];
  for (int w = 1; w < kSelThreads / 32; ++w) {
    if (s_red[w] > pm || (s_red[w] == pm && s_top[w] < top)) {
      pm = s_red[w];
      top = s_top[w];
    }
  }
  // The keep decision and the list in increasing j.
  int* lrow = kv_idx + (bh * nqb + i) * nkb;
  unsigned base = 0;
  for (int j0 = 0; j0 < nkb; j0 += kSelThreads) {
    const int j = j0 + threadIdx.x;
    const bool keep = j < nkb && (s_p[j] >= thr || j == top);
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    const unsigned within = __popc(bal & ((1u << lane) - 1u));
    __syncthreads();  // s_tot of the previous chunk is consumed
    if (lane == 0) s_tot[warp] = __popc(bal);
    __syncthreads();
    unsigned before = 0, all = 0;
    for (int w = 0; w < kSelThreads / 32; ++w) {
      before += w < warp ? s_tot[w] : 0u;
      all += s_tot[w];
    }
    if (keep) lrow[base + before + within] = j;
    base += all;
  }
  if (threadIdx.x == 0) kv_cnt[bh * nqb + i] = static_cast<int>(base);
}

}  // namespace sparse

cudaError_t launch_sparse_select(const SparseProblem& sp, cudaStream_t s) {
  using namespace sparse;
  const int nqb = (sp.N + kQBlock - 1) / kQBlock, nkb = (sp.N + kKBlock - 1) / kKBlock;
  dim3 pg(nqb, (sp.H + kPoolHeads - 1) / kPoolHeads, sp.B);
  sparse_pool_kernel<<<pg, kPoolThreads, 0, s>>>(static_cast<const __nv_bfloat16*>(sp.q),
                                                 static_cast<const __nv_bfloat16*>(sp.k), sp.H, sp.N, sp.qbar,
                                                 sp.kbar);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int smem = nkb * static_cast<int>(sizeof(float));
  if (smem > 48 * 1024) {
    if ((e = set_smem_attr(reinterpret_cast<const void*>(sparse_select_kernel), smem)) != cudaSuccess) return e;
  }
  // The threshold tau / n_kb, one correctly rounded fp32 division.
  const float thr = sp.tau / static_cast<float>(nkb);
  dim3 sg(nqb, sp.H, sp.B);
  sparse_select_kernel<<<sg, kSelThreads, smem, s>>>(sp.qbar, sp.kbar, sp.H, nqb, nkb, sp.softmax_scale, thr,
                                                     sp.probs, sp.kv_idx, sp.kv_cnt);
  return cudaGetLastError();
}

}  // namespace jattn
