// C-ABI of the jattn library (declared in include/jattn.h): argument
// checks, tensor-map encoding and kernel launches.  Built as one
// translation unit with the kernels so that device globals need no
// relocatable device code.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>

#include "jattn.h"
#include "jattn_internal.h"
#include "sm100_ptx.cuh"

#include "attn_bf16.cu"
#include "attn_fp8.cu"
#include "qkv_gemm.cu"
#include "prologue.cu"
#include "repair.cu"
#include "sparse.cu"

namespace jattn {

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<EncodeTiledFn>(p);
    }
  });
  return fn;
}

// Wait-timeout self test: one thread waits on a barrier nothing completes.
__global__ void wait_selftest_kernel(uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, timeout_ns);
  __syncthreads();
}

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // 2 s per wait

thread_local cudaError_t t_last_cuda_error = cudaSuccess;

int map_err(cudaError_t e) {
  if (e == cudaSuccess) return JATTN_OK;
  t_last_cuda_error = e;
  return JATTN_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_common(int B, int H, int N_txt, int N_img, int N_ref, int d) {
  if (B < 1 || H < 1 || N_txt < 0 || N_img < 0 || N_ref < 0) return JATTN_ERR_INVALID_ARG;
  if (B > 65535 || H > 65535) return JATTN_ERR_INVALID_ARG;
  const long long N = static_cast<long long>(N_txt) + N_img + N_ref;
  if (N < 1 || N > (1ll << 30)) return JATTN_ERR_INVALID_ARG;
  if (d != kHeadDim) return JATTN_ERR_UNSUPPORTED;
  // Element offsets are formed in 64 bits; keep B*N*H*d within int64 and
  // each tensor below 2^40 bytes (TMA global stride limit).
  if (static_cast<long long>(B) * N * H * d * 2 >= (1ll << 40)) return JATTN_ERR_INVALID_ARG;
  return JATTN_OK;
}

// Validates the position and RoPE parameters against the stream sizes and
// fills the position fields and frequencies of `a`; returns a jattn_status.
static_assert(JATTN_MAX_REF_GRIDS == kMaxRefGrids, "reference-grid limit");

int fill_positions(PrologueArgs& a, const jattn_prologue_params* p, int N_txt, int N_img, int N_ref) {
  if (p == nullptr) return JATTN_ERR_INVALID_ARG;
  if (p->img_h < 0 || p->img_w < 0 || static_cast<long long>(p->img_h) * p->img_w != N_img)
    return JATTN_ERR_INVALID_ARG;
  if (!(p->rope_theta > 0.f) || !std::isfinite(p->rope_theta)) return JATTN_ERR_INVALID_ARG;
  a.n_txt = N_txt;
  a.n_img = N_img;
  a.img_w = p->img_w > 0 ? p->img_w : 1;
  a.n_grids = 0;
  if (p->n_ref_grids == 0) {
    if (p->ref_h < 0 || p->ref_w < 0 || p->ref_row_offset < 0 ||
        static_cast<long long>(p->ref_h) * p->ref_w != N_ref)
      return JATTN_ERR_INVALID_ARG;
    if (N_ref > 0) {
      a.n_grids = 1;
      a.grid_end[0] = N_ref;
      a.grid_w[0] = p->ref_w;
      a.grid_row[0] = p->ref_row_offset;
      a.grid_col[0] = 0;
    }
  } else {
    if (p->n_ref_grids < 0 || p->n_ref_grids > JATTN_MAX_REF_GRIDS || p->ref_grids == nullptr)
      return JATTN_ERR_INVALID_ARG;
    long long end = 0;
    for (int g = 0; g < p->n_ref_grids; ++g) {
      const jattn_ref_grid& r = p->ref_grids[g];
      if (r.h < 1 || r.w < 1 || r.row_offset < 0 || r.col_offset < 0) return JATTN_ERR_INVALID_ARG;
      end += static_cast<long long>(r.h) * r.w;
      if (end > N_ref) return JATTN_ERR_INVALID_ARG;
      a.grid_end[g] = static_cast<int>(end);
      a.grid_w[g] = r.w;
      a.grid_row[g] = r.row_offset;
      a.grid_col[g] = r.col_offset;
    }
    if (end != N_ref) return JATTN_ERR_INVALID_ARG;
    a.n_grids = p->n_ref_grids;
  }
  for (int i = 0; i < 32; ++i) a.omega[i] = std::pow(static_cast<double>(p->rope_theta), -2.0 * i / 64.0);
  return JATTN_OK;
}

}  // namespace

cudaError_t make_act_map(CUtensorMap* map, const void* ptr, int B, int N, int H, int elem_bytes) {
  return make_act_map_box(map, ptr, B, N, H, elem_bytes, 128);
}

cudaError_t make_act_map_box(CUtensorMap* map, const void* ptr, int B, int N, int H, int elem_bytes,
                             int box_tokens) {
  EncodeTiledFn fn = encoder();
  if (fn == nullptr) return cudaErrorNotSupported;
  const cuuint64_t row = static_cast<cuuint64_t>(kHeadDim) * elem_bytes;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {row, row * H, row * H * N};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(128 / elem_bytes), 1, static_cast<cuuint32_t>(box_tokens), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUtensorMapDataType dt = elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  CUresult r = fn(map, dt, 4, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_rows_map(CUtensorMap* map, const void* ptr, int B, int N, int H, int box_heads, int box_tokens) {
  EncodeTiledFn fn = encoder();
  if (fn == nullptr) return cudaErrorNotSupported;
  const cuuint64_t row = static_cast<cuuint64_t>(kHeadDim) * 2;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {row, row * H, row * H * N};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(kHeadDim), static_cast<cuuint32_t>(box_heads),
                       static_cast<cuuint32_t>(box_tokens), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_kmajor_map(CUtensorMap* map, const void* ptr, long long rows, int cols, int box_rows) {
  EncodeTiledFn fn = encoder();
  if (fn == nullptr) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

int device_sm_count() {
  constexpr int kMaxDev = 64;
  static std::atomic<int> cached[kMaxDev];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < kMaxDev) {
    const int c = cached[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < kMaxDev) cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

cudaError_t set_smem_attr(const void* func, int bytes) {
  // Remembers the largest limit set per device and kernel; a kernel whose
  // shared memory depends on the problem size is raised again when a call
  // needs more.
  constexpr int kMaxDev = 64;
  constexpr int kMaxFuncs = 16;
  static std::mutex mu;
  static const void* done_func[kMaxDev][kMaxFuncs] = {};
  static int done_bytes[kMaxDev][kMaxFuncs] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  int slot = -1;
  if (dev >= 0 && dev < kMaxDev) {
    for (int i = 0; i < kMaxFuncs && slot < 0; ++i)
      if (done_func[dev][i] == func) slot = i;
    if (slot >= 0 && done_bytes[dev][slot] >= bytes) return cudaSuccess;
  }
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < kMaxDev) {
    for (int i = 0; i < kMaxFuncs && slot < 0; ++i)
      if (done_func[dev][i] == nullptr) slot = i;
    if (slot >= 0) {
      done_func[dev][slot] = func;
      done_bytes[dev][slot] = bytes;
    }
  }
  return cudaSuccess;
}

cudaError_t launch_wait_selftest(uint64_t timeout_ns, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>(timeout_ns);
  return cudaGetLastError();
}

}  // namespace jattn

using namespace jattn;

extern "C" {

const char* jattn_status_string(int status) {
  switch (status) {
    case JATTN_OK: return "JATTN_OK";
    case JATTN_ERR_INVALID_ARG: return "JATTN_ERR_INVALID_ARG";
    case JATTN_ERR_UNSUPPORTED: return "JATTN_ERR_UNSUPPORTED";
    case JATTN_ERR_MISALIGNED: return "JATTN_ERR_MISALIGNED";
    case JATTN_ERR_CUDA: return "JATTN_ERR_CUDA";
    case JATTN_ERR_TIMEOUT: return "JATTN_ERR_TIMEOUT";
    default: return "JATTN_ERR_UNKNOWN";
  }
}

int jattn_prologue(const void* q, const void* k, const void* v, void* q_out, void* k_out, void* v_out,
                   float* q_scale, float* k_scale, float* v_scale, int B, int H, int N_txt, int N_img, int N_ref,
                   int d, int mode, const jattn_prologue_params* p, void* cuda_stream) {
  int st = check_common(B, H, N_txt, N_img, N_ref, d);
  if (st != JATTN_OK) return st;
  if (p == nullptr || (mode != JATTN_PROLOGUE_BF16 && mode != JATTN_PROLOGUE_FP8)) return JATTN_ERR_INVALID_ARG;
  PrologueArgs a;
  std::memset(&a, 0, sizeof(a));
  if ((st = fill_positions(a, p, N_txt, N_img, N_ref)) != JATTN_OK) return st;
  if (!(p->eps >= 0.f) || !std::isfinite(p->eps)) return JATTN_ERR_INVALID_ARG;
  if (q == nullptr || k == nullptr || q_out == nullptr || k_out == nullptr) return JATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_out) || !aligned16(k_out)) return JATTN_ERR_MISALIGNED;
  if (!aligned16(p->q_norm_w) || !aligned16(p->k_norm_w)) return JATTN_ERR_MISALIGNED;
  if (mode == JATTN_PROLOGUE_FP8) {
    if (v == nullptr || v_out == nullptr || q_scale == nullptr || k_scale == nullptr || v_scale == nullptr)
      return JATTN_ERR_INVALID_ARG;
    if (!aligned16(v) || !aligned16(v_out)) return JATTN_ERR_MISALIGNED;
    if ((reinterpret_cast<uintptr_t>(q_scale) | reinterpret_cast<uintptr_t>(k_scale) |
         reinterpret_cast<uintptr_t>(v_scale)) & 3u)
      return JATTN_ERR_MISALIGNED;
  }
  a.q = q; a.k = k; a.v = v;
  a.q_out = q_out; a.k_out = k_out; a.v_out = v_out;
  a.q_scale = q_scale; a.k_scale = k_scale; a.v_scale = v_scale;
  a.q_w = p->q_norm_w; a.k_w = p->k_norm_w;
  a.B = B; a.H = H; a.N = N_txt + N_img + N_ref;
  a.eps = p->eps;
  a.timeout_ns = kDefaultTimeoutNs;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  return map_err(mode == JATTN_PROLOGUE_BF16 ? launch_prologue_bf16(a, s) : launch_prologue_fp8(a, s));
}

int jattn_fwd_bf16(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N_txt,
                   int N_img, int N_ref, int d, float softmax_scale, void* cuda_stream) {
  int st = check_common(B, H, N_txt, N_img, N_ref, d);
  if (st != JATTN_OK) return st;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return JATTN_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return JATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return JATTN_ERR_MISALIGNED;
  AttnProblem pr;
  std::memset(&pr, 0, sizeof(pr));
  pr.q = q; pr.k = k; pr.v = v; pr.o = o; pr.lse = lse;
  pr.B = B; pr.H = H; pr.N = N_txt + N_img + N_ref;
  pr.softmax_scale = softmax_scale;
  pr.timeout_ns = kDefaultTimeoutNs;
  return map_err(launch_attn_bf16(pr, static_cast<cudaStream_t>(cuda_stream)));
}

int jattn_sparse_select(const void* q, const void* k, float* qbar, float* kbar, float* probs, int* kv_idx,
                        int* kv_cnt, int B, int H, int N_txt, int N_img, int N_ref, int d, float softmax_scale,
                        float tau, void* cuda_stream) {
  int st = check_common(B, H, N_txt, N_img, N_ref, d);
  if (st != JATTN_OK) return st;
  if (q == nullptr || k == nullptr || qbar == nullptr || kbar == nullptr || kv_idx == nullptr || kv_cnt == nullptr)
    return JATTN_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return JATTN_ERR_INVALID_ARG;
  if (!(tau >= 0.f) || !std::isfinite(tau)) return JATTN_ERR_INVALID_ARG;
  const int N = N_txt + N_img + N_ref;
  if (N > (1 << 22)) return JATTN_ERR_INVALID_ARG;  // key-block scores are staged in shared memory
  if (!aligned16(q) || !aligned16(k) || !aligned16(qbar) || !aligned16(kbar) ||
      (reinterpret_cast<uintptr_t>(probs) & 3u) || (reinterpret_cast<uintptr_t>(kv_idx) & 3u) ||
      (reinterpret_cast<uintptr_t>(kv_cnt) & 3u))
    return JATTN_ERR_MISALIGNED;
  SparseProblem sp;
  std::memset(&sp, 0, sizeof(sp));
  sp.q = q; sp.k = k; sp.qbar = qbar; sp.kbar = kbar; sp.probs = probs; sp.kv_idx = kv_idx; sp.kv_cnt = kv_cnt;
  sp.B = B; sp.H = H; sp.N = N;
  sp.softmax_scale = softmax_scale;
  sp.tau = tau;
  return map_err(launch_sparse_select(sp, static_cast<cudaStream_t>(cuda_stream)));
}

int jattn_fwd_bf16_sparse(const void* q, const void* k, const void* v, void* o, float* lse, const int* kv_idx,
                          const int* kv_cnt, int B, int H, int N_txt, int N_img, int N_ref, int d,
                          float softmax_scale, void* cuda_stream) {
  int st = check_common(B, H, N_txt, N_img, N_ref, d);
  if (st != JATTN_OK) return st;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || kv_idx == nullptr || kv_cnt == nullptr)
    return JATTN_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return JATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(kv_idx) & 3u) ||
      (reinterpret_cast<uintptr_t>(kv_cnt) & 3u))
    return JATTN_ERR_MISALIGNED;
  AttnProblem pr;
  std::memset(&pr, 0, sizeof(pr));
  pr.q = q; pr.k = k; pr.v = v; pr.o = o; pr.lse = lse;
  pr.B = B; pr.H = H; pr.N = N_txt + N_img + N_ref;
  pr.softmax_scale = softmax_scale;
  pr.timeout_ns = kDefaultTimeoutNs;
  return map_err(launch_attn_bf16_sparse(pr, kv_idx, kv_cnt, static_cast<cudaStream_t>(cuda_stream)));
}

int jattn_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* q_scale, const float* k_scale,
                  const float* v_scale, void* o, float* lse, int B, int H, int N_txt, int N_img, int N_ref, int d,
                  float softmax_scale, void* cuda_stream) {
  int st = check_common(B, H, N_txt, N_img, N_ref, d);
  if (st != JATTN_OK) return st;
  if (q8 == nullptr || k8 == nullptr || v8 == nullptr || o == nullptr || q_scale == nullptr ||
      k_scale == nullptr || v_scale == nullptr)
    return JATTN_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return JATTN_ERR_INVALID_ARG;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8) || !aligned16(o) ||
      ((reinterpret_cast<uintptr_t>(lse) | reinterpret_cast<uintptr_t>(q_scale) |
        reinterpret_cast<uintptr_t>(k_scale) | reinterpret_cast<uintptr_t>(v_scale)) & 3u))
    return JATTN_ERR_MISALIGNED;
  AttnProblem pr;
  std::memset(&pr, 0, sizeof(pr));
  pr.q = q8; pr.k = k8; pr.v = v8;
  pr.q_scale = q_scale; pr.k_scale = k_scale; pr.v_scale = v_scale;
  pr.o = o; pr.lse = lse;
  pr.B = B; pr.H = H; pr.N = N_txt + N_img + N_ref;
  pr.softmax_scale = softmax_scale;
  pr.timeout_ns = kDefaultTimeoutNs;
  cudaError_t e = launch_attn_fp8(pr, static_cast<cudaStream_t>(cuda_stream));
  if (e == cudaErrorNotSupported) return JATTN_ERR_UNSUPPORTED;
  return map_err(e);
}

int jattn_rope_table(float* table, int N_txt, int N_img, int N_ref, const jattn_prologue_params* p,
                     void* cuda_stream) {
  int st = check_common(1, 1, N_txt, N_img, N_ref, kHeadDim);
  if (st != JATTN_OK) return st;
  if (table == nullptr || p == nullptr) return JATTN_ERR_INVALID_ARG;
  if (!aligned16(table)) return JATTN_ERR_MISALIGNED;
  PrologueArgs a;
  std::memset(&a, 0, sizeof(a));
  if ((st = fill_positions(a, p, N_txt, N_img, N_ref)) != JATTN_OK) return st;
  a.B = 1; a.H = 1; a.N = N_txt + N_img + N_ref;
  return map_err(launch_rope_table(a, table, static_cast<cudaStream_t>(cuda_stream)));
}

int jattn_qkv_fused(const void* x, const jattn_qkv_weights* w, const float* rope, void* q, void* k, void* v,
                    int B, int H, int N_txt, int N_img, int N_ref, int d, int C, void* cuda_stream) {
  int st = check_common(B, H, N_txt, N_img, N_ref, d);
  if (st != JATTN_OK) return st;
  if (H % 2 != 0) return JATTN_ERR_UNSUPPORTED;
  if (C < 64 || C > 16384 || C % 64 != 0) return JATTN_ERR_UNSUPPORTED;
  if (x == nullptr || w == nullptr || rope == nullptr || q == nullptr || k == nullptr || v == nullptr)
    return JATTN_ERR_INVALID_ARG;
  if ((N_txt > 0 && w->w_qkv[0] == nullptr) || (N_img + N_ref > 0 && w->w_qkv[1] == nullptr))
    return JATTN_ERR_INVALID_ARG;
  if (!(w->eps >= 0.f) || !std::isfinite(w->eps)) return JATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * (N_txt + N_img + N_ref) * C * 2 >= (1ll << 40)) return JATTN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(rope) || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
      !aligned16(w->w_qkv[0]) || !aligned16(w->w_qkv[1]))
    return JATTN_ERR_MISALIGNED;
  for (int s = 0; s < 2; ++s)
    if (!aligned16(w->q_norm_w[s]) || !aligned16(w->k_norm_w[s])) return JATTN_ERR_MISALIGNED;
  QkvProblem pr;
  std::memset(&pr, 0, sizeof(pr));
  pr.x = x;
  for (int s = 0; s < 2; ++s) {
    pr.w[s] = w->w_qkv[s];
    pr.qw[s] = w->q_norm_w[s];
    pr.kw[s] = w->k_norm_w[s];
  }
  pr.rope = rope;
  pr.q = q; pr.k = k; pr.v = v;
  pr.B = B; pr.H = H; pr.N = N_txt + N_img + N_ref; pr.n_txt = N_txt; pr.C = C;
  pr.eps = w->eps;
  pr.timeout_ns = kDefaultTimeoutNs;
  return map_err(launch_qkv_fused(pr, static_cast<cudaStream_t>(cuda_stream)));
}

namespace {

// Fills the prologue arguments (positions, RoPE frequencies, norm) shared
// by jattn_prologue and the repair selection; returns a jattn_status.
int fill_prologue_args(PrologueArgs& a, const void* q, const void* k, const void* v, int B, int H, int N_txt,
                       int N_img, int N_ref, const jattn_prologue_params* p) {
  std::memset(&a, 0, sizeof(a));
  const int st = fill_positions(a, p, N_txt, N_img, N_ref);
  if (st != JATTN_OK) return st;
  if (!(p->eps >= 0.f) || !std::isfinite(p->eps)) return JATTN_ERR_INVALID_ARG;
  if (!aligned16(p->q_norm_w) || !aligned16(p->k_norm_w)) return JATTN_ERR_MISALIGNED;
  a.q = q; a.k = k; a.v = v;
  a.q_w = p->q_norm_w; a.k_w = p->k_norm_w;
  a.B = B; a.H = H; a.N = N_txt + N_img + N_ref;
  a.eps = p->eps;
  a.timeout_ns = kDefaultTimeoutNs;
  return JATTN_OK;
}

}  // namespace

int jattn_fp8_repair_select(const void* k, const void* v, const void* k8, const void* v8, const float* k_scale,
                            const float* v_scale, const jattn_prologue_params* p, int m, float* err, int* idx,
                            void* k_sel, void* v_sel, int B, int H, int N_txt, int N_img, int N_ref, int d,
                            void* cuda_stream) {
  int st = check_common(B, H, N_txt, N_img, N_ref, d);
  if (st != JATTN_OK) return st;
  const int N = N_txt + N_img + N_ref;
  if (m < 0 || m > N) return JATTN_ERR_INVALID_ARG;
  if (k == nullptr || v == nullptr || k8 == nullptr || v8 == nullptr || k_scale == nullptr || v_scale == nullptr ||
      err == nullptr || (m > 0 && (idx == nullptr || k_sel == nullptr || v_sel == nullptr)))
    return JATTN_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k8) || !aligned16(v8) || !aligned16(k_sel) || !aligned16(v_sel) ||
      ((reinterpret_cast<uintptr_t>(k_scale) | reinterpret_cast<uintptr_t>(v_scale) |
        reinterpret_cast<uintptr_t>(err) | reinterpret_cast<uintptr_t>(idx)) & 3u))
    return JATTN_ERR_MISALIGNED;
  PrologueArgs a;
  if ((st = fill_prologue_args(a, nullptr, k, v, B, H, N_txt, N_img, N_ref, p)) != JATTN_OK) return st;
  RepairProblem r;
  std::memset(&r, 0, sizeof(r));
  r.k8 = k8; r.v8 = v8; r.k_scale = k_scale; r.v_scale = v_scale;
  r.err = err; r.idx = idx; r.k_sel = k_sel; r.v_sel = v_sel; r.m = m;
  return map_err(launch_repair_select(a, r, static_cast<cudaStream_t>(cuda_stream)));
}

int jattn_fp8_repair_apply(const void* q8, const float* q_scale, const void* k8, const void* v8, const float* k_scale,
                           const float* v_scale, const int* idx, const void* k_sel, const void* v_sel, int m,
                           void* o, float* lse, int B, int H, int N_txt, int N_img, int N_ref, int d,
                           float softmax_scale, void* cuda_stream) {
  int st = check_common(B, H, N_txt, N_img, N_ref, d);
  if (st != JATTN_OK) return st;
  const int N = N_txt + N_img + N_ref;
  if (m < 0 || m > N) return JATTN_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return JATTN_ERR_INVALID_ARG;
  if (q8 == nullptr || q_scale == nullptr || k8 == nullptr || v8 == nullptr || k_scale == nullptr ||
      v_scale == nullptr || o == nullptr || lse == nullptr ||
      (m > 0 && (idx == nullptr || k_sel == nullptr || v_sel == nullptr)))
    return JATTN_ERR_INVALID_ARG;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8) || !aligned16(k_sel) || !aligned16(v_sel) || !aligned16(o) ||
      ((reinterpret_cast<uintptr_t>(q_scale) | reinterpret_cast<uintptr_t>(k_scale) |
        reinterpret_cast<uintptr_t>(v_scale) | reinterpret_cast<uintptr_t>(idx) | reinterpret_cast<uintptr_t>(lse)) &
       3u))
    return JATTN_ERR_MISALIGNED;
  RepairProblem r;
  std::memset(&r, 0, sizeof(r));
  r.q8 = q8; r.q_scale = q_scale; r.k8 = k8; r.v8 = v8; r.k_scale = k_scale; r.v_scale = v_scale;
  r.idx = const_cast<int*>(idx); r.k_sel = const_cast<void*>(k_sel); r.v_sel = const_cast<void*>(v_sel);
  r.o = o; r.lse = lse; r.m = m;
  r.timeout_ns = kDefaultTimeoutNs;
  return map_err(launch_repair_apply(r, B, H, N, softmax_scale, static_cast<cudaStream_t>(cuda_stream)));
}

const char* jattn_last_cuda_error(void) { return cudaGetErrorName(t_last_cuda_error); }

int jattn_device_status(void* cuda_stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(cuda_stream));
  if (e != cudaSuccess) return map_err(e);
  unsigned int word = 0;
  if ((e = cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word))) != cudaSuccess) return map_err(e);
  if (word != 0) {
    const unsigned int zero = 0;
    if ((e = cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero))) != cudaSuccess) return map_err(e);
    return JATTN_ERR_TIMEOUT;
  }
  return JATTN_OK;
}

int jattn_selftest_wait_timeout(long long timeout_ns, void* cuda_stream) {
  if (timeout_ns < 1 || timeout_ns > 1000000000ll) return JATTN_ERR_INVALID_ARG;
  return map_err(launch_wait_selftest(static_cast<uint64_t>(timeout_ns), static_cast<cudaStream_t>(cuda_stream)));
}

}  // extern "C"

// Entry point that needs no device allocation by the caller.
#include "noalloc.cu"
