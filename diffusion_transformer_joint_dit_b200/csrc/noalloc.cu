// Block selection of the block-sparse attention without any device
// allocation by the caller: jattn_sparse_select_noalloc (include/jattn.h).
//
// jattn_sparse_select needs a workspace for the pooled block means (qbar,
// kbar) that the caller allocates.  Some callers cannot allocate device
// memory where they make this call: a plugin inside an inference engine
// whose enqueue step may not allocate (the engine owns every byte of device
// memory and hands out only inputs and outputs), code running between the
// begin and end of a stream capture (cudaMalloc is not a stream operation
// and may synchronise the device), or a process that has given all device
// memory to its own pool allocator.  For them the workspace lives in the
// fixed-size file-scope device array below, which every GPU that loads the
// library holds until the process exits.
//
// Included by jattn_api.cu (one translation unit with the kernels).

namespace jattn {

namespace noalloc {

// Capacity of the workspace: 16 MiB of fp32 pooled means, B * H *
// (ceil(N / 256) + ceil(N / 128)) * 128 floats.  That covers B = 2, H = 24
// up to N = 58112 (both 2048^2 workloads: 16896 and 33280 joint tokens).
constexpr size_t kScratchBytes = size_t(16) << 20;
constexpr size_t kScratchFloats = kScratchBytes / sizeof(float);

// The workspace.  In host code this name is only a stand-in for the device
// symbol, not a device address: the kernels get the address that
// cudaGetSymbolAddress returns for the current device (scratch_address).
static __device__ __align__(256) float g_sparse_scratch[kScratchFloats];

// Device address of g_sparse_scratch on the current device, looked up once
// per device (the first call on a device does it; later calls reuse it).
// Returns cudaSuccess and sets *out, or the lookup's error.
cudaError_t scratch_address(float** out) {
  constexpr int kMaxDev = 64;
  static std::atomic<float*> cached[kMaxDev];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < kMaxDev) {
    float* p = cached[dev].load(std::memory_order_acquire);
    if (p != nullptr) {
      *out = p;
      return cudaSuccess;
    }
  }
  float* ptr = nullptr;
  e = cudaGetSymbolAddress(reinterpret_cast<void**>(&ptr), g_sparse_scratch);
  if (e != cudaSuccess) return e;
  if (ptr == nullptr) return cudaErrorInvalidSymbol;
  if (dev >= 0 && dev < kMaxDev) cached[dev].store(ptr, std::memory_order_release);
  *out = ptr;
  return cudaSuccess;
}

}  // namespace noalloc

}  // namespace jattn

extern "C" {

int jattn_sparse_select_noalloc(const void* q, const void* k, float* probs, int* kv_idx, int* kv_cnt, int B, int H,
                                int N_txt, int N_img, int N_ref, int d, float softmax_scale, float tau,
                                void* cuda_stream) {
  using namespace jattn;
  int st = check_common(B, H, N_txt, N_img, N_ref, d);
  if (st != JATTN_OK) return st;
  if (q == nullptr || k == nullptr || kv_idx == nullptr || kv_cnt == nullptr) return JATTN_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return JATTN_ERR_INVALID_ARG;
  if (!(tau >= 0.f) || !std::isfinite(tau)) return JATTN_ERR_INVALID_ARG;
  const int N = N_txt + N_img + N_ref;
  if (N > (1 << 22)) return JATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || (reinterpret_cast<uintptr_t>(probs) & 3u) ||
      (reinterpret_cast<uintptr_t>(kv_idx) & 3u) || (reinterpret_cast<uintptr_t>(kv_cnt) & 3u))
    return JATTN_ERR_MISALIGNED;
  // The pooled means must fit the fixed workspace.
  const size_t nqb = (static_cast<size_t>(N) + JATTN_SPARSE_QBLOCK - 1) / JATTN_SPARSE_QBLOCK;
  const size_t nkb = (static_cast<size_t>(N) + JATTN_SPARSE_KBLOCK - 1) / JATTN_SPARSE_KBLOCK;
  const size_t q_floats = static_cast<size_t>(B) * H * nqb * kHeadDim;
  const size_t k_floats = static_cast<size_t>(B) * H * nkb * kHeadDim;
  if (q_floats + k_floats > noalloc::kScratchFloats) return JATTN_ERR_UNSUPPORTED;
  float* scratch = nullptr;
  cudaError_t e = noalloc::scratch_address(&scratch);
  if (e != cudaSuccess) return map_err(e);
  SparseProblem sp;
  std::memset(&sp, 0, sizeof(sp));
  sp.q = q; sp.k = k;
  sp.qbar = scratch;              // 256-byte aligned
  sp.kbar = scratch + q_floats;   // q_floats is a multiple of 128: 512-byte aligned
  sp.probs = probs; sp.kv_idx = kv_idx; sp.kv_cnt = kv_cnt;
  sp.B = B; sp.H = H; sp.N = N;
  sp.softmax_scale = softmax_scale;
  sp.tau = tau;
  return map_err(launch_sparse_select(sp, static_cast<cudaStream_t>(cuda_stream)));
}

}  // extern "C"
