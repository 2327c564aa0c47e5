// Internal launch interface between the C-ABI layer (jattn_api.cu) and the
// kernels.  Not installed; not part of the public C-ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace jattn {

constexpr int kHeadDim = 128;
constexpr int kQuantBlock = 64;
constexpr int kMaxRefGrids = 8;

// Arguments of the prologue kernels, passed by value (__grid_constant__).
struct PrologueArgs {
  const void* q;
  const void* k;
  const void* v;
  void* q_out;
  void* k_out;
  void* v_out;
  float* q_scale;
  float* k_scale;
  float* v_scale;
  const float* q_w;  // nullable: weight 1.0
  const float* k_w;
  int B, H, N;
  int n_txt, n_img, img_w;
  // Reference grids in sequence order: grid g covers reference tokens
  // [grid_end[g - 1], grid_end[g]) (grid_end[-1] = 0), row-major with width
  // grid_w[g], placed at (grid_row[g], grid_col[g]).
  int n_grids;
  int grid_end[kMaxRefGrids];
  int grid_w[kMaxRefGrids];
  int grid_row[kMaxRefGrids];
  int grid_col[kMaxRefGrids];
  float eps;
  uint64_t timeout_ns;  // bound of each barrier wait (FP8 mode)
  // RoPE frequencies of the 32 channel pairs of one axis half,
  // omega_i = theta^(-2i/64), in double so that angles are exact enough.
  double omega[32];
};

cudaError_t launch_prologue_bf16(const PrologueArgs& a, cudaStream_t s);
cudaError_t launch_prologue_fp8(const PrologueArgs& a, cudaStream_t s);

struct AttnProblem {
  const void* q;
  const void* k;
  const void* v;
  const float* q_scale;  // fp8 only
  const float* k_scale;
  const float* v_scale;
  void* o;
  float* lse;  // nullable
  int B, H, N;
  float softmax_scale;
  uint64_t timeout_ns;
};

// Fused QKV projection (qkv_gemm.cu).
struct QkvProblem {
  const void* x;        // bf16 [B, N, C]
  const void* w[2];     // bf16 [3 H d, C] per stream (text, image + reference)
  const float* qw[2];   // [d] per stream, nullable
  const float* kw[2];
  const float* rope;    // [N, 64, 2]
  void* q;
  void* k;
  void* v;
  int B, H, N, n_txt, C;
  float eps;
  uint64_t timeout_ns;
};

cudaError_t launch_qkv_fused(const QkvProblem& q, cudaStream_t s);
cudaError_t launch_rope_table(const PrologueArgs& a, float* table, cudaStream_t s);

// FP8 repair budget (repair.cu).
struct RepairProblem {
  const void* q8;
  const float* q_scale;
  const void* k8;
  const void* v8;
  const float* k_scale;
  const float* v_scale;
  float* err;         // [B, H, N]
  int* idx;           // [B, H, m]
  void* k_sel;        // bf16 [B, H, m, d]
  void* v_sel;
  void* o;            // bf16 [B, N, H, d], corrected in place
  float* lse;         // [B, H, N], corrected in place
  int m;
  uint64_t timeout_ns;  // bound of each barrier wait (apply)
};

cudaError_t launch_repair_select(const PrologueArgs& a, const RepairProblem& r, cudaStream_t s);
cudaError_t launch_repair_apply(const RepairProblem& r, int B, int H, int N, float softmax_scale, cudaStream_t s);

// Block-sparse attention (sparse.cu, attn_bf16.cu).
struct SparseProblem {
  const void* q;      // bf16 Q' [B, N, H, d]
  const void* k;      // bf16 K'
  float* qbar;        // [B, H, n_qb, d] query-block means
  float* kbar;        // [B, H, n_kb, d] key-block means
  float* probs;       // nullable [B, H, n_qb, n_kb]
  int* kv_idx;        // [B, H, n_qb, n_kb]
  int* kv_cnt;        // [B, H, n_qb]
  int B, H, N;
  float softmax_scale, tau;
};

cudaError_t launch_sparse_select(const SparseProblem& sp, cudaStream_t s);
cudaError_t launch_attn_bf16_sparse(const AttnProblem& p, const int* kv_idx, const int* kv_cnt, cudaStream_t s);

cudaError_t launch_attn_bf16(const AttnProblem& p, cudaStream_t s);
cudaError_t launch_attn_fp8(const AttnProblem& p, cudaStream_t s);
cudaError_t launch_wait_selftest(uint64_t timeout_ns, cudaStream_t s);

// 4-D tensor map over a token-major [B, N, H, d=128] tensor with
// `elem_bytes`-byte elements (2 = bf16, 1 = e4m3): dims (d, H, N, B), box
// (128 bytes of channels, 1 head, 128 tokens, 1 batch), 128-byte swizzle,
// zero fill out of bounds.  Encoded through cuTensorMapEncodeTiled, looked
// up via the runtime's driver entry point (no link-time libcuda dependency).
cudaError_t make_act_map(CUtensorMap* map, const void* ptr, int B, int N, int H, int elem_bytes);

// The same view with a box of `box_tokens` tokens (1 .. 256) instead of 128.
cudaError_t make_act_map_box(CUtensorMap* map, const void* ptr, int B, int N, int H, int elem_bytes,
                             int box_tokens);

// 4-D tensor map over a token-major bf16 [B, N, H, d=128] tensor for the
// prologue: box (128 channels, `box_heads` heads, `box_tokens` tokens, 1),
// no swizzle (rows land densely, 256 B each, token-major then head), zero
// fill out of bounds.
cudaError_t make_rows_map(CUtensorMap* map, const void* ptr, int B, int N, int H, int box_heads, int box_tokens);

// 2-D tensor map over a row-major bf16 [rows, cols] matrix read K-major:
// box (64 columns = 128 B, box_rows rows), 128-byte swizzle, zero fill out
// of bounds.
cudaError_t make_kmajor_map(CUtensorMap* map, const void* ptr, long long rows, int cols, int box_rows);

// Number of SMs of the current device (cached per device).
int device_sm_count();

// Raise a kernel's dynamic shared-memory limit on the current device (once
// per device and kernel).
cudaError_t set_smem_attr(const void* func, int bytes);

}  // namespace jattn
