/*
 * jattn — joint text + image (+ reference image) multi-head self-attention
 * forward of one DiT block, for NVIDIA B200 (sm_100a).
 *
 * What the calls compute.  The NVIDIA tutorial on accelerating FLUX 3 Image
 * Klein with TensorRT LLM VisualGen ("FLUX 3 inference with TensorRT LLM
 * VisualGen" section) describes a DiT that processes the text, noisy-target
 * and optional reference-image token streams separately and lets them meet
 * only in one joint attention.  Its "GEMM kernel optimization" section fuses
 * query/key normalisation and rotary position embedding into the QKV
 * projection epilogue; its "Quantized and sparse attention" section runs the
 * attention itself either in BF16 or with FP8 Q/K and FP8 V.  The three
 * calls below are those steps (jattn_qkv_fused, further down, is the
 * projection with the prologue fused into its epilogue):
 *
 *   jattn_prologue   per-head RMSNorm of Q and K, 2-D RoPE on the tokens'
 *                    (row, col) latent-grid positions, optionally followed
 *                    by E4M3 block quantisation of Q', K' and V;
 *   jattn_fwd_bf16   O = softmax(scale * Q' K'^T) V over the whole joint
 *                    sequence (no mask), bf16 in, fp32 accumulate, bf16 out;
 *   jattn_fwd_fp8    the same from E4M3 codes with per-64-token block scales.
 *
 * Layout.  Every activation tensor is token-major [B, N, H, d], the layout a
 * QKV projection writes: element (b, t, h, c) sits at
 * ((b * N + t) * H + h) * d + c.  The joint sequence is the concatenation
 * [text (N_txt) | noisy target image (N_img) | reference image (N_ref)],
 * N = N_txt + N_img + N_ref; the caller lays the streams out contiguously.
 * Image tokens are the latent grid flattened row-major.
 *
 * Ownership and execution.  The caller owns all memory (device pointers
 * unless stated otherwise).  The library never allocates, frees or
 * synchronises inside these calls: each enqueues its kernel(s) on
 * `cuda_stream` (a cudaStream_t; NULL = legacy default stream) and returns.
 * Results are valid once the stream has run the work.
 *
 * Errors.  Arguments are checked before any launch; a rejected call launches
 * nothing and returns a jattn_status below.  After a launch the return is the
 * launch status (cudaGetLastError, which also clears a pending non-sticky
 * error of the calling thread) mapped to JATTN_ERR_CUDA.  Every wait
 * inside the attention kernels is bounded; a wait that runs out sets a device
 * error word and the kernel returns early, leaving its outputs undefined;
 * jattn_device_status() reports and clears it.
 */
#ifndef JATTN_H_
#define JATTN_H_

#if defined(__GNUC__)
#define JATTN_API __attribute__((visibility("default")))
#else
#define JATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  JATTN_OK = 0,
  JATTN_ERR_INVALID_ARG = 1,  /* a size, pointer or enum out of range        */
  JATTN_ERR_UNSUPPORTED = 2,  /* valid, but not built (e.g. head_dim != 128)  */
  JATTN_ERR_MISALIGNED = 3,   /* a pointer is not 16-byte aligned             */
  JATTN_ERR_CUDA = 4,         /* the CUDA runtime reported an error           */
  JATTN_ERR_TIMEOUT = 5       /* a bounded in-kernel wait ran out             */
} jattn_status;

/* Prologue modes. */
#define JATTN_PROLOGUE_BF16 0  /* Q', K' written as bf16; V untouched               */
#define JATTN_PROLOGUE_FP8 1   /* Q', K', V written as E4M3 codes + block scales     */

/* Token block covered by one FP8 scale (tokens of one (batch, head)). */
#define JATTN_FP8_BLOCK 64

/*
 * Position and normalisation parameters of the prologue.
 *
 * RoPE positions (2-D, the reading of the workloads' "split 64/64 over
 * (row, col)"): text token t < N_txt sits at (0, 0); image token
 * t' = t - N_txt at (t' / img_w, t' % img_w); reference token
 * t'' = t - N_txt - N_img at (ref_row_offset + t'' / ref_w, t'' % ref_w).
 * Channels [0, d/2) rotate with the row position, [d/2, d) with the column
 * position; inside a half, adjacent pair (2i, 2i+1) rotates by
 * pos * rope_theta^(-2i/(d/2)).
 *
 * Several reference images (the tutorial's editing command takes one
 * --image per reference; the pages give no position rule for them): with
 * n_ref_grids > 0, the reference stream is the concatenation of
 * n_ref_grids grids in the order of ref_grids, token u of grid g at
 * (row_offset_g + u / w_g, col_offset_g + u % w_g), and ref_h, ref_w,
 * ref_row_offset are ignored; N_ref must equal the sum of h_g * w_g.  One
 * grid {ref_h, ref_w, ref_row_offset, 0} is the single-reference rule.
 *
 * RMSNorm: y = x / sqrt(mean_c(x^2) + eps) * w[c], per (b, t, h), fp32 math.
 * q_norm_w / k_norm_w are device pointers to d fp32 weights, or NULL for 1.0.
 */
#define JATTN_MAX_REF_GRIDS 8

typedef struct {
  int h, w;                /* grid size, each >= 1 */
  int row_offset;          /* position of the grid's first row, >= 0 */
  int col_offset;          /* position of the grid's first column, >= 0 */
} jattn_ref_grid;

typedef struct {
  int img_h, img_w;        /* noisy-target latent grid; N_img must equal img_h * img_w */
  int ref_h, ref_w;        /* reference grid; N_ref must equal ref_h * ref_w (0 x 0 = none) */
  int ref_row_offset;      /* row shift of the reference grid (e.g. img_h) */
  float rope_theta;        /* RoPE base, > 0 (workloads: 10000) */
  float eps;               /* RMSNorm epsilon, >= 0 (workloads: 1e-6) */
  const float* q_norm_w;   /* [d] fp32 device pointer or NULL */
  const float* k_norm_w;   /* [d] fp32 device pointer or NULL */
  int n_ref_grids;         /* 0: the single grid above; 1 .. JATTN_MAX_REF_GRIDS: ref_grids */
  const jattn_ref_grid* ref_grids;  /* host array of n_ref_grids grids, or NULL */
} jattn_prologue_params;

/*
 * jattn_prologue — RMSNorm + 2-D RoPE of Q and K, optional E4M3 quantisation.
 *
 * Source: the QKV-epilogue fusion of query/key normalisation and rotary
 * position embedding ("GEMM kernel optimization" section of the tutorial),
 * and the FP8 Q/K/V attention inputs ("Quantized and sparse attention").
 *
 * q, k, v : bf16 [B, N, H, d] inputs (v is read only in mode FP8).
 * mode JATTN_PROLOGUE_BF16:
 *   q_out, k_out : bf16 [B, N, H, d]; may equal q, k (in place);
 *   v_out, *_scale : ignored (may be NULL).
 * mode JATTN_PROLOGUE_FP8:
 *   q_out, k_out, v_out : E4M3FN codes, 1 byte each, [B, N, H, d];
 *   q_scale, k_scale, v_scale : fp32 [B, H, ceil(N / 64)].
 *   Per (b, h, 64-token block j): amax = max |x| over the block's tokens
 *   and all d channels of the bf16-rounded Q' (resp. K', V);
 *   code = E4M3_RNE_satfinite(x * (448 / amax)), scale = amax / 448, both
 *   fp32 operations correctly rounded; an all-zero block has scale 1 and
 *   zero codes.  The value a code stands for is decode(code) * scale.
 * Sizes: B, H >= 1; d == 128 (else UNSUPPORTED); N = N_txt + N_img + N_ref
 * >= 1; p must be non-NULL and consistent with N_img / N_ref.
 * All tensor pointers must be 16-byte aligned (else MISALIGNED).
 */
JATTN_API int jattn_prologue(const void* q, const void* k, const void* v,
                   void* q_out, void* k_out, void* v_out,
                   float* q_scale, float* k_scale, float* v_scale,
                   int B, int H, int N_txt, int N_img, int N_ref, int d, int mode,
                   const jattn_prologue_params* p, void* cuda_stream);

/*
 * jattn_fwd_bf16 — joint attention forward, BF16 operands.
 *
 * Source: the VANILLA BF16 attention the tutorial's "Quantized and sparse
 * attention" section names as the dominant DiT cost at 2048^2; the joint
 * sequence from "FLUX 3 inference with TensorRT LLM VisualGen".
 *
 * q, k, v : bf16 [B, N, H, d] (Q', K' as the prologue writes them).
 * o       : bf16 [B, N, H, d] output, O = softmax(softmax_scale * Q K^T) V,
 *           every query against all N keys of its (b, h).
 * lse     : optional fp32 [B, H, N] output, ln sum_j exp(scale * q.k_j);
 *           NULL skips it.
 * The stream split (N_txt / N_img / N_ref) is validated (each >= 0, sum
 * >= 1) but does not change the result: the sequence is attended as one.
 * d must be 128; softmax_scale must be finite and > 0.
 * o must not overlap q, k or v.
 * Work items are 256 query rows of one (b, h), taken in (b, h, block)
 * order, one per SM at a time.  When the items past the last whole wave
 * fill at most half of the SMs (and N > 128), each of them runs as a
 * cluster of two CTAs over the two halves of the keys, merged at the end;
 * those rows differ from a one-pass computation by the merge's rounding
 * only.  The result is deterministic: the same inputs on the same GPU give
 * the same bits.
 */
JATTN_API int jattn_fwd_bf16(const void* q, const void* k, const void* v, void* o, float* lse,
                   int B, int H, int N_txt, int N_img, int N_ref, int d,
                   float softmax_scale, void* cuda_stream);

/*
 * jattn_fwd_fp8 — joint attention forward from E4M3 block-quantised inputs.
 *
 * Source: FP8 Q/K and FP8 V attention ("Quantized and sparse attention"
 * section of the tutorial, qk_dtype / v_dtype fp8).
 *
 * q8, k8, v8 : E4M3FN codes [B, N, H, d] as jattn_prologue(mode FP8) writes.
 * q_scale, k_scale, v_scale : fp32 [B, H, ceil(N / 64)] block scales.
 * Computes O = softmax(softmax_scale * Qd Kd^T) Vd with Xd the dequantised
 * values decode(code) * scale.  QK^T runs on E4M3 operands with fp32
 * accumulation and the block scales applied to the fp32 scores; P.V runs
 * with P in FP16 and V's codes widened to FP16 (exact).
 * o : bf16 [B, N, H, d]; lse : optional fp32 [B, H, N].
 */
JATTN_API int jattn_fwd_fp8(const void* q8, const void* k8, const void* v8,
                  const float* q_scale, const float* k_scale, const float* v_scale,
                  void* o, float* lse,
                  int B, int H, int N_txt, int N_img, int N_ref, int d,
                  float softmax_scale, void* cuda_stream);

/*
 * jattn_rope_table — the (cos, sin) of every token's 64 RoPE channel pairs,
 * for jattn_qkv_fused.
 *
 * table : fp32 [N, 64, 2] device output; entry (t, j) = (cos phi, sin phi)
 *         with phi = pos * rope_theta^(-2 (j mod 32) / 64), pos = the row
 *         position of token t for j < 32, its column position for j >= 32
 *         (positions as for jattn_prologue; p's norm fields are ignored).
 * Angles are formed and reduced to [-pi, pi] in double, then evaluated in
 * float.  N = N_txt + N_img + N_ref >= 1; table 16-byte aligned.
 */
JATTN_API int jattn_rope_table(float* table, int N_txt, int N_img, int N_ref,
                     const jattn_prologue_params* p, void* cuda_stream);

/*
 * Weights of the fused QKV projection, per token stream.  The tutorial's DiT
 * processes the text and image streams separately until the joint
 * attention, so each stream has its own projection and Q/K norm weights;
 * reference-image tokens use the image stream's (they are latents of the
 * same kind).  Index 0 = text, 1 = image (and reference).
 *
 * w_qkv[s]    : bf16 [3 H d, C] device pointer, row-major: output feature f
 *               (f < H d: Q head f / d channel f mod d; then K, then V) is
 *               the dot product of a token's C inputs with row f.
 * q_norm_w[s], k_norm_w[s] : [d] fp32 device pointers, or NULL for 1.0.
 * eps         : RMSNorm epsilon (>= 0).
 */
typedef struct {
  const void* w_qkv[2];
  const float* q_norm_w[2];
  const float* k_norm_w[2];
  float eps;
} jattn_qkv_weights;

/*
 * jattn_qkv_fused — QKV projection with query/key RMSNorm and 2-D RoPE in
 * the GEMM epilogue, the fusion the tutorial's "GEMM kernel optimization"
 * section describes, in BF16 (tcgen05 MMAs, fp32 accumulation).
 *
 * x       : bf16 [B, N, C] token activations, the joint sequence
 *           [text | image | reference] of each batch element.
 * w       : per-stream weights (see jattn_qkv_weights); w_qkv[0] may be
 *           NULL when N_txt == 0, w_qkv[1] when N_img + N_ref == 0.
 * rope    : fp32 [N, 64, 2] from jattn_rope_table.
 * q, k, v : bf16 [B, N, H, d] outputs.  For token t of stream s:
 *           Q = RoPE(RMSNorm(x_t W_s,q) * q_norm_w[s]), K likewise with the
 *           K rows and k_norm_w[s], V = x_t W_s,v; each is rounded to bf16
 *           once, from the fp32 accumulator (no intermediate rounding).
 * Sizes: d == 128; H even (two heads per output tile); C a multiple of 64,
 * 64 <= C <= 16384; N >= 1.  Pointers 16-byte aligned.  The outputs must
 * not overlap x or the weights.
 */
JATTN_API int jattn_qkv_fused(const void* x, const jattn_qkv_weights* w, const float* rope,
                    void* q, void* k, void* v,
                    int B, int H, int N_txt, int N_img, int N_ref, int d, int C, void* cuda_stream);

/*
 * FP8 attention with a repair budget (the tutorial's VC-Attention FP8 runs
 * with a budget rho = 0.005: a share rho of the tokens, those that
 * quantisation hurt most, gets a residual correction; "Quantized and
 * sparse attention" section).  Reading implemented, per (batch, head):
 * the m tokens whose key and value rows lost the most in E4M3,
 *   e_t = sum_c (K'_tc - Kd_tc)^2 + sum_c (V_tc - Vd_tc)^2
 * (K' = the bf16 RMSNorm + RoPE of K the prologue quantises, V the bf16
 * input, Kd / Vd their dequantised codes), are attended with their exact
 * rows instead of the dequantised ones; queries stay dequantised.  The
 * tutorial's budget is m = ceil(rho N) (85 at N = 16896).
 *
 * Usage: jattn_prologue(mode FP8) -> jattn_fwd_fp8 (with lse) ->
 * jattn_fp8_repair_select -> jattn_fp8_repair_apply.
 */

/*
 * jattn_fp8_repair_select — per-token errors and the selected tokens.
 *
 * k, v              : bf16 [B, N, H, d] prologue inputs (raw K; V).
 * k8, v8, *_scale   : the prologue's FP8 output for K and V.
 * p                 : the prologue parameters used (positions, k_norm_w, eps).
 * m                 : tokens to repair per (b, h), 0 <= m <= N.
 * err               : fp32 [B, H, N] output, e_t above (fp32 arithmetic).
 * idx               : int32 [B, H, m] output, the m largest e_t of each
 *                     (b, h) (ties to the lower token), in token order.
 * k_sel, v_sel      : bf16 [B, H, m, d] outputs, the exact K' and V rows of
 *                     the selected tokens.
 * idx, k_sel, v_sel may be NULL when m == 0.  Sizes as jattn_prologue;
 * 16-byte aligned tensors, 4-byte aligned scales, err and idx.
 */
JATTN_API int jattn_fp8_repair_select(const void* k, const void* v, const void* k8, const void* v8,
                            const float* k_scale, const float* v_scale, const jattn_prologue_params* p,
                            int m, float* err, int* idx, void* k_sel, void* v_sel,
                            int B, int H, int N_txt, int N_img, int N_ref, int d, void* cuda_stream);

/*
 * jattn_fp8_repair_apply — correct jattn_fwd_fp8's O and LSE in place for
 * the selected keys.
 *
 * q8, q_scale, k8, v8, k_scale, v_scale : the FP8 attention's inputs.
 * idx, k_sel, v_sel, m : jattn_fp8_repair_select's outputs.
 * o, lse : jattn_fwd_fp8's outputs (lse is required), overwritten with
 *          attention in which the selected keys use their exact rows:
 *          with a = sum over them of exp(s_x - L) v_x - exp(s_q - L) v_q and
 *          z the same sum without v, O' = (O + a) / (1 + z), L' = L + ln(1+z),
 *          s_x = scale qd.k'_t and s_q = scale qd.kd_t (tensor-core products,
 *          fp32 accumulation: s_x from FP16 operands, s_q from the E4M3
 *          codes).  The exact K' and V rows are used as FP16, so they must
 *          lie within the FP16 range.
 * m == 0 leaves o and lse unchanged.  softmax_scale as for jattn_fwd_fp8.
 * Token indices in idx are clamped into [0, N); a list that is not
 * jattn_fp8_repair_select's gives undefined values, never an access
 * outside the tensors.
 */
JATTN_API int jattn_fp8_repair_apply(const void* q8, const float* q_scale, const void* k8, const void* v8,
                           const float* k_scale, const float* v_scale, const int* idx,
                           const void* k_sel, const void* v_sel, int m, void* o, float* lse,
                           int B, int H, int N_txt, int N_img, int N_ref, int d, float softmax_scale,
                           void* cuda_stream);

/* Block-sparse attention: query blocks of 256 tokens, key blocks of 128,
 * counted from token 0 of each (b, h); n_qb = ceil(N / 256),
 * n_kb = ceil(N / 128). */
#define JATTN_SPARSE_QBLOCK 256
#define JATTN_SPARSE_KBLOCK 128

/*
 * jattn_sparse_select — choose the key blocks each query block attends to.
 *
 * Source: Sol-Attention ("Quantized and sparse attention" section of the
 * tutorial), a generic block-sparse attention whose sparsity a parameter
 * tau sets (tau = 1.0 in the tutorial; a higher tau is sparser).  The pages
 * do not define tau; the rule implemented is this reading:
 *   qbar_i = mean of Q' over query block i, kbar_j = mean of K' over key
 *   block j (the last blocks partial); p_ij = softmax_j(scale qbar_i.kbar_j);
 *   key block j is kept for query block i iff p_ij >= tau / n_kb (fp32, the
 *   threshold one correctly rounded division), and the first j with the
 *   largest p_ij is always kept.  tau = 0 keeps every block.
 *
 * q, k    : bf16 Q', K' [B, N, H, d] (after jattn_prologue).
 * qbar    : fp32 [B, H, n_qb, d] output (workspace: the query-block means).
 * kbar    : fp32 [B, H, n_kb, d] output (the key-block means).
 * probs   : optional fp32 [B, H, n_qb, n_kb] output p_ij; NULL skips it.
 * kv_idx  : int32 [B, H, n_qb, n_kb] output; row (b, h, i) starts with the
 *           kept key blocks in increasing order (the rest is not written).
 * kv_cnt  : int32 [B, H, n_qb] output, the number kept (>= 1).
 * d == 128; softmax_scale finite > 0; tau finite >= 0; N <= 2^22.
 * q, k, qbar, kbar 16-byte aligned; probs, kv_idx, kv_cnt 4-byte aligned.
 */
JATTN_API int jattn_sparse_select(const void* q, const void* k, float* qbar, float* kbar, float* probs,
                        int* kv_idx, int* kv_cnt,
                        int B, int H, int N_txt, int N_img, int N_ref, int d,
                        float softmax_scale, float tau, void* cuda_stream);

/*
 * jattn_fwd_bf16_sparse — block-sparse joint attention, BF16 operands.
 *
 * Source: the generic block-sparse attention kernel Sol-Attention runs on
 * ("Quantized and sparse attention" section of the tutorial).
 *
 * As jattn_fwd_bf16, except that every query of query block i of (b, h)
 * attends only to the keys of the key blocks listed in kv_idx[b, h, i, 0 ..
 * kv_cnt[b, h, i] - 1] (jattn_sparse_select's layout): O = softmax over
 * those keys of scale * q.k, times their V rows; lse over the same keys.
 * A query block with count 0 gets O = 0 and lse = -inf.
 * The list must be strictly increasing key-block indices in [0, n_kb);
 * counts are clamped to [0, n_kb] and indices into [0, n_kb) so that any
 * list stays within the tensors, but a list that breaks the rule gives
 * undefined values (a repeated index, for one, counts its keys twice in O
 * and the LSE).  Nothing checks the rule at run time.
 */
JATTN_API int jattn_fwd_bf16_sparse(const void* q, const void* k, const void* v, void* o, float* lse,
                          const int* kv_idx, const int* kv_cnt,
                          int B, int H, int N_txt, int N_img, int N_ref, int d,
                          float softmax_scale, void* cuda_stream);

/*
 * jattn_sparse_select_noalloc — jattn_sparse_select for callers that cannot
 * allocate device memory.  The paper has no counterpart: this is a service
 * of the library, not a step of the method.
 *
 * Some callers cannot call cudaMalloc where they select blocks: a plugin
 * inside an inference engine whose enqueue step may not allocate (the
 * engine owns all device memory and passes in only inputs and outputs),
 * code between the begin and end of a stream capture (cudaMalloc is not a
 * stream operation and may synchronise the device), or a process that has
 * handed all device memory to its own pool allocator.  This call takes the
 * same inputs and outputs as jattn_sparse_select minus the qbar / kbar
 * workspace, which lives instead in a fixed 16 MiB device array inside the
 * library (held by every GPU that loads the library until the process
 * exits).  It allocates and frees nothing.
 *
 * q, k, probs, kv_idx, kv_cnt, sizes, softmax_scale, tau : as for
 * jattn_sparse_select, with the same results.
 * Limit: B * H * (ceil(N / 256) + ceil(N / 128)) * 128 * 4 bytes must not
 * exceed 16 MiB (B = 2, H = 24 up to N = 58112); a larger problem is
 * rejected with JATTN_ERR_UNSUPPORTED before anything is launched.
 * Set-up: the first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  Later calls on the device reuse the address.
 * Sharing: every call uses the same array and leaves its contents behind.
 * Each call overwrites every part of it that it reads, so nothing needs to
 * start at zero, but two calls whose work overlaps on the GPU (on
 * different streams, or from different threads) race on the array and
 * give undefined results: serialise them.
 */
JATTN_API int jattn_sparse_select_noalloc(const void* q, const void* k, float* probs, int* kv_idx, int* kv_cnt,
                                int B, int H, int N_txt, int N_img, int N_ref, int d,
                                float softmax_scale, float tau, void* cuda_stream);

/* Human-readable name of a jattn_status value (static string, never NULL). */
JATTN_API const char* jattn_status_string(int status);

/*
 * jattn_last_cuda_error — name of the CUDA runtime error behind the last
 * JATTN_ERR_CUDA returned on the calling thread ("cudaSuccess" if none).
 * Static string, never NULL.
 */
JATTN_API const char* jattn_last_cuda_error(void);

/*
 * jattn_device_status — synchronise `cuda_stream`, read and clear the device
 * error word the kernels set when a bounded wait runs out.  Returns JATTN_OK,
 * JATTN_ERR_TIMEOUT, or JATTN_ERR_CUDA if the synchronisation itself failed.
 * The error word is one per device and process: it collects timeouts of
 * every launch of the library on the current device since the last call,
 * from any stream or host thread, and this call clears it for all of them.
 * Synchronising `cuda_stream` only waits for that stream's work; a timeout
 * in a launch still running on another stream may be reported by a later
 * call.  A diagnostic call: it blocks the host and must not be
 * stream-captured.
 */
JATTN_API int jattn_device_status(void* cuda_stream);

/*
 * jattn_selftest_wait_timeout — launch one CTA that waits, with the same
 * bounded wait the attention kernels use, on a barrier nothing will ever
 * complete, for at most `timeout_ns` nanoseconds (1 .. 1e9), then returns.
 * Exercises the timeout path without a fault or a hang: afterwards
 * jattn_device_status() must report JATTN_ERR_TIMEOUT.
 */
JATTN_API int jattn_selftest_wait_timeout(long long timeout_ns, void* cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* JATTN_H_ */
