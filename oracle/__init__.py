"""Float64 CPU oracle for the joint text+image DiT attention forward.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
its Python binding) may import, call or link anything in this package.  Only
``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference
arm of ``bench.py`` use it.  It shares no code with the CUDA path: the two
meet only through the seeded input generators, which hold none of the
method's arithmetic.

Every function is a plain, slow, obviously correct restatement of what the
method computes, in float64 unless the quantisation rule fixes float32
arithmetic.  Sources (titles of the web pages the method is described on):

* "FLUX 3 inference with TensorRT LLM VisualGen" section of the NVIDIA
  tutorial on accelerating FLUX 3 Image Klein (everytik.com translation):
  the text, noisy-target and optional reference streams are processed
  separately and meet only in joint attention.
* "GEMM kernel optimization" section of the same tutorial: the QKV
  projection epilogue applies query/key normalisation and rotary position
  embedding (in that order).
* "Quantized and sparse attention" section of the same tutorial: FP8 Q/K
  and FP8 V attention (``qk_dtype: fp8``, ``v_dtype: fp8``), the
  VC-Attention FP8 repair budget and Sol-Attention block sparsity.

The pages fix no constants (head size, eps, RoPE base and axis split, block
size, quantisation format); those come from the workload definitions and
from readings of the pages, each stated in the docstring of the function
that applies it.

Pins: every function here is checked by ``tests/test_oracle_pins.py``
against closed forms, hand-derived worked values (``tests/golden/``),
library routines (torch float64 SDPA, ``torch.float8_e4m3fn``) and
invariants.  One reading is parity unpinned against the pages: the meaning
of Sol-Attention's tau (``sparse_probs`` / ``sparse_keep``), which the pages
name but do not define; the rule implemented is pinned as stated.
"""

from .jattn_oracle import (  # noqa: F401
    E4M3_MAX,
    SPARSE_KBLOCK,
    SPARSE_QBLOCK,
    bf16_round,
    bf16_ulp_distance,
    block_sparse_attention,
    block_quantize_e4m3,
    dequantize_e4m3,
    e4m3_decode,
    e4m3_encode,
    joint_attention,
    prologue,
    qkv_fused,
    repair_count,
    repair_select,
    repaired_attention,
    rmsnorm,
    rope_2d,
    rope_table,
    sparse_keep,
    sparse_pool,
    sparse_probs,
    token_positions,
)
