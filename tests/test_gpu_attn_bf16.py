"""GPU parity of jattn_fwd_bf16 against the float64 oracle.

Inputs are the same bf16 tensors on both sides.  Small problems and the
1024^2 workload are checked on every query row; the 2048^2 workloads run
the kernel at full size in the benchmark's launch configuration and compare
256 sampled query rows per (b, h) against all keys.  Tolerances: relative L2 <= 5e-3 and
max-abs <= 2e-2 on the output; 2^-8 absolute on the log-sum-exp (l counts
each tile's largest P at its bf16 value, so ln l can carry up to 2^-9 of
that term's rounding).
"""

import numpy as np
import pytest
import torch

from diffusion_transformer_joint_dit_b200 import binding as J
from diffusion_transformer_joint_dit_b200 import inputs as I
from tests.gpu_common import (check_attention, gpu_attn_bf16, gpu_prologue_bf16, oracle_prologue_bf16,
                              to_np)

pytestmark = pytest.mark.gpu


def _run(w, seed=0, q_gain=1.0, rows=None):
    q, k, v = I.make_qkv(w, seed=seed)
    if q_gain != 1.0:
        q = (q.float() * q_gain).to(torch.bfloat16)
    if w.k_outlier_frac > 0:
        k = I.apply_outliers(k, I.outlier_rows(w, seed), w.k_outlier_gain)
    o, lse = gpu_attn_bf16(w, q, k, v)
    return check_attention(w, o, lse, to_np(q), to_np(k), to_np(v), rows=rows)


def test_tiny_full(cuda_ok):
    _run(I.WORKLOADS["tiny"])


@pytest.mark.parametrize("N", [1, 2, 63, 64, 65, 127, 128, 129, 255, 256, 257, 383, 384, 385, 511, 513])
def test_ragged_lengths(cuda_ok, N):
    _run(I.custom(f"n{N}", B=1, H=1, n_txt=N, img_h=0, img_w=0), seed=N)


def test_batch_heads_ref_stream(cuda_ok):
    _run(I.custom("bh", B=2, H=3, n_txt=40, img_h=8, img_w=16, ref_h=4, ref_w=8, ref_row_offset=8), seed=9)


@pytest.mark.parametrize("gain", [4.0, 12.0])
def test_peaked_softmax_exercises_rescale(cuda_ok, gain):
    # Larger logits move the running max often (and by more than the lazy
    # rescale threshold), exercising the O correction path.
    _run(I.custom("peaked", B=1, H=2, n_txt=16, img_h=24, img_w=24), seed=11, q_gain=gain)


@pytest.mark.parametrize("gain", [1.0, 12.0])
def test_main_launch_and_split_tail_all_rows(cuda_ok, gain):
    """162 work items on 148 SMs: a whole wave in the main launch and 14
    items run split over KV halves (merged across a CTA pair), every row
    checked; with gain 12 the two halves of a row keep different reference
    maxima, which the merge has to reconcile."""
    _run(I.custom("tail", B=1, H=9, n_txt=512, img_h=64, img_w=64), seed=31, q_gain=gain)


def test_t2i_1024_all_rows(cuda_ok):
    """The 1024^2 workload checked on every query row of every (b, h)."""
    _run(I.WORKLOADS["t2i_1024"])


def test_t2i_2048_outliers_sampled(cuda_ok):
    w = I.WORKLOADS["t2i_2048"]
    _run(w, rows=I.sampled_rows(w, 256))


def test_i2i_2048_sampled(cuda_ok):
    w = I.WORKLOADS["i2i_2048"]
    _run(w, rows=I.sampled_rows(w, 256))


def test_pipeline_prologue_then_attention(cuda_ok):
    """Raw Q, K, V -> GPU prologue -> GPU attention, against the oracle chain."""
    w = I.WORKLOADS["tiny"]
    q, k, v = I.make_qkv(w, seed=12)
    qo, ko = gpu_prologue_bf16(w, q, k)
    o, lse = gpu_attn_bf16(w, qo, ko, v)
    _, _, qb, kb = oracle_prologue_bf16(w, q, k)
    check_attention(w, o, lse, qb, kb, to_np(v))


def test_output_canaries_and_no_unwritten_rows(cuda_ok):
    """Guard regions around O stay untouched; every element of O is written."""
    w = I.custom("canary", B=2, H=3, n_txt=5, img_h=10, img_w=30)
    q, k, v = (t.cuda() for t in I.make_qkv(w, seed=13))
    n = w.B * w.N * w.H * w.d
    guard = 4096
    buf = torch.full((n + 2 * guard,), float("nan"), dtype=torch.bfloat16, device="cuda")
    buf[:guard] = 7.0
    buf[-guard:] = -7.0
    o = buf[guard:guard + n].view(w.B, w.N, w.H, w.d)
    J.jattn_fwd_bf16(q, k, v, o, None, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d, w.softmax_scale)
    torch.cuda.synchronize()
    assert (buf[:guard] == 7.0).all() and (buf[-guard:] == -7.0).all()
    assert torch.isfinite(o.float()).all()
    check_attention(w, o, None, to_np(q), to_np(k), to_np(v))


def test_repeatable(cuda_ok):
    w = I.custom("rep", B=1, H=2, n_txt=100, img_h=10, img_w=10)
    q, k, v = I.make_qkv(w, seed=14)
    o1, l1 = gpu_attn_bf16(w, q, k, v)
    o2, l2 = gpu_attn_bf16(w, q, k, v)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
