"""GPU parity of jattn_fwd_fp8 against the float64 oracle.

The oracle quantises with the same E4M3 block rule and runs exact softmax
attention on the dequantised values; the kernel must match it within
relative L2 1e-2.  The error of the FP8 path against the unquantised
oracle is reported (printed), not gated: it is dominated by the E4M3
quantisation of Q, K, V itself.
"""

import numpy as np
import pytest
import torch

import oracle as O
from diffusion_transformer_joint_dit_b200 import binding as J
from diffusion_transformer_joint_dit_b200 import inputs as I
from tests.gpu_common import FP8_REL_L2, gpu_prologue_fp8, oracle_prologue_bf16, rel_l2, to_np

pytestmark = pytest.mark.gpu


def _oracle_quant(w, q, k, v):
    _, _, qb, kb = oracle_prologue_bf16(w, q, k)
    out = []
    for x in (qb, kb, to_np(v)):
        out.append(O.block_quantize_e4m3(x.astype(np.float32)))
    return out, (qb, kb, to_np(v))


def _gpu_fwd_fp8(w, codes, scales):
    o = torch.full((w.B, w.N, w.H, w.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((w.B, w.H, w.N), float("nan"), dtype=torch.float32, device="cuda")
    c = [torch.as_tensor(x).cuda() if isinstance(x, np.ndarray) else x for x in codes]
    s = [torch.as_tensor(x).cuda() if isinstance(x, np.ndarray) else x for x in scales]
    J.jattn_fwd_fp8(c[0], c[1], c[2], s[0], s[1], s[2], o, lse, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d,
                    w.softmax_scale)
    torch.cuda.synchronize()
    assert J.jattn_device_status() == J.JATTN_OK
    return o, lse


def _check(w, o, lse, codes, scales, rows=None, unquant=None):
    deq = [O.dequantize_e4m3(c, s) for c, s in zip(codes, scales)]
    ref, ref_lse = O.joint_attention(deq[0], deq[1], deq[2], w.softmax_scale, rows=rows)
    got = to_np(o)
    gl = to_np(lse)
    if rows is not None:
        got, gl = got[:, rows], gl[:, :, rows]
    assert np.isfinite(got).all()
    err = rel_l2(got, ref)
    assert err <= FP8_REL_L2, f"rel-L2 vs quantised oracle {err:.3e}"
    assert np.max(np.abs(gl - ref_lse)) <= 5e-3
    if unquant is not None:
        ref_u, _ = O.joint_attention(*unquant, w.softmax_scale, rows=rows)
        print(f"{w.name}: rel-L2 vs quantised oracle {err:.3e}, vs unquantised oracle {rel_l2(got, ref_u):.3e}")
    return err


@pytest.mark.parametrize("name", ["tiny", "ragged"])
def test_fp8_attention_small(cuda_ok, name):
    w = I.WORKLOADS["tiny"] if name == "tiny" else I.custom("ragged", B=2, H=3, n_txt=7, img_h=9, img_w=21,
                                                             gain_sigma=0.5)
    q, k, v = I.make_qkv(w, seed=31)
    qkv8, unq = _oracle_quant(w, q, k, v)
    codes, scales = zip(*qkv8)
    o, lse = _gpu_fwd_fp8(w, codes, scales)
    _check(w, o, lse, codes, scales, unquant=unq)


@pytest.mark.parametrize("N", [1, 63, 64, 65, 129, 200, 257, 300])
def test_fp8_ragged_lengths(cuda_ok, N):
    w = I.custom(f"n{N}", B=1, H=1, n_txt=N, img_h=0, img_w=0)
    q, k, v = I.make_qkv(w, seed=N + 100)
    qkv8, _ = _oracle_quant(w, q, k, v)
    codes, scales = zip(*qkv8)
    o, lse = _gpu_fwd_fp8(w, codes, scales)
    _check(w, o, lse, codes, scales)


def test_fp8_random_codes_and_scales(cuda_ok):
    """Arbitrary finite codes and scales spanning decades (not prologue output)."""
    w = I.custom("rand", B=1, H=2, n_txt=40, img_h=12, img_w=20)
    nblk = -(-w.N // 64)
    rng = np.random.default_rng(33)
    codes = [I.random_e4m3_codes((w.B, w.N, w.H, w.d), seed=34 + i) for i in range(3)]
    scales = [np.exp(rng.uniform(-6, -2, (w.B, w.H, nblk))).astype(np.float32) for _ in range(3)]
    o, lse = _gpu_fwd_fp8(w, codes, scales)
    _check(w, o, lse, codes, scales)


def test_fp8_pipeline_t2i_2048_sampled(cuda_ok):
    """Raw Q, K, V -> GPU FP8 prologue -> GPU FP8 attention, full 2048^2 size."""
    w = I.WORKLOADS["t2i_2048_fp8"]
    q, k, v = I.make_qkv(w, seed=0)
    codes_g, scales_g = gpu_prologue_fp8(w, q, k, v)
    o, lse = _gpu_fwd_fp8(w, codes_g, scales_g)
    qkv8, unq = _oracle_quant(w, q, k, v)
    codes, scales = zip(*qkv8)
    _check(w, o, lse, codes, scales, rows=I.sampled_rows(w, 256), unquant=unq)
