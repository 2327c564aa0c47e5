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


def _prologue_like_codes(w, seed, v_scale_fn):
    """Q, K, V codes as the prologue would write them for N(0,1) rows (random
    finite E4M3 codes would do too) with V block scales chosen by
    ``v_scale_fn(nblk, rng)``; Q and K keep ordinary scales."""
    rng = np.random.default_rng(seed)
    nblk = -(-w.N // 64)
    codes = [I.random_e4m3_codes((w.B, w.N, w.H, w.d), seed=seed + i) for i in range(3)]
    scales = [np.exp(rng.uniform(-5.5, -4.5, (w.B, w.H, nblk))).astype(np.float32) for _ in range(2)]
    scales.append(v_scale_fn(nblk, rng).astype(np.float32))
    return codes, scales


def test_fp8_all_zero_v_block(cuda_ok):
    """One 64-token V block is all zero (the prologue then stores scale 1
    and zero codes) while every other V block has a scale near 1e-2: the
    zero block must not cost the other blocks precision."""
    w = I.custom("zero_v", B=1, H=2, n_txt=64, img_h=16, img_w=20)

    def v_scales(nblk, rng):
        s = np.full((w.B, w.H, nblk), 0.01, dtype=np.float64) * np.exp(rng.uniform(-0.3, 0.3, (w.B, w.H, nblk)))
        s[:, :, 2] = 1.0
        return s

    codes, scales = _prologue_like_codes(w, 41, v_scales)
    codes[2][:, 128:192] = 0  # block 2 of every (b, h): zero codes, scale 1
    o, lse = _gpu_fwd_fp8(w, codes, scales)
    _check(w, o, lse, codes, scales)


def test_fp8_v_scales_spanning_three_decades(cuda_ok):
    """V block scales from 1e-4 to 1e-1 within each (b, h)."""
    w = I.custom("spread_v", B=2, H=2, n_txt=30, img_h=10, img_w=30)

    def v_scales(nblk, rng):
        return 10.0 ** rng.uniform(-4.0, -1.0, (w.B, w.H, nblk))

    codes, scales = _prologue_like_codes(w, 43, v_scales)
    o, lse = _gpu_fwd_fp8(w, codes, scales)
    _check(w, o, lse, codes, scales)
