"""GPU parity of jattn_prologue against the float64 oracle.

BF16 mode: the kernel works in fp32, so its value y differs from the exact
(float64) oracle value y* by the fp32 rounding of the norm and rotation,
at most about 2^-20 times the norm of the rotated channel pair.  Every
element must satisfy |y - y*| <= ulp_bf16(y*) + 2^-18 * |pair|; at least
99.99% must be within one bf16 code point of y* rounded to bf16 and at
least 99.9% identical to it.  (Near-zero outputs of a rotation lose their
relative accuracy by cancellation, so a pure ulp bound would not hold.)
FP8 mode: E4M3 codes at least 99.99% identical to the oracle's quantisation
of its own bf16-rounded Q', K' (and of V), every mismatch one code step
apart and at a rounding tie (within the 2^-7 relative rounding of a bf16
input); block scales identical, except where the block maximum itself is
one bf16 step away, which is then what the kernel's scale must show.
"""

import numpy as np
import pytest
import torch

import oracle as O
from diffusion_transformer_joint_dit_b200 import binding as J
from diffusion_transformer_joint_dit_b200 import inputs as I
from tests.gpu_common import (gpu_prologue_bf16, gpu_prologue_fp8, oracle_prologue_bf16, prologue_params,
                              to_np)

pytestmark = pytest.mark.gpu

EDGE = {
    "i2i_small": I.custom("i2i_small", B=2, H=3, n_txt=8, img_h=4, img_w=4, ref_h=4, ref_w=4, ref_row_offset=4),
    "text_only_1": I.custom("text_only_1", B=1, H=1, n_txt=1, img_h=0, img_w=0),
    "rect_grid": I.custom("rect_grid", B=1, H=5, n_txt=3, img_h=7, img_w=13, ref_h=2, ref_w=9, ref_row_offset=7),
    "tail_block": I.custom("tail_block", B=1, H=2, n_txt=70, img_h=0, img_w=0),
    # Three reference images, each with its own grid and (row, col) offsets.
    "multi_ref": I.custom("multi_ref", B=2, H=3, n_txt=9, img_h=6, img_w=10,
                          ref_grids=((4, 10, 6, 0), (3, 7, 10, 2), (2, 5, 0, 12))),
}


def _bf16_close(got, exact):
    g = to_np(got).astype(np.float64)
    ref = O.bf16_round(exact)
    pair = np.sqrt(exact[..., 0::2] ** 2 + exact[..., 1::2] ** 2).repeat(2, axis=-1)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -126))) - 7)
    bound = ulp + 2.0 ** -18 * pair
    worst = np.max(np.abs(g - exact) - bound)
    assert worst <= 0, f"error exceeds bound by {worst:.3e}"
    d = O.bf16_ulp_distance(g, ref)
    assert (d <= 1).mean() >= 0.9999, f"within-1-ulp fraction {(d <= 1).mean():.6f}"
    assert (d == 0).mean() >= 0.999, f"identical fraction {(d == 0).mean():.5f}"


@pytest.mark.parametrize("name", ["tiny", "t2i_1024", "i2i_small", "text_only_1", "rect_grid", "tail_block",
                                  "multi_ref"])
def test_prologue_bf16_matches_oracle(cuda_ok, name):
    w = I.WORKLOADS.get(name) or EDGE[name]
    q, k, _ = I.make_qkv(w, seed=3)
    qo, ko = gpu_prologue_bf16(w, q, k)
    qp, kp, _, _ = oracle_prologue_bf16(w, q, k)
    _bf16_close(qo, qp)
    _bf16_close(ko, kp)


def test_prologue_bf16_in_place_and_weights(cuda_ok):
    w = EDGE["i2i_small"]
    q, k, _ = I.make_qkv(w, seed=4)
    rng = np.random.default_rng(5)
    wq = rng.uniform(0.5, 1.5, 128).astype(np.float32)
    wk = rng.uniform(0.5, 1.5, 128).astype(np.float32)
    qd, kd = q.cuda(), k.cuda()
    wqd, wkd = torch.from_numpy(wq).cuda(), torch.from_numpy(wk).cuda()
    p = J.make_prologue_params(w.img_h, w.img_w, w.ref_h, w.ref_w, w.ref_row_offset, w.theta, w.eps,
                               q_norm_w=wqd, k_norm_w=wkd)
    J.jattn_prologue(qd, kd, None, qd, kd, None, None, None, None, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d,
                     J.JATTN_PROLOGUE_BF16, p)
    torch.cuda.synchronize()
    qp, kp = O.prologue(to_np(q), to_np(k), n_txt=w.n_txt, img_h=w.img_h, img_w=w.img_w, ref_h=w.ref_h,
                        ref_w=w.ref_w, ref_row_offset=w.ref_row_offset, theta=w.theta, eps=w.eps,
                        q_norm_w=wq, k_norm_w=wk)
    _bf16_close(qd, qp)
    _bf16_close(kd, kp)


def _bf16_neighbours(a):
    """The bf16 values one code point below and above each (positive) a."""
    a32 = np.asarray(a, dtype=np.float32)
    bits = a32.view(np.uint32).astype(np.int64)
    step = np.int64(1) << 16
    below = np.maximum(bits - step, 0).astype(np.uint32).view(np.float32)
    above = (bits + step).astype(np.uint32).view(np.float32)
    return below, above


def _check_quantised(got_codes, got_scales, x, block=64):
    """E4M3 codes and block scales of the kernel against the quantisation
    rule applied to the oracle's bf16 values ``x [B, N, H, d]``.

    Scales: identical to fl32(amax / 448) of the oracle's block maximum,
    except where the kernel's block maximum is one bf16 code point away
    (its fp32 norm and rotation rounded that element the other way); such
    a block is then checked with the maximum the kernel's scale implies.
    Codes: at least 99.99% identical to RNE_sat(fl32(x * fl32(448 / amax)))
    and every mismatch an adjacent code whose product lies within one bf16
    rounding of x (2^-7 relative) of the midpoint between the two codes:
    a rounding tie that a 1-ulp difference of the kernel's own bf16 value
    can cross, nothing else.
    """
    codes_k = got_codes.cpu().numpy()
    scales_k = got_scales.cpu().numpy()
    x32 = np.asarray(x, dtype=np.float32)
    B, N, H, d = x32.shape
    nblk = -(-N // block)
    pad = nblk * block - N
    xb = np.pad(x32, ((0, 0), (0, pad), (0, 0), (0, 0))).reshape(B, nblk, block, H, d)
    amax = np.abs(xb).max(axis=(2, 4)).transpose(0, 2, 1).astype(np.float32)     # [B, H, nblk]
    f448 = np.float32(448.0)
    scale_o = np.where(amax > 0, amax / f448, np.float32(1.0)).astype(np.float32)
    differ = scales_k != scale_o
    assert differ.mean() <= 0.01, f"{differ.mean():.4f} of the block scales differ"
    amax_used = amax.copy()
    if differ.any():
        below, above = _bf16_neighbours(amax[differ])
        s_below = (below / f448).astype(np.float32)
        s_above = (above / f448).astype(np.float32)
        sk = scales_k[differ]
        ok = (sk == s_below) | (sk == s_above)
        assert ok.all(), "a block scale differs by more than one bf16 step of its maximum"
        amax_used[differ] = np.where(sk == s_below, below, above)
    inv = np.where(amax_used > 0, f448 / np.maximum(amax_used, np.float32(1e-38)), np.float32(0.0)).astype(np.float32)
    inv_tok = np.repeat(inv.transpose(0, 2, 1), block, axis=1)[:, :N]               # [B, N, H]
    prod = (x32 * inv_tok[..., None]).astype(np.float32)                             # fl32 product
    want = O.e4m3_encode(prod)
    same = codes_k == want
    assert same.mean() >= 0.9999, f"identical code fraction {same.mean():.6f}"
    if not same.all():
        g, r = codes_k[~same].astype(np.int64), want[~same].astype(np.int64)
        assert ((g & 0x80) == (r & 0x80)).all() and (np.abs((g & 0x7F) - (r & 0x7F)) == 1).all(), \
            "a mismatching code is not adjacent"
        mid = 0.5 * (O.e4m3_decode(g) + O.e4m3_decode(r))
        pv = prod[~same].astype(np.float64)
        dist = np.abs(pv - mid)
        assert (dist <= 2.0 ** -7 * np.abs(pv) + 2.0 ** -20).all(), \
            f"a mismatch lies {np.max(dist / np.maximum(np.abs(pv), 1e-30)):.2e} (relative) from its tie"


@pytest.mark.parametrize("name", ["tiny", "i2i_small", "text_only_1", "tail_block", "rect_grid", "multi_ref",
                                  "t2i_2048_fp8"])
def test_prologue_fp8_matches_oracle(cuda_ok, name):
    w = I.WORKLOADS.get(name) or EDGE[name]
    q, k, v = I.make_qkv(w, seed=6)
    (q8, k8, v8), (qs, ks, vs) = gpu_prologue_fp8(w, q, k, v)
    _, _, qb, kb = oracle_prologue_bf16(w, q, k)
    for got_c, got_s, x in ((q8, qs, qb), (k8, ks, kb), (v8, vs, to_np(v))):
        _check_quantised(got_c, got_s, x)


@pytest.mark.parametrize("name", ["t2i_2048", "i2i_2048"])
def test_prologue_bf16_full_size_sampled_tokens(cuda_ok, name):
    """Full size, in the bench's launch configuration, checked on sampled
    tokens (every head): the oracle's RMSNorm and 2-D RoPE applied to those
    tokens at their positions in the whole sequence."""
    w = I.WORKLOADS[name]
    q, k, _ = I.make_qkv(w, seed=11)
    qo, ko = gpu_prologue_bf16(w, q, k)
    idx = I.sampled_rows(w, 256, seed=4)
    rows, cols = O.token_positions(w.n_txt, w.img_h, w.img_w, w.ref_h, w.ref_w, w.ref_row_offset)
    for got, x in ((qo, q), (ko, k)):
        exact = O.rope_2d(O.rmsnorm(to_np(x[:, idx]), eps=w.eps), rows[idx], cols[idx], theta=w.theta)
        _bf16_close(got[:, idx].cpu(), exact)
