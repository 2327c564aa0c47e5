"""GPU parity of the fused QKV projection (jattn_rope_table + jattn_qkv_fused)
against the float64 oracle.

The kernel accumulates the C-long dot products in fp32 and rounds each output
to bf16 once.  The fp32 accumulation of C products of unit-size factors is
off the exact sum by about sqrt(C) * 2^-24 of the row's size (below 2^-16 for
C <= 65536), far below a bf16 step, and the fp32 norm and rotation add about
2^-20 of the channel pair's size.  So every element must lie within one bf16
step of the exact value plus 2^-16 times the row's rms plus (Q, K) 2^-12
times the size of its rotated channel pair; at least 99.9% within one code
point of the exact value rounded to bf16 and 99% identical to it.
"""

import numpy as np
import pytest
import torch

import oracle as O
from diffusion_transformer_joint_dit_b200 import binding as J
from diffusion_transformer_joint_dit_b200 import inputs as I

pytestmark = pytest.mark.gpu

CASES = {
    # One text tile with 3 valid rows, one image tile; 3 output tiles.
    "small": (I.custom("small", B=1, H=2, n_txt=3, img_h=4, img_w=5), 128),
    # Text straddles a 128-row tile, reference grid, two batch elements.
    "ragged": (I.custom("ragged", B=2, H=4, n_txt=130, img_h=10, img_w=20, ref_h=3, ref_w=5,
                        ref_row_offset=10), 256),
    # No text tokens (text weights unused), K loop of 12 steps.
    "image_only": (I.custom("image_only", B=1, H=2, n_txt=0, img_h=9, img_w=15), 768),
    "text_only": (I.custom("text_only", B=1, H=2, n_txt=77, img_h=0, img_w=0), 192),
    # Three reference grids with their own row and column offsets.
    "multi_ref": (I.custom("multi_ref", B=1, H=2, n_txt=9, img_h=6, img_w=10,
                           ref_grids=((4, 10, 6, 0), (3, 7, 10, 2), (2, 5, 0, 12))), 128),
}


def _run(w, C, seed=0):
    x, (wt, wi), qn, kn = I.make_qkv_projection_inputs(w, C, seed)
    dev = torch.device("cuda")
    xd, wtd, wid = x.to(dev), wt.to(dev), wi.to(dev)
    qnd = [t.to(dev) for t in qn]
    knd = [t.to(dev) for t in kn]
    rope = torch.empty((w.N, 64, 2), dtype=torch.float32, device=dev)
    params = J.make_prologue_params(w.img_h, w.img_w, w.ref_h, w.ref_w, w.ref_row_offset, w.theta, w.eps,
                                    ref_grids=w.ref_grids or None)
    J.jattn_rope_table(rope, w.n_txt, w.n_img, w.n_ref, params)
    shape = (w.B, w.N, w.H, w.d)
    q, k, v = (torch.empty(shape, dtype=torch.bfloat16, device=dev) for _ in range(3))
    wts = J.make_qkv_weights(wtd if w.n_txt > 0 else None, wid if w.n_img + w.n_ref > 0 else None,
                             tuple(qnd), tuple(knd), w.eps)
    J.jattn_qkv_fused(xd, wts, rope, q, k, v, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d, C)
    torch.cuda.synchronize()
    assert J.jattn_device_status() == J.JATTN_OK
    return (x, wt, wi, qn, kn), rope.cpu().numpy(), (q.cpu(), k.cpu(), v.cpu())


def _check(got, exact, rotated):
    g = got.to(torch.float64).numpy()
    ref = O.bf16_round(exact)
    row = np.sqrt(np.mean(exact ** 2, axis=-1, keepdims=True))
    extra = 2.0 ** -16 * row
    if rotated:
        extra = extra + 2.0 ** -12 * np.sqrt(exact[..., 0::2] ** 2 + exact[..., 1::2] ** 2).repeat(2, axis=-1)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -126))) - 7)
    worst = np.max(np.abs(g - exact) - (ulp + extra))
    assert worst <= 0, f"error exceeds bound by {worst:.3e}"
    d = O.bf16_ulp_distance(g, ref)
    assert (d <= 1).mean() >= 0.999, f"within-1-ulp fraction {(d <= 1).mean():.6f}"
    assert (d == 0).mean() >= 0.99, f"identical fraction {(d == 0).mean():.5f}"


@pytest.mark.parametrize("name", sorted(CASES))
def test_qkv_fused_matches_oracle(cuda_ok, name):
    w, C = CASES[name]
    (x, wt, wi, qn, kn), rope, (q, k, v) = _run(w, C)
    grids = list(w.ref_grids) or None
    np.testing.assert_allclose(rope, O.rope_table(w.n_txt, w.img_h, w.img_w, w.ref_h, w.ref_w, w.ref_row_offset,
                                                  grids, w.theta), rtol=0, atol=2e-7)
    f = lambda t: t.to(torch.float64).numpy()
    qe, ke, ve = O.qkv_fused(f(x), f(wt), f(wi), n_txt=w.n_txt, img_h=w.img_h, img_w=w.img_w, H=w.H,
                             ref_h=w.ref_h, ref_w=w.ref_w, ref_row_offset=w.ref_row_offset, ref_grids=grids,
                             theta=w.theta,
                             eps=w.eps, q_norm_w=tuple(t.numpy() for t in qn),
                             k_norm_w=tuple(t.numpy() for t in kn))
    _check(q, qe, True)
    _check(k, ke, True)
    _check(v, ve, False)


def test_qkv_fused_t2i_2048_sampled_rows(cuda_ok):
    """Full-size projection (C = 3072 = H d, t2i_2048 shapes) checked on
    sampled tokens, the oracle steps applied to those rows only."""
    w = I.WORKLOADS["t2i_2048"]
    C = w.H * w.d
    (x, wt, wi, qn, kn), _, (q, k, v) = _run(w, C, seed=1)
    idx = I.sampled_rows(w, 64, seed=2)
    rows, cols = O.token_positions(w.n_txt, w.img_h, w.img_w)
    f = lambda t: t.to(torch.float64).numpy()
    for b in range(w.B):
        xs = f(x[b, idx])
        for s, sel in ((0, idx < w.n_txt), (1, idx >= w.n_txt)):
            if not sel.any():
                continue
            y = xs[sel] @ f(wt if s == 0 else wi).T                       # [R, 3 H d]
            hd = w.H * w.d
            qe = O.rmsnorm(y[:, :hd].reshape(-1, w.H, w.d), qn[s].numpy(), w.eps)[None]
            ke = O.rmsnorm(y[:, hd:2 * hd].reshape(-1, w.H, w.d), kn[s].numpy(), w.eps)[None]
            ve = y[:, 2 * hd:].reshape(1, -1, w.H, w.d)
            t = idx[sel]
            qe = O.rope_2d(qe, rows[t], cols[t], w.theta)
            ke = O.rope_2d(ke, rows[t], cols[t], w.theta)
            _check(q[b, t][None], qe, True)
            _check(k[b, t][None], ke, True)
            _check(v[b, t][None], ve, False)
