"""GPU parity of the FP8 repair budget (jattn_fp8_repair_select / _apply)
against the float64 oracle.

Both sides start from the GPU prologue's E4M3 codes and scales (the prologue
itself is checked in test_gpu_prologue.py).  The per-token errors must match
the oracle's float64 errors to fp32 rounding (up to the prologue's one-step
bf16 tolerance on K'); the selection is an integer
decision taken on the kernel's fp32 errors, so it must equal the oracle's
rule applied to those same values exactly.  The repaired output must match
the oracle's repaired attention within the FP8 tolerance (relative L2 1e-2;
log-sum-exp within 5e-3), and must not move away from exact attention.
"""

import numpy as np
import pytest
import torch

import oracle as O
from diffusion_transformer_joint_dit_b200 import binding as J
from diffusion_transformer_joint_dit_b200 import inputs as I
from tests.gpu_common import FP8_REL_L2, gpu_prologue_fp8, oracle_prologue_bf16, prologue_params, rel_l2, to_np

pytestmark = pytest.mark.gpu


def _run(w, m, seed=0):
    q, k, v = I.make_qkv(w, seed=seed)
    (q8, k8, v8), (qs, ks, vs) = gpu_prologue_fp8(w, q, k, v)
    o = torch.empty((w.B, w.N, w.H, w.d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device="cuda")
    J.jattn_fwd_fp8(q8, k8, v8, qs, ks, vs, o, lse, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d, w.softmax_scale)
    o0, lse0 = o.clone(), lse.clone()
    err = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device="cuda")
    idx = torch.empty((w.B, w.H, max(m, 1)), dtype=torch.int32, device="cuda")
    ksel = torch.empty((w.B, w.H, max(m, 1), w.d), dtype=torch.bfloat16, device="cuda")
    vsel = torch.empty_like(ksel)
    J.jattn_fp8_repair_select(k.cuda(), v.cuda(), k8, v8, ks, vs, prologue_params(w), m, err, idx, ksel, vsel,
                              w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d)
    J.jattn_fp8_repair_apply(q8, qs, k8, v8, ks, vs, idx, ksel, vsel, m, o, lse, w.B, w.H, w.n_txt, w.n_img,
                             w.n_ref, w.d, w.softmax_scale)
    torch.cuda.synchronize()
    assert J.jattn_device_status() == J.JATTN_OK
    codes = [to_np(t) for t in (q8, k8, v8)]
    scales = [to_np(t) for t in (qs, ks, vs)]
    return (q, k, v), codes, scales, (o0, lse0), (o, lse), err, idx[..., :m], ksel[:, :, :m], vsel[:, :, :m]


CASES = {
    # N = 196: a partial 64-token block, selections crossing 32-key chunks.
    "ragged": I.custom("ragged", B=1, H=2, n_txt=7, img_h=9, img_w=21, gain_sigma=0.5),
    "two_batch": I.custom("two_batch", B=2, H=3, n_txt=5, img_h=8, img_w=8, ref_h=2, ref_w=8, ref_row_offset=8,
                          gain_sigma=0.5),
    # Two reference grids: the exact K' rows are recomputed at their positions.
    "multi_ref": I.custom("multi_ref", B=1, H=2, n_txt=6, img_h=8, img_w=9,
                          ref_grids=((3, 9, 8, 0), (4, 5, 11, 9)), gain_sigma=0.5),
}


@pytest.mark.parametrize("name,m", [("ragged", 0), ("ragged", 1), ("ragged", 37), ("ragged", 196),
                                    ("two_batch", 9), ("multi_ref", 11)])
def test_repair_matches_oracle(cuda_ok, name, m):
    w = CASES[name]
    (q, k, v), codes, scales, (o0, lse0), (o, lse), err, idx, ksel, vsel = _run(w, m)
    deq = [O.dequantize_e4m3(c, s) for c, s in zip(codes, scales)]
    _, _, _, kb = oracle_prologue_bf16(w, q, k)          # exact K' (bf16 rounding, as quantised)
    vb = to_np(v)
    # Errors: float64 oracle against the kernel's fp32 sums.
    _, err_ref = O.repair_select(kb, vb, deq[1], deq[2], rho=0.0)
    # The kernel's K' may sit one bf16 step from the oracle's rounding in a
    # channel (the prologue's own tolerance), which moves e_t by about
    # 2^-7 |K'| |K' - Kd| there: all errors within 1e-3 relative, nearly all
    # within fp32 summation rounding.
    ge = to_np(err)
    rel = np.abs(ge - err_ref) / np.maximum(err_ref, 1e-30)
    assert rel.max() <= 1e-3, f"max relative error {rel.max():.3e}"
    assert (rel <= 2e-5).mean() >= 0.99
    if m == 0:
        assert torch.equal(o, o0) and torch.equal(lse, lse0)
        return
    # Selection: the oracle's rule on the kernel's own fp32 errors.
    e32 = to_np(err)
    got_idx = to_np(idx).astype(np.int64)
    for b in range(w.B):
        for h in range(w.H):
            want = np.sort(np.argsort(-e32[b, h], kind="stable")[:m])
            assert got_idx[b, h].tolist() == want.tolist()
    # Gathered exact rows.
    kbt = np.transpose(kb, (0, 2, 1, 3))
    vbt = np.transpose(vb, (0, 2, 1, 3))
    sel = lambda a: np.take_along_axis(a, got_idx[..., None], axis=2)
    d = O.bf16_ulp_distance(to_np(ksel), sel(kbt))
    assert (d <= 1).all() and (d == 0).mean() >= 0.999
    np.testing.assert_array_equal(to_np(vsel), sel(vbt))
    # Repaired attention.
    ref, ref_lse = O.repaired_attention(deq[0], deq[1], deq[2], kb, vb, got_idx, w.softmax_scale)
    got = to_np(o)
    assert rel_l2(got, ref) <= FP8_REL_L2, f"rel-L2 {rel_l2(got, ref):.3e}"
    assert np.max(np.abs(to_np(lse) - ref_lse)) <= 5e-3
    exact, _ = O.joint_attention(deq[0], kb, vb, w.softmax_scale)
    assert rel_l2(got, exact) <= rel_l2(to_np(o0), exact) + 1e-4


def test_repair_t2i_2048_fp8_budget(cuda_ok):
    """Full size, the tutorial's budget rho = 0.005 (85 tokens per head),
    checked on sampled query rows."""
    w = I.WORKLOADS["t2i_2048_fp8"]
    m = J.repair_count(w.N, 0.005)
    assert m == 85
    (q, k, v), codes, scales, (o0, _), (o, lse), err, idx, ksel, vsel = _run(w, m)
    rows = I.sampled_rows(w, 128, seed=5)
    deq = [O.dequantize_e4m3(c, s) for c, s in zip(codes, scales)]
    _, _, _, kb = oracle_prologue_bf16(w, q, k)
    vb = to_np(v)
    got_idx = to_np(idx).astype(np.int64)
    e32 = to_np(err)
    for h in range(w.H):
        want = np.sort(np.argsort(-e32[0, h], kind="stable")[:m])
        assert got_idx[0, h].tolist() == want.tolist()
    kr = np.array(deq[1])
    vr = np.array(deq[2])
    for h in range(w.H):
        t = got_idx[0, h]
        kr[0, t, h] = kb[0, t, h]
        vr[0, t, h] = vb[0, t, h]
    ref, ref_lse = O.joint_attention(deq[0], kr, vr, w.softmax_scale, rows=rows)
    got = to_np(o)[:, rows]
    assert rel_l2(got, ref) <= FP8_REL_L2
    assert np.max(np.abs(to_np(lse)[:, :, rows] - ref_lse)) <= 5e-3
    base, _ = O.joint_attention(deq[0], deq[1], deq[2], w.softmax_scale, rows=rows)
    exact, _ = O.joint_attention(deq[0], kb, vb, w.softmax_scale, rows=rows)
    print(f"rel-L2 vs exact-K/V attention: FP8 {rel_l2(to_np(o0)[:, rows], exact):.4e}, "
          f"repaired {rel_l2(got, exact):.4e} (oracle FP8 {rel_l2(base, exact):.4e})")
