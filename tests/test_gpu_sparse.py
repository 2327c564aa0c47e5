"""GPU parity of the block-sparse attention (jattn_sparse_select and
jattn_fwd_bf16_sparse) against the float64 oracle.

Selection: the pooled block means match the oracle's float64 means to fp32
summation rounding, the pooled probabilities likewise; the kept blocks are
an integer decision taken on the kernel's fp32 probabilities, so they must
equal the oracle's rule applied to those same values exactly.  Attention:
the output over the kept blocks matches the oracle's block-sparse attention
within the BF16 tolerances (relative L2 5e-3, max-abs 2e-2, LSE 2^-8).
"""

import numpy as np
import pytest
import torch

import oracle as O
from diffusion_transformer_joint_dit_b200 import binding as J
from diffusion_transformer_joint_dit_b200 import inputs as I
from tests.gpu_common import (BF16_LSE_ABS, BF16_MAX_ABS, BF16_REL_L2, assert_equal_but_split_tail, gpu_attn_bf16,
                              gpu_prologue_bf16, rel_l2, to_np)

pytestmark = pytest.mark.gpu


def _blocky_qk(w, seed, gain=1.5):
    """Q', K' stand-ins with a mean vector per 128-token block, so that the
    pooled block scores differ (and blocks are really dropped)."""
    g = torch.Generator().manual_seed(seed)
    shape = (w.B, w.N, w.H, w.d)
    nkb = -(-w.N // 128)
    out = []
    for _ in range(2):
        base = torch.randn(shape, generator=g)
        means = torch.randn((w.B, nkb, w.H, w.d), generator=g) * gain
        out.append((base + means.repeat_interleave(128, dim=1)[:, :w.N]).to(torch.bfloat16))
    v = torch.randn(shape, generator=g).to(torch.bfloat16)
    return out[0], out[1], v


def _select(w, q, k, tau):
    nqb, nkb = J.sparse_blocks(w.N)
    qbar = torch.empty((w.B, w.H, nqb, w.d), dtype=torch.float32, device="cuda")
    kbar = torch.empty((w.B, w.H, nkb, w.d), dtype=torch.float32, device="cuda")
    probs = torch.full((w.B, w.H, nqb, nkb), float("nan"), dtype=torch.float32, device="cuda")
    idx = torch.full((w.B, w.H, nqb, nkb), -1, dtype=torch.int32, device="cuda")
    cnt = torch.full((w.B, w.H, nqb), -1, dtype=torch.int32, device="cuda")
    J.jattn_sparse_select(q, k, qbar, kbar, probs, idx, cnt, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d,
                          w.softmax_scale, tau)
    torch.cuda.synchronize()
    return qbar, kbar, probs, idx, cnt


def _sparse_attn(w, q, k, v, idx, cnt):
    o = torch.full_like(q, float("nan"))
    lse = torch.full((w.B, w.H, w.N), float("nan"), dtype=torch.float32, device="cuda")
    J.jattn_fwd_bf16_sparse(q, k, v, o, lse, idx, cnt, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d, w.softmax_scale)
    torch.cuda.synchronize()
    assert J.jattn_device_status() == J.JATTN_OK
    return o, lse


def _keep_from_lists(idx, cnt, nkb):
    idx, cnt = to_np(idx).astype(np.int64), to_np(cnt).astype(np.int64)
    keep = np.zeros(idx.shape[:-1] + (nkb,), dtype=bool)
    for pos in np.ndindex(*cnt.shape):
        row = idx[pos][:cnt[pos]]
        assert np.all(np.diff(row) > 0), "list not strictly increasing"
        keep[pos][row] = True
    return keep


def _check_selection(w, q, k, tau, qbar, kbar, probs, idx, cnt, heads=None):
    qn, kn = to_np(q), to_np(k)
    if heads is not None:
        qn, kn = qn[:, :, heads], kn[:, :, heads]
        sl = lambda t: to_np(t)[:, heads]
    else:
        sl = to_np
    # Pooled means: fp32 sums of at most 256 bf16 values.
    for got, x, blk in ((sl(qbar), qn, 256), (sl(kbar), kn, 128)):
        ref = O.sparse_pool(x, blk)
        scale = np.max(np.abs(x)) + 1e-30
        assert np.max(np.abs(got - ref)) <= 2e-6 * scale
    ref_p = O.sparse_probs(qn, kn, w.softmax_scale)
    p = sl(probs)
    assert np.max(np.abs(p - ref_p) / np.maximum(ref_p, 1e-30)) <= 1e-4
    # The decision on the kernel's own probabilities.
    nkb = p.shape[-1]
    want = O.sparse_keep(p, tau)
    got = _keep_from_lists(idx, cnt, nkb)
    if heads is not None:
        got = got[:, heads]
    assert np.array_equal(got, want)
    assert np.array_equal(sl(cnt), want.sum(-1))
    return want


CASES = {
    # N = 700: 3 query blocks (the last partial), 6 key blocks (last 60 keys).
    "ragged": I.custom("ragged", B=1, H=2, n_txt=12, img_h=16, img_w=43),
    "two_batch": I.custom("two_batch", B=2, H=3, n_txt=40, img_h=16, img_w=24, ref_h=4, ref_w=24,
                          ref_row_offset=16),
}


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("tau", [0.0, 0.5, 1.0, 3.0])
def test_sparse_matches_oracle(cuda_ok, name, tau):
    w = CASES[name]
    q, k, v = _blocky_qk(w, seed=7)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    sel = _select(w, qd, kd, tau)
    keep = _check_selection(w, qd, kd, tau, *sel)
    if tau == 0.0:
        assert keep.all()
    o, lse = _sparse_attn(w, qd, kd, vd, sel[3], sel[4])
    ref, ref_lse = O.block_sparse_attention(to_np(q), to_np(k), to_np(v), keep, w.softmax_scale)
    got = to_np(o)
    assert np.isfinite(got).all()
    assert rel_l2(got, ref) <= BF16_REL_L2
    assert np.max(np.abs(got - ref)) <= BF16_MAX_ABS
    assert np.max(np.abs(to_np(lse) - ref_lse)) <= BF16_LSE_ABS


def test_all_blocks_kept_is_the_dense_kernel(cuda_ok):
    w = CASES["two_batch"]
    q, k, v = _blocky_qk(w, seed=8)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    sel = _select(w, qd, kd, 0.0)
    o, lse = _sparse_attn(w, qd, kd, vd, sel[3], sel[4])
    od, lsed = gpu_attn_bf16(w, q, k, v)
    assert_equal_but_split_tail(w, o, lse, od, lsed)


def test_hand_written_lists(cuda_ok):
    """Empty lists (O = 0, LSE = -inf), the partial last key block alone,
    non-contiguous lists."""
    w = CASES["ragged"]
    q, k, v = _blocky_qk(w, seed=9)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    nqb, nkb = J.sparse_blocks(w.N)
    lists = {(0, 0): [], (0, 1): [5], (0, 2): [0, 2, 5], (1, 0): [1, 3], (1, 1): list(range(nkb)), (1, 2): []}
    idx = torch.zeros((1, w.H, nqb, nkb), dtype=torch.int32)
    cnt = torch.zeros((1, w.H, nqb), dtype=torch.int32)
    keep = np.zeros((1, w.H, nqb, nkb), dtype=bool)
    for (h, i), row in lists.items():
        cnt[0, h, i] = len(row)
        idx[0, h, i, :len(row)] = torch.tensor(row, dtype=torch.int32)
        keep[0, h, i, row] = True
    o, lse = _sparse_attn(w, qd, kd, vd, idx.cuda(), cnt.cuda())
    ref, ref_lse = O.block_sparse_attention(to_np(q), to_np(k), to_np(v), keep, w.softmax_scale)
    got, gl = to_np(o), to_np(lse)
    for (h, i), row in lists.items():
        rows = slice(i * 256, min(w.N, (i + 1) * 256))
        if not row:
            assert np.all(got[0, rows, h] == 0.0)
            assert np.all(np.isneginf(gl[0, h, rows]))
    fin = np.isfinite(ref_lse)
    assert rel_l2(got, ref) <= BF16_REL_L2
    assert np.max(np.abs(got - ref)) <= BF16_MAX_ABS
    assert np.max(np.abs(gl[fin] - ref_lse[fin])) <= BF16_LSE_ABS


def test_t2i_2048_tau_1_sampled(cuda_ok):
    """Full size after the prologue, the tutorial's tau = 1.0; selection
    checked on four heads, attention on sampled query rows."""
    w = I.WORKLOADS["t2i_2048"]
    q, k, v = I.make_qkv(w, seed=0)
    qp, kp = gpu_prologue_bf16(w, q, k)
    sel = _select(w, qp, kp, 1.0)
    heads = [0, 7, 13, 23]
    _check_selection(w, qp, kp, 1.0, *sel, heads=heads)
    nkb = sel[2].shape[-1]
    keep = _keep_from_lists(sel[3], sel[4], nkb)
    vd = v.cuda()
    o, lse = _sparse_attn(w, qp, kp, vd, sel[3], sel[4])
    rows = I.sampled_rows(w, 256, seed=3)
    ref, ref_lse = O.block_sparse_attention(to_np(qp), to_np(kp), to_np(v), keep, w.softmax_scale, rows=rows)
    got = to_np(o)[:, rows]
    assert rel_l2(got, ref) <= BF16_REL_L2
    assert np.max(np.abs(got - ref)) <= BF16_MAX_ABS
    assert np.max(np.abs(to_np(lse)[:, :, rows] - ref_lse)) <= BF16_LSE_ABS
    print(f"t2i_2048 tau=1.0: kept {keep.mean():.3f} of the key blocks")


def test_select_on_a_sequence_that_needs_more_shared_memory(cuda_ok):
    """Key-block scores live in shared memory (4 B per key block): two
    calls whose sequences need more than 48 KB, the second more than the
    first, both launch (the kernel's shared-memory limit is raised again).
    Checked on sampled query blocks against the oracle's rule applied to the
    kernel's probabilities and against pooled means recomputed here."""
    B, H, d = 1, 1, 128
    for n in (1_600_000, 2_000_000):
        g = torch.Generator(device="cuda").manual_seed(n)
        q = torch.randn((B, n, H, d), generator=g, device="cuda").to(torch.bfloat16)
        k = torch.randn((B, n, H, d), generator=g, device="cuda").to(torch.bfloat16)
        nqb, nkb = J.sparse_blocks(n)
        assert nkb * 4 > 48 * 1024
        qbar = torch.empty((B, H, nqb, d), dtype=torch.float32, device="cuda")
        kbar = torch.empty((B, H, nkb, d), dtype=torch.float32, device="cuda")
        idx = torch.empty((B, H, nqb, nkb), dtype=torch.int32, device="cuda")
        cnt = torch.empty((B, H, nqb), dtype=torch.int32, device="cuda")
        scale = 0.0883883
        J.jattn_sparse_select(q, k, qbar, kbar, None, idx, cnt, B, H, n, 0, 0, d, scale, 1.0)
        torch.cuda.synchronize()
        # Pooled means of a few blocks, recomputed from the tensors (float64).
        for i in (0, nkb // 2, nkb - 1):
            ref = k[0, i * 128:(i + 1) * 128, 0].double().mean(0)
            assert torch.allclose(kbar[0, 0, i].double(), ref, atol=2e-6 * float(k.abs().max()))
        # The kept lists of sampled query blocks: the rule on probabilities
        # formed here in float64 from the kernel's pooled means.
        kb = kbar[0, 0].double()
        for i in (0, nqb // 3, nqb - 1):
            s = scale * (kb @ qbar[0, 0, i].double())
            p = torch.softmax(s, 0).cpu().numpy()
            c = int(cnt[0, 0, i])
            row = to_np(idx[0, 0, i, :c]).astype(np.int64)
            assert c >= 1 and np.all(np.diff(row) > 0)
            # Blocks clearly above or below the threshold agree with the rule.
            thr = 1.0 / nkb
            clear_in = np.nonzero(p >= thr * (1 + 1e-3))[0]
            clear_out = np.nonzero(p < thr * (1 - 1e-3))[0]
            assert set(clear_in.tolist()) <= set(row.tolist())
            assert not (set(clear_out.tolist()) & set(row.tolist()) - {int(np.argmax(p))})
        del q, k, idx
        torch.cuda.empty_cache()
