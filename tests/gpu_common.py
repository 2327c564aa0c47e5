"""Helpers shared by the GPU parity tests: run the CUDA path through the
C-ABI binding, run the oracle on the same seeded inputs, compare."""

from __future__ import annotations

import numpy as np
import torch

import oracle as O
from diffusion_transformer_joint_dit_b200 import binding as J
from diffusion_transformer_joint_dit_b200 import inputs as I

# Tolerances (workload definition): BF16 attention relative L2 <= 5e-3 and
# max-abs <= 2e-2 on N(0,1) inputs; FP8 attention relative L2 <= 1e-2 against
# the oracle that applies the same E4M3 block quantisation.
BF16_REL_L2 = 5e-3
BF16_MAX_ABS = 2e-2
FP8_REL_L2 = 1e-2


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def to_np(t: torch.Tensor) -> np.ndarray:
    """bf16 / fp32 torch tensor (any device) -> float32 numpy (exact)."""
    return t.detach().float().cpu().numpy()


def prologue_params(w: I.Workload):
    return J.make_prologue_params(w.img_h, w.img_w, w.ref_h, w.ref_w, w.ref_row_offset, w.theta, w.eps,
                                  ref_grids=w.ref_grids or None)


def gpu_prologue_bf16(w: I.Workload, q, k):
    qd, kd = q.cuda(), k.cuda()
    qo, ko = torch.empty_like(qd), torch.empty_like(kd)
    J.jattn_prologue(qd, kd, None, qo, ko, None, None, None, None, w.B, w.H, w.n_txt, w.n_img, w.n_ref,
                     w.d, J.JATTN_PROLOGUE_BF16, prologue_params(w))
    torch.cuda.synchronize()
    return qo, ko


def gpu_prologue_fp8(w: I.Workload, q, k, v):
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    shape = (w.B, w.N, w.H, w.d)
    nblk = -(-w.N // J.JATTN_FP8_BLOCK)
    q8, k8, v8 = (torch.empty(shape, dtype=torch.uint8, device="cuda") for _ in range(3))
    qs, ks, vs = (torch.empty((w.B, w.H, nblk), dtype=torch.float32, device="cuda") for _ in range(3))
    J.jattn_prologue(qd, kd, vd, q8, k8, v8, qs, ks, vs, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d,
                     J.JATTN_PROLOGUE_FP8, prologue_params(w))
    torch.cuda.synchronize()
    return (q8, k8, v8), (qs, ks, vs)


def gpu_attn_bf16(w: I.Workload, q, k, v, with_lse: bool = True):
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = torch.full_like(qd, float("nan"))
    lse = torch.full((w.B, w.H, w.N), float("nan"), dtype=torch.float32, device="cuda") if with_lse else None
    J.jattn_fwd_bf16(qd, kd, vd, o, lse, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d, w.softmax_scale)
    torch.cuda.synchronize()
    assert J.jattn_device_status() == J.JATTN_OK
    return o, lse


def split_tail_rows(B: int, H: int, N: int) -> np.ndarray:
    """Boolean [B, H, N] mask of the query rows that jattn_fwd_bf16 computes
    in its split tail (include/jattn.h: the work items, 256 query rows of
    one (b, h) in (b, h, block) order, past the last whole wave of one per
    SM, run split over KV halves when they fill at most half of the SMs and
    N spans at least two KV tiles).  Those rows differ from a one-pass
    computation by the rounding of the merge only."""
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    n_qb, n_kv = -(-N // 256), -(-N // 128)
    items = n_qb * H * B
    rem = items % sms
    tail = rem if n_kv >= 2 and 2 * rem <= sms else 0
    mask = np.zeros((B, H, n_qb), dtype=bool)
    mask.reshape(-1)[items - tail:] = True
    return np.repeat(mask, 256, axis=2)[:, :, :N]


def assert_equal_but_split_tail(w: I.Workload, o_a, lse_a, o_b, lse_b):
    """o_a / lse_a from a one-pass kernel (e.g. the block-sparse kernel with
    every block kept), o_b / lse_b from jattn_fwd_bf16 on the same inputs:
    bitwise equal on rows outside the split tail.  On its rows each half
    keeps its own lazy row maximum, so the bf16 P (relative rounding 2^-9)
    and the per-tile corrections of l differ from the one-pass run: the two
    agree to that rounding noise (rel-L2 <= 2e-3, max-abs <= 2^-6 of the
    largest |O|, LSE within the BF16 LSE bound), while each is checked
    against the oracle elsewhere."""
    split = split_tail_rows(w.B, w.H, w.N)                 # [B, H, N]
    rows = np.transpose(split, (0, 2, 1))                  # [B, N, H] like O
    oa, ob = to_np(o_a), to_np(o_b)
    assert np.array_equal(oa[~rows], ob[~rows])
    assert np.array_equal(to_np(lse_a)[~split], to_np(lse_b)[~split])
    if rows.any():
        assert rel_l2(oa[rows], ob[rows]) <= 2e-3
        assert np.max(np.abs(oa[rows] - ob[rows])) <= 2.0 ** -6 * max(1.0, float(np.max(np.abs(ob[rows]))))
        assert np.max(np.abs(to_np(lse_a)[split] - to_np(lse_b)[split])) <= BF16_LSE_ABS


def oracle_prologue_bf16(w: I.Workload, q, k):
    """Oracle Q', K' (float64) and their bf16 roundings (float64 arrays)."""
    qp, kp = O.prologue(to_np(q), to_np(k), n_txt=w.n_txt, img_h=w.img_h, img_w=w.img_w,
                        ref_h=w.ref_h, ref_w=w.ref_w, ref_row_offset=w.ref_row_offset,
                        ref_grids=list(w.ref_grids) or None, theta=w.theta, eps=w.eps)
    return qp, kp, O.bf16_round(qp), O.bf16_round(kp)


# LSE: the kernels sum the P values as rounded for the P.V product (bf16 on
# the BF16 path), so ln(l) carries up to 2^-9 relative rounding of l; the
# bound is 2^-8.
BF16_LSE_ABS = 2.0 ** -8


def check_attention(w: I.Workload, out, lse, q_np, k_np, v_np, rows=None, rel_tol=BF16_REL_L2,
                    abs_tol=BF16_MAX_ABS, lse_tol=BF16_LSE_ABS):
    """Compare GPU O (and LSE) with the oracle on `rows` (all if None)."""
    ref, ref_lse = O.joint_attention(q_np, k_np, v_np, w.softmax_scale, rows=rows)
    o = to_np(out)
    if rows is not None:
        o = o[:, rows]
    assert np.isfinite(o).all(), "unwritten or non-finite output"
    err = rel_l2(o, ref)
    mx = float(np.max(np.abs(o - ref)))
    assert err <= rel_tol, f"rel-L2 {err:.3e} > {rel_tol}"
    assert mx <= abs_tol, f"max-abs {mx:.3e} > {abs_tol}"
    if lse is not None:
        l = to_np(lse)
        if rows is not None:
            l = l[:, :, rows]
        lerr = float(np.max(np.abs(l - ref_lse)))
        assert lerr <= lse_tol, f"LSE max-abs {lerr:.3e} > {lse_tol:.3e}"
    return err, mx
