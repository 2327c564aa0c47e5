"""The one-call API (attention.joint_attention) against the float64 oracle
and against the same library calls made one by one."""

import pytest
import torch

import oracle as O
from diffusion_transformer_joint_dit_b200 import attention as A
from diffusion_transformer_joint_dit_b200 import binding as J
from diffusion_transformer_joint_dit_b200 import inputs as I
from tests.gpu_common import (BF16_REL_L2, FP8_REL_L2, assert_equal_but_split_tail, gpu_attn_bf16,
                              gpu_prologue_bf16, gpu_prologue_fp8, oracle_prologue_bf16, rel_l2, to_np)

pytestmark = pytest.mark.gpu

W = I.custom("api", B=2, H=2, n_txt=24, img_h=12, img_w=16, ref_h=4, ref_w=16, ref_row_offset=12)


def _call(mode, q, k, v, **kw):
    return A.joint_attention(q.cuda(), k.cuda(), v.cuda(), n_txt=W.n_txt, img_h=W.img_h, img_w=W.img_w,
                             ref_h=W.ref_h, ref_w=W.ref_w, ref_row_offset=W.ref_row_offset,
                             config=A.AttentionConfig(mode=mode, **kw), return_lse=True)


def test_bf16_mode_matches_the_oracle_and_the_calls(cuda_ok):
    q, k, v = I.make_qkv(W, seed=21)
    o, lse = _call("bf16", q, k, v)
    _, _, qb, kb = oracle_prologue_bf16(W, q, k)
    ref, _ = O.joint_attention(qb, kb, to_np(v), W.softmax_scale)
    assert rel_l2(to_np(o), ref) <= BF16_REL_L2
    qp, kp = gpu_prologue_bf16(W, q, k)
    od, lsed = gpu_attn_bf16(W, qp.cpu(), kp.cpu(), v)
    assert torch.equal(o, od) and torch.equal(lse, lsed)


@pytest.mark.parametrize("mode", ["fp8", "fp8_repair"])
def test_fp8_modes_match_the_quantised_oracle(cuda_ok, mode):
    q, k, v = I.make_qkv(W, seed=22)
    o, lse = _call(mode, q, k, v, rho=0.02)
    assert torch.isfinite(lse).all()
    # The oracle on the same E4M3 codes (re-run the prologue to read them).
    codes, scales = gpu_prologue_fp8(W, q, k, v)
    deq = [O.dequantize_e4m3(to_np(c), to_np(s)) for c, s in zip(codes, scales)]
    if mode == "fp8":
        ref, _ = O.joint_attention(deq[0], deq[1], deq[2], W.softmax_scale)
    else:
        _, _, _, kb = oracle_prologue_bf16(W, q, k)
        idx, _ = O.repair_select(kb, to_np(v), deq[1], deq[2], rho=0.02)
        ref, _ = O.repaired_attention(deq[0], deq[1], deq[2], kb, to_np(v), idx, W.softmax_scale)
    assert rel_l2(to_np(o), ref) <= FP8_REL_L2


def test_sparse_mode_at_tau_zero_is_the_bf16_mode(cuda_ok):
    q, k, v = I.make_qkv(W, seed=23)
    o_dense, l_dense = _call("bf16", q, k, v)
    o_sparse, l_sparse = _call("sparse", q, k, v, tau=0.0)
    assert_equal_but_split_tail(W, o_sparse, l_sparse, o_dense, l_dense)


def test_strided_views_give_the_contiguous_result(cuda_ok):
    """q, k, v as views of one packed [B, N, 3, H, d] projection output (not
    contiguous) give the same result as contiguous copies."""
    q, k, v = I.make_qkv(W, seed=24)
    packed = torch.stack([q, k, v], dim=2).cuda()
    qv, kv, vv = packed.unbind(2)
    assert not qv.is_contiguous()
    o_view, l_view = A.joint_attention(qv, kv, vv, n_txt=W.n_txt, img_h=W.img_h, img_w=W.img_w, ref_h=W.ref_h,
                                       ref_w=W.ref_w, ref_row_offset=W.ref_row_offset, return_lse=True)
    o, lse = _call("bf16", q, k, v)
    assert torch.equal(o_view, o) and torch.equal(l_view, lse)
