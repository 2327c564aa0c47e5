"""Host-side checks of the C-ABI library (no GPU needed).

The library must load, export every function ``include/jattn.h`` declares,
and reject bad arguments with the documented status before touching CUDA.
No call here launches a kernel.
"""

import os
import re

import pytest

from diffusion_transformer_joint_dit_b200 import binding as J

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "jattn.h")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(J.LIB_PATH):
        from diffusion_transformer_joint_dit_b200 import build
        build.build()
    return J.load_library()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"JATTN_API\s+[\w\s\*]*?\b(jattn_\w+)\s*\(", text)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    assert {"jattn_prologue", "jattn_fwd_bf16", "jattn_fwd_fp8", "jattn_status_string"} <= names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) == set(J.EXPORTED)


def test_status_strings(lib):
    assert J.status_name(0) == "JATTN_OK"
    assert J.status_name(J.JATTN_ERR_TIMEOUT) == "JATTN_ERR_TIMEOUT"
    assert J.status_name(99) == "JATTN_ERR_UNKNOWN"


A = 1 << 20          # a 16-byte aligned fake device address; never dereferenced
MIS = A + 8          # misaligned


def fwd(**kw):
    args = dict(q=A, k=A, v=A, o=A + 4096, lse=None, B=1, H=2, N_txt=32, N_img=256, N_ref=0, d=128,
                softmax_scale=0.088)
    args.update(kw)
    return J.jattn_fwd_bf16(args["q"], args["k"], args["v"], args["o"], args["lse"], args["B"], args["H"],
                            args["N_txt"], args["N_img"], args["N_ref"], args["d"], args["softmax_scale"],
                            stream=0, check=False)


@pytest.mark.parametrize("kw,status", [
    (dict(d=64), J.JATTN_ERR_UNSUPPORTED),
    (dict(N_txt=0, N_img=0), J.JATTN_ERR_INVALID_ARG),
    (dict(N_txt=-1), J.JATTN_ERR_INVALID_ARG),
    (dict(B=0), J.JATTN_ERR_INVALID_ARG),
    (dict(H=0), J.JATTN_ERR_INVALID_ARG),
    (dict(q=None), J.JATTN_ERR_INVALID_ARG),
    (dict(o=None), J.JATTN_ERR_INVALID_ARG),
    (dict(k=MIS), J.JATTN_ERR_MISALIGNED),
    (dict(lse=A + 2), J.JATTN_ERR_MISALIGNED),
    (dict(softmax_scale=0.0), J.JATTN_ERR_INVALID_ARG),
    (dict(softmax_scale=float("inf")), J.JATTN_ERR_INVALID_ARG),
    (dict(softmax_scale=float("nan")), J.JATTN_ERR_INVALID_ARG),
])
def test_fwd_bf16_rejects_bad_arguments(lib, kw, status):
    assert fwd(**kw) == status


def prologue(mode=J.JATTN_PROLOGUE_BF16, params="default", **kw):
    args = dict(q=A, k=A, v=A, q_out=A, k_out=A, v_out=A, qs=A, ks=A, vs=A,
                B=1, H=2, N_txt=32, N_img=256, N_ref=0, d=128)
    args.update(kw)
    if params == "default":
        params = J.make_prologue_params(16, 16)
    return J.jattn_prologue(args["q"], args["k"], args["v"], args["q_out"], args["k_out"], args["v_out"],
                            args["qs"], args["ks"], args["vs"], args["B"], args["H"], args["N_txt"],
                            args["N_img"], args["N_ref"], args["d"], mode, params, stream=0, check=False)


@pytest.mark.parametrize("kw,status", [
    (dict(params=None), J.JATTN_ERR_INVALID_ARG),
    (dict(mode=7), J.JATTN_ERR_INVALID_ARG),
    (dict(N_img=255), J.JATTN_ERR_INVALID_ARG),                       # != img_h * img_w
    (dict(N_ref=16), J.JATTN_ERR_INVALID_ARG),                        # ref grid 0 x 0
    (dict(params=J.make_prologue_params(16, 16, rope_theta=0.0)), J.JATTN_ERR_INVALID_ARG),
    (dict(params=J.make_prologue_params(16, 16, eps=-1.0)), J.JATTN_ERR_INVALID_ARG),
    (dict(params=J.make_prologue_params(16, 16, q_norm_w=A + 4)), J.JATTN_ERR_MISALIGNED),
    (dict(q_out=MIS), J.JATTN_ERR_MISALIGNED),
    (dict(d=256), J.JATTN_ERR_UNSUPPORTED),
    (dict(mode=J.JATTN_PROLOGUE_FP8, vs=None), J.JATTN_ERR_INVALID_ARG),
    (dict(mode=J.JATTN_PROLOGUE_FP8, v_out=MIS), J.JATTN_ERR_MISALIGNED),
    (dict(mode=J.JATTN_PROLOGUE_FP8, ks=A + 2), J.JATTN_ERR_MISALIGNED),
])
def test_prologue_rejects_bad_arguments(lib, kw, status):
    assert prologue(**kw) == status


def test_reference_grids_are_validated(lib):
    # 32 text + 16 x 16 image + references of 2 x 16 and 1 x 8 = 40 tokens.
    call = lambda grids, n_ref=40: prologue(N_ref=n_ref, params=J.make_prologue_params(16, 16, ref_grids=grids))
    assert call([(2, 16, 16, 0), (1, 8, 18, 0)], n_ref=41) == J.JATTN_ERR_INVALID_ARG    # sizes do not add up
    assert call([(2, 16, 16, 0), (0, 8, 18, 0)]) == J.JATTN_ERR_INVALID_ARG              # empty grid
    assert call([(2, 16, -1, 0), (1, 8, 18, 0)]) == J.JATTN_ERR_INVALID_ARG              # negative offset
    assert call([(2, 16, 16, 0), (1, 8, 18, -3)]) == J.JATTN_ERR_INVALID_ARG
    assert call([(1, 4, 0, 0)] * 10) == J.JATTN_ERR_INVALID_ARG                           # more than 8 grids
    p = J.make_prologue_params(16, 16)
    p.n_ref_grids = 2                                                                      # no array
    assert prologue(N_ref=40, params=p) == J.JATTN_ERR_INVALID_ARG
    rope = lambda grids, n_ref: J.jattn_rope_table(A, 32, 256, n_ref, J.make_prologue_params(16, 16, ref_grids=grids),
                                                   stream=0, check=False)
    assert rope([(2, 16, 16, 0)], 31) == J.JATTN_ERR_INVALID_ARG


def test_fwd_fp8_rejects_bad_arguments(lib):
    call = lambda **kw: J.jattn_fwd_fp8(
        kw.get("q", A), A, A, kw.get("qs", A), A, A, A, None, 1, 2, 32, 256, 0, kw.get("d", 128), 0.088,
        stream=0, check=False)
    assert call(d=96) == J.JATTN_ERR_UNSUPPORTED
    assert call(q=None) == J.JATTN_ERR_INVALID_ARG
    assert call(q=MIS) == J.JATTN_ERR_MISALIGNED
    assert call(qs=A + 1) == J.JATTN_ERR_MISALIGNED


def qkv(weights="default", **kw):
    args = dict(x=A, rope=A, q=A, k=A, v=A, B=1, H=2, N_txt=32, N_img=256, N_ref=0, d=128, C=256)
    args.update(kw)
    if weights == "default":
        weights = J.make_qkv_weights(A, A)
    return J.jattn_qkv_fused(args["x"], weights, args["rope"], args["q"], args["k"], args["v"], args["B"],
                             args["H"], args["N_txt"], args["N_img"], args["N_ref"], args["d"], args["C"],
                             stream=0, check=False)


@pytest.mark.parametrize("kw,status", [
    (dict(H=3), J.JATTN_ERR_UNSUPPORTED),                             # two heads per output tile
    (dict(C=96), J.JATTN_ERR_UNSUPPORTED),                            # not a multiple of 64
    (dict(C=0), J.JATTN_ERR_UNSUPPORTED),
    (dict(d=64), J.JATTN_ERR_UNSUPPORTED),
    (dict(weights=None), J.JATTN_ERR_INVALID_ARG),
    (dict(weights=J.make_qkv_weights(None, A)), J.JATTN_ERR_INVALID_ARG),   # text tokens, no text weights
    (dict(weights=J.make_qkv_weights(A, None)), J.JATTN_ERR_INVALID_ARG),   # image tokens, no image weights
    (dict(weights=J.make_qkv_weights(A, A, eps=-1.0)), J.JATTN_ERR_INVALID_ARG),
    (dict(weights=J.make_qkv_weights(A, A, q_norm_w=(A + 4, None))), J.JATTN_ERR_MISALIGNED),
    (dict(rope=None), J.JATTN_ERR_INVALID_ARG),
    (dict(x=MIS), J.JATTN_ERR_MISALIGNED),
    (dict(v=MIS), J.JATTN_ERR_MISALIGNED),
    (dict(N_txt=0, N_img=0), J.JATTN_ERR_INVALID_ARG),
])
def test_qkv_fused_rejects_bad_arguments(lib, kw, status):
    assert qkv(**kw) == status


def test_rope_table_rejects_bad_arguments(lib):
    call = lambda table=A, n_img=256, params="default": J.jattn_rope_table(
        table, 32, n_img, 0, J.make_prologue_params(16, 16) if params == "default" else params,
        stream=0, check=False)
    assert call(table=None) == J.JATTN_ERR_INVALID_ARG
    assert call(table=MIS) == J.JATTN_ERR_MISALIGNED
    assert call(params=None) == J.JATTN_ERR_INVALID_ARG
    assert call(n_img=255) == J.JATTN_ERR_INVALID_ARG
    assert call(params=J.make_prologue_params(16, 16, rope_theta=-1.0)) == J.JATTN_ERR_INVALID_ARG


def test_sparse_select_rejects_bad_arguments(lib):
    def call(**kw):
        a = dict(q=A, k=A, qbar=A, kbar=A, probs=None, idx=A, cnt=A, d=128, scale=0.088, tau=1.0, n_img=256)
        a.update(kw)
        return J.jattn_sparse_select(a["q"], a["k"], a["qbar"], a["kbar"], a["probs"], a["idx"], a["cnt"], 1, 2,
                                     32, a["n_img"], 0, a["d"], a["scale"], a["tau"], stream=0, check=False)
    assert call(d=64) == J.JATTN_ERR_UNSUPPORTED
    assert call(k=None) == J.JATTN_ERR_INVALID_ARG
    assert call(qbar=None) == J.JATTN_ERR_INVALID_ARG
    assert call(cnt=None) == J.JATTN_ERR_INVALID_ARG
    assert call(tau=-0.5) == J.JATTN_ERR_INVALID_ARG
    assert call(tau=float("nan")) == J.JATTN_ERR_INVALID_ARG
    assert call(scale=0.0) == J.JATTN_ERR_INVALID_ARG
    assert call(n_img=1 << 22) == J.JATTN_ERR_INVALID_ARG            # beyond 2^22 tokens
    assert call(kbar=MIS) == J.JATTN_ERR_MISALIGNED
    assert call(probs=A + 2) == J.JATTN_ERR_MISALIGNED
    assert call(idx=A + 1) == J.JATTN_ERR_MISALIGNED


def test_fwd_bf16_sparse_rejects_bad_arguments(lib):
    def call(**kw):
        a = dict(q=A, v=A, o=A + 4096, lse=None, idx=A, cnt=A, d=128, scale=0.088)
        a.update(kw)
        return J.jattn_fwd_bf16_sparse(a["q"], A, a["v"], a["o"], a["lse"], a["idx"], a["cnt"], 1, 2, 32, 256, 0,
                                       a["d"], a["scale"], stream=0, check=False)
    assert call(d=256) == J.JATTN_ERR_UNSUPPORTED
    assert call(idx=None) == J.JATTN_ERR_INVALID_ARG
    assert call(cnt=None) == J.JATTN_ERR_INVALID_ARG
    assert call(o=None) == J.JATTN_ERR_INVALID_ARG
    assert call(scale=float("inf")) == J.JATTN_ERR_INVALID_ARG
    assert call(v=MIS) == J.JATTN_ERR_MISALIGNED
    assert call(cnt=A + 2) == J.JATTN_ERR_MISALIGNED
    assert call(lse=A + 1) == J.JATTN_ERR_MISALIGNED


def test_sparse_block_counts():
    assert J.sparse_blocks(16896) == (66, 132)
    assert J.sparse_blocks(300) == (2, 3)
    assert J.sparse_blocks(1) == (1, 1)


def test_selftest_rejects_bad_timeout(lib):
    assert J.jattn_selftest_wait_timeout(0, stream=0, check=False) == J.JATTN_ERR_INVALID_ARG
    assert J.jattn_selftest_wait_timeout(2 * 10 ** 9, stream=0, check=False) == J.JATTN_ERR_INVALID_ARG


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(J, "_lib", None)
    monkeypatch.setattr(J, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(RuntimeError, match="not built"):
        J.load_library()


def test_attention_api_rejects_bad_inputs_without_a_launch():
    import torch
    from diffusion_transformer_joint_dit_b200 import attention as A
    x = torch.zeros((1, 4, 1, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        A.joint_attention(x, x, x, n_txt=4, img_h=0, img_w=0, config=A.AttentionConfig(mode="fp4"))
    with pytest.raises(ValueError):
        A.joint_attention(x, x, x, n_txt=4, img_h=0, img_w=0)      # CPU tensors
