"""Argument checks of attention.joint_attention that run before any CUDA
call (no GPU needed)."""

import pytest
import torch

from diffusion_transformer_joint_dit_b200 import attention as A

KW = dict(n_txt=4, img_h=2, img_w=2)


def _t(shape=(1, 8, 2, 128), dtype=torch.bfloat16):
    return torch.zeros(shape, dtype=dtype)


@pytest.mark.parametrize("k,v", [
    (_t((1, 8, 3, 128)), _t()),               # k shape differs
    (_t(), _t((1, 7, 2, 128))),               # v shape differs
    (_t(dtype=torch.float16), _t()),          # k dtype differs
    (_t(), _t(dtype=torch.float32)),          # v dtype differs
    (_t(), _t()),                             # all on the CPU
])
def test_mismatched_or_host_inputs_are_rejected(k, v):
    with pytest.raises(ValueError):
        A.joint_attention(_t(), k, v, **KW)


def test_three_dimensional_input_is_rejected():
    with pytest.raises(ValueError):
        A.joint_attention(_t((8, 2, 128)), _t((8, 2, 128)), _t((8, 2, 128)), **KW)


def test_unknown_mode_is_rejected():
    with pytest.raises(ValueError):
        A.joint_attention(_t(), _t(), _t(), config=A.AttentionConfig(mode="int4"), **KW)
