"""The softmax's polynomial exp2 (degree-3 minimax fit of 2^f on [-1/2, 1/2]
after Cody-Waite range reduction) stays within its stated relative error
bound, 7.5e-5 plus float32 rounding, over the argument range the lazy-max
softmax feeds it ([-125, 8]; below -125 the argument is clamped)."""

import numpy as np
import pytest
import torch

from diffusion_transformer_joint_dit_b200 import binding as J

pytestmark = pytest.mark.gpu


def test_exp2_poly_error_bound(cuda_ok):
    rng = np.random.default_rng(41)
    x = np.concatenate([np.linspace(-125.0, 8.0, 1_000_001), rng.uniform(-30, 8, 200_000),
                        np.arange(-125, 9, dtype=np.float64), np.arange(-125, 8) + 0.5]).astype(np.float32)
    xd = torch.from_numpy(x).cuda()
    yd = torch.empty_like(xd)
    J.jattn_selftest_exp2_poly(xd, yd, x.size)
    torch.cuda.synchronize()
    y = yd.cpu().numpy().astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() <= 7.5e-5 + 4 * 2.0 ** -24, f"max relative error {rel.max():.3e}"
