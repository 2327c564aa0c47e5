"""The dense-step cutoff of block-sparse attention against the worked
figures of the tutorial's "Quantized and sparse attention" section."""

import pytest

from diffusion_transformer_joint_dit_b200 import schedule as S


@pytest.mark.parametrize("steps,cutoff,dense", [(50, 0.96, 12), (16, 0.96, 4), (50, 0.94, 16)])
def test_dense_steps_match_the_pages(steps, cutoff, dense):
    assert S.dense_steps(steps, 6.93, cutoff) == dense
    assert not S.sparse_active(dense - 1, steps, 6.93, cutoff)
    assert S.sparse_active(dense, steps, 6.93, cutoff)


def test_shift_endpoints_and_identity():
    assert S.shifted_sigma(0, 50, 6.93) == 1.0
    # alpha = 1 is the unshifted linear grid.
    assert S.shifted_sigma(10, 50, 1.0) == pytest.approx(0.8)
    assert S.dense_steps(10, 6.93, 0.0) == 10
    assert S.dense_steps(10, 6.93, 1.5) == 0
    with pytest.raises(ValueError):
        S.shifted_sigma(5, 5, 6.93)
