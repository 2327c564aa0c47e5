"""Failure detection on the GPU without a fault: a bounded in-kernel wait
that runs out reports JATTN_ERR_TIMEOUT through the device error word, and
the context stays usable for the next launch."""

import pytest

from diffusion_transformer_joint_dit_b200 import binding as J
from diffusion_transformer_joint_dit_b200 import inputs as I
from tests.gpu_common import check_attention, gpu_attn_bf16, to_np

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_context_survives(cuda_ok):
    assert J.jattn_device_status() == J.JATTN_OK
    J.jattn_selftest_wait_timeout(20_000_000)       # 20 ms on a barrier nothing completes
    assert J.jattn_device_status() == J.JATTN_ERR_TIMEOUT
    assert J.jattn_device_status() == J.JATTN_OK    # read-and-clear
    w = I.WORKLOADS["tiny"]
    q, k, v = I.make_qkv(w, seed=21)
    o, lse = gpu_attn_bf16(w, q, k, v)
    check_attention(w, o, lse, to_np(q), to_np(k), to_np(v))
