"""jattn_sparse_select_noalloc: the block selection for callers that cannot
allocate device memory (an engine plugin whose enqueue may not allocate,
code inside a stream capture, a process whose device memory belongs to its
own pool allocator).  Its pooled-means workspace is a fixed 16 MiB device
array inside the library instead of caller-allocated qbar / kbar.

The GPU test calls it through the C-ABI twice in a row, on two different
problems, and requires the same lists, counts and probabilities as
jattn_sparse_select with a caller-allocated workspace: the second call runs
over the first call's leftovers in the shared array.  The file is named to
be collected last, so that a run stopping at the first failure has already
run every other test.
"""

import numpy as np
import pytest
import torch

from diffusion_transformer_joint_dit_b200 import binding as J
from diffusion_transformer_joint_dit_b200 import inputs as I

SCRATCH_BYTES = 16 << 20

FAKE = 1 << 20  # a 16-byte aligned stand-in address; never dereferenced


def _scratch_bytes(B, H, N):
    nqb, nkb = J.sparse_blocks(N)
    return B * H * (nqb + nkb) * 128 * 4


def test_noalloc_rejects_problems_beyond_its_workspace():
    # B = 2, H = 24 fits up to N = 58112; one more token does not.  The
    # check runs before any CUDA call, so no GPU is needed.
    assert _scratch_bytes(2, 24, 58112) <= SCRATCH_BYTES < _scratch_bytes(2, 24, 58113)
    args = (FAKE, FAKE, None, FAKE, FAKE)
    st = J.jattn_sparse_select_noalloc(*args, 2, 24, 512, 58113 - 512, 0, 128, 0.088, 1.0, stream=0, check=False)
    assert st == J.JATTN_ERR_UNSUPPORTED
    st = J.jattn_sparse_select_noalloc(*args, 1, 1, 0, 16, 0, 64, 0.088, 1.0, stream=0, check=False)
    assert st == J.JATTN_ERR_UNSUPPORTED  # head dim
    st = J.jattn_sparse_select_noalloc(FAKE, FAKE, None, None, FAKE, 1, 1, 0, 16, 0, 128, 0.088, 1.0, stream=0,
                                       check=False)
    assert st == J.JATTN_ERR_INVALID_ARG  # missing output
    st = J.jattn_sparse_select_noalloc(*args, 1, 1, 0, 16, 0, 128, 0.088, -1.0, stream=0, check=False)
    assert st == J.JATTN_ERR_INVALID_ARG  # tau


def _blocky(w, seed):
    """Q', K' with a mean vector per 128-token block, drawn on the GPU."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    shape = (w.B, w.N, w.H, w.d)
    nkb = -(-w.N // 128)
    out = []
    for _ in range(2):
        base = torch.randn(shape, generator=g, device="cuda")
        means = torch.randn((w.B, nkb, w.H, w.d), generator=g, device="cuda") * 1.5
        out.append((base + means.repeat_interleave(128, dim=1)[:, :w.N]).to(torch.bfloat16))
    return out


def _outputs(w):
    nqb, nkb = J.sparse_blocks(w.N)
    probs = torch.full((w.B, w.H, nqb, nkb), float("nan"), dtype=torch.float32, device="cuda")
    idx = torch.full((w.B, w.H, nqb, nkb), -1, dtype=torch.int32, device="cuda")
    cnt = torch.full((w.B, w.H, nqb), -1, dtype=torch.int32, device="cuda")
    return probs, idx, cnt


def _with_workspace(w, q, k, tau):
    nqb, nkb = J.sparse_blocks(w.N)
    qbar = torch.empty((w.B, w.H, nqb, w.d), dtype=torch.float32, device="cuda")
    kbar = torch.empty((w.B, w.H, nkb, w.d), dtype=torch.float32, device="cuda")
    probs, idx, cnt = _outputs(w)
    J.jattn_sparse_select(q, k, qbar, kbar, probs, idx, cnt, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d,
                          w.softmax_scale, tau)
    return probs, idx, cnt


def _without_workspace(w, q, k, tau):
    probs, idx, cnt = _outputs(w)
    J.jattn_sparse_select_noalloc(q, k, probs, idx, cnt, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d,
                                  w.softmax_scale, tau)
    return probs, idx, cnt


def _assert_same(w, got, want):
    probs, idx, cnt = (t.cpu().numpy() for t in got)
    probs_w, idx_w, cnt_w = (t.cpu().numpy() for t in want)
    # Counts and lists are integer results: identical.  Probabilities: the
    # relative bound the block-sparse parity tests use (1e-4).
    assert np.array_equal(cnt, cnt_w)
    for pos in np.ndindex(*cnt.shape):
        assert np.array_equal(idx[pos][:cnt[pos]], idx_w[pos][:cnt_w[pos]]), pos
    assert np.isfinite(probs).all()
    assert np.max(np.abs(probs - probs_w) / np.maximum(np.abs(probs_w), 1e-30)) <= 1e-4


@pytest.mark.gpu
def test_noalloc_matches_caller_workspace_on_two_calls_in_a_row(cuda_ok):
    torch.cuda.set_device(0)
    # Call 1: the 2048^2 text-to-image shapes (B = 2, H = 24, N = 16896,
    # 4.9 MB of the workspace).  Call 2: a small ragged problem (3 query
    # blocks, the last partial) over call 1's leftovers.
    big = I.WORKLOADS["t2i_2048"]
    small = I.custom("ragged", B=1, H=2, n_txt=12, img_h=16, img_w=43)
    runs = []
    for w, tau, seed in ((big, 1.0, 3), (small, 0.5, 4)):
        q, k = _blocky(w, seed)
        got = _without_workspace(w, q, k, tau)
        torch.cuda.synchronize()
        want = _with_workspace(w, q, k, tau)
        torch.cuda.synchronize()
        runs.append((w, got, want))
    assert J.jattn_device_status() == J.JATTN_OK
    for w, got, want in runs:
        _assert_same(w, got, want)
    # The small problem really drops blocks, so the lists are not trivial.
    assert (runs[1][1][2] < J.sparse_blocks(small.N)[1]).any()
