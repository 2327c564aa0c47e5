"""Every entry point is asynchronous on the caller's stream and never
allocates or synchronises, so a whole step can be captured in a CUDA graph
and replayed (the tutorial's "Multi-GPU inference" section runs FLUX 3 with
CUDA Graphs).  Each test captures one path once, replays it on new inputs
copied into the captured buffers, and requires bit equality with direct
launches of the same calls.  The kernels use no atomics on floating-point
data, so results are deterministic.
"""

import pytest
import torch

from diffusion_transformer_joint_dit_b200 import binding as J
from diffusion_transformer_joint_dit_b200 import inputs as I
from tests.gpu_common import prologue_params

pytestmark = pytest.mark.gpu

W = I.custom("graph", B=2, H=2, n_txt=13, img_h=12, img_w=20, ref_h=3, ref_w=20, ref_row_offset=12)


def _replay_matches(step, inputs, outputs, seeds):
    """Warm up, capture step() in a graph, then for each seed: fill the
    inputs, replay, copy the outputs; run step() directly; compare."""
    step()  # first launches set kernel attributes outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for seed in seeds:
        gen = torch.Generator(device="cuda").manual_seed(seed)
        for t in inputs:
            if t.dtype == torch.uint8:
                continue
            t.copy_(torch.randn(t.shape, generator=gen, device="cuda").to(t.dtype))
        g.replay()
        torch.cuda.synchronize()
        got = [t.clone() for t in outputs]
        step()
        torch.cuda.synchronize()
        for a, b in zip(got, outputs):
            assert torch.equal(a, b)
    assert J.jattn_device_status() == J.JATTN_OK


def test_bf16_step_in_a_graph(cuda_ok):
    w = W
    shape = (w.B, w.N, w.H, w.d)
    q, k, v = (torch.empty(shape, dtype=torch.bfloat16, device="cuda") for _ in range(3))
    qo, ko, o = (torch.empty(shape, dtype=torch.bfloat16, device="cuda") for _ in range(3))
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device="cuda")
    p = prologue_params(w)

    def step():
        J.jattn_prologue(q, k, None, qo, ko, None, None, None, None, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d,
                         J.JATTN_PROLOGUE_BF16, p)
        J.jattn_fwd_bf16(qo, ko, v, o, lse, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d, w.softmax_scale)

    for t in (q, k, v):
        t.normal_()
    _replay_matches(step, [q, k, v], [qo, ko, o, lse], seeds=[1, 2])


def test_bf16_call_with_split_tail_in_a_graph(cuda_ok):
    """A problem whose jattn_fwd_bf16 call is two launches on 148 SMs (162
    work items: one whole wave, then 14 items run split over KV halves with
    programmatic dependent launch) captured and replayed in a graph."""
    w = I.custom("graph_tail", B=1, H=9, n_txt=512, img_h=64, img_w=64)
    shape = (w.B, w.N, w.H, w.d)
    q, k, v = (torch.empty(shape, dtype=torch.bfloat16, device="cuda") for _ in range(3))
    o = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device="cuda")

    def step():
        J.jattn_fwd_bf16(q, k, v, o, lse, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d, w.softmax_scale)

    for t in (q, k, v):
        t.normal_()
    _replay_matches(step, [q, k, v], [o, lse], seeds=[3, 4])


def test_fp8_step_with_repair_in_a_graph(cuda_ok):
    w = W
    shape = (w.B, w.N, w.H, w.d)
    nblk = -(-w.N // J.JATTN_FP8_BLOCK)
    m = J.repair_count(w.N, 0.02)
    q, k, v = (torch.empty(shape, dtype=torch.bfloat16, device="cuda") for _ in range(3))
    q8, k8, v8 = (torch.empty(shape, dtype=torch.uint8, device="cuda") for _ in range(3))
    qs, ks, vs = (torch.empty((w.B, w.H, nblk), dtype=torch.float32, device="cuda") for _ in range(3))
    o = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device="cuda")
    err = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device="cuda")
    idx = torch.empty((w.B, w.H, m), dtype=torch.int32, device="cuda")
    ksel = torch.empty((w.B, w.H, m, w.d), dtype=torch.bfloat16, device="cuda")
    vsel = torch.empty_like(ksel)
    p = prologue_params(w)

    def step():
        J.jattn_prologue(q, k, v, q8, k8, v8, qs, ks, vs, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d,
                         J.JATTN_PROLOGUE_FP8, p)
        J.jattn_fwd_fp8(q8, k8, v8, qs, ks, vs, o, lse, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d, w.softmax_scale)
        J.jattn_fp8_repair_select(k, v, k8, v8, ks, vs, p, m, err, idx, ksel, vsel, w.B, w.H, w.n_txt, w.n_img,
                                  w.n_ref, w.d)
        J.jattn_fp8_repair_apply(q8, qs, k8, v8, ks, vs, idx, ksel, vsel, m, o, lse, w.B, w.H, w.n_txt, w.n_img,
                                 w.n_ref, w.d, w.softmax_scale)

    for t in (q, k, v):
        t.normal_()
    _replay_matches(step, [q, k, v], [q8, k8, v8, qs, ks, vs, o, lse, idx], seeds=[3, 4])


def test_block_sparse_step_in_a_graph(cuda_ok):
    w = W
    shape = (w.B, w.N, w.H, w.d)
    nqb, nkb = J.sparse_blocks(w.N)
    q, k, v, o = (torch.empty(shape, dtype=torch.bfloat16, device="cuda") for _ in range(4))
    qbar = torch.empty((w.B, w.H, nqb, w.d), dtype=torch.float32, device="cuda")
    kbar = torch.empty((w.B, w.H, nkb, w.d), dtype=torch.float32, device="cuda")
    probs = torch.empty((w.B, w.H, nqb, nkb), dtype=torch.float32, device="cuda")
    idx = torch.empty((w.B, w.H, nqb, nkb), dtype=torch.int32, device="cuda")
    cnt = torch.empty((w.B, w.H, nqb), dtype=torch.int32, device="cuda")
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device="cuda")

    def step():
        J.jattn_sparse_select(q, k, qbar, kbar, probs, idx, cnt, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d,
                              w.softmax_scale, 1.0)
        J.jattn_fwd_bf16_sparse(q, k, v, o, lse, idx, cnt, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d,
                                w.softmax_scale)

    for t in (q, k, v):
        t.normal_()
    _replay_matches(step, [q, k, v], [probs, cnt, o, lse], seeds=[5, 6])


def test_fused_qkv_in_a_graph(cuda_ok):
    w = W
    C = 256
    x = torch.empty((w.B, w.N, C), dtype=torch.bfloat16, device="cuda")
    wt = (torch.randn((3 * w.H * w.d, C), device="cuda") / C ** 0.5).to(torch.bfloat16)
    wi = (torch.randn((3 * w.H * w.d, C), device="cuda") / C ** 0.5).to(torch.bfloat16)
    rope = torch.empty((w.N, 64, 2), dtype=torch.float32, device="cuda")
    shape = (w.B, w.N, w.H, w.d)
    q, k, v = (torch.empty(shape, dtype=torch.bfloat16, device="cuda") for _ in range(3))
    wts = J.make_qkv_weights(wt, wi)
    p = prologue_params(w)

    def step():
        J.jattn_rope_table(rope, w.n_txt, w.n_img, w.n_ref, p)
        J.jattn_qkv_fused(x, wts, rope, q, k, v, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d, C)

    x.normal_()
    _replay_matches(step, [x], [rope, q, k, v], seeds=[7, 8])
