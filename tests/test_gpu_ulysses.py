"""Ulysses path on one GPU: a one-rank NCCL group, the all-to-all exchanges
and the jattn prologue + BF16 attention on the head shard.  With one rank the
exchanges are layout round trips, so the result must equal the direct
library call bit for bit, and it must match the float64 oracle within the
BF16 tolerances."""

import os

import pytest
import torch
import torch.distributed as dist

from diffusion_transformer_joint_dit_b200 import binding as J
from diffusion_transformer_joint_dit_b200 import inputs as I
from diffusion_transformer_joint_dit_b200 import ulysses as U
from tests.gpu_common import check_attention, oracle_prologue_bf16, to_np


@pytest.fixture(scope="module")
def nccl_group(cuda_ok):
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", str(29400 + os.getpid() % 500))
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    yield None
    dist.destroy_process_group()


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["tiny", "t2i_1024"])
def test_ulysses_one_rank_equals_direct(nccl_group, name):
    w = I.WORKLOADS[name]
    q, k, v = (t.cuda() for t in I.make_qkv(w, 0))
    prologue, attn = U.jattn_bf16_ops(w.n_txt, w.n_img, w.n_ref, w.softmax_scale, w.img_h, w.img_w,
                                      w.ref_h, w.ref_w, w.ref_row_offset)
    got = U.ulysses_attention(q, k, v, n_total=w.N, attn=attn, prologue=prologue)
    qp, kp, _ = prologue(q, k, v)
    want = attn(qp, kp, v)
    torch.cuda.synchronize()
    assert J.jattn_device_status() == J.JATTN_OK
    assert torch.equal(got, want)
    # And against the float64 oracle chain (prologue, bf16 rounding,
    # attention) on every row of tiny, 256 sampled rows of t2i_1024.
    rows = None if w.N <= 512 else I.sampled_rows(w, 256)
    _, _, qb, kb = oracle_prologue_bf16(w, q.cpu(), k.cpu())
    check_attention(w, got, None, qb, kb, to_np(v), rows=rows)
