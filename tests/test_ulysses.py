"""Ulysses sequence parallelism and the CFG x Ulysses rank layout, on CPU
ranks (gloo).  The exchange and layout code is the product's; the compute
injected here is the float64 oracle, so a rank's output must equal the rows
of the full-sequence oracle result that rank owns."""

import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from diffusion_transformer_joint_dit_b200 import ulysses as U  # noqa: E402


def test_shard_sizes_cover_and_balance():
    for n in (1, 7, 64, 100, 16896):
        for p in (1, 2, 3, 4, 8):
            s = U.shard_sizes(n, p)
            assert len(s) == p and sum(s) == n and max(s) - min(s) <= 1
            starts = [U.shard_bounds(n, p, r)[0] for r in range(p)]
            ends = [U.shard_bounds(n, p, r)[1] for r in range(p)]
            assert starts[0] == 0 and ends[-1] == n and starts[1:] == ends[:-1]
    with pytest.raises(ValueError):
        U.shard_sizes(10, 0)


def test_parallel_layout():
    lay = U.ParallelLayout.make(8, 2)
    assert (lay.cfg, lay.sp) == (2, 4)
    assert [lay.cfg_index(r) for r in range(8)] == [0, 0, 0, 0, 1, 1, 1, 1]
    assert [lay.sp_rank(r) for r in range(8)] == [0, 1, 2, 3, 0, 1, 2, 3]
    assert lay.sp_group_ranks(1) == [4, 5, 6, 7]
    with pytest.raises(ValueError):
        U.ParallelLayout.make(6, 4)


# Problem: joint sequence of 5 text + 4x6 image + 2x3 reference tokens, so
# shards straddle stream boundaries and are uneven for P = 3.
CASE = dict(B=2, H=6, d=16, n_txt=5, img_h=4, img_w=6, ref_h=2, ref_w=3, ref_row_offset=4)


def _case_tensors():
    rng = np.random.default_rng(7)
    n = CASE["n_txt"] + CASE["img_h"] * CASE["img_w"] + CASE["ref_h"] * CASE["ref_w"]
    shape = (CASE["B"], n, CASE["H"], CASE["d"])
    return n, [rng.standard_normal(shape) for _ in range(3)]


def _oracle_ops(scale):
    from oracle import jattn_oracle as O

    def prologue(q, k, v):
        qp, kp = O.prologue(q.numpy(), k.numpy(), n_txt=CASE["n_txt"], img_h=CASE["img_h"], img_w=CASE["img_w"],
                            ref_h=CASE["ref_h"], ref_w=CASE["ref_w"], ref_row_offset=CASE["ref_row_offset"])
        return torch.from_numpy(qp), torch.from_numpy(kp), v

    def attn(q, k, v):
        o, _ = O.joint_attention(q.numpy(), k.numpy(), v.numpy(), scale)
        return torch.from_numpy(o)

    return prologue, attn


def _worker(rank, world, port, out, cfg):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lay = U.ParallelLayout.make(world, cfg)
        group = U.new_sp_groups(lay) if cfg > 1 else None
        n, (q, k, v) = _case_tensors()
        # CFG branch c takes batch element c (B = cfg branches here), the
        # sequence rank its shard of the joint sequence.
        bsl = slice(lay.cfg_index(rank), lay.cfg_index(rank) + 1) if cfg > 1 else slice(None)
        s0, s1 = U.shard_bounds(n, lay.sp, lay.sp_rank(rank))
        shard = [torch.from_numpy(np.ascontiguousarray(t[bsl, s0:s1])) for t in (q, k, v)]
        prologue, attn = _oracle_ops(scale=0.25)
        o = U.ulysses_attention(*shard, n_total=n, attn=attn, prologue=prologue, group=group)
        out[rank] = (bsl.start, s0, s1, o.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,cfg", [(2, 1), (3, 1), (4, 2)])
def test_ulysses_matches_full_sequence_oracle(world, cfg):
    from oracle import jattn_oracle as O

    n, (q, k, v) = _case_tensors()
    qp, kp = O.prologue(q, k, n_txt=CASE["n_txt"], img_h=CASE["img_h"], img_w=CASE["img_w"],
                        ref_h=CASE["ref_h"], ref_w=CASE["ref_w"], ref_row_offset=CASE["ref_row_offset"])
    full, _ = O.joint_attention(qp, kp, v, 0.25)
    port = 29500 + (os.getpid() * 7 + world * 31 + cfg) % 1500
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out, cfg), nprocs=world, join=True)
        covered = np.zeros(full.shape[:2], dtype=int)
        for r in range(world):
            b0, s0, s1, o = out[r]
            ref = full[:, s0:s1] if b0 is None else full[b0:b0 + 1, s0:s1]
            # Same float64 arithmetic on the same head slices: exact.
            np.testing.assert_array_equal(o, ref)
            if b0 is None:
                covered[:, s0:s1] += 1
            else:
                covered[b0, s0:s1] += 1
        assert (covered == 1).all()  # every (batch, token) row produced by exactly one rank


def _layout_worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b, h, d = 2, 4, 3
        sizes = U.shard_sizes(7, world)
        s0, s1 = U.shard_bounds(7, world, rank)
        # Element value encodes (b, token, head, channel) of the full tensor.
        full = torch.arange(b * 7 * h * d, dtype=torch.float32).view(b, 7, h, d)
        heads = U.seq_to_heads(full[:, s0:s1].contiguous(), sizes)
        hp = h // world
        ok_heads = torch.equal(heads, full[:, :, rank * hp:(rank + 1) * hp])
        back = U.heads_to_seq(heads, sizes)
        out[rank] = (ok_heads, torch.equal(back, full[:, s0:s1]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_all_to_all_layouts_round_trip(world):
    port = 29500 + (os.getpid() * 11 + world * 17) % 1500
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_layout_worker, args=(world, port, out), nprocs=world, join=True)
        for r in range(world):
            assert out[r] == (True, True)
