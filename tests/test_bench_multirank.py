"""Host-side multi-rank logic of bench.py on CPU (gloo, world size 2): the
step time is the max over ranks, the value is whole-job (weak scaling),
and the reference arm runs on rank 0 only."""

import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 3.0], torch.device("cpu"))
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    world = 2
    port = 29500 + os.getpid() % 1000
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        for r in range(world):
            assert out[r] == [2.0, 10.0, 3.0]


def test_weak_scaling_value_and_single_rank_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.weak_scaling_value(4, 7e12, 7.0) == pytest.approx(4000.0)
    assert bench.max_over_ranks([5.0, 6.0], torch.device("cpu")) == [5.0, 6.0]


def test_reference_arm_only_on_rank0(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        workload = "tiny"
        steps = 1
        warmup = 0

    assert bench.run_reference(Args(), rank=1, world=2) == 0
    assert capsys.readouterr().out == ""


# ---- bench.py's multi-GPU path: CFG branches x Ulysses sequence shards ----

def _cfg_case():
    sys.path.insert(0, ROOT)
    from diffusion_transformer_joint_dit_b200 import inputs as I
    # d = 16 keeps the float64 oracle quick; 10% of K' rows are outliers so
    # that the head shard's K input must come from the right (b, t, h) rows.
    return I.custom("cfg_sp", B=2, H=4, d=16, n_txt=5, img_h=4, img_w=6, ref_h=2, ref_w=3, ref_row_offset=4,
                    k_outlier_frac=0.1)


def _cfg_oracle(w):
    import numpy as np

    from diffusion_transformer_joint_dit_b200 import inputs as I
    from oracle import jattn_oracle as O
    q, k, v = (t.double().numpy() for t in I.make_qkv(w, seed=0))
    kw = dict(n_txt=w.n_txt, img_h=w.img_h, img_w=w.img_w, ref_h=w.ref_h, ref_w=w.ref_w,
              ref_row_offset=w.ref_row_offset)
    qp, kp = O.prologue(q, k, **kw)
    kp_out = kp.copy()
    kp_out[I.outlier_rows(w, 0)] *= w.k_outlier_gain
    full, _ = O.joint_attention(qp, kp_out, v, 0.25)
    return (q, k, v), kp_out, full, kw, np


def _cfg_worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import bench
    from diffusion_transformer_joint_dit_b200 import ulysses as U
    from oracle import jattn_oracle as O
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = _cfg_case()
        (q, k, v), kp_out, _, kw, np = _cfg_oracle(w)
        layout, bsl, (s0, s1) = bench.cfg_ulysses_plan(w, world, rank, cfg=2)
        group = U.new_sp_groups(layout)
        hp = w.H // layout.sp
        me = layout.sp_rank(rank)
        shard = [torch.from_numpy(np.ascontiguousarray(t[bsl, s0:s1])) for t in (q, k, v)]
        k_heads = torch.from_numpy(np.ascontiguousarray(kp_out[bsl, :, me * hp:(me + 1) * hp]))

        def prologue(qh, kh, vh):
            qp, kp = O.prologue(qh.numpy(), kh.numpy(), **kw)
            return torch.from_numpy(qp), torch.from_numpy(kp), vh

        def attn(qh, kh, vh):
            o, _ = O.joint_attention(qh.numpy(), kh.numpy(), vh.numpy(), 0.25)
            return torch.from_numpy(o)

        o = bench.cfg_ulysses_step(*shard, k_heads, w.N, prologue, attn, group)
        out[rank] = (layout.cfg, layout.sp, bsl.start, bsl.stop, s0, s1, o.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_cfg_ulysses_step_matches_full_oracle(world):
    """cfg 2 x sp 1 (no exchange) and cfg 2 x sp 2 (all-to-all): every rank's
    rows equal the single-problem oracle result, each (b, t) row from
    exactly one rank."""
    import numpy as np
    w = _cfg_case()
    _, _, full, _, _ = _cfg_oracle(w)
    port = 29500 + (os.getpid() * 13 + world * 7) % 1500
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_cfg_worker, args=(world, port, out), nprocs=world, join=True)
        covered = np.zeros(full.shape[:2], dtype=int)
        for r in range(world):
            cfg, sp, b0, b1, s0, s1, o = out[r]
            assert (cfg, sp) == (2, world // 2)
            np.testing.assert_array_equal(o, full[b0:b1, s0:s1])
            covered[b0:b1, s0:s1] += 1
        assert (covered == 1).all()


def test_cfg_ulysses_plan_layouts():
    sys.path.insert(0, ROOT)
    import bench
    from diffusion_transformer_joint_dit_b200 import inputs as I
    w = I.WORKLOADS["t2i_2048"]
    for world, sp in ((2, 1), (4, 2), (8, 4)):
        seen = set()
        for r in range(world):
            lay, bsl, (s0, s1) = bench.cfg_ulysses_plan(w, world, r, cfg=2)
            assert (lay.cfg, lay.sp) == (2, sp) and bsl.stop - bsl.start == 1
            seen.add((bsl.start, s0, s1))
        assert len(seen) == world
    # A world that the CFG degree does not divide falls back to sequence
    # parallelism over all ranks (both batch elements on every rank).
    lay, bsl, _ = bench.cfg_ulysses_plan(w, 3, 0, cfg=2)
    assert (lay.cfg, lay.sp) == (1, 3) and (bsl.start, bsl.stop) == (0, 2)


def test_default_multi_gpu_mode_is_cfg_ulysses():
    sys.path.insert(0, ROOT)
    import bench
    assert not bench.parse_args(["--gpus", "8"]).replicas
    assert bench.parse_args(["--gpus", "8", "--replicas"]).replicas
