#!/usr/bin/env python
"""Joint text+image attention forward benchmark (B200, sm_100a).

One step = the whole hot path on one batch of synthetic input: the prologue
(RMSNorm + 2-D RoPE of Q and K) followed by the joint attention forward, on
the 2048^2 text-to-image workload with classifier-free guidance batched as
B=2 (24 heads of 128, 512 text tokens + a 128x128 latent grid = 16896 joint
tokens).  The metric is attention TFLOP/s with FLOPs = 4 * B * H * N^2 * d.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

The attention's K input carries the workload's outliers: the prologue's K'
with 1% of its (b, t, h) rows scaled by 8 (RMSNorm would erase an outlier in
raw K), built once before the timed region.

Under torchrun (N > 1) the ranks split one problem the way the tutorial's
multi-GPU section does: the two CFG branches (the batch) on separate rank
groups and Ulysses sequence parallelism inside a group, an all-to-all of Q,
K, V to head shards before the attention and one of O back after it, over
NCCL (strong scaling).  ``--replicas`` runs an independent full problem per
rank instead (weak scaling, no data-path collective).  The step time is the
max over ranks; rank 0 prints one JSON line.  ``--impl reference`` times the
float64 CPU oracle instead, on a bounded sample of the same workload, on
rank 0 only.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from diffusion_transformer_joint_dit_b200 import inputs as I  # noqa: E402

METRIC = "joint-attn fwd TFLOP/s & % tensor peak, 2048² T2I (16896 tok, 24×128)"
UNIT = "TFLOP/s"
WORKLOAD = "t2i_2048"
L2_BYTES = 126 * 2 ** 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "attn_bf16_traffic_t2i_2048.md")
KERNEL_SOURCES = ["attn_bf16.cu", "sm100_ptx.cuh", "softmax_sm100.cuh", "jattn_internal.h"]


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(I.WORKLOADS))
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU oracle baseline budget (rank 0, N=1)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-table", action="store_true",
                    help="time the float64 oracle on all five workloads (minutes of host CPU) and exit")
    ap.add_argument("--no-fp8", action="store_true", help="skip the FP8-path timing object")
    ap.add_argument("--no-qkv", action="store_true", help="skip the fused-QKV-projection timing object")
    ap.add_argument("--no-sparse", action="store_true", help="skip the block-sparse attention timing object")
    ap.add_argument("--replicas", action="store_true",
                    help="with N > 1 ranks: an independent full problem per rank (weak scaling) instead of "
                         "the CFG x Ulysses split of one problem")
    ap.add_argument("--cfg", type=int, default=2,
                    help="CFG degree of the multi-GPU layout (ranks = cfg x sequence-parallel degree)")
    return ap.parse_args(argv)


def workload_config(w: I.Workload, extra=None):
    cfg = {
        "workload": (f"{w.name}: B={w.B} H={w.H} d={w.d} N_txt={w.n_txt} N_img={w.n_img} "
                     f"({w.img_h}x{w.img_w}) N_ref={w.n_ref} -> N={w.N} joint tokens"),
        "B": w.B, "H": w.H, "N": w.N, "d": w.d, "path": w.path,
        "step": "jattn_prologue (RMSNorm + 2-D RoPE of Q, K; bf16) + jattn_fwd_bf16",
        "l2": f"inputs larger than L2: Q, K, V {3 * w.B * w.N * w.H * w.d * 2 / 1e6:.0f} MB read per step",
        "parallelism": "independent batch per GPU (weak scaling, no collective)",
    }
    if extra:
        cfg.update(extra)
    return cfg


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "diffusion_transformer_joint_dit_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def profiled_traffic():
    """DRAM bytes per attention launch from the committed ncu summary, if it
    was taken on the current kernel source; else None.  The summary is a
    Markdown file whose key lines read `- key: value`."""
    try:
        with open(PROFILE_SUMMARY) as f:
            kv = {}
            for line in f:
                if line.startswith("- ") and ": " in line:
                    key, val = line[2:].split(": ", 1)
                    kv[key.strip()] = val.strip().strip("`")
    except OSError:
        return None
    if kv.get("source_sha256") != kernel_source_sha():
        return None
    try:
        return int(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, local_rank: int):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        idx = local_rank
        if vis:
            parts = [p.strip() for p in vis.split(",") if p.strip()]
            if local_rank < len(parts) and parts[local_rank].isdigit():
                idx = int(parts[local_rank])
        self.idx = idx
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.idx)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ oracle ----

def oracle_unit(w: I.Workload, q, k, v, b: int, h: int, rows):
    """Oracle prologue + attention for one (b, h) on sampled query rows."""
    import oracle as O
    qs = q[b:b + 1, :, h:h + 1, :].float().numpy()
    ks = k[b:b + 1, :, h:h + 1, :].float().numpy()
    vs = v[b:b + 1, :, h:h + 1, :].float().numpy()
    # The prologue runs on the whole (b, h) slice (every key needs K'); the
    # attention only on the sampled query rows.
    qp, kp = O.prologue(qs, ks, n_txt=w.n_txt, img_h=w.img_h, img_w=w.img_w, ref_h=w.ref_h, ref_w=w.ref_w,
                        ref_row_offset=w.ref_row_offset, theta=w.theta, eps=w.eps)
    O.joint_attention(O.bf16_round(qp), O.bf16_round(kp), vs, w.softmax_scale, rows=rows)
    return 4.0 * len(rows) * w.N * w.d


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [int(i.get("num_threads", 0)) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_baseline(w: I.Workload, q, k, v, seconds: float):
    rows_per_unit = 256
    rows = I.sampled_rows(w, rows_per_unit)
    units = [(b, h) for b in range(w.B) for h in range(w.H)]
    flops, done, t0 = 0.0, 0, time.perf_counter()
    while done < len(units) and (time.perf_counter() - t0) < seconds:
        b, h = units[done]
        flops += oracle_unit(w, q, k, v, b, h, rows)
        done += 1
    dt = time.perf_counter() - t0
    rate = flops / dt / 1e12
    return {"value": rate, "unit": UNIT, "cores": blas_threads(), "kind": "oracle", "cpu_model": cpu_model(),
            "cpu_count": os.cpu_count(),
            "sample": (f"float64 oracle (prologue of one (b,h) slice + attention of {rows_per_unit} sampled "
                       f"query rows vs all {w.N} keys) on {done} of {len(units)} (b,h) pairs, {dt:.1f} s"),
            "full_step_s_extrapolated": w.flops / (rate * 1e12),
            "seconds": dt}


def cpu_model() -> str:
    """The host CPU's model name (lscpu, else /proc/cpuinfo)."""
    try:
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        for line in out.splitlines():
            if line.startswith("Model name:"):
                return line.split(":", 1)[1].strip()
    except (OSError, subprocess.SubprocessError):
        pass
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


CPU_TABLE_CONFIGS = ("tiny", "t2i_1024", "t2i_2048", "i2i_2048", "t2i_2048_fp8")


def cpu_baseline_table(rows_sampled: int = 256):
    """The float64 oracle on every workload, on the host cores: tiny and
    t2i_1024 in full; the 2048^2 workloads on ``rows_sampled`` sampled query
    rows per (b, h) against all keys, with the full-size time extrapolated
    (prologue time + attention time x N / rows).  Every (b, h) is run; the
    FP8 workload also quantises Q', K', V to E4M3 blocks and dequantises
    them before the attention.  One JSON object per workload."""
    import oracle as O
    out = []
    for name in CPU_TABLE_CONFIGS:
        w = I.WORKLOADS[name]
        q, k, v = I.make_qkv(w, seed=0)
        full = name in ("tiny", "t2i_1024")
        rows = None if full else I.sampled_rows(w, rows_sampled)
        n_rows = w.N if full else len(rows)
        t_pro = t_att = 0.0
        for b in range(w.B):
            for h in range(w.H):
                t0 = time.perf_counter()
                qs = q[b:b + 1, :, h:h + 1, :].float().numpy()
                ks = k[b:b + 1, :, h:h + 1, :].float().numpy()
                vs = v[b:b + 1, :, h:h + 1, :].float().numpy()
                qp, kp = O.prologue(qs, ks, n_txt=w.n_txt, img_h=w.img_h, img_w=w.img_w, ref_h=w.ref_h,
                                    ref_w=w.ref_w, ref_row_offset=w.ref_row_offset, theta=w.theta, eps=w.eps)
                qp, kp = O.bf16_round(qp), O.bf16_round(kp)
                if w.path == "fp8":
                    qp, kp, vs = (O.dequantize_e4m3(*O.block_quantize_e4m3(x)) for x in (qp, kp, vs))
                t1 = time.perf_counter()
                O.joint_attention(qp, kp, vs, w.softmax_scale, rows=rows)
                t2 = time.perf_counter()
                t_pro += t1 - t0
                t_att += t2 - t1
        flops_done = 4.0 * w.B * w.H * n_rows * w.N * w.d
        full_s = t_pro + t_att * (w.N / n_rows)
        out.append({
            "workload": name, "B": w.B, "H": w.H, "N": w.N, "path": w.path,
            "rows_per_head": n_rows, "sampled": not full,
            "measured_s": t_pro + t_att, "prologue_s": t_pro, "attention_s": t_att,
            "attention_gflops": flops_done / t_att / 1e9,
            "full_step_s": full_s, "full_step_extrapolated": not full,
            "flops_full": w.flops,
        })
    return {"cpu_model": cpu_model(), "cpu_count": os.cpu_count(), "blas_threads": blas_threads(),
            "kind": "oracle (float64 numpy)", "configs": out}


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return 0
    w = I.WORKLOADS[args.workload]
    q, k, v = I.make_qkv(w, seed=0)
    rows = I.sampled_rows(w, 256)
    units = [(b, h) for b in range(w.B) for h in range(w.H)]
    for i in range(args.warmup):
        b, h = units[i % len(units)]
        oracle_unit(w, q, k, v, b, h, rows)
    flops, t0 = 0.0, time.perf_counter()
    for i in range(args.steps):
        b, h = units[(args.warmup + i) % len(units)]
        flops += oracle_unit(w, q, k, v, b, h, rows)
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    sample = (f"each step: float64 oracle prologue of one (b,h) slice of {w.name} + attention of 256 "
              f"sampled query rows vs all {w.N} keys")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, {"sample": sample}),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# -------------------------------------------------------------------- ours ----

def time_fp8_path(J, dev, stream, rank: int, peaks, peaks_src, steps: int = 10):
    """FP8 path on its own workload (2048^2, no CFG): jattn_prologue in FP8
    mode (RMSNorm + RoPE + E4M3 block quantisation of Q, K, V) followed by
    jattn_fwd_fp8.  Reported beside the headline line, not instead of it."""
    w = I.WORKLOADS["t2i_2048_fp8"]
    q, k, v = (t.to(dev) for t in I.make_qkv(w, seed=rank))
    shape = (w.B, w.N, w.H, w.d)
    nblk = -(-w.N // J.JATTN_FP8_BLOCK)
    q8, k8, v8 = (torch.empty(shape, dtype=torch.uint8, device=dev) for _ in range(3))
    qs, ks, vs = (torch.empty((w.B, w.H, nblk), dtype=torch.float32, device=dev) for _ in range(3))
    o = torch.empty(shape, dtype=torch.bfloat16, device=dev)
    params = J.make_prologue_params(w.img_h, w.img_w, w.ref_h, w.ref_w, w.ref_row_offset, w.theta, w.eps)
    h = stream.cuda_stream

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        J.jattn_prologue(q, k, v, q8, k8, v8, qs, ks, vs, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d,
                         J.JATTN_PROLOGUE_FP8, params, h)
        if ev is not None:
            ev[1].record(stream)
        J.jattn_fwd_fp8(q8, k8, v8, qs, ks, vs, o, None, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d,
                        w.softmax_scale, h)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(3):
        step()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    torch.cuda.synchronize(dev)
    for e in evs:
        step(e)
    torch.cuda.synchronize(dev)
    if J.jattn_device_status(h) != J.JATTN_OK:
        raise RuntimeError("device error word set during FP8 timing")
    pro = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    att = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    # Repair budget rho = 0.005 on top of the FP8 attention: selection
    # (errors, top-m, exact rows) and the correction, timed separately.
    m = J.repair_count(w.N, 0.005)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    err = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    idx = torch.empty((w.B, w.H, m), dtype=torch.int32, device=dev)
    ksel = torch.empty((w.B, w.H, m, w.d), dtype=torch.bfloat16, device=dev)
    vsel = torch.empty_like(ksel)
    J.jattn_fwd_fp8(q8, k8, v8, qs, ks, vs, o, lse, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d, w.softmax_scale, h)

    def repair(e=None):
        if e is not None:
            e[0].record(stream)
        J.jattn_fp8_repair_select(k, v, k8, v8, ks, vs, params, m, err, idx, ksel, vsel, w.B, w.H, w.n_txt,
                                  w.n_img, w.n_ref, w.d, h)
        if e is not None:
            e[1].record(stream)
        J.jattn_fp8_repair_apply(q8, qs, k8, v8, ks, vs, idx, ksel, vsel, m, o, lse, w.B, w.H, w.n_txt, w.n_img,
                                 w.n_ref, w.d, w.softmax_scale, h)
        if e is not None:
            e[2].record(stream)

    # Warm-up: the first launches load the kernels (lazy module loading) and
    # set their attributes; each repair call updates o and lse in place, so
    # the timed calls see the same sizes and work as these.
    for _ in range(3):
        repair()
    rev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    torch.cuda.synchronize(dev)
    for e in rev:
        repair(e)
    torch.cuda.synchronize(dev)
    if J.jattn_device_status(h) != J.JATTN_OK:
        raise RuntimeError("device error word set during repair timing")
    sel_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in rev)
    app_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in rev)
    fp8_peak = 2.0 * peaks["bf16_tflops"]  # nominal dense fp8 : bf16 ratio 2
    achieved = w.flops / (att * 1e-3) / 1e12
    pro_bytes = w.B * w.N * w.H * w.d * (3 * 2 + 3 * 1) + 3 * w.B * w.H * nblk * 4
    return {
        "workload": f"{w.name}: B={w.B} H={w.H} N={w.N} d={w.d}, E4M3 Q/K/V with per-64-token scales",
        "steps": steps, "attention_ms": att, "prologue_ms": pro,
        "value": w.flops / ((att + pro) * 1e-3) / 1e12, "unit": UNIT,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": fp8_peak, "unit": "TFLOP/s",
                     "frac": achieved / fp8_peak,
                     "peak_source": f"{peaks_src} bf16_tflops x 2 (nominal dense fp8/bf16 ratio)",
                     "bf16_peak_frac": achieved / peaks["bf16_tflops"]},
        "prologue_roofline": {"bound": "hbm", "achieved": pro_bytes / (pro * 1e-3) / 1e9,
                              "peak": peaks["hbm_gbs"], "unit": "GB/s",
                              "frac": pro_bytes / (pro * 1e-3) / 1e9 / peaks["hbm_gbs"]},
        "repair": {"rho": 0.005, "tokens_per_head": m, "select_ms": sel_ms, "apply_ms": app_ms,
                   "note": "per-token K'/V quantisation error, top-m per head, exact rows, LSE correction"},
    }


def time_sparse_path(J, dev, stream, rank: int, peaks, peaks_src, dense_ms: float, steps: int = 10):
    """Block-sparse attention (Sol-Attention reading, tau = 1.0) on the
    t2i_2048 workload: jattn_prologue (BF16), jattn_sparse_select (pooled
    block scores, kept-block lists), jattn_fwd_bf16_sparse.  The work is the
    kept (query, key) pairs: 4 d per pair, counted from the lists.  Reported
    beside the headline line, not instead of it."""
    w = I.WORKLOADS["t2i_2048"]
    tau = 1.0
    q, k, v = (t.to(dev) for t in I.make_qkv(w, seed=rank))
    params = J.make_prologue_params(w.img_h, w.img_w, w.ref_h, w.ref_w, w.ref_row_offset, w.theta, w.eps)
    h = stream.cuda_stream
    J.jattn_prologue(q, k, None, q, k, None, None, None, None, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d,
                     J.JATTN_PROLOGUE_BF16, params, h)
    nqb, nkb = J.sparse_blocks(w.N)
    qbar = torch.empty((w.B, w.H, nqb, w.d), dtype=torch.float32, device=dev)
    kbar = torch.empty((w.B, w.H, nkb, w.d), dtype=torch.float32, device=dev)
    idx = torch.empty((w.B, w.H, nqb, nkb), dtype=torch.int32, device=dev)
    cnt = torch.empty((w.B, w.H, nqb), dtype=torch.int32, device=dev)
    o = torch.empty_like(q)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        J.jattn_sparse_select(q, k, qbar, kbar, None, idx, cnt, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d,
                              w.softmax_scale, tau, h)
        if ev is not None:
            ev[1].record(stream)
        J.jattn_fwd_bf16_sparse(q, k, v, o, None, idx, cnt, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d,
                                w.softmax_scale, h)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(3):
        step()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    torch.cuda.synchronize(dev)
    for e in evs:
        step(e)
    torch.cuda.synchronize(dev)
    if J.jattn_device_status(h) != J.JATTN_OK:
        raise RuntimeError("device error word set during sparse timing")
    sel = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    att = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    # Kept (query, key) pairs, from the lists (outside the timed region).
    ci, ii = cnt.cpu().numpy(), idx.cpu().numpy()
    qrows = np.minimum(w.N - np.arange(nqb) * J.JATTN_SPARSE_QBLOCK, J.JATTN_SPARSE_QBLOCK)
    kcols = np.minimum(w.N - np.arange(nkb) * J.JATTN_SPARSE_KBLOCK, J.JATTN_SPARSE_KBLOCK)
    pairs = 0
    for pos in np.ndindex(*ci.shape):
        pairs += int(qrows[pos[-1]]) * int(kcols[ii[pos][:ci[pos]]].sum())
    flops = 4.0 * pairs * w.d
    achieved = flops / (att * 1e-3) / 1e12
    return {
        "workload": f"t2i_2048 block-sparse: B={w.B} H={w.H} N={w.N} d={w.d}, tau={tau}, query blocks "
                    f"{J.JATTN_SPARSE_QBLOCK}, key blocks {J.JATTN_SPARSE_KBLOCK}",
        "steps": steps, "select_ms": sel, "attention_ms": att,
        "kept_fraction": pairs / (w.B * w.H * w.N * w.N), "flops_per_launch": flops,
        "value": achieved, "unit": UNIT,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops"], "peak_source": f"{peaks_src} bf16_tflops"},
        "speedup_vs_dense_attention": dense_ms / (sel + att),
        "note": "synthetic N(0,1) inputs after the prologue; kept fraction is data dependent",
    }


def time_qkv_fused(J, dev, stream, rank: int, peaks, peaks_src, steps: int = 10):
    """Fused QKV projection (RMSNorm + RoPE in the GEMM epilogue) on the
    t2i_2048 shapes: x [B, N, C = H d] -> Q, K, V [B, N, H, d], per-stream
    weights.  For context it also times the same projection unfused: torch's
    bf16 matmul (cuBLAS, one per stream) followed by jattn_prologue.
    Reported beside the headline line, not instead of it."""
    w = I.WORKLOADS["t2i_2048"]
    C = w.H * w.d
    x, (wt, wi), qn, kn = I.make_qkv_projection_inputs(w, C, seed=rank)
    x, wt, wi = x.to(dev), wt.to(dev), wi.to(dev)
    qn = tuple(t.to(dev) for t in qn)
    kn = tuple(t.to(dev) for t in kn)
    h = stream.cuda_stream
    rope = torch.empty((w.N, 64, 2), dtype=torch.float32, device=dev)
    params = J.make_prologue_params(w.img_h, w.img_w, w.ref_h, w.ref_w, w.ref_row_offset, w.theta, w.eps)
    J.jattn_rope_table(rope, w.n_txt, w.n_img, w.n_ref, params, h)
    shape = (w.B, w.N, w.H, w.d)
    q, k, v = (torch.empty(shape, dtype=torch.bfloat16, device=dev) for _ in range(3))
    wts = J.make_qkv_weights(wt, wi, qn, kn, w.eps)
    y = torch.empty((w.B, w.N, 3 * C), dtype=torch.bfloat16, device=dev)
    qu, ku = torch.empty(shape, dtype=torch.bfloat16, device=dev), torch.empty(shape, dtype=torch.bfloat16, device=dev)
    pparams = J.make_prologue_params(w.img_h, w.img_w, w.ref_h, w.ref_w, w.ref_row_offset, w.theta, w.eps,
                                     qn[1], kn[1])

    def fused():
        J.jattn_qkv_fused(x, wts, rope, q, k, v, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d, C, h)

    def unfused():
        torch.matmul(x[:, :w.n_txt], wt.T, out=y[:, :w.n_txt])
        torch.matmul(x[:, w.n_txt:], wi.T, out=y[:, w.n_txt:])
        yq = y[..., :C].unflatten(-1, (w.H, w.d))
        yk = y[..., C:2 * C].unflatten(-1, (w.H, w.d))
        qc, kc = yq.contiguous(), yk.contiguous()
        J.jattn_prologue(qc, kc, None, qu, ku, None, None, None, None, w.B, w.H, w.n_txt, w.n_img, w.n_ref,
                         w.d, J.JATTN_PROLOGUE_BF16, pparams, h)

    def timed(fn):
        with torch.cuda.stream(stream):
            for _ in range(3):
                fn()
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(steps)]
            torch.cuda.synchronize(dev)
            for a, b in evs:
                a.record(stream)
                fn()
                b.record(stream)
            torch.cuda.synchronize(dev)
        return statistics.mean(a.elapsed_time(b) for a, b in evs)

    ms = timed(fused)
    if J.jattn_device_status(h) != J.JATTN_OK:
        raise RuntimeError("device error word set during QKV timing")
    ms_unfused = timed(unfused)
    flops = 2.0 * w.B * w.N * C * 3 * C
    achieved = flops / (ms * 1e-3) / 1e12
    return {
        "workload": f"t2i_2048 QKV projection: x [{w.B}, {w.N}, {C}] bf16, per-stream W [{3 * C}, {C}], "
                    f"Q/K RMSNorm + 2-D RoPE fused",
        "steps": steps, "ms": ms, "value": achieved, "unit": UNIT,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops"], "peak_source": f"{peaks_src} bf16_tflops",
                     "flops_per_launch": flops},
        "unfused_ms": ms_unfused,
        "unfused_note": "torch bf16 matmul per stream (cuBLAS) + jattn_prologue on Q, K (context, not ours)",
        "gpu_launches_per_step": 1,
    }


def sm_count(dev) -> int:
    return torch.cuda.get_device_properties(dev).multi_processor_count


def attn_bf16_launches(B: int, H: int, N: int, sms: int) -> int:
    """Kernel launches of one jattn_fwd_bf16 call: one over the whole waves
    of 256-row work items (one CTA per SM), plus one for a last partial wave
    that fills at most half of the SMs, which runs split over KV halves."""
    n_qb, n_kv = -(-N // 256), -(-N // 128)
    items = n_qb * H * B
    rem = items % sms
    tail = rem if n_kv >= 2 and 2 * rem <= sms else 0
    return int(items - tail > 0) + int(tail > 0)


def mufu_roofline(w: I.Workload, att_ms: float, clocks, dev):
    """Secondary roofline of the attention kernel: one exp2 per score
    (B H N^2 per launch) against the SFU rate, 16 ex2 per clock per SM (a
    probe on this GPU measured 15.7), at the median SM clock sampled during
    the timed region (the maximum clock when no sample was taken)."""
    exps = float(w.B * w.H * w.N * w.N)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    mhz = (clocks or {}).get("sm_mhz") or (clocks or {}).get("sm_max_mhz") or 1965.0
    peak = 16.0 * sms * mhz * 1e6 / 1e9
    achieved = exps / (att_ms * 1e-3) / 1e9
    return {"bound": "mufu", "achieved": achieved, "peak": peak, "unit": "Gexp2/s", "frac": achieved / peak,
            "exp_per_launch": exps, "peak_source": f"16 ex2/clk/SM x {sms} SMs x {mhz:.0f} MHz"}


def max_over_ranks(values, device):
    """Element-wise max of per-rank timings over all ranks (identity at N=1)."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if torch.distributed.is_initialized() and torch.distributed.get_world_size() > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def weak_scaling_value(world: int, flops_per_rank: float, ms_per_step: float) -> float:
    """Whole-job TFLOP/s: every rank processes its own batch in the step time."""
    return world * flops_per_rank / (ms_per_step * 1e-3) / 1e12


def outlier_k(J, w, qd, kd, params, seed, stream):
    """The attention's K input of the stated workload: K' = the prologue of
    K, with the workload's outlier rows (1% of (b, t, h) rows on t2i_2048)
    scaled by the outlier gain.  RMSNorm would erase an outlier in raw K, so
    the scaling applies to K'.  Built once, outside the timed region."""
    qp, kp = torch.empty_like(qd), torch.empty_like(kd)
    J.jattn_prologue(qd, kd, None, qp, kp, None, None, None, None, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d,
                     J.JATTN_PROLOGUE_BF16, params, stream.cuda_stream)
    torch.cuda.synchronize(qd.device)
    if w.k_outlier_frac <= 0:
        return kp
    mask = I.outlier_rows(w, seed)
    return I.apply_outliers(kp.cpu(), mask, w.k_outlier_gain).to(qd.device)


def e2e_steps(steps: int) -> int:
    """Steps of the end-to-end leg: at least 10, at most 20."""
    return max(10, min(steps, 20))


def run_e2e(J, w, q, k, v, k_att, dev, params, steps):
    """The headline step with host buffers: each step copies Q, K, V from
    pinned host memory, runs the prologue and the attention (on the outlier
    K' `k_att`, resident like the weights of a layer) and reads O back."""
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    ins = [[torch.empty_like(qh, device=dev) for _ in range(3)] for _ in range(2)]
    mids = [torch.empty_like(qh, device=dev) for _ in range(2)]       # Q', K' (reused per step)
    outs = [torch.empty_like(qh, device=dev) for _ in range(2)]
    ohs = [torch.empty(qh.shape, dtype=qh.dtype, pin_memory=True) for _ in range(2)]
    h2d, comp, d2h = (torch.cuda.Stream(dev) for _ in range(3))
    h2d_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    d2h_done = [torch.cuda.Event() for _ in range(2)]
    Ke = e2e_steps(steps)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def issue_h2d(i):
        bi = i % 2
        with torch.cuda.stream(h2d):
            if i >= 2:
                h2d.wait_event(comp_done[bi])          # step i-2 finished reading this buffer
            for dst, src in zip(ins[bi], (qh, kh, vh)):
                dst.copy_(src, non_blocking=True)
            h2d_done[bi].record(h2d)

    torch.cuda.synchronize(dev)
    t0.record(h2d)
    issue_h2d(0)
    for i in range(Ke):
        bi = i % 2
        if i + 1 < Ke:
            issue_h2d(i + 1)
        with torch.cuda.stream(comp):
            comp.wait_event(h2d_done[bi])
            if i >= 2:
                comp.wait_event(d2h_done[bi])          # O buffer of step i-2 read back
            qd, kd, vd = ins[bi]
            qp, kp = mids
            J.jattn_prologue(qd, kd, None, qp, kp, None, None, None, None, w.B, w.H, w.n_txt, w.n_img,
                             w.n_ref, w.d, J.JATTN_PROLOGUE_BF16, params, comp)
            J.jattn_fwd_bf16(qp, k_att, vd, outs[bi], None, w.B, w.H, w.n_txt, w.n_img, w.n_ref, w.d,
                             w.softmax_scale, comp)
            comp_done[bi].record(comp)
        with torch.cuda.stream(d2h):
            d2h.wait_event(comp_done[bi])
            ohs[bi].copy_(outs[bi], non_blocking=True)
            d2h_done[bi].record(d2h)
    d2h.wait_event(d2h_done[(Ke - 1) % 2])
    t1.record(d2h)
    torch.cuda.synchronize(dev)
    return t0.elapsed_time(t1), Ke


def run_ours(args, rank: int, world: int, local_rank: int):
    """One full problem per rank: the headline at N = 1, and independent
    replicas (weak scaling, no data-path collective) with --replicas."""
    from diffusion_transformer_joint_dit_b200 import binding as J

    dist = world > 1
    torch.cuda.set_device(local_rank)
    if dist:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    w = I.WORKLOADS[args.workload]
    if w.path != "bf16":
        raise SystemExit("bench.py times the BF16 path")
    q, k, v = I.make_qkv(w, seed=rank)
    dev = torch.device("cuda", local_rank)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    qp, kp, o = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(qd)
    params = J.make_prologue_params(w.img_h, w.img_w, w.ref_h, w.ref_w, w.ref_row_offset, w.theta, w.eps)
    stream = torch.cuda.current_stream(dev)
    s_handle = stream.cuda_stream
    # The attention's K input carries the workload's outliers (see outlier_k);
    # plain K' (the prologue's output, no outliers) is timed beside it.
    k_att = outlier_k(J, w, qd, kd, params, rank, stream)

    def prologue():
        J.jattn_prologue(qd, kd, None, qp, kp, None, None, None, None, w.B, w.H, w.n_txt, w.n_img, w.n_ref,
                         w.d, J.JATTN_PROLOGUE_BF16, params, s_handle)

    def attention(kin=None):
        J.jattn_fwd_bf16(qp, k_att if kin is None else kin, vd, o, None, w.B, w.H, w.n_txt, w.n_img, w.n_ref,
                         w.d, w.softmax_scale, s_handle)

    for _ in range(max(args.warmup, 3)):
        prologue()
        attention()
    torch.cuda.synchronize(dev)
    if J.jattn_device_status(s_handle) != J.JATTN_OK:
        raise RuntimeError("device error word set during warm-up")

    # ---- device-timed region: inputs resident in HBM ----
    K = args.steps
    att_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    pro_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local_rank)
    if dist:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)  # let the sampler take its first reading
    e0.record(stream)
    for i in range(K):
        pro_ev[i][0].record(stream)
        prologue()
        pro_ev[i][1].record(stream)
        att_ev[i][0].record(stream)
        attention()
        att_ev[i][1].record(stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if dist:
        torch.distributed.barrier()
    elapsed = e0.elapsed_time(e1)
    att_ms = statistics.mean(a.elapsed_time(b) for a, b in att_ev)
    pro_ms = statistics.mean(a.elapsed_time(b) for a, b in pro_ev)
    att_med = statistics.median(a.elapsed_time(b) for a, b in att_ev)
    pro_med = statistics.median(a.elapsed_time(b) for a, b in pro_ev)
    if J.jattn_device_status(s_handle) != J.JATTN_OK:
        raise RuntimeError("device error word set during timed steps")
    # The same attention on plain K' (no outliers), for comparison.
    plain_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(min(K, 20))]
    for a, b in plain_ev:
        a.record(stream)
        attention(kp)
        b.record(stream)
    torch.cuda.synchronize(dev)
    att_plain = statistics.mean(a.elapsed_time(b) for a, b in plain_ev)

    # ---- end-to-end region: host buffers, copies inside the timed region ----
    # Every step copies its Q, K, V from pinned host memory and reads its O
    # back; the copies of neighbouring steps overlap the compute of this one
    # (an H2D stream, the compute stream and a D2H stream, with device inputs
    # and outputs double-buffered).  Timed from the first copy to the last.
    if dist:
        torch.distributed.barrier()
    e2e_elapsed, Ke = run_e2e(J, w, q, k, v, k_att, dev, params, K)
    elapsed, e2e_elapsed, att_ms, pro_ms, att_med, pro_med, att_plain = max_over_ranks(
        [elapsed, e2e_elapsed, att_ms, pro_ms, att_med, pro_med, att_plain], dev)
    if dist:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return 0

    ms_per_step = elapsed / K
    value = weak_scaling_value(world, w.flops, ms_per_step)
    e2e_value = weak_scaling_value(world, w.flops, e2e_elapsed / Ke)
    peaks, peaks_src = load_peaks()
    sustained = elapsed >= 1000.0
    peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    achieved = w.flops / (att_ms * 1e-3) / 1e12
    traffic = profiled_traffic()
    act_bytes = w.B * w.N * w.H * w.d * 2
    data = "synthetic (seeded N(0,1) bf16 Q, K, V"
    if w.k_outlier_frac > 0:
        data += (f"; the attention's K input is the prologue's K' with {w.k_outlier_frac:.0%} of (b, t, h) rows "
                 f"x{w.k_outlier_gain:g}")
    data += ")"
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": data,
        "config": workload_config(w, {"attention_ms": att_ms, "prologue_ms": pro_ms,
                                      "attention_ms_median": att_med, "prologue_ms_median": pro_med,
                                      "attention_ms_plain_k": att_plain,
                                      "attention_tflops_plain_k": w.flops / (att_plain * 1e-3) / 1e12,
                                      "prologue_gbs": 4 * act_bytes / (pro_ms * 1e-3) / 1e9,
                                      # time x median SM clock of the timed region: compares runs
                                      # taken in different power states
                                      "attention_mcycles_at_median_clock":
                                          att_ms * clocks["sm_mhz"] / 1e3 if (clocks or {}).get("sm_mhz")
                                          else None}),
        "roofline": {
            "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "traffic": traffic,
            "kernel": "attn_bf16_kernel", "flops_per_launch": w.flops,
            "data": "outlier K'" if w.k_outlier_frac > 0 else "plain",
            "peak_source": f"{peaks_src} {'bf16_tflops_sustained' if sustained else 'bf16_tflops'}"
                           f" ({'timed region >= 1 s' if sustained else 'timed region < 1 s'})",
            "algorithmic_bytes_per_launch": 4 * act_bytes,
        },
        "prologue_roofline": {
            "bound": "hbm", "achieved": 4 * act_bytes / (pro_ms * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": 4 * act_bytes / (pro_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
        },
        "mufu_roofline": mufu_roofline(w, att_ms, clocks, dev),
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": 3 * act_bytes,
                "d2h_bytes_per_step": act_bytes, "steps": Ke,
                "note": "copies of neighbouring steps overlap compute (H2D, compute, D2H streams)"},
        "gpu_launches": K * (1 + attn_bf16_launches(w.B, w.H, w.N, sm_count(dev))),
        "clocks": clocks,
    }
    if world > 1:
        line["config"]["parallelism"] = f"replicas: an independent {w.name} problem per GPU (no collective)"
    if not args.no_fp8:
        line["fp8_path"] = time_fp8_path(J, dev, stream, rank, peaks, peaks_src)
    if not args.no_qkv:
        line["qkv_fused"] = time_qkv_fused(J, dev, stream, rank, peaks, peaks_src)
    if not args.no_sparse:
        line["sparse_path"] = time_sparse_path(J, dev, stream, rank, peaks, peaks_src, att_ms)
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = {k_: v_ for k_, v_ in cpu_baseline(w, q, k, v, args.cpu_seconds).items()
                                if k_ != "seconds"}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------- CFG x Ulysses (N > 1) --

def cfg_ulysses_plan(w: I.Workload, world: int, rank: int, cfg: int):
    """This rank's share of one problem under the tutorial's multi-GPU
    layout: the CFG branches (the batch) split over ``cfg`` rank groups, and
    inside a group the joint sequence split over the ``world / cfg`` ranks
    (Ulysses).  Returns (layout, batch slice, sequence shard [s0, s1))."""
    from diffusion_transformer_joint_dit_b200 import ulysses as U

    if cfg < 1 or w.B % cfg != 0 or world % cfg != 0:
        cfg = 1
    layout = U.ParallelLayout.make(world, cfg)
    if w.H % layout.sp != 0:
        raise SystemExit(f"{w.H} heads do not split over {layout.sp} sequence ranks")
    per = w.B // layout.cfg
    c = layout.cfg_index(rank)
    s0, s1 = U.shard_bounds(w.N, layout.sp, layout.sp_rank(rank))
    return layout, slice(c * per, (c + 1) * per), (s0, s1)


def cfg_ulysses_step(q, k, v, k_att_heads, n_total, prologue, attn, group=None):
    """One step of a rank: exchange its sequence shard of Q, K, V to the head
    shard of the whole sequence, the prologue there (positions are global),
    attention with the head shard's K input ``k_att_heads`` (the prologue's
    K' carrying the workload's outliers), and O back to the sequence shard."""
    from diffusion_transformer_joint_dit_b200 import ulysses as U

    p = torch.distributed.get_world_size(group)
    if p == 1:  # the whole sequence is here: no exchange
        qp, _, vp = prologue(q, k, v)
        return attn(qp, k_att_heads, vp)
    sizes = U.shard_sizes(n_total, p)
    qh, kh, vh = (U.seq_to_heads(t, sizes, group) for t in (q, k, v))
    qp, _, vh = prologue(qh, kh, vh)
    return U.heads_to_seq(attn(qp, k_att_heads, vh), sizes, group)


def run_cfg_ulysses(args, rank: int, world: int, local_rank: int):
    """One problem split over all ranks (strong scaling): the CFG branches on
    separate rank groups (no exchange between them) and Ulysses sequence
    parallelism inside a group (one all-to-all before the attention, one
    after, over NCCL).  Every rank holds its shard of Q, K, V in HBM."""
    from diffusion_transformer_joint_dit_b200 import binding as J
    from diffusion_transformer_joint_dit_b200 import ulysses as U

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    group = None
    try:
        w = I.WORKLOADS[args.workload]
        if w.path != "bf16":
            raise SystemExit("bench.py times the BF16 path")
        layout, bsl, (s0, s1) = cfg_ulysses_plan(w, world, rank, args.cfg)
        group = U.new_sp_groups(layout)
        q, k, v = I.make_qkv(w, seed=0)
        qd, kd, vd = (t[bsl, s0:s1].contiguous().to(dev) for t in (q, k, v))
        nb = bsl.stop - bsl.start
        hp = w.H // layout.sp
        me = layout.sp_rank(rank)
        prologue, attn = U.jattn_bf16_ops(w.n_txt, w.n_img, w.n_ref, w.softmax_scale, w.img_h, w.img_w,
                                          w.ref_h, w.ref_w, w.ref_row_offset)
        # The head shard's attention K input: its K' with the workload's
        # outlier rows (the same (b, t, h) rows as on one GPU), built once.
        sizes = U.shard_sizes(w.N, layout.sp)
        qh, kh, vh = (U.seq_to_heads(t, sizes, group) for t in (qd, kd, vd))
        _, kph, _ = prologue(qh, kh, vh)
        if w.k_outlier_frac > 0:
            mask = I.outlier_rows(w, 0)[bsl, :, me * hp:(me + 1) * hp]
            kph = I.apply_outliers(kph.cpu(), mask.copy(), w.k_outlier_gain).to(dev)
        del qh, kh, vh

        def step():
            return cfg_ulysses_step(qd, kd, vd, kph, w.N, prologue, attn, group)

        for _ in range(max(args.warmup, 3)):
            step()
        torch.cuda.synchronize(dev)
        if J.jattn_device_status() != J.JATTN_OK:
            raise RuntimeError("device error word set during warm-up")
        K = args.steps
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        clocks = ClockSampler(local_rank)
        torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        clocks.start()
        time.sleep(0.3)
        e0.record()
        for _ in range(K):
            step()
        e1.record()
        torch.cuda.synchronize(dev)
        clk = clocks.stop()
        torch.distributed.barrier()
        if J.jattn_device_status() != J.JATTN_OK:
            raise RuntimeError("device error word set during the timed region")
        ms = max_over_ranks([e0.elapsed_time(e1) / K], dev)[0]
        if rank == 0:
            value = w.flops / (ms * 1e-3) / 1e12
            line = {
                "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
                "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True,
                "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded N(0,1) bf16 Q, K, V; the attention's K input is the prologue's K' "
                        f"with {w.k_outlier_frac:.0%} of (b, t, h) rows x{w.k_outlier_gain:g})",
                "config": workload_config(w, {
                    "parallelism": f"cfg{layout.cfg} x ulysses sp{layout.sp} (all-to-all over NCCL inside a "
                                   f"CFG group; no exchange between groups)",
                    "step": "all-to-all of Q, K, V to head shards + jattn_prologue + jattn_fwd_bf16 on "
                            f"H/{layout.sp} heads + all-to-all of O back",
                    "per_rank": f"batch {bsl.start}..{bsl.stop - 1}, tokens {s0}..{s1 - 1} of {w.N}",
                    "all_to_all_bytes_sent_per_rank_per_step":
                        4 * nb * (s1 - s0) * w.H * w.d * 2 * (layout.sp - 1) // layout.sp,
                    "l2": "inputs larger than L2"}),
                "gpu_launches": K * (1 + attn_bf16_launches(nb, hp, w.N, sm_count(dev))),
                "clocks": clk,
            }
            print(json.dumps(line), flush=True)
    finally:
        torch.distributed.destroy_process_group()
    return 0


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(args.gpus if args.gpus == 1 else 1)))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        raise SystemExit("--gpus N > 1 runs under torchrun (one process per GPU)")
    if args.cpu_table:
        if rank == 0:
            print(json.dumps(cpu_baseline_table()), flush=True)
        return 0
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if world > 1 and not args.replicas:
        return run_cfg_ulysses(args, rank, world, local_rank)
    return run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    sys.exit(main())
