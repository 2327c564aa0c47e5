"""Print the GPU path's error against the float64 oracle on each of the five
workloads (test infrastructure; run on a GPU machine:
``python -m tests.parity_report``).

BF16 workloads: jattn_fwd_bf16 on the oracle's own bf16 Q', K' (the
attention inputs of the workload: t2i_2048 with its outlier K' rows), all
query rows of tiny and t2i_1024, 256 sampled rows per (b, h) of the 2048^2
workloads.  FP8 workload: GPU FP8 prologue + jattn_fwd_fp8 against the
oracle run on the same E4M3 quantisation, and against the unquantised
oracle.  One JSON line per workload.
"""

from __future__ import annotations

import json

import numpy as np
import torch

import oracle as O
from diffusion_transformer_joint_dit_b200 import inputs as I
from tests.gpu_common import gpu_attn_bf16, gpu_prologue_fp8, oracle_prologue_bf16, rel_l2, to_np
from tests.test_gpu_attn_fp8 import _gpu_fwd_fp8, _oracle_quant


def bf16_case(name):
    w = I.WORKLOADS[name]
    q, k, v = I.make_qkv(w, seed=0)
    _, _, qb, kb = oracle_prologue_bf16(w, q, k)
    if w.k_outlier_frac > 0:
        kb = kb.copy()
        kb[I.outlier_rows(w, 0)] *= w.k_outlier_gain
    qt = torch.from_numpy(qb.astype(np.float32)).to(torch.bfloat16)
    kt = torch.from_numpy(kb.astype(np.float32)).to(torch.bfloat16)
    o, lse = gpu_attn_bf16(w, qt, kt, v)
    rows = None if w.N <= 4608 else I.sampled_rows(w, 256)
    ref, ref_lse = O.joint_attention(qb, kb, to_np(v), w.softmax_scale, rows=rows)
    got, gl = to_np(o), to_np(lse)
    if rows is not None:
        got, gl = got[:, rows], gl[:, :, rows]
    return {"workload": name, "rows_per_head": len(rows) if rows is not None else w.N,
            "rel_l2": rel_l2(got, ref), "max_abs": float(np.max(np.abs(got - ref))),
            "lse_max_abs": float(np.max(np.abs(gl - ref_lse)))}


def fp8_case(name="t2i_2048_fp8"):
    w = I.WORKLOADS[name]
    q, k, v = I.make_qkv(w, seed=0)
    codes_g, scales_g = gpu_prologue_fp8(w, q, k, v)
    o, lse = _gpu_fwd_fp8(w, codes_g, scales_g)
    qkv8, unq = _oracle_quant(w, q, k, v)
    codes, scales = zip(*qkv8)
    rows = I.sampled_rows(w, 256)
    deq = [O.dequantize_e4m3(c, s) for c, s in zip(codes, scales)]
    ref, ref_lse = O.joint_attention(deq[0], deq[1], deq[2], w.softmax_scale, rows=rows)
    ref_u, _ = O.joint_attention(*unq, w.softmax_scale, rows=rows)
    got, gl = to_np(o)[:, rows], to_np(lse)[:, :, rows]
    return {"workload": name, "rows_per_head": len(rows), "rel_l2": rel_l2(got, ref),
            "max_abs": float(np.max(np.abs(got - ref))), "lse_max_abs": float(np.max(np.abs(gl - ref_lse))),
            "rel_l2_vs_unquantised": rel_l2(got, ref_u)}


def main():
    torch.cuda.set_device(0)
    for name in ("tiny", "t2i_1024", "t2i_2048", "i2i_2048"):
        print(json.dumps(bf16_case(name)), flush=True)
    print(json.dumps(fp8_case()), flush=True)


if __name__ == "__main__":
    main()
