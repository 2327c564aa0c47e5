"""Write ``tiny_oracle.json``: oracle values for the tiny workload.

Calls only ``oracle/`` (plus the seeded input generator).  The pages print no
worked numeric example for this method, so the stored values are a
regression pin of the oracle itself (``tests/test_golden.py`` re-derives
them) and a cheap expected-value table for smoke checks.

Run from the repository root:  python tests/golden/make_golden.py
"""

import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle as O  # noqa: E402
from diffusion_transformer_joint_dit_b200 import inputs as I  # noqa: E402

# (token, head, channel) probes: first/last text token, first image token,
# a mid-grid image token, last token; both RoPE halves.
PROBES = [(0, 0, 0), (31, 1, 5), (32, 0, 64), (32 + 17, 1, 33), (32 + 137, 0, 127),
          (287, 1, 70), (287, 0, 1)]


def build():
    w = I.WORKLOADS["tiny"]
    q, k, v = I.make_qkv(w, seed=0)
    qd, kd, vd = (t.double().numpy() for t in (q, k, v))
    qp, kp = O.prologue(qd, kd, n_txt=w.n_txt, img_h=w.img_h, img_w=w.img_w,
                        theta=w.theta, eps=w.eps)
    qb, kb = O.bf16_round(qp), O.bf16_round(kp)
    out, lse = O.joint_attention(qb, kb, vd, w.softmax_scale)
    codes, scales = O.block_quantize_e4m3(qb)
    return {
        "workload": "tiny (B=1, H=2, d=128, N_txt=32, 16x16 grid, seed 0)",
        "softmax_scale": w.softmax_scale,
        "probes": [
            {"t": t, "h": h, "c": c,
             "q_prime": float(qp[0, t, h, c]), "k_prime": float(kp[0, t, h, c]),
             "o": float(out[0, t, h, c]), "lse": float(lse[0, h, t]),
             "q_code": int(codes[0, t, h, c])}
            for (t, h, c) in PROBES
        ],
        "q_scales": [[float(s) for s in row] for row in scales[0]],
        "o_sum": float(out.sum()),
        "o_sq_sum": float((out * out).sum()),
    }


if __name__ == "__main__":
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.json")
    with open(path, "w") as f:
        json.dump(build(), f, indent=1)
    print("wrote", path)
