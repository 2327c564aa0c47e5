"""Seeded synthetic inputs for the joint-attention workloads.

This module is shared by the tests, the benchmark and the oracle checks, and
holds none of the method's arithmetic: it only draws random numbers and casts
them to the storage dtype (bf16 via torch's round-to-nearest-even cast).

The five workloads are the shapes of a FLUX-3-Klein-style DiT block at the
resolutions the tutorial measures (1024^2 and 2048^2 text-to-image with
classifier-free guidance batched as B=2, 2048^2 image-to-image with one
reference image, and a 2048^2 no-guidance FP8 run).  The pages give no head
count, head size, text length or latent grid; the sizes below are the
stated workload definitions: 24 heads of 128, 512 text tokens, latent grid =
image side / 16.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    n_txt: int
    img_h: int
    img_w: int
    ref_h: int = 0
    ref_w: int = 0
    ref_row_offset: int = 0
    ref_grids: tuple = ()         # several references: ((h, w, row_offset, col_offset), ...)
    d: int = 128
    path: str = "bf16"            # "bf16" or "fp8"
    k_outlier_frac: float = 0.0   # fraction of K' rows scaled by k_outlier_gain
    k_outlier_gain: float = 8.0
    gain_sigma: float = 0.0       # per-channel LogNormal(0, sigma) gains (fp8 workload)
    theta: float = 10000.0
    eps: float = 1e-6
    sampled_rows: int = 0         # 0 = oracle checks every query row
    notes: str = field(default="", compare=False)

    @property
    def n_img(self) -> int:
        return self.img_h * self.img_w

    @property
    def n_ref(self) -> int:
        if self.ref_grids:
            return sum(h * w for h, w, _, _ in self.ref_grids)
        return self.ref_h * self.ref_w

    @property
    def N(self) -> int:
        return self.n_txt + self.n_img + self.n_ref

    @property
    def softmax_scale(self) -> float:
        return float(np.float32(1.0 / np.sqrt(self.d)))

    @property
    def flops(self) -> float:
        """Attention forward FLOPs: 4 * B * H * N^2 * d (QK^T plus PV)."""
        return 4.0 * self.B * self.H * self.N * self.N * self.d


WORKLOADS = {
    "tiny": Workload("tiny", B=1, H=2, n_txt=32, img_h=16, img_w=16),
    "t2i_1024": Workload("t2i_1024", B=2, H=24, n_txt=512, img_h=64, img_w=64),
    "t2i_2048": Workload("t2i_2048", B=2, H=24, n_txt=512, img_h=128, img_w=128,
                         k_outlier_frac=0.01, sampled_rows=256),
    "i2i_2048": Workload("i2i_2048", B=2, H=24, n_txt=512, img_h=128, img_w=128,
                         ref_h=128, ref_w=128, ref_row_offset=128, sampled_rows=256),
    "t2i_2048_fp8": Workload("t2i_2048_fp8", B=1, H=24, n_txt=512, img_h=128, img_w=128,
                             path="fp8", gain_sigma=0.5, sampled_rows=256),
}


def custom(name: str = "custom", **kw) -> Workload:
    """A workload with explicit sizes (edge-case tests)."""
    return Workload(name, **kw)


def _to_bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def make_qkv(w: Workload, seed: int = 0):
    """Q, K, V as bf16 CPU tensors ``[B, N, H, d]``.

    Draw order with ``numpy.random.default_rng(seed)``: Q, K, V standard
    normal (float32), then, for the FP8 workload, one gain vector of length d
    per tensor g = exp(N(0, sigma^2)) applied channel-wise before the cast.
    """
    rng = np.random.default_rng(seed)
    shape = (w.B, w.N, w.H, w.d)
    q = rng.standard_normal(shape, dtype=np.float32)
    k = rng.standard_normal(shape, dtype=np.float32)
    v = rng.standard_normal(shape, dtype=np.float32)
    if w.gain_sigma > 0:
        for t in (q, k, v):
            g = np.exp(rng.normal(0.0, w.gain_sigma, size=w.d)).astype(np.float32)
            t *= g
    return _to_bf16(q), _to_bf16(k), _to_bf16(v)


def outlier_rows(w: Workload, seed: int = 0) -> np.ndarray:
    """Boolean mask ``[B, N, H]`` of the K rows scaled by ``k_outlier_gain``.

    ``round(frac * B*N*H)`` rows drawn without replacement from
    ``default_rng(seed + 1)``.  Scaling a bf16 value by 8 is exact, so the
    scaled tensor is the same on every side that applies the mask.
    """
    mask = np.zeros((w.B, w.N, w.H), dtype=bool)
    if w.k_outlier_frac <= 0:
        return mask
    total = w.B * w.N * w.H
    n = int(round(w.k_outlier_frac * total))
    pick = np.random.default_rng(seed + 1).choice(total, size=n, replace=False)
    mask.reshape(-1)[pick] = True
    return mask


def apply_outliers(k: torch.Tensor, mask: np.ndarray, gain: float) -> torch.Tensor:
    """Return a copy of bf16 ``k`` with the masked rows multiplied by ``gain``."""
    out = k.clone()
    m = torch.from_numpy(mask)
    out[m] = out[m] * gain
    return out


def sampled_rows(w: Workload, count: int, seed: int = 0) -> np.ndarray:
    """Sorted query indices checked against the oracle on large workloads.

    Always includes the stream boundaries (first token, last text token,
    first and last image token, first reference token, last token); the
    rest are drawn without replacement from ``default_rng(seed + 2)``.  The
    same indices are used for every (b, h).
    """
    N = w.N
    fixed = {0, max(w.n_txt - 1, 0), min(w.n_txt, N - 1),
             min(w.n_txt + w.n_img - 1, N - 1), N - 1}
    if w.n_ref > 0:
        fixed.add(w.n_txt + w.n_img)
    fixed = sorted(fixed)
    if count >= N:
        return np.arange(N)
    rest = np.setdiff1d(np.arange(N), np.array(fixed))
    extra = np.random.default_rng(seed + 2).choice(rest, size=count - len(fixed), replace=False)
    return np.sort(np.concatenate([np.array(fixed), extra]))


def random_e4m3_codes(shape, seed: int = 0) -> np.ndarray:
    """Uniformly random finite E4M3 bytes (0x7F / 0xFF, the NaN codes, excluded)."""
    rng = np.random.default_rng(seed)
    c = rng.integers(0, 256, size=shape, dtype=np.int64)
    c = np.where((c & 0x7F) == 0x7F, c ^ 0x01, c)
    return c.astype(np.uint8)


def make_qkv_projection_inputs(w: Workload, C: int, seed: int = 0):
    """Inputs of the fused QKV projection as bf16 / fp32 CPU tensors.

    Draw order with ``numpy.random.default_rng(seed)``: activations
    x ``[B, N, C]`` standard normal; then per stream (text, image) the
    projection ``[3 H d, C]`` with entries N(0, 1/C), so projected features
    are about unit size; then per stream the Q and K norm weights
    ``[d]`` uniform in [0.5, 1.5).
    Returns ``x, (w_txt, w_img), (qn_txt, qn_img), (kn_txt, kn_img)``.
    """
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((w.B, w.N, C), dtype=np.float32)
    ws = [rng.standard_normal((3 * w.H * w.d, C), dtype=np.float32) / np.float32(np.sqrt(C)) for _ in range(2)]
    qn, kn = [], []
    for _ in range(2):
        qn.append(torch.from_numpy(rng.uniform(0.5, 1.5, w.d).astype(np.float32)))
        kn.append(torch.from_numpy(rng.uniform(0.5, 1.5, w.d).astype(np.float32)))
    return _to_bf16(x), (_to_bf16(ws[0]), _to_bf16(ws[1])), tuple(qn), tuple(kn)
