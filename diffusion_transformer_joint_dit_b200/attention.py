"""One-call joint attention on torch CUDA tensors.

The tutorial configures DiT attention with one of four settings ("Quantized
and sparse attention" section): VANILLA BF16 attention, FP8 Q/K/V attention,
VC-Attention FP8 with a repair budget rho, and Sol-Attention block sparsity
with a threshold tau.  :func:`joint_attention` runs the matching path of the
jattn library: the prologue (per-head Q/K RMSNorm and 2-D RoPE, plus E4M3
block quantisation on the FP8 paths) and the attention kernels, allocating
the intermediate and output buffers with torch.  Every step runs in the
library's CUDA kernels on the current stream; this module only allocates and
orders the calls.
"""

from __future__ import annotations

from dataclasses import dataclass

import torch

from . import binding as J

MODES = ("bf16", "fp8", "fp8_repair", "sparse")


@dataclass
class AttentionConfig:
    """Which path to run.  ``mode``: "bf16" (VANILLA BF16), "fp8" (FP8 Q/K/V),
    "fp8_repair" (FP8 with the repair budget ``rho``), "sparse" (block-sparse
    BF16 with threshold ``tau``)."""
    mode: str = "bf16"
    rho: float = 0.005
    tau: float = 1.0
    eps: float = 1e-6
    rope_theta: float = 10000.0


def joint_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, n_txt: int, img_h: int, img_w: int,
                    ref_h: int = 0, ref_w: int = 0, ref_row_offset: int = 0, ref_grids=None,
                    config: AttentionConfig | None = None, softmax_scale: float | None = None,
                    q_norm_w: torch.Tensor | None = None, k_norm_w: torch.Tensor | None = None,
                    return_lse: bool = False):
    """Attention of the raw (pre-norm) Q, K, V of one DiT block.

    q, k, v: bf16 CUDA tensors ``[B, N, H, 128]`` holding the streams
    [text | image | references] in that order; N = n_txt + img_h img_w +
    the reference tokens.  Returns O (bf16, same shape) and, with
    ``return_lse``, the fp32 log-sum-exp ``[B, H, N]`` of each query row.
    The inputs are left unchanged.
    """
    cfg = config or AttentionConfig()
    if cfg.mode not in MODES:
        raise ValueError(f"mode must be one of {MODES}")
    q, k, v = _checked_inputs(q, k, v)
    q_norm_w, k_norm_w = (_checked_weight(w_, q) for w_ in (q_norm_w, k_norm_w))
    with torch.cuda.device(q.device):
        return _joint_attention(q, k, v, n_txt, img_h, img_w, ref_h, ref_w, ref_row_offset, ref_grids, cfg,
                                softmax_scale, q_norm_w, k_norm_w, return_lse)


def _checked_inputs(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor):
    """q, k, v as the library needs them: bf16 CUDA tensors of one shape
    [B, N, H, d] on one device, contiguous (a strided view, e.g. from
    qkv.unbind(2), is copied)."""
    ts = (q, k, v)
    if any(not isinstance(t, torch.Tensor) for t in ts):
        raise TypeError("q, k, v must be torch tensors")
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError(f"q, k, v must share one [B, N, H, d] shape, got {tuple(q.shape)}, {tuple(k.shape)}, "
                         f"{tuple(v.shape)}")
    if any(t.dtype != torch.bfloat16 for t in ts):
        raise ValueError("q, k, v must be bf16")
    if any(not t.is_cuda for t in ts) or k.device != q.device or v.device != q.device:
        raise ValueError("q, k, v must be CUDA tensors on one device")
    return tuple(t.contiguous() for t in ts)


def _checked_weight(w_, q: torch.Tensor):
    if w_ is None:
        return None
    if w_.dtype != torch.float32 or w_.shape != (q.shape[-1],) or w_.device != q.device:
        raise ValueError("norm weights must be fp32 [d] tensors on q's device")
    return w_.contiguous()


def _joint_attention(q, k, v, n_txt, img_h, img_w, ref_h, ref_w, ref_row_offset, ref_grids, cfg, softmax_scale,
                     q_norm_w, k_norm_w, return_lse):
    B, N, H, d = q.shape
    n_img = img_h * img_w
    n_ref = N - n_txt - n_img
    scale = softmax_scale if softmax_scale is not None else float(d) ** -0.5
    p = J.make_prologue_params(img_h, img_w, ref_h, ref_w, ref_row_offset, cfg.rope_theta, cfg.eps,
                               q_norm_w, k_norm_w, ref_grids=ref_grids)
    dev = q.device
    o = torch.empty_like(q)
    want_lse = return_lse or cfg.mode == "fp8_repair"
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev) if want_lse else None

    if cfg.mode in ("bf16", "sparse"):
        qp, kp = torch.empty_like(q), torch.empty_like(k)
        J.jattn_prologue(q, k, None, qp, kp, None, None, None, None, B, H, n_txt, n_img, n_ref, d,
                         J.JATTN_PROLOGUE_BF16, p)
        if cfg.mode == "bf16":
            J.jattn_fwd_bf16(qp, kp, v, o, lse, B, H, n_txt, n_img, n_ref, d, scale)
        else:
            nqb, nkb = J.sparse_blocks(N)
            qbar = torch.empty((B, H, nqb, d), dtype=torch.float32, device=dev)
            kbar = torch.empty((B, H, nkb, d), dtype=torch.float32, device=dev)
            idx = torch.empty((B, H, nqb, nkb), dtype=torch.int32, device=dev)
            cnt = torch.empty((B, H, nqb), dtype=torch.int32, device=dev)
            J.jattn_sparse_select(qp, kp, qbar, kbar, None, idx, cnt, B, H, n_txt, n_img, n_ref, d, scale, cfg.tau)
            J.jattn_fwd_bf16_sparse(qp, kp, v, o, lse, idx, cnt, B, H, n_txt, n_img, n_ref, d, scale)
    else:
        nblk = -(-N // J.JATTN_FP8_BLOCK)
        q8, k8, v8 = (torch.empty((B, N, H, d), dtype=torch.uint8, device=dev) for _ in range(3))
        qs, ks, vs = (torch.empty((B, H, nblk), dtype=torch.float32, device=dev) for _ in range(3))
        J.jattn_prologue(q, k, v, q8, k8, v8, qs, ks, vs, B, H, n_txt, n_img, n_ref, d, J.JATTN_PROLOGUE_FP8, p)
        J.jattn_fwd_fp8(q8, k8, v8, qs, ks, vs, o, lse, B, H, n_txt, n_img, n_ref, d, scale)
        if cfg.mode == "fp8_repair":
            m = J.repair_count(N, cfg.rho)
            if m > 0:
                err = torch.empty((B, H, N), dtype=torch.float32, device=dev)
                idx = torch.empty((B, H, m), dtype=torch.int32, device=dev)
                ksel = torch.empty((B, H, m, d), dtype=torch.bfloat16, device=dev)
                vsel = torch.empty_like(ksel)
                J.jattn_fp8_repair_select(k, v, k8, v8, ks, vs, p, m, err, idx, ksel, vsel, B, H, n_txt, n_img,
                                          n_ref, d)
                J.jattn_fp8_repair_apply(q8, qs, k8, v8, ks, vs, idx, ksel, vsel, m, o, lse, B, H, n_txt, n_img,
                                         n_ref, d, scale)
    return (o, lse) if return_lse else o
