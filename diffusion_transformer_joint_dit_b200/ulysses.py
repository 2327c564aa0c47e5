"""Sequence-parallel (Ulysses) and CFG-parallel joint attention across GPUs.

The multi-GPU scheme of the NVIDIA tutorial on accelerating FLUX 3 Image
Klein with TensorRT LLM VisualGen ("Multi-GPU inference" section): the two
classifier-free-guidance branches run on separate GPU groups (no exchange),
and inside a group the joint sequence is split across the P ranks.  Attention
needs every key for its queries, so one all-to-all turns the sequence shards
of Q, K and V ([B, N_r, H, d] per rank) into head shards of the whole
sequence ([B, N, H/P, d]); the prologue and the attention kernels then run
unchanged on H/P heads, and a second all-to-all returns O to sequence shards.

Only the exchange and the layout changes live here (torch.distributed over
NCCL on GPUs); the compute is the jattn library.  ``prologue`` and ``attn``
are injectable so that the host logic can be exercised on CPU ranks.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist


def shard_sizes(n: int, parts: int) -> List[int]:
    """Balanced split of ``n`` tokens over ``parts`` ranks (first ranks take
    the remainder), in rank order."""
    if parts < 1:
        raise ValueError("parts must be >= 1")
    base, extra = divmod(n, parts)
    return [base + (1 if r < extra else 0) for r in range(parts)]


def shard_bounds(n: int, parts: int, rank: int) -> Tuple[int, int]:
    """[start, end) of ``rank``'s sequence shard."""
    sizes = shard_sizes(n, parts)
    start = sum(sizes[:rank])
    return start, start + sizes[rank]


@dataclass(frozen=True)
class ParallelLayout:
    """Rank placement for CFG x Ulysses: ``world = cfg * sp`` ranks; rank r
    is CFG branch ``r // sp`` and sequence rank ``r % sp`` inside it."""

    world: int
    cfg: int
    sp: int

    @staticmethod
    def make(world: int, cfg: int) -> "ParallelLayout":
        if cfg < 1 or world % cfg != 0:
            raise ValueError(f"world size {world} is not a multiple of the CFG degree {cfg}")
        return ParallelLayout(world, cfg, world // cfg)

    def cfg_index(self, rank: int) -> int:
        return rank // self.sp

    def sp_rank(self, rank: int) -> int:
        return rank % self.sp

    def sp_group_ranks(self, cfg_index: int) -> List[int]:
        return list(range(cfg_index * self.sp, (cfg_index + 1) * self.sp))


def new_sp_groups(layout: ParallelLayout):
    """Create one process group per CFG branch (every rank must call this, in
    the same order) and return the calling rank's group."""
    mine = None
    me = dist.get_rank()
    for c in range(layout.cfg):
        g = dist.new_group(layout.sp_group_ranks(c))
        if layout.cfg_index(me) == c:
            mine = g
    return mine


def seq_to_heads(x: torch.Tensor, sizes: Sequence[int], group=None) -> torch.Tensor:
    """All-to-all from a sequence shard [B, N_r, H, d] to the whole sequence
    of this rank's head shard [B, N, H/P, d] (heads of rank p are
    [p H/P, (p+1) H/P); tokens are concatenated in rank order)."""
    p = dist.get_world_size(group)
    me = dist.get_rank(group)
    b, n_r, h, d = x.shape
    if h % p != 0:
        raise ValueError(f"{h} heads do not split over {p} ranks")
    if n_r != sizes[me]:
        raise ValueError(f"rank {me} holds {n_r} tokens, expected {sizes[me]}")
    hp = h // p
    send = x.reshape(b, n_r, p, hp, d).permute(2, 0, 1, 3, 4).contiguous()  # [P, B, N_r, H/P, d]
    recv = torch.empty(b * sum(sizes) * hp * d, dtype=x.dtype, device=x.device)
    dist.all_to_all_single(recv, send.reshape(-1),
                           output_split_sizes=[b * s * hp * d for s in sizes],
                           input_split_sizes=[b * n_r * hp * d] * p, group=group)
    chunks, off = [], 0
    for s in sizes:
        chunks.append(recv[off:off + b * s * hp * d].view(b, s, hp, d))
        off += b * s * hp * d
    return torch.cat(chunks, dim=1)


def heads_to_seq(y: torch.Tensor, sizes: Sequence[int], group=None) -> torch.Tensor:
    """Inverse of :func:`seq_to_heads`: [B, N, H/P, d] -> [B, N_r, H, d]."""
    p = dist.get_world_size(group)
    me = dist.get_rank(group)
    b, n, hp, d = y.shape
    if n != sum(sizes):
        raise ValueError(f"{n} tokens, shards sum to {sum(sizes)}")
    send = torch.cat([y[:, s0:s0 + s].reshape(-1) for s0, s in zip(_starts(sizes), sizes)])
    n_r = sizes[me]
    recv = torch.empty(p * b * n_r * hp * d, dtype=y.dtype, device=y.device)
    dist.all_to_all_single(recv, send, output_split_sizes=[b * n_r * hp * d] * p,
                           input_split_sizes=[b * s * hp * d for s in sizes], group=group)
    return recv.view(p, b, n_r, hp, d).permute(1, 2, 0, 3, 4).reshape(b, n_r, p * hp, d)


def _starts(sizes: Sequence[int]) -> List[int]:
    out, acc = [], 0
    for s in sizes:
        out.append(acc)
        acc += s
    return out


Prologue = Callable[[torch.Tensor, torch.Tensor, torch.Tensor], Tuple[torch.Tensor, torch.Tensor, torch.Tensor]]
Attention = Callable[[torch.Tensor, torch.Tensor, torch.Tensor], torch.Tensor]


def ulysses_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, n_total: int,
                      attn: Attention, prologue: Optional[Prologue] = None, group=None) -> torch.Tensor:
    """Joint attention of this rank's sequence shard.

    q, k, v: [B, N_r, H, d] rows [start_r, end_r) of the joint sequence, the
    shard :func:`shard_bounds` assigns to this rank of ``group``.
    ``prologue`` (if given) maps the head-sharded full-sequence Q, K, V to
    the attention inputs (RMSNorm and RoPE use global token positions, so it
    runs after the first exchange); ``attn`` maps them to O [B, N, H/P, d].
    Returns O for this rank's tokens and all heads, [B, N_r, H, d].
    """
    sizes = shard_sizes(n_total, dist.get_world_size(group))
    qh, kh, vh = (seq_to_heads(t, sizes, group) for t in (q, k, v))
    if prologue is not None:
        qh, kh, vh = prologue(qh, kh, vh)
    return heads_to_seq(attn(qh, kh, vh), sizes, group)


def jattn_bf16_ops(n_txt: int, n_img: int, n_ref: int, softmax_scale: float, img_h: int, img_w: int,
                   ref_h: int = 0, ref_w: int = 0, ref_row_offset: int = 0, ref_grids=None):
    """(prologue, attn) for :func:`ulysses_attention` on CUDA tensors, both
    through the jattn library (BF16 path).  ``ref_grids`` as for
    ``binding.make_prologue_params`` (several reference images)."""
    from . import binding as J

    params = J.make_prologue_params(img_h, img_w, ref_h, ref_w, ref_row_offset, ref_grids=ref_grids)

    def prologue(q, k, v):
        b, n, h, d = q.shape
        qo, ko = torch.empty_like(q), torch.empty_like(k)
        J.jattn_prologue(q, k, v, qo, ko, None, None, None, None, b, h, n_txt, n_img, n_ref, d,
                         J.JATTN_PROLOGUE_BF16, params)
        return qo, ko, v

    def attn(q, k, v):
        b, n, h, d = q.shape
        o = torch.empty_like(q)
        J.jattn_fwd_bf16(q, k, v, o, None, b, h, n_txt, n_img, n_ref, d, softmax_scale)
        return o

    return prologue, attn
