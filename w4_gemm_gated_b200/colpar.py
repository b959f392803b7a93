"""Column-parallel sharding of one W4 + gated-EC layer over ranks (one GPU per
rank), with the one collective the layer needs: an all-gather of y.

The layer y = x W + g (x A) B splits over its output channels with no exchange
inside it.  (The gist.science technical summary quotes its multi-GPU results
under tensor parallelism, section 3.2; its own split, section 2.2 B, is over K
and must reduce the partial activations before the gate inside the GEMM
epilogue.  Splitting over N needs no such reduction.)  Rank p holds the
channels [n0, n1):

- W[:, n0:n1], quantised on the rank.  Round-to-nearest quantisation works
  per output channel (and per 128-row group along K), so the shard's codes and
  scales are exactly the full layer's for those channels;
- B[:, n0:n1], folded with those channels' scales like the full layer's;
- x, A, w_g and b_g replicated: every rank computes t = x A and the gate itself
  (M K (r + 1) multiply-adds, small beside M K N / world).

y[:, n0:n1] is then complete on the rank.  When the consumer needs whole rows,
`gather_columns` assembles them with one all-gather over the process group
(NCCL over NVLink on GPUs, gloo on CPU).
"""
from __future__ import annotations

import torch

from . import spear as S

ALIGN = 256  # channels: a tensor-core output tile, and 16 decode strips


def column_ranges(N: int, world: int, align: int = ALIGN) -> list[tuple[int, int]]:
    """Contiguous channel ranges [n0, n1), one per rank, each a multiple of
    `align` channels, their sizes differing by at most `align`."""
    if world < 1:
        raise ValueError("world must be >= 1")
    if N % align:
        raise ValueError(f"N={N} is not a multiple of {align}")
    units = N // align
    if units < world:
        raise ValueError(f"N={N} gives {units} blocks of {align} channels for {world} ranks")
    base, extra = divmod(units, world)
    out, n0 = [], 0
    for p in range(world):
        n = (base + (1 if p < extra else 0)) * align
        out.append((n0, n0 + n))
        n0 += n
    return out


def prepare_shard(W: torch.Tensor, group: int, A: torch.Tensor | None, B: torch.Tensor | None,
                  w_g: torch.Tensor | None, b_g: float, rank: int, world: int, gate_tau: float = 0.1,
                  align: int = ALIGN, stream=None) -> tuple[S.Layer, tuple[int, int]]:
    """Rank `rank`'s shard of the layer (W is K x N fp32 on this rank's device,
    B is r x N): its prepared layer and its channel range."""
    n0, n1 = column_ranges(W.shape[1], world, align)[rank]
    Wp = W[:, n0:n1].contiguous()
    Bp = B[:, n0:n1].contiguous() if B is not None else None
    return S.prepare_layer(Wp, group, A, Bp, w_g, b_g, gate_tau, stream), (n0, n1)


def assemble(parts: list[torch.Tensor], ranges: list[tuple[int, int]], N: int) -> torch.Tensor:
    """Whole rows [M, N] from the ranks' column blocks (parts[p] holds at least
    ranges[p]'s width of columns; extra padding columns are ignored)."""
    M = parts[0].shape[0]
    y = torch.empty((M, N), dtype=parts[0].dtype, device=parts[0].device)
    for (n0, n1), part in zip(ranges, parts):
        y[:, n0:n1] = part[:, : n1 - n0]
    return y


def gather_columns(y_part: torch.Tensor, N: int, group=None, align: int = ALIGN) -> torch.Tensor:
    """All-gather of the ranks' [M, n1 - n0] outputs into whole rows [M, N] on
    every rank.  Shards may differ in width by `align`; each is padded to the
    widest for the collective, which needs equal sizes."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    ranges = column_ranges(N, world, align)
    width = max(n1 - n0 for n0, n1 in ranges)
    M = y_part.shape[0]
    send = y_part
    if y_part.shape[1] != width:
        send = torch.zeros((M, width), dtype=y_part.dtype, device=y_part.device)
        send[:, : y_part.shape[1]] = y_part
    # the ranks' blocks stacked along rows (the layout both NCCL and gloo take)
    recv = torch.empty((world * M, width), dtype=y_part.dtype, device=y_part.device)
    dist.all_gather_into_tensor(recv, send.contiguous(), group=group)
    return assemble(list(recv.view(world, M, width).unbind(0)), ranges, N)
