"""The zone indicator with the heads spread over several GPUs.

Every stage after the indicator works head by head, so a layer whose heads
are split over G ranks needs one exchange only: the indicator's video
statistics are sums over all heads' channels (Portuguese reading guide,
"Método" 1: the channel average over D; one block shape per zone serves every
head).  Each rank sums over its own channels (``prism_zone_partials``), one
all-reduce adds the [Z, 4] sums over the ranks, and each rank finishes the
indicator alone (``prism_zone_finalize``).  The audio statistics come from
hhat, which every rank holds whole.

One process per GPU; the process group is NCCL's in a real run (the reduced
tensor lives on the GPU) and gloo in the CPU tests of the exchange.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import _abi


def reduce_zone_partials(partials: torch.Tensor, n_zones: int, group=None) -> torch.Tensor:
    """Sum the video half of ``partials`` ([2, Z, 4] float32) over the ranks of
    ``group``, in place; the audio half is the same on every rank."""
    video = partials.view(-1)[: n_zones * 4]
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(video, op=dist.ReduceOp.SUM, group=group)
    return partials


def head_slice(heads: int, rank: int, world: int) -> slice:
    """The heads rank `rank` of `world` holds: contiguous, as even as possible."""
    base, extra = divmod(heads, world)
    start = rank * base + min(rank, extra)
    return slice(start, start + base + (1 if rank < extra else 0))


class ShardedZoneIndicator:
    """Stage 1 of one layer whose heads ``head_slice(heads, rank, world)`` live on
    this rank: ``__call__(V_local, hhat)`` returns g [Z, 3], rho [Z], abar [Z] and
    the zone statistics [Z, 8], the same on every rank."""

    def __init__(self, T, H, W, heads, head_dim, audio_dim=64, dtype="bf16", eps=1e-6, guidance="joint",
                 group=None, device="cuda"):
        world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
        rank = dist.get_rank(group) if world > 1 else 0
        self.group = group
        self.heads = head_slice(heads, rank, world)
        n_local = self.heads.stop - self.heads.start
        if n_local < 1:
            raise ValueError(f"{heads} heads cannot be spread over {world} ranks")
        self.prob = _abi.problem(T, H, W, heads, head_dim, audio_dim, dtype)
        self.prob_local = _abi.problem(T, H, W, n_local, head_dim, audio_dim, dtype)
        self.eps, self.guidance = float(eps), guidance
        sz = _abi.query_sizes(self.prob_local)
        self.Z = int(sz.n_zones)
        dev = torch.device(device)
        self.ws = torch.empty(max(int(sz.ws_indicator), self.Z * 16), dtype=torch.uint8, device=dev)
        self.partials = torch.empty((2, self.Z, 4), dtype=torch.float32, device=dev)
        self.g = torch.empty((self.Z, 3), dtype=torch.float32, device=dev)
        self.rho = torch.empty(self.Z, dtype=torch.float32, device=dev)
        self.abar = torch.empty(self.Z, dtype=torch.float32, device=dev)
        self.zone_stats = torch.empty((self.Z, 8), dtype=torch.float32, device=dev)

    def __call__(self, V_local, hhat):
        """On the current CUDA stream, which the all-reduce also follows."""
        _abi.prism_zone_partials(self.prob_local, V_local, hhat, self.partials, self.ws)
        reduce_zone_partials(self.partials, self.Z, self.group)
        _abi.prism_zone_finalize(self.prob, self.partials, self.eps, self.guidance, self.g, self.rho, self.abar,
                                 self.zone_stats, self.ws)
        return self.g, self.rho, self.abar, self.zone_stats
