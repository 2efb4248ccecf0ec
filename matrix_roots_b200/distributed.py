"""Blocked Shampoo over several GPUs: each layer's factors, roots, grafting
state and update live on one rank, and one AllGather shares the updated
weights.

The layers are assigned greedily by the cost of their inverse roots: sorted
by that cost, largest first, each goes to the rank with the least work so far
("A Distributed Data-Parallel PyTorch Implementation of the Distributed
Shampoo Optimizer ...", abstract; "Shampoo" notes, "Spreading the
preconditioners across GPUs": assign each layer to one worker, balanced
greedily by size, compute only those layers' directions, gather with one
AllGather).  A rank runs the whole single-GPU step (``BlockedShampoo``) on
its own layers; the gather then moves the new weights of every layer from
its owner to all ranks over NCCL (NVLink / NVSwitch on one node).
"""
from __future__ import annotations

from typing import Callable, Sequence


def split_dim(d: int, block_size: int) -> list[int]:
    """Block sizes of one dimension: floor(d/B) blocks of B and the remainder."""
    if block_size <= 0 or d <= block_size:
        return [d]
    return [block_size] * (d // block_size) + ([d % block_size] if d % block_size else [])


def layer_cost(shape, block_size: int) -> float:
    """Inverse-root work of one layer: sum over its blocks of m_b^3 + n_b^3."""
    rows = split_dim(int(shape[0]), block_size)
    cols = split_dim(int(shape[1]), block_size)
    return float(sum(r ** 3 + c ** 3 for r in rows for c in cols))


def assign_layers(shapes: Sequence, block_size: int, world: int) -> list[int]:
    """Owner rank of every layer: largest cost first, each to the least-loaded
    rank (lowest rank on ties); the order among equal costs is the input order."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(shapes)), key=lambda i: (-layer_cost(shapes[i], block_size), i))
    load = [0.0] * world
    owner = [0] * len(shapes)
    for i in order:
        r = min(range(world), key=lambda k: (load[k], k))
        owner[i] = r
        load[r] += layer_cost(shapes[i], block_size)
    return owner


def local_config(cfg, mine: Sequence[int]):
    """The configuration of the per-rank optimizer over layers ``mine``:
    per-layer options (the one-sided layer indices) renumbered to the
    rank's own layer order; everything else unchanged."""
    import dataclasses
    one = set(getattr(cfg, "one_sided", ()) or ())
    if not one or not dataclasses.is_dataclass(cfg):
        return cfg
    return dataclasses.replace(cfg, one_sided=tuple(k for k, i in enumerate(mine) if i in one))


class DistributedShampoo:
    """One optimizer step over all layers on ``world`` ranks.

    ``local_step(W_local, G_local)`` updates the owned layers in place; by
    default it is a ``BlockedShampoo`` over those layers.  After it, one
    ``all_gather`` of a padded flat buffer per rank replicates every layer's
    new weights.
    """

    def __init__(self, shapes, cfg, group=None, device="cuda",
                 local_step: Callable | None = None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.shapes = [(int(m), int(n)) for m, n in shapes]
        self.owner = assign_layers(self.shapes, cfg.block_size, self.world)
        self.mine = [i for i, r in enumerate(self.owner) if r == self.rank]
        self.counts = [sum(self.shapes[i][0] * self.shapes[i][1] for i, r in enumerate(self.owner) if r == k)
                       for k in range(self.world)]
        if local_step is None and self.mine:
            from .optimizer import BlockedShampoo
            opt = BlockedShampoo([self.shapes[i] for i in self.mine], local_config(cfg, self.mine), device)
            local_step = opt.step
            self.local = opt
        self.local_step = local_step

    def step(self, W, G) -> None:
        """W <- the Shampoo update, for every layer on every rank, in place."""
        import torch
        if self.mine:
            self.local_step([W[i] for i in self.mine], [G[i] for i in self.mine])
        width = max(self.counts) if self.counts else 0
        if width == 0:
            return
        ref = W[0]
        buf = torch.zeros(width, dtype=ref.dtype, device=ref.device)
        if self.mine:
            flat = torch.cat([W[i].reshape(-1) for i in self.mine])
            buf[: flat.numel()] = flat
        parts = [torch.empty_like(buf) for _ in range(self.world)]
        self.dist.all_gather(parts, buf, group=self.group)
        for k in range(self.world):
            if k == self.rank:
                continue
            off = 0
            for i, r in enumerate(self.owner):
                if r != k:
                    continue
                n = self.shapes[i][0] * self.shapes[i][1]
                W[i].copy_(parts[k][off: off + n].view(self.shapes[i]))
                off += n
