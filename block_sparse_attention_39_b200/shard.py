"""Head-sharded PBSA: each rank owns a contiguous range of a layer's heads.

Sparse Forcing keeps the persistent memory, the block scores and the
selections of PBSA per (batch, head) (gist.science/es, section 2
"Arquitectura Propuesta", item "Memoria Persistente"; section 2 PBSA, item
"Atención Híbrida"): no step of the hot path reads another head's data.  A layer's heads therefore split across GPUs with
no exchange inside the path; only the caller, whose output projection needs
every head, gathers O, with one all-gather over the ranks (NCCL over
NVLink / NVSwitch between GPUs, gloo on the host).

``head_range`` fixes the partition, ``gather_heads`` assembles the output in
head order, and ``ShardedLayer`` runs one rank's share of a layer through the
same ``PbsaLayer`` the single-GPU path uses.
"""
from __future__ import annotations

import copy
import dataclasses

import torch
import torch.distributed as dist

from .engine import PbsaLayer


def head_range(H: int, world: int, rank: int) -> tuple[int, int]:
    """Heads [h0, h1) of ``rank`` among ``world`` ranks: contiguous ranges in
    rank order; the first H % world ranks take one head more."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if H < world:
        raise ValueError(f"{H} heads cannot give each of {world} ranks one")
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def gather_heads(x_local: torch.Tensor, H: int, world: int, group=None) -> torch.Tensor:
    """The whole layer's [B, H, ...] from every rank's [B, h1 - h0, ...] share,
    in head order.  Shares may differ by one head: each is padded to the
    largest before the all-gather and trimmed after.  One collective; every
    rank calls it with its own share."""
    if world == 1:
        return x_local
    h_max = -(-H // world)
    B, h_loc = x_local.shape[0], x_local.shape[1]
    send = x_local.new_zeros((B, h_max) + tuple(x_local.shape[2:]))
    send[:, :h_loc] = x_local
    recv = [torch.empty_like(send) for _ in range(world)]
    dist.all_gather(recv, send, group=group)
    parts = []
    for r in range(world):
        h0, h1 = head_range(H, world, r)
        parts.append(recv[r][:, :h1 - h0])
    return torch.cat(parts, dim=1)


def _with_heads(cfg, H):
    if dataclasses.is_dataclass(cfg):
        return dataclasses.replace(cfg, H=H)
    c = copy.copy(cfg)
    c.H = H
    return c


class ShardedLayer:
    """One rank's share of a layer: a ``PbsaLayer`` over heads [h0, h1).

    ``step`` takes the chunk's Q, K and V for every head ([B, H, T_c, D], the
    same tensors on every rank), keeps this rank's heads, appends the K/V
    into the rank's pool, runs score -> update -> select -> attend on them,
    and returns the whole layer's O gathered over the ranks (or, with
    ``gather=False``, this rank's [B, h1 - h0, T_c, D] share)."""

    def __init__(self, cfg, world: int = 1, rank: int = 0, device="cuda", group=None):
        self.H = cfg.H
        self.world, self.rank, self.group = world, rank, group
        self.h0, self.h1 = head_range(cfg.H, world, rank)
        self.layer = PbsaLayer(_with_heads(cfg, self.h1 - self.h0), device=device)

    def step(self, t, q, k, v, fused=False, gather=True, stream=None):
        L, sl = self.layer, slice(self.h0, self.h1)
        L.q.copy_(q[:, sl])
        L.append(t, k[:, sl].contiguous(), v[:, sl].contiguous(), stream=stream)
        L.step(t, stream=stream, fused=fused, appended=True)
        if not gather:
            return L.o
        return gather_heads(L.o, self.H, self.world, self.group)
