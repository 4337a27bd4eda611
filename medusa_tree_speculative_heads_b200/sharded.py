"""Medusa heads over vocabulary shards, one per GPU.

Each rank holds rows [v0, v1) of every head's W_head and the full residual
block; medusa_heads_shard reduces its rows to one 72-byte partial (m, l,
top-8) per (sequence, head); the ranks all-gather the partials in rank order
(the only exchange: B*K*72 bytes per rank); medusa_heads_merge turns them
into the full-vocabulary top-8, probabilities and tree tokens.  This module
is plumbing only (slicing, buffers, the collective); all arithmetic runs in
the library's kernels."""
from __future__ import annotations

from typing import Dict, Optional, Tuple

import torch

from . import binding as _b
from .binding import Tree


def vocab_shard(V: int, world: int, rank: int) -> Tuple[int, int]:
    """Rows [v0, v1) of rank `rank`: contiguous, in rank order, sizes
    differing by at most one (the first V % world ranks take one more)."""
    if world < 1 or not 0 <= rank < world or V < world:
        raise ValueError(f"cannot split V={V} over {world} ranks (rank {rank})")
    base, extra = divmod(V, world)
    v0 = rank * base + min(rank, extra)
    return v0, v0 + base + (1 if rank < extra else 0)


def exchange_partials(local: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather of every rank's partials ([B, K, 72] uint8) into
    [world, B, K, 72], rank r's block at index r."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    out = [torch.empty_like(local) for _ in range(world)]
    dist.all_gather(out, local.contiguous(), group=group)
    return torch.stack(out)


class ShardedHeads:
    """This rank's share of the heads: W_head rows [v0, v1) of a V-row
    vocabulary.  ``__call__`` runs the shard, exchanges the partials over
    ``group`` (None: a single process, the partial set is just this rank's)
    and merges them."""

    def __init__(self, *, B: int, d: int, V: int, K: int, v0: int, v1: int, dtype: torch.dtype,
                 tree: Optional[Tree] = None, device=None):
        dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.B, self.d, self.V, self.K, self.v0, self.v1 = B, d, V, K, v0, v1
        self.dt = _b.dtype_code(dtype)
        self.tree = tree
        self.partial = torch.empty((B, K, _b.PARTIAL_BYTES), dtype=torch.uint8, device=dev)
        self.ws_n = _b.medusa_heads_shard_workspace_size(B, d, v1 - v0, K, self.dt)
        self.ws = torch.empty(max(self.ws_n, 16), dtype=torch.uint8, device=dev)
        self.topk_idx = torch.empty((B, K, _b.TOPK), dtype=torch.int32, device=dev)
        self.topk_prob = torch.empty((B, K, _b.TOPK), dtype=torch.float32, device=dev)
        self.node_tokens = torch.empty((B, tree.T), dtype=torch.int32, device=dev) if tree is not None else None
        self.node_q = torch.empty((B, tree.T), dtype=torch.float32, device=dev) if tree is not None else None
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)

    def shard(self, h, W_res, W_head_shard) -> torch.Tensor:
        _b.medusa_heads_shard(h, W_res, W_head_shard, self.B, self.d, self.v1 - self.v0, self.v0, self.K, self.dt,
                              self.partial, self.ws, self.ws_n, self.status)
        return self.partial

    def merge(self, partials: torch.Tensor, root_token=None) -> Dict[str, torch.Tensor]:
        _b.medusa_heads_merge(partials, partials.shape[0], self.B, self.K, self.V, self.tree, root_token,
                              self.topk_idx, self.topk_prob, self.node_tokens, self.node_q, self.status)
        out = {"topk_idx": self.topk_idx, "topk_prob": self.topk_prob, "status": self.status}
        if self.tree is not None:
            out["node_tokens"], out["node_q"] = self.node_tokens, self.node_q
        return out

    def __call__(self, h, W_res, W_head_shard, root_token=None, group=None) -> Dict[str, torch.Tensor]:
        local = self.shard(h, W_res, W_head_shard)
        import torch.distributed as dist
        parts = exchange_partials(local, group) if dist.is_initialized() else local[None]
        return self.merge(parts, root_token)
