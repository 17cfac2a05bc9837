"""Head-parallel sparse MLA: the 128 attention heads split across ranks, one process per GPU.

The layout of the "RoPE coefficients" page's MLA init excerpt: each rank keeps n_heads / world_size
query heads (n_local_heads) and the whole latent cache, and computes the attention of its heads
only. The selected positions must be the same on every rank; the Indexer.forward excerpt of
"Rotate first features" broadcasts them from rank 0. Here the indexer runs on one rank (`src`) and
its int32 indices go to the others with one broadcast of the process group (NCCL on GPUs, gloo on
CPU), after which every rank runs dsa_sparse_mla_heads on its own heads: no other data crosses
ranks, and each rank's output rows are its heads' rows of the full result.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

HEADS = 128


def head_shard(rank: int, world: int, heads: int = HEADS) -> slice:
    """The heads rank `rank` of `world` holds (contiguous blocks of heads / world)."""
    if world < 1 or heads % world:
        raise ValueError(f"{heads} heads do not split evenly over {world} ranks")
    n = heads // world
    return slice(rank * n, (rank + 1) * n)


def broadcast_indices(idx: torch.Tensor, src: int = 0, group=None) -> torch.Tensor:
    """Every rank ends with rank `src`'s selected positions (int32 [B, T, k], same shape on every
    rank; the receiving ranks' contents are overwritten in place)."""
    if idx.dtype != torch.int32 or not idx.is_contiguous():
        raise ValueError("idx must be a contiguous int32 tensor")
    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.broadcast(idx, src=src, group=group)
    return idx


def sparse_mla_head_parallel(q_local, kv, idx, src: int = 0, group=None, attend=None, **kw):
    """This rank's part of the head-parallel sparse MLA: broadcast the indices from `src`, then
    attend with this rank's query heads q_local [B, T, 128 / world, 576]. Returns this rank's
    (out [B, T, 128 / world, 512], lse). `attend` defaults to the library's dsa_sparse_mla_heads."""
    if attend is None:
        from . import dsa_sparse_mla_heads as attend
    broadcast_indices(idx, src=src, group=group)
    return attend(q_local, kv, idx, **kw)
