"""Context-parallel split of decode attention: one process per GPU, each holding
a contiguous shard of every layer's keys.

Each rank decodes its shard (``kvq_decode_attn_shard``) and merges its own
chunks (``kvq_merge_lse``); the ranks then exchange their merged rows with one
all-gather and every rank merges the gathered parts (``kvq_merge_lse_parts``).
The log-sum-exp merge is the one the RX 9070 XT KV-streaming page applies
across pages ("Online Log-Sum-Exp prefill & pipelined prefetch"); splitting
the context over GPUs is this library's extension.  The exchange per rank is
rows x (head_dim + 1) fp32 values, about 1.6 MB for 16 layers of a 4-token
verify batch with 24 query heads at head_dim 256, against the 7 GB of keys
the ranks read between them.

This module holds the host side only: the shard ranges and the exchange.  The
arithmetic runs in the library's kernels (or, in the CPU tests, in whatever
merge function the caller passes).
"""
from __future__ import annotations

from typing import Callable


def shard_range(n_kv: int, world: int, rank: int, chunk: int, T: int = 1) -> tuple[int, int]:
    """Keys ``[key0, key0 + n_keys)`` of rank ``rank``: the ``ceil(n_kv / chunk)`` chunks
    of the context dealt out in contiguous, balanced runs (rank r takes chunks
    ``[r C / world, (r + 1) C / world)``), so that every shard boundary is a chunk
    boundary of the unsplit context.  Raises ValueError when a shard would hold no
    chunk or fewer than ``T`` keys (the decode of a shard needs ``T <= n_keys``)."""
    if world < 1 or not 0 <= rank < world or chunk < 1 or n_kv < 1:
        raise ValueError("bad shard arguments")
    C = -(-n_kv // chunk)
    if C < world:
        raise ValueError(f"{C} chunks cannot be split over {world} ranks")
    c0, c1 = rank * C // world, (rank + 1) * C // world
    key0, key1 = c0 * chunk, min(c1 * chunk, n_kv)
    if key1 - key0 < T:
        raise ValueError(f"shard {rank} holds {key1 - key0} keys < T={T}")
    return key0, key1 - key0


def gather_merge(out_r, lse_r, out, lse, merge_parts: Callable, group=None) -> None:
    """All-gather this rank's merged rows and merge them over the ranks, in place.

    out_r [rows, head_dim] and lse_r [rows] (fp32 tensors on this rank's device, the
    rank's shard merged over its chunks); out, lse: the results, same shapes.
    ``merge_parts(parts_out, parts_lse, out, lse)`` merges ``parts_out
    [world, rows, head_dim]`` / ``parts_lse [world, rows]`` (rank r's rows at part r)
    into out and lse.  Every rank takes the same collective steps."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    parts_out = torch.empty((world,) + tuple(out_r.shape), dtype=out_r.dtype, device=out_r.device)
    parts_lse = torch.empty((world,) + tuple(lse_r.shape), dtype=lse_r.dtype, device=lse_r.device)
    dist.all_gather(list(parts_out.unbind(0)), out_r.contiguous(), group=group)
    dist.all_gather(list(parts_lse.unbind(0)), lse_r.contiguous(), group=group)
    merge_parts(parts_out, parts_lse, out, lse)
