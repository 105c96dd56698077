"""Sequence-sharded decode over the ranks of a torch.distributed group.

The "Tree Attention Decoding" gist (tree_attn_decode) gives every rank one
chunk of the keys (``k.chunk(world_size, dim=-2)[rank]``), lets it compute
its partial attention, and finishes with three all-reduces (MAX of the local
maxima, then SUMs of the renormalised denominators and numerators).  Here a
rank's partial is a normalised output and its log-sum-exp, packed by the
``td_decode_shard`` kernel; the ranks exchange them with ONE all-gather (NCCL
on GPUs) and each merges them with the ``td_merge_shards`` kernel.  This module
only sizes and moves buffers; every step of the arithmetic is in the kernels.
"""
from typing import List, Optional, Tuple

import torch
import torch.distributed as dist

from . import decode_shard, merge_shards, state_floats


def shard_bounds(n: int, world: int, mode: str = "torch_chunk") -> List[Tuple[int, int]]:
    """(key_offset, length) of each rank's chunk of n keys.

    "torch_chunk" follows the gist's k.chunk(world_size): chunks of
    ceil(n / world) keys, the last shorter, and ranks past the end empty;
    "balanced" gives rank r the keys [floor(r n / W), floor((r+1) n / W)).
    """
    if world < 1 or n < 0:
        raise ValueError("world >= 1 and n >= 0 required")
    out = []
    if mode == "torch_chunk":
        cs = -(-n // world)
        for r in range(world):
            a = min(r * cs, n)
            b = min(a + cs, n)
            out.append((a, b - a))
    elif mode == "balanced":
        for r in range(world):
            a, b = r * n // world, (r + 1) * n // world
            out.append((a, b - a))
    else:
        raise ValueError("mode must be 'torch_chunk' or 'balanced'")
    return out


def _all_gather(gathered: torch.Tensor, local: torch.Tensor, group) -> None:
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(gathered, local, group=group)
    else:
        dist.all_gather(list(gathered.unbind(0)), local, group=group)


def decode_sharded(q: torch.Tensor, k_shard: torch.Tensor, v_shard: torch.Tensor,
                   key_offset: int, n_total: int, *, group=None,
                   slopes: Optional[torch.Tensor] = None, n_split: int = 0, stream=None,
                   shard_fn=None, merge_fn=None):
    """Decode q [B,H,1,D] over sequences of n_total keys whose keys
    [key_offset, key_offset + N_shard) this rank holds in k_shard/v_shard
    [B,H,N_shard,D].  Every rank of `group` calls it with its own chunk and
    gets the full result (out [B,H,1,D], lse [B,H,1]).

    shard_fn / merge_fn default to the library's kernels (decode_shard,
    merge_shards); a test may pass stand-ins with the same signatures.
    """
    shard_fn = shard_fn or decode_shard
    merge_fn = merge_fn or merge_shards
    # one process without a process group: a single shard, nothing to exchange
    alone = group is None and not (dist.is_available() and dist.is_initialized())
    world = 1 if alone else dist.get_world_size(group)
    B, H, _, D = q.shape
    state = shard_fn(q, k_shard, v_shard, key_offset, n_total, slopes=slopes, n_split=n_split,
                     stream=stream)
    if state.numel() != state_floats(B, H, D):
        raise ValueError("shard state has the wrong size")
    if alone:
        gathered = state.view(1, -1)
    else:
        gathered = torch.empty((world, state.numel()), dtype=torch.float32, device=state.device)
        _all_gather(gathered, state, group)
    return merge_fn(gathered, B, H, D, stream=stream)
