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

from . import decode_shard, decode_varlen, merge_shards, state_floats


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


def ragged_shard(lengths, world: int, rank: int, mode: str = "balanced"):
    """This rank's chunk of every sequence of a ragged batch: (offsets,
    lengths), one pair per sequence, from shard_bounds of each length."""
    offs, lens = [], []
    for n in lengths:
        a, ln = shard_bounds(int(n), world, mode)[rank]
        offs.append(a)
        lens.append(ln)
    return offs, lens


def pack_ragged_shard(x: torch.Tensor, offsets, lens) -> torch.Tensor:
    """Rows [offsets[b], offsets[b] + lens[b]) of every x[b, h] ([B,H,Nmax,D]),
    packed into a new [B, H, max(lens), D] tensor (the rest left zero)."""
    B, H, _, D = x.shape
    n = max(lens) if len(lens) else 0
    out = torch.zeros((B, H, n, D), dtype=x.dtype, device=x.device)
    for b, (a, ln) in enumerate(zip(offsets, lens)):
        if ln:
            out[b, :, :ln].copy_(x[b, :, a:a + ln])
    return out


def _varlen_state(q, k_shard, v_shard, shard_lens, shard_lens_host, n_split=0, stream=None):
    """td_decode_varlen on a rank's chunks, written as the packed shard state
    (the normalised outputs, then the log-sum-exps; an empty chunk gives the
    empty state 0 / -inf)."""
    B, H, _, D = q.shape
    state = torch.empty(state_floats(B, H, D), dtype=torch.float32, device=q.device)
    if k_shard.shape[2] == 0:
        # no keys on this rank for any sequence
        return decode_shard(q, k_shard, v_shard, 0, 1, state=state, stream=stream)
    decode_varlen(q, k_shard, v_shard, shard_lens, seqlens_host=shard_lens_host,
                  n_split=n_split, out=state[: B * H * D].view(B, H, 1, D),
                  lse=state[B * H * D:].view(B, H, 1), stream=stream)
    return state


def decode_sharded_varlen(q: torch.Tensor, k_shard: torch.Tensor, v_shard: torch.Tensor,
                          shard_lens: torch.Tensor, *, shard_lens_host=None, group=None,
                          n_split: int = 0, stream=None, state_fn=None, merge_fn=None):
    """decode_sharded for a ragged batch without a positional bias: this rank
    holds, in k_shard/v_shard [B,H,Nmax_r,D], chunk shard_lens[b] (device
    int32 [B]) of the keys of every sequence b (pack_ragged_shard).  The
    attention of a chunk does not depend on where its keys sit in the
    sequence when there is no bias, so each rank's state is a ragged decode of
    its chunks; one all-gather and the merge finish as in decode_sharded.

    state_fn(q, k, v, lens, lens_host, n_split, stream) / merge_fn default to
    the library's kernels; a test may pass stand-ins."""
    state_fn = state_fn or _varlen_state
    merge_fn = merge_fn or merge_shards
    alone = group is None and not (dist.is_available() and dist.is_initialized())
    world = 1 if alone else dist.get_world_size(group)
    B, H, _, D = q.shape
    state = state_fn(q, k_shard, v_shard, shard_lens, shard_lens_host, n_split, stream)
    if state.numel() != state_floats(B, H, D):
        raise ValueError("shard state has the wrong size")
    if alone:
        gathered = state.view(1, -1)
    else:
        gathered = torch.empty((world, state.numel()), dtype=torch.float32, device=state.device)
        _all_gather(gathered, state, group)
    return merge_fn(gathered, B, H, D, stream=stream)
