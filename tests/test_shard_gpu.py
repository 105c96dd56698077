"""Sequence-sharded decode through the library's kernels on one GPU: the W
ranks of the gist's scheme are emulated one after another (each rank's
td_decode_shard on its chunk of the keys, then td_merge_shards over the W
states), and the result must be the plain definition over the whole sequence
(the fp64 oracle).  Nothing here waits across ranks."""
import numpy as np
import pytest
import torch

import long_context_attention_td_b200 as td
from long_context_attention_td_b200 import sharded
from long_context_attention_td_b200.workloads import Workload, make_inputs
import oracle

from gpu_common import SPEC_OUT, SPEC_LSE

pytestmark = pytest.mark.gpu

DEV = "cuda"


def emulate(w, world, mode, n_split=0):
    inp = make_inputs(w, DEV)
    q, k, v, slopes = inp["q"], inp["k"], inp["v"], inp["slopes"]
    B, H, D, N = w.B, w.H, w.D, w.N
    states = torch.empty((world, td.state_floats(B, H, D)), dtype=torch.float32, device=DEV)
    n0 = td.launch_count()
    for r, (off, ln) in enumerate(sharded.shard_bounds(N, world, mode)):
        ks = k[:, :, off:off + ln].contiguous()
        vs = v[:, :, off:off + ln].contiguous()
        td.decode_shard(q, ks, vs, off, N, state=states[r], slopes=slopes, n_split=n_split)
    out, lse = td.merge_shards(states, B, H, D)
    td.check_device_error()
    assert td.launch_count() - n0 == world + 1
    s = None if slopes is None else slopes.cpu()
    ro, rl = oracle.full(q.cpu(), k.cpu(), v.cpu(), slopes=s)
    o = out.reshape(-1, D).double().cpu().numpy()
    l = lse.reshape(-1).double().cpu().numpy()
    err_o = float(np.abs(o - ro).max())
    err_l = float(np.abs(l - rl).max())
    assert err_o <= SPEC_OUT[w.dtype], err_o
    assert err_l <= SPEC_LSE, err_l
    return err_o, err_l


@pytest.mark.parametrize("world,N,mode", [(2, 3000, "torch_chunk"), (4, 5, "torch_chunk"),
                                          (3, 100003, "balanced"), (8, 777, "torch_chunk"),
                                          (8, 1 << 16, "balanced")])
@pytest.mark.parametrize("alibi", [False, True])
def test_sharded_decode_emulated_ranks(world, N, mode, alibi):
    w = Workload("shard", torch.bfloat16, 2, 4, 128, N, alibi=alibi, seed=1300 + world + N)
    emulate(w, world, mode)


def test_sharded_decode_gist_shape_fp32():
    # the gist's own test shape: one head, D = 512, fp32, 8 ranks
    w = Workload("shard_gist", torch.float32, 1, 1, 512, 4096, seed=1234)
    emulate(w, 8, "torch_chunk")
    emulate(w, 8, "torch_chunk", n_split=3)


def test_all_empty_states_merge_to_zero():
    B, H, D = 1, 2, 64
    q = torch.zeros((B, H, 1, D), dtype=torch.float16, device=DEV)
    states = torch.empty((3, td.state_floats(B, H, D)), dtype=torch.float32, device=DEV)
    empty = torch.empty((B, H, 0, D), dtype=torch.float16, device=DEV)
    for r in range(3):
        td.decode_shard(q, empty, empty, 10, 10, state=states[r])
    out, lse = td.merge_shards(states, B, H, D)
    td.check_device_error()
    assert torch.count_nonzero(out) == 0
    assert torch.all(torch.isinf(lse)) and torch.all(lse < 0)


def test_decode_sharded_in_one_process():
    """The distributed entry point without a process group: one shard holding
    the whole sequence, merged with itself."""
    w = Workload("shard_one", torch.float16, 1, 8, 64, 20000, alibi=True, seed=1400)
    inp = make_inputs(w, DEV)
    out, lse = sharded.decode_sharded(inp["q"], inp["k"], inp["v"], 0, w.N, slopes=inp["slopes"])
    td.check_device_error()
    ro, rl = oracle.full(inp["q"].cpu(), inp["k"].cpu(), inp["v"].cpu(), slopes=inp["slopes"].cpu())
    assert float(np.abs(out.reshape(-1, w.D).double().cpu().numpy() - ro).max()) <= SPEC_OUT[w.dtype]
    assert float(np.abs(lse.reshape(-1).double().cpu().numpy() - rl).max()) <= SPEC_LSE
