"""Stress of the fused last-CTA ticket merge.

1000 decode calls on one caller workspace, each with a random part count and
one of three problems of different B*H (so the ticket region and the part
records of earlier calls overlap the next call's), every result held to the
fp64 oracle, repeated part counts held to their first result bit for bit.
Every 20th call also runs the two-kernel path over the same chunk boundaries:
td_decode_shard on each chunk (the gist's per-rank local attention, written
out as a normalised state), then the standalone td_combine over those states
with (num, m, l) = (out_r, lse_r, 1) -- the gist's global max, renormalisation
and sums.  The fused and two-kernel results differ only in the order of their
fp32 operations, so both are held to the oracle and to each other within the
fp32 arithmetic bound.
"""
import numpy as np
import pytest
import torch

import long_context_attention_td_b200 as td
from long_context_attention_td_b200.workloads import Workload, make_inputs

from gpu_common import ARITH_OUT, SPEC_LSE, compare, oracle_all

pytestmark = pytest.mark.gpu

PROBLEMS = [
    Workload("st_bf16", torch.bfloat16, 2, 4, 128, 3001, seed=111),
    Workload("st_f16_alibi", torch.float16, 1, 3, 64, 777, alibi=True, seed=112),
    Workload("st_f32_d256", torch.float32, 3, 2, 256, 1500, seed=113),
]
CALLS = 1000
CROSS_EVERY = 20


def _two_kernel(inp, w, S):
    """td_decode_shard on the S balanced chunks of every sequence, then
    td_combine over the S states of each (b,h)."""
    B, H, N, D = w.B, w.H, w.N, w.D
    nums = torch.empty((B, H, S, D), dtype=torch.float32, device="cuda")
    ms = torch.empty((B, H, S), dtype=torch.float32, device="cuda")
    for i in range(S):
        a, b = i * N // S, (i + 1) * N // S
        k = inp["k"][:, :, a:b].contiguous()
        v = inp["v"][:, :, a:b].contiguous()
        st = td.decode_shard(inp["q"], k, v, a, N, slopes=inp["slopes"], n_split=1)
        nums[:, :, i] = st[: B * H * D].view(B, H, D)
        ms[:, :, i] = st[B * H * D:].view(B, H)
    return td.combine(nums, ms, torch.ones_like(ms))


def test_thousand_fused_merges_against_the_oracle_and_the_two_kernel_path():
    inputs = [make_inputs(w, "cuda") for w in PROBLEMS]
    refs = [oracle_all(inp) for inp in inputs]
    ws_bytes = max(td.workspace_bytes(w.B, w.H, w.D, w.B * w.H * w.N) for w in PROBLEMS)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    g = np.random.default_rng(2024)
    first = {}
    crossed = 0
    for it in range(CALLS):
        pi = int(g.integers(len(PROBLEMS)))
        w, inp = PROBLEMS[pi], inputs[pi]
        T = w.B * w.H * w.N
        if it % CROSS_EVERY == 0:
            S = int(g.integers(1, 17))
            parts = w.B * w.H * S            # S balanced chunks per sequence
        else:
            parts = int(min(T, np.exp(g.uniform(0, np.log(4 * T)))))
            parts = max(1, parts)
        out, lse = td.decode_ws(inp["q"], inp["k"], inp["v"], ws, parts=parts,
                                slopes=inp["slopes"])
        compare(out, lse, refs[pi][0], refs[pi][1], np.arange(w.B * w.H), w.dtype)
        key = (pi, parts)
        if key in first:
            assert torch.equal(out, first[key][0]) and torch.equal(lse, first[key][1]), key
        else:
            first[key] = (out.clone(), lse.clone())
        if it % CROSS_EVERY == 0:
            o2, l2 = _two_kernel(inp, w, S)
            compare(o2, l2, refs[pi][0], refs[pi][1], np.arange(w.B * w.H), w.dtype)
            assert float((o2 - out).abs().max()) <= ARITH_OUT
            assert float((l2 - lse).abs().max()) <= SPEC_LSE
            crossed += 1
    td.check_device_error(ws)
    assert crossed == CALLS // CROSS_EVERY
    # the tickets are all back to zero: the region right after the error word
    tickets = ws[256:256 + 4 * max(w.B * w.H for w in PROBLEMS)].view(torch.int32)
    assert int(tickets.abs().sum()) == 0
