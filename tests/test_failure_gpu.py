"""The split-KV kernel's bounded waits, made to run out on purpose.

Every pipeline wait of the kernel gives up after a time limit, records
TD_DEVERR_WAIT_TIMEOUT in the workspace's error word and lets the CTA wind
down, so a stalled pipeline ends as an error status the host reads instead of
a hung GPU.  td_set_wait_test sets that limit to 1 ms and has the first CTA's
loader stop issuing tiles from a chosen tile on (nothing else ever completes
that CTA's next stage), so the consumers' wait can only end by its limit.
Each test checks the reported bits, that the call returned within seconds, and
that the next normal call on the same workspace matches the fp64 oracle.
"""
import time

import numpy as np
import pytest
import torch

import long_context_attention_td_b200 as td
from long_context_attention_td_b200.workloads import Workload, make_inputs

from gpu_common import compare, oracle_all

pytestmark = pytest.mark.gpu

TD_ERR_DEVICE = 5
TIMEOUT_BIT = 0x1

W_UNIFORM = Workload("fail_bf16", torch.bfloat16, 2, 8, 128, 9000, seed=81)
W_RAGGED = Workload("fail_f16_ragged", torch.float16, 3, 4, 64, 6000, ragged=(1, 6000),
                    alibi=True, seed=82)


def _expect_timeout(check):
    with pytest.raises(td.TreeDecError) as ei:
        check()
    assert ei.value.status == TD_ERR_DEVICE
    assert "0x%x" % TIMEOUT_BIT in str(ei.value)


def _with_withheld_tile(tile, fn):
    td.set_wait_test(1_000_000, tile)
    try:
        return fn()
    finally:
        td.set_wait_test(0, -1)


@pytest.mark.parametrize("tile", [0, 1, 5])
@pytest.mark.parametrize("n_split", [0, 3])
def test_library_workspace_timeout_then_clean_call(tile, n_split):
    w = W_UNIFORM
    inp = make_inputs(w, "cuda")
    ref_o, ref_l = oracle_all(inp)
    td.decode(inp["q"], inp["k"], inp["v"], n_split=n_split)
    td.check_device_error()
    t0 = time.perf_counter()
    _with_withheld_tile(tile, lambda: td.decode(inp["q"], inp["k"], inp["v"], n_split=n_split))
    _expect_timeout(td.check_device_error)
    assert time.perf_counter() - t0 < 10.0
    td.check_device_error()  # cleared by the read above
    for _ in range(2):
        out, lse = td.decode(inp["q"], inp["k"], inp["v"], n_split=n_split)
        td.check_device_error()
        compare(out, lse, ref_o, ref_l, np.arange(w.B * w.H), w.dtype)


@pytest.mark.parametrize("tile", [0, 2])
def test_caller_workspace_timeout_then_clean_call(tile):
    w = W_RAGGED
    inp = make_inputs(w, "cuda")
    ref_o, ref_l = oracle_all(inp)
    B, H, N, D = inp["k"].shape
    parts = 40
    ws = torch.zeros(td.workspace_bytes(B, H, D, parts), dtype=torch.uint8, device="cuda")

    def call():
        return td.decode_ws(inp["q"], inp["k"], inp["v"], ws, seqlens=inp["seqlens"],
                            seqlens_host=inp["seqlens_host"], parts=parts,
                            slopes=inp["slopes"])

    t0 = time.perf_counter()
    _with_withheld_tile(tile, call)
    _expect_timeout(lambda: td.check_device_error(ws))
    assert time.perf_counter() - t0 < 10.0
    for _ in range(2):
        out, lse = call()
        td.check_device_error(ws)
        compare(out, lse, ref_o, ref_l, np.arange(w.B * w.H), w.dtype)


def test_a_withheld_tile_past_the_end_changes_nothing():
    """A withheld tile the first CTA never reaches leaves the call intact."""
    w = W_UNIFORM
    inp = make_inputs(w, "cuda")
    ref_o, ref_l = oracle_all(inp)
    out, lse = _with_withheld_tile(
        1 << 40, lambda: td.decode(inp["q"], inp["k"], inp["v"], n_split=3))
    td.check_device_error()
    compare(out, lse, ref_o, ref_l, np.arange(w.B * w.H), w.dtype)
