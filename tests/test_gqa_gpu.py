"""Grouped-query / multi-query decode on the tensor cores vs the fp64 oracle.

Tolerance: p is rounded to the input element type before the P V product on
the tensor cores (unit roundoff u = 2^-9 for bf16, 2^-12 for fp16), so out is
a weighted average of V whose weights carry a relative error <= u: the spec
bound max |out - oracle| <= 2e-2 for half-precision inputs is kept, and the
measured error must also stay under 4 u max|v| (the weight perturbation bound).
lse comes from the unrounded sum and keeps the 1e-4 bound.
"""
import numpy as np
import pytest
import torch

import long_context_attention_td_b200 as td
from long_context_attention_td_b200.workloads import Workload, make_gqa_inputs
import oracle

pytestmark = pytest.mark.gpu

DEV = "cuda"
UNIT = {torch.bfloat16: 2.0 ** -9, torch.float16: 2.0 ** -12}


def run_and_check(w, Hkv, n_split=0, parts=None, lens=None):
    inp = make_gqa_inputs(w, Hkv, DEV)
    if lens is not None:
        inp["seqlens_host"] = torch.tensor(lens, dtype=torch.int32)
        inp["seqlens"] = inp["seqlens_host"].to(DEV)
    q, k, v = inp["q"], inp["k"], inp["v"]
    if parts is None:
        out, lse = td.decode_gqa(q, k, v, seqlens=inp["seqlens"], seqlens_host=inp["seqlens_host"],
                                 slopes=inp["slopes"], n_split=n_split)
        td.check_device_error()
    else:
        ws = torch.zeros(td.gqa_workspace_bytes(w.B, w.H, Hkv, w.D, parts), dtype=torch.uint8,
                         device=DEV)
        out, lse = td.decode_gqa_ws(q, k, v, ws, seqlens=inp["seqlens"],
                                    seqlens_host=inp["seqlens_host"], parts=parts,
                                    slopes=inp["slopes"])
        td.check_device_error(ws)
    s = None if inp["slopes"] is None else inp["slopes"].cpu()
    ro, rl = oracle.full_gqa(q.cpu(), k.cpu(), v.cpu(), slopes=s, seqlens=inp["seqlens_host"])
    o = out.reshape(-1, w.D).double().cpu().numpy()
    l = lse.reshape(-1).double().cpu().numpy()
    assert np.all(np.isfinite(o))
    fin = np.isfinite(rl)
    assert np.array_equal(np.isfinite(l), fin)
    err_o = float(np.abs(o - ro).max())
    err_l = float(np.abs(l[fin] - rl[fin]).max()) if fin.any() else 0.0
    vmax = float(v.abs().max())
    assert err_o <= 2e-2, err_o
    assert err_o <= 4 * UNIT[w.dtype] * vmax, (err_o, vmax)
    assert err_l <= 1e-4, err_l
    return err_o, err_l


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 3, 4, 5, 8, 12, 16, 24, 32, 48, 128])
def test_gqa_group_sizes(dtype, D, G):
    Hkv = 2
    w = Workload("gqa", dtype, 2, G * Hkv, D, 700, seed=300 + G + D)
    run_and_check(w, Hkv)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("N", [1, 2, 63, 64, 65, 127, 128, 129, 1000])
def test_gqa_lengths_and_alibi(N, D):
    w = Workload("gqa_n", torch.bfloat16, 1, 16, D, N, alibi=True, seed=400 + N + D)
    for n_split in (0, 1, 3):
        run_and_check(w, 2, n_split=n_split)


@pytest.mark.parametrize("parts", [1, 2, 5, 37, 148, 300])
def test_gqa_parts_cross_sequences(parts):
    w = Workload("gqa_p", torch.float16, 2, 24, 64, 500, alibi=True, seed=500)
    run_and_check(w, 3, parts=parts)


def test_gqa_merge_of_more_than_a_chunk_of_parts():
    """1300 parts per sequence (128 keys each): the merge kernel takes the part
    statistics in chunks of 1024 and its widest (512-thread) form."""
    w = Workload("gqa_many", torch.bfloat16, 1, 8, 128, 1300 * 128, alibi=True, seed=800)
    run_and_check(w, 2, parts=2 * 1300)


@pytest.mark.parametrize("D", [64, 128])
def test_gqa_ragged_with_empty_sequences(D):
    w = Workload("gqa_r", torch.bfloat16, 5, 16, D, 900, alibi=True, seed=600 + D)
    run_and_check(w, 4, lens=[0, 1, 900, 333, 0])
    run_and_check(w, 4, parts=7, lens=[0, 1, 900, 333, 0])


def test_gqa_d64_bench_shape_sampled():
    """The grouped-query D = 64 workload at a reduced length (fp16, B16 Hq32
    Hkv4, G = 8), every query head against the oracle."""
    w = Workload("gqa_d64", torch.float16, 16, 32, 64, 8192, seed=1244)
    run_and_check(w, 4)


def test_gqa_multi_query_long():
    w = Workload("mqa", torch.bfloat16, 1, 32, 128, 50000, seed=700)
    run_and_check(w, 1)


def test_gqa_repeated_calls_bitwise_and_mha_agreement():
    w = Workload("gqa_rep", torch.bfloat16, 2, 16, 128, 3000, seed=800)
    inp = make_gqa_inputs(w, 2, DEV)
    a = td.decode_gqa(inp["q"], inp["k"], inp["v"])
    for _ in range(10):
        b = td.decode_gqa(inp["q"], inp["k"], inp["v"])
    td.check_device_error()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    # the CUDA-core MHA kernel on the repeated K/V computes the same attention
    kr = inp["k"].repeat_interleave(8, dim=1).contiguous()
    vr = inp["v"].repeat_interleave(8, dim=1).contiguous()
    m = td.decode(inp["q"], kr, vr)
    td.check_device_error()
    assert float((a[0] - m[0]).abs().max()) <= 4 * UNIT[torch.bfloat16] * float(inp["v"].abs().max())
    assert float((a[1] - m[1]).abs().max()) <= 1e-4


def test_gqa_rejects_unsupported():
    w = Workload("gqa_bad", torch.float32, 1, 8, 128, 64, seed=1)
    inp = make_gqa_inputs(w, 2, DEV)
    with pytest.raises(td.TreeDecError, match="UNSUPPORTED"):
        td.decode_gqa(inp["q"], inp["k"], inp["v"])
    w = Workload("gqa_bad2", torch.bfloat16, 1, 6, 128, 64, seed=1)
    inp = make_gqa_inputs(w, 4, DEV)
    with pytest.raises(td.TreeDecError, match="INVALID"):
        td.decode_gqa(inp["q"], inp["k"], inp["v"])


def test_gqa_short_pieces_leave_replica_slices_empty():
    """Pieces shorter than a tile (a part that ends one sequence after a few
    keys and starts the next) leave some key-column slices with no key."""
    w = Workload("gqa_short", torch.bfloat16, 3, 8, 128, 70, alibi=True, seed=900)
    for parts in (4, 5, 7, 11, 13, 50, 210):
        run_and_check(w, 2, parts=parts)
    w = Workload("gqa_tiny", torch.float16, 4, 4, 64, 5, seed=901)
    for parts in (1, 3, 20):
        run_and_check(w, 1, parts=parts)


@pytest.mark.parametrize("G", [4, 8, 16, 32])
def test_gqa_large_groups_alibi_ragged_parts(G):
    w = Workload("gqa_lg", torch.bfloat16, 3, G * 2, 128, 1500, alibi=True, seed=1000 + G)
    run_and_check(w, 2, lens=[1500, 260, 1])
    for parts in (5, 23):
        run_and_check(w, 2, parts=parts, lens=[1500, 260, 1])


@pytest.mark.parametrize("G", [1, 4, 8, 16, 32])
@pytest.mark.parametrize("direction", ["growing", "shrinking"])
def test_gqa_running_max_moves_between_tiles(G, direction):
    """Key norms ramp along the sequence, so the score maximum moves up by many
    log2 units from tile to tile (or only down): the kernels must rescale the
    O accumulators they already hold."""
    Hkv, N, D = 2, 2000, 128
    w = Workload("gqa_ramp", torch.bfloat16, 1, G * Hkv, D, N, seed=1100 + G)
    inp = make_gqa_inputs(w, Hkv, DEV)
    ramp = 1.0 + torch.arange(N, device=DEV, dtype=torch.float32) / 48.0
    if direction == "shrinking":
        ramp = ramp.flip(0)
    k = (inp["k"].float() * ramp[None, None, :, None]).to(w.dtype)
    q, v = inp["q"], inp["v"]
    for parts in (None, 3):
        if parts is None:
            out, lse = td.decode_gqa(q, k, v)
            td.check_device_error()
        else:
            ws = torch.zeros(td.gqa_workspace_bytes(1, G * Hkv, Hkv, D, parts), dtype=torch.uint8,
                             device=DEV)
            out, lse = td.decode_gqa_ws(q, k, v, ws, parts=parts)
            td.check_device_error(ws)
        ro, rl = oracle.full_gqa(q.cpu(), k.cpu(), v.cpu())
        o = out.reshape(-1, D).double().cpu().numpy()
        l = lse.reshape(-1).double().cpu().numpy()
        err_o = float(np.abs(o - ro).max())
        assert err_o <= 4 * UNIT[w.dtype] * float(v.abs().max()), err_o
        assert float(np.abs(l - rl).max()) <= 1e-4 * max(1.0, float(np.abs(rl).max()))


def test_launch_count_and_kernel_events():
    """The library reports what it launched: one kernel for a multi-head call,
    the grouped-query kernel plus the merge kernel when a long sequence is
    split over the whole GPU, and events recorded right around the main kernel."""
    w = Workload("hooks", torch.bfloat16, 1, 32, 128, 1 << 17, seed=1200)
    inp = make_gqa_inputs(w, 1, DEV)
    q, k, v = inp["q"], inp["k"], inp["v"]
    td.decode_gqa(q, k, v)
    torch.cuda.synchronize()
    n0 = td.launch_count()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c, d = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    td.set_kernel_events(a, b)
    c.record()
    td.decode_gqa(q, k, v)
    d.record()
    td.set_kernel_events(None, None)
    torch.cuda.synchronize()
    td.check_device_error()
    assert td.launch_count() - n0 == 2
    assert td.last_kernel() == "td_gqa_keys_kernel"
    k_ms, call_ms = a.elapsed_time(b), c.elapsed_time(d)
    assert 0 < k_ms <= call_ms
    kr = k[:, :1].expand(1, 32, w.N, 128).contiguous()
    vr = v[:, :1].expand(1, 32, w.N, 128).contiguous()
    n1 = td.launch_count()
    td.decode(q, kr, vr)
    td.check_device_error()
    assert td.launch_count() - n1 == 1
    assert td.last_kernel() == "td_partial_kernel"
