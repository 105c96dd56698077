"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small cases compare every output element; the five named workloads run at
full size in the launch configuration the benchmark times and compare sampled
(b,h) rows the oracle computes one by one, plus an exact key-count property
that holds at any size.
"""
import math

import numpy as np
import pytest
import torch

import long_context_attention_td_b200 as td
from long_context_attention_td_b200.workloads import WORKLOADS, Workload, make_inputs
import oracle

from gpu_common import (ARITH_OUT, compare, oracle_all, oracle_on, run_td, sample_bh)

pytestmark = pytest.mark.gpu

DEV = "cuda"


def small(name, **kw):
    return WORKLOADS[name].with_(**kw)


# ---------------------------------------------------------------- small, dense

SMALL = [
    # gist shape, fp32 D=512, 8 chunks as on the page and the heuristic
    (small("gist_f32_d512_n4k"), 8),
    (small("gist_f32_d512_n4k"), 0),
    (small("gist_f32_d512_n4k", N=31), 8),
    # bf16 D=128, several tiles and a ragged tail
    (small("bf16_h32_d128_n128k", H=4, N=4 * 64 * 7 + 37), 0),
    (small("bf16_h32_d128_n128k", H=4, N=4 * 64 * 7 + 37), 5),
    # ALiBi
    (small("bf16_alibi_b8_h32_d128_n32k", B=2, H=8, N=3000), 0),
    (small("bf16_alibi_b8_h32_d128_n32k", B=2, H=8, N=3000), 3),
    # peaked softmax
    (small("bf16_peaked_h8_d128_n1m", H=2, N=20000), 0),
    # ragged fp16 D=64
    (small("f16_ragged_b64_h16_d64", B=6, H=3, N=2000, ragged=(1, 2000)), 0),
    (small("f16_ragged_b64_h16_d64", B=6, H=3, N=2000, ragged=(1, 2000)), 4),
]


@pytest.mark.parametrize("w,n_split", SMALL, ids=lambda x: getattr(x, "name", str(x)))
def test_small_workloads_every_element(w, n_split):
    inp = make_inputs(w, DEV)
    out, lse = run_td(inp, n_split=n_split)
    ref_o, ref_l = oracle_all(inp)
    compare(out, lse, ref_o, ref_l, np.arange(w.B * w.H), w.dtype)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("D", [64, 128, 256, 512])
@pytest.mark.parametrize("alibi", [False, True])
def test_every_dtype_and_head_size(dtype, D, alibi):
    w = Workload("sweep", dtype, 2, 3, D, 1000, alibi=alibi, seed=7 + D)
    inp = make_inputs(w, DEV)
    for n_split in (0, 1, 3):
        out, lse = run_td(inp, n_split=n_split)
        ref_o, ref_l = oracle_all(inp)
        compare(out, lse, ref_o, ref_l, np.arange(6), dtype)


@pytest.mark.parametrize("N", [1, 2, 63, 64, 65, 127, 128, 129, 1000])
def test_short_and_tile_edge_lengths(N):
    w = Workload("edge", torch.bfloat16, 1, 5, 128, N, alibi=True, seed=N)
    inp = make_inputs(w, DEV)
    ref_o, ref_l = oracle_all(inp)
    for n_split in (0, 1, 2, 7, N + 5):
        out, lse = run_td(inp, n_split=n_split)
        compare(out, lse, ref_o, ref_l, np.arange(5), w.dtype)


@pytest.mark.parametrize("parts", [1, 2, 3, 7, 29, 148, 1000, 5 * 700])
def test_explicit_part_counts_cross_sequence_boundaries(parts):
    """Parts that start and end inside sequences, span several sequences, or
    hold a single key: the flattened partition and the ticket merge."""
    w = Workload("parts", torch.float16, 1, 5, 64, 700, alibi=True, seed=11)
    inp = make_inputs(w, DEV)
    ref_o, ref_l = oracle_all(inp)
    out, lse = run_td(inp, parts=parts)
    compare(out, lse, ref_o, ref_l, np.arange(5), w.dtype)


def test_ragged_with_empty_and_full_sequences():
    w = Workload("ragged", torch.float16, 7, 2, 64, 300, alibi=True, seed=3)
    inp = make_inputs(w, DEV)
    lens = torch.tensor([0, 1, 300, 0, 17, 299, 0], dtype=torch.int32)
    inp["seqlens_host"] = lens
    inp["seqlens"] = lens.to(DEV)
    ref_o, ref_l = oracle_all(inp)
    for parts in (None, 1, 2, 5, 14, 64, 600):
        out, lse = run_td(inp, parts=parts)
        compare(out, lse, ref_o, ref_l, np.arange(14), w.dtype)
        # without the host copy of the lengths too
    out, lse = td.decode_varlen(inp["q"], inp["k"], inp["v"], inp["seqlens"],
                                slopes=inp["slopes"])
    td.check_device_error()
    compare(out, lse, ref_o, ref_l, np.arange(14), w.dtype)


def test_many_short_sequences_per_cta():
    w = Workload("many", torch.bfloat16, 64, 16, 128, 37, seed=5)
    inp = make_inputs(w, DEV)
    ref_o, ref_l = oracle_all(inp)
    for parts in (None, 1, 10, 148):
        out, lse = run_td(inp, parts=parts)
        compare(out, lse, ref_o, ref_l, np.arange(64 * 16), w.dtype)


def test_chunked_gist_reading_agrees():
    """8 chunks on the GPU vs the oracle's own Algorithm-3 merge (both chunk
    modes) and the plain definition."""
    w = WORKLOADS["gist_f32_d512_n4k"]
    inp = make_inputs(w, DEV)
    out, lse = run_td(inp, n_split=8)
    q, k, v = inp["q"].cpu(), inp["k"].cpu(), inp["v"].cpu()
    for mode in ("torch_chunk", "balanced"):
        ro, rl = oracle.chunked(q, k, v, 8, mode)
        compare(out, lse, ro, rl, np.arange(1), w.dtype)


# ------------------------------------------------ determinism and the tickets

def test_repeated_calls_are_bitwise_identical_and_tickets_reset():
    w = Workload("rep", torch.bfloat16, 2, 8, 128, 5000, alibi=True, seed=21)
    inp = make_inputs(w, DEV)
    ref_o, ref_l = oracle_all(inp)
    g = np.random.default_rng(0)
    first = {}
    for it in range(60):
        P = int(g.choice([1, 3, 16, 37, 148, 296, 1000]))
        out, lse = run_td(inp, parts=P)
        if P in first:
            assert torch.equal(out, first[P][0]) and torch.equal(lse, first[P][1])
        else:
            first[P] = (out.clone(), lse.clone())
            compare(out, lse, ref_o, ref_l, np.arange(16), w.dtype)
    # the library-owned workspace path, many calls on one stream
    a = td.decode(inp["q"], inp["k"], inp["v"], slopes=inp["slopes"])
    for _ in range(20):
        b = td.decode(inp["q"], inp["k"], inp["v"], slopes=inp["slopes"])
    td.check_device_error()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_workspace_reuse_with_growing_and_shrinking_batch():
    """One workspace (library-owned, then caller-owned) serving calls whose
    B*H goes up and down: the ticket region must be zero whenever it grows
    over memory earlier calls used for part records."""
    shapes = [(1, 2, 5000), (64, 16, 40), (1, 3, 7000), (128, 16, 33), (2, 2, 900),
              (128, 16, 33)]
    cases = []
    for i, (B, H, N) in enumerate(shapes):
        w = Workload("reuse%d" % i, torch.bfloat16, B, H, 128, N, seed=60 + i)
        inp = make_inputs(w, DEV)
        cases.append((w, inp, oracle_all(inp)))
    for w, inp, (ro, rl) in cases:
        out, lse = run_td(inp)
        compare(out, lse, ro, rl, np.arange(w.B * w.H), w.dtype)
    ws = torch.zeros(4 << 20, dtype=torch.uint8, device=DEV)
    for w, inp, (ro, rl) in cases + cases[::-1]:
        for P in (37, 300):
            out, lse = td.decode_ws(inp["q"], inp["k"], inp["v"], ws, parts=P)
            td.check_device_error(ws)
            compare(out, lse, ro, rl, np.arange(w.B * w.H), w.dtype)


def test_caller_workspace_matches_library_workspace():
    w = Workload("ws", torch.bfloat16, 1, 4, 128, 9000, seed=31)
    inp = make_inputs(w, DEV)
    P = td.plan_parts(1, 4, 9000, 128, torch.bfloat16)
    ws = torch.zeros(td.workspace_bytes(1, 4, 128, P), dtype=torch.uint8, device=DEV)
    o1, l1 = td.decode_ws(inp["q"], inp["k"], inp["v"], ws)
    o2, l2 = td.decode(inp["q"], inp["k"], inp["v"])
    td.check_device_error(ws)
    td.check_device_error()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    small_ws = torch.zeros(64, dtype=torch.uint8, device=DEV)
    with pytest.raises(td.TreeDecError, match="WORKSPACE"):
        td.decode_ws(inp["q"], inp["k"], inp["v"], small_ws)


def test_host_buffer_entry_point_matches_device_path():
    w = Workload("host", torch.float16, 3, 2, 64, 777, alibi=True, ragged=(100, 777), seed=41)
    inp = make_inputs(w, DEV)
    o1, l1 = run_td(inp)
    qh = inp["q"].cpu().pin_memory()
    kh = inp["k"].cpu().pin_memory()
    vh = inp["v"].cpu().pin_memory()
    o2, l2 = td.decode_host(qh, kh, vh, seqlens=inp["seqlens_host"], slopes=inp["slopes"].cpu())
    assert torch.equal(o1.cpu(), o2) and torch.equal(l1.cpu(), l2)


def test_bad_device_lengths_are_clamped_and_reported():
    w = Workload("bad", torch.float16, 2, 2, 64, 100, seed=51)
    inp = make_inputs(w, DEV)
    bad = torch.tensor([50, 1000], dtype=torch.int32, device=DEV)
    td.decode_varlen(inp["q"], inp["k"], inp["v"], bad)
    with pytest.raises(td.TreeDecError, match="0x2"):
        td.check_device_error()
    td.check_device_error()  # cleared
    # the clamped call equals lengths [50, 100]
    good = torch.tensor([50, 100], dtype=torch.int32)
    inp["seqlens_host"], inp["seqlens"] = good, good.to(DEV)
    out, lse = run_td(inp)
    ref_o, ref_l = oracle_all(inp)
    compare(out, lse, ref_o, ref_l, np.arange(4), w.dtype)


# ---------------------------------------------------------------- combine

@pytest.mark.parametrize("S,D", [(1, 128), (8, 512), (37, 64), (1024, 128), (5, 100)])
def test_combine_of_caller_partials(S, D):
    g = torch.Generator().manual_seed(S * 1000 + D)
    B, H = 2, 3
    num = torch.randn(B, H, S, D, generator=g, dtype=torch.float64)
    m = torch.randn(B, H, S, generator=g, dtype=torch.float64) * 5
    l = torch.rand(B, H, S, generator=g, dtype=torch.float64) * 10 + 0.1
    if S > 2:  # empty parts
        m[:, :, 1] = -math.inf
        l[:, :, 1] = 0
        num[:, :, 1] = 0
    m[1, 2, :] = -math.inf  # an all-empty row
    l[1, 2, :] = 0
    num[1, 2] = 0
    n32, m32, l32 = num.float(), m.float(), l.float()
    out, lse = td.combine(n32.to(DEV), m32.to(DEV), l32.to(DEV))
    for b in range(B):
        for h in range(H):
            ro, rl = oracle.merge(n32[b, h].double().numpy(), m32[b, h].double().numpy(),
                                  l32[b, h].double().numpy())
            o = out[b, h, 0].double().cpu().numpy()
            scale = max(1.0, float(np.abs(ro).max()))
            assert np.abs(o - ro).max() <= 1e-5 * scale
            L = float(lse[b, h, 0])
            if rl == -math.inf:
                assert L == -math.inf and np.all(o == 0)
            else:
                assert abs(L - rl) <= 1e-4


# ------------------------------------------------ full-size named workloads

FULL = ["gist_f32_d512_n4k", "bf16_h32_d128_n128k", "bf16_alibi_b8_h32_d128_n32k",
        "bf16_peaked_h8_d128_n1m", "f16_ragged_b64_h16_d64"]


@pytest.mark.slow
@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled_rows(name):
    w = WORKLOADS[name]
    inp = make_inputs(w, DEV)
    out, lse = run_td(inp, n_split=w.n_split)
    bh = sample_bh(w.B, w.H, 12, seed=1)
    ref_o, ref_l = oracle_on(inp, bh)
    compare(out, lse, ref_o, ref_l, bh, w.dtype)


@pytest.mark.slow
@pytest.mark.parametrize("name", FULL)
def test_full_size_exact_key_counts(name):
    """q = 0 makes every score 0 (no bias): each key weighs exactly 1, the sums
    are exact integers in fp32, so with v_j = onehot(j mod D) every out[d] is
    exactly count{j < n_b : j = d mod D} / n_b and lse = ln n_b.  A key read
    twice or skipped anywhere in the partition changes an output."""
    w = WORKLOADS[name].with_(alibi=False)
    inp = make_inputs(w, DEV)
    B, H, N, D = w.B, w.H, w.N, w.D
    inp["q"].zero_()
    idx = torch.arange(N, device=DEV) % D
    onehot = torch.nn.functional.one_hot(idx, D).to(w.dtype)
    inp["v"].copy_(onehot.view(1, 1, N, D).expand(B, H, N, D))
    out, lse = run_td(inp, n_split=w.n_split)
    lens = inp["seqlens_host"]
    n_b = (lens.to(torch.float64) if lens is not None
           else torch.full((B,), float(N), dtype=torch.float64))
    d = torch.arange(D, dtype=torch.float64)
    cnt = torch.floor((n_b.view(B, 1) - 1 - d.view(1, D)) / D) + 1   # [B, D]
    expect = (cnt / n_b.view(B, 1)).view(B, 1, 1, D).expand(B, H, 1, D)
    got = out.double().cpu()
    assert torch.allclose(got, expect, rtol=2e-7, atol=0), float((got - expect).abs().max())
    lexp = torch.log(n_b).view(B, 1, 1).expand(B, H, 1)
    assert torch.allclose(lse.double().cpu(), lexp, rtol=0, atol=4e-6)


SPLIT_SWEEP = [16, 32, 64, 128, 256, 512, 1024]


@pytest.mark.slow
@pytest.mark.parametrize("mode", ["aligned", "scaled"])
def test_peaked_1m_split_count_sweep(mode):
    """bf16 B1 H8 D128 N=1M with 16 spiked keys per head, 16..1024 splits per
    head: every head against the oracle at every split count (the partition
    moves the spikes between parts, and the merge must rescale them)."""
    w = WORKLOADS["bf16_peaked_h8_d128_n1m"].with_(spike_mode=mode)
    inp = make_inputs(w, DEV)
    bh = np.arange(w.B * w.H)
    ref_o, ref_l = oracle_on(inp, bh)
    for n_split in SPLIT_SWEEP:
        out, lse = run_td(inp, n_split=n_split)
        compare(out, lse, ref_o, ref_l, bh, w.dtype)
