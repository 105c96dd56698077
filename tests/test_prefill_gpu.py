"""Prefill attention on the tensor cores vs the fp64 oracle.

Tolerance: p is rounded to the input type (unit roundoff u = 2^-9 bf16,
2^-11 fp16) before the P V product, so each output row is a weighted average
of V whose weights carry a relative error <= u: |out - oracle| <= 4 u max|v|
(and the half-precision spec bound 2e-2).  lse comes from fp32 scores and the
unrounded fp32 sum: |lse - oracle| <= 1e-4 + 4e-7 |lse| (the ALiBi term makes
|lse| grow with S, and the scores carry the fp32 rounding of that term).
"""
import numpy as np
import pytest
import torch

import long_context_attention_td_b200 as td
from long_context_attention_td_b200.workloads import alibi_slopes
import oracle

pytestmark = pytest.mark.gpu

DEV = "cuda"
UNIT = {torch.bfloat16: 2.0 ** -9, torch.float16: 2.0 ** -11}


def inputs(B, H, S, D, dtype, seed, alibi):
    g = torch.Generator(device=DEV).manual_seed(seed)
    q = torch.randn((B, H, S, D), generator=g, device=DEV).to(dtype)
    k = torch.randn((B, H, S, D), generator=g, device=DEV).to(dtype)
    v = torch.randn((B, H, S, D), generator=g, device=DEV).to(dtype)
    return q, k, v, (alibi_slopes(H, DEV) if alibi else None)


def check(q, k, v, slopes, causal, rows=None):
    out, lse = td.prefill(q, k, v, causal=causal, slopes=slopes)
    td.check_device_error()
    B, H, S, D = q.shape
    s = None if slopes is None else slopes.cpu()
    ro, rl = oracle.prefill(q.cpu(), k.cpu(), v.cpu(), causal=causal, slopes=s, rows=rows)
    o = out.reshape(-1, D).double().cpu().numpy()
    l = lse.reshape(-1).double().cpu().numpy()
    if rows is not None:
        o, l = o[rows], l[rows]
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(l))
    err_o = float(np.abs(o - ro).max())
    vmax = float(v.abs().max())
    assert err_o <= 2e-2, err_o
    assert err_o <= 4 * UNIT[q.dtype] * vmax, (err_o, vmax)
    tol_l = 1e-4 + 4e-7 * np.abs(rl)
    assert np.all(np.abs(l - rl) <= tol_l), float(np.abs(l - rl).max())
    return err_o


@pytest.mark.parametrize("S", [1, 5, 127, 128, 129, 300, 1000])
@pytest.mark.parametrize("causal", [True, False])
def test_prefill_lengths(S, causal):
    q, k, v, sl = inputs(1, 2, S, 128, torch.bfloat16, 100 + S, alibi=False)
    check(q, k, v, sl, causal)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("alibi", [False, True])
def test_prefill_dtypes_dims_alibi(dtype, D, alibi):
    q, k, v, sl = inputs(2, 3, 700, D, dtype, 200 + D, alibi=alibi)
    check(q, k, v, sl, True)
    check(q, k, v, sl, False)


def test_prefill_peaked_scores_move_the_running_max():
    """Key norms grow along the sequence, so every row's max moves by many log2
    units from key tile to key tile: O must be rescaled in TMEM."""
    B, H, S, D = 1, 2, 640, 128
    q, k, v, _ = inputs(B, H, S, D, torch.bfloat16, 300, alibi=False)
    ramp = (1.0 + torch.arange(S, device=DEV, dtype=torch.float32) / 64.0)
    k = (k.float() * ramp[None, None, :, None]).to(torch.bfloat16)
    check(q, k, v, None, True)
    check(q, k, v, None, False)


def test_prefill_last_row_is_the_decode():
    """The last causal row of a prefill is the decode of the whole sequence."""
    B, H, S, D = 1, 4, 3000, 128
    q, k, v, sl = inputs(B, H, S, D, torch.bfloat16, 400, alibi=True)
    out, lse = td.prefill(q, k, v, causal=True, slopes=sl)
    dout, dlse = td.decode(q[:, :, S - 1:].contiguous(), k, v, slopes=sl)
    td.check_device_error()
    assert float((out[:, :, S - 1] - dout[:, :, 0]).abs().max()) <= 4 * UNIT[torch.bfloat16] * float(v.abs().max())
    assert float((lse[:, :, S - 1] - dlse[:, :, 0]).abs().max()) <= 1e-4


def test_prefill_full_size_sampled_rows():
    """The benchmark's shape (bf16, H = 32, S = 8192, causal): rows sampled
    across every query tile, checked against the oracle row by row."""
    B, H, S, D = 1, 32, 8192, 128
    q, k, v, sl = inputs(B, H, S, D, torch.bfloat16, 500, alibi=False)
    g = np.random.default_rng(5)
    rows = sorted(set(int(x) for x in g.integers(0, B * H * S, 48)) | {0, S - 1, B * H * S - 1})
    check(q, k, v, sl, True, rows=rows)


@pytest.mark.parametrize("B,H,S,D,alibi", [(3, 5, 8192, 128, True), (1, 9, 16384, 64, False)])
def test_prefill_sequence_groups_with_a_partial_last_group(B, H, S, D, alibi):
    """The kernel schedules sequences in groups whose K and V fill about 32 MB
    (8 sequences here), heaviest query tiles first inside a group; with 15 and
    9 sequences the last group is partial.  The first, last and one random row
    of every sequence against the oracle."""
    q, k, v, sl = inputs(B, H, S, D, torch.bfloat16, 700 + H, alibi=alibi)
    g = np.random.default_rng(H)
    rows = set()
    for bh in range(B * H):
        rows |= {bh * S, bh * S + S - 1, bh * S + int(g.integers(0, S))}
    check(q, k, v, sl, True, rows=sorted(rows))


def test_prefill_repeat_is_bitwise_stable_and_counted():
    q, k, v, sl = inputs(1, 2, 513, 128, torch.float16, 600, alibi=True)
    n0 = td.launch_count()
    a = td.prefill(q, k, v, slopes=sl)
    b = td.prefill(q, k, v, slopes=sl)
    td.check_device_error()
    assert td.launch_count() - n0 == 2 and td.last_kernel() == "td_prefill_kernel"
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
