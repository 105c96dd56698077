"""Decode over an FP8 E4M3 K/V cache vs the fp64 oracle on the dequantised
cache (K = e4m3(k8) * k_scale[h], V = e4m3(v8) * v_scale[h]).

Tolerance, derived from the kernel's arithmetic:
  * q . k runs as 8-term chains of fused f16 multiply-adds (one rounding of
    u = 2^-11 each), so a score carries |ds| <= E = 8 u D^-1/2 k_scale
    sum_i |q_i| |k8_i| (natural-log units), plus the fp32 rest;
  * |lse - oracle| <= max_j E_j + 1e-4;
  * the softmax weights then move by at most a factor e^(+-2E), p is rounded
    to f16 (u) and p v is summed in f16 over at most 4 rows before fp32 (4u
    of the partial sums), so |out - oracle| <= (2 (e^(2E) - 1) + 6 u) max|v|.
"""
import math

import numpy as np
import pytest
import torch

import long_context_attention_td_b200 as td
from long_context_attention_td_b200.workloads import Workload, make_inputs
import oracle

pytestmark = pytest.mark.gpu

DEV = "cuda"
U16 = 2.0 ** -11


def run_and_check(w, n_split=0, lens=None):
    inp = make_inputs(w, DEV)
    if lens is not None:
        inp["seqlens_host"] = torch.tensor(lens, dtype=torch.int32)
        inp["seqlens"] = inp["seqlens_host"].to(DEV)
    q, k8, v8 = inp["q"], inp["k"], inp["v"]
    ks, vs = inp["k_scale"], inp["v_scale"]
    out, lse = td.decode_fp8(q, k8, v8, ks, vs, seqlens=inp["seqlens"],
                             seqlens_host=inp["seqlens_host"], slopes=inp["slopes"],
                             n_split=n_split)
    td.check_device_error()
    K = oracle.dequant_e4m3(k8, ks)
    V = oracle.dequant_e4m3(v8, vs)
    s = None if inp["slopes"] is None else inp["slopes"].cpu()
    ro, rl = oracle.full(q.double().cpu(), torch.from_numpy(K), torch.from_numpy(V), slopes=s,
                         seqlens=inp["seqlens_host"])
    B, H, N, D = w.B, w.H, w.N, w.D
    o = out.reshape(-1, D).double().cpu().numpy()
    l = lse.reshape(-1).double().cpu().numpy()
    # the bound E per (b,h) row from |q| and the codes' magnitudes
    lut = np.abs(np.array([oracle.decode_e4m3(b) if (b & 0x7F) != 0x7F else 0.0
                           for b in range(256)]))
    qa = np.abs(q.double().cpu().numpy()).reshape(B, H, D)
    ka = lut[k8.cpu().numpy()]                                   # [B,H,N,D]
    lens_b = [N] * B if inp["seqlens_host"] is None else [int(x) for x in inp["seqlens_host"]]
    E = np.zeros(B * H)
    for b in range(B):
        for h in range(H):
            n = lens_b[b]
            if n == 0:
                continue
            sums = ka[b, h, :n] @ qa[b, h]
            E[b * H + h] = 8 * U16 * float(ks[h]) / math.sqrt(D) * float(sums.max())
    vmax = float(np.abs(V).max())
    fin = np.isfinite(rl)
    assert np.array_equal(np.isfinite(l), fin)
    err_l = np.abs(l[fin] - rl[fin])
    assert np.all(err_l <= E[fin] + 1e-4), (float(err_l.max()), float(E.max()))
    bound_o = (2 * (np.exp(2 * E) - 1) + 6 * U16) * vmax
    err_o = np.abs(o - ro).max(axis=1)
    assert np.all(err_o <= bound_o + 1e-6), (float(err_o.max()), float(bound_o.max()))
    return float(err_o.max()), float(err_l.max()) if err_l.size else 0.0


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("qdt", [torch.bfloat16, torch.float16])
def test_fp8_dims_and_q_types(D, qdt):
    w = Workload("fp8", qdt, 2, 4, D, 3000, kv_fp8=True, seed=1500 + D)
    run_and_check(w)


@pytest.mark.parametrize("N", [1, 2, 127, 128, 129, 20000])
def test_fp8_lengths_alibi_and_splits(N):
    w = Workload("fp8_n", torch.bfloat16, 1, 8, 128, N, kv_fp8=True, alibi=True, seed=1600 + N)
    for n_split in (0, 1, 7):
        run_and_check(w, n_split=n_split)


def test_fp8_ragged_with_empty_sequences():
    w = Workload("fp8_r", torch.float16, 4, 4, 128, 5000, kv_fp8=True, alibi=True, seed=1700)
    run_and_check(w, lens=[0, 5000, 1, 2345])


def test_fp8_large_q_does_not_overflow_half_precision():
    """|q| far above 1: the power-of-two pre-scaling keeps the f16 chains finite."""
    w = Workload("fp8_big", torch.bfloat16, 1, 4, 128, 4000, kv_fp8=True, scale=40.0, seed=1800)
    run_and_check(w)


def test_fp8_bench_shape_all_heads():
    w = Workload("fp8kv_h32_d128_n128k", torch.bfloat16, 1, 32, 128, 131072, kv_fp8=True,
                 seed=1243)
    eo, el = run_and_check(w)
    assert td.last_kernel() == "td_partial_kernel (fp8 kv)"
