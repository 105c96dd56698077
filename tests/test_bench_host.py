"""bench.py's host-side helpers (no GPU): the sampled parity check it prints
beside the measurement."""
import torch

import bench
import oracle
from long_context_attention_td_b200.workloads import WORKLOADS, make_inputs


def _oracle_outputs(inp, w):
    q, k, v = inp["q"], inp["k"], inp["v"]
    s = None if inp["slopes"] is None else inp["slopes"]
    if w.kv_heads and w.kv_heads != w.H:
        o, l = oracle.full_gqa(q, k, v, slopes=s, seqlens=inp["seqlens_host"])
    else:
        o, l = oracle.full(q, k, v, slopes=s, seqlens=inp["seqlens_host"])
    out = torch.tensor(o, dtype=torch.float32).view(w.B, w.H, 1, w.D)
    lse = torch.tensor(l, dtype=torch.float32).view(w.B, w.H, 1)
    return out, lse


def test_sampled_parity_accepts_the_exact_result_and_flags_a_wrong_one():
    for name, kw in (("bf16_alibi_b8_h32_d128_n32k", dict(B=2, H=4, N=300)),
                     ("f16_ragged_b64_h16_d64", dict(B=3, H=2, N=200, ragged=(1, 200))),
                     ("gqa_bf16_h32_kv8_d128_n128k", dict(H=8, kv_heads=2, N=257))):
        w = WORKLOADS[name].with_(**kw)
        inp = make_inputs(w, "cpu")
        out, lse = _oracle_outputs(inp, w)
        r = bench.sampled_parity(inp, w, out, lse)
        assert r["ok"] and r["rows"] >= 2 and r["max_abs_out"] < 1e-6, r
        bad = out.clone()
        bad[0, 0, 0, 3] += 0.05
        assert not bench.sampled_parity(inp, w, bad, lse)["ok"]


def test_sampled_parity_skips_prefill_and_fp8():
    assert bench.sampled_parity({}, WORKLOADS["prefill_bf16_h32_d128_s8k"], None, None) is None
    assert bench.sampled_parity({}, WORKLOADS["fp8kv_h32_d128_n128k"], None, None) is None
