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


class _Proc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0

    def kill(self):
        pass


def test_clock_sampler_median_and_reasons(tmp_path):
    """nvidia-smi rows (clocks.sm, clocks.max.sm, power.draw, event-reason
    bits): unreadable rows are skipped, gpu_idle is not a throttle reason."""
    p = tmp_path / "clocks.csv"
    p.write_text("1965, 1965, 700.5, 0x0000000000000004\n"
                 "1800, 1965, 990.1, 0x0000000000000004\n"
                 "[N/A], 1965, 1.0, 0x0000000000000001\n"
                 "1900, 1965, 950.0, 0x0000000000000000\n"
                 "1500, 1965, 800.0, 0x0000000000000001\n"
                 "truncated line\n")
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.proc, s.path, s.f = _Proc(), str(p), open(tmp_path / "sink", "w")
    r = s.stop()
    assert r == {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                 "samples": 4}


def test_profiled_traffic_needs_the_current_source_hash(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "td_partial_wl.md").write_text(
        "kernel source hash: `0123456789abcdef`\n\ndram bytes per launch: 12345\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda k: "0123456789abcdef")
    assert bench.profiled_traffic("wl", "td_partial_kernel") == 12345
    # an instantiation suffix in the kernel's name maps to the same sources
    assert bench.profiled_traffic("wl", "td_partial_kernel (fp8 kv)") == 12345
    assert bench.profiled_traffic("other", "td_partial_kernel") is None
    assert bench.profiled_traffic("wl", "unknown_kernel") is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda k: "fedcba9876543210")
    assert bench.profiled_traffic("wl", "td_partial_kernel") is None


def test_reference_arm_prints_the_config_of_the_cuda_arm(capsys):
    """Both arms build `config` with workload_config (host arithmetic only), so
    the driver can pair their lines; the reference arm's sample stays small."""
    import argparse
    import json
    for wl in ("gist_f32_d512_n4k", "prefill_bf16_alibi_b4_h16_d128_s4k"):
        bench.main(["--impl", "reference", "--steps", "3", "--warmup", "3", "--workload", wl])
        line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
        args = argparse.Namespace(workload=wl, n_keys=0, n_split=None)
        expect = bench.workload_config(args, WORKLOADS[wl], bench.parallelism_name(1, False))
        assert line["impl"] == "reference" and line["config"] == expect
        assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["value"] > 0
