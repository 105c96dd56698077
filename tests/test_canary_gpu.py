"""Guard bytes around every buffer the kernels write.

Each output (out, lse, shard state) and each caller workspace is placed inside
a larger allocation whose 4 KiB margins on both sides hold a sentinel byte;
after the call the margins must be untouched.  This catches a write past the
end (or before the start) of a row that the parity tests, which read only the
valid elements, would miss.  Shapes sit on and next to tile edges.
"""
import pytest
import torch

import long_context_attention_td_b200 as td
from long_context_attention_td_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu

MARGIN = 4096
SENTINEL = 0xA5


class Guarded:
    """A device buffer of `nbytes` between two sentinel-filled margins."""

    def __init__(self, nbytes, fill=None):
        self.nbytes = int(nbytes)
        self.raw = torch.full((MARGIN + self.nbytes + MARGIN,), SENTINEL, dtype=torch.uint8,
                              device="cuda")
        if fill is not None:
            self.raw[MARGIN:MARGIN + self.nbytes].fill_(fill)

    def bytes(self):
        return self.raw[MARGIN:MARGIN + self.nbytes]

    def f32(self, *shape):
        return self.bytes().view(torch.float32).view(*shape)

    def check(self, what):
        torch.cuda.synchronize()
        lo = self.raw[:MARGIN]
        hi = self.raw[MARGIN + self.nbytes:]
        bad_lo = int((lo != SENTINEL).sum())
        bad_hi = int((hi != SENTINEL).sum())
        assert bad_lo == 0 and bad_hi == 0, "%s: %d bytes before, %d after changed" % (
            what, bad_lo, bad_hi)


def _outs(B, H, D, rows=1):
    go = Guarded(B * H * rows * D * 4)
    gl = Guarded(B * H * rows * 4)
    return go, gl


def _check_finite(*ts):
    for t in ts:
        assert torch.isfinite(t).all()


DECODE = [
    Workload("c_f32_d512", torch.float32, 1, 2, 512, 4097, seed=91),
    Workload("c_bf16_d128", torch.bfloat16, 2, 3, 128, 64 * 5 + 1, seed=92),
    Workload("c_bf16_d128_edge", torch.bfloat16, 1, 5, 128, 64 * 6, seed=93),
    Workload("c_f16_d64_ragged", torch.float16, 4, 3, 64, 700, ragged=(0, 700), seed=94),
    Workload("c_bf16_d256_alibi", torch.bfloat16, 2, 2, 256, 999, alibi=True, seed=95),
]


@pytest.mark.parametrize("w", DECODE, ids=lambda w: w.name)
@pytest.mark.parametrize("n_split", [0, 1, 7])
def test_decode_outputs_stay_in_bounds(w, n_split):
    inp = make_inputs(w, "cuda")
    go, gl = _outs(w.B, w.H, w.D)
    out, lse = go.f32(w.B, w.H, 1, w.D), gl.f32(w.B, w.H, 1)
    if inp["seqlens"] is not None:
        td.decode_varlen(inp["q"], inp["k"], inp["v"], inp["seqlens"],
                         seqlens_host=inp["seqlens_host"], slopes=inp["slopes"],
                         n_split=n_split, out=out, lse=lse)
    else:
        td.decode(inp["q"], inp["k"], inp["v"], slopes=inp["slopes"], n_split=n_split,
                  out=out, lse=lse)
    td.check_device_error()
    go.check("out")
    gl.check("lse")
    _check_finite(out)


@pytest.mark.parametrize("w", DECODE, ids=lambda w: w.name)
@pytest.mark.parametrize("parts_mul", [1, 3])
def test_caller_workspace_stays_in_bounds(w, parts_mul):
    inp = make_inputs(w, "cuda")
    B, H, N, D = inp["k"].shape
    total = -1 if inp["seqlens_host"] is None else int(inp["seqlens_host"].sum()) * H
    parts = td.plan_parts(B, H, N, D, w.dtype, 0, total) * parts_mul
    parts = max(1, min(parts, B * H * N))
    gw = Guarded(td.workspace_bytes(B, H, D, parts), fill=0)
    go, gl = _outs(B, H, D)
    for _ in range(2):
        td.decode_ws(inp["q"], inp["k"], inp["v"], gw.bytes(), seqlens=inp["seqlens"],
                     seqlens_host=inp["seqlens_host"], parts=parts, slopes=inp["slopes"],
                     out=go.f32(B, H, 1, D), lse=gl.f32(B, H, 1))
        td.check_device_error(gw.bytes())
        gw.check("workspace")
        go.check("out")
        gl.check("lse")


GQA = [
    Workload("c_gqa_g4", torch.bfloat16, 2, 8, 128, 128 * 3 + 5, kv_heads=2, seed=96),
    Workload("c_mqa_g32", torch.bfloat16, 1, 32, 128, 1000, kv_heads=1, alibi=True, seed=97),
    Workload("c_gqa_d64", torch.float16, 2, 16, 64, 64 * 9 - 1, kv_heads=2, seed=98),
    Workload("c_gqa_ragged", torch.float16, 3, 12, 128, 900, kv_heads=3, ragged=(1, 900),
             seed=99),
]


@pytest.mark.parametrize("w", GQA, ids=lambda w: w.name)
@pytest.mark.parametrize("n_split", [0, 5])
def test_gqa_outputs_and_workspace_stay_in_bounds(w, n_split):
    inp = make_inputs(w, "cuda")
    B, Hq, D = w.B, w.H, w.D
    Hkv, N = inp["k"].shape[1], inp["k"].shape[2]
    go, gl = _outs(B, Hq, D)
    td.decode_gqa(inp["q"], inp["k"], inp["v"], seqlens=inp["seqlens"],
                  seqlens_host=inp["seqlens_host"], slopes=inp["slopes"], n_split=n_split,
                  out=go.f32(B, Hq, 1, D), lse=gl.f32(B, Hq, 1))
    td.check_device_error()
    go.check("gqa out")
    gl.check("gqa lse")
    total = -1 if inp["seqlens_host"] is None else int(inp["seqlens_host"].sum()) * Hkv
    parts = td.plan_parts_gqa(B, Hq, Hkv, N, D, w.dtype, n_split, total)
    gw = Guarded(td.gqa_workspace_bytes(B, Hq, Hkv, D, parts), fill=0)
    go2, gl2 = _outs(B, Hq, D)
    td.decode_gqa_ws(inp["q"], inp["k"], inp["v"], gw.bytes(), seqlens=inp["seqlens"],
                     seqlens_host=inp["seqlens_host"], parts=parts, slopes=inp["slopes"],
                     out=go2.f32(B, Hq, 1, D), lse=gl2.f32(B, Hq, 1))
    td.check_device_error(gw.bytes())
    gw.check("gqa workspace")
    go2.check("gqa_ws out")
    gl2.check("gqa_ws lse")
    _check_finite(go2.f32(B, Hq, 1, D))


@pytest.mark.parametrize("n_split", [0, 4])
def test_fp8_outputs_stay_in_bounds(n_split):
    w = Workload("c_fp8", torch.bfloat16, 2, 4, 128, 64 * 4 + 3, kv_fp8=True, alibi=True,
                 seed=100)
    inp = make_inputs(w, "cuda")
    go, gl = _outs(w.B, w.H, w.D)
    td.decode_fp8(inp["q"], inp["k"], inp["v"], inp["k_scale"], inp["v_scale"],
                  slopes=inp["slopes"], n_split=n_split, out=go.f32(w.B, w.H, 1, w.D),
                  lse=gl.f32(w.B, w.H, 1))
    td.check_device_error()
    go.check("fp8 out")
    gl.check("fp8 lse")


@pytest.mark.parametrize("S,D,causal,alibi", [(129, 128, True, False), (255, 64, True, True),
                                              (200, 128, False, False)])
def test_prefill_outputs_stay_in_bounds(S, D, causal, alibi):
    w = Workload("c_prefill", torch.bfloat16, 2, 2, D, S, prefill=True, alibi=alibi,
                 causal=causal, seed=101)
    inp = make_inputs(w, "cuda")
    go, gl = _outs(w.B, w.H, D, rows=S)
    td.prefill(inp["q"], inp["k"], inp["v"], causal=causal, slopes=inp["slopes"],
               out=go.f32(w.B, w.H, S, D), lse=gl.f32(w.B, w.H, S))
    td.check_device_error()
    go.check("prefill out")
    gl.check("prefill lse")
    _check_finite(go.f32(w.B, w.H, S, D))


def test_combine_shard_and_merge_outputs_stay_in_bounds():
    B, H, S, D = 2, 3, 5, 128
    g = torch.Generator(device="cuda").manual_seed(102)
    num = torch.randn((B, H, S, D), generator=g, device="cuda")
    m = torch.randn((B, H, S), generator=g, device="cuda")
    m[0, 0, 1] = float("-inf")
    l = torch.rand((B, H, S), generator=g, device="cuda") + 0.5
    l[0, 0, 1] = 0.0
    num[0, 0, 1] = 0.0
    go, gl = _outs(B, H, D)
    td.combine(num, m, l, out=go.f32(B, H, 1, D), lse=gl.f32(B, H, 1))
    go.check("combine out")
    gl.check("combine lse")

    w = Workload("c_shard", torch.bfloat16, B, H, D, 1000, alibi=True, seed=103)
    inp = make_inputs(w, "cuda")
    W = 3
    gs = [Guarded(td.state_floats(B, H, D) * 4) for _ in range(W)]
    bounds = [(0, 300), (300, 650), (650, 1000)]
    for (a, b), gd in zip(bounds, gs):
        k = inp["k"][:, :, a:b].contiguous()
        v = inp["v"][:, :, a:b].contiguous()
        td.decode_shard(inp["q"], k, v, a, w.N, state=gd.f32(td.state_floats(B, H, D)),
                        slopes=inp["slopes"])
    td.check_device_error()
    for gd in gs:
        gd.check("shard state")
    states = torch.stack([gd.f32(td.state_floats(B, H, D)) for gd in gs])
    go2, gl2 = _outs(B, H, D)
    td.merge_shards(states, B, H, D, out=go2.f32(B, H, 1, D), lse=gl2.f32(B, H, 1))
    go2.check("merge out")
    gl2.check("merge lse")


def test_static_entry_outputs_stay_in_bounds():
    w = Workload("c_static", torch.float16, 3, 5, 64, 64 * 7 + 1, alibi=True, seed=104)
    inp = make_inputs(w, "cuda")
    go, gl = _outs(w.B, w.H, w.D)
    for n_split in (0, 3):
        td.decode_static(inp["q"], inp["k"], inp["v"], slopes=inp["slopes"], n_split=n_split,
                         out=go.f32(w.B, w.H, 1, w.D), lse=gl.f32(w.B, w.H, 1))
        td.check_static_error()
        go.check("static out")
        gl.check("static lse")
