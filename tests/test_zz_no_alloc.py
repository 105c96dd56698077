"""td_decode_static: the decode entry point that allocates nothing.

Callers that cannot allocate device memory (an engine whose memory pool owns
nearly all HBM, a host application that owns a plug-in's allocations, a decode
loop that cannot take cudaMalloc's synchronisation) use this entry point; its
scratch is a fixed array inside the library.  Every call reuses that array, so
its results are checked on two calls in a row, against the fp64 oracle and
against td_decode.  Its device errors are read with td_check_static_error.
This file is collected last so a stop at its first failure has run every
other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import long_context_attention_td_b200 as td
from long_context_attention_td_b200.workloads import Workload, make_inputs

from gpu_common import SPEC_LSE, SPEC_OUT, compare, oracle_all

pytestmark = pytest.mark.gpu

TD_ERR_WORKSPACE = 6
TD_ERR_DEVICE = 5
TD_DEVERR_WAIT_TIMEOUT = 0x1


def _entry():
    f = td.lib().td_decode_static
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    f.restype = i32
    f.argtypes = [vp, vp, vp, vp, vp, i32, i32, i64, i32, i32, vp, i32, vp]
    return f


def _call(f, inp, n_split, out, lse):
    q, k, v, sl = inp["q"], inp["k"], inp["v"], inp["slopes"]
    B, H, N, D = k.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return f(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, H, N, D,
             n_split, None if sl is None else sl.data_ptr(), td.DTYPE_CODE[q.dtype], stream)


def _static_error_bits():
    bits = ctypes.c_int(0)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = td.lib().td_check_static_error(ctypes.byref(bits), stream)
    return st, bits.value


CASES = [
    (Workload("static_bf16", torch.bfloat16, 2, 16, 128, 20000, seed=71), 0),
    (Workload("static_f16_alibi", torch.float16, 3, 4, 64, 5000, alibi=True, seed=72), 5),
    (Workload("static_f32_gist", torch.float32, 1, 1, 512, 4096, seed=73), 8),
]


@pytest.mark.parametrize("w,n_split", CASES, ids=[c[0].name for c in CASES])
def test_static_entry_matches_oracle_and_decode_on_two_calls(w, n_split):
    f = _entry()
    inp = make_inputs(w, "cuda")
    ref_o, ref_l = oracle_all(inp)
    dec_out, dec_lse = td.decode(inp["q"], inp["k"], inp["v"], slopes=inp["slopes"],
                                 n_split=n_split)
    torch.cuda.synchronize()
    for _ in range(2):
        out = torch.full_like(dec_out, float("nan"))
        lse = torch.full_like(dec_lse, float("nan"))
        assert _call(f, inp, n_split, out, lse) == 0
        torch.cuda.synchronize()
        compare(out, lse, ref_o, ref_l, np.arange(w.B * w.H), w.dtype)
        err_o = float((out.double() - dec_out.double()).abs().max())
        err_l = float((lse.double() - dec_lse.double()).abs().max())
        assert np.isfinite(err_o) and err_o <= SPEC_OUT[w.dtype], err_o
        assert np.isfinite(err_l) and err_l <= SPEC_LSE, err_l
    assert _static_error_bits() == (0, 0)


def test_static_entry_rejects_problems_beyond_its_scratch():
    f = _entry()
    w = Workload("static_big", torch.float32, 1, 1, 512, 100000, seed=74)
    inp = make_inputs(w, "cuda")
    out = torch.full((1, 1, 1, 512), float("nan"), device="cuda")
    lse = torch.full((1, 1, 1), float("nan"), device="cuda")
    # 2000 parts of D=512 need about 8 MB of part records: over the fixed array
    assert _call(f, inp, 2000, out, lse) == TD_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.isnan(out).all() and torch.isnan(lse).all()


@pytest.mark.parametrize("withhold_tile", [0, 2])
def test_static_entry_reports_a_wait_that_ran_out(withhold_tile):
    """A static call whose first CTA's loader stops issuing tiles: its next
    pipeline wait runs out after 1 ms, the error bit is readable through
    td_check_static_error, and the next static call is correct again."""
    f = _entry()
    w, n_split = CASES[0]
    inp = make_inputs(w, "cuda")
    ref_o, ref_l = oracle_all(inp)
    out = torch.empty((w.B, w.H, 1, w.D), dtype=torch.float32, device="cuda")
    lse = torch.empty((w.B, w.H, 1), dtype=torch.float32, device="cuda")
    td.set_wait_test(1_000_000, withhold_tile)
    try:
        assert _call(f, inp, n_split, out, lse) == 0
    finally:
        td.set_wait_test(0, -1)
    st, bits = _static_error_bits()
    assert st == TD_ERR_DEVICE and bits & TD_DEVERR_WAIT_TIMEOUT, (st, bits)
    assert _static_error_bits() == (0, 0)  # read and cleared
    for _ in range(2):
        assert _call(f, inp, n_split, out, lse) == 0
        torch.cuda.synchronize()
        compare(out, lse, ref_o, ref_l, np.arange(w.B * w.H), w.dtype)
    assert _static_error_bits() == (0, 0)
