"""td_decode_static: the decode entry point that allocates nothing.

Callers that cannot allocate device memory (an engine whose memory pool owns
nearly all HBM, a host application that owns a plug-in's allocations, a decode
loop that cannot take cudaMalloc's synchronisation) use this entry point; its
scratch is a fixed array inside the library.  Its results must match those of
td_decode, call after call, since every call reuses the same array.  This file
is collected last so a stop at its first failure has run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import long_context_attention_td_b200 as td
from long_context_attention_td_b200.workloads import Workload, make_inputs

from gpu_common import SPEC_LSE, SPEC_OUT

pytestmark = pytest.mark.gpu

TD_ERR_WORKSPACE = 6


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


CASES = [
    (Workload("static_bf16", torch.bfloat16, 2, 16, 128, 20000, seed=71), 0),
    (Workload("static_f16_alibi", torch.float16, 3, 4, 64, 5000, alibi=True, seed=72), 5),
    (Workload("static_f32_gist", torch.float32, 1, 1, 512, 4096, seed=73), 8),
]


@pytest.mark.parametrize("w,n_split", CASES, ids=[c[0].name for c in CASES])
def test_static_entry_matches_decode_on_two_calls(w, n_split):
    f = _entry()
    inp = make_inputs(w, "cuda")
    ref_out, ref_lse = td.decode(inp["q"], inp["k"], inp["v"], slopes=inp["slopes"],
                                 n_split=n_split)
    torch.cuda.synchronize()
    for _ in range(2):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        assert _call(f, inp, n_split, out, lse) == 0
        torch.cuda.synchronize()
        err_o = float((out.double() - ref_out.double()).abs().max())
        err_l = float((lse.double() - ref_lse.double()).abs().max())
        assert np.isfinite(err_o) and err_o <= SPEC_OUT[w.dtype], err_o
        assert np.isfinite(err_l) and err_l <= SPEC_LSE, err_l


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
