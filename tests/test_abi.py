"""The C-ABI library: it loads, exports every declared entry point, and its
host-side logic (validation, split heuristic, workspace sizing) behaves --
all without a GPU and without launching anything."""
import ctypes
import math
import os
import re

import pytest
import torch

import long_context_attention_td_b200 as td
from long_context_attention_td_b200 import build as tdbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "treedec.h")

INVALID, UNSUPPORTED = 1, 2


@pytest.fixture(scope="module")
def L():
    tdbuild.build()
    return td.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(td_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("td_decode", "td_decode_varlen", "td_decode_ws", "td_combine",
                     "td_auto_split", "td_workspace_bytes", "td_status_string",
                     "td_last_cuda_error", "td_release_workspace"):
        assert required in names


def test_every_declared_symbol_is_exported(L):
    raw = ctypes.CDLL(td.library_path())
    for name in declared_functions():
        assert hasattr(raw, name), name


def test_library_is_built_for_sm100a_only():
    assert "arch=compute_100a,code=sm_100a" in " ".join(tdbuild.NVCC_FLAGS)


def test_status_strings(L):
    assert L.td_status_string(0) == b"ok"
    assert L.td_status_string(1) == b"invalid argument"
    assert L.td_status_string(6) == b"workspace too small"
    assert L.td_version() >= 100


FAKE = 0x10000  # never dereferenced: every call below fails validation first


def _decode(L, q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=0, B=1, H=1, N=16, D=128, n_split=0,
            slopes=0, dtype=1):
    return L.td_decode(q or None, k or None, v or None, out or None, lse or None, B, H, N, D,
                       n_split, slopes or None, dtype, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=0), INVALID), (dict(k=0), INVALID), (dict(v=0), INVALID), (dict(out=0), INVALID),
    (dict(B=0), INVALID), (dict(H=0), INVALID), (dict(N=0), INVALID), (dict(N=-5), INVALID),
    (dict(n_split=-1), INVALID),
    (dict(D=96), UNSUPPORTED), (dict(D=1024), UNSUPPORTED), (dict(dtype=7), UNSUPPORTED),
    (dict(q=FAKE + 8), INVALID), (dict(k=FAKE + 4), INVALID), (dict(v=FAKE + 2), INVALID),
    (dict(out=FAKE + 2), INVALID), (dict(lse=FAKE + 1), INVALID), (dict(slopes=FAKE + 2), INVALID),
    (dict(B=1 << 20, H=1 << 20, N=1 << 30), INVALID),
])
def test_decode_rejects_bad_arguments_before_any_launch(L, kw, expect):
    assert _decode(L, **kw) == expect


def test_varlen_and_ws_reject_bad_arguments(L):
    f = FAKE
    # seqlens required
    assert L.td_decode_varlen(f, f, f, f, None, 1, 1, 16, 128, None, None, 0, None, 1, None) == INVALID
    # seqlens_host out of range
    sh = (ctypes.c_int32 * 2)(4, 17)
    assert L.td_decode_varlen(f, f, f, f, None, 2, 1, 16, 128, f, sh, 0, None, 1, None) == INVALID
    sh = (ctypes.c_int32 * 2)(-1, 3)
    assert L.td_decode_varlen(f, f, f, f, None, 2, 1, 16, 128, f, sh, 0, None, 1, None) == INVALID
    # misaligned seqlens
    assert L.td_decode_varlen(f, f, f, f, None, 1, 1, 16, 128, f + 2, None, 0, None, 1, None) == INVALID
    # workspace required, parts >= 0
    assert L.td_decode_ws(f, f, f, f, None, 1, 1, 16, 128, None, None, 0, None, 1, None, 0, None) == INVALID
    assert L.td_decode_ws(f, f, f, f, None, 1, 1, 16, 128, None, None, -2, None, 1, f, 1 << 20, None) == INVALID


def test_combine_rejects_bad_arguments(L):
    f = FAKE
    assert L.td_combine(None, f, f, f, None, 1, 1, 4, 128, None) == INVALID
    assert L.td_combine(f, f, f, f, None, 1, 1, 0, 128, None) == INVALID
    assert L.td_combine(f, f, f, f, None, 1, 1, 4, 0, None) == INVALID
    assert L.td_combine(f, f, f, f, None, 1, 1, 4, 513, None) == INVALID
    assert L.td_combine(f, f, f + 1, f, None, 1, 1, 4, 128, None) == INVALID


def test_decode_host_rejects_bad_arguments(L):
    f = FAKE
    assert L.td_decode_host(None, f, f, f, None, 1, 1, 16, 128, None, 0, None, 1, None, 0) == INVALID
    assert L.td_decode_host(f, f, f, f, None, 1, 1, 16, 100, None, 0, None, 1, None, 0) == UNSUPPORTED


def test_auto_split_fills_the_gpu_and_respects_part_size(L):
    sms = 148
    # long sequences: one CTA per SM slot, regardless of B*H
    for (B, H, N) in ((1, 32, 131072), (8, 32, 32768), (1, 8, 1 << 20), (1, 1, 1 << 22)):
        P = L.td_auto_split(B, H, N, 128, 1, sms)
        assert P % sms == 0 and P >= sms
        assert L.td_auto_split(B, H, N, 128, 1, 2 * sms) == 2 * P
    # tiny problem: no part below 64 KiB of K+V, never more parts than keys, and
    # no more parts per sequence than keep its merge cheap: floor(sqrt(0.62 N elt))
    P = L.td_auto_split(1, 1, 4096, 512, 0, sms)  # fp32 D=512: 4 KiB per key
    assert P == int(math.sqrt(0.62 * 4096 * 4))      # 100, the measured optimum 64..128
    fill = L.td_auto_split(1, 1, 1 << 22, 512, 0, sms)  # long sequence: every CTA slot
    assert fill % sms == 0
    assert L.td_auto_split(4, 2, 4096, 512, 0, sms) == min(8 * 100, fill)
    # long sequences never reach the cap
    assert L.td_auto_split(1, 32, 131072, 128, 1, sms) == 3 * sms
    assert L.td_auto_split(1, 1, 3, 64, 2, sms) == 1
    assert L.td_auto_split(1, 1, 5, 64, 2, sms) <= 5
    for bad in ((0, 1, 1, 128, 1, sms), (1, 1, 0, 128, 1, sms), (1, 1, 8, 96, 1, sms),
                (1, 1, 8, 128, 9, sms), (1, 1, 8, 128, 1, 0)):
        assert L.td_auto_split(*bad) == -1


def test_workspace_bytes(L):
    # error region 256 B + tickets (B*H int32, 256-B padded) + 2 records per part
    assert L.td_workspace_bytes(1, 32, 128, 148) == 256 + 256 + 148 * 2 * 130 * 4
    assert L.td_workspace_bytes(64, 16, 64, 296) == 256 + 4096 + 296 * 2 * 66 * 4
    assert L.td_workspace_bytes(1, 1, 128, 0) == 0


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    monkeypatch.setattr(td, "_LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(td, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        td.lib()


def test_binding_rejects_host_tensors_for_device_calls():
    q = torch.zeros(1, 1, 1, 128, dtype=torch.bfloat16)
    k = torch.zeros(1, 1, 8, 128, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        td.decode(q, k, k)


def test_measurement_hooks_without_a_launch(L):
    # nothing launched from this thread yet in a CPU-only process
    if not torch.cuda.is_available():
        assert td.launch_count() == 0
        assert td.last_kernel() == ""
    ev = ctypes.c_void_p(0x1234)
    assert L.td_set_kernel_events(ev, None) == INVALID
    assert L.td_set_kernel_events(None, ev) == INVALID
    assert L.td_set_kernel_events(None, None) == 0


def test_shard_entry_points_reject_bad_arguments(L):
    p = ctypes.c_void_p(256)
    # keys past the end of the full sequence, negative offset, empty total
    assert L.td_decode_shard(p, p, p, p, 1, 1, 10, 128, 5, 12, 0, None, 1, None) == INVALID
    assert L.td_decode_shard(p, p, p, p, 1, 1, 10, 128, -1, 12, 0, None, 1, None) == INVALID
    assert L.td_decode_shard(p, p, p, p, 1, 1, 0, 128, 0, 0, 0, None, 1, None) == INVALID
    assert L.td_decode_shard(p, None, None, None, 1, 1, 0, 128, 0, 4, 0, None, 1, None) == INVALID
    # keys present but no k/v pointers
    assert L.td_decode_shard(p, None, p, p, 1, 1, 3, 128, 0, 4, 0, None, 1, None) == INVALID
    assert L.td_merge_shards(p, 0, 1, 1, 128, p, p, None) == INVALID
    assert L.td_merge_shards(p, 2, 1, 1, 1024, p, p, None) == INVALID
    assert L.td_merge_shards(None, 2, 1, 1, 128, p, p, None) == INVALID


def test_prefill_rejects_bad_arguments(L):
    p = ctypes.c_void_p(256)
    odd = ctypes.c_void_p(258)
    assert L.td_prefill(p, p, p, p, p, 1, 1, 128, 128, 1, None, 0, None) == UNSUPPORTED  # fp32
    assert L.td_prefill(p, p, p, p, p, 1, 1, 128, 96, 1, None, 1, None) == UNSUPPORTED   # D
    assert L.td_prefill(p, p, p, p, p, 1, 1, 0, 128, 1, None, 1, None) == INVALID        # S
    assert L.td_prefill(odd, p, p, p, p, 1, 1, 64, 128, 1, None, 1, None) == INVALID     # align
    assert L.td_prefill(None, p, p, p, p, 1, 1, 64, 128, 1, None, 1, None) == INVALID
    # key indices are 32-bit in the kernel: S may not come within 256 of 2^31
    assert L.td_prefill(p, p, p, p, p, 1, 1, 2**31 - 256, 128, 1, None, 1, None) == INVALID


def test_wait_test_settings_are_validated(L):
    # limits outside 1 us .. 10 s and tiles below -1 are refused
    assert L.td_set_wait_test(999, -1) == INVALID
    assert L.td_set_wait_test(10_000_000_001, -1) == INVALID
    assert L.td_set_wait_test(0, -2) == INVALID
    assert L.td_set_wait_test(1_000_000, 3) == 0
    assert L.td_set_wait_test(0, -1) == 0  # back to the defaults


def test_static_entry_rejects_bad_arguments_before_setup(L):
    p = ctypes.c_void_p(256)
    # unsupported D / dtype and bad sizes are refused before the scratch is touched
    assert L.td_decode_static(p, p, p, p, p, 1, 1, 16, 96, 0, None, 1, None) == UNSUPPORTED
    assert L.td_decode_static(p, p, p, p, p, 1, 1, 16, 128, 0, None, 7, None) == UNSUPPORTED
    assert L.td_decode_static(p, p, p, p, p, 0, 1, 16, 128, 0, None, 1, None) == INVALID
    assert L.td_decode_static(p, p, p, p, p, 1, 1, 16, 128, -1, None, 1, None) == INVALID


def test_host_decode_rejects_ragged_lengths_outside_the_padding(L):
    p = ctypes.c_void_p(256)
    lens = (ctypes.c_int32 * 2)(5, 17)   # 17 > N = 16
    assert L.td_decode_host(p, p, p, p, p, 2, 1, 16, 128, lens, 0, None, 1, None, 0) == INVALID
    lens = (ctypes.c_int32 * 2)(-1, 3)
    assert L.td_decode_host(p, p, p, p, p, 2, 1, 16, 128, lens, 0, None, 1, None, 0) == INVALID
