"""Python binding of libtreedec (split-KV tree-decode attention on B200).

Argument marshalling only: every step of the decode runs in the library's CUDA
kernels, reached through the C ABI declared in include/treedec.h.  torch is
used for device memory and streams.  There is no fallback: if the compiled
library is missing, every call raises.

    import long_context_attention_td_b200 as td
    out, lse = td.decode(q, k, v)                 # q [B,H,1,D], k/v [B,H,N,D]
    out, lse = td.decode(q, k, v, slopes=alibi)   # ALiBi broadcast-row bias
    out, lse = td.decode_varlen(q, k, v, seqlens) # padded ragged batch
    out, lse = td.combine(num, m, l)              # merge caller partials
"""
import ctypes
import os

import torch

__all__ = [
    "TreeDecError", "lib", "library_path", "decode", "decode_varlen", "decode_ws", "combine",
    "auto_split", "plan_parts", "workspace_bytes", "decode_host", "check_device_error",
    "release_workspace", "DTYPE_CODE", "decode_gqa", "decode_gqa_ws", "plan_parts_gqa",
    "gqa_workspace_bytes", "decode_static", "check_static_error", "set_wait_test",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libtreedec.so")

DTYPE_CODE = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}
_STATUS = {0: "TD_OK", 1: "TD_ERR_INVALID_ARG", 2: "TD_ERR_UNSUPPORTED", 3: "TD_ERR_CUDA",
           4: "TD_ERR_NO_MEMORY", 5: "TD_ERR_DEVICE", 6: "TD_ERR_WORKSPACE"}


class TreeDecError(RuntimeError):
    def __init__(self, status, what, detail=""):
        self.status = status
        name = _STATUS.get(status, str(status))
        super().__init__("%s failed: %s%s" % (what, name, (" (%s)" % detail) if detail else ""))


_lib = None


def library_path():
    return _LIB_PATH


def lib():
    """The loaded libtreedec (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError("libtreedec.so is not built; run "
                           "`python -m long_context_attention_td_b200.build`")
    L = ctypes.CDLL(_LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    L.td_decode.restype = i32
    L.td_decode.argtypes = [vp, vp, vp, vp, vp, i32, i32, i64, i32, i32, vp, i32, vp]
    L.td_decode_varlen.restype = i32
    L.td_decode_varlen.argtypes = [vp, vp, vp, vp, vp, i32, i32, i64, i32, vp, vp, i32, vp,
                                   i32, vp]
    L.td_decode_ws.restype = i32
    L.td_decode_ws.argtypes = [vp, vp, vp, vp, vp, i32, i32, i64, i32, vp, vp, i64, vp, i32,
                               vp, sz, vp]
    L.td_decode_gqa.restype = i32
    L.td_decode_gqa.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i64, i32, vp, vp, i32, vp,
                                i32, vp]
    L.td_decode_gqa_ws.restype = i32
    L.td_decode_gqa_ws.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i64, i32, vp, vp, i64, vp,
                                   i32, vp, sz, vp]
    L.td_plan_parts_gqa.restype = i64
    L.td_plan_parts_gqa.argtypes = [i32, i32, i32, i64, i32, i32, i32, i64]
    L.td_gqa_workspace_bytes.restype = sz
    L.td_gqa_workspace_bytes.argtypes = [i32, i32, i32, i32, i64]
    L.td_combine.restype = i32
    L.td_combine.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, vp]
    L.td_auto_split.restype = i64
    L.td_auto_split.argtypes = [i32, i32, i64, i32, i32, i32]
    L.td_plan_parts.restype = i64
    L.td_plan_parts.argtypes = [i32, i32, i64, i32, i32, i32, i64]
    L.td_workspace_bytes.restype = sz
    L.td_workspace_bytes.argtypes = [i32, i32, i32, i64]
    L.td_decode_host.restype = i32
    L.td_decode_host.argtypes = [vp, vp, vp, vp, vp, i32, i32, i64, i32, vp, i32, vp, i32, vp,
                                 i32]
    L.td_check_device_error.restype = i32
    L.td_check_device_error.argtypes = [vp, sz, ctypes.POINTER(ctypes.c_int), vp]
    L.td_status_string.restype = ctypes.c_char_p
    L.td_status_string.argtypes = [i32]
    L.td_last_cuda_error.restype = i32
    L.td_last_cuda_error.argtypes = []
    L.td_release_workspace.restype = None
    L.td_release_workspace.argtypes = []
    L.td_version.restype = i32
    L.td_version.argtypes = []
    L.td_decode_shard.restype = i32
    L.td_decode_shard.argtypes = [vp, vp, vp, vp, i32, i32, i64, i32, i64, i64, i32, vp, i32, vp]
    L.td_merge_shards.restype = i32
    L.td_merge_shards.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp]
    L.td_decode_fp8.restype = i32
    L.td_decode_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i64, i32, vp, vp, i32, vp,
                                i32, vp]
    L.td_prefill.restype = i32
    L.td_prefill.argtypes = [vp, vp, vp, vp, vp, i32, i32, i64, i32, i32, vp, i32, vp]
    L.td_launch_count.restype = ctypes.c_uint64
    L.td_launch_count.argtypes = []
    L.td_set_kernel_events.restype = i32
    L.td_set_kernel_events.argtypes = [vp, vp]
    L.td_last_kernel.restype = ctypes.c_char_p
    L.td_last_kernel.argtypes = []
    L.td_decode_static.restype = i32
    L.td_decode_static.argtypes = [vp, vp, vp, vp, vp, i32, i32, i64, i32, i32, vp, i32, vp]
    L.td_check_static_error.restype = i32
    L.td_check_static_error.argtypes = [ctypes.POINTER(ctypes.c_int), vp]
    L.td_set_wait_test.restype = i32
    L.td_set_wait_test.argtypes = [ctypes.c_uint64, i64]
    _lib = L
    return L


def _check(st, what):
    if st != 0:
        detail = ""
        if st == 3:
            detail = "cudaError %d" % lib().td_last_cuda_error()
        raise TreeDecError(st, what, detail)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dev_tensor(t, name, dtype=None):
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise TypeError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must be %s" % (name, dtype))
    return t


def _shapes(q, k, v):
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("expected q [B,H,1,D], k and v [B,H,N,D]")
    B, H, one, D = q.shape
    if one != 1 or k.shape[:2] != (B, H) or k.shape[3] != D or v.shape != k.shape:
        raise ValueError("expected q [B,H,1,D], k and v [B,H,N,D]")
    if q.dtype != k.dtype or q.dtype != v.dtype or q.dtype not in DTYPE_CODE:
        raise TypeError("q, k, v must share one of float32, bfloat16, float16")
    return B, H, int(k.shape[2]), D


def _outputs(q, B, H, D, out, lse):
    if out is None:
        out = torch.empty((B, H, 1, D), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, 1), dtype=torch.float32, device=q.device)
    _dev_tensor(out, "out", torch.float32)
    _dev_tensor(lse, "lse", torch.float32)
    if out.numel() != B * H * D or lse.numel() != B * H:
        raise ValueError("out must hold B*H*D and lse B*H floats")
    return out, lse


def decode(q, k, v, *, slopes=None, n_split=0, out=None, lse=None, stream=None):
    """Decode attention: returns (out [B,H,1,D] fp32, lse [B,H,1] fp32)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev_tensor(t, n)
    B, H, N, D = _shapes(q, k, v)
    if slopes is not None:
        _dev_tensor(slopes, "slopes", torch.float32)
    out, lse = _outputs(q, B, H, D, out, lse)
    st = lib().td_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, N, D,
                         int(n_split), _ptr(slopes), DTYPE_CODE[q.dtype], _stream(stream))
    _check(st, "td_decode")
    return out, lse


def decode_fp8(q, k8, v8, k_scale, v_scale, *, seqlens=None, seqlens_host=None, slopes=None,
               n_split=0, out=None, lse=None, stream=None):
    """Decode over an FP8 E4M3 K/V cache: k8, v8 [B,H,Nmax,D] uint8 codes (or
    torch.float8_e4m3fn), dequantised per head by k_scale, v_scale fp32 [H];
    q [B,H,1,D] bf16 or fp16.  Returns (out [B,H,1,D], lse [B,H,1]) fp32."""
    k8 = k8.view(torch.uint8) if k8.dtype == torch.float8_e4m3fn else k8
    v8 = v8.view(torch.uint8) if v8.dtype == torch.float8_e4m3fn else v8
    _dev_tensor(q, "q")
    _dev_tensor(k8, "k8", torch.uint8)
    _dev_tensor(v8, "v8", torch.uint8)
    _dev_tensor(k_scale, "k_scale", torch.float32)
    _dev_tensor(v_scale, "v_scale", torch.float32)
    if q.dim() != 4 or k8.dim() != 4 or v8.dim() != 4 or k8.shape != v8.shape:
        raise ValueError("expected q [B,H,1,D], k8 and v8 [B,H,N,D]")
    B, H, _, D = q.shape
    N = int(k8.shape[2])
    if tuple(k8.shape) != (B, H, N, D) or q.shape[2] != 1:
        raise ValueError("expected q [B,H,1,D], k8 and v8 [B,H,N,D]")
    if k_scale.numel() != H or v_scale.numel() != H:
        raise ValueError("k_scale and v_scale hold one scale per head")
    if seqlens is not None:
        _dev_tensor(seqlens, "seqlens", torch.int32)
    sh = None if seqlens_host is None else seqlens_host.to(torch.int32).contiguous().cpu()
    if slopes is not None:
        _dev_tensor(slopes, "slopes", torch.float32)
    out, lse = _outputs(q, B, H, D, out, lse)
    st = lib().td_decode_fp8(_ptr(q), _ptr(k8), _ptr(v8), _ptr(k_scale), _ptr(v_scale),
                             _ptr(out), _ptr(lse), B, H, N, D, _ptr(seqlens), _ptr(sh),
                             int(n_split), _ptr(slopes), DTYPE_CODE[q.dtype], _stream(stream))
    _check(st, "td_decode_fp8")
    return out, lse


def decode_varlen(q, k, v, seqlens, *, seqlens_host=None, slopes=None, n_split=0, out=None,
                  lse=None, stream=None):
    """Ragged decode over padded k/v [B,H,Nmax,D]; seqlens int32 [B] on device."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev_tensor(t, n)
    B, H, N, D = _shapes(q, k, v)
    _dev_tensor(seqlens, "seqlens", torch.int32)
    sh = None
    if seqlens_host is not None:
        sh = seqlens_host.to(torch.int32).contiguous().cpu()
    if slopes is not None:
        _dev_tensor(slopes, "slopes", torch.float32)
    out, lse = _outputs(q, B, H, D, out, lse)
    st = lib().td_decode_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, N, D,
                                _ptr(seqlens), _ptr(sh), int(n_split), _ptr(slopes),
                                DTYPE_CODE[q.dtype], _stream(stream))
    _check(st, "td_decode_varlen")
    return out, lse


def decode_ws(q, k, v, workspace, *, seqlens=None, seqlens_host=None, parts=0, slopes=None,
              out=None, lse=None, stream=None):
    """Decode with a caller-owned (uint8 device) workspace and explicit parts."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev_tensor(t, n)
    B, H, N, D = _shapes(q, k, v)
    _dev_tensor(workspace, "workspace")
    if seqlens is not None:
        _dev_tensor(seqlens, "seqlens", torch.int32)
    sh = None if seqlens_host is None else seqlens_host.to(torch.int32).contiguous().cpu()
    if slopes is not None:
        _dev_tensor(slopes, "slopes", torch.float32)
    out, lse = _outputs(q, B, H, D, out, lse)
    nbytes = workspace.numel() * workspace.element_size()
    st = lib().td_decode_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, N, D,
                            _ptr(seqlens), _ptr(sh), int(parts), _ptr(slopes),
                            DTYPE_CODE[q.dtype], _ptr(workspace), nbytes, _stream(stream))
    _check(st, "td_decode_ws")
    return out, lse


def _gqa_shapes(q, k, v):
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("expected q [B,Hq,1,D], k and v [B,Hkv,N,D]")
    B, Hq, one, D = q.shape
    if one != 1 or k.shape[0] != B or k.shape[3] != D or v.shape != k.shape:
        raise ValueError("expected q [B,Hq,1,D], k and v [B,Hkv,N,D]")
    if q.dtype != k.dtype or q.dtype != v.dtype or q.dtype not in DTYPE_CODE:
        raise TypeError("q, k, v must share one of bfloat16, float16")
    return B, Hq, int(k.shape[1]), int(k.shape[2]), D


def decode_gqa(q, k, v, *, seqlens=None, seqlens_host=None, slopes=None, n_split=0, out=None,
               lse=None, stream=None):
    """Grouped-query decode (tensor cores): q [B,Hq,1,D], k/v [B,Hkv,N,D]."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev_tensor(t, n)
    B, Hq, Hkv, N, D = _gqa_shapes(q, k, v)
    if seqlens is not None:
        _dev_tensor(seqlens, "seqlens", torch.int32)
    sh = None if seqlens_host is None else seqlens_host.to(torch.int32).contiguous().cpu()
    if slopes is not None:
        _dev_tensor(slopes, "slopes", torch.float32)
    out, lse = _outputs(q, B, Hq, D, out, lse)
    st = lib().td_decode_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, N, D,
                             _ptr(seqlens), _ptr(sh), int(n_split), _ptr(slopes),
                             DTYPE_CODE[q.dtype], _stream(stream))
    _check(st, "td_decode_gqa")
    return out, lse


def decode_gqa_ws(q, k, v, workspace, *, seqlens=None, seqlens_host=None, parts=0, slopes=None,
                  out=None, lse=None, stream=None):
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev_tensor(t, n)
    B, Hq, Hkv, N, D = _gqa_shapes(q, k, v)
    _dev_tensor(workspace, "workspace")
    if seqlens is not None:
        _dev_tensor(seqlens, "seqlens", torch.int32)
    sh = None if seqlens_host is None else seqlens_host.to(torch.int32).contiguous().cpu()
    if slopes is not None:
        _dev_tensor(slopes, "slopes", torch.float32)
    out, lse = _outputs(q, B, Hq, D, out, lse)
    nbytes = workspace.numel() * workspace.element_size()
    st = lib().td_decode_gqa_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, N,
                                D, _ptr(seqlens), _ptr(sh), int(parts), _ptr(slopes),
                                DTYPE_CODE[q.dtype], _ptr(workspace), nbytes, _stream(stream))
    _check(st, "td_decode_gqa_ws")
    return out, lse


def plan_parts_gqa(B, Hq, Hkv, Nmax, D, dtype, n_split=0, total_keys=-1):
    return int(lib().td_plan_parts_gqa(int(B), int(Hq), int(Hkv), int(Nmax), int(D),
                                       DTYPE_CODE[dtype], int(n_split), int(total_keys)))


def gqa_workspace_bytes(B, Hq, Hkv, D, parts):
    return int(lib().td_gqa_workspace_bytes(int(B), int(Hq), int(Hkv), int(D), int(parts)))


def combine(num, m, l, *, out=None, lse=None, stream=None):
    """Merge partials num [B,H,S,D], m [B,H,S], l [B,H,S] (fp32, device)."""
    _dev_tensor(num, "num", torch.float32)
    _dev_tensor(m, "m", torch.float32)
    _dev_tensor(l, "l", torch.float32)
    if num.dim() != 4 or m.shape != num.shape[:3] or l.shape != num.shape[:3]:
        raise ValueError("expected num [B,H,S,D], m and l [B,H,S]")
    B, H, S, D = num.shape
    out, lse = _outputs(num, B, H, D, out, lse)
    st = lib().td_combine(_ptr(num), _ptr(m), _ptr(l), _ptr(out), _ptr(lse), B, H, S, D,
                          _stream(stream))
    _check(st, "td_combine")
    return out, lse


def auto_split(B, H, N, D, dtype, num_sms):
    return int(lib().td_auto_split(int(B), int(H), int(N), int(D), DTYPE_CODE[dtype],
                                   int(num_sms)))


def plan_parts(B, H, Nmax, D, dtype, n_split=0, total_keys=-1):
    return int(lib().td_plan_parts(int(B), int(H), int(Nmax), int(D), DTYPE_CODE[dtype],
                                   int(n_split), int(total_keys)))


def workspace_bytes(B, H, D, parts):
    return int(lib().td_workspace_bytes(int(B), int(H), int(D), int(parts)))


def decode_host(q, k, v, *, seqlens=None, slopes=None, n_split=0, out=None, lse=None,
                stream=None, sync=True):
    """Decode from HOST tensors (pinned for async copies) through td_decode_host.

    The library copies the inputs to device staging, decodes and copies out and
    lse back to the host tensors it returns."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        if t.device.type != "cpu" or not t.is_contiguous():
            raise TypeError("%s must be a contiguous host tensor" % n)
    B, H, N, D = _shapes(q, k, v)
    if out is None:
        out = torch.empty((B, H, 1, D), dtype=torch.float32, pin_memory=q.is_pinned())
    if lse is None:
        lse = torch.empty((B, H, 1), dtype=torch.float32, pin_memory=q.is_pinned())
    sq = None if seqlens is None else seqlens.to(torch.int32).contiguous()
    sl = None if slopes is None else slopes.to(torch.float32).contiguous().cpu()
    st = lib().td_decode_host(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, N, D,
                              _ptr(sq), int(n_split), _ptr(sl), DTYPE_CODE[q.dtype],
                              _stream(stream), 1 if sync else 0)
    _check(st, "td_decode_host")
    return out, lse


def check_device_error(workspace=None, stream=None):
    """Wait for the stream, then read and clear the kernels' error word."""
    bits = ctypes.c_int(0)
    ws = None if workspace is None else _ptr(workspace)
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().td_check_device_error(ws, nbytes, ctypes.byref(bits), _stream(stream))
    if st != 0:
        raise TreeDecError(st, "kernel", "error bits 0x%x" % bits.value)


def check_static_error(stream=None):
    """check_device_error for the fixed scratch array of decode_static."""
    bits = ctypes.c_int(0)
    st = lib().td_check_static_error(ctypes.byref(bits), _stream(stream))
    if st != 0:
        raise TreeDecError(st, "kernel (static scratch)", "error bits 0x%x" % bits.value)


def decode_static(q, k, v, *, slopes=None, n_split=0, out=None, lse=None, stream=None):
    """td_decode_static: decode whose scratch is a fixed array inside the
    library, so the call allocates no device memory (out/lse may be passed in
    for the same reason).  Calls that overlap on the GPU race on that array."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev_tensor(t, n)
    B, H, N, D = _shapes(q, k, v)
    if out is None:
        out = torch.empty((B, H, 1, D), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, 1), dtype=torch.float32, device=q.device)
    _dev_tensor(out, "out", torch.float32)
    _dev_tensor(lse, "lse", torch.float32)
    if slopes is not None:
        _dev_tensor(slopes, "slopes", torch.float32)
    st = lib().td_decode_static(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, N, D,
                                int(n_split), _ptr(slopes), DTYPE_CODE[q.dtype], _stream(stream))
    _check(st, "td_decode_static")
    return out, lse


def set_wait_test(wait_limit_ns=0, withhold_tile=-1):
    """td_set_wait_test: limit of the split-KV kernel's pipeline waits (0: the
    default 2 s) and the failure-path test's withheld tile (-1: off) for this
    thread's later decode calls."""
    _check(lib().td_set_wait_test(int(wait_limit_ns), int(withhold_tile)), "td_set_wait_test")


def prefill(q, k, v, *, causal=True, slopes=None, out=None, lse=None, stream=None):
    """Prefill attention of every query row: q, k, v [B,H,S,D] (bf16/fp16);
    returns out fp32 [B,H,S,D] and lse fp32 [B,H,S]."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev_tensor(t, n)
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must all be [B,H,S,D]")
    B, H, S, D = q.shape
    if out is None:
        out = torch.empty((B, H, S, D), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    _dev_tensor(out, "out", torch.float32)
    _dev_tensor(lse, "lse", torch.float32)
    if slopes is not None:
        _dev_tensor(slopes, "slopes", torch.float32)
    st = lib().td_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, S, D,
                          1 if causal else 0, _ptr(slopes), DTYPE_CODE[q.dtype], _stream(stream))
    _check(st, "td_prefill")
    return out, lse


def state_floats(B, H, D):
    """fp32 floats of one shard state (td_decode_shard)."""
    return B * H * (D + 1)


def decode_shard(q, k, v, key_offset, n_total, *, state=None, slopes=None, n_split=0,
                 stream=None):
    """One rank's part of a sequence-sharded decode: keys [key_offset,
    key_offset + N_shard) of sequences of n_total keys in k/v [B,H,N_shard,D].
    Returns the packed state (fp32 [B*H*(D+1)]: outputs, then log-sum-exps)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev_tensor(t, n)
    B, H, _, D = q.shape
    Ns = int(k.shape[2])
    if tuple(k.shape) != (B, H, Ns, D) or tuple(v.shape) != (B, H, Ns, D):
        raise ValueError("k/v must be [B,H,N_shard,D] with q [B,H,1,D]")
    if state is None:
        state = torch.empty(state_floats(B, H, D), dtype=torch.float32, device=q.device)
    _dev_tensor(state, "state", torch.float32)
    if state.numel() < state_floats(B, H, D):
        raise ValueError("state too small")
    if slopes is not None:
        _dev_tensor(slopes, "slopes", torch.float32)
    st = lib().td_decode_shard(_ptr(q), _ptr(k), _ptr(v), _ptr(state), B, H, Ns, D,
                               int(key_offset), int(n_total), int(n_split), _ptr(slopes),
                               DTYPE_CODE[q.dtype], _stream(stream))
    _check(st, "td_decode_shard")
    return state


def merge_shards(states, B, H, D, *, out=None, lse=None, stream=None):
    """Merge gathered shard states (fp32 [W, B*H*(D+1)]) into out [B,H,1,D],
    lse [B,H,1]."""
    _dev_tensor(states, "states", torch.float32)
    W = states.numel() // state_floats(B, H, D)
    if W < 1 or states.numel() != W * state_floats(B, H, D):
        raise ValueError("states must hold W whole shard states")
    if out is None:
        out = torch.empty((B, H, 1, D), dtype=torch.float32, device=states.device)
    if lse is None:
        lse = torch.empty((B, H, 1), dtype=torch.float32, device=states.device)
    st = lib().td_merge_shards(_ptr(states), W, B, H, D, _ptr(out), _ptr(lse), _stream(stream))
    _check(st, "td_merge_shards")
    return out, lse


def release_workspace():
    lib().td_release_workspace()


def launch_count():
    """Kernels launched so far by this thread's library calls."""
    return int(lib().td_launch_count())


def last_kernel():
    """Name of the main kernel of this thread's last library call."""
    return lib().td_last_kernel().decode()


def set_kernel_events(before=None, after=None):
    """Have later calls on this thread record the torch.cuda.Events `before` and
    `after` on their stream around their main attention kernel (None, None:
    stop).  Each event is recorded once here first so that it exists."""
    if (before is None) != (after is None):
        raise ValueError("give both events or neither")
    if before is None:
        _check(lib().td_set_kernel_events(None, None), "td_set_kernel_events")
        return
    for e in (before, after):
        if not e.cuda_event:
            e.record()
    _check(lib().td_set_kernel_events(ctypes.c_void_p(before.cuda_event),
                                      ctypes.c_void_p(after.cuda_event)),
           "td_set_kernel_events")
