"""fp64 CPU oracle for exact decode attention and the chunked tree merge.

TEST INFRASTRUCTURE ONLY: imported by the tests, by the smoke check and by the
CPU-baseline leg of the benchmark, never by the product package.  The
arithmetic lives in ``td_oracle.c``; this module only marshals arrays.

Inputs are CPU ``torch`` tensors (float32, bfloat16 or float16: the exact bits
the GPU sees) or numpy float32/float16 arrays.  Results are numpy float64.

Sources (page title -- section):
  "Tree Attention Decoding" gist, tree_attn_decode.py -- regular_decode and
  tree_attn_decode (Algorithm 3); llm-foundry issue #186 "ALiBi with
  causal=True unexpected bias?" -- the broadcast bias row and causal masking;
  "Flash Aandacht" (unite.ai) -- "De Wiskunde Achter Flash Aandacht", formulas
  1 and 2, and the blockwise forward it describes (whose rows prefill computes).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_F32, _BF16, _F16, _F64 = 0, 1, 2, 3
_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        c_i64p = ctypes.POINTER(ctypes.c_int64)
        c_dp = ctypes.POINTER(ctypes.c_double)
        vp = ctypes.c_void_p
        L.or_decode_bf16.restype = ctypes.c_double
        L.or_decode_bf16.argtypes = [ctypes.c_uint16]
        L.or_decode_f16.restype = ctypes.c_double
        L.or_decode_f16.argtypes = [ctypes.c_uint16]
        L.or_decode_e4m3.restype = ctypes.c_double
        L.or_decode_e4m3.argtypes = [ctypes.c_uint8]
        L.or_alibi_bias.restype = ctypes.c_double
        L.or_alibi_bias.argtypes = [ctypes.c_double, ctypes.c_int64, ctypes.c_int64]
        L.or_attend_one.restype = ctypes.c_int
        L.or_attend_one.argtypes = [vp, vp, vp, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                                    ctypes.c_double, vp, vp, vp]
        L.or_chunk_bounds.restype = ctypes.c_int
        L.or_chunk_bounds.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, c_i64p]
        L.or_chunk_partial.restype = ctypes.c_int
        L.or_chunk_partial.argtypes = [vp, vp, vp, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                                       ctypes.c_double, ctypes.c_int64, ctypes.c_int64,
                                       vp, c_dp, c_dp]
        L.or_merge.restype = ctypes.c_int
        L.or_merge.argtypes = [vp, vp, vp, ctypes.c_int64, ctypes.c_int, vp, c_dp]
        common = [vp, vp, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64,
                  ctypes.c_int, vp, vp, vp, ctypes.c_int64]
        L.or_full.restype = ctypes.c_int
        L.or_full.argtypes = common + [vp, vp, ctypes.c_int]
        L.or_chunked.restype = ctypes.c_int
        L.or_chunked.argtypes = common + [ctypes.c_int, ctypes.c_int, vp, vp, ctypes.c_int]
        L.or_full_gqa.restype = ctypes.c_int
        L.or_full_gqa.argtypes = [vp, vp, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                  ctypes.c_int, ctypes.c_int64, ctypes.c_int, vp, vp, vp,
                                  ctypes.c_int64, vp, vp, ctypes.c_int]
        L.or_prefill.restype = ctypes.c_int
        L.or_prefill.argtypes = [vp, vp, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                 ctypes.c_int64, ctypes.c_int, ctypes.c_int, vp, vp,
                                 ctypes.c_int64, vp, vp, ctypes.c_int]
        _lib = L
    return _lib


def _code_and_buf(x):
    """(dtype code, contiguous CPU buffer object, address) for a tensor/array."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            t = x.detach()
            if t.device.type != "cpu":
                raise ValueError("oracle inputs must be CPU tensors")
            t = t.contiguous()
            code = {torch.float32: _F32, torch.bfloat16: _BF16, torch.float16: _F16,
                    torch.float64: _F64}.get(t.dtype)
            if code is None:
                raise TypeError("unsupported dtype %s" % t.dtype)
            return code, t, t.data_ptr()
    except ImportError:
        pass
    a = np.ascontiguousarray(x)
    code = {np.dtype(np.float32): _F32, np.dtype(np.float16): _F16,
            np.dtype(np.float64): _F64}.get(a.dtype)
    if code is None:
        raise TypeError("unsupported dtype %s" % a.dtype)
    return code, a, a.ctypes.data


def _ptr(a):
    return None if a is None else a.ctypes.data


def _check(rc, what):
    if rc != 0:
        raise RuntimeError("oracle %s failed with code %d" % (what, rc))


def _batched(fn_name, q, k, v, slopes, seqlens, bh, threads, extra=()):
    cq, tq, pq = _code_and_buf(q)
    ck, tk, pk = _code_and_buf(k)
    cv, tv, pv = _code_and_buf(v)
    if not (cq == ck == cv):
        raise TypeError("q, k, v must share one element type")
    B, H, _, D = tuple(tq.shape)
    Nmax = int(tk.shape[2])
    if tuple(tk.shape) != (B, H, Nmax, D) or tuple(tv.shape) != (B, H, Nmax, D):
        raise ValueError("layout must be q[B,H,1,D], k/v[B,H,N,D]")
    sl = None if slopes is None else np.ascontiguousarray(np.asarray(slopes, dtype=np.float32))
    sq = None if seqlens is None else np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
    bl = None if bh is None else np.ascontiguousarray(np.asarray(bh, dtype=np.int64))
    n_bh = B * H if bl is None else len(bl)
    out = np.zeros((n_bh, D), dtype=np.float64)
    lse = np.zeros((n_bh,), dtype=np.float64)
    fn = getattr(lib(), fn_name)
    rc = fn(pq, pk, pv, cq, B, H, Nmax, D, _ptr(sq), _ptr(sl), _ptr(bl), n_bh,
            *extra, out.ctypes.data, lse.ctypes.data, int(threads))
    _check(rc, fn_name)
    return out, lse


def full(q, k, v, slopes=None, seqlens=None, bh=None, threads=0):
    """Plain softmax decode attention in fp64 for the listed (b,h) pairs.

    q [B,H,1,D]; k, v [B,H,N,D]; slopes fp32 [H] or None; seqlens int32 [B] or
    None (ragged: sequence b uses its first seqlens[b] keys).  Returns
    (out [n_bh, D], lse [n_bh]), lse the absolute natural-log log-sum-exp.
    """
    return _batched("or_full", q, k, v, slopes, seqlens, bh, threads)


def full_gqa(q, k, v, slopes=None, seqlens=None, bh=None, threads=0):
    """Grouped-query plain decode: q [B,H,1,D], k/v [B,Hkv,N,D] with H a
    multiple of Hkv (query head h reads kv head h // (H // Hkv)); slopes [H].
    Returns (out [n_bh, D], lse [n_bh]) over the listed b*H+h (all by default)."""
    cq, tq, pq = _code_and_buf(q)
    ck, tk, pk = _code_and_buf(k)
    cv, tv, pv = _code_and_buf(v)
    if not (cq == ck == cv):
        raise TypeError("q, k, v must share one element type")
    B, H, _, D = tuple(tq.shape)
    Hkv, Nmax = int(tk.shape[1]), int(tk.shape[2])
    if tuple(tk.shape) != (B, Hkv, Nmax, D) or tuple(tv.shape) != (B, Hkv, Nmax, D):
        raise ValueError("layout must be q[B,H,1,D], k/v[B,Hkv,N,D]")
    sl = None if slopes is None else np.ascontiguousarray(np.asarray(slopes, dtype=np.float32))
    sq = None if seqlens is None else np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
    bl = None if bh is None else np.ascontiguousarray(np.asarray(bh, dtype=np.int64))
    n_bh = B * H if bl is None else len(bl)
    out = np.zeros((n_bh, D), dtype=np.float64)
    lse = np.zeros((n_bh,), dtype=np.float64)
    _check(lib().or_full_gqa(pq, pk, pv, cq, B, H, Hkv, Nmax, D, _ptr(sq), _ptr(sl), _ptr(bl),
                             n_bh, out.ctypes.data, lse.ctypes.data, int(threads)), "full_gqa")
    return out, lse


def prefill(q, k, v, causal=True, slopes=None, rows=None, threads=0):
    """Prefill attention of every query row (or the listed row indices
    (b*H + h)*S + i): q, k, v [B,H,S,D]; slope_h (j - S + 1) bias; causal mask
    j <= i when causal.  Returns (out [n_rows, D], lse [n_rows]) in fp64."""
    cq, tq, pq = _code_and_buf(q)
    ck, tk, pk = _code_and_buf(k)
    cv, tv, pv = _code_and_buf(v)
    if not (cq == ck == cv):
        raise TypeError("q, k, v must share one element type")
    B, H, S, D = tuple(tq.shape)
    if tuple(tk.shape) != (B, H, S, D) or tuple(tv.shape) != (B, H, S, D):
        raise ValueError("layout must be q, k, v [B,H,S,D]")
    sl = None if slopes is None else np.ascontiguousarray(np.asarray(slopes, dtype=np.float32))
    rl = None if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    n = B * H * S if rl is None else len(rl)
    out = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    _check(lib().or_prefill(pq, pk, pv, cq, B, H, S, D, 1 if causal else 0, _ptr(sl), _ptr(rl), n,
                            out.ctypes.data, lse.ctypes.data, int(threads)), "prefill")
    return out, lse


def chunked(q, k, v, n_chunks, mode="torch_chunk", slopes=None, seqlens=None, bh=None,
            threads=0):
    """The gist's Algorithm 3 with n_chunks chunks per (b,h), merged in fp64.

    mode "torch_chunk" follows k.chunk(world_size) (chunk size ceil(n/w));
    mode "balanced" uses chunk i = [floor(i n / w), floor((i+1) n / w)).
    """
    m = {"torch_chunk": 0, "balanced": 1}[mode]
    return _batched("or_chunked", q, k, v, slopes, seqlens, bh, threads,
                    extra=(int(n_chunks), m))


def attend_one(q, k, v, slope=0.0, extra_bias=None):
    """One query q[D] over one sequence k,v[n,D]; optional extra per-key term."""
    cq, tq, pq = _code_and_buf(q)
    ck, tk, pk = _code_and_buf(k)
    cv, tv, pv = _code_and_buf(v)
    if not (cq == ck == cv):
        raise TypeError("q, k, v must share one element type")
    D = int(tq.shape[-1])
    n = int(tk.shape[0])
    eb = None
    if extra_bias is not None:
        eb = np.ascontiguousarray(np.asarray(extra_bias, dtype=np.float64))
        if eb.shape != (n,):
            raise ValueError("extra_bias must have one value per key")
    out = np.zeros((D,), dtype=np.float64)
    lse = np.zeros((1,), dtype=np.float64)
    _check(lib().or_attend_one(pq, pk, pv, cq, n, D, float(slope), _ptr(eb),
                               out.ctypes.data, lse.ctypes.data), "attend_one")
    return out, float(lse[0])


def chunk_bounds(n, w, mode="torch_chunk"):
    starts = (ctypes.c_int64 * (w + 1))()
    _check(lib().or_chunk_bounds(int(n), int(w), {"torch_chunk": 0, "balanced": 1}[mode],
                                 starts), "chunk_bounds")
    return [int(x) for x in starts]


def chunk_partial(q, k, v, j0, j1, slope=0.0):
    """(num[D], local_max, den) of keys [j0, j1) of one sequence (gist form)."""
    cq, tq, pq = _code_and_buf(q)
    ck, tk, pk = _code_and_buf(k)
    cv, tv, pv = _code_and_buf(v)
    D = int(tq.shape[-1])
    n = int(tk.shape[0])
    num = np.zeros((D,), dtype=np.float64)
    m = ctypes.c_double()
    den = ctypes.c_double()
    _check(lib().or_chunk_partial(pq, pk, pv, cq, n, D, float(slope), int(j0), int(j1),
                                  num.ctypes.data, ctypes.byref(m), ctypes.byref(den)),
           "chunk_partial")
    return num, m.value, den.value


def merge(num, m, l):
    """Merge S partials: num [S,D], m [S], l [S] (natural-log units)."""
    num = np.ascontiguousarray(np.asarray(num, dtype=np.float64))
    m = np.ascontiguousarray(np.asarray(m, dtype=np.float64))
    l = np.ascontiguousarray(np.asarray(l, dtype=np.float64))
    S, D = num.shape
    out = np.zeros((D,), dtype=np.float64)
    lse = ctypes.c_double()
    _check(lib().or_merge(num.ctypes.data, m.ctypes.data, l.ctypes.data, S, D,
                          out.ctypes.data, ctypes.byref(lse)), "merge")
    return out, lse.value


def decode_bf16(bits):
    return lib().or_decode_bf16(int(bits))


def decode_f16(bits):
    return lib().or_decode_f16(int(bits))


def decode_e4m3(bits):
    return lib().or_decode_e4m3(int(bits))


def dequant_e4m3(x8, scales):
    """FP8 E4M3 cache [B,H,N,D] (uint8 bits) times per-head scales [H] as fp64
    (exact: a 4-bit by 24-bit significand product)."""
    lut = np.array([decode_e4m3(b) for b in range(256)], dtype=np.float64)
    a = np.asarray(x8.cpu() if hasattr(x8, "cpu") else x8)
    if a.dtype != np.uint8:
        raise TypeError("FP8 caches are passed as their uint8 bits")
    sc = np.asarray(scales.cpu() if hasattr(scales, "cpu") else scales, dtype=np.float32)
    return lut[a] * sc.astype(np.float64)[None, :, None, None]


def alibi_bias(slope, j, n):
    return lib().or_alibi_bias(float(slope), int(j), int(n))


def threads_used(threads=0):
    return threads if threads > 0 else (os.cpu_count() or 1)
