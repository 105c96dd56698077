"""Seeded synthetic decode workloads (inputs only -- no attention arithmetic).

Every input of the tests and of the benchmark comes from here, so the CUDA
path and the fp64 oracle always see the same bits.  Recipe, per workload:

* values are drawn with ``torch.randn`` from a ``torch.Generator`` seeded with
  ``seed`` on the device the tensors live on, in fp32, in the fixed order
  q, k, v (k and v in slices of at most ``_SLICE`` elements along the
  flattened [B*H*N, D] rows), multiplied by ``scale`` and then rounded to the
  workload's element type;
* ALiBi slopes are the fp32 values 2^(-8(h+1)/H), h = 0..H-1;
* ragged lengths are ``torch.randint(lo, hi+1, (B,))`` from a CPU generator
  seeded with ``seed + 1``; keys at positions >= N_b of the padded [B,H,Nmax,D]
  buffers are filled like the rest but never read;
* "peaked" workloads pick, per (b,h), ``spikes`` distinct key positions with
  ``torch.randperm`` from a CPU generator seeded with ``seed + 2`` and set
  k_j <- 8 * ||k_j|| * q/||q|| (fp32, before rounding), so those keys score far
  above the rest (``spike_mode="aligned"``); ``spike_mode="scaled"`` takes
  the other reading of a key spiked to eight times its norm, k_j <- 8 * k_j in
  place, which keeps the random direction and so peaks the softmax far less.

The five named workloads are the shapes the decode kernel is measured on; any
field can be overridden (smaller N, B, H) for parity runs the oracle finishes
in seconds.
"""
from dataclasses import dataclass, replace
from typing import Optional, Tuple

import torch

_SLICE = 1 << 26


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: torch.dtype
    B: int
    H: int
    D: int
    N: int                      # keys per sequence (the padded Nmax when ragged)
    n_split: int = 0            # splits per (b,h); 0 = library heuristic
    alibi: bool = False
    ragged: Optional[Tuple[int, int]] = None   # inclusive [lo, hi] of N_b
    scale: float = 1.0
    spikes: int = 0
    spike_mode: str = "aligned"  # "aligned": 8||k|| q/||q||; "scaled": 8 k in place
    seed: int = 1234
    kv_heads: int = 0           # grouped-query: key/value heads (0 = H, plain multi-head)
    prefill: bool = False       # every query row of an N-token sequence (q, k, v [B,H,N,D])
    kv_fp8: bool = False        # K/V as FP8 E4M3 codes (uint8) with per-head fp32 scales
    causal: bool = True         # prefill: keys j <= i only

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def elt(self) -> int:
        """Bytes per K/V element."""
        if self.kv_fp8:
            return 1
        return torch.tensor([], dtype=self.dtype).element_size()


WORKLOADS = {
    # gist shape: one head, D=512, 4096 keys, split into 8 chunks, fp32
    "gist_f32_d512_n4k": Workload("gist_f32_d512_n4k", torch.float32, 1, 1, 512, 4096,
                                  n_split=8, seed=1234),
    # long-context bf16 decode, 32 heads, 128K keys, split count automatic
    "bf16_h32_d128_n128k": Workload("bf16_h32_d128_n128k", torch.bfloat16, 1, 32, 128,
                                    131072, seed=1235),
    # batched bf16 decode with the ALiBi broadcast row
    "bf16_alibi_b8_h32_d128_n32k": Workload("bf16_alibi_b8_h32_d128_n32k", torch.bfloat16,
                                            8, 32, 128, 32768, alibi=True, seed=1236),
    # 1M-key bf16 decode with a peaked softmax (16 spiked keys per head)
    "bf16_peaked_h8_d128_n1m": Workload("bf16_peaked_h8_d128_n1m", torch.bfloat16, 1, 8,
                                        128, 1 << 20, scale=0.5, spikes=16, seed=1237),
    # fp16 batched decode, ragged lengths U[1024, 65536], padded to 65536
    "f16_ragged_b64_h16_d64": Workload("f16_ragged_b64_h16_d64", torch.float16, 64, 16, 64,
                                       65536, ragged=(1024, 65536), seed=1238),
    # grouped-query decode (tensor cores): 32 query heads over 8 kv heads, 128K keys
    "gqa_bf16_h32_kv8_d128_n128k": Workload("gqa_bf16_h32_kv8_d128_n128k", torch.bfloat16, 1,
                                            32, 128, 131072, seed=1239, kv_heads=8),
    # multi-query decode: 32 query heads over one kv head, 1M keys
    "mqa_bf16_h32_kv1_d128_n1m": Workload("mqa_bf16_h32_kv1_d128_n1m", torch.bfloat16, 1, 32,
                                          128, 1 << 20, seed=1240, kv_heads=1),
    # grouped-query decode with D = 64: 32 query heads over 4 kv heads, 16 sequences of 64K keys
    "gqa_f16_b16_h32_kv4_d64_n64k": Workload("gqa_f16_b16_h32_kv4_d64_n64k", torch.float16, 16,
                                             32, 64, 65536, seed=1244, kv_heads=4),
    # multi-query decode with 48 query heads per kv head (more than 32 heads in one group)
    "mqa_bf16_h48_kv1_d128_n256k": Workload("mqa_bf16_h48_kv1_d128_n256k", torch.bfloat16, 1, 48,
                                            128, 1 << 18, seed=1246, kv_heads=1),
    # multi-query decode with 64 query heads (more than 32 heads in one group)
    "mqa_bf16_h64_kv1_d128_n256k": Workload("mqa_bf16_h64_kv1_d128_n256k", torch.bfloat16, 1, 64,
                                            128, 1 << 18, seed=1245, kv_heads=1),
    # the bench decode shape with an FP8 (E4M3) K/V cache and per-head scales
    "fp8kv_h32_d128_n128k": Workload("fp8kv_h32_d128_n128k", torch.bfloat16, 1, 32, 128, 131072,
                                     seed=1243, kv_fp8=True),
    # causal prefill of an 8K-token prompt, 32 heads (tensor cores)
    "prefill_bf16_h32_d128_s8k": Workload("prefill_bf16_h32_d128_s8k", torch.bfloat16, 1, 32,
                                          128, 8192, seed=1241, prefill=True),
    # batched causal prefill with the ALiBi row
    "prefill_bf16_alibi_b4_h16_d128_s4k": Workload("prefill_bf16_alibi_b4_h16_d128_s4k",
                                                   torch.bfloat16, 4, 16, 128, 4096, alibi=True,
                                                   seed=1242, prefill=True),
}


def alibi_slopes(H: int, device="cpu") -> torch.Tensor:
    """Per-head ALiBi slopes 2^(-8(h+1)/H) as fp32."""
    h = torch.arange(H, dtype=torch.float64)
    return torch.pow(2.0, -8.0 * (h + 1) / H).to(torch.float32).to(device)


def seqlens_for(w: Workload) -> Optional[torch.Tensor]:
    if w.ragged is None:
        return None
    lo, hi = w.ragged
    lo = min(lo, w.N)
    hi = min(hi, w.N)
    g = torch.Generator(device="cpu").manual_seed(w.seed + 1)
    return torch.randint(lo, hi + 1, (w.B,), generator=g, dtype=torch.int64).to(torch.int32)


def _randn_rows(gen, rows, D, device, scale, dtype):
    """[rows, D] of N(0,1)*scale in dtype, drawn in fp32 slices."""
    out = torch.empty((rows, D), dtype=dtype, device=device)
    step = max(1, _SLICE // D)
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        x = torch.randn((r1 - r0, D), generator=gen, device=device, dtype=torch.float32)
        if scale != 1.0:
            x.mul_(scale)
        out[r0:r1].copy_(x)
    return out


def make_gqa_inputs(w: Workload, Hkv: int, device="cpu"):
    """Grouped-query inputs: q [B, w.H, 1, D], k/v [B, Hkv, N, D] (same recipe
    as make_inputs, with the key/value tensors drawn for Hkv heads)."""
    device = torch.device(device)
    g = torch.Generator(device=device).manual_seed(w.seed)
    B, H, D, N = w.B, w.H, w.D, w.N
    qf = torch.randn((B, H, 1, D), generator=g, device=device, dtype=torch.float32)
    if w.scale != 1.0:
        qf.mul_(w.scale)
    q = qf.to(w.dtype)
    k = _randn_rows(g, B * Hkv * N, D, device, w.scale, w.dtype).view(B, Hkv, N, D)
    v = _randn_rows(g, B * Hkv * N, D, device, w.scale, w.dtype).view(B, Hkv, N, D)
    sl_host = seqlens_for(w)
    slopes = alibi_slopes(H, device) if w.alibi else None
    seqlens = sl_host.to(device) if sl_host is not None else None
    return dict(q=q, k=k, v=v, slopes=slopes, seqlens=seqlens, seqlens_host=sl_host)


def make_prefill_inputs(w: Workload, device="cpu"):
    """Prefill inputs: q, k, v [B, H, N, D] drawn like make_inputs (q first)."""
    device = torch.device(device)
    g = torch.Generator(device=device).manual_seed(w.seed)
    B, H, D, N = w.B, w.H, w.D, w.N
    q = _randn_rows(g, B * H * N, D, device, w.scale, w.dtype).view(B, H, N, D)
    k = _randn_rows(g, B * H * N, D, device, w.scale, w.dtype).view(B, H, N, D)
    v = _randn_rows(g, B * H * N, D, device, w.scale, w.dtype).view(B, H, N, D)
    slopes = alibi_slopes(H, device) if w.alibi else None
    return dict(q=q, k=k, v=v, slopes=slopes, seqlens=None, seqlens_host=None)


def prefill_flops(w: Workload) -> float:
    """Algorithmic FLOPs of a prefill: 4 D per visible (query, key) pair."""
    pairs = w.N * (w.N + 1) / 2 if w.causal else float(w.N) * w.N
    return 4.0 * w.D * pairs * w.B * w.H


E4M3_MAX = 448.0


def quantize_e4m3(x: torch.Tensor):
    """Per-head FP8 E4M3 codes of x [B,H,N,D] (fp32): scale_h = amax_h / 448,
    codes = round-to-nearest(x / scale_h), returned as their uint8 bits with the
    fp32 scales [H].  This prepares a cache the way a serving stack stores it;
    the attention arithmetic on it is the library's (and the oracle's)."""
    amax = x.abs().amax(dim=(0, 2, 3)).clamp_min(1e-30)
    scale = (amax / E4M3_MAX).to(torch.float32)
    y = (x / scale[None, :, None, None]).clamp(-E4M3_MAX, E4M3_MAX)
    return y.to(torch.float8_e4m3fn).view(torch.uint8), scale


def make_fp8_inputs(w: Workload, device="cpu"):
    """q [B,H,1,D] in w.dtype; k, v [B,H,N,D] FP8 E4M3 codes (uint8) drawn as
    N(0,1)*scale in fp32 then quantised per head; k_scale, v_scale [H]."""
    device = torch.device(device)
    g = torch.Generator(device=device).manual_seed(w.seed)
    B, H, D, N = w.B, w.H, w.D, w.N
    qf = torch.randn((B, H, 1, D), generator=g, device=device, dtype=torch.float32)
    if w.scale != 1.0:
        qf.mul_(w.scale)
    q = qf.to(w.dtype)
    kf = _randn_rows(g, B * H * N, D, device, w.scale, torch.float32).view(B, H, N, D)
    k, k_scale = quantize_e4m3(kf)
    del kf
    vf = _randn_rows(g, B * H * N, D, device, w.scale, torch.float32).view(B, H, N, D)
    v, v_scale = quantize_e4m3(vf)
    del vf
    sl_host = seqlens_for(w)
    slopes = alibi_slopes(H, device) if w.alibi else None
    seqlens = sl_host.to(device) if sl_host is not None else None
    return dict(q=q, k=k, v=v, k_scale=k_scale, v_scale=v_scale, slopes=slopes,
                seqlens=seqlens, seqlens_host=sl_host)


def make_inputs(w: Workload, device="cpu"):
    """Materialise a workload: dict(q, k, v, slopes, seqlens, seqlens_host)."""
    if w.kv_fp8:
        return make_fp8_inputs(w, device)
    if w.prefill:
        return make_prefill_inputs(w, device)
    if w.kv_heads and w.kv_heads != w.H:
        return make_gqa_inputs(w, w.kv_heads, device)
    device = torch.device(device)
    g = torch.Generator(device=device).manual_seed(w.seed)
    B, H, D, N = w.B, w.H, w.D, w.N
    qf = torch.randn((B, H, 1, D), generator=g, device=device, dtype=torch.float32)
    if w.scale != 1.0:
        qf.mul_(w.scale)
    q = qf.to(w.dtype)
    k = _randn_rows(g, B * H * N, D, device, w.scale, w.dtype).view(B, H, N, D)
    v = _randn_rows(g, B * H * N, D, device, w.scale, w.dtype).view(B, H, N, D)
    sl_host = seqlens_for(w)
    if w.spikes:
        gs = torch.Generator(device="cpu").manual_seed(w.seed + 2)
        for b in range(B):
            n_b = int(sl_host[b]) if sl_host is not None else N
            for h in range(H):
                pos = torch.randperm(n_b, generator=gs)[: min(w.spikes, n_b)].to(device)
                kj = k[b, h, pos].float()
                if w.spike_mode == "scaled":
                    k[b, h, pos] = (8.0 * kj).to(w.dtype)
                elif w.spike_mode == "aligned":
                    qd = qf[b, h, 0] / qf[b, h, 0].norm()
                    k[b, h, pos] = (8.0 * kj.norm(dim=-1, keepdim=True) * qd).to(w.dtype)
                else:
                    raise ValueError("spike_mode must be 'aligned' or 'scaled'")
    slopes = alibi_slopes(H, device) if w.alibi else None
    seqlens = sl_host.to(device) if sl_host is not None else None
    return dict(q=q, k=k, v=v, slopes=slopes, seqlens=seqlens, seqlens_host=sl_host)


def kv_lengths(w: Workload, seqlens_host: Optional[torch.Tensor]) -> int:
    """Sum over (b, kv head) of the keys actually read."""
    heads = w.kv_heads or w.H
    if seqlens_host is None:
        return w.B * heads * w.N
    return int(seqlens_host.to(torch.int64).sum()) * heads


def kv_bytes(w: Workload, seqlens_host: Optional[torch.Tensor]) -> int:
    """Algorithmic bytes of one decode step: every attended K and V row once."""
    return 2 * kv_lengths(w, seqlens_host) * w.D * w.elt
