"""Benchmark of one decode step of libtreedec on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one decode call over the whole workload: td_decode /
td_decode_varlen (the split-KV kernel with its fused ticket combine, one
launch) for multi-head workloads, or td_decode_gqa (the tensor-core kernel,
plus the merge kernel when sequences are split over many CTAs) for
grouped-query ones.  Inputs are seeded synthetic tensors already resident in
HBM; the default workload (fp16, B=64, H=16, D=64, ragged lengths U[1024,
65536]) moves about 8.7 GB of K+V per step, far beyond the 126 MB L2, so no
flush is needed between steps (a workload whose K+V fit in L2 rotates over
enough copies of K and V to exceed twice the L2).  Prints one JSON line on
rank 0.

Under torchrun (N > 1 ranks) every sequence of the workload is split over the
ranks, the gist's own multi-GPU scheme: rank r decodes chunk r of the keys of
every sequence, the ranks exchange their partial states with one NCCL
all-gather and each merges them (strong scaling: the total work is fixed).
`--replicas` gives every rank its own copy of the workload instead
(independent problems, weak scaling, no data-path collective).

`--impl reference` times the fp64 CPU oracle on the host cores instead (rank 0
only), each step a bounded sample of the same workload.
"""
import argparse
import hashlib
import json
import math
import os
import re
import shutil
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from long_context_attention_td_b200.workloads import (WORKLOADS, kv_bytes, kv_lengths,  # noqa: E402
                                                      make_inputs, prefill_flops, seqlens_for)

METRIC = "decode attention KV GB/s and % of B200 HBM peak (1 GPU); µs per decode step"
PREFILL_METRIC = "prefill attention TFLOP/s (4 D FLOPs per visible query-key pair; 1 GPU)"
DEFAULT_WORKLOAD = "f16_ragged_b64_h16_d64"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
DTYPE_NAME = {torch.float32: "f32", torch.bfloat16: "bf16", torch.float16: "f16"}
# sources whose text decides each main kernel's code (its ncu summary is valid
# while their hash matches the one recorded in it)
KERNEL_SOURCES = {
    "td_partial_kernel": ["td_partial.cu", "td_device.cuh", "td_internal.cuh"],
    "td_gqa_keys_kernel": ["td_gqa_keys.cu", "td_tc.cuh", "td_device.cuh", "td_internal.cuh"],
    "td_prefill_kernel": ["td_prefill.cu", "td_tc.cuh", "td_device.cuh", "td_internal.cuh"],
}


L2_BYTES = 126 << 20


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def measured_tensor_peak():
    """Dense bf16 TFLOP/s measured by cuBLAS on this machine (burst), or the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (burst)"
    except Exception:
        return 1590.0, "fallback"


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash(kernel="td_partial_kernel"):
    h = hashlib.sha256()
    for s in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "long_context_attention_td_b200", "csrc", s), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload, kernel="td_partial_kernel"):
    """DRAM bytes per launch of `kernel` from the committed ncu summary of this
    workload (profiles/<kernel without _kernel>_<workload>.md), or None if
    absent or taken on other sources."""
    kernel = kernel.split(" ")[0]  # "td_partial_kernel (fp8 kv)" -> its source set
    if kernel not in KERNEL_SOURCES:
        return None
    path = os.path.join(ROOT, "profiles", "%s_%s.md" % (kernel[: -len("_kernel")], workload))
    try:
        text = open(path).read()
    except OSError:
        return None
    m_hash = re.search(r"kernel source hash:\s*`?([0-9a-f]{16})", text)
    m_bytes = re.search(r"dram bytes per launch:\s*([0-9]+)", text)
    if not m_hash or not m_bytes or m_hash.group(1) != kernel_source_hash(kernel):
        return None
    return int(m_bytes.group(1))


def traffic_record(workload, kernel):
    """(traffic, where it came from) for the roofline record: the DRAM bytes
    per launch of a committed ncu capture taken on the current kernel source,
    or (None, why not)."""
    t = profiled_traffic(workload, kernel)
    base = kernel.split(" ")[0] if kernel else ""
    name = "profiles/%s_%s.md" % (base[: -len("_kernel")], workload) if base else "-"
    if t is None:
        return None, "none: no ncu capture of %s on the current kernel source" % name
    return t, ("ncu dram__bytes_read.sum + dram__bytes_write.sum from %s (kernel source hash "
               "%s), not measured in this run" % (name, kernel_source_hash(base)))


# ------------------------------------------------------------------ clocks

_REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
                0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
                0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
                0x100: "display_clock_setting"}


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons every 200 ms."""

    def __init__(self, device_index):
        self.proc = None
        self.path = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            ident = str(device_index)
        self.ident = ident

    def start(self):
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active")
        self.dir = tempfile.mkdtemp(prefix="td_clocks_")
        self.path = os.path.join(self.dir, "clocks.csv")
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.ident, "--query-gpu=" + q,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def _cleanup(self):
        d = getattr(self, "dir", None)
        if d:
            shutil.rmtree(d, ignore_errors=True)

    def stop(self):
        if self.proc is None:
            self._cleanup()
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], None, set()
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 4:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
                bits = int(parts[3], 16)
            except ValueError:
                continue
            for b, n in _REASON_BITS.items():
                if bits & b and n != "gpu_idle":
                    reasons.add(n)
        self._cleanup()
        sm.sort()
        med = sm[len(sm) // 2] if sm else None
        return {"sm_mhz": med, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------ distributed

def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def reduce_max(x, device):
    """Max of a float over ranks (x itself when not distributed)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(x, device):
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def hbm_roofline(achieved, peak, peak_kind, kernel, bytes_per_launch, traffic, traffic_src):
    """The roofline record of an HBM-bound kernel.  `peak` is a copy rate
    (read + write bytes of a device-to-device copy); a read-only stream can
    run a few per cent above it, so frac may exceed 1: frac_of_nominal gives
    the share of the 8 TB/s data-sheet bandwidth beside it."""
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
            "peak_note": "%s device copy (read+write), the stated denominator; a read-only "
                         "stream can exceed it" % peak_kind,
            "frac_of_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
            "traffic": traffic, "traffic_source": traffic_src, "kernel": kernel,
            "algorithmic_bytes_per_launch": int(bytes_per_launch)}


def rotation_copies(bytes_step):
    """Copies of K and V the timed steps rotate over so that a workload whose
    K+V fit in L2 is read from HBM: enough that the steps between two uses of
    one copy read more than twice the L2."""
    if bytes_step >= 2 * L2_BYTES:
        return 1
    return min(64, -(-2 * L2_BYTES // max(bytes_step, 1)))


def is_shardable(w):
    """Workloads the sequence-sharded step takes: multi-head decode (uniform,
    or ragged without a positional bias)."""
    if w.prefill or w.kv_fp8 or (w.kv_heads and w.kv_heads != w.H):
        return False
    return not (w.ragged is not None and w.alibi)


def parallelism_name(world, sharded):
    return ("sequence-sharded x%d" % world) if sharded else ("replicas x%d" % world)


def workload_config(args, w, parallelism):
    """The `config` object both arms print for a workload: its shape and the
    L2 handling, all host arithmetic (the same on a box without a GPU)."""
    if w.prefill:
        return {"workload": args.workload + ("" if not args.n_keys else "@S=%d" % w.N),
                "B": w.B, "H": w.H, "D": w.D, "S": w.N, "causal": w.causal, "alibi": w.alibi,
                "flops_per_step": prefill_flops(w),
                "l2": "no flush: q, k, v, out per step %.2f GB > 126 MB L2"
                      % ((3 * 2 + 4) * w.B * w.H * w.N * w.D / 1e9),
                "parallelism": parallelism}
    n_split = w.n_split if args.n_split is None else args.n_split
    bytes_step = kv_bytes(w, seqlens_for(w))
    n_rot = rotation_copies(bytes_step)
    return {"workload": args.workload + ("" if not args.n_keys else "@N=%d" % w.N),
            "B": w.B, "H": w.H, "kv_heads": w.kv_heads or w.H, "D": w.D, "N": w.N,
            "ragged": w.ragged is not None, "alibi": w.alibi,
            "n_split": n_split if n_split else "auto", "bytes_per_step": int(bytes_step),
            "l2": ("no flush: K+V per step %.2f GB > 126 MB L2" % (bytes_step / 1e9)
                   if n_rot == 1 else
                   "no flush: steps rotate over %d copies of K+V (%.1f MB each, %.0f MB "
                   "in all > 2 x 126 MB L2)" % (n_rot, bytes_step / 1e6, n_rot * bytes_step / 1e6)),
            "parallelism": parallelism}


# -------------------------------------------------------------- CPU oracle

def oracle_rate_gqa(inp, w, budget_s, min_s=0.0, threads=0):
    """The same for grouped-query workloads: every query head of batch 0 over
    the first keys of its kv head, shortened to the time budget."""
    import oracle
    cores = os.cpu_count() or 1
    threads = threads or cores
    Hkv = w.kv_heads
    nk = max(1024, min(w.N, int(budget_s * 0.5e9 * min(threads, w.H) / (2 * w.D * w.elt * w.H))))
    q = inp["q"][:1].cpu()
    k = inp["k"][:1, :, :nk].cpu().contiguous()
    v = inp["v"][:1, :, :nk].cpu().contiguous()
    bytes_once = 2 * Hkv * nk * w.D * w.elt
    passes, t0 = 0, time.perf_counter()
    while True:
        oracle.full_gqa(q, k, v, threads=threads)
        passes += 1
        dt = time.perf_counter() - t0
        if dt >= min_s:
            break
    desc = ("%d query heads over %d kv heads x %d keys (%s, D=%d), %d pass(es), %d thread(s)"
            % (w.H, Hkv, nk, DTYPE_NAME[w.dtype], w.D, passes, min(threads, w.H)))
    return bytes_once * passes / dt / 1e9, min(threads, w.H), desc, dt


def oracle_rate_prefill(inp, w, budget_s, min_s=0.0, threads=0):
    """The fp64 oracle on the last query rows of head 0 (the most keys each),
    as many as fit the budget; returns (TFLOP/s, threads, description, s)."""
    import oracle
    cores = os.cpu_count() or 1
    threads = threads or cores
    S, D = w.N, w.D
    # ~1 GFLOP/s of fp64 per core on the plain loops
    n_rows = int(max(threads, min(S, budget_s * 1e9 * threads / (4.0 * D * S))))
    rows = list(range(S - n_rows, S))
    q, k, v = (inp[x][:1, :1].cpu().contiguous() for x in ("q", "k", "v"))
    sl = None if inp["slopes"] is None else inp["slopes"][:1].cpu()
    flops_once = sum(4.0 * D * ((r + 1) if w.causal else S) for r in rows)
    passes, t0 = 0, time.perf_counter()
    while True:
        oracle.prefill(q, k, v, causal=w.causal, slopes=sl, rows=rows, threads=threads)
        passes += 1
        dt = time.perf_counter() - t0
        if dt >= min_s:
            break
    desc = ("%d query rows (the last of head 0) of a %d-token %s prefill (%s, D=%d), %d pass(es), "
            "%d thread(s)" % (n_rows, S, "causal" if w.causal else "full", DTYPE_NAME[w.dtype],
                              D, passes, threads))
    return flops_once * passes / dt / 1e12, threads, desc, dt


def oracle_rate_fp8(inp, w, budget_s, min_s=0.0, threads=0):
    """The fp64 oracle on the first keys of every head of batch 0 of an FP8
    cache, dequantised (outside the timed region) to the fp64 values it
    stands for; GB/s counts the FP8 bytes those keys occupy."""
    import oracle
    cores = os.cpu_count() or 1
    threads = threads or cores
    H, D = w.H, w.D
    nk = max(1024, min(w.N, int(budget_s * 0.25e9 * min(threads, H) / (2 * D * H))))
    q = inp["q"][:1].double().cpu()
    K = torch.from_numpy(oracle.dequant_e4m3(inp["k"][:1, :, :nk].cpu(), inp["k_scale"]))
    V = torch.from_numpy(oracle.dequant_e4m3(inp["v"][:1, :, :nk].cpu(), inp["v_scale"]))
    bytes_once = 2 * H * nk * D  # one byte per FP8 element
    passes, t0 = 0, time.perf_counter()
    while True:
        oracle.full(q, K, V, threads=threads)
        passes += 1
        dt = time.perf_counter() - t0
        if dt >= min_s:
            break
    desc = ("%d heads x %d keys of an FP8 cache (D=%d, dequantised to fp64 before timing), "
            "%d pass(es), %d thread(s)" % (H, nk, D, passes, min(threads, H)))
    return bytes_once * passes / dt / 1e9, min(threads, H), desc, dt


def sampled_parity(inp, w, out, lse, n_rows=8):
    """The decode step's output against the fp64 oracle on sampled full-length
    (b, h) rows of the workload: max |out - oracle| and |lse - oracle| next to
    the bounds the parity tests hold them to (multi-head and grouped-query
    decode; None for the other kinds)."""
    import numpy as np
    import oracle
    if w.prefill or w.kv_fp8:
        return None
    B, H, D = w.B, w.H, w.D
    G = H // (w.kv_heads or H)
    lens = inp["seqlens_host"]
    rng = np.random.default_rng(7)
    picks = rng.choice(B * H, size=min(n_rows, B * H), replace=False)
    rows = sorted({0, B * H - 1} | set(int(x) for x in picks))
    q, k, v, slopes = inp["q"], inp["k"], inp["v"], inp["slopes"]
    eo, el, used, keys = 0.0, 0.0, 0, 0
    for r in rows:
        b, h = divmod(r, H)
        n_b = int(lens[b]) if lens is not None else w.N
        if n_b == 0:
            continue
        qs = q[b, h].reshape(1, 1, 1, D).cpu()
        ks = k[b, h // G, :n_b].reshape(1, 1, n_b, D).cpu()
        vs = v[b, h // G, :n_b].reshape(1, 1, n_b, D).cpu()
        s1 = None if slopes is None else slopes[h:h + 1].cpu()
        ro, rl = oracle.full(qs, ks, vs, slopes=s1)
        eo = max(eo, float(np.abs(out[b, h, 0].double().cpu().numpy() - ro[0]).max()))
        el = max(el, abs(float(lse[b, h, 0]) - float(rl[0])))
        used += 1
        keys += n_b
    bound = 1e-5 if w.dtype == torch.float32 else 2e-2
    return {"kind": "oracle", "rows": used, "keys": keys, "max_abs_out": eo, "max_abs_lse": el,
            "bound_out": bound, "bound_lse": 1e-4, "ok": bool(eo <= bound and el <= 1e-4)}


def oracle_rate(inp, w, budget_s, min_s=0.0, threads=0):
    """Time the fp64 oracle on (b,h) rows of a host copy of the workload;
    returns (GB/s, threads used, description, seconds)."""
    if w.prefill:
        return oracle_rate_prefill(inp, w, budget_s, min_s, threads)
    if w.kv_fp8:
        return oracle_rate_fp8(inp, w, budget_s, min_s, threads)
    if w.kv_heads and w.kv_heads != w.H:
        return oracle_rate_gqa(inp, w, budget_s, min_s, threads)
    import oracle
    B, H = w.B, w.H
    cores = os.cpu_count() or 1
    threads = threads or cores
    q, k, v = inp["q"], inp["k"], inp["v"]
    lens = inp["seqlens_host"]
    per_head = [int(lens[b]) if lens is not None else w.N for b in range(B) for _ in range(H)]
    # rows to time: one per thread, first (b,h) pairs, shortened so one pass
    # stays within the budget at ~0.5 GB/s per core
    n_rows = min(B * H, threads)
    est_rate = 0.5e9 * n_rows
    keys_cap = max(1024, int(budget_s * est_rate / (2 * w.D * w.elt * n_rows)))
    rows = list(range(n_rows))
    nk = min(max(per_head[r] for r in rows), keys_cap)
    qs = q.reshape(B * H, 1, 1, w.D)[rows].cpu()
    ks = k.reshape(B * H, 1, w.N, w.D)[rows, :, :nk].cpu()
    vs = v.reshape(B * H, 1, w.N, w.D)[rows, :, :nk].cpu()
    sl = None
    if lens is not None:
        sl = torch.tensor([min(per_head[r], nk) for r in rows], dtype=torch.int32)
    slopes = inp["slopes"]
    s1 = None if slopes is None else slopes.cpu()[[r % H for r in rows]]
    bytes_once = sum(2 * (min(per_head[r], nk)) * w.D * w.elt for r in rows)
    passes, t0 = 0, time.perf_counter()
    while True:
        if s1 is None:
            oracle.full(qs.view(len(rows), 1, 1, w.D), ks.view(len(rows), 1, nk, w.D),
                        vs.view(len(rows), 1, nk, w.D), seqlens=None if sl is None else sl,
                        threads=threads)
        else:
            # per-row slope: rows are independent sequences with H = 1
            for i in range(len(rows)):
                oracle.full(qs[i:i + 1], ks[i:i + 1], vs[i:i + 1], slopes=s1[i:i + 1],
                            seqlens=None if sl is None else sl[i:i + 1], threads=1)
        passes += 1
        dt = time.perf_counter() - t0
        if dt >= min_s:
            break
    rate = bytes_once * passes / dt / 1e9
    desc = ("%d (b,h) rows x %d keys (%s, D=%d), %d pass(es), %d thread(s)"
            % (len(rows), nk, DTYPE_NAME[w.dtype], w.D, passes, min(threads, len(rows))))
    return rate, min(threads, len(rows)), desc, dt


# -------------------------------------------------------------- our arm

def run_ours(args):
    import long_context_attention_td_b200 as td

    world, rank, local = dist_setup(args.gpus)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    w = w.with_(seed=w.seed + 1000 * rank)
    if args.n_keys:
        w = w.with_(N=args.n_keys)
    inp = make_inputs(w, dev)
    q, k, v = inp["q"], inp["k"], inp["v"]
    n_split = w.n_split if args.n_split is None else args.n_split
    stream = torch.cuda.current_stream(dev)
    B, H, D, N = w.B, w.H, w.D, w.N
    total_keys = kv_lengths(w, inp["seqlens_host"])
    gqa = bool(w.kv_heads) and w.kv_heads != w.H
    if gqa:
        parts = td.plan_parts_gqa(B, H, w.kv_heads, N, D, w.dtype, n_split,
                                  total_keys if inp["seqlens"] is not None else -1)
    else:
        parts = td.plan_parts(B, H, N, D, w.dtype, n_split,
                              total_keys if inp["seqlens"] is not None else -1)

    bytes_step = kv_bytes(w, inp["seqlens_host"])
    # a step whose K and V fit in L2 would be timed from L2: rotate over enough
    # distinct copies of K and V that the steps between two uses of one copy
    # read more than twice the L2
    n_rot = rotation_copies(bytes_step)
    kv_sets = [(k, v)] + [(k.clone(), v.clone()) for _ in range(n_rot - 1)]
    step_no = [0]

    def step():
        k, v = kv_sets[step_no[0] % n_rot]
        step_no[0] += 1
        if w.kv_fp8:
            td.decode_fp8(q, k, v, inp["k_scale"], inp["v_scale"], seqlens=inp["seqlens"],
                          seqlens_host=inp["seqlens_host"], slopes=inp["slopes"],
                          n_split=n_split, out=out, lse=lse, stream=stream)
        elif gqa:
            td.decode_gqa(q, k, v, seqlens=inp["seqlens"], seqlens_host=inp["seqlens_host"],
                          slopes=inp["slopes"], n_split=n_split, out=out, lse=lse, stream=stream)
        elif inp["seqlens"] is not None:
            td.decode_varlen(q, k, v, inp["seqlens"], seqlens_host=inp["seqlens_host"],
                             slopes=inp["slopes"], n_split=n_split, out=out, lse=lse,
                             stream=stream)
        else:
            td.decode(q, k, v, slopes=inp["slopes"], n_split=n_split, out=out, lse=lse,
                      stream=stream)

    out = torch.empty((B, H, 1, D), dtype=torch.float32, device=dev)
    lse = torch.empty((B, H, 1), dtype=torch.float32, device=dev)

    sampler = ClockSampler(dev.index).start()
    t_load0 = time.perf_counter()
    for _ in range(args.warmup):
        step()
    td.check_device_error(stream=stream)
    barrier()
    torch.cuda.synchronize(dev)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    launches0 = td.launch_count()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    launches = td.launch_count() - launches0
    torch.cuda.synchronize(dev)
    barrier()
    ms_total = ev0.elapsed_time(ev1)
    kernel_name = td.last_kernel()
    # keep the GPU loaded until the clock sampler has seen >= 1 s of load
    while time.perf_counter() - t_load0 < 1.2:
        for _ in range(20):
            step()
        torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    td.check_device_error(stream=stream)

    # the dominant kernel of the step, launch by launch: the library records
    # the events on its stream right around that kernel
    n_kt = min(args.steps, 50)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n_kt)]
    with torch.cuda.stream(stream):
        for a, b in evs:
            td.set_kernel_events(a, b)
            step()
        td.set_kernel_events(None, None)
    torch.cuda.synchronize(dev)
    kernel_ms = sum(a.elapsed_time(b) for a, b in evs) / n_kt

    ms_max = reduce_max(ms_total, dev)
    bytes_all = reduce_sum(float(bytes_step) * args.steps, dev)
    kernel_ms_max = reduce_max(kernel_ms, dev)
    ms_per_step = ms_max / args.steps
    value = bytes_all / (ms_max * 1e-3) / 1e9
    per_gpu = bytes_step / (ms_per_step * 1e-3) / 1e9

    # end to end through the host-buffer entry point (pinned host inputs)
    e2e = None
    if not args.no_e2e and not gqa and not w.kv_fp8:
        def pinned(t):
            h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
            h.copy_(t)
            return h

        qh, kh, vh = pinned(q), pinned(k), pinned(v)
        sh = inp["seqlens_host"]
        slh = None if inp["slopes"] is None else inp["slopes"].cpu()
        oh = torch.empty((B, H, 1, D), dtype=torch.float32).pin_memory()
        lh = torch.empty((B, H, 1), dtype=torch.float32).pin_memory()
        e2e_steps = max(3, min(args.steps, args.e2e_steps))
        for _ in range(2):
            td.decode_host(qh, kh, vh, seqlens=sh, slopes=slh, n_split=n_split, out=oh, lse=lh,
                           stream=stream, sync=True)
        barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            td.decode_host(qh, kh, vh, seqlens=sh, slopes=slh, n_split=n_split, out=oh, lse=lh,
                           stream=stream, sync=False)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        e_ms = reduce_max(e0.elapsed_time(e1), dev)
        e_bytes = reduce_sum(float(bytes_step) * e2e_steps, dev)
        # what td_decode_host copies in: q, the attended K and V rows (all of
        # them, or the first seqlens[b] of each (b,h) of a ragged batch), the
        # slopes and the lengths
        h2d = qh.numel() * qh.element_size() + 2 * total_keys * D * w.elt
        h2d += 0 if slh is None else slh.numel() * 4
        h2d += 0 if sh is None else sh.numel() * 4
        d2h = oh.numel() * 4 + lh.numel() * 4
        e2e = {"value": round(e_bytes / (e_ms * 1e-3) / 1e9, 3), "unit": "GB/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": e2e_steps, "ms_per_step": round(e_ms / e2e_steps, 4),
               "entry_point": "td_decode_host"}
        del qh, kh, vh

    peak, peak_kind = measured_peak()
    achieved = bytes_step / (kernel_ms_max * 1e-3) / 1e9
    traffic, traffic_src = traffic_record(args.workload, kernel_name)
    roofline = hbm_roofline(achieved, peak, peak_kind, kernel_name, bytes_step, traffic,
                            traffic_src)

    cpu = None
    parity = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, used, desc, dt = oracle_rate(inp, w, budget_s=2.0, min_s=args.cpu_seconds)
        cpu = {"value": round(rate, 4), "unit": "GB/s", "cores": used, "kind": "oracle",
               "sample": desc, "seconds": round(dt, 2), "host_cores": os.cpu_count()}
        try:
            parity = sampled_parity(inp, w, out, lse)
        except Exception as e:  # reported, never fatal to the measurement
            parity = {"error": str(e)[:200]}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 6),
            "us_per_step": round(ms_per_step * 1e3, 3),
            "pct_of_measured_hbm_peak": round(100 * per_gpu / peak, 2),
            "pct_of_nominal_8tbs": round(100 * per_gpu / NOMINAL_HBM_GBS, 2),
            "tokens_of_kv_per_s": round(total_keys * world / (ms_per_step * 1e-3), 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "input_dtype": (DTYPE_NAME[w.dtype] + " q, e4m3 k/v (f16 products)"
                                            if w.kv_fp8 else DTYPE_NAME[w.dtype]),
            "data": "synthetic",
            "config": workload_config(args, w.with_(seed=WORKLOADS[args.workload].seed),
                                      parallelism_name(world, False)),
            "launch": {"parts": parts},
            "gpu_launches": int(launches), "clocks": clocks, "roofline": roofline, "parity": parity,
            "e2e": e2e, "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------------ prefill

def run_prefill(args):
    """A step is one td_prefill call over the whole workload (one kernel)."""
    import long_context_attention_td_b200 as td

    world, rank, local = dist_setup(args.gpus)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    w = w.with_(seed=w.seed + 1000 * rank)
    if args.n_keys:
        w = w.with_(N=args.n_keys)
    inp = make_inputs(w, dev)
    q, k, v, slopes = inp["q"], inp["k"], inp["v"], inp["slopes"]
    stream = torch.cuda.current_stream(dev)
    out = torch.empty((w.B, w.H, w.N, w.D), dtype=torch.float32, device=dev)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    flops = prefill_flops(w)

    def step():
        td.prefill(q, k, v, causal=w.causal, slopes=slopes, out=out, lse=lse, stream=stream)

    sampler = ClockSampler(dev.index).start()
    t_load0 = time.perf_counter()
    for _ in range(args.warmup):
        step()
    td.check_device_error(stream=stream)
    barrier()
    torch.cuda.synchronize(dev)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    launches0 = td.launch_count()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    launches = td.launch_count() - launches0
    torch.cuda.synchronize(dev)
    barrier()
    ms_total = ev0.elapsed_time(ev1)
    while time.perf_counter() - t_load0 < 1.2:
        for _ in range(5):
            step()
        torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    td.check_device_error(stream=stream)
    n_kt = min(args.steps, 20)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n_kt)]
    with torch.cuda.stream(stream):
        for a, b in evs:
            td.set_kernel_events(a, b)
            step()
        td.set_kernel_events(None, None)
    torch.cuda.synchronize(dev)
    kernel_name = td.last_kernel()
    kernel_ms = reduce_max(sum(a.elapsed_time(b) for a, b in evs) / n_kt, dev)
    ms_max = reduce_max(ms_total, dev)
    ms_per_step = ms_max / args.steps
    flops_all = reduce_sum(flops * args.steps, dev)
    peak, peak_kind = measured_tensor_peak()
    achieved = flops / (kernel_ms * 1e-3) / 1e12
    traffic, tsrc = traffic_record(args.workload, kernel_name)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, used, desc, dt = oracle_rate_prefill(inp, w, budget_s=2.0, min_s=args.cpu_seconds)
        cpu = {"value": round(rate, 6), "unit": "TFLOP/s", "cores": used, "kind": "oracle",
               "sample": desc, "seconds": round(dt, 2), "host_cores": os.cpu_count()}
    if rank == 0:
        line = {
            "metric": PREFILL_METRIC, "value": round(flops_all / (ms_max * 1e-3) / 1e12, 2),
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 6), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16 in, fp32 accumulate",
            "input_dtype": DTYPE_NAME[w.dtype], "data": "synthetic",
            "config": workload_config(args, w, parallelism_name(world, False)),
            "gpu_launches": int(launches), "clocks": clocks,
            "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                         "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                         "peak_kind": peak_kind, "traffic": traffic, "traffic_source": tsrc,
                         "kernel": kernel_name, "algorithmic_flops_per_launch": flops},
            "e2e": None, "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------- sequence-sharded (strong scaling)

def shard_workload(inp, w, world, rank):
    """This rank's chunk of every sequence of a materialised workload (the
    balanced bounds of each sequence's length): a uniform workload keeps one
    key range for all (b,h) (td_decode_shard places ALiBi terms by it); a
    ragged one packs each sequence's chunk into [B,H,max chunk,D] with its
    chunk lengths (no positional bias)."""
    from long_context_attention_td_b200 import sharded
    B, H, D, N = w.B, w.H, w.D, w.N
    if inp["seqlens_host"] is not None:
        if inp["slopes"] is not None:
            raise SystemExit("a sharded ragged workload takes no ALiBi bias")
        offs, lens = sharded.ragged_shard(inp["seqlens_host"].tolist(), world, rank, "balanced")
        k = sharded.pack_ragged_shard(inp["k"], offs, lens)
        v = sharded.pack_ragged_shard(inp["v"], offs, lens)
        lens_host = torch.tensor(lens, dtype=torch.int32)
        return {"kind": "ragged", "q": inp["q"], "k": k, "v": v,
                "lens": lens_host.to(inp["q"].device), "lens_host": lens_host,
                "keys": int(sum(lens)) * H, "slopes": None}
    off, ln = sharded.shard_bounds(N, world, "balanced")[rank]
    k = inp["k"][:, :, off:off + ln].contiguous()
    v = inp["v"][:, :, off:off + ln].contiguous()
    return {"kind": "uniform", "q": inp["q"], "k": k, "v": v, "off": off, "n_total": N,
            "keys": B * H * ln, "slopes": inp["slopes"]}


def sharded_step(ch, n_split=0, stream=None, state_fn=None, shard_fn=None, merge_fn=None):
    """One sequence-sharded decode step of a rank on its chunk: the rank's
    partial state, one all-gather, the merge.  The kernels may be replaced
    by stand-ins (tests on CPU ranks)."""
    from long_context_attention_td_b200 import sharded
    if ch["kind"] == "ragged":
        return sharded.decode_sharded_varlen(ch["q"], ch["k"], ch["v"], ch["lens"],
                                             shard_lens_host=ch["lens_host"], n_split=n_split,
                                             stream=stream, state_fn=state_fn,
                                             merge_fn=merge_fn)
    return sharded.decode_sharded(ch["q"], ch["k"], ch["v"], ch["off"], ch["n_total"],
                                  slopes=ch["slopes"], n_split=n_split, stream=stream,
                                  shard_fn=shard_fn, merge_fn=merge_fn)


def run_sharded(args):
    """The gist's multi-GPU scheme (the default under torchrun, or --shard-seq):
    every sequence of the workload is split over the N ranks (rank r holds
    chunk r of its keys); a step is the rank's partial decode of its chunks
    (td_decode_shard, or td_decode_varlen for a ragged batch), one all-gather
    of the packed states and td_merge_shards.  The total work is fixed, so
    this is strong scaling."""
    import long_context_attention_td_b200 as td
    from long_context_attention_td_b200 import sharded

    world, rank, local = dist_setup(args.gpus)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    if (w.kv_heads and w.kv_heads != w.H) or w.prefill or w.kv_fp8:
        raise SystemExit("the sequence-sharded step takes a multi-head decode workload")
    if args.n_keys:
        w = w.with_(N=args.n_keys)
    # the same seed on every rank: every rank holds the same sequences and
    # keeps only its chunk of them (the full tensors stay for the parity check)
    inp = make_inputs(w, dev)
    ch = shard_workload(inp, w, world, rank)
    stream = torch.cuda.current_stream(dev)
    n_split = w.n_split if args.n_split is None else args.n_split
    B, H, D = w.B, w.H, w.D
    bytes_all = float(kv_bytes(w, inp["seqlens_host"]))
    shard_bytes = 2 * ch["keys"] * D * w.elt
    box = {}

    def step():
        box["out"] = sharded_step(ch, n_split, stream)

    sampler = ClockSampler(dev.index).start()
    t_load0 = time.perf_counter()
    for _ in range(args.warmup):
        step()
    td.check_device_error(stream=stream)
    barrier()
    torch.cuda.synchronize(dev)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    launches0 = td.launch_count()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    launches = td.launch_count() - launches0
    torch.cuda.synchronize(dev)
    barrier()
    ms_total = ev0.elapsed_time(ev1)
    out, lse = box["out"]
    out, lse = out.clone(), lse.clone()
    # keep the GPUs loaded until the clock sampler has seen >= 1 s of load;
    # every rank runs the same number of steps (each holds an all-gather)
    need_s = max(0.0, 1.2 - (time.perf_counter() - t_load0))
    n_more = int(reduce_max(float(min(20000, math.ceil(need_s / max(ms_total / args.steps * 1e-3,
                                                                      1e-6)))), dev))
    for _ in range(n_more):
        step()
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    td.check_device_error(stream=stream)
    # this rank's partial-decode kernel alone, launch by launch
    n_kt = min(args.steps, 50)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n_kt)]
    state = torch.empty(td.state_floats(B, H, D), dtype=torch.float32, device=dev)
    with torch.cuda.stream(stream):
        for a, b in evs:
            td.set_kernel_events(a, b)
            if ch["kind"] == "ragged":
                sharded._varlen_state(ch["q"], ch["k"], ch["v"], ch["lens"], ch["lens_host"],
                                      n_split, stream)
            else:
                td.decode_shard(ch["q"], ch["k"], ch["v"], ch["off"], ch["n_total"],
                                state=state, slopes=ch["slopes"], n_split=n_split,
                                stream=stream)
        td.set_kernel_events(None, None)
    torch.cuda.synchronize(dev)
    kernel_name = td.last_kernel()
    kernel_ms = reduce_max(sum(a.elapsed_time(b) for a, b in evs) / n_kt, dev)
    ms_max = reduce_max(ms_total, dev)
    ms_per_step = ms_max / args.steps

    # end to end through the same public call: this rank's chunk copied in
    # from pinned host memory every step, the result copied back
    e2e = None
    if not args.no_e2e:
        kh = torch.empty(ch["k"].shape, dtype=ch["k"].dtype, pin_memory=True)
        vh = torch.empty(ch["v"].shape, dtype=ch["v"].dtype, pin_memory=True)
        qh = torch.empty(ch["q"].shape, dtype=ch["q"].dtype, pin_memory=True)
        kh.copy_(ch["k"])
        vh.copy_(ch["v"])
        qh.copy_(ch["q"])
        oh = torch.empty((B, H, 1, D), dtype=torch.float32, pin_memory=True)
        lh = torch.empty((B, H, 1), dtype=torch.float32, pin_memory=True)
        e2e_steps = max(3, min(args.steps, args.e2e_steps))

        def e2e_step():
            with torch.cuda.stream(stream):
                ch["q"].copy_(qh, non_blocking=True)
                ch["k"].copy_(kh, non_blocking=True)
                ch["v"].copy_(vh, non_blocking=True)
                o, l = sharded_step(ch, n_split, stream)
                oh.copy_(o, non_blocking=True)
                lh.copy_(l.view(B, H, 1), non_blocking=True)

        e2e_step()
        barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        e_ms = reduce_max(e0.elapsed_time(e1), dev)
        h2d = reduce_sum(float(sum(t.numel() * t.element_size() for t in (qh, kh, vh))), dev)
        d2h = reduce_sum(float(oh.numel() * 4 + lh.numel() * 4), dev)
        e2e = {"value": round(bytes_all * e2e_steps / (e_ms * 1e-3) / 1e9, 3), "unit": "GB/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": e2e_steps, "ms_per_step": round(e_ms / e2e_steps, 4),
               "entry_point": "sharded.decode_sharded%s (chunks copied from pinned host "
                              "memory each step; bytes summed over ranks)"
                              % ("_varlen" if ch["kind"] == "ragged" else "")}
        del kh, vh, qh

    peak, peak_kind = measured_peak()
    achieved = shard_bytes / (kernel_ms * 1e-3) / 1e9 if shard_bytes else 0.0
    parity = None
    if rank == 0 and not args.no_cpu_baseline:
        try:
            parity = sampled_parity(inp, w, out, lse.view(B, H, 1))
        except Exception as e:  # reported, never fatal to the measurement
            parity = {"error": str(e)[:200]}
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(bytes_all / (ms_per_step * 1e-3) / 1e9, 3),
            "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 6), "us_per_step": round(ms_per_step * 1e3, 3),
            "tokens_of_kv_per_s": round(kv_lengths(w, inp["seqlens_host"]) /
                                        (ms_per_step * 1e-3), 1),
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f32",
            "input_dtype": DTYPE_NAME[w.dtype], "data": "synthetic",
            "config": workload_config(args, w, parallelism_name(world, True)),
            "launch": {"collective": "one all_gather of B*H*(D+1) fp32 per rank (NCCL)",
                       "rank_bytes_per_step": int(shard_bytes),
                       "rank_l2": "K+V per rank per step %.2f GB > 126 MB L2" % (shard_bytes / 1e9)},
            "gpu_launches": int(launches), "clocks": clocks,
            "roofline": hbm_roofline(achieved, peak, peak_kind, kernel_name, shard_bytes, None,
                                     "none: per-rank chunk, not captured"),
            "parity": parity, "e2e": e2e, "cpu_baseline": None,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# -------------------------------------------------------- reference arm

def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    if args.n_keys:
        w = w.with_(N=args.n_keys)
    sharded = world > 1 and not args.replicas and is_shardable(w)
    config = workload_config(args, w, parallelism_name(world, sharded or args.shard_seq))
    # the oracle's sample reads the first rows of the first batch entries only
    # (one per host core at most): generate just those entries on the host
    cores = os.cpu_count() or 1
    plain = not (w.prefill or w.kv_fp8 or (w.kv_heads and w.kv_heads != w.H))
    b_need = min(w.B, max(1, -(-cores // w.H))) if plain else 1
    inp = make_inputs(w.with_(B=b_need), "cpu")
    w = w.with_(B=b_need)
    # each step is a bounded sample so the whole run stays within ~2 minutes
    per_step_budget = max(0.002, 120.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_rate(inp, w, budget_s=per_step_budget)
    t0 = time.perf_counter()
    rates = []
    desc, used = "", 1
    for _ in range(args.steps):
        r, used, desc, _ = oracle_rate(inp, w, budget_s=per_step_budget)
        rates.append(r)
    dt = time.perf_counter() - t0
    value = sum(rates) / len(rates)
    metric, unit = (PREFILL_METRIC, "TFLOP/s") if w.prefill else (METRIC, "GB/s")
    line = {
        "metric": metric, "value": round(value, 6), "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * dt / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "input_dtype": DTYPE_NAME[w.dtype], "data": "synthetic", "impl": "reference",
        "config": config,
        "cpu_baseline": {"value": round(value, 6), "unit": unit, "cores": used,
                         "kind": "oracle", "sample": "per step: " + desc},
        "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--n-split", type=int, default=None)
    ap.add_argument("--n-keys", type=int, default=0,
                    help="override keys per sequence (smaller profiling captures)")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--shard-seq", action="store_true",
                    help="split every sequence over the ranks (one all-gather per step); "
                         "the default when more than one rank runs")
    ap.add_argument("--replicas", action="store_true",
                    help="with more than one rank, give every rank its own copy of the "
                         "workload (no data-path collective) instead of sharding it")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args)
    elif args.shard_seq or (world > 1 and is_shardable(w) and not args.replicas):
        run_sharded(args)
    elif WORKLOADS[args.workload].prefill:
        run_prefill(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
