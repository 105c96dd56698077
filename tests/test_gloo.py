"""Multi-process paths on CPU ranks (gloo, world size 2 and 3).

1. The gist's own scheme ("Tree Attention Decoding", tree_attn_decode): every
   rank owns one chunk of the keys (k.chunk(world_size)), computes its
   (num, local_max, den) with the oracle, then all-reduce MAX, renormalise and
   two all-reduce SUMs -- the result must equal the plain definition.
2. bench.py's rank aggregation: max of the timed region over ranks, sum of the
   work, and one JSON line from rank 0 only.
3. The library's sequence-sharded decode (long_context_attention_td_b200.sharded):
   its plumbing on gloo ranks, with the oracle standing in for its two kernels.
"""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _init(rank, world, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))


def _gist_scheme(rank, world, port, n, D, slope, q, k, v, result):
    import oracle
    _init(rank, world, port)
    try:
        starts = oracle.chunk_bounds(n, world, "torch_chunk")
        j0, j1 = starts[rank], starts[rank + 1]
        num, m, den = oracle.chunk_partial(q, k, v, j0, j1, slope=slope)
        num = torch.from_numpy(num)
        gmax = torch.tensor([m], dtype=torch.float64)
        dist.all_reduce(gmax, op=dist.ReduceOp.MAX)
        r = math.exp(m - float(gmax)) if m != -math.inf else 0.0
        den_t = torch.tensor([den * r], dtype=torch.float64)
        num_t = num * r
        dist.all_reduce(den_t)
        dist.all_reduce(num_t)
        out = (num_t / den_t).numpy()
        if rank == 0:
            result.put((out.tolist(), float(gmax) + math.log(float(den_t))))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,n", [(2, 31), (3, 31), (2, 1)])
def test_gist_allreduce_scheme_on_cpu_ranks(world, n):
    import oracle
    D = 64
    g = torch.Generator().manual_seed(world * 100 + n)
    q = sum(torch.randn(D, generator=g) for _ in range(world))
    k = sum(torch.randn(n, D, generator=g) for _ in range(world))
    v = sum(torch.randn(n, D, generator=g) for _ in range(world))
    ctx = mp.get_context("spawn")
    result = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gist_scheme, args=(r, world, port, n, D, 0.25, q, k, v, result))
             for r in range(world)]
    for p in procs:
        p.start()
    out, lse = result.get(timeout=120)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    ref, ref_l = oracle.attend_one(q, k, v, slope=0.25)
    np.testing.assert_allclose(np.array(out), ref, rtol=0, atol=1e-12)
    assert abs(lse - ref_l) < 1e-12


def _bench_aggregate(rank, world, port, result):
    import bench
    _init(rank, world, port)
    try:
        ms = [3.0, 5.0, 4.0][rank]
        mx = bench.reduce_max(ms, "cpu")
        tot = bench.reduce_sum(100.0 * (rank + 1), "cpu")
        bench.barrier()
        result.put((rank, mx, tot))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_bench_takes_the_max_time_and_sums_work_over_ranks(world):
    ctx = mp.get_context("spawn")
    result = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bench_aggregate, args=(r, world, port, result))
             for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(result.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    expect_max = max([3.0, 5.0, 4.0][:world])
    expect_sum = sum(100.0 * (r + 1) for r in range(world))
    for rank, mx, tot in got:
        assert mx == expect_max and tot == expect_sum


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    bench.main(["--impl", "reference", "--steps", "3", "--warmup", "3"])
    assert capsys.readouterr().out == ""


# ------------------------------------------------ sequence-sharded decode

def _oracle_shard_state(q, k_s, v_s, off, n_total, slopes=None, n_split=0, stream=None):
    """td_decode_shard's contract computed by the oracle: each (b,h) attends
    its shard's keys with the ALiBi term of their place in the full sequence."""
    import oracle
    B, H, _, D = q.shape
    ns = k_s.shape[2]
    out = np.zeros((B * H, D))
    lse = np.full(B * H, -np.inf)
    for b in range(B):
        for h in range(H):
            if ns == 0:
                continue
            slope = 0.0 if slopes is None else float(slopes[h])
            extra = np.full(ns, slope * (off + ns - n_total))
            o, l = oracle.attend_one(q[b, h, 0], k_s[b, h], v_s[b, h], slope=slope,
                                     extra_bias=extra)
            out[b * H + h] = o
            lse[b * H + h] = l
    return torch.from_numpy(np.concatenate([out.ravel(), lse])).to(torch.float32)


def _oracle_merge(gathered, B, H, D, stream=None):
    import oracle
    W = gathered.shape[0]
    g = gathered.double().numpy()
    outs = g[:, : B * H * D].reshape(W, B * H, D)
    lses = g[:, B * H * D:]
    out = np.zeros((B * H, D))
    lse = np.zeros(B * H)
    for row in range(B * H):
        m = lses[:, row]
        o, l = oracle.merge(outs[:, row], m, np.isfinite(m).astype(np.float64))
        out[row], lse[row] = o, l
    return out, lse


def _sharded(rank, world, port, n, mode, alibi, result):
    from long_context_attention_td_b200 import sharded
    _init(rank, world, port)
    try:
        B, H, D = 2, 3, 32
        g = torch.Generator().manual_seed(7 + n)
        q = torch.randn(B, H, 1, D, generator=g)
        k = torch.randn(B, H, n, D, generator=g)
        v = torch.randn(B, H, n, D, generator=g)
        slopes = torch.tensor([0.5, 0.25, 0.125]) if alibi else None
        off, ln = sharded.shard_bounds(n, world, mode)[rank]
        out, lse = sharded.decode_sharded(q, k[:, :, off:off + ln], v[:, :, off:off + ln], off, n,
                                          slopes=slopes, shard_fn=_oracle_shard_state,
                                          merge_fn=_oracle_merge)
        result.put((rank, out.tolist(), lse.tolist()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,n,mode,alibi", [(2, 37, "torch_chunk", True), (3, 2, "torch_chunk", False),
                                                (3, 100, "balanced", True), (2, 1, "balanced", True)])
def test_sharded_decode_on_cpu_ranks(world, n, mode, alibi):
    """decode_sharded's plumbing -- chunk bounds, the packed state, the one
    all-gather in rank order, the merge -- on gloo ranks, with the two kernels
    replaced by the oracle computing their stated contracts; every rank must
    end with the plain definition over the whole sequence."""
    import oracle
    ctx = mp.get_context("spawn")
    result = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sharded, args=(r, world, port, n, mode, alibi, result))
             for r in range(world)]
    for p in procs:
        p.start()
    got = [result.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    B, H, D = 2, 3, 32
    g = torch.Generator().manual_seed(7 + n)
    q = torch.randn(B, H, 1, D, generator=g)
    k = torch.randn(B, H, n, D, generator=g)
    v = torch.randn(B, H, n, D, generator=g)
    slopes = np.array([0.5, 0.25, 0.125], dtype=np.float32) if alibi else None
    ref, ref_l = oracle.full(q, k, v, slopes=slopes)
    for _, out, lse in got:
        np.testing.assert_allclose(np.array(out), ref, rtol=0, atol=2e-6)
        np.testing.assert_allclose(np.array(lse), ref_l, rtol=0, atol=2e-6)


@pytest.mark.parametrize("n,world", [(0, 1), (1, 4), (5, 4), (31, 8), (4096, 8), (1000, 3)])
def test_shard_bounds_match_the_oracle_chunking(n, world):
    import oracle
    from long_context_attention_td_b200 import sharded
    for mode in ("torch_chunk", "balanced"):
        starts = oracle.chunk_bounds(n, world, mode)
        got = sharded.shard_bounds(n, world, mode)
        assert [(a, b - a) for a, b in zip(starts[:-1], starts[1:])] == got


def _oracle_varlen_state(q, k_s, v_s, lens, lens_host, n_split=0, stream=None):
    """The ragged shard state (td_decode_varlen on a rank's chunks) computed
    by the oracle: a chunk of length 0 gives the empty state (0, -inf)."""
    import oracle
    B, H, _, D = q.shape
    if k_s.shape[2] == 0:
        return torch.cat([torch.zeros(B * H * D), torch.full((B * H,), -math.inf)]).float()
    o, l = oracle.full(q, k_s, v_s, seqlens=lens_host)
    return torch.from_numpy(np.concatenate([o.ravel(), l])).to(torch.float32)


def _bench_sharded(rank, world, port, name, kw, result):
    import bench
    from long_context_attention_td_b200.workloads import WORKLOADS, make_inputs
    _init(rank, world, port)
    try:
        w = WORKLOADS[name].with_(**kw)
        inp = make_inputs(w, "cpu")
        ch = bench.shard_workload(inp, w, world, rank)
        out, lse = bench.sharded_step(ch, state_fn=_oracle_varlen_state,
                                      shard_fn=_oracle_shard_state, merge_fn=_oracle_merge)
        result.put((rank, ch["keys"], np.asarray(out).tolist(), np.asarray(lse).tolist()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,name,kw", [
    (2, "f16_ragged_b64_h16_d64", dict(B=5, H=2, N=40, ragged=(1, 40))),
    (3, "f16_ragged_b64_h16_d64", dict(B=4, H=3, N=9, ragged=(0, 9))),
    (2, "bf16_alibi_b8_h32_d128_n32k", dict(B=2, H=3, N=33)),
    (3, "bf16_h32_d128_n128k", dict(H=2, N=50)),
])
def test_bench_sharded_step_on_cpu_ranks(world, name, kw):
    """bench.py's multi-GPU step (each rank takes its chunk of every sequence
    with shard_workload, then decodes it, all-gathers the states and merges)
    on gloo ranks, with the oracle standing in for the kernels: every rank
    ends with the plain definition over the whole workload, and the chunks
    cover every attended key exactly once."""
    import oracle
    from long_context_attention_td_b200.workloads import WORKLOADS, kv_lengths, make_inputs
    ctx = mp.get_context("spawn")
    result = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bench_sharded, args=(r, world, port, name, kw, result))
             for r in range(world)]
    for p in procs:
        p.start()
    got = [result.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    w = WORKLOADS[name].with_(**kw)
    inp = make_inputs(w, "cpu")
    s = None if inp["slopes"] is None else inp["slopes"].numpy()
    ref, ref_l = oracle.full(inp["q"], inp["k"], inp["v"], slopes=s, seqlens=inp["seqlens_host"])
    assert sum(g[1] for g in got) == kv_lengths(w, inp["seqlens_host"])
    fin = np.isfinite(ref_l)
    for _, _, out, lse in got:
        out = np.array(out).reshape(ref.shape)
        lse = np.array(lse).reshape(-1)
        np.testing.assert_allclose(out, ref, rtol=0, atol=2e-6)
        np.testing.assert_allclose(lse[fin], ref_l[fin], rtol=0, atol=2e-6)
        assert np.all(lse[~fin] == -np.inf)
