"""Pins of the fp64 oracle to things other than itself (CPU only).

Each test names what it pins and where that fact comes from: values printed on
the pages (tests/golden), library routines (torch SDPA / logsumexp / chunk,
numpy float16), closed forms, invariants the pages state, and brute force.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_sections(name):
    sec, out = None, {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("["):
                sec = line.strip("[]")
                out[sec] = []
                continue
            out[sec].append([None if t == "X" else float(t) for t in line.split()])
    return out


def _rand(shape, dtype, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g, dtype=torch.float32) * scale).to(dtype)


def _sdpa_fp64(q, k, v, slope=0.0, n=None):
    """Library reference: torch SDPA on the exactly widened inputs (fp64).

    The bias is the broadcast row slope * arange(1 - n, 1) of the ALiBi thread.
    Returns (out[D], lse) with lse from torch.logsumexp of the biased scores.
    """
    q64, k64, v64 = q.double(), k.double(), v.double()
    n = k64.shape[0] if n is None else n
    bias = slope * torch.arange(1 - n, 1, dtype=torch.float64)
    out = torch.nn.functional.scaled_dot_product_attention(
        q64.view(1, 1, 1, -1), k64.view(1, 1, n, -1), v64.view(1, 1, n, -1),
        attn_mask=bias.view(1, 1, 1, n))
    s = (k64 @ q64) / math.sqrt(q64.shape[-1]) + bias
    return out.view(-1).numpy(), float(torch.logsumexp(s, 0))


# ------------------------------------------------------------------ decoders

def test_decode_bf16_exhaustive_vs_torch():
    bits = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16)
    ref = bits.view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.decode_bf16(b & 0xFFFF) for b in range(1 << 16)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_decode_f16_exhaustive_vs_numpy():
    ref = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16).view(np.float16).astype(np.float64)
    got = np.array([oracle.decode_f16(b) for b in range(1 << 16)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


# ------------------------------------------------------ plain definition pins

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("D", [1, 2, 4, 64, 128])
@pytest.mark.parametrize("n", [1, 2, 7, 33])
@pytest.mark.parametrize("slope", [0.0, 0.37])
def test_attend_one_vs_sdpa(dtype, D, n, slope):
    q = _rand((D,), dtype, 1 + D + n)
    k = _rand((n, D), dtype, 2 + D + n)
    v = _rand((n, D), dtype, 3 + D + n)
    out, lse = oracle.attend_one(q, k, v, slope=slope)
    ref, ref_lse = _sdpa_fp64(q, k, v, slope)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    assert abs(lse - ref_lse) < 1e-12


def test_brute_force_integer_inputs():
    """Tiny integer-valued cases against SDPA, every D in {1,2,4}, N in 1..16."""
    g = torch.Generator().manual_seed(7)
    for D in (1, 2, 4):
        for n in range(1, 17):
            q = torch.randint(-3, 4, (D,), generator=g).float()
            k = torch.randint(-3, 4, (n, D), generator=g).float()
            v = torch.randint(-5, 6, (n, D), generator=g).float()
            out, lse = oracle.attend_one(q, k, v)
            ref, ref_lse = _sdpa_fp64(q, k, v)
            np.testing.assert_allclose(out, ref, rtol=0, atol=1e-13)
            assert abs(lse - ref_lse) < 1e-13


def test_batched_full_matches_per_head_and_bh_subset():
    B, H, N, D = 2, 3, 40, 16
    q = _rand((B, H, 1, D), torch.bfloat16, 11)
    k = _rand((B, H, N, D), torch.bfloat16, 12)
    v = _rand((B, H, N, D), torch.bfloat16, 13)
    slopes = torch.tensor([0.5, 0.25, 0.125], dtype=torch.float32)
    out, lse = oracle.full(q, k, v, slopes=slopes)
    for b in range(B):
        for h in range(H):
            ref, ref_lse = _sdpa_fp64(q[b, h, 0], k[b, h], v[b, h], float(slopes[h]))
            np.testing.assert_allclose(out[b * H + h], ref, rtol=0, atol=1e-12)
            assert abs(lse[b * H + h] - ref_lse) < 1e-12
    sub = [5, 0, 3]
    o2, l2 = oracle.full(q, k, v, slopes=slopes, bh=sub, threads=2)
    np.testing.assert_array_equal(o2, out[sub])
    np.testing.assert_array_equal(l2, lse[sub])


def test_ragged_lengths_match_truncation_and_empty():
    B, H, N, D = 3, 2, 24, 8
    q = _rand((B, H, 1, D), torch.float16, 21)
    k = _rand((B, H, N, D), torch.float16, 22)
    v = _rand((B, H, N, D), torch.float16, 23)
    slopes = torch.tensor([0.3, 0.7], dtype=torch.float32)
    seqlens = [5, 24, 0]
    out, lse = oracle.full(q, k, v, slopes=slopes, seqlens=seqlens)
    for b in range(B):
        for h in range(H):
            i = b * H + h
            if seqlens[b] == 0:
                assert np.all(out[i] == 0.0) and lse[i] == -math.inf
                continue
            n = seqlens[b]
            ref, ref_lse = _sdpa_fp64(q[b, h, 0], k[b, h, :n], v[b, h, :n], float(slopes[h]))
            np.testing.assert_allclose(out[i], ref, rtol=0, atol=1e-12)
            assert abs(lse[i] - ref_lse) < 1e-12


# ---------------------------------------------------------- closed forms

def test_equal_scores_mean_and_log_n():
    """q = 0 and no bias: every score is 0, so out = mean(v) and lse = ln N."""
    n, D = 37, 16
    q = torch.zeros(D)
    k = _rand((n, D), torch.float32, 31)
    v = _rand((n, D), torch.float32, 32)
    out, lse = oracle.attend_one(q, k, v)
    np.testing.assert_allclose(out, v.double().numpy().mean(axis=0), rtol=0, atol=1e-14)
    assert abs(lse - math.log(n)) < 1e-14


def test_single_key():
    D = 32
    q = _rand((D,), torch.float32, 41)
    k = _rand((1, D), torch.float32, 42)
    v = _rand((1, D), torch.float32, 43)
    out, lse = oracle.attend_one(q, k, v, slope=0.9)
    np.testing.assert_array_equal(out, v[0].double().numpy())
    s0 = float(np.dot(q.double().numpy(), k[0].double().numpy())) / math.sqrt(D)
    assert abs(lse - s0) < 1e-14


@pytest.mark.parametrize("beta", [0.0625, 0.5, 1.0, 2.0])
@pytest.mark.parametrize("n", [1, 5, 64, 1000])
def test_alibi_closed_form_geometric(beta, n):
    """q = 0, v_j = j: s_j = beta (j - n + 1), so with r = e^-beta and t = n-1-j
    l = (1 - r^n)/(1 - r), out = (n-1) - sum_t t r^t / l,
    sum_t t r^t = r (1 - n r^(n-1) + (n-1) r^n) / (1 - r)^2, lse = ln l."""
    D = 4
    q = torch.zeros(D)
    k = _rand((n, D), torch.float32, 51)
    v = torch.arange(n, dtype=torch.float32).view(n, 1).repeat(1, D)
    out, lse = oracle.attend_one(q, k, v, slope=beta)
    r = math.exp(-beta)
    l = (1 - r ** n) / (1 - r)
    st = r * (1 - n * r ** (n - 1) + (n - 1) * r ** n) / (1 - r) ** 2
    expect = (n - 1) - st / l
    np.testing.assert_allclose(out, np.full(D, expect), rtol=1e-13, atol=1e-12)
    assert abs(lse - math.log(l)) < 1e-13


def test_uniform_v_returns_v():
    n, D = 50, 8
    q = _rand((D,), torch.float32, 61, scale=3.0)
    k = _rand((n, D), torch.float32, 62, scale=3.0)
    c = torch.linspace(-2, 2, D)
    v = c.view(1, D).repeat(n, 1)
    out, _ = oracle.attend_one(q, k, v, slope=0.4)
    np.testing.assert_allclose(out, c.double().numpy(), rtol=0, atol=1e-14)


def test_one_dominant_key():
    """A key whose score exceeds the others by >= 50 returns its value row."""
    n, D = 200, 16
    q = _rand((D,), torch.float32, 71)
    k = _rand((n, D), torch.float32, 72, scale=0.1)
    j = 123
    k[j] = q / q.norm() * (60.0 * math.sqrt(D) / float(q.norm()))
    v = _rand((n, D), torch.float32, 73)
    out, _ = oracle.attend_one(q, k, v)
    np.testing.assert_allclose(out, v[j].double().numpy(), rtol=0, atol=n * math.exp(-50) * 10)


# ----------------------------------------------------------- invariants

@pytest.mark.parametrize("c", [-1e3, 0.0, 1e3])
def test_shift_invariance(c):
    """softmax(x) = softmax(x + c): out unchanged, lse shifted by c."""
    n, D = 64, 32
    q = _rand((D,), torch.bfloat16, 81)
    k = _rand((n, D), torch.bfloat16, 82)
    v = _rand((n, D), torch.bfloat16, 83)
    o0, l0 = oracle.attend_one(q, k, v, slope=0.2)
    o1, l1 = oracle.attend_one(q, k, v, slope=0.2, extra_bias=np.full(n, c))
    np.testing.assert_allclose(o1, o0, rtol=0, atol=1e-12)
    assert abs((l1 - l0) - c) < 1e-12 * max(1.0, abs(c))


def test_alibi_row_matches_printed_values():
    g = _golden_sections("alibi_n5.txt")
    row = [oracle.alibi_bias(1.0, j, 5) for j in range(5)]
    assert row == g["row"][0]


@pytest.mark.parametrize("beta", [0.25, 1.0])
def test_alibi_full_form_equivalence_printed(beta):
    """The ALiBi thread: under causal masking the symmetric -|i-j| form and the
    broadcast row differ by a per-row constant, so they give the same
    attention; the oracle's row form (n = i+1) equals the symmetric row."""
    g = _golden_sections("alibi_n5.txt")
    full, bc = g["full"], g["causal_broadcast"]
    n, D = 5, 8
    q = _rand((D,), torch.float32, 91)
    k = _rand((n, D), torch.float32, 92)
    v = _rand((n, D), torch.float32, 93)
    for i in range(n):
        kk, vv = k[: i + 1], v[: i + 1]
        fb = beta * np.array(full[i][: i + 1])
        bb = beta * np.array(bc[i][: i + 1])
        assert all(x is None for x in bc[i][i + 1:])
        o_full, l_full = oracle.attend_one(q, kk, vv, extra_bias=fb)
        o_bc, l_bc = oracle.attend_one(q, kk, vv, extra_bias=bb)
        o_row, l_row = oracle.attend_one(q, kk, vv, slope=beta)
        np.testing.assert_allclose(o_bc, o_full, rtol=0, atol=1e-14)
        np.testing.assert_allclose(o_row, o_full, rtol=0, atol=1e-14)
        assert abs(l_row - l_full) < 1e-14
        # the per-row constant between the two printed forms
        const = bc[i][0] - full[i][0]
        assert abs((l_bc - l_full) - beta * const) < 1e-13


# --------------------------------------------------- chunked Algorithm 3

def test_chunk_bounds_follow_torch_chunk():
    for n in range(0, 41):
        for w in range(1, 11):
            st = oracle.chunk_bounds(n, w, "torch_chunk")
            lens = [st[i + 1] - st[i] for i in range(w)]
            ref = [len(c) for c in torch.arange(n).chunk(w)] if n else []
            assert [x for x in lens if x > 0] == ref
            assert st[0] == 0 and st[-1] == n
            bal = oracle.chunk_bounds(n, w, "balanced")
            bl = [bal[i + 1] - bal[i] for i in range(w)]
            assert sum(bl) == n and max(bl) - min(bl) <= 1


@pytest.mark.parametrize("mode", ["torch_chunk", "balanced"])
def test_chunked_equals_full_every_chunk_count(mode):
    B, H, N, D = 1, 2, 45, 16
    q = _rand((B, H, 1, D), torch.bfloat16, 101)
    k = _rand((B, H, N, D), torch.bfloat16, 102)
    v = _rand((B, H, N, D), torch.bfloat16, 103)
    slopes = torch.tensor([0.05, 1.5])
    out, lse = oracle.full(q, k, v, slopes=slopes)
    for w in range(1, 65):
        o, l = oracle.chunked(q, k, v, w, mode, slopes=slopes)
        np.testing.assert_allclose(o, out, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l, lse, rtol=0, atol=1e-12)


@pytest.mark.parametrize("dtype", [torch.float64, torch.float32, torch.float16])
@pytest.mark.parametrize("mode", ["torch_chunk", "balanced"])
def test_chunked_equals_full_for_every_element_type_and_row(dtype, mode):
    """The gist's claim that the chunked decode equals regular decode, on
    every (b,h) row of a batch (so each row's q, k, v are found at their own
    offsets) and for every element width the oracle reads (8, 4, 2 bytes),
    with ragged lengths; the rows are also held against fp64 SDPA."""
    B, H, N, D = 2, 3, 20, 8
    q = _rand((B, H, 1, D), torch.float32, 111).to(dtype)
    k = _rand((B, H, N, D), torch.float32, 112).to(dtype)
    v = _rand((B, H, N, D), torch.float32, 113).to(dtype)
    slopes = np.array([0.0, 0.25, 1.0], dtype=np.float32)
    lens = torch.tensor([20, 13], dtype=torch.int32)
    out, lse = oracle.full(q, k, v, slopes=slopes, seqlens=lens)
    for w in range(1, 17):
        o, l = oracle.chunked(q, k, v, w, mode, slopes=slopes, seqlens=lens)
        np.testing.assert_allclose(o, out, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l, lse, rtol=0, atol=1e-12)
    for b in range(B):
        n = int(lens[b])
        for h in range(H):
            ref, ref_lse = _sdpa_fp64(q[b, h, 0], k[b, h, :n], v[b, h, :n],
                                      slope=float(slopes[h]))
            np.testing.assert_allclose(out[b * H + h], ref, rtol=0, atol=1e-12)
            assert abs(lse[b * H + h] - ref_lse) < 1e-12


def test_gist_worked_case_n31_w8_d512():
    """The gist's own check: 8 ranks, 31 keys, D=512, inputs the sum of 8
    standard normal draws; Algorithm 3 must match regular decode (the page's
    CPU tolerance is 1e-5; fp64 gives far less)."""
    W, n, D = 8, 31, 512
    g = torch.Generator().manual_seed(5)
    q = sum(torch.randn(1, 1, 1, D, generator=g) for _ in range(W))
    k = sum(torch.randn(1, 1, n, D, generator=g) for _ in range(W))
    v = sum(torch.randn(1, 1, n, D, generator=g) for _ in range(W))
    st = oracle.chunk_bounds(n, W, "torch_chunk")
    assert [st[i + 1] - st[i] for i in range(W)] == [4] * 7 + [3]
    out, lse = oracle.full(q, k, v)
    o, l = oracle.chunked(q, k, v, W, "torch_chunk")
    np.testing.assert_allclose(o, out, rtol=0, atol=1e-12)
    assert abs(l[0] - lse[0]) < 1e-12
    ref, _ = _sdpa_fp64(q[0, 0, 0], k[0, 0], v[0, 0])
    np.testing.assert_allclose(o[0], ref, rtol=0, atol=1e-5)


def test_more_chunks_than_keys():
    """torch.chunk gives fewer chunks than ranks (the gist's harness would
    index past them); balanced mode gives empty chunks; both merge exactly."""
    B, H, N, D = 1, 1, 5, 8
    q = _rand((B, H, 1, D), torch.float32, 111)
    k = _rand((B, H, N, D), torch.float32, 112)
    v = _rand((B, H, N, D), torch.float32, 113)
    out, lse = oracle.full(q, k, v)
    for mode in ("torch_chunk", "balanced"):
        o, l = oracle.chunked(q, k, v, 4 if mode == "torch_chunk" else 13, mode)
        np.testing.assert_allclose(o, out, rtol=0, atol=1e-13)
        np.testing.assert_allclose(l, lse, rtol=0, atol=1e-13)


def test_merge_of_normalised_parts_and_empty_parts():
    """Parts given as (out_c, lse_c, l=1) plus empty parts merge to the full."""
    n, D = 30, 8
    q = _rand((D,), torch.float32, 121)
    k = _rand((n, D), torch.float32, 122)
    v = _rand((n, D), torch.float32, 123)
    full_o, full_l = oracle.attend_one(q, k, v)
    cuts = [0, 7, 8, 19, 30]
    nums, ms, ls = [], [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        o, l = oracle.attend_one(q, k[a:b], v[a:b],
                                 extra_bias=np.zeros(b - a))
        nums.append(o)
        ms.append(l)
        ls.append(1.0)
    nums.append(np.zeros(D))
    ms.append(-math.inf)
    ls.append(0.0)
    o, l = oracle.merge(np.array(nums), ms, ls)
    np.testing.assert_allclose(o, full_o, rtol=0, atol=1e-13)
    assert abs(l - full_l) < 1e-13
    o, l = oracle.merge(np.zeros((3, D)), [-math.inf] * 3, [0.0] * 3)
    assert np.all(o == 0) and l == -math.inf


def test_chunk_partial_matches_definition_of_num_den():
    """num = sum e^(s - m_c) v and den = sum e^(s - m_c) over the chunk, with
    m_c the chunk max: checked through the page's fusion of two chunks."""
    n, D = 20, 4
    q = _rand((D,), torch.float32, 131)
    k = _rand((n, D), torch.float32, 132)
    v = _rand((n, D), torch.float32, 133)
    na, ma, da = oracle.chunk_partial(q, k, v, 0, 9, slope=0.3)
    nb, mb, db = oracle.chunk_partial(q, k, v, 9, 20, slope=0.3)
    M = max(ma, mb)
    o = (na * math.exp(ma - M) + nb * math.exp(mb - M)) / (da * math.exp(ma - M) + db * math.exp(mb - M))
    ref, _ = _sdpa_fp64(q, k, v, 0.3)
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-13)
    s = (k.double() @ q.double()).numpy() / math.sqrt(D) + 0.3 * (np.arange(n) - n + 1)
    assert ma == s[:9].max() and mb == s[9:].max()


def _flash_block_loop_as_printed(q, k, v, block):
    """The blockwise update of the Flash Aandacht listing, re-expressed for one
    query row: O <- (e^(M-M') O + e^(S-M') V) / L'.  It leaves out the factor L
    on the already-normalised O, so it is wrong as soon as there are 2 blocks."""
    s = (k @ q) / math.sqrt(q.shape[0])
    O, L, M = np.zeros(v.shape[1]), 0.0, -math.inf
    for j in range(0, len(s), block):
        sb = s[j:j + block]
        Mn = max(M, sb.max())
        e = np.exp(sb - Mn)
        a = math.exp(M - Mn) if M != -math.inf else 0.0
        Ln = a * L + e.sum()
        O = (a * O + e @ v[j:j + block]) / Ln
        L, M = Ln, Mn
    return O


def _flash_block_loop_corrected(q, k, v, block):
    s = (k @ q) / math.sqrt(q.shape[0])
    O, L, M = np.zeros(v.shape[1]), 0.0, -math.inf
    for j in range(0, len(s), block):
        sb = s[j:j + block]
        Mn = max(M, sb.max())
        e = np.exp(sb - Mn)
        a = math.exp(M - Mn) if M != -math.inf else 0.0
        Ln = a * L + e.sum()
        O = (a * L * O + e @ v[j:j + block]) / Ln
        L, M = Ln, Mn
    return O


def test_negative_control_printed_block_loop_is_caught():
    """The same block-count invariance that pins the oracle rejects the
    printed blockwise loop (>= 2 blocks) and accepts the corrected one."""
    n, D = 64, 8
    q = _rand((D,), torch.float32, 141).double().numpy()
    k = _rand((n, D), torch.float32, 142).double().numpy()
    v = _rand((n, D), torch.float32, 143).double().numpy()
    ref, _ = oracle.attend_one(torch.from_numpy(q).float(), torch.from_numpy(k).float(),
                               torch.from_numpy(v).float())
    np.testing.assert_allclose(_flash_block_loop_as_printed(q, k, v, n), ref, atol=1e-12)
    assert np.abs(_flash_block_loop_as_printed(q, k, v, 16) - ref).max() > 1e-3
    for blk in (1, 5, 16, 64):
        np.testing.assert_allclose(_flash_block_loop_corrected(q, k, v, blk), ref, atol=1e-12)


def test_threads_do_not_change_results():
    B, H, N, D = 2, 4, 100, 16
    q = _rand((B, H, 1, D), torch.bfloat16, 151)
    k = _rand((B, H, N, D), torch.bfloat16, 152)
    v = _rand((B, H, N, D), torch.bfloat16, 153)
    o1, l1 = oracle.full(q, k, v, threads=1)
    o8, l8 = oracle.full(q, k, v, threads=8)
    np.testing.assert_array_equal(o1, o8)
    np.testing.assert_array_equal(l1, l8)


# ------------------------------------------------------- grouped-query form

@pytest.mark.parametrize("H,Hkv", [(8, 1), (8, 2), (8, 8), (6, 3)])
def test_gqa_equals_mha_on_repeated_kv(H, Hkv):
    """Grouped-query attention is plain attention with each kv head repeated
    for the query heads that share it."""
    B, N, D = 2, 37, 16
    q = _rand((B, H, 1, D), torch.bfloat16, 161)
    k = _rand((B, Hkv, N, D), torch.bfloat16, 162)
    v = _rand((B, Hkv, N, D), torch.bfloat16, 163)
    slopes = torch.linspace(0.05, 0.9, H).float()
    seqlens = [20, 37]
    o, l = oracle.full_gqa(q, k, v, slopes=slopes, seqlens=seqlens)
    G = H // Hkv
    kr = k.repeat_interleave(G, dim=1).contiguous()
    vr = v.repeat_interleave(G, dim=1).contiguous()
    ro, rl = oracle.full(q, kr, vr, slopes=slopes, seqlens=seqlens)
    np.testing.assert_array_equal(o, ro)
    np.testing.assert_array_equal(l, rl)


def test_gqa_vs_torch_sdpa_enable_gqa():
    B, H, Hkv, N, D = 1, 8, 2, 29, 32
    q = _rand((B, H, 1, D), torch.float32, 171)
    k = _rand((B, Hkv, N, D), torch.float32, 172)
    v = _rand((B, Hkv, N, D), torch.float32, 173)
    o, l = oracle.full_gqa(q, k, v)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double(), k.double(), v.double(), enable_gqa=True)
    np.testing.assert_allclose(o, ref.reshape(B * H, D).numpy(), rtol=0, atol=1e-12)


# ----------------------------------------------------------------- prefill

def _prefill_block_loop_corrected(q, k, v, slope, causal, qblk, kblk):
    """The Flash Aandacht blockwise forward (outer loop over query blocks,
    inner over key blocks, running M, L and O per query row), with the
    normalised O rescaled by L before it is updated, the ALiBi broadcast row
    slope (j - S + 1) and, when causal, the mask j > i; fp64 numpy."""
    S, D = q.shape
    s_all = (q @ k.T) / math.sqrt(D) + slope * (np.arange(S) - S + 1)[None, :]
    O = np.zeros((S, D))
    L = np.zeros(S)
    M = np.full(S, -math.inf)
    for i0 in range(0, S, qblk):
        rows = np.arange(i0, min(S, i0 + qblk))
        for j0 in range(0, S, kblk):
            cols = np.arange(j0, min(S, j0 + kblk))
            sb = s_all[np.ix_(rows, cols)].copy()
            if causal:
                sb[cols[None, :] > rows[:, None]] = -math.inf
            Mn = np.maximum(M[rows], sb.max(axis=1))
            ok = Mn != -math.inf
            e = np.where(ok[:, None], np.exp(sb - np.where(ok, Mn, 0.0)[:, None]), 0.0)
            a = np.where(M[rows] != -math.inf, np.exp(M[rows] - np.where(ok, Mn, 0.0)), 0.0)
            Ln = a * L[rows] + e.sum(axis=1)
            O[rows] = np.where(Ln[:, None] > 0,
                               (a[:, None] * L[rows][:, None] * O[rows] + e @ v[cols])
                               / np.where(Ln > 0, Ln, 1.0)[:, None], 0.0)
            L[rows], M[rows] = Ln, Mn
    return O, M + np.log(L)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("slope", [0.0, 0.37])
@pytest.mark.parametrize("qblk,kblk", [(1, 1), (4, 7), (16, 5), (64, 64)])
def test_prefill_matches_the_corrected_blockwise_forward(causal, slope, qblk, kblk):
    S, D = 37, 16
    q = _rand((S, D), torch.float32, 181).double().numpy()
    k = _rand((S, D), torch.float32, 182).double().numpy()
    v = _rand((S, D), torch.float32, 183).double().numpy()
    o, l = oracle.prefill(torch.from_numpy(q).float()[None, None], torch.from_numpy(k).float()[None, None],
                          torch.from_numpy(v).float()[None, None], causal=causal,
                          slopes=np.array([slope], dtype=np.float32))
    bo, bl = _prefill_block_loop_corrected(q, k, v, np.float32(slope), causal, qblk, kblk)
    np.testing.assert_allclose(o, bo, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l, bl, rtol=0, atol=1e-12)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_prefill_vs_torch_sdpa_causal(dtype):
    """Library pin: fp64 SDPA with the causal mask plus the ALiBi row as an
    additive mask, on the exactly widened inputs."""
    B, H, S, D = 2, 3, 29, 32
    q = _rand((B, H, S, D), dtype, 191)
    k = _rand((B, H, S, D), dtype, 192)
    v = _rand((B, H, S, D), dtype, 193)
    slopes = np.array([0.5, 0.0, 0.125], dtype=np.float32)
    o, _ = oracle.prefill(q, k, v, causal=True, slopes=slopes)
    row = torch.arange(S, dtype=torch.float64) - S + 1
    mask = torch.full((S, S), -math.inf, dtype=torch.float64).triu(1)
    bias = torch.from_numpy(slopes.astype(np.float64))[:, None, None] * row[None, None, :] + mask
    ref = torch.nn.functional.scaled_dot_product_attention(q.double(), k.double(), v.double(),
                                                           attn_mask=bias[None])
    np.testing.assert_allclose(o, ref.reshape(-1, D).numpy(), rtol=0, atol=1e-12)


def test_prefill_rows_are_decodes_of_their_prefixes():
    """Causal row i is a decode of the first i + 1 keys whose ALiBi row is
    shifted by the constant slope (i + 1 - S): out equal, lse shifted; the last
    row is exactly the decode of the whole sequence; non-causal rows are
    decodes of the whole sequence."""
    S, D, slope = 23, 8, 0.25
    q = _rand((1, 1, S, D), torch.bfloat16, 201)
    k = _rand((1, 1, S, D), torch.bfloat16, 202)
    v = _rand((1, 1, S, D), torch.bfloat16, 203)
    o, l = oracle.prefill(q, k, v, causal=True, slopes=np.array([slope], dtype=np.float32))
    for i in range(S):
        ro, rl = oracle.attend_one(q[0, 0, i], k[0, 0, :i + 1], v[0, 0, :i + 1], slope=slope)
        np.testing.assert_allclose(o[i], ro, rtol=0, atol=1e-12)
        assert abs(l[i] - (rl + slope * (i + 1 - S))) < 1e-12
    ro, rl = oracle.attend_one(q[0, 0, S - 1], k[0, 0], v[0, 0], slope=slope)
    np.testing.assert_array_equal(o[S - 1], ro)
    assert l[S - 1] == rl
    on, ln = oracle.prefill(q, k, v, causal=False, slopes=np.array([slope], dtype=np.float32))
    for i in (0, 7, S - 1):
        ro, rl = oracle.attend_one(q[0, 0, i], k[0, 0], v[0, 0], slope=slope)
        np.testing.assert_allclose(on[i], ro, rtol=0, atol=1e-12)
        assert abs(ln[i] - rl) < 1e-12


def test_prefill_first_row_closed_form_and_row_selection():
    S, D, slope = 9, 4, 0.5
    q = _rand((2, 2, S, D), torch.float32, 211)
    k = _rand((2, 2, S, D), torch.float32, 212)
    v = _rand((2, 2, S, D), torch.float32, 213)
    o, l = oracle.prefill(q, k, v, causal=True, slopes=np.array([slope, 0.0], dtype=np.float32))
    # row 0 of a causal prefill sees key 0 only
    np.testing.assert_array_equal(o[0], v[0, 0, 0].double().numpy())
    s00 = float((q[0, 0, 0].double() * k[0, 0, 0].double()).sum()) / 2.0 + slope * (1 - S)
    assert abs(l[0] - s00) < 1e-12
    rows = [0, S + 3, 3 * S + 8, 2 * S]
    os_, ls_ = oracle.prefill(q, k, v, causal=True, slopes=np.array([slope, 0.0], dtype=np.float32),
                              rows=rows)
    np.testing.assert_array_equal(os_, o[rows])
    np.testing.assert_array_equal(ls_, l[rows])


# --------------------------------------------------------- FP8 (E4M3) caches

def test_e4m3_decoder_matches_torch_on_every_code():
    """Library pin: torch's float8_e4m3fn widening, all 256 codes."""
    bits = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = bits.view(torch.float8_e4m3fn).double().numpy()
    got = np.array([oracle.decode_e4m3(b) for b in range(256)])
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])


def test_e4m3_decoder_closed_forms():
    assert oracle.decode_e4m3(0x7E) == 448.0           # largest finite
    assert oracle.decode_e4m3(0x01) == 2.0 ** -9        # smallest subnormal
    assert oracle.decode_e4m3(0x08) == 2.0 ** -6        # smallest normal
    assert oracle.decode_e4m3(0x38) == 1.0
    assert oracle.decode_e4m3(0xB8) == -1.0
    assert math.isnan(oracle.decode_e4m3(0x7F)) and math.isnan(oracle.decode_e4m3(0xFF))
    assert oracle.decode_e4m3(0x00) == 0.0 and math.copysign(1, oracle.decode_e4m3(0x80)) < 0


def test_fp64_inputs_agree_with_fp32_inputs():
    """The widened-input path reads the same numbers as the fp32 path."""
    B, H, N, D = 1, 3, 41, 16
    q = _rand((B, H, 1, D), torch.float32, 221)
    k = _rand((B, H, N, D), torch.float32, 222)
    v = _rand((B, H, N, D), torch.float32, 223)
    slopes = np.array([0.1, 0.2, 0.3], dtype=np.float32)
    a = oracle.full(q, k, v, slopes=slopes)
    b = oracle.full(q.double(), k.double(), v.double(), slopes=slopes)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_fp8_cache_attention_is_attention_on_the_dequantised_cache():
    """An FP8 cache with per-head scales means K = e4m3(k8) * k_scale[h] (and V
    alike); fp64 SDPA on those dequantised values is the library pin."""
    B, H, N, D = 2, 2, 50, 32
    g = torch.Generator().manual_seed(231)
    q = torch.randn((B, H, 1, D), generator=g).to(torch.bfloat16)
    k8 = torch.randint(0, 256, (B, H, N, D), generator=g, dtype=torch.int32).to(torch.uint8)
    v8 = torch.randint(0, 256, (B, H, N, D), generator=g, dtype=torch.int32).to(torch.uint8)
    k8[(k8 & 0x7F) == 0x7F] = 0x38   # no NaN codes in a cache
    v8[(v8 & 0x7F) == 0x7F] = 0x38
    ks = np.array([0.01, 0.002], dtype=np.float32)
    vs = np.array([0.5, 0.03125], dtype=np.float32)
    K = oracle.dequant_e4m3(k8, ks)
    V = oracle.dequant_e4m3(v8, vs)
    o, l = oracle.full(q.double(), torch.from_numpy(K), torch.from_numpy(V))
    ref = torch.nn.functional.scaled_dot_product_attention(q.double(), torch.from_numpy(K),
                                                           torch.from_numpy(V))
    np.testing.assert_allclose(o, ref.reshape(B * H, D).numpy(), rtol=0, atol=1e-12)
