"""Pins for the CPU oracle: each check ties it to something other than itself.

Library routines (torch scaled_dot_product_attention in fp64), closed forms,
brute force on tiny inputs, invariants and hand-derived fixtures.  No GPU.
"""
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from dynamic_sparse_attention_02_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_qkv(Hq, Hkv, N, d, seed, bf16=True):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(Hq, N, d, generator=g)
    k = torch.randn(Hkv, N, d, generator=g)
    v = torch.randn(Hkv, N, d, generator=g)
    if bf16:
        q, k, v = (t.to(torch.bfloat16).float() for t in (q, k, v))
    return q, k, v


def sdpa_rows(q, k, v, h, mask=None, causal=False):
    """Library reference: torch SDPA in fp64 for query head h (GQA: contiguous groups)."""
    g = h * k.shape[0] // q.shape[0]
    qh = q[h].double()[None, None]
    kh = k[g].double()[None, None]
    vh = v[g].double()[None, None]
    if mask is not None:
        return F.scaled_dot_product_attention(qh, kh, vh, attn_mask=torch.as_tensor(mask)[None, None])[0, 0].numpy()
    return F.scaled_dot_product_attention(qh, kh, vh, is_causal=causal)[0, 0].numpy()


# ---------------------------------------------------------------- dense (P1)

@pytest.mark.parametrize("Hq,Hkv,N,d", [(1, 1, 128, 64), (4, 2, 192, 128), (8, 2, 256, 64)])
def test_dense_matches_sdpa(Hq, Hkv, N, d):
    q, k, v = rand_qkv(Hq, Hkv, N, d, 1)
    for h in range(Hq):
        out, lse = oracle.attn_dense(q, k, v, h)
        ref = sdpa_rows(q, k, v, h, causal=True)
        np.testing.assert_allclose(out, ref, atol=1e-12, rtol=1e-10)
        # lse against logsumexp of the scaled causal scores (torch fp64)
        g = h * Hkv // Hq
        s = (q[h].double() @ k[g].double().T) / np.sqrt(d)
        s = s.masked_fill(torch.triu(torch.ones(N, N, dtype=torch.bool), 1), float("-inf"))
        np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), atol=1e-12)


def test_full_budgets_reduce_to_dense():
    """Budgets that cover everything give dense causal attention."""
    Hq, Hkv, N, d = 2, 1, 256, 64
    q, k, v = rand_qkv(Hq, Hkv, N, d, 2)
    ref = sdpa_rows(q, k, v, 1, causal=True)
    every = np.arange(N)
    out, _ = oracle.attn_vs(q, k, v, 1, every, [], rows=None)          # all columns
    np.testing.assert_allclose(out, ref, atol=1e-12)
    out, _ = oracle.attn_vs(q, k, v, 1, [], every)                     # all diagonals
    np.testing.assert_allclose(out, ref, atol=1e-12)
    nB = N // 64
    blk = np.tile(np.arange(nB, dtype=np.int32), (nB, 1))
    out, _ = oracle.attn_bs(q, k, v, 1, blk, np.full(nB, nB, np.int32))  # all blocks
    np.testing.assert_allclose(out, ref, atol=1e-12)
    out, _ = oracle.attn_ashape(q, k, v, 1, sink=0, window=N)          # window covers all
    np.testing.assert_allclose(out, ref, atol=1e-12)
    # and the index pipeline with budgets >= N selects every column / diagonal
    v_idx, s_idx, _, _ = oracle.vs_index(q, k, 1, 64, N + 5, 10 * N)
    assert np.array_equal(v_idx, every) and np.array_equal(s_idx, every)
    bi, bc = oracle.bs_index(q, k, 1, nB + 3)
    assert np.array_equal(bc, np.arange(1, nB + 1))


# ------------------------------------------------------------- A-shape (P2)

@pytest.mark.parametrize("sink,window", [(64, 128), (1, 1), (0, 64), (10, 37), (64, 1024)])
def test_ashape_matches_brute_force_mask(sink, window):
    Hq, Hkv, N, d = 2, 1, 384, 64
    q, k, v = rand_qkv(Hq, Hkv, N, d, 3)
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    mask = (j <= i) & ((j < sink) | (i - j < window))
    for h in range(Hq):
        out, _ = oracle.attn_ashape(q, k, v, h, sink, window)
        ref = sdpa_rows(q, k, v, h, mask=mask)
        np.testing.assert_allclose(out, ref, atol=1e-12)


def test_ashape_window_one_returns_own_value():
    """sink = 0, window = 1: each row sees only itself, so out_i = v_i exactly (P5)."""
    q, k, v = rand_qkv(4, 2, 192, 64, 4)
    for h in (0, 3):
        out, lse = oracle.attn_ashape(q, k, v, h, sink=0, window=1)
        g = h * 2 // 4
        np.testing.assert_array_equal(out, v[g].double().numpy())
        s_ii = (q[h].double() * k[g].double()).sum(-1) / 8.0
        np.testing.assert_allclose(lse, s_ii.numpy(), atol=1e-12)


def test_ashape_window_two_closed_form():
    """window = 2: two keys (i-1, i) -> sigmoid weights, written out by hand."""
    q, k, v = rand_qkv(1, 1, 128, 64, 5)
    out, _ = oracle.attn_ashape(q, k, v, 0, sink=0, window=2)
    qd, kd, vd = (t[0].double().numpy() for t in (q, k, v))
    for i in (1, 50, 127):
        a = qd[i] @ kd[i - 1] / 8.0
        b = qd[i] @ kd[i] / 8.0
        w = 1.0 / (1.0 + np.exp(b - a))
        np.testing.assert_allclose(out[i], w * vd[i - 1] + (1 - w) * vd[i], atol=1e-12)
    np.testing.assert_allclose(out[0], vd[0], atol=1e-15)


# -------------------------------------------------------- row sums (P4)

def test_rows_sum_to_one_every_pattern():
    """With v = 1 every non-empty row outputs exactly 1: the weights sum to 1."""
    Hq, Hkv, N, d = 2, 1, 256, 64
    q, k, _ = rand_qkv(Hq, Hkv, N, d, 6)
    ones = torch.ones(Hkv, N, d)
    outs = [oracle.attn_dense(q, k, ones, 0)[0],
            oracle.attn_ashape(q, k, ones, 0, 16, 40)[0],
            oracle.attn_vs(q, k, ones, 1, [0, 7, 99], [0, 130])[0]]
    bi, bc = oracle.bs_index(q, k, 0, 2)
    outs.append(oracle.attn_bs(q, k, ones, 0, bi, bc)[0])
    for o in outs:
        np.testing.assert_allclose(o, 1.0, atol=1e-12)


# ----------------------------------------------------- Vertical-Slash (P6-P9)

def test_vs_single_column_closed_form():
    """V = {0}, no diagonals: every row attends only to key 0, out_i = v_0 (P6)."""
    q, k, v = rand_qkv(2, 1, 256, 64, 7)
    out, _ = oracle.attn_vs(q, k, v, 0, [0], [])
    np.testing.assert_array_equal(out, np.broadcast_to(v[0, 0].double().numpy(), out.shape))


def test_vs_empty_rows_are_zero():
    """Rows before the only selected column have no key: 0 and lse = -inf."""
    q, k, v = rand_qkv(1, 1, 128, 64, 8)
    out, lse = oracle.attn_vs(q, k, v, 0, [5], [])
    assert np.all(out[:5] == 0) and np.all(np.isneginf(lse[:5]))
    np.testing.assert_array_equal(out[5:], np.broadcast_to(v[0, 5].double().numpy(), (123, 64)))


def test_vs_mask_matches_brute_force():
    """VS attention equals SDPA with the mask built element by element."""
    Hq, Hkv, N, d = 2, 1, 512, 64
    q, k, v = rand_qkv(Hq, Hkv, N, d, 9)
    v_idx = np.array([3, 77, 200, 201, 450], np.int32)
    s_idx = np.array([0, 100, 300, 385], np.int32)  # 385 = 6*64 + 1 touches deltas 6 and 7
    D = set()
    for o in s_idx:  # tiles touched by each diagonal, by scanning its elements
        for i in range(N):
            if i - o >= 0:
                D.add(i // 64 - (i - o) // 64)
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    delta = i // 64 - j // 64
    mask = (j <= i) & (np.isin(j, v_idx) | np.isin(delta, sorted(D)))
    out, _ = oracle.attn_vs(q, k, v, 1, v_idx, s_idx)
    np.testing.assert_allclose(out, sdpa_rows(q, k, v, 1, mask=mask), atol=1e-12)


def _golden_slash():
    cases = []
    with open(os.path.join(GOLDEN, "slash_deltas.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            n, offs, deltas = (c.strip() for c in line.split("|"))
            cases.append((int(n), [int(x) for x in offs.split()], [int(x) for x in deltas.split()]))
    return cases


@pytest.mark.parametrize("N,offs,deltas", _golden_slash())
def test_slash_deltas_golden(N, offs, deltas):
    D = oracle.slash_deltas(np.array(offs, np.int32), N)
    assert sorted(np.nonzero(D)[0].tolist()) == deltas


def test_slash_deltas_brute_force_scan():
    """Delta set equals a scan of every element of every selected diagonal (P7)."""
    rng = np.random.default_rng(11)
    N = 1024
    for _ in range(20):
        offs = rng.choice(N, size=rng.integers(0, 12), replace=False).astype(np.int32)
        want = set()
        for o in offs:
            for i in range(o, N):
                want.add(i // 64 - (i - o) // 64)
        D = oracle.slash_deltas(offs, N)
        assert set(np.nonzero(D)[0].tolist()) == want
    # each offset alone at and beside a block boundary, where a bound is easiest to get wrong
    for o in [64 * a + r for a in (0, 1, 7, 15) for r in (0, 1, 2, 62, 63)]:
        want = {i // 64 - (i - o) // 64 for i in range(o, N)}
        D = oracle.slash_deltas(np.array([o], np.int32), N)
        assert set(np.nonzero(D)[0].tolist()) == want, o


def _softmax_weights_via_sdpa(q, k, h, rows):
    """Attention weights of the given rows, read out of torch SDPA with v = identity."""
    N = k.shape[1]
    g = h * k.shape[0] // q.shape[0]
    eye = torch.eye(N, dtype=torch.float64)[None, None]
    qh = q[h].double()[None, None]
    kh = k[g].double()[None, None]
    W = F.scaled_dot_product_attention(qh, kh, eye, is_causal=True)[0, 0].numpy()
    return W[rows]


@pytest.mark.parametrize("N,d,L,Hq,Hkv", [(256, 64, 64, 1, 1), (640, 128, 64, 4, 2), (192, 64, 128, 2, 2)])
def test_vs_scores_match_materialised_softmax(N, d, L, Hq, Hkv):
    """vertical = column sums and slash = diagonal sums of the last-L softmax rows (P8)."""
    q, k, _ = rand_qkv(Hq, Hkv, N, d, 12)
    rows = np.arange(N - L, N)
    for h in range(Hq):
        W = _softmax_weights_via_sdpa(q, k, h, rows)
        vert_ref = W.sum(0)
        slash_ref = np.zeros(N)
        for r, i in enumerate(rows):
            for j in range(i + 1):
                slash_ref[i - j] += W[r, j]
        vert, sl = oracle.vs_scores(q, k, h, L)
        np.testing.assert_allclose(vert, vert_ref, rtol=1e-10, atol=1e-15)
        np.testing.assert_allclose(sl, slash_ref, rtol=1e-10, atol=1e-15)
        # P9: every row sums to one
        assert abs(vert.sum() - L) < 1e-9 and abs(sl.sum() - L) < 1e-9


def test_vs_scores_single_query_row():
    """last_q = 1: slash is the last row's weights read backwards (closed form)."""
    q, k, _ = rand_qkv(1, 1, 256, 64, 13)
    vert, sl = oracle.vs_scores(q, k, 0, 1)
    np.testing.assert_allclose(sl, vert[::-1], rtol=1e-14, atol=1e-18)


# --------------------------------------------------------------- top-k (R5)

def test_topk_ties_prefer_lower_index():
    s = np.array([1.0, 3.0, 3.0, 2.0, 3.0, 0.5])
    assert oracle.topk(s, 2).tolist() == [1, 2]
    assert oracle.topk(s, 4).tolist() == [1, 2, 3, 4]
    assert oracle.topk(s, 100).tolist() == list(range(6))
    assert oracle.topk(s, 0).tolist() == []


# --------------------------------------------------------- Block-Sparse (P3)

@pytest.mark.parametrize("N,d,topk", [(512, 64, 3), (1024, 128, 5), (256, 64, 1), (320, 64, 10)])
def test_bs_index_matches_exhaustive_numpy(N, d, topk):
    Hq, Hkv = 4, 2
    q, k, _ = rand_qkv(Hq, Hkv, N, d, 14)
    nB = N // 64
    for h in range(Hq):
        g = h * Hkv // Hq
        Qm = q[h].double().numpy().reshape(nB, 64, d).mean(1)
        Km = k[g].double().numpy().reshape(nB, 64, d).mean(1)
        S = Qm @ Km.T / np.sqrt(d)
        bi, bc, sc = oracle.bs_index(q, k, h, topk, want_scores=True)
        for bq in range(nB):
            cand = np.arange(bq + 1)
            order = np.lexsort((cand, -S[bq, :bq + 1]))  # score desc, then index asc
            want = np.sort(cand[order[:min(topk, bq + 1)]])
            assert bc[bq] == len(want)
            assert bi[bq, :bc[bq]].tolist() == want.tolist()
            assert np.all(bi[bq, bc[bq]:] == -1)
            np.testing.assert_allclose(sc[bq, :bq + 1], S[bq, :bq + 1], rtol=1e-12, atol=1e-15)


def test_bs_ties_prefer_lower_block():
    """All key blocks identical: every block score ties, so the lowest blocks win."""
    N, d = 512, 64
    q, k, _ = rand_qkv(1, 1, N, d, 15)
    k = k[:, :64].repeat(1, 8, 1).contiguous()
    bi, bc, sc = oracle.bs_index(q, k, 0, 3, want_scores=True)
    for bq in range(8):
        assert np.all(sc[bq, :bq + 1] == sc[bq, 0])
        want = list(range(min(3, bq + 1)))
        assert bc[bq] == len(want) and bi[bq, :bc[bq]].tolist() == want


def test_bs_attention_matches_brute_force_mask():
    Hq, Hkv, N, d = 2, 1, 512, 64
    q, k, v = rand_qkv(Hq, Hkv, N, d, 16)
    bi, bc = oracle.bs_index(q, k, 0, 3)
    sel = np.zeros((8, 8), bool)
    for bq in range(8):
        sel[bq, bi[bq, :bc[bq]]] = True
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    mask = (j <= i) & sel[i // 64, j // 64]
    out, _ = oracle.attn_bs(q, k, v, 0, bi, bc)
    np.testing.assert_allclose(out, sdpa_rows(q, k, v, 0, mask=mask), atol=1e-12)


# -------------------------------------------------------------- GQA mapping

def test_gqa_contiguous_groups():
    """Query head h reads KV head floor(h * Hkv / Hq): heads 0-3 share KV 0 at 8:2."""
    q, k, v = rand_qkv(8, 2, 128, 64, 17)
    for h in range(8):
        out, _ = oracle.attn_dense(q, k, v, h)
        g = h // 4
        k1 = k[g:g + 1].expand(8, -1, -1)
        v1 = v[g:g + 1].expand(8, -1, -1)
        ref = sdpa_rows(q, k1.contiguous(), v1.contiguous(), h, causal=True)
        np.testing.assert_allclose(out, ref, atol=1e-12)


def test_generator_deterministic_and_planted():
    w = synth.workload("vs_n2k_h1_d64", N=512)
    a = synth.make_inputs(w)
    b = synth.make_inputs(w)
    for key in ("q", "k", "v"):
        assert torch.equal(a[key], b[key]) and a[key].dtype == torch.bfloat16
    assert a["q"].shape == (1, 512, 64) and a["k"].shape == (1, 512, 64)
    assert set(range(4)) <= set(a["planted"].tolist())
    assert len(a["planted"]) == 4 + round(0.01 * 512) or len(a["planted"]) >= 4
    m = synth.workload("mixed_n256k_llama3_8b")
    pt = synth.pattern_table(m, torch.Generator().manual_seed(1))
    assert sorted(np.bincount(pt, minlength=3).tolist()) == [10, 11, 11]


# ------------------------------------------- hand-worked fixtures (golden/)

def _golden_cases(name):
    """Blank-line separated `key: value` blocks of a hand-worked fixture file."""
    cases, cur = [], {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].rstrip()
            if not line:
                if cur:
                    cases.append(cur)
                    cur = {}
                continue
            key, _, val = line.partition(":")
            cur[key.strip()] = val.strip()
    if cur:
        cases.append(cur)
    return [pytest.param(c, id=c.get("case")) for c in cases]


def _fracs(s):
    from fractions import Fraction
    return np.array([float(Fraction(t)) for t in s.split()], np.float64)


def _rows(s):
    """'a b | c d ; e f | g h' -> float32 [heads, rows, cols]."""
    heads = [[[float(x) for x in r.split()] for r in h.split("|")] for h in s.split(";")]
    return torch.tensor(heads, dtype=torch.float32)


def _ints(s):
    return [int(t) for t in s.split()]


@pytest.mark.parametrize("c", _golden_cases("vs_scores_hand.txt"))
def test_vs_scores_hand_worked(c):
    """Column and diagonal sums equal fractions worked by hand (weights 2^(q.k))."""
    q, k = _rows(c["q"]), _rows(c["k"])
    h, L = int(c["h"]), int(c["last_q"])
    assert q.shape == (int(c["Hq"]), int(c["N"]), int(c["d"])) and k.shape[0] == int(c["Hkv"])
    vert, sl = oracle.vs_scores(q, k, h, L, scale=np.log(2.0))
    np.testing.assert_allclose(vert, _fracs(c["vertical"]), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(sl, _fracs(c["slash"]), rtol=1e-14, atol=1e-15)
    for kk in (1, 2):
        assert oracle.topk(vert, kk).tolist() == _ints(c[f"v_top{kk}"])
        assert oracle.topk(sl, kk).tolist() == _ints(c[f"s_top{kk}"])


@pytest.mark.parametrize("c", _golden_cases("bs_index_hand.txt"))
def test_bs_index_hand_worked(c):
    """Block means, causal block scores and top-k equal values worked by hand."""
    N, d, B = int(c["N"]), int(c["d"]), int(c["block"])
    q, k = _rows(c["q"]), _rows(c["k"])
    assert q.shape == (1, N, d) and k.shape == (1, N, d)
    nB = N // B
    want_s = [[float(x) for x in r.split()] for r in c["scores"].split(";")]
    for kk in (1, 2):
        bi, bc, sc = oracle.bs_index(q, k, 0, kk, block=B, scale=1.0, want_scores=True)
        want = [_ints(r) for r in c[f"top{kk}"].split(";")]
        for bq in range(nB):
            np.testing.assert_allclose(sc[bq, :bq + 1], want_s[bq], rtol=0, atol=1e-15)
            assert bc[bq] == len(want[bq]) and bi[bq, :bc[bq]].tolist() == want[bq]


@pytest.mark.parametrize("c", _golden_cases("attn_hand.txt"))
def test_attention_hand_worked(c):
    """A-shape and Vertical-Slash rows (window, gathered column, no double count,
    empty rows) equal fractions worked by hand."""
    N = int(c["N"])
    q = torch.ones(1, N, 1)
    k = torch.tensor(_ints(c["k"]), dtype=torch.float32).reshape(1, N, 1)
    v = torch.tensor(_ints(c["v"]), dtype=torch.float32).reshape(1, N, 1)
    if c["case"] == "ashape":
        out, lse = oracle.attn_ashape(q, k, v, 0, int(c["sink"]), int(c["window"]),
                                      scale=np.log(2.0))
    else:
        out, lse = oracle.attn_vs(q, k, v, 0, _ints(c["v_idx"]), _ints(c["s_idx"]),
                                  block=int(c["block"]), scale=np.log(2.0))
    np.testing.assert_allclose(out[:, 0], _fracs(c["out"]), rtol=1e-14, atol=1e-15)
    lse_of = _fracs(c["lse_of"])
    empty = lse_of == 0
    assert np.all(np.isneginf(lse[empty]))
    np.testing.assert_allclose(lse[~empty], np.log(lse_of[~empty]), rtol=1e-14, atol=1e-15)


# ------------------------------------------- range-based slash tiles (§ next)

def _brute_range_mask(N, v_idx, s_idx, block=64):
    """The range predicate built diagonal by diagonal: for every selected o and
    every query block bq, mark keys [64 bq - o, 64 bq + 63 - o] for the rows of
    bq; then the selected columns; then the causal limit."""
    m = np.zeros((N, N), bool)
    for o in s_idx:
        if not 0 <= o < N:
            continue
        for bq in range(N // block):
            lo, hi = max(0, block * bq - o), block * bq + block - 1 - o
            if hi >= lo:
                m[block * bq:block * bq + block, lo:hi + 1] = True
    for c in v_idx:
        if 0 <= c < N:
            m[:, c] = True
    return m & np.tril(np.ones((N, N), bool))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_vs_range_mask_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    N = 512
    s_idx = rng.choice(N, size=12, replace=False).astype(np.int32)
    v_idx = rng.choice(N, size=5, replace=False).astype(np.int32)
    got = oracle.vs_mask(N, v_idx, s_idx, range_tiles=True)
    np.testing.assert_array_equal(got, _brute_range_mask(N, v_idx, s_idx))


def test_vs_range_between_exact_diagonals_and_whole_tiles():
    """Exact diagonals (j = i - o) lie inside the ranges, which lie inside the
    whole 64x64 tiles the same diagonals touch; equality on neither side."""
    rng = np.random.default_rng(5)
    N = 640
    s_idx = rng.choice(N, size=20, replace=False).astype(np.int32)
    rng_m = oracle.vs_mask(N, [], s_idx, range_tiles=True)
    tile_m = oracle.vs_mask(N, [], s_idx, range_tiles=False)
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    exact = (j <= i) & np.isin(i - j, s_idx)
    assert np.all(rng_m[exact]) and np.all(tile_m[rng_m])
    assert rng_m.sum() > exact.sum() and tile_m.sum() > rng_m.sum()


def test_vs_range_hand_cases():
    """Worked by hand, N = 192 (three query blocks), no columns:
    o = 0 -> each query block takes its own block (causal);
    o = 64 -> each query block takes the previous block whole, block 0 none;
    o = 1 -> query block bq takes keys 64 bq - 1 .. 64 bq + 62."""
    N = 192
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    bq = i // 64
    m0 = oracle.vs_mask(N, [], [0], range_tiles=True)
    np.testing.assert_array_equal(m0, (j // 64 == bq) & (j <= i))
    m64 = oracle.vs_mask(N, [], [64], range_tiles=True)
    np.testing.assert_array_equal(m64, j // 64 == bq - 1)
    m1 = oracle.vs_mask(N, [], [1], range_tiles=True)
    np.testing.assert_array_equal(m1, (j >= 64 * bq - 1) & (j <= 64 * bq + 62) & (j <= i))


def test_vs_range_attention_matches_sdpa_with_the_mask():
    Hq, Hkv, N, d = 2, 1, 384, 64
    q, k, v = rand_qkv(Hq, Hkv, N, d, 17)
    v_idx = np.array([2, 90, 300], np.int32)
    s_idx = np.array([0, 33, 130, 200], np.int32)
    mask = _brute_range_mask(N, v_idx, s_idx)
    out, lse = oracle.attn_vs_range(q, k, v, 1, v_idx, s_idx)
    np.testing.assert_allclose(out, sdpa_rows(q, k, v, 1, mask=mask), atol=1e-12)


def test_vs_range_full_slash_budget_is_dense():
    """Every diagonal selected: every causal key is covered (P1 for ranges)."""
    Hq, Hkv, N, d = 1, 1, 256, 64
    q, k, v = rand_qkv(Hq, Hkv, N, d, 18)
    out, _ = oracle.attn_vs_range(q, k, v, 0, [], np.arange(N))
    np.testing.assert_allclose(out, sdpa_rows(q, k, v, 0, causal=True), atol=1e-12)
