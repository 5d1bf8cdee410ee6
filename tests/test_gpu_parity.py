"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Sizes span several 256-row super tiles, ragged tails (N not a multiple of
256), GQA 4:1 and 1:1, d = 64 and 128, and the degenerate cases of each
pattern.  Attention is always fed the oracle's own indices.
"""
import numpy as np
import pytest
import torch

import oracle
from dynamic_sparse_attention_02_b200 import binding as B
from dynamic_sparse_attention_02_b200 import synth
from parity_util import check_attn, check_index_set, head_slices, rand_bf16

pytestmark = pytest.mark.gpu

needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from dynamic_sparse_attention_02_b200 import build
    build.build()


@pytest.fixture(params=[B.BS_ENGINE_ROW, B.BS_ENGINE_KEY], ids=["row", "key"])
def bs_engine(request):
    """Each Block-Sparse attention case runs on both engines."""
    B.mi_set_bs_engine(request.param)
    yield request.param
    B.mi_set_bs_engine(B.BS_ENGINE_ROW)


# ------------------------------------------------------------ VS index

@pytest.mark.parametrize("Hq,Hkv,N,d,L,kv,ks", [
    (1, 1, 2048, 64, 64, 128, 256),     # the 2K single-head workload
    (4, 1, 1088, 128, 64, 100, 300),    # GQA 4:1, ragged N
    (2, 2, 640, 128, 130, 700, 17),     # last_q not a multiple of 64 (3 row groups), kv > N
    (2, 1, 192, 64, 64, 0, 1),          # tiny: one super tile, zero vertical budget
    # several 2048-key chunks, so diagonals that start near a chunk's end are finished
    # in the next key tile, plus ragged tails
    (2, 1, 4160, 128, 64, 300, 900),    # 3 chunks, the last one 64 keys
    (3, 1, 6144, 64, 48, 200, 500),     # 3 full chunks, 16 padding rows per head, odd head count
    (1, 1, 4096, 128, 1, 100, 300),     # last_q = 1: a single row, diagonals of one element
    (4, 2, 2112, 128, 33, 64, 128),     # 2 chunks, the second one tile; 31 padding rows
    (1, 1, 64, 128, 64, 10, 20),        # one 64-key tile
    # last_q > 64: several 64-row groups per head, partial sums merged per head
    (2, 1, 4160, 128, 200, 300, 900),   # 4 row groups (the first 8 rows), 3 chunks
    (1, 1, 2112, 64, 1000, 400, 800),   # 16 row groups, nearly every row of the sequence
    (3, 1, 2048, 128, 128, 150, 400),   # 2 full row groups per head, odd head count
])
def test_vs_index_matches_oracle(Hq, Hkv, N, d, L, kv, ks):
    w = synth.workload("vs_n2k_h1_d64", Hq=Hq, Hkv=Hkv, N=N, d=d)
    x = synth.make_inputs(w, device="cuda")
    v_idx, s_idx, vsc, ssc = B.mi_vs_index(x["q"], x["k"], L, kv, ks, want_scores=True)
    torch.cuda.synchronize()
    # Score tolerance from the arithmetic: the products q.k run on the bf16 tensor cores,
    # exact per product but summed over d in fp32, so a logit carries an error of a few
    # units of 2^-24 x sqrt(d) x |q||k| x scale (1e-7 .. 1e-6 here) and a probability the
    # same relative error; a score that sums a single row (last_q = 1) shows it unaveraged
    # (1.3e-6 measured).  1e-5 bounds that with margin; a wrong term, sign or index would
    # show as 1e-3 or more.  The index sets are held to the 1e-6 window below.
    rtol = 1e-5
    for h in range(Hq):
        qs, ks_, _ = head_slices(x["q"], x["k"], None, h)
        vert, sl = oracle.vs_scores(qs, ks_, 0, L)
        np.testing.assert_allclose(vsc[h].cpu().numpy(), vert, rtol=rtol, atol=1e-30)
        np.testing.assert_allclose(ssc[h].cpu().numpy(), sl, rtol=rtol, atol=1e-30)
        check_index_set(v_idx[h].cpu().numpy(), vert, kv, what=f"vertical h{h}")
        check_index_set(s_idx[h].cpu().numpy(), sl, ks, what=f"slash h{h}")


def test_vs_index_head_subset():
    q, k, _ = rand_bf16(8, 2, 512, 128, 3)
    heads = [6, 1, 3]
    v_idx, s_idx = B.mi_vs_index(q, k, 64, 50, 60, heads=heads)
    torch.cuda.synchronize()
    for pos, h in enumerate(heads):
        qs, ks_, _ = head_slices(q, k, None, h)
        vert, sl = oracle.vs_scores(qs, ks_, 0, 64)
        check_index_set(v_idx[pos].cpu().numpy(), vert, 50, what=f"vertical h{h}")
        check_index_set(s_idx[pos].cpu().numpy(), sl, 60, what=f"slash h{h}")


# ------------------------------------------------------------ BS index

@pytest.mark.parametrize("Hq,Hkv,N,d,topk", [
    (4, 1, 1024, 128, 5), (2, 2, 576, 64, 3), (1, 1, 256, 128, 10), (2, 1, 4096, 128, 100)])
def test_bs_index_matches_oracle(Hq, Hkv, N, d, topk):
    w = synth.workload("bs_n128k_llama3_8b", Hq=Hq, Hkv=Hkv, N=N, d=d)
    x = synth.make_inputs(w, device="cuda")
    blk_idx, blk_cnt = B.mi_bs_index(x["q"], x["k"], topk)
    torch.cuda.synchronize()
    nB = N // 64
    for h in range(Hq):
        qs, ks_, _ = head_slices(x["q"], x["k"], None, h)
        ref_idx, ref_cnt, S = oracle.bs_index(qs, ks_, 0, topk, want_scores=True)
        cnt = blk_cnt[h].cpu().numpy()
        assert np.array_equal(cnt, ref_cnt)
        bi = blk_idx[h].cpu().numpy()
        for bq in range(nB):
            row = S[bq, :bq + 1]
            # tie window scaled by the row's largest |score| (logits sit near 0)
            check_index_set(bi[bq], row, topk, window_scale=np.abs(row).max(),
                            what=f"h{h} bq{bq}")


# ------------------------------------------------------------ attention

def _all_rows(N):
    return np.arange(N)


@pytest.mark.parametrize("Hq,Hkv,N,d,sink,window", [
    (2, 1, 512, 128, 64, 128),
    (4, 2, 1088, 128, 64, 1024),   # ragged tail
    (1, 1, 192, 64, 0, 1),         # out_i = v_i
    (2, 2, 320, 64, 10, 37),       # unaligned sink / window
    (1, 1, 64, 128, 64, 1024),     # one block
])
def test_ashape_attn_matches_oracle(Hq, Hkv, N, d, sink, window):
    q, k, v = rand_bf16(Hq, Hkv, N, d, 11)
    out, lse = B.mi_ashape_attn(q, k, v, sink, window)
    torch.cuda.synchronize()
    for h in range(Hq):
        qs, ks_, vs_ = head_slices(q, k, v, h)
        ro, rl = oracle.attn_ashape(qs, ks_, vs_, 0, sink, window)
        check_attn(out[h], lse[h], ro, rl, what=f"ashape h{h}")


@pytest.mark.parametrize("Hq,Hkv,N,d,topk", [
    (4, 1, 1024, 128, 4), (2, 2, 576, 64, 3), (2, 1, 2048, 128, 100),
    (6, 2, 4096, 128, 9),    # more items than one CTA per SM takes at once, odd topk
    (1, 1, 64, 128, 1)])     # a single query block
def test_block_sparse_attn_matches_oracle(Hq, Hkv, N, d, topk, bs_engine):
    q, k, v = rand_bf16(Hq, Hkv, N, d, 12)
    nB = N // 64
    bi = np.full((Hq, nB, topk), -1, np.int32)
    bc = np.zeros((Hq, nB), np.int32)
    refs = []
    for h in range(Hq):
        qs, ks_, vs_ = head_slices(q, k, v, h)
        bi[h], bc[h] = oracle.bs_index(qs, ks_, 0, topk)
        refs.append(oracle.attn_bs(qs, ks_, vs_, 0, bi[h], bc[h]))
    out, lse = B.mi_block_sparse_attn(q, k, v, torch.from_numpy(bi).cuda(),
                                      torch.from_numpy(bc).cuda())
    torch.cuda.synchronize()
    for h in range(Hq):
        check_attn(out[h], lse[h], *refs[h], what=f"bs h{h}")


def test_block_sparse_attn_unusual_lists_and_empty_rows(bs_engine):
    """Block lists as a caller may pass them: unsorted, with duplicates, -1
    padding in the middle, entries past the query block or outside [0, N/64)
    (skipped and counted), counts above topk (clamped to topk) and rows with no
    block at all (out 0, lse -inf).  Odd counts leave half of a key-major tile
    unused; query blocks whose own block is chosen need the causal mask."""
    Hq, Hkv, N, d, topk = 4, 2, 1536, 128, 7
    q, k, v = rand_bf16(Hq, Hkv, N, d, 61)
    nB = N // 64
    rng = np.random.default_rng(3)
    bi = np.full((Hq, nB, topk), -1, np.int32)
    bc = np.zeros((Hq, nB), np.int32)
    for h in range(Hq):
        for bq in range(nB):
            c = int(rng.integers(0, topk + 3))  # above topk: clamped
            row = rng.integers(0, bq + 1, size=topk).astype(np.int32)
            for t in range(topk):
                r = rng.random()
                if r < 0.1:
                    row[t] = -1                    # padding, not counted
                elif r < 0.15:
                    row[t] = bq + 1 + int(rng.integers(0, 3))  # past the query block
                elif r < 0.18:
                    row[t] = -5                    # negative, not padding
            bi[h, bq], bc[h, bq] = row, c
    bc[0, 3] = 0                     # an empty query block
    bi[1, 5, :] = -1                 # only padding: empty too
    bc[1, 5] = topk
    n_bad = 0
    for h in range(Hq):
        for bq in range(nB):
            for t in range(min(int(bc[h, bq]), topk)):
                e = int(bi[h, bq, t])
                n_bad += e != -1 and (e < 0 or e > bq)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = B.mi_block_sparse_attn(q, k, v, torch.from_numpy(bi).cuda(),
                                      torch.from_numpy(bc).cuda(), err_count=err)
    torch.cuda.synchronize()
    assert int(err.item()) == n_bad
    for h in range(Hq):
        qs, ks_, vs_ = head_slices(q, k, v, h)
        ro, rl = oracle.attn_bs(qs, ks_, vs_, 0, bi[h], bc[h])
        check_attn(out[h], lse[h], ro, rl, what=f"bs lists h{h}")
    assert (out[0, 192:256] == 0).all() and torch.isneginf(lse[0, 192:256]).all()


def test_block_sparse_attn_rescales_mid_item(bs_engine):
    """A query block whose later key blocks score far above its first ones:
    the per-query reference max must move up mid-item (the lazy rescale of
    O and of the running sums), and a block scoring far below must not."""
    Hq, Hkv, N, d = 2, 1, 1024, 128
    q, k, v = rand_bf16(Hq, Hkv, N, d, 62)
    q, k = q.clone(), k.clone()
    qd = q[:, 640:704].float().mean(dim=(0, 1))
    k[0, 320:384] = (100.0 * qd / qd.norm()).to(torch.bfloat16)   # block 5: large scores
    k[0, 128:192] = (-100.0 * qd / qd.norm()).to(torch.bfloat16)  # block 2: tiny weights
    nB, topk = N // 64, 6
    bi = np.full((Hq, nB, topk), -1, np.int32)
    bc = np.zeros((Hq, nB), np.int32)
    for h in range(Hq):
        for bq in range(nB):
            lst = sorted({0, bq, bq // 2, 2 if bq >= 2 else 0, 5 if bq >= 5 else 0})
            bi[h, bq, :len(lst)] = lst
            bc[h, bq] = len(lst)
    out, lse = B.mi_block_sparse_attn(q, k, v, torch.from_numpy(bi).cuda(),
                                      torch.from_numpy(bc).cuda())
    torch.cuda.synchronize()
    for h in range(Hq):
        qs, ks_, vs_ = head_slices(q, k, v, h)
        ro, rl = oracle.attn_bs(qs, ks_, vs_, 0, bi[h], bc[h])
        check_attn(out[h], lse[h], ro, rl, what=f"bs rescale h{h}")


@pytest.mark.parametrize("Hq,Hkv,N,d,L,kv,ks", [
    (1, 1, 2048, 64, 64, 128, 256),
    (4, 1, 1088, 128, 64, 60, 40),
    (2, 2, 512, 128, 64, 5, 3),
])
def test_vs_attn_matches_oracle(Hq, Hkv, N, d, L, kv, ks):
    w = synth.workload("vs_n2k_h1_d64", Hq=Hq, Hkv=Hkv, N=N, d=d)
    x = synth.make_inputs(w, device="cuda")
    q, k, v = x["q"], x["k"], x["v"]
    vi = np.full((Hq, kv), -1, np.int32)
    si = np.full((Hq, ks), -1, np.int32)
    refs = []
    for h in range(Hq):
        qs, ks_, vs_ = head_slices(q, k, v, h)
        a, b, _, _ = oracle.vs_index(qs, ks_, 0, L, kv, ks)
        vi[h, :a.size], si[h, :b.size] = a, b
        refs.append(oracle.attn_vs(qs, ks_, vs_, 0, a, b))
    out, lse = B.mi_vs_sparse_attn(q, k, v, torch.from_numpy(vi).cuda(), torch.from_numpy(si).cuda())
    torch.cuda.synchronize()
    for h in range(Hq):
        check_attn(out[h], lse[h], *refs[h], what=f"vs h{h}")


@pytest.mark.parametrize("Hq,Hkv,N,d", [
    (4, 1, 1088, 128),   # GQA 4:1, ragged tail
    (2, 2, 576, 64),
    (1, 1, 64, 128),     # one block
])
def test_dense_attn_matches_oracle(Hq, Hkv, N, d):
    q, k, v = rand_bf16(Hq, Hkv, N, d, 31)
    out, lse = B.mi_dense_attn(q, k, v)
    torch.cuda.synchronize()
    for h in range(Hq):
        qs, ks_, vs_ = head_slices(q, k, v, h)
        check_attn(out[h], lse[h], *oracle.attn_dense(qs, ks_, vs_, 0), what=f"dense h{h}")


def test_vs_attn_unsorted_duplicates_and_empty_rows():
    """Unsorted, repeated index entries count once; rows before every key are empty."""
    q, k, v = rand_bf16(2, 1, 512, 128, 13)
    vi = np.array([[300, 5, 300, 77, 5, 200], [5, 5, 5, 5, 5, 5]], np.int32)
    si = np.array([[130, 0, 130], [-1, -1, -1]], np.int32)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = B.mi_vs_sparse_attn(q, k, v, torch.from_numpy(vi).cuda(),
                                   torch.from_numpy(si).cuda(), err_count=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for h in range(2):
        qs, ks_, vs_ = head_slices(q, k, v, h)
        ro, rl = oracle.attn_vs(qs, ks_, vs_, 0, vi[h], si[h][si[h] >= 0])
        check_attn(out[h], lse[h], ro, rl, what=f"h{h}")
    assert torch.all(out[1, :5] == 0) and torch.all(torch.isneginf(lse[1, :5]))


def test_vs_attn_gathered_columns_inside_query_blocks():
    """Many vertical columns, most of them inside the rows' own query blocks,
    with only far slash diagonals (so no diagonal tile covers them): each
    gathered chunk holds columns of several query blocks, and every row must
    take exactly the gathered columns j <= i.  Rows before the first column
    and every diagonal are empty."""
    q, k, v = rand_bf16(2, 1, 1088, 128, 21)
    rng = np.random.default_rng(5)
    vi = np.stack([rng.choice(1088, 400, replace=False) for _ in range(2)]).astype(np.int32)
    si = np.array([[700, 901], [512, 640]], np.int32)
    out, lse = B.mi_vs_sparse_attn(q, k, v, torch.from_numpy(vi).cuda(),
                                   torch.from_numpy(si).cuda())
    torch.cuda.synchronize()
    for h in range(2):
        qs, ks_, vs_ = head_slices(q, k, v, h)
        ro, rl = oracle.attn_vs(qs, ks_, vs_, 0, np.unique(vi[h]), np.unique(si[h]))
        check_attn(out[h], lse[h], ro, rl, what=f"vs gathered h{h}")


def test_vs_attn_counts_out_of_range_entries():
    q, k, v = rand_bf16(1, 1, 256, 64, 14)
    vi = torch.tensor([[3, 256, -7, 9]], dtype=torch.int32, device="cuda")
    si = torch.tensor([[0, 999]], dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, _ = B.mi_vs_sparse_attn(q, k, v, vi, si, err_count=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 3
    qs, ks_, vs_ = head_slices(q, k, v, 0)
    ro, rl = oracle.attn_vs(qs, ks_, vs_, 0, [3, 9], [0])
    check_attn(out[0], None, ro, rl)


def test_full_budgets_equal_dense_sdpa():
    """Budgets covering all columns / diagonals / blocks reproduce dense causal
    attention; cross-checked against torch SDPA on the GPU (library routine)."""
    Hq, Hkv, N, d = 4, 2, 768, 128
    q, k, v = rand_bf16(Hq, Hkv, N, d, 15)
    rep = Hq // Hkv
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.float()[None], k.float().repeat_interleave(rep, 0)[None],
        v.float().repeat_interleave(rep, 0)[None], is_causal=True)[0]
    every = torch.arange(N, dtype=torch.int32, device="cuda").repeat(Hq, 1)
    outs = [B.mi_vs_sparse_attn(q, k, v, every, every[:, :1] * 0 - 1)[0],
            B.mi_vs_sparse_attn(q, k, v, every[:, :1] * 0 - 1, every)[0],
            B.mi_ashape_attn(q, k, v, 0, N)[0]]
    nB = N // 64
    bi = torch.arange(nB, dtype=torch.int32, device="cuda").repeat(Hq, nB, 1)
    bc = torch.arange(1, nB + 1, dtype=torch.int32, device="cuda").repeat(Hq, 1)
    outs.append(B.mi_block_sparse_attn(q, k, v, bi, bc)[0])
    torch.cuda.synchronize()
    for o in outs:
        err = (o.float() - ref).abs()
        assert err.max().item() <= 1e-2 and err.mean().item() <= 1e-3


@pytest.mark.parametrize("N,d,L", [(1024, 128, 64), (576, 64, 64), (2560, 128, 100)])
def test_prefill_layer_mixed_matches_oracle(N, d, L, bs_engine):
    """The pattern router: mixed A-shape / VS / BS / dense heads in one launch
    (last_q = 100: the VS index merges two 64-row groups per head)."""
    w = synth.workload("mixed_n256k_llama3_8b", Hq=8, Hkv=2, N=N, d=d)
    x = synth.make_inputs(w, device="cuda")
    pattern = np.array([0, 1, 2, 3, 2, 0, 1, 3], np.int8)
    p = B.make_params(last_q=L, vertical_size=40, slash_size=60, topk_blocks=4, sink=64,
                      window=256)
    out, lse = B.mi_prefill_layer(x["q"], x["k"], x["v"], pattern, p, want_lse=True)
    torch.cuda.synchronize()
    for h in range(8):
        qs, ks_, vs_ = head_slices(x["q"], x["k"], x["v"], h)
        if pattern[h] == 0:
            ro, rl = oracle.attn_ashape(qs, ks_, vs_, 0, 64, 256)
        elif pattern[h] == 1:
            a, b, _, _ = oracle.vs_index(qs, ks_, 0, L, 40, 60)
            ro, rl = oracle.attn_vs(qs, ks_, vs_, 0, a, b)
        elif pattern[h] == 3:
            ro, rl = oracle.attn_dense(qs, ks_, vs_, 0)
        else:
            bi, bc = oracle.bs_index(qs, ks_, 0, 4)
            ro, rl = oracle.attn_bs(qs, ks_, vs_, 0, bi, bc)
        check_attn(out[h], lse[h], ro, rl, what=f"layer h{h} pattern {pattern[h]}")


def test_prefill_layer_per_head_parameters():
    """mi_prefill_layer_heads: every head with its own budgets (VS vertical /
    slash sizes, BS block count, A-shape sink and window), one launch."""
    w = synth.workload("mixed_n256k_llama3_8b", Hq=8, Hkv=2, N=1024, d=128)
    x = synth.make_inputs(w, device="cuda")
    pattern = np.array([1, 1, 2, 2, 0, 0, 3, 1], np.int8)
    ps = [B.make_params(vertical_size=20, slash_size=30),
          B.make_params(vertical_size=60, slash_size=90),
          B.make_params(topk_blocks=3),
          B.make_params(topk_blocks=6),
          B.make_params(sink=64, window=256),
          B.make_params(sink=10, window=100),
          B.make_params(),
          B.make_params(vertical_size=35, slash_size=50)]
    out, lse = B.mi_prefill_layer_heads(x["q"], x["k"], x["v"], pattern, ps, want_lse=True)
    torch.cuda.synchronize()
    for h in range(8):
        qs, ks_, vs_ = head_slices(x["q"], x["k"], x["v"], h)
        p = ps[h]
        if pattern[h] == 0:
            ro, rl = oracle.attn_ashape(qs, ks_, vs_, 0, p.sink, p.window)
        elif pattern[h] == 1:
            a, b, _, _ = oracle.vs_index(qs, ks_, 0, p.last_q, p.vertical_size, p.slash_size)
            ro, rl = oracle.attn_vs(qs, ks_, vs_, 0, a, b)
        elif pattern[h] == 2:
            bi, bc = oracle.bs_index(qs, ks_, 0, p.topk_blocks)
            ro, rl = oracle.attn_bs(qs, ks_, vs_, 0, bi, bc)
        else:
            ro, rl = oracle.attn_dense(qs, ks_, vs_, 0)
        check_attn(out[h], lse[h], ro, rl, what=f"per-head h{h} pattern {pattern[h]}")


def test_prefill_layer_stage_events_and_stream():
    q, k, v = rand_bf16(4, 1, 512, 128, 16)
    s = torch.cuda.Stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(B.MI_STAGE_EVENTS)]
    with torch.cuda.stream(s):
        out, _ = B.mi_prefill_layer(q, k, v, np.ones(4, np.int8),
                                    B.make_params(vertical_size=32, slash_size=32),
                                    stage_events=ev, stream=s)
    s.synchronize()
    assert ev[0].elapsed_time(ev[B.MI_STAGE_ATTN_DONE]) > 0
    assert ev[B.MI_STAGE_PREP_DONE].elapsed_time(ev[B.MI_STAGE_ATTN_DONE]) > 0
    assert torch.isfinite(out.float()).all()


def test_single_row_max_jump_rescales_within_warp():
    """One row's running max jumps by far more than 2^8 mid-stream while its
    warp neighbours' does not: the lazy O rescale runs for that row only."""
    N, d = 512, 128
    q, k, v = rand_bf16(1, 1, N, d, 21)
    q, k = q.clone(), k.clone()
    qd = q[0, 300].float()
    k[0, 256] = (20.0 * qd / qd.norm()).to(torch.bfloat16)  # s(300, 256) ~ 20 * |q|/sqrt(d)
    every = torch.arange(N, dtype=torch.int32, device="cuda")[None]
    none = torch.full((1, 1), -1, dtype=torch.int32, device="cuda")
    out, lse = B.mi_vs_sparse_attn(q, k, v, every, none)
    torch.cuda.synchronize()
    qs, ks_, vs_ = head_slices(q, k, v, 0)
    ro, rl = oracle.attn_dense(qs, ks_, vs_, 0)
    check_attn(out[0], lse[0], ro, rl)


def test_zz_no_device_wait_gave_up():
    """Every bounded wait of every launch above completed: nothing was recorded."""
    rec = B.mi_debug_wait_failure()
    assert rec["site"] == 0, rec
