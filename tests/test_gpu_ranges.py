"""Range slash tiles (MI_SLASH_RANGES) against the oracle's range reading.

Diagonal o gives query block bq the keys 64 bq - o .. 64 bq + 63 - o; the
engine covers each super tile's kept keys with 64-key windows that start at
any key, and masks every row to the keys of its own block.  Cases: the
generator's indices at several sizes (ragged tails, GQA, d = 64 and 128),
hand-placed diagonals at and around multiples of 64 (where a range is
aligned, or splits across two blocks), clusters that merge into long runs,
diagonals near N, vertical columns inside and outside the ranges, unsorted
and repeated entries, and the layer entry points with the flag set per head.
"""
import numpy as np
import pytest
import torch

import oracle
from dynamic_sparse_attention_02_b200 import binding as B
from dynamic_sparse_attention_02_b200 import synth
from parity_util import check_attn, head_slices, rand_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from dynamic_sparse_attention_02_b200 import build
    build.build()


def _check_heads(q, k, v, vi, si, out, lse, what):
    for h in range(q.shape[0]):
        qs, ks_, vs_ = head_slices(q, k, v, h)
        ro, rl = oracle.attn_vs_range(qs, ks_, vs_, 0, vi[h], si[h])
        check_attn(out[h], lse[h], ro, rl, what=f"{what} h{h}")


@pytest.mark.parametrize("Hq,Hkv,N,d,L,kv,ks", [
    (1, 1, 2048, 64, 64, 128, 256),
    (4, 1, 1088, 128, 64, 60, 40),     # GQA 4:1, ragged tail (N % 256 != 0)
    (2, 2, 512, 128, 64, 5, 3),
    (2, 1, 4160, 128, 64, 300, 900),   # many windows per super tile, ragged
])
def test_vs_range_attn_matches_oracle(Hq, Hkv, N, d, L, kv, ks):
    w = synth.workload("vs_n2k_h1_d64", Hq=Hq, Hkv=Hkv, N=N, d=d)
    x = synth.make_inputs(w, device="cuda")
    q, k, v = x["q"], x["k"], x["v"]
    vi = np.full((Hq, kv), -1, np.int32)
    si = np.full((Hq, ks), -1, np.int32)
    for h in range(Hq):
        qs, ks_, _ = head_slices(q, k, v, h)
        a, b, _, _ = oracle.vs_index(qs, ks_, 0, L, kv, ks)
        vi[h, :a.size], si[h, :b.size] = a, b
    out, lse = B.mi_vs_sparse_attn(q, k, v, torch.from_numpy(vi).cuda(),
                                   torch.from_numpy(si).cuda(), ranges=True)
    torch.cuda.synchronize()
    _check_heads(q, k, v, vi, si, out, lse, "range")


@pytest.mark.parametrize("d", [64, 128])
def test_vs_range_attn_hand_placed_diagonals(d):
    """Aligned and unaligned ranges, clusters, far and near-N diagonals,
    columns inside and outside the ranges, unsorted and repeated entries."""
    N = 1344  # 5.25 super tiles
    q, k, v = rand_bf16(3, 1, N, d, 71)
    si = np.array([
        [0, 1, 63, 64, 65, 127, 128, 200, N - 1, 300, 301, 305, 310, 64, 0],   # repeats
        [700, 64, 128, 192, 256, 512, 1024, 1280, -1, -1, -1, -1, -1, -1, -1],  # aligned only
        [33, 97, 161, 900, 901, 902, 1200, 1300, 1343, 5, 6, 7, 8, 9, 10],
    ], np.int32)
    vi = np.array([
        [3, 900, 64, 1000, 1343, 500, 501, 3, 640, 641],
        [0, 1, 2, 700, 701, 130, 129, 128, 1100, 1200],
        [1300, 20, 40, 60, 80, 100, 1330, 1331, 1332, 1333],
    ], np.int32)
    out, lse = B.mi_vs_sparse_attn(q, k, v, torch.from_numpy(vi).cuda(),
                                   torch.from_numpy(si).cuda(), ranges=True)
    torch.cuda.synchronize()
    _check_heads(q, k, v, vi, [s[s >= 0] for s in si], out, lse, f"hand d{d}")


def test_vs_range_attn_differs_from_tiles_where_ranges_are_narrower():
    """One unaligned diagonal: tiles take two whole 64x64 blocks per query
    block, ranges one 64-key run, so the outputs differ, each matching its
    own reading of the oracle."""
    N, d = 768, 128
    q, k, v = rand_bf16(1, 1, N, d, 72)
    vi = np.array([[0]], np.int32)
    si = np.array([[100]], np.int32)
    vt, st = torch.from_numpy(vi).cuda(), torch.from_numpy(si).cuda()
    out_r, lse_r = B.mi_vs_sparse_attn(q, k, v, vt, st, ranges=True)
    out_t, lse_t = B.mi_vs_sparse_attn(q, k, v, vt, st)
    torch.cuda.synchronize()
    qs, ks_, vs_ = head_slices(q, k, v, 0)
    ro, rl = oracle.attn_vs_range(qs, ks_, vs_, 0, vi[0], si[0])
    to, tl = oracle.attn_vs(qs, ks_, vs_, 0, vi[0], si[0])
    check_attn(out_r[0], lse_r[0], ro, rl, what="ranges")
    check_attn(out_t[0], lse_t[0], to, tl, what="tiles")
    assert (out_r[0].float() - out_t[0].float()).abs().max().item() > 0.05


def test_vs_range_attn_counts_out_of_range_entries():
    N, d = 512, 128
    q, k, v = rand_bf16(1, 1, N, d, 73)
    vi = torch.tensor([[5, N, -3, 7]], dtype=torch.int32, device="cuda")
    si = torch.tensor([[70, -1, N + 4, 0]], dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = B.mi_vs_sparse_attn(q, k, v, vi, si, err_count=err, ranges=True)
    torch.cuda.synchronize()
    assert int(err.item()) == 3  # N, -3 and N + 4; -1 is padding
    qs, ks_, vs_ = head_slices(q, k, v, 0)
    ro, rl = oracle.attn_vs_range(qs, ks_, vs_, 0, np.array([5, 7]), np.array([70, 0]))
    check_attn(out[0], lse[0], ro, rl, what="out-of-range entries")


def test_prefill_layer_with_range_heads():
    """mi_prefill_layer_heads with the flag on some VS heads only, beside
    tile-read VS heads and the other patterns in the same launch."""
    w = synth.workload("mixed_n256k_llama3_8b", Hq=8, Hkv=2, N=1088, d=128)
    x = synth.make_inputs(w, device="cuda")
    pattern = np.array([1, 1, 2, 0, 1, 3, 1, 2], np.int8)
    R, T = B.MI_SLASH_RANGES, B.MI_SLASH_BLOCKS
    ps = [B.make_params(vertical_size=40, slash_size=60, slash_tiles=R),
          B.make_params(vertical_size=40, slash_size=60, slash_tiles=T),
          B.make_params(topk_blocks=4),
          B.make_params(sink=64, window=256),
          B.make_params(vertical_size=20, slash_size=90, slash_tiles=R),
          B.make_params(),
          B.make_params(vertical_size=70, slash_size=30, slash_tiles=T),
          B.make_params(topk_blocks=3)]
    out, lse = B.mi_prefill_layer_heads(x["q"], x["k"], x["v"], pattern, ps, want_lse=True)
    torch.cuda.synchronize()
    for h in range(8):
        qs, ks_, vs_ = head_slices(x["q"], x["k"], x["v"], h)
        p = ps[h]
        if pattern[h] == 1:
            a, b, _, _ = oracle.vs_index(qs, ks_, 0, p.last_q, p.vertical_size, p.slash_size)
            fn = oracle.attn_vs_range if p.slash_tiles == R else oracle.attn_vs
            ro, rl = fn(qs, ks_, vs_, 0, a, b)
        elif pattern[h] == 2:
            bi, bc = oracle.bs_index(qs, ks_, 0, p.topk_blocks)
            ro, rl = oracle.attn_bs(qs, ks_, vs_, 0, bi, bc)
        elif pattern[h] == 0:
            ro, rl = oracle.attn_ashape(qs, ks_, vs_, 0, p.sink, p.window)
        else:
            ro, rl = oracle.attn_dense(qs, ks_, vs_, 0)
        check_attn(out[h], lse[h], ro, rl, what=f"layer h{h} pattern {pattern[h]}")


def test_prefill_layer_all_range_heads_one_params():
    """mi_prefill_layer with one mi_params whose slash_tiles is RANGES."""
    w = synth.workload("vs_n128k_llama3_8b", Hq=4, Hkv=1, N=2112, d=128)
    x = synth.make_inputs(w, device="cuda")
    pattern = np.ones(4, np.int8)
    p = B.make_params(vertical_size=100, slash_size=200, slash_tiles=B.MI_SLASH_RANGES)
    out, lse = B.mi_prefill_layer(x["q"], x["k"], x["v"], pattern, p, want_lse=True)
    torch.cuda.synchronize()
    for h in range(4):
        qs, ks_, vs_ = head_slices(x["q"], x["k"], x["v"], h)
        a, b, _, _ = oracle.vs_index(qs, ks_, 0, 64, 100, 200)
        ro, rl = oracle.attn_vs_range(qs, ks_, vs_, 0, a, b)
        check_attn(out[h], lse[h], ro, rl, what=f"all-range layer h{h}")


@pytest.mark.parametrize("N,d,si,vi", [
    (64, 128, [0, 5, 63], [-1]),            # one block: every range starts at or before key 0
    (192, 64, [191, 1, 64], [100]),         # the last diagonal reaches key 0 of the last block only
    (320, 128, [130, 129, 128, 127], []),   # four adjacent diagonals merge into one run
    (256, 128, [-1, -1], [0, 255]),         # no diagonal: the verticals alone
])
def test_vs_range_attn_small_edges(N, d, si, vi):
    q, k, v = rand_bf16(1, 1, N, d, 74)
    s = np.array([si], np.int32)
    c = np.array([vi if vi else [-1]], np.int32)
    out, lse = B.mi_vs_sparse_attn(q, k, v, torch.from_numpy(c).cuda(), torch.from_numpy(s).cuda(),
                                   ranges=True)
    torch.cuda.synchronize()
    qs, ks_, vs_ = head_slices(q, k, v, 0)
    ro, rl = oracle.attn_vs_range(qs, ks_, vs_, 0, c[0][c[0] >= 0], s[0][s[0] >= 0])
    check_attn(out[0], lse[0], ro, rl, what=f"range edge N={N}")
