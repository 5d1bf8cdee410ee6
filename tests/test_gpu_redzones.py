"""Out-of-bounds-write checks: every output lives inside a larger buffer whose
other bytes hold a sentinel, and after each entry point the sentinel must
survive everywhere the call is not documented to write.

What the header promises, checked here:
  * index outputs ([n_heads, ...], indexed by position in the head list) are
    written in full and nothing past them;
  * out / lse are written for the listed heads only (absolute head index),
    "heads not listed are not touched";
  * budgets past N (or past the causal block count) write -1 padding inside
    the row, never beyond it;
  * the workspace is used only up to the size the size query returns.
compute-sanitizer is not available on these machines; guard regions are the
stand-in for its out-of-bounds write check.
"""
import numpy as np
import pytest
import torch

from dynamic_sparse_attention_02_b200 import binding as B
from parity_util import rand_bf16

pytestmark = pytest.mark.gpu

GUARD = 4096  # elements of sentinel after every buffer
BF16_SENTINEL = 0x7FA1  # a bf16 NaN: attention never writes one
F32_SENTINEL_BITS = 0x7FC0BEEF  # a quiet NaN with a payload
I32_SENTINEL = -7


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from dynamic_sparse_attention_02_b200 import build
    build.build()


class Guarded:
    """A tensor of `shape` at the front of a flat buffer with GUARD sentinel
    elements behind it; `view` is the contiguous tensor handed to the library."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape))
        self.n = n
        if dtype == torch.bfloat16:
            self.raw = torch.full((n + GUARD,), BF16_SENTINEL, dtype=torch.int16, device="cuda")
            self.view = self.raw[:n].view(torch.bfloat16).view(*shape)
        elif dtype == torch.float32:
            self.raw = torch.full((n + GUARD,), F32_SENTINEL_BITS, dtype=torch.int32,
                                  device="cuda")
            self.view = self.raw[:n].view(torch.float32).view(*shape)
        else:
            self.raw = torch.full((n + GUARD,), I32_SENTINEL, dtype=torch.int32, device="cuda")
            self.view = self.raw[:n].view(*shape)
        self.sentinel = self.raw[-1].item()

    def guard_intact(self):
        return bool((self.raw[self.n:] == self.sentinel).all().item())

    def untouched(self, mask_rows):
        """True where every element of the leading-dimension rows in mask_rows
        still holds the sentinel."""
        rows = self.raw[:self.n].view(self.view.shape[0], -1)
        return bool((rows[mask_rows] == self.sentinel).all().item())

    def written(self, rows_sel):
        rows = self.raw[:self.n].view(self.view.shape[0], -1)
        return bool((rows[rows_sel] != self.sentinel).all().item())


def workspace(nbytes):
    """Workspace of exactly nbytes (256-aligned start) plus a sentinel tail."""
    raw = torch.full((nbytes + 4 * GUARD,), 0x5A, dtype=torch.uint8, device="cuda")
    return raw, raw[:nbytes]


def test_vs_index_head_subset_and_budgets_past_n():
    Hq, Hkv, N, d = 8, 2, 512, 128
    q, k, _ = rand_bf16(Hq, Hkv, N, d, 41)
    heads = [6, 1, 3]
    n = len(heads)
    kv, ks = N + 37, 100  # vertical budget past N: -1 padding inside the row
    vi, si = Guarded((n, kv), torch.int32), Guarded((n, ks), torch.int32)
    vsc, ssc = Guarded((n, N), torch.float32), Guarded((n, N), torch.float32)
    nb = B.mi_workspace_bytes(B.MI_OP_VS_INDEX, Hq, Hkv, N, d, n, 64, kv, ks)
    raw, ws = workspace(nb)
    import ctypes
    harr = (ctypes.c_int32 * n)(*heads)
    rc = B.lib().mi_vs_index(B._ptr(q), B._ptr(k), Hq, Hkv, N, d, 0.0, 64, kv, ks,
                             ctypes.cast(harr, ctypes.c_void_p), n, B._ptr(vi.view),
                             B._ptr(si.view), B._ptr(vsc.view), B._ptr(ssc.view), B._ptr(ws), nb,
                             B._stream(None))
    assert rc == B.MI_OK
    torch.cuda.synchronize()
    for g in (vi, si, vsc, ssc):
        assert g.guard_intact()
        assert g.written(slice(None))
    assert (vi.view[:, N:] == -1).all()
    assert (raw[nb:] == 0x5A).all(), "workspace used past its queried size"


def test_bs_index_head_subset():
    Hq, Hkv, N, d, topk = 4, 1, 1024, 128, 20
    q, k, _ = rand_bf16(Hq, Hkv, N, d, 42)
    heads = [3, 0]
    n, nB = len(heads), N // 64
    bi, bc = Guarded((n, nB, topk), torch.int32), Guarded((n, nB), torch.int32)
    nb = B.mi_workspace_bytes(B.MI_OP_BS_INDEX, Hq, Hkv, N, d, n)
    raw, ws = workspace(nb)
    import ctypes
    harr = (ctypes.c_int32 * n)(*heads)
    rc = B.lib().mi_bs_index(B._ptr(q), B._ptr(k), Hq, Hkv, N, d, 0.0, 64, topk,
                             ctypes.cast(harr, ctypes.c_void_p), n, B._ptr(bi.view),
                             B._ptr(bc.view), B._ptr(ws), nb, B._stream(None))
    assert rc == B.MI_OK
    torch.cuda.synchronize()
    assert bi.guard_intact() and bc.guard_intact()
    assert bi.written(slice(None)) and bc.written(slice(None))
    cnt = bc.view.cpu().numpy()
    assert np.array_equal(cnt, np.minimum(topk, np.arange(nB) + 1)[None].repeat(n, 0))
    # entries past the count are -1 padding
    b = bi.view.cpu().numpy()
    for p in range(n):
        for bq in range(nB):
            assert np.all(b[p, bq, cnt[p, bq]:] == -1)
    assert (raw[nb:] == 0x5A).all(), "workspace used past its queried size"


def _attn_call(which, q, k, v, heads, out, lse, ws):
    N = q.shape[1]
    if which in ("vs", "vs_range"):
        vi = torch.tensor([[0, 5, 300, N - 1, -1]] * len(heads), dtype=torch.int32,
                          device="cuda")
        si = torch.tensor([[0, 64, 200, -1]] * len(heads), dtype=torch.int32, device="cuda")
        B.mi_vs_sparse_attn(q, k, v, vi, si, heads=heads, out=out, lse=lse, ws=ws,
                            ranges=which == "vs_range")
    elif which in ("bs", "bs_key"):
        nB = N // 64
        bi = torch.full((len(heads), nB, 3), -1, dtype=torch.int32, device="cuda")
        for bq in range(nB):
            bi[:, bq, 0] = bq
            bi[:, bq, 1] = 0
        bc = torch.full((len(heads), nB), 2, dtype=torch.int32, device="cuda")
        bc[:, 0] = 1
        B.mi_set_bs_engine(B.BS_ENGINE_KEY if which == "bs_key" else B.BS_ENGINE_ROW)
        try:
            B.mi_block_sparse_attn(q, k, v, bi, bc, heads=heads, out=out, lse=lse)
        finally:
            B.mi_set_bs_engine(B.BS_ENGINE_ROW)
    elif which == "ashape":
        B.mi_ashape_attn(q, k, v, 64, 128, heads=heads, out=out, lse=lse)
    else:
        B.mi_dense_attn(q, k, v, heads=heads, out=out, lse=lse)


@pytest.mark.parametrize("which", ["vs", "vs_range", "bs", "bs_key", "ashape", "dense"])
def test_attention_touches_listed_heads_only(which):
    Hq, Hkv, N, d = 6, 2, 640, 128
    q, k, v = rand_bf16(Hq, Hkv, N, d, 43)
    heads = [5, 0, 2]
    out, lse = Guarded((Hq, N, d), torch.bfloat16), Guarded((Hq, N), torch.float32)
    ws = None
    if which in ("vs", "vs_range"):
        nb = B.mi_workspace_bytes(B.MI_OP_VS_ATTN, Hq, Hkv, N, d, len(heads), 0, 5)
        raw, ws = workspace(nb)
    _attn_call(which, q, k, v, heads, out.view, lse.view, ws)
    torch.cuda.synchronize()
    listed = torch.zeros(Hq, dtype=torch.bool, device="cuda")
    listed[heads] = True
    for g in (out, lse):
        assert g.guard_intact()
        assert g.untouched(~listed), "a head that was not listed was written"
        assert g.written(listed)
    if ws is not None:
        assert (raw[nb:] == 0x5A).all(), "workspace used past its queried size"


def test_prefill_layer_stays_inside_out_lse_and_workspace():
    Hq, Hkv, N, d = 6, 2, 768, 128
    q, k, v = rand_bf16(Hq, Hkv, N, d, 44)
    pattern = np.array([0, 1, 2, 3, 1, 2], np.int8)
    p = B.make_params(last_q=64, vertical_size=48, slash_size=64, topk_blocks=4, sink=64,
                      window=256)
    out, lse = Guarded((Hq, N, d), torch.bfloat16), Guarded((Hq, N), torch.float32)
    nb = B.mi_prefill_workspace_bytes(Hq, Hkv, N, d, pattern, p)
    raw, ws = workspace(nb)
    B.mi_prefill_layer(q, k, v, pattern, p, out=out.view, lse=lse.view, ws=ws)
    torch.cuda.synchronize()
    for g in (out, lse):
        assert g.guard_intact()
        assert g.written(slice(None))
    assert (raw[nb:] == 0x5A).all(), "workspace used past its queried size"
