"""The C-ABI library: it loads without a GPU, exports every symbol the header
declares, and rejects bad arguments on the host with the documented status
(on this GPU-less machine any launch would fail with MI_ERR_CUDA instead, so
getting the validation code shows nothing was launched)."""
import ctypes
import os
import re

import numpy as np
import pytest

from dynamic_sparse_attention_02_b200 import binding as B
from dynamic_sparse_attention_02_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.lib()


def header_functions():
    txt = open(os.path.join(ROOT, "include", "minfer.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(mi_\w+)\s*\(", txt)))


def test_exports_every_declared_symbol(lib):
    names = header_functions()
    assert len(names) == 19
    assert sorted(B.EXPORTS) == names
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code in range(5):
        assert B.mi_status_str(code)
    assert B.mi_status_str(99) == "unknown status"
    assert "sm_100a" in B.mi_version()


def test_bs_engine_selector(lib):
    assert lib.mi_set_bs_engine(2) == B.MI_ERR_INVALID_ARG
    assert lib.mi_set_bs_engine(-1) == B.MI_ERR_INVALID_ARG
    assert lib.mi_set_bs_engine(B.BS_ENGINE_KEY) == B.MI_OK
    assert lib.mi_set_bs_engine(B.BS_ENGINE_ROW) == B.MI_OK


FAKE = ctypes.c_void_p(0x1000)  # never dereferenced: validation runs first


def vs_index(lib, **kw):
    a = dict(q=FAKE, k=FAKE, Hq=4, Hkv=2, N=512, d=128, scale=0.0, last_q=64, kv=16, ks=32,
             heads=None, n_heads=0, v_idx=FAKE, s_idx=FAKE, vs=None, ss=None, ws=FAKE,
             ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return lib.mi_vs_index(a["q"], a["k"], a["Hq"], a["Hkv"], a["N"], a["d"], a["scale"],
                           a["last_q"], a["kv"], a["ks"], a["heads"], a["n_heads"], a["v_idx"],
                           a["s_idx"], a["vs"], a["ss"], a["ws"], a["ws_bytes"], a["stream"])


def test_vs_index_validation(lib):
    assert vs_index(lib, q=None) == B.MI_ERR_INVALID_ARG
    assert vs_index(lib, Hq=3) == B.MI_ERR_INVALID_ARG              # Hq % Hkv
    assert vs_index(lib, d=96) == B.MI_ERR_UNSUPPORTED
    assert vs_index(lib, N=500) == B.MI_ERR_UNSUPPORTED             # N % 64
    assert vs_index(lib, last_q=1024 + 64, N=4096) == B.MI_ERR_UNSUPPORTED
    assert vs_index(lib, last_q=1024) == B.MI_ERR_UNSUPPORTED       # last_q > N
    assert vs_index(lib, last_q=0) == B.MI_ERR_INVALID_ARG
    assert vs_index(lib, kv=-1) == B.MI_ERR_INVALID_ARG
    assert vs_index(lib, v_idx=None) == B.MI_ERR_INVALID_ARG
    assert vs_index(lib, ws_bytes=16) == B.MI_ERR_WORKSPACE
    assert vs_index(lib, ws=ctypes.c_void_p(0x1001)) == B.MI_ERR_WORKSPACE  # misaligned
    dup = (ctypes.c_int32 * 2)(1, 1)
    assert vs_index(lib, heads=dup, n_heads=2) == B.MI_ERR_INVALID_ARG
    bad = (ctypes.c_int32 * 1)(4)
    assert vs_index(lib, heads=bad, n_heads=1) == B.MI_ERR_INVALID_ARG
    assert vs_index(lib, Hq=512, Hkv=2) == B.MI_ERR_UNSUPPORTED     # > MI_MAX_HEADS


def test_attention_validation(lib):
    f = FAKE
    # block-sparse: block must be 64, topk >= 0
    assert lib.mi_block_sparse_attn(f, f, f, 4, 2, 512, 128, 0.0, f, f, 8, 32, None, 0, f, None,
                                    None, None, 0, None) == B.MI_ERR_UNSUPPORTED
    assert lib.mi_block_sparse_attn(f, f, f, 4, 2, 512, 128, 0.0, f, f, -1, 64, None, 0, f, None,
                                    None, None, 0, None) == B.MI_ERR_INVALID_ARG
    assert lib.mi_block_sparse_attn(f, f, None, 4, 2, 512, 128, 0.0, f, f, 8, 64, None, 0, f,
                                    None, None, None, 0, None) == B.MI_ERR_INVALID_ARG
    # A-shape: window >= 1, sink >= 0
    assert lib.mi_ashape_attn(f, f, f, 4, 2, 512, 128, 0.0, 64, 0, None, 0, f, None, None, None,
                              0, None) == B.MI_ERR_INVALID_ARG
    assert lib.mi_ashape_attn(f, f, f, 4, 2, 512, 128, 0.0, -1, 8, None, 0, f, None, None, None,
                              0, None) == B.MI_ERR_INVALID_ARG
    assert lib.mi_ashape_attn(f, f, f, 4, 2, 520, 128, 0.0, 4, 8, None, 0, f, None, None, None,
                              0, None) == B.MI_ERR_UNSUPPORTED
    # dense: v and out required, same shape rules
    assert lib.mi_dense_attn(f, f, None, 4, 2, 512, 128, 0.0, None, 0, f, None, None, None, 0,
                             None) == B.MI_ERR_INVALID_ARG
    assert lib.mi_dense_attn(f, f, f, 4, 2, 520, 128, 0.0, None, 0, f, None, None, None, 0,
                             None) == B.MI_ERR_UNSUPPORTED
    # VS attention: workspace
    assert lib.mi_vs_sparse_attn(f, f, f, 4, 2, 512, 128, 0.0, f, 8, f, 8, None, 0, f, None,
                                 None, f, 8, None) == B.MI_ERR_WORKSPACE
    # BS index
    assert lib.mi_bs_index(f, f, 4, 2, 512, 128, 0.0, 32, 8, None, 0, f, f, f, 1 << 30,
                           None) == B.MI_ERR_UNSUPPORTED


def test_prefill_layer_validation(lib):
    f = FAKE
    p = B.make_params()
    bad = np.array([0, 1, 2, 7], np.int8)
    assert lib.mi_prefill_layer(f, f, f, 4, 2, 512, 128, 0.0, bad.ctypes.data_as(ctypes.c_void_p),
                                ctypes.byref(p), f, None, None, f, 1 << 30, None,
                                None) == B.MI_ERR_INVALID_ARG
    good = np.array([0, 1, 2, 3], np.int8)  # A-shape, VS, BS, dense
    assert lib.mi_prefill_layer(f, f, f, 4, 2, 512, 128, 0.0, good.ctypes.data_as(ctypes.c_void_p),
                                ctypes.byref(p), f, None, None, f, 16, None,
                                None) == B.MI_ERR_WORKSPACE
    assert lib.mi_prefill_layer(f, f, f, 4, 2, 512, 128, 0.0, None, ctypes.byref(p), f, None,
                                None, f, 1 << 30, None, None) == B.MI_ERR_INVALID_ARG
    p2 = B.make_params(last_q=1024)
    assert lib.mi_prefill_layer(f, f, f, 4, 2, 512, 128, 0.0, good.ctypes.data_as(ctypes.c_void_p),
                                ctypes.byref(p2), f, None, None, f, 1 << 30, None,
                                None) == B.MI_ERR_UNSUPPORTED


def test_prefill_layer_heads_validation(lib):
    f = FAKE
    pat = np.array([1, 1, 2, 0], np.int8)
    ps = [B.make_params(vertical_size=10 * (h + 1), topk_blocks=h + 1, sink=h, window=h + 8)
          for h in range(4)]
    assert B.mi_prefill_workspace_bytes_heads(4, 2, 512, 128, pat, ps) > 0
    arr = (B.mi_params * 4)(*ps)
    ok = lib.mi_prefill_layer_heads(f, f, f, 4, 2, 512, 128, 0.0,
                                    pat.ctypes.data_as(ctypes.c_void_p),
                                    ctypes.cast(arr, ctypes.c_void_p), f, None, None, f, 16, None,
                                    None)
    assert ok == B.MI_ERR_WORKSPACE                      # valid plan, workspace too small
    ps[1] = B.make_params(last_q=128)                    # VS heads must share last_q
    arr = (B.mi_params * 4)(*ps)
    assert lib.mi_prefill_layer_heads(f, f, f, 4, 2, 512, 128, 0.0,
                                      pat.ctypes.data_as(ctypes.c_void_p),
                                      ctypes.cast(arr, ctypes.c_void_p), f, None, None, f,
                                      1 << 30, None, None) == B.MI_ERR_INVALID_ARG
    assert B.mi_prefill_workspace_bytes_heads(4, 2, 512, 128, pat, ps) == 0
    ps[1] = B.make_params(slash_tiles=2)                 # neither tiles nor ranges
    arr = (B.mi_params * 4)(*ps)
    assert lib.mi_prefill_layer_heads(f, f, f, 4, 2, 512, 128, 0.0,
                                      pat.ctypes.data_as(ctypes.c_void_p),
                                      ctypes.cast(arr, ctypes.c_void_p), f, None, None, f,
                                      1 << 30, None, None) == B.MI_ERR_INVALID_ARG
    ps[1] = B.make_params(slash_tiles=B.MI_SLASH_RANGES)  # one range head: a valid plan
    assert B.mi_prefill_workspace_bytes_heads(4, 2, 512, 128, pat, ps) > 0
    ps[1] = B.make_params()
    ps[3] = B.make_params(window=0)                      # A-shape window >= 1
    arr = (B.mi_params * 4)(*ps)
    assert lib.mi_prefill_layer_heads(f, f, f, 4, 2, 512, 128, 0.0,
                                      pat.ctypes.data_as(ctypes.c_void_p),
                                      ctypes.cast(arr, ctypes.c_void_p), f, None, None, f,
                                      1 << 30, None, None) == B.MI_ERR_INVALID_ARG


def test_vs_range_attn_validation(lib):
    f = FAKE
    args = [f, f, f, 4, 2, 512, 128, 0.0, f, 16, f, 32, None, 0, f, None, None]
    ws = B.mi_workspace_bytes(B.MI_OP_VS_ATTN, 4, 2, 512, 128, 0, 0, 16, 32)
    assert lib.mi_vs_range_attn(*args, f, ws - 256, None) == B.MI_ERR_WORKSPACE
    bad = list(args)
    bad[0] = None
    assert lib.mi_vs_range_attn(*bad, f, ws, None) == B.MI_ERR_INVALID_ARG
    bad = list(args)
    bad[3] = 3                                            # Hq % Hkv
    assert lib.mi_vs_range_attn(*bad, f, ws, None) == B.MI_ERR_INVALID_ARG
    bad = list(args)
    bad[5] = 500                                          # N % 64
    assert lib.mi_vs_range_attn(*bad, f, ws, None) == B.MI_ERR_UNSUPPORTED


def test_workspace_queries(lib):
    a = B.mi_workspace_bytes(B.MI_OP_VS_INDEX, 32, 8, 131072, 128, 32, 64, 1000, 6096)
    b = B.mi_workspace_bytes(B.MI_OP_VS_INDEX, 32, 8, 131072, 128, 4, 64, 1000, 6096)
    assert a > b > 0 and a % 256 == 0
    assert B.mi_workspace_bytes(B.MI_OP_VS_INDEX, 32, 8, 131072, 128, 32, 200000) == 0
    assert B.mi_workspace_bytes(B.MI_OP_BS_INDEX, 32, 8, 131072, 128) > 0
    assert B.mi_workspace_bytes(B.MI_OP_VS_ATTN, 32, 8, 131072, 128, 0, 0, 1000) > 0
    assert B.mi_workspace_bytes(99, 32, 8, 131072, 128) == 0
    p = B.make_params()
    full = B.mi_prefill_workspace_bytes(32, 8, 131072, 128, None, p)
    vs_only = B.mi_prefill_workspace_bytes(32, 8, 131072, 128, np.ones(32, np.int8), p)
    a_only = B.mi_prefill_workspace_bytes(32, 8, 131072, 128, np.zeros(32, np.int8), p)
    assert full >= vs_only > a_only >= 0


def test_vs_index_workspace_grows_with_row_groups(lib):
    """last_q > 64 splits each head's rows into 64-row groups whose partial
    column and diagonal scores (fp32 [heads][groups][N], two lists) live in the
    workspace until they are merged; last_q <= 64 needs none of them."""
    n, N = 32, 131072
    w64 = B.mi_workspace_bytes(B.MI_OP_VS_INDEX, 32, 8, N, 128, n, 64, 1000, 6096)
    w1 = B.mi_workspace_bytes(B.MI_OP_VS_INDEX, 32, 8, N, 128, n, 1, 1000, 6096)
    w200 = B.mi_workspace_bytes(B.MI_OP_VS_INDEX, 32, 8, N, 128, n, 200, 1000, 6096)
    row_stats = lambda L: 2 * n * L * (N // 2048) * 8 + 2 * n * L * 8
    assert w64 - w1 >= row_stats(64) - row_stats(1)
    groups = (200 + 63) // 64
    assert w200 - w64 >= 2 * n * groups * N * 4 + row_stats(200) - row_stats(64)


def test_vs_index_static_validation_and_capacity(lib):
    """The no-workspace entry point validates like mi_vs_index and rejects
    shapes whose scratch exceeds its fixed array -- both before any CUDA call."""
    f = FAKE
    assert lib.mi_vs_index_static(None, f, 4, 2, 512, 128, 0.0, 64, 16, 32, None, 0, f, f, None,
                                  None, None) == B.MI_ERR_INVALID_ARG
    assert lib.mi_vs_index_static(f, f, 4, 2, 500, 128, 0.0, 64, 16, 32, None, 0, f, f, None,
                                  None, None) == B.MI_ERR_UNSUPPORTED
    # 32 heads at N = 131072 need 36 MiB of scratch: more than the 16 MiB array
    assert lib.mi_vs_index_static(f, f, 32, 8, 131072, 128, 0.0, 64, 1000, 6096, None, 0, f, f,
                                  None, None, None) == B.MI_ERR_UNSUPPORTED
