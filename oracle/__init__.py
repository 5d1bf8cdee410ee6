"""CPU oracle for MInference dynamic sparse prefill -- test infrastructure only.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  It wraps ``minfer_oracle.c`` (plain fp64 loops,
see that file's header for the definitions and readings it follows) through
ctypes and never touches the CUDA library.

All array arguments are numpy arrays; bf16 tensors are widened to float32
(exact) before they are passed in.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "minfer_oracle.c")
_LIB = os.path.join(_HERE, "libminfer_oracle.so")
# A prebuilt variant of the oracle to load instead (the mutation test plants
# mistakes in copies of minfer_oracle.c and runs the pins against each).
_VARIANT = os.environ.get("MINFER_ORACLE_LIB")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle (gcc, -O2 -fopenmp) into oracle/libminfer_oracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(_VARIANT or build())
            P = ctypes.c_void_p
            I, I64, D = ctypes.c_int, ctypes.c_int64, ctypes.c_double
            lib.oracle_vs_scores.argtypes = [P, P, I, I, I, I, D, I, I, P, P]
            lib.oracle_topk.argtypes = [P, I64, I64, P]
            lib.oracle_topk.restype = I64
            lib.oracle_bs_index.argtypes = [P, P, I, I, I, I, D, I, I, I, P, P, P]
            lib.oracle_slash_deltas.argtypes = [P, I64, I, I, P]
            lib.oracle_attn_dense_rows.argtypes = [P, P, P, I, I, I, I, D, I, P, I64, P, P]
            lib.oracle_attn_ashape_rows.argtypes = [P, P, P, I, I, I, I, D, I, I, I, P, I64, P, P]
            lib.oracle_attn_vs_rows.argtypes = [P, P, P, I, I, I, I, D, I, P, I64, P, I64, I, P,
                                                I64, P, P]
            lib.oracle_attn_bs_rows.argtypes = [P, P, P, I, I, I, I, D, I, P, P, I, I, P, I64, P,
                                                P]
            lib.oracle_attn_vs_range_rows.argtypes = [P, P, P, I, I, I, I, D, I, P, I64, P, I64,
                                                      I, P, I64, P, P]
            lib.oracle_vs_mask.argtypes = [I, P, I64, P, I64, I, I, P]
            lib.oracle_num_threads.restype = I
            _lib = lib
    return _lib


def _f32(x):
    import torch  # local: the oracle itself does not need torch
    if isinstance(x, torch.Tensor):
        x = x.detach().to("cpu", torch.float32).numpy()
    return np.ascontiguousarray(x, dtype=np.float32)


def _i32(x):
    return np.ascontiguousarray(np.asarray(x), dtype=np.int32)


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None and a.size else None


def _check(rc, name):
    if rc != 0:
        raise RuntimeError(f"oracle {name} failed with code {rc}")


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def vs_scores(q, k, h, last_q, scale=None):
    """(vertical, slash) fp64 [N] for query head h (see oracle_vs_scores)."""
    q, k = _f32(q), _f32(k)
    Hq, N, d = q.shape
    Hkv = k.shape[0]
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    vert = np.zeros(N, np.float64)
    sl = np.zeros(N, np.float64)
    _check(_load().oracle_vs_scores(_ptr(q), _ptr(k), Hq, Hkv, N, d, scale, last_q, h,
                                    _ptr(vert), _ptr(sl)), "vs_scores")
    return vert, sl


def topk(score, k):
    """Indices of the top-k by (score desc, index asc), returned sorted ascending."""
    s = np.ascontiguousarray(score, dtype=np.float64)
    out = np.zeros(max(1, min(k, s.size)), np.int64)
    m = _load().oracle_topk(_ptr(s), s.size, k, _ptr(out))
    if m < 0:
        raise RuntimeError("oracle topk failed")
    return out[:m]


def vs_index(q, k, h, last_q, vertical_size, slash_size, scale=None):
    """(v_idx, s_idx, vertical, slash) for query head h."""
    vert, sl = vs_scores(q, k, h, last_q, scale)
    return topk(vert, vertical_size), topk(sl, slash_size), vert, sl


def bs_index(q, k, h, topk_blocks, block=64, scale=None, want_scores=False):
    """(blk_idx int32 [nB, topk] (-1 padded), blk_cnt int32 [nB][, scores fp64 [nB, nB]])."""
    q, k = _f32(q), _f32(k)
    Hq, N, d = q.shape
    Hkv = k.shape[0]
    nB = N // block
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    idx = np.full((nB, max(topk_blocks, 1)), -1, np.int32)
    cnt = np.zeros(nB, np.int32)
    sc = np.zeros((nB, nB), np.float64) if want_scores else None
    _check(_load().oracle_bs_index(_ptr(q), _ptr(k), Hq, Hkv, N, d, scale, block, topk_blocks,
                                   h, _ptr(idx), _ptr(cnt), _ptr(sc)), "bs_index")
    idx = idx[:, :topk_blocks]
    return (idx, cnt, sc) if want_scores else (idx, cnt)


def slash_deltas(s_idx, N, block=64):
    """uint8 [N/block]: 1 where a selected diagonal touches block-diagonal delta."""
    s = _i32(s_idx)
    D = np.zeros(N // block, np.uint8)
    _check(_load().oracle_slash_deltas(_ptr(s), s.size, N, block, _ptr(D)), "slash_deltas")
    return D


def _attn_common(q, k, v, rows):
    q, k, v = _f32(q), _f32(k), _f32(v)
    Hq, N, d = q.shape
    rows = np.ascontiguousarray(np.arange(N) if rows is None else rows, dtype=np.int64)
    out = np.zeros((rows.size, d), np.float64)
    lse = np.zeros(rows.size, np.float64)
    return q, k, v, Hq, k.shape[0], N, d, rows, out, lse


def attn_dense(q, k, v, h, rows=None, scale=None):
    """Dense causal attention rows of head h: (out fp64 [rows, d], lse fp64 [rows])."""
    q, k, v, Hq, Hkv, N, d, rows, out, lse = _attn_common(q, k, v, rows)
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    _check(_load().oracle_attn_dense_rows(_ptr(q), _ptr(k), _ptr(v), Hq, Hkv, N, d, scale, h,
                                          _ptr(rows), rows.size, _ptr(out), _ptr(lse)), "dense")
    return out, lse


def attn_ashape(q, k, v, h, sink, window, rows=None, scale=None):
    q, k, v, Hq, Hkv, N, d, rows, out, lse = _attn_common(q, k, v, rows)
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    _check(_load().oracle_attn_ashape_rows(_ptr(q), _ptr(k), _ptr(v), Hq, Hkv, N, d, scale, h,
                                           sink, window, _ptr(rows), rows.size, _ptr(out),
                                           _ptr(lse)), "ashape")
    return out, lse


def attn_vs(q, k, v, h, v_idx, s_idx, rows=None, block=64, scale=None):
    q, k, v, Hq, Hkv, N, d, rows, out, lse = _attn_common(q, k, v, rows)
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    vi, si = _i32(v_idx), _i32(s_idx)
    _check(_load().oracle_attn_vs_rows(_ptr(q), _ptr(k), _ptr(v), Hq, Hkv, N, d, scale, h,
                                       _ptr(vi), vi.size, _ptr(si), si.size, block, _ptr(rows),
                                       rows.size, _ptr(out), _ptr(lse)), "vs")
    return out, lse


def attn_vs_range(q, k, v, h, v_idx, s_idx, rows=None, block=64, scale=None):
    """Vertical-Slash attention rows with range-based slash tiles: diagonal o
    covers keys [64 bq - o, 64 bq + 63 - o] for query block bq."""
    q, k, v, Hq, Hkv, N, d, rows, out, lse = _attn_common(q, k, v, rows)
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    vi, si = _i32(v_idx), _i32(s_idx)
    _check(_load().oracle_attn_vs_range_rows(_ptr(q), _ptr(k), _ptr(v), Hq, Hkv, N, d, scale, h,
                                             _ptr(vi), vi.size, _ptr(si), si.size, block,
                                             _ptr(rows), rows.size, _ptr(out), _ptr(lse)),
           "vs_range")
    return out, lse


def vs_mask(N, v_idx, s_idx, range_tiles=False, block=64):
    """The causal Vertical-Slash mask, bool [N, N]: whole 64x64 slash tiles, or
    range-based ones (range_tiles=True)."""
    vi, si = _i32(v_idx), _i32(s_idx)
    m = np.zeros((N, N), np.uint8)
    _check(_load().oracle_vs_mask(N, _ptr(vi), vi.size, _ptr(si), si.size, block,
                                  1 if range_tiles else 0, _ptr(m)), "vs_mask")
    return m.astype(bool)


def attn_bs(q, k, v, h, blk_idx, blk_cnt, rows=None, block=64, scale=None):
    q, k, v, Hq, Hkv, N, d, rows, out, lse = _attn_common(q, k, v, rows)
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    bi, bc = _i32(blk_idx), _i32(blk_cnt)
    topk_ = bi.shape[1] if bi.ndim == 2 else 0
    _check(_load().oracle_attn_bs_rows(_ptr(q), _ptr(k), _ptr(v), Hq, Hkv, N, d, scale, h,
                                       _ptr(bi), _ptr(bc), topk_, block, _ptr(rows), rows.size,
                                       _ptr(out), _ptr(lse)), "bs")
    return out, lse
