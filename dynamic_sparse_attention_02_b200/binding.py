"""Thin ctypes binding over libminfer.so (include/minfer.h).

Argument marshalling only: every step of the computation runs in the
library's CUDA kernels.  Functions carry the C names; they take torch CUDA
tensors (torch is used for device memory and streams), allocate outputs and
workspace with torch when the caller does not pass them, and raise
``MinferError`` on a non-zero status.  There is no fallback: if the library
is missing or a CUDA call fails, the call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libminfer.so")

MI_OK, MI_ERR_INVALID_ARG, MI_ERR_UNSUPPORTED, MI_ERR_WORKSPACE, MI_ERR_CUDA = range(5)
MI_PATTERN_ASHAPE, MI_PATTERN_VS, MI_PATTERN_BS, MI_PATTERN_DENSE = 0, 1, 2, 3
MI_OP_VS_INDEX, MI_OP_BS_INDEX, MI_OP_VS_ATTN, MI_OP_BS_ATTN, MI_OP_ASHAPE_ATTN = 1, 2, 3, 4, 5
MI_OP_DENSE_ATTN = 6
MI_STAGE_START, MI_STAGE_INDEX_DONE, MI_STAGE_PREP_DONE, MI_STAGE_ATTN_DONE, MI_STAGE_EVENTS = (
    0, 1, 2, 3, 4)
MI_MAX_HEADS = 256
MI_BLOCK = 64

# every symbol include/minfer.h declares
EXPORTS = ["mi_status_str", "mi_last_cuda_error", "mi_version", "mi_workspace_bytes",
           "mi_prefill_workspace_bytes", "mi_vs_index", "mi_bs_index", "mi_vs_sparse_attn",
           "mi_vs_range_attn", "mi_block_sparse_attn", "mi_ashape_attn", "mi_prefill_layer",
           "mi_debug_wait_failure",
           "mi_vs_index_static", "mi_dense_attn", "mi_prefill_workspace_bytes_heads",
           "mi_prefill_layer_heads", "mi_debug_set_wait_budget", "mi_set_bs_engine"]


class MinferError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = f"{fn}: {_lib_handle().mi_status_str(status).decode()} (status {status})"
        if status == MI_ERR_CUDA:
            msg += f", cudaError {_lib_handle().mi_last_cuda_error()}"
        super().__init__(msg)


class mi_params(ctypes.Structure):
    _fields_ = [("last_q", ctypes.c_int), ("vertical_size", ctypes.c_int),
                ("slash_size", ctypes.c_int), ("topk_blocks", ctypes.c_int),
                ("sink", ctypes.c_int), ("window", ctypes.c_int), ("slash_tiles", ctypes.c_int)]


_lib = None


def _lib_handle():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run "
                               "`python -m dynamic_sparse_attention_02_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        P, I, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        lib.mi_status_str.argtypes = [I]
        lib.mi_status_str.restype = ctypes.c_char_p
        lib.mi_last_cuda_error.restype = I
        lib.mi_version.restype = ctypes.c_char_p
        lib.mi_workspace_bytes.argtypes = [I] * 10
        lib.mi_workspace_bytes.restype = SZ
        lib.mi_prefill_workspace_bytes.argtypes = [I, I, I, I, P, ctypes.POINTER(mi_params)]
        lib.mi_prefill_workspace_bytes.restype = SZ
        lib.mi_vs_index.argtypes = [P, P, I, I, I, I, F, I, I, I, P, I, P, P, P, P, P, SZ, P]
        lib.mi_bs_index.argtypes = [P, P, I, I, I, I, F, I, I, P, I, P, P, P, SZ, P]
        lib.mi_vs_sparse_attn.argtypes = [P, P, P, I, I, I, I, F, P, I, P, I, P, I, P, P, P, P,
                                          SZ, P]
        lib.mi_vs_range_attn.argtypes = lib.mi_vs_sparse_attn.argtypes
        lib.mi_block_sparse_attn.argtypes = [P, P, P, I, I, I, I, F, P, P, I, I, P, I, P, P, P,
                                             P, SZ, P]
        lib.mi_ashape_attn.argtypes = [P, P, P, I, I, I, I, F, I, I, P, I, P, P, P, P, SZ, P]
        lib.mi_prefill_layer.argtypes = [P, P, P, I, I, I, I, F, P, ctypes.POINTER(mi_params),
                                         P, P, P, P, SZ, P, P]
        lib.mi_debug_wait_failure.argtypes = [P]
        lib.mi_vs_index_static.argtypes = [P, P, I, I, I, I, F, I, I, I, P, I, P, P, P, P, P]
        lib.mi_dense_attn.argtypes = [P, P, P, I, I, I, I, F, P, I, P, P, P, P, SZ, P]
        lib.mi_prefill_workspace_bytes_heads.argtypes = [I, I, I, I, P, P]
        lib.mi_prefill_workspace_bytes_heads.restype = SZ
        lib.mi_prefill_layer_heads.argtypes = [P, P, P, I, I, I, I, F, P, P, P, P, P, P, SZ, P,
                                               P]
        lib.mi_debug_set_wait_budget.argtypes = [ctypes.c_longlong]
        lib.mi_set_bs_engine.argtypes = [ctypes.c_int]
        for name in EXPORTS[5:]:
            if name != "mi_prefill_workspace_bytes_heads":
                getattr(lib, name).restype = I
        _lib = lib
    return _lib


def lib():
    """The loaded ctypes library (raises if it is not built)."""
    return _lib_handle()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _heads(heads, Hq):
    if heads is None:
        return None, Hq, None
    arr = np.ascontiguousarray(np.asarray(heads, dtype=np.int32))
    return arr, int(arr.size), arr.ctypes.data_as(ctypes.c_void_p)


def _check(fn, rc):
    if rc != MI_OK:
        raise MinferError(fn, rc)


def _dev(name, t, dtype, shape, device):
    """The library reads raw device pointers with the layout the header states:
    refuse anything else before a pointer reaches a kernel (a host pointer, a
    wrong element type or a strided view would be read as dense device data)."""
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor, got {type(t).__name__}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if not _device_ok(t, device):
        raise ValueError(f"{name} must be on {device or 'a CUDA device'}, got {t.device}")


def _device_ok(t, device):
    return t.device.type == "cuda" and (device is None or t.device == device)


def _shape(q, k, v=None):
    """(Hq, Hkv, N, d) of bf16 [Hq, N, d] q and [Hkv, N, d] k (and v) on one device."""
    if not isinstance(q, torch.Tensor) or q.dim() != 3:
        raise ValueError("q must be a 3-D tensor [Hq, N, d]")
    Hq, N, d = q.shape
    _dev("q", q, torch.bfloat16, None, None)
    if not isinstance(k, torch.Tensor) or k.dim() != 3:
        raise ValueError("k must be a 3-D tensor [Hkv, N, d]")
    Hkv = k.shape[0]
    _dev("k", k, torch.bfloat16, (Hkv, N, d), q.device)
    _dev("v", v, torch.bfloat16, (Hkv, N, d), q.device)
    return Hq, Hkv, N, d


def _host_array(name, a, dtype, n):
    arr = np.ascontiguousarray(np.asarray(a, dtype=dtype))
    if arr.ndim != 1 or arr.size != n:
        raise ValueError(f"{name} must hold {n} entries, got shape {arr.shape}")
    return arr


def _workspace(nbytes, device, ws):
    """(tensor, its size in bytes): the caller's workspace, checked, or a new one."""
    if ws is not None:
        if not isinstance(ws, torch.Tensor) or not ws.is_contiguous():
            raise ValueError("ws must be a contiguous tensor")
        if not _device_ok(ws, device):
            raise ValueError(f"ws must be on {device}, got {ws.device}")
        size = ws.numel() * ws.element_size()
        if size < nbytes:
            raise ValueError(f"workspace too small: {size} < {nbytes} bytes")
        return ws, size
    ws = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    return ws, ws.numel()


def mi_debug_wait_failure():
    """First device wait that gave up since the last read (all zeros if none); clears it."""
    rec = (ctypes.c_int32 * 8)()
    _check("mi_debug_wait_failure", _lib_handle().mi_debug_wait_failure(rec))
    keys = ["seq", "site", "block", "thread", "group", "parity", "r6", "r7"]
    return dict(zip(keys, list(rec)))


def mi_debug_set_wait_budget(cycles: int) -> None:
    """Clock budget of the kernels' abortable waits for later launches
    (<= 0: the default).  Failure-path tests only."""
    _check("mi_debug_set_wait_budget", _lib_handle().mi_debug_set_wait_budget(int(cycles)))


BS_ENGINE_ROW = 0
BS_ENGINE_KEY = 1


def mi_set_bs_engine(engine: int) -> None:
    """Engine for Block-Sparse heads in later launches: BS_ENGINE_ROW (the
    default) or BS_ENGINE_KEY (key-major tiles, d = 128)."""
    _check("mi_set_bs_engine", _lib_handle().mi_set_bs_engine(int(engine)))


def mi_status_str(status: int) -> str:
    return _lib_handle().mi_status_str(status).decode()


def mi_version() -> str:
    return _lib_handle().mi_version().decode()


def mi_workspace_bytes(op, Hq, Hkv, N, d, n_heads=0, last_q=0, vertical_size=0, slash_size=0,
                       topk_blocks=0) -> int:
    return int(_lib_handle().mi_workspace_bytes(op, Hq, Hkv, N, d, n_heads, last_q,
                                                vertical_size, slash_size, topk_blocks))


MI_SLASH_BLOCKS = 0
MI_SLASH_RANGES = 1


def make_params(last_q=64, vertical_size=1000, slash_size=6096, topk_blocks=100, sink=64,
                window=1024, slash_tiles=MI_SLASH_BLOCKS) -> mi_params:
    return mi_params(last_q, vertical_size, slash_size, topk_blocks, sink, window, slash_tiles)


def mi_prefill_workspace_bytes(Hq, Hkv, N, d, pattern, params: mi_params) -> int:
    pat = None if pattern is None else _host_array("pattern", pattern, np.int8, Hq)
    pp = None if pat is None else pat.ctypes.data_as(ctypes.c_void_p)
    return int(_lib_handle().mi_prefill_workspace_bytes(Hq, Hkv, N, d, pp, ctypes.byref(params)))


def _params_array(params, Hq):
    if len(params) != Hq:
        raise ValueError(f"one mi_params per query head: {Hq} expected, got {len(params)}")
    return (mi_params * Hq)(*params)


def mi_prefill_workspace_bytes_heads(Hq, Hkv, N, d, pattern, params) -> int:
    """Workspace of mi_prefill_layer_heads: `params` holds one mi_params per head."""
    pat = _host_array("pattern", pattern, np.int8, Hq)
    arr = _params_array(params, Hq)
    return int(_lib_handle().mi_prefill_workspace_bytes_heads(
        Hq, Hkv, N, d, pat.ctypes.data_as(ctypes.c_void_p), ctypes.cast(arr, ctypes.c_void_p)))


def _index_outputs(n, N, vertical_size, slash_size, want_scores, dev):
    if vertical_size < 0 or slash_size < 0:
        raise ValueError("budgets must be non-negative")
    v_idx = torch.empty(n, vertical_size, dtype=torch.int32, device=dev)
    s_idx = torch.empty(n, slash_size, dtype=torch.int32, device=dev)
    vs = torch.empty(n, N, dtype=torch.float32, device=dev) if want_scores else None
    ss = torch.empty(n, N, dtype=torch.float32, device=dev) if want_scores else None
    return v_idx, s_idx, vs, ss


def mi_vs_index(q, k, last_q, vertical_size, slash_size, heads: Optional[Sequence[int]] = None,
                scale=0.0, ws=None, want_scores=False, stream=None):
    """Vertical-Slash index: (v_idx, s_idx[, v_score, s_score]) per listed head."""
    Hq, Hkv, N, d = _shape(q, k)
    harr, n, hp = _heads(heads, Hq)
    dev = q.device
    v_idx, s_idx, vs, ss = _index_outputs(n, N, vertical_size, slash_size, want_scores, dev)
    nb = mi_workspace_bytes(MI_OP_VS_INDEX, Hq, Hkv, N, d, n, last_q, vertical_size, slash_size)
    ws, ws_bytes = _workspace(nb, dev, ws)
    rc = _lib_handle().mi_vs_index(_ptr(q), _ptr(k), Hq, Hkv, N, d, scale, last_q, vertical_size,
                                   slash_size, hp, n, _ptr(v_idx), _ptr(s_idx), _ptr(vs), _ptr(ss),
                                   _ptr(ws), ws_bytes, _stream(stream))
    _check("mi_vs_index", rc)
    return (v_idx, s_idx, vs, ss) if want_scores else (v_idx, s_idx)


def mi_vs_index_static(q, k, last_q, vertical_size, slash_size, heads=None, scale=0.0,
                       want_scores=False, stream=None):
    """mi_vs_index for callers that cannot provide a workspace: the library keeps
    the scratch in a fixed 16 MiB device array (calls must not overlap)."""
    Hq, Hkv, N, d = _shape(q, k)
    harr, n, hp = _heads(heads, Hq)
    v_idx, s_idx, vs, ss = _index_outputs(n, N, vertical_size, slash_size, want_scores, q.device)
    rc = _lib_handle().mi_vs_index_static(_ptr(q), _ptr(k), Hq, Hkv, N, d, scale, last_q,
                                          vertical_size, slash_size, hp, n, _ptr(v_idx),
                                          _ptr(s_idx), _ptr(vs), _ptr(ss), _stream(stream))
    _check("mi_vs_index_static", rc)
    return (v_idx, s_idx, vs, ss) if want_scores else (v_idx, s_idx)


def mi_bs_index(q, k, topk, heads=None, scale=0.0, ws=None, stream=None):
    """Block-Sparse index: (blk_idx [n, N/64, topk], blk_cnt [n, N/64])."""
    Hq, Hkv, N, d = _shape(q, k)
    harr, n, hp = _heads(heads, Hq)
    if topk < 0:
        raise ValueError("topk must be non-negative")
    dev = q.device
    nB = N // MI_BLOCK
    blk_idx = torch.empty(n, nB, topk, dtype=torch.int32, device=dev)
    blk_cnt = torch.empty(n, nB, dtype=torch.int32, device=dev)
    ws, ws_bytes = _workspace(mi_workspace_bytes(MI_OP_BS_INDEX, Hq, Hkv, N, d, n), dev, ws)
    rc = _lib_handle().mi_bs_index(_ptr(q), _ptr(k), Hq, Hkv, N, d, scale, MI_BLOCK, topk, hp, n,
                                   _ptr(blk_idx), _ptr(blk_cnt), _ptr(ws), ws_bytes,
                                   _stream(stream))
    _check("mi_bs_index", rc)
    return blk_idx, blk_cnt


def _attn_out(q, out, lse, want_lse, err_count):
    """Check or allocate out (bf16 [Hq, N, d]) and lse (fp32 [Hq, N]); check err_count."""
    Hq, N, _ = q.shape
    _dev("out", out, torch.bfloat16, q.shape, q.device)
    _dev("lse", lse, torch.float32, (Hq, N), q.device)
    _dev("err_count", err_count, torch.int32, None, q.device)
    if err_count is not None and err_count.numel() < 1:
        raise ValueError("err_count must hold one int32")
    if out is None:
        out = torch.zeros_like(q)
    if lse is None and want_lse:
        lse = torch.full((Hq, N), float("nan"), dtype=torch.float32, device=q.device)
    return out, lse


def _index_rows(name, t, n, q):
    """An int32 index tensor with one row per listed head; returns its row length."""
    if t is None:
        return 0
    if not isinstance(t, torch.Tensor) or t.dim() != 2 or t.shape[0] != n:
        raise ValueError(f"{name} must be a 2-D int32 tensor with {n} rows")
    _dev(name, t, torch.int32, None, q.device)
    return int(t.shape[1])


def mi_vs_sparse_attn(q, k, v, v_idx, s_idx, heads=None, scale=0.0, out=None, lse=None,
                      want_lse=True, err_count=None, ws=None, stream=None, ranges=False):
    """Vertical-Slash attention; ranges=True reads each diagonal as one
    unaligned 64-key range per query block (mi_vs_range_attn)."""
    Hq, Hkv, N, d = _shape(q, k, v)
    harr, n, hp = _heads(heads, Hq)
    kv = _index_rows("v_idx", v_idx, n, q)
    ks = _index_rows("s_idx", s_idx, n, q)
    out, lse = _attn_out(q, out, lse, want_lse, err_count)
    ws, ws_bytes = _workspace(mi_workspace_bytes(MI_OP_VS_ATTN, Hq, Hkv, N, d, n, 0, kv, ks),
                              q.device, ws)
    name = "mi_vs_range_attn" if ranges else "mi_vs_sparse_attn"
    rc = getattr(_lib_handle(), name)(_ptr(q), _ptr(k), _ptr(v), Hq, Hkv, N, d, scale,
                                      _ptr(v_idx), kv, _ptr(s_idx), ks, hp, n, _ptr(out),
                                      _ptr(lse), _ptr(err_count), _ptr(ws), ws_bytes,
                                      _stream(stream))
    _check(name, rc)
    return out, lse


def mi_block_sparse_attn(q, k, v, blk_idx, blk_cnt, heads=None, scale=0.0, out=None, lse=None,
                         want_lse=True, err_count=None, stream=None):
    Hq, Hkv, N, d = _shape(q, k, v)
    harr, n, hp = _heads(heads, Hq)
    nB = N // MI_BLOCK
    if not isinstance(blk_idx, torch.Tensor) or blk_idx.dim() != 3:
        raise ValueError("blk_idx must be a 3-D int32 tensor [n_heads, N/64, topk]")
    topk = int(blk_idx.shape[-1])
    _dev("blk_idx", blk_idx, torch.int32, (n, nB, topk), q.device)
    _dev("blk_cnt", blk_cnt, torch.int32, (n, nB), q.device)
    out, lse = _attn_out(q, out, lse, want_lse, err_count)
    rc = _lib_handle().mi_block_sparse_attn(_ptr(q), _ptr(k), _ptr(v), Hq, Hkv, N, d, scale,
                                            _ptr(blk_idx), _ptr(blk_cnt), topk, MI_BLOCK, hp, n,
                                            _ptr(out), _ptr(lse), _ptr(err_count), None, 0,
                                            _stream(stream))
    _check("mi_block_sparse_attn", rc)
    return out, lse


def mi_ashape_attn(q, k, v, sink, window, heads=None, scale=0.0, out=None, lse=None,
                   want_lse=True, err_count=None, stream=None):
    Hq, Hkv, N, d = _shape(q, k, v)
    harr, n, hp = _heads(heads, Hq)
    out, lse = _attn_out(q, out, lse, want_lse, err_count)
    rc = _lib_handle().mi_ashape_attn(_ptr(q), _ptr(k), _ptr(v), Hq, Hkv, N, d, scale, sink,
                                      window, hp, n, _ptr(out), _ptr(lse), _ptr(err_count), None,
                                      0, _stream(stream))
    _check("mi_ashape_attn", rc)
    return out, lse


def mi_dense_attn(q, k, v, heads=None, scale=0.0, out=None, lse=None, want_lse=True,
                  err_count=None, stream=None):
    """Dense causal attention (every key j <= i) on the same engine."""
    Hq, Hkv, N, d = _shape(q, k, v)
    harr, n, hp = _heads(heads, Hq)
    out, lse = _attn_out(q, out, lse, want_lse, err_count)
    rc = _lib_handle().mi_dense_attn(_ptr(q), _ptr(k), _ptr(v), Hq, Hkv, N, d, scale, hp, n,
                                     _ptr(out), _ptr(lse), _ptr(err_count), None, 0,
                                     _stream(stream))
    _check("mi_dense_attn", rc)
    return out, lse


def mi_prefill_layer_heads(q, k, v, pattern, params, scale=0.0, out=None, lse=None,
                           want_lse=False, err_count=None, ws=None, stream=None):
    """One layer with one mi_params per head (host int8 pattern [Hq], params [Hq])."""
    Hq, Hkv, N, d = _shape(q, k, v)
    pat = _host_array("pattern", pattern, np.int8, Hq)
    arr = _params_array(params, Hq)
    out, lse = _attn_out(q, out, lse, want_lse, err_count)
    need = mi_prefill_workspace_bytes_heads(Hq, Hkv, N, d, pat, params)
    ws, ws_bytes = _workspace(need, q.device, ws)
    rc = _lib_handle().mi_prefill_layer_heads(
        _ptr(q), _ptr(k), _ptr(v), Hq, Hkv, N, d, scale, pat.ctypes.data_as(ctypes.c_void_p),
        ctypes.cast(arr, ctypes.c_void_p), _ptr(out), _ptr(lse), _ptr(err_count), _ptr(ws),
        ws_bytes, _stream(stream), None)
    _check("mi_prefill_layer_heads", rc)
    return out, lse


def mi_prefill_layer(q, k, v, pattern, params: mi_params, scale=0.0, out=None, lse=None,
                     want_lse=False, err_count=None, ws=None, stage_events=None, stream=None):
    """One layer: per-head pattern table (host int8 [Hq]) -> index + sparse attention."""
    Hq, Hkv, N, d = _shape(q, k, v)
    pat = _host_array("pattern", pattern, np.int8, Hq)
    out, lse = _attn_out(q, out, lse, want_lse, err_count)
    ws, ws_bytes = _workspace(mi_prefill_workspace_bytes(Hq, Hkv, N, d, pat, params), q.device,
                              ws)
    ev = None
    if stage_events is not None:
        if len(stage_events) != MI_STAGE_EVENTS:
            raise ValueError(f"stage_events must hold {MI_STAGE_EVENTS} events")
        for e in stage_events:
            if not e.cuda_event:  # torch creates the CUDA event on first record
                e.record()
        ev = (ctypes.c_void_p * MI_STAGE_EVENTS)(*[e.cuda_event for e in stage_events])
    rc = _lib_handle().mi_prefill_layer(_ptr(q), _ptr(k), _ptr(v), Hq, Hkv, N, d, scale,
                                        pat.ctypes.data_as(ctypes.c_void_p), ctypes.byref(params),
                                        _ptr(out), _ptr(lse), _ptr(err_count), _ptr(ws),
                                        ws_bytes, _stream(stream), ev)
    _check("mi_prefill_layer", rc)
    return out, lse
