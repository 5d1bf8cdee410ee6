"""Host-side checks of the Python binding (no GPU).

The library reads raw pointers with the layouts its header states, so the
binding must refuse host tensors, wrong element types, strided views and
mis-shaped index, output and host arrays before any pointer reaches a kernel,
and must hand the library the sizes the tensors really have.  A fake library
records the calls; the device test is relaxed to CPU for the marshalling cases.
"""
import numpy as np
import pytest
import torch

from dynamic_sparse_attention_02_b200 import binding as B


def bf16(*shape):
    return torch.zeros(*shape, dtype=torch.bfloat16)


class FakeLib:
    """Records every library call; workspace queries answer 4096 bytes."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def call(*args):
            self.calls.append((name, args))
            return 4096 if "workspace_bytes" in name else B.MI_OK
        return call


@pytest.fixture
def fake(monkeypatch):
    lib = FakeLib()
    monkeypatch.setattr(B, "_lib_handle", lambda: lib)
    monkeypatch.setattr(B, "_device_ok", lambda t, dev: dev is None or t.device == dev)
    return lib


def test_host_tensors_are_refused_before_the_library():
    q, k, v = bf16(2, 128, 64), bf16(1, 128, 64), bf16(1, 128, 64)
    with pytest.raises(ValueError, match="CUDA device"):
        B.mi_dense_attn(q, k, v, stream=0)
    with pytest.raises(ValueError, match="CUDA device"):
        B.mi_vs_index(q, k, 64, 10, 10, stream=0)


def test_wrong_dtype_and_strided_views_are_refused():
    with pytest.raises(TypeError, match="bfloat16"):
        B.mi_dense_attn(torch.zeros(2, 128, 64), bf16(1, 128, 64), bf16(1, 128, 64), stream=0)
    q = bf16(128, 2, 64).transpose(0, 1)
    with pytest.raises(ValueError, match="contiguous"):
        B.mi_dense_attn(q, bf16(1, 128, 64), bf16(1, 128, 64), stream=0)
    with pytest.raises(ValueError, match="3-D"):
        B.mi_dense_attn(bf16(128, 64), bf16(1, 128, 64), bf16(1, 128, 64), stream=0)


def test_kv_shapes_must_match_q(fake):
    q = bf16(4, 256, 64)
    with pytest.raises(ValueError, match="k must have shape"):
        B.mi_dense_attn(q, bf16(2, 192, 64), bf16(2, 192, 64), stream=0)
    with pytest.raises(ValueError, match="v must have shape"):
        B.mi_dense_attn(q, bf16(2, 256, 64), bf16(2, 256, 128), stream=0)
    with pytest.raises(TypeError, match="v must be"):
        B.mi_dense_attn(q, bf16(2, 256, 64), torch.zeros(2, 256, 64), stream=0)
    assert fake.calls == []


def test_outputs_are_checked(fake):
    q, k, v = bf16(4, 256, 64), bf16(2, 256, 64), bf16(2, 256, 64)
    with pytest.raises(ValueError, match="out must have shape"):
        B.mi_ashape_attn(q, k, v, 64, 128, out=bf16(4, 256, 128), stream=0)
    with pytest.raises(TypeError, match="lse must be"):
        B.mi_ashape_attn(q, k, v, 64, 128, lse=torch.zeros(4, 256, dtype=torch.float64),
                         stream=0)
    with pytest.raises(TypeError, match="err_count must be"):
        B.mi_ashape_attn(q, k, v, 64, 128, err_count=torch.zeros(1, dtype=torch.int64),
                         stream=0)
    assert fake.calls == []


def test_index_tensors_need_one_row_per_listed_head(fake):
    q, k, v = bf16(4, 256, 64), bf16(2, 256, 64), bf16(2, 256, 64)
    vi = torch.zeros(4, 10, dtype=torch.int32)
    si = torch.zeros(4, 20, dtype=torch.int32)
    with pytest.raises(ValueError, match="v_idx must be"):
        B.mi_vs_sparse_attn(q, k, v, vi, si, heads=[1, 3], stream=0)
    with pytest.raises(TypeError, match="s_idx must be"):
        B.mi_vs_sparse_attn(q, k, v, vi, si.long(), stream=0)
    bi = torch.zeros(4, 4, 3, dtype=torch.int32)
    with pytest.raises(ValueError, match="blk_cnt must have shape"):
        B.mi_block_sparse_attn(q, k, v, bi, torch.zeros(4, 3, dtype=torch.int32), stream=0)
    with pytest.raises(ValueError, match="blk_idx must have shape"):
        B.mi_block_sparse_attn(q, k, v, torch.zeros(4, 5, 3, dtype=torch.int32),
                               torch.zeros(4, 4, dtype=torch.int32), stream=0)
    assert fake.calls == []


def test_host_tables_need_one_entry_per_head(fake):
    q, k, v = bf16(4, 256, 64), bf16(2, 256, 64), bf16(2, 256, 64)
    p = B.make_params()
    with pytest.raises(ValueError, match="pattern must hold 4"):
        B.mi_prefill_layer(q, k, v, np.ones(3, np.int8), p, stream=0)
    with pytest.raises(ValueError, match="one mi_params per query head"):
        B.mi_prefill_layer_heads(q, k, v, np.ones(4, np.int8), [p] * 3, stream=0)
    assert fake.calls == []


def test_workspace_size_is_passed_in_bytes(fake):
    q, k, v = bf16(4, 256, 64), bf16(2, 256, 64), bf16(2, 256, 64)
    vi = torch.zeros(2, 10, dtype=torch.int32)
    si = torch.zeros(2, 20, dtype=torch.int32)
    with pytest.raises(ValueError, match="workspace too small"):
        B.mi_vs_sparse_attn(q, k, v, vi, si, heads=[1, 3], ws=torch.empty(100, dtype=torch.uint8),
                            stream=0)
    ws = torch.empty(1024, dtype=torch.float32)  # 4096 bytes in 1024 elements
    B.mi_vs_sparse_attn(q, k, v, vi, si, heads=[1, 3], ws=ws, stream=0)
    name, args = fake.calls[-1]
    assert name == "mi_vs_sparse_attn"
    # (q, k, v, Hq, Hkv, N, d, scale, v_idx, kv, s_idx, ks, heads, n, out, lse, err, ws, bytes, s)
    assert args[3:7] == (4, 2, 256, 64)
    assert args[9] == 10 and args[11] == 20 and args[13] == 2
    assert args[18] == 4096


def test_valid_layer_call_marshals_the_tables(fake):
    q, k, v = bf16(4, 256, 64), bf16(2, 256, 64), bf16(2, 256, 64)
    out, lse = B.mi_prefill_layer(q, k, v, [0, 1, 2, 3], B.make_params(), want_lse=True,
                                  stream=0)
    assert out.shape == q.shape and out.dtype == torch.bfloat16
    assert lse.shape == (4, 256) and lse.dtype == torch.float32
    names = [c[0] for c in fake.calls]
    assert names == ["mi_prefill_workspace_bytes", "mi_prefill_layer"]
    args = fake.calls[-1][1]
    assert args[3:7] == (4, 2, 256, 64)
    assert args[14] == 4096


def test_missing_library_raises_instead_of_falling_back(monkeypatch):
    """Without the built library every entry point raises: there is no CPU path."""
    monkeypatch.setattr(B, "_lib", None)
    monkeypatch.setattr(B, "LIB_PATH", B.LIB_PATH + ".absent")
    monkeypatch.setattr(B, "_device_ok", lambda t, dev: dev is None or t.device == dev)
    q, k, v = bf16(2, 128, 64), bf16(1, 128, 64), bf16(1, 128, 64)
    with pytest.raises(RuntimeError, match="is not built"):
        B.mi_dense_attn(q, k, v, stream=0)
    with pytest.raises(RuntimeError, match="is not built"):
        B.mi_prefill_layer(q, k, v, [1, 2], B.make_params(), stream=0)
