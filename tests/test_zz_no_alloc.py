"""mi_vs_index_static: the Vertical-Slash index for callers that cannot give
the library device scratch (e.g. a server whose allocator owns all HBM, or a
latency-critical path that cannot afford cudaMalloc's synchronisation).

Through the C ABI it must return what the workspace entry point mi_vs_index
returns on the same inputs, on two calls in a row (the second call finds the
first call's leftovers in the shared static scratch).  This file is collected
last; it also passes alone in a fresh process.
"""
import ctypes

import pytest
import torch

from dynamic_sparse_attention_02_b200 import binding as B
from dynamic_sparse_attention_02_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from dynamic_sparse_attention_02_b200 import build
    build.build()


def call_static(q, k, L, kv, ks, heads=None):
    """Raw C-ABI call of mi_vs_index_static (no workspace argument)."""
    Hq, N, d = q.shape
    Hkv = k.shape[0]
    n = Hq if heads is None else len(heads)
    harr = None if heads is None else (ctypes.c_int32 * n)(*heads)
    v_idx = torch.full((n, kv), -7, dtype=torch.int32, device="cuda")
    s_idx = torch.full((n, ks), -7, dtype=torch.int32, device="cuda")
    vs = torch.full((n, N), float("nan"), dtype=torch.float32, device="cuda")
    ss = torch.full((n, N), float("nan"), dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = B.lib().mi_vs_index_static(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), Hq, Hkv, N, d, 0.0, L, kv,
        ks, None if harr is None else ctypes.cast(harr, ctypes.c_void_p), 0 if heads is None else n,
        ctypes.c_void_p(v_idx.data_ptr()), ctypes.c_void_p(s_idx.data_ptr()),
        ctypes.c_void_p(vs.data_ptr()), ctypes.c_void_p(ss.data_ptr()), stream)
    assert rc == B.MI_OK, B.mi_status_str(rc)
    return v_idx, s_idx, vs, ss


def test_static_scratch_matches_workspace_entry_point_twice():
    # Calls in a row with different shapes.  The third one (last_q = 128, a
    # head subset) uses the per-row-group partial score buffers, where an
    # earlier call's leftovers would matter most.  Same kernels, same inputs:
    # every output must be bit-identical to the workspace entry point's.
    cases = [("vs_n2k_h1_d64", dict(Hq=4, Hkv=1, N=4096, d=128), 64, None),
             ("vs_n2k_h1_d64", dict(Hq=2, Hkv=2, N=2048, d=64), 64, None),
             ("vs_n2k_h1_d64", dict(Hq=4, Hkv=2, N=4096, d=128), 128, [1, 3])]
    for name, shape, L, heads in cases:
        w = synth.workload(name, **shape)
        x = synth.make_inputs(w, device="cuda")
        got = call_static(x["q"], x["k"], L, 100, 200, heads)
        want = B.mi_vs_index(x["q"], x["k"], L, 100, 200, heads=heads, want_scores=True)
        torch.cuda.synchronize()
        for g, e in zip(got, want):
            assert torch.equal(g, e)
