"""mi_vs_index_static: the Vertical-Slash index for callers that cannot give
the library device scratch (e.g. a server whose allocator owns all HBM, or a
latency-critical path that cannot afford cudaMalloc's synchronisation).

Through the C ABI it must return what the workspace entry point mi_vs_index
returns on the same inputs, on two calls in a row (the second call finds the
first call's leftovers in the shared static scratch).  This file is collected
last; it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
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


def call_static(q, k, L, kv, ks):
    """Raw C-ABI call of mi_vs_index_static (no workspace argument)."""
    Hq, N, d = q.shape
    Hkv = k.shape[0]
    v_idx = torch.full((Hq, kv), -7, dtype=torch.int32, device="cuda")
    s_idx = torch.full((Hq, ks), -7, dtype=torch.int32, device="cuda")
    vs = torch.full((Hq, N), float("nan"), dtype=torch.float32, device="cuda")
    ss = torch.full((Hq, N), float("nan"), dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = B.lib().mi_vs_index_static(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), Hq, Hkv, N, d, 0.0, L, kv,
        ks, None, 0, ctypes.c_void_p(v_idx.data_ptr()), ctypes.c_void_p(s_idx.data_ptr()),
        ctypes.c_void_p(vs.data_ptr()), ctypes.c_void_p(ss.data_ptr()), stream)
    assert rc == B.MI_OK, B.mi_status_str(rc)
    return v_idx, s_idx, vs, ss


def test_static_scratch_matches_workspace_entry_point_twice():
    cases = [("vs_n2k_h1_d64", dict(Hq=4, Hkv=1, N=4096, d=128)),
             ("vs_n2k_h1_d64", dict(Hq=2, Hkv=2, N=2048, d=64))]
    for name, shape in cases:  # two calls in a row, different shapes
        w = synth.workload(name, **shape)
        x = synth.make_inputs(w, device="cuda")
        got = call_static(x["q"], x["k"], 64, 100, 200)
        want = B.mi_vs_index(x["q"], x["k"], 64, 100, 200, want_scores=True)
        torch.cuda.synchronize()
        assert torch.equal(got[0], want[0]) and torch.equal(got[1], want[1])
        np.testing.assert_allclose(got[2].cpu().numpy(), want[2].cpu().numpy(), rtol=1e-6)
        np.testing.assert_allclose(got[3].cpu().numpy(), want[3].cpu().numpy(), rtol=1e-6)
