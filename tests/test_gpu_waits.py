"""The give-up path of the kernels' bounded waits, exercised on purpose.

Every abortable wait inside the attention kernel and the tensor-core
Vertical-Slash score passes has a clock budget (about half a second).  A
diagnostic setter lowers that budget for later launches to one cycle, so the
first wait that does not find its phase already complete gives up.  The launch
must then end cleanly: the host call returns, the attention launch sets bit 30
of err_count, the first give-up is recorded with its site, and the device and
the library stay usable -- the next normal call matches the oracle.  Waits that
guard the release of tensor memory and the landing of copies in flight keep
the full budget, which is what makes the clean ending possible.  Nothing here
faults, traps or hangs: the budget only makes waits return early.
"""
import numpy as np
import pytest
import torch

import oracle
from dynamic_sparse_attention_02_b200 import binding as B
from parity_util import check_attn, check_index_set, head_slices, rand_bf16

pytestmark = pytest.mark.gpu

ATTN_SITES = range(1, 8)    # producer / MMA / softmax waits of the attention kernel
SCORE_SITES = range(11, 16)  # producer / MMA / epilogue waits of the VS score passes
KT_SITES = range(21, 28)     # producer / MMA / softmax waits of the key-major engine


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from dynamic_sparse_attention_02_b200 import build
    build.build()
    yield
    B.mi_debug_set_wait_budget(0)


def _vs_inputs(N):
    every = torch.arange(0, N, 3, dtype=torch.int32, device="cuda")[None].repeat(2, 1)
    diag = torch.tensor([[0, 1, 100, 257]] * 2, dtype=torch.int32, device="cuda")
    return every, diag


def test_attention_wait_gives_up_then_device_is_usable():
    N, d = 512, 128
    q, k, v = rand_bf16(2, 1, N, d, 51)
    vi, si = _vs_inputs(N)
    B.mi_debug_wait_failure()  # clear any earlier record
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.mi_debug_set_wait_budget(1)
    try:
        out, lse = B.mi_vs_sparse_attn(q, k, v, vi, si, err_count=err)
        torch.cuda.synchronize()
    finally:
        B.mi_debug_set_wait_budget(0)
    assert int(err.item()) & (1 << 30), "no wait gave up with a one-cycle budget"
    rec = B.mi_debug_wait_failure()
    assert rec["site"] in ATTN_SITES, rec
    # a launch that gave up writes finite rows (zeros where it stopped), nothing else
    assert torch.isfinite(out.float()).all()

    # the same call with the default budget: nothing gives up and the rows match
    err.zero_()
    out, lse = B.mi_vs_sparse_attn(q, k, v, vi, si, err_count=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for h in range(2):
        qs, ks_, vs_ = head_slices(q, k, v, h)
        ro, rl = oracle.attn_vs(qs, ks_, vs_, 0, vi[h].cpu().numpy(), si[h].cpu().numpy())
        check_attn(out[h], lse[h], ro, rl, what=f"after the give-up, head {h}")
    assert B.mi_debug_wait_failure()["site"] == 0


def test_key_major_engine_wait_gives_up_then_device_is_usable():
    """The same for the key-major Block-Sparse engine (sites 21-27)."""
    Hq, Hkv, N, d, topk = 2, 1, 1024, 128, 6
    q, k, v = rand_bf16(Hq, Hkv, N, d, 53)
    bi = np.full((Hq, N // 64, topk), -1, np.int32)
    bc = np.zeros((Hq, N // 64), np.int32)
    for h in range(Hq):
        qs, ks_, _ = head_slices(q, k, None, h)
        bi[h], bc[h] = oracle.bs_index(qs, ks_, 0, topk)
    bit, bct = torch.from_numpy(bi).cuda(), torch.from_numpy(bc).cuda()
    B.mi_debug_wait_failure()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.mi_set_bs_engine(B.BS_ENGINE_KEY)
    try:
        B.mi_debug_set_wait_budget(1)
        try:
            out, lse = B.mi_block_sparse_attn(q, k, v, bit, bct, err_count=err)
            torch.cuda.synchronize()
        finally:
            B.mi_debug_set_wait_budget(0)
        assert int(err.item()) & (1 << 30), "no wait gave up with a one-cycle budget"
        rec = B.mi_debug_wait_failure()
        assert rec["site"] in KT_SITES, rec
        assert torch.isfinite(out.float()).all()
        err.zero_()
        out, lse = B.mi_block_sparse_attn(q, k, v, bit, bct, err_count=err)
        torch.cuda.synchronize()
    finally:
        B.mi_set_bs_engine(B.BS_ENGINE_ROW)
    assert int(err.item()) == 0
    for h in range(Hq):
        qs, ks_, vs_ = head_slices(q, k, v, h)
        ro, rl = oracle.attn_bs(qs, ks_, vs_, 0, bi[h], bc[h])
        check_attn(out[h], lse[h], ro, rl, what=f"key-major after the give-up, head {h}")
    assert B.mi_debug_wait_failure()["site"] == 0


def test_score_pass_waits_end_cleanly_with_a_tiny_budget():
    """The score passes wait with mbarrier.try_wait, which may itself block
    until its phase completes, so a one-cycle budget need not make them give
    up; what must hold is that the launch ends, any give-up is recorded at a
    score-pass site, and the next normal call matches the oracle."""
    Hq, Hkv, N, d, L, kv, ks = 4, 1, 4160, 128, 64, 300, 900
    q, k, _ = rand_bf16(Hq, Hkv, N, d, 52)
    B.mi_debug_wait_failure()
    B.mi_debug_set_wait_budget(1)
    try:
        B.mi_vs_index(q, k, L, kv, ks)
        torch.cuda.synchronize()
    finally:
        B.mi_debug_set_wait_budget(0)
    rec = B.mi_debug_wait_failure()
    print(f"score passes with a one-cycle budget: wait record {rec}")
    assert rec["site"] == 0 or rec["site"] in SCORE_SITES, rec

    v_idx, s_idx = B.mi_vs_index(q, k, L, kv, ks)
    torch.cuda.synchronize()
    for h in range(Hq):
        qs, ks_, _ = head_slices(q, k, None, h)
        vert, sl = oracle.vs_scores(qs, ks_, 0, L)
        check_index_set(v_idx[h].cpu().numpy(), vert, kv, what=f"vertical h{h}")
        check_index_set(s_idx[h].cpu().numpy(), sl, ks, what=f"slash h{h}")
    assert B.mi_debug_wait_failure()["site"] == 0
    assert np.isfinite(vert).all()
