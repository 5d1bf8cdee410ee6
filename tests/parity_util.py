"""Shared checks for the GPU parity tests (CUDA path vs the CPU oracle)."""
import numpy as np
import torch

import oracle

# required accuracy of the bf16 attention output against the oracle
ATTN_MAX_ABS = 1e-2
ATTN_MEAN_ABS = 1e-3
# index sets may differ only at entries within this relative distance of the k-th score
INDEX_REL = 1e-6


def head_slices(q, k, v, h):
    """The oracle's inputs for query head h: that head and its KV head (contiguous groups)."""
    Hq, Hkv = q.shape[0], k.shape[0]
    g = h * Hkv // Hq
    qs = q[h:h + 1].float().cpu()
    ks = k[g:g + 1].float().cpu()
    vs = v[g:g + 1].float().cpu() if v is not None else None
    return qs, ks, vs


def check_index_set(gpu_idx, scores, k, window_scale=None, what=""):
    """GPU indices (ascending, -1 padded) against oracle fp64 scores.

    The sets must be equal except for entries whose score lies within
    INDEX_REL * window_scale of the k-th largest score (window_scale defaults
    to |k-th score|).  Returns the number of tolerated differences.
    """
    gpu = np.asarray(gpu_idx).astype(np.int64)
    n = scores.size
    kk = min(k, n)
    assert np.all(gpu[kk:] == -1), f"{what}: padding"
    sel = gpu[:kk]
    assert np.all(sel >= 0) and np.all(sel < n), f"{what}: range"
    assert np.all(np.diff(sel) > 0), f"{what}: not strictly ascending"
    if kk == 0:
        return 0
    ref = oracle.topk(scores, kk)
    sk = np.sort(scores)[::-1][kk - 1]
    scale = abs(sk) if window_scale is None else window_scale
    diff = np.setxor1d(sel, ref)
    bad = [j for j in diff if abs(scores[j] - sk) > INDEX_REL * scale]
    assert not bad, (f"{what}: {len(bad)} entries differ beyond the tie window, e.g. "
                     f"{bad[:5]} scores {[scores[j] for j in bad[:5]]} k-th {sk}")
    return len(diff)


def check_attn(out_gpu, lse_gpu, out_ref, lse_ref, what=""):
    """bf16 GPU rows against fp64 oracle rows: max-abs <= 1e-2 and mean-abs <= 1e-3."""
    o = out_gpu.float().cpu().numpy().astype(np.float64)
    err = np.abs(o - out_ref)
    assert np.all(np.isfinite(o)), f"{what}: non-finite output"
    assert err.max() <= ATTN_MAX_ABS, f"{what}: max abs {err.max():.3e}"
    assert err.mean() <= ATTN_MEAN_ABS, f"{what}: mean abs {err.mean():.3e}"
    if lse_gpu is not None:
        lg = lse_gpu.float().cpu().numpy().astype(np.float64)
        empty = np.isneginf(lse_ref)
        assert np.all(np.isneginf(lg[empty])), f"{what}: empty rows must have lse = -inf"
        if (~empty).any():
            le = np.abs(lg[~empty] - lse_ref[~empty])
            assert le.max() <= 1e-3, f"{what}: lse max abs {le.max():.3e}"
    return float(err.max()), float(err.mean())


def rand_bf16(Hq, Hkv, N, d, seed, device="cuda"):
    g = torch.Generator(device="cpu").manual_seed(seed)
    q = torch.randn(Hq, N, d, generator=g).to(torch.bfloat16)
    k = torch.randn(Hkv, N, d, generator=g).to(torch.bfloat16)
    v = torch.randn(Hkv, N, d, generator=g).to(torch.bfloat16)
    return q.to(device), k.to(device), v.to(device)
