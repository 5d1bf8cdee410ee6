"""Seeded synthetic inputs shaped like a LLaMA-3-8B attention layer.

This module is input synthesis only: it draws q, k, v and the per-head
pattern table, and holds none of the method's arithmetic (no scores, no
softmax, no index selection).  Both the CUDA path and the CPU oracle are fed
from it by the tests and by the benchmark; neither imports the other.

Recipe (the pages measure on LLaMA-3-8B long-context prompts, MInference 1.0
abstract and "Results"; no prompt text or weights are used here, the shapes
and the planted column/block structure stand in for them):

* one ``torch.Generator`` on the target device, seeded ``20260000 + workload.index``;
  draw order q, k, v, planted key positions, planted key blocks, pattern table;
* q, k ~ N(0, 1) in fp32, shape [heads, N, d]; rotary position embedding
  (rotate-half pairs (t, t + d/2), inverse frequency theta^(-2t/d),
  theta = 500000, positions 0..N-1) applied to q and k;
* u_g = unit vector along the mean post-RoPE query of KV group g (all
  positions, all query heads of the group);
* keys 0..3 plus a seeded 1% of positions (without replacement) get
  k += 3 u_g ("vertical" landmark columns);
* block-clustered workloads also pick a seeded 2% of the 64-key blocks and
  add 2 u_g to all 64 keys of each;
* v ~ N(0, 1);
* everything is rounded to bf16 (round to nearest even) at the end.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

PATTERN_ASHAPE = 0
PATTERN_VS = 1
PATTERN_BS = 2
PATTERN_DENSE = 3

ROPE_THETA = 500000.0
SEED_BASE = 20260000


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic prefill layer: shapes, per-pattern budgets, generator knobs."""

    index: int          # seeds the generator (SEED_BASE + index)
    name: str
    Hq: int
    Hkv: int
    N: int
    d: int
    pattern: str        # "vs", "bs", "ashape" or "mixed"
    last_q: int = 64
    vertical_size: int = 1000
    slash_size: int = 6096
    block: int = 64
    topk_blocks: int = 100
    sink: int = 64
    window: int = 1024
    planted_frac: float = 0.01
    block_bias_frac: float = 0.0

    @property
    def nB(self) -> int:
        return self.N // self.block

    @property
    def seed(self) -> int:
        return SEED_BASE + self.index


# The five layers the benchmark and the parity tests use.
WORKLOADS = {
    w.name: w
    for w in [
        Workload(1, "vs_n2k_h1_d64", Hq=1, Hkv=1, N=2048, d=64, pattern="vs",
                 vertical_size=128, slash_size=256),
        Workload(2, "vs_n128k_llama3_8b", Hq=32, Hkv=8, N=131072, d=128, pattern="vs"),
        Workload(3, "bs_n128k_llama3_8b", Hq=32, Hkv=8, N=131072, d=128, pattern="bs",
                 block_bias_frac=0.02),
        Workload(4, "mixed_n256k_llama3_8b", Hq=32, Hkv=8, N=262144, d=128, pattern="mixed"),
        Workload(5, "vs_n1m_llama3_8b", Hq=32, Hkv=8, N=1048576, d=128, pattern="vs"),
    ]
}


def workload(name: str, **overrides) -> Workload:
    """Look up a named workload, optionally with fields replaced (small test variants)."""
    w = WORKLOADS[name]
    return dataclasses.replace(w, **overrides) if overrides else w


def _rope_inplace(x: torch.Tensor, chunk_rows: int = 1 << 16) -> None:
    """Rotate-half rotary embedding over positions 0..N-1 of x [H, N, d], in place."""
    H, N, d = x.shape
    half = d // 2
    t = torch.arange(half, dtype=torch.float64, device=x.device)
    inv_freq = ROPE_THETA ** (-2.0 * t / d)
    for r0 in range(0, N, chunk_rows):
        r1 = min(N, r0 + chunk_rows)
        pos = torch.arange(r0, r1, dtype=torch.float64, device=x.device)
        ang = pos[:, None] * inv_freq[None, :]
        c = torch.cos(ang).to(torch.float32)
        s = torch.sin(ang).to(torch.float32)
        x1 = x[:, r0:r1, :half].clone()
        x2 = x[:, r0:r1, half:]
        x[:, r0:r1, :half] = x1 * c - x2 * s
        x[:, r0:r1, half:] = x2 * c + x1 * s


def pattern_table(w: Workload, gen: Optional[torch.Generator] = None,
                  device: str = "cpu") -> np.ndarray:
    """Per-query-head pattern codes (int8 [Hq]): 0 A-shape, 1 Vertical-Slash, 2 Block-Sparse."""
    if w.pattern == "vs":
        return np.full(w.Hq, PATTERN_VS, np.int8)
    if w.pattern == "bs":
        return np.full(w.Hq, PATTERN_BS, np.int8)
    if w.pattern == "ashape":
        return np.full(w.Hq, PATTERN_ASHAPE, np.int8)
    # mixed: a seeded permutation of roughly one third of each pattern
    n_a = (w.Hq + 2) // 3
    n_vs = (w.Hq + 1) // 3
    n_bs = w.Hq - n_a - n_vs
    base = np.array([PATTERN_ASHAPE] * n_a + [PATTERN_VS] * n_vs + [PATTERN_BS] * n_bs, np.int8)
    perm = torch.randperm(w.Hq, generator=gen, device=device).cpu().numpy()
    return base[perm]


def make_inputs(w: Workload, device: str = "cpu", seed: Optional[int] = None):
    """Draw the seeded bf16 q [Hq,N,d], k [Hkv,N,d], v [Hkv,N,d] and the pattern table.

    Returns a dict with ``q``, ``k``, ``v`` (bf16 tensors on ``device``),
    ``pattern`` (np.int8 [Hq]), ``planted`` (sorted int64 key positions) and
    ``planted_blocks`` (sorted int64 block ids).
    """
    assert w.Hq % w.Hkv == 0 and w.N % w.block == 0
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed if seed is None else seed)
    q = torch.randn(w.Hq, w.N, w.d, generator=gen, device=device, dtype=torch.float32)
    k = torch.randn(w.Hkv, w.N, w.d, generator=gen, device=device, dtype=torch.float32)
    v = torch.randn(w.Hkv, w.N, w.d, generator=gen, device=device, dtype=torch.float32)
    n_pl = int(round(w.planted_frac * w.N))
    planted = torch.randperm(w.N, generator=gen, device=device)[:n_pl]
    planted = torch.unique(torch.cat([torch.arange(4, device=device), planted]))
    n_blk = int(round(w.block_bias_frac * w.nB))
    if n_blk > 0:
        pblocks = torch.sort(torch.randperm(w.nB, generator=gen, device=device)[:n_blk]).values
    else:
        pblocks = torch.zeros(0, dtype=torch.int64, device=device)
    pattern = pattern_table(w, gen, device)

    _rope_inplace(q)
    _rope_inplace(k)
    group = w.Hq // w.Hkv
    for g in range(w.Hkv):
        u = q[g * group:(g + 1) * group].double().mean(dim=(0, 1))
        u = (u / u.norm()).to(torch.float32)
        k[g, planted] += 3.0 * u
        if n_blk > 0:
            rows = (pblocks[:, None] * w.block + torch.arange(w.block, device=device)[None, :]).reshape(-1)
            k[g, rows] += 2.0 * u
    return {
        "q": q.to(torch.bfloat16),
        "k": k.to(torch.bfloat16),
        "v": v.to(torch.bfloat16),
        "pattern": pattern,
        "planted": planted.cpu(),
        "planted_blocks": pblocks.cpu(),
    }


def sample_heads_rows(w: Workload, n_heads: int, n_rows: int, seed: Optional[int] = None):
    """Seeded subset for full-size checks: query heads in distinct KV groups, sorted rows.

    Uses its own numpy generator so that the draw does not disturb the tensors.
    """
    rng = np.random.default_rng((w.seed if seed is None else seed) + 7919)
    group = w.Hq // w.Hkv
    groups = rng.permutation(w.Hkv)[:min(n_heads, w.Hkv)]
    heads = sorted(int(g * group + rng.integers(group)) for g in groups)
    rows = np.sort(rng.choice(w.N, size=min(n_rows, w.N), replace=False)).astype(np.int64)
    return heads, rows


def kv_bytes(w: Workload) -> int:
    return 2 * w.Hkv * w.N * w.d * 2


def q_bytes(w: Workload) -> int:
    return w.Hq * w.N * w.d * 2

