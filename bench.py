#!/usr/bin/env python
"""Benchmark: one MInference dynamic-sparse prefill layer per step on B200.

A step is one pass of the whole hot path over one layer of synthetic input:
mi_prefill_layer = per-head index estimation + slash/vertical prep + one
sparse-attention launch.  Default workload: the LLaMA-3-8B-shaped 128K layer
(32 query heads, 8 KV heads, d = 128, N = 131072, every head Vertical-Slash
with last_q = 64, vertical 1000, slash 6096).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl minfer|reference]

Multi-GPU runs (torchrun, one process per GPU) are independent replicas: the
layer does not shard, so there is no data-path collective; the step time is
the max over ranks and the reported ms/layer is that time divided by the
number of layers all ranks processed.

--impl reference times the CPU oracle (the only reference implementation of
this method here) on a bounded sample of the same workload, extrapolated to
the same metric.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from dynamic_sparse_attention_02_b200 import synth  # noqa: E402

METRIC = "sparse prefill attn ms/layer (index+attn) at 128K/1M; tensor-pipe util %"
UNIT = "ms/layer"
_T0 = time.time()


def log(msg):
    """Progress on stderr (the JSON result goes to stdout)."""
    print(f"[bench {time.time() - _T0:7.1f}s] {msg}", file=sys.stderr, flush=True)


FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
ATTN_SOURCES = ["attn.cu", "softmax_math.cuh", "exp2_poly.h", "ptx.cuh", "internal.h"]


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="minfer", choices=["minfer", "reference"])
    ap.add_argument("--workload", default="vs_n128k_llama3_8b", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--seq-len", type=int, default=0,
                    help="override N of the workload (smaller profiling cases)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-dense", action="store_true",
                    help="skip the dense-prefill comparison (every head dense causal)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-1m", action="store_true",
                    help="skip the 1M-token layer measured after the main workload (at_1m)")
    ap.add_argument("--no-1m-ranges", action="store_true",
                    help="skip the 1M layer with range slash tiles (at_1m.slash_ranges)")
    ap.add_argument("--slash-tiles", default="blocks", choices=["blocks", "ranges"],
                    help="how VS heads of the main workload read their diagonals")
    ap.add_argument("--bs-engine", default="row", choices=["row", "key"],
                    help="engine for Block-Sparse heads (row-major tiles, or key-major)")
    ap.add_argument("--cpu-budget-s", type=float, default=15.0,
                    help="approximate CPU seconds for the oracle baseline sample")
    return ap.parse_args(argv)


# ----------------------------------------------------------------- helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


def params_of(w, B, ranges=False):
    return B.make_params(last_q=w.last_q, vertical_size=w.vertical_size, slash_size=w.slash_size,
                         topk_blocks=w.topk_blocks, sink=w.sink, window=w.window,
                         slash_tiles=B.MI_SLASH_RANGES if ranges else B.MI_SLASH_BLOCKS)


def _code_only(src):
    """C/C++ source with comments and whitespace removed (string literals kept),
    so that a comment edit does not orphan measurements taken on the code."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif c == '"' or c == "'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        else:
            if not c.isspace():
                out.append(c)
            i += 1
    return "".join(out)


def attn_source_sha():
    """Hash of the attention kernel's code (comments and whitespace ignored): the
    key under which ncu records of that kernel are kept."""
    h = hashlib.sha256()
    for name in ATTN_SOURCES:
        with open(os.path.join(ROOT, "dynamic_sparse_attention_02_b200", "csrc", name)) as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload):
    """DRAM bytes per attention launch from a committed ncu summary, if it was
    taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "attn_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    entry = rec.get(workload)
    if not entry or entry.get("source_sha") != attn_source_sha():
        return None
    return entry.get("dram_bytes_per_launch")


def recorded_tensor_pipe(workload):
    """Tensor-pipe utilisation of the attention kernel from a committed ncu
    summary taken on the current kernel source (else None).  The capture is a
    small case of the same pattern (the record says which)."""
    path = os.path.join(ROOT, "profiles", "attn_tensor_pipe.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    entry = rec.get(workload)
    if not entry or entry.get("source_sha") != attn_source_sha():
        return None
    return {k: entry[k] for k in ("pct", "metric", "case") if k in entry}


class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait(timeout=10)
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        return parse_clock_samples(lines)


def parse_clock_samples(lines):
    """Summary of `nvidia-smi --query-gpu=<ClockSampler.QUERY> --format=csv,noheader,nounits`
    lines: median SM clock, highest max clock, and every slowdown reason seen Active."""
    rows = []
    for line in lines:
        parts = [p.strip() for p in line.split(",")]
        if len(parts) >= 9:
            rows.append(parts)
    if not rows:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
    sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
    smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
    return {"sm_mhz": float(np.median(sm)) if sm else None,
            "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
            "samples": len(rows)}


def vs_useful_flops(v_idx, s_idx, N, d):
    """Useful FLOPs of one VS head: 4*d per (row, key) pair over computed 64x64
    tiles (slash diagonals -> block diagonals D) plus 64 rows per gathered
    column per query block (columns outside D tiles).  Returns (flops, tiles,
    gathered column-blocks)."""
    nB = N // 64
    s = s_idx[(s_idx >= 0) & (s_idx < N)]
    D = np.zeros(nB + 1, bool)
    a = s // 64
    D[a] = True
    D[np.minimum(a + 1, nB)[(s % 64) != 0]] = True
    D = D[:nB]
    deltas = np.nonzero(D)[0]
    tiles = int(np.sum(nB - deltas))
    V = np.unique(v_idx[(v_idx >= 0) & (v_idx < N)])
    cnt_le = np.cumsum(D)  # |{delta in D : delta <= x}|
    bj = V // 64
    cols = int(np.sum((nB - bj) - cnt_le[nB - 1 - bj]))
    return 4.0 * d * (64 * 64 * tiles + 64 * cols), tiles, cols


def vs_range_useful_flops(v_idx, s_idx, N, d):
    """Useful FLOPs of one VS head whose diagonals are read as ranges: query
    block bq takes key u iff some selected o has 64 bq - u <= o <= 64 bq - u + 63,
    i.e. R[64 bq - u] with R[x] = "a selected offset in [x, x + 63]" (x >= -63).
    Per query block, the kept keys form runs of R; each run of length n costs
    ceil(n / 64) 64-key tiles of 64 rows.  Gathered columns: those outside the
    block's runs, 64 rows each.  Returns (flops, 64x64-equivalent tiles,
    gathered column-blocks)."""
    nB = N // 64
    s = np.unique(s_idx[(s_idx >= 0) & (s_idx < N)])
    S = np.zeros(N + 64, np.int64)
    S[s] = 1
    cs = np.concatenate([[0], np.cumsum(S)])
    x = np.arange(-63, N)                              # R over x in [-63, N)
    lo, hi = np.clip(x, 0, N), np.clip(x + 63, -1, N - 1)
    R = (cs[hi + 1] - cs[lo]) > 0
    # runs of R, then per query block bq the windows of the runs clipped to x <= 64 bq
    m = np.concatenate([[0], R.astype(np.int8), [0]])
    dm = np.diff(m)
    rs = np.nonzero(dm == 1)[0] - 63                   # run starts (x coordinates)
    re = np.nonzero(dm == -1)[0] - 1 - 63              # run ends, inclusive
    full = (re - rs + 64) // 64
    cf = np.concatenate([[0], np.cumsum(full)])
    lim = 64 * np.arange(nB)
    j = np.searchsorted(re, lim, side="right")         # runs ending at or before lim
    win = cf[j]
    jj = np.minimum(j, max(len(rs) - 1, 0))
    part = (j < len(rs)) & (rs[jj] <= lim) if len(rs) else np.zeros(nB, bool)
    win = win + np.where(part, (lim - rs[jj] + 64) // 64, 0) if len(rs) else win
    tiles = int(win.sum())
    # column c is kept by blocks bq >= c // 64; covered there iff R[64 bq - c], i.e. entry
    # 64 (bq - c // 64) + 63 - c % 64 of R (which starts at x = -63): a stride-64 count
    V = np.unique(v_idx[(v_idx >= 0) & (v_idx < N)])
    Rp = np.zeros(64 * (nB + 1), np.int64)
    Rp[:R.size] = R
    C = np.cumsum(Rp.reshape(nB + 1, 64), axis=0)
    cb, cl = V // 64, V % 64
    covered = C[nB - 1 - cb, 63 - cl]
    cols = int(np.sum((nB - cb) - covered))
    return 4.0 * d * (64 * 64 * tiles + 64 * cols), tiles, cols


def ashape_tiles(N, sink, window):
    """64x64 causal tiles an A-shape head computes: key block b of query block qb
    holds a sink key (64 b < sink) or a key inside the local window of some row
    (64 (qb - b) - 63 < window)."""
    nB = N // 64
    qb = np.arange(nB)
    a = np.minimum(qb + 1, -(-sink // 64))        # sink blocks: b < ceil(sink / 64)
    dmax = -(-(window + 63) // 64) - 1            # window blocks: qb - b <= dmax
    lo = np.maximum(0, qb - dmax)
    both = np.maximum(0, np.minimum(a, qb + 1) - lo)
    return int(np.sum(a + (qb - lo + 1) - both))


# ----------------------------------------------------------------- oracle timing

def oracle_sample(w, x, budget_s, rng, h=0, min_rows=32, max_rows=16384):
    """Time the CPU oracle on a bounded sample of head h: its index, then seeded
    random rows of its attention in chunks until `budget_s` of CPU time is used.
    Returns (extrapolated ms/layer, description, threads used)."""
    import oracle
    pattern = x["pattern"]
    g = h * w.Hkv // w.Hq
    qs = x["q"][h:h + 1].float().cpu()
    ks = x["k"][g:g + 1].float().cpu()
    vs = x["v"][g:g + 1].float().cpu()
    pt = int(pattern[h])
    t0 = time.perf_counter()
    if pt == synth.PATTERN_VS:
        vi, si, _, _ = oracle.vs_index(qs, ks, 0, w.last_q, w.vertical_size, w.slash_size)
    elif pt == synth.PATTERN_BS:
        bi, bc = oracle.bs_index(qs, ks, 0, w.topk_blocks)
    t_index = time.perf_counter() - t0
    order = rng.permutation(w.N)
    t_rows, done, chunk = 0.0, 0, min_rows
    while done < min(max_rows, w.N) and (done < min_rows or t_index + t_rows < budget_s):
        rows = np.sort(order[done:done + chunk])
        t1 = time.perf_counter()
        if pt == synth.PATTERN_VS:
            oracle.attn_vs(qs, ks, vs, 0, vi, si, rows=rows)
        elif pt == synth.PATTERN_BS:
            oracle.attn_bs(qs, ks, vs, 0, bi, bc, rows=rows)
        else:
            oracle.attn_ashape(qs, ks, vs, 0, w.sink, w.window, rows=rows)
        t_rows += time.perf_counter() - t1
        done += rows.size
        chunk = min(2 * chunk, 2048)
    ms = 1e3 * (t_index * w.Hq + t_rows / done * w.N * w.Hq)
    desc = (f"index of head {h} ({t_index:.1f} s) + {done} seeded random rows of its attention "
            f"at N={w.N} ({t_rows:.1f} s), extrapolated to {w.Hq} heads x {w.N} rows")
    return ms, desc, oracle.num_threads()


# ----------------------------------------------------------------- arms

def workload_of(args):
    w = synth.workload(args.workload)
    return synth.workload(args.workload, N=args.seq_len) if args.seq_len else w


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = workload_of(args)
    x = synth.make_inputs(w, device="cuda" if torch.cuda.is_available() else "cpu")
    rng = np.random.default_rng(w.seed)
    total = args.steps + args.warmup
    budget = max(2.0, 150.0 / max(total, 1))  # the whole run stays within a few minutes
    for _ in range(args.warmup):
        oracle_sample(w, x, budget, rng)
    vals = []
    desc, cores = "", 1
    for _ in range(args.steps):
        ms, desc, cores = oracle_sample(w, x, budget, rng)
        vals.append(ms)
    v = float(np.median(vals))
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": v,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(w),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_of(w):
    return {"workload": w.name, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d,
            "pattern": w.pattern, "last_q": w.last_q, "vertical_size": w.vertical_size,
            "slash_size": w.slash_size, "topk_blocks": w.topk_blocks, "sink": w.sink,
            "window": w.window, "parallelism": "replicas",
            "l2": (f"inputs larger than L2 (q+k+v {(w.Hq + 2 * w.Hkv) * w.N * w.d * 2 / 2**20:.0f} MiB"
                   " > 126 MB); no flush")}


class Ranks:
    """One process per GPU, launched by torchrun: rank and world size from its
    environment, and a process group for the barriers around the timed region
    and the max-over-ranks step time (NCCL on GPUs; the tests drive the
    same code over gloo on CPU).  The layer is run as independent replicas:
    no collective touches the data path."""

    def __init__(self, backend="nccl", device=None, timeout_s=300):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.device = device
        self.dist = None
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
            self.dist = dist

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def max_over_ranks(self, val):
        if self.dist is None:
            return val
        t = torch.tensor([val], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.dist is not None:
            self.dist.barrier()
            self.dist.destroy_process_group()
            self.dist = None


def job_value(ms_step_max, world):
    """Whole-job ms per layer: `world` replicas each finish one layer per step,
    timed by the slowest rank."""
    return ms_step_max / world


def time_layer(B, w, x, params, ws, out, steps, warmup, ranks, dev):
    """Warm up, then time `steps` mi_prefill_layer calls with CUDA events (stage
    events inside each step) and nvidia-smi clock samples over the timed
    region.  Returns (ms per step on this rank, ms index, ms prep, ms attention,
    clock summary)."""
    q, k, v, pattern = x["q"], x["k"], x["v"], x["pattern"]

    def step(ev):
        B.mi_prefill_layer(q, k, v, pattern, params, out=out, ws=ws, stage_events=ev)

    warm_ev = [torch.cuda.Event(enable_timing=True) for _ in range(B.MI_STAGE_EVENTS)]
    for i in range(warmup):
        step(warm_ev)
        torch.cuda.synchronize()
        log(f"{w.name} warmup step {i}: index {warm_ev[0].elapsed_time(warm_ev[1]):.2f} ms, "
            f"attn {warm_ev[2].elapsed_time(warm_ev[3]):.2f} ms")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(B.MI_STAGE_EVENTS)]
           for _ in range(steps)]
    for e in evs:
        for ee in e:
            ee.record()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index)
    clocks.start()
    ranks.barrier()
    torch.cuda.synchronize()
    t_start.record()
    for i in range(steps):
        step(evs[i])
    t_end.record()
    torch.cuda.synchronize()
    ranks.barrier()
    clk = clocks.stop()
    ms_step = t_start.elapsed_time(t_end) / steps
    ms_index = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    ms_prep = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    ms_attn = float(np.mean([e[2].elapsed_time(e[3]) for e in evs]))
    log(f"{w.name}: timed {steps} steps: {ms_step:.2f} ms/step (attn {ms_attn:.2f} ms)")
    return ms_step, ms_index, ms_prep, ms_attn, clk


def useful_work(B, w, x, ranges=False):
    """Algorithmic work of the layer's attention launch, from its own index:
    (computed-tile FLOPs, 64x64 tiles, gathered column-blocks); ranges: the
    VS heads read their diagonals as 64-key ranges."""
    useful, tiles, cols = 0.0, 0, 0
    q, k, pat = x["q"], x["k"], np.asarray(x["pattern"])
    vs_heads = [h for h in range(w.Hq) if pat[h] == synth.PATTERN_VS]
    bs_heads = [h for h in range(w.Hq) if pat[h] == synth.PATTERN_BS]
    n_ash = int(np.sum(pat == synth.PATTERN_ASHAPE))
    if vs_heads:
        v_idx, s_idx = B.mi_vs_index(q, k, w.last_q, w.vertical_size, w.slash_size,
                                     heads=vs_heads)
        vi, si = v_idx.cpu().numpy(), s_idx.cpu().numpy()
        for i in range(len(vs_heads)):
            f, t, c = (vs_range_useful_flops if ranges else vs_useful_flops)(vi[i], si[i], w.N,
                                                                              w.d)
            useful += f
            tiles += t
            cols += c
    if bs_heads:
        _, blk_cnt = B.mi_bs_index(q, k, w.topk_blocks, heads=bs_heads)
        t = int(blk_cnt.sum().item())
        useful += 4.0 * w.d * 64 * 64 * t
        tiles += t
    if n_ash:
        t = ashape_tiles(w.N, w.sink, w.window) * n_ash
        useful += 4.0 * w.d * 64 * 64 * t
        tiles += t
    return useful, tiles, cols


def tile_density(w, tiles):
    return tiles / (w.Hq * (w.N // 64) * (w.N // 64 + 1) / 2) if tiles else None


def measure_1m(B, ranks, dev, peak, with_ranges=True):
    """The metric's 1M half, measured in the same run: the 1M-token
    Vertical-Slash layer (32 query heads, 8 KV heads, d = 128, last_q 64,
    vertical 1000, slash 6096), 1 warm-up + 2 timed steps, with its own clock
    record.  attn_kcycles = attention ms x median SM MHz (thousands of cycles at
    the sampled clock), so that runs at different power-capped clocks compare."""
    w = synth.workload("vs_n1m_llama3_8b")
    log(f"generating {w.name} (N={w.N})")
    x = synth.make_inputs(w, device=str(dev))
    torch.cuda.synchronize()
    out = torch.empty_like(x["q"])
    steps, warmup = 2, 1

    def leg(ranges):
        params = params_of(w, B, ranges)
        ws = torch.empty(B.mi_prefill_workspace_bytes(w.Hq, w.Hkv, w.N, w.d, x["pattern"],
                                                      params), dtype=torch.uint8, device=dev)
        ms_step, ms_index, ms_prep, ms_attn, clk = time_layer(B, w, x, params, ws, out, steps,
                                                              warmup, ranks, dev)
        del ws
        useful, tiles, cols = useful_work(B, w, x, ranges)
        eff = useful / (ms_attn * 1e-3) / 1e12
        mhz = clk.get("sm_mhz")
        return {"ms_per_layer": ms_step, "ms_index": ms_index, "ms_prep": ms_prep,
                "ms_attn": ms_attn, "eff_tflops": eff, "frac_of_peak": eff / peak,
                "flops_per_launch": useful, "tile_density": tile_density(w, tiles),
                "gathered_column_blocks": cols,
                "attn_kcycles": ms_attn * mhz if mhz else None, "clocks": clk}

    rec = {"workload": w.name, "N": w.N, "steps": steps, "warmup": warmup}
    rec.update(leg(False))
    rec["tensor_pipe"] = recorded_tensor_pipe(w.name)
    # VS index (2 score passes, row merge, top-k), prep, attention
    rec["gpu_launches"] = 6 * steps
    if with_ranges:
        # the same layer with every diagonal read as 64-key ranges (MI_SLASH_RANGES):
        # a different, sparser mask, so its time is not the metric's
        log("1M layer with range slash tiles")
        rec["slash_ranges"] = leg(True)
    del x, out
    torch.cuda.empty_cache()
    return rec


def run_minfer(args):
    from dynamic_sparse_attention_02_b200 import binding as B
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    dev = torch.device("cuda", torch.cuda.current_device())
    ranks = Ranks("nccl", dev)
    world, rank = ranks.world, ranks.rank
    barrier, max_over_ranks = ranks.barrier, ranks.max_over_ranks

    w = workload_of(args)
    B.mi_set_bs_engine(B.BS_ENGINE_KEY if args.bs_engine == "key" else B.BS_ENGINE_ROW)
    log(f"generating {w.name} (N={w.N})")
    x = synth.make_inputs(w, device=str(dev))
    torch.cuda.synchronize()
    q, k, v = x["q"], x["k"], x["v"]
    pattern = x["pattern"]
    ranges = args.slash_tiles == "ranges"
    params = params_of(w, B, ranges)
    ws = torch.empty(B.mi_prefill_workspace_bytes(w.Hq, w.Hkv, w.N, w.d, pattern, params),
                     dtype=torch.uint8, device=dev)
    out = torch.empty_like(q)
    n_vs = int(np.sum(pattern == synth.PATTERN_VS))
    n_bs = int(np.sum(pattern == synth.PATTERN_BS))
    # VS: two score passes, the row merge, one top-k launch for both lists, the
    # slash/vertical prep, and for last_q > 64 the merge of row-group partials;
    # BS: mean-pool of Q, of K, block score + top-k; then one attention launch
    n_vs_launches = 5 + (1 if w.last_q > 64 else 0)
    launches_per_step = (n_vs_launches if n_vs else 0) + (3 if n_bs else 0) + 1

    ms_step, ms_index, ms_prep, ms_attn, clk = time_layer(B, w, x, params, ws, out, args.steps,
                                                          args.warmup, ranks, dev)
    ms_step_max = max_over_ranks(ms_step)

    # end to end through the public API: host inputs in, host output back
    e2e = None
    if not args.no_e2e:
        hq = q.cpu().pin_memory()
        hk = k.cpu().pin_memory()
        hv = v.cpu().pin_memory()
        hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        n_e2e = max(1, min(args.steps, 5))

        # Each KV group (its query heads and their shared K/V) is an independent
        # layer call through the public API, so the copies of one group overlap
        # the compute of its neighbours: host->device of group g+1 and
        # device->host of group g-1 run on their own streams while group g
        # computes.  Every byte still crosses PCIe inside the timed region.
        comp = torch.cuda.current_stream()
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        gq = w.Hq // w.Hkv
        ev_in = [torch.cuda.Event() for _ in range(w.Hkv)]
        ev_done = [torch.cuda.Event() for _ in range(w.Hkv)]
        ev_out = torch.cuda.Event()

        def step_e2e():
            s_in.wait_stream(comp)  # the previous step has finished with dq/dk/dv
            for g in range(w.Hkv):
                hs = slice(g * gq, (g + 1) * gq)
                with torch.cuda.stream(s_in):
                    dq[hs].copy_(hq[hs], non_blocking=True)
                    dk[g].copy_(hk[g], non_blocking=True)
                    dv[g].copy_(hv[g], non_blocking=True)
                    ev_in[g].record(s_in)
            for g in range(w.Hkv):
                hs = slice(g * gq, (g + 1) * gq)
                comp.wait_event(ev_in[g])
                B.mi_prefill_layer(dq[hs], dk[g:g + 1], dv[g:g + 1], pattern[hs], params,
                                   out=out[hs], ws=ws, stream=comp)
                ev_done[g].record(comp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_done[g])
                    hout[hs].copy_(out[hs], non_blocking=True)
            ev_out.record(s_out)
            comp.wait_event(ev_out)  # the step ends when its result is on the host

        step_e2e()
        torch.cuda.synchronize()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(n_e2e):
            step_e2e()
        b.record()
        torch.cuda.synchronize()
        barrier()
        ms_e2e = max_over_ranks(a.elapsed_time(b) / n_e2e)
        log(f"e2e {ms_e2e:.2f} ms/step")
        e2e = {"value": job_value(ms_e2e, world), "unit": UNIT,
               "h2d_bytes_per_step": int(hq.numel() * 2 + hk.numel() * 2 + hv.numel() * 2),
               "d2h_bytes_per_step": int(hout.numel() * 2), "steps": n_e2e}
        assert torch.equal(hout, out.cpu()), "e2e output differs from the device output"

    # The pages' headline comparison: the same layer with every head dense
    # causal (the prefill MInference is measured against), on the same engine.
    dense = None
    if not args.no_dense:
        dout = torch.empty_like(out)
        n_dense = 1 if w.N > 262144 else max(1, min(args.steps, 3))
        B.mi_dense_attn(q, k, v, out=dout, want_lse=False)
        torch.cuda.synchronize()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(n_dense):
            B.mi_dense_attn(q, k, v, out=dout, want_lse=False)
        b.record()
        torch.cuda.synchronize()
        barrier()
        ms_dense = max_over_ranks(a.elapsed_time(b) / n_dense)
        log(f"dense causal attention {ms_dense:.2f} ms")
        dense = {"ms": ms_dense, "steps": n_dense,
                 "speedup_vs_dense": ms_dense / ms_step_max,
                 "tflops": 4.0 * w.d * w.N * (w.N + 1) / 2 * w.Hq / (ms_dense * 1e-3) / 1e12}
        del dout

    useful, tiles, cols = useful_work(B, w, x, ranges)
    dense_eq = 4.0 * w.d * w.N * (w.N + 1) / 2 * w.Hq
    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    achieved = useful / (ms_attn * 1e-3) / 1e12 if useful else None
    traffic = recorded_traffic(w.name)

    # The metric's 1M half on a single GPU (the default 128K run only).
    at_1m = None
    if (world == 1 and not args.no_1m and not args.seq_len
            and w.name == "vs_n128k_llama3_8b"):
        # the oracle baseline samples head 0 only: keep its tensors on the host
        x = {"q": q[0:1].cpu(), "k": k[0:1].cpu(), "v": v[0:1].cpu(), "pattern": pattern}
        del q, k, v, ws, out
        torch.cuda.empty_cache()
        at_1m = measure_1m(B, ranks, dev, peak, with_ranges=not args.no_1m_ranges)

    line = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            rng = np.random.default_rng(w.seed)
            log(f"oracle baseline: ~{args.cpu_budget_s:.0f} s of CPU work")
            ms_cpu, desc, cores = oracle_sample(w, x, args.cpu_budget_s, rng)
            log("oracle baseline done: " + desc)
            cpu = {"value": ms_cpu, "unit": UNIT, "cores": cores, "kind": "oracle",
                   "sample": desc}
        line = {
            "metric": METRIC, "value": job_value(ms_step_max, world), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step_max,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": dict(config_of(w), **({"bs_engine": "key"} if args.bs_engine == "key" else {}),
                           **({"slash_tiles": "ranges"} if ranges else {})),
            "ms_index": ms_index, "ms_prep": ms_prep, "ms_attn": ms_attn,
            "tile_density": tile_density(w, tiles),
            "gathered_column_blocks": cols,
            "eff_tflops": achieved,
            "dense_eq_tflops": dense_eq / (ms_step_max * 1e-3) / 1e12,
            "roofline": {"bound": "tensor", "kernel": "sparse_attn_kernel<128>",
                         "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": (achieved / peak) if achieved else None,
                         "peak_source": f"bf16_tflops_sustained ({peak_src})",
                         "traffic": traffic,
                         "flops_per_launch": useful},
            "tensor_pipe": recorded_tensor_pipe(w.name),
            "at_1m": at_1m,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "dense_prefill": dense,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    ranks.close()
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_minfer(args)


if __name__ == "__main__":
    sys.exit(main())
