"""Host-side logic of bench.py: useful-FLOP accounting of a Vertical-Slash
head, against a brute-force count of the 64x64 tiles and gathered columns."""
import numpy as np

import bench
import oracle


def brute(v_idx, s_idx, N, d):
    nB = N // 64
    D = oracle.slash_deltas(np.asarray(s_idx, np.int32), N).astype(bool)
    tiles = sum(1 for bq in range(nB) for bk in range(bq + 1) if D[bq - bk])
    cols = 0
    for j in sorted(set(int(x) for x in v_idx if 0 <= x < N)):
        for bq in range(j // 64, nB):
            if not D[bq - j // 64]:
                cols += 1
    return 4.0 * d * (64 * 64 * tiles + 64 * cols), tiles, cols


def test_vs_useful_flops_matches_brute_force():
    rng = np.random.default_rng(0)
    for N in (512, 1024, 2048):
        for _ in range(5):
            v = rng.integers(-1, N, size=rng.integers(0, 40)).astype(np.int32)
            s = rng.integers(-1, N, size=rng.integers(0, 30)).astype(np.int32)
            assert bench.vs_useful_flops(v, s, N, 128) == brute(v, s, N, 128)


def brute_range(v_idx, s_idx, N, d):
    """Range reading, from the oracle's element mask: per query block, the kept
    slash keys (seen by the block's last row) as runs, each run of n keys
    costing ceil(n / 64) tiles; gathered columns are the kept columns outside
    the block's slash keys."""
    nB = N // 64
    s = np.asarray([x for x in s_idx if 0 <= x < N], np.int32)
    v = np.asarray(sorted(set(int(x) for x in v_idx if 0 <= x < N)), np.int32)
    ms = oracle.vs_mask(N, np.zeros(0, np.int32), s, range_tiles=True)
    tiles = cols = 0
    for bq in range(nB):
        row = ms[64 * bq + 63].astype(np.int8)
        m = np.diff(np.concatenate([[0], row, [0]]))
        st, en = np.nonzero(m == 1)[0], np.nonzero(m == -1)[0]
        tiles += int(np.sum((en - st + 63) // 64))
        cols += int(np.sum(~ms[64 * bq + 63, v[v <= 64 * bq + 63]]))
    return 4.0 * d * (64 * 64 * tiles + 64 * cols), tiles, cols


def test_vs_range_useful_flops_matches_the_oracle_mask():
    rng = np.random.default_rng(1)
    for N in (512, 1024, 1600):
        for _ in range(4):
            v = rng.integers(-1, N, size=rng.integers(0, 40)).astype(np.int32)
            s = rng.integers(-1, N, size=rng.integers(1, 30)).astype(np.int32)
            assert bench.vs_range_useful_flops(v, s, N, 128) == brute_range(v, s, N, 128)


def test_ashape_tile_count_matches_brute_force():
    """The closed-form count of 64x64 tiles an A-shape head computes (bench FLOP
    accounting) equals a direct count over every causal (query block, key block)."""
    rng = np.random.default_rng(7)
    for _ in range(200):
        N = 64 * int(rng.integers(1, 70))
        sink = int(rng.integers(0, 300))
        window = int(rng.integers(0, 1500))
        nB = N // 64
        qb = np.arange(nB)[:, None]
        b = np.arange(nB)[None, :]
        want = int(np.sum((b <= qb) & ((64 * b < sink) | (64 * (qb - b) - 63 < window))))
        assert bench.ashape_tiles(N, sink, window) == want


def test_clock_samples_summary():
    """Median SM clock, highest max clock, and every slowdown reason seen Active;
    unreadable fields and short lines are skipped."""
    idle = "Not Active"
    lines = [
        f"0, 1700, 1965, 900.1, 0x4, {idle}, {idle}, {idle}, Active\n",
        f"0, 1650, 1965, 990.0, 0x4, {idle}, {idle}, {idle}, Active\n",
        f"0, 1800, 1965, 700.0, 0x0, {idle}, {idle}, {idle}, {idle}\n",
        f"0, [N/A], 1965, 700.0, 0x0, {idle}, Active, {idle}, {idle}\n",
        "garbage line\n",
    ]
    got = bench.parse_clock_samples(lines)
    assert got["sm_mhz"] == 1700.0 and got["sm_max_mhz"] == 1965.0
    assert got["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert got["samples"] == 4
    assert bench.parse_clock_samples([])["reasons"] == ["no samples"]


def test_job_value_is_whole_job_time_per_layer():
    """N replicas each finish one layer per step, timed by the slowest rank."""
    assert bench.job_value(130.0, 1) == 130.0
    assert bench.job_value(132.0, 4) == 33.0


def test_reference_arm_json_line(capsys, monkeypatch):
    """`--impl reference` prints one JSON line with the contract's keys: the
    oracle timed on a bounded sample, host-only (no copies), time-like metric."""
    import json
    for key in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(key, raising=False)
    args = bench.parse_args(["--impl", "reference", "--steps", "2", "--warmup", "3",
                             "--workload", "vs_n2k_h1_d64"])
    assert bench.run_reference(args) == 0
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["n_gpus"] == 1
    assert (d["steps"], d["warmup"]) == (2, 3)
    assert d["higher_is_better"] is False and d["vs_baseline"] is None
    assert d["value"] > 0 and d["ms_per_step"] == d["value"]
    assert d["config"]["workload"] == "vs_n2k_h1_d64" and d["config"]["N"] == 2048
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert "2048 seeded random rows" in cb["sample"]  # the whole small layer was sampled
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_code_only_hash_ignores_comments_not_code():
    a = 'int f() { // one\n  return 1; /* two */ }\nconst char* s = "// kept";\n'
    b = 'int f() {   // other words\n return 1; }\n/* c */ const char* s = "// kept";'
    c = 'int f() { return 2; }\nconst char* s = "// kept";'
    d = 'int f() { return 1; }\nconst char* s = "// other";'
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)
    assert bench._code_only(a) != bench._code_only(d)
