"""Strength of the oracle's pins: plant one plausible mistake at a time in a copy
of the C oracle and require the pin suite (test_oracle_pins.py) to fail on it.

Each mutant is a wrong index, a dropped term, an off-by-one bound, a transposed
operand or a flipped rule of the kind a careless restatement of the pages would
make.  All of them keep every memory access in bounds.  The unmutated source,
built the same way, must pass, which shows the failures come from the mistakes.
Builds go to _build/oracle_mutants/ inside the repository.
"""
import concurrent.futures as cf
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "minfer_oracle.c")
OUT = os.path.join(ROOT, "_build", "oracle_mutants")

# (name, text in minfer_oracle.c, replacement)
MUTANTS = [
    ("vs_rows_first_not_last",
     "const int64_t i = (int64_t)N - L + r;\n        const float* qi",
     "const int64_t i = r;\n        const float* qi"),
    ("vs_scale_dropped",
     "Pr[j] = dot_scaled(qi, row_ptr(k, g, N, d, j), d, scale);",
     "Pr[j] = dot_scaled(qi, row_ptr(k, g, N, d, j), d, 1.0);"),
    ("vs_softmax_not_normalised",
     "for (int64_t j = 0; j <= i; ++j) Pr[j] /= l;", ""),
    ("vs_vertical_skips_first_row",
     "for (int r = 0; r < L; ++r) acc += P[(size_t)r * N + j];",
     "for (int r = 1; r < L; ++r) acc += P[(size_t)r * N + j];"),
    ("vs_slash_reads_column_not_diagonal",
     "const int64_t j = i - o;", "const int64_t j = o;"),
    ("topk_ties_prefer_higher_index",
     "return (x->i > y->i) - (x->i < y->i);", "return (x->i < y->i) - (x->i > y->i);"),
    ("topk_output_not_sorted",
     "qsort(out, (size_t)m, sizeof(int64_t), cmp_i64);", ""),
    ("bs_pools_half_the_block",
     "const int64_t i = (int64_t)b * block + r;", "const int64_t i = (int64_t)b * block + r / 2;"),
    ("bs_scores_transposed",
     "acc += Qm[(size_t)bq * d + t] * Km[(size_t)bk * d + t];",
     "acc += Qm[(size_t)bk * d + t] * Km[(size_t)bq * d + t];"),
    ("slash_tile_bound_off_by_one",
     "if (diff <= block - 1 && diff >= -(block - 1)) hit = 1;",
     "if (diff < block - 1 && diff > -(block - 1)) hit = 1;"),
    ("ashape_window_one_too_wide",
     "return j < c->sink || i - j < c->window;", "return j < c->sink || i - j <= c->window;"),
    ("ashape_sink_one_too_wide",
     "return j < c->sink || i - j < c->window;", "return j <= c->sink || i - j < c->window;"),
    ("gqa_interleaved_groups",
     "return (int)(((int64_t)h * Hkv) / Hq);", "return h % Hkv;"),
    ("attn_excludes_the_diagonal_key",
     "for (int64_t j = 0; j <= i; ++j) {\n                if (!allow(ctx, i, j)) continue;",
     "for (int64_t j = 0; j < i; ++j) {\n                if (!allow(ctx, i, j)) continue;"),
    ("attn_weights_not_normalised",
     "const double p = s[t] / l;", "const double p = s[t];"),
    ("attn_lse_drops_the_max",
     "lse[r] = m + log(l);", "lse[r] = log(l);"),
    ("vs_attn_delta_from_key_block_only",
     "return c->D[i / c->block - j / c->block] != 0;", "return c->D[j / c->block] != 0;"),
    ("vs_range_upper_bound_off_by_one",
     "int64_t lo = base - j, hi = base + c->block - 1 - j;",
     "int64_t lo = base - j, hi = base + c->block - j;"),
    ("vs_range_from_the_row_not_its_block",
     "const int64_t base = (i / c->block) * c->block; /* 64 bq */",
     "const int64_t base = i; /* 64 bq */"),
    ("vs_range_prefix_count_shifted",
     "return c->s_cnt[hi + 1] - c->s_cnt[lo] > 0;", "return c->s_cnt[hi] - c->s_cnt[lo] > 0;"),
    ("bs_attn_block_table_transposed",
     "return c->sel[(size_t)(i / c->block) * c->nB + (size_t)(j / c->block)] != 0;",
     "return c->sel[(size_t)(j / c->block) * c->nB + (size_t)(i / c->block)] != 0;"),
]


def _build(name, text):
    os.makedirs(OUT, exist_ok=True)
    c = os.path.join(OUT, name + ".c")
    so = os.path.join(OUT, "lib" + name + ".so")
    with open(c, "w") as f:
        f.write(text)
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", so, c,
                           "-lm"])
    return so


def _pins_pass(so):
    env = dict(os.environ, MINFER_ORACLE_LIB=so, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests",
                        "test_oracle_pins.py"), "-x", "-q", "-p", "no:cacheprovider"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode == 0, r.stdout[-400:]


def _run(item):
    name, text = item
    passed, tail = _pins_pass(_build(name, text))
    return name, passed, tail


def test_every_planted_mistake_fails_a_pin():
    with open(SRC) as f:
        src = f.read()
    jobs = [("control", src)]
    for name, old, new in MUTANTS:
        assert src.count(old) == 1, f"{name}: mutation site not unique in the oracle source"
        jobs.append((name, src.replace(old, new)))
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = {name: (passed, tail) for name, passed, tail in ex.map(_run, jobs)}
    assert results["control"][0], "unmutated oracle fails its pins:\n" + results["control"][1]
    survivors = [n for n, (passed, _) in results.items() if n != "control" and passed]
    assert not survivors, f"mistakes no pin catches: {survivors}"
