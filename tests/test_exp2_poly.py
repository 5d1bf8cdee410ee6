"""Error bound of the FMA-pipe exp2 used for part of the softmax
(csrc/exp2_poly.h), evaluated step by step in fp32 arithmetic on the CPU
against numpy's fp64 exp2."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "dynamic_sparse_attention_02_b200", "csrc", "exp2_poly.h")


def constants():
    txt = open(HDR).read()
    vals = dict(re.findall(r"constexpr float (kExp2\w+) = ([^;]+?)f?;", txt))
    out = {}
    for k, v in vals.items():
        out[k] = float.fromhex(v) if "0x" in v else float(v)
    return out


def f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def fma32(a, b, c):
    # fp32 fused multiply-add: exact product and sum in fp64, one rounding to fp32
    return f32(a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64))


def exp2_poly(x):
    c = constants()
    x = f32(x)
    xc = np.maximum(x, np.float32(c["kExp2Clamp"]))
    t = f32(xc.astype(np.float64) + c["kExp2Round"])
    tn = f32(t.astype(np.float64) - c["kExp2Round"])
    fr = fma32(tn, np.float32(-1.0), xc)
    p = fma32(np.full_like(fr, c["kExp2C3"]), fr, np.full_like(fr, c["kExp2C2"]))
    p = fma32(p, fr, np.full_like(fr, c["kExp2C1"]))
    p = fma32(p, fr, np.full_like(fr, c["kExp2C0"]))
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    # normal results only: below 2^-126 the output is denormal and flushed downstream
    x = np.concatenate([np.linspace(-125.0, 9.0, 2_000_001), np.arange(-125, 9) + 0.5])
    y = exp2_poly(x).astype(np.float64)
    ref = np.exp2(f32(x).astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 1e-4, rel.max()


def test_clamped_and_masked_inputs_are_tiny_and_nonnegative():
    x = np.array([-np.inf, -1e30, -200.0, -127.0, -126.7], np.float32)
    y = exp2_poly(x)
    assert np.all(y >= 0) and np.all(y < 2.0 ** -125)
    # flush-to-zero arithmetic reads anything below 2^-126 as zero
    assert np.all(y[:4] < np.finfo(np.float32).tiny)


def test_constants_reproduced_by_the_fitting_script():
    """csrc/fit_exp2.py (Remez exchange, relative error) prints the header's
    coefficients exactly."""
    import importlib.util
    path = os.path.join(os.path.dirname(HDR), "fit_exp2.py")
    spec = importlib.util.spec_from_file_location("fit_exp2", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    c32, e, e32 = mod.fp32_coefficients(3)
    k = constants()
    for j in range(4):
        assert float(c32[j]) == k[f"kExp2C{j}"], j
        assert mod.c_hex(c32[j]) in open(HDR).read()
    assert e < 7.6e-5 and e32 < 7.6e-5
