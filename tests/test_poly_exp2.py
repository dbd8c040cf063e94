"""CPU check of the fine kernel's FMA-pipe exponential (csrc/poly_exp2.cuh).

The kernel computes part of its softmax numerators 2^x with a fitted cubic
instead of the MUFU instruction. This test reads the coefficients and the
clamp range from the header and replays the device function's float32
operation sequence in numpy (the clamp, the 1.5 * 2^23 rounding add, the
reduced argument, three fused multiply-adds, the integer add into the
exponent field), then checks the header's stated bound against exp2 in
float64 on a dense grid.
"""
import os
import re

import numpy as np

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "trainable_block_sparse_cube_b200",
                      "csrc", "poly_exp2.cuh")
BOUND = 7.8e-5


def _constants():
    src = open(HEADER).read()
    vals = {}
    for name in ("C3", "C2", "C1", "C0", "XMIN", "XMAX"):
        m = re.search(r"#define VSA_POLY_EXP2_%s\s+\(?\s*([-+0-9.eE]+)f\)?" % name, src)
        assert m, f"VSA_POLY_EXP2_{name} not found in the header"
        vals[name] = np.float32(float(m.group(1)))
    return vals


def _fma32(a, b, c):
    # a*b of two float32 values is exact in float64; one rounding to float32
    # after the add models fmaf (a double rounding would move the result by an
    # ulp at most, far below the bound checked here)
    return (a.astype(np.float64) * b.astype(np.float64) + np.float64(c)).astype(np.float32)


def poly_exp2_emulated(x):
    k = _constants()
    x = np.minimum(np.maximum(np.asarray(x, dtype=np.float32), k["XMIN"]), k["XMAX"]).astype(np.float32)
    big = np.float32(12582912.0)                       # 1.5 * 2^23
    t = (x + big).astype(np.float32)
    f = (x - (t - big).astype(np.float32)).astype(np.float32)
    p = _fma32(np.full_like(f, k["C3"]), f, k["C2"])
    p = _fma32(p, f, k["C1"])
    p = _fma32(p, f, k["C0"])
    bits = (p.view(np.uint32).astype(np.int64) + ((t.view(np.uint32).astype(np.int64) << 23) & 0xFFFFFFFF)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_within_stated_bound():
    k = _constants()
    rng = np.random.default_rng(0)
    grid = np.linspace(float(k["XMIN"]), float(k["XMAX"]), 4_000_001).astype(np.float32)
    rand = rng.uniform(float(k["XMIN"]), float(k["XMAX"]), 1_000_000).astype(np.float32)
    # the half-integers are where the reduced argument reaches +-1/2
    halves = (np.arange(int(k["XMIN"]), int(k["XMAX"])) + 0.5).astype(np.float32)
    x = np.concatenate([grid, rand, halves, np.nextafter(halves, np.float32(0))])
    y = poly_exp2_emulated(x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= BOUND, f"max relative error {rel.max():.3e} at x = {x[np.argmax(rel)]}"
    # the fit is not looser than it needs to be either: the bound is attained to 1%
    assert rel.max() >= 0.99 * 7.7e-5


def test_clamped_ends():
    k = _constants()
    lo = np.array([-1e4, -300.0, -126.0, float(k["XMIN"])], dtype=np.float32)
    y = poly_exp2_emulated(lo).astype(np.float64)
    assert np.all(np.isfinite(y)) and np.all(y > 0)
    assert np.all(np.abs(y - 2.0 ** -125) <= 2.0 ** -124)     # about 2^-125: never a subnormal pattern
    hi = poly_exp2_emulated(np.array([64.0, 100.0], dtype=np.float32)).astype(np.float64)
    assert np.all(np.abs(hi / 2.0 ** 64 - 1) <= BOUND)


def test_emulation_catches_a_wrong_coefficient():
    """The replay is sensitive to the coefficients: a perturbed cubic term
    breaks the bound (so the check above is not vacuous)."""
    k = _constants()
    x = np.linspace(-20, 20, 100_001).astype(np.float32)
    base = poly_exp2_emulated(x).astype(np.float64)
    big = np.float32(12582912.0)
    t = (x + big).astype(np.float32)
    f = (x - (t - big).astype(np.float32)).astype(np.float32)
    p = _fma32(np.full_like(f, np.float32(k["C3"] * 1.05)), f, k["C2"])
    p = _fma32(p, f, k["C1"])
    p = _fma32(p, f, k["C0"])
    bits = (p.view(np.uint32).astype(np.int64) + ((t.view(np.uint32).astype(np.int64) << 23) & 0xFFFFFFFF)) & 0xFFFFFFFF
    bad = bits.astype(np.uint32).view(np.float32).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.abs(base / ref - 1).max() <= BOUND
    assert np.abs(bad / ref - 1).max() > BOUND
