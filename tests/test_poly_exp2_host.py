"""The attention kernel's optional FMA-pipe exp2 (poly_ex2x2, compiled out unless
DSA_POLY_PERIOD > 0) checked on the CPU against the mathematics: its constants are
read from the kernel source, its float32 steps replayed in numpy (each FMA as an
exact product and sum rounded once to float32), and 2^x compared with the exact
value over the whole clamped range.  CPU only."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "dynamic_sparse_attention_build_b200", "csrc", "dsa_attn.cu")


def _constants():
    src = open(SRC, encoding="utf-8").read()
    body = src[src.index("poly_ex2x2(float x0"):]
    shift = float(re.search(r"kShift\s*=\s*([0-9.eE+-]+)f", body).group(1))
    cs = re.search(r"c0\s*=\s*([0-9.eE+-]+)f,\s*c1\s*=\s*([0-9.eE+-]+)f,\s*c2\s*=\s*([0-9.eE+-]+)f,"
                   r"\s*c3\s*=\s*([0-9.eE+-]+)f", body)
    clamp = float(re.search(r"fmaxf\(x0,\s*(-?[0-9.]+)f\)", body).group(1))
    return np.float32(shift), [np.float32(c) for c in cs.groups()], np.float32(clamp)


def _fma32(a, b, c):
    # a*b is exact in float64 for float32 inputs; one rounding of the sum to float32
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _poly_ex2(x):
    shift, (c0, c1, c2, c3), clamp = _constants()
    x = x.astype(np.float32)
    cx = np.maximum(x, clamp)
    y = (cx + shift).astype(np.float32)         # add.rn.f32
    j = (y - shift).astype(np.float32)          # round(x)
    f = (cx - j).astype(np.float32)             # in [-1/2, 1/2]
    p = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.full_like(f, c0))
    bits = (p.view(np.uint32).astype(np.uint64) + (y.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    out = bits.astype(np.uint32).view(np.float32)
    return np.where(x > clamp, out, np.float32(0.0))


def test_relative_error_within_documented_bound():
    x = np.linspace(-124.999, 0.0, 2_000_001, dtype=np.float64).astype(np.float32)
    y = _poly_ex2(x).astype(np.float64)
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(y - exact) / exact
    assert rel.max() < 1e-4, rel.max()   # the source states 7.5e-5 from the fit


def test_reduced_argument_and_masked_keys():
    # integers are exact powers of two up to the polynomial's value at f = 0
    shift, (c0, _, _, _), _ = _constants()
    for k in (-100, -7, -1, 0):
        got = float(_poly_ex2(np.array([k], np.float32))[0])
        assert abs(got / 2.0 ** k - float(c0)) < 1e-7
    # at or below the clamp (masked keys are -inf) the result is exactly 0, like ex2.approx.ftz
    z = _poly_ex2(np.array([-125.0, -126.0, -1e30, -np.inf], np.float32))
    assert (z == 0).all()
