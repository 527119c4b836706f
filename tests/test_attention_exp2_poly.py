"""The attention kernel takes a quarter of its exponentials 2^x on the FMA pipe:
x = n + f with n = rint(x) read from the low mantissa bits of x + 1.5 * 2^23,
2^f from a cubic on [-1/2, 1/2], and n added to the exponent field.  This test
replays those fp32 steps in numpy with the kernel's own constants (read from
its source) and holds the result to the bound the kernel states: relative
error at most 1e-4 (25 times below the bf16 rounding the weights get) for
x in [-125, 8], 2^-125 (to the same bound) below that, NaN kept NaN."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "test_rnn_layer_b200", "csrc",
                   "attn_seg_tc.cu")


def _constants():
    text = open(SRC).read()
    got = {k: float(v) for k, v in re.findall(r"(kExp2C[0-3]) = ([0-9.eE+-]+)f", text)}
    assert set(got) == {"kExp2C0", "kExp2C1", "kExp2C2", "kExp2C3"}
    return [np.float32(got[f"kExp2C{i}"]) for i in range(4)]


def _ex2_poly(x):
    """The kernel's steps in fp32 (fma rounded once: computed in fp64, then rounded)."""
    c0, c1, c2, c3 = _constants()
    x = np.asarray(x, dtype=np.float32)
    x = np.where(x < np.float32(-125.0), np.float32(-125.0), x).astype(np.float32)   # NaN stays NaN
    shift = np.float32(12582912.0)
    t = (x + shift).astype(np.float32)
    f = (x - (t - shift).astype(np.float32)).astype(np.float32)
    fma = lambda a, b, c: (a.astype(np.float64) * b + c).astype(np.float32)
    p = fma(np.full_like(f, c3), f, np.full_like(f, c2))
    p = fma(p, f, np.full_like(f, c1))
    p = fma(p, f, np.full_like(f, c0))
    bits = (p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_within_bound():
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001), np.arange(-125, 9) + 0.5,
                        np.random.default_rng(0).uniform(-30, 8, 200_000)]).astype(np.float32)
    got = _ex2_poly(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 1e-4, rel.max()


def test_below_range_and_nan():
    got = _ex2_poly(np.array([-126.0, -1e4, -np.inf, np.nan], dtype=np.float32))
    assert np.all(np.abs(got[:3].astype(np.float64) / 2.0 ** -125 - 1.0) < 1e-4)   # the cubic's value at f = 0
    assert np.isnan(got[3])


def test_integers_are_nearly_exact():
    n = np.arange(-125, 9, dtype=np.float32)
    got = _ex2_poly(n).astype(np.float64)
    assert np.all(np.abs(got / np.exp2(n.astype(np.float64)) - 1.0) < 1e-4)
