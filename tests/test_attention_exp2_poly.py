"""2^x on the FMA pipe (csrc/fma_exp2.cuh): x = n + f with n = rint(x) read
from the low mantissa bits of x + 1.5 * 2^23, 2^f from a polynomial on
[-1/2, 1/2], and n added to the exponent field.  The attention kernel takes a
quarter of its exponentials this way (the cubic), the scan's GELU its
exp(-a^2/2) (the quartic).  This test replays those fp32 steps in numpy with
the header's own constants and holds them to the stated bounds: relative
error at most 1e-4 (cubic) and 4e-6 (quartic) for x in [-125, 8], about
2^-125 below that, NaN kept NaN."""
import os
import re

import numpy as np
import pytest

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "test_rnn_layer_b200", "csrc",
                   "fma_exp2.cuh")
BOUND = {"kC3": 1e-4, "kC4": 4e-6}


def _constants(name):
    got = dict(re.findall(r"(" + name + r"_\d) = ([0-9.eE+-]+)f", open(SRC).read()))
    return [np.float32(float(got[f"{name}_{k}"])) for k in range(len(got))]


def _ex2(x, name):
    """The header's steps in fp32 (each fma rounded once: computed in fp64, then rounded)."""
    c = _constants(name)
    x = np.asarray(x, dtype=np.float32)
    x = np.where(x < np.float32(-125.0), np.float32(-125.0), x).astype(np.float32)   # NaN stays NaN
    shift = np.float32(12582912.0)
    t = (x + shift).astype(np.float32)
    f = (x - (t - shift).astype(np.float32)).astype(np.float32)
    p = np.full_like(f, c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = (p.astype(np.float64) * f + c[k]).astype(np.float32)
    bits = (p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


@pytest.mark.parametrize("name", ["kC3", "kC4"])
def test_relative_error_within_bound(name):
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001), np.arange(-125, 9) + 0.5,
                        np.random.default_rng(0).uniform(-30, 8, 200_000)]).astype(np.float32)
    got = _ex2(x, name).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < BOUND[name], rel.max()


@pytest.mark.parametrize("name", ["kC3", "kC4"])
def test_below_range_and_nan(name):
    got = _ex2(np.array([-126.0, -1e4, -np.inf, np.nan], dtype=np.float32), name)
    assert np.all(np.abs(got[:3].astype(np.float64) / 2.0 ** -125 - 1.0) < BOUND[name])   # the polynomial at f = 0
    assert np.isnan(got[3])


def test_the_attention_kernel_uses_the_header():
    src = open(os.path.join(os.path.dirname(SRC), "attn_seg_tc.cu")).read()
    assert '#include "fma_exp2.cuh"' in src and "kC3_3" in src
