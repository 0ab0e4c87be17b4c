"""CPU check of the FMA-pipe 2^x used by the forward kernel (ex2_poly2 in
csrc/ssm_common.cuh): its coefficients are read from the source and the exact
fp32 operation sequence is emulated in numpy, then compared with 2^x in fp64
over the whole range the kernel uses it on (x <= 0)."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "selective_state_space_50_b200", "csrc", "ssm_common.cuh")


def coefficients():
    src = open(SRC).read()
    body = src[src.index("float2 ex2_poly2("):]
    body = body[:body.index("return make_float2(__int_as_float")]
    vals = [float(v) for v in re.findall(r"make_float2\(([-0-9.e]+)f, \1f\)", body)]
    # order in the source: clamp, +M, -M, -1, c5, c4, c3, c2, c1, c0
    return vals


def emulate(x):
    x = np.asarray(x, dtype=np.float32)
    vals = coefficients()
    M = np.float32(12582912.0)
    assert vals[0] == 12582912.0 and vals[1] == -12582912.0 and vals[2] == -1.0
    c5, c4, c3, c2, c1, c0 = [np.float32(v) for v in vals[3:9]]
    x = np.maximum(x, np.float32(-126.0))
    t = (x + M).astype(np.float32)
    j = (t - M).astype(np.float32)
    r = (x - j).astype(np.float32)           # fma(j, -1, x) is exact here
    p = np.float32(c5)
    for c in (c4, c3, c2, c1, c0):
        p = (p * r + c).astype(np.float32)   # fma rounding differs by < 1 ulp
    bits = (p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_coefficients_parse():
    vals = coefficients()
    assert len(vals) == 9 and vals[8] == 1.0


def test_relative_error_matches_sfu_class():
    x = np.concatenate([np.linspace(-126.0, 0.0, 2_000_001), -np.logspace(-8, 2, 100_001)])
    x = x.astype(np.float32)
    got = emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    # degree-5 minimax on [-1/2, 1/2]: 2^-22 plus the rounding of the Horner steps
    assert rel.max() < 4e-7, rel.max()


def test_integers_and_clamp():
    for k in range(0, 127):
        assert emulate(np.float32(-k)) == np.float32(2.0 ** -k)
    # below the clamp the result stays the smallest normal power, never garbage
    for v in (-126.5, -200.0, -1e6, -3.0e38):
        out = float(emulate(np.float32(v)))
        assert 0.0 < out <= 2.0 ** -125
