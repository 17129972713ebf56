"""Host-side model of the polynomial exp2 used by the prefill softmax.

The kernel computes part of its probabilities 2^x on the FMA pipes
(csrc/exp2_poly.cuh): x is clamped at -126, split into j = rint(x) and
f = x - j, 2^f comes from a degree-3 polynomial, the result is rounded to
bf16 and j is added to its exponent field.  This test replays those fp32
steps bit for bit in numpy, with the coefficients read from the header, and
checks the result against 2^x computed in fp64 and rounded to bf16.

The pins are mathematical facts, not the kernel: 2^x for integer x is exact,
the bf16 result is within one ulp of the correctly rounded value everywhere
on [-126, 9], and the clamp keeps -inf and very negative inputs at a tiny
non-negative value instead of NaN or a wrapped exponent.
"""
import os
import re

import numpy as np
import pytest

HDR = os.path.join(os.path.dirname(__file__), "..", "block_skipping_softmax_b200", "csrc",
                   "exp2_poly.cuh")


def _consts():
    txt = open(HDR).read()
    vals = {}
    for name in ("kExp2C0", "kExp2C1", "kExp2C2", "kExp2C3", "kExp2Round", "kExp2Lo"):
        m = re.search(rf"constexpr float {name} = ([-0-9.e]+)f;", txt)
        assert m, name
        vals[name] = np.float32(float(m.group(1)))
    return vals


def _fma32(a, b, c):
    # a*b is exact in fp64 for fp32 operands; the sum is rounded once to fp64
    # and once to fp32, which equals the fused result except in double-rounding
    # ties that this test's one-ulp bound does not depend on
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _bf16_bits_rne(x32):
    u = x32.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) & 0xFFFF
    return r.astype(np.uint32)


def model_exp2_bf16(x):
    """bf16 bit patterns the kernel produces for fp32 inputs x."""
    c = _consts()
    x = np.maximum(np.asarray(x, np.float32), c["kExp2Lo"])
    t = (x + c["kExp2Round"]).astype(np.float32)
    j = (t - c["kExp2Round"]).astype(np.float32)
    f = _fma32(j, np.full_like(j, -1.0), x)
    p = _fma32(f, np.full_like(f, c["kExp2C3"]), np.full_like(f, c["kExp2C2"]))
    p = _fma32(f, p, np.full_like(f, c["kExp2C1"]))
    p = _fma32(f, p, np.full_like(f, c["kExp2C0"]))
    w = _bf16_bits_rne(p)
    tb = t.view(np.uint32).astype(np.uint64)
    # low-half form of the packed update: bf16(p) + 128 j, with j read from t's bits
    out = (w.astype(np.uint64) + (tb << 7) + 0x60000000) & 0xFFFFFFFF
    return (out & 0xFFFF).astype(np.uint32)


def _bf16_to_f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _ref_bits(x):
    return _bf16_bits_rne(np.exp2(x.astype(np.float64)).astype(np.float32))


def test_integer_powers_are_exact():
    x = np.arange(-126, 9, dtype=np.float32)
    got = _bf16_to_f64(model_exp2_bf16(x))
    np.testing.assert_array_equal(got, np.exp2(x.astype(np.float64)))


def test_within_one_ulp_and_mostly_correctly_rounded():
    rng = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-126, 9, 2_000_001, dtype=np.float32),
                        rng.uniform(-30, 8, 500_000).astype(np.float32)])
    got = model_exp2_bf16(x).astype(np.int64)
    ref = _ref_bits(x).astype(np.int64)
    # positive bf16 patterns are ordered like their values: one ulp = 1
    assert np.max(np.abs(got - ref)) <= 1
    assert np.mean(got == ref) > 0.95


def test_relative_error_bound():
    x = np.linspace(-20, 8, 400_001, dtype=np.float32)
    got = _bf16_to_f64(model_exp2_bf16(x))
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1)
    assert np.max(rel) < 2.0 ** -8 + 1e-4  # one bf16 ulp at most


@pytest.mark.parametrize("x", [-np.inf, -1e30, -1000.0, -200.0, -127.0, -126.6])
def test_clamped_inputs_stay_tiny_and_nonnegative(x):
    got = _bf16_to_f64(model_exp2_bf16(np.array([x], np.float32)))[0]
    assert np.isfinite(got) and 0.0 <= got <= 2.0 ** -125


def test_high_half_update_matches_low_half():
    # the kernel adds 2^23 j to the high half; the same exponent arithmetic
    # on the high half must give the same bf16 as the low-half form
    c = _consts()
    x = np.linspace(-126, 8, 100_001, dtype=np.float32)
    lo = model_exp2_bf16(x)
    xc = np.maximum(x, c["kExp2Lo"])
    t = (xc + c["kExp2Round"]).astype(np.float32)
    tb = t.view(np.uint32).astype(np.uint64)
    j = (t - c["kExp2Round"]).astype(np.float32)
    f = _fma32(j, np.full_like(j, -1.0), xc)
    p = _fma32(f, np.full_like(f, c["kExp2C3"]), np.full_like(f, c["kExp2C2"]))
    p = _fma32(f, p, np.full_like(f, c["kExp2C1"]))
    p = _fma32(f, p, np.full_like(f, c["kExp2C0"]))
    word = (_bf16_bits_rne(p).astype(np.uint64) << 16)
    hi = ((word + (tb << 23) + 0x60000000 + (0x4B400000 << 7)) & 0xFFFFFFFF) >> 16
    # the 0xA0000000 that (low-half t) << 7 contributes is absent when only
    # the high half is updated, so it is added back above
    np.testing.assert_array_equal(hi.astype(np.uint32), lo)
