"""Pins of the oracle's FP8 (E4M3) path (oracle/fp8.py) against what the
format and the mathematics fix, independently of the oracle's own code:

* every E4M3 value, decoded here byte by byte from the format's definition
  (sign, 4 exponent bits with bias 7, 3 mantissa bits, subnormals m * 2^-9,
  the all-ones pattern not a number), and the nearest of them found by brute
  force (ties to the code with the even mantissa) -- the oracle's rounding
  must pick it for every probe, ties and the saturation point included;
* torch's own float8_e4m3fn conversion agrees inside the finite range;
* codes of up to 5 bits are exact in E4M3 and 17 is not (why the path stops
  at b = 5, as DynaQuant "Custom kernel architecture" implies);
* the per-token scale: every nonzero token reaches +-448 exactly, zero
  tokens give zeros, the sign of every element is kept;
* the linear against a Fraction triple loop on tiny inputs;
* the bound on the error the rounding of x causes, on random inputs;
* planted mistakes (ties away from zero, truncation, a 480 maximum, one scale
  for the whole tensor, a dropped activation scale) each fail a pin.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import fp8


def e4m3_table():
    """{byte: value} of the 254 finite E4M3 codes, from the bit layout."""
    out = {}
    for byte in range(256):
        sign = -1.0 if byte & 0x80 else 1.0
        e = (byte >> 3) & 0xF
        m = byte & 0x7
        if e == 0xF and m == 0x7:
            continue                                  # not a number
        if e == 0:
            mag = m * 2.0 ** -9                       # subnormal
        else:
            mag = (1.0 + m / 8.0) * 2.0 ** (e - 7)
        out[byte] = sign * mag
    return out


TABLE = e4m3_table()
VALUES = np.array(sorted(set(TABLE.values())))
EVEN = {v for b, v in TABLE.items() if (b & 1) == 0}


def nearest_brute(v: float) -> float:
    """Nearest finite E4M3 value, ties to the even mantissa, saturating."""
    if v >= 448.0:
        return 448.0
    if v <= -448.0:
        return -448.0
    d = np.abs(VALUES - v)
    best = VALUES[d == d.min()]
    if len(best) == 1:
        return float(best[0])
    even = [b for b in best if b in EVEN]
    assert len(even) == 1
    return float(even[0])


def probes():
    rng = np.random.default_rng(0)
    pts = list(VALUES)
    mids = (VALUES[1:] + VALUES[:-1]) / 2             # every tie
    pts += list(mids)
    pts += list(np.nextafter(mids.astype(np.float32), np.float32(np.inf)))
    pts += list(np.nextafter(mids.astype(np.float32), np.float32(-np.inf)))
    pts += list(rng.uniform(-470, 470, 4000)) + list(rng.standard_normal(4000) * 3)
    pts += list(rng.standard_normal(2000) * 2.0 ** -8)   # the subnormal range
    pts += [448.0, 449.0, 463.9, 464.0, 464.1, 479.0, 1e6, -1e6, 0.0]
    return np.array(pts, dtype=np.float32)


def test_table_shape():
    assert len(TABLE) == 254 and max(VALUES) == 448.0 and min(VALUES) == -448.0
    assert 2.0 ** -9 in VALUES and 2.0 ** -6 in VALUES


def test_rounding_is_the_nearest_value_ties_to_even():
    p = probes()
    got = oracle.e4m3_round(p)
    want = np.array([nearest_brute(float(v)) for v in p], dtype=np.float32)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, [(float(p[i]), float(got[i]), float(want[i])) for i in bad[:5]]


def test_rounding_agrees_with_torch_inside_the_range():
    import torch

    p = probes()
    p = p[np.abs(p) <= 448]
    t = torch.from_numpy(p).to(torch.float8_e4m3fn).to(torch.float32).numpy()
    assert np.array_equal(oracle.e4m3_round(p), t)


def test_codes_up_to_five_bits_are_exact():
    for q in range(-15, 16):
        assert float(q) in TABLE.values()
    assert 17.0 not in TABLE.values()          # a 6-bit code (|q| <= 31) would round
    for b in (4, 5):
        Q = oracle.qmax(b)
        q = np.arange(-Q, Q + 1, dtype=np.float32)
        assert np.array_equal(oracle.e4m3_round(q), q)
    fp8.check_bits(5)
    with pytest.raises(ValueError):
        fp8.check_bits(6)


def test_per_token_scale():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((6, 300)).astype(np.float32)
    x[2] = 0
    x[3] *= np.float32(1e-30)
    xq, sx = oracle.quantize_x_fp8(x)
    assert sx.dtype == np.float32 and xq.dtype == np.float32
    assert sx[2] == np.float32(1.0) / np.float32(448.0)
    assert not xq[2].any()
    for m in (0, 1, 3, 4, 5):
        assert np.max(np.abs(xq[m])) == 448.0
        assert sx[m] == np.float32(np.max(np.abs(x[m])) / np.float32(448.0))
    assert np.all(np.isin(xq, VALUES))
    assert np.all((np.sign(xq) == np.sign(x)) | (xq == 0))


def test_linear_against_fractions():
    rng = np.random.default_rng(2)
    for b in (4, 5):
        W = rng.standard_normal((5, 7)).astype(np.float32)
        q, s = oracle.quantize(W, b)
        x = rng.standard_normal((3, 7)).astype(np.float32)
        y, bound = oracle.qlinear_fp8_ref(x, q, s)
        xq, sx = oracle.quantize_x_fp8(x)
        for m in range(3):
            for n in range(5):
                exact = sum(Fraction(float(xq[m, k])) * int(q[n, k]) for k in range(7))
                exact *= Fraction(float(sx[m])) * Fraction(float(s[n]))
                assert abs(Fraction(float(y[m, n])) - exact) <= abs(exact) * Fraction(1, 2 ** 50)
        assert np.all(bound > 0)


def test_input_rounding_bound_holds():
    rng = np.random.default_rng(3)
    for b in (4, 5):
        W = rng.standard_normal((40, 512)).astype(np.float32) * np.float32(0.02)
        q, s = oracle.quantize(W, b)
        x = rng.standard_normal((9, 512)).astype(np.float32)
        x[4] *= np.float32(1e-3)
        x[5, :100] *= np.float32(1e-6)             # elements in E4M3's subnormal range
        y8, _ = oracle.qlinear_fp8_ref(x, q, s)
        y, _ = oracle.qlinear_ref(x, q, s)
        eb = oracle.fp8_input_error_bound(x, q, s)
        assert np.all(np.abs(y8 - y) <= eb)
        # and it is not vacuous: the typical error is well inside it
        assert np.median(np.abs(y8 - y) / eb) < 0.5


# ---- planted mistakes: each must break a pin above ----

def _ties_away(v):
    v = np.asarray(v, np.float32)
    a = np.abs(v.astype(np.float64))
    _, e = np.frexp(a)
    quantum = np.ldexp(1.0, np.maximum(e - 1, -6) - 3)
    r = np.minimum(np.floor(a / quantum + 0.5) * quantum, 448.0)
    return (np.sign(v) * r).astype(np.float32)


def _truncate(v):
    v = np.asarray(v, np.float32)
    a = np.abs(v.astype(np.float64))
    _, e = np.frexp(a)
    quantum = np.ldexp(1.0, np.maximum(e - 1, -6) - 3)
    r = np.minimum(np.floor(a / quantum) * quantum, 448.0)
    return (np.sign(v) * r).astype(np.float32)


def _max480(v):
    v = np.asarray(v, np.float32)
    a = np.abs(v.astype(np.float64))
    _, e = np.frexp(a)
    quantum = np.ldexp(1.0, np.maximum(e - 1, -6) - 3)
    r = np.minimum(np.rint(a / quantum) * quantum, 480.0)
    return (np.sign(v) * r).astype(np.float32)


@pytest.mark.parametrize("mutant", [_ties_away, _truncate, _max480])
def test_planted_rounding_mistakes_are_caught(mutant):
    p = probes()
    want = np.array([nearest_brute(float(v)) for v in p], dtype=np.float32)
    assert not np.array_equal(mutant(p), want)


def test_planted_scale_mistakes_are_caught():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((4, 64)).astype(np.float32)
    x[1] *= 10
    # one scale for the whole tensor: a token that does not hold the tensor
    # maximum no longer reaches 448
    amax = np.float32(np.max(np.abs(x)))
    xq_tensor = oracle.e4m3_round(x / (amax / np.float32(448)))
    assert any(np.max(np.abs(xq_tensor[m])) != 448.0 for m in range(4))
    # a dropped activation scale changes the linear by orders of magnitude
    W = rng.standard_normal((3, 64)).astype(np.float32)
    q, s = oracle.quantize(W, 5)
    xq, sx = oracle.quantize_x_fp8(x)
    y, bound = oracle.qlinear_fp8_ref(x, q, s)
    wrong = xq.astype(np.float64) @ (q * s.astype(np.float64)[:, None]).T
    assert not oracle.check_qlinear(wrong, y, bound).all()
