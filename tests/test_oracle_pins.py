"""Pins for the CPU oracle: it is checked against things other than itself.

* hand-derived fixtures (tests/golden/) built from the printed formulas;
* exact rational arithmetic (IEEE rounding re-derived with Fractions) on small
  random inputs, including ties and subnormals;
* a packer written as one big Python integer;
* special cases that reduce to library routines (b = 8 is an int8 view,
  b = 4 is two nibbles per byte);
* closed-form invariants (code range, the row maximum hits +-Q, signs,
  monotonicity, the rounding-error bound);
* size formulas and the bandwidth ratios printed on the DynaQuant page;
* brute-force dequantize-then-multiply with Fractions for the linear layer.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests import _exact as ex

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
SUB = np.finfo(np.float32).smallest_subnormal


def _parse_value(tok: str) -> float:
    if tok.startswith("sub:"):
        return float(np.float32(float(tok[4:]) * float(SUB))) if tok[4:] != "0" else 0.0
    if tok.startswith("hex:"):
        return ex.f32_from_bits(int(tok[4:], 16))
    return float(tok)


def _load_golden():
    cases = []
    for name in sorted(os.listdir(GOLDEN)):
        if not name.endswith(".txt") or name == "README.txt":
            continue
        d = {}
        for line in open(os.path.join(GOLDEN, name)):
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            k, v = line.split(":", 1)
            d[k.strip()] = v.strip()
        b = int(d["bits"])
        w = np.array([_parse_value(t) for t in d["w"].split()], dtype=np.float32)
        scale = np.float32(_parse_value(d["scale"]))
        codes = [int(t) for t in d["codes"].split()]
        packed = bytes(int(t, 16) for t in d["packed"].split())
        cases.append(pytest.param(b, w, scale, codes, packed, id=name[:-4]))
    return cases


def _subnormal_from_multiple(k: int) -> np.float32:
    return np.float32(k * float(SUB))


# ----------------------------------------------------------------------------
# hand-derived fixtures
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("b,w,scale,codes,packed", _load_golden())
def test_golden_fixture(b, w, scale, codes, packed):
    W = w[None, :]
    q, s = oracle.quantize(W, b)
    assert ex.f32_bits(float(s[0])) == ex.f32_bits(float(scale))
    assert q[0].tolist() == codes
    p = oracle.pack(q, b)
    assert p[0].tobytes() == packed
    assert oracle.unpack(p, W.shape[1], b)[0].tolist() == codes


def test_golden_subnormal_values_are_exact():
    # the fixture notation sub:k means k * 2^-149, exactly representable
    for k in (1, 3, 10, -10):
        v = _subnormal_from_multiple(k)
        assert Fraction(float(v)) == k * ex.SUB_ULP


# ----------------------------------------------------------------------------
# exact arithmetic on small random inputs
# ----------------------------------------------------------------------------

def _tiny_rows(rng, n_rows, K):
    rows = []
    for i in range(n_rows):
        kind = i % 6
        if kind == 0:
            r = rng.standard_normal(K).astype(np.float32) * np.float32(0.02)
        elif kind == 1:       # ties: multiples of half a step of a power-of-two scale
            b_hint = 4 + (i % 12)
            Q = (1 << (b_hint - 1)) - 1
            r = (rng.integers(-2 * Q, 2 * Q + 1, size=K) / 2.0).astype(np.float32)
            r[0] = np.float32(Q)
        elif kind == 2:       # subnormals
            r = (rng.integers(-50, 51, size=K) * float(SUB)).astype(np.float32)
        elif kind == 3:       # wide dynamic range
            r = (np.exp2(rng.uniform(-40, 40, size=K)) * rng.choice([-1, 1], size=K)).astype(np.float32)
        elif kind == 4:       # sparse, with an outlier
            r = np.zeros(K, np.float32)
            r[rng.integers(0, K, size=3)] = rng.standard_normal(3).astype(np.float32)
            r[rng.integers(0, K)] *= np.float32(20)
        else:                 # zero row
            r = np.zeros(K, np.float32)
        rows.append(r)
    return np.stack(rows)


@pytest.mark.parametrize("b", list(range(4, 16)))
def test_scales_and_codes_match_exact_arithmetic(b):
    rng = np.random.default_rng(100 + b)
    W = _tiny_rows(rng, 24, 37)
    q, s = oracle.quantize(W, b)
    for n in range(W.shape[0]):
        codes, s_exact = ex.exact_codes(W[n], b)
        assert Fraction(float(s[n])) == s_exact, (n, s[n], s_exact)
        assert q[n].tolist() == codes, n


def test_round_to_f32_matches_hardware_conversion():
    # the exact rounding helper agrees with numpy's own float64 -> float32
    # conversion wherever that conversion rounds once (values exact in float64)
    rng = np.random.default_rng(3)
    vals = np.concatenate([rng.standard_normal(2000), np.exp2(rng.uniform(-149, 120, 2000))])
    for v in vals:
        assert ex.round_to_f32(Fraction(float(v))) == Fraction(float(np.float32(v)))


@pytest.mark.parametrize("b", list(range(4, 16)))
def test_pack_matches_big_integer_packer(b):
    rng = np.random.default_rng(200 + b)
    Q = oracle.qmax(b)
    for K in (1, 2, 7, 31, 32, 33, 64, 127, 128, 129, 300):
        q = rng.integers(-Q, Q + 1, size=(3, K)).astype(np.int32)
        p = oracle.pack(q, b)
        assert p.shape == (3, 16 * math.ceil(K * b / 128))
        for n in range(3):
            assert p[n].tobytes() == ex.pack_row_int(q[n].tolist(), b, K)
            assert oracle.unpack(p, K, b)[n].tolist() == ex.unpack_row_int(p[n].tobytes(), b, K)


@pytest.mark.parametrize("b", list(range(4, 16)))
def test_unpack_inverts_pack(b):
    rng = np.random.default_rng(300 + b)
    Q = oracle.qmax(b)
    q = rng.integers(-Q, Q + 1, size=(5, 1000)).astype(np.int32)
    q[0, :] = Q
    q[1, :] = -Q
    assert np.array_equal(oracle.unpack(oracle.pack(q, b), 1000, b), q)


# ----------------------------------------------------------------------------
# special cases that reduce to library routines
# ----------------------------------------------------------------------------

def test_b8_is_int8_view():
    rng = np.random.default_rng(4)
    q = rng.integers(-127, 128, size=(4, 64)).astype(np.int32)
    p = oracle.pack(q, 8)
    assert np.array_equal(p, q.astype(np.int8).view(np.uint8))


def test_b4_is_two_nibbles_per_byte():
    rng = np.random.default_rng(5)
    q = rng.integers(-7, 8, size=(4, 64)).astype(np.int32)
    p = oracle.pack(q, 4)
    lo = q[:, 0::2] & 15
    hi = q[:, 1::2] & 15
    assert np.array_equal(p[:, :32], (lo | (hi << 4)).astype(np.uint8))


# ----------------------------------------------------------------------------
# invariants
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("b", list(range(4, 16)))
def test_code_invariants(b):
    rng = np.random.default_rng(400 + b)
    W = rng.standard_normal((64, 257)).astype(np.float32) * np.float32(0.02)
    W[5] = 0
    q, s = oracle.quantize(W, b)
    Q = oracle.qmax(b)
    assert np.all(np.abs(q) <= Q)
    nz = np.any(W != 0, axis=1)
    # the row maximum lands on +-Q
    am = np.argmax(np.abs(W), axis=1)
    assert np.all(np.abs(q[np.arange(64), am])[nz] == Q)
    # signs agree or the code is zero
    assert np.all((np.sign(q) == np.sign(W)) | (q == 0))
    # monotone within each row
    for n in range(0, 64, 7):
        order = np.argsort(W[n], kind="stable")
        assert np.all(np.diff(q[n][order]) >= 0)
    # zero row: codes 0, scale fl32(1/Q)
    assert np.all(q[5] == 0)
    assert s[5] == np.float32(1.0) / np.float32(Q)
    # re-quantizing the reconstruction with the same scale returns the codes
    w_hat = oracle.dequantize(q, s)
    with np.errstate(divide="ignore", invalid="ignore"):
        q2 = np.clip(np.rint(w_hat / s[:, None]), -Q, Q).astype(np.int32)
    assert np.array_equal(q2, q)


@pytest.mark.parametrize("b", list(range(4, 16)))
def test_rounding_error_bound(b):
    # Tutorial, "How quantization works": each value is off by at most scale/2.
    # With the quotient rounded to fp32 first, |w - q s| <= s (1/2 + Q 2^-23).
    rng = np.random.default_rng(500 + b)
    W = rng.standard_normal((32, 500)).astype(np.float32)
    W.flat[rng.integers(0, W.size, 50)] *= np.float32(20)
    q, s = oracle.quantize(W, b)
    Q = oracle.qmax(b)
    err = np.abs(W.astype(np.float64) - q.astype(np.float64) * s.astype(np.float64)[:, None])
    lim = s.astype(np.float64)[:, None] * (0.5 + Q * 2.0 ** -23)
    assert np.all(err <= lim)
    strict = int(np.sum(err > s.astype(np.float64)[:, None] / 2))
    assert strict <= W.size // 1000


def test_snr_rises_about_6db_per_bit():
    # Tutorial, "Step 2: quality metrics" / "Step 3: bit-width sweep".
    rng = np.random.default_rng(7)
    W = rng.standard_normal((256, 1024)).astype(np.float32)
    snr = []
    for b in range(4, 16):
        q, s = oracle.quantize(W, b)
        snr.append(oracle.quality(W, oracle.dequantize(q, s))["snr_db"])
    # uniform rounding noise ~ (s^2 / 12) with s = max / Q: the SNR step from b
    # to b+1 is 20 log10(Q(b+1) / Q(b)), which tends to 6.02 dB per bit
    steps = np.diff(snr)
    expect = np.array([20 * np.log10(oracle.qmax(b + 1) / oracle.qmax(b)) for b in range(4, 15)])
    assert np.all(np.abs(steps - expect) < 0.1), (steps, expect)
    assert abs(expect[-1] - 6.02) < 0.01


# ----------------------------------------------------------------------------
# sizes and the ratios printed on the DynaQuant page
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("b", list(range(4, 16)))
def test_packed_sizes(b):
    for K in (1, 3, 16, 100, 512, 4096, 5120, 17408):
        assert oracle.unpadded_row_bytes(K, b) == math.ceil(K * b / 8)
        rb = oracle.packed_row_bytes(K, b)
        assert rb % 16 == 0 and rb >= math.ceil(K * b / 8) and rb - math.ceil(K * b / 8) < 16


def test_bandwidth_saving_ratios():
    # DynaQuant, "Custom kernel architecture": savings (8-N)/8 for 5-7 bits and
    # (16-N)/16 for 9-15 bits.  At the benchmark shapes K*b is a multiple of
    # 128, so packed bytes / (N*K) is exactly b/8.
    for K in (4096, 5120, 6144, 17408):
        for b in range(5, 8):
            r = Fraction(oracle.packed_row_bytes(K, b), K)
            assert 1 - r / 1 == Fraction(8 - b, 8)
        for b in range(9, 16):
            r = Fraction(oracle.packed_row_bytes(K, b), 2 * K)
            assert 1 - r == Fraction(16 - b, 16)
    # "5-7 bits at 62% of the FP8 cost": 5/8
    assert Fraction(oracle.packed_row_bytes(4096, 5), 4096) == Fraction(5, 8)


def test_benchmark_sizes():
    assert 4096 * oracle.packed_row_bytes(4096, 5) == 10_485_760
    assert 4096 * oracle.packed_row_bytes(4096, 12) == 25_165_824
    assert 17408 * oracle.packed_row_bytes(5120, 6) == 66_846_720
    assert 256 * oracle.packed_row_bytes(512, 5) == 81_920


# ----------------------------------------------------------------------------
# the linear layer
# ----------------------------------------------------------------------------

def _bf16_values(rng, shape):
    import torch

    return torch.from_numpy(rng.standard_normal(shape).astype(np.float32)).to(torch.bfloat16).float().numpy()


@pytest.mark.parametrize("b", [4, 5, 8, 9, 12, 15])
def test_qlinear_against_fraction_triple_loop(b):
    rng = np.random.default_rng(600 + b)
    M, N, K = 3, 5, 19
    W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)
    x = _bf16_values(rng, (M, K))
    q, s = oracle.quantize(W, b)
    y, bound = oracle.qlinear_ref(x, q, s)
    for m in range(M):
        for n in range(N):
            exact = Fraction(float(s[n])) * sum(Fraction(float(x[m, k])) * int(q[n, k]) for k in range(K))
            assert abs(Fraction(float(y[m, n])) - exact) <= abs(exact) * Fraction(1, 2 ** 45) + Fraction(1, 2 ** 200)
            babs = sum(abs(Fraction(float(x[m, k])) * int(q[n, k]) * Fraction(float(s[n]))) for k in range(K))
            assert abs(Fraction(float(bound[m, n])) - (Fraction(8, 1000) * babs + Fraction(1, 10 ** 6))) <= babs * Fraction(1, 2 ** 40) + Fraction(1, 10 ** 12)


def test_qlinear_b8_matches_torch_dequantized_matmul():
    import torch

    rng = np.random.default_rng(8)
    W = rng.standard_normal((40, 64)).astype(np.float32)
    x = _bf16_values(rng, (4, 64))
    q, s = oracle.quantize(W, 8)
    y, _ = oracle.qlinear_ref(x, q, s)
    w_hat = torch.from_numpy(q.astype(np.float64)) * torch.from_numpy(s.astype(np.float64))[:, None]
    yt = torch.from_numpy(x.astype(np.float64)) @ w_hat.T
    assert np.allclose(y, yt.numpy(), rtol=1e-14, atol=1e-14)


@pytest.mark.parametrize("b", list(range(10, 16)))
def test_hi_lo_split_is_exact_in_bf16(b):
    # Codes wider than the bf16 significand are split q = 256*hi + lo with
    # lo = q & 255 in [0, 255] and hi = q >> 8 (arithmetic); both 256*hi and lo
    # are exact in bf16, so no code is rounded on the tensor cores.
    import torch

    Q = oracle.qmax(b)
    q = np.arange(-Q, Q + 1, dtype=np.int64)
    lo = q & 255
    hi = q >> 8
    assert np.array_equal(256 * hi + lo, q)
    for part in (lo, 256 * hi):
        t = torch.from_numpy(part.astype(np.float32))
        assert torch.equal(t.to(torch.bfloat16).float(), t)


def test_codes_up_to_nine_bits_are_exact_in_bf16():
    import torch

    for b in range(4, 10):
        Q = oracle.qmax(b)
        t = torch.arange(-Q, Q + 1, dtype=torch.float32)
        assert torch.equal(t.to(torch.bfloat16).float(), t)
    t = torch.tensor([257.0])
    assert not torch.equal(t.to(torch.bfloat16).float(), t)


def test_nonfinite_weights_are_rejected():
    W = np.zeros((2, 4), np.float32)
    W[1, 2] = np.inf
    with pytest.raises(ValueError):
        oracle.quantize(W, 6)
    W[1, 2] = np.nan
    with pytest.raises(ValueError):
        oracle.quantize(W, 6)


def test_bits_out_of_range_are_rejected():
    with pytest.raises(ValueError):
        oracle.qmax(3)
    with pytest.raises(ValueError):
        oracle.qmax(16)


def test_rms_scale_closed_forms():
    # constant rows: mean(v^2) = c^2, so r = 1 / sqrt(c^2 + 1e-6)
    v = np.array([[2.0] * 10, [-0.5] * 4 + [0.5] * 4, [0.0] * 3], dtype=object)
    r0 = oracle.rms_scale(np.full((1, 10), 2.0))[0, 0]
    assert abs(r0 - 1.0 / np.sqrt(4.0 + 1e-6)) < 1e-15
    r1 = oracle.rms_scale(np.array([[-0.5, 0.5, -0.5, 0.5]]))[0, 0]
    assert abs(r1 - 1.0 / np.sqrt(0.25 + 1e-6)) < 1e-15
    r2 = oracle.rms_scale(np.zeros((1, 3)))[0, 0]
    assert abs(r2 - 1000.0) < 1e-9
    # the scaled row has mean square 1 up to the epsilon
    rng = np.random.default_rng(2)
    x = rng.standard_normal((3, 500)) * 7.0
    xs = x * oracle.rms_scale(x)
    assert np.allclose(np.mean(xs ** 2, axis=1), 1.0, atol=1e-6)
    # the rms-scaled linear is the plain linear scaled per token
    W = rng.standard_normal((6, 500)).astype(np.float32)
    q, s = oracle.quantize(W, 7)
    y1, _ = oracle.qlinear_rms_ref(x, q, s)
    y0, _ = oracle.qlinear_ref(x, q, s)
    assert np.allclose(y1, y0 * oracle.rms_scale(x), rtol=1e-12)


# ----------------------------------------------------------------------------
# Paired-halves layout (kernel-private ordering of the packed bits)
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("b", list(range(4, 16)))
def test_paired_matches_big_integer_packer(b):
    rng = np.random.default_rng(700 + b)
    Q = oracle.qmax(b)
    K = 96
    q = rng.integers(-Q, Q + 1, size=(3, K)).astype(np.int32)
    q[0, :32] = Q
    q[1, 32:64] = -Q
    got = oracle.pack_paired(q, b)
    rb = oracle.packed_row_bytes(K, b)
    for n in range(q.shape[0]):
        want = ex.pack_paired_row_int([int(v) for v in q[n]], b)
        assert bytes(got[n, : len(want)]) == want
        assert not got[n, len(want):rb].any()


@pytest.mark.parametrize("b", [4, 5, 7, 8, 11, 15])
def test_unpack_paired_inverts_pack_paired(b):
    rng = np.random.default_rng(800 + b)
    Q = oracle.qmax(b)
    q = rng.integers(-Q, Q + 1, size=(4, 160)).astype(np.int32)
    assert np.array_equal(oracle.unpack_paired(oracle.pack_paired(q, b), 160, b), q)


def test_paired_b8_bytes_are_2x2_transposes():
    # b = 8: word h of a group holds codes (4h, 4h+2) in its low half and
    # (4h+1, 4h+3) in its high half, i.e. each block of four int8 codes
    # [a0, a1, a2, a3] is stored as [a0, a2, a1, a3].
    rng = np.random.default_rng(81)
    q = rng.integers(-127, 128, size=(3, 64)).astype(np.int32)
    p = oracle.pack_paired(q, 8).view(np.int8).astype(np.int32)
    want = q.reshape(3, 16, 2, 2).transpose(0, 1, 3, 2).reshape(3, 64)
    assert np.array_equal(p, want)


def test_paired_b4_nibble_order():
    # b = 4: the eight nibbles of word h (low nibble first) are codes
    # 8h + (0, 2, 4, 6, 1, 3, 5, 7) of the group.
    rng = np.random.default_rng(41)
    q = rng.integers(-7, 8, size=(2, 64)).astype(np.int32)
    p = oracle.pack_paired(q, 4)
    words = p.view("<u4")
    for n in range(2):
        for w in range(8):
            nib = [(int(words[n, w]) >> (4 * t)) & 15 for t in range(8)]
            codes = [v - 16 if v >= 8 else v for v in nib]
            want = [int(q[n, 8 * w + j]) for j in (0, 2, 4, 6, 1, 3, 5, 7)]
            assert codes == want


@pytest.mark.parametrize("b", [5, 6, 9, 13])
def test_paired_is_a_permutation_of_each_canonical_group(b):
    # For K a multiple of 32 a canonical group also fills exactly b words, so
    # the two layouts hold the same multiset of bits word-group by word-group.
    rng = np.random.default_rng(900 + b)
    Q = oracle.qmax(b)
    q = rng.integers(-Q, Q + 1, size=(5, 128)).astype(np.int32)
    c = np.unpackbits(oracle.pack(q, b), axis=1).reshape(5, -1)
    p = np.unpackbits(oracle.pack_paired(q, b), axis=1).reshape(5, -1)
    g_bits = 32 * b
    for g in range(4):
        assert np.array_equal(c[:, g * g_bits:(g + 1) * g_bits].sum(1), p[:, g * g_bits:(g + 1) * g_bits].sum(1))
    assert np.array_equal(oracle.pair_halves(oracle.pack(q, b), 128, b), oracle.pack_paired(q, b))


def test_paired_needs_k_multiple_of_32():
    with pytest.raises(ValueError):
        oracle.pack_paired(np.zeros((1, 48), np.int32), 5)
    with pytest.raises(ValueError):
        oracle.unpack_paired(np.zeros((1, oracle.packed_row_bytes(48, 5)), np.uint8), 48, 5)
