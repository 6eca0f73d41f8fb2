"""Planted mistakes: each plausible slip in the oracle must fail a pin.

The mistakes are planted in the oracle on the CPU (monkeypatched copies of its
functions); the pin tests from test_oracle_pins are then run against them and
must raise.
"""
import numpy as np
import pytest

import oracle
import oracle.quant as oq
from tests import test_oracle_pins as pins

GOLDEN = pins._load_golden()


def _run_pins():
    """Run a fixed subset of pins; return True if any of them fails."""
    failures = 0
    checks = [lambda: [pins.test_golden_fixture(*c.values) for c in GOLDEN]]
    checks += [lambda b=b: pins.test_scales_and_codes_match_exact_arithmetic(b) for b in (4, 5, 6, 11)]
    checks += [lambda b=b: pins.test_pack_matches_big_integer_packer(b) for b in (4, 6, 13)]
    checks += [lambda b=b: pins.test_unpack_inverts_pack(b) for b in (5, 12)]
    checks += [lambda: pins.test_b8_is_int8_view(), lambda: pins.test_b4_is_two_nibbles_per_byte()]
    checks += [lambda b=b: pins.test_qlinear_against_fraction_triple_loop(b) for b in (5, 12)]
    checks += [lambda b=b: pins.test_packed_sizes(b) for b in (5, 7)]
    checks += [lambda b=b: pins.test_rounding_error_bound(b) for b in (4, 9)]
    checks += [lambda b=b: pins.test_paired_matches_big_integer_packer(b) for b in (5, 8)]
    checks += [lambda: pins.test_paired_b8_bytes_are_2x2_transposes(), lambda: pins.test_paired_b4_nibble_order()]
    checks += [lambda b=b: pins.test_unpack_paired_inverts_pack_paired(b) for b in (7,)]
    for c in checks:
        try:
            c()
        except (AssertionError, ValueError, IndexError):
            failures += 1
    return failures


def _patch(monkeypatch, name, fn):
    monkeypatch.setattr(oq, name, fn)
    monkeypatch.setattr(oracle, name, fn)


def test_unmutated_oracle_passes_the_subset():
    assert _run_pins() == 0


def _quantize_with(rounder=np.rint, clamp=True, q_of=oq.qmax, zero_scale=None):
    def quantize(W, b):
        Q = np.float32(q_of(b))
        m = np.max(np.abs(W), axis=1).astype(np.float32)
        zs = np.float32(1.0) / Q if zero_scale is None else np.float32(zero_scale)
        with np.errstate(all="ignore"):
            s = np.where(m == 0, zs, m / Q).astype(np.float32)
            t = W / s[:, None]
        r = rounder(t)
        r = np.where(np.isnan(r), np.float32(0), r)
        if clamp:
            r = np.clip(r, -oq.qmax(b), oq.qmax(b))
        else:
            r = np.where(np.isinf(r), np.sign(r) * oq.qmax(b), r)
        return r.astype(np.int32), s
    return quantize


MUTANTS = {
    "floor_instead_of_rint": lambda mp: _patch(mp, "quantize", _quantize_with(rounder=np.floor)),
    "round_half_away": lambda mp: _patch(mp, "quantize", _quantize_with(
        rounder=lambda t: np.sign(t) * np.floor(np.abs(t) + 0.5))),
    "scale_uses_2_pow_b_minus_1": lambda mp: _patch(mp, "quantize", _quantize_with(q_of=lambda b: 1 << (b - 1))),
    "no_clamp": lambda mp: _patch(mp, "quantize", _quantize_with(clamp=False)),
    "zero_row_scale_one": lambda mp: _patch(mp, "quantize", _quantize_with(zero_scale=1.0)),
    "msb_first_bits": lambda mp: _patch(mp, "pack", lambda q, b: np.packbits(
        np.unpackbits(oq.pack.__wrapped__(q, b) if hasattr(oq.pack, "__wrapped__") else ORIG_PACK(q, b),
                      axis=1, bitorder="little"), axis=1, bitorder="big")),
    "pad_to_8_bytes": lambda mp: _patch(mp, "packed_row_bytes", lambda K, b: 8 * ((K * b + 63) // 64)),
    "unpack_without_sign_extension": lambda mp: _patch(mp, "unpack", lambda p, K, b: np.where(
        ORIG_UNPACK(p, K, b) < 0, ORIG_UNPACK(p, K, b) + (1 << b), ORIG_UNPACK(p, K, b)).astype(np.int32)),
    "qlinear_drops_scale": lambda mp: _patch(mp, "qlinear_ref", lambda x, q, s: ORIG_QLINEAR(x, q, np.ones_like(s))),
    "paired_streams_swapped": lambda mp: _patch(mp, "pack_paired", lambda q, b: ORIG_PACK_PAIRED(
        np.ascontiguousarray(q.reshape(q.shape[0], -1, 2)[:, :, ::-1].reshape(q.shape)), b)),
    "paired_codes_adjacent_not_even_odd": lambda mp: _patch(mp, "pack_paired", lambda q, b: ORIG_PACK_PAIRED(
        np.ascontiguousarray(q.reshape(q.shape[0], -1, 2, 16).transpose(0, 1, 3, 2).reshape(q.shape)), b)),
    "qlinear_transposed_codes": lambda mp: _patch(mp, "qlinear_ref", lambda x, q, s: ORIG_QLINEAR(
        x, np.ascontiguousarray(q[::-1]), s[::-1])),
}

ORIG_PACK = oq.pack
ORIG_UNPACK = oq.unpack
ORIG_QLINEAR = oq.qlinear_ref
ORIG_PACK_PAIRED = oq.pack_paired


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    MUTANTS[name](monkeypatch)
    assert _run_pins() > 0, f"mutant {name} passed every pin"
