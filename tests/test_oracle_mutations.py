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


# ---------------------------------------------------------------------------
# the bit allocator (oracle/alloc.py)
# ---------------------------------------------------------------------------

import heapq  # noqa: E402

import oracle.alloc as oa  # noqa: E402
from tests import test_allocator as apins  # noqa: E402

ORIG_ALLOCATE = oa.allocate


def _run_alloc_pins():
    failures = 0
    checks = [apins.test_matrix_bytes_matches_the_packed_format, apins.test_loss_model_follows_the_quantizer,
              apins.test_end_points]
    checks += [lambda m=m: apins.test_filling_states_are_optimal_for_their_budget(m) for m in ("native", "full")]
    checks += [lambda m=m: apins.test_filling_leaves_no_upgrade_that_fits(m) for m in ("native", "full")]
    checks += [lambda m=m: apins.test_filling_contains_the_largest_prefix_that_fits(m) for m in ("native", "full")]
    checks += [lambda m=m: apins.test_prefix_states_are_optimal_by_exhaustive_search(m) for m in ("native",)]
    for c in checks:
        try:
            c()
        except (AssertionError, ValueError, IndexError, ZeroDivisionError):
            failures += 1
    return failures


def _allocate_with(priority=lambda gain, extra: gain / extra, stop_at_first_drop=False):
    def allocate(sens, shapes, budget, mode="full"):
        lv = oa.step_levels(mode)
        level = [0] * len(shapes)
        spent = sum(oa.matrix_bytes(N, K, lv[0]) for N, K in shapes)
        if spent > budget:
            raise ValueError("budget")
        heap = []

        def push(i):
            if level[i] + 1 < len(lv):
                N, K = shapes[i]
                b0, b1 = lv[level[i]], lv[level[i] + 1]
                gain = oa.distortion(sens[i], b0) - oa.distortion(sens[i], b1)
                extra = oa.matrix_bytes(N, K, b1) - oa.matrix_bytes(N, K, b0)
                heapq.heappush(heap, (-(float("inf") if extra <= 0 else priority(gain, extra)), i, extra))

        for i in range(len(shapes)):
            push(i)
        while heap:
            _, i, extra = heapq.heappop(heap)
            if spent + extra > budget:
                if stop_at_first_drop:
                    break
                continue
            spent += extra
            level[i] += 1
            push(i)
        return [lv[l] for l in level], spent
    return allocate


ALLOC_MUTANTS = {
    "priority_is_gain_not_gain_per_byte": lambda mp: mp.setattr(oa, "allocate", _allocate_with(lambda g, e: g)),
    "priority_is_bytes_per_gain": lambda mp: mp.setattr(oa, "allocate", _allocate_with(lambda g, e: e / g if g else 0)),
    "filling_stops_at_first_misfit": lambda mp: mp.setattr(oa, "allocate", _allocate_with(stop_at_first_drop=True)),
    "loss_not_squared": lambda mp: mp.setattr(oa, "distortion",
                                              lambda s, b: 0.0 if b == 16 else s / float(2 ** (b - 1) - 1)),
    "bf16_costed_as_packed_codes": lambda mp: mp.setattr(
        oa, "matrix_bytes",
        lambda N, K, b: N * (16 * ((K * b + 127) // 128)) + 4 * N),
}


def test_unmutated_allocator_oracle_passes_its_pins():
    assert oa.allocate is ORIG_ALLOCATE
    assert _run_alloc_pins() == 0


@pytest.mark.parametrize("name", sorted(ALLOC_MUTANTS))
def test_planted_allocator_mistake_is_caught(name, monkeypatch):
    ALLOC_MUTANTS[name](monkeypatch)
    assert _run_alloc_pins() > 0, name


# ---------------------------------------------------------------------------
# group-wise scales (oracle/quant.py)
# ---------------------------------------------------------------------------

from tests import test_oracle_groups as gpins  # noqa: E402


def _run_group_pins():
    failures = 0
    checks = [lambda b=b: gpins.test_one_group_per_row_is_the_per_row_quantizer(b) for b in (4, 9)]
    checks += [lambda b=b, g=g: gpins.test_groups_are_rows_of_the_reshaped_matrix(b, g)
               for b in (5, 12) for g in (8, 128)]
    checks += [lambda b=b: gpins.test_groups_match_exact_arithmetic(b) for b in (4, 11)]
    checks += [lambda b=b: gpins.test_error_bound_per_group(b) for b in (6,)]
    checks += [gpins.test_smaller_groups_reconstruct_better, gpins.test_group_linear_against_fraction_triple_loop]
    for c in checks:
        try:
            c()
        except (AssertionError, ValueError, IndexError):
            failures += 1
    return failures


def _group_scales_with(axis_rows=False, last_from_row=False, shift=0):
    def group_scales(W, b, g):
        W = np.asarray(W)
        N, K = W.shape
        Q = np.float32(oq.qmax(b))
        G = oq.group_count(K, g)
        s = np.empty((N, G), np.float32)
        for j in range(G):
            if axis_rows:
                blk = W[(j * g) % max(N, 1):(j * g) % max(N, 1) + g, :]
                m = np.full(N, np.max(np.abs(blk)) if blk.size else 0, np.float32)
            elif last_from_row and j == G - 1 and K % g:
                m = np.max(np.abs(W), axis=1).astype(np.float32)
            else:
                lo = max(0, j * g + shift)
                m = np.max(np.abs(W[:, lo:(j + 1) * g + shift]), axis=1).astype(np.float32) \
                    if lo < K else np.zeros(N, np.float32)
            s[:, j] = np.where(m == 0, np.float32(1) / Q, m / Q).astype(np.float32)
        return s
    return group_scales


GROUP_MUTANTS = {
    "groups_across_rows": lambda mp: _patch(mp, "group_scales", _group_scales_with(axis_rows=True)),
    "last_partial_group_takes_the_row_max": lambda mp: _patch(mp, "group_scales",
                                                              _group_scales_with(last_from_row=True)),
    "group_boundaries_off_by_one": lambda mp: _patch(mp, "group_scales", _group_scales_with(shift=1)),
    "linear_uses_the_first_group_scale_only": lambda mp: _patch(
        mp, "group_scale_of_weight",
        lambda s, K, g: np.repeat(np.asarray(s, np.float32)[:, :1], K, axis=1)),
}


def test_unmutated_group_oracle_passes_its_pins():
    assert _run_group_pins() == 0


@pytest.mark.parametrize("name", sorted(GROUP_MUTANTS))
def test_planted_group_mistake_is_caught(name, monkeypatch):
    GROUP_MUTANTS[name](monkeypatch)
    assert _run_group_pins() > 0, name
