"""The per-matrix bit allocator (DynaQuant, "Step 2: bit allocation").

The oracle (oracle/alloc.py) is pinned by:
* its loss model against the oracle's own quantizer: the measured rounding
  error of Gaussian rows falls with the bit width as the model says;
* exhaustive search: every prefix of the upgrades sorted by loss removed per
  extra byte is the least total loss any assignment reaches within its own
  bytes (the marginal-allocation optimality of convex per-matrix
  trade-offs), in both modes, and the filling reaches exactly those states
  at those budgets;
* at any budget the filling has taken at least the longest such prefix that
  fits;
* maximality: after the filling no single further upgrade fits the budget;
* the end points: the lowest level's cost leaves every matrix at 4 bits,
  the cost of bf16 everywhere gives 16 bits everywhere.
The library's mpw_allocate_bits must then return the oracle's bits and total
byte for byte.  All of this runs on the host.
"""
import ctypes
import itertools

import numpy as np
import pytest

import mixed_precision_weight_row_b200 as mpw
import oracle
import workloads as wl
from oracle import alloc


def _instance(rng, n, k_mult=128):
    shapes = [(int(rng.integers(1, 9)) * 64, int(rng.integers(1, 9)) * k_mult) for _ in range(n)]
    sens = list(np.exp(rng.uniform(-3, 3, size=n)))
    return sens, shapes


def test_matrix_bytes_matches_the_packed_format():
    for N, K in [(1, 1), (7, 100), (256, 512), (5120, 17408)]:
        for b in range(4, 16):
            assert alloc.matrix_bytes(N, K, b) == N * oracle.packed_row_bytes(K, b) + 4 * N
        assert alloc.matrix_bytes(N, K, 16) == 2 * N * K
    # the pages' saving ratios at shapes where K*b is a multiple of 128
    N, K = 4096, 4096
    for b in range(5, 8):
        packed = alloc.matrix_bytes(N, K, b) - 4 * N
        assert 1 - packed / (N * K) == (8 - b) / 8
    for b in range(9, 16):
        packed = alloc.matrix_bytes(N, K, b) - 4 * N
        assert 1 - packed / (2 * N * K) == (16 - b) / 16


def test_loss_model_follows_the_quantizer():
    """D(b) / D(b+1) is the ratio of the rounding-error powers the oracle's
    quantizer produces on the same Gaussian rows (within 5%)."""
    rng = np.random.default_rng(5)
    W = rng.standard_normal((64, 4096)).astype(np.float32)
    mse = {}
    for b in range(4, 13):
        q, s = oracle.quantize(W, b)
        mse[b] = float(np.mean((np.float64(W) - oracle.dequantize(q, s)) ** 2))
    for b in range(4, 12):
        model = alloc.distortion(1.0, b) / alloc.distortion(1.0, b + 1)
        assert abs(mse[b] / mse[b + 1] / model - 1) < 0.05, b
    assert alloc.distortion(3.0, 16) == 0.0


def _prefix_states(sens, shapes, mode):
    """(bytes, bits) after each upgrade when every upgrade of every matrix is
    sorted by loss removed per extra byte (the order an unbounded filling
    takes; with convex trade-offs a matrix's upgrades come in order)."""
    lv = alloc.step_levels(mode)
    level = [0] * len(shapes)
    spent = sum(alloc.matrix_bytes(N, K, lv[0]) for N, K in shapes)
    out = [(spent, [lv[0]] * len(shapes))]
    cand = []
    for i, (N, K) in enumerate(shapes):
        for l in range(len(lv) - 1):
            g = alloc.distortion(sens[i], lv[l]) - alloc.distortion(sens[i], lv[l + 1])
            e = alloc.matrix_bytes(N, K, lv[l + 1]) - alloc.matrix_bytes(N, K, lv[l])
            cand.append((-(g / e), i, l, e))
    for _, i, l, e in sorted(cand):
        assert level[i] == l
        level[i] += 1
        spent += e
        out.append((spent, [lv[x] for x in level]))
    return out


def _greedy_prefix_budgets(sens, shapes, mode):
    """Bytes after each upgrade of the unbounded filling."""
    lv = alloc.step_levels(mode)
    full, _ = alloc.allocate(sens, shapes, 1 << 62, mode)
    assert full == [lv[-1]] * len(shapes)
    return [c for c, _ in _prefix_states(sens, shapes, mode)]


@pytest.mark.parametrize("mode", ["native", "full"])
def test_prefix_states_are_optimal_by_exhaustive_search(mode):
    """The ratio order itself: each prefix state is the least loss within its
    own bytes (exhaustive search), which pins the order the filling must
    follow."""
    rng = np.random.default_rng(17)
    for trial in range(10 if mode == "native" else 4):
        sens, shapes = _instance(rng, 4 if mode == "native" else 3)
        states = _prefix_states(sens, shapes, mode)
        for cost, bits in states[:: max(1, len(states) // 10)]:
            d = sum(alloc.distortion(s_, b) for s_, b in zip(sens, bits))
            best, _ = alloc.exhaustive(sens, shapes, cost, mode)
            assert d <= best * (1 + 1e-12) + 1e-300


@pytest.mark.parametrize("mode", ["native", "full"])
def test_filling_contains_the_largest_prefix_that_fits(mode):
    """At any budget the filling has taken, at least, every upgrade of the
    longest prefix of the ratio order that fits."""
    rng = np.random.default_rng(23)
    for trial in range(30):
        sens, shapes = _instance(rng, 5)
        states = _prefix_states(sens, shapes, mode)
        for _ in range(8):
            B = int(rng.integers(states[0][0], states[-1][0] + 1))
            bits, _ = alloc.allocate(sens, shapes, B, mode)
            pref = max((st for st in states if st[0] <= B), key=lambda st: st[0])[1]
            assert all(b >= p for b, p in zip(bits, pref)), (trial, B)


@pytest.mark.parametrize("mode", ["native", "full"])
def test_filling_states_are_optimal_for_their_budget(mode):
    rng = np.random.default_rng(11 if mode == "native" else 12)
    n_cases = 0
    for trial in range(12 if mode == "native" else 6):
        n = 4 if mode == "native" else 3
        sens, shapes = _instance(rng, n)
        budgets = _greedy_prefix_budgets(sens, shapes, mode)
        for B in budgets[:: max(1, len(budgets) // 12)] + budgets[-1:]:
            bits, spent = alloc.allocate(sens, shapes, B, mode)
            assert spent == B
            d = sum(alloc.distortion(s, b) for s, b in zip(sens, bits))
            best, _ = alloc.exhaustive(sens, shapes, B, mode)
            assert d <= best * (1 + 1e-12) + 1e-300, (trial, B)
            n_cases += 1
    assert n_cases > 30


@pytest.mark.parametrize("mode", ["native", "full"])
def test_filling_leaves_no_upgrade_that_fits(mode):
    rng = np.random.default_rng(21)
    lv = alloc.step_levels(mode)
    for trial in range(40):
        sens, shapes = _instance(rng, 6, k_mult=int(rng.choice([100, 128, 96])))
        lo = sum(alloc.matrix_bytes(N, K, 4) for N, K in shapes)
        hi = sum(alloc.matrix_bytes(N, K, 16) for N, K in shapes)
        B = int(rng.integers(lo, hi + 1))
        bits, spent = alloc.allocate(sens, shapes, B, mode)
        assert spent <= B
        assert spent == sum(alloc.matrix_bytes(N, K, b) for (N, K), b in zip(shapes, bits))
        for (N, K), b in zip(shapes, bits):
            if b != lv[-1]:
                nxt = lv[lv.index(b) + 1]
                assert alloc.matrix_bytes(N, K, nxt) - alloc.matrix_bytes(N, K, b) > B - spent


def test_end_points():
    rng = np.random.default_rng(3)
    sens, shapes = _instance(rng, 5)
    for mode in ("native", "full"):
        lo = sum(alloc.matrix_bytes(N, K, 4) for N, K in shapes)
        hi = sum(alloc.matrix_bytes(N, K, 16) for N, K in shapes)
        assert alloc.allocate(sens, shapes, lo, mode) == ([4] * 5, lo)
        assert alloc.allocate(sens, shapes, hi, mode) == ([16] * 5, hi)
        with pytest.raises(ValueError):
            alloc.allocate(sens, shapes, lo - 1, mode)


def test_exhaustive_is_brute_force():
    # two matrices, native mode: the nine assignments by hand
    sens, shapes = [1.0, 4.0], [(64, 128), (64, 128)]
    B = alloc.matrix_bytes(64, 128, 8) + alloc.matrix_bytes(64, 128, 4)
    d, bits = alloc.exhaustive(sens, shapes, B, "native")
    cands = []
    for b0, b1 in itertools.product((4, 8, 16), repeat=2):
        if alloc.matrix_bytes(64, 128, b0) + alloc.matrix_bytes(64, 128, b1) <= B:
            cands.append((alloc.distortion(1.0, b0) + alloc.distortion(4.0, b1), [b0, b1]))
    assert (d, bits) == min(cands)
    assert bits == [4, 8]   # the more sensitive matrix gets the bits


# ---------------------------------------------------------------------------
# the library against the oracle
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("mode", ["native", "full"])
def test_library_matches_oracle(mode):
    rng = np.random.default_rng(31)
    for trial in range(30):
        n = int(rng.integers(1, 40))
        sens, shapes = _instance(rng, n, k_mult=int(rng.choice([100, 128, 17])))
        if trial % 5 == 0:
            sens[0] = 0.0                        # a matrix with no measured sensitivity
            sens[-1] = sens[min(1, n - 1)]       # a tie
        lo = sum(alloc.matrix_bytes(N, K, 4) for N, K in shapes)
        hi = sum(alloc.matrix_bytes(N, K, 16) for N, K in shapes)
        for B in (lo, int(rng.integers(lo, hi + 1)), hi, hi * 2):
            assert mpw.allocate_bits(sens, shapes, B, mode) == alloc.allocate(sens, shapes, B, mode)


def test_library_matches_oracle_on_the_recipe_stack():
    shapes = [(N, K) for _, _, N, K in wl.recipe_shapes()]
    rng = np.random.default_rng(41)
    sens = list(np.exp(rng.normal(0, 1.5, size=len(shapes))))
    lo = sum(alloc.matrix_bytes(N, K, 4) for N, K in shapes)
    for mode in ("native", "full"):
        for mean_bits in (4.5, 5.7, 7.0, 9.0):
            B = int(lo * mean_bits / 4)
            bits, total = mpw.allocate_bits(sens, shapes, B, mode)
            assert (bits, total) == alloc.allocate(sens, shapes, B, mode)
            assert total <= B


def test_allocate_bits_validation():
    L = mpw.lib
    d = (ctypes.c_double * 2)(1.0, 2.0)
    n = (ctypes.c_int64 * 2)(64, 64)
    k = (ctypes.c_int64 * 2)(128, 128)
    bits = (ctypes.c_int32 * 2)(-1, -1)
    big = 1 << 40
    ok = L.mpw_allocate_bits(d, n, k, 2, big, 1, bits, None)
    assert ok == 0 and list(bits) == [16, 16]
    for args in [(None, n, k, 2, big, 1, bits, None), (d, n, k, 0, big, 1, bits, None),
                 (d, n, k, 2, big, 2, bits, None), (d, n, k, 2, 10, 1, bits, None)]:
        assert L.mpw_allocate_bits(*args) == mpw.MPW_E_INVALID_ARG
    bad = (ctypes.c_double * 2)(1.0, float("nan"))
    assert L.mpw_allocate_bits(bad, n, k, 2, big, 1, bits, None) == mpw.MPW_E_INVALID_ARG
    neg = (ctypes.c_double * 2)(1.0, -1.0)
    assert L.mpw_allocate_bits(neg, n, k, 2, big, 1, bits, None) == mpw.MPW_E_INVALID_ARG
    zero_k = (ctypes.c_int64 * 2)(128, 0)
    assert L.mpw_allocate_bits(d, n, zero_k, 2, big, 1, bits, None) == mpw.MPW_E_INVALID_ARG


# ---------------------------------------------------------------------------
# the frontier the filling walks
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("mode", ["native", "full"])
def test_frontier_is_the_sorted_prefix_states(mode):
    """Bytes of every frontier point are those of the ratio-sorted prefix
    states (which exhaustive search pins), the loss is that state's total,
    and the filling at that budget returns that state."""
    rng = np.random.default_rng(61)
    for trial in range(10):
        sens, shapes = _instance(rng, 5)
        pts = alloc.frontier(sens, shapes, mode)
        states = _prefix_states(sens, shapes, mode)
        assert len(pts) == len(states) == 1 + len(shapes) * (len(alloc.step_levels(mode)) - 1)
        for (b, l), (c, bits) in zip(pts, states):
            assert b == c
            d = sum(alloc.distortion(s_, x) for s_, x in zip(sens, bits))
            assert abs(l - d) <= 1e-9 * max(1.0, abs(d))
            assert alloc.allocate(sens, shapes, b, mode)[0] == bits
        losses = [l for _, l in pts]
        assert all(a >= c - 1e-12 * abs(a) for a, c in zip(losses, losses[1:]))
        assert pts[-1][1] == pytest.approx(0.0, abs=1e-12 * losses[0])


@pytest.mark.parametrize("mode", ["native", "full"])
def test_library_frontier_matches_oracle(mode):
    rng = np.random.default_rng(71)
    for trial in range(10):
        sens, shapes = _instance(rng, int(rng.integers(1, 30)), k_mult=int(rng.choice([100, 128, 17])))
        b_lib, l_lib = mpw.allocation_frontier(sens, shapes, mode)
        pts = alloc.frontier(sens, shapes, mode)
        assert b_lib == [b for b, _ in pts]
        assert l_lib == [l for _, l in pts]          # same fp64 operations in the same order
    shapes = [(N, K) for _, _, N, K in wl.recipe_shapes()]
    sens = list(np.exp(np.random.default_rng(72).normal(0, 1.5, size=len(shapes))))
    b_lib, l_lib = mpw.allocation_frontier(sens, shapes, mode)
    pts = alloc.frontier(sens, shapes, mode)
    assert b_lib == [b for b, _ in pts] and l_lib == [l for _, l in pts]


def test_allocate_frontier_validation():
    L = mpw.lib
    d = (ctypes.c_double * 2)(1.0, 2.0)
    n = (ctypes.c_int64 * 2)(64, 64)
    k = (ctypes.c_int64 * 2)(128, 128)
    cnt = ctypes.c_int64(-1)
    assert L.mpw_allocate_frontier(d, n, k, 2, 0, None, None, 0, ctypes.byref(cnt)) == 0 and cnt.value == 5
    assert L.mpw_allocate_frontier(d, n, k, 2, 1, None, None, 0, ctypes.byref(cnt)) == 0 and cnt.value == 25
    assert L.mpw_allocate_frontier(d, n, k, 2, 1, None, None, 3, ctypes.byref(cnt)) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_allocate_frontier(d, n, k, 0, 1, None, None, 0, ctypes.byref(cnt)) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_allocate_frontier(d, n, k, 2, 7, None, None, 0, ctypes.byref(cnt)) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_allocate_frontier(d, n, k, 2, 1, None, None, 0, None) == mpw.MPW_E_INVALID_ARG
    # a short buffer gets the first points and the full count
    b3 = (ctypes.c_uint64 * 3)()
    l3 = (ctypes.c_double * 3)()
    assert L.mpw_allocate_frontier(d, n, k, 2, 1, b3, l3, 3, ctypes.byref(cnt)) == 0 and cnt.value == 25
    pts = alloc.frontier([1.0, 2.0], [(64, 128), (64, 128)], "full")
    assert [int(v) for v in b3] == [p[0] for p in pts[:3]] and list(l3) == [p[1] for p in pts[:3]]
