"""Plain CPU definition of the per-matrix bit allocator (water filling on a
max-heap of marginal upgrades).

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this module; only the
tests and the CPU leg of ``bench.py`` use it.  It shares no code or table with
the library's allocator.

Source (page title, section): DynaQuant (zingnex forum thread), "Step 2: bit
allocation": water filling over a max-heap of marginal bit upgrades; every
step raises one weight matrix to its next bit level, the priority being the
marginal quality gain per byte of cost; two modes, hardware-native {4, 8, 16}
and full {4, 5, ..., 16}.  "Step 1" measures one sensitivity per matrix; the
sensitivities are an input here.

Readings taken where the page is silent (each also listed in the design
notes):

* Quality loss of a matrix at b bits: D(b) = sens / Q_b^2 with
  Q_b = 2^(b-1) - 1 (the quantization step is max|w| / Q_b and uniform
  rounding noise has variance step^2 / 12; constants common to all matrices
  drop out of the ordering).  16 bits is the unquantized bf16 matrix: D = 0.
* Cost of a matrix at b bits: the bytes this library stores, N rows of
  16 * ceil(K*b/128) bytes plus a 4-byte scale per row; at 16 bits the bf16
  matrix, 2*N*K bytes.
* Every matrix starts at the lowest level of the mode (4 bits); the starting
  cost must fit the budget.
* Upgrades are taken in order of gain / extra bytes (fp64, in that operation
  order); ties go to the lower matrix index.  An upgrade that adds no bytes
  (very short rows, where the padded codes and scales can take as much room
  as bf16) has infinite priority.  An upgrade that no longer fits
  the remaining budget is dropped for good (the matrix keeps its level) and
  the filling goes on with the others.
"""
from __future__ import annotations

import heapq
import itertools

MODES = {"native": (4, 8, 16), "full": tuple(range(4, 17))}


def step_levels(mode: str):
    """Bit levels of a mode (DynaQuant, "Step 2": {4, 8, 16} or 4..16)."""
    return MODES[mode]


def matrix_bytes(N: int, K: int, b: int) -> int:
    """Stored bytes of an N x K matrix at b bits (b = 16: bf16)."""
    if b == 16:
        return 2 * N * K
    return N * (16 * ((K * b + 127) // 128)) + 4 * N


def distortion(sens: float, b: int) -> float:
    """D(b) = sens / Q_b^2, and 0 at 16 bits."""
    if b == 16:
        return 0.0
    q = float(2 ** (b - 1) - 1)
    return sens / (q * q)


def allocate(sens, shapes, budget: int, mode: str = "full"):
    """Water filling: returns (bits per matrix, total bytes).

    sens: sensitivities (floats >= 0); shapes: (N, K) per matrix; budget:
    bytes.  Raises ValueError when the lowest level does not fit.
    """
    lv = step_levels(mode)
    n = len(shapes)
    level = [0] * n
    spent = sum(matrix_bytes(N, K, lv[0]) for N, K in shapes)
    if spent > budget:
        raise ValueError("budget below the cost of the lowest level")
    heap = []

    def push(i):
        if level[i] + 1 < len(lv):
            N, K = shapes[i]
            b0, b1 = lv[level[i]], lv[level[i] + 1]
            gain = distortion(sens[i], b0) - distortion(sens[i], b1)
            extra = matrix_bytes(N, K, b1) - matrix_bytes(N, K, b0)
            # an upgrade that costs no bytes (short rows, where bf16 can take
            # no more room than padded codes and scales) goes first
            prio = float("inf") if extra <= 0 else gain / extra
            # max-heap on the priority, then the lower index
            heapq.heappush(heap, (-prio, i, extra))

    for i in range(n):
        push(i)
    while heap:
        _, i, extra = heapq.heappop(heap)
        if spent + extra > budget:
            continue
        spent += extra
        level[i] += 1
        push(i)
    return [lv[l] for l in level], spent


def frontier(sens, shapes, mode: str = "full"):
    """The curve the filling walks without a budget: (bytes, total loss)
    after each upgrade, from the lowest level everywhere to the highest.
    The total starts as the sum of the losses in matrix order and each
    upgrade subtracts its gain (fp64, in that order)."""
    lv = step_levels(mode)
    level = [0] * len(shapes)
    spent = sum(matrix_bytes(N, K, lv[0]) for N, K in shapes)
    total = 0.0
    for i in range(len(shapes)):
        total += distortion(sens[i], lv[0])
    heap = []

    def push(i):
        if level[i] + 1 < len(lv):
            N, K = shapes[i]
            b0, b1 = lv[level[i]], lv[level[i] + 1]
            gain = distortion(sens[i], b0) - distortion(sens[i], b1)
            extra = matrix_bytes(N, K, b1) - matrix_bytes(N, K, b0)
            prio = float("inf") if extra <= 0 else gain / extra
            heapq.heappush(heap, (-prio, i, extra))

    for i in range(len(shapes)):
        push(i)
    points = [(spent, total)]
    while heap:
        _, i, extra = heapq.heappop(heap)
        l = level[i]
        total -= distortion(sens[i], lv[l]) - distortion(sens[i], lv[l + 1])
        spent += extra
        level[i] += 1
        push(i)
        points.append((spent, total))
    return points


def exhaustive(sens, shapes, budget: int, mode: str = "full"):
    """Brute force over every assignment of levels (tiny inputs only):
    (least total distortion within the budget, its bits)."""
    lv = step_levels(mode)
    best = None
    for bits in itertools.product(lv, repeat=len(shapes)):
        cost = sum(matrix_bytes(N, K, b) for (N, K), b in zip(shapes, bits))
        if cost > budget:
            continue
        d = sum(distortion(s, b) for s, b in zip(sens, bits))
        if best is None or d < best[0]:
            best = (d, list(bits))
    return best
