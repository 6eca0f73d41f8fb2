"""How the recipe runner schedules a stack (host only: mpw_recipe_plan).

Each linear gets MPW_QLINEAR_X_READY when its input bytes were written
neither by the linear before the current run of flagged linears nor inside
that run, and MPW_QLINEAR_Y_UNSHARED as well when its output bytes are
neither read nor written there.  Slot addresses are fake (never read).
"""
import ctypes

import pytest

import mixed_precision_weight_row_b200 as mpw
import workloads as wl

X, XY = mpw.X_READY, mpw.X_READY | mpw.Y_UNSHARED
BASE = 0x10000000


def _plan(links, widths, slot_addr, M=1, shapes=None):
    n = len(links)
    arr = (mpw._Linear * n)()
    for i, (si, so) in enumerate(links):
        N, K = shapes[i] if shapes else (widths[so], widths[si])
        arr[i] = mpw._Linear(0x1000, 0x2000, N, K, 6, si, so, 0, 1, 0)
    ptrs = (ctypes.c_void_p * len(slot_addr))(*slot_addr)
    flags = (ctypes.c_uint32 * n)()
    st = mpw.lib.mpw_recipe_plan(arr, n, ptrs, len(slot_addr), M, flags)
    assert st == mpw.MPW_OK, mpw.status_str(st)
    return list(flags)


def test_the_decoder_stack_overlaps_k_v_and_up():
    links = [(si, so) for si, so, _ in wl.recipe_links()]
    widths = wl.SLOT_WIDTH
    addr = [BASE * (s + 1) for s in range(8)]
    flags = _plan(links, widths, addr)
    # q, k, v, o, gate, up, down in every layer
    assert flags == [0, XY, XY, 0, 0, XY, 0] * (len(links) // 7)


def test_aliased_slots_are_compared_by_bytes():
    widths = {0: 2048, 1: 3072, 2: 3072, 3: 3072, 4: 1024}
    addr = [BASE, 2 * BASE, 3 * BASE, 2 * BASE, 4 * BASE]        # slot 3 is slot 1
    # the third linear reads slot 3 = the second's output: it must wait
    assert _plan([(0, 2), (0, 1), (3, 4)], widths, addr) == [0, XY, 0]
    # a partial overlap counts too
    addr2 = [BASE, 2 * BASE, 3 * BASE, 2 * BASE + 1024, 4 * BASE]
    assert _plan([(0, 2), (0, 1), (3, 4)], widths, addr2) == [0, XY, 0]


def test_output_over_an_input_of_the_run_is_not_unshared():
    widths = {0: 1024, 1: 1024, 2: 1024, 3: 1024}
    addr = [BASE, 2 * BASE, 3 * BASE, BASE]                       # slot 3 is slot 0
    # the third linear writes over the input the first two read
    assert _plan([(0, 1), (0, 2), (0, 3)], widths, addr) == [0, XY, X]


def test_runs_are_bounded():
    widths = {s: 512 for s in range(12)}
    addr = [BASE * (s + 1) for s in range(12)]
    links = [(0, s) for s in range(1, 11)]
    flags = _plan(links, widths, addr)
    # eight linears per run at most: the ninth starts a new run
    assert flags == [0] + [XY] * 7 + [0, XY]


def test_plan_validates_like_the_runner():
    arr = (mpw._Linear * 1)()
    arr[0] = mpw._Linear(0x1000, 0x2000, 64, 64, 6, 0, 0, 0, 1, 0)   # in == out
    ptrs = (ctypes.c_void_p * 2)(BASE, 2 * BASE)
    flags = (ctypes.c_uint32 * 1)()
    assert mpw.lib.mpw_recipe_plan(arr, 1, ptrs, 2, 1, flags) == mpw.MPW_E_INVALID_ARG
    arr[0] = mpw._Linear(0x1000, 0x2000, 64, 64, 6, 0, 1, 0, 1, 0)
    assert mpw.lib.mpw_recipe_plan(arr, 1, ptrs, 2, 1, None) == mpw.MPW_E_INVALID_ARG
    assert mpw.lib.mpw_recipe_plan(arr, 1, ptrs, 2, 33, flags) == mpw.MPW_E_INVALID_ARG
    assert mpw.lib.mpw_recipe_plan(arr, 1, ptrs, 2, 1, flags) == mpw.MPW_OK and flags[0] == 0
