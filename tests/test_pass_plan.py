"""Host checks of the planned decode pass's dependency lists
(mpw_pass_dependencies; no GPU: slot addresses are compared, never read).

The pins are independent of the library's code: a brute-force list of every
earlier linear that conflicts with a later one (it writes bytes the later one
reads, or reads or writes bytes the later one writes), which must all be
reachable through the listed dependencies, and the recipe stack's lists as
the decoder layer's data flow gives them by hand.
"""
import pytest

import workloads as wl


def _mpw():
    import mixed_precision_weight_row_b200 as mpw

    return mpw


def _fake_layers(mpw, specs):
    # (N, K, in_slot, out_slot): packed / scales at distinct aligned fake addresses
    return [mpw.Linear(0x10000000 + 0x100000 * i, 0x20000000 + 0x1000 * i, N, K, 6, si, so, True,
                       layout="paired") for i, (N, K, si, so) in enumerate(specs)]


def _conflicts(specs, addr):
    """Brute force: pairs (j, i), j < i, whose byte ranges conflict."""
    def rng(slot, n):
        return addr[slot], addr[slot] + 2 * n

    def ov(a, b):
        return a[0] < b[1] and b[0] < a[1]

    out = set()
    for i, (Ni, Ki, si, so) in enumerate(specs):
        xi, yi = rng(si, Ki), rng(so, Ni)
        for j in range(i):
            Nj, Kj, sj, soj = specs[j]
            xj, yj = rng(sj, Kj), rng(soj, Nj)
            if ov(yj, xi) or ov(xj, yi) or ov(yj, yi):
                out.add((j, i))
    return out


def _closure(deps):
    anc = []
    for i, d in enumerate(deps):
        a = set()
        for j in d:
            assert j < i
            a |= anc[j] | {j}
        anc.append(a)
    return anc


def _check(specs, addr, M=1):
    mpw = _mpw()
    layers = _fake_layers(mpw, specs)
    deps = mpw.pass_dependencies(layers, list(addr), M)
    anc = _closure(deps)
    for j, i in _conflicts(specs, addr):
        assert j in anc[i], (j, i)
    for i, d in enumerate(deps):
        # no listed dependency is already covered by another listed one
        for a in d:
            for b in d:
                assert a == b or a not in anc[b], (i, a, b)
        # nothing listed that does not conflict
        assert set(d) <= {j for j, k in _conflicts(specs, addr) if k == i}
    return deps


def _recipe_specs(layers):
    shapes, links = wl.recipe_shapes(layers), wl.recipe_links(layers)
    return [(N, K, si, so) for (_, _, N, K), (si, so, _) in zip(shapes, links)]


def test_recipe_stack_dependencies():
    layers = 16
    specs = _recipe_specs(layers)
    # separate slot buffers, far apart
    addr = [0x40000000 + (s << 22) for s in range(8)]
    deps = _check(specs, addr)
    names = [n for (_, n, _, _) in wl.recipe_shapes(layers)]
    assert deps[0] == deps[1] == deps[2] == []
    for layer in range(1, layers):
        b = 7 * layer
        idx = {names[b + t]: b + t for t in range(7)}
        prev = {names[b - 7 + t]: b - 7 + t for t in range(7)}
        # q reads the previous down's output; its own slot's last reader (the
        # previous o) is covered by that down
        assert deps[idx["q"]] == [prev["down"]]
        # o reads q's output and overwrites the slot the previous gate read
        assert set(deps[idx["o"]]) == {idx["q"], prev["gate"]}
        assert deps[idx["gate"]] == [idx["o"]] and deps[idx["up"]] == [idx["o"]]
        # down reads up's output and overwrites the slot that k and v read
        assert set(deps[idx["down"]]) == {idx["up"], idx["k"], idx["v"]}
        assert prev["down"] in deps[idx["k"]] and prev["down"] in deps[idx["v"]]
    # layer 0's down only waits for up (nothing read slot D before it)
    assert deps[6] == [5]


def test_aliased_slots_dependencies():
    # slot 2 is the upper half of slot 1; slot 3 separate
    base = 0x50000000
    addr = [base, base + 1024, base + 2048, base + 0x100000]
    specs = [(1024, 512, 0, 1), (640, 512, 2, 3), (512, 640, 3, 0), (512, 512, 0, 2), (256, 512, 0, 3)]
    deps = _check(specs, addr)
    assert deps[1] == [0]               # reads part of what 0 wrote
    assert set(deps[3]) == {2}          # 2 covers 0 and 1 transitively
    # 4 reads what 2 wrote and overwrites what 2 read and 1 wrote; 2 waits for 1
    assert deps[4] == [2]


def test_random_stacks_dependencies():
    import numpy as np

    rng = np.random.default_rng(0)
    for trial in range(30):
        nslots = int(rng.integers(3, 7))
        # slots as windows of one buffer, some overlapping
        starts = sorted(int(v) for v in rng.integers(0, 64, nslots))
        addr = [0x60000000 + 256 * s for s in starts]
        specs = []
        for _ in range(int(rng.integers(2, 24))):
            si, so = rng.choice(nslots, 2, replace=False)
            K = 128 * int(rng.integers(1, 4))
            N = 16 * int(rng.integers(1, 40))
            # skip linears whose input and output bytes overlap (refused)
            x0, y0 = addr[si], addr[so]
            if x0 < y0 + 2 * N and y0 < x0 + 2 * K:
                continue
            specs.append((N, K, int(si), int(so)))
        if specs:
            _check(specs, addr)


def test_dependency_errors():
    mpw = _mpw()
    addr = [0x70000000, 0x70000000 + 512]   # overlapping windows
    layers = _fake_layers(mpw, [(512, 512, 0, 1)])
    with pytest.raises(mpw.MPWError) as e:
        mpw.pass_dependencies(layers, addr, 1)
    assert e.value.status == mpw.MPW_E_INVALID_ARG
    addr = [0x70000000, 0x71000000]
    with pytest.raises(mpw.MPWError) as e:
        mpw.pass_dependencies(layers, addr, 2)
    assert e.value.status == mpw.MPW_E_UNSUPPORTED
    canon = [mpw.Linear(0x10000000, 0x20000000, 512, 512, 6, 0, 1, False, layout="canonical")]
    with pytest.raises(mpw.MPWError) as e:
        mpw.pass_dependencies(canon, addr, 1)
    assert e.value.status == mpw.MPW_E_UNSUPPORTED
    wide = [mpw.Linear(0x10000000, 0x20000000, 512, 512, 9, 0, 1, False, layout="paired")]
    with pytest.raises(mpw.MPWError) as e:
        mpw.pass_dependencies(wide, addr, 1)
    assert e.value.status == mpw.MPW_E_UNSUPPORTED
    ragged_k = [mpw.Linear(0x10000000, 0x20000000, 512, 480, 6, 0, 1, False, layout="paired")]
    with pytest.raises(mpw.MPWError) as e:
        mpw.pass_dependencies(ragged_k, addr, 1)
    assert e.value.status == mpw.MPW_E_UNSUPPORTED
