"""The planned decode pass (mpw_pass_*: a stack of linears as one persistent
kernel) against the oracle.

Each linear is checked with the GPU's own bf16 input to it: a pass planned
over the linears up to and including that one is run, after which the
linear's input slot still holds what it read (later linears are not in the
plan) and its output slot what it wrote.  The oracle quantizes the matrix,
applies the rms scale where the linear reads a normalised input and bounds
every output (small stacks) or sampled rows (the 448-matrix recipe stack).
Runs are deterministic (K parts are added in a fixed order) and a captured
CUDA graph replays the same bits.
"""
import numpy as np
import pytest

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu

# a decoder-like layer at small sizes: (name, N, K, in slot, out slot); k, v
# and gate have ragged N (not read as another linear's input)
H, QD, FF = 512, 768, 1408
SMALL_LAYER = [("q", QD, H), ("k", 200, H), ("v", 136, H), ("o", H, QD), ("gate", 1400, H), ("up", FF, H),
               ("down", H, FF)]
S_H, S_Q, S_K, S_V, S_O, S_G, S_U, S_D = range(8)
SMALL_WIDTH = [H, QD, 200, 136, H, 1400, FF, H]


def _small_links(layers):
    out = []
    for layer in range(layers):
        h = S_H if layer == 0 else S_D
        out += [(h, S_Q, layer > 0), (h, S_K, layer > 0), (h, S_V, layer > 0), (S_Q, S_O, True),
                (S_O, S_G, True), (S_O, S_U, True), (S_U, S_D, True)]
    return out


def _build_small(mpw, torch, layers=3, seed=0, bits=None):
    rng = np.random.default_rng(seed)
    out, Ws = [], []
    links = _small_links(layers)
    for i, (si, so, nrm) in enumerate(links):
        name, N, K = SMALL_LAYER[i % 7]
        b = int(bits[i]) if bits is not None else int(rng.integers(4, 9))
        W = (0.02 * rng.standard_normal((N, K))).astype(np.float32)
        packed, scales = mpw.quantize_pack(torch.from_numpy(W).cuda(), b)
        mpw.repack(packed, K, b, "canonical", "paired", out=packed)
        out.append(mpw.Linear(packed, scales, N, K, b, si, so, nrm, layout="paired"))
        Ws.append(W)
    return out, Ws


def _slots(torch, widths, x0):
    slots = [torch.zeros((1, w), dtype=torch.bfloat16, device="cuda") for w in widths]
    slots[0].copy_(x0)
    return slots


def _check_link(L, W, x_in, y_out, rows=None):
    q, s = oracle.quantize(W if rows is None else W[rows], L.bits)
    if L.norm_input:
        y_ref, bound = oracle.qlinear_rms_ref(x_in, q, s)
    else:
        y_ref, bound = oracle.qlinear_ref(x_in, q, s)
    y = y_out if rows is None else y_out[:, rows]
    return oracle.check_qlinear(y, y_ref, bound)


def test_pass_small_stack_every_link_every_output():
    import torch

    import mixed_precision_weight_row_b200 as mpw

    layers, Ws = _build_small(mpw, torch, layers=3, seed=1)
    x0 = wl.gen_x(1, H, 11).cuda()
    for i, L in enumerate(layers):
        slots = _slots(torch, SMALL_WIDTH, x0)
        p = mpw.Pass(layers[: i + 1], slots, 1)
        p.run()
        torch.cuda.synchronize()
        x_in = slots[L.in_slot].float().cpu().numpy()
        y_out = slots[L.out_slot].float().cpu().numpy()
        p.close()
        ok = _check_link(L, Ws[i], x_in, y_out)
        assert ok.all(), f"link {i} ({SMALL_LAYER[i % 7][0]}, b={L.bits}): {(~ok).sum()} outputs out of bound"
    assert mpw.device_error() == 0


@pytest.mark.parametrize("b", [4, 5, 6, 7, 8])
def test_pass_each_width_alone(b):
    # one width for the whole stack, every output of every link
    import torch

    import mixed_precision_weight_row_b200 as mpw

    layers, Ws = _build_small(mpw, torch, layers=1, seed=20 + b, bits=[b] * 7)
    x0 = wl.gen_x(1, H, 30 + b).cuda()
    for i in (0, 3, 6):
        slots = _slots(torch, SMALL_WIDTH, x0)
        p = mpw.Pass(layers[: i + 1], slots, 1)
        p.run()
        torch.cuda.synchronize()
        ok = _check_link(layers[i], Ws[i], slots[layers[i].in_slot].float().cpu().numpy(),
                         slots[layers[i].out_slot].float().cpu().numpy())
        p.close()
        assert ok.all(), (b, i)
    assert mpw.device_error() == 0


def test_pass_deterministic_and_graph_replay():
    import torch

    import mixed_precision_weight_row_b200 as mpw

    layers, _ = _build_small(mpw, torch, layers=4, seed=3)
    x0 = wl.gen_x(1, H, 12).cuda()
    slots = _slots(torch, SMALL_WIDTH, x0)
    p = mpw.Pass(layers, slots, 1)
    info = p.info()
    assert info["grid"] >= 1 and 2 <= info["stages"] <= 8 and info["items"] >= len(layers)
    p.run()
    torch.cuda.synchronize()
    first = [s.clone() for s in slots]
    for _ in range(3):
        slots[0].copy_(x0)
        p.run()
    torch.cuda.synchronize()
    for a, c in zip(first, slots):
        assert torch.equal(a, c)
    # the same run captured in a CUDA graph
    for s in slots[1:]:
        s.zero_()
    slots[0].copy_(x0)
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        p.run(st)
    for s in slots[1:]:
        s.zero_()
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    for a, c in zip(first, slots):
        assert torch.equal(a, c)
    del g
    p.close()
    assert mpw.device_error() == 0


def test_pass_matches_per_linear_run():
    # the same stack through mpw_recipe_run: every slot within the decode
    # tolerance of the planned pass's (the fp32 sums differ in order only)
    import torch

    import mixed_precision_weight_row_b200 as mpw

    layers, Ws = _build_small(mpw, torch, layers=2, seed=5)
    x0 = wl.gen_x(1, H, 13).cuda()
    a = _slots(torch, SMALL_WIDTH, x0)
    b = _slots(torch, SMALL_WIDTH, x0)
    p = mpw.Pass(layers, a, 1)
    p.run()
    mpw.recipe_run(layers, b, 1)
    torch.cuda.synchronize()
    p.close()
    for i, (u, v) in enumerate(zip(a, b)):
        u, v = u.float(), v.float()
        tol = 2e-2 * float(v.abs().max()) + 1e-6
        assert float((u - v).abs().max()) <= tol, i


def test_pass_aliased_slots():
    # slots that are overlapping views of one buffer: the plan orders the
    # linears by the bytes they touch, not by slot index
    import torch

    import mixed_precision_weight_row_b200 as mpw

    rng = np.random.default_rng(8)
    buf = torch.zeros((4096,), dtype=torch.bfloat16, device="cuda")
    slots = [buf[0:512].view(1, 512), buf[512:1536].view(1, 1024), buf[1024:1536].view(1, 512),
             torch.zeros((1, 640), dtype=torch.bfloat16, device="cuda")]
    # slot 2 is the upper half of slot 1
    spec = [(1024, 512, 0, 1, False, 5), (640, 512, 2, 3, True, 6), (512, 640, 3, 0, True, 7),
            (512, 512, 0, 2, True, 4)]
    layers, Ws = [], []
    for N, K, si, so, nrm, b in spec:
        W = (0.02 * rng.standard_normal((N, K))).astype(np.float32)
        packed, scales = mpw.quantize_pack(torch.from_numpy(W).cuda(), b)
        mpw.repack(packed, K, b, "canonical", "paired", out=packed)
        layers.append(mpw.Linear(packed, scales, N, K, b, si, so, nrm, layout="paired"))
        Ws.append(W)
    x0 = wl.gen_x(1, 512, 14).cuda()
    for i, L in enumerate(layers):
        buf.zero_()
        slots[3].zero_()
        slots[0].copy_(x0)
        p = mpw.Pass(layers[: i + 1], slots, 1)
        p.run()
        torch.cuda.synchronize()
        ok = _check_link(L, Ws[i], slots[L.in_slot].float().cpu().numpy(), slots[L.out_slot].float().cpu().numpy())
        p.close()
        assert ok.all(), i
    # a linear whose input and output overlap is refused
    bad = [mpw.Linear(layers[0].packed, layers[0].scales, 1024, 512, 5, 0, 0, False, layout="paired")]
    with pytest.raises(mpw.MPWError):
        mpw.Pass(bad, slots, 1)


def test_pass_unsupported():
    import torch

    import mixed_precision_weight_row_b200 as mpw

    layers, _ = _build_small(mpw, torch, layers=1, seed=6, bits=[5] * 7)
    slots = _slots(torch, SMALL_WIDTH, wl.gen_x(1, H, 1).cuda())
    with pytest.raises(mpw.MPWError) as e:
        mpw.Pass(layers, [torch.zeros((2, w), dtype=torch.bfloat16, device="cuda") for w in SMALL_WIDTH], 2)
    assert e.value.status == mpw.MPW_E_UNSUPPORTED
    # a 9-bit linear, and a canonical one
    W = (0.02 * np.random.default_rng(0).standard_normal((QD, H))).astype(np.float32)
    for b, layout in ((9, "paired"), (6, "canonical")):
        packed, scales = mpw.quantize_pack(torch.from_numpy(W).cuda(), b)
        if layout == "paired":
            mpw.repack(packed, H, b, "canonical", "paired", out=packed)
        odd = [mpw.Linear(packed, scales, QD, H, b, S_H, S_Q, False, layout=layout)]
        with pytest.raises(mpw.MPWError) as e:
            mpw.Pass(odd, slots, 1)
        assert e.value.status == mpw.MPW_E_UNSUPPORTED


@pytest.fixture(scope="module")
def recipe_stack():
    import torch

    import mixed_precision_weight_row_b200 as mpw

    shapes, bits, links = wl.recipe_shapes(), wl.recipe_bits(), wl.recipe_links()
    layers = []
    for i, ((layer, name, N, K), b, (si, so, nrm)) in enumerate(zip(shapes, bits, links)):
        W = wl.gen_weight_torch(N, K, wl.RECIPE["sigma"], wl.recipe_weight_seed(i))
        packed, scales = mpw.quantize_pack(W, b)
        del W
        mpw.repack(packed, K, b, "canonical", "paired", out=packed)
        layers.append(mpw.Linear(packed, scales, N, K, b, si, so, nrm, layout="paired"))
    torch.cuda.synchronize()
    yield mpw, layers, shapes, bits
    del layers
    torch.cuda.empty_cache()


def test_pass_recipe_stack_sampled_links(recipe_stack):
    # the 448-matrix recipe stack (paired rows, the layout the benchmark
    # times): sampled links, each with its own GPU input, on sampled rows
    import torch

    mpw, layers, shapes, bits = recipe_stack
    x0 = wl.gen_x(1, 5120, wl.RECIPE["x_seed"]).cuda()
    rng = np.random.default_rng(77)
    check = sorted(set(range(7)) | {447} | set(rng.choice(448, 10, replace=False).tolist()))
    for i in check:
        slots = [torch.zeros((1, wl.SLOT_WIDTH[s]), dtype=torch.bfloat16, device="cuda") for s in range(8)]
        slots[wl.SLOT_H].copy_(x0)
        p = mpw.Pass(layers[: i + 1], slots, 1)
        p.run()
        torch.cuda.synchronize()
        L = layers[i]
        x_in = slots[L.in_slot].float().cpu().numpy()
        y_out = slots[L.out_slot].float().cpu().numpy()
        p.close()
        (_, name, N, K), b = shapes[i], bits[i]
        W = wl.gen_weight_torch(N, K, wl.RECIPE["sigma"], wl.recipe_weight_seed(i))
        rows = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(i).choice(N, 30, replace=False)]))
        W_rows = W[torch.from_numpy(rows).cuda()].cpu().numpy()
        del W
        q, s = oracle.quantize(W_rows, b)
        if L.norm_input:
            y_ref, bound = oracle.qlinear_rms_ref(x_in, q, s)
        else:
            y_ref, bound = oracle.qlinear_ref(x_in, q, s)
        ok = oracle.check_qlinear(y_out[:, rows], y_ref, bound)
        assert ok.all(), f"link {i} ({name}, b={b}): {(~ok).sum()} outputs out of bound"
    # the whole pass: finite, non-degenerate, and error word clear
    slots = [torch.zeros((1, wl.SLOT_WIDTH[s]), dtype=torch.bfloat16, device="cuda") for s in range(8)]
    slots[wl.SLOT_H].copy_(x0)
    p = mpw.Pass(layers, slots, 1)
    p.run()
    torch.cuda.synchronize()
    p.close()
    d = slots[wl.SLOT_D].float()
    assert torch.isfinite(d).all() and float(d.abs().max()) > 0
    assert mpw.device_error() == 0
