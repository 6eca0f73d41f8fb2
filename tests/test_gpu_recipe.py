"""The mixed-bit recipe decode pass (448 chained linears, M = 1) against the
oracle, at full size.

Every linear is checked against the oracle with the GPU's own bf16 input to
that link (so errors do not compound along the chain): the oracle normalises
that input itself where the link reads the rms-scaled input, quantizes a seeded sample of the
matrix's rows and bounds the sampled outputs.  The whole pass issued as one
mpw_recipe_run call must equal the link-by-link run bit for bit.  Both
packed layouts are run at full size: the canonical rows and the paired
halves the benchmark times.
"""
import numpy as np
import pytest

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", params=["paired", "canonical"])
def stack(request):
    """The 448-matrix stack in the layout under test (paired: the layout the
    benchmark times, re-ordered in place after quantization)."""
    import torch

    import mixed_precision_weight_row_b200 as mpw

    layout = request.param

    shapes = wl.recipe_shapes()
    bits = wl.recipe_bits()
    links = wl.recipe_links()
    layers = []
    for i, ((layer, name, N, K), b, (si, so, nrm)) in enumerate(zip(shapes, bits, links)):
        W = wl.gen_weight_torch(N, K, wl.RECIPE["sigma"], wl.recipe_weight_seed(i))
        packed, scales = mpw.quantize_pack(W, b)
        del W
        if layout != "canonical":
            mpw.repack(packed, K, b, "canonical", layout, out=packed)
        layers.append(mpw.Linear(packed, scales, N, K, b, si, so, nrm, layout=layout))
    torch.cuda.synchronize()
    yield mpw, layers, shapes, bits
    del layers
    torch.cuda.empty_cache()


def _slots(torch):
    return [torch.zeros((1, wl.SLOT_WIDTH[s]), dtype=torch.bfloat16, device="cuda") for s in range(8)]


def test_recipe_bit_multiset(stack):
    _, _, shapes, bits = stack
    assert len(shapes) == 448 and len(bits) == 448
    assert sorted(set(bits)) == [5, 6, 7, 8]
    assert bits.count(6) == 283 and bits.count(5) == 98 and bits.count(7) + bits.count(8) == 67
    params = sum(n * k for _, _, n, k in shapes)
    assert params == 64 * 340_787_200
    # mean bits over weights, not over matrices
    mean_bits = sum(n * k * b for (_, _, n, k), b in zip(shapes, bits)) / params
    assert 5.5 < mean_bits < 6.6


def test_recipe_chain_links_and_whole_pass(stack):
    import torch

    mpw, layers, shapes, bits = stack
    x0 = wl.gen_x(1, 5120, wl.RECIPE["x_seed"]).cuda()
    # link by link, keeping the input and output of sampled links
    slots = _slots(torch)
    slots[wl.SLOT_H].copy_(x0)
    rng = np.random.default_rng(99)
    check = set(range(7)) | set(range(441, 448)) | set(rng.choice(448, 20, replace=False).tolist())
    kept = {}
    for i, L in enumerate(layers):
        if i in check:
            kept[i] = slots[L.in_slot].float().cpu().numpy().copy()
        mpw.recipe_run([L], slots, 1)
        if i in check:
            kept[i] = (kept[i], slots[L.out_slot].float().cpu().numpy().copy())
    torch.cuda.synchronize()
    final = [s.clone() for s in slots]
    # the whole pass in one call gives the same bits
    slots2 = _slots(torch)
    slots2[wl.SLOT_H].copy_(x0)
    mpw.recipe_run(layers, slots2, 1)
    torch.cuda.synchronize()
    for a, b in zip(final, slots2):
        assert torch.equal(a, b)
    # the chain stays finite and non-degenerate
    d = final[wl.SLOT_D].float()
    assert torch.isfinite(d).all() and float(d.abs().max()) > 0
    # per-link parity on sampled rows
    for i in sorted(check):
        x_in, y_out = kept[i]
        (_, name, N, K), b = shapes[i], bits[i]
        L = layers[i]
        x_used = x_in * oracle.rms_scale(x_in) if L.norm_input else x_in
        W = wl.gen_weight_torch(N, K, wl.RECIPE["sigma"], wl.recipe_weight_seed(i))
        rows = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(i).choice(N, 30, replace=False)]))
        W_rows = W[torch.from_numpy(rows).cuda()].cpu().numpy()
        del W
        q, s = oracle.quantize(W_rows, b)
        y_ref, bound = oracle.qlinear_ref(x_used, q, s)
        ok = oracle.check_qlinear(y_out[:, rows], y_ref, bound)
        assert ok.all(), f"link {i} ({name}, b={b}): {(~ok).sum()} outputs out of bound"


def test_recipe_small_stack_every_output(stack):
    # a 3-link chain on small matrices where the oracle recomputes every output
    import torch

    mpw = stack[0]
    rng = np.random.default_rng(4)
    dims = [(96, 64), (80, 96), (64, 80)]          # (N, K) per link
    Ws, links = [], []
    for j, ((N, K), b) in enumerate(zip(dims, (5, 9, 13))):
        W = rng.standard_normal((N, K)).astype(np.float32)
        packed, scales = mpw.quantize_pack(torch.from_numpy(W).cuda(), b)
        links.append(mpw.Linear(packed, scales, N, K, b, j, j + 1, j > 0))
        Ws.append((W, b))
    for M in (1, 3, 32):
        x = wl.gen_x(M, 64, 5 + M)
        slots = [x.cuda()] + [torch.zeros((M, n), dtype=torch.bfloat16, device="cuda") for n, _ in dims]
        mpw.recipe_run(links, slots, M)
        torch.cuda.synchronize()
        for j, L in enumerate(links):
            W, b = Ws[j]
            q, s = oracle.quantize(W, b)
            xin = slots[j].float().cpu().numpy()
            if L.norm_input:
                y_ref, bound = oracle.qlinear_rms_ref(xin, q, s)
            else:
                y_ref, bound = oracle.qlinear_ref(xin, q, s)
            assert oracle.check_qlinear(slots[j + 1].float().cpu().numpy(), y_ref, bound).all(), (M, j)
