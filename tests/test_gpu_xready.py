"""MPW_QLINEAR_X_READY on the GPU.

* A flagged call gives the same bytes as the unflagged one: the flag moves
  the loads of x ahead of the wait on the preceding launch and changes no
  arithmetic.
* Ordering, within the flag's contract (x written before the launch that
  precedes the run of flagged calls): A writes ya, B runs unflagged, then C
  (reading ya) and D (reading A's input) run flagged.  In eager launches and
  in a replayed CUDA graph, with fresh inputs every iteration so that a stale
  read would show, every output meets the oracle's bound
  |y - y_ref| <= 8e-3 * sum_k |x w_hat| + 1e-6, and the ys written by a run
  of flagged calls land in call order (the last write to a shared y wins).
"""
import numpy as np
import pytest

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mpw():
    import mixed_precision_weight_row_b200 as m

    return m


def _matrix(mpw, rng, N, K, b, layout, n_rows=None):
    """Packed on the GPU (quantize_pack, then repack), which other tests pin
    to the oracle byte for byte; the oracle quantizes the checked rows (all,
    or a seeded sample of n_rows) and its scales must equal the GPU's."""
    import torch

    W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)
    packed, scales = mpw.quantize_pack(torch.from_numpy(W).cuda(), b)
    if layout == "paired":
        mpw.repack(packed, K, b, "canonical", "paired", out=packed)
    rows = np.arange(N) if n_rows is None else np.unique(np.r_[0, N - 1, rng.choice(N, n_rows, replace=False)])
    q, s = oracle.quantize(W[rows], b)
    assert np.array_equal(scales.cpu().numpy()[rows].view(np.uint32), s.view(np.uint32))
    return q, s, packed, scales, rows


@pytest.mark.parametrize("layout", ["paired", "canonical"])
@pytest.mark.parametrize("b", [4, 6, 8, 12])
def test_flag_changes_no_result(mpw, layout, b):
    import torch

    rng = np.random.default_rng(700 + b)
    for N, K, M in [(4096, 4096, 1), (1000, 5120, 3), (17, 2048, 8), (300, 1024, 16), (64, 512, 40)]:
        q, s, packed, scales, rows = _matrix(mpw, rng, N, K, b, layout, n_rows=min(N - 2, 200))
        x = workloads.gen_x(M, K, seed=N + M).cuda()
        y0 = mpw.qlinear(x, packed, scales, b, layout=layout)
        y1 = mpw.qlinear(x, packed, scales, b, layout=layout, x_ready=True)
        torch.cuda.synchronize()
        assert torch.equal(y0.view(torch.int16), y1.view(torch.int16)), (N, K, M)
        y_ref, bound = oracle.qlinear_ref(x.float().cpu().numpy(), q, s)
        assert oracle.check_qlinear(y1.float().cpu().numpy()[:, rows], y_ref, bound).all(), (N, K, M)
    assert mpw.device_error() == 0


def _round(mpw, mats, x0, ya, yb, yc, yd, layout):
    """A: ya = W_A x0 and B: yb = W_B x0, unflagged (x0 is written just
    before A); C: yc = W_C ya and D: yd = W_D x0, flagged (their inputs were
    written before B, the launch preceding their run)."""
    (_, _, pa, sa, ba, _), (_, _, pb, sb, bb, _), (_, _, pc, sc, bc, _), (_, _, pd, sd, bd, _) = mats
    mpw.qlinear(x0, pa, sa, ba, y=ya, layout=layout)
    mpw.qlinear(x0, pb, sb, bb, y=yb, layout=layout)
    mpw.qlinear(ya, pc, sc, bc, y=yc, layout=layout, x_ready=True)
    mpw.qlinear(x0, pd, sd, bd, y=yd, layout=layout, x_ready=True)


def _check_round(mats, x_in, ya, yb, yc, yd):
    """Every output row is checked for A (it is C's input); the others on the
    sampled rows kept with their matrices (a stale input moves all rows)."""
    xin = x_in.float().cpu().numpy()
    a = ya.float().cpu().numpy()
    for (q, s, _, _, _, rows), got, xx in zip(mats, (a, yb.float().cpu().numpy(), yc.float().cpu().numpy(),
                                                     yd.float().cpu().numpy()), (xin, xin, a, xin)):
        y_ref, bound = oracle.qlinear_ref(xx, q, s)
        assert oracle.check_qlinear(got[:, rows], y_ref, bound).all()


@pytest.mark.parametrize("layout", ["paired", "canonical"])
def test_flagged_run_sees_inputs_written_before_it(mpw, layout):
    import torch

    rng = np.random.default_rng(4242)
    # A (a q-sized projection) writes C's input; B and D are small projections
    mats = []
    for i, (N, K, b) in enumerate([(6144, 5120, 6), (1024, 5120, 5), (5120, 6144, 8), (1024, 5120, 7)]):
        q, s, p, sc, rows = _matrix(mpw, rng, N, K, b, layout, n_rows=None if i == 0 else 254)
        mats.append((q, s, p, sc, b, rows))
    x0 = torch.empty((1, 5120), dtype=torch.bfloat16, device="cuda")
    ya = torch.empty((1, 6144), dtype=torch.bfloat16, device="cuda")
    yb = torch.empty((1, 1024), dtype=torch.bfloat16, device="cuda")
    yc = torch.empty((1, 5120), dtype=torch.bfloat16, device="cuda")
    yd = torch.empty((1, 1024), dtype=torch.bfloat16, device="cuda")
    # eager rounds with fresh inputs; the output of A is cleared first so
    # that a read of it before A finished would see zeros
    for r in range(12):
        x_in = workloads.gen_x(1, 5120, seed=900 + r).cuda()
        ya.zero_()
        x0.copy_(x_in)
        _round(mpw, mats, x0, ya, yb, yc, yd, layout)
        torch.cuda.synchronize()
        _check_round(mats, x_in, ya, yb, yc, yd)
    # the same launches captured once and replayed
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        x0.zero_()
        _round(mpw, mats, x0, ya, yb, yc, yd, layout)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            ya.zero_()
            _round(mpw, mats, x0, ya, yb, yc, yd, layout)
    torch.cuda.current_stream().wait_stream(s)
    for r in range(12):
        x_in = workloads.gen_x(1, 5120, seed=950 + r).cuda()
        x0.copy_(x_in)
        g.replay()
        torch.cuda.synchronize()
        _check_round(mats, x_in, ya, yb, yc, yd)
    del g
    assert mpw.device_error() == 0


def test_flagged_run_writes_y_in_call_order(mpw):
    """A run of flagged calls into one y: the last call's result stays."""
    import torch

    rng = np.random.default_rng(77)
    mats = [_matrix(mpw, rng, 4096, 4096, b, "paired", n_rows=200) for b in (4, 6, 8, 5, 7, 6)]
    x = workloads.gen_x(1, 4096, seed=5).cuda()
    y = torch.empty((1, 4096), dtype=torch.bfloat16, device="cuda")
    for rnd in range(20):
        order = rng.permutation(len(mats))
        for i in order:
            q, s, p, sc, rows = mats[i]
            mpw.qlinear(x, p, sc, (4, 6, 8, 5, 7, 6)[i], y=y, layout="paired", x_ready=True)
        torch.cuda.synchronize()
        q, s, p, sc, rows = mats[order[-1]]
        y_ref, bound = oracle.qlinear_ref(x.float().cpu().numpy(), q, s)
        assert oracle.check_qlinear(y.float().cpu().numpy()[:, rows], y_ref, bound).all(), rnd
    assert mpw.device_error() == 0


@pytest.mark.parametrize("norm", [False, True])
def test_recipe_run_with_aliased_slots(mpw, norm):
    """The recipe runner flags a linear only when its input bytes were not
    written by the current run (nor the linear before it); slot 3 is a view
    of slot 1's buffer, so the third linear must wait for the second."""
    import torch

    rng = np.random.default_rng(31 + norm)
    K0, N1, N2 = 2048, 3072, 1024
    mats = [_matrix(mpw, rng, N, K, b, "paired", n_rows=None) for N, K, b in
            [(N1, K0, 6), (N1, K0, 5), (N2, N1, 7)]]
    big = torch.zeros((2, N1), dtype=torch.bfloat16, device="cuda")
    slots = [torch.empty((1, K0), dtype=torch.bfloat16, device="cuda"),
             big[0:1],
             torch.empty((1, N1), dtype=torch.bfloat16, device="cuda"),
             big[0:1],
             torch.empty((1, N2), dtype=torch.bfloat16, device="cuda")]
    links = [(0, 2), (0, 1), (3, 4)]
    layers = [mpw.Linear(p, sc, p.shape[0], K, b, si, so, norm and i > 0, layout="paired")
              for i, ((q, s, p, sc, rows), (N, K, b), (si, so)) in
              enumerate(zip(mats, [(N1, K0, 6), (N1, K0, 5), (N2, N1, 7)], links))]
    for r in range(10):
        x_in = workloads.gen_x(1, K0, seed=300 + r).cuda()
        big.zero_()
        slots[0].copy_(x_in)
        mpw.recipe_run(layers, slots, 1)
        torch.cuda.synchronize()
        xin = x_in.float().cpu().numpy()
        y1 = slots[1].float().cpu().numpy()
        for (q, s, _, _, _), x, got, nrm in ((mats[0], xin, slots[2], False), (mats[1], xin, slots[1], norm),
                                            (mats[2], y1, slots[4], norm)):
            y_ref, bound = (oracle.qlinear_rms_ref if nrm else oracle.qlinear_ref)(x, q, s)
            assert oracle.check_qlinear(got.float().cpu().numpy(), y_ref, bound).all(), r
    assert mpw.device_error() == 0


@pytest.mark.parametrize("layout", ["paired", "canonical"])
def test_unshared_outputs_then_an_unflagged_reader(mpw, layout):
    """A and E unflagged; B and C flagged x_ready + y_unshared (inputs written
    before E, distinct outputs), so they write y without waiting; F,
    unflagged, reads B's output and must see it complete."""
    import torch

    rng = np.random.default_rng(515)
    K0, NA = 5120, 6144
    shapes = [(NA, K0, 6), (1024, K0, 5), (4096, NA, 8), (4096, K0, 7), (2048, 4096, 6)]
    mats = [_matrix(mpw, rng, N, K, b, layout, n_rows=None if i == 0 else 254) for i, (N, K, b) in
            enumerate(shapes)]
    x0 = torch.empty((1, K0), dtype=torch.bfloat16, device="cuda")
    ys = [torch.empty((1, N), dtype=torch.bfloat16, device="cuda") for N, _, _ in shapes]
    yf = torch.empty((1, 2048), dtype=torch.bfloat16, device="cuda")

    def launch():
        (_, _, pa, sa, _), (_, _, pe, se, _), (_, _, pb, sb, _), (_, _, pc, sc, _), (_, _, pf, sf, _) = mats
        mpw.qlinear(x0, pa, sa, 6, y=ys[0], layout=layout)                                  # A
        mpw.qlinear(x0, pe, se, 5, y=ys[1], layout=layout)                                  # E
        mpw.qlinear(ys[0], pb, sb, 8, y=ys[2], layout=layout, x_ready=True, y_unshared=True)  # B
        mpw.qlinear(x0, pc, sc, 7, y=ys[3], layout=layout, x_ready=True, y_unshared=True)     # C
        mpw.qlinear(ys[2][:, :4096], pf, sf, 6, y=yf, layout=layout)                        # F

    def check(x_in):
        xin = x_in.float().cpu().numpy()
        a = ys[0].float().cpu().numpy()
        bout = ys[2].float().cpu().numpy()
        for (q, s, _, _, rows), got, xx in zip(mats, (a, ys[1], ys[2], ys[3], yf),
                                               (xin, xin, a, xin, bout)):
            g = got if isinstance(got, np.ndarray) else got.float().cpu().numpy()
            y_ref, bound = oracle.qlinear_ref(xx, q, s)
            assert oracle.check_qlinear(g[:, rows], y_ref, bound).all()

    for r in range(10):
        x_in = workloads.gen_x(1, K0, seed=600 + r).cuda()
        for t in ys:
            t.zero_()
        x0.copy_(x_in)
        launch()
        torch.cuda.synchronize()
        check(x_in)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        launch()
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            ys[2].zero_()
            launch()
    torch.cuda.current_stream().wait_stream(s)
    for r in range(10):
        x_in = workloads.gen_x(1, K0, seed=650 + r).cuda()
        x0.copy_(x_in)
        g.replay()
        torch.cuda.synchronize()
        check(x_in)
    del g
    assert mpw.device_error() == 0
