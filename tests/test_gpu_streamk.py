"""The stream-K decode kernel (work split evenly over a persistent grid, split
tiles combined through the caller's workspace).

* Outputs meet the bound against the oracle on shapes whose tiles are split
  between CTAs (few rows, long rows, one tile, one chunk), both layouts.
* Results are bit-identical from call to call (the combine order is fixed)
  and identical to the per-tile kernel's within the bound.
* The workspace comes back with its counters at zero: a second call on the
  same workspace, with a different shape, is still correct.
* The C ABI rejects a workspace that is misaligned or too small.
"""
import ctypes

import numpy as np
import pytest

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mpw():
    import mixed_precision_weight_row_b200 as m

    return m


def _t():
    import torch

    return torch


SHAPES = [(16, 128), (16, 4096), (1024, 5120), (40, 17408), (100, 2048), (3000, 384), (4096, 4096)]


def _run(mpw, W, x, b, layout, use_workspace=True):  # stream-K unless told otherwise
    torch = _t()
    q, s = oracle.quantize(W, b)
    packed = oracle.pack_paired(q, b) if layout == "paired" else oracle.pack(q, b)
    y = mpw.qlinear(x.cuda(), torch.from_numpy(packed).cuda(), torch.from_numpy(s).cuda(), b, layout=layout,
                    use_workspace=use_workspace)
    torch.cuda.synchronize()
    return y, q, s


@pytest.mark.parametrize("b", [4, 5, 6, 8, 11, 15])
@pytest.mark.parametrize("layout", ["paired", "canonical"])
@pytest.mark.parametrize("M", [1, 3, 8, 9, 17, 32])
def test_streamk_matches_oracle(mpw, b, layout, M):
    rng = np.random.default_rng(9000 + 10 * b + M)
    for N, K in SHAPES[:6]:
        W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)
        W[min(3, N - 1)] = 0
        x = workloads.gen_x(M, K, seed=N + K + M)
        y, q, s = _run(mpw, W, x, b, layout)
        y_ref, bound = oracle.qlinear_ref(x.float().numpy(), q, s)
        ok = oracle.check_qlinear(y.float().cpu().numpy(), y_ref, bound)
        assert ok.all(), f"{N}x{K}: {(~ok).sum()} outputs out of bound"


def test_streamk_is_deterministic_and_agrees_with_per_tile_kernel(mpw):
    torch = _t()
    rng = np.random.default_rng(9100)
    for N, K in [(1024, 5120), (4096, 4096), (40, 17408)]:
        W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)
        x = workloads.gen_x(1, K, seed=K)
        y1, q, s = _run(mpw, W, x, 6, "paired")
        y2, _, _ = _run(mpw, W, x, 6, "paired")
        assert torch.equal(y1.view(torch.int16), y2.view(torch.int16)), "stream-K result changed between calls"
        y3, _, _ = _run(mpw, W, x, 6, "paired", use_workspace=False)
        y_ref, bound = oracle.qlinear_ref(x.float().numpy(), q, s)
        assert oracle.check_qlinear(y3.float().cpu().numpy(), y_ref, bound).all()


def test_workspace_is_left_ready_for_the_next_call(mpw):
    # one explicit workspace reused by calls of different shapes: each call
    # must find the counters at zero
    torch = _t()
    rng = np.random.default_rng(9200)
    shapes = [(1024, 5120, 6), (40, 17408, 5), (1024, 5120, 8), (3000, 384, 4)]
    need = max(mpw.qlinear_workspace_bytes(b, 4, n, k, "paired") for n, k, b in shapes)
    assert need > 0
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for rep in range(2):
        for N, K, b in shapes:
            W = rng.standard_normal((N, K)).astype(np.float32)
            q, s = oracle.quantize(W, b)
            packed = torch.from_numpy(oracle.pack_paired(q, b)).cuda()
            x = workloads.gen_x(4, K, seed=N + rep).cuda()
            y = torch.empty((4, N), dtype=torch.bfloat16, device="cuda")
            st = mpw.lib.mpw_qlinear_ws(x.data_ptr(), packed.data_ptr(), torch.from_numpy(s).cuda().data_ptr(), b,
                                        1, 4, N, K, y.data_ptr(), 0, ws.data_ptr(), need,
                                        torch.cuda.current_stream().cuda_stream)
            assert st == 0
            torch.cuda.synchronize()
            y_ref, bound = oracle.qlinear_ref(x.float().cpu().numpy(), q, s)
            assert oracle.check_qlinear(y.float().cpu().numpy(), y_ref, bound).all(), (rep, N, K, b)


def test_workspace_validation(mpw):
    torch = _t()
    N, K, b = 1024, 5120, 6
    need = mpw.qlinear_workspace_bytes(b, 1, N, K, "paired")
    assert need > 0
    ws = torch.zeros(need + 64, dtype=torch.uint8, device="cuda")
    x = torch.zeros((1, K), dtype=torch.bfloat16, device="cuda")
    packed = torch.zeros((N, mpw.packed_row_bytes(K, b)), dtype=torch.uint8, device="cuda")
    scales = torch.ones(N, dtype=torch.float32, device="cuda")
    y = torch.empty((1, N), dtype=torch.bfloat16, device="cuda")
    call = lambda ptr, nbytes: mpw.lib.mpw_qlinear_ws(x.data_ptr(), packed.data_ptr(), scales.data_ptr(), b, 1, 1,
                                                      N, K, y.data_ptr(), 0, ptr, nbytes, 0)
    assert call(ws.data_ptr() + 4, need) == mpw.MPW_E_MISALIGNED
    assert call(ws.data_ptr(), need - 16) == mpw.MPW_E_INVALID_ARG
    assert call(ws.data_ptr(), need) == mpw.MPW_OK
    assert call(None, 0) == mpw.MPW_OK
    torch.cuda.synchronize()
    assert mpw.device_error() == 0


def test_streamk_recipe_with_norm_links(mpw):
    # a chain whose later links read the rms-scaled input (the sum of squares
    # is combined across split tiles too)
    torch = _t()
    rng = np.random.default_rng(9300)
    dims = [(64, 4096), (1024, 64), (40, 1024)]          # (N, K): split tiles in every link
    bits = [6, 5, 8]
    M = 3
    bufs = [torch.zeros(M * 4096, dtype=torch.bfloat16, device="cuda") for _ in range(4)]
    x0 = workloads.gen_x(M, 4096, seed=93)
    views = [bufs[0][: M * 4096].view(M, 4096)]
    for i, (N, K) in enumerate(dims):
        views.append(bufs[i + 1][: M * N].view(M, N))
    views[0].copy_(x0.cuda())
    layers, refs = [], []
    for i, ((N, K), b) in enumerate(zip(dims, bits)):
        W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.05)
        q, s = oracle.quantize(W, b)
        refs.append((q, s))
        layers.append(mpw.Linear(torch.from_numpy(oracle.pack_paired(q, b)).cuda(), torch.from_numpy(s).cuda(),
                                 N, K, b, i, i + 1, i > 0, layout="paired"))
    mpw.recipe_run(layers, views, M, use_workspace=True)
    torch.cuda.synchronize()
    for i, (q, s) in enumerate(refs):
        x_in = views[i].float().cpu().numpy()
        y = views[i + 1].float().cpu().numpy()
        y_ref, bound = (oracle.qlinear_ref if i == 0 else oracle.qlinear_rms_ref)(x_in, q, s)
        assert oracle.check_qlinear(y, y_ref, bound).all(), f"link {i}"
    assert mpw.device_error() == 0
