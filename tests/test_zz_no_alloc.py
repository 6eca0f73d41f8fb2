"""mpw_qlinear_noalloc: the decode linear for callers that cannot allocate
device memory (it takes its workspace from a fixed array in the library).

Collected last on purpose.  Each check calls the entry point through the C
ABI twice in a row and compares it with the existing entry point
(mpw_qlinear_ex) and with the oracle, within the bound every decode test
uses: |y - y_ref| <= 8e-3 * sum_k |x w_hat| + 1e-6.  Nothing here depends on
what ran before, so the file passes alone or after the rest of the suite.

Calls queued back to back on one stream, with no synchronisation between
them, check that each call's clearing of the shared array lands after the
previous call's kernel is done with it.
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


def _call_noalloc(mpw, x, packed, scales, b, layout, y):
    import torch

    M, K = x.shape
    N = packed.shape[0]
    return mpw.lib.mpw_qlinear_noalloc(x.data_ptr(), packed.data_ptr(), scales.data_ptr(), b,
                                       mpw.LAYOUTS[layout], M, N, K, y.data_ptr(),
                                       torch.cuda.current_stream().cuda_stream)


def _call_existing(mpw, x, packed, scales, b, layout, y):
    import torch

    M, K = x.shape
    N = packed.shape[0]
    return mpw.lib.mpw_qlinear_ex(x.data_ptr(), packed.data_ptr(), scales.data_ptr(), b, mpw.LAYOUTS[layout],
                                  M, N, K, y.data_ptr(), 0, torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("layout", ["paired", "canonical"])
def test_noalloc_matches_existing_entry_point_two_calls_in_a_row(mpw, layout):
    import torch

    rng = np.random.default_rng(1234)
    # split tiles (few rows, long rows) and whole tiles; M of 1 and 5
    for (N, K, b, M) in [(1024, 5120, 6, 1), (40, 17408, 5, 5), (4096, 4096, 8, 1)]:
        W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)
        q, s = oracle.quantize(W, b)
        packed = torch.from_numpy(oracle.pack_paired(q, b) if layout == "paired" else oracle.pack(q, b)).cuda()
        scales = torch.from_numpy(s).cuda()
        y_ex = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        for call in range(2):
            x = workloads.gen_x(M, K, seed=10 * N + call).cuda()
            y_na = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
            assert _call_noalloc(mpw, x, packed, scales, b, layout, y_na) == mpw.MPW_OK
            assert _call_existing(mpw, x, packed, scales, b, layout, y_ex) == mpw.MPW_OK
            torch.cuda.synchronize()
            y_ref, bound = oracle.qlinear_ref(x.float().cpu().numpy(), q, s)
            a = y_na.float().cpu().numpy()
            e = y_ex.float().cpu().numpy()
            assert oracle.check_qlinear(a, y_ref, bound).all(), (N, K, b, call)
            # both within the bound of the exact value, hence within twice it of each other
            assert (np.abs(a - e) <= 2 * bound).all()
    assert mpw.device_error() == 0


def test_noalloc_rejects_what_its_scratch_cannot_hold(mpw):
    import torch

    # nothing is launched when the limit is exceeded, so small dummy buffers do
    x = torch.zeros((1, 64), dtype=torch.bfloat16, device="cuda")
    packed = torch.zeros((16, 64), dtype=torch.uint8, device="cuda")
    scales = torch.ones(16, dtype=torch.float32, device="cuda")
    y = torch.empty((1, 16), dtype=torch.bfloat16, device="cuda")
    N_huge = 16 * 70000                       # more tiles than the scratch keeps counters for
    st = mpw.lib.mpw_qlinear_noalloc(x.data_ptr(), packed.data_ptr(), scales.data_ptr(), 6, 0, 1, N_huge, 64,
                                     y.data_ptr(), 0)
    assert st == mpw.MPW_E_SCRATCH_LIMIT
    assert "scratch" in mpw.status_str(st)
    # M beyond the decode range and misaligned x are argument errors
    assert mpw.lib.mpw_qlinear_noalloc(x.data_ptr(), packed.data_ptr(), scales.data_ptr(), 6, 0, 33, 16, 64,
                                       y.data_ptr(), 0) == mpw.MPW_E_INVALID_ARG
    assert mpw.lib.mpw_qlinear_noalloc(x.data_ptr() + 2, packed.data_ptr(), scales.data_ptr(), 6, 0, 1, 16, 64,
                                       y.data_ptr(), 0) == mpw.MPW_E_MISALIGNED


@pytest.mark.parametrize("layout", ["paired", "canonical"])
def test_noalloc_calls_queued_back_to_back(mpw, layout):
    """Three calls on one stream (different x, separate outputs), one sync at
    the end, on shapes with split tiles; M of 12 and 32 take the two- and
    four-tile-wide kernels."""
    import torch

    rng = np.random.default_rng(4321)
    for (N, K, b, M) in [(40, 17408, 5, 12), (40, 17408, 6, 32), (1024, 5120, 8, 32), (100, 2048, 11, 12)]:
        W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)
        q, s = oracle.quantize(W, b)
        packed = torch.from_numpy(oracle.pack_paired(q, b) if layout == "paired" else oracle.pack(q, b)).cuda()
        scales = torch.from_numpy(s).cuda()
        xs = [workloads.gen_x(M, K, seed=77 * N + call).cuda() for call in range(3)]
        ys = [torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda") for _ in range(3)]
        ye = [torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
        for x, y in zip(xs, ys):
            assert _call_noalloc(mpw, x, packed, scales, b, layout, y) == mpw.MPW_OK
        for x, y in zip(xs, ye):
            assert _call_existing(mpw, x, packed, scales, b, layout, y) == mpw.MPW_OK
        torch.cuda.synchronize()
        for x, y, e in zip(xs, ys, ye):
            y_ref, bound = oracle.qlinear_ref(x.float().cpu().numpy(), q, s)
            a = y.float().cpu().numpy()
            assert oracle.check_qlinear(a, y_ref, bound).all(), (N, K, b, M)
            assert (np.abs(a - e.float().cpu().numpy()) <= 2 * bound).all()
    assert mpw.device_error() == 0


def test_noalloc_limit_agrees_with_workspace_size(mpw):
    """On the 27B-class MLP shapes, the call is refused exactly when the
    workspace it needs (mpw_qlinear_workspace_bytes) exceeds the array.  The
    buffers have their full sizes (zero weights, zero x), so a call that does
    run reads only what it owns and writes zeros."""
    import torch

    limit = 4 << 20
    refused = 0
    for (N, K) in [(17408, 5120), (5120, 17408)]:
        for b in (5, 6):
            rb = mpw.packed_row_bytes(K, b)
            packed = torch.zeros((N, rb), dtype=torch.uint8, device="cuda")
            scales = torch.ones(N, dtype=torch.float32, device="cuda")
            for M in (1, 8, 32):
                need = mpw.lib.mpw_qlinear_workspace_bytes(b, mpw.LAYOUTS["paired"], M, N, K)
                x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
                y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
                if N == 17408:
                    # what the header states for the gate/up shape
                    assert (need > limit) == (M == 32), (b, M, need)
                st = _call_noalloc(mpw, x, packed, scales, b, "paired", y)
                if need > limit:
                    refused += 1
                    assert st == mpw.MPW_E_SCRATCH_LIMIT, (N, K, b, M, need)
                else:
                    assert st == mpw.MPW_OK, (N, K, b, M, need)
                    torch.cuda.synchronize()
                    assert float(y.float().abs().max()) == 0.0
    # gate/up at M = 32 needs more than the array holds
    assert refused >= 1
    assert mpw.device_error() == 0
