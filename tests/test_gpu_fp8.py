"""FP8 (E4M3) prefill for 4- and 5-bit codes against the oracle's reading
(oracle/fp8.py).

* mpw_quantize_x_fp8: the per-token scales (bit patterns) and every E4M3
  byte equal the oracle's, including zero tokens, values in E4M3's
  subnormal range, ties and outliers.
* mpw_qlinear_fp8: every output within 8e-3 * sum|sx xq w_hat| + 1e-6 of
  the oracle's fp64 value of the FP8 definition, for b = 4, 5, both layouts,
  ragged M, N and K, one and several 256-token tiles; the full prefill
  shapes (x 2048 x 5120 against 17408 x 5120 and 5120 x 5120) on sampled
  rows.  Against the exact bf16 linear the difference stays within the bound
  of the activation rounding (plus the same tolerance).
* Wider codes are refused.
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


def _torch():
    import torch

    return torch


def _x(M, K, seed):
    torch = _torch()
    x = workloads.gen_x(M, K, seed)
    if M > 3:
        x[1] = 0                                      # a zero token
        x[2] = x[2] * 1e-6                            # elements in E4M3's subnormal range
        x[3, :7] = torch.tensor([448.0, -3.0, 0.5, 2.0 ** -9, 17.0, -33.0, 1e-30]).to(torch.bfloat16)
    return x


def _decode_e4m3(xq):
    torch = _torch()
    return xq.view(torch.float8_e4m3fn).to(torch.float32).cpu().numpy()


@pytest.mark.parametrize("M,K", [(1, 16), (5, 64), (300, 5120), (33, 4112), (2048, 5120)])
def test_quantize_x_fp8_bit_exact(mpw, M, K):
    torch = _torch()
    x = _x(M, K, M + K)
    xq, sx = mpw.quantize_x_fp8(x.cuda())
    torch.cuda.synchronize()
    xq_ref, sx_ref = oracle.quantize_x_fp8(x.float().numpy())
    assert np.array_equal(sx.cpu().numpy().view(np.uint32), sx_ref.view(np.uint32)), "activation scales differ"
    got = _decode_e4m3(xq)
    bad = np.argwhere(got != xq_ref)
    assert bad.size == 0, f"{len(bad)} E4M3 values differ, first {bad[:3].tolist()}"


def _check_fp8(mpw, W, b, M, layout, seed, rows=None):
    torch = _torch()
    N, K = W.shape
    packed, scales = mpw.quantize_pack(torch.from_numpy(W).cuda() if isinstance(W, np.ndarray) else W, b)
    if layout != "canonical":
        packed = mpw.repack(packed, K, b, "canonical", layout)
    x = _x(M, K, seed)
    y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    mpw.qlinear_fp8(x.cuda(), packed, scales, b, y=y, layout=layout)
    torch.cuda.synchronize()
    Wr = W if rows is None else W[rows]
    if not isinstance(Wr, np.ndarray):
        Wr = Wr.cpu().numpy()
    q, s = oracle.quantize(Wr, b)
    xf = x.float().numpy()
    y_ref, bound = oracle.qlinear_fp8_ref(xf, q, s)
    yg = y.float().cpu().numpy()
    if rows is not None:
        yg = yg[:, rows]
    ok = oracle.check_qlinear(yg, y_ref, bound)
    assert ok.all(), f"b={b} M={M} {layout}: {(~ok).sum()} outputs out of bound"
    # against the exact bf16 linear: within the bound of the activation rounding
    y_bf, bound_bf = oracle.qlinear_ref(xf, q, s)
    eb = oracle.fp8_input_error_bound(xf, q, s)
    assert np.all(np.abs(yg - y_bf) <= eb + bound_bf + bound)


@pytest.mark.parametrize("layout", ["paired", "canonical"])
@pytest.mark.parametrize("b", [4, 5])
def test_qlinear_fp8_small(mpw, layout, b):
    rng = np.random.default_rng(10 + b)
    for (N, K, M) in [(100, 256, 1), (128, 512, 40), (257, 1024, 300), (130, 5120, 513), (64, 4096, 256)]:
        W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)
        W[min(5, N - 1)] = 0
        _check_fp8(mpw, W, b, M, layout, seed=N + M)
    assert mpw.device_error() == 0


@pytest.mark.parametrize("shape", ["up", "o"])
@pytest.mark.parametrize("b", [4, 5])
def test_qlinear_fp8_prefill_workload_sampled(mpw, shape, b):
    torch = _torch()
    c = workloads.PREFILL
    name, N, K = [s for s in c["shapes"] if s[0] == shape][0]
    Wt = workloads.gen_weight_torch(N, K, c["sigma"], 11 + N)
    rows = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(N + b).choice(N, 40, replace=False)]))
    W_rows = Wt[torch.from_numpy(rows).cuda()].cpu().numpy()
    packed, scales = mpw.quantize_pack(Wt, b)
    packed = mpw.repack(packed, K, b, "canonical", "paired")
    x = workloads.gen_x(c["M"], K, c["x_seed"])
    y = mpw.qlinear_fp8(x.cuda(), packed, scales, b, layout="paired")
    torch.cuda.synchronize()
    q, s = oracle.quantize(W_rows, b)
    y_ref, bound = oracle.qlinear_fp8_ref(x.float().numpy(), q, s)
    ok = oracle.check_qlinear(y.float().cpu().numpy()[:, rows], y_ref, bound)
    assert ok.all(), f"{(~ok).sum()} outputs out of bound"
    assert mpw.device_error() == 0


def test_qlinear_fp8_refuses_wide_codes(mpw):
    torch = _torch()
    W = torch.randn(32, 64, device="cuda")
    for b in (6, 8):
        packed, scales = mpw.quantize_pack(W, b)
        xq = torch.zeros((4, 64), dtype=torch.uint8, device="cuda")
        sx = torch.ones(4, dtype=torch.float32, device="cuda")
        y = torch.empty((4, 32), dtype=torch.bfloat16, device="cuda")
        st = mpw.lib.mpw_qlinear_fp8(xq.data_ptr(), sx.data_ptr(), packed.data_ptr(), scales.data_ptr(), b, 0,
                                     4, 32, 64, y.data_ptr(), 0)
        assert st == mpw.MPW_E_UNSUPPORTED_BITS
