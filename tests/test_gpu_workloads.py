"""CUDA path vs the CPU oracle at the benchmark workloads' full sizes.

* single  (256x512, b=5, M=1): everything compared.
* decode  (4096x4096 with 0.1% outliers, every listed b, M in {1,4,16}):
  packed bytes and scales compared in full, outputs in full.
* mlp27b  (17408x5120 and 5120x17408, b in {5,6}, M in {1,8,32}): the
  quantizer and the linear run at full size in the configuration the benchmark
  uses; a seeded sample of rows is compared (each output column depends on one
  row of W only, so the oracle can compute the sampled columns one by one).
* prefill (x 2048x5120; 17408x5120 and 5120x5120, b in {5,6,8,10,12}): the
  tensor-core GEMM on sampled rows.
Each linear runs on the canonical rows and on their paired-halves re-ordering
(made on the GPU and compared with the oracle's byte for byte).
"""
import numpy as np
import pytest

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mpw():
    import mixed_precision_weight_row_b200 as m

    return m


def _t():
    import torch

    return torch


def test_single_matrix_workload(mpw):
    torch = _t()
    c = wl.SINGLE
    W = wl.gen_weight(c["N"], c["K"], c["sigma"], c["w_seed"])
    x = wl.gen_x(1, c["K"], c["x_seed"])
    b = c["bits"][0]
    packed, scales = mpw.quantize_pack(torch.from_numpy(W).cuda(), b)
    p_ref, s_ref = oracle.quantize_pack(W, b)
    assert np.array_equal(packed.cpu().numpy(), p_ref)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    y = mpw.qlinear(x.cuda(), packed, scales, b)
    q, s = oracle.quantize(W, b)
    y_ref, bound = oracle.qlinear_ref(x.float().numpy(), q, s)
    assert oracle.check_qlinear(y.float().cpu().numpy(), y_ref, bound).all()


@pytest.fixture(scope="module")
def decode_w():
    c = wl.DECODE
    return wl.gen_weight(c["N"], c["K"], c["sigma"], c["w_seed"], c["outlier_frac"], c["outlier_scale"])


@pytest.mark.parametrize("b", wl.DECODE["bits"])
def test_decode_workload(mpw, decode_w, b):
    torch = _t()
    c = wl.DECODE
    W = decode_w
    packed, scales = mpw.quantize_pack(torch.from_numpy(W).cuda(), b)
    q, s = oracle.quantize(W, b)
    p_ref = oracle.pack(q, b)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), s.view(np.uint32))
    assert np.array_equal(packed.cpu().numpy(), p_ref)
    paired = mpw.repack(packed, c["K"], b)
    assert np.array_equal(paired.cpu().numpy(), oracle.pack_paired(q, b))
    for M in c["Ms"]:
        x = wl.gen_x(M, c["K"], c["x_seed"])
        y_ref, bound = oracle.qlinear_ref(x.float().numpy(), q, s)
        for layout, p in (("canonical", packed), ("paired", paired)):
            y = mpw.qlinear(x.cuda(), p, scales, b, layout=layout)
            ok = oracle.check_qlinear(y.float().cpu().numpy(), y_ref, bound)
            assert ok.all(), f"{layout} M={M}: {(~ok).sum()} outputs out of bound"


@pytest.mark.parametrize("name,N,K", wl.MLP27B["shapes"][1:], ids=["gate", "down"])
@pytest.mark.parametrize("b", wl.MLP27B["bits"])
def test_mlp27b_workload_sampled(mpw, name, N, K, b):
    torch = _t()
    c = wl.MLP27B
    W = wl.gen_weight(N, K, c["sigma"], c["w_seed"])
    packed, scales = mpw.quantize_pack(torch.from_numpy(W).cuda(), b)
    rng = np.random.default_rng(123)
    rows = np.unique(np.concatenate([[0, N - 1], rng.choice(N, 254, replace=False)]))
    q, s = oracle.quantize(W[rows], b)
    p_gpu = packed.cpu().numpy()[rows]
    assert np.array_equal(p_gpu, oracle.pack(q, b))
    assert np.array_equal(scales.cpu().numpy()[rows].view(np.uint32), s.view(np.uint32))
    paired = mpw.repack(packed, K, b)
    assert np.array_equal(paired.cpu().numpy()[rows], oracle.pack_paired(q, b))
    for M in c["Ms"]:
        x = wl.gen_x(M, K, c["x_seed"])
        y_ref, bound = oracle.qlinear_ref(x.float().numpy(), q, s)
        for layout, p in (("canonical", packed), ("paired", paired)):
            y = mpw.qlinear(x.cuda(), p, scales, b, layout=layout).float().cpu().numpy()[:, rows]
            ok = oracle.check_qlinear(y, y_ref, bound)
            assert ok.all(), f"{layout} M={M}: {(~ok).sum()} sampled outputs out of bound"


@pytest.mark.parametrize("name,N,K", wl.PREFILL["shapes"], ids=["up", "o"])
@pytest.mark.parametrize("b", wl.PREFILL["bits"])
def test_prefill_workload_sampled(mpw, name, N, K, b):
    torch = _t()
    c = wl.PREFILL
    W = wl.gen_weight(N, K, c["sigma"], c["w_seed"])
    x = wl.gen_x(c["M"], K, c["x_seed"])
    packed, scales = mpw.quantize_pack(torch.from_numpy(W).cuda(), b)
    rng = np.random.default_rng(321)
    rows = np.unique(np.concatenate([[0, 127, 128, N - 1], rng.choice(N, 124, replace=False)]))
    q, s = oracle.quantize(W[rows], b)
    y_ref, bound = oracle.qlinear_ref(x.float().numpy(), q, s)
    for layout in ("canonical", "paired"):
        p = packed if layout == "canonical" else mpw.repack(packed, K, b)
        y = mpw.qlinear(x.cuda(), p, scales, b, layout=layout)          # M = 2048 -> tensor-core GEMM
        torch.cuda.synchronize()
        ok = oracle.check_qlinear(y.float().cpu().numpy()[:, rows], y_ref, bound)
        assert ok.all(), f"{layout}: {(~ok).sum()} sampled outputs out of bound"
    assert mpw.device_error() == 0
