"""Group-wise scales (quantization tutorial, exercises, item 1: one scale per
g consecutive weights of a row instead of one per row) on the GPU against the
oracle.

* mpw_quantize_pack_groups: scales (as bit patterns) and packed bytes equal
  oracle.quantize_groups + oracle.pack, for every bit width and every group
  size 32..1024, on ragged shapes (K not a multiple of 32 or of g), rows with
  zero groups, ties, outliers and tiny values; guard bytes catch writes past
  the buffers.  The 4096x4096 decode matrix at g = 32 .. 256 and sampled rows
  of the 27B-class shapes at g = 128 are compared too.
* mpw_qlinear_groups: every output within |y - y_ref| <= 8e-3 * sum|x w_hat|
  + 1e-6 of the oracle's fp64 reference from w_hat = q * s_group, for
  g = 128 .. 1024, both layouts, M = 1 .. 40 (two passes of 32 above 32),
  and on the full-size decode and 27B-class shapes (sampled rows there).
"""
import numpy as np
import pytest

import oracle
import workloads

pytestmark = pytest.mark.gpu

BITS = list(range(4, 16))
GROUPS = [32, 64, 128, 256, 512, 1024]
SHAPES = [(1, 32), (3, 100), (17, 129), (40, 1000), (64, 1024), (129, 2560), (5, 4099)]


@pytest.fixture(scope="module")
def mpw():
    import mixed_precision_weight_row_b200 as m

    return m


def _torch():
    import torch

    return torch


def _weights(N, K, seed):
    rng = np.random.default_rng(seed)
    W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)
    if N > 2:
        W[1, : min(K, 300)] = 0.0                    # zero groups, and a partly zero row
    if N > 3:
        W[2] = np.round(W[2] * 64) / 64              # many ties after the division
    W.flat[rng.integers(0, W.size, max(1, W.size // 500))] *= np.float32(20)
    if N > 4:
        W[3] *= np.float32(1e-30)                    # tiny values, subnormal scales
    return W


def _gpu_quantize_groups(mpw, W_np, b, g, guard=256):
    torch = _torch()
    N, K = W_np.shape
    rb = oracle.packed_row_bytes(K, b)
    G = oracle.group_count(K, g)
    W = torch.from_numpy(W_np).cuda()
    pbuf = torch.full((N * rb + guard,), 0xAB, dtype=torch.uint8, device="cuda")
    sbuf = torch.full((N * G + 64,), -7.0, dtype=torch.float32, device="cuda")
    packed = pbuf[: N * rb].view(N, rb)
    scales = sbuf[: N * G].view(N, G)
    mpw.quantize_pack_groups(W, b, g, packed=packed, scales=scales)
    torch.cuda.synchronize()
    assert bool((pbuf[N * rb:] == 0xAB).all()), "write past the packed buffer"
    assert bool((sbuf[N * G:] == -7.0).all()), "write past the scales"
    return packed, scales


def _assert_groups_equal(mpw, W_np, b, g):
    packed, scales = _gpu_quantize_groups(mpw, W_np, b, g)
    q_ref, s_ref = oracle.quantize_groups(W_np, b, g)
    s_gpu = scales.cpu().numpy()
    assert np.array_equal(s_gpu.view(np.uint32), s_ref.view(np.uint32)), "group scales differ"
    p_ref = oracle.pack(q_ref, b)
    p_gpu = packed.cpu().numpy()
    if not np.array_equal(p_gpu, p_ref):
        bad = np.argwhere(p_gpu != p_ref)
        raise AssertionError(f"packed bytes differ at {bad[:5].tolist()} ({len(bad)} bytes)")
    return packed, scales, q_ref, s_ref


@pytest.mark.parametrize("b", BITS)
@pytest.mark.parametrize("g", GROUPS)
def test_quantize_pack_groups_bit_exact(mpw, b, g):
    for i, (N, K) in enumerate(SHAPES):
        _assert_groups_equal(mpw, _weights(N, K, 100 * b + g + i), b, g)


@pytest.mark.parametrize("g", [32, 64, 128, 256])
@pytest.mark.parametrize("b", [4, 6])
def test_quantize_pack_groups_decode_matrix(mpw, b, g):
    c = workloads.DECODE
    W = workloads.gen_weight(c["N"], c["K"], c["sigma"], c["w_seed"], c["outlier_frac"], c["outlier_scale"])
    _assert_groups_equal(mpw, W, b, g)


def test_quantize_pack_groups_single_group_equals_per_row(mpw):
    """g >= K: one group per row, so the group quantizer must reproduce the
    per-row quantizer's bytes and scales exactly."""
    torch = _torch()
    W = _weights(33, 1000, 5)
    for b in (4, 7, 12):
        p_g, s_g = _gpu_quantize_groups(mpw, W, b, 1024)
        p_r, s_r = mpw.quantize_pack(torch.from_numpy(W).cuda(), b)
        torch.cuda.synchronize()
        assert torch.equal(p_g, p_r)
        assert torch.equal(s_g[:, 0].view(torch.int32), s_r.view(torch.int32))


def _qlinear_groups_check(mpw, W, b, g, M, layout, x_seed, rows=None):
    torch = _torch()
    N, K = W.shape
    packed, scales = mpw.quantize_pack_groups(torch.from_numpy(W).cuda(), b, g)
    if layout != "canonical":
        packed = mpw.repack(packed, K, b, "canonical", layout)
    x = workloads.gen_x(M, K, x_seed)
    y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    mpw.qlinear_groups(x.cuda(), packed, scales, b, g, y=y, layout=layout)
    torch.cuda.synchronize()
    Wr = W if rows is None else W[rows]
    q, s = oracle.quantize_groups(Wr, b, g)
    y_ref, bound = oracle.qlinear_groups_ref(x.float().numpy(), q, s, g)
    yg = y.float().cpu().numpy()
    if rows is not None:
        yg = yg[:, rows]
    ok = oracle.check_qlinear(yg, y_ref, bound)
    assert ok.all(), f"b={b} g={g} M={M} {layout}: {(~ok).sum()} outputs out of bound"


@pytest.mark.parametrize("layout", ["paired", "canonical"])
@pytest.mark.parametrize("g", [128, 256, 512, 1024])
@pytest.mark.parametrize("b", [4, 5, 6, 8, 9, 10, 12, 15])
def test_qlinear_groups_small(mpw, layout, g, b):
    shapes = [(16, 128), (40, 1024), (100, 2560), (257, 1280), (33, 4096)]
    for i, (N, K) in enumerate(shapes):
        for M in (1, 3, 8, 9, 16, 17, 32, 40):
            _qlinear_groups_check(mpw, _weights(N, K, 7 * i + b + g), b, g, M, layout, x_seed=M + N)
    assert mpw.device_error() == 0


@pytest.mark.parametrize("b", [4, 6, 8])
@pytest.mark.parametrize("M", [1, 4, 16])
def test_qlinear_groups_decode_workload(mpw, b, M):
    c = workloads.DECODE
    W = workloads.gen_weight(c["N"], c["K"], c["sigma"], c["w_seed"], c["outlier_frac"], c["outlier_scale"])
    _qlinear_groups_check(mpw, W, b, 128, M, "paired", x_seed=c["x_seed"])
    assert mpw.device_error() == 0


@pytest.mark.parametrize("shape", ["gate", "down"])
@pytest.mark.parametrize("M", [1, 8, 32])
def test_qlinear_groups_mlp27b_sampled(mpw, shape, M):
    torch = _torch()
    name, N, K = [s for s in workloads.MLP27B["shapes"] if s[0] == shape][0]
    Wt = workloads.gen_weight_torch(N, K, workloads.MLP27B["sigma"], 17 + N)
    rows = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(N + M).choice(N, 48, replace=False)]))
    b = 5
    packed, scales = mpw.quantize_pack_groups(Wt, b, 128)
    # quantizer parity on the sampled rows
    W_rows = Wt[torch.from_numpy(rows).cuda()].cpu().numpy()
    q_ref, s_ref = oracle.quantize_groups(W_rows, b, 128)
    assert np.array_equal(scales.cpu().numpy()[rows].view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(packed.cpu().numpy()[rows], oracle.pack(q_ref, b))
    packed = mpw.repack(packed, K, b, "canonical", "paired")
    x = workloads.gen_x(M, K, 1)
    y = mpw.qlinear_groups(x.cuda(), packed, scales, b, 128, layout="paired")
    torch.cuda.synchronize()
    y_ref, bound = oracle.qlinear_groups_ref(x.float().numpy(), q_ref, s_ref, 128)
    ok = oracle.check_qlinear(y.float().cpu().numpy()[:, rows], y_ref, bound)
    assert ok.all(), f"{(~ok).sum()} outputs out of bound"
    assert mpw.device_error() == 0


def test_qlinear_groups_flagged_calls(mpw):
    """Flagged calls (x_ready, y_unshared) back to back on one stream, each
    matrix into its own output, after an unflagged call: every output still
    meets the bound (the flags only let the calls overlap)."""
    torch = _torch()
    N, K, b, g = 1000, 2048, 5, 128
    mats = []
    for i in range(5):
        W = _weights(N, K, 900 + i)
        packed, scales = mpw.quantize_pack_groups(torch.from_numpy(W).cuda(), b, g)
        mats.append((W, mpw.repack(packed, K, b, "canonical", "paired"), scales))
    for M in (1, 8, 32):
        x = workloads.gen_x(M, K, 77 + M)
        xd = x.cuda()
        ys = [torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda") for _ in mats]
        for i, (_, p, s) in enumerate(mats):
            mpw.qlinear_groups(xd, p, s, b, g, y=ys[i], layout="paired", x_ready=i > 0, y_unshared=i > 0)
        torch.cuda.synchronize()
        for (W, _, _), y in zip(mats, ys):
            q, s = oracle.quantize_groups(W, b, g)
            y_ref, bound = oracle.qlinear_groups_ref(x.float().numpy(), q, s, g)
            assert oracle.check_qlinear(y.float().cpu().numpy(), y_ref, bound).all(), M
    assert mpw.device_error() == 0
