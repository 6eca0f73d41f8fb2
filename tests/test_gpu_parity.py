"""CUDA path vs the CPU oracle on small and ragged shapes (every bit width).

Codes, scales and packed bytes must match bit for bit; qlinear outputs must
satisfy |y - y_ref| <= 8e-3 * sum_k |x w_hat| + 1e-6 elementwise.
"""
import numpy as np
import pytest

import oracle
import workloads

pytestmark = pytest.mark.gpu

BITS = list(range(4, 16))
SHAPES = [(1, 1), (3, 5), (7, 31), (17, 33), (64, 127), (129, 257), (256, 512), (33, 1000), (5, 4099)]


@pytest.fixture(scope="module")
def mpw():
    import mixed_precision_weight_row_b200 as m

    return m


def _torch():
    import torch

    return torch


def _gpu_quantize(mpw, W_np, b, guard=256):
    """Quantize on the GPU into buffers with guard bytes after them."""
    torch = _torch()
    N, K = W_np.shape
    rb = oracle.packed_row_bytes(K, b)
    W = torch.from_numpy(W_np).cuda()
    pbuf = torch.full((N * rb + guard,), 0xAB, dtype=torch.uint8, device="cuda")
    sbuf = torch.full((N + 64,), -7.0, dtype=torch.float32, device="cuda")
    packed = pbuf[: N * rb].view(N, rb)
    scales = sbuf[:N]
    mpw.quantize_pack(W, b, packed=packed, scales=scales)
    torch.cuda.synchronize()
    assert bool((pbuf[N * rb:] == 0xAB).all()), "write past the packed buffer"
    assert bool((sbuf[N:] == -7.0).all()), "write past the scales"
    return packed, scales


def _assert_quant_equal(mpw, W_np, b):
    packed, scales = _gpu_quantize(mpw, W_np, b)
    p_ref, s_ref = oracle.quantize_pack(W_np, b)
    s_gpu = scales.cpu().numpy()
    assert np.array_equal(s_gpu.view(np.uint32), s_ref.view(np.uint32)), "scales differ"
    p_gpu = packed.cpu().numpy()
    if not np.array_equal(p_gpu, p_ref):
        bad = np.argwhere(p_gpu != p_ref)
        raise AssertionError(f"packed bytes differ at {bad[:5].tolist()} ({len(bad)} bytes)")
    return packed, scales


@pytest.mark.parametrize("b", BITS)
@pytest.mark.parametrize("shape", SHAPES, ids=[f"{n}x{k}" for n, k in SHAPES])
def test_quantize_pack_bit_exact(mpw, b, shape):
    N, K = shape
    rng = np.random.default_rng(N * 1000 + K + b)
    W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)
    if N > 4:
        W[2] = 0.0
        W.flat[rng.integers(0, W.size, max(1, W.size // 1000))] *= np.float32(20)
    _assert_quant_equal(mpw, W, b)


@pytest.mark.parametrize("b", [4, 5, 8, 11, 15])
@pytest.mark.parametrize("K", [37, 1000, 4096])
def test_quantize_pack_special_rows(mpw, b, K):
    _assert_quant_equal(mpw, workloads.special_rows(K), b)


@pytest.mark.parametrize("b", [4, 9, 15])
@pytest.mark.parametrize("K", [45000, 60000])
def test_quantize_pack_long_rows(mpw, b, K):
    # rows longer than the shared-memory stage take the two-pass variant
    rng = np.random.default_rng(K + b)
    W = rng.standard_normal((3, K)).astype(np.float32)
    _assert_quant_equal(mpw, W, b)


def test_quantize_pack_ties_exact(mpw):
    # rows whose quotients hit .5 exactly (power-of-two scales)
    rng = np.random.default_rng(11)
    for b in BITS:
        Q = oracle.qmax(b)
        W = (rng.integers(-2 * Q, 2 * Q + 1, size=(16, 300)) / 2.0).astype(np.float32)
        W[:, 0] = np.float32(Q)
        _assert_quant_equal(mpw, W, b)


def test_quantize_pack_golden_rows(mpw):
    from tests import test_oracle_pins as pins

    for case in pins._load_golden():
        b, w, scale, codes, packed = case.values
        p, s = _gpu_quantize(mpw, w[None, :].astype(np.float32), b)
        assert p.cpu().numpy()[0].tobytes() == packed, case.id
        assert s.cpu().numpy()[0].view(np.uint32) == np.float32(scale).view(np.uint32), case.id


def test_nonfinite_flag(mpw):
    torch = _torch()
    W = torch.zeros((4, 64), dtype=torch.float32, device="cuda")
    flag = torch.zeros((1,), dtype=torch.int32, device="cuda")
    mpw.quantize_pack(W, 6, nonfinite_flag=flag)
    assert int(flag.item()) == 0
    W[2, 17] = float("inf")
    mpw.quantize_pack(W, 6, nonfinite_flag=flag)
    assert int(flag.item()) == 1
    flag.zero_()
    W[2, 17] = float("nan")
    mpw.quantize_pack(W, 6, nonfinite_flag=flag)
    assert int(flag.item()) == 1


@pytest.mark.parametrize("b", BITS)
def test_unpack_and_dequantize_bit_exact(mpw, b):
    torch = _torch()
    rng = np.random.default_rng(50 + b)
    for N, K in [(1, 1), (9, 33), (70, 513), (33, 1000)]:
        W = rng.standard_normal((N, K)).astype(np.float32)
        q_ref, s_ref = oracle.quantize(W, b)
        p_ref = oracle.pack(q_ref, b)
        packed = torch.from_numpy(p_ref).cuda()
        scales = torch.from_numpy(s_ref).cuda()
        codes = mpw.unpack(packed, K, b)
        assert np.array_equal(codes.cpu().numpy().astype(np.int32), q_ref)
        w_hat = mpw.dequantize(packed, scales, K, b)
        assert np.array_equal(w_hat.cpu().numpy().view(np.uint32), oracle.dequantize(q_ref, s_ref).view(np.uint32))


def _check_qlinear(mpw, W, x_t, b, path="auto"):
    torch = _torch()
    q, s = oracle.quantize(W, b)
    packed = torch.from_numpy(oracle.pack(q, b)).cuda()
    scales = torch.from_numpy(s).cuda()
    y = mpw.qlinear(x_t.cuda(), packed, scales, b, path=path)
    torch.cuda.synchronize()
    y_ref, bound = oracle.qlinear_ref(x_t.float().numpy(), q, s)
    ok = oracle.check_qlinear(y.float().cpu().numpy(), y_ref, bound)
    if not ok.all():
        i = np.argwhere(~ok)[0]
        raise AssertionError(f"{(~ok).sum()} outputs out of bound, first at {i.tolist()}: "
                             f"gpu {y.float().cpu().numpy()[tuple(i)]} ref {y_ref[tuple(i)]} bound {bound[tuple(i)]}")


QL_SHAPES = [(1, 1), (3, 37), (64, 512), (129, 1000), (256, 4099), (40, 64)]


@pytest.mark.parametrize("b", BITS)
@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 16, 17, 32])
def test_qlinear_decode_small(mpw, b, M):
    rng = np.random.default_rng(1000 * b + M)
    for N, K in QL_SHAPES:
        W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)
        if N > 3:
            W[1] = 0
        x = workloads.gen_x(M, K, seed=b * 31 + M)
        _check_qlinear(mpw, W, x, b)


@pytest.mark.parametrize("b", [4, 6, 9, 10, 15])
@pytest.mark.parametrize("M", [33, 64, 130])
def test_qlinear_gemv_path_any_m(mpw, b, M):
    rng = np.random.default_rng(2000 * b + M)
    W = rng.standard_normal((96, 300)).astype(np.float32)
    x = workloads.gen_x(M, 300, seed=M)
    _check_qlinear(mpw, W, x, b, path="gemv")


@pytest.mark.parametrize("b", [5, 8, 12])
def test_qlinear_large_k_chunks_x(mpw, b):
    # K beyond the shared-memory budget for x makes the kernel stage x per chunk
    rng = np.random.default_rng(77 + b)
    for M, K in [(1, 45000), (2, 25000)]:
        W = rng.standard_normal((24, K)).astype(np.float32)
        x = workloads.gen_x(M, K, seed=K)
        _check_qlinear(mpw, W, x, b)


def test_qlinear_does_not_write_past_y(mpw):
    torch = _torch()
    b, M, N, K = 6, 3, 50, 200
    rng = np.random.default_rng(5)
    W = rng.standard_normal((N, K)).astype(np.float32)
    q, s = oracle.quantize(W, b)
    packed = torch.from_numpy(oracle.pack(q, b)).cuda()
    scales = torch.from_numpy(s).cuda()
    x = workloads.gen_x(M, K, seed=3).cuda()
    ybuf = torch.full((M * N + 128,), 7.0, dtype=torch.bfloat16, device="cuda")
    mpw.qlinear(x, packed, scales, b, y=ybuf[: M * N].view(M, N))
    torch.cuda.synchronize()
    assert bool((ybuf[M * N:] == 7.0).all())


def test_quantize_then_qlinear_roundtrip(mpw):
    # the packed bytes the GPU writes are what the GPU linear reads
    torch = _torch()
    rng = np.random.default_rng(9)
    W = rng.standard_normal((300, 777)).astype(np.float32) * np.float32(0.02)
    x = workloads.gen_x(4, 777, seed=9)
    for b in (4, 7, 13):
        packed, scales = mpw.quantize_pack(torch.from_numpy(W).cuda(), b)
        y = mpw.qlinear(x.cuda(), packed, scales, b)
        q, s = oracle.quantize(W, b)
        y_ref, bound = oracle.qlinear_ref(x.float().numpy(), q, s)
        assert oracle.check_qlinear(y.float().cpu().numpy(), y_ref, bound).all()


# ----------------------------------------------------------------------------
# tensor-core prefill GEMM
# ----------------------------------------------------------------------------

GEMM_SHAPES = [(33, 1, 8), (64, 40, 64), (256, 128, 128), (300, 200, 520), (513, 129, 1000), (40, 260, 4104)]


@pytest.mark.parametrize("b", BITS)
def test_qlinear_gemm_small(mpw, b):
    rng = np.random.default_rng(3000 + b)
    for M, N, K in GEMM_SHAPES:
        W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)
        if N > 3:
            W[2] = 0
        x = workloads.gen_x(M, K, seed=M + K + b)
        _check_qlinear(mpw, W, x, b, path="gemm")


@pytest.mark.parametrize("b", [4, 8, 9, 10, 15])
@pytest.mark.parametrize("M", [1, 16, 32])
def test_qlinear_gemm_path_small_m(mpw, b, M):
    rng = np.random.default_rng(4000 + b + M)
    W = rng.standard_normal((150, 256)).astype(np.float32)
    x = workloads.gen_x(M, 256, seed=M)
    _check_qlinear(mpw, W, x, b, path="gemm")


def test_qlinear_auto_routes_odd_k_to_gemv(mpw):
    # K % 8 != 0 cannot be a TMA operand: auto falls back to the decode kernel
    rng = np.random.default_rng(6)
    W = rng.standard_normal((64, 301)).astype(np.float32)
    x = workloads.gen_x(70, 301, seed=6)
    _check_qlinear(mpw, W, x, 7)
    with pytest.raises(mpw.MPWError):
        _check_qlinear(mpw, W, x, 7, path="gemm")


def test_gemm_extreme_codes(mpw):
    # rows that hit +-Q everywhere and x of both signs: exercises the hi/lo split
    rng = np.random.default_rng(8)
    for b in (9, 10, 12, 15):
        W = np.where(rng.random((128, 512)) < 0.5, -1.0, 1.0).astype(np.float32)
        x = workloads.gen_x(256, 512, seed=b)
        _check_qlinear(mpw, W, x, b, path="gemm")


def test_gemm_device_error_word_clear(mpw):
    rng = np.random.default_rng(10)
    W = rng.standard_normal((128, 256)).astype(np.float32)
    x = workloads.gen_x(64, 256, seed=1)
    _check_qlinear(mpw, W, x, 6, path="gemm")
    assert mpw.device_error() == 0
