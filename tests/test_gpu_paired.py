"""Paired-halves layout on the GPU.

* The re-ordering kernel matches the oracle's definition byte for byte, in
  both directions, out of place (no write past the buffer) and in place.
* The decode and prefill kernels reading paired rows meet the output bound
  |y - y_ref| <= 8e-3 * sum_k |x w_hat| + 1e-6 on every bit width.
* With one-hot x every output is exactly bf16(fl32(s_n * q)): the expansion
  of every code to the tensor-core operand is exact, in both layouts and on
  both kernels.
"""
import numpy as np
import pytest

import oracle
import workloads

pytestmark = pytest.mark.gpu

BITS = list(range(4, 16))
PAIR_SHAPES = [(1, 32), (3, 64), (17, 96), (64, 512), (129, 1024), (40, 4096), (33, 5120)]


@pytest.fixture(scope="module")
def mpw():
    import mixed_precision_weight_row_b200 as m

    return m


def _torch():
    import torch

    return torch


def _codes(rng, N, K, b):
    Q = oracle.qmax(b)
    q = rng.integers(-Q, Q + 1, size=(N, K)).astype(np.int32)
    q[0, : min(K, 40)] = Q
    if N > 1:
        q[1, : min(K, 40)] = -Q
    if N > 2:
        q[2] = 0
    return q


@pytest.mark.parametrize("b", BITS)
def test_repack_matches_oracle(mpw, b):
    torch = _torch()
    rng = np.random.default_rng(60 + b)
    for N, K in PAIR_SHAPES:
        q = _codes(rng, N, K, b)
        canon = oracle.pack(q, b)
        want = oracle.pack_paired(q, b)
        rb = oracle.packed_row_bytes(K, b)
        src = torch.from_numpy(canon).cuda()
        buf = torch.full((N * rb + 256,), 0xAB, dtype=torch.uint8, device="cuda")
        out = buf[: N * rb].view(N, rb)
        mpw.repack(src, K, b, out=out)
        torch.cuda.synchronize()
        assert np.array_equal(out.cpu().numpy(), want), f"{N}x{K}"
        assert bool((buf[N * rb:] == 0xAB).all()), "write past the output"
        back = mpw.repack(out, K, b, "paired", "canonical")
        assert np.array_equal(back.cpu().numpy(), canon)
        inplace = src.clone()
        mpw.repack(inplace, K, b, out=inplace)
        assert np.array_equal(inplace.cpu().numpy(), want)


def test_repack_then_unpack_roundtrip_on_quantized_rows(mpw):
    torch = _torch()
    rng = np.random.default_rng(61)
    W = rng.standard_normal((300, 640)).astype(np.float32)
    for b in (4, 6, 8, 11, 15):
        packed, _ = mpw.quantize_pack(torch.from_numpy(W).cuda(), b)
        paired = mpw.repack(packed, 640, b)
        q, _ = oracle.quantize(W, b)
        assert np.array_equal(oracle.unpack_paired(paired.cpu().numpy(), 640, b), q)
        codes = mpw.unpack(mpw.repack(paired, 640, b, "paired", "canonical"), 640, b)
        assert np.array_equal(codes.cpu().numpy().astype(np.int32), q)


def _check_paired(mpw, W, x_t, b, path="auto"):
    torch = _torch()
    q, s = oracle.quantize(W, b)
    packed = torch.from_numpy(oracle.pack_paired(q, b)).cuda()
    scales = torch.from_numpy(s).cuda()
    y = mpw.qlinear(x_t.cuda(), packed, scales, b, path=path, layout="paired")
    torch.cuda.synchronize()
    y_ref, bound = oracle.qlinear_ref(x_t.float().numpy(), q, s)
    ok = oracle.check_qlinear(y.float().cpu().numpy(), y_ref, bound)
    if not ok.all():
        i = np.argwhere(~ok)[0]
        raise AssertionError(f"{(~ok).sum()} outputs out of bound, first at {i.tolist()}: "
                             f"gpu {y.float().cpu().numpy()[tuple(i)]} ref {y_ref[tuple(i)]} bound {bound[tuple(i)]}")


QL_SHAPES = [(1, 32), (64, 512), (129, 1024), (40, 4096), (33, 160), (16, 17408)]


@pytest.mark.parametrize("b", BITS)
@pytest.mark.parametrize("M", [1, 2, 3, 8, 9, 16, 17, 32])
def test_qlinear_paired_decode(mpw, b, M):
    rng = np.random.default_rng(7000 + 40 * b + M)
    for N, K in QL_SHAPES:
        W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)
        if N > 3:
            W[1] = 0
            W[2, ::7] *= np.float32(30)
        x = workloads.gen_x(M, K, seed=b * 17 + M)
        _check_paired(mpw, W, x, b)


@pytest.mark.parametrize("b", [4, 6, 9, 15])
@pytest.mark.parametrize("M", [33, 70])
def test_qlinear_paired_gemv_path_any_m(mpw, b, M):
    rng = np.random.default_rng(7100 + b + M)
    W = rng.standard_normal((96, 320)).astype(np.float32)
    _check_paired(mpw, W, workloads.gen_x(M, 320, seed=M), b, path="gemv")


@pytest.mark.parametrize("b", BITS)
def test_qlinear_paired_gemm(mpw, b):
    rng = np.random.default_rng(7200 + b)
    for M, N, K in [(33, 1, 32), (64, 40, 64), (256, 128, 128), (300, 200, 512), (40, 260, 4096)]:
        W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)
        if N > 3:
            W[2] = 0
        _check_paired(mpw, W, workloads.gen_x(M, K, seed=M + K + b), b, path="gemm")


@pytest.mark.parametrize("b", BITS)
@pytest.mark.parametrize("layout", ["canonical", "paired"])
@pytest.mark.parametrize("path", ["gemv", "gemm"])
def test_one_hot_x_gives_exact_products(mpw, b, layout, path):
    torch = _torch()
    N, K, M = 96, 512, 8
    rng = np.random.default_rng(7300 + b)
    q = _codes(rng, N, K, b)
    s = (rng.random(N).astype(np.float32) + np.float32(0.5)) * np.float32(0.01)
    ks = np.array([0, 1, 31, 32, 200, 255, 256, 511])
    x = torch.zeros((M, K), dtype=torch.bfloat16)
    for m, k in enumerate(ks):
        x[m, k] = 1.0
    packed = oracle.pack_paired(q, b) if layout == "paired" else oracle.pack(q, b)
    y = mpw.qlinear(x.cuda(), torch.from_numpy(packed).cuda(), torch.from_numpy(s).cuda(), b, path=path,
                    layout=layout)
    prod = (q[:, ks].T.astype(np.float32) * s[None, :]).astype(np.float32)       # fl32(q * s)
    want = torch.from_numpy(prod).to(torch.bfloat16)                             # round to nearest even
    assert torch.equal(y.cpu().view(torch.int16), want.view(torch.int16))


def test_recipe_stack_paired_layers(mpw):
    # three chained links, the last two reading the rms-scaled input, in the
    # paired layout, against the oracle link by link
    torch = _torch()
    rng = np.random.default_rng(7400)
    dims = [(256, 320), (192, 256), (320, 192)]        # (N, K) per link
    bits = [5, 8, 12]
    x0 = workloads.gen_x(3, 320, seed=74)
    slots = [torch.zeros((3, 512), dtype=torch.bfloat16, device="cuda") for _ in range(4)]
    slots[0][:, :320] = x0.cuda()
    # slot buffers are [3, 512]; each link reads/writes a contiguous [M, K] / [M, N] prefix
    flat = [sl.view(-1) for sl in slots]
    layers, refs = [], []
    for i, ((N, K), b) in enumerate(zip(dims, bits)):
        W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.05)
        q, s = oracle.quantize(W, b)
        refs.append((q, s))
        layers.append(mpw.Linear(torch.from_numpy(oracle.pack_paired(q, b)).cuda(), torch.from_numpy(s).cuda(),
                                 N, K, b, i, i + 1, i > 0, layout="paired"))
    views = [flat[0][: 3 * 320].view(3, 320)]
    for i, (N, K) in enumerate(dims):
        views.append(flat[i + 1][: 3 * N].view(3, N))
    views[0].copy_(x0.cuda())
    mpw.recipe_run(layers, views, 3)
    torch.cuda.synchronize()
    for i, (q, s) in enumerate(refs):
        x_in = views[i].float().cpu().numpy()
        y = views[i + 1].float().cpu().numpy()
        if i == 0:
            y_ref, bound = oracle.qlinear_ref(x_in, q, s)
        else:
            y_ref, bound = oracle.qlinear_rms_ref(x_in, q, s)
        assert oracle.check_qlinear(y, y_ref, bound).all(), f"link {i}"
