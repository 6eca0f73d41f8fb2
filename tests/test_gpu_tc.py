"""The tensor-memory decode kernel (weights expanded into tensor memory,
tcgen05 MMAs with a 32-token tile), which the decode path selects for M > 16
on shapes with long K slices (M = 16 is also run: the per-tile kernel then).  Sampled rows are compared with the oracle
(each output row depends on one weight row only); the whole kernel was also
run over the full decode parity suite with it forced (MPW_GEMV_KERNEL=tc).
"""
import numpy as np
import pytest

import oracle
import workloads

pytestmark = pytest.mark.gpu

N, K = 16384, 3072      # 128 row tiles, 24 weight blocks per CTA: the kernel is selected


@pytest.fixture(scope="module")
def mpw():
    import mixed_precision_weight_row_b200 as m

    return m


@pytest.fixture(scope="module")
def weights():
    return workloads.gen_weight(N, K, 0.02, 77, 0.001, 20.0)


@pytest.mark.parametrize("b", [5, 6, 8, 12])
@pytest.mark.parametrize("layout", ["paired", "canonical"])
@pytest.mark.parametrize("M", [16, 17, 32, 45])
def test_tc_decode_sampled_rows(mpw, weights, b, layout, M):
    import torch

    assert mpw.lib.mpw_version() > 0
    packed, scales = mpw.quantize_pack(torch.from_numpy(weights).cuda(), b)
    if layout == "paired":
        packed = mpw.repack(packed, K, b)
    x = workloads.gen_x(M, K, seed=M + b)
    y = mpw.qlinear(x.cuda(), packed, scales, b, layout=layout, path="gemv")
    torch.cuda.synchronize()
    rng = np.random.default_rng(b * 100 + M)
    rows = np.unique(np.concatenate([[0, 127, 128, N - 1], rng.choice(N, 200, replace=False)]))
    q, s = oracle.quantize(weights[rows], b)
    y_ref, bound = oracle.qlinear_ref(x.float().numpy(), q, s)
    ok = oracle.check_qlinear(y.float().cpu().numpy()[:, rows], y_ref, bound)
    assert ok.all(), f"{(~ok).sum()} sampled outputs out of bound"
    assert mpw.device_error() == 0


def test_tc_one_hot_exact(mpw):
    import torch

    b, M = 8, 17
    rng = np.random.default_rng(5)
    q = rng.integers(-127, 128, size=(N, K)).astype(np.int32)
    s = (rng.random(N).astype(np.float32) + np.float32(0.5)) * np.float32(0.01)
    ks = np.array([0, 1, 127, 128, 1000, 2047, 2048, 3071, 5, 6, 7, 8, 9, 10, 11, 12, 3000])
    x = torch.zeros((M, K), dtype=torch.bfloat16)
    for m, k in enumerate(ks):
        x[m, k] = 1.0
    packed = torch.from_numpy(oracle.pack_paired(q, b)).cuda()
    y = mpw.qlinear(x.cuda(), packed, torch.from_numpy(s).cuda(), b, layout="paired")
    prod = (q[:, ks].T.astype(np.float32) * s[None, :]).astype(np.float32)
    want = torch.from_numpy(prod).to(torch.bfloat16)
    assert torch.equal(y.cpu().view(torch.int16), want.view(torch.int16))


def test_tc_recipe_norm_links(mpw, weights):
    # two linears on the tensor-memory kernel, the second reading the
    # rms-scaled input (its sums of squares are gathered over a K split)
    import torch

    M, b = 20, 6
    N2, K2 = 4096, N                          # 32 row tiles, K split over a cluster of 4
    x0 = workloads.gen_x(M, K, seed=31).cuda()
    W2 = workloads.gen_weight_torch(N2, K2, 0.02, 12)
    pa, sa = mpw.quantize_pack(torch.from_numpy(weights).cuda(), b)
    pb, sb = mpw.quantize_pack(W2, b)
    slots = [x0.contiguous(), torch.zeros((M, N), dtype=torch.bfloat16, device="cuda"),
             torch.zeros((M, N2), dtype=torch.bfloat16, device="cuda")]
    layers = [mpw.Linear(pa, sa, N, K, b, 0, 1, False), mpw.Linear(pb, sb, N2, K2, b, 1, 2, True)]
    assert mpw.lib.mpw_version() > 0
    mpw.recipe_run(layers, slots, M)
    torch.cuda.synchronize()
    rows1 = np.array([0, 1, 500, 8191, 16383])
    q1, s1 = oracle.quantize(weights[rows1], b)
    y_ref, bound = oracle.qlinear_ref(x0.float().cpu().numpy(), q1, s1)
    assert oracle.check_qlinear(slots[1][:, rows1].float().cpu().numpy(), y_ref, bound).all()
    rows2 = np.array([0, 7, 2048, 4095])
    q2, s2 = oracle.quantize(W2[rows2].cpu().numpy(), b)
    y_ref, bound = oracle.qlinear_rms_ref(slots[1].float().cpu().numpy(), q2, s2)
    assert oracle.check_qlinear(slots[2][:, rows2].float().cpu().numpy(), y_ref, bound).all()
    assert mpw.device_error() == 0
