"""Output-row sharding on one GPU: every rank's share is run on this GPU
(no collective: the blocks are laid out as an all-gather would leave them),
and mpw_gather_shards puts the columns in order.  The result must meet the
decode bound against the oracle over the whole matrix, for world sizes
1..4, M = 1 and M > 1, both layouts.  The re-ordering kernel alone is
compared value for value with its formula.
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


def test_gather_shards_formula(mpw):
    import torch

    for world, M, Nl, N in [(3, 5, 32, 90), (2, 2, 16, 17), (4, 32, 4352, 17408), (1, 7, 48, 40)]:
        blocks = torch.arange(world * M * Nl, dtype=torch.float32).remainder(4093).to(torch.bfloat16).cuda()
        y = mpw.gather_shards(blocks, world, M, Nl, N)
        torch.cuda.synchronize()
        b = blocks.cpu().float().numpy().reshape(world, M, Nl)
        n = np.arange(N)
        want = b[n // Nl, :, n % Nl].T
        assert np.array_equal(y.float().cpu().numpy(), want)


@pytest.mark.parametrize("layout", ["paired", "canonical"])
@pytest.mark.parametrize("world", [1, 2, 3, 4])
def test_sharded_ranks_on_one_gpu(mpw, layout, world):
    import torch

    from mixed_precision_weight_row_b200 import shard

    rng = np.random.default_rng(50 + world)
    for N, K, b in [(1000, 512, 5), (17408 // 8, 5120, 6), (130, 4096, 12)]:
        W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)
        packed, scales = mpw.quantize_pack(torch.from_numpy(W).cuda(), b)
        if layout != "canonical":
            packed = mpw.repack(packed, K, b, "canonical", layout)
        q, s = oracle.quantize(W, b)
        lins = [shard.ShardedLinear.from_full(packed, scales, N, K, b, world, r, layout=layout)
                for r in range(world)]
        for M in (1, 4, 33):
            x = workloads.gen_x(M, K, seed=N + M)
            xd = x.cuda()
            blocks = torch.cat([mpw.qlinear(xd, L.packed, L.scales, b, layout=layout).reshape(-1) for L in lins])
            Nl = lins[0].Nl
            if M == 1:
                y = blocks[:N].view(1, N)
            else:
                y = mpw.gather_shards(blocks, world, M, Nl, N)
            torch.cuda.synchronize()
            y_ref, bound = oracle.qlinear_ref(x.float().numpy(), q, s)
            ok = oracle.check_qlinear(y.float().cpu().numpy(), y_ref, bound)
            assert ok.all(), (N, K, b, M, int((~ok).sum()))


def test_single_rank_call_needs_no_process_group(mpw):
    import torch

    from mixed_precision_weight_row_b200 import shard

    rng = np.random.default_rng(3)
    N, K, b = 300, 1024, 6
    W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)
    packed, scales = mpw.quantize_pack(torch.from_numpy(W).cuda(), b)
    lin = shard.ShardedLinear.from_full(packed, scales, N, K, b, 1, 0)
    q, s = oracle.quantize(W, b)
    for M in (1, 5):
        x = workloads.gen_x(M, K, seed=M)
        y = shard.qlinear_sharded(x.cuda(), lin)
        torch.cuda.synchronize()
        y_ref, bound = oracle.qlinear_ref(x.float().numpy(), q, s)
        assert oracle.check_qlinear(y.float().cpu().numpy(), y_ref, bound).all()
