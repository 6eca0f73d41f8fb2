"""Output-row sharding of a packed linear (mixed_precision_weight_row_b200.shard)
on CPU ranks: gloo, world size 2 and 3, 127.0.0.1.

The partition (rows per rank, zero rows past N, each rank's packed rows and
scales), the one all-gather and the order in which the gathered blocks form
y are the product's own code; only the rank-local product and the column
re-ordering are CPU stand-ins here (the oracle's fp64 linear on the rank's
rows, and the documented formula y[m, n] = blocks[n // Nl, m, n % Nl]),
because the library's kernels need a GPU.  Every rank's y must equal the
oracle's linear over the whole matrix.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from mixed_precision_weight_row_b200 import shard  # noqa: E402


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_partition_covers_every_row_once():
    for N in (1, 15, 16, 17, 50, 1024, 5120, 17408):
        for world in (1, 2, 3, 4, 8):
            Nl = shard.rows_per_rank(N, world)
            assert Nl % 16 == 0 and Nl * world >= N and Nl - 16 < -(-N // world) <= Nl
            seen = []
            for r in range(world):
                n0, n1 = shard.rank_rows(N, world, r)
                assert n0 == min(r * Nl, N) and n1 - n0 <= Nl
                seen.extend(range(n0, n1))
            assert seen == list(range(N))
    with pytest.raises(ValueError):
        shard.rank_rows(10, 2, 2)


def _cpu_local(oracle, K, b):
    import torch

    def local(x, lin):
        q = oracle.unpack(lin.packed.numpy(), K, b)
        y, _ = oracle.qlinear_ref(x.numpy(), q, lin.scales.numpy())
        return torch.from_numpy(y)
    return local


def _cpu_reorder(blocks, world, M, Nl, N, y):
    import torch

    b = blocks.reshape(world, M, Nl)
    for n in range(N):
        y[:, n] = b[n // Nl, :, n % Nl]
    return y


def _rank_main(rank, world, port, queue):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch
    import torch.distributed as dist

    import oracle
    from mixed_precision_weight_row_b200 import shard as sh

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        rng = np.random.default_rng(11)
        N, K, b = 50, 64, 6
        W = rng.standard_normal((N, K)).astype(np.float32)
        packed, s = oracle.quantize_pack(W, b)
        q, _ = oracle.quantize(W, b)
        lin = sh.ShardedLinear.from_full(torch.from_numpy(packed), torch.from_numpy(s), N, K, b, world, rank)
        errs = []
        for M in (1, 3):
            x = torch.from_numpy(rng.standard_normal((M, K)))
            y = sh.qlinear_sharded(x, lin, local=_cpu_local(oracle, K, b), reorder=_cpu_reorder)
            y_ref, _ = oracle.qlinear_ref(x.numpy(), q, s)
            errs.append(float(np.max(np.abs(y.numpy() - y_ref) / (np.abs(y_ref) + 1e-12))))
        # the rank's own rows, zero rows past N
        n0, n1 = sh.rank_rows(N, world, rank)
        ok_rows = bool(np.array_equal(lin.packed[: n1 - n0].numpy(), packed[n0:n1])) and \
            bool((lin.packed[n1 - n0:] == 0).all()) and bool((lin.scales[n1 - n0:] == 1).all())
        queue.put((rank, errs, ok_rows, lin.Nl))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_linear_equals_the_whole_matrix(world):
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, queue)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(queue.get(timeout=5) for _ in range(world))
    for rank, errs, ok_rows, Nl in got:
        assert ok_rows, rank
        assert Nl == shard.rows_per_rank(50, world)
        assert max(errs) < 1e-12, (rank, errs)
