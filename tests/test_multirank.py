"""World-size-2 checks of the token-sharded multi-rank path, on CPU with gloo.

Each rank takes its rows of a global batch, runs the forward on them (the
oracle stands in for the GPU kernels here), gathers the row-sharded outputs,
and the result must equal the single-process forward. Also checks the row
split and the max-over-ranks timing reduction used by bench.py.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from hadamard_bit_quant_b200 import inputs
from hadamard_bit_quant_b200.shard import gather_rows, max_over_ranks, row_range


def test_row_range_partitions():
    for M in (0, 1, 5, 16, 4096, 4097):
        for world in (1, 2, 3, 8):
            spans = [row_range(M, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == M
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        row_range(4, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, M, q):
    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        case = inputs.tiny_case()
        X = inputs.gaussian_with_outliers(M, case.K, 7, [3, 77], 40.0).to(torch.float64).numpy()
        a, T = oracle.weight_quant(case.make_w().numpy())
        lo, hi = row_range(M, rank, world)
        y_local = torch.from_numpy(oracle.forward(X[lo:hi], T, a, 4, 1)["Y"])
        y = gather_rows(y_local, M)
        t = max_over_ranks(1.0 + rank)
        q.put((rank, y.numpy(), t))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("M", [5, 16])
def test_two_rank_sharded_forward_matches_single(M):
    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, M, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    case = inputs.tiny_case()
    X = inputs.gaussian_with_outliers(M, case.K, 7, [3, 77], 40.0).to(torch.float64).numpy()
    a, T = oracle.weight_quant(case.make_w().numpy())
    want = oracle.forward(X, T, a, 4, 1)["Y"]
    for rank, y, t in res:
        assert np.array_equal(y, want)
        assert t == 2.0
