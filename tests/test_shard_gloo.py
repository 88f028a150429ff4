"""Multi-process (world_size 2, gloo, CPU) tests of the N > 1 host logic.

The path shards by tokens with no data-path collective; these tests check the
shard arithmetic, the max/sum reductions the benchmark times with, and that
running the oracle path on each rank's token shard and concatenating gives
exactly the unsharded result (so no exchange step is missing).
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from rotation_ptq_b200 import shard as S


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case_reduce(rank, world):
    mx = S.max_over_ranks([rank + 1.5, -rank, 10.0 * rank])
    assert mx == [world + 0.5, 0.0, 10.0 * (world - 1)], mx
    sm = S.sum_over_ranks([1.0, rank])
    assert sm == [float(world), float(sum(range(world)))], sm
    # the benchmark's figure: all ranks' units over the slowest rank's time
    ms = S.max_over_ranks([2.0 + rank])[0]
    units = S.sum_over_ranks([100.0])[0]
    assert S.job_rate(units, ms * 1e-3) == pytest.approx(100.0 * world / ((1.0 + world) * 1e-3))


def _case_sharded_oracle(rank, world, total):
    from oracle import oracle as O
    from workloads import synthetic as W
    K, N = 768, 48                       # H12 x H64 rotation, 12 * 64 = 768
    wl = W.down_proj(M=total, K=K, N=N, seed=4242)
    x = wl.x.double().numpy()
    wp, ws, _ = O.quantize_weights(wl.w.double().numpy(), 12, 64)
    lo, hi = S.token_shard(total, world, rank)
    part = None
    if hi > lo:
        ap, sa, _, _ = O.rotate_quant(x[lo:hi], 12, 64)
        acc, out = O.w4a4_linear(ap, sa, wp, ws)
        part = (lo, hi, ap, sa, acc, out)
    parts = [None] * world
    dist.all_gather_object(parts, part)
    if rank == 0:
        parts = [p for p in parts if p is not None]
        assert [p[0] for p in parts] == sorted(p[0] for p in parts)
        assert sum(p[1] - p[0] for p in parts) == total
        ap, sa, _, _ = O.rotate_quant(x, 12, 64)
        acc, out = O.w4a4_linear(ap, sa, wp, ws)
        assert np.array_equal(np.concatenate([p[2] for p in parts]), ap)
        assert np.array_equal(np.concatenate([p[3] for p in parts]), sa)
        assert np.array_equal(np.concatenate([p[4] for p in parts]), acc)
        assert np.array_equal(np.concatenate([p[5] for p in parts]), out)


def _worker(rank, world, port, case, arg):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        if case == "reduce":
            _case_reduce(rank, world)
        else:
            _case_sharded_oracle(rank, world, arg)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _spawn(case, arg=None, world=2):
    mp.start_processes(_worker, args=(world, _free_port(), case, arg), nprocs=world,
                       join=True, start_method="spawn")


def test_token_shard_covers_disjoint_balanced():
    for total in (0, 1, 2, 7, 4096, 4097):
        for world in (1, 2, 3, 8):
            spans = [S.token_shard(total, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == total
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [hi - lo for lo, hi in spans]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 0
    with pytest.raises(ValueError):
        S.token_shard(8, 2, 2)


def test_reductions_without_a_group_are_identity():
    assert S.max_over_ranks([1.0, 2.0]) == [1.0, 2.0]
    assert S.shard_seed(1001, 0) == 1001 and S.shard_seed(1001, 3) != 1001


def test_gloo_max_and_sum_over_two_ranks():
    _spawn("reduce")


@pytest.mark.parametrize("total", [7, 1])
def test_gloo_token_sharded_oracle_path_is_exact(total):
    # total 7: ragged shards 4 + 3; total 1: rank 1 owns no tokens
    _spawn("sharded_oracle", total)
