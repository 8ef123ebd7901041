"""The multi-rank host path of bench.py on CPU: two gloo ranks, as torchrun
would start them (RANK / WORLD_SIZE / LOCAL_RANK, rendezvous on 127.0.0.1).

The layer shards by tokens with no exchange step (replicas only): each rank
draws its own token shard, the step time is the maximum over ranks, and the
job's throughput counts every rank's tokens."""
import datetime
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r, ws, lr = bench.dist_env()
        step_ms = 0.040 + 0.010 * rank  # rank 1 is the slower one
        slowest = bench.max_over_ranks(step_ms)
        w = bench.wl.WORKLOADS["tiny"]
        inp = bench.wl.make_inputs(w.name, T=16, seed=bench.rank_seed(w, rank))
        out[rank] = (r, ws, lr, slowest, bench.job_tokens_per_s(ws, w.T, slowest), inp.x.copy(), inp.logits.copy())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_disjoint_shards():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        codes = [p.exitcode for p in procs]
        res = dict(out)
    assert codes == [0, 0], codes
    import bench
    tiny_T = bench.wl.WORKLOADS["tiny"].T
    for rank in range(world):
        r, ws, lr, slowest, tps, _, _ = res[rank]
        assert (r, ws, lr) == (rank, world, rank)
        assert slowest == pytest.approx(0.050)  # every rank sees the slowest rank's time
        assert tps == pytest.approx(world * tiny_T / 0.050e-3)
    # each rank routes its own tokens
    assert not np.array_equal(res[0][5], res[1][5])
    assert not np.array_equal(res[0][6], res[1][6])


def test_single_process_needs_no_group():
    import bench
    assert bench.max_over_ranks(0.25) == 0.25
    assert bench.job_tokens_per_s(1, 4096, 0.04) == pytest.approx(4096 / 0.04e-3)
