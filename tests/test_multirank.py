"""The multi-GPU path of bench.py on the CPU: two gloo ranks (spawned processes) run the same
plumbing torchrun drives on GPUs — process group from the environment, barrier, max over ranks of
each rank's time, weak-scaling aggregate, and independent seeded inputs per rank.  The path has
no data-path collective: each rank solves its own problems."""
import multiprocessing as _mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import synthetic
    r = bench.Ranks.from_env("gloo")
    r.barrier()
    local_ms = 10.0 + 3.0 * rank           # this rank's timed region
    m = r.max(local_ms)
    thr = bench.weak_scaling_throughput(r.world, 5, 2.0e9, m)
    w = synthetic.WORKLOADS["mha_causal"]
    x = synthetic.normal_bf16(w.seed(0) + bench.rank_seed_offset(rank), (16,))
    r.barrier()
    r.close()
    out.put((rank, r.world, m, thr, x.tolist()))


@pytest.mark.parametrize("world", [2])
def test_two_gloo_ranks(world):
    ctx = _mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    slowest = 10.0 + 3.0 * (world - 1)
    for rank, w, m, thr, _ in res:
        assert w == world
        assert m == slowest                                  # every rank reports the max
        assert thr == pytest.approx(world * 5 * 2.0e9 / (slowest * 1e-3))
    # each rank drew its own inputs
    assert res[0][4] != res[1][4]


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    r = bench.Ranks(1, 0, 0, "gloo")
    assert r.dist is None
    assert r.max(4.5) == 4.5
    r.barrier()
    r.close()
    assert bench.weak_scaling_throughput(1, 10, 3.0, 2.0) == pytest.approx(15000.0)
