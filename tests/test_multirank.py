"""The replica path of bench.py on two ranks (gloo, CPU): each rank decodes its
own batch, ranks meet only at barriers and in the max over ranks of the device
times, and the job rate divides all ranks' tokens by the slowest rank's time."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    r, w, local = bench.dist_setup(world, backend="gloo")
    bench.barrier(w)
    elapsed = 1.0 + 0.5 * r                 # rank 1 is the slower one
    emax = bench.max_over_ranks(elapsed, w, torch.device("cpu"))
    rate = bench.job_throughput(w, 4096, 10, emax)
    bench.barrier(w)
    torch.distributed.destroy_process_group()
    q.put((r, w, local, emax, rate))


def test_two_rank_replicas_take_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[0] for o in out] == [0, 1] and all(o[1] == 2 for o in out)
    assert all(o[3] == pytest.approx(1.5) for o in out)          # slowest rank's time on both
    assert all(o[4] == pytest.approx(2 * 4096 * 10 / 1.5) for o in out)


def test_world_size_must_match_gpus(monkeypatch):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    with pytest.raises(SystemExit):
        bench.dist_setup(1)
