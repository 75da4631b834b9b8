"""The multi-rank host logic of bench.py on CPU: two gloo ranks, each timing its own replica;
the reported step time is the slowest rank's and the value is whole-job tokens/s."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    r, w, local = bench.dist_env()
    bench.dist_init(w, local, backend="gloo")
    bench.dist_barrier(w)
    local_ms = 100.0 + 50.0 * r          # rank 1 is the slow one
    ms = bench.dist_max(local_ms, w, device="cpu")
    out[r] = (ms, bench.weak_scaling_value(65536, 10, w, ms))
    bench.dist_done(w)


def test_two_gloo_ranks_take_max_and_weak_scale():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, _free_port() if r < 0 else port, out))
                 for port in [_free_port()] for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0][0] == pytest.approx(150.0) and res[1][0] == pytest.approx(150.0)
    # 2 ranks x 10 steps x 65536 tokens in 150 ms
    assert res[0][1] == pytest.approx(2 * 10 * 65536 / 0.150)


def test_single_rank_is_local():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    assert bench.dist_max(3.5, 1) == 3.5
    assert bench.weak_scaling_value(100, 4, 1, 2000.0) == pytest.approx(200.0)
