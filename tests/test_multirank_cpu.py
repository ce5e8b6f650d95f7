"""The multi-rank host logic of bench.py on CPU: two gloo ranks agree on the max-over-ranks step time and
on the whole-job (weak-scaling) throughput."""
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), LOCAL_RANK=str(rank),
                      WORLD_SIZE=str(world))
    import bench

    r, local, w = bench.dist_init("gloo")
    ms = [12.5, 17.25][r]  # rank 1 is the slow one
    mx = bench.reduce_max(ms)
    bench.barrier()
    out[r] = (mx, bench.weak_scaling_value(2 * 32768, w, mx / 1e3))
    import torch.distributed as dist

    dist.destroy_process_group()


def test_two_gloo_ranks_reduce_max_and_weak_scaling():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0] == res[1]
    mx, value = res[0]
    assert mx == 17.25
    assert abs(value - 2 * 2 * 32768 / 0.01725) < 1e-6 * value
