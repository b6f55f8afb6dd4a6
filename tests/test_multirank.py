"""Multi-process host logic of bench.py on CPU (gloo, world size 2):
every rank scans its own independent sessions (reseeded workload, same
shapes) and the timed region's length is the maximum over ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    from long_context_decode_bit_b200 import inputs
    r, wsz, local = bench.dist_env()
    w = bench.rank_workload(inputs.STEP_1M, r)
    bench.barrier()
    t = bench.reduce_max(10.0 + 5.0 * rank)           # this rank's elapsed time
    q = inputs.queries(w, 0, 1)
    out.put((rank, r, wsz, w.seed, w.H, w.n, t, float(q.float().sum())))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_reseed_and_reduce_max():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, rr0, w0, seed0, H0, n0, t0, q0), (r1, rr1, w1, seed1, H1, n1, t1, q1) = res
    assert (rr0, rr1) == (0, 1) and w0 == w1 == 2
    assert (H0, n0) == (H1, n1) == (288, 2 ** 20)      # same shapes on every rank
    assert seed0 != seed1 and q0 != q1                  # independent sessions
    assert t0 == t1 == 15.0                             # max over ranks
