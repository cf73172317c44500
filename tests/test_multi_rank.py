"""Multi-rank host logic of bench.py on CPU (gloo, world_size 2): every rank
draws its own equally shaped batch (weak scaling, no data-path exchange) and
the step time is the max over ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    r, w, _ = bench.dist_env()
    wl = bench.make_workload("cfg1", r)
    t = bench.reduce_max(10.0 + 5.0 * r, w)      # rank-specific "elapsed ms"
    bench.barrier(w)
    q.put((r, t, wl.num_seqs, tuple(wl.query.shape), float(wl.query.sum()),
           sorted(wl.seq_lens.tolist())))
    dist.destroy_process_group()


def test_two_ranks_weak_scaling_and_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    (r0, t0, s0, sh0, sum0, l0), (r1, t1, s1, sh1, sum1, l1) = res
    assert t0 == t1 == 15.0                      # max over ranks
    assert s0 == s1 and sh0 == sh1 and l0 == l1  # same shapes and length mix
    assert sum0 != sum1                          # but a different batch per rank
