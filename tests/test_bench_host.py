"""Host-side logic of bench.py: rank aggregation over two gloo ranks on CPU
(max of time, sum of units), the algorithmic byte count, the argument
defaults."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    bench.barrier()
    t, u = bench.aggregate(10.0 * (rank + 1), 100.0 + rank)
    assert bench.dist_env() == (world, rank, rank)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, t, u))


def test_aggregate_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, t, u in res:
        assert t == 20.0 and u == 201.0


def test_aggregate_single_process_is_identity():
    assert bench.aggregate(3.5, 7.0) == (3.5, 7.0)


def test_algorithmic_bytes_match_hand_count():
    s = bench.workload(4)
    # 4 experts x 7,077,888 + shared 3*4096*1024*2 + router 512*4096*2 + bias 512*4
    # + gamma 4096*2 + x, residual, h_out, y_norm 4*4096*2 + idx, w 2*4*4
    expect = 4 * 7077888 + 25165824 + 4194304 + 2048 + 8192 + 32768 + 32
    assert bench.algorithmic_bytes(s, 1) == expect
    s2 = bench.workload(2)
    assert bench.algorithmic_bytes(s2, 1) == expect - 4 * (7077888 - 3932160)


def test_defaults():
    a = bench.parse_args([])
    assert a.gpus == 1 and a.warmup >= 3 and a.impl == "ours" and a.replicas == 8
