"""World-size-2 replica bookkeeping on CPU (gloo): every rank ends with the
slowest rank's time, the job throughput counts both ranks, and the ranks'
token streams are disjoint."""
import multiprocessing as mp
import os
import socket

import pytest

from bit_expert_ffn_fp32_b200 import replicas


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, local_ms, q):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        slow = replicas.max_over_ranks(local_ms[rank])
        thr = replicas.job_throughput(100, world, slow[0])
        streams = replicas.token_streams(rank, 5)
        q.put((rank, slow, thr, streams))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_agree_on_the_slowest_time():
    world = 2
    local_ms = {0: [10.0, 3.0], 1: [12.5, 2.0]}
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, local_ms, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, slow, thr, streams in res:
        assert slow == [12.5, 3.0]
        assert thr == pytest.approx(2 * 100 / 0.0125)
    s0, s1 = set(res[0][3]), set(res[1][3])
    assert len(s0) == 5 and len(s1) == 5 and not (s0 & s1)


def test_single_process_is_identity():
    assert replicas.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert replicas.job_throughput(4, 1, 2.0) == pytest.approx(2000.0)
    with pytest.raises(ValueError):
        replicas.job_throughput(4, 1, 0.0)
    with pytest.raises(ValueError):
        replicas.token_streams(-1, 3)
