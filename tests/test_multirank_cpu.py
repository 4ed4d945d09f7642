"""The replica path of bench.py on two CPU ranks over gloo: every rank decodes
its own seeded batch (no data crosses ranks) and the job's time is the
slowest rank's, taken by an all-reduce MAX.  No GPU is needed."""

import datetime
import hashlib
import os
import socket

import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist

    import bench
    from workloads import WORKLOADS, make_queries
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = bench.rank_shard(WORKLOADS["tiny_4k"], rank)
        digest = hashlib.sha256(make_queries(w).tobytes()).hexdigest()
        digests = [None] * world
        dist.all_gather_object(digests, digest)
        # per-rank timings: the element-wise maximum must come back everywhere
        mine = [1.0 + rank, 5.0 - rank, 0.25 * rank]
        got = bench.max_over_ranks(mine, dist, "cpu", world)
        out.put((rank, got, digests, w.seed))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_and_take_the_slowest():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    results = [out.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
        assert p.exitcode == 0
    results.sort()
    assert [r[1] for r in results] == [[2.0, 5.0, 0.25]] * 2
    digests = results[0][2]
    assert digests == results[1][2] and digests[0] != digests[1]   # distinct batches
    assert results[0][3] != results[1][3]


def test_one_rank_is_identity():
    import bench
    from workloads import WORKLOADS
    w = WORKLOADS["tiny_4k"]
    assert bench.rank_shard(w, 0) is w
    assert bench.max_over_ranks([3.0, 1.5], None, "cpu", 1) == [3.0, 1.5]
