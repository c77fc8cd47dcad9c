"""The N > 1 bench path on CPU: two gloo ranks (no GPU).  Every rank indexes
its own chunk of the same shape (same keys, its own query permutation), the
timing is the maximum over ranks, and the whole-job value divides it by the
number of ranks; no collective touches the data path."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench
    from long_context_sparse_block_b200 import workloads as W
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        inp = W.generate(W.WORKLOADS["tiny_1k"])
        mine = bench.rank_inputs(inp, rank, world)
        got = [None] * world
        dist.all_gather_object(got, (mine["Q"].tobytes(), mine["w"].tobytes()))
        t_max = bench.max_over_ranks(1.5 + rank, "cpu")     # rank r "took" 1.5 + r ms
        q.put((rank, got, t_max, bench.whole_job_ms(t_max, world),
               mine["K"].tobytes() == inp["K"].tobytes(),
               sorted(map(tuple, mine["Q"].reshape(mine["Q"].shape[0], -1).tolist()))
               == sorted(map(tuple, inp["Q"].reshape(inp["Q"].shape[0], -1).tolist()))))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_index_their_own_chunks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, got, t_max, whole, same_keys, same_queries in res:
        assert t_max == pytest.approx(1.5 + (world - 1))     # the slowest rank
        assert whole == pytest.approx(t_max / world)
        assert same_keys                                     # the keys are shared
        assert same_queries                                  # a permutation of the chunk's queries
        assert got[0] != got[1]                              # but a different order per rank
    assert res[0][1] == res[1][1]                            # both ranks saw the same exchange


def test_single_rank_is_unchanged():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from long_context_sparse_block_b200 import workloads as W
    inp = W.generate(W.WORKLOADS["tiny_1k"])
    assert bench.rank_inputs(inp, 0, 1) is inp
    assert bench.max_over_ranks(2.5, "cpu") == 2.5
    assert bench.whole_job_ms(2.5, 1) == 2.5
    assert np.array_equal(inp["Q"], W.generate(W.WORKLOADS["tiny_1k"])["Q"])
