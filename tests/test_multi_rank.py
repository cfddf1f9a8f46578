"""The multi-GPU path on CPU: two gloo ranks exercise bench.py's rank logic.

Each (b, h) is an independent recurrence, so ranks shard the batch with no
exchange on the data path; the only collectives are the barrier and the
max-over-ranks of the timings.  The test checks that the max is taken across
ranks, that ranks get distinct seeded batches, and that a rank's result does
not depend on the other rank (it equals a single-process run of its shard).
"""
import multiprocessing as mp
import os
import socket

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _shard(p):
    return p.replace(B=1, H=2, T=40)


def _worker(rank, world, port, q):
    import sys

    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    import oracle
    from synth import make_inputs

    ws, r, _ = bench.dist_env()
    m = bench.max_over_ranks(10.0 * (rank + 1), ws, torch.device("cpu"))
    p = _shard(bench.rank_problem(r))
    x = make_inputs(p)
    o, S = oracle.delta_rule_sequential(x["q"], x["k"], x["v"], x["beta_k"], alpha=x["alpha"],
                                        beta_v=x["beta_v"], S0=x["S0"], threads=1)
    bench.barrier(ws)
    q.put((rank, ws, m, p.seed, o, S))
    dist.destroy_process_group()


def test_two_gloo_ranks_shard_without_exchange():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for pr in procs:
        pr.start()
    res = sorted([q.get(timeout=300) for _ in procs], key=lambda t: t[0])
    for pr in procs:
        pr.join(timeout=120)
        assert pr.exitcode == 0
    assert [r[1] for r in res] == [2, 2]
    assert all(r[2] == 20.0 for r in res)          # max over ranks, seen by both
    assert res[0][3] != res[1][3]                  # distinct seeded batches
    import sys

    sys.path.insert(0, ROOT)
    import bench
    import oracle
    from synth import make_inputs

    for rank, _, _, seed, o, S in res:
        x = make_inputs(_shard(bench.rank_problem(rank)))
        o1, S1 = oracle.delta_rule_sequential(x["q"], x["k"], x["v"], x["beta_k"], alpha=x["alpha"],
                                              beta_v=x["beta_v"], S0=x["S0"], threads=1)
        np.testing.assert_array_equal(o, o1)
        np.testing.assert_array_equal(S, S1)
