"""Sequence-parallel prefill end to end on the GPU: two gloo ranks, each a process on the one GPU,
each holding one segment of every (b, h) of one sequence.

Every rank runs weight_recurrence_chunkwise_b200.seqpar.seqpar_chunk_fwd with the CUDA prefill and
the CUDA state-map kernel; the one collective step (the all-gather of the affine state maps) goes
through gloo with host staging.  The ranks' kernels never wait on one another -- each rank's work
is independent until the host-side exchange -- so the two processes may share the GPU.  The rank
outputs, concatenated, and every rank's final state must match the float64 oracle run on the whole
sequence, at the bf16 bounds of the parity tests.
"""
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CASES = [("kda_bf16", dict(S0="normal", s_scale="channel"), (257, 190)),
         ("fg2plus_bf16", dict(S0="normal"), (320, 333)),
         ("gdn_bf16", dict(), (64, 1))]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(base, kw, split):
    import sys

    sys.path.insert(0, ROOT)
    from synth import make_inputs, problem

    return make_inputs(problem(base, B=1, H=3, T=sum(split), seed=23, **kw))


def _worker(rank, world, port, case, q):
    import datetime
    import sys

    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        from weight_recurrence_chunkwise_b200 import seqpar

        base, kw, split = case
        x = {k: (None if t is None else t.cuda()) for k, t in _inputs(base, kw, split).items()}
        t0 = sum(split[:rank])
        sl = lambda t: None if t is None else t[:, t0:t0 + split[rank]].contiguous()
        o, S = seqpar.seqpar_chunk_fwd(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["beta_k"]), alpha=sl(x["alpha"]),
                                       beta_v=sl(x["beta_v"]), s=sl(x["s"]), S0=x["S0"])
        torch.cuda.synchronize()
        q.put((rank, o.float().cpu().numpy(), S.cpu().numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_two_ranks_on_one_gpu_split_one_sequence(case):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import oracle
    from tests.test_gpu_parity import OUT_ROUND, TOL, err

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, case, q)) for r in range(2)]
    for pr in procs:
        pr.start()
    res = sorted([q.get(timeout=600) for _ in procs], key=lambda t: t[0])
    for pr in procs:
        pr.join(timeout=120)
        assert pr.exitcode == 0
    x = _inputs(*case)
    ref_o, ref_S = oracle.delta_rule_sequential(x["q"], x["k"], x["v"], x["beta_k"], alpha=x["alpha"],
                                                beta_v=x["beta_v"], S0=x["S0"], s_scale=x["s"])
    o = np.concatenate([r[1] for r in res], axis=1)
    assert err(o, ref_o, OUT_ROUND["bf16"]) <= TOL["bf16"][0]
    for r in res:
        assert err(r[2], ref_S) <= TOL["bf16"][1], r[0]
