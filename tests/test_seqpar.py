"""Sequence-parallel prefill on the CPU: two gloo ranks, each holding one segment of T.

The ranks run weight_recurrence_chunkwise_b200.seqpar with the float64 oracle standing in for the
prefill kernel and a float64 product for the map composition, so the test checks the algebra and the
collective step (one all-gather of the affine state maps) without a GPU.  Each rank's outputs and the
composed final state must equal the oracle run on the whole sequence.
"""
import multiprocessing as mp
import os
import socket

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SPLIT = (37, 70)  # segment lengths of ranks 0 and 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_prefill(q, k, v, beta_k, alpha=None, beta_v=None, s=None, S0=None, chunk=64):
    import oracle

    o, S = oracle.delta_rule_sequential(q, k, v, beta_k, alpha=alpha, beta_v=beta_v, S0=S0, s_scale=s, threads=1)
    return torch.from_numpy(o), torch.from_numpy(S)


def _f64_apply(M, S, N):
    return torch.matmul(M.double(), S.double()) + N.double()


def _inputs():
    import sys

    sys.path.insert(0, ROOT)
    from synth import make_inputs, problem

    return make_inputs(problem("kda_bf16", B=2, H=2, T=sum(SPLIT), dk=8, dv=6, S0="normal", beta_v="channel",
                               s_scale="channel", seed=5))


def _worker(rank, world, port, q):
    import sys

    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from weight_recurrence_chunkwise_b200 import seqpar

    x = _inputs()
    t0 = sum(SPLIT[:rank])
    sl = lambda t: None if t is None else t[:, t0:t0 + SPLIT[rank]].contiguous()
    o, S = seqpar.seqpar_chunk_fwd(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["beta_k"]), alpha=sl(x["alpha"]),
                                   beta_v=sl(x["beta_v"]), s=sl(x["s"]), S0=x["S0"].double(),
                                   prefill=_oracle_prefill, apply=_f64_apply)
    q.put((rank, o.numpy(), S.numpy()))
    dist.destroy_process_group()


def test_two_ranks_split_one_sequence():
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
    import sys

    sys.path.insert(0, ROOT)
    import oracle

    x = _inputs()
    o_ref, S_ref = oracle.delta_rule_sequential(x["q"], x["k"], x["v"], x["beta_k"], alpha=x["alpha"],
                                                beta_v=x["beta_v"], S0=x["S0"], s_scale=x["s"], threads=1)
    o = np.concatenate([r[1] for r in res], axis=1)
    np.testing.assert_allclose(o, o_ref, rtol=1e-10, atol=1e-12)
    for r in res:  # every rank holds the whole sequence's final state
        np.testing.assert_allclose(r[2], S_ref, rtol=1e-10, atol=1e-12)
