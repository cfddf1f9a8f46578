"""GPU parity of the packed variable-length prefill (dr_chunk_fwd_varlen) and the prefill -> decode
handoff, against the float64 oracle run on each sequence on its own.

Sequences of mixed lengths (empty, one token, around a chunk boundary, several chunks) are laid end
to end; each must match the oracle from its own initial state, with rows past its end inside a chunk
holding the next sequence's tokens.  A packed batch of equal lengths must reproduce the dense batch
bit for bit, and decode steps continuing every sequence from its S_T must match the oracle on the
sequence extended by those tokens.
"""
import numpy as np
import pytest
import torch

import oracle
from synth import make_inputs, problem
from tests.test_gpu_parity import OUT_ROUND, TOL, err, to_dev

pytestmark = pytest.mark.gpu

LENGTHS = [1, 63, 0, 64, 65, 300, 129]


@pytest.fixture(scope="module")
def dr():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_recurrence_chunkwise_b200 as m
    from weight_recurrence_chunkwise_b200 import build

    build.build()
    m.lib()
    return m


def packed_inputs(base, lengths, extra=0, **kw):
    """One input draw per sequence (length + extra tokens), concatenated along T; S0 stacked."""
    seqs = [make_inputs(problem(base, B=1, T=n + extra, seed=1000 + i, **kw)) for i, n in enumerate(lengths)]
    cat = {}
    for name in ("q", "k", "v", "alpha", "beta_k", "beta_v", "s"):
        parts = [x[name][:, :n] for x, n in zip(seqs, lengths)] if seqs[0][name] is not None else None
        cat[name] = None if parts is None else torch.cat(parts, dim=1)
    cat["S0"] = None if seqs[0]["S0"] is None else torch.cat([x["S0"] for x in seqs], dim=0)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    return cat, cu, seqs


def oracle_seq(x, n):
    sl = lambda t: None if t is None else t[:, :n]
    return oracle.delta_rule_sequential(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["beta_k"]), alpha=sl(x["alpha"]),
                                        beta_v=sl(x["beta_v"]), S0=x["S0"], s_scale=sl(x["s"]))


CASES = [
    # (base, overrides)                       kernel
    ("gdn_bf16", dict(S0="normal")),                                          # ring, scalar gates
    ("kda_bf16", dict()),                                                     # ring, channel gates, S0
    ("fg2plus_bf16", dict(S0="normal", s_scale="channel")),                   # ring, beta_v, OSDN scale
    ("kda_bf16", dict(chunk=32)),                                             # CUDA-core kernel, bf16
    ("deltanet_f32", dict(S0="normal")),                                      # CUDA-core kernel, fp32
]


@pytest.mark.parametrize("base,kw", CASES, ids=["gdn", "kda", "fg2plus_osdn", "kda_C32", "deltanet_f32"])
def test_varlen_prefill(dr, base, kw):
    kw = dict(kw)
    chunk = kw.pop("chunk", 64)
    kw["H"] = 2
    x, cu, seqs = packed_inputs(base, LENGTHS, **kw)
    g = to_dev(x)
    o, S_T = dr.dr_chunk_fwd_varlen(g["q"], g["k"], g["v"], g["beta_k"], cu.cuda(), alpha=g["alpha"],
                                    beta_v=g["beta_v"], s=g["s"], S0=g["S0"], chunk=chunk)
    torch.cuda.synchronize()
    io = problem(base).io
    to, ts = TOL[io]
    for i, n in enumerate(LENGTHS):
        ref_o, ref_S = oracle_seq(seqs[i], n)
        e_S = err(S_T[i:i + 1].cpu().numpy(), ref_S)
        assert e_S <= ts, (i, n, e_S)
        if n:
            got = o[:, int(cu[i]):int(cu[i + 1])].float().cpu().numpy()
            e_o = err(got, ref_o, OUT_ROUND[io])
            assert e_o <= to, (i, n, e_o)


@pytest.mark.parametrize("base,chunk", [("gdn_bf16", 64), ("kda_bf16", 64), ("deltanet_f32", 64)])
def test_varlen_equal_lengths_match_dense_batch(dr, base, chunk):
    """Equal lengths: the packed call is the dense call, bit for bit (rows past each end are inert)."""
    p = problem(base, B=3, H=2, T=200, S0="normal", seed=7)
    g = to_dev(make_inputs(p))
    o_d, S_d = dr.dr_chunk_fwd(g["q"], g["k"], g["v"], g["beta_k"], alpha=g["alpha"], beta_v=g["beta_v"],
                               S0=g["S0"], chunk=chunk)
    pk = lambda t: None if t is None else t.reshape((1, -1) + tuple(t.shape[2:])).contiguous()
    cu = torch.tensor([0, 200, 400, 600], dtype=torch.int32, device="cuda")
    o_p, S_p = dr.dr_chunk_fwd_varlen(pk(g["q"]), pk(g["k"]), pk(g["v"]), pk(g["beta_k"]), cu, alpha=pk(g["alpha"]),
                                      beta_v=pk(g["beta_v"]), S0=g["S0"], chunk=chunk)
    torch.cuda.synchronize()
    assert torch.equal(o_p.reshape(o_d.shape), o_d) and torch.equal(S_p, S_d)


def test_varlen_prefill_then_decode_handoff(dr):
    """Packed prefill of each prompt, then three decode steps continuing every sequence from S_T."""
    lengths, steps = [5, 64, 130, 1], 3
    x, cu, seqs = packed_inputs("kda_bf16", lengths, extra=steps, H=2)
    g = to_dev(x)
    o, S = dr.dr_chunk_fwd_varlen(g["q"], g["k"], g["v"], g["beta_k"], cu.cuda(), alpha=g["alpha"], S0=g["S0"])
    outs = []
    for t in range(steps):
        tok = lambda name: torch.cat([seqs[i][name][:, n + t:n + t + 1] for i, n in enumerate(lengths)], 0).cuda()
        outs.append(dr.dr_decode_step(tok("q"), tok("k"), tok("v"), tok("beta_k"), S, alpha=tok("alpha")))
    torch.cuda.synchronize()
    for i, n in enumerate(lengths):
        ref_o, ref_S = oracle_seq(seqs[i], n + steps)
        got = torch.stack([outs[t][i, 0] for t in range(steps)]).float().cpu().numpy()  # [steps, H, dv]
        assert err(got, ref_o[0, n:], OUT_ROUND["bf16"]) <= TOL["bf16"][0]
        assert err(S[i:i + 1].cpu().numpy(), ref_S) <= TOL["bf16"][1]


def test_varlen_requires_offsets(dr):
    p = problem("gdn_bf16", B=1, H=2, T=64, seed=3)
    g = to_dev(make_inputs(p))
    with pytest.raises(ValueError):
        dr.dr_chunk_fwd_varlen(g["q"], g["k"], g["v"], g["beta_k"], torch.tensor([0, 64], device="cuda"),
                               alpha=g["alpha"])  # int64 offsets
