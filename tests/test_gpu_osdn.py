"""GPU parity of OSDN's write-side key scaling (write key a = s * b, erase key b) against the oracle.

Covers the tensor-core ring kernel (scalar and channel gates, decoupled write strength, ragged
lengths, many chunks), the CUDA-core kernel (fp32 I/O; bf16 shapes the ring kernel does not take),
the decode step chained over a short sequence, and the plumbing check that s = 1 reproduces the
entry points without s bit for bit.
"""
import zlib

import numpy as np
import pytest
import torch

import oracle
from synth import make_inputs, problem
from tests.test_gpu_parity import OUT_ROUND, TOL, check, err, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dr():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_recurrence_chunkwise_b200 as m
    from weight_recurrence_chunkwise_b200 import build

    build.build()
    m.lib()
    return m


def ref(x):
    return oracle.delta_rule_sequential(x["q"], x["k"], x["v"], x["beta_k"], alpha=x["alpha"], beta_v=x["beta_v"],
                                        S0=x["S0"], s_scale=x["s"])


PREFILL = [
    # (base, B, H, T, dk, dv, chunk, io, alpha, beta_k, beta_v, S0)
    ("gdn_bf16", 1, 3, 200, 128, 128, 64, "bf16", "scalar", "scalar", "none", "normal"),
    ("gdn_bf16", 1, 2, 2048, 128, 128, 64, "bf16", "scalar", "scalar", "none", "zero"),
    ("gdn_bf16", 2, 2, 63, 128, 128, 64, "bf16", "none", "scalar", "scalar", "normal"),
    ("kda_bf16", 1, 3, 333, 128, 128, 64, "bf16", "channel", "channel", "none", "normal"),
    ("kda_bf16", 1, 2, 517, 128, 128, 64, "bf16", "channel", "channel", "channel", "zero"),
    ("kda_bf16", 1, 2, 130, 128, 128, 32, "bf16", "channel", "channel", "none", "normal"),
    ("kda_bf16", 1, 2, 150, 128, 64, 64, "bf16", "scalar", "channel", "channel", "normal"),
    ("deltanet_f32", 1, 2, 150, 64, 64, 64, "f32", "none", "scalar", "none", "normal"),
    ("kda_bf16", 1, 2, 77, 128, 128, 16, "f32", "channel", "channel", "channel", "zero"),
]


@pytest.mark.parametrize("case", PREFILL, ids=lambda c: "{}_T{}_dk{}_dv{}_C{}_{}_a{}_bk{}_bv{}".format(
    c[0], c[3], c[4], c[5], c[6], c[7], c[8], c[9], c[10]))
def test_osdn_prefill(dr, case):
    base, B, H, T, dk, dv, C, io, a, bk, bv, s0 = case
    p = problem(base, B=B, H=H, T=T, dk=dk, dv=dv, chunk=C, io=io, alpha=a, beta_k=bk, beta_v=bv, S0=s0,
                s_scale="channel", seed=zlib.crc32(repr(case).encode()) % 1000)
    x = make_inputs(p)
    g = to_dev(x)
    o, S_T = dr.dr_chunk_fwd_osdn(g["q"], g["k"], g["v"], g["beta_k"], g["s"], alpha=g["alpha"],
                                  beta_v=g["beta_v"], S0=g["S0"], chunk=C)
    torch.cuda.synchronize()
    ref_o, ref_S = ref(x)
    check(p, o, S_T, ref_o, ref_S)


@pytest.mark.parametrize("base,C,io", [("gdn_bf16", 64, "bf16"), ("kda_bf16", 64, "bf16"), ("kda_bf16", 32, "bf16"),
                                       ("deltanet_f32", 64, "f32")])
def test_osdn_unit_scale_equals_plain_entry_point(dr, base, C, io):
    """s = 1 goes through the scaled code and must give exactly the result without s."""
    dk = 64 if io == "f32" else 128
    p = problem(base, B=1, H=2, T=200, dk=dk, dv=dk, chunk=C, io=io, S0="normal", s_scale="channel", seed=11)
    g = to_dev(make_inputs(p))
    ones = torch.ones_like(g["s"])
    o1, S1 = dr.dr_chunk_fwd_osdn(g["q"], g["k"], g["v"], g["beta_k"], ones, alpha=g["alpha"], beta_v=g["beta_v"],
                                  S0=g["S0"], chunk=C)
    o0, S0 = dr.dr_chunk_fwd(g["q"], g["k"], g["v"], g["beta_k"], alpha=g["alpha"], beta_v=g["beta_v"], S0=g["S0"],
                             chunk=C)
    torch.cuda.synchronize()
    assert torch.equal(o1, o0) and torch.equal(S1, S0)


@pytest.mark.parametrize("beta_v", ["none", "channel"])
def test_osdn_decode_chain(dr, beta_v):
    """Eight chained decode steps with s equal the oracle's recurrence over those eight tokens."""
    p = problem("kda_bf16", B=3, H=4, T=8, beta_v=beta_v, S0="normal", s_scale="channel", seed=21)
    x = make_inputs(p)
    g = to_dev(x)
    S = g["S0"].clone()
    outs = []
    for t in range(p.T):
        sl = lambda z: None if z is None else z[:, t:t + 1].contiguous()
        outs.append(dr.dr_decode_step_osdn(sl(g["q"]), sl(g["k"]), sl(g["v"]), sl(g["beta_k"]), S, sl(g["s"]),
                                           alpha=sl(g["alpha"]), beta_v=sl(g["beta_v"])))
    torch.cuda.synchronize()
    o = torch.cat(outs, dim=1)
    ref_o, ref_S = ref(x)
    e_o = err(o.float().cpu().numpy(), ref_o, OUT_ROUND["bf16"])
    e_S = err(S.cpu().numpy(), ref_S)
    # the decode step is the recurrence itself in fp32: far inside the chunkwise bounds
    assert e_o <= 1e-2 and e_S <= 1e-4, (e_o, e_S)


def test_osdn_decode_unit_scale_equals_plain(dr):
    p = problem("kda_bf16", B=2, H=3, T=1, S0="normal", s_scale="channel", seed=5)
    g = to_dev(make_inputs(p))
    S_a, S_b = g["S0"].clone(), g["S0"].clone()
    o_a = dr.dr_decode_step_osdn(g["q"], g["k"], g["v"], g["beta_k"], S_a, torch.ones_like(g["s"]), alpha=g["alpha"])
    o_b = dr.dr_decode_step(g["q"], g["k"], g["v"], g["beta_k"], S_b, alpha=g["alpha"])
    torch.cuda.synchronize()
    assert torch.equal(o_a, o_b) and torch.equal(S_a, S_b)


def test_osdn_rejects_misshaped_scale(dr):
    p = problem("gdn_bf16", B=1, H=2, T=64, s_scale="channel", seed=3)
    g = to_dev(make_inputs(p))
    with pytest.raises(ValueError):
        dr.dr_chunk_fwd_osdn(g["q"], g["k"], g["v"], g["beta_k"], g["s"][:, :, :, :64].contiguous(),
                             alpha=g["alpha"])
