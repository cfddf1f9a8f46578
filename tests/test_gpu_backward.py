"""GPU parity of the backward pass (dr_backward) against the float64 autograd reference.

Every gradient -- q, k, v, the gates, OSDN's scale and the initial state -- in every gate mode,
with ragged lengths across the recomputation spans and the chunks, fp32 and bf16 I/O, and both head
sizes.  Error measure as for the forward: max |g - g_ref| / rms(g_ref) per tensor.  The bounds follow
the forward's precision classes: the token-sequential kernel computes in fp32 throughout (2e-4); the
chunkwise kernel, the library's choice for bf16 I/O with dk = dv = 128, multiplies fp16 operands on
the tensor cores (the forward's bf16 bound, 2e-2).
"""
import zlib

import numpy as np
import pytest
import torch

from oracle import backward as ob
from synth import make_inputs, problem
from tests.test_gpu_parity import err, to_dev

pytestmark = pytest.mark.gpu

TOL_SEQ, TOL_CHUNK = 2e-4, 2e-2

CASES = [
    # (base, T, dk, dv, io, alpha, beta_k, beta_v, s)
    ("gdn_bf16", 200, 128, 128, "bf16", "scalar", "scalar", "none", "none"),     # four chunks, ragged
    ("kda_bf16", 130, 128, 128, "bf16", "channel", "channel", "none", "none"),
    ("fg2plus_bf16", 256, 128, 128, "bf16", "channel", "channel", "channel", "channel"),
    ("gdn_bf16", 77, 128, 128, "bf16", "scalar", "scalar", "none", "none"),
    ("gdn_bf16", 1, 128, 128, "bf16", "none", "scalar", "none", "none"),
    ("kda_bf16", 100, 128, 128, "bf16", "channel", "channel", "none", "channel"),
    ("fg2plus_bf16", 65, 128, 128, "bf16", "channel", "channel", "channel", "none"),
    ("kda_bf16", 96, 128, 64, "bf16", "scalar", "channel", "scalar", "channel"),
    ("deltanet_f32", 70, 64, 64, "f32", "none", "scalar", "none", "none"),
    ("kda_bf16", 33, 64, 128, "f32", "channel", "scalar", "channel", "none"),
]


@pytest.fixture(scope="module")
def dr():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_recurrence_chunkwise_b200 as m
    from weight_recurrence_chunkwise_b200 import build

    build.build()
    m.lib()
    return m


def _chunk_path(case):
    _, _, dk, dv, io, _, _, _, _ = case
    return io == "bf16" and dk == 128 and dv == 128


@pytest.mark.parametrize("variant", ["default", "sequential"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "{}_T{}_dk{}_dv{}_{}_a{}_bk{}_bv{}_s{}".format(*c))
def test_backward_matches_reference(dr, case, variant):
    base, T, dk, dv, io, a, bk, bv, sc = case
    p = problem(base, B=2, H=2, T=T, dk=dk, dv=dv, io=io, alpha=a, beta_k=bk, beta_v=bv, S0="normal",
                s_scale=sc, seed=zlib.crc32(repr(case).encode()) % 1000)
    x = make_inputs(p)
    rng = np.random.default_rng(1)
    do = torch.from_numpy(rng.standard_normal((p.B, p.T, p.H, dv)).astype(np.float32)).to(x["v"].dtype)
    dST = torch.from_numpy(rng.standard_normal((p.B, p.H, dk, dv)).astype(np.float32))
    g = to_dev(x)
    got = dr.dr_diag_backward_variant(variant, g["q"], g["k"], g["v"], g["beta_k"], do.cuda(), alpha=g["alpha"],
                                      beta_v=g["beta_v"], s=g["s"], S0=g["S0"], dS_T=dST.cuda())
    torch.cuda.synchronize()
    ref = ob.backward(x["q"], x["k"], x["v"], x["beta_k"], do, alpha=x["alpha"], beta_v=x["beta_v"], S0=x["S0"],
                      s_scale=x["s"], dS_T=dST)
    names = {"q": "q", "k": "k", "v": "v", "beta_k": "beta_k", "alpha": "alpha", "beta_v": "beta_v",
             "s": "s_scale", "S0": "S0"}
    for mine, theirs in names.items():
        if ref[theirs] is None:
            assert got[mine] is None
            continue
        e = err(got[mine].cpu().numpy(), ref[theirs].numpy())
        tol = TOL_CHUNK if (variant == "default" and _chunk_path(case)) else TOL_SEQ
        assert e <= tol, (mine, e)


def test_backward_without_final_state_gradient(dr):
    """dS_T omitted means zero; dS0 not requested is skipped."""
    p = problem("gdn_bf16", B=1, H=2, T=40, S0="normal", seed=9)
    x = make_inputs(p)
    do = torch.randn(p.B, p.T, p.H, p.dv, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16)
    g = to_dev(x)
    got = dr.dr_backward(g["q"], g["k"], g["v"], g["beta_k"], do.cuda(), alpha=g["alpha"], S0=g["S0"], want_dS0=False)
    torch.cuda.synchronize()
    ref = ob.backward(x["q"], x["k"], x["v"], x["beta_k"], do, alpha=x["alpha"], S0=x["S0"])
    assert got["S0"] is None
    assert err(got["v"].cpu().numpy(), ref["v"].numpy()) <= TOL_CHUNK
    assert err(got["alpha"].cpu().numpy(), ref["alpha"].numpy()) <= TOL_CHUNK


@pytest.mark.parametrize("base", ["gdn_bf16", "kda_bf16"])
def test_backward_workload_full_size(dr, base):
    """The backward at the workload's full size, in the launch configuration ``bench.py --backward``
    times, checked two ways:

    * Linearity, over the whole batch.  With the gates and keys fixed, o and S_T are linear in
      (v, S0) jointly and o is linear in q, so for L = sum(do o) + sum(dS_T S_T)
          <dv, v> + <dS0, S0> = L   and   <dq, q> = sum(do o),
      with o and S_T from the forward kernel.  The forward's bf16 output rounding (2^-9 relative)
      bounds the mismatch by 5e-3 of sum |do o| + sum |dS_T S_T|.
    * One sampled head (the last (b, h), whose gradients depend on that head's inputs alone)
      against the float64 reference, to the bound of the kernel the library runs here (the
      chunkwise one: 2e-2 of each gradient's RMS; GDN only: the reference needs about ten seconds
      per 4096 tokens).
    """
    p = problem(base, S0="normal")
    x = make_inputs(p)
    g = to_dev(x)
    gen = torch.Generator().manual_seed(5)
    do = torch.randn(x["v"].shape, generator=gen).to(x["v"].dtype)
    dST = torch.randn((p.B, p.H, p.dk, p.dv), generator=gen)
    do_d, dST_d = do.cuda(), dST.cuda()
    got = dr.dr_backward(g["q"], g["k"], g["v"], g["beta_k"], do_d, alpha=g["alpha"], beta_v=g["beta_v"], s=g["s"],
                         S0=g["S0"], dS_T=dST_d)
    o, S_T = dr.dr_chunk_fwd(g["q"], g["k"], g["v"], g["beta_k"], alpha=g["alpha"], beta_v=g["beta_v"], S0=g["S0"],
                             chunk=p.chunk)
    torch.cuda.synchronize()
    f64 = lambda t: t.double()
    Lo = (f64(do_d) * f64(o)).sum()
    LS = (f64(dST_d) * f64(S_T)).sum()
    scale = float((f64(do_d) * f64(o)).abs().sum() + (f64(dST_d) * f64(S_T)).abs().sum())
    lin_v = float((got["v"].double() * f64(g["v"])).sum() + (got["S0"].double() * f64(g["S0"])).sum())
    lin_q = float((got["q"].double() * f64(g["q"])).sum())
    assert abs(lin_v - float(Lo + LS)) <= 5e-3 * scale, (lin_v, float(Lo + LS), scale)
    assert abs(lin_q - float(Lo)) <= 5e-3 * scale, (lin_q, float(Lo), scale)

    if base != "gdn_bf16":
        return
    b, h = p.B - 1, p.H - 1
    one = lambda t: None if t is None else t[b:b + 1, :, h:h + 1]
    ref = ob.backward(one(x["q"]), one(x["k"]), one(x["v"]), one(x["beta_k"]), one(do), alpha=one(x["alpha"]),
                      beta_v=one(x["beta_v"]), S0=x["S0"][b:b + 1, h:h + 1], s_scale=one(x["s"]),
                      dS_T=dST[b:b + 1, h:h + 1])
    pick = {"q": one, "k": one, "v": one, "beta_k": one, "alpha": one, "beta_v": one,
            "S0": lambda t: t[b:b + 1, h:h + 1]}
    names = {"q": "q", "k": "k", "v": "v", "beta_k": "beta_k", "alpha": "alpha", "beta_v": "beta_v", "S0": "S0"}
    for mine, theirs in names.items():
        if ref[theirs] is None:
            continue
        e = err(pick[mine](got[mine]).cpu().numpy(), ref[theirs].numpy())
        assert e <= TOL_CHUNK, (mine, e)
