"""The prefill entry point that allocates nothing (dr_chunk_fwd_noalloc).

It serves callers that cannot allocate device memory -- runtimes that
pre-plan all device memory and offer a kernel no workspace, or loops that
cannot pay for cudaMalloc/cudaFree -- by keeping its scratch in a static
device array inside the library.  For the cluster-kernel shapes it runs the
two-CTA kernel (the four-CTA kernel's factor staging does not fit the array),
so its results must be the bits of that kernel run through the allocating
entry point (dr_diag_chunk_fwd_variant "ring"), call after call: the shared
array keeps the previous call's contents, so two different problems are run
back to back.  Its device status word is
read back through dr_noalloc_status.  The file is named to be collected last.
"""
import pytest
import torch

from synth import make_inputs, problem

pytestmark = pytest.mark.gpu


def _dev(x):
    return {n: (None if t is None else t.cuda()) for n, t in x.items()}


def test_noalloc_matches_allocating_entry_point_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_recurrence_chunkwise_b200 as dr
    from weight_recurrence_chunkwise_b200 import build

    build.build()
    cases = [problem("kda_bf16", B=2, H=3, T=200),                 # channel gates, S0 given
             problem("gdn_bf16", B=1, H=4, T=333, S0="normal")]    # scalar gates, ragged tail
    for p in cases:
        x = _dev(make_inputs(p))
        args = (x["q"], x["k"], x["v"], x["beta_k"])
        kw = dict(alpha=x["alpha"], beta_v=x["beta_v"], S0=x["S0"], chunk=p.chunk)
        o_ref, S_ref = dr.dr_diag_chunk_fwd_variant("ring", *args, **kw)
        o_new = torch.full_like(o_ref, float("nan"))
        S_new = torch.full_like(S_ref, float("nan"))
        dr.dr_chunk_fwd_noalloc(*args, **kw, o=o_new, S_T=S_new)
        torch.cuda.synchronize()
        assert torch.equal(o_new, o_ref)
        assert torch.equal(S_new, S_ref)
        assert dr.dr_noalloc_status() == dr.DR_OK


def test_noalloc_reports_device_status():
    """A chunk whose cumulative decay leaves the factorised range sets DR_ERR_RANGE in the static
    array's status word, and the next in-range call clears it."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_recurrence_chunkwise_b200 as dr

    p = problem("gdn_bf16", B=1, H=1, T=64)
    x = make_inputs(p)
    x["alpha"] = torch.full_like(x["alpha"], 1e-3)  # sum of log alpha over the chunk ~ -442
    g = _dev(x)
    dr.dr_chunk_fwd_noalloc(g["q"], g["k"], g["v"], g["beta_k"], alpha=g["alpha"], chunk=64)
    assert dr.dr_noalloc_status() == dr.DR_ERR_RANGE
    g2 = _dev(make_inputs(p))
    dr.dr_chunk_fwd_noalloc(g2["q"], g2["k"], g2["v"], g2["beta_k"], alpha=g2["alpha"], chunk=64)
    assert dr.dr_noalloc_status() == dr.DR_OK


def test_noalloc_rejects_invalid_problem_before_launch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_recurrence_chunkwise_b200 as dr

    q = torch.zeros(1, 8, 1, 96, dtype=torch.bfloat16, device="cuda")   # dk = 96 unsupported
    b = torch.zeros(1, 8, 1, device="cuda")
    with pytest.raises(dr.DeltaRuleError) as e:
        dr.dr_chunk_fwd_noalloc(q, q, q, b)
    assert e.value.code == dr.DR_ERR_UNSUPPORTED
