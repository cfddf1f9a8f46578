"""The prefill entry point that allocates nothing (dr_chunk_fwd_noalloc).

It serves callers that cannot allocate device memory -- runtimes that
pre-plan all device memory and offer a kernel no workspace, or loops that
cannot pay for cudaMalloc/cudaFree -- by keeping its scratch in a static
device array inside the library.  Its results must match the allocating
entry point dr_chunk_fwd on the same inputs, call after call: the shared
array keeps the previous call's contents, so two different problems are run
back to back.  The file is named to be collected last.
"""
import numpy as np
import pytest
import torch

from synth import make_inputs, problem

pytestmark = pytest.mark.gpu

OUT_ROUND_BF16 = 2.0 ** -8


def _err(x, ref, round_rel=0.0):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = np.maximum(np.abs(x - ref) - round_rel * np.abs(ref), 0.0)
    return float(d.max() / max(np.sqrt(np.mean(ref ** 2)), 1e-30))


def test_noalloc_matches_allocating_entry_point_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_recurrence_chunkwise_b200 as dr
    from weight_recurrence_chunkwise_b200 import build

    build.build()
    cases = [problem("kda_bf16", B=2, H=3, T=200),                 # channel gates, S0 given
             problem("gdn_bf16", B=1, H=4, T=333, S0="normal")]    # scalar gates, ragged tail
    for p in cases:
        x = {n: (None if t is None else t.cuda()) for n, t in make_inputs(p).items()}
        args = (x["q"], x["k"], x["v"], x["beta_k"])
        kw = dict(alpha=x["alpha"], beta_v=x["beta_v"], S0=x["S0"], chunk=p.chunk)
        o_ref, S_ref = dr.dr_chunk_fwd(*args, **kw)
        o_new = torch.full_like(o_ref, float("nan"))
        S_new = torch.full_like(S_ref, float("nan"))
        dr.dr_chunk_fwd_noalloc(*args, **kw, o=o_new, S_T=S_new)
        torch.cuda.synchronize()
        assert _err(o_new.float().cpu(), o_ref.float().cpu(), 2 * OUT_ROUND_BF16) <= 2e-2
        assert _err(S_new.cpu(), S_ref.cpu()) <= 1e-2
        assert torch.isfinite(o_new.float()).all() and torch.isfinite(S_new).all()


def test_noalloc_rejects_invalid_problem_before_launch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_recurrence_chunkwise_b200 as dr

    q = torch.zeros(1, 8, 1, 96, dtype=torch.bfloat16, device="cuda")   # dk = 96 unsupported
    b = torch.zeros(1, 8, 1, device="cuda")
    with pytest.raises(dr.DeltaRuleError) as e:
        dr.dr_chunk_fwd_noalloc(q, q, q, b)
    assert e.value.code == dr.DR_ERR_UNSUPPORTED
