"""Failure detection on the GPU, without a fault.

Every wait in the prefill kernels is bounded: after its wall-time limit it gives up, records a
timeout bit in the workspace status word and lets the kernel exit.  dr_diag_wait_timeout runs those
same wait helpers on an mbarrier that nothing completes (CTA scope on one CTA; cluster-scope acquire
on a cluster of two), with a short limit.  The host must read DR_ERR_TIMEOUT, each CTA must have
waited at least the limit and not much longer, and the context must stay usable: a prefill right
after still matches the oracle and reports DR_OK.
"""
import pytest
import torch

import oracle
from synth import make_inputs, problem
from tests.test_gpu_parity import OUT_ROUND, TOL, err, to_dev

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


@pytest.mark.parametrize("cluster", [False, True], ids=["cta", "cluster"])
def test_bounded_wait_times_out_and_reports(dr, cluster):
    limit = 20_000_000  # 20 ms
    status, waited = dr.dr_diag_wait_timeout(cluster, limit)
    assert status == dr.DR_ERR_TIMEOUT
    assert len(waited) == (2 if cluster else 1)
    assert all(limit <= w < limit + 500_000_000 for w in waited), waited

    # the context is still usable
    p = problem("kda_bf16", B=1, H=2, T=100, S0="normal", seed=3)
    x = make_inputs(p)
    g = to_dev(x)
    ws = torch.zeros(dr.workspace_bytes(dr.make_problem(g["q"], g["v"], g["alpha"], g["beta_k"], g["beta_v"], 64)),
                     dtype=torch.uint8, device="cuda")
    o, S_T = dr.dr_chunk_fwd(g["q"], g["k"], g["v"], g["beta_k"], alpha=g["alpha"], S0=g["S0"], workspace=ws)
    assert dr.dr_workspace_status(ws) == dr.DR_OK
    ref_o, ref_S = oracle.delta_rule_sequential(x["q"], x["k"], x["v"], x["beta_k"], alpha=x["alpha"], S0=x["S0"])
    assert err(o.float().cpu().numpy(), ref_o, OUT_ROUND["bf16"]) <= TOL["bf16"][0]
    assert err(S_T.cpu().numpy(), ref_S) <= TOL["bf16"][1]


def test_wait_limit_is_validated(dr):
    with pytest.raises(dr.DeltaRuleError):
        dr.dr_diag_wait_timeout(False, 0)
    with pytest.raises(dr.DeltaRuleError):
        dr.dr_diag_wait_timeout(True, 2_000_000_000)  # above the one-second cap
