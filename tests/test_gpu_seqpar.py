"""GPU parts of the sequence-parallel prefill: the affine state-map kernel, and a split of one sequence
into segments emulated on one GPU (maps by the prefill kernel, composition by dr_state_map_apply, one
prefill per segment from its composed initial state) against the oracle on the whole sequence.
The collective step itself is covered on CPU ranks in test_seqpar.py.
"""
import numpy as np
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


@pytest.mark.parametrize("n,dk,dv,with_S", [(5, 128, 128, True), (3, 64, 96, True), (4, 128, 64, False)])
def test_state_map_apply(dr, n, dk, dv, with_S):
    g = torch.Generator().manual_seed(n * 100 + dk + dv)
    M = torch.randn(n, dk, dk, generator=g) / dk ** 0.5
    S = torch.randn(n, dk, dv, generator=g) if with_S else None
    N = torch.randn(n, dk, dv, generator=g)
    out = dr.dr_state_map_apply(M.cuda(), N.cuda(), S=None if S is None else S.cuda())
    torch.cuda.synchronize()
    ref = N.double() + (M.double() @ S.double() if S is not None else 0)
    np.testing.assert_allclose(out.cpu().double().numpy(), ref.numpy(), rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("base,kw,split", [
    ("gdn_bf16", dict(S0="normal"), (300, 257, 343)),
    ("kda_bf16", dict(s_scale="channel"), (64, 191, 128, 100)),
    ("fg2plus_bf16", dict(S0="normal"), (500, 500)),
])
def test_split_sequence_emulated(dr, base, kw, split):
    from weight_recurrence_chunkwise_b200 import seqpar

    p = problem(base, B=1, H=3, T=sum(split), seed=17, **kw)
    x = make_inputs(p)
    g = to_dev(x)
    bounds = np.concatenate([[0], np.cumsum(split)])
    # each segment in its own allocation, as a rank would hold it (the library wants 16-byte aligned arrays)
    seg = lambda t, i: None if t is None else t[:, bounds[i]:bounds[i + 1]].clone()
    args = lambda i: dict(alpha=seg(g["alpha"], i), beta_v=seg(g["beta_v"], i), s=seg(g["s"], i))
    maps = [seqpar.segment_map(seg(g["q"], i), seg(g["k"], i), seg(g["v"], i), seg(g["beta_k"], i), **args(i))
            for i in range(len(split))]
    outs, S_final = [], None
    for i in range(len(split)):
        S_in = seqpar.compose(maps[:i], g["S0"])
        o, S_seg = seqpar._cuda_prefill(seg(g["q"], i), seg(g["k"], i), seg(g["v"], i), seg(g["beta_k"], i),
                                        S0=S_in, **args(i))
        outs.append(o)
        if i == len(split) - 1:
            S_final = S_seg
    torch.cuda.synchronize()
    ref_o, ref_S = oracle.delta_rule_sequential(x["q"], x["k"], x["v"], x["beta_k"], alpha=x["alpha"],
                                                beta_v=x["beta_v"], S0=x["S0"], s_scale=x["s"])
    o = torch.cat(outs, dim=1).float().cpu().numpy()
    assert err(o, ref_o, OUT_ROUND["bf16"]) <= TOL["bf16"][0]
    assert err(S_final.cpu().numpy(), ref_S) <= TOL["bf16"][1]
