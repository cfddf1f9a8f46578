"""GPU parity in the method's degenerate cases, on every prefill kernel path and the decode step,
against the float64 oracle:

* zero strength everywhere (beta = 0): nothing is erased or written, S_T = (prod alpha) S0;
* zero strength on every other token inside chunks (holes in the chunk's UT system);
* decoupled strengths with a zero write (beta_v = 0): erase only;
* no decay and full strength on unit keys (alpha = 1, beta = 1): exact recall, S_t^T k_t = v_t;
* no decay (alpha absent) with channel strengths.

The oracle pins fix the closed forms of the first and fourth cases; here the kernels are compared
with the oracle on the same inputs, element by element, at the usual bounds.
"""
import numpy as np
import pytest
import torch

from synth import make_inputs, problem
from tests.test_gpu_parity import OUT_ROUND, TOL, check, err, ref_prefill, run_prefill, to_dev

pytestmark = pytest.mark.gpu

PATHS = [
    # (base, chunk): the tensor-core ring kernel, the CUDA-core kernel in bf16 and in fp32
    ("kda_bf16", 64),
    ("kda_bf16", 32),
    ("deltanet_f32", 64),
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


def _case(base, name, T=150):
    dk = 64 if base == "deltanet_f32" else 128
    common = dict(B=1, H=2, T=T, dk=dk, dv=dk, S0="normal", seed=77)
    if name == "zero_strength":
        p = problem(base, alpha="channel", beta_k="channel", **common)
        x = make_inputs(p)
        x["beta_k"] = torch.zeros_like(x["beta_k"])
        x["alpha"] = x["alpha"] ** 0.1  # keep the decayed state well above fp16's subnormals
    elif name == "holes":
        p = problem(base, alpha="scalar", beta_k="scalar", **common)
        x = make_inputs(p)
        x["beta_k"][:, 1::2] = 0.0
    elif name == "erase_only":
        p = problem(base, alpha="channel", beta_k="channel", beta_v="channel", **common)
        x = make_inputs(p)
        x["beta_v"] = torch.zeros_like(x["beta_v"])
        x["alpha"] = x["alpha"] ** 0.1
    elif name == "exact_recall":
        p = problem(base, alpha="none", beta_k="scalar", **common)
        x = make_inputs(p)
        x["beta_k"] = torch.ones_like(x["beta_k"])
    elif name == "no_decay_channel":
        p = problem(base, alpha="none", beta_k="channel", **common)
        x = make_inputs(p)
    else:
        raise ValueError(name)
    return p, x


CASES = ["zero_strength", "holes", "erase_only", "exact_recall", "no_decay_channel"]


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("base,chunk", PATHS, ids=["ring", "cudacore_bf16", "cudacore_f32"])
def test_degenerate_prefill(dr, base, chunk, case):
    p, x = _case(base, case)
    o, S_T = run_prefill(dr, x, chunk)
    ref_o, ref_S = ref_prefill(x)
    check(p, o, S_T, ref_o, ref_S)
    if case == "zero_strength":  # closed form: S_T = Diag(prod_t alpha_t) S0
        decay = np.prod(x["alpha"].double().numpy(), axis=1)  # [B, H, dk]
        want = decay[..., None] * x["S0"].double().numpy()
        assert err(S_T.cpu().numpy(), want) <= TOL[p.io][1]


@pytest.mark.parametrize("case", CASES)
def test_degenerate_decode(dr, case):
    p, x = _case("kda_bf16", case, T=6)
    g = to_dev(x)
    S = g["S0"].clone()
    outs = []
    for t in range(p.T):
        tok = lambda n: None if g[n] is None else g[n][:, t:t + 1].clone()  # own, 16-byte-aligned copy
        outs.append(dr.dr_decode_step(tok("q"), tok("k"), tok("v"), tok("beta_k"), S, alpha=tok("alpha"),
                                      beta_v=tok("beta_v")))
    torch.cuda.synchronize()
    ref_o, ref_S = ref_prefill(x)
    got = torch.cat(outs, dim=1).float().cpu().numpy()
    assert err(got, ref_o, OUT_ROUND["bf16"]) <= TOL["bf16"][0]
    assert err(S.cpu().numpy(), ref_S) <= TOL["bf16"][1]
