"""The dk = dv = 128 decode kernels against one another and against the oracle.

Kernels, named through dr_diag_decode_step_variant (include/deltarule_diag.h): one CTA per head;
four CTAs per head of 32 value columns each (the library's choice when there are no more heads
than SMs); and the persistent streaming kernel, two CTAs per SM, with the next head's state copied
ahead into shared memory (the library's choice for more heads than SMs).  Inputs: the decode
workload (all 8192 heads, four chained in-place steps), head counts just above the SM count and
not a multiple of it, and small batches, in every gate mode and with OSDN's write-key scale.
Every kernel does the same operations in the same order per value column, so outputs and states
must agree bit for bit; the small cases are also checked against the float64 oracle.
"""
import pytest

pytestmark = pytest.mark.gpu

SMALL = [
    # (B, H, alpha, beta_k, beta_v, s)
    (149, 1, "channel", "channel", "none", "none"),
    (10, 30, "scalar", "scalar", "none", "none"),
    (3, 101, "channel", "scalar", "channel", "channel"),
    (7, 43, "none", "channel", "scalar", "none"),
    (4, 16, "scalar", "scalar", "none", "none"),         # the handoff batch: 64 heads, split 4 ways
    (2, 74, "channel", "channel", "channel", "channel"),  # 148 heads
    (1, 1, "channel", "scalar", "none", "channel"),
]
VARIANTS = ("default", "per_head", "split4", "stream")


def _run(variant):
    import torch

    import weight_recurrence_chunkwise_b200 as dr
    from synth import decode_inputs, make_inputs, problem

    res = {}
    d = decode_inputs()
    S = d["S"].cuda()
    outs = []
    for t in range(4):
        step = {n: (None if d[n] is None else d[n][t].cuda()) for n in ("q", "k", "v", "alpha", "beta_k")}
        outs.append(dr.dr_diag_decode_step_variant(variant, step["q"], step["k"], step["v"], step["beta_k"], S,
                                                   alpha=step["alpha"]))
    torch.cuda.synchronize()
    res["workload"] = (torch.stack(outs).cpu(), S.cpu())
    del S, outs
    for i, (B, H, a, bk, bv, sc) in enumerate(SMALL):
        p = problem("kda_bf16", B=B, H=H, T=1, alpha=a, beta_k=bk, beta_v=bv, S0="normal", s_scale=sc, seed=40 + i)
        x = {n: (None if t is None else t.cuda()) for n, t in make_inputs(p).items()}
        S = x["S0"].clone()
        o = dr.dr_diag_decode_step_variant(variant, x["q"], x["k"], x["v"], x["beta_k"], S, alpha=x["alpha"],
                                           beta_v=x["beta_v"], s=x["s"])
        torch.cuda.synchronize()
        res[i] = (o.cpu(), S.cpu())
    return res


def test_decode_kernels_agree_and_match_oracle():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import oracle
    from synth import make_inputs, problem
    from tests.test_gpu_parity import OUT_ROUND, TOL, err

    got = {v: _run(v) for v in VARIANTS}
    for v in VARIANTS[1:]:
        for key in got["per_head"]:
            (o_c, S_c), (o_s, S_s) = got["per_head"][key], got[v][key]
            assert torch.equal(o_c, o_s) and torch.equal(S_c, S_s), (v, key)
    for i, (B, H, a, bk, bv, sc) in enumerate(SMALL):
        p = problem("kda_bf16", B=B, H=H, T=1, alpha=a, beta_k=bk, beta_v=bv, S0="normal", s_scale=sc, seed=40 + i)
        x = make_inputs(p)
        ref_o, ref_S = oracle.delta_rule_sequential(x["q"], x["k"], x["v"], x["beta_k"], alpha=x["alpha"],
                                                    beta_v=x["beta_v"], S0=x["S0"], s_scale=x["s"])
        o, S = got["default"][i]
        assert err(o.float().numpy(), ref_o, OUT_ROUND["bf16"]) <= TOL["bf16"][0], i
        assert err(S.numpy(), ref_S) <= TOL["bf16"][1], i
