"""The dk = dv = 128 decode paths against the one-CTA-per-head kernel and the oracle: the streaming
kernel (persistent, two CTAs per SM, the next head's state copied ahead into shared memory) for more
heads than SMs, and four CTAs per head (32 value columns each) for fewer.

The library picks the path once per process (DR_DECODE_KERNEL=classic keeps one CTA per head), so
each runs in a child process on the same inputs: the decode workload (all 8192 heads, four chained
in-place steps), head counts just above the SM count and not a multiple of it, and small batches,
in every gate mode and with OSDN's write-key scale.  Every path does the same operations in the
same order per value column, so outputs and states must agree bit for bit; the small cases are also
checked against the float64 oracle.
"""
import os
import subprocess
import sys
import tempfile

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

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


def _run(out_path):
    import torch

    sys.path.insert(0, ROOT)
    import weight_recurrence_chunkwise_b200 as dr
    from synth import decode_inputs, make_inputs, problem

    dr.lib()
    res = {}
    d = decode_inputs()
    S = d["S"].cuda()
    outs = []
    for t in range(4):
        step = {n: (None if d[n] is None else d[n][t].cuda()) for n in ("q", "k", "v", "alpha", "beta_k")}
        outs.append(dr.dr_decode_step(step["q"], step["k"], step["v"], step["beta_k"], S, alpha=step["alpha"]))
    torch.cuda.synchronize()
    res["workload"] = (torch.stack(outs).cpu(), S.cpu())
    for i, (B, H, a, bk, bv, sc) in enumerate(SMALL):
        p = problem("kda_bf16", B=B, H=H, T=1, alpha=a, beta_k=bk, beta_v=bv, S0="normal", s_scale=sc, seed=40 + i)
        x = {n: (None if t is None else t.cuda()) for n, t in make_inputs(p).items()}
        S = x["S0"].clone()
        if x["s"] is None:
            o = dr.dr_decode_step(x["q"], x["k"], x["v"], x["beta_k"], S, alpha=x["alpha"], beta_v=x["beta_v"])
        else:
            o = dr.dr_decode_step_osdn(x["q"], x["k"], x["v"], x["beta_k"], S, x["s"], alpha=x["alpha"],
                                       beta_v=x["beta_v"])
        torch.cuda.synchronize()
        res[i] = (o.cpu(), S.cpu())
    torch.save(res, out_path)


def _child(variant, path):
    env = dict(os.environ)
    env.pop("DR_DECODE_KERNEL", None)
    if variant == "classic":
        env["DR_DECODE_KERNEL"] = "classic"
    r = subprocess.run([sys.executable, os.path.abspath(__file__), path], env=env, cwd=ROOT, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]


def test_stream_decode_equals_classic_and_oracle():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import oracle
    from synth import make_inputs, problem
    from tests.test_gpu_parity import OUT_ROUND, TOL, err

    with tempfile.TemporaryDirectory() as tmp:
        paths = {v: os.path.join(tmp, v + ".pt") for v in ("stream", "classic")}
        for v, pth in paths.items():
            _child(v, pth)
        got = {v: torch.load(pth) for v, pth in paths.items()}
    for key in got["classic"]:
        (o_c, S_c), (o_s, S_s) = got["classic"][key], got["stream"][key]
        assert torch.equal(o_c, o_s) and torch.equal(S_c, S_s), key
    for i, (B, H, a, bk, bv, sc) in enumerate(SMALL):
        p = problem("kda_bf16", B=B, H=H, T=1, alpha=a, beta_k=bk, beta_v=bv, S0="normal", s_scale=sc, seed=40 + i)
        x = make_inputs(p)
        ref_o, ref_S = oracle.delta_rule_sequential(x["q"], x["k"], x["v"], x["beta_k"], alpha=x["alpha"],
                                                    beta_v=x["beta_v"], S0=x["S0"], s_scale=x["s"])
        o, S = got["stream"][i]
        assert err(o.float().numpy(), ref_o, OUT_ROUND["bf16"]) <= TOL["bf16"][0], i
        assert err(S.numpy(), ref_S) <= TOL["bf16"][1], i


if __name__ == "__main__":
    _run(sys.argv[1])
