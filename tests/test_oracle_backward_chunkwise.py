"""Pins of the chunkwise form of the backward (oracle/backward_chunkwise.py): every gradient equals
reverse-mode differentiation of the sequential recurrence (oracle/backward.py, itself pinned to
finite differences of the C oracle), in every gate mode, with decoupled write strengths and OSDN's
write-side scale, for chunk sizes from one token to longer than the sequence (ragged last chunks
included).  Chunk size 1 reduces every chunk's UT system to the identity, the other sizes exercise
the inverse, the masks and the gate products across chunk boundaries."""
import numpy as np
import pytest

from oracle import backward as ob
from oracle import backward_chunkwise as obc

MODES = [
    dict(alpha="none", beta_k="scalar", beta_v="none", s=False),
    dict(alpha="scalar", beta_k="scalar", beta_v="none", s=False),
    dict(alpha="channel", beta_k="channel", beta_v="none", s=False),
    dict(alpha="channel", beta_k="channel", beta_v="channel", s=True),
    dict(alpha="scalar", beta_k="channel", beta_v="scalar", s=True),
    dict(alpha="channel", beta_k="scalar", beta_v="channel", s=False),
]


def _inputs(mode, B=2, T=11, H=2, dk=6, dv=6, seed=0):
    rng = np.random.default_rng(seed)
    lead = (B, T, H)
    gate = lambda m, w, lo, hi: None if m == "none" else rng.uniform(lo, hi, lead if m == "scalar" else lead + (w,))
    x = dict(q=rng.standard_normal(lead + (dk,)), k=rng.standard_normal(lead + (dk,)) / np.sqrt(dk),
             v=rng.standard_normal(lead + (dv,)), alpha=gate(mode["alpha"], dk, 0.6, 1.0),
             beta_k=gate(mode["beta_k"], dk, 0.2, 0.9), beta_v=gate(mode["beta_v"], dv, 0.2, 0.9),
             S0=0.3 * rng.standard_normal((B, H, dk, dv)),
             s_scale=rng.uniform(0.5, 1.5, lead + (dk,)) if mode["s"] else None)
    return x, rng.standard_normal(lead + (dv,)), rng.standard_normal((B, H, dk, dv))


@pytest.mark.parametrize("chunk", [1, 3, 4, 16])
@pytest.mark.parametrize("mode", MODES, ids=lambda m: "a{alpha}_bk{beta_k}_bv{beta_v}_s{s}".format(**m))
def test_chunkwise_backward_equals_autograd(mode, chunk):
    x, do, dST = _inputs(mode, seed=chunk)
    ref = ob.backward(x["q"], x["k"], x["v"], x["beta_k"], do, alpha=x["alpha"], beta_v=x["beta_v"], S0=x["S0"],
                      s_scale=x["s_scale"], dS_T=dST)
    got = obc.backward(x["q"], x["k"], x["v"], x["beta_k"], do, alpha=x["alpha"], beta_v=x["beta_v"], S0=x["S0"],
                       s_scale=x["s_scale"], dS_T=dST, chunk=chunk)
    for name in ("q", "k", "v", "beta_k", "alpha", "beta_v", "S0", "s_scale"):
        if ref[name] is None:
            assert got[name] is None, name
            continue
        r = ref[name].numpy()
        np.testing.assert_allclose(got[name], r, rtol=1e-9, atol=1e-9 * max(1.0, float(np.abs(r).max())),
                                   err_msg=name)


def test_chunkwise_backward_without_final_state_gradient():
    """dS_T omitted means zero, as in the sequential form."""
    mode = MODES[2]
    x, do, _ = _inputs(mode, T=9, seed=4)
    ref = ob.backward(x["q"], x["k"], x["v"], x["beta_k"], do, alpha=x["alpha"], S0=x["S0"])
    got = obc.backward(x["q"], x["k"], x["v"], x["beta_k"], do, alpha=x["alpha"], S0=x["S0"], chunk=4)
    for name in ("q", "k", "v", "alpha", "S0"):
        np.testing.assert_allclose(got[name], ref[name].numpy(), rtol=1e-9, atol=1e-10, err_msg=name)
