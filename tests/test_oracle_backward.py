"""Pins of the float64 backward reference (oracle/backward.py).

* Its forward, a second statement of the recurrence in torch ops, equals the C oracle's forward.
* Every gradient equals a central finite difference of the C oracle's forward along a random
  direction, in every gate mode, with decoupled write strengths and OSDN's write-side scale.
* A closed form: with zero write and erase strength the state never moves, so o_t = S0^T q_t,
  dq_t = S0 do_t and dS0 = sum_t q_t do_t^T + dS_T.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as ob

MODES = [
    dict(alpha="none", beta_k="scalar", beta_v="none", s=False),
    dict(alpha="scalar", beta_k="scalar", beta_v="none", s=False),
    dict(alpha="channel", beta_k="channel", beta_v="none", s=False),
    dict(alpha="channel", beta_k="channel", beta_v="channel", s=True),
    dict(alpha="scalar", beta_k="channel", beta_v="scalar", s=True),
]


def _inputs(mode, B=2, T=7, H=2, dk=5, dv=5, seed=0):
    rng = np.random.default_rng(seed)
    lead = (B, T, H)
    gate = lambda m, w, lo, hi: None if m == "none" else rng.uniform(lo, hi, lead if m == "scalar" else lead + (w,))
    x = dict(q=rng.standard_normal(lead + (dk,)), k=rng.standard_normal(lead + (dk,)) / np.sqrt(dk),
             v=rng.standard_normal(lead + (dv,)), alpha=gate(mode["alpha"], dk, 0.6, 1.0),
             beta_k=gate(mode["beta_k"], dk, 0.2, 0.9), beta_v=gate(mode["beta_v"], dv, 0.2, 0.9),
             S0=0.3 * rng.standard_normal((B, H, dk, dv)),
             s_scale=rng.uniform(0.5, 1.5, lead + (dk,)) if mode["s"] else None)
    do = rng.standard_normal(lead + (dv,))
    dST = rng.standard_normal((B, H, dk, dv))
    return x, do, dST


def _c_forward(x):
    return oracle.delta_rule_sequential(x["q"], x["k"], x["v"], x["beta_k"], alpha=x["alpha"], beta_v=x["beta_v"],
                                        S0=x["S0"], s_scale=x["s_scale"], threads=1)


@pytest.mark.parametrize("mode", MODES, ids=lambda m: "a{alpha}_bk{beta_k}_bv{beta_v}_s{s}".format(**m))
def test_torch_forward_equals_c_oracle(mode):
    x, _, _ = _inputs(mode)
    t = {n: (None if a is None else torch.from_numpy(a)) for n, a in x.items()}
    o, S = ob.forward(t["q"], t["k"], t["v"], t["beta_k"], t["alpha"], t["beta_v"], t["S0"], t["s_scale"])
    o_c, S_c = _c_forward(x)
    np.testing.assert_allclose(o.numpy(), o_c, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S.numpy(), S_c, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mode", MODES, ids=lambda m: "a{alpha}_bk{beta_k}_bv{beta_v}_s{s}".format(**m))
def test_gradients_match_finite_differences_of_c_oracle(mode):
    x, do, dST = _inputs(mode, seed=3)
    g = ob.backward(x["q"], x["k"], x["v"], x["beta_k"], do, alpha=x["alpha"], beta_v=x["beta_v"], S0=x["S0"],
                    s_scale=x["s_scale"], dS_T=dST)
    rng = np.random.default_rng(11)
    eps = 1e-6

    def loss(xx):
        o, S = _c_forward(xx)
        return float((o * do).sum() + (S * dST).sum())

    for name in ("q", "k", "v", "beta_k", "alpha", "beta_v", "S0", "s_scale"):
        if x[name] is None:
            continue
        d = rng.standard_normal(x[name].shape)
        xp = dict(x, **{name: x[name] + eps * d})
        xm = dict(x, **{name: x[name] - eps * d})
        fd = (loss(xp) - loss(xm)) / (2 * eps)
        an = float((g[name].numpy() * d).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, fd, an)


def test_closed_form_without_writes():
    """beta_k tiny and alpha = 1: the state stays S0 (up to O(beta)); dq and dS0 follow in closed form."""
    mode = dict(alpha="none", beta_k="scalar", beta_v="scalar", s=False)
    x, do, dST = _inputs(mode, seed=5)
    x["beta_k"] = np.full_like(x["beta_k"], 1e-30)
    x["beta_v"] = np.zeros_like(x["beta_v"])
    g = ob.backward(x["q"], x["k"], x["v"], x["beta_k"], do, beta_v=x["beta_v"], S0=x["S0"], dS_T=dST)
    S0 = x["S0"]
    np.testing.assert_allclose(g["o"].numpy(), np.einsum("bhij,bthi->bthj", S0, x["q"]), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["q"].numpy(), np.einsum("bhij,bthj->bthi", S0, do), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["S0"].numpy(), np.einsum("bthi,bthj->bhij", x["q"], do) + dST, rtol=1e-12,
                               atol=1e-12)
    np.testing.assert_allclose(g["v"].numpy(), 0.0, atol=1e-12)
