"""Pins of the float64 oracle against facts fixed by the pages and by the mathematics.

Each test checks the oracle against something other than itself: a hand-worked
example, an algebraic identity of the delta rule, a textbook special case
(additive linear attention, Householder reflections), or an independent dense
product-form evaluation.  Together they catch a dropped term, a wrong sign or
index, a transposed operand, or decay applied after the erase.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from synth import make_inputs, problem

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _case(rng, B=1, T=9, H=2, dk=6, dv=6, alpha="channel", beta_k="channel", beta_v="none",
          s_scale=False, S0=True):
    lead = (B, T, H)
    q = _rand(rng, *lead, dk)
    k = _unit(_rand(rng, *lead, dk))
    v = _rand(rng, *lead, dv)
    gshape = lambda m, w: lead if m == "scalar" else lead + (w,)
    al = None if alpha == "none" else rng.uniform(0.3, 1.0, gshape(alpha, dk))
    bk = rng.uniform(0.05, 1.0, gshape(beta_k, dk))
    bv = None if beta_v == "none" else rng.uniform(0.05, 1.0, gshape(beta_v, dv))
    s = rng.uniform(0.5, 1.5, lead + (dk,)) if s_scale else None
    s0 = 0.3 * _rand(rng, B, H, dk, dv) if S0 else None
    return dict(q=q, k=k, v=v, alpha=al, beta_k=bk, beta_v=bv, s_scale=s, S0=s0)


MODES = [
    dict(alpha="none", beta_k="scalar", beta_v="none"),          # DeltaNet
    dict(alpha="scalar", beta_k="scalar", beta_v="none"),        # Gated DeltaNet
    dict(alpha="channel", beta_k="channel", beta_v="none"),      # KDA / FG2-GDN
    dict(alpha="channel", beta_k="channel", beta_v="channel"),   # FG2-GDN+
    dict(alpha="scalar", beta_k="scalar", beta_v="scalar"),      # decoupled scalar strengths
    dict(alpha="channel", beta_k="channel", beta_v="none", s_scale=True),  # write-side scaling
]


# ---------------------------------------------------------------- hand-worked examples
def test_hand_worked_examples():
    with open(os.path.join(GOLDEN, "hand_worked.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        T, dk, dv = c["T"], c["dk"], c["dv"]
        a = lambda x, w: None if x is None else np.asarray(x, float).reshape(1, T, 1, *([w] if np.ndim(x) == 2 else []))
        q = np.asarray(c["q"], float).reshape(1, T, 1, dk)
        k = np.asarray(c["k"], float).reshape(1, T, 1, dk)
        v = np.asarray(c["v"], float).reshape(1, T, 1, dv)
        s = None if c["s_scale"] is None else np.asarray(c["s_scale"], float).reshape(1, T, 1, dk)
        S0 = np.asarray(c["S0"], float).reshape(1, 1, dk, dv)
        o, ST = oracle.delta_rule_sequential(q, k, v, a(c["beta_k"], dk), alpha=a(c["alpha"], dk),
                                             beta_v=a(c["beta_v"], dv), S0=S0, s_scale=s)
        np.testing.assert_allclose(o.reshape(T, dv), np.asarray(c["o"], float), rtol=0, atol=1e-14)
        np.testing.assert_allclose(ST.reshape(dk, dv), np.asarray(c["ST"], float), rtol=0, atol=1e-14)


# ---------------------------------------------------------------- pin (a): exact recall
@pytest.mark.parametrize("S0", [False, True])
def test_pin_a_read_after_write_returns_value(S0):
    """alpha = 1, beta = 1, unit keys: after the write, S_t^T k_t == v_t exactly."""
    rng = np.random.default_rng(10)
    B, T, H, d = 2, 40, 3, 16
    k = _unit(_rand(rng, B, T, H, d))
    v = _rand(rng, B, T, H, d)
    s0 = _rand(rng, B, H, d, d) if S0 else None
    o, _ = oracle.delta_rule_sequential(k, k, v, np.ones((B, T, H)), S0=s0)  # q := k
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- pin (b): zero strength
@pytest.mark.parametrize("mode", ["scalar", "channel"])
def test_pin_b_zero_strength_keeps_state(mode):
    rng = np.random.default_rng(11)
    c = _case(rng, alpha="none", beta_k=mode, beta_v="channel", T=12)
    c["beta_k"] = np.zeros_like(c["beta_k"])
    c["beta_v"] = np.zeros_like(c["beta_v"])
    o, ST = oracle.delta_rule_sequential(**c)
    np.testing.assert_array_equal(ST, c["S0"])
    # and every output reads the unchanged state
    np.testing.assert_allclose(o, np.einsum("bthi,bhij->bthj", c["q"], c["S0"]), rtol=0, atol=1e-13)


# ---------------------------------------------------------------- pin (c): linear attention
def test_pin_c_orthonormal_keys_reduce_to_linear_attention():
    """Mutually orthonormal keys with beta = 1, alpha = 1, S0 = 0: S_T = sum_t k_t v_t^T."""
    rng = np.random.default_rng(12)
    d, dv, T = 12, 7, 10
    Qm, _ = np.linalg.qr(_rand(rng, d, d))
    k = Qm[:, :T].T.reshape(1, T, 1, d)
    v = _rand(rng, 1, T, 1, dv)
    q = _rand(rng, 1, T, 1, d)
    o, ST = oracle.delta_rule_sequential(q, k, v, np.ones((1, T, 1)))
    K, V, Qr = k[0, :, 0], v[0, :, 0], q[0, :, 0]
    np.testing.assert_allclose(ST[0, 0], K.T @ V, rtol=0, atol=1e-13)
    mask = np.tril(np.ones((T, T)))
    np.testing.assert_allclose(o[0, :, 0], (mask * (Qr @ K.T)) @ V, rtol=0, atol=1e-13)


# ---------------------------------------------------------------- pin (d): chunkwise == sequential
@pytest.mark.parametrize("modes", MODES)
@pytest.mark.parametrize("chunk", [1, 2, 5, 16, 37])
def test_pin_d_chunkwise_equals_sequential(modes, chunk):
    rng = np.random.default_rng(13)
    c = _case(rng, T=37, **modes)
    o1, S1 = oracle.delta_rule_sequential(**c)
    o2, S2 = oracle.delta_rule_chunkwise(**c, chunk=chunk)
    scale = max(1.0, np.abs(o1).max())
    assert np.abs(o1 - o2).max() <= 1e-12 * scale
    assert np.abs(S1 - S2).max() <= 1e-12 * max(1.0, np.abs(S1).max())


# ---------------------------------------------------------------- closed forms
def test_constant_decay_without_writes_is_geometric():
    rng = np.random.default_rng(14)
    c = _case(rng, alpha="scalar", beta_k="scalar", T=17)
    c["alpha"] = np.full_like(c["alpha"], 0.9)
    c["beta_k"] = np.zeros_like(c["beta_k"])
    _, ST = oracle.delta_rule_sequential(**c)
    np.testing.assert_allclose(ST, 0.9 ** 17 * c["S0"], rtol=1e-13, atol=0)


def test_householder_reflections_preserve_frobenius_norm():
    """beta = 2, unit keys, zero write: each step applies the reflection I - 2 k k^T."""
    rng = np.random.default_rng(15)
    B, T, H, d = 1, 50, 2, 8
    k = _unit(_rand(rng, B, T, H, d))
    s0 = _rand(rng, B, H, d, d)
    _, ST = oracle.delta_rule_sequential(_rand(rng, B, T, H, d), k, np.zeros((B, T, H, d)),
                                         np.full((B, T, H), 2.0), S0=s0)
    np.testing.assert_allclose(np.linalg.norm(ST, axis=(2, 3)), np.linalg.norm(s0, axis=(2, 3)),
                               rtol=1e-12)
    # and the reflection is not the identity: the state really moved
    assert np.abs(ST - s0).max() > 1e-2


def test_spectral_norm_non_increasing_without_writes():
    """w = 0, alpha <= 1, beta |k|^2 in [0, 2]: the transition is a contraction."""
    rng = np.random.default_rng(16)
    d = 6
    S = _rand(rng, 1, 1, d, d)
    norm = np.linalg.norm(S[0, 0], 2)
    for _ in range(30):
        k = _unit(_rand(rng, 1, 1, 1, d))
        beta = rng.uniform(0.0, 2.0, (1, 1, 1, d))
        alpha = rng.uniform(0.5, 1.0, (1, 1, 1, d))
        # channel beta: the erase key is sqrt(beta) * k, |b|^2 <= 2 needs sum(beta k^2) <= 2
        _, S = oracle.delta_rule_sequential(k, k, np.zeros((1, 1, 1, d)), beta, alpha=alpha,
                                            beta_v=np.zeros((1, 1, 1, d)), S0=S)
        new = np.linalg.norm(S[0, 0], 2)
        assert new <= norm * (1 + 1e-12)
        norm = new


# ---------------------------------------------------------------- independent dense product form
def _dense_product_form(c):
    """S_T = (prod_t A_t) S0 + sum_t (prod_{s>t} A_s) a_t w_t^T with A_t = (I - a_t b_t^T) D_t,
    and o_t from S_t, built from explicit dk x dk matrices (no vector updates)."""
    q, k, v = c["q"], c["k"], c["v"]
    B, T, H, dk = q.shape
    dv = v.shape[3]

    def g(x, b, t, h, w):
        if x is None:
            return np.ones(w)
        return np.full(w, x[b, t, h]) if x.ndim == 3 else x[b, t, h]

    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S0 = c["S0"][b, h] if c["S0"] is not None else np.zeros((dk, dv))
            As, writes = [], []
            for t in range(T):
                bt = np.sqrt(g(c["beta_k"], b, t, h, dk)) * k[b, t, h]
                at = bt * (c["s_scale"][b, t, h] if c["s_scale"] is not None else 1.0)
                if c["beta_v"] is not None:
                    wt = g(c["beta_v"], b, t, h, dv) * v[b, t, h]
                else:
                    wt = np.sqrt(g(c["beta_k"], b, t, h, dv)) * v[b, t, h]
                As.append((np.eye(dk) - np.outer(at, bt)) @ np.diag(g(c["alpha"], b, t, h, dk)))
                writes.append(np.outer(at, wt))
                # state after token t from the product form
                St = np.linalg.multi_dot([*reversed(As), np.eye(dk)]) @ S0 if t else As[0] @ S0
                for s in range(t + 1):
                    M = np.eye(dk)
                    for r in range(s + 1, t + 1):
                        M = As[r] @ M
                    St = St + M @ writes[s]
                o[b, t, h] = St.T @ q[b, t, h]
            ST[b, h] = St
    return o, ST


@pytest.mark.parametrize("modes", MODES)
def test_brute_force_product_form(modes):
    rng = np.random.default_rng(17)
    c = _case(rng, B=2, T=8, H=2, dk=4, dv=4, **modes)
    o1, S1 = oracle.delta_rule_sequential(**c)
    o2, S2 = _dense_product_form(c)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(S1, S2, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- exact rational recurrence
def test_exact_rationals_on_tiny_input():
    """Fraction arithmetic (no rounding at all) on a 3x3 case with square-number strengths."""
    rng = np.random.default_rng(18)
    T, d = 5, 3
    F = Fraction
    k = [[F(int(x), 4) for x in rng.integers(-4, 5, d)] for _ in range(T)]
    v = [[F(int(x), 2) for x in rng.integers(-4, 5, d)] for _ in range(T)]
    q = [[F(int(x), 3) for x in rng.integers(-3, 4, d)] for _ in range(T)]
    sq = [F(1), F(1, 2), F(3, 4), F(1, 4), F(2, 3)]       # sqrt of beta, exact
    al = [[F(int(x), 8) for x in rng.integers(4, 9, d)] for _ in range(T)]
    S = [[F(int(x), 5) for x in rng.integers(-5, 6, d)] for _ in range(d)]
    S0 = [row[:] for row in S]
    outs = []
    for t in range(T):
        b = [sq[t] * x for x in k[t]]
        w = [sq[t] * x for x in v[t]]
        S = [[al[t][i] * S[i][j] for j in range(d)] for i in range(d)]
        u = [w[j] - sum(S[i][j] * b[i] for i in range(d)) for j in range(d)]
        S = [[S[i][j] + b[i] * u[j] for j in range(d)] for i in range(d)]
        outs.append([sum(S[i][j] * q[t][i] for i in range(d)) for j in range(d)])
    f = lambda x: np.array(x, dtype=float)
    o, ST = oracle.delta_rule_sequential(
        f(q).reshape(1, T, 1, d), f(k).reshape(1, T, 1, d), f(v).reshape(1, T, 1, d),
        (f(sq) ** 2).reshape(1, T, 1), alpha=f(al).reshape(1, T, 1, d),
        S0=f(S0).reshape(1, 1, d, d))
    np.testing.assert_allclose(o.reshape(T, d), f(outs), rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(ST.reshape(d, d), f(S), rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- structure
def test_heads_and_batches_are_independent():
    rng = np.random.default_rng(19)
    c = _case(rng, B=2, T=11, H=3, alpha="channel", beta_k="channel", beta_v="channel")
    o, ST = oracle.delta_rule_sequential(**c)
    sub = {n: (None if x is None else x[1:2, :, 2:3] if n != "S0" else x[1:2, 2:3])
           for n, x in c.items()}
    o1, S1 = oracle.delta_rule_sequential(**sub)
    np.testing.assert_array_equal(o1, o[1:2, :, 2:3])
    np.testing.assert_array_equal(S1, ST[1:2, 2:3])


def test_split_sequence_carries_state():
    rng = np.random.default_rng(20)
    c = _case(rng, T=20, alpha="scalar", beta_k="scalar")
    o, ST = oracle.delta_rule_sequential(**c)
    first = {n: (x[:, :8] if (x is not None and n != "S0") else x) for n, x in c.items()}
    second = {n: (x[:, 8:] if (x is not None and n != "S0") else x) for n, x in c.items()}
    oa, Sa = oracle.delta_rule_sequential(**first)
    second["S0"] = Sa
    ob, Sb = oracle.delta_rule_sequential(**second)
    np.testing.assert_allclose(np.concatenate([oa, ob], axis=1), o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(Sb, ST, rtol=0, atol=1e-13)


def test_scalar_gate_equals_constant_channel_gate():
    rng = np.random.default_rng(21)
    c = _case(rng, alpha="scalar", beta_k="scalar")
    o1, S1 = oracle.delta_rule_sequential(**c)
    d = c["q"].shape[-1]
    c2 = dict(c, alpha=np.repeat(c["alpha"][..., None], d, -1),
              beta_k=np.repeat(c["beta_k"][..., None], d, -1))
    o2, S2 = oracle.delta_rule_sequential(**c2)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-14)
    np.testing.assert_allclose(S1, S2, rtol=0, atol=1e-14)


def test_symmetric_channel_mode_needs_equal_dims():
    rng = np.random.default_rng(22)
    c = _case(rng, dk=6, dv=5, alpha="channel", beta_k="channel", beta_v="none")
    with pytest.raises(ValueError):
        oracle.delta_rule_sequential(**c)


def test_synthetic_inputs_follow_the_recipe():
    p = problem("kda_bf16", B=1, H=2, T=64)
    x = make_inputs(p)
    n = x["q"].float().norm(dim=-1)
    assert float((n - 1).abs().max()) < 1e-2           # L2-normalised (then bf16-rounded)
    assert 0 < float(x["alpha"].min()) and float(x["alpha"].max()) < 1
    assert 0 < float(x["beta_k"].min()) and float(x["beta_k"].max()) < 1
    assert x["alpha"].shape == (1, 64, 2, 128) and x["S0"].shape == (1, 2, 128, 128)
    y = make_inputs(p)
    assert all((x[k] is None and y[k] is None) or bool((x[k] == y[k]).all()) for k in x)
