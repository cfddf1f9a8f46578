"""Float64 reference for the backward pass of the gated delta-rule recurrence.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only ``tests/`` and the CPU leg of
``bench.py`` may import it; the CUDA library never does.

The forward here is a second, independent float64 statement of the recurrence the C oracle
computes (DeltaNet page, steps 3-6; FG2-GDN page, section 2 and "Erweiterung: FG2-GDN+";
OSDN summary, "Method"), written with plain PyTorch CPU ops, one token at a time:

    b_t = sqrt(beta_k_t) * k_t,   a_t = s_t * b_t  (s = 1 unless given)
    w_t = beta_v_t * v_t if beta_v is given else sqrt(beta_k_t) * v_t
    X_t = Diag(alpha_t) S_{t-1},  S_t = X_t + a_t (w_t - X_t^T b_t)^T,   o_t = S_t^T q_t

and the backward is reverse-mode differentiation of that forward by torch.autograd: the
gradients of L = sum(do * o) + sum(dS_T * S_T) with respect to every input.  The tests pin the
forward to the C oracle and the gradients to central finite differences of the C oracle.
"""
from __future__ import annotations

import torch


def _f64(x):
    return None if x is None else torch.as_tensor(x).detach().to("cpu", torch.float64)


def _per_row(g, t):
    """Gate at step t as a [B, H, d] (channel) or [B, H, 1] (scalar) factor."""
    x = g[:, t]
    return x if x.dim() == 3 else x[..., None]


def forward(q, k, v, beta_k, alpha=None, beta_v=None, S0=None, s_scale=None):
    """The recurrence in float64 torch ops (differentiable).  Returns ``(o, S_T)``."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    S = S0 if S0 is not None else torch.zeros(B, H, dk, dv, dtype=q.dtype)
    outs = []
    for t in range(T):
        sb = torch.sqrt(_per_row(beta_k, t))                     # [B,H,dk] or [B,H,1]
        b = sb * k[:, t]
        a = b * s_scale[:, t] if s_scale is not None else b
        if beta_v is not None:
            w = _per_row(beta_v, t) * v[:, t]
        else:
            w = sb * v[:, t]                                     # channel form needs dk == dv
        X = S * _per_row(alpha, t)[..., None] if alpha is not None else S
        u = w - torch.einsum("bhij,bhi->bhj", X, b)
        S = X + a[..., :, None] * u[..., None, :]
        outs.append(torch.einsum("bhij,bhi->bhj", S, q[:, t]))
    return torch.stack(outs, dim=1), S


def backward(q, k, v, beta_k, do, alpha=None, beta_v=None, S0=None, s_scale=None, dS_T=None):
    """Gradients of sum(do * o) + sum(dS_T * S_T) in float64.

    Returns a dict with keys q, k, v, beta_k, alpha, beta_v, S0, s_scale (None where the input is
    absent) and the forward's ``o``, ``S_T``.
    """
    names = ("q", "k", "v", "beta_k", "alpha", "beta_v", "S0", "s_scale")
    xs = {n: _f64(x) for n, x in zip(names, (q, k, v, beta_k, alpha, beta_v, S0, s_scale))}
    for x in xs.values():
        if x is not None:
            x.requires_grad_(True)
    o, S_T = forward(xs["q"], xs["k"], xs["v"], xs["beta_k"], xs["alpha"], xs["beta_v"], xs["S0"], xs["s_scale"])
    loss = (o * _f64(do)).sum()
    if dS_T is not None:
        loss = loss + (S_T * _f64(dS_T)).sum()
    present = [n for n in names if xs[n] is not None]
    grads = torch.autograd.grad(loss, [xs[n] for n in present])
    out = {n: None for n in names}
    out.update({n: g.detach() for n, g in zip(present, grads)})
    out["o"], out["S_T"] = o.detach(), S_T.detach()
    return out
