"""Chunkwise (WY/UT) form of the backward pass, in float64 -- the algebra a chunk-parallel backward
kernel follows, checked against reverse-mode differentiation of the recurrence.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only ``tests/`` may import it; the CUDA
library never does.  Parity unpinned it is not: ``tests/test_oracle_backward_chunkwise.py`` pins
every gradient to ``oracle.backward`` (torch autograd of the sequential recurrence, itself pinned
to finite differences of the C oracle).

Forward per chunk (DeltaNet page, step 7; FG2-GDN page, section 2), rows r of the chunk, S its
initial state, gamma_r = prod_{j<=r} alpha_j per key channel:
    Qh = gamma (.) q,  Bh = gamma (.) b,  Ac = a / gamma,  What = w
    A = strictly-lower(Bh Ac^T),  T = (I + A)^-1,  Y = What - Bh S,  U = T Y
    P = lower(Qh Ac^T),  O = Qh S + P U,  M = S + Ac^T U,  S_end = Diag(gamma_last) M
Backward per chunk, from the last chunk to the first, with dO and dS_end (the next chunk's dS):
    dM = Diag(gamma_last) dS_end
    dU = P^T dO + Ac dM
    dS = Qh^T dO + dM - Bh^T (T^T dU)            (the serial recurrence between chunks)
    dV = T^T dU:   dWhat = dV,   dBh = -dV S^T,   dA = strictly-lower(-dV U^T)
    dP = lower(dO U^T)
    dQh = dO S^T + dP Ac
    dBh += dA Ac
    dAc = dA^T Bh + dP^T Qh + U dM^T
    dgamma_r = q_r (.) dQh_r + b_r (.) dBh_r - Ac_r (.) dAc_r / gamma_r,
    dgamma_last += rowsum(dS_end (.) M)
    dq = gamma (.) dQh,  db = gamma (.) dBh,  da = dAc / gamma
    dalpha_j = (sum_{r >= j} dgamma_r (.) gamma_r) / alpha_j
then b = sqrt(beta_k) (.) k, a = s (.) b and w = beta_v (.) v or sqrt(beta_k) (.) v by the chain
rule, with scalar gates summed over their channels.
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    return None if x is None else np.asarray(x, dtype=np.float64)


def _rows(g, width):
    """Gate [B,T,H] or [B,T,H,d] (or None) as [B,T,H,width] float64."""
    if g is None:
        return None
    g = _f64(g)
    return np.broadcast_to(g[..., None], g.shape + (width,)) if g.ndim == 3 else g


def backward(q, k, v, beta_k, do, alpha=None, beta_v=None, S0=None, s_scale=None, dS_T=None, chunk=64):
    """Gradients of sum(do * o) + sum(dS_T * S_T), by the chunkwise form.  Same keys as
    ``oracle.backward.backward``: q, k, v, beta_k, alpha, beta_v, S0, s_scale (None where absent)."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    al = _rows(alpha, dk) if alpha is not None else np.ones((B, T, H, dk))
    bk = _rows(beta_k, dk)
    sb = np.sqrt(bk)
    b = sb * k
    sc = _f64(s_scale) if s_scale is not None else np.ones_like(b)
    a = sc * b
    if beta_v is not None:
        wsc = _rows(beta_v, dv)
    else:
        if _f64(beta_k).ndim == 4 and dk != dv:
            raise ValueError("the symmetric channel write needs dk == dv")
        wsc = np.sqrt(_rows(beta_k, dv)) if _f64(beta_k).ndim == 3 else sb
    w = wsc * v
    S0 = np.zeros((B, H, dk, dv)) if S0 is None else _f64(S0)
    dST = np.zeros((B, H, dk, dv)) if dS_T is None else _f64(dS_T)

    g_q, g_b, g_a, g_w = (np.zeros_like(x) for x in (q, b, a, w))
    g_al = np.zeros_like(al)
    g_S0 = np.zeros_like(S0)
    starts = list(range(0, T, chunk))
    for bi in range(B):
        for hi in range(H):
            # forward over the chunks, keeping each chunk's initial state
            S = S0[bi, hi].copy()
            S_in = []
            for t0 in starts:
                t1 = min(t0 + chunk, T)
                f = _chunk_factors(q[bi, t0:t1, hi], b[bi, t0:t1, hi], a[bi, t0:t1, hi], w[bi, t0:t1, hi],
                                   al[bi, t0:t1, hi], S)
                S_in.append(S)
                S = f["S_end"]
            # backward over the chunks
            dS = dST[bi, hi].copy()
            for ci in range(len(starts) - 1, -1, -1):
                t0 = starts[ci]
                t1 = min(t0 + chunk, T)
                sl = (bi, slice(t0, t1), hi)
                f = _chunk_factors(q[sl], b[sl], a[sl], w[sl], al[sl], S_in[ci])
                gr = _chunk_backward(f, q[sl], b[sl], a[sl], al[sl], do[sl], dS)
                g_q[sl], g_b[sl], g_a[sl], g_w[sl], g_al[sl] = gr["q"], gr["b"], gr["a"], gr["w"], gr["alpha"]
                dS = gr["S"]
            g_S0[bi, hi] = dS

    # chain rule through b = sqrt(beta_k) k, a = s b, w = wsc v
    g_b_tot = g_b + sc * g_a
    out = {"q": g_q, "k": sb * g_b_tot, "v": wsc * g_w, "S0": g_S0, "s_scale": None, "alpha": None, "beta_v": None}
    d_sb = k * g_b_tot  # d / d sqrt(beta_k), per channel, through b
    if s_scale is not None:
        out["s_scale"] = b * g_a
    d_wsc = v * g_w  # d / d (write scale), per value column
    if beta_v is not None:
        out["beta_v"] = d_wsc.sum(-1) if _f64(beta_v).ndim == 3 else d_wsc
    with np.errstate(divide="ignore", invalid="ignore"):
        d_bk = np.where(sb > 0, 0.5 * d_sb / np.where(sb > 0, sb, 1.0), 0.0)  # d sqrt(x) / dx
        if beta_v is None:  # w = sqrt(beta_k) v as well
            d_bk_w = np.where(wsc > 0, 0.5 * d_wsc / np.where(wsc > 0, wsc, 1.0), 0.0)
    if _f64(beta_k).ndim == 3:
        out["beta_k"] = d_bk.sum(-1) + (d_bk_w.sum(-1) if beta_v is None else 0.0)
    else:
        out["beta_k"] = d_bk + (d_bk_w if beta_v is None else 0.0)
    if alpha is not None:
        out["alpha"] = g_al.sum(-1) if _f64(alpha).ndim == 3 else g_al
    return out


def _chunk_factors(q, b, a, w, al, S):
    """The chunk's forward factors (rows of q, b, a, w, al: [L, d]) from its initial state S."""
    L = q.shape[0]
    gam = np.cumprod(al, axis=0)  # gamma_r per key channel
    Qh, Bh, Ac = gam * q, gam * b, a / gam
    A = np.tril(Bh @ Ac.T, -1)
    Tm = np.linalg.inv(np.eye(L) + A)
    Y = w - Bh @ S
    U = Tm @ Y
    P = np.tril(Qh @ Ac.T)
    M = S + Ac.T @ U
    return dict(gam=gam, Qh=Qh, Bh=Bh, Ac=Ac, T=Tm, U=U, P=P, M=M, S=S, S_end=gam[-1][:, None] * M,
                O=Qh @ S + P @ U)


def _chunk_backward(f, q, b, a, al, dO, dS_end):
    gam, Qh, Bh, Ac, Tm, U, P, M, S = (f[n] for n in ("gam", "Qh", "Bh", "Ac", "T", "U", "P", "M", "S"))
    dM = gam[-1][:, None] * dS_end
    dU = P.T @ dO + Ac @ dM
    dV = Tm.T @ dU
    dS = Qh.T @ dO + dM - Bh.T @ dV
    dW = dV
    dA = np.tril(-dV @ U.T, -1)
    dP = np.tril(dO @ U.T)
    dQh = dO @ S.T + dP @ Ac
    dBh = -dV @ S.T + dA @ Ac
    dAc = dA.T @ Bh + dP.T @ Qh + U @ dM.T
    dgam = q * dQh + b * dBh - Ac * dAc / gam
    dgam[-1] += np.sum(dS_end * M, axis=1)
    # gamma_r = prod_{j <= r} alpha_j:  dalpha_j = sum_{r >= j} dgamma_r gamma_r / alpha_j
    rev = np.cumsum((dgam * gam)[::-1], axis=0)[::-1]
    return {"q": gam * dQh, "b": gam * dBh, "a": dAc / gam, "w": dW, "alpha": rev / al, "S": dS}
