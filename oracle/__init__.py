"""Float64 CPU oracle of the gated delta-rule forward pass.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this package.  The
CUDA library and its Python binding never import it, and it imports nothing of
theirs.

The arithmetic lives in ``dr_oracle.c`` (plain C, float64, one recurrence per
(batch, head), OpenMP across heads).  This module only marshals arrays:
inputs of any float dtype (torch or numpy) are up-cast exactly to float64.

Recurrence (see the C file for the passages it follows):
    b_t = sqrt(beta_k_t) * k_t,  a_t = s_t * b_t (s = 1 unless given)
    w_t = beta_v_t * v_t if beta_v is given else sqrt(beta_k_t) * v_t
    S_t = (I - a_t b_t^T) Diag(alpha_t) S_{t-1} + a_t w_t^T,   o_t = S_t^T q_t
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build as _build

_lib = None

ABSENT, SCALAR, CHANNEL = 0, 1, 2


def _load():
    global _lib
    if _lib is None:
        path = _build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        ints5 = [ctypes.c_int] * 5
        tail = [dp, dp, dp, dp, ctypes.c_int, dp, ctypes.c_int, dp, ctypes.c_int, dp, dp, dp, dp,
                ctypes.c_int]
        lib.dro_sequential.argtypes = ints5 + tail
        lib.dro_sequential.restype = ctypes.c_int
        lib.dro_chunkwise.argtypes = ints5 + [ctypes.c_int] + tail
        lib.dro_chunkwise.restype = ctypes.c_int
        lib.dro_max_threads.argtypes = []
        lib.dro_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().dro_max_threads())


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: exact up-cast on the CPU
        import torch

        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _mode(x, ndim_scalar: int) -> int:
    if x is None:
        return ABSENT
    return SCALAR if x.ndim == ndim_scalar else CHANNEL


def _run(chunk, q, k, v, beta_k, alpha=None, beta_v=None, S0=None, s_scale=None, threads=None):
    q, k, v = _f64(q), _f64(k), _f64(v)
    alpha, beta_k, beta_v, S0, s_scale = map(_f64, (alpha, beta_k, beta_v, S0, s_scale))
    if q.ndim != 4 or k.shape != q.shape or v.ndim != 4 or v.shape[:3] != q.shape[:3]:
        raise ValueError("q, k must be [B,T,H,dk] and v [B,T,H,dv]")
    B, T, H, dk = q.shape
    dv = v.shape[3]
    if beta_k is None:
        raise ValueError("beta_k is required")
    for name, x, width in (("alpha", alpha, dk), ("beta_k", beta_k, dk), ("beta_v", beta_v, dv)):
        if x is not None and x.shape not in ((B, T, H), (B, T, H, width)):
            raise ValueError(f"{name} must be [B,T,H] or [B,T,H,{width}], got {x.shape}")
    if s_scale is not None and s_scale.shape != q.shape:
        raise ValueError("s_scale must be [B,T,H,dk]")
    if S0 is not None and S0.shape != (B, H, dk, dv):
        raise ValueError("S0 must be [B,H,dk,dv]")
    o = np.zeros((B, T, H, dv), dtype=np.float64)
    ST = np.zeros((B, H, dk, dv), dtype=np.float64)
    lib = _load()
    common = (_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _mode(alpha, 3), _ptr(beta_k), _mode(beta_k, 3),
              _ptr(beta_v), _mode(beta_v, 3), _ptr(s_scale), _ptr(S0), _ptr(o), _ptr(ST),
              int(threads or 0))
    if chunk is None:
        rc = lib.dro_sequential(B, T, H, dk, dv, *common)
    else:
        rc = lib.dro_chunkwise(B, T, H, dk, dv, int(chunk), *common)
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (code {rc})")
    return o, ST


def delta_rule_sequential(q, k, v, beta_k, alpha=None, beta_v=None, S0=None, s_scale=None,
                          threads=None):
    """The recurrence one token at a time, in float64.  Returns ``(o, S_T)``."""
    return _run(None, q, k, v, beta_k, alpha, beta_v, S0, s_scale, threads)


def delta_rule_chunkwise(q, k, v, beta_k, alpha=None, beta_v=None, S0=None, s_scale=None,
                         chunk=64, threads=None):
    """The chunkwise WY/UT evaluation of the same recurrence, in float64."""
    return _run(chunk, q, k, v, beta_k, alpha, beta_v, S0, s_scale, threads)
