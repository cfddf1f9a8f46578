"""Input recipe for the gated delta-rule forward pass.

Distributions (one numpy PCG64 stream per problem, seeded; draws are taken in
the fixed order q, k, v, x_alpha, x_beta_k, x_beta_v, S0, skipping absent ones):

* q, k ~ N(0, 1), then L2-normalised per (token, head) -- the key/query map
  with L2 normalisation that the DeltaNet page lists as standard (step 2).
* v ~ N(0, 1).
* alpha = exp(-0.1 * softplus(x)), x ~ N(0, 1): scalar per (b, t, h) or one
  value per key channel.
* beta = sigmoid(x), x ~ N(0, 1): scalar or per channel (erase strength
  beta_k, and the decoupled write strength beta_v when present).
* S0 = 0, or N(0, 0.01) read as variance 0.01 (standard deviation 0.1).
* s (OSDN write-side key scale, optional; drawn last so the other draws do not
  change) = exp(0.25 x), x ~ N(0, 1) per (b, t, h, key channel): a positive
  per-feature scale around 1.  The OSDN summary gives no distribution for it.

Draws are float32; q, k, v are then rounded to the I/O dtype (bf16 by
round-to-nearest-even through torch) and the gates stay float32.  Arrays are
returned as CPU torch tensors in the library's layouts:
q, k [B,T,H,dk]; v [B,T,H,dv]; alpha, beta_k [B,T,H] or [B,T,H,dk];
beta_v [B,T,H] or [B,T,H,dv]; S0 [B,H,dk,dv].
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import numpy as np
import torch

_IO = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Problem:
    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int
    chunk: int
    io: str            # "f32" or "bf16"
    alpha: str         # "none", "scalar" or "channel"
    beta_k: str        # "scalar" or "channel"
    beta_v: str        # "none", "scalar" or "channel"
    S0: str            # "zero" or "normal"
    seed: int
    s_scale: str = "none"  # "none" or "channel": OSDN write-side key scale s [B,T,H,dk]

    @property
    def token_heads(self) -> int:
        return self.B * self.T * self.H

    def replace(self, **kw) -> "Problem":
        return dataclasses.replace(self, **kw)


@dataclass(frozen=True)
class DecodeProblem:
    name: str
    B: int
    H: int
    dk: int
    dv: int
    io: str
    alpha: str
    beta_k: str
    beta_v: str
    pool: int          # distinct step inputs; step s uses pool[s % pool]
    steps: int
    seed: int


# The five workloads: pure DeltaNet (fp32), Gated DeltaNet, KDA / FG2-GDN
# (channel-wise gate and strength), FG2-GDN+ (decoupled erase/write, long
# prefill) and a single-token recurrent decode step.
CONFIGS = {
    "deltanet_f32": Problem("deltanet_f32", 1, 2, 256, 64, 64, 64, "f32", "none", "scalar",
                            "none", "zero", 0),
    "gdn_bf16": Problem("gdn_bf16", 4, 16, 4096, 128, 128, 64, "bf16", "scalar", "scalar",
                        "none", "zero", 1),
    "kda_bf16": Problem("kda_bf16", 2, 16, 8192, 128, 128, 64, "bf16", "channel", "channel",
                        "none", "normal", 2),
    "fg2plus_bf16": Problem("fg2plus_bf16", 1, 32, 32768, 128, 128, 64, "bf16", "channel",
                            "channel", "channel", "zero", 3),
}
DECODE = DecodeProblem("decode_bf16", 256, 32, 128, 128, "bf16", "channel", "channel", "none",
                       16, 1000, 4)


def problem(name: str, **overrides) -> Problem:
    return CONFIGS[name].replace(**overrides) if overrides else CONFIGS[name]


def _normal(rng, shape):
    return rng.standard_normal(size=shape, dtype=np.float32)


def _l2_rows(x):
    n = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True))
    return (x / n).astype(np.float32)


def _alpha_from(x):
    # exp(-0.1 * softplus(x)); softplus computed as logaddexp(0, x)
    return np.exp(-0.1 * np.logaddexp(np.float32(0.0), x)).astype(np.float32)


def _sigmoid(x):
    return (1.0 / (1.0 + np.exp(-x))).astype(np.float32)


def _gate_shape(mode, lead, width):
    return lead if mode == "scalar" else lead + (width,)


def make_inputs(p: Problem) -> dict:
    """Draw one problem's inputs.  Keys: q, k, v, alpha, beta_k, beta_v, S0, s (absent -> None)."""
    rng = np.random.Generator(np.random.PCG64(p.seed))
    lead = (p.B, p.T, p.H)
    q = _l2_rows(_normal(rng, lead + (p.dk,)))
    k = _l2_rows(_normal(rng, lead + (p.dk,)))
    v = _normal(rng, lead + (p.dv,))
    alpha = _alpha_from(_normal(rng, _gate_shape(p.alpha, lead, p.dk))) if p.alpha != "none" else None
    beta_k = _sigmoid(_normal(rng, _gate_shape(p.beta_k, lead, p.dk)))
    beta_v = _sigmoid(_normal(rng, _gate_shape(p.beta_v, lead, p.dv))) if p.beta_v != "none" else None
    S0 = (np.float32(0.1) * _normal(rng, (p.B, p.H, p.dk, p.dv))) if p.S0 == "normal" else None
    s = np.exp(np.float32(0.25) * _normal(rng, lead + (p.dk,))).astype(np.float32) if p.s_scale != "none" else None
    io = _IO[p.io]
    t = torch.from_numpy
    return {
        "q": t(q).to(io), "k": t(k).to(io), "v": t(v).to(io),
        "alpha": None if alpha is None else t(alpha),
        "beta_k": t(beta_k),
        "beta_v": None if beta_v is None else t(beta_v),
        "S0": None if S0 is None else t(S0),
        "s": None if s is None else t(s),
    }


def decode_inputs(p: DecodeProblem = DECODE, B: int | None = None) -> dict:
    """State and a pool of single-token step inputs for the recurrent decode workload.

    Keys: S [B,H,dk,dv] fp32; q, k [P,B,1,H,dk], v [P,B,1,H,dv] in the I/O dtype;
    alpha, beta_k [P,B,1,H,dk] (channel) fp32; beta_v None.  ``B`` overrides the
    batch (for smaller test cases) without changing the recipe.
    """
    B = p.B if B is None else B
    rng = np.random.Generator(np.random.PCG64(p.seed))
    S = np.float32(0.1) * _normal(rng, (B, p.H, p.dk, p.dv))
    lead = (p.pool, B, 1, p.H)
    q = _l2_rows(_normal(rng, lead + (p.dk,)))
    k = _l2_rows(_normal(rng, lead + (p.dk,)))
    v = _normal(rng, lead + (p.dv,))
    alpha = _alpha_from(_normal(rng, _gate_shape(p.alpha, lead, p.dk)))
    beta_k = _sigmoid(_normal(rng, _gate_shape(p.beta_k, lead, p.dk)))
    io = _IO[p.io]
    t = torch.from_numpy
    return {"S": t(S), "q": t(q).to(io), "k": t(k).to(io), "v": t(v).to(io),
            "alpha": t(alpha), "beta_k": t(beta_k), "beta_v": None}
