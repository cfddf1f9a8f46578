"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Error measure (both sides see the same rounded inputs):
    err_o = max |o_gpu - o_ref| / rms(o_ref),   err_S = max |S_gpu - S_ref| / rms(S_ref)
Bounds: fp32 I/O 1e-4 for both; bf16 I/O err_o <= 2e-2 and err_S <= 1e-2.
"""
import zlib

import numpy as np
import pytest
import torch

import oracle
from synth import CONFIGS, DECODE, decode_inputs, make_inputs, problem

pytestmark = pytest.mark.gpu

TOL = {"f32": (1e-4, 1e-4), "bf16": (2e-2, 1e-2)}


@pytest.fixture(scope="module")
def dr():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_recurrence_chunkwise_b200 as m
    from weight_recurrence_chunkwise_b200 import build

    build.build()
    m.lib()
    return m


# Relative rounding bound of the output's own dtype (round-to-nearest-even): the
# CUDA path must return o in the I/O dtype, so each element may carry this much
# on top of the stated tolerance.
OUT_ROUND = {"f32": 2.0 ** -24, "bf16": 2.0 ** -8}


def err(x, ref, round_rel=0.0):
    """max_i (|x_i - ref_i| - round_rel |ref_i|)_+ / rms(ref)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = np.maximum(np.abs(x - ref) - round_rel * np.abs(ref), 0.0)
    return float(d.max() / max(np.sqrt(np.mean(ref ** 2)), 1e-30))


def to_dev(x):
    return {k: (None if t is None else t.cuda()) for k, t in x.items()}


def run_prefill(dr, x, chunk, S0=None):
    g = to_dev(x)
    o, S_T = dr.dr_chunk_fwd(g["q"], g["k"], g["v"], g["beta_k"], alpha=g["alpha"], beta_v=g["beta_v"],
                             S0=g["S0"] if S0 is None else S0, chunk=chunk)
    torch.cuda.synchronize()
    return o, S_T


def ref_prefill(x, heads=None):
    if heads is not None:
        x = slice_heads(x, heads)
    return oracle.delta_rule_sequential(x["q"], x["k"], x["v"], x["beta_k"], alpha=x["alpha"],
                                        beta_v=x["beta_v"], S0=x["S0"])


def slice_heads(x, heads):
    """Stack the selected (b, h) heads as a batch of single-head problems."""
    out = {}
    for n, t in x.items():
        if t is None:
            out[n] = None
        elif n == "S0":
            out[n] = torch.stack([t[b, h] for b, h in heads])[:, None]
        else:
            out[n] = torch.stack([t[b, :, h] for b, h in heads])[:, :, None]
    return out


def check(p, o, S_T, ref_o, ref_S):
    to, ts = TOL[p.io]
    e_o, e_S = err(o.float().cpu().numpy(), ref_o, OUT_ROUND[p.io]), err(S_T.cpu().numpy(), ref_S)
    assert e_o <= to and e_S <= ts, f"{p}: err_o={e_o:.3e} (<= {to}), err_S={e_S:.3e} (<= {ts})"
    return e_o, e_S


# ------------------------------------------------------------------------- tcgen05 building blocks
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("N,K", [(64, 64), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1), (1, 0), (1, 1)])
def test_umma_building_blocks(dr, N, K, a_mn, b_mn, dtype):
    g = torch.Generator().manual_seed(N * 1000 + K + 10 * a_mn + b_mn)
    A = torch.randn(128, K, generator=g).to(dtype)
    Bm = torch.randn(K, N, generator=g).to(dtype)
    D, status = dr.dr_diag_umma_selftest(A.cuda(), Bm.cuda(), bool(a_mn), bool(b_mn))
    assert status == dr.DR_OK
    ref = A.double() @ Bm.double()
    np.testing.assert_allclose(D.cpu().double().numpy(), ref.numpy(), rtol=1e-4, atol=1e-3)


def _unit_lower_case(seed, scale):
    g = torch.Generator().manual_seed(seed)
    return torch.tril(scale * torch.randn(64, 64, generator=g, dtype=torch.float64), -1)


@pytest.mark.parametrize("variant", [0, 1])
@pytest.mark.parametrize("seed,scale", [(0, 0.05), (1, 0.15), (2, 0.3)])
def test_tri_inverse_building_block(dr, seed, scale, variant):
    """The warp-MMA UT-transform inverse (the ring prefill's, and the one-CTA prefill's) against a
    float64 matrix inverse."""
    A = _unit_lower_case(seed, scale)
    ref = torch.linalg.inv(torch.eye(64, dtype=torch.float64) + A)
    T = dr.dr_diag_tri_inverse(A.float().cuda(), variant=variant).double().cpu()
    assert torch.equal(torch.triu(T, 1), torch.zeros_like(T))          # lower triangular
    assert torch.allclose(torch.diagonal(T), torch.ones(64, dtype=torch.float64), atol=1e-6)
    assert float((T - ref).abs().max() / ref.abs().max()) <= 5e-3


@pytest.mark.parametrize("variant", [0, 1])
def test_tri_inverse_on_key_gram_matrix(dr, variant):
    """A shaped like a real chunk: A_ij = sqrt(b_i b_j) k_i . k_j (unit keys, strengths in (0,1))."""
    g = torch.Generator().manual_seed(7)
    k = torch.nn.functional.normalize(torch.randn(64, 128, generator=g, dtype=torch.float64), dim=-1)
    beta = torch.sigmoid(torch.randn(64, generator=g, dtype=torch.float64))
    kb = k * beta.sqrt()[:, None]
    A = torch.tril(kb @ kb.T, -1)
    ref = torch.linalg.inv(torch.eye(64, dtype=torch.float64) + A)
    T = dr.dr_diag_tri_inverse(A.float().cuda(), variant=variant).double().cpu()
    assert float((T - ref).abs().max() / ref.abs().max()) <= 5e-3


# ------------------------------------------------------------------------- prefill, small shapes
SMALL = [
    # (dk, dv, T, chunk, io, alpha, beta_k, beta_v, S0)
    (64, 64, 256, 64, "f32", "none", "scalar", "none", "zero"),
    (64, 64, 1, 64, "f32", "scalar", "scalar", "none", "normal"),
    (128, 128, 200, 64, "f32", "channel", "channel", "none", "normal"),
    (128, 128, 200, 32, "f32", "channel", "channel", "channel", "zero"),
    (128, 64, 77, 16, "f32", "scalar", "scalar", "channel", "normal"),
    (128, 128, 1, 64, "bf16", "scalar", "scalar", "none", "zero"),
    (128, 128, 63, 64, "bf16", "scalar", "scalar", "none", "normal"),
    (128, 128, 200, 64, "bf16", "scalar", "scalar", "none", "zero"),
    (128, 128, 200, 64, "bf16", "channel", "channel", "none", "normal"),
    (128, 128, 333, 64, "bf16", "channel", "channel", "channel", "zero"),
    (128, 128, 130, 32, "bf16", "channel", "channel", "channel", "normal"),
    (128, 128, 130, 16, "bf16", "none", "scalar", "none", "normal"),
    (64, 64, 150, 64, "bf16", "channel", "channel", "none", "normal"),
    (128, 64, 150, 64, "bf16", "channel", "channel", "scalar", "zero"),
    (64, 128, 150, 32, "bf16", "scalar", "channel", "channel", "normal"),
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "dk{}_dv{}_T{}_C{}_{}_a{}_bk{}_bv{}_{}".format(*c))
def test_prefill_small(dr, case):
    dk, dv, T, C, io, a, bk, bv, s0 = case
    p = problem("kda_bf16", B=2, H=3, T=T, dk=dk, dv=dv, chunk=C, io=io, alpha=a, beta_k=bk, beta_v=bv,
                S0=s0, seed=zlib.crc32(repr(case).encode()) % 1000)
    x = make_inputs(p)
    o, S_T = run_prefill(dr, x, C)
    ref_o, ref_S = ref_prefill(x)
    check(p, o, S_T, ref_o, ref_S)


def test_prefill_T0_returns_initial_state(dr):
    p = problem("kda_bf16", B=1, H=2, T=0)
    x = make_inputs(p)
    o, S_T = run_prefill(dr, x, 64)
    assert o.numel() == 0
    np.testing.assert_array_equal(S_T.cpu().numpy(), x["S0"].numpy())


def test_prefill_final_state_may_alias_initial(dr):
    p = problem("gdn_bf16", B=1, H=2, T=130, S0="normal")
    x = make_inputs(p)
    g = to_dev(x)
    S = g["S0"].clone()
    o, _ = dr.dr_chunk_fwd(g["q"], g["k"], g["v"], g["beta_k"], alpha=g["alpha"], S0=S, S_T=S, chunk=64)
    torch.cuda.synchronize()
    ref_o, ref_S = ref_prefill(x)
    check(p, o, S, ref_o, ref_S)


# ------------------------------------------------------------------------- prefill, the four workloads
def _sample_heads(p, n, seed=0):
    rng = np.random.default_rng(seed)
    allh = [(b, h) for b in range(p.B) for h in range(p.H)]
    if len(allh) <= n:
        return allh
    idx = rng.choice(len(allh), size=n, replace=False)
    return [allh[i] for i in sorted(idx)]


@pytest.mark.parametrize("name", list(CONFIGS))
def test_prefill_workload_full_size(dr, name):
    """Full-size launch; the oracle checks every output of a sample of heads."""
    p = CONFIGS[name]
    x = make_inputs(p)
    o, S_T = run_prefill(dr, x, p.chunk)
    heads = _sample_heads(p, 4)
    ref_o, ref_S = ref_prefill(x, heads)
    o_s = torch.stack([o[b, :, h] for b, h in heads])[:, :, None]
    S_s = torch.stack([S_T[b, h] for b, h in heads])[:, None]
    check(p, o_s, S_s, ref_o, ref_S)
    assert torch.isfinite(o.float()).all() and torch.isfinite(S_T).all()


# ------------------------------------------------------------------------- decode
def _decode_run(dr, d, steps, heads=None):
    S = d["S"].cuda()
    pool = {k: (None if d[k] is None else d[k].cuda()) for k in ("q", "k", "v", "alpha", "beta_k", "beta_v")}
    outs = []
    for s in range(steps):
        i = s % d["q"].shape[0]
        o = dr.dr_decode_step(pool["q"][i], pool["k"][i], pool["v"][i], pool["beta_k"][i], S,
                              alpha=pool["alpha"][i])
        outs.append(o[:, 0] if heads is None else torch.stack([o[b, 0, h] for b, h in heads]))
    torch.cuda.synchronize()
    return torch.stack(outs), S


def _decode_ref(d, steps, heads):
    P = d["q"].shape[0]
    idx = [s % P for s in range(steps)]
    seq = {}
    for n in ("q", "k", "v", "alpha", "beta_k"):
        # per head: the pool's rows for that head, then the step order -> [nh, steps, 1, d]
        seq[n] = torch.stack([d[n][:, b, 0, h][idx] for b, h in heads])[:, :, None]
    S0 = torch.stack([d["S"][b, h] for b, h in heads])[:, None]
    return oracle.delta_rule_sequential(seq["q"], seq["k"], seq["v"], seq["beta_k"], alpha=seq["alpha"], S0=S0)


def test_decode_small_all_heads(dr):
    d = decode_inputs(B=4)
    steps = 24
    o, S = _decode_run(dr, d, steps)
    heads = [(b, h) for b in range(4) for h in range(DECODE.H)]
    ref_o, ref_S = _decode_ref(d, steps, heads)
    o_h = torch.stack([o[:, b, h] for b, h in heads])[:, :, None]  # [nh, steps, 1, dv]
    S_h = torch.stack([S[b, h] for b, h in heads])[:, None]
    e_o, e_S = err(o_h.float().cpu().numpy(), ref_o, OUT_ROUND["bf16"]), err(S_h.cpu().numpy(), ref_S)
    assert e_o <= 2e-2 and e_S <= 1e-2, (e_o, e_S)


def test_decode_workload_full_size(dr):
    """All 8192 heads, 1000 chained in-place steps; the oracle checks 64 sampled heads."""
    d = decode_inputs()
    heads = _sample_heads(DECODE, 64, seed=4)
    o, S = _decode_run(dr, d, DECODE.steps, heads)
    ref_o, ref_S = _decode_ref(d, DECODE.steps, heads)
    o_h = o.permute(1, 0, 2)[:, :, None]  # [nh, steps, 1, dv]
    S_h = torch.stack([S[b, h] for b, h in heads])[:, None]
    e_o, e_S = err(o_h.float().cpu().numpy(), ref_o, OUT_ROUND["bf16"]), err(S_h.cpu().numpy(), ref_S)
    assert e_o <= 2e-2 and e_S <= 1e-2, (e_o, e_S)
    assert torch.isfinite(S).all()


# ------------------------------------------------------------------------- cross-entry consistency
def test_prefill_equals_chained_decode(dr):
    p = problem("kda_bf16", B=2, H=4, T=40)
    x = make_inputs(p)
    o_p, S_p = run_prefill(dr, x, 64)
    g = to_dev(x)
    S = g["S0"].clone()
    outs = []
    for t in range(p.T):
        sl = lambda z: None if z is None else z[:, t:t + 1].contiguous()
        outs.append(dr.dr_decode_step(sl(g["q"]), sl(g["k"]), sl(g["v"]), sl(g["beta_k"]), S,
                                      alpha=sl(g["alpha"])))
    o_d = torch.cat(outs, dim=1)
    torch.cuda.synchronize()
    assert err(o_d.float().cpu().numpy(), o_p.float().cpu().numpy(), 2 * OUT_ROUND["bf16"]) <= 2e-2
    assert err(S.cpu().numpy(), S_p.cpu().numpy()) <= 1e-2


def test_split_prefill_carries_state(dr):
    p = problem("fg2plus_bf16", B=1, H=4, T=300, S0="normal")
    x = make_inputs(p)
    o_full, S_full = run_prefill(dr, x, 64)
    half = 128
    first = {k: (None if t is None else (t if k == "S0" else t[:, :half].contiguous())) for k, t in x.items()}
    second = {k: (None if t is None else (t if k == "S0" else t[:, half:].contiguous())) for k, t in x.items()}
    o1, S1 = run_prefill(dr, first, 64)
    o2, S2 = run_prefill(dr, second, 64, S0=S1)
    assert err(torch.cat([o1, o2], 1).float().cpu().numpy(), o_full.float().cpu().numpy(), 2 * OUT_ROUND["bf16"]) <= 2e-2
    assert err(S2.cpu().numpy(), S_full.cpu().numpy()) <= 1e-2


def test_constant_channel_gate_equals_scalar_gate(dr):
    p = problem("gdn_bf16", B=1, H=2, T=200, S0="normal")
    x = make_inputs(p)
    o1, S1 = run_prefill(dr, x, 64)
    y = dict(x, alpha=x["alpha"][..., None].expand(-1, -1, -1, p.dk).contiguous(),
             beta_k=x["beta_k"][..., None].expand(-1, -1, -1, p.dk).contiguous())
    o2, S2 = run_prefill(dr, y, 64)
    assert err(o2.float().cpu().numpy(), o1.float().cpu().numpy(), 2 * OUT_ROUND["bf16"]) <= 1e-2
    assert err(S2.cpu().numpy(), S1.cpu().numpy()) <= 5e-3


# ------------------------------------------------------------------------- device-side status
def test_extreme_decay_sets_range_status(dr):
    p = problem("gdn_bf16", B=1, H=1, T=64)
    x = make_inputs(p)
    x["alpha"] = torch.full_like(x["alpha"], 1e-3)  # sum log alpha over a chunk ~ -442
    g = to_dev(x)
    need = dr.workspace_bytes(dr.make_problem(g["q"], g["v"], g["alpha"], g["beta_k"], None, 64))
    ws = torch.zeros(max(need, 256), dtype=torch.uint8, device="cuda")
    dr.dr_chunk_fwd(g["q"], g["k"], g["v"], g["beta_k"], alpha=g["alpha"], chunk=64, workspace=ws)
    assert dr.dr_workspace_status(ws) == dr.DR_ERR_RANGE
    # and a normal call afterwards clears it
    x2 = make_inputs(p)
    g2 = to_dev(x2)
    dr.dr_chunk_fwd(g2["q"], g2["k"], g2["v"], g2["beta_k"], alpha=g2["alpha"], chunk=64, workspace=ws)
    assert dr.dr_workspace_status(ws) == dr.DR_OK
