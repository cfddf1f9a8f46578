"""Out-of-bounds writes of every kernel, caught by canary padding (the stand-in for a memory checker).

Each output (and the in-place decode state, and the backward pass's workspace) is a view into a
larger buffer whose guard bytes -- 64 KiB before and after -- hold a sentinel pattern.  After the
call through the C ABI every guard byte must be unchanged, and the output must equal the same
call's output into a plain buffer.  The cases are the ones where a store past the end would hide:
ragged last chunks (T = 1, 63, 65, 333), packed sequences of length 0 and 1, decode on every
kernel, the state-map kernel and the backward pass.
"""
import ctypes
import math

import pytest
import torch

from synth import make_inputs, problem

pytestmark = pytest.mark.gpu

PAD = 1 << 16
FILL = 0xA7


def _guarded(shape, dtype, init=None):
    """A contiguous tensor of `shape` inside a sentinel-filled byte buffer, 16-byte aligned."""
    esize = torch.tensor([], dtype=dtype).element_size()
    n = math.prod(shape) * esize
    buf = torch.full((PAD + n + PAD,), FILL, dtype=torch.uint8, device="cuda")
    view = buf[PAD:PAD + n].view(dtype).view(shape)
    if init is not None:
        view.copy_(init)
    return buf, view, n


def _intact(buf, n):
    torch.cuda.synchronize()
    return bool((buf[:PAD] == FILL).all()) and bool((buf[PAD + n:] == FILL).all())


def _dev(x):
    return {k: (None if t is None else t.cuda()) for k, t in x.items()}


PREFILL = [
    ("gdn_bf16", dict(B=1, H=2, T=1)),
    ("gdn_bf16", dict(B=2, H=2, T=63, S0="normal")),
    ("kda_bf16", dict(B=1, H=3, T=65)),
    ("fg2plus_bf16", dict(B=1, H=2, T=333)),
    ("kda_bf16", dict(B=1, H=2, T=130, dv=64, beta_v="channel")),            # one CTA per value slice
    ("gdn_bf16", dict(B=1, H=2, T=77, chunk=32)),                            # CUDA-core kernel, bf16
    ("deltanet_f32", dict(T=100)),                                           # CUDA-core kernel, fp32
    ("deltanet_f32", dict(T=1, dk=128, dv=128)),
]


@pytest.mark.parametrize("name,kw", PREFILL)
def test_prefill_writes_stay_inside_outputs(name, kw):
    import weight_recurrence_chunkwise_b200 as dr

    p = problem(name, **kw)
    g = _dev(make_inputs(p))
    o_ref, S_ref = dr.dr_chunk_fwd(g["q"], g["k"], g["v"], g["beta_k"], alpha=g["alpha"], beta_v=g["beta_v"],
                                   S0=g["S0"], chunk=p.chunk)
    ob, o, on = _guarded(o_ref.shape, o_ref.dtype)
    sb, S, sn = _guarded(S_ref.shape, torch.float32)
    dr.dr_chunk_fwd(g["q"], g["k"], g["v"], g["beta_k"], alpha=g["alpha"], beta_v=g["beta_v"], S0=g["S0"],
                    chunk=p.chunk, o=o, S_T=S)
    assert _intact(ob, on) and _intact(sb, sn)
    assert torch.equal(o, o_ref) and torch.equal(S, S_ref)


@pytest.mark.parametrize("io,lengths", [("bf16", [0, 1, 63, 65, 0, 130]), ("bf16", [1]), ("f32", [0, 1, 17, 0])])
def test_varlen_writes_stay_inside_outputs(io, lengths):
    import weight_recurrence_chunkwise_b200 as dr

    name = "kda_bf16" if io == "bf16" else "deltanet_f32"
    tot = sum(lengths)
    p = problem(name, B=1, H=2, T=tot, S0="normal")
    g = _dev(make_inputs(p))
    cu = torch.tensor([0] + list(torch.tensor(lengths).cumsum(0).tolist()), dtype=torch.int32, device="cuda")
    n = len(lengths)
    S0 = torch.randn(n, p.H, p.dk, p.dv, device="cuda") * 0.1
    o_ref, S_ref = dr.dr_chunk_fwd_varlen(g["q"], g["k"], g["v"], g["beta_k"], cu, alpha=g["alpha"],
                                          beta_v=g["beta_v"], S0=S0, chunk=p.chunk)
    ob, o, on = _guarded(o_ref.shape, o_ref.dtype)
    sb, S, sn = _guarded(S_ref.shape, torch.float32)
    dr.dr_chunk_fwd_varlen(g["q"], g["k"], g["v"], g["beta_k"], cu, alpha=g["alpha"], beta_v=g["beta_v"], S0=S0,
                           chunk=p.chunk, o=o, S_T=S)
    assert _intact(ob, on) and _intact(sb, sn)
    assert torch.equal(o, o_ref) and torch.equal(S, S_ref)


@pytest.mark.parametrize("variant", ["per_head", "split4", "stream"])
@pytest.mark.parametrize("B,H,d", [(1, 3, 128), (5, 31, 128), (2, 3, 64)])
def test_decode_writes_stay_inside_state_and_output(variant, B, H, d):
    import weight_recurrence_chunkwise_b200 as dr

    if d != 128 and variant != "per_head":
        pytest.skip("the split and streaming decode kernels take dk = dv = 128")
    p = problem("kda_bf16", B=B, H=H, T=1, dk=d, dv=d, S0="normal")
    g = _dev(make_inputs(p))
    S_ref = g["S0"].clone()
    o_ref = dr.dr_diag_decode_step_variant(variant, g["q"], g["k"], g["v"], g["beta_k"], S_ref, alpha=g["alpha"])
    sb, S, sn = _guarded(S_ref.shape, torch.float32, init=g["S0"])
    ob, o, on = _guarded(o_ref.shape, o_ref.dtype)
    dr.dr_diag_decode_step_variant(variant, g["q"], g["k"], g["v"], g["beta_k"], S, alpha=g["alpha"], o=o)
    assert _intact(sb, sn) and _intact(ob, on)
    assert torch.equal(o, o_ref) and torch.equal(S, S_ref)


@pytest.mark.parametrize("n,dk,dv", [(3, 128, 128), (5, 64, 96), (1, 128, 32)])
def test_state_map_writes_stay_inside_output(n, dk, dv):
    import weight_recurrence_chunkwise_b200 as dr

    gen = torch.Generator().manual_seed(n * dk + dv)
    M = torch.randn(n, dk, dk, generator=gen).cuda()
    S = torch.randn(n, dk, dv, generator=gen).cuda()
    N = torch.randn(n, dk, dv, generator=gen).cuda()
    ref = dr.dr_state_map_apply(M, N, S)
    ob, out, on = _guarded(ref.shape, torch.float32)
    dr.dr_state_map_apply(M, N, S, out=out)
    assert _intact(ob, on)
    assert torch.equal(out, ref)


@pytest.mark.parametrize("name,kw", [("gdn_bf16", dict(B=1, H=2, T=77, S0="normal")),
                                     ("fg2plus_bf16", dict(B=1, H=2, T=33, s_scale="channel")),
                                     ("deltanet_f32", dict(T=50))])
def test_backward_writes_stay_inside_gradients_and_workspace(name, kw):
    import weight_recurrence_chunkwise_b200 as dr
    from weight_recurrence_chunkwise_b200 import _binding as Bd

    p = problem(name, **kw)
    g = _dev(make_inputs(p))
    gen = torch.Generator().manual_seed(7)
    dout = torch.randn(g["v"].shape, generator=gen).to(g["v"].dtype).cuda()
    dST = torch.randn((p.B, p.H, p.dk, p.dv), generator=gen).cuda()
    ref = dr.dr_backward(g["q"], g["k"], g["v"], g["beta_k"], dout, alpha=g["alpha"], beta_v=g["beta_v"], s=g["s"],
                         S0=g["S0"], dS_T=dST)
    prob = Bd.make_problem(g["q"], g["v"], g["alpha"], g["beta_k"], g["beta_v"], 64)
    need = int(Bd.lib().dr_backward_workspace(ctypes.byref(prob)))
    grads = {}
    for key, t in ref.items():
        if t is not None:
            grads[key] = _guarded(t.shape, torch.float32)
    wb, wsp, wn = _guarded((need,), torch.uint8)
    P = lambda key: Bd._ptr(grads[key][1]) if key in grads else None
    rc = Bd.lib().dr_backward(ctypes.byref(prob), Bd._ptr(g["q"]), Bd._ptr(g["k"]), Bd._ptr(g["v"]),
                              Bd._ptr(g["alpha"]), Bd._ptr(g["beta_k"]), Bd._ptr(g["beta_v"]), Bd._ptr(g["s"]),
                              Bd._ptr(g["S0"]), Bd._ptr(dout), Bd._ptr(dST), P("q"), P("k"), P("v"), P("alpha"),
                              P("beta_k"), P("beta_v"), P("s"), P("S0"), Bd._ptr(wsp), ctypes.c_size_t(need),
                              Bd._stream(None, "cuda"))
    assert rc == dr.DR_OK
    assert _intact(wb, wn)
    for key, (buf, view, n) in grads.items():
        assert _intact(buf, n), key
        # per-key-channel gradients are sums over value slices taken with atomics: equal up to the
        # order of those additions
        tol = 1e-5 * float(ref[key].abs().max()) + 1e-30
        assert torch.allclose(view, ref[key], rtol=1e-4, atol=tol), key
