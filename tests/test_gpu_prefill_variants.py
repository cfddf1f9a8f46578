"""GPU parity of every prefill kernel on the same problems, for dk = dv = 128 and chunk 64.

The library's choice (dr_chunk_fwd) and the other kernels, named through
dr_diag_chunk_fwd_variant (include/deltarule_diag.h): the tensor-core kernel with one CTA per
64-column value slice, the CUDA-core kernel, and the two cluster kernels (two CTAs per head with a
ring of factor slots; four CTAs per head with the factor blocks staged through global memory).
Cases cover ragged lengths, one to many chunks (the factor slots and staging entries wrap several
times), fewer chunks than CTAs in a cluster, scalar and channel gates, and the symmetric and
separate write strengths; each result is checked against the float64 oracle.
"""
import zlib

import pytest

pytestmark = pytest.mark.gpu

CASES = [
    # (T, alpha, beta_k, beta_v, S0)
    (1, "scalar", "scalar", "none", "zero"),
    (129, "channel", "scalar", "none", "normal"),
    (63, "scalar", "scalar", "none", "normal"),
    (200, "scalar", "scalar", "scalar", "normal"),
    (453, "none", "scalar", "none", "zero"),
    (2048, "scalar", "scalar", "none", "normal"),
    (130, "channel", "channel", "none", "normal"),
    (333, "channel", "channel", "channel", "zero"),
    (389, "scalar", "channel", "channel", "normal"),
    (260, "channel", "scalar", "scalar", "normal"),
]


@pytest.mark.parametrize("variant", ["default", "single", "simt", "ring", "quad"])
def test_prefill_kernel_variant(variant):
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_recurrence_chunkwise_b200 as dr
    from synth import make_inputs, problem
    from tests.test_gpu_parity import check, ref_prefill

    for case in CASES:
        T, a, bk, bv, s0 = case
        p = problem("kda_bf16", B=1, H=3, T=T, dk=128, dv=128, chunk=64, io="bf16", alpha=a, beta_k=bk,
                    beta_v=bv, S0=s0, seed=zlib.crc32(repr(case).encode()) % 1000)
        x = make_inputs(p)
        g = {n: (None if t is None else t.cuda()) for n, t in x.items()}
        o, S_T = dr.dr_diag_chunk_fwd_variant(variant, g["q"], g["k"], g["v"], g["beta_k"], alpha=g["alpha"],
                                              beta_v=g["beta_v"], S0=g["S0"], chunk=64)
        torch.cuda.synchronize()
        ref_o, ref_S = ref_prefill(x)
        check(p, o.cpu(), S_T.cpu(), ref_o, ref_S)


def test_unsupported_variant_is_refused():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_recurrence_chunkwise_b200 as dr
    from synth import make_inputs, problem

    p = problem("deltanet_f32", B=1, H=1, T=64)  # fp32 I/O: no tensor-core kernel
    g = {n: (None if t is None else t.cuda()) for n, t in make_inputs(p).items()}
    with pytest.raises(dr.DeltaRuleError) as e:
        dr.dr_diag_chunk_fwd_variant("single", g["q"], g["k"], g["v"], g["beta_k"], alpha=g["alpha"], chunk=64)
    assert e.value.code == dr.DR_ERR_UNSUPPORTED


def test_workspace_size_selects_the_cluster_kernel():
    """The library's choice with a workspace that holds only the status word is the two-CTA kernel's
    result, bit for bit; with dr_chunk_fwd_workspace bytes it is the four-CTA kernel's."""
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import weight_recurrence_chunkwise_b200 as dr
    from synth import make_inputs, problem

    p = problem("kda_bf16", B=1, H=2, T=300, dk=128, dv=128, chunk=64, io="bf16", alpha="channel",
                beta_k="channel", beta_v="none", S0="normal", seed=11)
    g = {n: (None if t is None else t.cuda()) for n, t in make_inputs(p).items()}
    args = (g["q"], g["k"], g["v"], g["beta_k"])
    kw = dict(alpha=g["alpha"], beta_v=g["beta_v"], S0=g["S0"], chunk=64)
    need = dr.workspace_bytes(dr.make_problem(g["q"], g["v"], g["alpha"], g["beta_k"], g["beta_v"], 64))
    assert need > 256  # two heads: the four-CTA kernel's clusters are resident
    o_small, S_small = dr.dr_chunk_fwd(*args, **kw, workspace=torch.zeros(256, dtype=torch.uint8, device="cuda"))
    o_ring, S_ring = dr.dr_diag_chunk_fwd_variant("ring", *args, **kw)
    o_full, S_full = dr.dr_chunk_fwd(*args, **kw)
    o_quad, S_quad = dr.dr_diag_chunk_fwd_variant("quad", *args, **kw)
    torch.cuda.synchronize()
    assert torch.equal(o_small, o_ring) and torch.equal(S_small, S_ring)
    assert torch.equal(o_full, o_quad) and torch.equal(S_full, S_quad)
