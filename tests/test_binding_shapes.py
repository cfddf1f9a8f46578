"""The Python binding refuses tensors whose shapes disagree with q [B, T, H, dk] and v [B, T, H, dv]
before anything reaches the library (which sizes every access from those dimensions).  CPU only:
the shape check comes before the device check, so CPU tensors exercise it."""
import pytest
import torch

import weight_recurrence_chunkwise_b200 as dr

B, T, H, DK, DV = 2, 5, 3, 8, 8


def _t(*shape, dtype=torch.float32):
    return torch.zeros(shape, dtype=dtype)


def _inputs():
    bf = torch.bfloat16
    return dict(q=_t(B, T, H, DK, dtype=bf), k=_t(B, T, H, DK, dtype=bf), v=_t(B, T, H, DV, dtype=bf),
                beta_k=_t(B, T, H), alpha=_t(B, T, H, DK), S0=_t(B, H, DK, DV))


@pytest.mark.parametrize("name,bad", [
    ("k", (B, T + 1, H, DK)), ("v", (B, T, H + 1, DV)), ("beta_k", (B, T, H, DK + 1)), ("alpha", (B, T - 1, H)),
    ("S0", (B, H, DK, DV + 8)),
])
def test_prefill_refuses_mismatched_shapes(name, bad):
    x = _inputs()
    x[name] = _t(*bad, dtype=x[name].dtype)
    with pytest.raises(ValueError, match="shape"):
        dr.dr_chunk_fwd(x["q"], x["k"], x["v"], x["beta_k"], alpha=x["alpha"], S0=x["S0"])


def test_prefill_with_matching_shapes_reaches_the_device_check():
    x = _inputs()
    with pytest.raises(ValueError, match="CUDA"):
        dr.dr_chunk_fwd(x["q"], x["k"], x["v"], x["beta_k"], alpha=x["alpha"], S0=x["S0"])


def test_decode_refuses_mismatched_state_and_multi_token_input():
    x = _inputs()
    q1 = x["q"][:, :1].contiguous()
    k1, v1 = x["k"][:, :1].contiguous(), x["v"][:, :1].contiguous()
    b1 = x["beta_k"][:, :1].contiguous()
    with pytest.raises(ValueError, match="shape"):
        dr.dr_decode_step(q1, k1, v1, b1, _t(B, H, DK + 1, DV))
    with pytest.raises(ValueError, match="one token"):
        dr.dr_decode_step(x["q"], x["k"], x["v"], x["beta_k"], x["S0"])


def test_backward_refuses_mismatched_output_gradient():
    x = _inputs()
    with pytest.raises(ValueError, match="shape"):
        dr.dr_backward(x["q"], x["k"], x["v"], x["beta_k"], _t(B, T, H, DV + 1, dtype=torch.bfloat16),
                       alpha=x["alpha"])


def test_varlen_requires_offsets_on_the_device():
    x = {n: (t[:1].contiguous() if n != "S0" else t) for n, t in _inputs().items()}
    cu = torch.tensor([0, 2, 5], dtype=torch.int32)
    with pytest.raises(ValueError):  # cu_seqlens must live on the GPU: refused before any launch
        dr.dr_chunk_fwd_varlen(x["q"], x["k"], x["v"], x["beta_k"], cu, alpha=x["alpha"])
