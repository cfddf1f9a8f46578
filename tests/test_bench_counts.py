"""The algorithmic work counts behind bench.py's roofline fractions, against the per-token figures
derived from the recurrence (chunkwise FLOPs with the triangular masks exploited; HBM bytes with
every input read once and every output written once) and checked by hand for each workload."""
import pytest

import bench
from synth import problem


@pytest.mark.parametrize("name,per_token_bytes", [
    ("deltanet_f32", 4 * (2 * 64 + 2 * 64) + 4),                     # fp32 q, k, v, o; scalar beta
    ("gdn_bf16", 2 * (2 * 128 + 2 * 128) + 4 + 4),                    # bf16; scalar alpha, beta
    ("kda_bf16", 2 * (2 * 128 + 2 * 128) + 4 * 128 + 4 * 128),        # channel alpha, beta
    ("fg2plus_bf16", 2 * (2 * 128 + 2 * 128) + 3 * 4 * 128),          # channel alpha, beta_k, beta_v
])
def test_prefill_bytes(name, per_token_bytes):
    p = problem(name)
    state = p.B * p.H * p.dk * p.dv * 4
    assert bench.prefill_bytes(p, with_S0=False) == p.token_heads * per_token_bytes + state
    assert bench.prefill_bytes(p, with_S0=True) == p.token_heads * per_token_bytes + 2 * state


def test_headline_workload_totals():
    p = problem("gdn_bf16")
    assert p.token_heads == 262_144
    assert bench.prefill_bytes(p, with_S0=False) == 274_726_912  # 1,032 B per token-head + the final states
    assert round(bench.flops_per_token_head(128, 128, 64)) == 140_629
    assert round(bench.flops_per_token_head(64, 64, 64)) == 46_421


def test_decode_bytes():
    # per head and step: fp32 state read and written, bf16 q, k, v, o, channel alpha and beta
    per_head = 2 * 128 * 128 * 4 + 2 * (2 * 128 + 2 * 128) + 4 * 128 + 4 * 128
    assert per_head == 133_120
    assert bench.decode_bytes(256, 32, 128, 128) == 8192 * per_head == 1_090_519_040


def test_backward_bytes():
    p = problem("gdn_bf16")
    per_in = 2 * (2 * 128 + 2 * 128) + 4 + 4                        # q, k, v, dout, scalar gates
    per_out = 4 * (2 * 128 + 128) + 4 + 4                           # fp32 dq, dk, dv, gate gradients
    state = p.B * p.H * 128 * 128 * 4                               # S0, dS_T read; dS0 written
    assert bench.backward_bytes(p) == p.token_heads * (per_in + per_out) + 3 * state


def test_prefill_kernel_names_follow_the_dispatch():
    """The bench names the kernel the library runs: for the cluster shapes, the four-CTA kernel
    exactly when dr_chunk_fwd_workspace asks for more than the 256-byte status word (its factor
    staging), else the two-CTA ring; other shapes their own kernels."""
    fg2 = problem("fg2plus_bf16")
    assert bench.prefill_kernel_name(fg2, 256) == "chunk_fwd_ring_kernel"
    assert bench.prefill_kernel_name(fg2, 256 + fg2.B * fg2.H * 266240) == "chunk_fwd_quad_kernel"
    assert bench.prefill_kernel_name(problem("gdn_bf16", dv=64), 256) == "chunk_fwd_tc_kernel"
    assert bench.prefill_kernel_name(problem("deltanet_f32"), 256) == "chunk_fwd_simt_kernel"
    # traffic is keyed per (kernel, workload) and tied to the kernel's sources
    for kern, wl in (("chunk_fwd_quad_kernel", "fg2plus_bf16"), ("chunk_fwd_quad_kernel", "kda_bf16"),
                     ("chunk_fwd_ring_kernel", "gdn_bf16")):
        assert (kern, wl) in bench.MEASURED_TRAFFIC
