"""GPU parity of each tensor-core prefill kernel for dk = dv = 128, chunk 64.

The library picks its kernel once per process from DR_PREFILL_KERNEL (ring: default, two CTAs
and three factor slots; pair: two CTAs and two slots; single: one CTA per value slice), so each
variant runs in a child process.  Cases cover ragged lengths, one to many chunks (the slot ring
wraps several times), scalar and channel gates, and the symmetric and separate write strengths.
"""
import os
import subprocess
import sys
import zlib

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = [
    # (T, alpha, beta_k, beta_v, S0)
    (1, "scalar", "scalar", "none", "zero"),
    (63, "scalar", "scalar", "none", "normal"),
    (200, "scalar", "scalar", "scalar", "normal"),
    (453, "none", "scalar", "none", "zero"),
    (2048, "scalar", "scalar", "none", "normal"),
    (130, "channel", "channel", "none", "normal"),
    (333, "channel", "channel", "channel", "zero"),
    (389, "scalar", "channel", "channel", "normal"),
    (260, "channel", "scalar", "scalar", "normal"),
]


def _run_cases():
    import numpy as np  # noqa: F401
    import torch

    sys.path.insert(0, ROOT)
    import weight_recurrence_chunkwise_b200 as dr
    from synth import make_inputs, problem
    from tests.test_gpu_parity import check, ref_prefill, run_prefill

    dr.lib()
    for case in CASES:
        T, a, bk, bv, s0 = case
        p = problem("kda_bf16", B=1, H=3, T=T, dk=128, dv=128, chunk=64, io="bf16", alpha=a, beta_k=bk,
                    beta_v=bv, S0=s0, seed=zlib.crc32(repr(case).encode()) % 1000)
        x = make_inputs(p)
        o, S_T = run_prefill(dr, x, 64)
        ref_o, ref_S = ref_prefill(x)
        e_o, e_S = check(p, o, S_T, ref_o, ref_S)
        print(f"{os.environ.get('DR_PREFILL_KERNEL', 'ring')} {case}: err_o={e_o:.2e} err_S={e_S:.2e}")
    assert torch.cuda.is_available()


@pytest.mark.parametrize("variant", ["ring", "pair", "single"])
def test_prefill_kernel_variant(variant):
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    env = dict(os.environ, DR_PREFILL_KERNEL=variant)
    r = subprocess.run([sys.executable, os.path.abspath(__file__)], env=env, cwd=ROOT, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]


if __name__ == "__main__":
    _run_cases()
