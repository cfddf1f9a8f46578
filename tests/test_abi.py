"""Host-side checks of the C ABI: the library loads without a GPU, exports every
symbol the headers declare, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

import weight_recurrence_chunkwise_b200 as dr
from weight_recurrence_chunkwise_b200 import _binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", f)).read()
            names |= set(re.findall(r"DR_API\s+[\w\s\*]+?\b(dr_\w+)\s*\(", txt))
    return names


def _declared_arity():
    """Parameter count of every DR_API function, from the headers."""
    out = {}
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", f)).read()
            for name, params in re.findall(r"DR_API\s+[\w\s\*]+?\b(dr_\w+)\s*\(([^)]*)\)", txt):
                params = params.strip()
                out[name] = 0 if params in ("", "void") else params.count(",") + 1
    return out


@pytest.fixture(scope="module")
def lib():
    from weight_recurrence_chunkwise_b200 import build

    build.build()
    return dr.lib()


def test_every_declared_symbol_is_exported(lib):
    names = _declared_symbols()
    assert {"dr_chunk_fwd", "dr_decode_step", "dr_chunk_fwd_workspace", "dr_workspace_status",
            "dr_status_string", "dr_version"} <= names
    for n in names:
        assert hasattr(lib, n), f"{n} declared but not exported"
    assert set(B.EXPORTS) == names


def test_binding_argument_counts_match_the_headers(lib):
    """Every ctypes prototype the binding sets up has the declared number of parameters."""
    arity = _declared_arity()
    assert set(arity) == set(B.EXPORTS)
    for name, n in arity.items():
        assert len(getattr(lib, name).argtypes) == n, (name, len(getattr(lib, name).argtypes), n)


def test_version_and_status_strings(lib):
    assert lib.dr_version() >= 100
    for code in range(8):
        assert dr.status_string(code).startswith("DR_")


def _prob(**kw):
    base = dict(B=1, T=8, H=1, dk=128, dv=128, chunk=64, io_dtype=B.DR_BF16, alpha_mode=B.DR_SCALAR,
                beta_k_mode=B.DR_SCALAR, beta_v_mode=B.DR_ABSENT)
    base.update(kw)
    return B.dr_problem(*[base[f] for f, _ in B.dr_problem._fields_])


FAKE = ctypes.c_void_p(0x10000)      # aligned, never dereferenced: validation fails first
MISALIGNED = ctypes.c_void_p(0x10004)


def _chunk(lib, p, q=FAKE, alpha=FAKE, beta_v=None, ws=FAKE, ws_bytes=256):
    return lib.dr_chunk_fwd(ctypes.byref(p), q, FAKE, FAKE, alpha, FAKE, beta_v, None, FAKE, FAKE, ws,
                            ctypes.c_size_t(ws_bytes), None)


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), B.DR_ERR_INVALID_ARG),
    (dict(T=-1), B.DR_ERR_INVALID_ARG),
    (dict(dk=96), B.DR_ERR_UNSUPPORTED),
    (dict(dv=256), B.DR_ERR_UNSUPPORTED),
    (dict(chunk=48), B.DR_ERR_UNSUPPORTED),
    (dict(H=70000), B.DR_ERR_UNSUPPORTED),  # the prefill grids index H and B in y and z
    (dict(B=65536), B.DR_ERR_UNSUPPORTED),
    (dict(chunk=0), B.DR_ERR_INVALID_ARG),
    (dict(io_dtype=7), B.DR_ERR_INVALID_ARG),
    (dict(beta_k_mode=B.DR_ABSENT), B.DR_ERR_INVALID_ARG),
    (dict(beta_k_mode=B.DR_CHANNEL, dv=64), B.DR_ERR_INVALID_ARG),  # sqrt(beta_k) (.) v needs dk == dv
])
def test_chunk_fwd_rejects_bad_problems(lib, kw, code):
    assert _chunk(lib, _prob(**kw)) == code
    assert lib.dr_chunk_fwd_workspace(ctypes.byref(_prob(**kw))) == 0


def test_chunk_fwd_pointer_checks(lib):
    p = _prob()
    assert _chunk(lib, p, q=None) == B.DR_ERR_INVALID_ARG
    assert _chunk(lib, p, alpha=None) == B.DR_ERR_INVALID_ARG            # mode says scalar
    assert _chunk(lib, _prob(alpha_mode=B.DR_ABSENT)) == B.DR_ERR_INVALID_ARG  # pointer but mode absent
    assert _chunk(lib, p, beta_v=FAKE) == B.DR_ERR_INVALID_ARG           # mode says absent
    assert _chunk(lib, p, q=MISALIGNED) == B.DR_ERR_ALIGNMENT
    assert _chunk(lib, p, ws=None) == B.DR_ERR_WORKSPACE
    assert _chunk(lib, p, ws_bytes=8) == B.DR_ERR_WORKSPACE
    assert lib.dr_chunk_fwd_workspace(ctypes.byref(p)) >= 4


def test_decode_checks(lib):
    p = _prob(T=2)
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, None]
    assert lib.dr_decode_step(ctypes.byref(p), *args) == B.DR_ERR_INVALID_ARG  # T must be 1
    p = _prob(T=1)
    bad = list(args)
    bad[6] = None  # S
    assert lib.dr_decode_step(ctypes.byref(p), *bad) == B.DR_ERR_INVALID_ARG
    bad = list(args)
    bad[6] = MISALIGNED
    assert lib.dr_decode_step(ctypes.byref(p), *bad) == B.DR_ERR_ALIGNMENT
    assert lib.dr_decode_step(None, *args) == B.DR_ERR_INVALID_ARG


def test_python_binding_requires_cuda_tensors():
    import torch

    q = torch.zeros(1, 4, 1, 64)
    with pytest.raises((ValueError, TypeError)):
        dr.dr_chunk_fwd(q, q, q, torch.zeros(1, 4, 1))
