"""ctypes binding of ``libdeltarule.so`` (include/deltarule.h).

Argument marshalling only: shapes become a ``dr_problem``, tensors become
device pointers, status codes become exceptions.  Every step of the operation
runs inside the library's CUDA kernels; there is no host or PyTorch fallback,
and a missing library is an error.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdeltarule.so")

DR_OK, DR_ERR_INVALID_ARG, DR_ERR_UNSUPPORTED, DR_ERR_ALIGNMENT = 0, 1, 2, 3
DR_ERR_WORKSPACE, DR_ERR_RANGE, DR_ERR_TIMEOUT, DR_ERR_CUDA = 4, 5, 6, 7
DR_F32, DR_BF16 = 0, 1
DR_ABSENT, DR_SCALAR, DR_CHANNEL = 0, 1, 2

_DTYPE = {torch.float32: DR_F32, torch.bfloat16: DR_BF16}


class dr_problem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int),
                ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("chunk", ctypes.c_int),
                ("io_dtype", ctypes.c_int), ("alpha_mode", ctypes.c_int),
                ("beta_k_mode", ctypes.c_int), ("beta_v_mode", ctypes.c_int)]


class DeltaRuleError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {status_string(code)}")


_lib = None

EXPORTS = ("dr_chunk_fwd_workspace", "dr_chunk_fwd", "dr_chunk_fwd_osdn", "dr_chunk_fwd_varlen",
           "dr_chunk_fwd_noalloc", "dr_decode_step",
           "dr_decode_step_osdn", "dr_state_map_apply", "dr_backward_workspace", "dr_backward",
           "dr_workspace_status", "dr_noalloc_status", "dr_status_string", "dr_version", "dr_diag_umma_selftest",
           "dr_diag_tri_inverse", "dr_diag_wait_timeout", "dr_diag_chunk_fwd_workspace", "dr_diag_chunk_fwd_variant",
           "dr_diag_decode_step_variant",
           "dr_diag_backward_workspace", "dr_diag_backward_variant")

# kernels of dr_diag_chunk_fwd_variant / dr_diag_decode_step_variant (include/deltarule_diag.h)
PREFILL_VARIANTS = {"default": 0, "single": 1, "simt": 2, "ring": 3, "quad": 4}
DECODE_VARIANTS = {"default": 0, "per_head": 1, "split4": 2, "stream": 3}
BACKWARD_VARIANTS = {"default": 0, "sequential": 1, "chunk": 2}


def lib():
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with weight_recurrence_chunkwise_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, P = ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(dr_problem)
        L.dr_chunk_fwd_workspace.argtypes = [P]
        L.dr_chunk_fwd_workspace.restype = sz
        L.dr_chunk_fwd.argtypes = [P] + [vp] * 9 + [vp, sz, vp]
        L.dr_chunk_fwd.restype = ctypes.c_int
        L.dr_chunk_fwd_noalloc.argtypes = [P] + [vp] * 9 + [vp]
        L.dr_chunk_fwd_noalloc.restype = ctypes.c_int
        L.dr_decode_step.argtypes = [P] + [vp] * 8 + [vp]
        L.dr_decode_step.restype = ctypes.c_int
        L.dr_chunk_fwd_osdn.argtypes = [P] + [vp] * 10 + [vp, sz, vp]
        L.dr_chunk_fwd_osdn.restype = ctypes.c_int
        L.dr_chunk_fwd_varlen.argtypes = [P] + [vp] * 11 + [vp, sz, vp]
        L.dr_chunk_fwd_varlen.restype = ctypes.c_int
        L.dr_state_map_apply.argtypes = [ctypes.c_int] * 3 + [vp] * 5
        L.dr_state_map_apply.restype = ctypes.c_int
        L.dr_backward_workspace.argtypes = [P]
        L.dr_backward_workspace.restype = sz
        L.dr_backward.argtypes = [P] + [vp] * 18 + [vp, sz, vp]
        L.dr_backward.restype = ctypes.c_int
        L.dr_decode_step_osdn.argtypes = [P] + [vp] * 9 + [vp]
        L.dr_decode_step_osdn.restype = ctypes.c_int
        L.dr_workspace_status.argtypes = [vp, vp]
        L.dr_workspace_status.restype = ctypes.c_int
        L.dr_noalloc_status.argtypes = [vp]
        L.dr_noalloc_status.restype = ctypes.c_int
        L.dr_status_string.argtypes = [ctypes.c_int]
        L.dr_status_string.restype = ctypes.c_char_p
        L.dr_version.argtypes = []
        L.dr_version.restype = ctypes.c_int
        L.dr_diag_umma_selftest.argtypes = [ctypes.c_int] * 5 + [vp, vp, vp, vp, vp]
        L.dr_diag_umma_selftest.restype = ctypes.c_int
        L.dr_diag_tri_inverse.argtypes = [ctypes.c_int, vp, vp, vp]
        L.dr_diag_tri_inverse.restype = ctypes.c_int
        L.dr_diag_wait_timeout.argtypes = [ctypes.c_int, ctypes.c_ulonglong, vp, vp, vp]
        L.dr_diag_wait_timeout.restype = ctypes.c_int
        L.dr_diag_chunk_fwd_workspace.argtypes = [ctypes.c_int, P]
        L.dr_diag_chunk_fwd_workspace.restype = sz
        L.dr_diag_chunk_fwd_variant.argtypes = [ctypes.c_int, P] + [vp] * 9 + [vp, sz, vp]
        L.dr_diag_chunk_fwd_variant.restype = ctypes.c_int
        L.dr_diag_decode_step_variant.argtypes = [ctypes.c_int, P] + [vp] * 9 + [vp]
        L.dr_diag_decode_step_variant.restype = ctypes.c_int
        L.dr_diag_backward_workspace.argtypes = [ctypes.c_int, P]
        L.dr_diag_backward_workspace.restype = sz
        L.dr_diag_backward_variant.argtypes = [ctypes.c_int, P] + [vp] * 18 + [vp, sz, vp]
        L.dr_diag_backward_variant.restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().dr_status_string(int(code)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device):
    """The raw handle of ``stream``, else of ``device``'s current stream; a stream of another device
    than the data's is refused (its kernels would run on one GPU with another GPU's pointers)."""
    device = _dev(device)
    if stream is None:
        stream = torch.cuda.current_stream(device)
    elif stream.device != device:
        raise ValueError(f"stream is on {stream.device}, the tensors on {device}")
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(device):
    """``device`` as a CUDA device with an index (a bare "cuda" is the current device)."""
    device = torch.device(device)
    if device.type != "cuda":
        raise ValueError(f"expected a CUDA device, got {device}")
    return device if device.index is not None else torch.device("cuda", torch.cuda.current_device())


def _call(name, device, *args):
    """Call library function ``name`` with ``device`` current: the library launches on, and looks up
    per-device state of, the current device."""
    with torch.cuda.device(_dev(device)):
        return getattr(lib(), name)(*args)


def _mode(x, scalar_ndim):
    if x is None:
        return DR_ABSENT
    return DR_SCALAR if x.dim() == scalar_ndim else DR_CHANNEL


def make_problem(q, v, alpha, beta_k, beta_v, chunk=64) -> dr_problem:
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if q.dtype not in _DTYPE:
        raise TypeError(f"unsupported I/O dtype {q.dtype}")
    return dr_problem(B, T, H, dk, dv, int(chunk), _DTYPE[q.dtype], _mode(alpha, 3),
                      _mode(beta_k, 3), _mode(beta_v, 3))


def _check_shapes(q, v, named, state_batch=None):
    """Every tensor's shape against q [B, T, H, dk] and v [B, T, H, dv], and its device against q's.

    The library sizes every access from these dimensions, so a mismatched tensor is refused here,
    before anything is launched.  ``state_batch``: the leading size of the states when it is not B
    (a packed batch: the number of sequences).
    """
    if q.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be 4-D: [B, T, H, d]")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    SB = B if state_batch is None else state_batch
    tok, st = (B, T, H), (SB, H, dk, dv)
    want = {"k": [tok + (dk,)], "s": [tok + (dk,)], "v": [tok + (dv,)], "o": [tok + (dv,)],
            "dout": [tok + (dv,)], "alpha": [tok, tok + (dk,)], "beta_k": [tok, tok + (dk,)],
            "beta_v": [tok, tok + (dv,)], "S0": [st], "S_T": [st], "S": [st], "dS_T": [st]}
    for name, t in named:
        if t is None:
            continue
        if tuple(t.shape) not in want[name]:
            raise ValueError(f"{name} has shape {tuple(t.shape)}; expected "
                             + " or ".join(str(w) for w in want[name]))
        if t.device != q.device:
            raise ValueError(f"{name} is on {t.device}, q on {q.device}")


def _check_tensors(io_dtype, named):
    for name, t in named:
        if t is None:
            continue
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
        want = io_dtype if name in ("q", "k", "v", "o", "dout") else torch.float32
        if t.dtype != want:
            raise TypeError(f"{name} must be {want}, got {t.dtype}")


def workspace_bytes(problem: dr_problem) -> int:
    return int(lib().dr_chunk_fwd_workspace(ctypes.byref(problem)))


def dr_chunk_fwd(q, k, v, beta_k, alpha=None, beta_v=None, S0=None, chunk=64, o=None, S_T=None,
                 workspace=None, stream=None, final_state=True):
    """Chunkwise prefill.  Returns ``(o, S_T)``; S_T is None when ``final_state`` is False."""
    return _chunk_fwd(None, q, k, v, beta_k, alpha, beta_v, S0, chunk, o, S_T, workspace, stream, final_state)


def dr_diag_chunk_fwd_variant(variant, q, k, v, beta_k, alpha=None, beta_v=None, S0=None, chunk=64, o=None,
                              S_T=None, workspace=None, stream=None):
    """dr_chunk_fwd through a named kernel (``PREFILL_VARIANTS``) instead of the library's choice."""
    return _chunk_fwd(None, q, k, v, beta_k, alpha, beta_v, S0, chunk, o, S_T, workspace, stream, True,
                      variant=PREFILL_VARIANTS[variant])


def dr_chunk_fwd_osdn(q, k, v, beta_k, s, alpha=None, beta_v=None, S0=None, chunk=64, o=None, S_T=None,
                      workspace=None, stream=None, final_state=True):
    """Chunkwise prefill with OSDN's write-side key scale ``s`` [B, T, H, dk] (write key a = s * b)."""
    return _chunk_fwd(s, q, k, v, beta_k, alpha, beta_v, S0, chunk, o, S_T, workspace, stream, final_state)


def dr_chunk_fwd_varlen(q, k, v, beta_k, cu_seqlens, alpha=None, beta_v=None, s=None, S0=None, chunk=64, o=None,
                        S_T=None, workspace=None, stream=None):
    """Prefill of a packed batch: sequence n is tokens cu_seqlens[n] .. cu_seqlens[n+1]-1.

    q, k, v (and gates, s): [1, Ttot, H, d]; cu_seqlens: int32 CUDA tensor [N + 1]; S0 and the
    returned S_T: [N, H, dk, dv].  Returns ``(o, S_T)``.
    """
    if q.shape[0] != 1:
        raise ValueError("a packed batch has leading dimension 1: [1, Ttot, H, d]")
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda or cu_seqlens.dim() != 1:
        raise ValueError("cu_seqlens must be a 1-D int32 CUDA tensor")
    n = cu_seqlens.numel() - 1
    if n < 1:
        raise ValueError("cu_seqlens needs at least two entries")
    _check_shapes(q, v, [("k", k), ("v", v), ("o", o), ("alpha", alpha), ("beta_k", beta_k), ("beta_v", beta_v),
                         ("s", s), ("S0", S0), ("S_T", S_T)], state_batch=n)
    p = make_problem(q, v, alpha, beta_k, beta_v, chunk)
    p.B = n
    dev = q.device
    if o is None:
        o = torch.empty(q.shape[:3] + (p.dv,), dtype=q.dtype, device=dev)
    if S_T is None:
        S_T = torch.empty((n, p.H, p.dk, p.dv), dtype=torch.float32, device=dev)
    _check_tensors(q.dtype, [("q", q), ("k", k), ("v", v), ("o", o), ("alpha", alpha),
                             ("beta_k", beta_k), ("beta_v", beta_v), ("s", s), ("S0", S0), ("S_T", S_T)])
    if s is not None and tuple(s.shape) != tuple(q.shape):
        raise ValueError("s must have the shape of q / k")
    if S0 is not None and tuple(S0.shape) != (n, p.H, p.dk, p.dv):
        raise ValueError("S0 must be [N, H, dk, dv]")
    need = workspace_bytes(p)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    if cu_seqlens.device != dev:
        raise ValueError(f"cu_seqlens is on {cu_seqlens.device}, q on {dev}")
    rc = _call("dr_chunk_fwd_varlen", dev, ctypes.byref(p), _ptr(cu_seqlens), _ptr(q), _ptr(k), _ptr(v),
               _ptr(alpha), _ptr(beta_k), _ptr(beta_v), _ptr(s), _ptr(S0), _ptr(o), _ptr(S_T), _ptr(workspace),
               ctypes.c_size_t(workspace.numel()), _stream(stream, dev))
    if rc != DR_OK:
        raise DeltaRuleError(rc, "dr_chunk_fwd_varlen")
    return o, S_T


def _chunk_fwd(s, q, k, v, beta_k, alpha, beta_v, S0, chunk, o, S_T, workspace, stream, final_state, variant=None):
    _check_shapes(q, v, [("k", k), ("v", v), ("o", o), ("alpha", alpha), ("beta_k", beta_k), ("beta_v", beta_v),
                         ("s", s), ("S0", S0), ("S_T", S_T)])
    p = make_problem(q, v, alpha, beta_k, beta_v, chunk)
    dev = q.device
    if o is None:
        o = torch.empty(q.shape[:3] + (p.dv,), dtype=q.dtype, device=dev)
    if S_T is None and final_state:
        S_T = torch.empty((p.B, p.H, p.dk, p.dv), dtype=torch.float32, device=dev)
    _check_tensors(q.dtype, [("q", q), ("k", k), ("v", v), ("o", o), ("alpha", alpha),
                             ("beta_k", beta_k), ("beta_v", beta_v), ("s", s), ("S0", S0), ("S_T", S_T)])
    if s is not None and tuple(s.shape) != tuple(q.shape):
        raise ValueError("s must have the shape of q / k: [B, T, H, dk]")
    need = workspace_bytes(p) if variant is None else int(lib().dr_diag_chunk_fwd_workspace(int(variant), ctypes.byref(p)))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    elif workspace.device != dev:
        raise ValueError(f"workspace is on {workspace.device}, q on {dev}")
    if variant is not None:
        rc = _call("dr_diag_chunk_fwd_variant", dev, int(variant), ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v),
                   _ptr(alpha), _ptr(beta_k), _ptr(beta_v), _ptr(S0), _ptr(o), _ptr(S_T), _ptr(workspace),
                   ctypes.c_size_t(workspace.numel()), _stream(stream, dev))
        name = "dr_diag_chunk_fwd_variant"
    elif s is None:
        rc = _call("dr_chunk_fwd", dev, ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta_k),
                   _ptr(beta_v), _ptr(S0), _ptr(o), _ptr(S_T), _ptr(workspace),
                   ctypes.c_size_t(workspace.numel()), _stream(stream, dev))
        name = "dr_chunk_fwd"
    else:
        rc = _call("dr_chunk_fwd_osdn", dev, ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                   _ptr(beta_k), _ptr(beta_v), _ptr(s), _ptr(S0), _ptr(o), _ptr(S_T), _ptr(workspace),
                   ctypes.c_size_t(workspace.numel()), _stream(stream, dev))
        name = "dr_chunk_fwd_osdn"
    if rc != DR_OK:
        raise DeltaRuleError(rc, name)
    return o, S_T


def dr_chunk_fwd_noalloc(q, k, v, beta_k, alpha=None, beta_v=None, S0=None, chunk=64, o=None, S_T=None,
                         stream=None):
    """dr_chunk_fwd without a workspace, for callers that cannot allocate device memory.

    The library keeps the scratch in a static device array; ``o`` and ``S_T``
    must be passed in by such callers (they are only allocated here when
    omitted, as a convenience for tests).  Returns ``(o, S_T)``.
    """
    _check_shapes(q, v, [("k", k), ("v", v), ("o", o), ("alpha", alpha), ("beta_k", beta_k), ("beta_v", beta_v),
                         ("S0", S0), ("S_T", S_T)])
    p = make_problem(q, v, alpha, beta_k, beta_v, chunk)
    if o is None:
        o = torch.empty(q.shape[:3] + (p.dv,), dtype=q.dtype, device=q.device)
    if S_T is None:
        S_T = torch.empty((p.B, p.H, p.dk, p.dv), dtype=torch.float32, device=q.device)
    _check_tensors(q.dtype, [("q", q), ("k", k), ("v", v), ("o", o), ("alpha", alpha),
                             ("beta_k", beta_k), ("beta_v", beta_v), ("S0", S0), ("S_T", S_T)])
    dev = q.device
    rc = _call("dr_chunk_fwd_noalloc", dev, ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
               _ptr(beta_k), _ptr(beta_v), _ptr(S0), _ptr(o), _ptr(S_T), _stream(stream, dev))
    if rc != DR_OK:
        raise DeltaRuleError(rc, "dr_chunk_fwd_noalloc")
    return o, S_T


def dr_decode_step(q, k, v, beta_k, S, alpha=None, beta_v=None, o=None, stream=None):
    """One recurrent step for every (b, h); updates ``S`` in place and returns ``o``.

    q, k: [B, 1, H, dk]; v: [B, 1, H, dv]; gates [B, 1, H] or [B, 1, H, d]; S [B, H, dk, dv].
    """
    return _decode_step(None, q, k, v, beta_k, S, alpha, beta_v, o, stream)


def dr_decode_step_osdn(q, k, v, beta_k, S, s, alpha=None, beta_v=None, o=None, stream=None):
    """dr_decode_step with OSDN's write-side key scale ``s`` [B, 1, H, dk] (write key a = s * b)."""
    return _decode_step(s, q, k, v, beta_k, S, alpha, beta_v, o, stream)


def dr_diag_decode_step_variant(variant, q, k, v, beta_k, S, alpha=None, beta_v=None, s=None, o=None, stream=None):
    """dr_decode_step (or its OSDN form when ``s`` is given) through a named kernel (``DECODE_VARIANTS``)."""
    return _decode_step(s, q, k, v, beta_k, S, alpha, beta_v, o, stream, variant=DECODE_VARIANTS[variant])


def _decode_step(s, q, k, v, beta_k, S, alpha, beta_v, o, stream, variant=None):
    if q.dim() == 4 and q.shape[1] != 1:
        raise ValueError("a decode step takes one token: q [B, 1, H, dk]")
    _check_shapes(q, v, [("k", k), ("v", v), ("o", o), ("alpha", alpha), ("beta_k", beta_k), ("beta_v", beta_v),
                         ("s", s), ("S", S)])
    if S is None:
        raise ValueError("S (the state to update in place) is required")
    p = make_problem(q, v, alpha, beta_k, beta_v, 0)
    dev = q.device
    if o is None:
        o = torch.empty(q.shape[:3] + (p.dv,), dtype=q.dtype, device=q.device)
    _check_tensors(q.dtype, [("q", q), ("k", k), ("v", v), ("o", o), ("alpha", alpha),
                             ("beta_k", beta_k), ("beta_v", beta_v), ("s", s), ("S", S)])
    if s is not None and tuple(s.shape) != tuple(q.shape):
        raise ValueError("s must have the shape of q / k: [B, 1, H, dk]")
    if variant is not None:
        rc = _call("dr_diag_decode_step_variant", dev, int(variant), ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v),
                   _ptr(alpha), _ptr(beta_k), _ptr(beta_v), _ptr(s), _ptr(S), _ptr(o), _stream(stream, dev))
        name = "dr_diag_decode_step_variant"
    elif s is None:
        rc = _call("dr_decode_step", dev, ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                   _ptr(beta_k), _ptr(beta_v), _ptr(S), _ptr(o), _stream(stream, dev))
        name = "dr_decode_step"
    else:
        rc = _call("dr_decode_step_osdn", dev, ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                   _ptr(beta_k), _ptr(beta_v), _ptr(s), _ptr(S), _ptr(o), _stream(stream, dev))
        name = "dr_decode_step_osdn"
    if rc != DR_OK:
        raise DeltaRuleError(rc, name)
    return o


def dr_state_map_apply(M, N, S=None, out=None, stream=None):
    """out = M @ S + N per head (S None: zero).  M [..., dk, dk], S / N / out [..., dk, dv], fp32 CUDA."""
    dk, dv = N.shape[-2], N.shape[-1]
    n = N.numel() // (dk * dv)
    if out is None:
        out = torch.empty_like(N)
    for name, t in (("M", M), ("N", N), ("S", S), ("out", out)):
        if t is not None and (not t.is_cuda or not t.is_contiguous() or t.dtype != torch.float32):
            raise ValueError(f"{name} must be a contiguous fp32 CUDA tensor")
    if M.numel() != n * dk * dk or (S is not None and S.shape != N.shape) or out.shape != N.shape:
        raise ValueError("shapes: M [n, dk, dk], S / N / out [n, dk, dv]")
    dev = N.device
    for name, t in (("M", M), ("S", S), ("out", out)):
        if t is not None and t.device != dev:
            raise ValueError(f"{name} is on {t.device}, N on {dev}")
    rc = _call("dr_state_map_apply", dev, n, dk, dv, _ptr(M), _ptr(S), _ptr(N), _ptr(out), _stream(stream, dev))
    if rc != DR_OK:
        raise DeltaRuleError(rc, "dr_state_map_apply")
    return out


def dr_backward(q, k, v, beta_k, dout, alpha=None, beta_v=None, s=None, S0=None, dS_T=None, want_dS0=True,
                workspace=None, stream=None):
    """Gradients of sum(dout * o) + sum(dS_T * S_T) w.r.t. the forward's inputs (fp32 tensors).

    Returns a dict with keys q, k, v, beta_k, alpha, beta_v, s, S0 (None where absent / not wanted).
    """
    return _backward(None, q, k, v, beta_k, dout, alpha, beta_v, s, S0, dS_T, want_dS0, workspace, stream)


def dr_diag_backward_variant(variant, q, k, v, beta_k, dout, alpha=None, beta_v=None, s=None, S0=None, dS_T=None,
                             want_dS0=True, workspace=None, stream=None):
    """dr_backward through a named kernel (``BACKWARD_VARIANTS``) instead of the library's choice."""
    return _backward(BACKWARD_VARIANTS[variant], q, k, v, beta_k, dout, alpha, beta_v, s, S0, dS_T, want_dS0,
                     workspace, stream)


def _backward(variant, q, k, v, beta_k, dout, alpha, beta_v, s, S0, dS_T, want_dS0, workspace, stream):
    _check_shapes(q, v, [("k", k), ("v", v), ("dout", dout), ("alpha", alpha), ("beta_k", beta_k),
                         ("beta_v", beta_v), ("s", s), ("S0", S0), ("dS_T", dS_T)])
    p = make_problem(q, v, alpha, beta_k, beta_v, 64)
    dev = q.device
    f32 = lambda t: None if t is None else torch.empty(t.shape, dtype=torch.float32, device=dev)
    g = {"q": f32(q), "k": f32(k), "v": f32(v), "alpha": f32(alpha), "beta_k": f32(beta_k), "beta_v": f32(beta_v),
         "s": f32(s), "S0": torch.empty((p.B, p.H, p.dk, p.dv), dtype=torch.float32, device=dev) if want_dS0 else None}
    _check_tensors(q.dtype, [("q", q), ("k", k), ("v", v), ("dout", dout), ("alpha", alpha), ("beta_k", beta_k),
                             ("beta_v", beta_v), ("s", s), ("S0", S0), ("S_T", dS_T)])
    if s is not None and tuple(s.shape) != tuple(q.shape):
        raise ValueError("s must have the shape of q / k")
    if variant is None:
        need = int(lib().dr_backward_workspace(ctypes.byref(p)))
    else:
        need = int(lib().dr_diag_backward_workspace(int(variant), ctypes.byref(p)))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    args = [ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta_k), _ptr(beta_v), _ptr(s), _ptr(S0),
            _ptr(dout), _ptr(dS_T), _ptr(g["q"]), _ptr(g["k"]), _ptr(g["v"]), _ptr(g["alpha"]), _ptr(g["beta_k"]),
            _ptr(g["beta_v"]), _ptr(g["s"]), _ptr(g["S0"]), _ptr(workspace), ctypes.c_size_t(workspace.numel()),
            _stream(stream, dev)]
    if variant is None:
        rc = _call("dr_backward", dev, *args)
        name = "dr_backward"
    else:
        rc = _call("dr_diag_backward_variant", dev, int(variant), *args)
        name = "dr_diag_backward_variant"
    if rc != DR_OK:
        raise DeltaRuleError(rc, name)
    return g


def dr_workspace_status(workspace, stream=None) -> int:
    dev = workspace.device
    return int(_call("dr_workspace_status", dev, _ptr(workspace), _stream(stream, dev)))


def dr_noalloc_status(device=None, stream=None) -> int:
    """Status word of the last dr_chunk_fwd_noalloc call on ``device`` (default: the current device),
    read after synchronising the stream: DR_OK, DR_ERR_RANGE or DR_ERR_TIMEOUT."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    return int(_call("dr_noalloc_status", dev, _stream(stream, dev)))


def dr_diag_umma_selftest(A, B, a_mn: bool, b_mn: bool, stream=None):
    """128 x N product of bf16 or fp16 A, B through the tcgen05 building blocks; returns (D, status)."""
    K, N = B.shape
    if A.dtype != B.dtype or A.dtype not in (torch.bfloat16, torch.float16):
        raise TypeError("A and B must both be bf16 or both fp16")
    D = torch.empty((A.shape[0], N), dtype=torch.float32, device=A.device)
    ws = torch.zeros(256, dtype=torch.uint8, device=A.device)
    dev = A.device
    rc = _call("dr_diag_umma_selftest", dev, N, K, int(a_mn), int(b_mn), int(A.dtype == torch.bfloat16), _ptr(A),
               _ptr(B), _ptr(D), _ptr(ws), _stream(stream, dev))
    if rc != DR_OK:
        raise DeltaRuleError(rc, "dr_diag_umma_selftest")
    return D, dr_workspace_status(ws, stream)


def dr_diag_tri_inverse(A, stream=None, variant=0):
    """(I + strictly-lower(A))^-1 for a 64 x 64 fp32 CUDA tensor, via a prefill kernel's warp-MMA routine
    (variant 0: the ring prefill's, 1: the one-CTA prefill's)."""
    if A.shape != (64, 64) or A.dtype != torch.float32 or not A.is_cuda:
        raise ValueError("A must be a 64 x 64 fp32 CUDA tensor")
    A = A.contiguous()
    T = torch.zeros_like(A)
    rc = _call("dr_diag_tri_inverse", A.device, int(variant), _ptr(A), _ptr(T), _stream(stream, A.device))
    if rc != DR_OK:
        raise DeltaRuleError(rc, "dr_diag_tri_inverse")
    return T


def dr_diag_wait_timeout(cluster_scope: bool, limit_ns: int, device=None, stream=None):
    """Run the prefill kernels' bounded wait out on a barrier nothing completes.

    Returns ``(status, waited_ns)``: the workspace status code (DR_ERR_TIMEOUT when the wait gave
    up) and the nanoseconds each CTA waited (one CTA, or a cluster of two with ``cluster_scope``).
    """
    dev = torch.device("cuda") if device is None else torch.device(device)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    waited = torch.zeros(2, dtype=torch.int64, device=dev)
    rc = _call("dr_diag_wait_timeout", ws.device, int(bool(cluster_scope)), int(limit_ns), _ptr(ws), _ptr(waited),
               _stream(stream, ws.device))
    if rc != DR_OK:
        raise DeltaRuleError(rc, "dr_diag_wait_timeout")
    status = dr_workspace_status(ws, stream)
    return status, [int(x) for x in waited[:2 if cluster_scope else 1].cpu()]
