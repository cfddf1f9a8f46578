"""Gated delta-rule forward pass on NVIDIA B200 (sm_100a): chunkwise prefill and
recurrent decode behind a C ABI (``include/deltarule.h``, ``libdeltarule.so``).

Python entry points carry the C names:
    dr_chunk_fwd(q, k, v, beta_k, alpha=None, beta_v=None, S0=None, chunk=64) -> (o, S_T)
    dr_decode_step(q, k, v, beta_k, S, alpha=None, beta_v=None) -> o   (S updated in place)
    dr_chunk_fwd_osdn / dr_decode_step_osdn: the same with a write-side key scale s (a = s * b)
    dr_chunk_fwd_varlen(q, k, v, beta_k, cu_seqlens, ...) -> (o, S_T): packed variable-length batch
    dr_backward(q, k, v, beta_k, dout, ...) -> dict of gradients
"""
from ._binding import (DR_ABSENT, DR_BF16, DR_CHANNEL, DR_ERR_ALIGNMENT, DR_ERR_CUDA,
                       DR_ERR_INVALID_ARG, DR_ERR_RANGE, DR_ERR_TIMEOUT, DR_ERR_UNSUPPORTED,
                       DR_ERR_WORKSPACE, DR_F32, DR_OK, DR_SCALAR, EXPORTS, LIB_PATH, DeltaRuleError,
                       dr_chunk_fwd, dr_chunk_fwd_noalloc, dr_chunk_fwd_osdn, dr_chunk_fwd_varlen, dr_decode_step,
                       dr_decode_step_osdn, dr_diag_tri_inverse, dr_diag_wait_timeout, dr_state_map_apply, dr_backward,
                       dr_diag_umma_selftest, dr_diag_chunk_fwd_variant, dr_diag_decode_step_variant,
                       dr_diag_backward_variant, dr_problem, PREFILL_VARIANTS, DECODE_VARIANTS, BACKWARD_VARIANTS,
                       dr_noalloc_status, dr_workspace_status, lib, make_problem, status_string, workspace_bytes)

__all__ = [
    "dr_chunk_fwd", "dr_chunk_fwd_noalloc", "dr_chunk_fwd_osdn", "dr_chunk_fwd_varlen", "dr_decode_step", "dr_decode_step_osdn", "dr_state_map_apply", "dr_backward", "dr_workspace_status", "dr_noalloc_status", "dr_diag_umma_selftest", "dr_diag_tri_inverse", "dr_diag_wait_timeout", "dr_diag_chunk_fwd_variant",
    "dr_diag_decode_step_variant", "dr_diag_backward_variant", "PREFILL_VARIANTS", "DECODE_VARIANTS",
    "BACKWARD_VARIANTS", "dr_problem",
    "DeltaRuleError", "lib", "make_problem", "status_string", "workspace_bytes", "EXPORTS", "LIB_PATH",
    "DR_OK", "DR_ERR_INVALID_ARG", "DR_ERR_UNSUPPORTED", "DR_ERR_ALIGNMENT", "DR_ERR_WORKSPACE",
    "DR_ERR_RANGE", "DR_ERR_TIMEOUT", "DR_ERR_CUDA", "DR_F32", "DR_BF16", "DR_ABSENT", "DR_SCALAR",
    "DR_CHANNEL",
]
