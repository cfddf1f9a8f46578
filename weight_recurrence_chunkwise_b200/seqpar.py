"""Sequence-parallel prefill: one long sequence split along T across ranks.

The chunkwise recurrence is linear in the state (DeltaNet page, step 7; FG2-GDN page, section 2):
a segment of tokens maps its initial state to its final state as S_out = M S_in + N, per (b, h).
Each rank holds one contiguous segment of every (b, h) and

1. computes its segment's map with two prefill calls:
   N = final state from a zero initial state; M = final state with zero write vectors from S0 = I
   (the product of the segment's transitions, dk x dk);
2. exchanges the maps with all ranks (one NCCL all-gather of M and N; the only collective);
3. composes the maps of the segments before it into its initial state (dr_state_map_apply);
4. reruns its segment's prefill from that state for the outputs.

Every rank also composes the global final state.  The cost per rank is three segment prefills (the
map pass with dv = dk), so the split pays from about four ranks on.  The maps are [B, H, dk, dk] and
[B, H, dk, dv] fp32: 8 MiB per rank for 64 heads of 128 x 128, small next to NVLink's bandwidth.
"""
from __future__ import annotations

import torch

from . import _binding as _b


def _cuda_prefill(q, k, v, beta_k, alpha=None, beta_v=None, s=None, S0=None, chunk=64):
    if s is None:
        return _b.dr_chunk_fwd(q, k, v, beta_k, alpha=alpha, beta_v=beta_v, S0=S0, chunk=chunk)
    return _b.dr_chunk_fwd_osdn(q, k, v, beta_k, s, alpha=alpha, beta_v=beta_v, S0=S0, chunk=chunk)


def _cuda_apply(M, S, N):
    return _b.dr_state_map_apply(M, N, S=S)


def segment_map(q, k, v, beta_k, alpha=None, beta_v=None, s=None, chunk=64, prefill=_cuda_prefill):
    """(M, N) of this segment: S_out = M S_in + N per (b, h); M [B,H,dk,dk], N [B,H,dk,dv] fp32."""
    B, T, H, dk = q.shape
    _, N = prefill(q, k, v, beta_k, alpha=alpha, beta_v=beta_v, s=s, S0=None, chunk=chunk)
    eye = torch.eye(dk, dtype=torch.float32, device=q.device).expand(B, H, dk, dk).contiguous()
    # zero write vectors: v = 0 and no separate write strength (w = sqrt(beta_k) * 0 = 0)
    _, M = prefill(q, k, torch.zeros_like(k), beta_k, alpha=alpha, beta_v=None, s=s, S0=eye, chunk=chunk)
    return M, N


def compose(maps, S0=None, apply=_cuda_apply):
    """Initial state after the segments `maps` = [(M, N), ...] in order, starting from S0 (None: 0)."""
    S = S0
    for M, N in maps:
        S = N.clone() if S is None else apply(M, S, N)
    return S


def _all_gather(x, group):
    """Every rank's copy of `x`, in rank order.  Over NCCL the device tensors are exchanged directly;
    a gloo group (CPU ranks, or ranks sharing one GPU in tests) exchanges through host copies."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    staged = x.is_cuda and dist.get_backend(group) == "gloo"
    src = x.detach().cpu() if staged else x.contiguous()
    out = [torch.empty_like(src) for _ in range(world)]
    dist.all_gather(out, src, group=group)
    return [t.to(x.device) for t in out] if staged else out


def seqpar_chunk_fwd(q, k, v, beta_k, alpha=None, beta_v=None, s=None, S0=None, chunk=64, group=None,
                     prefill=_cuda_prefill, apply=_cuda_apply):
    """Prefill of this rank's segment of a sequence split along T over the ranks of `group`.

    Rank r holds tokens of segment r (any lengths, in rank order) of every (b, h); S0 is the initial
    state of the whole sequence (same on every rank, or None).  Returns (o of this segment, final
    state of the whole sequence).  Every rank takes the same collective step (one all-gather).
    """
    import torch.distributed as dist

    rank, world = dist.get_rank(group), dist.get_world_size(group)
    M, N = segment_map(q, k, v, beta_k, alpha=alpha, beta_v=beta_v, s=s, chunk=chunk, prefill=prefill)
    maps = list(zip(_all_gather(M, group), _all_gather(N, group)))
    S_in = compose(maps[:rank], S0, apply)
    o, S_seg = prefill(q, k, v, beta_k, alpha=alpha, beta_v=beta_v, s=s, S0=S_in, chunk=chunk)
    # this segment's own final state is exact; the later segments' maps carry it to the end
    return o, compose(maps[rank + 1:], S_seg, apply)
