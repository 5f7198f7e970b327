"""Sequence-parallel forward: one sequence split into segments that run at the same time.

Across a segment the recurrence of the Gated DeltaNet-2 note (sec. 3, forward-pass
paragraph) is affine in the state it starts from: S_out = A_g S_in + B_g. B_g is the
segment's final state from a zero state; A_g, the product of its (I - k e^T) Diag(alpha)
factors, is its final state from the identity with the write gate off (value channels
then carry A_g's d_k columns). One batched forward gives every segment's B_g, one more
its A_g, ``gdr2_segment_states`` scans S_{g+1} = A_g S_g + B_g, and a last forward runs
every segment from its own entering state. That is three forwards' work instead of one,
in exchange for a scan chain G times shorter per head, or for G GPUs sharing one sequence.

Every arithmetic step runs in libgdr2.so; this module only arranges the calls (views,
zero and identity inputs, and, across ranks, the exchange of the (A_g, B_g) pairs).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from .binding import gdr2_forward, gdr2_segment_states


def _transition_inputs(v, w, dk):
    """Zero values with d_k channels and a zero write gate (scalar: one value per token-head)."""
    lead = tuple(v.shape[:-1])
    return torch.zeros(lead + (dk,), dtype=v.dtype, device=v.device), torch.zeros(lead, dtype=w.dtype,
                                                                                   device=w.device)


def _identity(n, H, dk, device):
    return torch.eye(dk, dtype=torch.float32, device=device).expand(n, H, dk, dk).contiguous()


def gdr2_forward_segmented(q, k, v, log_alpha, b, w, S0=None, *, segments, final_state=True, stream=None):
    """gdr2_forward with each sequence cut into ``segments`` equal parts run side by side on
    one GPU. Inputs as gdr2_forward ([B, T, H, .], T a multiple of ``segments``). Returns
    (o [B, T, H, dv], S_T or None)."""
    B, T, H, dk = q.shape
    G = int(segments)
    if G < 1 or T % G:
        raise ValueError(f"T={T} must be a positive multiple of segments={G}")
    L = T // G
    seg = lambda t: t.reshape(B * G, L, *t.shape[2:])  # noqa: E731  (a view: segments inside the batch)
    qs, ks, vs, las, bs, ws = (seg(t) for t in (q, k, v, log_alpha, b, w))
    _, Bst, _ = gdr2_forward(qs, ks, vs, las, bs, ws, None, stream=stream)
    vz, wz = _transition_inputs(vs, ws, dk)
    _, A, _ = gdr2_forward(qs, ks, vz, las, bs, wz, _identity(B * G, H, dk, q.device), stream=stream)
    S_starts, S_T = gdr2_segment_states(A.view(B, G, H, dk, dk), Bst.view(B, G, H, dk, -1), S0,
                                        final_state=final_state, stream=stream)
    o, _, _ = gdr2_forward(qs, ks, vs, las, bs, ws, S_starts.view(B * G, H, dk, -1), final_state=False,
                           stream=stream)
    return o.view(B, T, H, -1), S_T


def gdr2_forward_sequence_parallel(q, k, v, log_alpha, b, w, S0=None, *, group=None, forward=None,
                                   segment_states=None):
    """One segment per rank: rank r holds tokens r L .. (r + 1) L - 1 of every sequence
    ([B, L, H, .] on its device) and S0 is the whole sequences' initial state (any rank's
    copy; rank 0's chain starts from it). Only the (A_g, B_g) pairs cross ranks (one
    all-gather). Returns (this rank's o [B, L, H, dv], the sequences' final state S_T on
    every rank). ``forward`` and ``segment_states`` default to the library's; they take and
    return what gdr2_forward and gdr2_segment_states do."""
    forward = forward or gdr2_forward
    segment_states = segment_states or gdr2_segment_states
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, L, H, dk = q.shape
    _, Bst, _ = forward(q, k, v, log_alpha, b, w, None)
    vz, wz = _transition_inputs(v, w, dk)
    _, A, _ = forward(q, k, vz, log_alpha, b, wz, _identity(B, H, dk, q.device))
    As = [torch.empty_like(A) for _ in range(world)]
    Bs = [torch.empty_like(Bst) for _ in range(world)]
    dist.all_gather(As, A.contiguous(), group=group)
    dist.all_gather(Bs, Bst.contiguous(), group=group)
    # every rank scans the short chain itself: [B, G, H, ...] with the segment (rank) index inside
    S_starts, S_T = segment_states(torch.stack(As, 1), torch.stack(Bs, 1), S0)
    o, _, _ = forward(q, k, v, log_alpha, b, w, S_starts[:, rank].contiguous(), final_state=False)
    return o, S_T
