"""Ulysses head<->sequence layout exchange, as an index map (test infrastructure only).

Source: "Context parallelism", section "Ulysses Attention".  The first
all-to-all regroups the data so that each GPU holds every token for a subset
of the attention heads; after attention, a second all-to-all regroups the
results by token.  Section table: sequence length and head count must both be
divisible by ``ulysses_degree``.

Layout reading (the pages give no byte layout; this is the plainest one):

* sequence-sharded ("src" of the forward exchange): ``P`` shards stacked
  rank-major, shard ``p`` holds tokens ``[p*S/P, (p+1)*S/P)`` of every head:
  ``src[p, b, s_local, h, d]`` with shape ``[P, B, S/P, H, D]``.
* head-sharded ("dst" of the forward exchange): shard ``p`` holds heads
  ``[p*H/P, (p+1)*H/P)`` for every token: ``dst[p, b, s, j, d]`` with shape
  ``[P, B, S, H/P, D]``.

The map is ``dst[p, b, s, j, :] = src[s // (S/P), b, s % (S/P), p*(H/P) + j, :]``
and the inverse exchange is its exact inverse.  Both are pure copies, so the
oracle is bit-exact for any dtype.
"""

from __future__ import annotations

import numpy as np


def _arr(x):
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
    return x


def ulysses_fwd(src, degree: int):
    """Sequence-sharded ``[P, B, S/P, H, D]`` -> head-sharded ``[P, B, S, H/P, D]``."""
    src = _arr(src)
    P = int(degree)
    Pn, B, Sp, H, D = src.shape
    assert Pn == P and H % P == 0
    S, Hp = Sp * P, H // P
    dst = src.new_empty((P, B, S, Hp, D)) if hasattr(src, "new_empty") else np.empty((P, B, S, Hp, D), src.dtype)
    for p in range(P):                       # destination rank (head group)
        for s in range(S):                   # global token index
            owner, s_local = s // Sp, s % Sp  # rank that holds token s before the exchange
            dst[p, :, s, :, :] = src[owner, :, s_local, p * Hp:(p + 1) * Hp, :]
    return dst


def ulysses_inv(dst, degree: int):
    """Head-sharded ``[P, B, S, H/P, D]`` -> sequence-sharded ``[P, B, S/P, H, D]``."""
    dst = _arr(dst)
    P = int(degree)
    Pn, B, S, Hp, D = dst.shape
    assert Pn == P and S % P == 0
    Sp, H = S // P, Hp * P
    src = dst.new_empty((P, B, Sp, H, D)) if hasattr(dst, "new_empty") else np.empty((P, B, Sp, H, D), dst.dtype)
    for p in range(P):                       # rank that held the head group
        for s in range(S):
            owner, s_local = s // Sp, s % Sp
            src[owner, :, s_local, p * Hp:(p + 1) * Hp, :] = dst[p, :, s, :, :]
    return src


def _owner(bounds, s):
    """The shard p with bounds[p] <= s < bounds[p+1] (empty shards hold nothing)."""
    for p in range(len(bounds) - 1):
        if bounds[p] <= s < bounds[p + 1]:
            return p
    raise IndexError(s)


def ulysses_anything_fwd(src_shards, seq_bounds, head_bounds):
    """Ulysses exchange for shards of unequal size ("Context parallelism", section "Ulysses
    Anything Attention": sequence length and head count need not be divisible by the
    degree).  Reading: sequence shard p holds tokens ``[seq_bounds[p], seq_bounds[p+1])``
    of every head; head shard q holds heads ``[head_bounds[q], head_bounds[q+1])`` of every
    token.

    ``src_shards``: list of P arrays ``[B, S_p, H, D]`` -> list of P arrays ``[B, S, H_q, D]``.
    """
    src_shards = [_arr(x) for x in src_shards]
    P = len(src_shards)
    assert len(seq_bounds) == P + 1 and len(head_bounds) == P + 1
    B, _, H, D = src_shards[0].shape
    S = int(seq_bounds[-1])
    assert int(head_bounds[-1]) == H
    x0 = src_shards[0]
    out = []
    for q in range(P):
        hq0, hq1 = int(head_bounds[q]), int(head_bounds[q + 1])
        shape = (B, S, hq1 - hq0, D)
        dst = x0.new_empty(shape) if hasattr(x0, "new_empty") else np.empty(shape, x0.dtype)
        for s in range(S):
            owner = _owner(seq_bounds, s)
            dst[:, s, :, :] = src_shards[owner][:, s - int(seq_bounds[owner]), hq0:hq1, :]
        out.append(dst)
    return out


def ulysses_anything_inv(dst_shards, seq_bounds, head_bounds):
    """Inverse of :func:`ulysses_anything_fwd`: list of ``[B, S, H_q, D]`` -> list of ``[B, S_p, H, D]``."""
    dst_shards = [_arr(x) for x in dst_shards]
    P = len(dst_shards)
    B, S, _, D = dst_shards[0].shape
    H = int(head_bounds[-1])
    x0 = dst_shards[0]
    out = []
    for p in range(P):
        s0, s1 = int(seq_bounds[p]), int(seq_bounds[p + 1])
        shape = (B, s1 - s0, H, D)
        src = x0.new_empty(shape) if hasattr(x0, "new_empty") else np.empty(shape, x0.dtype)
        for q in range(P):
            hq0, hq1 = int(head_bounds[q]), int(head_bounds[q + 1])
            for s in range(s0, s1):
                src[:, s - s0, hq0:hq1, :] = dst_shards[q][:, s, :, :]
        out.append(src)
    return out
