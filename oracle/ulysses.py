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
