"""Unified sequence parallelism (Ulysses x ring) on one host (test infrastructure only).

Source: "Context parallelism", section "Unified Attention": an all-to-all regroups heads
and tokens, Ring Attention runs on the result, and the all-to-all in the reverse
direction restores the original layout; the GPUs form a ulysses_degree x ring_degree
grid.  On one host this is the composition of the oracle's own parts: the forward
exchange :func:`ulysses_fwd` on Q, K and V, :func:`ring` on every head shard (the ring
blocks are K/V row ranges of the whole sequence, which every head shard holds after the
exchange), and the inverse exchange :func:`ulysses_inv` on O.  Pinned in
``tests/test_oracle_pins.py``: the composition equals unsplit :func:`attention`, which
is what both all-to-alls and the ring merge must preserve.
"""

from __future__ import annotations

import numpy as np

from .attention import ring
from .ulysses import ulysses_fwd, ulysses_inv


def usp(q_shards, k_shards, v_shards, degree: int, scale: float, chunk_bounds):
    """q, k, v sequence-sharded ``[P, B, S/P, H, D]`` -> ``(o [P, B, S/P, H, D], lse [B, H, S])``.

    Head group p of the exchange holds heads ``[p*H/P, (p+1)*H/P)``, so its LSE rows are
    those heads of the unsharded ``[B, H, S]`` layout.
    """
    qh, kh, vh = (ulysses_fwd(t, degree) for t in (q_shards, k_shards, v_shards))
    outs, lses = [], []
    for p in range(int(degree)):  # head group p: [B, S, H/P, D]
        o_p, lse_p, _, _ = ring(qh[p], kh[p], vh[p], scale, chunk_bounds)
        outs.append(o_p)
        lses.append(lse_p)
    o = ulysses_inv(np.stack(outs), degree)
    lse = np.concatenate(lses, axis=1)
    return o, lse
