"""Ring Anything's pad -> all-gather -> slice of K/V blocks, as an index map (test
infrastructure only).

Source: "Context parallelism", section "Ring Anything Attention": when the ranks' K/V
blocks have different lengths, every rank pads its local block to the longest block,
the padded blocks are all-gathered, and each gathered block is cut back to its true
length before attention, so the padding never enters the softmax.

Reading (the pages give no byte layout or padding value; the plainest ones):

* the blocks are rows ``[c_r, c_{r+1})`` of a ``[B, S, H, D]`` tensor, as in the ring;
* a padded block is its true rows followed by zero rows up to ``max_len``;
* the all-gather stacks the padded blocks in rank order: ``[n, B, max_len, H, D]``.

Both functions are pure copies, exact for any dtype.
"""

from __future__ import annotations

import numpy as np


def _bounds(chunk_bounds):
    b = [int(c) for c in chunk_bounds]
    assert len(b) >= 2 and b[0] == 0 and all(x <= y for x, y in zip(b[:-1], b[1:]))
    return b


def ring_anything_gather(x, chunk_bounds, max_len: int):
    """The gathered buffer: ``out[c, b, r] = x[b, c_c + r]`` for ``r < len_c``, zero after.

    ``x`` is a ``[B, S, H, D]`` numpy array or CPU torch tensor; the result has its dtype.
    """
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
    bounds = _bounds(chunk_bounds)
    B, S, H, D = x.shape
    n = len(bounds) - 1
    assert bounds[-1] == S
    if hasattr(x, "new_zeros"):
        out = x.new_zeros((n, B, max_len, H, D))
    else:
        out = np.zeros((n, B, max_len, H, D), dtype=x.dtype)
    for c in range(n):                       # the rank that owns block c
        lo, hi = bounds[c], bounds[c + 1]
        assert hi - lo <= max_len, "max_len below the longest block"
        for b in range(B):
            for r in range(hi - lo):         # the block's true rows; the rest stay zero
                out[c, b, r] = x[b, lo + r]
    return out


def ring_anything_slice(gathered, chunk_bounds):
    """Cut every gathered block back to its true length: a list of ``[B, len_c, H, D]``."""
    bounds = _bounds(chunk_bounds)
    return [gathered[c, :, :bounds[c + 1] - bounds[c]] for c in range(len(bounds) - 1)]
