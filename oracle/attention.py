"""Attention, LSE merge and simulated ring: the fp64 oracle (test infrastructure only).

Sources (pages that define what is computed):

* "Attention backends", section "Available backends": the default ``native``
  backend is PyTorch ``scaled_dot_product_attention``, i.e. non-causal
  ``softmax(Q K^T * scale) V``.  Tensors are laid out ``(batch, seq, heads,
  head_dim)``; the section "Checks" uses a ``(1, 10, 8, 64)`` example.
* "Context parallelism", section "Ring Attention": every GPU attends its
  queries to one K/V block after another until it has seen every token.
  Section "Ring Anything Attention": blocks may have unequal lengths; padded
  rows are cut off again before attention.
* "Parallelism" (API page), ``ContextParallelConfig.convert_to_fp32``: the
  output and its LSE are kept in float32 so that the ring's accumulation over
  blocks is numerically stable.  The pages never print the merge formula; the
  plainest reading, used here, is the log-sum-exp merge written out in
  :func:`merge`.

Everything is computed in float64 from the inputs widened exactly (bf16 and
fp32 values are exactly representable in fp64).  The softmax is the plain
two-pass form (row max, then exponentials), never an online/streaming form.
"""

from __future__ import annotations

import numpy as np


def _f64(x) -> np.ndarray:
    """Widen a numpy array or a CPU torch tensor (bf16/fp16/fp32/fp64) to fp64 exactly."""
    if hasattr(x, "detach"):  # torch tensor: numpy has no bf16, go through fp32 (exact)
        import torch

        x = x.detach().to("cpu")
        if x.dtype in (torch.bfloat16, torch.float16):
            x = x.to(torch.float32)
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


def attention(q, k, v, scale: float):
    """Non-causal scaled-dot-product attention with its log-sum-exp.

    Definition ("Attention backends", "Available backends": ``native`` is
    ``scaled_dot_product_attention``), for batch ``b``, head ``h``, query row
    ``i`` and keys ``j``::

        s_ij  = scale * sum_d q_id k_jd
        m_i   = max_j s_ij
        l_i   = sum_j exp(s_ij - m_i)
        o_i   = (sum_j exp(s_ij - m_i) v_j) / l_i
        lse_i = m_i + ln(l_i)                       (natural log)

    Args:
        q: ``[B, Sq, H, D]``; k, v: ``[B, Skv, H, D]`` (any float dtype).
        scale: the logit scale (``1/sqrt(D)`` by default in SDPA).

    Returns:
        ``(o, lse)``: ``o`` fp64 ``[B, Sq, H, D]``; ``lse`` fp64 ``[B, H, Sq]``.
        With no keys (``Skv == 0``) the softmax has an empty support: the
        reading taken is ``o = 0`` and ``lse = -inf`` (the neutral element of
        the merge).
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    B, Sq, H, D = q.shape
    Skv = k.shape[1]
    assert k.shape == (B, Skv, H, D) and v.shape == (B, Skv, H, D)
    o = np.zeros((B, Sq, H, D), dtype=np.float64)
    lse = np.full((B, H, Sq), -np.inf, dtype=np.float64)
    if Skv == 0 or Sq == 0:
        return o, lse
    for b in range(B):
        for h in range(H):
            qh = q[b, :, h, :]          # [Sq, D]
            kh = k[b, :, h, :]          # [Skv, D]
            vh = v[b, :, h, :]          # [Skv, D]
            s = scale * (qh @ kh.T)     # [Sq, Skv] logits
            m = s.max(axis=1)           # pass 1: row max
            e = np.exp(s - m[:, None])  # pass 2: shifted exponentials
            l = e.sum(axis=1)
            o[b, :, h, :] = (e @ vh) / l[:, None]
            lse[b, h, :] = m + np.log(l)
    return o, lse


def merge(partials, lses):
    """Merge per-block attention results by their log-sum-exps.

    Plainest reading of the ring's accumulation over K/V blocks ("Context
    parallelism", "Ring Attention"; fp32 output + LSE per block from
    ``ContextParallelConfig.convert_to_fp32``).  With ``M = max_i lse_i``::

        L = M + ln(sum_i exp(lse_i - M))
        O = sum_i exp(lse_i - L) * O_i

    A block with ``lse_i = -inf`` (no keys) has weight 0.  If every block has
    ``lse_i = -inf`` the result is ``O = 0``, ``L = -inf``.

    Args:
        partials: ``[n, B, Sq, H, D]``; lses: ``[n, B, H, Sq]``.

    Returns:
        ``(o, lse)`` fp64 with shapes ``[B, Sq, H, D]`` and ``[B, H, Sq]``.
    """
    P = _f64(partials)
    Ls = _f64(lses)
    n, B, Sq, H, D = P.shape
    assert Ls.shape == (n, B, H, Sq)
    M = Ls.max(axis=0)                                   # [B, H, Sq]
    finite = np.isfinite(M)
    Msafe = np.where(finite, M, 0.0)
    with np.errstate(invalid="ignore", divide="ignore"):
        tot = np.exp(Ls - Msafe[None]).sum(axis=0)       # exp(-inf) = 0
        L = np.where(finite, Msafe + np.log(tot), -np.inf)
        w = np.where(finite[None], np.exp(Ls - np.where(finite, L, 0.0)[None]), 0.0)  # [n,B,H,Sq]
    wt = np.transpose(w, (0, 1, 3, 2))[..., None]        # [n, B, Sq, H, 1]
    O = (wt * P).sum(axis=0)
    return O, L


def ring(q, k, v, scale: float, chunk_bounds):
    """Simulated ring / ring-anything attention on one host.

    K/V rows ``[c_r, c_{r+1})`` form block ``r``; every block is attended with
    :func:`attention` in ring order ``r = 0 .. n-1`` and the per-block results
    are combined with :func:`merge` ("Context parallelism", sections "Ring
    Attention" and "Ring Anything Attention": padded rows are removed before
    attention, so each block is exactly its true-length rows).

    Returns ``(o, lse, partials, lses)``.
    """
    bounds = [int(c) for c in chunk_bounds]
    k = _f64(k)
    v = _f64(v)
    assert bounds[0] == 0 and bounds[-1] == k.shape[1]
    assert all(a <= b for a, b in zip(bounds[:-1], bounds[1:]))
    parts, ls = [], []
    for r in range(len(bounds) - 1):
        o_r, l_r = attention(q, k[:, bounds[r]:bounds[r + 1]], v[:, bounds[r]:bounds[r + 1]], scale)
        parts.append(o_r)
        ls.append(l_r)
    P = np.stack(parts)
    Ls = np.stack(ls)
    o, lse = merge(P, Ls)
    return o, lse, P, Ls


def attention_rows(q, k, v, scale: float, rows):
    """:func:`attention` restricted to the query rows ``rows`` (a list of ints).

    Used for sequences where the full oracle would take minutes: attention of
    a query row depends only on that row and on all of K/V, so the selected
    rows are exact.  Returns ``(o [B, len(rows), H, D], lse [B, H, len(rows)])``.
    """
    q = _f64(q)
    return attention(q[:, list(rows)], k, v, scale)
