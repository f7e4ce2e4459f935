"""The fp64 oracle evaluated over a process pool (test infrastructure only).

Attention of one (batch, head, query row) depends only on that query row and on the
head's keys and values, so disjoint (batch, head, row range) pieces, each computed by
``oracle.attention`` on its own slice, together give the oracle's full output.  This lets
a long sequence (the 32760-token video workload: 2.2e13 fp64 FLOP) be checked on every
element in minutes on the host's cores.  Nothing here computes attention itself.

The pool uses the ``spawn`` start method (a forked child of a process that has touched
the GPU can hang), and every worker limits its BLAS to one thread.
"""

from __future__ import annotations

import multiprocessing as mp
import os
import tempfile

import numpy as np

_STATE = {}


def _bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 values (raw uint16 bits) widened exactly: bf16 is the top half of a float32."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _init(path, shape, scale):
    from threadpoolctl import threadpool_limits

    threadpool_limits(1)
    _STATE["mm"] = np.memmap(path, dtype=np.uint16, mode="r", shape=(3,) + tuple(shape))
    _STATE["scale"] = scale


def _piece(args):
    import oracle

    b, h, r0, r1, sub = args
    mm, scale = _STATE["mm"], _STATE["scale"]
    k = _bf16_bits_to_f64(np.asarray(mm[1, b, :, h, :]))[None, :, None, :]
    v = _bf16_bits_to_f64(np.asarray(mm[2, b, :, h, :]))[None, :, None, :]
    q = _bf16_bits_to_f64(np.asarray(mm[0, b, r0:r1, h, :]))
    outs, lses = [], []
    for s0 in range(0, r1 - r0, sub):
        o, lse = oracle.attention(q[None, s0:s0 + sub, None, :], k, v, scale)
        outs.append(o[0, :, 0, :])
        lses.append(lse[0, 0, :])
    return b, h, r0, r1, np.concatenate(outs), np.concatenate(lses)


def attention_pieces(q, k, v, scale: float, workers: int | None = None, rows_per_piece: int = 2048,
                     sub_rows: int = 512):
    """Yield ``(b, h, r0, r1, o [r1-r0, D] fp64, lse [r1-r0] fp64)`` pieces of
    ``oracle.attention(q, k, v, scale)`` in completion order.

    q, k, v: bf16 CPU torch tensors ``[B, S, H, D]`` of one shape (self-attention).
    """
    import torch

    assert q.dtype == k.dtype == v.dtype == torch.bfloat16 and q.shape == k.shape == v.shape
    B, S, H, D = q.shape
    workers = workers or max(1, len(os.sched_getaffinity(0)))
    with tempfile.TemporaryDirectory() as tmp:
        path = os.path.join(tmp, "qkv.u16")
        mm = np.memmap(path, dtype=np.uint16, mode="w+", shape=(3, B, S, H, D))
        for i, t in enumerate((q, k, v)):
            mm[i] = t.contiguous().view(torch.int16).numpy().view(np.uint16)
        mm.flush()
        del mm
        tasks = [(b, h, r0, min(S, r0 + rows_per_piece), sub_rows)
                 for b in range(B) for h in range(H) for r0 in range(0, S, rows_per_piece)]
        ctx = mp.get_context("spawn")
        with ctx.Pool(workers, initializer=_init, initargs=(path, (B, S, H, D), scale)) as pool:
            for res in pool.imap_unordered(_piece, tasks):
                yield res


class ErrorAccumulator:
    """The acceptance statistics of ``gpu_util.assert_attn_close`` (max-abs, mean-abs and
    relative L2 of the output, max-abs of finite LSEs and the -inf pattern), accumulated over
    pieces so that a full output never has to be held in fp64."""

    def __init__(self):
        self.max_abs = 0.0
        self.sum_abs = 0.0
        self.count = 0
        self.sum_sq_diff = 0.0
        self.sum_sq_ref = 0.0
        self.lse_max_abs = 0.0
        self.inf_pattern_ok = True
        self.finite = True

    def add(self, o_gpu: np.ndarray, o_ref: np.ndarray, lse_gpu: np.ndarray, lse_ref: np.ndarray):
        d = np.abs(o_gpu.astype(np.float64) - o_ref)
        self.finite &= bool(np.isfinite(d).all())
        self.max_abs = max(self.max_abs, float(d.max()))
        self.sum_abs += float(d.sum())
        self.count += d.size
        self.sum_sq_diff += float((d * d).sum())
        self.sum_sq_ref += float((o_ref * o_ref).sum())
        lg = lse_gpu.astype(np.float64)
        fin = np.isfinite(lse_ref)
        self.inf_pattern_ok &= bool(np.array_equal(np.isneginf(lg), np.isneginf(lse_ref)))
        if fin.any():
            self.lse_max_abs = max(self.lse_max_abs, float(np.abs(lg[fin] - lse_ref[fin]).max()))

    def summary(self):
        rel = (self.sum_sq_diff ** 0.5) / max(self.sum_sq_ref ** 0.5, 1e-300)
        return {"max_abs": self.max_abs, "mean_abs": self.sum_abs / max(self.count, 1), "rel_l2": rel,
                "lse_max_abs": self.lse_max_abs, "elements": self.count}
