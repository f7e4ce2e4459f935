"""Context-parallel DiT attention for B200: blockwise attention + LSE merge + Ulysses exchange.

The compute runs in ``libcpattn.so`` (hand-written sm_100a CUDA behind a C ABI,
``include/cpattn.h``); :mod:`.binding` marshals torch tensors into it.  The
library is loaded on first use and every op raises if it is missing.
"""

from .binding import (  # noqa: F401
    CpError,
    attn_fwd,
    attn_fwd_blocks,
    attn_merge,
    last_device_status,
    load,
    ring_bounds,
    ring_sim,
    ring_sim_fused,
    ring_workspace_size,
    ring_workspace_views,
    status_string,
    ulysses_permute,
    ulysses_permute_n,
)

__all__ = [
    "CpError", "attn_fwd", "attn_fwd_blocks", "attn_merge", "last_device_status", "load", "ring_bounds", "ring_sim", "ring_sim_fused",
    "ring_workspace_size", "ring_workspace_views", "status_string", "ulysses_permute", "ulysses_permute_n",
]
