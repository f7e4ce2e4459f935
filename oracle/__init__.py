"""fp64 CPU oracle for context-parallel DiT attention.

TEST INFRASTRUCTURE ONLY.  This package is the slow, plainly written reference
that the CUDA path is checked against.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py`` (its ``cpu_baseline`` leg and its
``--impl reference`` arm) may import it.  The product library
(``context_attention_dit_b200``) never imports it and has no CPU fallback.

It shares no code with the CUDA path: no kernels, headers, helpers or tables.
Inputs come from the seeded generator in ``context_attention_dit_b200.inputs``,
which holds no arithmetic of the method.

Every function here is pinned by ``tests/test_oracle_pins.py`` to closed forms,
invariants, a brute-force high-precision evaluation, a library routine
(``torch.nn.functional.scaled_dot_product_attention`` in fp64) and a simulated
message-passing all-to-all.  No function here is "parity unpinned".
"""

from .attention import attention, merge, ring, attention_rows
from .ring_anything import ring_anything_gather, ring_anything_slice
from .ulysses import ulysses_anything_fwd, ulysses_anything_inv, ulysses_fwd, ulysses_inv
from .usp import usp

__all__ = ["attention", "merge", "ring", "attention_rows", "ring_anything_gather", "ring_anything_slice", "ulysses_fwd", "ulysses_inv", "ulysses_anything_fwd",
           "ulysses_anything_inv", "usp"]
