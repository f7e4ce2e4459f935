"""cp_ring_sim_static: ring attention that allocates nothing.

Some callers of this library may not allocate device memory at the point where they
attend: code running inside another framework's memory pool or under a fixed memory
budget (a cudaMalloc there bypasses the pool's accounting or fails), and real-time
loops that cannot afford an allocation's latency.  cp_ring_sim_static gives them
cp_ring_sim with the per-block partials in the library's own static device array
(32 MiB) instead of a caller-provided workspace.

This file is collected last on purpose, so that a run that stops at the first
failure has already run every other test.  It must pass alone in a fresh process
and after the rest of the suite.
"""

import ctypes

import pytest
import torch

import oracle
from context_attention_dit_b200 import binding
from tests.gpu_util import assert_attn_close, qkv

pytestmark = pytest.mark.gpu


def _call_static(q, k, v, bounds, out, out_lse):
    """Call the entry point through the C ABI with preallocated outputs (no allocation anywhere)."""
    B, Sq, H, D = q.shape
    Skv = k.shape[1]
    n = len(bounds) - 1
    cb = (ctypes.c_int * (n + 1))(*bounds)
    return binding.load().cp_ring_sim_static(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()), cb, n,
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(out_lse.data_ptr()), B, H, Sq, Skv, D, D ** -0.5,
        binding.CP_BF16, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_static_scratch_matches_workspace_version_twice():
    """Two calls in a row, with different inputs and block splits.  Each runs the same
    kernels on the same inputs as cp_ring_sim with a caller workspace, so the outputs must
    be bit-identical; the first case is also checked against the fp64 oracle."""
    cases = [((1, 4, 700, 700, 128), [0, 250, 251, 700], 101),
             ((2, 3, 333, 1000, 64), [0, 0, 400, 1000, 1000], 202)]
    for i, ((B, H, Sq, Skv, D), bounds, seed) in enumerate(cases):
        q_h, k_h, v_h = qkv(B, H, Sq, Skv, D, seed=seed)
        q, k, v = q_h.cuda(), k_h.cuda(), v_h.cuda()
        out = torch.full((B, Sq, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        out_lse = torch.full((B, H, Sq), float("nan"), dtype=torch.float32, device="cuda")
        st = _call_static(q, k, v, bounds, out, out_lse)
        assert st == binding.CP_OK, binding.status_string(st)
        ref, ref_lse, _ = binding.ring_sim(q, k, v, bounds)          # workspace version
        torch.cuda.synchronize()
        assert binding.last_device_status() == binding.CP_OK
        assert torch.equal(out, ref), f"case {i}: output differs from cp_ring_sim"
        assert torch.equal(out_lse, ref_lse), f"case {i}: lse differs from cp_ring_sim"
        if i == 0:
            o_ref, l_ref, _, _ = oracle.ring(q_h, k_h, v_h, D ** -0.5, bounds)
            assert_attn_close(out, out_lse, o_ref, l_ref, "cp_ring_sim_static vs oracle")


def test_static_scratch_rejects_too_large():
    """FLUX ring-8 partials (~457 MB) do not fit the 32 MiB array: a clear error, nothing launched."""
    fake = ctypes.c_void_p(1 << 20)  # aligned stand-in: the size check precedes any device access
    cb = (ctypes.c_int * 9)(*[576 * i for i in range(9)])
    st = binding.load().cp_ring_sim_static(fake, fake, fake, cb, 8, fake, None, 1, 24, 4608, 4608, 128, 0.088,
                                           binding.CP_BF16, None)
    assert st == binding.CP_ERR_UNSUPPORTED
    q, k, v = (t.cuda() for t in qkv(1, 24, 4608, 4608, 128))
    with pytest.raises(binding.CpError) as e:
        binding.ring_sim_static(q, k, v, [576 * i for i in range(9)])
    assert e.value.status == binding.CP_ERR_UNSUPPORTED and "static" in str(e.value)
