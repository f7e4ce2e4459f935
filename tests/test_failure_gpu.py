"""Failure detection on the GPU without a fault: a bounded device wait that runs out.

The test hook makes the attention kernel's TMA producer skip one K tile, so the MMA
thread's wait for it can never complete.  Every wait in the kernel is bounded: after
about a second the waiter records CP_ERR_TIMEOUT, the other warps see the abort flag and
leave, in-flight copies and MMAs drain, TMEM is freed and the kernel returns.  The host
reads the status and the context stays usable for the next call.
"""

import pytest
import torch

from context_attention_dit_b200 import binding
from tests.gpu_util import assert_attn_close, cuda, qkv

pytestmark = pytest.mark.gpu


def test_bounded_wait_timeout_is_reported_and_context_survives():
    import oracle

    q, k, v = qkv(1, 2, 300, 500, 128, seed=3)
    dq, dk, dv = cuda(q, k, v)
    assert binding.last_device_status() == binding.CP_OK
    binding.debug_set_fault(1)
    binding.attn_fwd(dq, dk, dv)
    assert binding.last_device_status() == binding.CP_ERR_TIMEOUT
    assert binding.last_device_status() == binding.CP_OK      # reading clears it
    o, lse = binding.attn_fwd(dq, dk, dv)                     # the next call is unaffected
    torch.cuda.synchronize()
    assert binding.last_device_status() == binding.CP_OK
    o_ref, lse_ref = oracle.attention(q, k, v, 128 ** -0.5)
    assert_attn_close(o, lse, o_ref, lse_ref, "after timeout")


def test_fault_hook_rejects_unknown_mode():
    with pytest.raises(binding.CpError):
        binding.debug_set_fault(7)
