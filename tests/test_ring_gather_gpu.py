"""cp_ring_anything_gather: the Ring Anything pad -> all-gather buffer ("Context
parallelism", "Ring Anything Attention"), bit for bit against the oracle's index map, and
ring attention over the sliced gathered blocks bit for bit against cp_ring_sim."""

import math

import pytest
import torch

import oracle
from context_attention_dit_b200 import binding
from context_attention_dit_b200.inputs import make_qkv
from tests.gpu_util import LSE_ABS, assert_attn_close, assert_split_close, cuda, qkv

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.view(torch.int16) if t.element_size() == 2 else t.view(torch.int32)


@pytest.mark.parametrize("B,S,H,D,bounds,max_len,dtype", [
    (1, 4481, 24, 128, [0, 1121, 2241, 3361, 4481], 1121, torch.bfloat16),   # FLUX 1008^2 over 4
    (2, 4173, 24, 128, [0, 1392, 2783, 4173], 1392, torch.bfloat16),         # uneven 1392/1391/1390
    (2, 300, 3, 64, [0, 0, 101, 300], 210, torch.bfloat16),                  # empty block, extra padding
    (3, 50, 5, 8, [0, 7, 20, 33, 50], 17, torch.float32),                    # 4-byte elements, odd rows
])
def test_gather_bit_exact(B, S, H, D, bounds, max_len, dtype):
    g = torch.Generator().manual_seed(81)
    k = torch.randn(B, S, H, D, generator=g).to(dtype)
    v = torch.randn(B, S, H, D, generator=g).to(dtype)
    dk, dv = cuda(k, v)
    yk, yv = binding.ring_anything_gather([dk, dv], bounds, max_len)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    for src, y in ((k, yk), (v, yv)):
        want = oracle.ring_anything_gather(_bits(src), bounds, max_len)
        assert torch.equal(_bits(y.cpu()), want)


def test_ring_over_sliced_blocks_equals_ring_sim():
    """Attention of every true-length slice of the gathered K/V (strided views, no copy),
    merged by LSE: the same launches and arithmetic as attention of each block cut from the
    unpadded K/V, so the same bits; and the same result as cp_ring_sim (which runs every
    block in one launch) up to fp32 rounding order."""
    B, H, S, D = 2, 4, 4481, 128
    bounds = binding.ring_bounds(S, 4, anything=True)      # 1121/1120/1120/1120
    q, k, v = cuda(*make_qkv(B, H, S, S, D, seed=82, rms_norm_qk=True))
    max_len = max(b - a for a, b in zip(bounds[:-1], bounds[1:]))
    gk, gv = binding.ring_anything_gather([k, v], bounds, max_len)
    n = len(bounds) - 1
    parts = torch.empty((n, B, S, H, D), dtype=torch.float32, device="cuda")
    lses = torch.empty((n, B, H, S), dtype=torch.float32, device="cuda")
    for c in range(n):
        L = bounds[c + 1] - bounds[c]
        binding.attn_fwd_strided(q, gk[c, :, :L], gv[c, :, :L], out_dtype=torch.float32, out=parts[c], lse=lses[c])
    o, lse = binding.attn_merge(parts, lses)
    for c in range(n):
        kb, vb = (x[:, bounds[c]:bounds[c + 1]].contiguous() for x in (k, v))
        binding.attn_fwd(q, kb, vb, out_dtype=torch.float32, out=parts[c], lse=lses[c])
    ref, ref_lse = binding.attn_merge(parts, lses)
    o_ring, lse_ring, _ = binding.ring_sim(q, k, v, bounds)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    assert torch.equal(o, ref) and torch.equal(lse, ref_lse)
    assert_split_close(o, o_ring, "sliced gathered blocks vs cp_ring_sim")
    assert float((lse - lse_ring).abs().max()) <= LSE_ABS


def test_ring_over_sliced_blocks_matches_oracle():
    B, H, S, D = 1, 3, 1000, 64
    bounds = [0, 401, 402, 1000]
    q, k, v = qkv(B, H, S, S, D, seed=83)
    scale = 1 / math.sqrt(D)
    dq, dk, dv = cuda(q, k, v)
    gk, gv = binding.ring_anything_gather([dk, dv], bounds, 600)
    n = len(bounds) - 1
    parts = torch.empty((n, B, S, H, D), dtype=torch.float32, device="cuda")
    lses = torch.empty((n, B, H, S), dtype=torch.float32, device="cuda")
    for c in range(n):
        L = bounds[c + 1] - bounds[c]
        binding.attn_fwd_strided(dq, gk[c, :, :L], gv[c, :, :L], out_dtype=torch.float32, out=parts[c], lse=lses[c])
    o, lse = binding.attn_merge(parts, lses)
    o_ref, lse_ref = oracle.attention(q, k, v, scale)
    assert_attn_close(o, lse, o_ref, lse_ref, "ring anything over gathered slices")
