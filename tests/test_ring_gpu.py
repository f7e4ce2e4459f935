"""cp_ring_sim and cp_attn_merge against the oracle, and split-degree invariance.

The pages report outputs drifting across parallel degrees ("FLUX with SP: images
differ across parallel degrees"): a split changes the summation order, and both
results are correct.  Here every split must match the fp64 oracle within the
attention tolerances and the unsplit GPU result within 1e-2 max-abs.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from context_attention_dit_b200 import binding
from context_attention_dit_b200.inputs import bounds_from_sizes, even_bounds
from tests.gpu_util import (assert_attn_close, assert_split_close, cuda, qkv, sample_rows, workload_inputs,
                            workload_oracle)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize(
    "shape,bounds",
    [
        ((1, 2, 256, 256, 64), [0, 128, 256]),
        ((2, 3, 300, 300, 128), [0, 100, 200, 300]),
        ((1, 2, 200, 450, 128), [0, 0, 130, 130, 450]),     # empty blocks
        ((1, 1, 129, 17, 64), [0, 5, 6, 17]),               # blocks far below one tile
        ((1, 2, 150, 640, 128), [0, 640, 640]),             # trailing empty block
    ],
)
def test_ring_small_matches_oracle(shape, bounds):
    B, H, Sq, Skv, D = shape
    q, k, v = qkv(B, H, Sq, Skv, D, seed=31)
    scale = 1 / math.sqrt(D)
    o_ref, lse_ref, parts_ref, lses_ref = oracle.ring(q, k, v, scale, bounds)
    dq, dk, dv = cuda(q, k, v)
    o, lse, ws = binding.ring_sim(dq, dk, dv, bounds, scale=scale)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    assert_attn_close(o, lse, o_ref, lse_ref, f"ring {bounds}")
    n = len(bounds) - 1
    if n > 1:  # the per-block partials in the workspace match the oracle's blocks
        parts, lses = binding.ring_workspace_views(ws, n, B, H, Sq, D)
        for r in range(n):
            assert_attn_close(parts[r], lses[r], parts_ref[r], lses_ref[r], f"block {r}")
    o_full, _ = binding.attn_fwd(dq, dk, dv, scale=scale)
    assert_split_close(o, o_full, f"ring {bounds}")


def test_tiny_workload_two_blocks():
    w, (q, k, v) = workload_inputs("tiny_s256_d64")
    o_ref, lse_ref = oracle.attention(q, k, v, w.scale)
    dq, dk, dv = cuda(q, k, v)
    o, lse, _ = binding.ring_sim(dq, dk, dv, bounds_from_sizes(w.splits[0]), scale=w.scale)
    assert_attn_close(o, lse, o_ref, lse_ref, "tiny split 2x128")
    o1, _ = binding.attn_fwd(dq, dk, dv, scale=w.scale)
    assert_split_close(o, o1, "tiny")


def test_flux_ring8_all_elements():
    w, (q, k, v) = workload_inputs("flux_1024_ring8_ulysses8")
    o_ref, lse_ref = workload_oracle("flux_1024_ring1")  # same inputs (seed, shape, QK-norm)
    dq, dk, dv = cuda(q, k, v)
    o, lse, _ = binding.ring_sim(dq, dk, dv, even_bounds(w.S, 8), scale=w.scale)
    assert_attn_close(o, lse, o_ref, lse_ref, "flux ring-8")
    o1, _ = binding.attn_fwd(dq, dk, dv, scale=w.scale)
    assert_split_close(o, o1, "flux ring-8 vs ring-1")


@pytest.mark.parametrize("split", [0, 1], ids=["1391x3", "1392-1391-1390"])
def test_uneven_ring_anything_all_elements(split):
    w, (q, k, v) = workload_inputs("uneven_s4173_ring3")
    o_ref, lse_ref = workload_oracle("uneven_s4173_ring3")
    dq, dk, dv = cuda(q, k, v)
    o, lse, _ = binding.ring_sim(dq, dk, dv, bounds_from_sizes(w.splits[split]), scale=w.scale)
    assert_attn_close(o, lse, o_ref, lse_ref, f"uneven split {w.splits[split]}")
    o1, _ = binding.attn_fwd(dq, dk, dv, scale=w.scale)
    assert_split_close(o, o1, "uneven vs unsplit")


def test_flux_1008_ring_anything_4():
    """FLUX at 1008^2 (4481 tokens, not divisible by 4): ring-anything over 4 blocks."""
    B, H, S, D = 1, 24, 4481, 128
    q, k, v = qkv(B, H, S, S, D, seed=42, rms=True)
    bounds = binding.ring_bounds(S, 4, anything=True)
    rows = sample_rows(S, bounds, n_random=200)
    o_ref, lse_ref = oracle.attention_rows(q, k, v, 1 / math.sqrt(D), rows)
    dq, dk, dv = cuda(q, k, v)
    o, lse, _ = binding.ring_sim(dq, dk, dv, bounds)
    assert_attn_close(o[:, rows], lse[:, :, rows], o_ref, lse_ref, "flux-1008 ring-anything-4")
    o1, _ = binding.attn_fwd(dq, dk, dv)
    assert_split_close(o, o1, "flux-1008")


def test_video_ring4_sampled_rows():
    """Video DiT (B1 H40 S32760 D128): sampled query rows vs fp64, every element vs unsplit GPU."""
    w, (q, k, v) = workload_inputs("video_s32760_ring4")
    bounds = bounds_from_sizes(w.splits[0])
    rows = sample_rows(w.S, bounds, n_random=400)
    o_ref, lse_ref = oracle.attention_rows(q, k, v, w.scale, rows)
    dq, dk, dv = cuda(q, k, v)
    o, lse, _ = binding.ring_sim(dq, dk, dv, bounds, scale=w.scale)
    assert_attn_close(o[:, rows], lse[:, :, rows], o_ref, lse_ref, "video ring-4 (sampled rows)")
    o1, lse1 = binding.attn_fwd(dq, dk, dv, scale=w.scale)
    assert_attn_close(o1[:, rows], lse1[:, :, rows], o_ref, lse_ref, "video ring-1 (sampled rows)")
    assert_split_close(o, o1, "video ring-4 vs ring-1")


def test_merge_kernel_against_oracle_merge():
    """cp_attn_merge alone: random partials/LSEs (incl. -inf blocks) vs the fp64 merge."""
    n, B, H, Sq, D = 5, 2, 3, 97, 128
    g = torch.Generator().manual_seed(9)
    parts = torch.randn(n, B, Sq, H, D, generator=g)
    lses = torch.randn(n, B, H, Sq, generator=g) * 4
    lses[1, 0, 0, :10] = -math.inf
    lses[:, 1, 2, 5] = -math.inf  # a row with every block empty
    o_ref, l_ref = oracle.merge(parts, lses)
    o, l = binding.attn_merge(parts.cuda(), lses.cuda(), out_dtype=torch.float32)
    torch.cuda.synchronize()
    ob, _ = binding.attn_merge(parts.cuda(), lses.cuda(), out_dtype=torch.bfloat16)
    assert np.abs(o.cpu().double().numpy() - o_ref).max() < 1e-5
    fin = np.isfinite(l_ref)
    assert np.array_equal(np.isneginf(l.cpu().numpy()), ~fin)
    assert np.abs(l.cpu().double().numpy()[fin] - l_ref[fin]).max() < 1e-5
    assert np.abs(ob.cpu().double().numpy() - o_ref).max() < 2e-2
    assert (o[1, 5, 2] == 0).all()


@pytest.mark.parametrize("D", [64, 128])
def test_merge_single_block_is_identity(D):
    parts = torch.randn(1, 1, 33, 2, D).cuda()
    lses = torch.randn(1, 1, 2, 33).cuda()
    o, l = binding.attn_merge(parts, lses, out_dtype=torch.float32)
    assert torch.allclose(o, parts[0], atol=1e-6, rtol=1e-6)
    assert torch.allclose(l, lses[0], atol=1e-5)


def test_ring_deterministic():
    q, k, v = cuda(*qkv(1, 2, 500, 700, 128, seed=23))
    outs = [binding.ring_sim(q, k, v, [0, 300, 301, 700], out_dtype=torch.float32)[:2] for _ in range(3)]
    for o, l in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(l, outs[0][1])


@pytest.mark.parametrize(
    "shape,bounds",
    [
        ((1, 2, 256, 256, 64), [0, 128, 256]),
        ((2, 3, 300, 300, 128), [0, 100, 200, 300]),
        ((1, 2, 200, 450, 128), [0, 0, 130, 130, 450]),     # empty blocks
        ((1, 1, 129, 17, 64), [0, 5, 6, 17]),
        ((1, 2, 150, 640, 128), [0, 640, 640]),
    ],
)
def test_fused_ring_matches_oracle_and_unfused(shape, bounds):
    """Fused merge (running softmax carried across blocks) == oracle ring == unfused ring."""
    B, H, Sq, Skv, D = shape
    q, k, v = qkv(B, H, Sq, Skv, D, seed=41)
    scale = 1 / math.sqrt(D)
    o_ref, lse_ref, _, _ = oracle.ring(q, k, v, scale, bounds)
    dq, dk, dv = cuda(q, k, v)
    o, lse = binding.ring_sim_fused(dq, dk, dv, bounds, scale=scale)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    assert_attn_close(o, lse, o_ref, lse_ref, f"fused ring {bounds}")
    o2, _, _ = binding.ring_sim(dq, dk, dv, bounds, scale=scale)
    assert_split_close(o, o2, f"fused vs unfused {bounds}")


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
@pytest.mark.parametrize(
    "shape,bounds",
    [
        ((1, 24, 4608, 4608, 128), [576 * i for i in range(9)]),  # FLUX ring-8
        ((2, 3, 300, 300, 128), [0, 100, 200, 300]),
        ((1, 2, 200, 450, 64), [0, 0, 130, 130, 450]),          # empty blocks
        ((1, 2, 129, 17, 64), [0, 5, 6, 17]),
    ],
)
def test_fused_ring_equals_unsplit_bit_for_bit(shape, bounds, out_dtype):
    """The fused ring's blocks are consecutive ranges of one K/V tensor feeding one running
    softmax, so the launch tiles their union exactly as unsplit attention tiles the keys:
    the result does not depend on the split at all, bit for bit."""
    B, H, Sq, Skv, D = shape
    q, k, v = cuda(*qkv(B, H, Sq, Skv, D, seed=47, rms=True))
    o, lse = binding.ring_sim_fused(q, k, v, bounds, out_dtype=out_dtype)
    o1, l1 = binding.attn_fwd(q, k, v, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    assert torch.equal(o, o1) and torch.equal(lse, l1)


def test_fused_ring_all_blocks_empty():
    q, k, v = cuda(*qkv(1, 2, 130, 0, 128))
    o, lse = binding.ring_sim_fused(q, k, v, [0, 0, 0])
    torch.cuda.synchronize()
    assert not o.float().abs().sum().item() and torch.isneginf(lse).all()


def test_fused_flux_ring8_and_uneven():
    w, (q, k, v) = workload_inputs("flux_1024_ring8_ulysses8")
    o_ref, lse_ref = workload_oracle("flux_1024_ring1")
    o, lse = binding.ring_sim_fused(*cuda(q, k, v), even_bounds(w.S, 8), scale=w.scale)
    assert_attn_close(o, lse, o_ref, lse_ref, "fused flux ring-8")
    w2, (q2, k2, v2) = workload_inputs("uneven_s4173_ring3")
    o_ref2, lse_ref2 = workload_oracle("uneven_s4173_ring3")
    o2, lse2 = binding.ring_sim_fused(*cuda(q2, k2, v2), bounds_from_sizes(w2.splits[1]), scale=w2.scale)
    assert_attn_close(o2, lse2, o_ref2, lse_ref2, "fused uneven 1392/1391/1390")


def test_bench_step_launch_configuration():
    """The hot path exactly as bench.py times it on FLUX: the Ulysses-8 exchange of Q, K, V
    in one launch, ring-8 attention over the head-sharded tensors (batch 8, 3 heads) in one
    launch, the LSE merge, the inverse exchange of O.  Every element against fp64."""
    w, (q, k, v) = workload_inputs("flux_1024_ring8_ulysses8")
    o_ref, lse_ref = workload_oracle("flux_1024_ring1")  # same inputs (seed, shape, QK-norm)
    P, B, S, H, D = 8, w.B, w.S, w.H, w.D
    xs = [t.reshape(B, P, S // P, H, D).permute(1, 0, 2, 3, 4).contiguous().cuda() for t in (q, k, v)]
    ys = binding.ulysses_permute_n(xs, P, 0)
    view = lambda t: t.view(P * B, S, H // P, D)
    parts, lses = binding.attn_fwd_blocks(view(ys[0]), view(ys[1]), view(ys[2]), even_bounds(S, 8), scale=w.scale)
    o_h, lse_h = binding.attn_merge(parts, lses)
    o_seq = binding.ulysses_permute(o_h.view(P, B, S, H // P, D), P, 1)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    o = o_seq.permute(1, 0, 2, 3, 4).reshape(B, S, H, D)
    lse = lse_h.view(P, B, H // P, S).permute(1, 0, 2, 3).reshape(B, H, S)  # head group p = heads 3p..3p+2
    assert_attn_close(o, lse, o_ref, lse_ref, "bench step (FLUX Ulysses-8 x ring-8)")


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
@pytest.mark.parametrize("P,B,S,H,D,n", [(8, 1, 4608, 24, 128, 8), (4, 2, 200, 8, 64, 3), (3, 1, 99, 6, 128, 1)])
def test_merge_ulysses_equals_merge_then_inverse_exchange(P, B, S, H, D, n, out_dtype):
    g = torch.Generator().manual_seed(P * 7 + S)
    parts = torch.randn(n, P * B, S, H // P, D, generator=g).cuda()
    lses = (torch.randn(n, P * B, H // P, S, generator=g) * 3).cuda()
    lses[0, 0, 0, :5] = -math.inf                    # an empty block for some rows
    if n > 1:
        lses[:, -1, -1, -1] = -math.inf              # a row with every block empty
    o_h, l_h = binding.attn_merge(parts, lses, out_dtype=out_dtype)
    want = binding.ulysses_permute(o_h.view(P, B, S, H // P, D), P, 1)
    want_lse = l_h.view(P, B, H // P, S).permute(1, 0, 2, 3).reshape(B, H, S)
    o, lse = binding.attn_merge_ulysses(parts, lses, P, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert torch.equal(o, want)
    assert torch.equal(lse, want_lse)


def test_bench_step_fused_merge_matches_oracle():
    """The bench step with the merge fused into the inverse exchange, every element vs fp64."""
    w, (q, k, v) = workload_inputs("flux_1024_ring8_ulysses8")
    o_ref, lse_ref = workload_oracle("flux_1024_ring1")
    P, B, S, H, D = 8, w.B, w.S, w.H, w.D
    xs = [t.reshape(B, P, S // P, H, D).permute(1, 0, 2, 3, 4).contiguous().cuda() for t in (q, k, v)]
    ys = binding.ulysses_permute_n(xs, P, 0)
    view = lambda t: t.view(P * B, S, H // P, D)
    parts, lses = binding.attn_fwd_blocks(view(ys[0]), view(ys[1]), view(ys[2]), even_bounds(S, 8), scale=w.scale)
    o_seq, lse = binding.attn_merge_ulysses(parts, lses, P)
    o = o_seq.permute(1, 0, 2, 3, 4).reshape(B, S, H, D)
    assert_attn_close(o, lse, o_ref, lse_ref, "bench step, fused merge + inverse exchange")
