"""cp_usp_sim (Ulysses x ring, "Context parallelism", section "Unified Attention") against the
fp64 oracle, and split invariance against unsplit GPU attention."""

import math

import pytest
import torch

import oracle
from context_attention_dit_b200 import binding
from context_attention_dit_b200.inputs import bounds_from_sizes, even_bounds
from tests.gpu_util import (assert_attn_close, assert_split_close, cuda, qkv, sample_rows, workload_inputs,
                            workload_oracle)

pytestmark = pytest.mark.gpu


def shard(x, P):
    """[B,S,H,D] -> sequence-sharded [P,B,S/P,H,D] (shard p = tokens [p*S/P, (p+1)*S/P))."""
    B, S, H, D = x.shape
    return x.reshape(B, P, S // P, H, D).permute(1, 0, 2, 3, 4).contiguous()


def unshard(x):
    """Sequence-sharded [P,B,S/P,H,D] -> [B,S,H,D]."""
    P, B, Sp, H, D = x.shape
    return x.permute(1, 0, 2, 3, 4).reshape(B, P * Sp, H, D)


@pytest.mark.parametrize(
    "shape,degree,bounds",
    [
        ((2, 4, 256, 64), 2, [0, 100, 256]),
        ((1, 8, 384, 128), 4, [0, 128, 129, 384]),   # an empty-ish 1-key block
        ((1, 6, 300, 128), 3, [0, 300]),             # one ring block: the unmerged path
        ((1, 4, 200, 128), 2, [0, 0, 77, 200]),      # an empty block
    ],
)
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
def test_usp_small_matches_oracle(shape, degree, bounds, out_dtype):
    B, H, S, D = shape
    q, k, v = qkv(B, H, S, S, D, seed=61)
    scale = 1 / math.sqrt(D)
    qs, ks, vs = (shard(t, degree) for t in (q, k, v))
    o_ref, lse_ref = oracle.usp(qs, ks, vs, degree, scale, bounds)
    o, lse, _ = binding.usp_sim(*cuda(qs, ks, vs), degree, bounds, scale=scale, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    assert_attn_close(unshard(o), lse, unshard(torch.from_numpy(o_ref)), lse_ref, f"usp {degree} x {bounds}")


@pytest.mark.parametrize("degree,ring", [(2, 4), (4, 2)], ids=["ulysses2_ring4", "ulysses4_ring2"])
def test_usp_flux_all_elements(degree, ring):
    w, (q, k, v) = workload_inputs("flux_1024_ring1")
    o_ref, lse_ref = workload_oracle("flux_1024_ring1")  # USP equals unsplit attention
    qs, ks, vs = cuda(*(shard(t, degree) for t in (q, k, v)))
    o, lse, _ = binding.usp_sim(qs, ks, vs, degree, even_bounds(w.S, ring), scale=w.scale)
    assert_attn_close(unshard(o), lse, o_ref, lse_ref, f"flux usp {degree}x{ring}")
    o1, _ = binding.attn_fwd(*cuda(q, k, v), scale=w.scale)
    assert_split_close(unshard(o), o1, f"flux usp {degree}x{ring} vs unsplit")


@pytest.mark.parametrize("degree,ring", [(2, 4), (4, 2)], ids=["ulysses2_ring4", "ulysses4_ring2"])
def test_usp_video_sampled_rows(degree, ring):
    """Video DiT (B1 H40 S32760 D128): sampled rows vs fp64, every element vs unsplit GPU."""
    w, (q, k, v) = workload_inputs("video_s32760_ring4")
    bounds = even_bounds(w.S, ring)
    rows = sample_rows(w.S, bounds, n_random=300)
    o_ref, lse_ref = oracle.attention_rows(q, k, v, w.scale, rows)
    qs, ks, vs = cuda(*(shard(t, degree) for t in (q, k, v)))
    o, lse, _ = binding.usp_sim(qs, ks, vs, degree, bounds, scale=w.scale)
    o = unshard(o)
    assert_attn_close(o[:, rows], lse[:, :, rows], o_ref, lse_ref, f"video usp {degree}x{ring} (sampled rows)")
    o1, _ = binding.attn_fwd(*cuda(q, k, v), scale=w.scale)
    assert_split_close(o, o1, f"video usp {degree}x{ring} vs unsplit")


def test_usp_ulysses_only_is_bit_exact():
    """Ring degree 1: each head is computed by identical code on identical data after the
    exchange, so the result equals unsplit attention bit for bit."""
    q, k, v = qkv(1, 8, 1024, 1024, 128, seed=63, rms=True)
    o1, l1 = binding.attn_fwd(*cuda(q, k, v))
    o, lse, _ = binding.usp_sim(*cuda(*(shard(t, 4) for t in (q, k, v))), 4, [0, 1024])
    assert torch.equal(unshard(o), o1) and torch.equal(lse, l1)


def test_usp_rejects_indivisible():
    q = torch.zeros(3, 1, 5, 4, 64, dtype=torch.bfloat16, device="cuda")  # S = 15, H = 4, degree 3
    with pytest.raises(binding.CpError) as e:
        binding.usp_sim(q, q, q, 3, [0, 15])
    assert e.value.status == binding.CP_ERR_NOT_DIVISIBLE
