"""cp_attn_fwd_strided (attention on views inside larger tensors) and
cp_ring_sim_fused_ulysses (the fused ring writing the token-sharded output), against the
fp64 oracle and bit for bit against the dense entry points they generalise.

"Context parallelism", "Ring Attention": a ring step attends the local queries to one
K/V block, which a caller often holds as a slice of a longer sequence; "Unified
Attention": an exchange, the ring on the head shards, and the reverse exchange."""

import math

import pytest
import torch

import oracle
from context_attention_dit_b200 import binding
from context_attention_dit_b200.inputs import even_bounds
from tests.gpu_util import assert_attn_close, assert_split_close, cuda, qkv, workload_inputs, workload_oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,Sq,S_full,c0,c1,D", [
    (1, 4, 300, 1000, 250, 700, 128),    # a K/V block inside a longer sequence
    (2, 3, 129, 640, 0, 77, 64),         # a short block at the start, batch stride = the full length
    (2, 2, 200, 500, 371, 500, 128),     # a ragged block at the end
])
def test_kv_block_view_matches_oracle_and_dense(B, H, Sq, S_full, c0, c1, D):
    q, k_full, v_full = qkv(B, H, Sq, S_full, D, seed=71)
    scale = 1 / math.sqrt(D)
    o_ref, lse_ref = oracle.attention(q, k_full[:, c0:c1], v_full[:, c0:c1], scale)
    dq, dk, dv = cuda(q, k_full, v_full)
    kv, vv = dk[:, c0:c1], dv[:, c0:c1]                 # views: no copy
    assert not kv.is_contiguous() or B == 1
    o, lse = binding.attn_fwd_strided(dq, kv, vv, scale=scale)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    assert_attn_close(o, lse, o_ref, lse_ref, f"kv view [{c0}, {c1})")
    o_d, lse_d = binding.attn_fwd(dq, kv.contiguous(), vv.contiguous(), scale=scale)
    assert torch.equal(o, o_d) and torch.equal(lse, lse_d), "strided != dense on the same data"


def test_packed_qkv_and_strided_output():
    """Q, K, V as slices of one packed [B, S, 3, H, D] tensor; the output written into rows
    [5, 5 + S) of a larger fp32 tensor, whose other rows stay untouched."""
    B, S, H, D = 2, 333, 4, 128
    q, k, v = qkv(B, H, S, S, D, seed=72, rms=True)
    packed = torch.stack([q, k, v], dim=2).cuda()        # [B, S, 3, H, D]
    pq, pk, pv = packed[:, :, 0], packed[:, :, 1], packed[:, :, 2]
    big = torch.full((B, S + 10, H, D), float("nan"), dtype=torch.float32, device="cuda")
    out = big[:, 5:5 + S]
    o, lse = binding.attn_fwd_strided(pq, pk, pv, out_dtype=torch.float32, out=out)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    assert o.data_ptr() == out.data_ptr()
    o_ref, lse_ref = oracle.attention(q, k, v, 1 / math.sqrt(D))
    assert_attn_close(big[:, 5:5 + S], lse, o_ref, lse_ref, "packed qkv, strided fp32 output")
    assert torch.isnan(big[:, :5]).all() and torch.isnan(big[:, 5 + S:]).all(), "wrote outside the output view"
    o_d, lse_d = binding.attn_fwd(*cuda(q, k, v), out_dtype=torch.float32)
    assert torch.equal(big[:, 5:5 + S], o_d) and torch.equal(lse, lse_d)


def test_empty_kv_view():
    """A K/V block of no rows (an empty slice): O = 0 and lse = -inf, as with cp_attn_fwd."""
    q, k_full, v_full = cuda(*qkv(2, 3, 77, 100, 64, seed=75))
    o, lse = binding.attn_fwd_strided(q, k_full[:, 40:40], v_full[:, 40:40], out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    assert torch.equal(o, torch.zeros_like(o)) and bool(torch.isneginf(lse).all())


def test_interleaved_output_layout():
    """An output whose batches sit side by side within each sequence row ([S][B][H][D])."""
    B, S, H, D = 3, 200, 2, 64
    q, k, v = qkv(B, H, S, S, D, seed=73)
    sbhd = torch.empty((S, B, H, D), dtype=torch.bfloat16, device="cuda")
    out = sbhd.permute(1, 0, 2, 3)                        # strides (H*D, B*H*D, D, 1)
    binding.attn_fwd_strided(*cuda(q, k, v), out=out)
    o_d, _ = binding.attn_fwd(*cuda(q, k, v))
    torch.cuda.synchronize()
    assert torch.equal(out, o_d)


def shard(x, P):
    B, S, H, D = x.shape
    return x.reshape(B, P, S // P, H, D).permute(1, 0, 2, 3, 4).contiguous()


def unshard(x):
    P, B, Sp, H, D = x.shape
    return x.permute(1, 0, 2, 3, 4).reshape(B, P * Sp, H, D)


@pytest.mark.parametrize("B,H,S,D,P,bounds", [
    (2, 4, 256, 64, 2, [0, 100, 256]),
    (1, 6, 300, 128, 3, [0, 300]),
    (2, 8, 384, 128, 4, [0, 128, 129, 384]),
    (1, 4, 200, 128, 2, [0, 0, 77, 200]),
])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
def test_fused_ulysses_small_matches_oracle(B, H, S, D, P, bounds, out_dtype):
    q, k, v = qkv(B, H, S, S, D, seed=74)
    scale = 1 / math.sqrt(D)
    o_ref, lse_ref = oracle.attention(q, k, v, scale)
    heads = binding.ulysses_permute_n([shard(t, P).cuda() for t in (q, k, v)], P, 0)
    o, lse = binding.ring_sim_fused_ulysses(*heads, P, bounds, scale=scale, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    assert o.shape == (P, B, S // P, H, D) and lse.shape == (B, H, S)
    assert_attn_close(unshard(o), lse, o_ref, lse_ref, f"fused ulysses {P} x {bounds}")
    # The fused kernel with a plain output, followed by the inverse exchange, gives the same
    # bits: only the output address differs.
    view = lambda t: t.view(P * B, S, H // P, D)  # noqa: E731
    of, lf = binding.ring_sim_fused(*(view(t) for t in heads), bounds, scale=scale, out_dtype=out_dtype)
    assert torch.equal(o, binding.ulysses_permute(of.view(P, B, S, H // P, D), P, 1))
    assert torch.equal(lse, lf.view(P, B, H // P, S).permute(1, 0, 2, 3).reshape(B, H, S))


def test_fused_ulysses_flux_all_elements():
    """FLUX B1 H24 S4608 D128: Ulysses-8 exchange, then the fused ring-8 writing the
    token-sharded output; every element against the fp64 oracle and the unsplit GPU result."""
    w, (q, k, v) = workload_inputs("flux_1024_ring1")
    o_ref, lse_ref = workload_oracle("flux_1024_ring1")
    P = 8
    heads = binding.ulysses_permute_n([shard(t, P).cuda() for t in (q, k, v)], P, 0)
    o, lse = binding.ring_sim_fused_ulysses(*heads, P, even_bounds(w.S, 8), scale=w.scale)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    assert_attn_close(unshard(o), lse, o_ref, lse_ref, "flux fused ulysses-8 x ring-8")
    o1, _ = binding.attn_fwd(*cuda(q, k, v), scale=w.scale)
    assert_split_close(unshard(o), o1, "flux fused ulysses-8 x ring-8 vs unsplit")


def test_fused_ulysses_rejects_indivisible():
    x = torch.zeros(3, 1, 16, 2, 64, dtype=torch.bfloat16, device="cuda")  # S = 16 not divisible by 3
    with pytest.raises(ValueError):
        binding.ring_sim_fused_ulysses(x, x, x, 3, [0, 16])


def test_fused_ulysses_video_sampled_rows():
    """Video DiT (B1 H40 S32760 D128) over Ulysses-8 (5 heads per shard) x ring-4: sampled
    rows against the fp64 oracle, every element against unsplit GPU attention."""
    from tests.gpu_util import sample_rows

    w, (q, k, v) = workload_inputs("video_s32760_ring4")
    P, bounds = 8, even_bounds(w.S, 4)
    rows = sample_rows(w.S, bounds + [i * w.S // P for i in range(P + 1)], n_random=200)
    o_ref, lse_ref = oracle.attention_rows(q, k, v, w.scale, rows)
    heads = binding.ulysses_permute_n([shard(t, P).cuda() for t in (q, k, v)], P, 0)
    o, lse = binding.ring_sim_fused_ulysses(*heads, P, bounds, scale=w.scale)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    o = unshard(o)
    assert_attn_close(o[:, rows], lse[:, :, rows], o_ref, lse_ref, "video fused ulysses-8 x ring-4 (sampled rows)")
    o1, _ = binding.attn_fwd(*cuda(q, k, v), scale=w.scale)
    assert_split_close(o, o1, "video fused ulysses-8 x ring-4 vs unsplit")
