"""cp_ulysses_anything_permute ("Context parallelism", section "Ulysses Anything Attention"):
bit-exact against the oracle's index map for shards of unequal size, equal to the even
exchange on equal shards, and Ulysses-Anything attention bit-exact against unsplit."""

import pytest
import torch

import oracle
from context_attention_dit_b200 import binding
from tests.gpu_util import cuda, qkv

pytestmark = pytest.mark.gpu


def near_even(count, parts):
    return binding.ring_bounds(count, parts, anything=True)


def pack_seq(x, sb):
    """[B,S,H,D] -> packed sequence shards (shard p = tokens [sb[p], sb[p+1]) as [B][S_p][H][D])."""
    return torch.cat([x[:, sb[p]:sb[p + 1]].reshape(-1) for p in range(len(sb) - 1)])


def pack_head(x, hb):
    """[B,S,H,D] -> packed head shards (shard q = heads [hb[q], hb[q+1]) as [B][S][H_q][D])."""
    return torch.cat([x[:, :, hb[q]:hb[q + 1]].reshape(-1) for q in range(len(hb) - 1)])


CASES = [
    # (P, B, S, H, D, dtype, seq_bounds or None = near even, head_bounds or None)
    (4, 1, 4481, 24, 128, torch.bfloat16, None, None),      # FLUX 1008^2: 4481 tokens over 4
    (5, 2, 1000, 24, 128, torch.bfloat16, None, None),      # 24 heads over 5
    (4, 2, 10, 3, 64, torch.bfloat16, None, [0, 1, 2, 3, 3]),  # an empty head group
    (3, 1, 9, 6, 64, torch.float32, [0, 0, 4, 9], None),    # an empty sequence shard, fp32
    (3, 2, 7, 5, 5, torch.bfloat16, None, None),            # odd head_dim: 2-byte vectors
    (2, 1, 33, 3, 128, torch.float32, None, None),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "P%d_B%d_S%d_H%d_D%d_%s" % (*c[:5], str(c[5])[6:]))
def test_anything_bit_exact(case):
    P, B, S, H, D, dtype, sb, hb = case
    sb = sb or near_even(S, P)
    hb = hb or near_even(H, P)
    g = torch.Generator().manual_seed(S * 31 + H)
    x = torch.randn(B, S, H, D, generator=g).to(dtype)
    ref = oracle.ulysses_anything_fwd([x[:, sb[p]:sb[p + 1]] for p in range(P)], sb, hb)
    ref_flat = torch.cat([r.reshape(-1) for r in ref])
    assert torch.equal(ref_flat, pack_head(x, hb))
    y = binding.ulysses_anything_permute(pack_seq(x, sb).cuda(), P, sb, hb, B, S, H, D, 0)
    assert torch.equal(y.cpu(), ref_flat)
    back = binding.ulysses_anything_permute(y, P, sb, hb, B, S, H, D, 1)
    assert torch.equal(back.cpu(), pack_seq(x, sb))


@pytest.mark.parametrize("case", [CASES[0], CASES[2], CASES[3]], ids=["flux1008_p4", "empty_heads", "empty_seq"])
def test_anything_batched_bit_exact(case):
    """Q, K and V in one launch: each equals the oracle's exchange of that tensor."""
    P, B, S, H, D, dtype, sb, hb = case
    sb = sb or near_even(S, P)
    hb = hb or near_even(H, P)
    g = torch.Generator().manual_seed(S * 17 + H)
    xs = [torch.randn(B, S, H, D, generator=g).to(dtype) for _ in range(3)]
    ys = binding.ulysses_anything_permute_n([pack_seq(x, sb).cuda() for x in xs], P, sb, hb, B, S, H, D, 0)
    for x, y in zip(xs, ys):
        ref = oracle.ulysses_anything_fwd([x[:, sb[p]:sb[p + 1]] for p in range(P)], sb, hb)
        assert torch.equal(y.cpu(), torch.cat([r.reshape(-1) for r in ref]))
    backs = binding.ulysses_anything_permute_n(ys, P, sb, hb, B, S, H, D, 1)
    for x, b in zip(xs, backs):
        assert torch.equal(b.cpu(), pack_seq(x, sb))


def test_anything_equals_even_exchange_on_equal_shards():
    P, B, S, H, D = 8, 1, 4608, 24, 128
    x = torch.randn(P, B, S // P, H, D, generator=torch.Generator().manual_seed(3)).bfloat16().cuda()
    even = binding.ulysses_permute(x, P, 0)
    any_ = binding.ulysses_anything_permute(x, P, near_even(S, P), near_even(H, P), B, S, H, D, 0)
    assert torch.equal(any_, even.reshape(-1))


@pytest.mark.parametrize("P,S,H", [(4, 4481, 24), (5, 2048, 24), (3, 1000, 8)], ids=["flux1008_p4", "h24_p5", "s1000_h8_p3"])
def test_anything_attention_bit_exact_vs_unsplit(P, S, H):
    """Exchange -> attention on each head shard (unequal head counts) -> inverse exchange:
    every head is computed by identical code on identical data, so the result equals unsplit
    attention bit for bit."""
    B, D = 1, 128
    q, k, v = cuda(*qkv(B, H, S, S, D, seed=71, rms=True))
    o_full, _ = binding.attn_fwd(q, k, v)
    sb, hb = near_even(S, P), near_even(H, P)
    heads = [binding.ulysses_anything_permute(pack_seq(t, sb), P, sb, hb, B, S, H, D, 0) for t in (q, k, v)]
    o_heads = torch.empty(B * S * H * D, dtype=torch.bfloat16, device="cuda")
    for g in range(P):
        Hq = hb[g + 1] - hb[g]
        if Hq == 0:
            continue
        lo, hi = B * S * hb[g] * D, B * S * hb[g + 1] * D
        view = lambda t: t[lo:hi].view(B, S, Hq, D)
        binding.attn_fwd(view(heads[0]), view(heads[1]), view(heads[2]), out=view(o_heads), want_lse=False)
    o_seq = binding.ulysses_anything_permute(o_heads, P, sb, hb, B, S, H, D, 1)
    assert torch.equal(o_seq, pack_seq(o_full, sb))
