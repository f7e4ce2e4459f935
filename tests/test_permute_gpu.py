"""cp_ulysses_permute: bit-exact against the oracle's index map, and Ulysses attention
(exchange -> per-head-group attention -> inverse exchange) bit-exact against unsplit."""

import pytest
import torch

import oracle
from context_attention_dit_b200 import binding
from tests.gpu_util import cuda, qkv, workload_inputs

pytestmark = pytest.mark.gpu


def seq_shards(x, P):
    """[B,S,H,D] -> sequence-sharded [P,B,S/P,H,D] (shard p holds tokens [p*S/P, (p+1)*S/P))."""
    B, S, H, D = x.shape
    return x.reshape(B, P, S // P, H, D).permute(1, 0, 2, 3, 4).contiguous()


@pytest.mark.parametrize(
    "P,B,S,H,D,dtype",
    [
        (2, 1, 4, 4, 1, torch.bfloat16),
        (8, 1, 4608, 24, 128, torch.bfloat16),
        (4, 2, 64, 8, 64, torch.float32),
        (3, 2, 9, 6, 5, torch.bfloat16),     # odd sizes -> 2-byte vector path
        (1, 1, 33, 3, 128, torch.bfloat16),  # degree 1 is the identity
        (5, 1, 25, 40, 128, torch.float32),
    ],
)
def test_permute_bit_exact(P, B, S, H, D, dtype):
    g = torch.Generator().manual_seed(P * 100 + S)
    x = torch.randn(P, B, S // P, H, D, generator=g).to(dtype)
    y_ref = oracle.ulysses_fwd(x, P)
    y = binding.ulysses_permute(x.cuda(), P, 0)
    assert torch.equal(y.cpu(), y_ref)
    back = binding.ulysses_permute(y, P, 1)
    assert torch.equal(back.cpu(), x)
    assert torch.equal(oracle.ulysses_inv(y_ref, P), x)


def test_flux_qkv_ulysses8_bit_exact():
    w, (q, k, v) = workload_inputs("flux_1024_ring8_ulysses8")
    for t in (q, k, v):
        xs = seq_shards(t, 8)
        y = binding.ulysses_permute(xs.cuda(), 8, 0)
        assert torch.equal(y.cpu(), oracle.ulysses_fwd(xs, 8))


def test_ulysses_attention_bit_exact_vs_unsplit():
    """Each head is computed by identical code on identical data after the exchange, so the
    simulated Ulysses attention equals unsplit attention bit for bit (no cross-degree drift)."""
    P, B, S, H, D = 4, 1, 1024, 8, 128
    q, k, v = qkv(B, H, S, S, D, seed=77, rms=True)
    o_full, lse_full = binding.attn_fwd(*cuda(q, k, v), out_dtype=torch.bfloat16)
    hq, hk, hv = (binding.ulysses_permute(seq_shards(t, P).cuda(), P, 0) for t in (q, k, v))  # [P,B,S,H/P,D]
    o_h, _ = binding.attn_fwd(hq.view(P * B, S, H // P, D), hk.view(P * B, S, H // P, D),
                              hv.view(P * B, S, H // P, D))
    o_seq = binding.ulysses_permute(o_h.view(P, B, S, H // P, D), P, 1)             # [P,B,S/P,H,D]
    o_back = o_seq.permute(1, 0, 2, 3, 4).reshape(B, S, H, D)
    assert torch.equal(o_back, o_full)


def test_batched_permute_matches_single():
    g = torch.Generator().manual_seed(5)
    xs = [torch.randn(8, 1, 576, 24, 128, generator=g).bfloat16().cuda() for _ in range(3)]
    ys = binding.ulysses_permute_n(xs, 8, 0)
    for x, y in zip(xs, ys):
        assert torch.equal(y, binding.ulysses_permute(x, 8, 0))
    back = binding.ulysses_permute_n(ys, 8, 1)
    for x, b in zip(xs, back):
        assert torch.equal(x, b)


def test_batched_permute_rejects_overlap():
    x = torch.zeros(2, 1, 4, 4, 64, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(2, 1, 8, 2, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(binding.CpError):
        binding.ulysses_permute_n([x, x], 2, 0, dsts=[y, y])  # two destinations alias
