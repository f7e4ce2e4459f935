"""The one-process-per-GPU exchange kernels on one GPU, with the ranks emulated by turns.

cp_ulysses_push_n: every rank's push, launched one after another with each rank's
"peer" buffers being local ones, must fill exactly the oracle's stacked exchange
(bit-exact), in both directions.  cp_peer_barrier: passes when every signal is there
(other ranks' signals written by the host), and runs out, bounded, reporting
CP_ERR_TIMEOUT, when one never comes; the context stays usable.  cp_ring_fetch_block:
a bit-exact row copy.  No kernel here waits on another kernel.
"""

import time

import pytest
import torch

import oracle
from context_attention_dit_b200 import binding
from tests.gpu_util import cuda, qkv

pytestmark = pytest.mark.gpu


def _push_all(srcs, P, B, S, H, D, direction, dst_shape, dtype):
    """Run every rank's push; returns the P destination buffers of every tensor."""
    dsts = [[torch.zeros(dst_shape, dtype=dtype, device="cuda") for _ in range(P)] for _ in srcs]
    stream = torch.cuda.current_stream().cuda_stream
    for r in range(P):
        binding.ulysses_push_n([s[r].data_ptr() for s in srcs], [[d.data_ptr() for d in row] for row in dsts], r, P,
                               B, S, H, D, direction, srcs[0].element_size(), stream)
    torch.cuda.synchronize()
    return [torch.stack(row) for row in dsts]


@pytest.mark.parametrize(
    "P,B,S,H,D,dtype,n",
    [
        (2, 1, 256, 2, 64, torch.bfloat16, 1),
        (8, 1, 4608, 24, 128, torch.bfloat16, 3),  # FLUX-like, Q/K/V in one launch
        (4, 2, 4 * 37, 8, 128, torch.bfloat16, 3),  # ragged row groups
        (3, 2, 9, 6, 5, torch.bfloat16, 1),  # odd piece size -> 2-byte vectors
        (4, 2, 64, 8, 64, torch.float32, 2),
        (16, 1, 160, 16, 128, torch.bfloat16, 1),  # the largest group
        (1, 1, 33, 3, 128, torch.bfloat16, 1),  # degree 1: a local copy
    ],
)
def test_push_fills_the_stacked_exchange(P, B, S, H, D, dtype, n):
    g = torch.Generator().manual_seed(1000 + P * 10 + S)
    xs = [torch.randn(P, B, S // P, H, D, generator=g).to(dtype) for _ in range(n)]
    ys = _push_all([x.cuda() for x in xs], P, B, S, H, D, 0, (B, S, H // P, D), dtype)
    for x, y in zip(xs, ys):
        assert torch.equal(y.cpu(), oracle.ulysses_fwd(x, P))
    back = _push_all(ys, P, B, S, H, D, 1, (B, S // P, H, D), dtype)
    for x, b in zip(xs, back):
        assert torch.equal(b.cpu(), x)


ANYTHING = [  # (P, B, S, H, D, dtype): uneven sequence and head shards, empty ones included
    (4, 1, 4481, 24, 128, torch.bfloat16),  # FLUX-1008^2 over 4 ranks
    (5, 1, 4608, 24, 128, torch.bfloat16),  # 24 heads over 5 ranks
    (3, 2, 10, 7, 3, torch.bfloat16),  # odd head_dim -> 2-byte vectors
    (5, 1, 4, 3, 64, torch.float32),  # more ranks than tokens and heads: empty shards
    (2, 2, 9, 1, 64, torch.bfloat16),
]


@pytest.mark.parametrize("P,B,S,H,D,dtype", ANYTHING)
def test_anything_push_fills_the_oracle_shards(P, B, S, H, D, dtype):
    g = torch.Generator().manual_seed(2000 + P * 10 + S)
    x = torch.randn(B, S, H, D, generator=g).to(dtype)
    sb = binding.ring_bounds(S, P, anything=True)
    hb = binding.ring_bounds(H, P, anything=True)
    xs = [x[:, sb[p]:sb[p + 1]].contiguous() for p in range(P)]
    want = oracle.ulysses_anything_fwd(xs, sb, hb)
    stream = torch.cuda.current_stream().cuda_stream
    # Separate allocations stand in for the ranks' buffers (sizes differ per shard).
    xg = [t.cuda() for t in xs]
    ys = [torch.zeros(B, S, hb[q + 1] - hb[q], D, dtype=dtype, device="cuda") for q in range(P)]
    ptr = lambda t: t.data_ptr() if t.numel() else 16  # noqa: E731  (an empty shard is never touched)
    for r in range(P):
        binding.ulysses_anything_push_n([ptr(xg[r])], [[ptr(y) for y in ys]], r, sb, hb, B, H, D, 0,
                                        x.element_size(), stream)
    torch.cuda.synchronize()
    for q in range(P):
        assert torch.equal(ys[q].cpu(), torch.as_tensor(want[q]))
    back = [torch.zeros(B, sb[p + 1] - sb[p], H, D, dtype=dtype, device="cuda") for p in range(P)]
    for r in range(P):
        binding.ulysses_anything_push_n([ptr(ys[r])], [[ptr(t) for t in back]], r, sb, hb, B, H, D, 1,
                                        x.element_size(), stream)
    torch.cuda.synchronize()
    for p in range(P):
        assert torch.equal(back[p].cpu(), xs[p])


def test_push_ulysses_attention_equals_unsplit():
    """Ulysses attention by pushes (exchange, attention per head shard, inverse) is
    bit-identical to attention of the unsplit sequence."""
    P, B, S, H, D = 4, 1, 1024, 8, 128
    q, k, v = cuda(*qkv(B, H, S, S, D, seed=7, rms=True))
    shard = lambda x: x.reshape(B, P, S // P, H, D).permute(1, 0, 2, 3, 4).contiguous()  # noqa: E731
    yq, yk, yv = _push_all([shard(q), shard(k), shard(v)], P, B, S, H, D, 0, (B, S, H // P, D), torch.bfloat16)
    oh = torch.stack([binding.attn_fwd(yq[r], yk[r], yv[r], want_lse=False)[0] for r in range(P)])
    (xo,) = _push_all([oh], P, B, S, H, D, 1, (B, S // P, H, D), torch.bfloat16)
    full, _ = binding.attn_fwd(q, k, v, want_lse=False)
    assert torch.equal(xo.permute(1, 0, 2, 3, 4).reshape(B, S, H, D), full)


def test_push_rejects_bad_arguments():
    x = torch.zeros(2, 8, 4, 64, dtype=torch.bfloat16, device="cuda")
    y = [torch.zeros(2, 16, 2, 64, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    stream = torch.cuda.current_stream().cuda_stream
    ptrs = [[t.data_ptr() for t in y]]
    for rank, S, H, code in ((2, 16, 4, binding.CP_ERR_INVALID_ARG), (0, 15, 4, binding.CP_ERR_NOT_DIVISIBLE),
                             (0, 16, 3, binding.CP_ERR_NOT_DIVISIBLE)):
        with pytest.raises(binding.CpError) as e:
            binding.ulysses_push_n([x.data_ptr()], ptrs, rank, 2, 2, S, H, 64, 0, 2, stream)
        assert e.value.status == code
    with pytest.raises(binding.CpError) as e:  # a destination overlapping the source
        binding.ulysses_push_n([x.data_ptr()], [[x.data_ptr(), y[1].data_ptr()]], 0, 2, 2, 16, 4, 64, 0, 2, stream)
    assert e.value.status == binding.CP_ERR_INVALID_ARG


@pytest.mark.parametrize("P,n,B,S,H,D,dtype", [
    (8, 8, 1, 4608, 24, 128, torch.bfloat16),  # the bench's merge, one rank's head shard at a time
    (2, 3, 2, 100, 4, 64, torch.float32),
    (4, 2, 1, 36, 8, 128, torch.bfloat16),
])
def test_merge_push_equals_fused_merge(P, n, B, S, H, D, dtype):
    """Each rank's merge of its head shard, stored into the ranks' sequence shards, gives
    exactly cp_attn_merge_ulysses's output (bit for bit)."""
    g = torch.Generator().manual_seed(3000 + S)
    Hp = H // P
    parts = torch.randn(n, P * B, S, Hp, D, generator=g).cuda()
    lses = (4 * torch.randn(n, P * B, Hp, S, generator=g)).cuda()
    lses[0, :, :, :3] = -float("inf")  # a block with no keys for some rows
    want, _ = binding.attn_merge_ulysses(parts, lses, P, out_dtype=dtype)
    outs = [torch.full((B, S // P, H, D), float("nan"), dtype=dtype, device="cuda") for _ in range(P)]
    for u in range(P):
        binding.attn_merge_push(parts[:, u * B:(u + 1) * B].contiguous(), lses[:, u * B:(u + 1) * B].contiguous(),
                                [o.data_ptr() for o in outs], u, out_dtype=dtype)
    torch.cuda.synchronize()
    assert torch.equal(torch.stack(outs), want)


def _pads(n):
    return [torch.zeros(binding.CP_PEER_MAX, dtype=torch.int32, device="cuda") for _ in range(n)]


def test_barrier_passes_when_every_rank_signalled():
    stream = torch.cuda.current_stream().cuda_stream
    (pad,) = _pads(1)
    for epoch in (1, 2, 3):  # degree 1: only its own signal
        binding.peer_barrier([pad.data_ptr()], 0, epoch, stream)
    assert binding.last_device_status() == binding.CP_OK
    assert pad[0].item() == 3
    # Degree 4, rank 2; ranks 0, 1, 3 have already signalled rank 2's pad (written here).
    pads = _pads(4)
    pads[2][:4] = torch.tensor([5, 5, 0, 6], dtype=torch.int32)
    binding.peer_barrier([p.data_ptr() for p in pads], 2, 5, stream)
    assert binding.last_device_status() == binding.CP_OK
    for p in pads:  # rank 2's signal reached every pad
        assert p[2].item() == 5
    # Epochs compare modulo 2^32: rank 1 has already signalled epoch 1 (its counter
    # wrapped past 0xFFFFFFFF), so rank 0's wait for 0xFFFFFFFF is over at once.
    pads = _pads(2)
    pads[0][1] = 1
    binding.peer_barrier([p.data_ptr() for p in pads], 0, 0xFFFFFFFF, stream)
    assert binding.last_device_status() == binding.CP_OK
    assert pads[1][0].item() == -1  # 0xFFFFFFFF as int32


def test_barrier_wait_runs_out_and_the_context_stays_usable():
    stream = torch.cuda.current_stream().cuda_stream
    pads = _pads(2)  # rank 1 never signals
    t0 = time.time()
    binding.peer_barrier([p.data_ptr() for p in pads], 0, 1, stream, timeout_ms=300)
    assert binding.last_device_status() == binding.CP_ERR_TIMEOUT
    waited = time.time() - t0
    assert 0.3 <= waited < 30, waited  # the limit is wall-clock time
    assert pads[1][0].item() == 1  # rank 0 still signalled before waiting
    q, k, v = cuda(*qkv(1, 2, 256, 256, 64, seed=3))
    o, _ = binding.attn_fwd(q, k, v)
    assert binding.last_device_status() == binding.CP_OK
    assert torch.isfinite(o.float()).all()


@pytest.mark.parametrize("B,rows,H,D,dst_S,dst_row0,src_S,src_row0,dtype", [
    (2, 1391, 24, 128, 4173, 1391, 1391, 0, torch.bfloat16),  # a ring-anything block into the gathered K
    (1, 0, 4, 64, 10, 3, 10, 2, torch.bfloat16),
    (3, 5, 3, 5, 7, 2, 9, 4, torch.float32),
])
def test_ring_fetch_block_copies_rows(B, rows, H, D, dst_S, dst_row0, src_S, src_row0, dtype):
    g = torch.Generator().manual_seed(rows + dst_S)
    src = torch.randn(B, src_S, H, D, generator=g).to(dtype).cuda()
    dst = torch.zeros(B, dst_S, H, D, dtype=dtype, device="cuda")
    binding.ring_fetch_block(dst.data_ptr(), src.data_ptr(), B, rows, H, D, dst_S, dst_row0, src_S, src_row0,
                             src.element_size(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    want = torch.zeros_like(dst)
    want[:, dst_row0:dst_row0 + rows] = src[:, src_row0:src_row0 + rows]
    assert torch.equal(dst, want)
    with pytest.raises(binding.CpError):
        binding.ring_fetch_block(dst.data_ptr(), src.data_ptr(), B, dst_S + 1, H, D, dst_S, 0, src_S, 0,
                                 src.element_size(), 0)
