"""A deterministic set of calls touching every kernel path (ragged shapes, empty blocks and
shards, both output types), used by tests/test_debug_bounds_gpu.py to run the same work
through the release and the bounds-checking debug library.  Prints one JSON object:
call name -> SHA-256 of its outputs, plus the device status after every call."""

import hashlib
import json
import sys

import torch

from context_attention_dit_b200 import binding
from context_attention_dit_b200.inputs import make_qkv


def _digest(*ts):
    h = hashlib.sha256()
    for t in ts:
        h.update(t.detach().contiguous().view(torch.uint8).cpu().numpy().tobytes())
    return h.hexdigest()[:24]


def run():
    torch.cuda.set_device(0)
    out = {}

    def record(name, *ts):
        torch.cuda.synchronize()
        out[name] = {"status": binding.last_device_status(), "digest": _digest(*ts)}

    for B, H, Sq, Skv, D, dt in ((1, 2, 1, 1, 128, torch.bfloat16), (2, 3, 129, 300, 128, torch.float32),
                                 (1, 2, 300, 77, 64, torch.bfloat16), (1, 4, 1391, 1391, 128, torch.bfloat16)):
        q, k, v = (t.cuda() for t in make_qkv(B, H, Sq, Skv, D, seed=3))
        record(f"attn_{B}x{H}x{Sq}x{Skv}x{D}", *binding.attn_fwd(q, k, v, out_dtype=dt))
    q, k, v = (t.cuda() for t in make_qkv(1, 2, 450, 450, 128, seed=4))
    for bounds in ([0, 0, 130, 130, 450], [0, 5, 6, 450], [0, 450, 450]):
        o, lse, _ = binding.ring_sim(q, k, v, bounds)
        record(f"ring_{bounds}", o, lse)
        record(f"ring_fused_{bounds}", *binding.ring_sim_fused(q, k, v, bounds, out_dtype=torch.float32))
    # The allocation-free ring on a shape whose partials and LSEs nearly fill the static
    # array (2 blocks x 4 heads x 8128 rows: 33,552,384 of 33,554,432 bytes).
    qs, ks, vs = (t.cuda() for t in make_qkv(1, 4, 8128, 300, 128, seed=10))
    assert binding.ring_workspace_size(2, 1, 4, 8128, 128) > binding.STATIC_SCRATCH_BYTES - 4096
    record("ring_static_near_limit", *binding.ring_sim_static(qs, ks, vs, [0, 150, 300]))
    # Views: a K/V block inside a longer sequence, an output written into a larger tensor,
    # and the fused ring writing the Ulysses token-sharded layout.
    qv, kv_full, vv_full = (t.cuda() for t in make_qkv(2, 3, 200, 700, 128, seed=11))
    big = torch.zeros(2, 210, 3, 128, dtype=torch.bfloat16, device="cuda")
    binding.attn_fwd_strided(qv, kv_full[:, 123:600], vv_full[:, 123:600], out=big[:, 5:205])
    record("attn_strided", big)
    Pu, Bu, Su, Hu = 2, 2, 256, 4
    xs = [t.reshape(Bu, Pu, Su // Pu, Hu, 64).permute(1, 0, 2, 3, 4).contiguous().cuda()
          for t in make_qkv(Bu, Hu, Su, Su, 64, seed=12)]
    heads = binding.ulysses_permute_n(xs, Pu, 0)
    record("fused_ulysses", *binding.ring_sim_fused_ulysses(*heads, Pu, [0, 100, 101, 256]))
    # The Ring Anything gather with an empty block and padding.
    gk = binding.ring_anything_gather([kv_full.contiguous()], [0, 0, 301, 700], 410)
    record("gather", *gk)
    P, B, S, H, D = 4, 2, 384, 8, 128
    x = [t.cuda() for t in make_qkv(P * B, H // P, S, S, D, seed=5)]
    parts, lses = binding.attn_fwd_blocks(*x, [0, 100, 101, 384])
    record("blocks", parts, lses)
    record("merge", *binding.attn_merge(parts, lses))
    record("merge_ulysses", *binding.attn_merge_ulysses(parts, lses, P))
    src = torch.randn(P, B, S // P, H, D, generator=torch.Generator().manual_seed(6)).bfloat16().cuda()
    y = binding.ulysses_permute(src, P, 0)
    record("permute", y, binding.ulysses_permute(y, P, 1))
    record("permute_n", *binding.ulysses_permute_n([src, src.clone()], P, 0))
    for Pa, Sa, Ha, Da, sb, hb in ((4, 10, 3, 64, [0, 3, 6, 8, 10], [0, 1, 2, 3, 3]),
                                   (3, 9, 6, 5, [0, 0, 4, 9], [0, 2, 4, 6])):
        xa = torch.randn(2 * Sa * Ha * Da, generator=torch.Generator().manual_seed(7)).bfloat16().cuda()
        ya = binding.ulysses_anything_permute(xa, Pa, sb, hb, 2, Sa, Ha, Da, 0)
        record(f"anything_{Pa}_{Sa}_{Ha}_{Da}", ya, binding.ulysses_anything_permute(ya, Pa, sb, hb, 2, Sa, Ha, Da, 1))
    yn = binding.ulysses_anything_permute_n([xa, xa.clone()], Pa, sb, hb, 2, Sa, Ha, Da, 0)
    record("anything_n", *yn)
    # One process per GPU, the ranks taken in turn with local buffers for their peers'.
    st = torch.cuda.current_stream().cuda_stream
    ys = [torch.zeros(B, S, H // P, D, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    for r in range(P):
        binding.ulysses_push_n([src[r].data_ptr()], [[t.data_ptr() for t in ys]], r, P, B, S, H, D, 0, 2, st)
    xb = [torch.zeros(B, S // P, H, D, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    for r in range(P):
        binding.ulysses_push_n([ys[r].data_ptr()], [[t.data_ptr() for t in xb]], r, P, B, S, H, D, 1, 2, st)
    record("push", *ys, *xb)
    outs = [torch.zeros(B, S // P, H, D, dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    for u in range(P):
        binding.attn_merge_push(parts[:, u * B:(u + 1) * B].contiguous(), lses[:, u * B:(u + 1) * B].contiguous(),
                                [o.data_ptr() for o in outs], u)
    record("merge_push", *outs)
    xf = torch.randn(2, Sa, Ha, Da, generator=torch.Generator().manual_seed(9)).bfloat16().cuda()
    xs = [xf[:, sb[p]:sb[p + 1]].contiguous() for p in range(Pa)]
    ya = [torch.zeros(2, Sa, hb[q + 1] - hb[q], Da, dtype=torch.bfloat16, device="cuda") for q in range(Pa)]
    xr = [torch.zeros(2, sb[p + 1] - sb[p], Ha, Da, dtype=torch.bfloat16, device="cuda") for p in range(Pa)]
    ptr = lambda t: t.data_ptr() if t.numel() else 16  # noqa: E731  (an empty shard is never touched)
    for r in range(Pa):
        binding.ulysses_anything_push_n([ptr(xs[r])], [[ptr(t) for t in ya]], r, sb, hb, 2, Ha, Da, 0, 2, st)
    for r in range(Pa):
        binding.ulysses_anything_push_n([ptr(ya[r])], [[ptr(t) for t in xr]], r, sb, hb, 2, Ha, Da, 1, 2, st)
    record("anything_push", *ya, *xr)
    pad = torch.zeros(16, dtype=torch.int32, device="cuda")
    binding.peer_barrier([pad.data_ptr()], 0, 1, st)
    record("barrier", pad)
    shards = [t.reshape(1, 2, 128, 4, 128).permute(1, 0, 2, 3, 4).contiguous().cuda()
              for t in make_qkv(1, 4, 256, 256, 128, seed=8)]
    o, lse, _ = binding.usp_sim(*shards, 2, [0, 100, 256])
    record("usp", o, lse)
    return out


if __name__ == "__main__":
    print(json.dumps(run()))
    sys.stdout.flush()
