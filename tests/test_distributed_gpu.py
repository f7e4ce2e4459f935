"""ContextParallel with real processes: 2 to 8 ranks, each its own process and CUDA
context, sharing the one GPU of the test box through CUDA IPC.

The peer buffers, the pushes into other processes' memory, the copy-engine fetches and
the host orchestration run exactly as with one GPU per rank.  The barriers are the
host's (stream synchronise + the gloo group's barrier): device-side barriers of ranks
that share one GPU would be kernels waiting on one another, which these tests never
launch.  Every rank's output is compared bit for bit with the single-process path on
the unsplit tensors (``attn_fwd`` for Ulysses alone; otherwise, as each rank computes it,
``attn_fwd`` of every ring block into an fp32 partial and ``attn_merge`` of the partials),
and a small case also with the fp64 oracle.
"""

import os
import socket
import sys
from datetime import timedelta

import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, cfg, out_q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    try:
        torch.cuda.set_device(0)
        dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                                timeout=timedelta(seconds=180))
        from context_attention_dit_b200 import binding
        from context_attention_dit_b200.distributed import ContextParallel
        from context_attention_dit_b200.inputs import make_qkv

        U, R, B, H, D, lens, oracle_check = cfg
        S = sum(lens)
        q, k, v = make_qkv(B, H, S, S, D, seed=11, rms_norm_qk=True)
        s0 = sum(lens[:rank])
        loc = [x[:, s0:s0 + lens[rank]].contiguous().cuda() for x in (q, k, v)]
        cp = ContextParallel(U, R, barrier="host")
        outs = []
        for _ in range(2):  # the second call reuses every buffer
            outs.append(cp.attention(*loc).clone())
        torch.cuda.synchronize()
        status = binding.last_device_status()
        gathered = [None] * world
        dist.all_gather_object(gathered, [o.cpu() for o in outs])
        cp.close()
        result = None
        if rank == 0:
            qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
            if R == 1:
                ref, _ = binding.attn_fwd(qc, kc, vc, want_lse=False)
            else:
                blk = [sum(lens[g * U:(g + 1) * U]) for g in range(R)]
                bounds = [0]
                for n in blk:
                    bounds.append(bounds[-1] + n)
                parts, lses = [], []
                for c in range(R):
                    kb, vb = (x[:, bounds[c]:bounds[c + 1]].contiguous() for x in (kc, vc))
                    o_c, l_c = binding.attn_fwd(qc, kb, vb, out_dtype=torch.float32)
                    parts.append(o_c)
                    lses.append(l_c)
                ref, _ = binding.attn_merge(torch.stack(parts), torch.stack(lses))
            ref = ref.cpu()
            result = {"status": status}
            for it in range(2):
                full = torch.cat([gathered[r][it] for r in range(world)], dim=1)
                result[f"equal{it}"] = bool(torch.equal(full, ref))
                result[f"maxdiff{it}"] = float((full.float() - ref.float()).abs().max())
            if oracle_check:
                import oracle
                from tests.gpu_util import attn_errors

                o_ref, _ = oracle.attention(q, k, v, D ** -0.5)
                full = torch.cat([gathered[r][0] for r in range(world)], dim=1)
                result["oracle_max"], result["oracle_mean"], result["oracle_rel_l2"] = attn_errors(full, o_ref)
        dist.barrier()
        dist.destroy_process_group()
        out_q.put((rank, result, None))
    except Exception as e:  # report, so that the parent fails with the reason
        import traceback

        out_q.put((rank, None, traceback.format_exc()))
        raise


def _run(U, R, B, H, D, lens, oracle_check=False):
    world = U * R
    assert len(lens) == world
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, (U, R, B, H, D, lens, oracle_check), q))
             for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    try:
        for _ in range(world):
            rank, res, err = q.get(timeout=600)
            assert err is None, f"rank {rank} failed:\n{err}"
            results[rank] = res
    finally:
        for p in procs:
            p.join(timeout=120)
            if p.is_alive():
                p.kill()
    for p in procs:
        assert p.exitcode == 0
    return results[0]


@pytest.mark.parametrize(
    "U,R,B,H,D,lens,oracle_check",
    [
        (2, 1, 1, 4, 128, [512, 512], True),  # Ulysses
        (3, 1, 1, 5, 128, [101, 100, 99], True),  # Ulysses anything: uneven tokens, 5 heads over 3
        (3, 1, 2, 2, 64, [64, 64, 63], False),  # Ulysses anything with an empty head shard
        (2, 1, 1, 24, 128, [2304, 2304], False),  # Ulysses on the FLUX-like shape
        (1, 2, 2, 3, 128, [301, 300], True),  # ring anything: uneven blocks
        (1, 3, 1, 2, 64, [384, 384, 384], False),  # ring of three
        (2, 2, 1, 4, 64, [256, 256, 256, 256], True),  # unified: 2 x 2 mesh
        (8, 1, 1, 24, 128, [576] * 8, False),  # Ulysses-8 on the FLUX-like shape: eight processes
        (4, 2, 1, 8, 128, [128] * 8, True),  # unified 4 x 2
        (2, 4, 1, 4, 64, [96] * 8, True),  # unified 2 x 4
        (4, 2, 1, 24, 128, [576] * 8, True),  # unified 4 x 2 on the FLUX-like shape
        (2, 4, 1, 24, 128, [576] * 8, True),  # unified 2 x 4 on the FLUX-like shape
    ],
)
def test_context_parallel_matches_single_process(U, R, B, H, D, lens, oracle_check):
    from tests.gpu_util import O_MAX_ABS, O_MEAN_ABS, O_REL_L2

    res = _run(U, R, B, H, D, lens, oracle_check)
    assert res["status"] == 0
    for it in range(2):
        assert res[f"equal{it}"], f"call {it}: max diff {res[f'maxdiff{it}']:.3e} from the single-process result"
    if oracle_check:
        assert res["oracle_max"] <= O_MAX_ABS and res["oracle_mean"] <= O_MEAN_ABS, res
        assert res["oracle_rel_l2"] <= O_REL_L2, res
