"""The host side of one process per GPU, on CPU: the mesh, the ring's block order and
bounds, the handle exchange and the failure detection, with real gloo ranks.

Failures are made on the host (a rank that reports one, a rank that never arrives);
nothing here touches a GPU.
"""

import os
import socket
import time
from datetime import timedelta

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from context_attention_dit_b200 import binding
from context_attention_dit_b200.distributed import (ContextParallel, HealthMonitor, PeerFailure, block_bounds,
                                                    mesh_coord, mesh_groups, ring_order, shard_shapes)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("U,R", [(1, 1), (2, 1), (1, 4), (2, 2), (2, 4), (4, 2), (8, 1), (3, 5)])
def test_mesh_partitions_the_ranks(U, R):
    world = U * R
    coords = [mesh_coord(r, U, R) for r in range(world)]
    ul = {c.ulysses_ranks for c in coords}
    rg = {c.ring_ranks for c in coords}
    # Ulysses groups: R disjoint groups of U consecutive ranks; ring groups: U disjoint
    # groups of R ranks, one from every Ulysses group.
    assert sorted(r for g in ul for r in g) == list(range(world)) and len(ul) == R
    assert sorted(r for g in rg for r in g) == list(range(world)) and len(rg) == U
    for c in coords:
        assert c.ulysses_ranks[c.ulysses_index] == c.rank and c.ring_ranks[c.ring_index] == c.rank
        assert list(c.ulysses_ranks) == list(range(c.ring_index * U, (c.ring_index + 1) * U))
        assert all(mesh_coord(r, U, R).ulysses_index == c.ulysses_index for r in c.ring_ranks)
        assert all(mesh_coord(r, U, R).ring_index == c.ring_index for r in c.ulysses_ranks)
    with pytest.raises(ValueError):
        mesh_coord(world, U, R)


@pytest.mark.parametrize("R", [1, 2, 3, 8])
def test_ring_order_visits_every_block_once_own_first(R):
    for me in range(R):
        order = ring_order(me, R)
        assert order[0] == me and sorted(order) == list(range(R))
        # Step i holds the block that started i ranks back (K/V move from rank j to j+1).
        assert all(order[i] == (me - i) % R for i in range(R))


@pytest.mark.parametrize("S,n", [(4173, 3), (4608, 8), (301, 2), (7, 4), (0, 2)])
def test_block_bounds_of_a_ring_anything_split(S, n):
    want = binding.ring_bounds(S, n, anything=True)
    lengths = [want[i + 1] - want[i] for i in range(n)]
    assert block_bounds(lengths) == want
    with pytest.raises(ValueError):
        block_bounds([3, -1])


def test_constructor_checks_the_mesh_before_any_device_call():
    # One gloo rank, a 2 x 1 mesh: rejected before any CUDA call.
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_mesh_check_worker, args=(_free_port(), q))
    p.start()
    msg = q.get(timeout=120)
    p.join(timeout=60)
    assert p.exitcode == 0 and "ulysses_degree 2 x ring_degree 1 != world 1" in msg


def _mesh_check_worker(port, out):
    import sys

    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        ContextParallel(2, 1)
        out.put("no error")
    except ValueError as e:
        out.put(str(e))
    dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _spawn(fn, world, *args):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=fn, args=(r, world, port, q, *args)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    try:
        for _ in range(world):
            rank, res = q.get(timeout=180)
            out[rank] = res
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    return out, [p.exitcode for p in procs]


def _init(rank, world, port):
    import sys

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))


def _exchange_worker(rank, world, port, out):
    _init(rank, world, port)
    from context_attention_dit_b200.distributed import exchange

    handle = bytes([rank]) * binding.CP_IPC_HANDLE_BYTES  # a stand-in IPC handle
    everyone = exchange(handle)
    c = mesh_coord(rank, 2, world // 2)
    # Ring-anything lengths over the ring sub-group (every rank creates every group).
    groups = [dist.new_group(list(mesh_coord(u, 2, world // 2).ring_ranks)) for u in range(2)]
    lens = exchange(100 + rank, groups[c.ulysses_index])
    out.put((rank, (everyone, lens)))
    dist.barrier()
    dist.destroy_process_group()


def test_handles_and_ring_lengths_are_exchanged_by_rank():
    world = 4
    res, codes = _spawn(_exchange_worker, world)
    assert codes == [0] * world
    for rank, (everyone, lens) in res.items():
        assert everyone == [bytes([r]) * binding.CP_IPC_HANDLE_BYTES for r in range(world)]
        c = mesh_coord(rank, 2, 2)
        assert lens == [100 + r for r in c.ring_ranks]


def _failure_worker(rank, world, port, out, mode):
    _init(rank, world, port)
    mon = HealthMonitor(dist.distributed_c10d._get_default_store(), rank, world, prefix=f"t{mode}", timeout_s=3.0)
    res = None
    if mode == "raises":
        # Rank 1 fails before its step and says so; rank 0 learns it before launching.
        if rank == 1:
            mon.report("out of memory in step 3")
            dist.barrier()
        else:
            dist.barrier()
            try:
                mon.check()
                res = "no failure seen"
            except PeerFailure as e:
                res = (e.ranks, str(e))
    elif mode == "never_arrives":
        # Rank 1 leaves without reaching step 7; rank 0's bounded wait names it.
        if rank == 0:
            t0 = time.time()
            try:
                mon.arrive(7, timeout_s=2.0)
                res = "arrived"
            except PeerFailure as e:
                res = (e.ranks, time.time() - t0)
        out.put((rank, res))
        return  # no collective after a rank has left
    elif mode == "all_arrive":
        mon.arrive(1)
        mon.arrive(2)
        mon.check()
        dist.barrier()
        # Step 1's keys are gone once every rank passed step 2; step 2's stay.
        store = dist.distributed_c10d._get_default_store()
        gone = not any(store.check([f"t{mode}/step/1/{r}"]) for r in range(world))
        kept = all(store.check([f"t{mode}/step/2/{r}"]) for r in range(world))
        res = "ok" if gone and kept else f"keys: step 1 gone {gone}, step 2 kept {kept}"
    out.put((rank, res))
    dist.barrier()
    dist.destroy_process_group()


def test_reported_failure_is_seen_before_the_next_step():
    res, codes = _spawn(_failure_worker, 2, "raises")
    assert codes == [0, 0]
    ranks, msg = res[0]
    assert ranks == [1] and "out of memory in step 3" in msg


def test_rank_that_never_arrives_is_named_within_the_limit():
    res, codes = _spawn(_failure_worker, 2, "never_arrives")
    ranks, waited = res[0]
    assert ranks == [1]
    assert 1.5 <= waited < 30


def test_every_rank_arriving_passes():
    res, codes = _spawn(_failure_worker, 3, "all_arrive")
    assert codes == [0, 0, 0] and all(r == "ok" for r in res.values()), res


def _groups_worker(rank, world, port, out, U, R, sub):
    _init(rank, world, port)
    import torch

    # With `sub`, the mesh lives on the odd ranks only: the even ranks take no part.
    group_ranks = list(range(1, world, 2)) if sub else list(range(world))
    res = None
    if rank in group_ranks:
        group = dist.new_group(group_ranks, use_local_synchronization=True) if sub else None
        me = dist.get_rank(group)
        c = mesh_coord(me, U, R)
        ulysses, ring = mesh_groups(c, group)
        # Sum of the global ranks in each group: shows who is in it.
        su = torch.tensor([rank])
        dist.all_reduce(su, group=ulysses)
        sr = torch.tensor([rank])
        dist.all_reduce(sr, group=ring)
        res = (me, int(su), int(sr))
    out.put((rank, res))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("U,R,world,sub", [(2, 2, 4, False), (4, 1, 4, False), (1, 3, 3, False), (2, 2, 8, True)])
def test_mesh_groups_hold_the_right_ranks(U, R, world, sub):
    res, codes = _spawn(_groups_worker, world, U, R, sub)
    assert codes == [0] * world
    group_ranks = list(range(1, world, 2)) if sub else list(range(world))
    for rank, r in res.items():
        if rank not in group_ranks:
            assert r is None
            continue
        me, su, sr = r
        c = mesh_coord(me, U, R)
        assert su == sum(group_ranks[x] for x in c.ulysses_ranks)
        assert sr == sum(group_ranks[x] for x in c.ring_ranks)


def _shapes_worker(rank, world, port, out, mismatch):
    _init(rank, world, port)
    # Uneven sequence shards are fine; a rank with other heads is an error on every rank.
    H = 8 if not (mismatch and rank == 1) else 6
    try:
        res = shard_shapes((1, 100 + rank, H, 128))
    except ValueError as e:
        res = "error: " + str(e)
    out.put((rank, res))
    dist.barrier()
    dist.destroy_process_group()


def test_shard_shapes_are_shared_and_mismatches_raise_everywhere():
    res, codes = _spawn(_shapes_worker, 3, False)
    assert codes == [0, 0, 0]
    for r in range(3):
        assert res[r] == [(1, 100, 8, 128), (1, 101, 8, 128), (1, 102, 8, 128)]
    res, codes = _spawn(_shapes_worker, 3, True)
    assert codes == [0, 0, 0]
    assert all(isinstance(v, str) and v.startswith("error: ranks disagree") for v in res.values())
