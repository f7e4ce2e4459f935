"""Context parallelism with one process per GPU: Ulysses, ring and unified attention
between real GPUs.

"Context parallelism", sections "Ring Attention", "Ulysses Attention", "Unified
Attention" and "Ring Anything Attention"; "Parallelism", ``ContextParallelConfig``
(``ulysses_degree``, ``ring_degree``, a device mesh with a "ring" and a "ulysses"
dimension).  Every rank holds one sequence shard of Q, K and V, ``[B, S_local, H, D]``
bf16, and gets back the attention output of its own tokens over the whole sequence.

Data moves through this package's library only:

* the Ulysses all-to-alls are ``cp_ulysses_push_n`` kernels that store each rank's pieces
  straight into the owning ranks' buffers (peer memory mapped with CUDA IPC);
* a ring rank fetches the other ring ranks' K/V blocks with ``cp_ring_fetch_block`` (the
  copy engines, on a side stream, one event per block), and attends each block as soon as
  it has landed: its own block first, while the others are still in flight;
* the blocks' fp32 partials are merged by their LSEs (``cp_attn_merge``); in unified
  attention the merge stores each row straight into its owner's sequence shard
  (``cp_attn_merge_push``: the merge and the second all-to-all in one kernel);
* ``cp_peer_barrier`` orders the steps, with a bounded device-side wait.

``torch.distributed`` (NCCL on GPUs, gloo in the CPU tests) carries the plumbing only: the
IPC handles, the block lengths of a ring-anything split and the health checks.  Nothing
here computes attention on the host, and there is no fallback: without the library every
call raises.

Mesh (a reading: the pages name the two mesh dimensions but not the rank order): rank =
ring_index * ulysses_degree + ulysses_index, so a Ulysses group is ``ulysses_degree``
consecutive ranks and a ring group takes one rank of every Ulysses group.  The sequence is
split over all ranks in rank order; after the Ulysses exchange, Ulysses group g holds
ring block g (its ranks' shards, concatenated) for H/ulysses_degree heads per rank.
"""

from __future__ import annotations

import datetime
from dataclasses import dataclass
from typing import Dict, List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

from . import binding

_PAD_WORDS = binding.CP_PEER_MAX  # signal words per barrier group
_GROUPS = ("world", "ulysses", "ring")
_PAD_BYTES = 256
assert len(_GROUPS) * _PAD_WORDS * 4 <= _PAD_BYTES


# ------------------------------------------------------------------ host-only plan


@dataclass(frozen=True)
class MeshCoord:
    rank: int
    ulysses_index: int
    ring_index: int
    ulysses_ranks: Tuple[int, ...]  # the Ulysses group, by Ulysses index
    ring_ranks: Tuple[int, ...]     # the ring group, by ring index


def mesh_coord(rank: int, ulysses_degree: int, ring_degree: int) -> MeshCoord:
    """Position of ``rank`` in the ``ring_degree x ulysses_degree`` mesh."""
    U, R = int(ulysses_degree), int(ring_degree)
    if U < 1 or R < 1 or not 0 <= rank < U * R:
        raise ValueError(f"rank {rank} outside a {R} x {U} mesh")
    u, g = rank % U, rank // U
    return MeshCoord(rank, u, g, tuple(g * U + j for j in range(U)), tuple(c * U + u for c in range(R)))


def mesh_groups(coord: MeshCoord, group=None):
    """This rank's Ulysses and ring process groups (for host barriers and exchanges).

    Only the members of a group create it (``use_local_synchronization``), so every rank
    makes two calls, and a group of some of the world's ranks works as well as the world.
    """
    ranks = dist.get_process_group_ranks(group) if group is not None else list(range(dist.get_world_size()))
    ulysses = dist.new_group([ranks[r] for r in coord.ulysses_ranks], use_local_synchronization=True)
    ring = dist.new_group([ranks[r] for r in coord.ring_ranks], use_local_synchronization=True)
    return ulysses, ring


def ring_order(ring_index: int, ring_degree: int) -> List[int]:
    """Blocks in the order a ring rank sees them: its own, then the block of the rank
    before it, and so on (K/V pass from rank i to rank i+1, "Ring Attention")."""
    return [(ring_index - i) % ring_degree for i in range(ring_degree)]


def block_bounds(lengths: Sequence[int]) -> List[int]:
    """Row bounds of blocks of the given lengths, concatenated in rank order."""
    out = [0]
    for n in lengths:
        if n < 0:
            raise ValueError("negative block length")
        out.append(out[-1] + int(n))
    return out


def exchange(obj, group=None) -> list:
    """Every rank's ``obj``, by rank within ``group`` (host plumbing only)."""
    out = [None] * dist.get_world_size(group)
    dist.all_gather_object(out, obj, group=group)
    return out


def shard_shapes(shape, group=None) -> List[Tuple[int, int, int, int]]:
    """Every rank's (B, S_local, H, D) shard shape, by rank (a host exchange).  Every rank
    gets the same list, so a mismatch in batch, heads or head_dim raises on all ranks
    alike, before anyone launches an exchange that could not complete."""
    shapes = [tuple(int(x) for x in t) for t in exchange(tuple(int(x) for x in shape), group)]
    if any(len(t) != 4 for t in shapes) or len({(b, h, d) for b, _, h, d in shapes}) != 1:
        raise ValueError(f"ranks disagree on batch, heads or head_dim: {shapes}")
    return shapes


# ------------------------------------------------------------------ failure detection


class PeerFailure(RuntimeError):
    """Another rank reported a failure, or did not reach a step in time."""

    def __init__(self, ranks, what: str):
        self.ranks = sorted(ranks)
        super().__init__(f"rank(s) {self.ranks}: {what}")


class HealthMonitor:
    """Host-side failure detection through the process group's key-value store.

    A rank that fails calls :meth:`report`; the others see it in :meth:`check`, which
    the attention calls run before their first launch, so that no rank starts a step
    whose exchanges a dead peer would never complete.  :meth:`arrive` waits, bounded, for
    every rank to reach a step, and names the ranks that did not.
    """

    def __init__(self, store, rank: int, world: int, prefix: str = "cp", timeout_s: float = 30.0):
        self.store, self.rank, self.world = store, rank, world
        self.prefix, self.timeout = prefix, datetime.timedelta(seconds=timeout_s)

    def _key(self, kind: str, *parts) -> str:
        return "/".join([self.prefix, kind, *map(str, parts)])

    def report(self, reason: str):
        self.store.set(self._key("failed", self.rank), reason)

    def failed(self) -> Dict[int, str]:
        out = {}
        for r in range(self.world):
            k = self._key("failed", r)
            if self.store.check([k]):
                out[r] = self.store.get(k).decode(errors="replace")
        return out

    def check(self):
        bad = self.failed()
        if bad:
            raise PeerFailure(bad, "reported failure: " + "; ".join(f"{r}: {m}" for r, m in sorted(bad.items())))

    def arrive(self, step: int, timeout_s: Optional[float] = None):
        self.store.set(self._key("step", step, self.rank), "1")
        keys = [self._key("step", step, r) for r in range(self.world)]
        limit = self.timeout if timeout_s is None else datetime.timedelta(seconds=timeout_s)
        try:
            self.store.wait(keys, limit)
        except Exception as e:  # the store raises on timeout; name who is missing
            missing = [r for r, k in enumerate(keys) if not self.store.check([k])]
            self.check()
            raise PeerFailure(missing, f"did not reach step {step} within {limit.total_seconds()} s") from e
        # Every rank has set its key of this step, so every rank is done waiting on the
        # previous one: this rank's key of that step can go (the store stays small).
        try:
            self.store.delete_key(self._key("step", step - 1, self.rank))
        except Exception:
            pass


# ------------------------------------------------------------------ peer buffers


class _PeerBuffer:
    """One peer-visible allocation per rank: ``ptrs[q]`` is rank q's, mapped here."""

    def __init__(self, nbytes: int, rank: int, group):
        self.nbytes, self.rank = int(nbytes), rank
        self.local, handle = binding.peer_alloc(self.nbytes)
        self.ptrs: List[int] = []
        self._opened: List[int] = []
        try:
            handles = exchange(handle, group)
            for q, h in enumerate(handles):
                if q == rank:
                    self.ptrs.append(self.local)
                else:
                    p = binding.peer_open(h)
                    self._opened.append(p)
                    self.ptrs.append(p)
        except Exception:
            self.close_mappings()
            self.free()
            raise

    def close_mappings(self):
        for p in self._opened:
            binding.peer_close(p)
        self._opened = []

    def free(self):
        if self.local:
            binding.peer_free(self.local)
            self.local = 0


class ContextParallel:
    """Ulysses x ring attention over the ranks of a process group, one GPU per rank.

    Every rank calls the constructor and every method in the same order (the buffers are
    allocated collectively), with its own GPU already current (``torch.cuda.set_device``).  ``barrier="device"`` orders steps with ``cp_peer_barrier``
    (stream-ordered, no host sync), whose wait gives up after ``barrier_timeout_ms``: ranks
    are driven by their hosts, so the limit must cover the host-side skew between ranks.
    A barrier that gave up leaves the step's outputs undefined; :meth:`check_device`
    reports it.  ``barrier="host"`` synchronises the stream and calls the process group's
    barrier instead.
    """

    def __init__(self, ulysses_degree: int = 1, ring_degree: int = 1, group=None, barrier: str = "device",
                 monitor: Optional[HealthMonitor] = None, barrier_timeout_ms: int = 30000):
        if barrier not in ("device", "host"):
            raise ValueError("barrier must be 'device' or 'host'")
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if ulysses_degree * ring_degree != self.world:
            raise ValueError(f"ulysses_degree {ulysses_degree} x ring_degree {ring_degree} != world {self.world}")
        if max(ulysses_degree, ring_degree) > binding.CP_PEER_MAX:
            raise ValueError(f"a group holds at most {binding.CP_PEER_MAX} ranks")
        self.U, self.R = int(ulysses_degree), int(ring_degree)
        self.coord = mesh_coord(self.rank, self.U, self.R)
        self.barrier_mode = barrier
        self.barrier_timeout_ms = int(barrier_timeout_ms)
        self.monitor = monitor
        self.device = torch.device("cuda", torch.cuda.current_device())
        ulysses, ring = mesh_groups(self.coord, group)
        self._pg = {"world": group, "ulysses": ulysses, "ring": ring}
        self._epoch = {g: 0 for g in _GROUPS}
        self._pads = _PeerBuffer(_PAD_BYTES, self.rank, group)
        self._bufs: Dict[str, _PeerBuffer] = {}
        self._copy_stream = torch.cuda.Stream(self.device)

    # -- plumbing

    def _members(self, name: str) -> Tuple[int, ...]:
        return {"world": tuple(range(self.world)), "ulysses": self.coord.ulysses_ranks,
                "ring": self.coord.ring_ranks}[name]

    def barrier(self, name: str = "world", stream: Optional[torch.cuda.Stream] = None):
        """All ranks of group ``name`` reach this point of their streams."""
        s = torch.cuda.current_stream(self.device) if stream is None else stream
        members = self._members(name)
        if len(members) == 1:
            return
        if self.barrier_mode == "host":
            s.synchronize()
            dist.barrier(group=self._pg[name])
            return
        self._epoch[name] += 1
        off = _GROUPS.index(name) * _PAD_WORDS * 4
        pads = [self._pads.ptrs[r] + off for r in members]
        binding.peer_barrier(pads, members.index(self.rank), self._epoch[name], s.cuda_stream,
                             self.barrier_timeout_ms)

    def _retire(self, bufs: Sequence[_PeerBuffer]):
        """Free peer buffers: every rank stops using them, unmaps the others', then frees
        its own (host barriers: this is not on the step's path)."""
        torch.cuda.current_stream(self.device).synchronize()
        self._copy_stream.synchronize()
        dist.barrier(group=self.group)
        for b in bufs:
            b.close_mappings()
        dist.barrier(group=self.group)
        for b in bufs:
            b.free()

    def _buffer(self, name: str, nbytes: int) -> _PeerBuffer:
        """Peer buffer ``name`` of at least ``nbytes`` (the same on every rank)."""
        b = self._bufs.get(name)
        if b is None or b.nbytes < nbytes:
            if b is not None:
                self._retire([b])
            b = _PeerBuffer(max(int(nbytes), 256), self.rank, self.group)
            self._bufs[name] = b
        return b

    def _view(self, ptr: int, shape) -> torch.Tensor:
        return binding.device_tensor(ptr, shape, torch.bfloat16, self.device)

    def check_health(self):
        if self.monitor is not None:
            self.monitor.check()

    def check_device(self):
        """Wait for the stream and raise if a device-side barrier wait ran out since the
        last check (the group is then to be treated as failed)."""
        st = binding.last_device_status()
        if st != binding.CP_OK:
            if self.monitor is not None:
                self.monitor.report(binding.status_string(st))
            raise binding.CpError(st, "ContextParallel")

    def close(self):
        """Free the peer buffers (collective: every rank calls it)."""
        self._retire(list(self._bufs.values()) + [self._pads])
        self._bufs = {}

    # -- the step

    def shard_shapes(self, q) -> List[Tuple[int, int, int, int]]:
        """Every rank's (B, S_local, H, D), by rank (see :func:`shard_shapes`)."""
        return shard_shapes(tuple(q.shape), self.group)

    def attention(self, q, k, v, scale: Optional[float] = None,
                  seq_lengths: Optional[Sequence[int]] = None) -> torch.Tensor:
        """Attention of this rank's tokens over the whole sequence.

        q, k, v: this rank's sequence shard ``[B, S_local, H, D]``, contiguous bf16 on the
        current device; the shards follow rank order along the sequence.  seq_lengths:
        every rank's S_local, by rank; given, it saves a host exchange per call.  Returns
        ``[B, S_local, H, D]`` bf16; with ulysses_degree > 1 the result lives in a peer
        buffer that the next call overwrites (copy it to keep it).

        Uneven shards follow the pages' variants table: with ring_degree 1 they are
        "Ulysses Anything Attention" (S_local and H need not divide), with ulysses_degree 1
        "Ring Anything Attention"; unified attention needs equal shards and H divisible by
        ulysses_degree.
        """
        binding._check_qkv(q, k, v)
        if q.shape != k.shape:
            raise ValueError("query and key shards must have one shape")
        B, Sl, H, D = q.shape
        U, R = self.U, self.R
        scale = float(D ** -0.5 if scale is None else scale)
        if seq_lengths is None:
            lengths = [s[1] for s in self.shard_shapes(q)]
        else:
            lengths = [int(x) for x in seq_lengths]
        if len(lengths) != self.world or lengths[self.rank] != Sl:
            raise ValueError(f"seq_lengths {lengths} do not hold this rank's {Sl} tokens at {self.rank}")
        even = len(set(lengths)) == 1 and H % U == 0
        if U > 1 and R > 1 and not even:
            raise ValueError("unified attention needs equal shards and heads divisible by ulysses_degree")
        self.check_health()
        s = torch.cuda.current_stream(self.device)
        es = q.element_size()
        self.barrier("world")  # every rank is done with the previous step's buffers
        if U > 1 and not even:
            return self._ulysses_anything(q, k, v, lengths, scale)
        if U > 1:
            S_blk, Hh = Sl * U, H // U
            blk = B * S_blk * Hh * D * es
            bufs = [self._buffer(n, blk) for n in ("yq", "yk", "yv")]
            binding.ulysses_push_n([q.data_ptr(), k.data_ptr(), v.data_ptr()],
                                   [[b.ptrs[r] for r in self.coord.ulysses_ranks] for b in bufs],
                                   self.coord.ulysses_index, U, B, S_blk, H, D, 0, es, s.cuda_stream)
            self.barrier("ulysses")
            qh, kh, vh = (self._view(b.local, (B, S_blk, Hh, D)) for b in bufs)
            kv_bufs = bufs[1:]
            ring = [S_blk] * R
        else:
            qh, kh, vh = q, k, v
            kv_bufs = None
            ring = lengths  # U == 1: the ring group is the whole group, in rank order
        if R > 1:
            if kv_bufs is None:  # K/V into this rank's peer-visible buffers (sized alike on every rank)
                kv_bufs = [self._buffer(n, B * max(ring) * H * D * es) for n in ("rk", "rv")]
                for src, b in ((k, kv_bufs[0]), (v, kv_bufs[1])):
                    binding.ring_fetch_block(b.local, src.data_ptr(), B, Sl, H, D, Sl, 0, Sl, 0, es, s.cuda_stream)
            self.barrier("ring")  # every ring rank's K/V block is in place
            partials, lses = self._ring(qh, kh, vh, kv_bufs, ring, scale)
            if U == 1:
                return binding.attn_merge(partials, lses)[0]
            # Unified: the merge stores every row straight into its owner's sequence shard
            # (the second all-to-all fused into the merge).
            out = self._buffer("xo", B * Sl * H * D * es)
            binding.attn_merge_push(partials, lses, [out.ptrs[r] for r in self.coord.ulysses_ranks],
                                    self.coord.ulysses_index)
            self.barrier("ulysses")
            return self._view(out.local, (B, Sl, H, D))
        oh, _ = binding.attn_fwd(qh, kh, vh, scale=scale, want_lse=False)
        if U == 1:
            return oh
        out = self._buffer("xo", B * Sl * H * D * es)
        binding.ulysses_push_n([oh.data_ptr()], [[out.ptrs[r] for r in self.coord.ulysses_ranks]],
                               self.coord.ulysses_index, U, B, Sl * U, H, D, 1, es, s.cuda_stream)
        self.barrier("ulysses")
        return self._view(out.local, (B, Sl, H, D))

    def _ulysses_anything(self, q, k, v, lengths: List[int], scale: float) -> torch.Tensor:
        """Ulysses with uneven sequence and head shards (ring_degree 1): sequence shards in
        rank order, head shards as even as possible with the first ones larger."""
        B, Sl, H, D = q.shape
        U, me = self.U, self.rank
        es = q.element_size()
        s = torch.cuda.current_stream(self.device)
        sb = block_bounds(lengths)
        hb = binding.ring_bounds(H, U, anything=True)
        S, Hr = sb[-1], hb[me + 1] - hb[me]
        max_h = max(hb[i + 1] - hb[i] for i in range(U))
        bufs = [self._buffer(n, B * S * max_h * D * es) for n in ("yq", "yk", "yv")]
        binding.ulysses_anything_push_n([q.data_ptr(), k.data_ptr(), v.data_ptr()], [b.ptrs for b in bufs], me, sb,
                                        hb, B, H, D, 0, es, s.cuda_stream)
        self.barrier("ulysses")
        qh, kh, vh = (self._view(b.local, (B, S, Hr, D)) for b in bufs)
        oh, _ = binding.attn_fwd(qh, kh, vh, scale=scale, want_lse=False)
        out = self._buffer("xo", B * max(lengths) * H * D * es)
        binding.ulysses_anything_push_n([oh.data_ptr()], [out.ptrs], me, sb, hb, B, H, D, 1, es, s.cuda_stream)
        self.barrier("ulysses")
        return self._view(out.local, (B, Sl, H, D))

    def _ring(self, qh, kh, vh, kv_bufs, lengths: List[int], scale: float):
        """Ring attention of the local queries over every ring rank's K/V block: returns
        the blocks' fp32 partials and LSEs, in block order."""
        B, Sq, Hh, D = qh.shape
        R, me = self.R, self.coord.ring_index
        es = qh.element_size()
        s = torch.cuda.current_stream(self.device)
        cs = self._copy_stream
        # Landing buffers: block c as a contiguous [B, len_c, Hh, D] tensor.
        offs = block_bounds([B * n * Hh * D for n in lengths])
        land_k = torch.empty(offs[-1], dtype=qh.dtype, device=self.device)
        land_v = torch.empty(offs[-1], dtype=qh.dtype, device=self.device)
        partials = torch.empty((R, B, Sq, Hh, D), dtype=torch.float32, device=self.device)
        lses = torch.empty((R, B, Hh, Sq), dtype=torch.float32, device=self.device)
        start = torch.cuda.Event()
        start.record(s)
        cs.wait_event(start)
        landed = {}
        for c in ring_order(me, R)[1:]:
            n, peer = lengths[c], self.coord.ring_ranks[c]
            for b, land in ((kv_bufs[0], land_k), (kv_bufs[1], land_v)):
                binding.ring_fetch_block(land.data_ptr() + offs[c] * es, b.ptrs[peer], B, n, Hh, D, n, 0, n, 0, es,
                                         cs.cuda_stream)
            ev = torch.cuda.Event()
            ev.record(cs)
            landed[c] = ev
        land_k.record_stream(cs)
        land_v.record_stream(cs)
        for c in ring_order(me, R):
            n = lengths[c]
            if c == me:
                kc, vc = kh, vh
            else:
                s.wait_event(landed[c])
                kc = land_k[offs[c]: offs[c + 1]].view(B, n, Hh, D)
                vc = land_v[offs[c]: offs[c + 1]].view(B, n, Hh, D)
            binding.attn_fwd(qh, kc, vc, scale=scale, out_dtype=torch.float32, out=partials[c], lse=lses[c])
        return partials, lses
