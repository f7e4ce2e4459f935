"""Benchmark of the context-parallel attention hot path on B200.

One step = the whole hot path on the FLUX.1-dev 1024x1024 joint-attention shape
(B=1, H=24, S=4608, D=128, bf16, QK-normed synthetic inputs), in two launches:
  1. Ulysses degree-8 exchange of Q, K and V (sequence-sharded -> head-sharded),
  2. ring attention over 8 K/V blocks of 576 keys on the head-sharded tensors, each
     block merged into the running output by LSE rescaling in TMEM (the ring's merge,
     pairwise in ring order), each finished row stored to its sequence-sharded place
     (the inverse Ulysses exchange of O).
The same path in three launches (blockwise attention writing every block's fp32
partial and LSE to HBM, then the LSE merge kernel fused with the inverse exchange) is
timed beside it and reported under "kernels".
Metric: attention TFLOP/s = 4*B*H*S*S*D per step / step time (device time, CUDA
events, L2 flushed between steps).  Also reported: the dominant kernel's roofline,
the single-block (ring-1) attention kernel, merge and permute GB/s, the fp64 CPU
oracle as a baseline, and an end-to-end number through host buffers.

--impl reference times the fp64 CPU oracle (the only reference this project has)
on a bounded sample of the same workload.  Multi-GPU (torchrun): every rank runs an
independent replica (the single-GPU path has no data exchange between GPUs).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "flux_1024_ring8_ulysses8"
METRIC = "attention TFLOP/s (4*B*H*Sq*Skv*D) and % of B200 BF16 peak; merge/permute GB/s"
UNIT = "TFLOP/s"
STEP_WORKLOAD = ("FLUX.1-dev 1024x1024 joint attention B1 H24 S4608 D128: Ulysses-8 exchange of Q/K/V, "
                 "ring-8 blockwise attention (8 x 576 keys) merged by LSE, inverse exchange of O")


def step_config(world: int, B: int, S: int, H: int, D: int, P: int, n_blocks: int, l2: str) -> dict:
    """The workload description shared by both arms of the bench (same keys, same workload)."""
    return {"workload": STEP_WORKLOAD, "global_batch": world * B, "seq_len": S, "heads": H, "head_dim": D,
            "ulysses_degree": P, "ring_degree": n_blocks,
            "parallelism": f"replicas x{world} (single-GPU simulated degrees)", "l2": l2}

# DRAM traffic of the timed attention launch (the fused ring over 8 blocks with the Ulysses
# output map, FLUX B1), from one ncu capture of the same kernel on the B2 shape
# (profiles/attn_fwd_sm100__flux_b2_ring8_fused_ulysses.md):
# dram__bytes_read.sum + dram__bytes_write.sum = 169.96 + 43.90 MB, halved to one B1 launch
# (the B1 launch processes half the units; Q/K/V reads and output writes scale with them).
# It describes only the kernel source it was captured on, identified by its SHA-256.
ATTN_TRAFFIC = {
    "kernel_sha256": "96aa2b09ae7037d97cfbd2edf9061b75e74a772e14ff93a248fb5e517b36cdf5",
    "bytes_per_launch": (169_955_072 + 43_901_952) // 2,
}


def attn_traffic():
    """Measured DRAM bytes per attention launch, or None if the kernel changed since."""
    import hashlib

    src = os.path.join(os.path.dirname(os.path.abspath(__file__)), "context_attention_dit_b200", "csrc",
                       "attn_fwd_sm100.cuh")
    with open(src, "rb") as f:
        digest = hashlib.sha256(f.read()).hexdigest()
    return ATTN_TRAFFIC["bytes_per_launch"] if digest == ATTN_TRAFFIC["kernel_sha256"] else None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks + throttle reasons sampled every 100 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
            return
        threading.Thread(target=self._read, daemon=True).start()
        time.sleep(0.8)  # nvidia-smi start-up

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        if self.proc:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = [s for t, s in self.samples if self.t0 and self.t1 and self.t0 - 0.15 <= t <= self.t1 + 0.15]
        if not rows:
            rows = [s for _, s in self.samples]
        mhz, maxmhz, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            parts = [p.strip() for p in r.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz.append(float(parts[1]))
                maxmhz = float(parts[2])
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": maxmhz,
                "reasons": sorted(reasons), "samples": len(mhz)}


def reduce_max(value: float, device) -> float:
    """Maximum of `value` over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, flop_per_step: float, total_ms: float, steps: int) -> float:
    """Whole-job TFLOP/s: every rank runs `steps` steps of `flop_per_step`; time = slowest rank."""
    return world * flop_per_step / (total_ms / steps * 1e-3) / 1e12


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# --------------------------------------------------------------------------- our arm


def run_ours(args):
    import datetime

    import torch
    import torch.distributed as dist

    from context_attention_dit_b200 import binding
    from context_attention_dit_b200.inputs import WORKLOADS, bounds_from_sizes, even_bounds, sha256

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    w = WORKLOADS[WORKLOAD]
    P, B, S, H, D = w.ulysses_degree, w.B, w.S, w.H, w.D
    n_blocks = len(w.splits[0])
    q_h, k_h, v_h = w.qkv()
    sha = {n: sha256(t)[:16] for n, t in zip("qkv", (q_h, k_h, v_h))}

    def seq_shards(x):
        return x.reshape(B, P, S // P, H, D).permute(1, 0, 2, 3, 4).contiguous()

    xq, xk, xv = (seq_shards(t).to(dev) for t in (q_h, k_h, v_h))  # sequence-sharded inputs
    Bp, Hp = P * B, H // P
    bounds = even_bounds(S, n_blocks)
    parts = torch.empty((n_blocks, Bp, S, Hp, D), dtype=torch.float32, device=dev)
    lses = torch.empty((n_blocks, Bp, Hp, S), dtype=torch.float32, device=dev)
    yq, yk, yv = (torch.empty((P, B, S, Hp, D), dtype=torch.bfloat16, device=dev) for _ in range(3))
    o_h = torch.empty((Bp, S, Hp, D), dtype=torch.bfloat16, device=dev)
    lse_h = torch.empty((Bp, Hp, S), dtype=torch.float32, device=dev)
    lse_full = torch.empty((B, H, S), dtype=torch.float32, device=dev)
    o_seq = torch.empty((P, B, S // P, H, D), dtype=torch.bfloat16, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    # L2 flush between timed steps: a read-only sweep of a buffer larger than L2.  A write
    # would leave L2 full of dirty lines that the next kernel has to write back; a read
    # evicts the previous step's dirty lines during the flush and leaves only clean ones.
    flush_buf = torch.ones(max(2 * l2, 256 << 20) // 4, dtype=torch.float32, device=dev)
    flush_sink = torch.empty((), dtype=torch.float32, device=dev)
    flush_mib = flush_buf.numel() * 4 >> 20

    def flush_l2():
        torch.sum(flush_buf, dim=0, out=flush_sink)
    scale = w.scale
    flop = w.flop
    launches_per_step = 1 + 1  # exchange of Q, K, V; ring attention with the merge and the inverse exchange
    view = lambda t: t.view(Bp, S, Hp, D)  # noqa: E731  (head shards as one BSHD tensor)

    def step(evs=None, x=None, out=None):
        """The hot path in two launches: the Ulysses exchange of Q, K and V, then ring
        attention over the 8 K/V blocks on every head shard with the LSE merge carried in
        TMEM from block to block and each finished row stored to its token-sharded place
        (the inverse exchange), cp_ring_sim_fused_ulysses."""
        x = x or (xq, xk, xv)
        out = o_seq if out is None else out
        if evs:
            evs[0].record()
        binding.ulysses_permute_n(x, P, 0, dsts=(yq, yk, yv))
        if evs:
            evs[1].record()
        binding.ring_sim_fused_ulysses(yq, yk, yv, P, bounds, scale=scale, out=out, out_lse=lse_full)
        if evs:
            evs[2].record()

    def step3(evs=None):
        """The same hot path in three launches, each block's fp32 partial and LSE written to
        HBM: the exchange, blockwise attention over the 8 blocks, then the LSE merge writing
        each merged row to its token-sharded place (cp_attn_merge_ulysses)."""
        if evs:
            evs[0].record()
        binding.ulysses_permute_n((xq, xk, xv), P, 0, dsts=(yq, yk, yv))
        if evs:
            evs[1].record()
        binding.attn_fwd_blocks(view(yq), view(yk), view(yv), bounds, scale=scale, partials=parts, lses=lses)
        if evs:
            evs[2].record()
        binding.attn_merge_ulysses(parts, lses, P, out=o_seq3, out_lse=lse3)
        if evs:
            evs[3].record()

    o_seq3 = torch.empty_like(o_seq)
    lse3 = torch.empty_like(lse_full)
    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0

    clocks = ClockSampler(local)
    clocks.start()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.mark_start()
    for i in range(args.steps):
        flush_l2()
        step(evs[i])
    torch.cuda.synchronize()
    clocks.mark_end()
    if world > 1:
        dist.barrier()
    clocks.stop()
    assert binding.last_device_status() == 0, "device status not OK after timed region"

    step_ms = [e[0].elapsed_time(e[2]) for e in evs]
    perm_ms = [e[0].elapsed_time(e[1]) for e in evs]
    attn_ms = [e[1].elapsed_time(e[2]) for e in evs]
    total_ms = reduce_max(sum(step_ms), dev)

    # The three-launch form, timed the same way (its merge is the merge kernel's number).
    n3 = min(args.steps, 200)
    for _ in range(max(args.warmup, 3)):
        flush_l2()
        step3()
    evs3 = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n3)]
    for i in range(n3):
        flush_l2()
        step3(evs3[i])
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    step3_ms = statistics.mean(e[0].elapsed_time(e[3]) for e in evs3)
    perm3_ms = [e[0].elapsed_time(e[1]) for e in evs3]
    attn3_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs3)
    merge_ms = [e[2].elapsed_time(e[3]) for e in evs3]
    # The merge on its own: inside the step it follows the attention launch, whose last
    # ~100 MB of partials are still dirty in L2 and are written back while the merge runs.
    # Here the partials of the last step are in HBM and L2 is flushed before each merge.
    iso = []
    for i in range(max(args.warmup, 3) + 50):
        flush_l2()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        binding.attn_merge_ulysses(parts, lses, P, out=o_seq3, out_lse=lse3)
        b.record()
        iso.append((a, b))
    torch.cuda.synchronize()
    merge_iso_ms = statistics.mean(a.elapsed_time(b) for a, b in iso[max(args.warmup, 3):])

    # Single-block attention (the FLUX ring-1 case) timed on its own.
    qd, kd, vd = (t.to(dev) for t in (q_h, k_h, v_h))
    o1 = torch.empty_like(qd)
    l1 = torch.empty((B, H, S), dtype=torch.float32, device=dev)
    r1 = []
    for i in range(max(args.warmup, 3) + 50):
        flush_l2()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        binding.attn_fwd(qd, kd, vd, scale=scale, out=o1, lse=l1)
        b.record()
        r1.append((a, b))
    torch.cuda.synchronize()
    ring1_ms = statistics.mean(a.elapsed_time(b) for a, b in r1[max(args.warmup, 3):])

    # The ring with the LSE merge fused into the attention kernel (no partials, no merge
    # pass), on the same head-sharded tensors as the step, head-sharded output.
    fo = torch.empty_like(o_h)
    fl = torch.empty_like(lse_h)
    rf = []
    for i in range(max(args.warmup, 3) + 50):
        flush_l2()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        binding.ring_sim_fused(view(yq), view(yk), view(yv), bounds, scale=scale, out=fo, out_lse=fl)
        b.record()
        rf.append((a, b))
    torch.cuda.synchronize()
    fused_ms = statistics.mean(a.elapsed_time(b) for a, b in rf[max(args.warmup, 3):])

    def timed_ms(fn, reps=20):
        evs = []
        for i in range(max(args.warmup, 3) + reps):
            flush_l2()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            evs.append((a, b))
        torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in evs[max(args.warmup, 3):])

    # Unified SP: Ulysses 2 x ring 4 and Ulysses 4 x ring 2 on the same tensors, through
    # cp_usp_sim (exchange, ring attention + merge, inverse exchange, LSE regroup).
    usp = {}
    for U, R in ((2, 4), (4, 2)):
        sh = [t.reshape(B, U, S // U, H, D).permute(1, 0, 2, 3, 4).contiguous().to(dev) for t in (q_h, k_h, v_h)]
        ws = torch.empty(binding.usp_workspace_size(U, R, B, S, H, D), dtype=torch.uint8, device=dev)
        uo = torch.empty_like(sh[0])
        ul = torch.empty((B, H, S), dtype=torch.float32, device=dev)
        ub = even_bounds(S, R)
        ms = timed_ms(lambda: binding.usp_sim(*sh, U, ub, scale=scale, workspace=ws, out=uo, out_lse=ul))
        usp[f"usp_u{U}_r{R}_ms"] = round(ms, 4)
        usp[f"usp_u{U}_r{R}_tflops"] = round(flop / (ms * 1e-3) / 1e12, 2)
        del sh, ws, uo, ul

    # Ulysses Anything exchange: FLUX at 1008x1008 (4481 tokens) over 4 ranks, Q/K/V in one launch.
    Sa = 4481
    xa = [torch.randn(B * Sa * H * D, generator=torch.Generator().manual_seed(5 + i)).bfloat16().to(dev)
          for i in range(3)]
    ya = [torch.empty_like(t) for t in xa]
    sba, hba = binding.ring_bounds(Sa, 4, anything=True), binding.ring_bounds(H, 4, anything=True)
    any_ms = timed_ms(lambda: binding.ulysses_anything_permute_n(xa, 4, sba, hba, B, Sa, H, D, 0, dsts=ya))
    any_bytes = 2 * sum(t.numel() * t.element_size() for t in xa)
    # Ring Anything's pad -> all-gather buffer of K and V for the same 4481 tokens over 4.
    ka = [t.view(B, Sa, H, D) for t in xa[1:]]
    ga = [torch.empty((4, B, 1121, H, D), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    gather_ms = timed_ms(lambda: binding.ring_anything_gather(ka, sba, 1121, dsts=ga))
    gather_bytes = sum(t.numel() * t.element_size() for t in ka) + sum(t.numel() * t.element_size() for t in ga)
    del xa, ya, ka, ga

    # The other workloads (parity cases, reported beside the bench line, not as it): ring /
    # ring-anything attention, blocks + LSE merge (cp_ring_sim), over each of their splits.
    other_configs = {}
    for name in ("tiny_s256_d64", "uneven_s4173_ring3", "video_s32760_ring4"):
        wl = WORKLOADS[name]
        cq, ck, cv = (t.to(dev) for t in wl.qkv())
        for i, sizes in enumerate(wl.splits):
            bnd = bounds_from_sizes(sizes)
            cws = torch.empty(max(binding.ring_workspace_size(len(sizes), wl.B, wl.H, wl.S, wl.D), 1),
                              dtype=torch.uint8, device=dev)
            co = torch.empty_like(cq)
            cl = torch.empty((wl.B, wl.H, wl.S), dtype=torch.float32, device=dev)
            ms = timed_ms(lambda: binding.ring_sim(cq, ck, cv, bnd, scale=wl.scale, workspace=cws, out=co,
                                                   out_lse=cl), reps=5 if wl.S > 20000 else 20)
            fms = timed_ms(lambda: binding.ring_sim_fused(cq, ck, cv, bnd, scale=wl.scale, out=co, out_lse=cl),
                           reps=5 if wl.S > 20000 else 20)
            key = name if len(wl.splits) == 1 else f"{name}_split{i}"
            other_configs[key] = {"blocks": list(sizes), "ms": round(ms, 4),
                                  "tflops": round(wl.flop / (ms * 1e-3) / 1e12, 2),
                                  "fused_ms": round(fms, 4), "fused_tflops": round(wl.flop / (fms * 1e-3) / 1e12, 2)}
            del cws, co, cl
        del cq, ck, cv
    torch.cuda.empty_cache()

    # One process per GPU: every rank's push of Q/K/V (cp_ulysses_push_n), the ranks taken
    # in turn on this GPU with local buffers for their peers' (NVLink is not measured here).
    def push_all():
        st = torch.cuda.current_stream().cuda_stream
        for r in range(P):
            binding.ulysses_push_n([xq[r].data_ptr(), xk[r].data_ptr(), xv[r].data_ptr()],
                                   [[t[p].data_ptr() for p in range(P)] for t in (yq, yk, yv)], r, P, B, S, H, D,
                                   0, 2, st)

    # The eight launches are replayed from a CUDA graph, so that the host's launch cost
    # does not pace them.
    push_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(push_graph):
        push_all()
    push_ms = timed_ms(push_graph.replay)

    # End to end through the public API with host buffers (pinned), per step: H2D of the
    # sequence-sharded Q/K/V, the hot path, D2H of O.  Steps are pipelined over three
    # streams with two buffer slots, as a serving loop would run them: the upload of step
    # i+1 and the download of step i-1 overlap the compute of step i (PCIe is full duplex).
    # Every step still moves all of its bytes and computes everything.
    hq, hk, hv = (seq_shards(t).pin_memory() for t in (q_h, k_h, v_h))
    ho = [torch.empty(o_seq.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    xs = [(xq, xk, xv), tuple(torch.empty_like(t) for t in (xq, xk, xv))]
    outs = [o_seq, torch.empty_like(o_seq)]
    s_up, s_cmp, s_dn = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    up_done, cmp_done, dn_done = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))

    def e2e_run(n):
        for i in range(n):
            sl = i % 2
            with torch.cuda.stream(s_up):
                if i >= 2:
                    s_up.wait_event(cmp_done[sl])  # the slot's previous inputs are consumed
                for d, h in zip(xs[sl], (hq, hk, hv)):
                    d.copy_(h, non_blocking=True)
                up_done[sl].record(s_up)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(up_done[sl])
                if i >= 2:
                    s_cmp.wait_event(dn_done[sl])  # the slot's previous output is downloaded
                step(x=xs[sl], out=outs[sl])
                cmp_done[sl].record(s_cmp)
            with torch.cuda.stream(s_dn):
                s_dn.wait_event(cmp_done[sl])
                ho[sl].copy_(outs[sl], non_blocking=True)
                dn_done[sl].record(s_dn)

    e2e_steps = max(5, min(50, args.steps // 20))
    torch.cuda.synchronize()
    e2e_run(2)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    e2e_run(e2e_steps)
    s_dn.wait_event(cmp_done[(e2e_steps - 1) % 2])
    e1.record(s_dn)  # after the last download, which follows every upload and compute
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    d2h = ho[0].numel() * ho[0].element_size()
    e2e_ms = reduce_max(e0.elapsed_time(e1) / e2e_steps, dev)

    if rank == 0:
        peaks = load_peaks()
        step_mean = total_ms / args.steps
        value = job_throughput(world, flop, total_ms, args.steps)
        attn_mean = statistics.mean(attn_ms)
        attn_tflops = flop / (attn_mean * 1e-3) / 1e12
        ring1_tflops = flop / (ring1_ms * 1e-3) / 1e12
        rows = Bp * Hp * S
        merge_bytes = n_blocks * rows * (4 * D + 4) + rows * (2 * D + 4)
        perm_bytes = 3 * 2 * B * S * H * D * 2
        part_bytes = n_blocks * rows * (4 * D + 4)
        merge_gbs = merge_bytes / (statistics.mean(merge_ms) * 1e-3) / 1e9
        merge_iso_gbs = merge_bytes / (merge_iso_ms * 1e-3) / 1e9
        perm_gbs = perm_bytes / (statistics.mean(perm_ms + perm3_ms) * 1e-3) / 1e9
        line = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": UNIT,
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(step_mean, 4),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16, per-head RMS-normed Q/K; sha256 " + ",".join(
                f"{k}:{v}" for k, v in sha.items()) + ")",
            "config": step_config(world, B, S, H, D, P, n_blocks,
                                  "flushed between timed steps (read of %d MiB > L2)" % flush_mib),
            "roofline": {
                "kernel": "attention, 8 ring blocks in one launch, merge in TMEM, inverse exchange in the epilogue",
                "bound": "tensor",
                "achieved": round(attn_tflops, 2),
                "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s",
                "frac": round(attn_tflops / peaks["bf16_tflops"], 4),
                "frac_of_sustained": round(attn_tflops / peaks["bf16_tflops_sustained"], 4)
                if peaks["bf16_tflops_sustained"] else None,
                "frac_of_spec_2250": round(attn_tflops / 2250.0, 4),
                "peak_source": peaks["source"] + " (burst bf16 GEMM)",
                "flop_per_launch": flop,
                "traffic": attn_traffic(),
                "traffic_unit": "bytes per launch (ncu dram read + write)",
            },
            "kernels": {
                "attn_ring1_tflops": round(ring1_tflops, 2),
                "attn_ring1_ms": round(ring1_ms, 4),
                "attn_ring8_fused_ulysses_ms": round(attn_mean, 4),
                "ring8_fused_ms": round(fused_ms, 4),
                "ring8_fused_tflops": round(flop / (fused_ms * 1e-3) / 1e12, 2),
                "step_3launch_ms": round(step3_ms, 4),
                "step_3launch_tflops": round(flop / (step3_ms * 1e-3) / 1e12, 2),
                "attn_ring8_blocks_ms": round(attn3_ms, 4),
                "attn_ring8_blocks_tflops": round(flop / (attn3_ms * 1e-3) / 1e12, 2),
                "attn_ring8_partial_bytes": part_bytes,
                "merge_inverse_exchange_ms": round(merge_iso_ms, 4),
                "merge_inverse_exchange_gbs": round(merge_iso_gbs, 1),
                "merge_inverse_exchange_frac_of_measured_hbm": round(merge_iso_gbs / peaks["hbm_gbs"], 4),
                "merge_inverse_exchange_frac_of_spec_8000": round(merge_iso_gbs / 8000.0, 4),
                "merge_inverse_exchange_in_3launch_step_ms": round(statistics.mean(merge_ms), 4),
                "merge_inverse_exchange_in_3launch_step_gbs": round(merge_gbs, 1),
                "permute_qkv_ms": round(statistics.mean(perm_ms), 4),
                "permute_qkv_gbs": round(perm_gbs, 1),
                "permute_qkv_frac_of_measured_hbm": round(perm_gbs / peaks["hbm_gbs"], 4),
                "permute_qkv_frac_of_spec_8000": round(perm_gbs / 8000.0, 4),
                "hbm_peak_gbs": peaks["hbm_gbs"],
                "ring_anything_gather_kv_flux1008_r4_ms": round(gather_ms, 4),
                "ring_anything_gather_kv_flux1008_r4_gbs": round(gather_bytes / (gather_ms * 1e-3) / 1e9, 1),
                **usp,
                "anything_permute_qkv_flux1008_p4_ms": round(any_ms, 4),
                "anything_permute_qkv_flux1008_p4_gbs": round(any_bytes / (any_ms * 1e-3) / 1e9, 1),
                "push_qkv_8_ranks_by_turns_ms": round(push_ms, 4),
                "push_qkv_8_ranks_by_turns_gbs": round(perm_bytes / (push_ms * 1e-3) / 1e9, 1),
            },
            "other_configs": other_configs,
            "e2e": {"value": round(world * flop / (e2e_ms * 1e-3) / 1e12, 2), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4)},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks.summary(),
        }
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(budget_s=args.cpu_budget)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# --------------------------------------------------------------------------- the oracle


def _oracle_step(q, k, v, scale, bounds, rows):
    """One oracle pass: ring attention (per block + LSE merge) for the sampled query rows."""
    import oracle

    return oracle.ring(q[:, rows], k, v, scale, bounds)


def _threads_used():
    try:
        from threadpoolctl import threadpool_info

        info = threadpool_info()
        return max((i.get("num_threads", 1) for i in info), default=1)
    except Exception:
        return 1


def _sample_rows(S, n):
    import numpy as np

    return sorted(np.random.default_rng(0).choice(S, size=n, replace=False).tolist())


def cpu_baseline(budget_s: float = 15.0):
    """Time the fp64 oracle as it stands on a bounded sample of the workload (rank 0 only)."""
    from context_attention_dit_b200.inputs import WORKLOADS, even_bounds

    w = WORKLOADS[WORKLOAD]
    q, k, v = w.qkv()
    bounds = even_bounds(w.S, len(w.splits[0]))
    # calibrate the sample size on 64 rows, then size it to the budget
    t0 = time.time()
    _oracle_step(q, k, v, w.scale, bounds, _sample_rows(w.S, 64))
    per_row = (time.time() - t0) / 64
    n_rows = int(max(64, min(w.S, budget_s / max(per_row, 1e-6))))
    rows = _sample_rows(w.S, n_rows)
    # The calibration overestimates the cost per row, so the sample can run short of the
    # budget: repeat it until at least two thirds of the budget have passed.
    passes = 0
    t0 = time.time()
    while True:
        _oracle_step(q, k, v, w.scale, bounds, rows)
        passes += 1
        dt = time.time() - t0
        if dt >= budget_s * 2 / 3:
            break
    flop = 4 * w.B * w.H * n_rows * w.S * w.D * passes
    what = f"{n_rows} of {w.S} query rows" + (f", {passes} passes" if passes > 1 else "")
    return {"value": round(flop / dt / 1e12, 6), "unit": UNIT, "cores": _threads_used(), "kind": "oracle",
            "sample": f"ring-8 attention + LSE merge (fp64 numpy) for {what}, all 24 heads, {dt:.1f} s",
            "seconds": round(dt, 2)}


def run_reference(args):
    world, rank, _ = dist_setup()
    if rank != 0:
        return
    from context_attention_dit_b200.inputs import WORKLOADS, even_bounds

    w = WORKLOADS[WORKLOAD]
    q, k, v = w.qkv()
    bounds = even_bounds(w.S, len(w.splits[0]))
    budget_per_step = max(0.05, args.ref_budget / max(1, args.steps + args.warmup))
    t0 = time.time()
    _oracle_step(q, k, v, w.scale, bounds, _sample_rows(w.S, 16))
    per_row = (time.time() - t0) / 16
    n_rows = int(max(1, min(w.S, budget_per_step / max(per_row, 1e-6))))
    rows = _sample_rows(w.S, n_rows)
    for _ in range(args.warmup):
        _oracle_step(q, k, v, w.scale, bounds, rows)
    times = []
    for _ in range(args.steps):
        t0 = time.time()
        _oracle_step(q, k, v, w.scale, bounds, rows)
        times.append(time.time() - t0)
    total = sum(times)
    flop = 4 * w.B * w.H * n_rows * w.S * w.D
    value = flop * args.steps / total / 1e12
    line = {
        "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": step_config(1, w.B, w.S, w.H, w.D, w.ulysses_degree, len(w.splits[0]),
                              "host cores (fp64 oracle; no GPU cache involved)"),
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": _threads_used(), "kind": "oracle",
                         "sample": f"{n_rows} of {w.S} query rows per step, all heads, 8 K/V blocks + merge "
                                   "(the exchanges are index maps with no arithmetic: not timed)"},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_profile_case(args):
    """Run one kernel of the hot path a few times on the FLUX shape (batch scaled by
    --profile-batch so that inputs exceed L2) for an ncu capture; prints nothing timed."""
    import torch

    from context_attention_dit_b200 import binding
    from context_attention_dit_b200.inputs import WORKLOADS, even_bounds, make_qkv

    torch.cuda.set_device(0)
    w = WORKLOADS[WORKLOAD]
    B, S, H, D, P = w.B * args.profile_batch, w.S, w.H, w.D, w.ulysses_degree
    q, k, v = (t.cuda() for t in make_qkv(B, H, S, S, D, rms_norm_qk=True))
    bounds = even_bounds(S, 8)
    case = args.profile_case
    for _ in range(args.profile_reps):
        if case == "attn_ring1":
            binding.attn_fwd(q, k, v)
        elif case == "attn_ring8":
            binding.attn_fwd_blocks(q, k, v, bounds)
        elif case == "attn_fused_ulysses":  # the step's attention: head shards in, token shards out
            heads = [t.view(B, P, S // P, H, D).permute(1, 0, 2, 3, 4).contiguous() for t in (q, k, v)]
            heads = binding.ulysses_permute_n(heads, P, 0)
            binding.ring_sim_fused_ulysses(*heads, P, bounds)
        elif case == "merge":  # the step's merge: head-shard partials, fused with the inverse exchange
            parts = torch.randn(8, P * B, S, H // P, D, device="cuda")
            lses = torch.randn(8, P * B, H // P, S, device="cuda")
            binding.attn_merge_ulysses(parts, lses, P)
        elif case == "permute":
            xs = [t.view(B, P, S // P, H, D).permute(1, 0, 2, 3, 4).contiguous() for t in (q, k, v)]
            ys = binding.ulysses_permute_n(xs, P, 0)
            binding.ulysses_permute(ys[0], P, 1)
        elif case == "anything":  # Q/K/V Ulysses-Anything exchange, FLUX-1008^2 (4481 tokens) over 4
            Sa = 4481
            xa = [torch.randn(B * Sa * H * D, device="cuda").bfloat16() for _ in range(3)]
            binding.ulysses_anything_permute_n(xa, 4, binding.ring_bounds(Sa, 4, anything=True),
                                               binding.ring_bounds(H, 4, anything=True), B, Sa, H, D, 0)
        elif case == "gather":  # Ring Anything pad -> all-gather buffer of K/V, FLUX-1008^2 over 4
            Sa = 4481
            ka = [torch.randn(B, Sa, H, D, device="cuda").bfloat16() for _ in range(2)]
            binding.ring_anything_gather(ka, binding.ring_bounds(Sa, 4, anything=True))
        elif case == "push":  # every rank's Q/K/V push, ranks by turns, local buffers for the peers'
            xs = [t.view(B, P, S // P, H, D).permute(1, 0, 2, 3, 4).contiguous() for t in (q, k, v)]
            ys = [torch.empty(P, B, S, H // P, D, dtype=torch.bfloat16, device="cuda") for _ in range(3)]
            st = torch.cuda.current_stream().cuda_stream
            for r in range(P):
                binding.ulysses_push_n([x[r].data_ptr() for x in xs], [[y[p].data_ptr() for p in range(P)] for y in ys],
                                       r, P, B, S, H, D, 0, 2, st)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    print(f"profile case {case} x{args.profile_reps} batch {B}: ok")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-budget", type=float, default=90.0)
    ap.add_argument("--profile-case", choices=["attn_ring1", "attn_ring8", "attn_fused_ulysses", "merge", "permute", "push", "anything",
                                                      "gather"], default=None)
    ap.add_argument("--profile-batch", type=int, default=2)
    ap.add_argument("--profile-reps", type=int, default=3)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.profile_case:
        run_profile_case(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
