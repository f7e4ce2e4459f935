"""Every element of the video-DiT workload (B1 H40 S32760 D128, QK-normed; "Context
parallelism" on long video sequences) against the fp64 oracle: ring-4 through
cp_ring_sim (blocks + LSE merge), the same ring with the merge fused into the kernel
(cp_ring_sim_fused), and unsplit attention (cp_attn_fwd).

The oracle's 2.2e13 fp64 FLOP run on a pool of host processes, one (head, row range)
piece at a time (tests/oracle_pool.py); the statistics are those of
gpu_util.assert_attn_close, accumulated over the pieces, and they are printed in the
session's parity summary."""

import numpy as np
import pytest
import torch

from context_attention_dit_b200 import binding
from context_attention_dit_b200.inputs import even_bounds
from tests import oracle_pool
from tests.gpu_util import LSE_ABS, O_MAX_ABS, O_MEAN_ABS, O_REL_L2, assert_split_close, cuda, workload_inputs

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def test_video_every_element_vs_oracle(parity_report):
    w, (q, k, v) = workload_inputs("video_s32760_ring4")
    bounds = even_bounds(w.S, 4)
    dq, dk, dv = cuda(q, k, v)
    o4, l4, ws = binding.ring_sim(dq, dk, dv, bounds, scale=w.scale)
    del ws
    o1, l1 = binding.attn_fwd(dq, dk, dv, scale=w.scale)
    of, lf = binding.ring_sim_fused(dq, dk, dv, bounds, scale=w.scale)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    assert_split_close(o4, o1, "video ring-4 vs unsplit")
    assert_split_close(of, o1, "video fused ring-4 vs unsplit")
    outs = {name: (o.float().cpu().numpy(), l.cpu().numpy())
            for name, (o, l) in {"cp_ring_sim ring-4": (o4, l4), "cp_ring_sim_fused ring-4": (of, lf),
                                 "cp_attn_fwd ring-1": (o1, l1)}.items()}
    del dq, dk, dv, o4, l4, o1, l1, of, lf
    torch.cuda.empty_cache()
    accs = {name: oracle_pool.ErrorAccumulator() for name in outs}
    seen = np.zeros((w.B, w.H, w.S), dtype=np.int8)
    for b, h, r0, r1, o_ref, l_ref in oracle_pool.attention_pieces(q, k, v, w.scale):
        seen[b, h, r0:r1] += 1
        for name, (og, lg) in outs.items():
            accs[name].add(og[b, r0:r1, h], o_ref, lg[b, h, r0:r1], l_ref)
    assert (seen == 1).all(), "the pieces must cover every (head, row) once"
    for name, acc in accs.items():
        s = acc.summary()
        parity_report(f"video B1 H40 S32760 D128, {name}, every element vs fp64 oracle: max-abs {s['max_abs']:.3e}, "
                      f"mean-abs {s['mean_abs']:.3e}, rel-L2 {s['rel_l2']:.3e}, lse max-abs {s['lse_max_abs']:.3e} "
                      f"({s['elements']} elements)")
        assert acc.finite and acc.inf_pattern_ok, name
        assert s["max_abs"] <= O_MAX_ABS and s["mean_abs"] <= O_MEAN_ABS and s["rel_l2"] <= O_REL_L2, (name, s)
        assert s["lse_max_abs"] <= LSE_ABS, (name, s)
