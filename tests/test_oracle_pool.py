"""The pooled oracle evaluation equals the oracle itself (CPU)."""

import numpy as np

import oracle
from context_attention_dit_b200.inputs import make_qkv
from tests import oracle_pool


def test_pooled_pieces_equal_the_oracle():
    q, k, v = make_qkv(2, 3, 700, 700, 64, seed=91, rms_norm_qk=True)
    o_ref, lse_ref = oracle.attention(q, k, v, 0.125)
    seen = np.zeros((2, 700, 3), dtype=int)
    acc = oracle_pool.ErrorAccumulator()
    for b, h, r0, r1, o, lse in oracle_pool.attention_pieces(q, k, v, 0.125, workers=2, rows_per_piece=300,
                                                             sub_rows=128):
        assert np.allclose(o, o_ref[b, r0:r1, h], rtol=0, atol=1e-13)
        assert np.allclose(lse, lse_ref[b, h, r0:r1], rtol=0, atol=1e-13)
        seen[b, r0:r1, h] += 1
        acc.add(o_ref[b, r0:r1, h].astype(np.float32), o, lse_ref[b, h, r0:r1].astype(np.float32), lse)
    assert (seen == 1).all(), "every (batch, row, head) exactly once"
    s = acc.summary()
    assert s["elements"] == o_ref.size and s["max_abs"] < 1e-6 and s["rel_l2"] < 1e-6
