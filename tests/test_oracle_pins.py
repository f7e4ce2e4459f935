"""The fp64 oracle against its pins (CPU only)."""

import numpy as np
import pytest

import oracle
from tests import pins


@pytest.mark.parametrize("pin", pins.ATTENTION_PINS, ids=lambda p: p.__name__)
def test_attention_pin(pin):
    pin(oracle.attention)


@pytest.mark.parametrize("pin", [pins.pin_merge_closed_form, pins.pin_merge_all_empty, pins.pin_merge_large_lse],
                         ids=lambda p: p.__name__)
def test_merge_pin(pin):
    pin(oracle.merge)


def test_chunk_merge_identity():
    pins.pin_chunk_merge_identity(oracle.attention, oracle.ring)


def test_usp_equals_unsplit():
    pins.pin_usp_equals_unsplit(oracle.attention, oracle.usp)


def test_ulysses_anything_origin():
    pins.pin_anything_origin(oracle.ulysses_anything_fwd, oracle.ulysses_anything_inv)


def test_ulysses_anything_reduces_to_even():
    pins.pin_anything_reduces_to_even(oracle.ulysses_anything_fwd, oracle.ulysses_fwd)


def test_ulysses_message_passing():
    pins.pin_ulysses_messages(oracle.ulysses_fwd)


def test_ulysses_roundtrip():
    pins.pin_ulysses_roundtrip(oracle.ulysses_fwd, oracle.ulysses_inv)


def test_ulysses_golden():
    pins.pin_ulysses_golden(oracle.ulysses_fwd)


def test_attention_rows_matches_full():
    r = np.random.default_rng(12)
    q = r.standard_normal((1, 40, 2, 8))
    k = r.standard_normal((1, 31, 2, 8))
    v = r.standard_normal((1, 31, 2, 8))
    o, lse = oracle.attention(q, k, v, 0.3)
    rows = [0, 7, 39]
    o2, l2 = oracle.attention_rows(q, k, v, 0.3, rows)
    assert np.array_equal(o[:, rows], o2) and np.array_equal(lse[:, :, rows], l2)


def test_ulysses_attention_is_per_head():
    """Exchange -> attention on H/P heads per shard -> inverse exchange == full attention (fp64)."""
    r = np.random.default_rng(13)
    P, B, S, H, D = 4, 1, 16, 8, 4
    q, k, v = (r.standard_normal((B, S, H, D)) for _ in range(3))
    o_full, _ = oracle.attention(q, k, v, 0.5)
    shard = lambda x: x.reshape(B, P, S // P, H, D).transpose(1, 0, 2, 3, 4)  # [P,B,S/P,H,D]
    qh, kh, vh = (oracle.ulysses_fwd(shard(x), P) for x in (q, k, v))         # [P,B,S,H/P,D]
    oh = np.stack([oracle.attention(qh[p], kh[p], vh[p], 0.5)[0] for p in range(P)])
    o_seq = oracle.ulysses_inv(oh, P)                                          # [P,B,S/P,H,D]
    o_back = o_seq.transpose(1, 0, 2, 3, 4).reshape(B, S, H, D)
    assert np.allclose(o_back, o_full, rtol=0, atol=1e-13)


def test_bf16_inputs_widen_exactly():
    import torch

    from context_attention_dit_b200.inputs import make_qkv

    q, k, v = make_qkv(1, 2, 5, 6, 8, seed=3)
    o1, l1 = oracle.attention(q, k, v, 0.25)
    o2, l2 = oracle.attention(q.float().numpy(), k.float().numpy(), v.float().numpy(), 0.25)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    assert q.dtype == torch.bfloat16


def test_ring_anything_gather_golden():
    pins.pin_gather_golden(oracle.ring_anything_gather)


def test_ring_anything_gather_per_rank():
    pins.pin_gather_per_rank(oracle.ring_anything_gather)


def test_ring_anything_gather_slice_roundtrip():
    pins.pin_gather_slice_roundtrip(oracle.ring_anything_gather, oracle.ring_anything_slice)


def test_ring_anything_gather_ring_equals_unsplit():
    pins.pin_gather_ring_equals_unsplit(oracle.attention, oracle.merge, oracle.ring_anything_gather,
                                        oracle.ring_anything_slice)
