"""Pins of the fp64 oracle to things other than itself.

Each ``pin_*`` takes the functions under test as arguments and raises
``AssertionError`` when the pinned property fails.  ``test_oracle_pins.py``
runs them on the real oracle; ``test_oracle_mutants.py`` runs them on copies of
the oracle with planted mistakes and checks that every mistake is caught.

What pins what:

* closed forms: identical keys (mean of V, LSE = ln Skv + logit), one key
  orthogonal-basis case (exact softmax weights), constant V, a single key,
  no keys, the two-block merge with hand-picked LSEs;
* invariants: key shift (softmax is shift invariant per row), joint
  permutation of K/V rows, the chunk-merge identity (split == unsplit);
* brute force: a 40-digit ``decimal`` evaluation of the un-shifted softmax;
* a library routine: ``torch.nn.functional.scaled_dot_product_attention`` and
  ``torch.logsumexp`` in fp64;
* the Ulysses exchange: a message-passing simulation of the all-to-all, a
  hand-written golden table and the round trip.
"""

from __future__ import annotations

import decimal
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


# --------------------------------------------------------------------------- attention


def pin_identical_keys(attention):
    """All keys equal: every weight is 1/Skv, so o_i = mean_j v_j and lse_i = ln(Skv) + scale*q_i.k."""
    r = _rng(1)
    B, Sq, Skv, H, D = 2, 5, 7, 3, 4
    q = r.standard_normal((B, Sq, H, D))
    k0 = r.standard_normal((B, 1, H, D))
    k = np.repeat(k0, Skv, axis=1)
    v = r.standard_normal((B, Skv, H, D))
    scale = 0.37
    o, lse = attention(q, k, v, scale)
    want_o = np.broadcast_to(v.mean(axis=1, keepdims=True), o.shape)
    assert np.allclose(o, want_o, rtol=0, atol=1e-12), "identical keys: o != mean(v)"
    logit = scale * np.einsum("bshd,bhd->bhs", q, k0[:, 0])
    assert np.allclose(lse, math.log(Skv) + logit, rtol=0, atol=1e-12), "identical keys: lse"


def pin_basis_keys(attention):
    """Keys are the basis vectors e_0..e_{D-1}; q = a*e_t gives logits scale*a at t and 0 elsewhere.

    Exact weights: w_t = e^{c} / (e^{c} + D - 1), w_j = 1 / (e^{c} + D - 1) with c = scale*a.
    With a large the row selects v_t (the one-dominant-logit case) within the
    bound (D-1) e^{-c} max|v|.
    """
    D = 6
    r = _rng(2)
    v = r.standard_normal((1, D, 1, D))
    k = np.eye(D).reshape(1, D, 1, D)
    scale = 0.5
    for t, a in [(0, 1.0), (3, -2.5), (5, 40.0)]:
        q = np.zeros((1, 1, 1, D))
        q[0, 0, 0, t] = a
        o, lse = attention(q, k, v, scale)
        c = scale * a
        den = math.exp(c) + D - 1
        w = np.full(D, 1.0 / den)
        w[t] = math.exp(c) / den
        want = (w[:, None] * v[0, :, 0, :]).sum(axis=0)
        assert np.allclose(o[0, 0, 0], want, rtol=0, atol=1e-12), f"basis keys t={t}"
        assert abs(lse[0, 0, 0] - math.log(den)) < 1e-12, f"basis keys lse t={t}"
        if c > 10:
            bound = (D - 1) * math.exp(-c) * np.abs(v).max() * 2
            assert np.abs(o[0, 0, 0] - v[0, t, 0]).max() <= bound, "dominant logit must select its row"
            assert abs(lse[0, 0, 0] - c) <= (D - 1) * math.exp(-c) * 2


def pin_constant_v(attention):
    """All value rows equal c: o_i = c for any logits (weights sum to one)."""
    r = _rng(3)
    B, Sq, Skv, H, D = 1, 9, 13, 2, 8
    q = r.standard_normal((B, Sq, H, D)) * 3
    k = r.standard_normal((B, Skv, H, D)) * 3
    c = r.standard_normal((B, 1, H, D))
    v = np.repeat(c, Skv, axis=1)
    o, _ = attention(q, k, v, 0.6)
    assert np.allclose(o, np.broadcast_to(c, o.shape), rtol=0, atol=1e-13), "constant v"


def pin_single_key(attention):
    """One key: o_i = v_0 and lse_i = scale*q_i.k_0."""
    r = _rng(4)
    q = r.standard_normal((2, 4, 3, 5))
    k = r.standard_normal((2, 1, 3, 5))
    v = r.standard_normal((2, 1, 3, 5))
    o, lse = attention(q, k, v, 0.8)
    assert np.allclose(o, np.broadcast_to(v, o.shape), rtol=0, atol=1e-14), "single key o"
    want = 0.8 * np.einsum("bshd,bhd->bhs", q, k[:, 0])
    assert np.allclose(lse, want, rtol=0, atol=1e-13), "single key lse"


def pin_no_keys(attention):
    """No keys: o = 0 and lse = -inf (the merge's neutral element)."""
    q = np.ones((1, 3, 2, 4))
    k = np.zeros((1, 0, 2, 4))
    o, lse = attention(q, k, k, 0.5)
    assert o.shape == (1, 3, 2, 4) and not o.any(), "no keys: o must be 0"
    assert lse.shape == (1, 2, 3) and np.all(np.isneginf(lse)), "no keys: lse must be -inf"


def pin_key_shift(attention):
    """k_j -> k_j + u for every j shifts row i's logits by scale*q_i.u: o unchanged, lse shifted."""
    r = _rng(5)
    B, Sq, Skv, H, D = 1, 6, 11, 2, 4
    q = r.standard_normal((B, Sq, H, D))
    k = r.standard_normal((B, Skv, H, D))
    v = r.standard_normal((B, Skv, H, D))
    u = r.standard_normal((B, 1, H, D))
    o1, l1 = attention(q, k, v, 0.9)
    o2, l2 = attention(q, k + u, v, 0.9)
    assert np.allclose(o1, o2, rtol=0, atol=1e-12), "key shift must not change o"
    shift = 0.9 * np.einsum("bshd,bhd->bhs", q, u[:, 0])
    assert np.allclose(l2 - l1, shift, rtol=0, atol=1e-12), "key shift must shift lse"


def pin_kv_permutation(attention):
    """Permuting K and V rows together leaves o and lse unchanged."""
    r = _rng(6)
    B, Sq, Skv, H, D = 2, 5, 17, 2, 4
    q = r.standard_normal((B, Sq, H, D))
    k = r.standard_normal((B, Skv, H, D))
    v = r.standard_normal((B, Skv, H, D))
    perm = r.permutation(Skv)
    o1, l1 = attention(q, k, v, 0.7)
    o2, l2 = attention(q, k[:, perm], v[:, perm], 0.7)
    assert np.allclose(o1, o2, rtol=0, atol=1e-12) and np.allclose(l1, l2, rtol=0, atol=1e-12), "kv permutation"


def _decimal_attention(q, k, v, scale):
    """Brute force: 40-digit decimal, un-shifted exponentials, scalar loops."""
    ctx = decimal.Context(prec=40)
    Dd = decimal.Decimal
    B, Sq, H, D = q.shape
    Skv = k.shape[1]
    o = np.zeros(q.shape)
    lse = np.zeros((B, H, Sq))
    sc = Dd(repr(float(scale)))
    for b in range(B):
        for h in range(H):
            for i in range(Sq):
                es = []
                for j in range(Skv):
                    dot = Dd(0)
                    for d in range(D):
                        dot = ctx.add(dot, ctx.multiply(Dd(repr(float(q[b, i, h, d]))), Dd(repr(float(k[b, j, h, d])))))
                    es.append(ctx.exp(ctx.multiply(sc, dot)))
                tot = Dd(0)
                for e in es:
                    tot = ctx.add(tot, e)
                for d in range(D):
                    acc = Dd(0)
                    for j in range(Skv):
                        acc = ctx.add(acc, ctx.multiply(es[j], Dd(repr(float(v[b, j, h, d])))))
                    o[b, i, h, d] = float(ctx.divide(acc, tot))
                lse[b, h, i] = float(ctx.ln(tot))
    return o, lse


def pin_brute_force(attention):
    """Tiny random inputs: oracle == 40-digit decimal evaluation of the definition."""
    r = _rng(7)
    for (B, Sq, Skv, H, D) in [(1, 3, 5, 1, 2), (2, 4, 8, 2, 4), (1, 8, 3, 1, 3)]:
        q = r.standard_normal((B, Sq, H, D)) * 2
        k = r.standard_normal((B, Skv, H, D)) * 2
        v = r.standard_normal((B, Skv, H, D))
        scale = 1.0 / math.sqrt(D)
        o, lse = attention(q, k, v, scale)
        o2, l2 = _decimal_attention(q, k, v, scale)
        assert np.allclose(o, o2, rtol=0, atol=1e-13), "brute force o"
        assert np.allclose(lse, l2, rtol=0, atol=1e-13), "brute force lse"


def pin_library_sdpa(attention):
    """fp64 torch SDPA (math path on CPU) and torch.logsumexp agree with the oracle."""
    import torch

    r = _rng(8)
    B, Sq, Skv, H, D = 2, 33, 47, 3, 16
    q = r.standard_normal((B, Sq, H, D))
    k = r.standard_normal((B, Skv, H, D))
    v = r.standard_normal((B, Skv, H, D))
    scale = 1.0 / math.sqrt(D)
    o, lse = attention(q, k, v, scale)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))  # BSHD -> BHSD
    to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=scale)
    assert np.allclose(o, to.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12), "torch sdpa o"
    tl = torch.logsumexp(scale * (tq @ tk.transpose(-1, -2)), dim=-1)  # [B,H,Sq]
    assert np.allclose(lse, tl.numpy(), rtol=0, atol=1e-12), "torch logsumexp"


ATTENTION_PINS = [
    pin_identical_keys, pin_basis_keys, pin_constant_v, pin_single_key, pin_no_keys,
    pin_key_shift, pin_kv_permutation, pin_brute_force, pin_library_sdpa,
]


# --------------------------------------------------------------------------- merge / ring


def pin_merge_closed_form(merge):
    """Two blocks with lse ln2 and ln6: L = ln8, weights 1/4 and 3/4; a third empty block is ignored."""
    P = np.zeros((3, 1, 1, 1, 2))
    P[0, ..., :] = [1.0, -2.0]
    P[1, ..., :] = [5.0, 4.0]
    P[2, ..., :] = [1e9, 1e9]  # empty block's output must not leak in
    L = np.array([math.log(2), math.log(6), -math.inf]).reshape(3, 1, 1, 1)
    o, lse = merge(P, L)
    assert abs(lse[0, 0, 0] - math.log(8)) < 1e-14, "merge lse"
    assert np.allclose(o[0, 0, 0], [0.25 * 1 + 0.75 * 5, 0.25 * -2 + 0.75 * 4], rtol=0, atol=1e-14), "merge o"


def pin_merge_all_empty(merge):
    """Every block empty: O = 0 and L = -inf."""
    P = np.ones((2, 1, 3, 1, 4))
    L = np.full((2, 1, 1, 3), -math.inf)
    o, lse = merge(P, L)
    assert not o.any() and np.all(np.isneginf(lse)), "all-empty merge"


def pin_merge_large_lse(merge):
    """Large LSEs (|L| ~ 1e3) must not overflow: the max shift makes the merge exact."""
    P = np.stack([np.full((1, 1, 1, 1), 2.0), np.full((1, 1, 1, 1), 4.0)])
    L = np.array([1000.0, 1000.0 + math.log(3)]).reshape(2, 1, 1, 1)
    o, lse = merge(P, L)
    assert abs(o[0, 0, 0, 0] - (0.25 * 2 + 0.75 * 4)) < 1e-12
    assert abs(lse[0, 0, 0] - (1000.0 + math.log(4))) < 1e-12


def pin_chunk_merge_identity(attention, ring):
    """Split == unsplit for even, uneven and empty blocks (fp64, 1e-12)."""
    r = _rng(9)
    B, S, H, D = 2, 23, 2, 4
    q = r.standard_normal((B, S, H, D))
    k = r.standard_normal((B, S, H, D))
    v = r.standard_normal((B, S, H, D))
    o, lse = attention(q, k, v, 0.5)
    for bounds in ([0, 23], [0, 11, 23], [0, 8, 16, 23], [0, 0, 5, 5, 23], [0, 1, 2, 3, 23], [0, 23, 23]):
        o2, l2, _, _ = ring(q, k, v, 0.5, bounds)
        assert np.allclose(o, o2, rtol=0, atol=1e-12), f"split {bounds}: o"
        assert np.allclose(lse, l2, rtol=0, atol=1e-12), f"split {bounds}: lse"


def pin_usp_equals_unsplit(attention, usp):
    """Unified SP (Ulysses exchange -> ring over each head shard -> inverse exchange) equals
    unsplit attention (fp64, 1e-12): both all-to-alls are pure data movement and the ring
    merge is exact, so every degree and block split must give the same O and LSE."""
    r = _rng(21)
    B, S, H, D = 2, 12, 4, 3
    q, k, v = (r.standard_normal((B, S, H, D)) for _ in range(3))
    o, lse = attention(q, k, v, 0.6)
    for degree, bounds in ((2, [0, 6, 12]), (4, [0, 5, 5, 12]), (2, [0, 12]), (1, [0, 4, 8, 12]), (4, [0, 1, 12])):
        shard = lambda x: x.reshape(B, degree, S // degree, H, D).transpose(1, 0, 2, 3, 4)
        o_sh, l2 = usp(shard(q), shard(k), shard(v), degree, 0.6, bounds)
        o2 = np.asarray(o_sh).transpose(1, 0, 2, 3, 4).reshape(B, S, H, D)
        assert np.allclose(o, o2, rtol=0, atol=1e-12), f"usp {degree} x {bounds}: o"
        assert np.allclose(lse, l2, rtol=0, atol=1e-12), f"usp {degree} x {bounds}: lse"


# --------------------------------------------------------------------------- Ulysses


def _alltoall_messages(src, degree):
    """Message-passing simulation of the first all-to-all.

    Rank p holds its sequence shard ``src[p]`` (``[B, S/P, H, D]``).  It cuts
    the head axis into P groups and sends group q to rank q.  Rank q receives
    one message from every rank and concatenates them in sender order along
    the sequence axis: every token, heads ``[q*H/P, (q+1)*H/P)``.
    """
    P = degree
    H = src.shape[3]
    Hp = H // P
    inbox = [[None] * P for _ in range(P)]          # inbox[receiver][sender]
    for sender in range(P):
        local = src[sender]
        for receiver in range(P):
            inbox[receiver][sender] = local[:, :, receiver * Hp:(receiver + 1) * Hp, :]
    return np.stack([np.concatenate(inbox[q], axis=1) for q in range(P)])


def pin_ulysses_messages(ulysses_fwd):
    """The index map equals a message-passing all-to-all (bit-exact)."""
    r = _rng(10)
    for (P, B, S, H, D) in [(2, 1, 4, 2, 3), (4, 2, 12, 8, 2), (8, 1, 16, 24, 1), (3, 2, 9, 6, 4)]:
        src = r.standard_normal((P, B, S // P, H, D)).astype(np.float32)
        assert np.array_equal(ulysses_fwd(src, P), _alltoall_messages(src, P)), f"ulysses P={P}"


def pin_ulysses_roundtrip(ulysses_fwd, ulysses_inv):
    r = _rng(11)
    src = r.standard_normal((4, 2, 5, 8, 3)).astype(np.float32)
    dst = ulysses_fwd(src, 4)
    assert dst.shape == (4, 2, 20, 2, 3)
    assert np.array_equal(ulysses_inv(dst, 4), src), "ulysses round trip"


def load_golden_ulysses():
    """tests/golden/ulysses_p2_s4_h4.txt: hand-written expected layout (values encode token*10+head)."""
    rows = []
    with open(os.path.join(GOLDEN, "ulysses_p2_s4_h4.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append([int(t) for t in line.split()])
    return rows


def pin_ulysses_golden(ulysses_fwd):
    """P=2, B=1, S=4, H=4, D=1; src value = 10*token + head; compare with the hand-written table."""
    P, S, H = 2, 4, 4
    src = np.zeros((P, 1, S // P, H, 1), dtype=np.int64)
    for p in range(P):
        for sl in range(S // P):
            for h in range(H):
                src[p, 0, sl, h, 0] = 10 * (p * (S // P) + sl) + h
    dst = ulysses_fwd(src, P)
    rows = load_golden_ulysses()       # one row per (rank, token): rank token v_head0 v_head1
    for rank, tok, *vals in rows:
        assert list(dst[rank, 0, tok, :, 0]) == vals, f"golden rank {rank} token {tok}"
    assert len(rows) == P * S


# --------------------------------------------------------------------------- Ulysses Anything

def _near_even(count, parts):
    """Bounds of ``parts`` shards as even as possible, the first ``count % parts`` one longer."""
    base, extra = divmod(count, parts)
    b = [0]
    for p in range(parts):
        b.append(b[-1] + base + (1 if p < extra else 0))
    return b


ANYTHING_CASES = [
    # (S, H, seq_bounds, head_bounds)
    (7, 5, [0, 3, 5, 7], [0, 2, 4, 5]),                  # both uneven, P = 3
    (10, 3, [0, 3, 6, 8, 10], [0, 1, 2, 3, 3]),          # an empty head group, P = 4
    (9, 6, [0, 0, 4, 9], [0, 2, 4, 6]),                  # an empty sequence shard
    (13, 24, _near_even(13, 5), _near_even(24, 5)),      # heads not divisible by 5
    (17, 4, _near_even(17, 4), _near_even(4, 4)),        # FLUX-1008-like: tokens not divisible by 4
]


def pin_anything_origin(ulysses_anything_fwd, ulysses_anything_inv):
    """Every input value encodes its origin (b, s, h, d) exactly in fp64; after the exchange,
    position (b, s, j, d) of head shard q must hold the code of (b, s, head_bounds[q] + j, d),
    computed here by formula, and the inverse must restore every sequence shard."""
    B, D = 2, 3
    code = lambda b, s, h, d: ((b * 100.0 + s) * 100.0 + h) * 10.0 + d
    for S, H, sb, hb in ANYTHING_CASES:
        X = np.fromfunction(code, (B, S, H, D))
        shards = [X[:, sb[p]:sb[p + 1]] for p in range(len(sb) - 1)]
        out = ulysses_anything_fwd(shards, sb, hb)
        for q in range(len(hb) - 1):
            want = np.fromfunction(lambda b, s, j, d: code(b, s, hb[q] + j, d), (B, S, hb[q + 1] - hb[q], D))
            assert np.asarray(out[q]).shape == want.shape and np.array_equal(np.asarray(out[q]), want), (S, H, q)
        back = ulysses_anything_inv(out, sb, hb)
        for p in range(len(sb) - 1):
            assert np.array_equal(np.asarray(back[p]), shards[p]), (S, H, p)


def pin_anything_reduces_to_even(ulysses_anything_fwd, ulysses_fwd):
    """With equal shards the Anything exchange is the (golden-pinned) even exchange."""
    r = _rng(23)
    P, B, S, H, D = 4, 2, 8, 8, 2
    stacked = r.standard_normal((P, B, S // P, H, D))
    even = ulysses_fwd(stacked, P)
    any_ = ulysses_anything_fwd([stacked[p] for p in range(P)], _near_even(S, P), _near_even(H, P))
    for q in range(P):
        assert np.array_equal(np.asarray(any_[q]), np.asarray(even[q]))


# --------------------------------------------------------------------------- Ring Anything gather

def load_golden_gather():
    """tests/golden/ring_anything_gather_s5.txt: hand-written gathered buffer (block, row, value)."""
    rows = []
    with open(os.path.join(GOLDEN, "ring_anything_gather_s5.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(tuple(int(t) for t in line.split()))
    return rows


def pin_gather_golden(ring_anything_gather):
    """B=1, S=5, H=D=1, blocks 2/1/2 padded to 2; token t holds 10*t + 1."""
    x = np.array([10 * t + 1 for t in range(5)], dtype=np.int64).reshape(1, 5, 1, 1)
    out = ring_anything_gather(x, [0, 2, 3, 5], 2)
    rows = load_golden_gather()
    assert np.asarray(out).shape == (3, 1, 2, 1, 1)
    for c, r, val in rows:
        assert int(out[c, 0, r, 0, 0]) == val, f"golden block {c} row {r}"
    assert len(rows) == 3 * 2


def _pad_then_allgather(x, bounds, max_len):
    """The pages' procedure by ranks: rank c holds rows [c_c, c_{c+1}), pads them at the
    end to max_len with zero rows, and the all-gather stacks every rank's padded block."""
    blocks = [x[:, bounds[c]:bounds[c + 1]] for c in range(len(bounds) - 1)]
    padded = [np.pad(blk, ((0, 0), (0, max_len - blk.shape[1]), (0, 0), (0, 0))) for blk in blocks]
    return np.stack(padded)


GATHER_CASES = [
    # (B, S, H, D, bounds, max_len)
    (1, 7, 2, 3, [0, 3, 5, 7], 3),                # uneven
    (2, 9, 3, 2, [0, 0, 4, 9], 5),                # an empty block
    (2, 8, 1, 4, [0, 2, 4, 6, 8], 2),             # even: no padding rows
    (3, 17, 2, 1, [0, 5, 9, 13, 17], 7),          # FLUX-1008-like split, extra padding
]


def pin_gather_per_rank(ring_anything_gather):
    """The index map equals padding on every rank followed by an all-gather (bit-exact)."""
    r = _rng(31)
    for B, S, H, D, bounds, max_len in GATHER_CASES:
        x = r.standard_normal((B, S, H, D)).astype(np.float32)
        assert np.array_equal(np.asarray(ring_anything_gather(x, bounds, max_len)),
                              _pad_then_allgather(x, bounds, max_len)), (B, S, bounds)


def pin_gather_slice_roundtrip(ring_anything_gather, ring_anything_slice):
    """Cutting the gathered blocks back to their true lengths and joining them along the
    sequence restores the input exactly; every padding row is zero."""
    r = _rng(32)
    for B, S, H, D, bounds, max_len in GATHER_CASES:
        x = r.standard_normal((B, S, H, D)) + 3.0  # no zero rows in the data
        g = np.asarray(ring_anything_gather(x, bounds, max_len))
        blocks = ring_anything_slice(g, bounds)
        assert np.array_equal(np.concatenate([np.asarray(b) for b in blocks], axis=1), x), (B, S, bounds)
        for c in range(len(bounds) - 1):
            assert not np.any(g[c, :, bounds[c + 1] - bounds[c]:]), f"padding of block {c} not zero"


def pin_gather_ring_equals_unsplit(attention, merge, ring_anything_gather, ring_anything_slice):
    """Attention over the sliced gathered blocks, merged by LSE, equals unsplit attention
    (fp64, 1e-12): the padding has no numerical effect once sliced off."""
    r = _rng(33)
    B, S, H, D = 2, 11, 2, 4
    q, k, v = (r.standard_normal((B, S, H, D)) for _ in range(3))
    bounds, max_len = [0, 4, 7, 11], 6
    kb = ring_anything_slice(ring_anything_gather(k, bounds, max_len), bounds)
    vb = ring_anything_slice(ring_anything_gather(v, bounds, max_len), bounds)
    parts = [attention(q, kc, vc, 0.7) for kc, vc in zip(kb, vb)]
    o, lse = merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    o_full, lse_full = attention(q, k, v, 0.7)
    assert np.allclose(o, o_full, rtol=0, atol=1e-12) and np.allclose(lse, lse_full, rtol=0, atol=1e-12)
