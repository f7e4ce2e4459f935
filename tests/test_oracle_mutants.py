"""Plant plausible mistakes in the oracle's source and check that a pin catches each one.

Each mutant is the oracle module's own text with one edit (a dropped term, a
wrong sign, index or axis, a swapped operand), executed into a fresh namespace
on the CPU.  A mutant that passes every pin would mean the pins cannot see that
class of mistake.
"""

import os

import pytest

from tests import pins

ORACLE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle")


def _load_mutant(fname, old, new):
    src = open(os.path.join(ORACLE, fname)).read()
    assert src.count(old) == 1, f"mutation anchor not unique/found: {old!r}"
    # The mutant runs outside the package: its relative imports take the (unmutated) oracle.
    src = src.replace("from .attention import", "from oracle.attention import").replace(
        "from .ulysses import", "from oracle.ulysses import")
    ns = {"__name__": "oracle_mutant"}
    exec(compile(src.replace(old, new), f"<mutant {fname}>", "exec"), ns)
    return ns


def _fails(fn):
    try:
        fn()
    except AssertionError:
        return True
    except (ValueError, IndexError, FloatingPointError):
        return True
    return False


ATTN_MUTANTS = [
    ("scale dropped", "s = scale * (qh @ kh.T)", "s = (qh @ kh.T)"),
    ("logit sign flipped", "s = scale * (qh @ kh.T)", "s = -scale * (qh @ kh.T)"),
    ("normaliser summed over queries", "l = e.sum(axis=1)", "l = np.resize(e.sum(axis=0), e.shape[0])"),
    ("keys used as values", "o[b, :, h, :] = (e @ vh) / l[:, None]", "o[b, :, h, :] = (e @ kh) / l[:, None]"),
    ("division by l dropped", "o[b, :, h, :] = (e @ vh) / l[:, None]", "o[b, :, h, :] = (e @ vh)"),
    ("max dropped from lse", "lse[b, h, :] = m + np.log(l)", "lse[b, h, :] = np.log(l)"),
    ("head index mixed", "kh = k[b, :, h, :]          # [Skv, D]", "kh = k[b, :, (h + 1) % H, :]"),
    ("probabilities transposed", "o[b, :, h, :] = (e @ vh) / l[:, None]",
     "o[b, :, h, :] = (np.resize(e.T, e.shape) @ vh) / l[:, None]"),
    ("exp of unscaled logits in the sum", "l = e.sum(axis=1)", "l = np.exp(s).sum(axis=1)"),
]

MERGE_MUTANTS = [
    ("weights not normalised", "np.exp(Ls - np.where(finite, L, 0.0)[None])", "np.exp(Ls - Msafe[None])"),
    ("log-sum term dropped", "L = np.where(finite, Msafe + np.log(tot), -np.inf)", "L = np.where(finite, Msafe, -np.inf)"),
    ("empty block not ignored", "M = Ls.max(axis=0)                                   # [B, H, Sq]",
     "Ls = np.where(np.isneginf(Ls), 0.0, Ls); M = Ls.max(axis=0)"),
    ("block order reversed in weights", "wt = np.transpose(w, (0, 1, 3, 2))[..., None]", "wt = np.transpose(w[::-1], (0, 1, 3, 2))[..., None]"),
]

ULYSSES_MUTANTS = [
    ("head group from owner", "dst[p, :, s, :, :] = src[owner, :, s_local, p * Hp:(p + 1) * Hp, :]",
     "dst[p, :, s, :, :] = src[owner, :, s_local, owner * Hp:(owner + 1) * Hp, :]"),
    ("local index wrong", "owner, s_local = s // Sp, s % Sp  # rank that holds token s before the exchange",
     "owner, s_local = s % P, s // P"),
    ("heads interleaved", "dst[p, :, s, :, :] = src[owner, :, s_local, p * Hp:(p + 1) * Hp, :]",
     "dst[p, :, s, :, :] = src[owner, :, s_local, p::P, :]"),
]


ANYTHING_MUTANTS = [
    ("owner by average shard size", "owner = _owner(seq_bounds, s)", "owner = min(s // -(-S // P), P - 1)"),
    ("head groups by floor split", "hq0, hq1 = int(head_bounds[q]), int(head_bounds[q + 1])\n        shape = (B, S, hq1 - hq0, D)",
     "hq0, hq1 = q * H // P, (q + 1) * H // P\n        shape = (B, S, hq1 - hq0, D)"),
    ("local index from an even stride", "s - int(seq_bounds[owner])", "s - owner * (S // P)"),
]

USP_MUTANTS = [
    ("LSE head groups reversed", "lse = np.concatenate(lses, axis=1)", "lse = np.concatenate(lses[::-1], axis=1)"),
    ("K/V of the first head group everywhere", "o_p, lse_p, _, _ = ring(qh[p], kh[p], vh[p], scale, chunk_bounds)",
     "o_p, lse_p, _, _ = ring(qh[p], kh[0], vh[0], scale, chunk_bounds)"),
    ("keys used as values", "o_p, lse_p, _, _ = ring(qh[p], kh[p], vh[p], scale, chunk_bounds)",
     "o_p, lse_p, _, _ = ring(qh[p], kh[p], kh[p], scale, chunk_bounds)"),
]


GATHER_MUTANTS = [
    ("block start off by one", "out[c, b, r] = x[b, lo + r]", "out[c, b, r] = x[b, min(lo + r + 1, S - 1)]"),
    ("padding in front of the block", "out[c, b, r] = x[b, lo + r]", "out[c, b, max_len - (hi - lo) + r] = x[b, lo + r]"),
    ("blocks gathered in reverse rank order", "out[c, b, r] = x[b, lo + r]", "out[n - 1 - c, b, r] = x[b, lo + r]"),
    ("slice keeps the padding", "gathered[c, :, :bounds[c + 1] - bounds[c]]", "gathered[c]"),
]


@pytest.mark.parametrize("name,old,new", ATTN_MUTANTS, ids=[m[0] for m in ATTN_MUTANTS])
def test_attention_mutant_is_caught(name, old, new):
    ns = _load_mutant("attention.py", old, new)
    caught = [p.__name__ for p in pins.ATTENTION_PINS if _fails(lambda p=p: p(ns["attention"]))]
    caught += ["chunk_merge"] if _fails(lambda: pins.pin_chunk_merge_identity(ns["attention"], ns["ring"])) else []
    assert caught, f"mutant '{name}' passed every pin"


@pytest.mark.parametrize("name,old,new", MERGE_MUTANTS, ids=[m[0] for m in MERGE_MUTANTS])
def test_merge_mutant_is_caught(name, old, new):
    ns = _load_mutant("attention.py", old, new)
    checks = [lambda: pins.pin_merge_closed_form(ns["merge"]), lambda: pins.pin_merge_all_empty(ns["merge"]),
              lambda: pins.pin_merge_large_lse(ns["merge"]),
              lambda: pins.pin_chunk_merge_identity(ns["attention"], ns["ring"])]
    assert any(_fails(c) for c in checks), f"mutant '{name}' passed every pin"


@pytest.mark.parametrize("name,old,new", ULYSSES_MUTANTS, ids=[m[0] for m in ULYSSES_MUTANTS])
def test_ulysses_mutant_is_caught(name, old, new):
    ns = _load_mutant("ulysses.py", old, new)
    checks = [lambda: pins.pin_ulysses_messages(ns["ulysses_fwd"]), lambda: pins.pin_ulysses_golden(ns["ulysses_fwd"]),
              lambda: pins.pin_ulysses_roundtrip(ns["ulysses_fwd"], ns["ulysses_inv"])]
    assert any(_fails(c) for c in checks), f"mutant '{name}' passed every pin"


@pytest.mark.parametrize("name,old,new", USP_MUTANTS, ids=[m[0] for m in USP_MUTANTS])
def test_usp_mutant_is_caught(name, old, new):
    import oracle

    ns = _load_mutant("usp.py", old, new)
    assert _fails(lambda: pins.pin_usp_equals_unsplit(oracle.attention, ns["usp"])), f"mutant '{name}' passed"


@pytest.mark.parametrize("name,old,new", ANYTHING_MUTANTS, ids=[m[0] for m in ANYTHING_MUTANTS])
def test_ulysses_anything_mutant_is_caught(name, old, new):
    import oracle

    ns = _load_mutant("ulysses.py", old, new)
    checks = [lambda: pins.pin_anything_origin(ns["ulysses_anything_fwd"], oracle.ulysses_anything_inv),
              lambda: pins.pin_anything_reduces_to_even(ns["ulysses_anything_fwd"], oracle.ulysses_fwd)]
    assert any(_fails(c) for c in checks), f"mutant '{name}' passed every pin"


@pytest.mark.parametrize("name,old,new", GATHER_MUTANTS, ids=[m[0] for m in GATHER_MUTANTS])
def test_ring_anything_gather_mutant_is_caught(name, old, new):
    import oracle

    ns = _load_mutant("ring_anything.py", old, new)
    checks = [lambda: pins.pin_gather_golden(ns["ring_anything_gather"]),
              lambda: pins.pin_gather_per_rank(ns["ring_anything_gather"]),
              lambda: pins.pin_gather_slice_roundtrip(ns["ring_anything_gather"], ns["ring_anything_slice"]),
              lambda: pins.pin_gather_ring_equals_unsplit(oracle.attention, oracle.merge, ns["ring_anything_gather"],
                                                          ns["ring_anything_slice"])]
    assert any(_fails(c) for c in checks), f"mutant '{name}' passed every pin"
