"""The C ABI on the host: the library loads, exports every declared entry point and
rejects bad arguments before launching anything (no GPU needed)."""

import ctypes
import os
import re

import pytest

from context_attention_dit_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "cpattn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(cp_[a-z0-9_]+)\s*\(", text)))


def test_library_loads_and_exports_header(lib):
    names = declared_functions()
    assert "cp_attn_fwd" in names and "cp_ulysses_permute" in names
    for name in names:
        assert hasattr(lib, name), f"libcpattn.so does not export {name}"
    assert set(binding.EXPORTS) <= set(names)


def test_exported_symbols_in_dynamic_table():
    import subprocess

    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\b(cp_[a-z0-9_]+)\b", out))
    assert set(declared_functions()) <= exported


def test_in_tree_debug_library_is_current():
    """The debug build that travels with the tree exports every declared entry point (a
    stale one would fail only on the GPU)."""
    import subprocess

    from context_attention_dit_b200 import build

    if not os.path.exists(build.LIB_DEBUG):
        pytest.skip("debug library not built")
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB_DEBUG], capture_output=True, text=True).stdout
    assert set(declared_functions()) <= set(re.findall(r"\b(cp_[a-z0-9_]+)\b", out))


def test_sources_compile_and_export_header(tmp_path):
    """The current sources (not only the in-tree binary) build for sm_100a and export every
    declared entry point."""
    import subprocess

    from context_attention_dit_b200 import build

    out = build.build(out=str(tmp_path / "libcpattn_check.so"))
    syms = subprocess.run(["nm", "-D", "--defined-only", out], capture_output=True, text=True).stdout
    assert set(declared_functions()) <= set(re.findall(r"\b(cp_[a-z0-9_]+)\b", syms))


def test_version_and_strings(lib):
    assert lib.cp_version() == 101
    for code in (0, -1, -2, -3, -4, -5, -6, -7):
        assert binding.status_string(code).startswith("CP_")


I = binding


@pytest.mark.parametrize(
    "args,want",
    [
        # q, k, v, out, lse, B, H, Sq, Skv, D, scale, dtype
        ((None, None, None, None, None, 1, 2, 16, 16, 96, 0.1, 0), I.CP_ERR_UNSUPPORTED),   # head_dim
        ((None, None, None, None, None, -1, 2, 16, 16, 64, 0.1, 0), I.CP_ERR_INVALID_ARG),  # negative size
        ((None, None, None, None, None, 1, 2, 16, 16, 64, 0.0, 0), I.CP_ERR_INVALID_ARG),   # scale <= 0
        ((None, None, None, None, None, 1, 2, 16, 16, 64, float("nan"), 0), I.CP_ERR_INVALID_ARG),
        ((None, None, None, None, None, 1, 2, 16, 16, 64, 0.1, 7), I.CP_ERR_INVALID_ARG),   # dtype code
        ((None, None, None, None, None, 1, 2, 16, 16, 64, 0.1, 0), I.CP_ERR_INVALID_ARG),   # null pointers
        ((16, 32, 48, 8, None, 1, 2, 16, 16, 64, 0.1, 0), I.CP_ERR_MISALIGNED),            # out not 16B aligned
        ((None, None, None, None, None, 0, 2, 16, 16, 64, 0.1, 0), I.CP_OK),                # empty batch: no-op
    ],
)
def test_attn_fwd_rejects_before_launch(lib, args, want):
    *ptrs, B, H, Sq, Skv, D, scale, dt = args
    st = lib.cp_attn_fwd(*[ctypes.c_void_p(p) if p else None for p in ptrs], B, H, Sq, Skv, D, scale, dt, None)
    assert st == want


def test_lse_needs_only_float_alignment(lib):
    """LSE arrays are accessed one float at a time: 4-byte alignment is enough (a block's
    LSE slice of an odd-length ring-anything block is not 16-byte aligned)."""
    vp = ctypes.c_void_p
    args = (vp(1 << 20), vp(2 << 20), vp(3 << 20), vp(4 << 20))
    assert lib.cp_attn_fwd(*args, vp((5 << 20) + 2), 1, 2, 16, 16, 64, 0.1, 0, None) == I.CP_ERR_MISALIGNED
    assert lib.cp_attn_fwd(*args, vp((5 << 20) + 4), 1, 2, 16, 16, 64, 0.1, 0, None) != I.CP_ERR_MISALIGNED
    assert lib.cp_attn_merge(vp(1 << 20), vp((2 << 20) + 2), 2, vp(3 << 20), None, 1, 1, 1, 64, 0,
                             None) == I.CP_ERR_MISALIGNED
    assert lib.cp_attn_merge(vp(1 << 20), vp((2 << 20) + 4), 2, vp(3 << 20), vp((4 << 20) + 4), 1, 1, 1, 64, 0,
                             None) != I.CP_ERR_MISALIGNED


def test_merge_rejects(lib):
    assert lib.cp_attn_merge(None, None, 0, None, None, 1, 1, 1, 64, 0, None) == I.CP_ERR_INVALID_ARG
    assert lib.cp_attn_merge(None, None, 65, None, None, 1, 1, 1, 64, 0, None) == I.CP_ERR_UNSUPPORTED
    assert lib.cp_attn_merge(None, None, 2, None, None, 1, 1, 1, 32, 0, None) == I.CP_ERR_UNSUPPORTED
    assert lib.cp_attn_merge(None, None, 2, None, None, 1, 1, 1, 64, 0, None) == I.CP_ERR_INVALID_ARG
    assert lib.cp_attn_merge(ctypes.c_void_p(32), ctypes.c_void_p(64), 2, ctypes.c_void_p(4), None, 1, 1, 1, 64, 0,
                             None) == I.CP_ERR_MISALIGNED


def _bounds(*c):
    return (ctypes.c_int * len(c))(*c)


@pytest.mark.parametrize(
    "bounds,n,skv,want",
    [
        ((0, 8, 16), 2, 16, I.CP_ERR_INVALID_ARG),     # null q etc. after bounds pass
        ((1, 8, 16), 2, 16, I.CP_ERR_INVALID_ARG),     # does not start at 0
        ((0, 8, 15), 2, 16, I.CP_ERR_INVALID_ARG),     # does not end at Skv
        ((0, 9, 8, 16), 3, 16, I.CP_ERR_INVALID_ARG),  # not monotonic
        ((0, 16), 0, 16, I.CP_ERR_INVALID_ARG),        # no blocks
    ],
)
def test_ring_sim_rejects_bad_bounds(lib, bounds, n, skv, want):
    st = lib.cp_ring_sim(None, None, None, _bounds(*bounds), n, None, None, 1, 2, 16, skv, 64, 0.1, 0, None, 0, None)
    assert st == want


def test_ring_sim_rejects_small_workspace(lib):
    # pointers are fake but aligned; the workspace check comes before any CUDA call
    p = ctypes.c_void_p(1 << 20)
    st = lib.cp_ring_sim(p, p, p, _bounds(0, 8, 16), 2, p, None, 1, 2, 16, 16, 64, 0.1, 0, p, 100, None)
    assert st == I.CP_ERR_INVALID_ARG


def test_workspace_size(lib):
    assert binding.ring_workspace_size(1, 1, 24, 4608, 128) == 0
    n, B, H, S, D = 8, 1, 24, 4608, 128
    want = n * B * H * S * D * 4 + n * B * H * S * 4
    assert binding.ring_workspace_size(n, B, H, S, D) == want


def test_usp_sim_checks_before_launch(lib):
    p = ctypes.c_void_p(1 << 20)
    # (degree, S, H, bounds, ws_bytes, want); pointers are fake, every check precedes CUDA
    cases = [
        (3, 16, 6, (0, 16), 1 << 30, I.CP_ERR_NOT_DIVISIBLE),   # S % degree
        (4, 16, 6, (0, 16), 1 << 30, I.CP_ERR_NOT_DIVISIBLE),   # H % degree
        (2, 16, 4, (0, 9, 15), 1 << 30, I.CP_ERR_INVALID_ARG),  # bounds do not span [0, S]
        (2, 16, 4, (0, 8, 16), 100, I.CP_ERR_INVALID_ARG),      # workspace too small
        (0, 16, 4, (0, 16), 1 << 30, I.CP_ERR_INVALID_ARG),     # degree < 1
    ]
    for degree, S, H, b, ws, want in cases:
        st = lib.cp_usp_sim(p, p, p, degree, _bounds(*b), len(b) - 1, p, None, 1, S, H, 64, 0.1, 0, p, ws, None)
        assert st == want, (degree, S, H, b, ws, st)


def test_ulysses_anything_checks_before_launch(lib):
    p = ctypes.c_void_p(1 << 20)
    q = ctypes.c_void_p((1 << 20) + 8)
    ok_s, ok_h = _bounds(0, 3, 5, 7), _bounds(0, 2, 4, 5)
    call = lambda src, dst, deg, sb, hb, eb=2, direction=0: lib.cp_ulysses_anything_permute(
        src, dst, deg, sb, hb, 1, 7, 5, 64, direction, eb, None)
    assert call(p, p, 3, _bounds(0, 3, 5, 6), ok_h) == I.CP_ERR_INVALID_ARG   # does not end at S
    assert call(p, p, 3, ok_s, _bounds(0, 3, 2, 5)) == I.CP_ERR_INVALID_ARG   # decreasing
    assert call(p, p, 3, ok_s, ok_h, eb=8) == I.CP_ERR_UNSUPPORTED
    assert call(p, p, 3, ok_s, ok_h, direction=2) == I.CP_ERR_INVALID_ARG
    assert call(p, p, 3, ok_s, ok_h) == I.CP_ERR_INVALID_ARG                  # src and dst overlap
    assert call(p, q, 3, ok_s, ok_h) == I.CP_ERR_MISALIGNED
    big = list(range(66))
    assert lib.cp_ulysses_anything_permute(p, p, 65, _bounds(*big), _bounds(*big), 1, 65, 65, 64, 0, 2,
                                           None) == I.CP_ERR_UNSUPPORTED        # degree > 64


def test_usp_workspace_size():
    U, n, B, S, H, D = 2, 4, 1, 4608, 24, 128
    elems = B * S * H * D
    ring = binding.ring_workspace_size(n, U * B, H // U, S, D)
    assert binding.usp_workspace_size(U, n, B, S, H, D) == 3 * elems * 2 + elems * 2 + B * H * S * 4 + ring
    assert binding.usp_workspace_size(5, n, B, S, H, D) == 0  # 24 heads are not divisible by 5


def test_ring_bounds():
    assert binding.ring_bounds(4608, 8) == [576 * i for i in range(9)]
    assert binding.ring_bounds(4173, 3, anything=True) == [0, 1391, 2782, 4173]
    assert binding.ring_bounds(4481, 4, anything=True) == [0, 1121, 2241, 3361, 4481]
    with pytest.raises(binding.CpError) as e:
        binding.ring_bounds(4481, 4)
    assert e.value.status == I.CP_ERR_NOT_DIVISIBLE


def test_permute_rejects(lib):
    assert lib.cp_ulysses_permute(None, None, 0, 1, 8, 8, 64, 0, 2, None) == I.CP_ERR_INVALID_ARG
    assert lib.cp_ulysses_permute(None, None, 2, 1, 8, 8, 64, 2, 2, None) == I.CP_ERR_INVALID_ARG
    assert lib.cp_ulysses_permute(None, None, 2, 1, 8, 8, 64, 0, 3, None) == I.CP_ERR_UNSUPPORTED
    assert lib.cp_ulysses_permute(None, None, 3, 1, 8, 9, 64, 0, 2, None) == I.CP_ERR_NOT_DIVISIBLE
    assert lib.cp_ulysses_permute(None, None, 3, 1, 9, 8, 64, 0, 2, None) == I.CP_ERR_NOT_DIVISIBLE
    p = ctypes.c_void_p(1 << 20)
    assert lib.cp_ulysses_permute(p, p, 2, 1, 8, 8, 64, 0, 2, None) == I.CP_ERR_INVALID_ARG  # overlap


def _golden_rows():
    rows = []
    for line in open(os.path.join(ROOT, "tests", "golden", "divisibility_flux.txt")):
        line = line.split("#", 1)[0].strip()
        if line:
            res, tok, heads, variant, deg, want = line.split()
            rows.append((int(res), int(tok), int(heads), variant, int(deg), want))
    return rows


@pytest.mark.parametrize("row", _golden_rows(), ids=lambda r: f"{r[0]}-{r[3]}-{r[4]}")
def test_pages_divisibility_rules(lib, row):
    res, tokens, heads, variant, degree, want = row
    if variant in ("ring", "ring_anything"):
        out = (ctypes.c_int * (degree + 1))()
        st = lib.cp_ring_bounds(tokens, degree, 1 if variant == "ring_anything" else 0, out)
        assert (st == I.CP_OK) == (want == "ok")
        if st == I.CP_OK:
            sizes = [out[i + 1] - out[i] for i in range(degree)]
            assert sum(sizes) == tokens and max(sizes) - min(sizes) <= 1
    else:  # ulysses: null pointers pass the divisibility check and stop at the pointer check
        st = lib.cp_ulysses_permute(None, None, degree, 1, tokens, heads, 128, 0, 2, None)
        assert st == (I.CP_ERR_INVALID_ARG if want == "ok" else I.CP_ERR_NOT_DIVISIBLE)


def test_peer_calls_check_before_cuda(lib):
    """The one-process-per-GPU calls reject bad arguments before any CUDA call."""
    vp = ctypes.c_void_p
    ptr = vp()
    handle = ctypes.create_string_buffer(binding.CP_IPC_HANDLE_BYTES)
    assert lib.cp_peer_alloc(0, ctypes.byref(ptr), handle) == I.CP_ERR_INVALID_ARG
    assert lib.cp_peer_alloc(256, None, handle) == I.CP_ERR_INVALID_ARG
    assert lib.cp_peer_open(None, ctypes.byref(ptr)) == I.CP_ERR_INVALID_ARG
    assert lib.cp_peer_close(None) == I.CP_ERR_INVALID_ARG
    assert lib.cp_peer_free(None) == I.CP_ERR_INVALID_ARG

    src, dsts = (vp * 1)(1 << 20), (vp * 2)(2 << 20, 3 << 20)
    push = lambda s, d, n, rank, deg, B, S, H, D, direc, eb: lib.cp_ulysses_push_n(  # noqa: E731
        s, d, n, rank, deg, B, S, H, D, direc, eb, None)
    assert push(src, dsts, 1, 2, 2, 1, 4, 4, 8, 0, 2) == I.CP_ERR_INVALID_ARG  # rank >= degree
    assert push(src, dsts, 1, -1, 2, 1, 4, 4, 8, 0, 2) == I.CP_ERR_INVALID_ARG
    assert push(src, dsts, 1, 0, 2, 1, 4, 4, 8, 2, 2) == I.CP_ERR_INVALID_ARG  # direction
    assert push(src, dsts, 1, 0, 2, 1, 4, 4, 8, 0, 3) == I.CP_ERR_UNSUPPORTED  # element size
    assert push(src, dsts, 9, 0, 2, 1, 4, 4, 8, 0, 2) == I.CP_ERR_UNSUPPORTED  # tensors
    assert push(src, dsts, 1, 0, 17, 1, 34, 34, 8, 0, 2) == I.CP_ERR_UNSUPPORTED  # ranks
    assert push(src, dsts, 1, 0, 2, 1, 5, 4, 8, 0, 2) == I.CP_ERR_NOT_DIVISIBLE
    assert push(src, dsts, 1, 0, 2, 1, 4, 3, 8, 0, 2) == I.CP_ERR_NOT_DIVISIBLE
    assert push(src, dsts, 1, 0, 2, 0, 4, 4, 8, 0, 2) == I.CP_OK  # empty: nothing to launch
    assert push((vp * 1)((1 << 20) + 1), dsts, 1, 0, 2, 1, 4, 4, 8, 0, 2) == I.CP_ERR_MISALIGNED
    assert push(src, (vp * 2)(2 << 20, (3 << 20) + 2), 1, 0, 2, 1, 4, 4, 8, 0, 4) == I.CP_ERR_MISALIGNED
    assert push(src, (vp * 2)(1 << 20, 3 << 20), 1, 0, 2, 1, 4, 4, 8, 0, 2) == I.CP_ERR_INVALID_ARG  # overlap
    assert push(src, (vp * 2)(2 << 20, 2 << 20), 1, 0, 2, 1, 4, 4, 8, 0, 2) == I.CP_ERR_INVALID_ARG
    assert push(src, (vp * 2)(2 << 20, None), 1, 0, 2, 1, 4, 4, 8, 0, 2) == I.CP_ERR_INVALID_ARG

    pads = (vp * 2)(1 << 20, 2 << 20)
    assert lib.cp_peer_barrier(pads, 2, 2, 1, 0, None) == I.CP_ERR_INVALID_ARG
    assert lib.cp_peer_barrier(None, 0, 2, 1, 0, None) == I.CP_ERR_INVALID_ARG
    assert lib.cp_peer_barrier(pads, 0, 17, 1, 0, None) == I.CP_ERR_UNSUPPORTED
    assert lib.cp_peer_barrier((vp * 2)(1 << 20, None), 0, 2, 1, 0, None) == I.CP_ERR_INVALID_ARG
    assert lib.cp_peer_barrier((vp * 2)(1 << 20, (2 << 20) + 2), 0, 2, 1, 0, None) == I.CP_ERR_MISALIGNED

    fetch = lib.cp_ring_fetch_block
    assert fetch(vp(1 << 20), vp(2 << 20), 1, 5, 2, 8, 4, 0, 8, 0, 2, None) == I.CP_ERR_INVALID_ARG  # past dst
    assert fetch(vp(1 << 20), vp(2 << 20), 1, 5, 2, 8, 8, 0, 8, 4, 2, None) == I.CP_ERR_INVALID_ARG  # past src
    assert fetch(vp(1 << 20), vp(2 << 20), 1, 1, 2, 8, 8, 0, 8, 0, 3, None) == I.CP_ERR_UNSUPPORTED
    assert fetch(vp(1 << 20), vp(1 << 20), 1, 4, 2, 8, 8, 0, 8, 2, 2, None) == I.CP_ERR_INVALID_ARG  # overlap
    assert fetch(None, None, 1, 0, 2, 8, 8, 0, 8, 0, 2, None) == I.CP_OK  # nothing to copy


def test_anything_push_checks_before_cuda(lib):
    vp = ctypes.c_void_p
    src, dsts = (vp * 1)(1 << 20), (vp * 2)(2 << 20, 3 << 20)
    sb, hb = _bounds(0, 3, 5), _bounds(0, 2, 3)
    call = lambda s, d, rank, sbd, hbd, H, direc=0, eb=2: lib.cp_ulysses_anything_push_n(  # noqa: E731
        s, d, 1, rank, 2, sbd, hbd, 1, H, 8, direc, eb, None)
    assert call(src, dsts, 2, sb, hb, 3) == I.CP_ERR_INVALID_ARG  # rank >= degree
    assert call(src, dsts, 0, None, hb, 3) == I.CP_ERR_INVALID_ARG
    assert call(src, dsts, 0, _bounds(1, 3, 5), hb, 3) == I.CP_ERR_INVALID_ARG  # bounds must start at 0
    assert call(src, dsts, 0, _bounds(0, 4, 3), hb, 3) == I.CP_ERR_INVALID_ARG  # decreasing
    assert call(src, dsts, 0, sb, hb, 4) == I.CP_ERR_INVALID_ARG  # head bounds must end at H
    assert call(src, dsts, 0, sb, hb, 3, 2) == I.CP_ERR_INVALID_ARG  # direction
    assert call(src, dsts, 0, sb, hb, 3, 0, 3) == I.CP_ERR_UNSUPPORTED
    assert call(src, dsts, 0, _bounds(0, 0, 5), hb, 3) == I.CP_OK  # this rank holds no tokens: nothing to push
    assert call(src, dsts, 1, sb, _bounds(0, 3, 3), 3, 1) == I.CP_OK  # this rank holds no heads
    assert call((vp * 1)((1 << 20) + 1), dsts, 0, sb, hb, 3) == I.CP_ERR_MISALIGNED
    assert call(src, (vp * 2)(1 << 20, 3 << 20), 0, sb, hb, 3) == I.CP_ERR_INVALID_ARG  # overlap
    assert call(src, (vp * 2)(None, 3 << 20), 0, sb, hb, 3) == I.CP_ERR_INVALID_ARG
    assert lib.cp_ulysses_anything_push_n(src, dsts, 1, 0, 17, sb, hb, 1, 3, 8, 0, 2, None) == I.CP_ERR_UNSUPPORTED


def test_merge_push_checks_before_cuda(lib):
    vp = ctypes.c_void_p
    outs = (vp * 2)(3 << 20, 4 << 20)
    call = lambda parts, outs_, shard, deg, S, H, D=64, n=2, dt=0: lib.cp_attn_merge_push(  # noqa: E731
        parts, vp(2 << 20), n, outs_, shard, deg, 1, S, H, D, dt, None)
    assert call(vp(1 << 20), outs, 2, 2, 8, 4) == I.CP_ERR_INVALID_ARG  # shard >= degree
    assert call(vp(1 << 20), outs, 0, 17, 34, 34) == I.CP_ERR_UNSUPPORTED
    assert call(vp(1 << 20), outs, 0, 2, 7, 4) == I.CP_ERR_NOT_DIVISIBLE
    assert call(vp(1 << 20), outs, 0, 2, 8, 3) == I.CP_ERR_NOT_DIVISIBLE
    assert call(vp(1 << 20), outs, 0, 2, 8, 4, D=96) == I.CP_ERR_UNSUPPORTED
    assert call(vp(1 << 20), outs, 0, 2, 8, 4, n=0) == I.CP_ERR_INVALID_ARG
    assert call(vp(1 << 20), outs, 0, 2, 8, 4, dt=5) == I.CP_ERR_INVALID_ARG
    assert call(vp((1 << 20) + 4), outs, 0, 2, 8, 4) == I.CP_ERR_MISALIGNED
    assert call(vp(1 << 20), (vp * 2)(3 << 20, (4 << 20) + 8), 0, 2, 8, 4) == I.CP_ERR_MISALIGNED
    assert call(vp(1 << 20), (vp * 2)(3 << 20, None), 0, 2, 8, 4) == I.CP_ERR_INVALID_ARG
    assert call(None, None, 0, 2, 0, 4) == I.CP_OK  # empty


def test_anything_permute_n_checks_before_cuda(lib):
    vp = ctypes.c_void_p
    sb, hb = _bounds(0, 3, 5), _bounds(0, 2, 3)
    srcs, dsts = (vp * 2)(1 << 20, 2 << 20), (vp * 2)(3 << 20, 4 << 20)
    call = lambda s, d, n, sbd=sb, hbd=hb, S=5, H=3: lib.cp_ulysses_anything_permute_n(  # noqa: E731
        s, d, n, 2, sbd, hbd, 1, S, H, 8, 0, 2, None)
    assert call(srcs, dsts, 0) == I.CP_ERR_INVALID_ARG
    assert call(srcs, dsts, 9) == I.CP_ERR_UNSUPPORTED
    assert call(srcs, dsts, 2, S=6) == I.CP_ERR_INVALID_ARG  # seq bounds must end at S
    assert call(srcs, (vp * 2)(3 << 20, 3 << 20), 2) == I.CP_ERR_INVALID_ARG  # destinations overlap
    assert call(srcs, (vp * 2)(3 << 20, 1 << 20), 2) == I.CP_ERR_INVALID_ARG  # a destination on a source
    assert call(srcs, (vp * 2)(3 << 20, (4 << 20) + 8), 2) == I.CP_ERR_MISALIGNED
    assert call(srcs, (vp * 2)(3 << 20, None), 2) == I.CP_ERR_INVALID_ARG
    assert call(srcs, dsts, 2, S=0, sbd=_bounds(0, 0, 0)) == I.CP_OK  # empty


def test_peer_bindings_reject_bad_arguments_before_the_library():
    import torch

    with pytest.raises(ValueError):
        binding.peer_open(b"\0" * 10)  # an IPC handle has 64 bytes
    with pytest.raises(ValueError):
        binding.ulysses_push_n([1 << 20], [[2 << 20]], 0, 2, 1, 4, 4, 8, 0, 2, 0)  # one row of 1 != degree 2
    with pytest.raises(ValueError):
        binding.ulysses_push_n([1 << 20, 2 << 20], [[3 << 20, 4 << 20]], 0, 2, 1, 4, 4, 8, 0, 2, 0)  # rows != sources
    with pytest.raises(ValueError):
        binding.ulysses_anything_push_n([1 << 20], [[2 << 20, 3 << 20]], 0, [0, 2, 4], [0, 2], 1, 2, 8, 0, 2, 0)
    with pytest.raises(ValueError):  # host tensors never reach the library
        binding.attn_merge_push(torch.zeros(1, 1, 4, 1, 64), torch.zeros(1, 1, 1, 4), [1 << 20, 2 << 20], 0)
    with pytest.raises(ValueError):
        binding.ulysses_anything_permute_n([torch.zeros(8)], 2, [0, 1, 2], [0, 1, 2], 1, 2, 2, 2, 0)


def test_attn_fwd_strided_checks_before_cuda(lib):
    """Strides and the output's row layout are checked on the host, before any CUDA call."""
    vp = ctypes.c_void_p
    q, k, v, o = vp(1 << 20), vp(2 << 20), vp(3 << 20), vp(4 << 20)
    B, H, S, D = 2, 3, 16, 64
    row = H * D

    def call(q_sb=S * row, q_ss=row, kv_sb=S * row, kv_ss=row, o_sb=S * row, o_ss=row, dt=0, b=B):
        return lib.cp_attn_fwd_strided(q, k, v, o, None, b, H, S, S, D, q_sb, q_ss, kv_sb, kv_ss, o_sb, o_ss, 0.1,
                                       dt, None)

    assert call(q_ss=0) == I.CP_ERR_INVALID_ARG
    assert call(kv_sb=-8) == I.CP_ERR_INVALID_ARG
    assert call(o_ss=-row) == I.CP_ERR_INVALID_ARG
    assert call(q_ss=row + 4) == I.CP_ERR_MISALIGNED                  # TMA: 16-byte strides
    assert call(kv_sb=S * row + 4) == I.CP_ERR_MISALIGNED
    assert call(o_ss=row + 4) == I.CP_ERR_MISALIGNED                  # bf16 rows on 16-byte bounds
    assert call(o_ss=row + 4, dt=1) != I.CP_ERR_MISALIGNED            # fp32: 4 elements are 16 bytes
    assert call(q_ss=1 << 39) == I.CP_ERR_UNSUPPORTED
    assert call(o_ss=row - 8) == I.CP_ERR_INVALID_ARG                 # output rows overlap
    assert call(o_sb=row * 4) == I.CP_ERR_INVALID_ARG                 # batches overlap along the sequence
    # An interleaved output (the sequence outermost, batches side by side) passes the checks
    # and reaches CUDA, which is absent here: CP_ERR_CUDA, not an argument error.
    assert call(o_sb=row, o_ss=B * row) not in (I.CP_ERR_INVALID_ARG, I.CP_ERR_MISALIGNED, I.CP_ERR_UNSUPPORTED)
    assert call(o_sb=0, b=1) not in (I.CP_ERR_INVALID_ARG, I.CP_ERR_MISALIGNED)  # batch stride unused for B = 1
    assert lib.cp_attn_fwd_strided(None, None, None, None, None, 0, H, S, S, D, 0, 0, 0, 0, 0, 0, 0.1, 0,
                                   None) == I.CP_OK                   # empty batch: nothing to do


def test_ring_sim_fused_ulysses_checks_before_cuda(lib):
    p = ctypes.c_void_p(1 << 20)
    call = lambda deg, S, H, b: lib.cp_ring_sim_fused_ulysses(  # noqa: E731
        p, p, p, deg, _bounds(*b), len(b) - 1, p, None, 1, S, H, 64, 0.1, 0, None)
    assert call(3, 16, 6, (0, 16)) == I.CP_ERR_NOT_DIVISIBLE    # S % degree
    assert call(4, 16, 6, (0, 16)) == I.CP_ERR_NOT_DIVISIBLE    # H % degree
    assert call(2, 16, 4, (0, 9, 15)) == I.CP_ERR_INVALID_ARG   # bounds do not span [0, S]
    assert call(0, 16, 4, (0, 16)) == I.CP_ERR_INVALID_ARG


def test_ring_anything_gather_checks_before_cuda(lib):
    vp = ctypes.c_void_p
    srcs, dsts = (vp * 2)(1 << 20, 2 << 20), (vp * 2)(3 << 20, 4 << 20)
    call = lambda s, d, n, b, max_len, eb=2: lib.cp_ring_anything_gather(  # noqa: E731
        s, d, n, _bounds(*b), len(b) - 1, max_len, 1, b[-1], 2, 8, eb, None)
    assert call(srcs, dsts, 2, (0, 3, 5), 2) == I.CP_ERR_INVALID_ARG      # max_len below the longest block
    assert call(srcs, dsts, 2, (0, 3, 2, 5), 3) == I.CP_ERR_INVALID_ARG   # decreasing bounds
    assert call(srcs, dsts, 2, (0, 3, 5), 3, eb=8) == I.CP_ERR_UNSUPPORTED
    assert call(srcs, dsts, 9, (0, 3, 5), 3) == I.CP_ERR_UNSUPPORTED      # more than 8 tensors
    assert call(srcs, dsts, 0, (0, 3, 5), 3) == I.CP_ERR_INVALID_ARG
    assert call(srcs, (vp * 2)(3 << 20, 1 << 20), 2, (0, 3, 5), 3) == I.CP_ERR_INVALID_ARG  # dst on a source
    assert call(srcs, (vp * 2)(3 << 20, 3 << 20), 2, (0, 3, 5), 3) == I.CP_ERR_INVALID_ARG  # dsts overlap
    assert call(srcs, (vp * 2)(3 << 20, (4 << 20) + 8), 2, (0, 3, 5), 3) == I.CP_ERR_MISALIGNED
    assert call(srcs, dsts, 2, (0, 0, 0), 0) == I.CP_OK                   # no rows: nothing to copy


def test_new_bindings_reject_bad_outputs_before_the_library():
    """The Python side of the strided, fused-Ulysses and gather calls checks the tensors it
    is given (host tensors and wrong shapes never reach the library)."""
    import torch

    with pytest.raises(ValueError):
        binding.attn_fwd_strided(torch.zeros(1, 4, 2, 64, dtype=torch.bfloat16), torch.zeros(1, 4, 2, 64, dtype=torch.bfloat16),
                                 torch.zeros(1, 4, 2, 64, dtype=torch.bfloat16))  # host tensors
    with pytest.raises(ValueError):
        binding.ring_sim_fused_ulysses(*(torch.zeros(2, 1, 8, 2, 64, dtype=torch.bfloat16) for _ in range(3)), 2, [0, 8])
    with pytest.raises(ValueError):
        binding.ring_anything_gather([torch.zeros(1, 5, 1, 8, dtype=torch.bfloat16)], [0, 2, 5])  # host source
