"""Thin ctypes binding of libcpattn.so (argument marshalling only).

Torch tensors supply device memory and the current stream; every step of the
computation runs in the library's CUDA kernels.  The binding checks what the
C ABI cannot see, mirroring the attention dispatcher's checks ("Attention
backends", section "Checks": query/key/value on one device, matching dtypes,
usually bfloat16, and valid shapes) and raises ``ValueError``.  A non-OK status
from the library raises ``RuntimeError`` with the status name.  There is no
fallback: if the library is missing or fails to load, every call raises.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# The debug build (libcpattn_debug.so, device-side bounds checks) is selected with
# CPATTN_LIB=debug; any other value is taken as a path.
_lib_env = os.environ.get("CPATTN_LIB", "")
LIB_PATH = (os.path.join(_PKG, "libcpattn_debug.so") if _lib_env == "debug"
            else _lib_env or os.path.join(_PKG, "libcpattn.so"))

CP_OK = 0
CP_ERR_INVALID_ARG = -1
CP_ERR_UNSUPPORTED = -2
CP_ERR_NOT_DIVISIBLE = -3
CP_ERR_MISALIGNED = -4
CP_ERR_CUDA = -5
CP_ERR_TIMEOUT = -6
CP_ERR_BOUNDS = -7
CP_BF16 = 0
CP_F32 = 1
CP_MAX_CHUNKS = 64

EXPORTS = (
    "cp_attn_fwd", "cp_attn_fwd_blocks", "cp_attn_merge", "cp_ring_sim_workspace_size", "cp_ring_sim",
    "cp_ring_sim_fused", "cp_ring_sim_static", "cp_ulysses_permute", "cp_ulysses_permute_n", "cp_ring_bounds",
    "cp_debug_set_fault", "cp_last_device_status", "cp_status_string", "cp_version", "cp_usp_sim_workspace_size",
    "cp_usp_sim", "cp_ulysses_anything_permute", "cp_attn_merge_ulysses", "cp_peer_alloc", "cp_peer_open",
    "cp_peer_close", "cp_peer_free", "cp_ulysses_push_n", "cp_peer_barrier", "cp_ring_fetch_block",
    "cp_ulysses_anything_push_n", "cp_attn_merge_push", "cp_ulysses_anything_permute_n", "cp_attn_fwd_strided",
    "cp_ring_sim_fused_ulysses", "cp_ring_anything_gather",
)
CP_PEER_MAX = 16
CP_IPC_HANDLE_BYTES = 64

_lib = None


class CpError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def load() -> ctypes.CDLL:
    """Load libcpattn.so (built in-tree); raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libcpattn.so not built at {LIB_PATH}; run python -m context_attention_dit_b200.build")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    ip = ctypes.POINTER(ctypes.c_int)
    lib.cp_attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp]
    ll = ctypes.c_longlong
    lib.cp_attn_fwd_strided.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, ll, ll, ll, ll, ll, ll, f, i, vp]
    lib.cp_attn_fwd_strided.restype = ctypes.c_int
    lib.cp_ring_sim_fused_ulysses.argtypes = [vp, vp, vp, i, ip, i, vp, vp, i, i, i, i, f, i, vp]
    lib.cp_ring_sim_fused_ulysses.restype = ctypes.c_int
    lib.cp_ring_anything_gather.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(vp), i, ip, i, i, i, i, i, i, i, vp]
    lib.cp_ring_anything_gather.restype = ctypes.c_int
    lib.cp_attn_fwd_blocks.argtypes = [vp, vp, vp, ip, i, vp, vp, i, i, i, i, i, f, vp]
    lib.cp_attn_merge.argtypes = [vp, vp, i, vp, vp, i, i, i, i, i, vp]
    lib.cp_attn_merge_ulysses.argtypes = [vp, vp, i, vp, vp, i, i, i, i, i, i, vp]
    lib.cp_ring_sim_workspace_size.argtypes = [i, i, i, i, i]
    lib.cp_ring_sim_workspace_size.restype = sz
    lib.cp_ring_sim.argtypes = [vp, vp, vp, ip, i, vp, vp, i, i, i, i, i, f, i, vp, sz, vp]
    lib.cp_ring_sim_fused.argtypes = [vp, vp, vp, ip, i, vp, vp, i, i, i, i, i, f, i, vp]
    lib.cp_usp_sim_workspace_size.argtypes = [i, i, i, i, i, i, i]
    lib.cp_usp_sim_workspace_size.restype = sz
    lib.cp_usp_sim.argtypes = [vp, vp, vp, i, ip, i, vp, vp, i, i, i, i, f, i, vp, sz, vp]
    lib.cp_ring_sim_fused.restype = ctypes.c_int
    lib.cp_ring_sim_static.argtypes = [vp, vp, vp, ip, i, vp, vp, i, i, i, i, i, f, i, vp]
    lib.cp_ulysses_permute.argtypes = [vp, vp, i, i, i, i, i, i, i, vp]
    lib.cp_ulysses_anything_permute.argtypes = [vp, vp, i, ip, ip, i, i, i, i, i, i, vp]
    lib.cp_ulysses_anything_permute_n.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(vp), i, i, ip, ip, i, i, i, i, i,
                                                  i, vp]
    lib.cp_ulysses_anything_permute_n.restype = ctypes.c_int
    lib.cp_ulysses_permute_n.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(vp), i, i, i, i, i, i, i, i, vp]
    lib.cp_ulysses_permute_n.restype = ctypes.c_int
    lib.cp_ring_bounds.argtypes = [i, i, i, ip]
    lib.cp_peer_alloc.argtypes = [sz, ctypes.POINTER(vp), ctypes.c_char_p]
    lib.cp_peer_open.argtypes = [ctypes.c_char_p, ctypes.POINTER(vp)]
    lib.cp_peer_close.argtypes = [vp]
    lib.cp_peer_free.argtypes = [vp]
    lib.cp_ulysses_push_n.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(vp), i, i, i, i, i, i, i, i, i, vp]
    lib.cp_ulysses_anything_push_n.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(vp), i, i, i, ip, ip, i, i, i, i,
                                                i, vp]
    lib.cp_ulysses_anything_push_n.restype = ctypes.c_int
    lib.cp_attn_merge_push.argtypes = [vp, vp, i, ctypes.POINTER(vp), i, i, i, i, i, i, i, vp]
    lib.cp_attn_merge_push.restype = ctypes.c_int
    lib.cp_peer_barrier.argtypes = [ctypes.POINTER(vp), i, i, ctypes.c_uint, ctypes.c_uint, vp]
    lib.cp_ring_fetch_block.argtypes = [vp, vp, i, i, i, i, i, i, i, i, i, vp]
    lib.cp_debug_set_fault.argtypes = [i]
    lib.cp_debug_set_fault.restype = ctypes.c_int
    lib.cp_last_device_status.argtypes = [vp]
    lib.cp_status_string.argtypes = [i]
    lib.cp_status_string.restype = ctypes.c_char_p
    lib.cp_version.argtypes = []
    for name in ("cp_attn_fwd", "cp_attn_fwd_blocks", "cp_attn_merge", "cp_ring_sim", "cp_ring_sim_static", "cp_ulysses_permute",
                 "cp_ring_bounds", "cp_last_device_status", "cp_peer_alloc", "cp_peer_open", "cp_peer_close",
                 "cp_peer_free", "cp_ulysses_push_n", "cp_peer_barrier", "cp_ring_fetch_block"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().cp_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != CP_OK:
        raise CpError(status, where)


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _out_code(dtype) -> int:
    if dtype == torch.bfloat16:
        return CP_BF16
    if dtype == torch.float32:
        return CP_F32
    raise ValueError(f"output dtype must be bfloat16 or float32, got {dtype}")


def _check_qkv(q, k, v):
    for name, t in (("query", q), ("key", k), ("value", v)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if t.dtype != torch.bfloat16:
            raise ValueError(f"{name} must be bfloat16, got {t.dtype}")
        if t.dim() != 4:
            raise ValueError(f"{name} must be 4-D (batch, seq, heads, head_dim), got {tuple(t.shape)}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous (BSHD)")
    if not (q.device == k.device == v.device):
        raise ValueError("query, key and value must be on the same device")
    B, Sq, H, D = q.shape
    if k.shape != v.shape or k.shape[0] != B or k.shape[2] != H or k.shape[3] != D:
        raise ValueError(f"incompatible shapes q{tuple(q.shape)} k{tuple(k.shape)} v{tuple(v.shape)}")
    return B, Sq, k.shape[1], H, D


def attn_fwd(q, k, v, scale: Optional[float] = None, out_dtype=torch.bfloat16, out=None, lse=None,
             want_lse: bool = True):
    """Attention of q over one K/V block; returns ``(out [B,Sq,H,D], lse [B,H,Sq] fp32)``."""
    B, Sq, Skv, H, D = _check_qkv(q, k, v)
    code = _out_code(out_dtype)
    scale = float(D ** -0.5 if scale is None else scale)
    if out is None:
        out = torch.empty((B, Sq, H, D), dtype=out_dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    st = load().cp_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Sq, Skv, D, scale, code,
                            ctypes.c_void_p(_stream(q)))
    _check(st, "cp_attn_fwd")
    return out, lse


def _check_view(name: str, t, D: Optional[int] = None):
    """A 4-D bf16 CUDA view whose heads and head_dim are dense (strides (., ., D, 1))."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dim() != 4:
        raise ValueError(f"{name} must be 4-D (batch, seq, heads, head_dim), got {tuple(t.shape)}")
    d = t.shape[3]
    if t.stride(3) != 1 or (t.shape[2] > 1 and t.stride(2) != d):
        raise ValueError(f"{name}: heads and head_dim must be dense (strides (., ., {d}, 1)), got {t.stride()}")
    return t.stride(0), t.stride(1)


def attn_fwd_strided(q, k, v, scale: Optional[float] = None, out_dtype=torch.bfloat16, out=None, lse=None,
                     want_lse: bool = True):
    """:func:`attn_fwd` on views: q, k, v (and ``out`` if given) may be slices of larger
    tensors along batch and sequence (e.g. ``k_full[:, c0:c1]``), with heads and head_dim
    dense.  Returns ``(out, lse)``; ``lse`` is dense ``[B, H, Sq]``."""
    for name, t in (("query", q), ("key", k), ("value", v)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16:
            raise ValueError(f"{name} must be a bfloat16 tensor")
    q_sb, q_ss = _check_view("query", q)
    kv_sb, kv_ss = _check_view("key", k)
    if _check_view("value", v) != (kv_sb, kv_ss):
        raise ValueError("key and value must have the same strides")
    if not (q.device == k.device == v.device):
        raise ValueError("query, key and value must be on the same device")
    B, Sq, H, D = q.shape
    Skv = k.shape[1]
    if k.shape != v.shape or k.shape[0] != B or k.shape[2] != H or k.shape[3] != D:
        raise ValueError(f"incompatible shapes q{tuple(q.shape)} k{tuple(k.shape)} v{tuple(v.shape)}")
    code = _out_code(out_dtype)
    scale = float(D ** -0.5 if scale is None else scale)
    if out is None:
        out = torch.empty((B, Sq, H, D), dtype=out_dtype, device=q.device)
    if out.dtype != out_dtype or tuple(out.shape) != (B, Sq, H, D) or out.device != q.device:
        raise ValueError(f"out must be {out_dtype} of shape {(B, Sq, H, D)} on {q.device}")
    o_sb, o_ss = _check_view("out", out)
    if lse is None and want_lse:
        lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    if lse is not None and (lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, Sq) or not lse.is_contiguous()
                            or lse.device != q.device):
        raise ValueError(f"lse must be a contiguous float32 tensor of shape {(B, H, Sq)}")
    st = load().cp_attn_fwd_strided(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Sq, Skv, D, q_sb, q_ss,
                                    kv_sb, kv_ss, o_sb, o_ss, scale, code, ctypes.c_void_p(_stream(q)))
    _check(st, "cp_attn_fwd_strided")
    return out, lse


def attn_fwd_blocks(q, k, v, chunk_bounds: Sequence[int], scale: Optional[float] = None, partials=None,
                    lses=None):
    """Attention of q over each K/V block ``[c_r, c_{r+1})`` in one launch (no merge).

    Returns fp32 ``(partials [n,B,Sq,H,D], lses [n,B,H,Sq])``, the inputs of :func:`attn_merge`.
    """
    B, Sq, Skv, H, D = _check_qkv(q, k, v)
    scale = float(D ** -0.5 if scale is None else scale)
    n = len(chunk_bounds) - 1
    if n < 1:
        raise ValueError("chunk_bounds needs at least two entries")
    bounds = (ctypes.c_int * (n + 1))(*[int(c) for c in chunk_bounds])
    if partials is None:
        partials = torch.empty((n, B, Sq, H, D), dtype=torch.float32, device=q.device)
    if lses is None:
        lses = torch.empty((n, B, H, Sq), dtype=torch.float32, device=q.device)
    st = load().cp_attn_fwd_blocks(_ptr(q), _ptr(k), _ptr(v), bounds, n, _ptr(partials), _ptr(lses), B, H, Sq, Skv,
                                   D, scale, ctypes.c_void_p(_stream(q)))
    _check(st, "cp_attn_fwd_blocks")
    return partials, lses


def attn_merge(partials, lses, out_dtype=torch.bfloat16, out=None, out_lse=None):
    """Merge fp32 partials ``[n,B,Sq,H,D]`` with LSEs ``[n,B,H,Sq]``; returns ``(out, lse)``."""
    if partials.dtype != torch.float32 or lses.dtype != torch.float32:
        raise ValueError("partials and lses must be float32")
    if not (partials.is_cuda and lses.is_cuda) or partials.device != lses.device:
        raise ValueError("partials and lses must be CUDA tensors on one device")
    if not (partials.is_contiguous() and lses.is_contiguous()):
        raise ValueError("partials and lses must be contiguous")
    n, B, Sq, H, D = partials.shape
    if tuple(lses.shape) != (n, B, H, Sq):
        raise ValueError(f"lses shape {tuple(lses.shape)} != {(n, B, H, Sq)}")
    code = _out_code(out_dtype)
    if out is None:
        out = torch.empty((B, Sq, H, D), dtype=out_dtype, device=partials.device)
    if out_lse is None:
        out_lse = torch.empty((B, H, Sq), dtype=torch.float32, device=partials.device)
    st = load().cp_attn_merge(_ptr(partials), _ptr(lses), n, _ptr(out), _ptr(out_lse), B, H, Sq, D, code,
                              ctypes.c_void_p(_stream(partials)))
    _check(st, "cp_attn_merge")
    return out, out_lse


def ring_workspace_size(n_chunks: int, B: int, H: int, Sq: int, D: int) -> int:
    return int(load().cp_ring_sim_workspace_size(n_chunks, B, H, Sq, D))


def attn_merge_ulysses(partials, lses, degree: int, out_dtype=torch.bfloat16, out=None, out_lse=None):
    """Merge of Ulysses head-shard partials ``[n, degree*B, S, H/degree, D]`` (LSEs ``[n,
    degree*B, H/degree, S]``) fused with the inverse exchange: returns ``(out [degree, B,
    S/degree, H, D], lse [B, H, S])``, identical to :func:`attn_merge` then the inverse
    :func:`ulysses_permute`."""
    if partials.dtype != torch.float32 or lses.dtype != torch.float32:
        raise ValueError("partials and lses must be float32")
    if not (partials.is_cuda and lses.is_cuda and partials.is_contiguous() and lses.is_contiguous()):
        raise ValueError("partials and lses must be contiguous CUDA tensors")
    n, PB, S, Hp, D = partials.shape
    if PB % degree != 0 or lses.shape != (n, PB, Hp, S):
        raise ValueError(f"incompatible shapes partials{tuple(partials.shape)} lses{tuple(lses.shape)}")
    B, H = PB // degree, Hp * degree
    code = _out_code(out_dtype)
    if out is None:
        out = torch.empty((degree, B, S // degree, H, D), dtype=out_dtype, device=partials.device)
    if out_lse is None:
        out_lse = torch.empty((B, H, S), dtype=torch.float32, device=partials.device)
    st = load().cp_attn_merge_ulysses(_ptr(partials), _ptr(lses), n, _ptr(out), _ptr(out_lse), degree, B, S, H, D, code,
                                      ctypes.c_void_p(_stream(partials)))
    _check(st, "cp_attn_merge_ulysses")
    return out, out_lse


def ring_sim(q, k, v, chunk_bounds: Sequence[int], scale: Optional[float] = None, out_dtype=torch.bfloat16,
             workspace=None, out=None, out_lse=None):
    """Ring / ring-anything attention over K/V blocks ``[c_r, c_{r+1})``; returns ``(out, lse, workspace)``."""
    B, Sq, Skv, H, D = _check_qkv(q, k, v)
    code = _out_code(out_dtype)
    scale = float(D ** -0.5 if scale is None else scale)
    n = len(chunk_bounds) - 1
    if n < 1:
        raise ValueError("chunk_bounds needs at least two entries")
    bounds = (ctypes.c_int * (n + 1))(*[int(c) for c in chunk_bounds])
    need = ring_workspace_size(n, B, H, Sq, D)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if out is None:
        out = torch.empty((B, Sq, H, D), dtype=out_dtype, device=q.device)
    if out_lse is None:
        out_lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    st = load().cp_ring_sim(_ptr(q), _ptr(k), _ptr(v), bounds, n, _ptr(out), _ptr(out_lse), B, H, Sq, Skv, D, scale,
                            code, _ptr(workspace), ws_bytes, ctypes.c_void_p(_stream(q)))
    _check(st, "cp_ring_sim")
    return out, out_lse, workspace


def usp_workspace_size(degree: int, n_chunks: int, B: int, S: int, H: int, D: int, out_dtype=torch.bfloat16) -> int:
    return int(load().cp_usp_sim_workspace_size(degree, n_chunks, B, S, H, D, _out_code(out_dtype)))


def usp_sim(q, k, v, degree: int, chunk_bounds: Sequence[int], scale: Optional[float] = None,
            out_dtype=torch.bfloat16, workspace=None, out=None, out_lse=None):
    """Ulysses (``degree``) x ring (``chunk_bounds`` over the whole sequence) attention.

    q, k, v: sequence-sharded ``[degree, B, S/degree, H, D]`` bf16 (shard p = tokens
    ``[p*S/degree, (p+1)*S/degree)``).  Returns ``(out, lse, workspace)``: out in the same
    layout, lse ``[B, H, S]`` fp32.
    """
    for name, t in (("query", q), ("key", k), ("value", v)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.bfloat16 or t.dim() != 5:
            raise ValueError(f"{name} must be a 5-D bf16 CUDA tensor [degree, B, S/degree, H, D]")
        if not t.is_contiguous() or t.shape != q.shape or t.device != q.device:
            raise ValueError("query, key and value must be contiguous, of one shape, on one device")
    P, B, Sp, H, D = q.shape
    if P != degree:
        raise ValueError(f"leading dimension {P} != degree {degree}")
    S = P * Sp
    code = _out_code(out_dtype)
    scale = float(D ** -0.5 if scale is None else scale)
    n = len(chunk_bounds) - 1
    if n < 1:
        raise ValueError("chunk_bounds needs at least two entries")
    bounds = (ctypes.c_int * (n + 1))(*[int(c) for c in chunk_bounds])
    need = usp_workspace_size(degree, n, B, S, H, D, out_dtype)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
    if out_lse is None:
        out_lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    st = load().cp_usp_sim(_ptr(q), _ptr(k), _ptr(v), degree, bounds, n, _ptr(out), _ptr(out_lse), B, S, H, D, scale,
                           code, _ptr(workspace), ws_bytes, ctypes.c_void_p(_stream(q)))
    _check(st, "cp_usp_sim")
    return out, out_lse, workspace


def ring_sim_fused(q, k, v, chunk_bounds: Sequence[int], scale: Optional[float] = None, out_dtype=torch.bfloat16,
                   out=None, out_lse=None):
    """Ring attention over K/V blocks with the LSE merge fused into the kernel; returns ``(out, lse)``."""
    B, Sq, Skv, H, D = _check_qkv(q, k, v)
    code = _out_code(out_dtype)
    scale = float(D ** -0.5 if scale is None else scale)
    n = len(chunk_bounds) - 1
    if n < 1:
        raise ValueError("chunk_bounds needs at least two entries")
    bounds = (ctypes.c_int * (n + 1))(*[int(c) for c in chunk_bounds])
    if out is None:
        out = torch.empty((B, Sq, H, D), dtype=out_dtype, device=q.device)
    if out_lse is None:
        out_lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    st = load().cp_ring_sim_fused(_ptr(q), _ptr(k), _ptr(v), bounds, n, _ptr(out), _ptr(out_lse), B, H, Sq, Skv, D,
                                  scale, code, ctypes.c_void_p(_stream(q)))
    _check(st, "cp_ring_sim_fused")
    return out, out_lse


def ring_sim_fused_ulysses(q, k, v, degree: int, chunk_bounds: Sequence[int], scale: Optional[float] = None,
                           out_dtype=torch.bfloat16, out=None, out_lse=None):
    """Fused ring attention on Ulysses head shards writing the token-sharded output.

    q, k, v: head-sharded ``[degree, B, S, H/degree, D]`` bf16 (the output of
    :func:`ulysses_permute` direction 0).  Returns ``(out [degree, B, S/degree, H, D],
    lse [B, H, S])``: what :func:`usp_sim` returns for the same sequence-sharded inputs.
    """
    for name, t in (("query", q), ("key", k), ("value", v)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.bfloat16 or t.dim() != 5:
            raise ValueError(f"{name} must be a 5-D bf16 CUDA tensor [degree, B, S, H/degree, D]")
        if not t.is_contiguous() or t.shape != q.shape or t.device != q.device:
            raise ValueError("query, key and value must be contiguous, of one shape, on one device")
    P, B, S, Hp, D = q.shape
    if P != degree:
        raise ValueError(f"leading dimension {P} != degree {degree}")
    if S % P:
        raise ValueError(f"sequence {S} not divisible by degree {P}")
    H = Hp * P
    code = _out_code(out_dtype)
    scale = float(D ** -0.5 if scale is None else scale)
    n = len(chunk_bounds) - 1
    if n < 1:
        raise ValueError("chunk_bounds needs at least two entries")
    bounds = (ctypes.c_int * (n + 1))(*[int(c) for c in chunk_bounds])
    if out is None:
        out = torch.empty((P, B, S // P, H, D), dtype=out_dtype, device=q.device)
    if out_lse is None:
        out_lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    if out.dtype != out_dtype or tuple(out.shape) != (P, B, S // P, H, D) or not out.is_contiguous() \
            or out.device != q.device:
        raise ValueError(f"out must be a contiguous {out_dtype} tensor of shape {(P, B, S // P, H, D)}")
    if out_lse.dtype != torch.float32 or tuple(out_lse.shape) != (B, H, S) or not out_lse.is_contiguous() \
            or out_lse.device != q.device:
        raise ValueError(f"out_lse must be a contiguous float32 tensor of shape {(B, H, S)}")
    st = load().cp_ring_sim_fused_ulysses(_ptr(q), _ptr(k), _ptr(v), P, bounds, n, _ptr(out), _ptr(out_lse), B, S, H,
                                          D, scale, code, ctypes.c_void_p(_stream(q)))
    _check(st, "cp_ring_sim_fused_ulysses")
    return out, out_lse


def ring_anything_gather(srcs, chunk_bounds: Sequence[int], max_len: Optional[int] = None, dsts=None):
    """Ring Anything pad -> all-gather buffers of the ``[B, S, H, D]`` tensors ``srcs``:
    each returned tensor is ``[n, B, max_len, H, D]`` with block c in ``[c, :, :len_c]``
    and zeros after it (``max_len`` defaults to the longest block)."""
    srcs = list(srcs)
    if not srcs:
        raise ValueError("need at least one tensor")
    ref = srcs[0]
    for t in srcs:
        if not isinstance(t, torch.Tensor) or not t.is_cuda or not t.is_contiguous() or t.dim() != 4 \
                or t.shape != ref.shape or t.dtype != ref.dtype or t.device != ref.device:
            raise ValueError("sources must be contiguous 4-D CUDA tensors of one shape, dtype and device")
    if ref.element_size() not in (2, 4):
        raise ValueError("elements must be 2 or 4 bytes")
    B, S, H, D = ref.shape
    n = len(chunk_bounds) - 1
    if n < 1:
        raise ValueError("chunk_bounds needs at least two entries")
    lens = [int(b) - int(a) for a, b in zip(chunk_bounds[:-1], chunk_bounds[1:])]
    if max_len is None:
        max_len = max(lens)
    if dsts is None:
        dsts = [torch.empty((n, B, max_len, H, D), dtype=ref.dtype, device=ref.device) for _ in srcs]
    dsts = list(dsts)
    if len(dsts) != len(srcs):
        raise ValueError(f"{len(srcs)} sources but {len(dsts)} destinations")
    for d in dsts:
        if not isinstance(d, torch.Tensor) or not d.is_cuda or not d.is_contiguous() or d.dtype != ref.dtype \
                or d.device != ref.device or d.numel() != n * B * max_len * H * D:
            raise ValueError(f"destinations must be contiguous CUDA tensors of {ref.dtype} with "
                             f"{n}*{B}*{max_len}*{H}*{D} elements on {ref.device}")
    cnt = len(srcs)
    sp = (ctypes.c_void_p * cnt)(*[t.data_ptr() for t in srcs])
    dp = (ctypes.c_void_p * cnt)(*[t.data_ptr() for t in dsts])
    bounds = (ctypes.c_int * (n + 1))(*[int(c) for c in chunk_bounds])
    st = load().cp_ring_anything_gather(sp, dp, cnt, bounds, n, int(max_len), B, S, H, D, ref.element_size(),
                                        ctypes.c_void_p(_stream(ref)))
    _check(st, "cp_ring_anything_gather")
    return dsts


STATIC_SCRATCH_BYTES = 32 << 20


def ring_sim_static(q, k, v, chunk_bounds: Sequence[int], scale: Optional[float] = None, out_dtype=torch.bfloat16,
                    out=None, out_lse=None):
    """:func:`ring_sim` without a workspace, for callers that cannot allocate device memory.

    The per-block partials live in the library's static 32 MiB device array, so the
    library call allocates nothing (``out``/``out_lse`` are allocated here only when not
    given; pass them to allocate nothing at all).  Problems whose partials exceed the
    array raise ``CpError`` (``CP_ERR_UNSUPPORTED``).  Calls that overlap on the GPU share
    the array and race.  Make the first call on a device before any stream capture.
    """
    B, Sq, Skv, H, D = _check_qkv(q, k, v)
    code = _out_code(out_dtype)
    scale = float(D ** -0.5 if scale is None else scale)
    n = len(chunk_bounds) - 1
    if n < 1:
        raise ValueError("chunk_bounds needs at least two entries")
    need = ring_workspace_size(n, B, H, Sq, D)
    if need > STATIC_SCRATCH_BYTES:
        raise CpError(CP_ERR_UNSUPPORTED, f"cp_ring_sim_static (needs {need} bytes of scratch, the static array "
                                          f"holds {STATIC_SCRATCH_BYTES})")
    bounds = (ctypes.c_int * (n + 1))(*[int(c) for c in chunk_bounds])
    if out is None:
        out = torch.empty((B, Sq, H, D), dtype=out_dtype, device=q.device)
    if out_lse is None:
        out_lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    st = load().cp_ring_sim_static(_ptr(q), _ptr(k), _ptr(v), bounds, n, _ptr(out), _ptr(out_lse), B, H, Sq, Skv, D,
                                   scale, code, ctypes.c_void_p(_stream(q)))
    _check(st, "cp_ring_sim_static")
    return out, out_lse


def ring_workspace_views(workspace, n: int, B: int, H: int, Sq: int, D: int):
    """Views of the per-block fp32 partials ``[n,B,Sq,H,D]`` and LSEs ``[n,B,H,Sq]`` in a ring workspace."""
    rows = B * H * Sq
    pbytes = (n * rows * D * 4 + 255) // 256 * 256
    parts = workspace[: n * rows * D * 4].view(torch.float32).view(n, B, Sq, H, D)
    lses = workspace[pbytes: pbytes + n * rows * 4].view(torch.float32).view(n, B, H, Sq)
    return parts, lses


def ulysses_permute(src, degree: int, direction: int, dst=None):
    """Ulysses exchange.  direction 0: ``[P,B,S/P,H,D] -> [P,B,S,H/P,D]``; direction 1: the inverse."""
    if not src.is_cuda or not src.is_contiguous():
        raise ValueError("src must be a contiguous CUDA tensor")
    if src.element_size() not in (2, 4):
        raise ValueError("src elements must be 2 or 4 bytes")
    P = int(degree)
    if src.dim() != 5 or src.shape[0] != P:
        raise ValueError(f"src must be 5-D with leading dim {P}, got {tuple(src.shape)}")
    if direction == 0:
        _, B, Sp, H, D = src.shape
        S = Sp * P
        if H % P:
            raise ValueError(f"heads {H} not divisible by degree {P}")
        shape = (P, B, S, H // P, D)
    elif direction == 1:
        _, B, S, Hp, D = src.shape
        H = Hp * P
        if S % P:
            raise ValueError(f"sequence {S} not divisible by degree {P}")
        shape = (P, B, S // P, H, D)
    else:
        raise ValueError("direction must be 0 or 1")
    if dst is None:
        dst = torch.empty(shape, dtype=src.dtype, device=src.device)
    st = load().cp_ulysses_permute(_ptr(src), _ptr(dst), P, B, S, H, D, direction, src.element_size(),
                                   ctypes.c_void_p(_stream(src)))
    _check(st, "cp_ulysses_permute")
    return dst


def ulysses_permute_n(srcs, degree: int, direction: int, dsts=None):
    """Ulysses exchange of several same-shaped tensors (e.g. Q, K, V) in one launch."""
    srcs = list(srcs)
    if not srcs:
        raise ValueError("need at least one tensor")
    ref = srcs[0]
    for t in srcs:
        if not t.is_cuda or not t.is_contiguous() or t.shape != ref.shape or t.dtype != ref.dtype \
                or t.device != ref.device:
            raise ValueError("tensors must be contiguous CUDA tensors of one shape, dtype and device")
    if dsts is None:
        dsts = [None] * len(srcs)
    dsts = list(dsts)
    P = int(degree)
    if ref.dim() != 5 or ref.shape[0] != P:
        raise ValueError(f"src must be 5-D with leading dim {P}, got {tuple(ref.shape)}")
    if direction == 0:
        _, B, Sp, H, D = ref.shape
        S = Sp * P
        if H % P:
            raise ValueError(f"heads {H} not divisible by degree {P}")
        shape = (P, B, S, H // P, D)
    elif direction == 1:
        _, B, S, Hp, D = ref.shape
        H = Hp * P
        if S % P:
            raise ValueError(f"sequence {S} not divisible by degree {P}")
        shape = (P, B, S // P, H, D)
    else:
        raise ValueError("direction must be 0 or 1")
    dsts = [torch.empty(shape, dtype=ref.dtype, device=ref.device) if d is None else d for d in dsts]
    n = len(srcs)
    sp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in srcs])
    dp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in dsts])
    st = load().cp_ulysses_permute_n(sp, dp, n, P, B, S, H, D, direction, ref.element_size(),
                                     ctypes.c_void_p(_stream(ref)))
    _check(st, "cp_ulysses_permute_n")
    return dsts


def ulysses_anything_permute(src, degree: int, seq_bounds: Sequence[int], head_bounds: Sequence[int], B: int, S: int,
                             H: int, D: int, direction: int, dst=None):
    """Ulysses exchange with unequal shards (see cp_ulysses_anything_permute): src and the
    returned dst are packed buffers of B*S*H*D elements (1-D views)."""
    if not isinstance(src, torch.Tensor) or not src.is_cuda or not src.is_contiguous():
        raise ValueError("src must be a contiguous CUDA tensor")
    if src.numel() != B * S * H * D:
        raise ValueError(f"src has {src.numel()} elements, expected B*S*H*D = {B * S * H * D}")
    if len(seq_bounds) != degree + 1 or len(head_bounds) != degree + 1:
        raise ValueError("seq_bounds and head_bounds need degree + 1 entries")
    sb = (ctypes.c_int * (degree + 1))(*[int(x) for x in seq_bounds])
    hb = (ctypes.c_int * (degree + 1))(*[int(x) for x in head_bounds])
    if dst is None:
        dst = torch.empty(src.numel(), dtype=src.dtype, device=src.device)
    st = load().cp_ulysses_anything_permute(_ptr(src), _ptr(dst), degree, sb, hb, B, S, H, D, direction,
                                            src.element_size(), ctypes.c_void_p(_stream(src)))
    _check(st, "cp_ulysses_anything_permute")
    return dst.view(-1)


def ulysses_anything_permute_n(srcs, degree: int, seq_bounds: Sequence[int], head_bounds: Sequence[int], B: int,
                               S: int, H: int, D: int, direction: int, dsts=None):
    """:func:`ulysses_anything_permute` of several same-shaped packed buffers (e.g. Q, K, V)
    in one launch; returns the destination buffers."""
    srcs = list(srcs)
    if not srcs:
        raise ValueError("need at least one tensor")
    ref = srcs[0]
    for t in srcs:
        if not isinstance(t, torch.Tensor) or not t.is_cuda or not t.is_contiguous() or t.dtype != ref.dtype \
                or t.device != ref.device or t.numel() != B * S * H * D:
            raise ValueError(f"sources must be contiguous CUDA tensors of B*S*H*D = {B * S * H * D} elements, "
                             f"one dtype and device")
    if len(seq_bounds) != degree + 1 or len(head_bounds) != degree + 1:
        raise ValueError("seq_bounds and head_bounds need degree + 1 entries")
    dsts = [torch.empty(ref.numel(), dtype=ref.dtype, device=ref.device) for _ in srcs] if dsts is None else list(dsts)
    n = len(srcs)
    sp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in srcs])
    dp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in dsts])
    sb = (ctypes.c_int * (degree + 1))(*[int(x) for x in seq_bounds])
    hb = (ctypes.c_int * (degree + 1))(*[int(x) for x in head_bounds])
    st = load().cp_ulysses_anything_permute_n(sp, dp, n, degree, sb, hb, B, S, H, D, direction, ref.element_size(),
                                              ctypes.c_void_p(_stream(ref)))
    _check(st, "cp_ulysses_anything_permute_n")
    return [d.view(-1) for d in dsts]


def ring_bounds(S: int, n: int, anything: bool = False):
    """Block bounds of a ring of ``n`` over ``S`` rows (host only)."""
    out = (ctypes.c_int * (n + 1))()
    _check(load().cp_ring_bounds(int(S), int(n), 1 if anything else 0, out), "cp_ring_bounds")
    return list(out)


def debug_set_fault(mode: int):
    """Test hook: mode 1 makes the next attention launch time out (see cpattn.h)."""
    _check(load().cp_debug_set_fault(int(mode)), "cp_debug_set_fault")


def last_device_status(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return int(load().cp_last_device_status(ctypes.c_void_p(s.cuda_stream)))


# ------------------------------------------------------------------ one process per GPU
# Raw device pointers (ints) in and out: peer buffers are not torch allocations.


def peer_alloc(nbytes: int):
    """A zero-filled device buffer other processes can map; returns ``(ptr, handle bytes)``."""
    ptr = ctypes.c_void_p()
    handle = ctypes.create_string_buffer(CP_IPC_HANDLE_BYTES)
    _check(load().cp_peer_alloc(int(nbytes), ctypes.byref(ptr), handle), "cp_peer_alloc")
    return int(ptr.value), handle.raw


def peer_open(handle: bytes) -> int:
    """Map another process's :func:`peer_alloc` buffer; returns the device pointer."""
    if len(handle) != CP_IPC_HANDLE_BYTES:
        raise ValueError(f"an IPC handle has {CP_IPC_HANDLE_BYTES} bytes, got {len(handle)}")
    ptr = ctypes.c_void_p()
    _check(load().cp_peer_open(ctypes.create_string_buffer(bytes(handle), CP_IPC_HANDLE_BYTES), ctypes.byref(ptr)),
           "cp_peer_open")
    return int(ptr.value)


def peer_close(ptr: int):
    _check(load().cp_peer_close(ctypes.c_void_p(ptr)), "cp_peer_close")


def peer_free(ptr: int):
    _check(load().cp_peer_free(ctypes.c_void_p(ptr)), "cp_peer_free")


def ulysses_push_n(srcs: Sequence[int], dsts: Sequence[Sequence[int]], rank: int, degree: int, B: int, S: int, H: int,
                   D: int, direction: int, elem_bytes: int, stream: int):
    """This rank's half of a Ulysses all-to-all (see cp_ulysses_push_n): ``dsts[t][q]`` is
    tensor t's buffer on rank q."""
    n = len(srcs)
    if n < 1 or len(dsts) != n or any(len(row) != degree for row in dsts):
        raise ValueError("dsts needs one row of degree pointers per source")
    sp = (ctypes.c_void_p * n)(*[int(x) for x in srcs])
    dp = (ctypes.c_void_p * (n * degree))(*[int(x) for row in dsts for x in row])
    _check(load().cp_ulysses_push_n(sp, dp, n, rank, degree, B, S, H, D, direction, elem_bytes, ctypes.c_void_p(stream)),
           "cp_ulysses_push_n")


def ulysses_anything_push_n(srcs: Sequence[int], dsts: Sequence[Sequence[int]], rank: int,
                            seq_bounds: Sequence[int], head_bounds: Sequence[int], B: int, H: int, D: int,
                            direction: int, elem_bytes: int, stream: int):
    """This rank's half of a Ulysses-Anything all-to-all (see cp_ulysses_anything_push_n)."""
    degree = len(seq_bounds) - 1
    n = len(srcs)
    if degree < 1 or len(head_bounds) != degree + 1:
        raise ValueError("seq_bounds and head_bounds need degree + 1 entries")
    if n < 1 or len(dsts) != n or any(len(row) != degree for row in dsts):
        raise ValueError("dsts needs one row of degree pointers per source")
    sp = (ctypes.c_void_p * n)(*[int(x) for x in srcs])
    dp = (ctypes.c_void_p * (n * degree))(*[int(x) for row in dsts for x in row])
    sb = (ctypes.c_int * (degree + 1))(*[int(x) for x in seq_bounds])
    hb = (ctypes.c_int * (degree + 1))(*[int(x) for x in head_bounds])
    _check(load().cp_ulysses_anything_push_n(sp, dp, n, rank, degree, sb, hb, B, H, D, direction, elem_bytes,
                                             ctypes.c_void_p(stream)), "cp_ulysses_anything_push_n")


def attn_merge_push(partials, lses, peer_outs: Sequence[int], shard: int, out_dtype=torch.bfloat16):
    """Merge this rank's head-shard partials ``[n, B, S, H/P, D]`` (LSEs ``[n, B, H/P, S]``)
    and store every merged row into its owner's sequence shard ``[B, S/P, H, D]``:
    ``peer_outs[p]`` is rank p's (see cp_attn_merge_push)."""
    if partials.dtype != torch.float32 or lses.dtype != torch.float32:
        raise ValueError("partials and lses must be float32")
    if not (partials.is_cuda and lses.is_cuda and partials.is_contiguous() and lses.is_contiguous()):
        raise ValueError("partials and lses must be contiguous CUDA tensors")
    n, B, S, Hp, D = partials.shape
    if tuple(lses.shape) != (n, B, Hp, S):
        raise ValueError(f"incompatible shapes partials{tuple(partials.shape)} lses{tuple(lses.shape)}")
    P = len(peer_outs)
    po = (ctypes.c_void_p * P)(*[int(x) for x in peer_outs])
    _check(load().cp_attn_merge_push(_ptr(partials), _ptr(lses), n, po, shard, P, B, S, Hp * P, D,
                                     _out_code(out_dtype), ctypes.c_void_p(_stream(partials))), "cp_attn_merge_push")


def peer_barrier(pads: Sequence[int], rank: int, epoch: int, stream: int, timeout_ms: int = 1000):
    """Signal every rank's pad and wait, at most ``timeout_ms``, for every rank's signal
    (see cp_peer_barrier)."""
    n = len(pads)
    pp = (ctypes.c_void_p * n)(*[int(x) for x in pads])
    _check(load().cp_peer_barrier(pp, rank, n, ctypes.c_uint(epoch & 0xFFFFFFFF), ctypes.c_uint(int(timeout_ms)),
                                  ctypes.c_void_p(stream)), "cp_peer_barrier")


def ring_fetch_block(dst: int, src: int, B: int, rows: int, H: int, D: int, dst_S: int, dst_row0: int, src_S: int,
                     src_row0: int, elem_bytes: int, stream: int):
    """Copy-engine copy of rows of a ``[B][S][H][D]`` tensor (see cp_ring_fetch_block)."""
    _check(load().cp_ring_fetch_block(ctypes.c_void_p(dst), ctypes.c_void_p(src), B, rows, H, D, dst_S, dst_row0,
                                      src_S, src_row0, elem_bytes, ctypes.c_void_p(stream)), "cp_ring_fetch_block")


class _DeviceMemory:
    """A raw device range seen by torch through the CUDA array interface (no copy)."""

    def __init__(self, ptr: int, nbytes: int):
        self.__cuda_array_interface__ = {"shape": (int(nbytes),), "typestr": "|u1", "data": (int(ptr), False),
                                         "version": 3, "strides": None, "stream": None}


def device_tensor(ptr: int, shape, dtype, device) -> torch.Tensor:
    """A contiguous torch tensor over ``ptr`` (memory owned elsewhere; no copy)."""
    nbytes = int(torch.Size(shape).numel()) * torch.empty((), dtype=dtype).element_size()
    raw = torch.as_tensor(_DeviceMemory(ptr, max(nbytes, 1)), device=device)
    return raw[:nbytes].view(dtype).view(shape)
