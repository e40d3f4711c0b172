"""Thin ctypes binding of libla_b200.so (include/la_b200.h).

Argument marshalling only: torch tensors are described to the C ABI by data
pointer, shape, strides and dtype, outputs and workspace are allocated with
torch (device memory plumbing), and the call is enqueued on the current torch
stream.  Every step of the computation runs in the library's CUDA kernels; if
the library is missing this module raises -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libla_b200.so")

LA_OK, LA_ERR_INVALID_ARG, LA_ERR_UNSUPPORTED, LA_ERR_WORKSPACE, LA_ERR_CUDA = range(5)
LA_PHI_IDENTITY, LA_PHI_ELU1 = 0, 1
LA_F32, LA_BF16 = 0, 1
LA_FLAG_NONE, LA_FLAG_SIMT = 0, 1
LA_FLAG_TEST_WAIT_TIMEOUT = 0x100  # tests of the failure path only (see include/la_b200.h)

_PHI = {"identity": LA_PHI_IDENTITY, "elu1": LA_PHI_ELU1, LA_PHI_IDENTITY: LA_PHI_IDENTITY,
        LA_PHI_ELU1: LA_PHI_ELU1}
_DT = {torch.float32: LA_F32, torch.bfloat16: LA_BF16}

# Every function include/la_b200.h declares.
EXPORTS = ("la_fwd_chunk", "la_fwd_chunk_z", "la_fwd_chunk_gated", "la_fwd_chunk_workspace_size", "la_step",
           "la_step_norm", "la_step_gated", "la_status_string", "la_last_error", "la_version", "la_device_error",
           "la_fwd_chunk_noalloc", "la_bwd_chunk", "la_norm_gate", "la_fwd_chunk_normgate",
           "la_fwd_gated_delta", "la_fwd_gated_delta_chunk", "la_fwd_gated_delta_workspace_size",
           "la_fwd_chunk_path", "la_fwd_chunk_host", "la_fwd_chunk_host_arena_size", "la_bwd_chunk_gated",
           "la_bwd_chunk_norm", "la_bwd_chunk_norm_workspace_size", "la_bwd_chunk_gated_norm",
           "la_bwd_chunk_gated_norm_workspace_size")


class LaTensor(ctypes.Structure):
    _fields_ = [
        ("data", ctypes.c_void_p),
        ("dtype", ctypes.c_int32),
        ("B", ctypes.c_int64), ("T", ctypes.c_int64), ("H", ctypes.c_int64), ("D", ctypes.c_int64),
        ("stride_b", ctypes.c_int64), ("stride_t", ctypes.c_int64), ("stride_h", ctypes.c_int64),
    ]


class LaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(msg)
        self.status = status


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libla_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            "libla_b200.so is not built (%s); run `python -c 'import __graft_entry__ as g; g.build()'`" % path)
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(LaTensor)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    lib.la_fwd_chunk.argtypes = [P, P, P, vp, vp, i64, i32, i32, i32, P, vp, i32, vp, sz, vp]
    lib.la_fwd_chunk.restype = i32
    lib.la_fwd_chunk_z.argtypes = [P, P, P, vp, vp, i64, i32, i32, i32, P, vp, vp, i32, vp, sz, vp]
    lib.la_fwd_chunk_z.restype = i32
    lib.la_fwd_chunk_gated.argtypes = [P, P, P, vp, vp, i64, i32, i32, i32, P, vp, vp, i32, vp, sz, vp]
    lib.la_fwd_chunk_gated.restype = i32
    lib.la_fwd_chunk_workspace_size.argtypes = [i64, i64, i64, i64, i64, i64, i32, i32, i32, i32]
    lib.la_fwd_chunk_workspace_size.restype = sz
    lib.la_step.argtypes = [P, P, P, vp, vp, P, i32, vp]
    lib.la_step.restype = i32
    lib.la_step_norm.argtypes = [P, P, P, vp, vp, vp, P, i32, vp]
    lib.la_step_norm.restype = i32
    lib.la_step_gated.argtypes = [P, P, P, vp, vp, vp, P, i32, vp]
    lib.la_step_gated.restype = i32
    lib.la_bwd_chunk.argtypes = [P, P, P, P, vp, vp, i64, i32, i32, P, P, P, i32, vp]
    lib.la_bwd_chunk.restype = i32
    lib.la_norm_gate.argtypes = [P, P, vp, ctypes.c_float, P, vp]
    lib.la_norm_gate.restype = i32
    lib.la_fwd_chunk_normgate.argtypes = [P, P, P, vp, vp, i64, i32, i32, i32, P, vp, ctypes.c_float, P, vp, i32,
                                          vp, sz, vp]
    lib.la_fwd_chunk_normgate.restype = i32
    lib.la_fwd_gated_delta.argtypes = [P, P, P, vp, vp, vp, i64, vp, P, vp, vp]
    lib.la_fwd_gated_delta.restype = i32
    lib.la_fwd_gated_delta_chunk.argtypes = [P, P, P, vp, vp, vp, i64, vp, P, vp, i32, vp, sz, vp]
    lib.la_fwd_gated_delta_chunk.restype = i32
    lib.la_fwd_gated_delta_workspace_size.argtypes = [i64, i64, i64, i64, i64, i64, i32, i32, i32]
    lib.la_fwd_gated_delta_workspace_size.restype = sz
    lib.la_fwd_chunk_path.argtypes = [i64, i64, i64, i64, i32, i32, i32]
    lib.la_fwd_chunk_path.restype = i32
    lib.la_fwd_chunk_host_arena_size.argtypes = [i64, i64, i64, i64, i64, i64, i32, i32, i32, i32, i32]
    lib.la_fwd_chunk_host_arena_size.restype = sz
    lib.la_fwd_chunk_host.argtypes = [P, P, P, vp, vp, i64, i32, i32, i32, P, vp, i32, vp, sz, vp]
    lib.la_fwd_chunk_host.restype = i32
    lib.la_bwd_chunk_gated.argtypes = [P, P, P, P, vp, vp, i64, i32, i32, P, P, P, vp, i32, vp]
    lib.la_bwd_chunk_gated.restype = i32
    lib.la_bwd_chunk_norm.argtypes = [P, P, P, P, vp, vp, i64, i32, i32, P, P, P, i32, vp, sz, vp]
    lib.la_bwd_chunk_norm.restype = i32
    lib.la_bwd_chunk_norm_workspace_size.argtypes = [i64, i64, i64, i64, i64, i32, i32, i32]
    lib.la_bwd_chunk_norm_workspace_size.restype = sz
    lib.la_bwd_chunk_gated_norm.argtypes = [P, P, P, P, vp, vp, i64, i32, i32, P, P, P, vp, i32, vp, sz, vp]
    lib.la_bwd_chunk_gated_norm.restype = i32
    lib.la_bwd_chunk_gated_norm_workspace_size.argtypes = [i64, i64, i64, i64, i64, i32, i32, i32]
    lib.la_bwd_chunk_gated_norm_workspace_size.restype = sz
    lib.la_status_string.argtypes = [i32]
    lib.la_status_string.restype = ctypes.c_char_p
    lib.la_last_error.argtypes = []
    lib.la_last_error.restype = ctypes.c_char_p
    lib.la_version.argtypes = []
    lib.la_version.restype = i32
    lib.la_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32), ctypes.POINTER(ctypes.c_uint32), i32]
    lib.la_device_error.restype = i32
    lib.la_fwd_chunk_noalloc.argtypes = [P, P, P, vp, vp, i64, i32, i32, i32, P, vp, i32, vp]
    lib.la_fwd_chunk_noalloc.restype = i32
    _lib = lib
    return lib


def describe(t: torch.Tensor) -> LaTensor:
    """la_tensor for a [B, T, H, D] torch tensor whose last dim is contiguous."""
    if t.dim() != 4:
        raise ValueError("expected a [B, T, H, D] tensor, got shape %s" % (tuple(t.shape),))
    if t.dtype not in _DT:
        raise TypeError("dtype %s not supported (float32 or bfloat16)" % t.dtype)
    if t.shape[3] > 1 and t.stride(3) != 1:
        raise ValueError("the head dim must be contiguous")
    B, T, H, D = t.shape
    return LaTensor(t.data_ptr(), _DT[t.dtype], B, T, H, D, t.stride(0), t.stride(1), t.stride(2))


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(lib, status: int, what: str):
    if status != LA_OK:
        detail = lib.la_last_error().decode(errors="replace")
        raise LaError(status, "%s failed: %s (%s)" % (what, lib.la_status_string(status).decode(), detail))


def workspace_size(B, T, H, d_k, d_v, n_seqs, varlen, chunk, dtype=torch.bfloat16, flags=0) -> int:
    lib = load_library()
    n = lib.la_fwd_chunk_workspace_size(B, T, H, d_k, d_v, n_seqs, int(bool(varlen)), chunk, _DT[dtype], flags)
    if n == ctypes.c_size_t(-1).value:
        raise LaError(LA_ERR_INVALID_ARG, "la_fwd_chunk_workspace_size rejected the arguments")
    return int(n)


LA_PATH_TENSOR_CORE, LA_PATH_CUDA_CORE = 1, 2


def fwd_chunk_path(d_k, d_v, T, H, chunk=64, dtype=torch.bfloat16, flags=LA_FLAG_NONE) -> int:
    """Kernel la_fwd_chunk runs for this shape: LA_PATH_TENSOR_CORE, LA_PATH_CUDA_CORE,
    or -1 for arguments it rejects (see la_fwd_chunk_path in include/la_b200.h)."""
    return int(load_library().la_fwd_chunk_path(d_k, d_v, T, H, chunk, _DT[dtype], flags))


def la_fwd_chunk(q, k, v, gamma, cu_seqlens=None, chunk=64, phi="identity", normalize=False,
                 out=None, final_state=None, return_final_state=True, flags=LA_FLAG_NONE,
                 workspace=None, stream=None):
    """Chunkwise causal linear attention forward (see la_fwd_chunk in include/la_b200.h).

    q, k [B,T,H,d_k], v [B,T,H,d_v] (CUDA, float32 or bfloat16); gamma float32 [H];
    cu_seqlens int32 [N+1] or None.  Returns (out, final_state or None).
    """
    out, final_state, _ = _fwd(q, k, v, gamma, cu_seqlens, chunk, phi, normalize, out, final_state,
                               return_final_state, None, flags, workspace, stream)
    return out, final_state


def host_arena_size(B, T, H, d_k, d_v, n_seqs, varlen, chunk=64, dtype=torch.bfloat16, flags=0,
                    final_state=True) -> int:
    """Device bytes la_fwd_chunk_host needs as its arena."""
    n = load_library().la_fwd_chunk_host_arena_size(B, T, H, d_k, d_v, n_seqs, int(bool(varlen)), chunk, _DT[dtype],
                                                     flags, int(bool(final_state)))
    if n == ctypes.c_size_t(-1).value:
        raise LaError(LA_ERR_INVALID_ARG, "la_fwd_chunk_host_arena_size rejected the arguments")
    return int(n)


def la_fwd_chunk_host(q, k, v, gamma, cu_seqlens=None, chunk=64, phi="identity", normalize=False, out=None,
                      final_state=None, return_final_state=True, flags=LA_FLAG_NONE, arena=None, stream=None):
    """la_fwd_chunk on host tensors (see la_fwd_chunk_host in include/la_b200.h): q, k, v, gamma,
    cu_seqlens, out and final_state are CPU tensors (pin them for asynchronous copies); the arena is a
    device uint8 tensor (allocated here if None).  The copies and the forward are enqueued on the
    stream; synchronise it before reading out / final_state.  Returns (out, final_state or None)."""
    lib = load_library()
    B, T, H, dk = q.shape
    dv = v.shape[3]
    n_seqs = B if cu_seqlens is None else cu_seqlens.numel() - 1
    for name, t in (("q", q), ("k", k), ("v", v), ("gamma", gamma)):
        if t.device.type != "cpu" or not t.is_contiguous():
            raise TypeError("%s must be a contiguous host tensor" % name)
    if cu_seqlens is not None and (cu_seqlens.dtype != torch.int32 or cu_seqlens.device.type != "cpu"):
        raise TypeError("cu_seqlens must be a host int32 tensor")
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, pin_memory=True)
    if final_state is None and return_final_state:
        final_state = torch.empty((n_seqs, H, dk, dv), dtype=torch.float32, pin_memory=True)
    need = host_arena_size(B, T, H, dk, dv, n_seqs, cu_seqlens is not None, chunk, q.dtype, flags,
                           final_state is not None)
    if arena is None or arena.numel() * arena.element_size() < need:
        arena = torch.empty(need, dtype=torch.uint8, device="cuda")
    tq, tk, tv, to = describe(q), describe(k), describe(v), describe(out)
    st = lib.la_fwd_chunk_host(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv), gamma.data_ptr(),
                               None if cu_seqlens is None else cu_seqlens.data_ptr(), n_seqs, int(chunk), _PHI[phi],
                               int(bool(normalize)), ctypes.byref(to),
                               None if final_state is None else final_state.data_ptr(), int(flags),
                               arena.data_ptr(), arena.numel() * arena.element_size(), _stream(stream))
    _check(lib, st, "la_fwd_chunk_host")
    return out, final_state


def la_fwd_chunk_gated(q, k, v, g, cu_seqlens=None, chunk=64, phi="identity", normalize=False, out=None,
                       final_state=None, final_z=None, return_final_z=False, flags=LA_FLAG_NONE, workspace=None,
                       stream=None):
    """Forward with a data-dependent decay exp(g[b, t, h]) (see la_fwd_chunk_gated in
    include/la_b200.h).  g float32 [B, T, H], <= 0.  Returns (out, final_state, final_z or None);
    final_z needs normalize."""
    B, T, H, dk = q.shape
    if g.dtype != torch.float32 or tuple(g.shape) != (B, T, H) or not g.is_contiguous():
        raise TypeError("g must be a contiguous float32 [B, T, H] tensor")
    n_seqs = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if final_z is None and return_final_z:
        final_z = torch.empty((n_seqs, H, dk), dtype=torch.float32, device=q.device)
    return _fwd(q, k, v, None, cu_seqlens, chunk, phi, normalize, out, final_state, True, final_z, flags,
                workspace, stream, g=g)


def la_fwd_chunk_z(q, k, v, gamma, cu_seqlens=None, chunk=64, phi="elu1", out=None, final_state=None,
                   final_z=None, flags=LA_FLAG_NONE, workspace=None, stream=None):
    """Normalised forward that also returns z after each sequence's last token
    (see la_fwd_chunk_z in include/la_b200.h).  Returns (out, final_state, final_z)."""
    B, T, H, dk = q.shape
    n_seqs = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if final_z is None:
        final_z = torch.empty((n_seqs, H, dk), dtype=torch.float32, device=q.device)
    return _fwd(q, k, v, gamma, cu_seqlens, chunk, phi, True, out, final_state, True, final_z, flags, workspace,
                stream)


def _fwd(q, k, v, gamma, cu_seqlens, chunk, phi, normalize, out, final_state, return_final_state, final_z,
         flags, workspace, stream, g=None):
    lib = load_library()
    B, T, H, dk = q.shape
    dv = v.shape[3]
    n_seqs = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if cu_seqlens is not None and cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    if g is None and (gamma.dtype != torch.float32 or gamma.numel() != H):
        raise TypeError("gamma must be float32 with H entries")
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if final_state is None and return_final_state:
        final_state = torch.empty((n_seqs, H, dk, dv), dtype=torch.float32, device=q.device)
    need = workspace_size(B, T, H, dk, dv, n_seqs, cu_seqlens is not None, chunk, q.dtype, flags)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    tq, tk, tv, to = describe(q), describe(k), describe(v), describe(out)
    args = [ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv), (gamma if g is None else g).data_ptr(),
            None if cu_seqlens is None else cu_seqlens.data_ptr(), n_seqs, int(chunk), _PHI[phi],
            int(bool(normalize)), ctypes.byref(to), None if final_state is None else final_state.data_ptr()]
    tail = [int(flags), None if workspace is None else workspace.data_ptr(),
            0 if workspace is None else workspace.numel() * workspace.element_size(), _stream(stream)]
    fz = None if final_z is None else final_z.data_ptr()
    if final_z is not None and (final_z.dtype != torch.float32 or not final_z.is_contiguous()):
        raise TypeError("final_z must be a contiguous float32 tensor")
    if g is not None:
        _check(lib, lib.la_fwd_chunk_gated(*args, fz, *tail), "la_fwd_chunk_gated")
    elif final_z is None:
        _check(lib, lib.la_fwd_chunk(*args, *tail), "la_fwd_chunk")
    else:
        _check(lib, lib.la_fwd_chunk_z(*args, fz, *tail), "la_fwd_chunk_z")
    return out, final_state, final_z


def device_error(reset: bool = True):
    """(flags, detail) of the tensor-core kernel's bounded-wait error word (synchronises the device)."""
    lib = load_library()
    f, d = ctypes.c_uint32(0), ctypes.c_uint32(0)
    _check(lib, lib.la_device_error(ctypes.byref(f), ctypes.byref(d), int(reset)), "la_device_error")
    return int(f.value), int(d.value)


def la_step(q, k, v, gamma, state, out=None, phi="identity", stream=None):
    """One decode token (see la_step in include/la_b200.h).

    q, k [N,H,d_k] or [N,1,H,d_k]; v [N,H,d_v] likewise; state float32 [N,H,d_k,d_v]
    updated in place.  Returns out shaped like v.
    """
    lib = load_library()
    squeeze = q.dim() == 3
    q4, k4, v4 = (x.unsqueeze(1) if squeeze else x for x in (q, k, v))
    if out is None:
        out = torch.empty_like(v4)
    o4 = out.unsqueeze(1) if out.dim() == 3 else out
    if state.dtype != torch.float32 or not state.is_contiguous():
        raise TypeError("state must be a contiguous float32 tensor")
    tq, tk, tv, to = describe(q4), describe(k4), describe(v4), describe(o4)
    st = lib.la_step(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv), gamma.data_ptr(), state.data_ptr(),
                     ctypes.byref(to), _PHI[phi], _stream(stream))
    _check(lib, st, "la_step")
    return o4.squeeze(1) if squeeze else o4


def la_step_norm(q, k, v, gamma, state, z, out=None, phi="elu1", stream=None):
    """One normalised decode token (see la_step_norm in include/la_b200.h).

    As la_step, plus z float32 [N,H,d_k] updated in place; out = S phi(q) / (z . phi(q)).
    """
    lib = load_library()
    squeeze = q.dim() == 3
    q4, k4, v4 = (x.unsqueeze(1) if squeeze else x for x in (q, k, v))
    if out is None:
        out = torch.empty_like(v4)
    o4 = out.unsqueeze(1) if out.dim() == 3 else out
    for name, t in (("state", state), ("z", z)):
        if t.dtype != torch.float32 or not t.is_contiguous():
            raise TypeError("%s must be a contiguous float32 tensor" % name)
    tq, tk, tv, to = describe(q4), describe(k4), describe(v4), describe(o4)
    st = lib.la_step_norm(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv), gamma.data_ptr(),
                          state.data_ptr(), z.data_ptr(), ctypes.byref(to), _PHI[phi], _stream(stream))
    _check(lib, st, "la_step_norm")
    return o4.squeeze(1) if squeeze else o4


def la_step_gated(q, k, v, g, state, z=None, out=None, phi="identity", stream=None):
    """One decode token with decay exp(g[n, h]) (see la_step_gated in include/la_b200.h).

    g float32 [N, H]; state [N,H,d_k,d_v] and, when given, z [N,H,d_k] (normalised) updated in place.
    """
    lib = load_library()
    squeeze = q.dim() == 3
    q4, k4, v4 = (x.unsqueeze(1) if squeeze else x for x in (q, k, v))
    if out is None:
        out = torch.empty_like(v4)
    o4 = out.unsqueeze(1) if out.dim() == 3 else out
    for name, t in (("state", state), ("z", z), ("g", g)):
        if t is not None and (t.dtype != torch.float32 or not t.is_contiguous()):
            raise TypeError("%s must be a contiguous float32 tensor" % name)
    tq, tk, tv, to = describe(q4), describe(k4), describe(v4), describe(o4)
    st = lib.la_step_gated(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv), g.data_ptr(), state.data_ptr(),
                           None if z is None else z.data_ptr(), ctypes.byref(to), _PHI[phi], _stream(stream))
    _check(lib, st, "la_step_gated")
    return o4.squeeze(1) if squeeze else o4


def la_bwd_chunk(q, k, v, dout, gamma, cu_seqlens=None, chunk=64, phi="identity", dq=None, dk=None, dv=None,
                 flags=LA_FLAG_NONE, stream=None):
    """Gradients (dq, dk, dv) of the unnormalised forward given dout (see la_bwd_chunk in
    include/la_b200.h).  All tensors [B, T, H, d], one dtype."""
    lib = load_library()
    B, T, H, d_k = q.shape
    n_seqs = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if cu_seqlens is not None and cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    t = [describe(x) for x in (q, k, v, dout, dq, dk, dv)]
    st = lib.la_bwd_chunk(*(ctypes.byref(x) for x in t[:4]), gamma.data_ptr(),
                          None if cu_seqlens is None else cu_seqlens.data_ptr(), n_seqs, int(chunk), _PHI[phi],
                          *(ctypes.byref(x) for x in t[4:]), int(flags), _stream(stream))
    _check(lib, st, "la_bwd_chunk")
    return dq, dk, dv


def la_bwd_chunk_gated(q, k, v, dout, g, cu_seqlens=None, chunk=64, phi="identity", dq=None, dk=None, dv=None,
                       dg=None, flags=LA_FLAG_NONE, stream=None):
    """Gradients of la_fwd_chunk_gated's unnormalised forward (see la_bwd_chunk_gated in
    include/la_b200.h): returns (dq, dk, dv, dg), dg float32 [B, T, H] for the log decays g."""
    lib = load_library()
    B, T, H, _ = q.shape
    n_seqs = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if g.dtype != torch.float32 or tuple(g.shape) != (B, T, H) or not g.is_contiguous():
        raise TypeError("g must be a contiguous float32 [B, T, H] tensor")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    dg = torch.empty_like(g) if dg is None else dg
    t = [describe(x) for x in (q, k, v, dout, dq, dk, dv)]
    st = lib.la_bwd_chunk_gated(*[ctypes.byref(x) for x in t[:4]], g.data_ptr(),
                                None if cu_seqlens is None else cu_seqlens.data_ptr(), n_seqs, int(chunk), _PHI[phi],
                                *[ctypes.byref(x) for x in t[4:]], dg.data_ptr(), int(flags), _stream(stream))
    _check(lib, st, "la_bwd_chunk_gated")
    return dq, dk, dv, dg


def bwd_norm_workspace_size(B, T, H, d_k, d_v, chunk=64, dtype=torch.bfloat16, flags=LA_FLAG_NONE) -> int:
    """Bytes of workspace la_bwd_chunk_norm needs; -1 for arguments it rejects."""
    n = load_library().la_bwd_chunk_norm_workspace_size(B, T, H, d_k, d_v, int(chunk), _DT[dtype], int(flags))
    return -1 if n == ctypes.c_size_t(-1).value else int(n)


def la_bwd_chunk_norm(q, k, v, dout, gamma, cu_seqlens=None, chunk=64, phi="elu1", dq=None, dk=None, dv=None,
                      flags=LA_FLAG_NONE, workspace=None, stream=None):
    """Gradients of la_fwd_chunk's normalised forward (see la_bwd_chunk_norm in
    include/la_b200.h): returns (dq, dk, dv)."""
    lib = load_library()
    B, T, H, d_k = q.shape
    n_seqs = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if gamma.dtype != torch.float32 or gamma.numel() != H:
        raise TypeError("gamma must be float32 with H entries")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = bwd_norm_workspace_size(B, T, H, d_k, v.shape[3], chunk, q.dtype, flags)
    if need > 0 and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    t = [describe(x) for x in (q, k, v, dout, dq, dk, dv)]
    st = lib.la_bwd_chunk_norm(*[ctypes.byref(x) for x in t[:4]], gamma.data_ptr(),
                               None if cu_seqlens is None else cu_seqlens.data_ptr(), n_seqs, int(chunk), _PHI[phi],
                               *[ctypes.byref(x) for x in t[4:]], int(flags),
                               None if workspace is None else workspace.data_ptr(),
                               0 if workspace is None else workspace.numel() * workspace.element_size(),
                               _stream(stream))
    _check(lib, st, "la_bwd_chunk_norm")
    return dq, dk, dv


def la_bwd_chunk_gated_norm(q, k, v, dout, g, cu_seqlens=None, chunk=64, phi="elu1", dq=None, dk=None, dv=None,
                            dg=None, flags=LA_FLAG_NONE, workspace=None, stream=None):
    """Gradients of la_fwd_chunk_gated's normalised forward (see la_bwd_chunk_gated_norm in
    include/la_b200.h): returns (dq, dk, dv, dg), dg float32 [B, T, H] for the log decays g."""
    lib = load_library()
    B, T, H, d_k = q.shape
    n_seqs = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if g.dtype != torch.float32 or tuple(g.shape) != (B, T, H) or not g.is_contiguous():
        raise TypeError("g must be a contiguous float32 [B, T, H] tensor")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    dg = torch.empty_like(g) if dg is None else dg
    need = bwd_norm_workspace_size(B, T, H, d_k, v.shape[3], chunk, q.dtype, flags)
    if need > 0 and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    t = [describe(x) for x in (q, k, v, dout, dq, dk, dv)]
    st = lib.la_bwd_chunk_gated_norm(*[ctypes.byref(x) for x in t[:4]], g.data_ptr(),
                                     None if cu_seqlens is None else cu_seqlens.data_ptr(), n_seqs, int(chunk),
                                     _PHI[phi], *[ctypes.byref(x) for x in t[4:]], dg.data_ptr(), int(flags),
                                     None if workspace is None else workspace.data_ptr(),
                                     0 if workspace is None else workspace.numel() * workspace.element_size(),
                                     _stream(stream))
    _check(lib, st, "la_bwd_chunk_gated_norm")
    return dq, dk, dv, dg


def la_norm_gate(o, gate, w, eps=1e-5, y=None, stream=None):
    """y = RMSNorm(o) * w * swish(gate) per (token, head) over d_v (see la_norm_gate in
    include/la_b200.h).  y defaults to a new tensor; pass y=o to work in place."""
    lib = load_library()
    if y is None:
        y = torch.empty_like(o)
    if w.dtype != torch.float32 or w.numel() != o.shape[3]:
        raise TypeError("w must be float32 with d_v entries")
    to, tg, ty = describe(o), describe(gate), describe(y)
    st = lib.la_norm_gate(ctypes.byref(to), ctypes.byref(tg), w.data_ptr(), float(eps), ctypes.byref(ty),
                          _stream(stream))
    _check(lib, st, "la_norm_gate")
    return y


def la_fwd_chunk_normgate(q, k, v, gamma, gate, w, eps=1e-5, cu_seqlens=None, chunk=64, phi="identity",
                          normalize=False, out=None, final_state=None, flags=LA_FLAG_NONE, workspace=None,
                          stream=None):
    """Forward whose output is la_norm_gate(o, gate, w, eps) (see la_fwd_chunk_normgate in
    include/la_b200.h).  Returns (out, final_state)."""
    lib = load_library()
    B, T, H, dk = q.shape
    dv = v.shape[3]
    n_seqs = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if w.dtype != torch.float32 or w.numel() != dv:
        raise TypeError("w must be float32 with d_v entries")
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if final_state is None:
        final_state = torch.empty((n_seqs, H, dk, dv), dtype=torch.float32, device=q.device)
    need = workspace_size(B, T, H, dk, dv, n_seqs, cu_seqlens is not None, chunk, q.dtype, flags)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    t = [describe(x) for x in (q, k, v, gate, out)]
    st = lib.la_fwd_chunk_normgate(
        ctypes.byref(t[0]), ctypes.byref(t[1]), ctypes.byref(t[2]), gamma.data_ptr(),
        None if cu_seqlens is None else cu_seqlens.data_ptr(), n_seqs, int(chunk), _PHI[phi], int(bool(normalize)),
        ctypes.byref(t[3]), w.data_ptr(), float(eps), ctypes.byref(t[4]), final_state.data_ptr(), int(flags),
        None if workspace is None else workspace.data_ptr(),
        0 if workspace is None else workspace.numel() * workspace.element_size(), _stream(stream))
    _check(lib, st, "la_fwd_chunk_normgate")
    return out, final_state


def la_fwd_gated_delta(q, k, v, g, beta, cu_seqlens=None, initial_state=None, out=None, final_state=None,
                       return_final_state=True, stream=None):
    """Gated delta rule (see la_fwd_gated_delta in include/la_b200.h).  g, beta float32 [B, T, H];
    initial_state / final_state float32 [N, H, d_k, d_v] (S^T).  Returns (out, final_state)."""
    lib = load_library()
    B, T, H, dk = q.shape
    dv = v.shape[3]
    n_seqs = B if cu_seqlens is None else cu_seqlens.numel() - 1
    for name, t in (("g", g), ("beta", beta)):
        if t.dtype != torch.float32 or tuple(t.shape) != (B, T, H) or not t.is_contiguous():
            raise TypeError("%s must be a contiguous float32 [B, T, H] tensor" % name)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if final_state is None and return_final_state:
        final_state = torch.empty((n_seqs, H, dk, dv), dtype=torch.float32, device=q.device)
    t = [describe(x) for x in (q, k, v, out)]
    st = lib.la_fwd_gated_delta(ctypes.byref(t[0]), ctypes.byref(t[1]), ctypes.byref(t[2]), g.data_ptr(),
                                beta.data_ptr(), None if cu_seqlens is None else cu_seqlens.data_ptr(), n_seqs,
                                None if initial_state is None else initial_state.data_ptr(), ctypes.byref(t[3]),
                                None if final_state is None else final_state.data_ptr(), _stream(stream))
    _check(lib, st, "la_fwd_gated_delta")
    return out, final_state


def gated_delta_workspace_size(B, T, H, d_k, d_v, n_seqs, varlen, dtype=torch.bfloat16, flags=0) -> int:
    """Bytes of workspace la_fwd_gated_delta_chunk needs (0: none)."""
    lib = load_library()
    n = lib.la_fwd_gated_delta_workspace_size(B, T, H, d_k, d_v, n_seqs, int(bool(varlen)), _DT[dtype], flags)
    if n == ctypes.c_size_t(-1).value:
        raise LaError(LA_ERR_INVALID_ARG, "la_fwd_gated_delta_workspace_size rejected the arguments")
    return n


def la_fwd_gated_delta_chunk(q, k, v, g, beta, cu_seqlens=None, initial_state=None, out=None, final_state=None,
                             return_final_state=True, flags=0, workspace=None, stream=None):
    """Gated delta rule in chunks (see la_fwd_gated_delta_chunk in include/la_b200.h): same
    arguments and results as :func:`la_fwd_gated_delta`, plus flags and an optional
    caller-owned workspace (allocated here when None)."""
    lib = load_library()
    B, T, H, dk = q.shape
    dv = v.shape[3]
    n_seqs = B if cu_seqlens is None else cu_seqlens.numel() - 1
    for name, t in (("g", g), ("beta", beta)):
        if t.dtype != torch.float32 or tuple(t.shape) != (B, T, H) or not t.is_contiguous():
            raise TypeError("%s must be a contiguous float32 [B, T, H] tensor" % name)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if final_state is None and return_final_state:
        final_state = torch.empty((n_seqs, H, dk, dv), dtype=torch.float32, device=q.device)
    if cu_seqlens is not None and cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    need = gated_delta_workspace_size(B, T, H, dk, dv, n_seqs, cu_seqlens is not None, q.dtype, flags)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    t = [describe(x) for x in (q, k, v, out)]
    st = lib.la_fwd_gated_delta_chunk(ctypes.byref(t[0]), ctypes.byref(t[1]), ctypes.byref(t[2]), g.data_ptr(),
                                      beta.data_ptr(), None if cu_seqlens is None else cu_seqlens.data_ptr(),
                                      n_seqs, None if initial_state is None else initial_state.data_ptr(),
                                      ctypes.byref(t[3]), None if final_state is None else final_state.data_ptr(),
                                      int(flags), None if workspace is None else workspace.data_ptr(),
                                      0 if workspace is None else workspace.numel() * workspace.element_size(),
                                      _stream(stream))
    _check(lib, st, "la_fwd_gated_delta_chunk")
    return out, final_state
