"""float64 CPU oracle for causal linear attention -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The product
path (the CUDA library and its Python binding) never imports it, and this
package imports nothing from the product.

The arithmetic lives in ``la_oracle.c`` (plain C, float64, OpenMP over
independent (sequence, head, state-row) tasks); this module builds it with gcc
and marshals numpy arrays to it.  What each function computes, and the passage
it follows, is stated in the C file's header:

* ``recurrent`` -- the token-by-token recurrence of "1.6 长上下文与高效注意力",
  section 线性注意力 (displayed equation for o_t, S_t, z_t), with a per-head
  constant decay gamma on the old state and the normaliser.
* ``chunked``   -- the same result regrouped into chunks (a restatement used to
  pin chunk-size invariance).
* ``step``      -- one decode token on a given state.
* ``final_z``   -- the normaliser's key sum z after each sequence's last token.
* ``step_norm`` -- one normalised decode token (state and z updated).
* ``backward``  -- dq, dk, dv of sum_t dout_t . o_t (unnormalised; the adjoint
  of the recurrence, token by token).
* ``backward_gated`` -- the same for the per-token decay, plus dg (the log
  decays' gradient); keeps every state, so for test sizes.
* ``backward_norm`` -- dq, dk, dv of sum_t dout_t . o_t through the normalised
  recurrence (o_t divided by z_t . phi(q_t)), token by token.
* ``backward_gated_norm`` -- dq, dk, dv and dg through the normalised recurrence
  with the per-token decay; keeps every state, so for test sizes.
* ``gated_delta`` -- the gated delta rule (section Gated delta rule of the same
  page), token by token, unit-norm keys.
* ``norm_gate``  -- y = RMSNorm(o) * w * swish(g) per (token, head) over d_v.
* ``recurrent_gated``, ``step_gated`` -- the same with a data-dependent decay
  alpha_t = exp(g_t) per token and head (section 状态空间模型与 Mamba of the
  same page: Mamba-2 as linear attention with a decay mask).

Inputs may be numpy float32, float64, or bfloat16 given as raw ``uint16`` bits
(use :func:`bf16_bits`); they are upcast to float64 exactly.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "la_oracle.c")
_LIB = os.path.join(_HERE, "liblaoracle.so")

F32, BF16, F64 = 0, 1, 2
PHI_IDENTITY, PHI_ELU1 = 0, 1
_PHI = {"identity": PHI_IDENTITY, "elu1": PHI_ELU1, PHI_IDENTITY: PHI_IDENTITY, PHI_ELU1: PHI_ELU1}

_lib = None


def build(force: bool = False) -> str:
    """Compile la_oracle.c into liblaoracle.so (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, i32, vp, dp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p
        lib.oracle_recurrent.argtypes = [vp, vp, vp, i32, i64, i64, i64, i64, i64, dp, vp, i64, i32, i32, dp, dp, i32]
        lib.oracle_recurrent.restype = i32
        lib.oracle_chunked.argtypes = [vp, vp, vp, i32, i64, i64, i64, i64, i64, dp, vp, i64, i64, i32, i32, dp, dp, i32]
        lib.oracle_chunked.restype = i32
        lib.oracle_step.argtypes = [vp, vp, vp, i32, i64, i64, i64, i64, dp, dp, dp, i32, i32]
        lib.oracle_final_z.argtypes = [vp, i32, i64, i64, i64, i64, dp, vp, i64, i32, dp, i32]
        lib.oracle_final_z.restype = i32
        lib.oracle_step_norm.argtypes = [vp, vp, vp, i32, i64, i64, i64, i64, dp, dp, dp, dp, i32, i32]
        lib.oracle_step_norm.restype = i32
        lib.oracle_recurrent_gated.argtypes = [vp, vp, vp, i32, i64, i64, i64, i64, i64, dp, vp, i64, i32, i32,
                                               dp, dp, dp, i32]
        lib.oracle_recurrent_gated.restype = i32
        lib.oracle_step_gated.argtypes = [vp, vp, vp, i32, i64, i64, i64, i64, dp, dp, dp, dp, i32, i32]
        lib.oracle_step_gated.restype = i32
        lib.oracle_backward.argtypes = [vp, vp, vp, vp, i32, i64, i64, i64, i64, i64, dp, vp, i64, i32, i32,
                                        dp, dp, dp, i32]
        lib.oracle_backward.restype = i32
        lib.oracle_backward_norm.argtypes = [vp, vp, vp, vp, i32, i64, i64, i64, i64, i64, dp, vp, i64, i32, dp, dp,
                                             dp, i32]
        lib.oracle_backward_norm.restype = i32
        lib.oracle_backward_gated.argtypes = [vp, vp, vp, vp, i32, i64, i64, i64, i64, i64, dp, vp, i64, i32,
                                              dp, dp, dp, dp, i32]
        lib.oracle_backward_gated.restype = i32
        lib.oracle_backward_gated_norm.argtypes = [vp, vp, vp, vp, i32, i64, i64, i64, i64, i64, dp, vp, i64, i32,
                                                   dp, dp, dp, dp, i32]
        lib.oracle_backward_gated_norm.restype = i32
        lib.oracle_norm_gate.argtypes = [dp, vp, i32, i64, i64, dp, ctypes.c_double, dp, i32]
        lib.oracle_norm_gate.restype = i32
        lib.oracle_gated_delta.argtypes = [vp, vp, vp, i32, i64, i64, i64, i64, i64, dp, dp, vp, i64, dp, dp, dp, i32]
        lib.oracle_gated_delta.restype = i32
        lib.oracle_gated_delta_chunked.argtypes = [vp, vp, vp, i32, i64, i64, i64, i64, i64, dp, dp, vp, i64, dp,
                                                   i64, dp, dp, i32]
        lib.oracle_gated_delta_chunked.restype = i32
        lib.oracle_step.restype = i32
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = i32
        _lib = lib
    return _lib


def _oracle_error(name: str, rc: int) -> Exception:
    """The exception for a non-zero return code of the C oracle."""
    if rc == -20:
        return MemoryError("%s could not allocate its working buffers on this host" % name)
    return ValueError("%s rejected its arguments (code %d)" % (name, rc))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def bf16_bits(x) -> np.ndarray:
    """Raw bfloat16 bits (uint16) of a torch bfloat16 tensor, for the oracle."""
    import torch  # local: only used to view torch bf16 storage

    assert x.dtype == torch.bfloat16
    return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _as_input(a):
    """(contiguous array, oracle dtype code) for a numpy array or torch tensor."""
    try:
        import torch

        if isinstance(a, torch.Tensor):
            if a.dtype == torch.bfloat16:
                return bf16_bits(a), BF16
            a = a.detach().cpu().contiguous().numpy()
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(a)
    if a.dtype == np.float32:
        return a, F32
    if a.dtype == np.float64:
        return a, F64
    if a.dtype == np.uint16:
        return a, BF16
    raise TypeError("oracle inputs must be float32, float64 or bfloat16 bits, got %s" % a.dtype)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _prep(q, k, v, gamma, cu_seqlens):
    q, dq = _as_input(q)
    k, dk_ = _as_input(k)
    v, dv_ = _as_input(v)
    if not (dq == dk_ == dv_):
        raise TypeError("q, k, v must share one dtype")
    if q.ndim != 4 or k.shape != q.shape or v.shape[:3] != q.shape[:3]:
        raise ValueError("q, k must be [B, T, H, d_k] and v [B, T, H, d_v]")
    B, T, H, dk = q.shape
    dv = v.shape[3]
    g = np.ascontiguousarray(np.asarray(gamma, dtype=np.float64).reshape(-1))
    if g.size == 1 and H > 1:
        g = np.full(H, g[0])
    if g.size != H:
        raise ValueError("gamma must have H entries")
    cu = None
    n_seqs = B
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        n_seqs = cu.size - 1
    return q, k, v, dq, B, T, H, dk, dv, g, cu, n_seqs


def recurrent(q, k, v, gamma, cu_seqlens=None, phi="identity", normalize=False, nthreads=0):
    """Token-by-token recurrence; returns (out [B,T,H,d_v], final_state [N,H,d_k,d_v]) in float64."""
    q, k, v, dt, B, T, H, dk, dv, g, cu, n = _prep(q, k, v, gamma, cu_seqlens)
    out = np.zeros((B, T, H, dv), np.float64)
    fs = np.zeros((n, H, dk, dv), np.float64)
    rc = _load().oracle_recurrent(
        _ptr(q), _ptr(k), _ptr(v), dt, B, T, H, dk, dv, _ptr(g), _ptr(cu), n,
        _PHI[phi], int(bool(normalize)), _ptr(out), _ptr(fs), int(nthreads),
    )
    if rc != 0:
        raise _oracle_error("oracle_recurrent", rc)
    return out, fs


def chunked(q, k, v, gamma, chunk, cu_seqlens=None, phi="identity", normalize=False, nthreads=0):
    """Chunked restatement (float64); same outputs as :func:`recurrent` up to rounding."""
    q, k, v, dt, B, T, H, dk, dv, g, cu, n = _prep(q, k, v, gamma, cu_seqlens)
    out = np.zeros((B, T, H, dv), np.float64)
    fs = np.zeros((n, H, dk, dv), np.float64)
    rc = _load().oracle_chunked(
        _ptr(q), _ptr(k), _ptr(v), dt, B, T, H, dk, dv, _ptr(g), _ptr(cu), n, int(chunk),
        _PHI[phi], int(bool(normalize)), _ptr(out), _ptr(fs), int(nthreads),
    )
    if rc != 0:
        raise _oracle_error("oracle_chunked", rc)
    return out, fs


def step(q, k, v, gamma, state, phi="identity", nthreads=0):
    """One decode token.  q,k [N,H,d_k], v [N,H,d_v], state [N,H,d_k,d_v] (S^T).

    Returns (out [N,H,d_v], new_state) in float64; the input state is not modified.
    """
    q, dq = _as_input(q)
    k, _ = _as_input(k)
    v, _ = _as_input(v)
    N, H, dk = q.shape
    dv = v.shape[2]
    st = np.array(state, dtype=np.float64, copy=True, order="C")
    if st.shape != (N, H, dk, dv):
        raise ValueError("state must be [N, H, d_k, d_v]")
    g = np.ascontiguousarray(np.asarray(gamma, dtype=np.float64).reshape(-1))
    if g.size == 1 and H > 1:
        g = np.full(H, g[0])
    out = np.zeros((N, H, dv), np.float64)
    rc = _load().oracle_step(
        _ptr(q), _ptr(k), _ptr(v), dq, N, H, dk, dv, _ptr(g), _ptr(st), _ptr(out), _PHI[phi], int(nthreads)
    )
    if rc != 0:
        raise _oracle_error("oracle_step", rc)
    return out, st


def final_z(k, gamma, cu_seqlens=None, phi="identity", nthreads=0):
    """z after the last token of each sequence: z_t = gamma z_{t-1} + phi(k_t).

    k [B, T, H, d_k]; returns [N, H, d_k] float64.
    """
    k, dt = _as_input(k)
    if k.ndim != 4:
        raise ValueError("k must be [B, T, H, d_k]")
    B, T, H, dk = k.shape
    g = np.ascontiguousarray(np.asarray(gamma, dtype=np.float64).reshape(-1))
    if g.size == 1 and H > 1:
        g = np.full(H, g[0])
    if g.size != H:
        raise ValueError("gamma must have H entries")
    cu, n = None, B
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        n = cu.size - 1
    z = np.zeros((n, H, dk), np.float64)
    rc = _load().oracle_final_z(_ptr(k), dt, B, T, H, dk, _ptr(g), _ptr(cu), n, _PHI[phi], _ptr(z), int(nthreads))
    if rc != 0:
        raise _oracle_error("oracle_final_z", rc)
    return z


def step_norm(q, k, v, gamma, state, z, phi="identity", nthreads=0):
    """One normalised decode token.  q,k [N,H,d_k], v [N,H,d_v], state [N,H,d_k,d_v]
    (S^T), z [N,H,d_k].  Returns (out [N,H,d_v], new_state, new_z) in float64; the
    inputs are not modified."""
    q, dq = _as_input(q)
    k, _ = _as_input(k)
    v, _ = _as_input(v)
    N, H, dk = q.shape
    dv = v.shape[2]
    st = np.array(state, dtype=np.float64, copy=True, order="C")
    zz = np.array(z, dtype=np.float64, copy=True, order="C")
    if st.shape != (N, H, dk, dv) or zz.shape != (N, H, dk):
        raise ValueError("state must be [N, H, d_k, d_v] and z [N, H, d_k]")
    g = np.ascontiguousarray(np.asarray(gamma, dtype=np.float64).reshape(-1))
    if g.size == 1 and H > 1:
        g = np.full(H, g[0])
    out = np.zeros((N, H, dv), np.float64)
    rc = _load().oracle_step_norm(_ptr(q), _ptr(k), _ptr(v), dq, N, H, dk, dv, _ptr(g), _ptr(st), _ptr(zz),
                                  _ptr(out), _PHI[phi], int(nthreads))
    if rc != 0:
        raise _oracle_error("oracle_step_norm", rc)
    return out, st, zz


def recurrent_gated(q, k, v, g, cu_seqlens=None, phi="identity", normalize=False, nthreads=0):
    """Token-by-token recurrence with a per-token decay exp(g[b, t, h]), g <= 0.

    g [B, T, H].  Returns (out [B,T,H,d_v], final_state [N,H,d_k,d_v], final_z [N,H,d_k]) in float64.
    """
    q, k, v, dt, B, T, H, dk, dv, _, cu, n = _prep(q, k, v, np.ones(q.shape[2] if hasattr(q, "shape") else 1),
                                                    cu_seqlens)
    gg = np.ascontiguousarray(np.asarray(g, dtype=np.float64))
    if gg.shape != (B, T, H):
        raise ValueError("g must be [B, T, H]")
    out = np.zeros((B, T, H, dv), np.float64)
    fs = np.zeros((n, H, dk, dv), np.float64)
    fz = np.zeros((n, H, dk), np.float64)
    rc = _load().oracle_recurrent_gated(
        _ptr(q), _ptr(k), _ptr(v), dt, B, T, H, dk, dv, _ptr(gg), _ptr(cu), n,
        _PHI[phi], int(bool(normalize)), _ptr(out), _ptr(fs), _ptr(fz), int(nthreads),
    )
    if rc != 0:
        raise _oracle_error("oracle_recurrent_gated", rc)
    return out, fs, fz


def step_gated(q, k, v, g, state, z=None, phi="identity", nthreads=0):
    """One decode token with decay exp(g[n, h]).  z None: unnormalised; else normalised.

    Returns (out, new_state, new_z or None) in float64; inputs are not modified."""
    q, dq = _as_input(q)
    k, _ = _as_input(k)
    v, _ = _as_input(v)
    N, H, dk = q.shape
    dv = v.shape[2]
    st = np.array(state, dtype=np.float64, copy=True, order="C")
    zz = None if z is None else np.array(z, dtype=np.float64, copy=True, order="C")
    gg = np.ascontiguousarray(np.asarray(g, dtype=np.float64))
    if st.shape != (N, H, dk, dv) or gg.shape != (N, H) or (zz is not None and zz.shape != (N, H, dk)):
        raise ValueError("state [N,H,d_k,d_v], g [N,H], z [N,H,d_k] expected")
    out = np.zeros((N, H, dv), np.float64)
    rc = _load().oracle_step_gated(_ptr(q), _ptr(k), _ptr(v), dq, N, H, dk, dv, _ptr(gg), _ptr(st), _ptr(zz),
                                   _ptr(out), _PHI[phi], int(nthreads))
    if rc != 0:
        raise _oracle_error("oracle_step_gated", rc)
    return out, st, zz


def backward(q, k, v, dout, gamma, cu_seqlens=None, phi="identity", nthreads=0):
    """Gradients of L = sum(dout * o) for the unnormalised recurrence.

    Returns (dq [B,T,H,d_k], dk [B,T,H,d_k], dv [B,T,H,d_v]) in float64."""
    q, k, v, dt, B, T, H, dk, dv, g, cu, n = _prep(q, k, v, gamma, cu_seqlens)
    do, ddt = _as_input(dout)
    if ddt != dt or do.shape != v.shape:
        raise ValueError("dout must be [B, T, H, d_v] of the inputs' dtype")
    gq = np.zeros(q.shape, np.float64)
    gk = np.zeros(k.shape, np.float64)
    gv = np.zeros(v.shape, np.float64)
    rc = _load().oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(do), dt, B, T, H, dk, dv, _ptr(g), _ptr(cu), n,
                                 _PHI[phi], 0, _ptr(gq), _ptr(gk), _ptr(gv), int(nthreads))
    if rc != 0:
        raise _oracle_error("oracle_backward", rc)
    return gq, gk, gv


def backward_norm(q, k, v, dout, gamma, cu_seqlens=None, phi="elu1", nthreads=0):
    """Gradients of L = sum(dout * o) for the normalised recurrence (o_t = S_t qh_t / z_t . qh_t).

    Returns (dq [B,T,H,d_k], dk [B,T,H,d_k], dv [B,T,H,d_v]) in float64."""
    q, k, v, dt, B, T, H, dk, dv, g, cu, n = _prep(q, k, v, gamma, cu_seqlens)
    do, ddt = _as_input(dout)
    if ddt != dt or do.shape != v.shape:
        raise ValueError("dout must be [B, T, H, d_v] of the inputs' dtype")
    gq = np.zeros(q.shape, np.float64)
    gk = np.zeros(k.shape, np.float64)
    gv = np.zeros(v.shape, np.float64)
    rc = _load().oracle_backward_norm(_ptr(q), _ptr(k), _ptr(v), _ptr(do), dt, B, T, H, dk, dv, _ptr(g), _ptr(cu),
                                      n, _PHI[phi], _ptr(gq), _ptr(gk), _ptr(gv), int(nthreads))
    if rc != 0:
        raise _oracle_error("oracle_backward_norm", rc)
    return gq, gk, gv


def backward_gated(q, k, v, dout, g, cu_seqlens=None, phi="identity", nthreads=0):
    """Gradients of L = sum(dout * o) for the unnormalised recurrence with the
    per-token decay exp(g[b, t, h]).

    Returns (dq, dk, dv, dg) in float64; dg [B, T, H] is the gradient of the log decays."""
    q, k, v, dt, B, T, H, dk, dv, _, cu, n = _prep(q, k, v, np.ones(q.shape[2] if hasattr(q, "shape") else 1),
                                                    cu_seqlens)
    do, ddt = _as_input(dout)
    if ddt != dt or do.shape != v.shape:
        raise ValueError("dout must be [B, T, H, d_v] of the inputs' dtype")
    gg = np.ascontiguousarray(np.asarray(g, dtype=np.float64))
    if gg.shape != (B, T, H):
        raise ValueError("g must be [B, T, H]")
    gq = np.zeros(q.shape, np.float64)
    gk = np.zeros(k.shape, np.float64)
    gv = np.zeros(v.shape, np.float64)
    gd = np.zeros((B, T, H), np.float64)
    rc = _load().oracle_backward_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(do), dt, B, T, H, dk, dv, _ptr(gg), _ptr(cu),
                                       n, _PHI[phi], _ptr(gq), _ptr(gk), _ptr(gv), _ptr(gd), int(nthreads))
    if rc != 0:
        raise _oracle_error("oracle_backward_gated", rc)
    return gq, gk, gv, gd


def backward_gated_norm(q, k, v, dout, g, cu_seqlens=None, phi="elu1", nthreads=0):
    """Gradients of L = sum(dout * o) for the normalised recurrence with the per-token
    decay exp(g[b, t, h]) (o_t = S_t qh_t / z_t . qh_t).

    Returns (dq, dk, dv, dg) in float64; dg [B, T, H] is the gradient of the log decays."""
    q, k, v, dt, B, T, H, dk, dv, _, cu, n = _prep(q, k, v, np.ones(q.shape[2] if hasattr(q, "shape") else 1),
                                                    cu_seqlens)
    do, ddt = _as_input(dout)
    if ddt != dt or do.shape != v.shape:
        raise ValueError("dout must be [B, T, H, d_v] of the inputs' dtype")
    gg = np.ascontiguousarray(np.asarray(g, dtype=np.float64))
    if gg.shape != (B, T, H):
        raise ValueError("g must be [B, T, H]")
    gq = np.zeros(q.shape, np.float64)
    gk = np.zeros(k.shape, np.float64)
    gv = np.zeros(v.shape, np.float64)
    gd = np.zeros((B, T, H), np.float64)
    rc = _load().oracle_backward_gated_norm(_ptr(q), _ptr(k), _ptr(v), _ptr(do), dt, B, T, H, dk, dv, _ptr(gg),
                                            _ptr(cu), n, _PHI[phi], _ptr(gq), _ptr(gk), _ptr(gv), _ptr(gd),
                                            int(nthreads))
    if rc != 0:
        raise _oracle_error("oracle_backward_gated_norm", rc)
    return gq, gk, gv, gd


def norm_gate(o, g, w, eps=1e-5, nthreads=0):
    """y = o / sqrt(mean(o^2) + eps) * w * g * sigmoid(g) over the last axis (d_v).

    o float64 [..., d_v]; g [..., d_v] (float32 / float64 / bfloat16); w [d_v].  Returns float64."""
    oo = np.ascontiguousarray(np.asarray(o, dtype=np.float64))
    gg, dt = _as_input(g)
    ww = np.ascontiguousarray(np.asarray(w, dtype=np.float64).reshape(-1))
    dv = oo.shape[-1]
    if gg.shape != oo.shape or ww.size != dv:
        raise ValueError("g must match o and w must have d_v entries")
    y = np.zeros_like(oo)
    rc = _load().oracle_norm_gate(_ptr(oo), _ptr(gg), dt, oo.size // dv, dv, _ptr(ww), float(eps), _ptr(y),
                                  int(nthreads))
    if rc != 0:
        raise _oracle_error("oracle_norm_gate", rc)
    return y


def gated_delta(q, k, v, g, beta, cu_seqlens=None, init=None, nthreads=0):
    """Gated delta rule: S_t = exp(g_t) S_{t-1} (I - beta_t kt kt^T) + beta_t v_t kt^T, o_t = S_t q_t,
    kt = k_t / |k_t|.  g, beta [B, T, H]; init None or [N, H, d_k, d_v] (S^T).

    Returns (out [B,T,H,d_v], final_state [N,H,d_k,d_v]) in float64."""
    q, k, v, dt, B, T, H, dk, dv, _, cu, n = _prep(q, k, v, np.ones(q.shape[2]), cu_seqlens)
    gg = np.ascontiguousarray(np.asarray(g, dtype=np.float64))
    bb = np.ascontiguousarray(np.asarray(beta, dtype=np.float64))
    if gg.shape != (B, T, H) or bb.shape != (B, T, H):
        raise ValueError("g and beta must be [B, T, H]")
    ii = None if init is None else np.ascontiguousarray(np.asarray(init, dtype=np.float64))
    if ii is not None and ii.shape != (n, H, dk, dv):
        raise ValueError("init must be [N, H, d_k, d_v]")
    out = np.zeros((B, T, H, dv), np.float64)
    fs = np.zeros((n, H, dk, dv), np.float64)
    rc = _load().oracle_gated_delta(_ptr(q), _ptr(k), _ptr(v), dt, B, T, H, dk, dv, _ptr(gg), _ptr(bb), _ptr(cu),
                                    n, _ptr(ii), _ptr(out), _ptr(fs), int(nthreads))
    if rc != 0:
        raise _oracle_error("oracle_gated_delta", rc)
    return out, fs


def gated_delta_chunked(q, k, v, g, beta, chunk, cu_seqlens=None, init=None, nthreads=0):
    """The gated delta rule regrouped into chunks of `chunk` tokens (float64): per chunk
    the unit lower-triangular system for the writes u_i is solved by T = (I + A)^{-1}.
    Same arguments and results as :func:`gated_delta`, equal to them up to rounding."""
    q, k, v, dt, B, T, H, dk, dv, _, cu, n = _prep(q, k, v, np.ones(q.shape[2]), cu_seqlens)
    gg = np.ascontiguousarray(np.asarray(g, dtype=np.float64))
    bb = np.ascontiguousarray(np.asarray(beta, dtype=np.float64))
    if gg.shape != (B, T, H) or bb.shape != (B, T, H):
        raise ValueError("g and beta must be [B, T, H]")
    ii = None if init is None else np.ascontiguousarray(np.asarray(init, dtype=np.float64))
    if ii is not None and ii.shape != (n, H, dk, dv):
        raise ValueError("init must be [N, H, d_k, d_v]")
    out = np.zeros((B, T, H, dv), np.float64)
    fs = np.zeros((n, H, dk, dv), np.float64)
    rc = _load().oracle_gated_delta_chunked(_ptr(q), _ptr(k), _ptr(v), dt, B, T, H, dk, dv, _ptr(gg), _ptr(bb),
                                            _ptr(cu), n, _ptr(ii), int(chunk), _ptr(out), _ptr(fs), int(nthreads))
    if rc != 0:
        raise _oracle_error("oracle_gated_delta_chunked", rc)
    return out, fs
