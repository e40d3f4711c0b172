"""The oracle's pins catch plausible mistakes.

Each case copies oracle/la_oracle.c to a temporary directory, plants one
mistake in the copy (the committed oracle is untouched), compiles it with gcc
and checks that the pins of test_oracle.py reject the mutant: the brute-force
quadratic form and the hand-derived fixture.
"""
import ctypes
import json
import os
import subprocess

import numpy as np
import pytest

from test_oracle import GOLD, quadratic_form, rand_qkv, rel

SRC = os.path.join(os.path.dirname(__file__), "..", "oracle", "la_oracle.c")

MUTATIONS = {
    "decay dropped from the state": (
        "Sr[c] = g * Sr[c] + vr * kh[c];", "Sr[c] = Sr[c] + vr * kh[c];"),
    "decay dropped from the normaliser": (
        "z[c] = g * z[c] + kh[c];", "z[c] = z[c] + kh[c];"),
    "output read before the update (diagonal excluded)": (
        "Sr[c] = g * Sr[c] + vr * kh[c];\n          num += Sr[c] * qh[c];",
        "num += Sr[c] * qh[c];\n          Sr[c] = g * Sr[c] + vr * kh[c];"),
    "elu+1 missing the +1": (
        "return x > 0.0 ? x + 1.0 : exp(x);", "return x > 0.0 ? x : exp(x);"),
    "final state stored untransposed": (
        "F[c * dv + r0 + i] = S[i * dk + c];", "F[(r0 + i) * dk + c] = S[i * dk + c];"),
    "decay applied twice": (
        "Sr[c] = g * Sr[c] + vr * kh[c];", "Sr[c] = g * g * Sr[c] + vr * kh[c];"),
}


def _build(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, name
    mpath = tmp_path / "mut.c"
    mpath.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC", "-shared", str(mpath), "-o", str(so), "-lm"])
    lib = ctypes.CDLL(str(so))
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.oracle_recurrent.argtypes = [vp, vp, vp, i32, i64, i64, i64, i64, i64, vp, vp, i64, i32, i32, vp, vp, i32]
    lib.oracle_recurrent.restype = i32
    return lib


def _run(lib, q, k, v, gamma, phi, normalize):
    B, T, H, dk = q.shape
    dv = v.shape[3]
    q, k, v = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v))
    g = np.ascontiguousarray(gamma, dtype=np.float64)
    out = np.zeros((B, T, H, dv))
    fs = np.zeros((B, H, dk, dv))
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)  # noqa: E731
    rc = lib.oracle_recurrent(p(q), p(k), p(v), 2, B, T, H, dk, dv, p(g), None, B,
                              1 if phi == "elu1" else 0, int(normalize), p(out), p(fs), 1)
    assert rc == 0
    return out, fs


def _pins_pass(lib):
    """True when the mutant passes every pin used here."""
    ok = True
    q, k, v = rand_qkv(1, 24, 1, 4, 4, seed=4)
    for gamma, phi, norm in ((0.9, "identity", False), (1.0, "elu1", True), (0.8, "elu1", True)):
        out, _ = _run(lib, q, k, v, [gamma], phi, norm)
        ok &= rel(out[0, :, 0], quadratic_form(q[0, :, 0], k[0, :, 0], v[0, :, 0], gamma, phi, norm)) < 1e-12
    with open(os.path.join(GOLD, "hand_d2_T2.json")) as f:
        G = json.load(f)
    qg, kg, vg = (np.array(G[x], float)[None, :, None] for x in "qkv")
    out, fs = _run(lib, qg, kg, vg, [G["gamma"]], "identity", False)
    ok &= np.allclose(out[0, :, 0], G["out"], atol=1e-15) and np.allclose(fs[0, 0], G["final_state"], atol=1e-15)
    return bool(ok)


def test_unmutated_copy_passes(tmp_path):
    lib = _build(tmp_path, "none", "#define ROWS_PER_TASK 8", "#define ROWS_PER_TASK 8")
    assert _pins_pass(lib)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutant_is_caught(tmp_path, name):
    old, new = MUTATIONS[name]
    lib = _build(tmp_path, name, old, new)
    assert not _pins_pass(lib), name


# ---------------------------------------------------------------- per-token-decay backward
GATED_BWD_MUTATIONS = {
    "dg without the decay's own factor": (
        "dg[row * H + h] = a * inner;", "dg[row * H + h] = inner;"),
    "reverse carry decayed by the current token's factor": (
        "D[r * dk + c] = a_next * D[r * dk + c] + d * qh[c];", "D[r * dk + c] = a * D[r * dk + c] + d * qh[c];"),
    "dg paired with the state after the token": (
        "const double *P = prev + (size_t)t * sz;",
        "const double *P = t + 1 < len ? prev + (size_t)(t + 1) * sz : S;"),
}


def _gated_bwd(lib, q, k, v, dout, g):
    B, T, H, dk = q.shape
    dv = v.shape[3]
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.oracle_backward_gated.argtypes = [vp, vp, vp, vp, i32, i64, i64, i64, i64, i64, vp, vp, i64, i32,
                                          vp, vp, vp, vp, i32]
    lib.oracle_backward_gated.restype = i32
    q, k, v, dout, g = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v, dout, g))
    outs = [np.zeros(q.shape), np.zeros(k.shape), np.zeros(v.shape), np.zeros((B, T, H))]
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)  # noqa: E731
    rc = lib.oracle_backward_gated(p(q), p(k), p(v), p(dout), 2, B, T, H, dk, dv, p(g), None, B, 0,
                                   *(p(o) for o in outs), 1)
    assert rc == 0
    return outs


def _gated_bwd_pin_passes(lib):
    """The autograd pin of test_oracle.py: torch float64 gradients through the
    masked form with the cumulative-decay mask."""
    import torch

    T, dk, dv = 12, 3, 2
    q, k, v = rand_qkv(1, T, 1, dk, dv, seed=90)
    rng = np.random.default_rng(91)
    dout = rng.standard_normal((1, T, 1, dv))
    g = np.log(rng.uniform(0.3, 1.0, (1, T, 1)))
    got = _gated_bwd(lib, q, k, v, dout, g)
    qt, kt, vt, lg = (torch.tensor(x[0, :, 0], dtype=torch.float64, requires_grad=True) for x in (q, k, v, g))
    b = torch.cumsum(lg, 0)
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    M = torch.where(i >= j, torch.exp(b[:, None] - b[None, :]), torch.zeros((), dtype=torch.float64))
    (((qt @ kt.T) * M) @ vt * torch.tensor(dout[0, :, 0])).sum().backward()
    want = [qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy(), lg.grad.numpy()]
    return all(rel(a[0, :, 0], w) < 1e-11 for a, w in zip(got, want))


def test_unmutated_copy_passes_gated_backward_pin(tmp_path):
    lib = _build(tmp_path, "none", "#define ROWS_PER_TASK 8", "#define ROWS_PER_TASK 8")
    assert _gated_bwd_pin_passes(lib)


@pytest.mark.parametrize("name", sorted(GATED_BWD_MUTATIONS))
def test_gated_backward_mutant_is_caught(tmp_path, name):
    old, new = GATED_BWD_MUTATIONS[name]
    lib = _build(tmp_path, name, old, new)
    assert not _gated_bwd_pin_passes(lib), name


NORM_BWD_MUTATIONS = {
    "dq without the denominator's term e_t z_t": (
        "        double acc = E[t] * z[c];\n        for (int64_t r = 0; r < dv; ++r) acc += S[r * dk + c] * u[r];",
        "        double acc = 0.0;\n        for (int64_t r = 0; r < dv; ++r) acc += S[r * dk + c] * u[r];"),
    "dk without the z adjoint g_t": (
        "        double acc = z[c];\n        for (int64_t r = 0; r < dv; ++r) acc += S[r * dk + c] * orc_load(v, dtype, vb + r);",
        "        double acc = 0.0;\n        for (int64_t r = 0; r < dv; ++r) acc += S[r * dk + c] * orc_load(v, dtype, vb + r);"),
    "denominator's adjoint with the wrong sign": (
        "E[t] = -dot / den;", "E[t] = dot / den;"),
    "z adjoint not decayed": (
        "for (int64_t c = 0; c < dk; ++c) z[c] = g * z[c] + E[t] * qh[c];",
        "for (int64_t c = 0; c < dk; ++c) z[c] = z[c] + E[t] * qh[c];"),
}


def _norm_bwd(lib, q, k, v, dout, gamma):
    B, T, H, dk = q.shape
    dv = v.shape[3]
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.oracle_backward_norm.argtypes = [vp, vp, vp, vp, i32, i64, i64, i64, i64, i64, vp, vp, i64, i32,
                                         vp, vp, vp, i32]
    lib.oracle_backward_norm.restype = i32
    q, k, v, dout, gamma = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v, dout, gamma))
    outs = [np.zeros(q.shape), np.zeros(k.shape), np.zeros(v.shape)]
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)  # noqa: E731
    rc = lib.oracle_backward_norm(p(q), p(k), p(v), p(dout), 2, B, T, H, dk, dv, p(gamma), None, B, 1,
                                  *(p(o) for o in outs), 1)
    assert rc == 0
    return outs


def _norm_bwd_pin_passes(lib):
    """The autograd pin of test_oracle.py: torch float64 gradients through the
    normalised masked form with elu + 1."""
    import torch

    T, dk, dv = 12, 3, 2
    q, k, v = rand_qkv(1, T, 1, dk, dv, seed=97)
    dout = np.random.default_rng(98).standard_normal((1, T, 1, dv))
    gam = 0.85
    got = _norm_bwd(lib, q, k, v, dout, np.array([gam]))
    qt, kt, vt = (torch.tensor(x[0, :, 0], dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    f = lambda x: torch.where(x > 0, x + 1.0, torch.exp(torch.clamp(x, max=0.0)))  # noqa: E731
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    M = torch.where(i >= j, torch.tensor(gam, dtype=torch.float64) ** (i - j).clamp(min=0).double(),
                    torch.zeros((), dtype=torch.float64))
    P = (f(qt) @ f(kt).T) * M
    ((P @ vt) / P.sum(dim=1, keepdim=True) * torch.tensor(dout[0, :, 0])).sum().backward()
    want = [qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()]
    return all(rel(a[0, :, 0], w) < 1e-11 for a, w in zip(got, want))


def test_unmutated_copy_passes_norm_backward_pin(tmp_path):
    lib = _build(tmp_path, "none", "#define ROWS_PER_TASK 8", "#define ROWS_PER_TASK 8")
    assert _norm_bwd_pin_passes(lib)


@pytest.mark.parametrize("name", sorted(NORM_BWD_MUTATIONS))
def test_norm_backward_mutant_is_caught(tmp_path, name):
    old, new = NORM_BWD_MUTATIONS[name]
    lib = _build(tmp_path, name, old, new)
    assert not _norm_bwd_pin_passes(lib), name


GATED_NORM_BWD_MUTATIONS = {
    "dg without the normaliser's term gz . z_{t-1}": (
        "      for (int64_t c = 0; c < dk; ++c) inner += gz[c] * Z[c];\n", ""),
    "z adjoint gz not decayed": (
        "gz[c] = a_next * gz[c] + E[t] * qh[c];", "gz[c] = gz[c] + E[t] * qh[c];"),
    "denominator's adjoint with the wrong sign (per-token decay)": (
        "E[t] = -(dot / den);", "E[t] = dot / den;"),
    "dg paired with z after the token": (
        "*Z = prevz + (size_t)t * dk;", "*Z = t + 1 < len ? prevz + (size_t)(t + 1) * dk : z;"),
}


def _gated_norm_bwd(lib, q, k, v, dout, g):
    B, T, H, dk = q.shape
    dv = v.shape[3]
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.oracle_backward_gated_norm.argtypes = [vp, vp, vp, vp, i32, i64, i64, i64, i64, i64, vp, vp, i64, i32,
                                               vp, vp, vp, vp, i32]
    lib.oracle_backward_gated_norm.restype = i32
    q, k, v, dout, g = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v, dout, g))
    outs = [np.zeros(q.shape), np.zeros(k.shape), np.zeros(v.shape), np.zeros(g.shape)]
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)  # noqa: E731
    rc = lib.oracle_backward_gated_norm(p(q), p(k), p(v), p(dout), 2, B, T, H, dk, dv, p(g), None, B, 1,
                                        *(p(o) for o in outs), 1)
    assert rc == 0
    return outs


def _gated_norm_bwd_pin_passes(lib):
    """The autograd pin of test_oracle.py: torch float64 gradients (dq, dk, dv, dg)
    through the normalised masked form with the cumulative-decay mask and elu + 1."""
    import torch

    T, dk, dv = 12, 3, 2
    q, k, v = rand_qkv(1, T, 1, dk, dv, seed=112)
    dout = np.random.default_rng(113).standard_normal((1, T, 1, dv))
    g = np.log(np.random.default_rng(114).uniform(0.3, 1.0, (1, T, 1)))
    got = _gated_norm_bwd(lib, q, k, v, dout, g)
    qt, kt, vt, lg = (torch.tensor(x[0, :, 0], dtype=torch.float64, requires_grad=True) for x in (q, k, v, g))
    f = lambda x: torch.where(x > 0, x + 1.0, torch.exp(torch.clamp(x, max=0.0)))  # noqa: E731
    b = torch.cumsum(lg, 0)
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    M = torch.where(i >= j, torch.exp(b[:, None] - b[None, :]), torch.zeros((), dtype=torch.float64))
    P = (f(qt) @ f(kt).T) * M
    ((P @ vt) / P.sum(dim=1, keepdim=True) * torch.tensor(dout[0, :, 0])).sum().backward()
    want = [qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy(), lg.grad.numpy()]
    return all(rel(a[0, :, 0], w) < 1e-10 for a, w in zip(got, want))


def test_unmutated_copy_passes_gated_norm_backward_pin(tmp_path):
    lib = _build(tmp_path, "none", "#define ROWS_PER_TASK 8", "#define ROWS_PER_TASK 8")
    assert _gated_norm_bwd_pin_passes(lib)


@pytest.mark.parametrize("name", sorted(GATED_NORM_BWD_MUTATIONS))
def test_gated_norm_backward_mutant_is_caught(tmp_path, name):
    old, new = GATED_NORM_BWD_MUTATIONS[name]
    lib = _build(tmp_path, name, old, new)
    assert not _gated_norm_bwd_pin_passes(lib), name
