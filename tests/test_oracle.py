"""Pins for the float64 oracle (CPU only).

Each test pins the oracle to something other than itself:
  * the quadratic (parallel) masked form written out here by brute force --
    a different formula for the same result ("1.6 长上下文与高效注意力",
    section 线性注意力: training may run in parallel form; the page's listing
    asserts parallel form == recurrent form);
  * hand-derived values (tests/golden/*.json, derivations inside);
  * closed forms for constant inputs, and special cases (T = 1, gamma = 0,
    d = 1, varlen == independent runs, prefill + one decode step == prefill
    of one more token);
  * invariance of the chunked restatement to the chunk size.
A plausible slip anywhere -- a dropped decay, the diagonal excluded, S used
transposed, the normaliser taken before the update, a wrong power of gamma in
the chunk carry -- fails at least one of these.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

GOLD = os.path.join(os.path.dirname(__file__), "golden")
TOL = 1e-12


def phi_np(x, kind):
    if kind == "elu1":
        return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))
    return x


def quadratic_form(q, k, v, gamma, phi, normalize):
    """O = ((phi(Q) phi(K)^T) * M_gamma) V [/ row sums], M[i,j] = gamma^(i-j) for i >= j.

    One sequence, one head: q, k [T, d_k], v [T, d_v] (float64).
    """
    T = q.shape[0]
    A = phi_np(q, phi) @ phi_np(k, phi).T
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    with np.errstate(divide="ignore", invalid="ignore"):
        M = np.where(i >= j, np.power(float(gamma), np.maximum(i - j, 0).astype(np.float64)), 0.0)
    P = A * M
    O = P @ v
    if normalize:
        O = O / P.sum(axis=1, keepdims=True)
    return O


def rel(x, ref):
    den = np.max(np.abs(ref))
    return float(np.max(np.abs(x - ref)) / (den if den > 0 else 1.0))


def rand_qkv(B, T, H, dk, dv, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, dk)) * scale
    k = rng.standard_normal((B, T, H, dk)) * scale
    v = rng.standard_normal((B, T, H, dv))
    return q, k, v


# ---------------------------------------------------------------- brute force
@pytest.mark.parametrize("T", [1, 2, 3, 17, 64])
@pytest.mark.parametrize("d", [1, 4, 16])
@pytest.mark.parametrize("gamma", [0.0, 0.5, 0.9, 1.0])
@pytest.mark.parametrize("phi,normalize", [("identity", False), ("elu1", False), ("elu1", True)])
def test_recurrent_equals_quadratic(oracle_mod, T, d, gamma, phi, normalize):
    B, H = 2, 2
    q, k, v = rand_qkv(B, T, H, d, d + 1, seed=T * 131 + d)
    out, _ = oracle_mod.recurrent(q, k, v, [gamma] * H, phi=phi, normalize=normalize)
    for b in range(B):
        for h in range(H):
            ref = quadratic_form(q[b, :, h], k[b, :, h], v[b, :, h], gamma, phi, normalize)
            assert rel(out[b, :, h], ref) < TOL


def test_final_state_equals_weighted_outer_sum(oracle_mod):
    """S_T = sum_j gamma^(T-1-j) v_j phi(k_j)^T, stored transposed ([d_k][d_v])."""
    T, dk, dv, g = 37, 5, 3, 0.8
    q, k, v = rand_qkv(1, T, 1, dk, dv, seed=3)
    _, fs = oracle_mod.recurrent(q, k, v, [g], phi="elu1")
    kh = phi_np(k[0, :, 0], "elu1")
    S = sum(g ** (T - 1 - j) * np.outer(v[0, j, 0], kh[j]) for j in range(T))
    assert rel(fs[0, 0], S.T) < TOL


def test_page_listing_check(oracle_mod):
    """The page's listing compares parallel and recurrent forms at T=50, d=16,
    phi = elu+1, normalised, gamma = 1, and reports agreement within atol 1e-5.
    Here the parallel form is computed independently (float64) and compared
    with the oracle on inputs drawn the same way (torch.manual_seed(0), three
    standard-normal [T, d] tensors)."""
    torch.manual_seed(0)
    qt, kt, vt = (torch.randn(50, 16) for _ in range(3))
    q, k, v = (x.double().numpy() for x in (qt, kt, vt))
    par = quadratic_form(q, k, v, 1.0, "elu1", True)
    out, _ = oracle_mod.recurrent(q[None, :, None], k[None, :, None], v[None, :, None], [1.0],
                                  phi="elu1", normalize=True)
    assert np.max(np.abs(out[0, :, 0] - par)) < 1e-5
    assert rel(out[0, :, 0], par) < TOL


# ---------------------------------------------------------------- hand values
def test_golden_hand_d2(oracle_mod):
    with open(os.path.join(GOLD, "hand_d2_T2.json")) as f:
        G = json.load(f)
    q = np.array(G["q"], float)[None, :, None]
    k = np.array(G["k"], float)[None, :, None]
    v = np.array(G["v"], float)[None, :, None]
    out, fs = oracle_mod.recurrent(q, k, v, [G["gamma"]])
    np.testing.assert_allclose(out[0, :, 0], G["out"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(fs[0, 0], G["final_state"], rtol=0, atol=1e-15)
    outn, _ = oracle_mod.recurrent(q, k, v, [G["gamma"]], normalize=True)
    np.testing.assert_allclose(outn[0, :, 0], G["out_normalized"], rtol=0, atol=1e-15)
    s = G["step"]
    o, st = oracle_mod.step(np.array(s["q"], float)[None, None], np.array(s["k"], float)[None, None],
                            np.array(s["v"], float)[None, None], [G["gamma"]], fs)
    np.testing.assert_allclose(st[0, 0], s["state_out"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(o[0, 0], s["out"], rtol=0, atol=1e-15)


def test_golden_hand_d1_elu(oracle_mod):
    with open(os.path.join(GOLD, "hand_d1_elu.json")) as f:
        G = json.load(f)
    ev = lambda e: eval(e, {"exp": math.exp})  # noqa: E731  (expressions from the fixture)
    q = np.array(G["q"], float)[None, :, None, None]
    k = np.array(G["k"], float)[None, :, None, None]
    v = np.array(G["v"], float)[None, :, None, None]
    out, fs = oracle_mod.recurrent(q, k, v, [G["gamma"]], phi="elu1")
    np.testing.assert_allclose(out.reshape(-1), [ev(e) for e in G["expr_out"]], rtol=1e-15)
    np.testing.assert_allclose(fs.reshape(-1), [ev(G["expr_final_state"])], rtol=1e-15)
    outn, _ = oracle_mod.recurrent(q, k, v, [G["gamma"]], phi="elu1", normalize=True)
    np.testing.assert_allclose(outn.reshape(-1), [ev(e) for e in G["expr_out_normalized"]], rtol=1e-15)


# ---------------------------------------------------------------- closed forms
@pytest.mark.parametrize("phi", ["identity", "elu1"])
@pytest.mark.parametrize("gamma", [1.0, 0.9, 0.3])
def test_constant_inputs_closed_form(oracle_mod, phi, gamma):
    T, dk, dv = 40, 6, 4
    rng = np.random.default_rng(11)
    qv, kv, vv = rng.standard_normal(dk), np.abs(rng.standard_normal(dk)), rng.standard_normal(dv)
    q = np.broadcast_to(qv, (1, T, 1, dk)).copy()
    k = np.broadcast_to(kv, (1, T, 1, dk)).copy()
    v = np.broadcast_to(vv, (1, T, 1, dv)).copy()
    out, fs = oracle_mod.recurrent(q, k, v, [gamma], phi=phi)
    qh, kh = phi_np(qv, phi), phi_np(kv, phi)
    t = np.arange(1, T + 1, dtype=np.float64)
    w = t if gamma == 1.0 else (1 - gamma ** t) / (1 - gamma)  # sum_{j<t} gamma^j
    ref = w[:, None] * (qh @ kh) * vv[None, :]
    assert rel(out[0, :, 0], ref) < TOL
    assert rel(fs[0, 0], w[-1] * np.outer(kh, vv)) < TOL
    if phi == "elu1":  # normalised: every output equals v exactly
        outn, _ = oracle_mod.recurrent(q, k, v, [gamma], phi=phi, normalize=True)
        assert np.max(np.abs(outn[0, :, 0] - vv[None, :])) < 1e-13


# ---------------------------------------------------------------- special cases
def test_single_token_and_gamma_zero(oracle_mod):
    q, k, v = rand_qkv(1, 30, 2, 8, 5, seed=5)
    for phi in ("identity", "elu1"):
        qh, kh = phi_np(q, phi), phi_np(k, phi)
        o1, _ = oracle_mod.recurrent(q[:, :1], k[:, :1], v[:, :1], [0.7, 1.0], phi=phi)
        ref1 = np.einsum("bthc,bthc->bth", qh[:, :1], kh[:, :1])[..., None] * v[:, :1]
        assert rel(o1, ref1) < TOL
        o0, fs0 = oracle_mod.recurrent(q, k, v, [0.0, 0.0], phi=phi)
        ref0 = np.einsum("bthc,bthc->bth", qh, kh)[..., None] * v
        assert rel(o0, ref0) < TOL
        assert rel(fs0[0], np.einsum("hc,hr->hcr", kh[0, -1], v[0, -1])) < TOL


def test_d1_scalar_ewma(oracle_mod):
    T, g = 25, 0.75
    q, k, v = rand_qkv(1, T, 1, 1, 1, seed=9)
    out, _ = oracle_mod.recurrent(q, k, v, [g])
    s, ref = 0.0, []
    for t in range(T):
        s = g * s + v[0, t, 0, 0] * k[0, t, 0, 0]
        ref.append(s * q[0, t, 0, 0])
    assert rel(out.reshape(-1), np.array(ref)) < TOL


def test_varlen_equals_independent_runs(oracle_mod):
    lengths = [5, 0, 17, 1, 64, 33]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    Tt, H, dk, dv = int(cu[-1]), 3, 8, 6
    q, k, v = rand_qkv(1, Tt, H, dk, dv, seed=21)
    gam = [1.0, 0.95, 0.5]
    for phi, norm in (("identity", False), ("elu1", True)):
        out, fs = oracle_mod.recurrent(q, k, v, gam, cu_seqlens=cu, phi=phi, normalize=norm)
        for n, L in enumerate(lengths):
            s, e = cu[n], cu[n + 1]
            o1, f1 = oracle_mod.recurrent(q[:, s:e], k[:, s:e], v[:, s:e], gam, phi=phi, normalize=norm)
            assert np.array_equal(out[:, s:e], o1)
            assert np.array_equal(fs[n], f1[0])
            if L == 0:
                assert not fs[n].any()


def test_prefill_then_step_equals_longer_prefill(oracle_mod):
    T, H, dk, dv = 20, 2, 8, 8
    q, k, v = rand_qkv(3, T + 1, H, dk, dv, seed=31)
    gam = [0.9, 0.99]
    for phi in ("identity", "elu1"):
        _, fsT = oracle_mod.recurrent(q[:, :T], k[:, :T], v[:, :T], gam, phi=phi)
        oT1, fsT1 = oracle_mod.recurrent(q, k, v, gam, phi=phi)
        o, st = oracle_mod.step(q[:, T], k[:, T], v[:, T], gam, fsT, phi=phi)
        assert rel(o, oT1[:, T]) < TOL
        assert rel(st, fsT1) < TOL


def test_final_z_closed_form_and_direct_sum(oracle_mod):
    """z after the last token: with constant keys z_T = sum_{j<T} gamma^j phi(k);
    for random keys it equals the direct weighted sum sum_t gamma^(T-1-t) phi(k_t)."""
    T, dk = 37, 6
    rng = np.random.default_rng(41)
    kv = rng.standard_normal(dk)
    for phi in ("identity", "elu1"):
        for g in (1.0, 0.9, 0.0):
            k = np.broadcast_to(kv, (1, T, 1, dk)).copy()
            z = oracle_mod.final_z(k, [g], phi=phi)
            w = float(T) if g == 1.0 else (1 - g ** T) / (1 - g)
            assert rel(z[0, 0], w * phi_np(kv, phi)) < TOL
    lengths = [9, 0, 30, 1]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    _, k, _ = rand_qkv(1, int(cu[-1]), 2, dk, 1, seed=43)
    gam = [0.8, 1.0]
    for phi in ("identity", "elu1"):
        z = oracle_mod.final_z(k, gam, cu_seqlens=cu, phi=phi)
        for n, L in enumerate(lengths):
            for h, g in enumerate(gam):
                kh = phi_np(k[0, cu[n]:cu[n + 1], h], phi)
                ref = (g ** np.arange(L - 1, -1, -1, dtype=np.float64))[:, None] * kh
                assert rel(z[n, h], ref.sum(axis=0) if L else np.zeros(dk)) < TOL


def test_prefill_then_normalised_step_equals_longer_prefill(oracle_mod):
    """A normalised decode token continuing from (final state, final z) of a
    prefill equals the normalised prefill of one more token."""
    T, H, dk, dv = 20, 2, 8, 8
    q, k, v = rand_qkv(3, T + 1, H, dk, dv, seed=33)
    gam = [0.9, 1.0]
    _, fsT = oracle_mod.recurrent(q[:, :T], k[:, :T], v[:, :T], gam, phi="elu1", normalize=True)
    zT = oracle_mod.final_z(k[:, :T], gam, phi="elu1")
    oT1, fsT1 = oracle_mod.recurrent(q, k, v, gam, phi="elu1", normalize=True)
    o, st, z = oracle_mod.step_norm(q[:, T], k[:, T], v[:, T], gam, fsT, zT, phi="elu1")
    assert rel(o, oT1[:, T]) < TOL
    assert rel(st, fsT1) < TOL
    assert rel(z, oracle_mod.final_z(k, gam, phi="elu1")) < TOL
    # constant inputs: the normalised output is v exactly, from a zero start too
    vv = v[:, 0]
    o1, _, _ = oracle_mod.step_norm(q[:, 0], np.abs(k[:, 0]) + 0.1, vv, gam, np.zeros((3, H, dk, dv)),
                                    np.zeros((3, H, dk)), phi="elu1")
    assert np.max(np.abs(o1 - vv)) < 1e-13


# ---------------------------------------------------------------- data-dependent decay
def gated_quadratic_form(q, k, v, g, phi, normalize):
    """O = ((phi(Q) phi(K)^T) * M) V [/ row sums], M[i,j] = prod_{j<t<=i} exp(g_t) for i >= j
    (the cumulative-product decay mask).  One sequence, one head."""
    T = q.shape[0]
    A = phi_np(q, phi) @ phi_np(k, phi).T
    M = np.zeros((T, T))
    for i in range(T):
        for j in range(i + 1):
            M[i, j] = math.exp(float(np.sum(g[j + 1:i + 1])))
    P = A * M
    O = P @ v
    if normalize:
        O = O / P.sum(axis=1, keepdims=True)
    return O


@pytest.mark.parametrize("phi,normalize", [("identity", False), ("elu1", False), ("elu1", True)])
def test_gated_equals_cumulative_mask_quadratic(oracle_mod, phi, normalize):
    T, H, dk, dv = 40, 2, 6, 5
    q, k, v = rand_qkv(1, T, H, dk, dv, seed=51)
    g = -np.random.default_rng(52).uniform(0.0, 1.5, (1, T, H))
    out, _, _ = oracle_mod.recurrent_gated(q, k, v, g, phi=phi, normalize=normalize)
    for h in range(H):
        ref = gated_quadratic_form(q[0, :, h], k[0, :, h], v[0, :, h], g[0, :, h], phi, normalize)
        assert rel(out[0, :, h], ref) < 1e-11


def test_gated_with_constant_gate_equals_per_head_decay(oracle_mod):
    """g_t = log gamma_h for every token reproduces the per-head-decay oracle,
    including the final state and z."""
    T, H, dk, dv = 50, 3, 8, 4
    q, k, v = rand_qkv(2, T, H, dk, dv, seed=53)
    gam = np.array([0.9, 0.5, 1.0])
    g = np.broadcast_to(np.log(gam), (2, T, H)).copy()
    for phi, norm in (("identity", False), ("elu1", True)):
        out, fs, fz = oracle_mod.recurrent_gated(q, k, v, g, phi=phi, normalize=norm)
        ref, fref = oracle_mod.recurrent(q, k, v, gam, phi=phi, normalize=norm)
        assert rel(out, ref) < TOL and rel(fs, fref) < TOL
        assert rel(fz, oracle_mod.final_z(k, gam, phi=phi)) < TOL


def test_gated_varlen_and_decode_handover(oracle_mod):
    lengths = [7, 0, 30, 1]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    Tt, H, dk, dv = int(cu[-1]), 2, 6, 6
    q, k, v = rand_qkv(1, Tt, H, dk, dv, seed=55)
    g = -np.random.default_rng(56).uniform(0.0, 0.5, (1, Tt, H))
    out, fs, fz = oracle_mod.recurrent_gated(q, k, v, g, cu_seqlens=cu, phi="elu1", normalize=True)
    for n, L in enumerate(lengths):
        s_, e = cu[n], cu[n + 1]
        o1, f1, z1 = oracle_mod.recurrent_gated(q[:, s_:e], k[:, s_:e], v[:, s_:e], g[:, s_:e], phi="elu1",
                                                normalize=True)
        assert np.array_equal(out[:, s_:e], o1) and np.array_equal(fs[n], f1[0]) and np.array_equal(fz[n], z1[0])
    # prefill of T tokens + one gated decode step == prefill of T + 1 tokens
    T = 25
    q, k, v = rand_qkv(3, T + 1, H, dk, dv, seed=57)
    g = -np.random.default_rng(58).uniform(0.0, 0.5, (3, T + 1, H))
    for norm in (False, True):
        _, fsT, fzT = oracle_mod.recurrent_gated(q[:, :T], k[:, :T], v[:, :T], g[:, :T], phi="elu1", normalize=norm)
        oT1, fsT1, fzT1 = oracle_mod.recurrent_gated(q, k, v, g, phi="elu1", normalize=norm)
        o, st, z = oracle_mod.step_gated(q[:, T], k[:, T], v[:, T], g[:, T], fsT, fzT if norm else None, phi="elu1")
        assert rel(o, oT1[:, T]) < TOL and rel(st, fsT1) < TOL
        if norm:
            assert rel(z, fzT1) < TOL


# ---------------------------------------------------------------- backward
@pytest.mark.parametrize("phi", ["identity", "elu1"])
@pytest.mark.parametrize("gamma", [0.8, 1.0, 0.0])
def test_backward_matches_finite_differences(oracle_mod, phi, gamma):
    """Central differences of L = sum(dout * o) through the forward oracle."""
    B, T, H, dk, dv = 1, 7, 2, 3, 2
    q, k, v = rand_qkv(B, T, H, dk, dv, seed=61)
    dout = np.random.default_rng(62).standard_normal((B, T, H, dv))
    gam = [gamma, 0.5]
    gq, gk, gv = oracle_mod.backward(q, k, v, dout, gam, phi=phi)

    def loss(q_, k_, v_):
        o, _ = oracle_mod.recurrent(q_, k_, v_, gam, phi=phi)
        return float(np.sum(o * dout))

    eps = 1e-6
    for x, gref, which in ((q, gq, 0), (k, gk, 1), (v, gv, 2)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[which], args_m[which] = xp, xm
            fd[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        assert rel(gref, fd) < 1e-7, which


def test_backward_matches_autograd_of_quadratic_form(oracle_mod):
    """torch autograd (float64) through the quadratic masked form, a different
    formula for the same outputs."""
    T, H, dk, dv = 30, 2, 5, 4
    q, k, v = rand_qkv(1, T, H, dk, dv, seed=63)
    dout = np.random.default_rng(64).standard_normal((1, T, H, dv))
    gam = [0.9, 1.0]
    for phi in ("identity", "elu1"):
        gq, gk, gv = oracle_mod.backward(q, k, v, dout, gam, phi=phi)
        for h in range(H):
            qt, kt, vt = (torch.tensor(x[0, :, h], dtype=torch.float64, requires_grad=True) for x in (q, k, v))
            f = (lambda x: torch.where(x > 0, x + 1.0, torch.exp(torch.clamp(x, max=0.0)))) if phi == "elu1" \
                else (lambda x: x)
            A = f(qt) @ f(kt).T
            i = torch.arange(T)[:, None]
            j = torch.arange(T)[None, :]
            M = torch.where(i >= j, torch.tensor(gam[h], dtype=torch.float64) ** (i - j).clamp(min=0).double(),
                            torch.zeros((), dtype=torch.float64))
            O = (A * M) @ vt
            (O * torch.tensor(dout[0, :, h])).sum().backward()
            assert rel(gq[0, :, h], qt.grad.numpy()) < 1e-11
            assert rel(gk[0, :, h], kt.grad.numpy()) < 1e-11
            assert rel(gv[0, :, h], vt.grad.numpy()) < 1e-11


def test_backward_varlen_equals_independent_runs(oracle_mod):
    lengths = [5, 0, 17, 1]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    Tt, H, dk, dv = int(cu[-1]), 2, 4, 3
    q, k, v = rand_qkv(1, Tt, H, dk, dv, seed=65)
    dout = np.random.default_rng(66).standard_normal((1, Tt, H, dv))
    gam = [0.7, 1.0]
    gq, gk, gv = oracle_mod.backward(q, k, v, dout, gam, cu_seqlens=cu, phi="elu1")
    for n in range(len(lengths)):
        s_, e = cu[n], cu[n + 1]
        a, b, c = oracle_mod.backward(q[:, s_:e], k[:, s_:e], v[:, s_:e], dout[:, s_:e], gam, phi="elu1")
        assert np.array_equal(gq[:, s_:e], a) and np.array_equal(gk[:, s_:e], b) and np.array_equal(gv[:, s_:e], c)


# ---------------------------------------------------------------- normalised backward
# elu + 1 keeps every denominator positive (phi > 0, positive weights); the identity
# map with the normaliser can make it vanish, so the pins use elu + 1 (and one
# identity case on positive inputs).
@pytest.mark.parametrize("gamma", [1.0, 0.8])
def test_backward_norm_matches_finite_differences(oracle_mod, gamma):
    """Central differences of L = sum(dout * o) through the normalised forward oracle."""
    B, T, H, dk, dv = 1, 7, 2, 3, 2
    q, k, v = rand_qkv(B, T, H, dk, dv, seed=91)
    dout = np.random.default_rng(92).standard_normal((B, T, H, dv))
    gam = [gamma, 0.5]
    gq, gk, gv = oracle_mod.backward_norm(q, k, v, dout, gam, phi="elu1")

    def loss(q_, k_, v_):
        o, _ = oracle_mod.recurrent(q_, k_, v_, gam, phi="elu1", normalize=True)
        return float(np.sum(o * dout))

    eps = 1e-6
    for x, gref, which in ((q, gq, 0), (k, gk, 1), (v, gv, 2)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[which], args_m[which] = xp, xm
            fd[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        assert rel(gref, fd) < 1e-7, which


def test_backward_norm_matches_autograd_of_masked_form(oracle_mod):
    """torch autograd (float64) through the normalised quadratic masked form,
    O = ((phi(Q) phi(K)^T * M) V) / rowsum(phi(Q) phi(K)^T * M): a different formula."""
    T, H, dk, dv = 30, 2, 5, 4
    q, k, v = rand_qkv(1, T, H, dk, dv, seed=93)
    dout = np.random.default_rng(94).standard_normal((1, T, H, dv))
    gam = [0.9, 1.0]
    cases = [("elu1", q, k)]
    cases.append(("identity", np.abs(q) + 0.1, np.abs(k) + 0.1))  # positive keys and queries: den > 0
    for phi, qq, kk in cases:
        gq, gk, gv = oracle_mod.backward_norm(qq, kk, v, dout, gam, phi=phi)
        for h in range(H):
            qt, kt, vt = (torch.tensor(x[0, :, h], dtype=torch.float64, requires_grad=True) for x in (qq, kk, v))
            f = (lambda x: torch.where(x > 0, x + 1.0, torch.exp(torch.clamp(x, max=0.0)))) if phi == "elu1" \
                else (lambda x: x)
            A = f(qt) @ f(kt).T
            i = torch.arange(T)[:, None]
            j = torch.arange(T)[None, :]
            M = torch.where(i >= j, torch.tensor(gam[h], dtype=torch.float64) ** (i - j).clamp(min=0).double(),
                            torch.zeros((), dtype=torch.float64))
            P = A * M
            O = (P @ vt) / P.sum(dim=1, keepdim=True)
            (O * torch.tensor(dout[0, :, h])).sum().backward()
            assert rel(gq[0, :, h], qt.grad.numpy()) < 1e-11
            assert rel(gk[0, :, h], kt.grad.numpy()) < 1e-11
            assert rel(gv[0, :, h], vt.grad.numpy()) < 1e-11


def test_backward_norm_varlen_equals_independent_runs(oracle_mod):
    lengths = [5, 0, 17, 1]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    Tt, H, dk, dv = int(cu[-1]), 2, 4, 3
    q, k, v = rand_qkv(1, Tt, H, dk, dv, seed=95)
    dout = np.random.default_rng(96).standard_normal((1, Tt, H, dv))
    gam = [0.7, 1.0]
    full = oracle_mod.backward_norm(q, k, v, dout, gam, cu_seqlens=cu, phi="elu1")
    for n in range(len(lengths)):
        s_, e = cu[n], cu[n + 1]
        part = oracle_mod.backward_norm(q[:, s_:e], k[:, s_:e], v[:, s_:e], dout[:, s_:e], gam, phi="elu1")
        for a, b in zip(full, part):
            assert np.array_equal(a[:, s_:e], b)


def _rand_log_decay(B, T, H, seed, lo=0.3):
    return np.log(np.random.default_rng(seed).uniform(lo, 1.0, (B, T, H)))


@pytest.mark.parametrize("phi", ["identity", "elu1"])
def test_backward_gated_matches_finite_differences(oracle_mod, phi):
    """Central differences of L = sum(dout * o) through the per-token-decay forward
    oracle, for q, k, v and the log decays g."""
    B, T, H, dk, dv = 1, 6, 2, 3, 2
    q, k, v = rand_qkv(B, T, H, dk, dv, seed=71)
    dout = np.random.default_rng(72).standard_normal((B, T, H, dv))
    g = _rand_log_decay(B, T, H, 73)
    gq, gk, gv, gg = oracle_mod.backward_gated(q, k, v, dout, g, phi=phi)

    def loss(q_, k_, v_, g_):
        o, _, _ = oracle_mod.recurrent_gated(q_, k_, v_, g_, phi=phi)
        return float(np.sum(o * dout))

    eps = 1e-6
    for x, gref, which in ((q, gq, 0), (k, gk, 1), (v, gv, 2), (g, gg, 3)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = [q, k, v, g]
            args_m = [q, k, v, g]
            args_p[which], args_m[which] = xp, xm
            fd[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        assert rel(gref, fd) < 1e-7, which


def test_backward_gated_matches_autograd_of_masked_form(oracle_mod):
    """torch autograd (float64) through O = ((phi(Q) phi(K)^T) .* M) V with the
    cumulative-decay mask M_ij = exp(b_i - b_j) (i >= j), b = cumsum(g): a
    different formula for the same outputs, including dg."""
    T, H, dk, dv = 25, 2, 4, 3
    q, k, v = rand_qkv(1, T, H, dk, dv, seed=74)
    dout = np.random.default_rng(75).standard_normal((1, T, H, dv))
    g = _rand_log_decay(1, T, H, 76)
    for phi in ("identity", "elu1"):
        gq, gk, gv, gg = oracle_mod.backward_gated(q, k, v, dout, g, phi=phi)
        for h in range(H):
            qt, kt, vt, lg = (torch.tensor(x[0, :, h], dtype=torch.float64, requires_grad=True) for x in (q, k, v, g))
            f = (lambda x: torch.where(x > 0, x + 1.0, torch.exp(torch.clamp(x, max=0.0)))) if phi == "elu1" \
                else (lambda x: x)
            b = torch.cumsum(lg, 0)
            i = torch.arange(T)[:, None]
            j = torch.arange(T)[None, :]
            M = torch.where(i >= j, torch.exp(b[:, None] - b[None, :]), torch.zeros((), dtype=torch.float64))
            O = ((f(qt) @ f(kt).T) * M) @ vt
            (O * torch.tensor(dout[0, :, h])).sum().backward()
            assert rel(gq[0, :, h], qt.grad.numpy()) < 1e-11
            assert rel(gk[0, :, h], kt.grad.numpy()) < 1e-11
            assert rel(gv[0, :, h], vt.grad.numpy()) < 1e-11
            assert rel(gg[0, :, h], lg.grad.numpy()) < 1e-11


def test_backward_gated_reduces_to_per_head_decay_and_dg_identity(oracle_mod):
    """g constant over time per head: dq, dk, dv equal the per-head-decay backward
    with gamma = exp(g).  And for any g (identity feature map), dg_t equals the
    reverse cumulative sum over s >= t of q_s . dq_s - k_s . dk_s, which follows
    from o_s = sum_{j<=s} exp(b_s - b_j) (q_s . k_j) v_j with b the prefix sum of g."""
    B, T, H, dk, dv = 2, 40, 3, 5, 4
    q, k, v = rand_qkv(B, T, H, dk, dv, seed=77)
    dout = np.random.default_rng(78).standard_normal((B, T, H, dv))
    lg = np.log(np.array([0.6, 0.95, 1.0]))
    g = np.broadcast_to(lg, (B, T, H)).copy()
    gq, gk, gv, _ = oracle_mod.backward_gated(q, k, v, dout, g, phi="elu1")
    rq, rk, rv = oracle_mod.backward(q, k, v, dout, np.exp(lg), phi="elu1")
    assert rel(gq, rq) < 1e-12 and rel(gk, rk) < 1e-12 and rel(gv, rv) < 1e-12
    g = _rand_log_decay(B, T, H, 79)
    gq, gk, _, gg = oracle_mod.backward_gated(q, k, v, dout, g, phi="identity")
    per_t = np.sum(q * gq, axis=-1) - np.sum(k * gk, axis=-1)  # [B, T, H]
    want = np.flip(np.cumsum(np.flip(per_t, axis=1), axis=1), axis=1)
    assert rel(gg, want) < 1e-11


def test_backward_gated_varlen_equals_independent_runs(oracle_mod):
    lengths = [6, 0, 13, 1]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    Tt, H, dk, dv = int(cu[-1]), 2, 4, 3
    q, k, v = rand_qkv(1, Tt, H, dk, dv, seed=80)
    dout = np.random.default_rng(81).standard_normal((1, Tt, H, dv))
    g = _rand_log_decay(1, Tt, H, 82)
    full = oracle_mod.backward_gated(q, k, v, dout, g, cu_seqlens=cu, phi="elu1")
    for n in range(len(lengths)):
        s_, e = cu[n], cu[n + 1]
        part = oracle_mod.backward_gated(q[:, s_:e], k[:, s_:e], v[:, s_:e], dout[:, s_:e], g[:, s_:e], phi="elu1")
        for a, b in zip(full, part):
            assert np.array_equal(a[:, s_:e], b)


# ---------------------------------------------------------------- output norm and gate
def test_norm_gate_closed_forms(oracle_mod):
    """Constant rows: o = c * 1 gives y = sign(c) * w * swish(g) (up to eps); scaling
    o leaves y unchanged with eps = 0; g = 0 gives y = 0; a large gate passes
    the normalised row times w (swish(g) -> g)."""
    rng = np.random.default_rng(71)
    dv = 16
    w = rng.uniform(0.5, 1.5, dv)
    g = rng.standard_normal((3, dv))
    o = np.broadcast_to(np.array([2.0, -0.5, 3.0])[:, None], (3, dv)).copy()
    y = oracle_mod.norm_gate(o, g, w, eps=0.0)
    swish = g / (1.0 + np.exp(-g))
    assert rel(y, np.sign(o) * w * swish) < TOL
    x = rng.standard_normal((5, dv))
    g2 = rng.standard_normal((5, dv))
    assert rel(oracle_mod.norm_gate(7.5 * x, g2, w, eps=0.0), oracle_mod.norm_gate(x, g2, w, eps=0.0)) < TOL
    assert not oracle_mod.norm_gate(x, np.zeros_like(x), w).any()
    big = np.full_like(x, 40.0)
    rms = np.sqrt(np.mean(x * x, axis=1, keepdims=True) + 1e-5)
    assert rel(oracle_mod.norm_gate(x, big, w), x / rms * w * 40.0) < 1e-12


# ---------------------------------------------------------------- gated delta rule
def test_gated_delta_exact_recall(oracle_mod):
    """alpha = beta = 1 and the same unit key written again and again: reading with
    that key returns the value exactly, every time (the page's associative-memory
    check), where linear attention would return t times the value."""
    rng = np.random.default_rng(81)
    d, T = 16, 5
    key = rng.standard_normal(d)
    key /= np.linalg.norm(key)
    val = rng.standard_normal(d)
    k = np.broadcast_to(3.0 * key, (1, T, 1, d)).copy()   # the rule normalises k
    q = np.broadcast_to(key, (1, T, 1, d)).copy()
    v = np.broadcast_to(val, (1, T, 1, d)).copy()
    z = np.zeros((1, T, 1))
    out, fs = oracle_mod.gated_delta(q, k, v, z, np.ones((1, T, 1)))
    assert np.max(np.abs(out[0, :, 0] - val[None, :])) < 1e-12
    lin, _ = oracle_mod.recurrent(q, k / 3.0, v, [1.0])
    assert rel(lin[0, -1, 0], T * val) < 1e-12


def test_gated_delta_orthonormal_keys_closed_form(oracle_mod):
    """Keys on the standard basis: column j of S only ever sees key e_j, so
    S[:, j] <- alpha (1 - beta) S[:, j] + beta v on a write to j and alpha S[:, j]
    otherwise; alpha = beta = 1 reduces to plain linear attention."""
    rng = np.random.default_rng(83)
    T, d, dv = 12, 6, 4
    idx = rng.integers(0, d, T)
    k = np.zeros((1, T, 1, d))
    k[0, np.arange(T), 0, idx] = rng.uniform(0.5, 2.0, T)
    q = rng.standard_normal((1, T, 1, d))
    v = rng.standard_normal((1, T, 1, dv))
    g = np.log(rng.uniform(0.5, 1.0, (1, T, 1)))
    b = rng.uniform(0.1, 1.0, (1, T, 1))
    out, fs = oracle_mod.gated_delta(q, k, v, g, b)
    S = np.zeros((dv, d))
    for t in range(T):
        a, bt, j = math.exp(g[0, t, 0]), b[0, t, 0], idx[t]
        S *= a
        S[:, j] = (1 - bt) * S[:, j] + bt * v[0, t, 0]
        assert rel(out[0, t, 0], S @ q[0, t, 0]) < 1e-12
    assert rel(fs[0, 0], S.T) < 1e-12
    kk = k / np.linalg.norm(k, axis=-1, keepdims=True)
    o1, _ = oracle_mod.gated_delta(q, kk, v, np.zeros((1, T, 1)), np.ones((1, T, 1)))
    ref, _ = oracle_mod.recurrent(q, kk, v, [1.0])
    # a repeated basis key overwrites instead of adding; compare only while keys are distinct
    first_repeat = next((t for t in range(T) if idx[t] in idx[:t]), T)
    assert rel(o1[0, :first_repeat], ref[0, :first_repeat]) < 1e-12


def test_gated_delta_beta_zero_decay_and_handover(oracle_mod):
    """beta = 0 leaves only the decayed initial state, o_t = prod_{s<=t} alpha_s S0 q_t;
    a prefill continued from its final state equals the longer prefill; a packed
    batch equals independent runs."""
    rng = np.random.default_rng(85)
    T, H, dk, dv = 9, 2, 5, 3
    q, k, v = rand_qkv(1, T, H, dk, dv, seed=86)
    g = np.log(rng.uniform(0.6, 1.0, (1, T, H)))
    S0 = rng.standard_normal((1, H, dk, dv))
    out, _ = oracle_mod.gated_delta(q, k, v, g, np.zeros((1, T, H)), init=S0)
    cum = np.exp(np.cumsum(g[0], axis=0))
    for h in range(H):
        ref = cum[:, h:h + 1] * (q[0, :, h] @ S0[0, h])
        assert rel(out[0, :, h], ref) < 1e-12
    b = rng.uniform(0.2, 1.0, (1, T, H))
    full, ffull = oracle_mod.gated_delta(q, k, v, g, b)
    _, f5 = oracle_mod.gated_delta(q[:, :5], k[:, :5], v[:, :5], g[:, :5], b[:, :5])
    rest, frest = oracle_mod.gated_delta(q[:, 5:], k[:, 5:], v[:, 5:], g[:, 5:], b[:, 5:], init=f5)
    assert rel(rest, full[:, 5:]) < 1e-12 and rel(frest, ffull) < 1e-12
    lengths = [4, 0, 5]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    pk, pf = oracle_mod.gated_delta(q, k, v, g, b, cu_seqlens=cu)
    for n in range(3):
        s_, e = cu[n], cu[n + 1]
        o1, f1 = oracle_mod.gated_delta(q[:, s_:e], k[:, s_:e], v[:, s_:e], g[:, s_:e], b[:, s_:e])
        assert np.array_equal(pk[:, s_:e], o1) and np.array_equal(pf[n], f1[0])


@pytest.mark.parametrize("chunk", [1, 2, 3, 7, 16, 64, 100])
def test_gated_delta_chunked_equals_recurrence(oracle_mod, chunk):
    """The chunk (WY / UT) form of the gated delta rule: per chunk the writes solve
    a unit lower-triangular system.  It must equal the token-by-token rule for
    every chunk size, with a partial last chunk, strong and weak decay, beta
    near 0 and 1, an initial state and a packed batch with an empty sequence."""
    rng = np.random.default_rng(87 + chunk)
    T, H, dk, dv = 100, 2, 7, 5
    q, k, v = rand_qkv(1, T, H, dk, dv, seed=88 + chunk)
    g = np.log(rng.uniform(0.05, 1.0, (1, T, H)))
    g[0, :, 1] *= 0.01
    b = rng.uniform(0.0, 1.0, (1, T, H))
    b[0, ::5, 0] = 1.0
    S0 = rng.standard_normal((1, H, dk, dv))
    ref, fref = oracle_mod.gated_delta(q, k, v, g, b, init=S0)
    out, fs = oracle_mod.gated_delta_chunked(q, k, v, g, b, chunk, init=S0)
    assert rel(out, ref) < 1e-10 and rel(fs, fref) < 1e-10
    cu = np.array([0, 37, 37, 38, 100], np.int32)
    ref, fref = oracle_mod.gated_delta(q, k, v, g, b, cu_seqlens=cu)
    out, fs = oracle_mod.gated_delta_chunked(q, k, v, g, b, chunk, cu_seqlens=cu)
    assert rel(out, ref) < 1e-10 and rel(fs, fref) < 1e-10
    assert not fs[1].any()


def test_gated_delta_chunked_single_chunk_matrix_form(oracle_mod):
    """One chunk holding the whole sequence, written out with numpy matrices from
    the same derivation (A, T = (I + A)^{-1}, U, then O and the final state), and
    the rule itself at alpha = 1: W = T diag(beta) Kt recovers plain delta-rule
    outputs.  Catches a transposed Kt Kt^T, a missing beta or a decay on the wrong side."""
    rng = np.random.default_rng(89)
    T, dk, dv = 11, 4, 3
    q, k, v = rand_qkv(1, T, 1, dk, dv, seed=90)
    g = np.log(rng.uniform(0.3, 1.0, (1, T, 1)))
    b = rng.uniform(0.1, 1.0, (1, T, 1))
    out, fs = oracle_mod.gated_delta_chunked(q, k, v, g, b, T)
    kt = k[0, :, 0] / np.linalg.norm(k[0, :, 0], axis=1, keepdims=True)
    bc = np.cumsum(g[0, :, 0])
    bt = b[0, :, 0]
    D = np.exp(bc[:, None] - bc[None, :])
    A = np.tril(bt[:, None] * D * (kt @ kt.T), -1)
    U = np.linalg.solve(np.eye(T) + A, bt[:, None] * v[0, :, 0])
    O = (np.tril(D) * (q[0, :, 0] @ kt.T)) @ U
    Sf = (np.exp(bc[-1] - bc)[:, None] * kt).T @ U
    assert rel(out[0, :, 0], O) < 1e-12 and rel(fs[0, 0], Sf) < 1e-12
    ref, fref = oracle_mod.gated_delta(q, k, v, g, b)
    assert rel(out, ref) < 1e-10 and rel(fs, fref) < 1e-10


# ---------------------------------------------------------------- chunked form
@pytest.mark.parametrize("chunk", [1, 2, 3, 7, 16, 64, 100, 130])
@pytest.mark.parametrize("phi,normalize", [("identity", False), ("elu1", True)])
def test_chunk_invariance(oracle_mod, chunk, phi, normalize):
    T, H, dk, dv = 130, 3, 6, 5
    q, k, v = rand_qkv(2, T, H, dk, dv, seed=chunk)
    gam = [1.0, 0.93, 0.0]
    ref, fref = oracle_mod.recurrent(q, k, v, gam, phi=phi, normalize=normalize)
    out, fs = oracle_mod.chunked(q, k, v, gam, chunk, phi=phi, normalize=normalize)
    assert rel(out, ref) < TOL
    assert rel(fs, fref) < TOL


def test_chunk_invariance_varlen(oracle_mod):
    lengths = [64, 65, 1, 0, 130, 63]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    q, k, v = rand_qkv(1, int(cu[-1]), 2, 8, 8, seed=77)
    gam = [0.97, 1.0]
    ref, fref = oracle_mod.recurrent(q, k, v, gam, cu_seqlens=cu, phi="elu1", normalize=True)
    for chunk in (16, 64):
        out, fs = oracle_mod.chunked(q, k, v, gam, chunk, cu_seqlens=cu, phi="elu1", normalize=True)
        assert rel(out, ref) < TOL and rel(fs, fref) < TOL


# ---------------------------------------------------------------- input types
def test_bf16_and_f32_inputs_upcast_exactly(oracle_mod):
    qf, kf, vf = (torch.randn(1, 33, 2, 8, dtype=torch.float32) for _ in range(3))
    qb, kb, vb = (x.to(torch.bfloat16) for x in (qf, kf, vf))
    o_b, f_b = oracle_mod.recurrent(qb, kb, vb, [0.9, 1.0])
    o_d, f_d = oracle_mod.recurrent(*(x.double().numpy() for x in (qb, kb, vb)), [0.9, 1.0])
    assert np.array_equal(o_b, o_d) and np.array_equal(f_b, f_d)
    o_f, _ = oracle_mod.recurrent(qf.numpy(), kf.numpy(), vf.numpy(), [0.9, 1.0])
    o_f64, _ = oracle_mod.recurrent(*(x.double().numpy() for x in (qf, kf, vf)), [0.9, 1.0])
    assert np.array_equal(o_f, o_f64)


def test_rejects_bad_arguments(oracle_mod):
    q, k, v = rand_qkv(2, 4, 1, 2, 2, seed=1)
    with pytest.raises(ValueError):
        oracle_mod.recurrent(q, k, v, [1.0], cu_seqlens=[0, 2, 4])  # B must be 1 with cu_seqlens
    with pytest.raises(ValueError):
        oracle_mod.recurrent(q[:1], k[:1], v[:1], [1.0], cu_seqlens=[0, 3, 2])  # decreasing
    with pytest.raises(ValueError):
        oracle_mod.chunked(q, k, v, [1.0], 0)


def test_oracle_is_independent_of_the_product():
    """The oracle package imports nothing from the CUDA library's package."""
    src = open(os.path.join(os.path.dirname(__file__), "..", "oracle", "__init__.py")).read()
    src += open(os.path.join(os.path.dirname(__file__), "..", "oracle", "la_oracle.c")).read()
    assert "chunkwise_causal_linear_la_b200" not in src


def test_backward_norm_splits_into_numerator_and_denominator_adjoints(oracle_mod):
    """The normalised adjoint is the unnormalised one twice: once for the numerator
    (values v, output gradient dout / den) and once for the denominator (values 1,
    output gradient e_t = -(dout_t . o_t) / den_t), with den and o from the forward."""
    gen = torch.Generator()
    gen.manual_seed(71)
    B, T, H, dk, dv = 2, 37, 2, 5, 4
    q, k, v, do = (torch.randn((B, T, H, d), generator=gen, dtype=torch.float64) for d in (dk, dk, dv, dv))
    gamma = np.array([1.0, 0.85])
    for phi in ("elu1",):
        ones = torch.ones((B, T, H, 1), dtype=torch.float64)
        den, _ = oracle_mod.recurrent(q, k, ones, gamma, phi=phi, normalize=False)
        o, _ = oracle_mod.recurrent(q, k, v, gamma, phi=phi, normalize=True)
        den, o = torch.from_numpy(den), torch.from_numpy(o)
        a = oracle_mod.backward(q, k, v, do / den, gamma, phi=phi)
        b = oracle_mod.backward(q, k, ones, -(do * o).sum(-1, keepdim=True) / den, gamma, phi=phi)
        ref = oracle_mod.backward_norm(q, k, v, do, gamma, phi=phi)
        for x, y, r in zip(a[:2], b[:2], ref[:2]):
            np.testing.assert_allclose(x + y, r, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(a[2], ref[2], rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- normalised backward, per-token decay
def test_backward_gated_norm_matches_finite_differences(oracle_mod):
    """Central differences of L = sum(dout * o) through the normalised per-token-decay
    forward oracle, for q, k, v and the log decays g."""
    B, T, H, dk, dv = 1, 6, 2, 3, 2
    q, k, v = rand_qkv(B, T, H, dk, dv, seed=101)
    dout = np.random.default_rng(102).standard_normal((B, T, H, dv))
    g = _rand_log_decay(B, T, H, 103)
    gq, gk, gv, gg = oracle_mod.backward_gated_norm(q, k, v, dout, g, phi="elu1")

    def loss(q_, k_, v_, g_):
        o, _, _ = oracle_mod.recurrent_gated(q_, k_, v_, g_, phi="elu1", normalize=True)
        return float(np.sum(o * dout))

    eps = 1e-6
    for x, gref, which in ((q, gq, 0), (k, gk, 1), (v, gv, 2), (g, gg, 3)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = [q, k, v, g]
            args_m = [q, k, v, g]
            args_p[which], args_m[which] = xp, xm
            fd[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        assert rel(gref, fd) < 1e-7, which


def test_backward_gated_norm_matches_autograd_of_masked_form(oracle_mod):
    """torch autograd (float64) through O = ((phi(Q) phi(K)^T .* M) V) / rowsum(phi(Q) phi(K)^T .* M)
    with the cumulative-decay mask M_ij = exp(b_i - b_j) (i >= j), b = cumsum(g)."""
    T, H, dk, dv = 25, 2, 4, 3
    q, k, v = rand_qkv(1, T, H, dk, dv, seed=104)
    dout = np.random.default_rng(105).standard_normal((1, T, H, dv))
    g = _rand_log_decay(1, T, H, 106)
    cases = [("elu1", q, k), ("identity", np.abs(q) + 0.1, np.abs(k) + 0.1)]
    for phi, qq, kk in cases:
        gq, gk, gv, gg = oracle_mod.backward_gated_norm(qq, kk, v, dout, g, phi=phi)
        for h in range(H):
            qt, kt, vt, lg = (torch.tensor(x[0, :, h], dtype=torch.float64, requires_grad=True)
                              for x in (qq, kk, v, g))
            f = (lambda x: torch.where(x > 0, x + 1.0, torch.exp(torch.clamp(x, max=0.0)))) if phi == "elu1" \
                else (lambda x: x)
            b = torch.cumsum(lg, 0)
            i = torch.arange(T)[:, None]
            j = torch.arange(T)[None, :]
            M = torch.where(i >= j, torch.exp(b[:, None] - b[None, :]), torch.zeros((), dtype=torch.float64))
            P = (f(qt) @ f(kt).T) * M
            O = (P @ vt) / P.sum(dim=1, keepdim=True)
            (O * torch.tensor(dout[0, :, h])).sum().backward()
            assert rel(gq[0, :, h], qt.grad.numpy()) < 1e-11
            assert rel(gk[0, :, h], kt.grad.numpy()) < 1e-11
            assert rel(gv[0, :, h], vt.grad.numpy()) < 1e-11
            assert rel(gg[0, :, h], lg.grad.numpy()) < 1e-10


def test_backward_gated_norm_reduces_to_per_head_decay(oracle_mod):
    """g constant over time per head: dq, dk, dv equal the normalised per-head-decay
    backward with gamma = exp(g)."""
    B, T, H, dk, dv = 2, 30, 3, 4, 3
    q, k, v = rand_qkv(B, T, H, dk, dv, seed=107)
    dout = np.random.default_rng(108).standard_normal((B, T, H, dv))
    lg = np.log(np.array([0.6, 0.95, 1.0]))
    g = np.broadcast_to(lg, (B, T, H)).copy()
    gq, gk, gv, _ = oracle_mod.backward_gated_norm(q, k, v, dout, g, phi="elu1")
    rq, rk, rv = oracle_mod.backward_norm(q, k, v, dout, np.exp(lg), phi="elu1")
    assert rel(gq, rq) < 1e-12 and rel(gk, rk) < 1e-12 and rel(gv, rv) < 1e-12


def test_backward_gated_norm_varlen_equals_independent_runs(oracle_mod):
    lengths = [6, 0, 13, 1]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    Tt, H, dk, dv = int(cu[-1]), 2, 4, 3
    q, k, v = rand_qkv(1, Tt, H, dk, dv, seed=109)
    dout = np.random.default_rng(110).standard_normal((1, Tt, H, dv))
    g = _rand_log_decay(1, Tt, H, 111)
    full = oracle_mod.backward_gated_norm(q, k, v, dout, g, cu_seqlens=cu, phi="elu1")
    for n in range(len(lengths)):
        s_, e = cu[n], cu[n + 1]
        part = oracle_mod.backward_gated_norm(q[:, s_:e], k[:, s_:e], v[:, s_:e], dout[:, s_:e], g[:, s_:e],
                                              phi="elu1")
        for a, b in zip(full, part):
            assert np.array_equal(a[:, s_:e], b)
