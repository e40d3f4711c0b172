"""GPU parity of the data-dependent decay (la_fwd_chunk_gated, la_step_gated)
against the float64 oracle (oracle.recurrent_gated / step_gated).

The decay of token t in head h is exp(g[t][h]).  Cases: both tensor-core
shapes (d_k = 128, 256) and the CUDA-core kernel (f32), mild decays (as in
the sweep workloads) and strong ones (exp(g) down to 0.05, so the decay over
a 64-token chunk underflows), both feature maps with and without the
normaliser, packed batches with empty sequences, a segmented long sequence,
and the decode step continuing a prefill.
"""
import math

import numpy as np
import pytest
import torch

from parity_util import TOL, seq_slices, slice_rel_err, state_rel_err, to_np

pytestmark = pytest.mark.gpu

BF = torch.bfloat16


@pytest.fixture(scope="module")
def la():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import chunkwise_causal_linear_la_b200 as la

    la.load_library()
    return la


def _inputs(B, T, H, dk, dv, dtype, seed, lo, hi):
    from chunkwise_causal_linear_la_b200.workloads import make_log_decay, make_qkv

    q, k, v = make_qkv(B, T, H, dk, dv, dtype, dk ** -0.5, seed=seed)
    gen = torch.Generator()
    gen.manual_seed(seed + 1)
    return q, k, v, make_log_decay(B, T, H, lo, hi, gen)


def _check(la, oracle_mod, q, k, v, g, cu=None, phi="identity", normalize=False, flags=0):
    dev = torch.device("cuda")
    out, fs, fz = la.la_fwd_chunk_gated(q.to(dev), k.to(dev), v.to(dev), g.to(dev),
                                        cu_seqlens=None if cu is None else cu.to(dev), phi=phi,
                                        normalize=normalize, return_final_z=normalize, flags=flags)
    torch.cuda.synchronize()
    ref, fref, zref = oracle_mod.recurrent_gated(q, k, v, g.double().numpy(),
                                                 cu_seqlens=None if cu is None else cu.numpy(), phi=phi,
                                                 normalize=normalize)
    B, T = q.shape[:2]
    tol = TOL[q.dtype]
    assert np.isfinite(to_np(out)).all()
    e1 = slice_rel_err(to_np(out), ref, seq_slices(B, T, None if cu is None else cu.tolist()))
    e2 = state_rel_err(to_np(fs), fref)
    assert e1 < tol and e2 < tol, (e1, e2)
    if normalize:
        assert state_rel_err(to_np(fz)[..., None], zref[..., None]) < 1e-4


@pytest.mark.parametrize("dk", [128, 256])
@pytest.mark.parametrize("T", [1, 65, 300])
@pytest.mark.parametrize("lo,hi", [(0.9, 0.999), (0.05, 1.0)])
def test_gated_tc_shapes(la, oracle_mod, dk, T, lo, hi):
    q, k, v, g = _inputs(2, T, 2, dk, dk, BF, T + dk, lo, hi)
    _check(la, oracle_mod, q, k, v, g)


@pytest.mark.parametrize("phi,normalize", [("elu1", True), ("elu1", False)])
@pytest.mark.parametrize("dk", [128, 256])
def test_gated_tc_feature_maps(la, oracle_mod, phi, normalize, dk):
    q, k, v, g = _inputs(1, 333, 2, dk, dk, BF, 3, 0.5, 1.0)
    _check(la, oracle_mod, q, k, v, g, phi=phi, normalize=normalize)


def test_gated_tc_varlen(la, oracle_mod):
    from chunkwise_causal_linear_la_b200.workloads import cu_seqlens_from_lengths

    cu = cu_seqlens_from_lengths([130, 0, 1, 64, 65, 300])
    q, k, v, g = _inputs(1, int(cu[-1]), 3, 128, 128, BF, 5, 0.8, 1.0)
    _check(la, oracle_mod, q, k, v, g, cu=cu, phi="elu1", normalize=True)
    _check(la, oracle_mod, q, k, v, g, cu=cu)


@pytest.mark.parametrize("phi,normalize", [("identity", False), ("elu1", True)])
def test_gated_tc_segmented(la, oracle_mod, phi, normalize):
    """One long sequence (few units): state pass, scan with per-segment decays, output pass."""
    q, k, v, g = _inputs(1, 5000, 2, 128, 128, BF, 17, 0.99, 1.0)
    assert la.workspace_size(1, 5000, 2, 128, 128, 1, False, 64) > 0
    _check(la, oracle_mod, q, k, v, g, phi=phi, normalize=normalize)


@pytest.mark.parametrize("chunk", [16, 64, 128])
@pytest.mark.parametrize("phi,normalize", [("identity", False), ("elu1", True)])
def test_gated_simt_f32(la, oracle_mod, chunk, phi, normalize):
    q, k, v, g = _inputs(2, 3 * chunk + 5, 3, 64, 64, torch.float32, chunk, 0.3, 1.0)
    _check(la, oracle_mod, q, k, v, g, phi=phi, normalize=normalize)


def test_gated_constant_gate_matches_per_head_decay(la):
    """g = log gamma on every token gives the per-head-decay kernel's result."""
    from chunkwise_causal_linear_la_b200.workloads import make_qkv

    q, k, v = (x.cuda() for x in make_qkv(2, 500, 4, 128, 128, BF, 128 ** -0.5, seed=9))
    gam = torch.tensor([0.9, 0.95, 0.99, 1.0], device="cuda")
    g = torch.log(gam).expand(2, 500, 4).contiguous()
    o1, f1 = la.la_fwd_chunk(q, k, v, gam)
    o2, f2, _ = la.la_fwd_chunk_gated(q, k, v, g)
    torch.cuda.synchronize()
    assert slice_rel_err(to_np(o2), to_np(o1), seq_slices(2, 500)) < TOL[BF]
    assert state_rel_err(to_np(f2), to_np(f1)) < TOL[BF]


@pytest.mark.parametrize("dtype", [torch.float32, BF])
@pytest.mark.parametrize("normalised", [False, True])
def test_step_gated_against_oracle(la, oracle_mod, dtype, normalised):
    from chunkwise_causal_linear_la_b200.workloads import make_decode_inputs

    x = make_decode_inputs(37, 4, 128, 128, 128 ** -0.5, 0.01, (1.0,) * 4, seed=3, dtype=dtype)
    rng = np.random.default_rng(7)
    g = torch.from_numpy(np.log(rng.uniform(0.5, 1.0, (37, 4))).astype(np.float32))
    z0 = torch.from_numpy(np.abs(rng.standard_normal((37, 4, 128))).astype(np.float32)) if normalised else None
    dev = torch.device("cuda")
    state = x["state"].to(dev)
    z = None if z0 is None else z0.to(dev)
    o = la.la_step_gated(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), g.to(dev), state, z, phi="elu1")
    torch.cuda.synchronize()
    ref_o, ref_s, ref_z = oracle_mod.step_gated(x["q"], x["k"], x["v"], g.double().numpy(),
                                                x["state"].double().numpy(),
                                                None if z0 is None else z0.double().numpy(), phi="elu1")
    assert state_rel_err(to_np(state), ref_s) < 1e-6
    if normalised:
        assert state_rel_err(to_np(z)[..., None], ref_z[..., None]) < 1e-6
    err = max(float(np.max(np.abs(to_np(o)[n, h] - ref_o[n, h])) / np.max(np.abs(ref_o[n, h])))
              for n in range(37) for h in range(4))
    assert err < TOL[dtype], err


def test_gated_prefill_then_decode(la, oracle_mod):
    B, T, H, d = 3, 300, 2, 128
    q, k, v, g = _inputs(B, T + 1, H, d, d, BF, 21, 0.7, 1.0)
    dev = torch.device("cuda")
    qd, kd, vd, gd = q.to(dev), k.to(dev), v.to(dev), g.to(dev)
    _, fs, z = la.la_fwd_chunk_gated(qd[:, :T].contiguous(), kd[:, :T].contiguous(), vd[:, :T].contiguous(),
                                     gd[:, :T].contiguous(), phi="elu1", normalize=True, return_final_z=True)
    o = la.la_step_gated(qd[:, T], kd[:, T], vd[:, T], gd[:, T].contiguous(), fs, z, phi="elu1")
    torch.cuda.synchronize()
    ref, _, _ = oracle_mod.recurrent_gated(q, k, v, g.double().numpy(), phi="elu1", normalize=True)
    for b in range(B):
        for h in range(H):
            r = ref[b, T, h]
            assert float(np.max(np.abs(to_np(o)[b, h] - r)) / np.max(np.abs(r))) < TOL[BF]


def test_gated_config_sample(la, oracle_mod):
    """The gated workload (B=8, H=16, d=128, T=16384, decays in [0.9, 0.999]) at
    full size; the oracle checks two (sequence, head) slices."""
    from chunkwise_causal_linear_la_b200.workloads import WORKLOADS, make_inputs

    w = WORKLOADS["gated_T16384"]
    x = make_inputs(w, seed=0)
    dev = torch.device("cuda")
    out, fs, _ = la.la_fwd_chunk_gated(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), x["g"].to(dev))
    torch.cuda.synchronize()
    for b, h in [(0, 0), (7, 15)]:
        qs, ks, vs = (x[n][b:b + 1, :, h:h + 1] for n in ("q", "k", "v"))
        gs = x["g"][b:b + 1, :, h:h + 1].double().numpy()
        ref, fref, _ = oracle_mod.recurrent_gated(qs, ks, vs, gs)
        assert slice_rel_err(to_np(out[b:b + 1, :, h:h + 1]), ref, seq_slices(1, w.T)) < TOL[BF]
        assert state_rel_err(to_np(fs[b:b + 1, h:h + 1]), fref) < TOL[BF]


def test_device_error_word_clear_after_gated(la):
    assert la.device_error(reset=True) == (0, 0)
