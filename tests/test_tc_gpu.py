"""GPU parity of the tensor-core (tcgen05) chunk kernel against the float64 oracle.

bf16 inputs, tolerance 2e-2 (slice-relative, see parity_util), for outputs and
final states.  Shapes span several chunks and ragged tails; gammas cover the
normal decay path (gamma^(C-1) >= 2^-64), the small-gamma path (gamma = 0,
0.3) and gamma = 1; both feature maps; with and without the normaliser;
dense and packed (cu_seqlens) batches.
"""
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


def _inputs(B, T, H, dk, dv, scale, seed):
    from chunkwise_causal_linear_la_b200.workloads import make_qkv

    return make_qkv(B, T, H, dk, dv, BF, scale, seed=seed)


def _check(la, oracle_mod, q, k, v, gamma, cu=None, phi="identity", normalize=False, chunk=64):
    dev = torch.device("cuda")
    out, fs = la.la_fwd_chunk(q.to(dev), k.to(dev), v.to(dev), gamma.to(dev),
                              cu_seqlens=None if cu is None else cu.to(dev), chunk=chunk, phi=phi,
                              normalize=normalize)
    torch.cuda.synchronize()
    ref, fref = oracle_mod.recurrent(q, k, v, gamma.double().numpy(), cu_seqlens=None if cu is None else cu.numpy(),
                                     phi=phi, normalize=normalize)
    B, T = q.shape[:2]
    e1 = slice_rel_err(to_np(out), ref, seq_slices(B, T, None if cu is None else cu.tolist()))
    e2 = state_rel_err(to_np(fs), fref)
    assert np.isfinite(to_np(out)).all()
    assert e1 < TOL[BF] and e2 < TOL[BF], (e1, e2)
    return e1, e2


@pytest.mark.parametrize("T", [1, 63, 64, 65, 200, 4 * 64 + 17])
def test_tc_lengths(la, oracle_mod, T):
    q, k, v = _inputs(2, T, 3, 128, 128, 128 ** -0.5, seed=T)
    _check(la, oracle_mod, q, k, v, torch.tensor([0.9, 0.999, 1.0]))


@pytest.mark.parametrize("gamma", [0.0, 0.3, 0.5, 0.9, 0.97, 1.0])
def test_tc_gammas(la, oracle_mod, gamma):
    q, k, v = _inputs(1, 300, 2, 128, 128, 128 ** -0.5, seed=7)
    _check(la, oracle_mod, q, k, v, torch.tensor([gamma, gamma]))


@pytest.mark.parametrize("phi,normalize", [("elu1", True), ("elu1", False), ("identity", False)])
@pytest.mark.parametrize("gamma", [1.0, 0.95, 0.2])
def test_tc_feature_maps(la, oracle_mod, phi, normalize, gamma):
    q, k, v = _inputs(2, 333, 2, 128, 128, 128 ** -0.5, seed=3)
    _check(la, oracle_mod, q, k, v, torch.tensor([gamma, 1.0]), phi=phi, normalize=normalize)


def test_tc_dv256(la, oracle_mod):
    q, k, _ = _inputs(2, 150, 2, 128, 128, 128 ** -0.5, seed=9)
    _, _, v = _inputs(2, 150, 2, 128, 256, 128 ** -0.5, seed=10)
    _check(la, oracle_mod, q, k, v, torch.tensor([0.98, 1.0]))


def test_tc_varlen(la, oracle_mod):
    from chunkwise_causal_linear_la_b200.workloads import cu_seqlens_from_lengths

    lengths = [130, 0, 1, 64, 65, 300, 17, 128]
    cu = cu_seqlens_from_lengths(lengths)
    q, k, v = _inputs(1, int(cu[-1]), 4, 128, 128, 128 ** -0.5, seed=5)
    _check(la, oracle_mod, q, k, v, torch.tensor([1.0, 0.9, 0.99, 0.0]), cu=cu, phi="elu1", normalize=True)
    _check(la, oracle_mod, q, k, v, torch.tensor([1.0, 0.9, 0.99, 0.0]), cu=cu)


def test_tc_varlen_config_sample(la, oracle_mod):
    """The packed-batch workload (64 sequences, lengths U[128, 2048], H=8, d=128,
    elu+1 with normaliser, gamma=1) at full size; the oracle checks 2 heads."""
    from chunkwise_causal_linear_la_b200.workloads import WORKLOADS, make_inputs

    w = WORKLOADS["varlen"]
    x = make_inputs(w, seed=0)
    dev = torch.device("cuda")
    out, fs = la.la_fwd_chunk(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), x["gamma"].to(dev),
                              cu_seqlens=x["cu_seqlens"].to(dev), chunk=64, phi="elu1", normalize=True)
    torch.cuda.synchronize()
    heads = [0, 5]
    cu = x["cu_seqlens"]
    ref, fref = oracle_mod.recurrent(x["q"][:, :, heads], x["k"][:, :, heads], x["v"][:, :, heads],
                                     np.ones(len(heads)), cu_seqlens=cu.numpy(), phi="elu1", normalize=True)
    o = to_np(out[:, :, heads])
    assert slice_rel_err(o, ref, seq_slices(1, 0, cu.tolist())) < TOL[BF]
    assert state_rel_err(to_np(fs[:, heads]), fref) < TOL[BF]


def test_tc_matches_simt(la):
    """Tensor-core and CUDA-core kernels agree on the same bf16 inputs."""
    q, k, v = _inputs(2, 500, 4, 128, 128, 128 ** -0.5, seed=1)
    dev = torch.device("cuda")
    g = torch.tensor([0.9, 0.95, 0.99, 1.0], device=dev)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o1, f1 = la.la_fwd_chunk(qd, kd, vd, g, chunk=64)
    o2, f2 = la.la_fwd_chunk(qd, kd, vd, g, chunk=64, flags=la.LA_FLAG_SIMT)
    torch.cuda.synchronize()
    assert slice_rel_err(to_np(o1), to_np(o2), seq_slices(2, 500)) < TOL[BF]
    assert state_rel_err(to_np(f1), to_np(f2)) < TOL[BF]


def test_tc_repeatable(la):
    """Two runs on the same inputs give bit-identical results (no races)."""
    q, k, v = _inputs(2, 700, 4, 128, 128, 128 ** -0.5, seed=2)
    dev = torch.device("cuda")
    g = torch.tensor([0.9, 0.95, 0.99, 1.0], device=dev)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o1, f1 = la.la_fwd_chunk(qd, kd, vd, g, phi="elu1", normalize=True)
    o2, f2 = la.la_fwd_chunk(qd, kd, vd, g, phi="elu1", normalize=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(f1, f2)


# ---------------------------------------------------------------- segmented sequences
@pytest.mark.parametrize("phi,normalize", [("identity", False), ("elu1", True)])
@pytest.mark.parametrize("gamma", [1.0, 0.995, 0.9, 0.3, 0.0])
def test_tc_segmented_long_sequence(la, oracle_mod, phi, normalize, gamma):
    """Few (sequence, head) units and a long sequence: the sequence is split into
    segments (state pass, scan, output pass) -- 79 chunks with a ragged tail."""
    B, T, H = 1, 5000, 2
    q, k, v = _inputs(B, T, H, 128, 128, 128 ** -0.5, seed=17)
    need = la.workspace_size(B, T, H, 128, 128, B, False, 64)
    assert need > 0  # this shape is segmented
    _check(la, oracle_mod, q, k, v, torch.tensor([gamma, 0.97]), phi=phi, normalize=normalize)


def test_tc_segmented_matches_unsegmented(la):
    """The same sequences with and without segmentation agree (the 4-unit batch is
    segmented, the 160-unit batch with the same first sequences is not)."""
    dev = torch.device("cuda")
    q, k, v = _inputs(40, 2048, 4, 128, 128, 128 ** -0.5, seed=23)
    g = torch.tensor([0.99, 0.9, 1.0, 0.95], device=dev)
    assert la.workspace_size(1, 2048, 4, 128, 128, 1, False, 64) > 0
    assert la.workspace_size(40, 2048, 4, 128, 128, 40, False, 64) == 0
    o_all, f_all = la.la_fwd_chunk(q.to(dev), k.to(dev), v.to(dev), g)
    o_one, f_one = la.la_fwd_chunk(q[:1].to(dev), k[:1].to(dev), v[:1].to(dev), g)
    torch.cuda.synchronize()
    assert slice_rel_err(to_np(o_one), to_np(o_all[:1]), seq_slices(1, 2048)) < TOL[BF]
    assert state_rel_err(to_np(f_one), to_np(f_all[:1])) < TOL[BF]


def test_tc_device_error_word_clear(la):
    """After every tensor-core launch above, no bounded wait timed out."""
    assert la.device_error(reset=True) == (0, 0)


# ---------------------------------------------------------------- d_k = 256
# d_k = 256 runs with 64-wide value slices (each CTA's state is 256 x 64 fp32)
@pytest.mark.parametrize("dv", [64, 128, 256])
@pytest.mark.parametrize("T", [1, 65, 200])
def test_tc_dk256_shapes(la, oracle_mod, dv, T):
    q, k, v = _inputs(2, T, 3, 256, dv, 256 ** -0.5, seed=T + dv)
    _check(la, oracle_mod, q, k, v, torch.tensor([0.97, 1.0, 0.3]))


@pytest.mark.parametrize("phi,normalize", [("elu1", True), ("elu1", False), ("identity", False)])
@pytest.mark.parametrize("gamma", [1.0, 0.96875, 0.2, 0.0])
def test_tc_dk256_feature_maps(la, oracle_mod, phi, normalize, gamma):
    q, k, v = _inputs(1, 333, 2, 256, 256, 256 ** -0.5, seed=11)
    _check(la, oracle_mod, q, k, v, torch.tensor([gamma, 0.99]), phi=phi, normalize=normalize)


def test_tc_dk256_varlen(la, oracle_mod):
    from chunkwise_causal_linear_la_b200.workloads import cu_seqlens_from_lengths

    cu = cu_seqlens_from_lengths([130, 0, 1, 64, 65, 300])
    q, k, v = _inputs(1, int(cu[-1]), 2, 256, 256, 256 ** -0.5, seed=13)
    _check(la, oracle_mod, q, k, v, torch.tensor([0.9, 1.0]), cu=cu, phi="elu1", normalize=True)
    _check(la, oracle_mod, q, k, v, torch.tensor([0.99, 0.1]), cu=cu)


@pytest.mark.parametrize("phi,normalize", [("identity", False), ("elu1", True)])
def test_tc_dk256_segmented(la, oracle_mod, phi, normalize):
    """One long sequence at d = 256: 8 (head, value-slice) units, split into segments."""
    q, k, v = _inputs(1, 5000, 2, 256, 256, 256 ** -0.5, seed=19)
    assert la.workspace_size(1, 5000, 2, 256, 256, 1, False, 64) > 0
    _check(la, oracle_mod, q, k, v, torch.tensor([0.995, 0.9]), phi=phi, normalize=normalize)


def test_tc_retnet_config_sample(la, oracle_mod):
    """The RetNet-style workload (B=32, H=4, T=2048, d_k=d_v=256, gamma_h = 1-2^(-5-h))
    at full size; the oracle checks the first and last (sequence, head) slices."""
    from chunkwise_causal_linear_la_b200.workloads import WORKLOADS, make_inputs

    w = WORKLOADS["retnet_d256"]
    x = make_inputs(w, seed=0)
    dev = torch.device("cuda")
    out, fs = la.la_fwd_chunk(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), x["gamma"].to(dev), chunk=w.chunk,
                              phi=w.phi, normalize=w.normalize)
    torch.cuda.synchronize()
    for b, h in [(0, 0), (31, 3)]:
        qs, ks, vs = (x[n][b:b + 1, :, h:h + 1] for n in ("q", "k", "v"))
        ref, fref = oracle_mod.recurrent(qs, ks, vs, [float(x["gamma"][h])], phi=w.phi, normalize=w.normalize)
        assert slice_rel_err(to_np(out[b:b + 1, :, h:h + 1]), ref, seq_slices(1, 2048)) < TOL[BF]
        assert state_rel_err(to_np(fs[b:b + 1, h:h + 1]), fref) < TOL[BF]


def test_tc_dk256_matches_simt(la):
    q, k, v = _inputs(2, 300, 2, 256, 256, 256 ** -0.5, seed=21)
    dev = torch.device("cuda")
    g = torch.tensor([0.97, 1.0], device=dev)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o1, f1 = la.la_fwd_chunk(qd, kd, vd, g)
    o2, f2 = la.la_fwd_chunk(qd, kd, vd, g, flags=la.LA_FLAG_SIMT)
    torch.cuda.synchronize()
    assert slice_rel_err(to_np(o1), to_np(o2), seq_slices(2, 300)) < TOL[BF]
    assert state_rel_err(to_np(f1), to_np(f2)) < TOL[BF]


def test_tc_device_error_word_clear_after_dk256(la):
    assert la.device_error(reset=True) == (0, 0)
