"""GPU parity of the backward (la_bwd_chunk) against the float64 oracle's
adjoint (oracle.backward), for f32 inputs (tolerance 1e-4) and bf16 inputs
(2e-2): several chunks and a ragged tail, every supported chunk size, both
feature maps, decays including 0 and 1, packed batches with empty sequences.
"""
import numpy as np
import pytest
import torch

from parity_util import TOL, seq_slices, slice_rel_err, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def la():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import chunkwise_causal_linear_la_b200 as la

    la.load_library()
    return la


def _inputs(B, T, H, dk, dv, dtype, seed):
    from chunkwise_causal_linear_la_b200.workloads import make_qkv

    q, k, v = make_qkv(B, T, H, dk, dv, dtype, dk ** -0.5, seed=seed)
    gen = torch.Generator()
    gen.manual_seed(seed + 7)
    dout = torch.randn((B, T, H, dv), generator=gen).to(dtype)
    return q, k, v, dout


def _check(la, oracle_mod, q, k, v, dout, gamma, cu=None, phi="identity", chunk=64):
    dev = torch.device("cuda")
    dq, dk, dv = la.la_bwd_chunk(q.to(dev), k.to(dev), v.to(dev), dout.to(dev), gamma.to(dev),
                                 cu_seqlens=None if cu is None else cu.to(dev), chunk=chunk, phi=phi)
    torch.cuda.synchronize()
    rq, rk, rv = oracle_mod.backward(q, k, v, dout, gamma.double().numpy(),
                                     cu_seqlens=None if cu is None else cu.numpy(), phi=phi)
    B, T = q.shape[:2]
    sl = seq_slices(B, T, None if cu is None else cu.tolist())
    tol = TOL[q.dtype]
    errs = [slice_rel_err(to_np(x), r, sl) for x, r in ((dq, rq), (dk, rk), (dv, rv))]
    assert all(np.isfinite(to_np(x)).all() for x in (dq, dk, dv))
    assert max(errs) < tol, errs


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("chunk", [16, 32, 64, 128])
@pytest.mark.parametrize("phi", ["identity", "elu1"])
def test_bwd_shapes(la, oracle_mod, dtype, chunk, phi):
    q, k, v, dout = _inputs(2, 3 * chunk + 5, 3, 64, 64, dtype, chunk)
    _check(la, oracle_mod, q, k, v, dout, torch.tensor([1.0, 0.95, 0.5]), phi=phi, chunk=chunk)


@pytest.mark.parametrize("dk,dv", [(128, 128), (32, 64), (16, 16), (128, 32)])
def test_bwd_head_dims(la, oracle_mod, dk, dv):
    q, k, v, dout = _inputs(1, 150, 2, dk, dv, torch.float32, dk + dv)
    _check(la, oracle_mod, q, k, v, dout, torch.tensor([0.99, 0.0]))


def test_bwd_varlen(la, oracle_mod):
    from chunkwise_causal_linear_la_b200.workloads import cu_seqlens_from_lengths

    cu = cu_seqlens_from_lengths([100, 0, 1, 64, 65, 200])
    q, k, v, dout = _inputs(1, int(cu[-1]), 4, 64, 64, torch.bfloat16, 5)
    _check(la, oracle_mod, q, k, v, dout, torch.tensor([1.0, 0.9, 0.99, 0.0]), cu=cu, phi="elu1")


def test_bwd_headline_shape_sample(la, oracle_mod):
    """B=8, H=16, d=128, T=2048 prefix of the sweep workload (bf16); the oracle
    checks the first and last (sequence, head) slices."""
    from chunkwise_causal_linear_la_b200.workloads import WORKLOADS, make_inputs

    w = WORKLOADS["sweep_T16384"]
    x = make_inputs(w, seed=0, T=2048)
    gen = torch.Generator()
    gen.manual_seed(3)
    dout = torch.randn(x["v"].shape, generator=gen).to(torch.bfloat16)
    dev = torch.device("cuda")
    dq, dk, dv = la.la_bwd_chunk(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), dout.to(dev), x["gamma"].to(dev))  # tensor cores
    torch.cuda.synchronize()
    for b, h in [(0, 0), (7, 15)]:
        sl = lambda t: t[b:b + 1, :, h:h + 1]  # noqa: E731
        rq, rk, rv = oracle_mod.backward(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(dout), [float(x["gamma"][h])])
        for got, ref in ((dq, rq), (dk, rk), (dv, rv)):
            assert slice_rel_err(to_np(sl(got)), ref, seq_slices(1, 2048)) < TOL[torch.bfloat16]


# ---------------------------------------------------------------- tensor-core backward
# bf16, chunk 64, d_k = d_v in {128, 256}: three tensor-core forward passes,
# two of them in reverse time (windows at negative token offsets, masked rows
# of the previous sequence in packed batches).
@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("T", [1, 65, 300])
@pytest.mark.parametrize("phi", ["identity", "elu1"])
def test_bwd_tc_shapes(la, oracle_mod, d, T, phi):
    q, k, v, dout = _inputs(2, T, 2, d, d, torch.bfloat16, T + d)
    _check(la, oracle_mod, q, k, v, dout, torch.tensor([0.97, 1.0]), phi=phi)


@pytest.mark.parametrize("gamma", [0.0, 0.3, 0.9, 1.0])
def test_bwd_tc_gammas(la, oracle_mod, gamma):
    """gamma <= 0.3 takes the forward kernel's value-decay mode."""
    q, k, v, dout = _inputs(1, 200, 2, 128, 128, torch.bfloat16, 11)
    _check(la, oracle_mod, q, k, v, dout, torch.tensor([gamma, 0.99]), phi="elu1")


def test_bwd_tc_varlen(la, oracle_mod):
    from chunkwise_causal_linear_la_b200.workloads import cu_seqlens_from_lengths

    cu = cu_seqlens_from_lengths([130, 0, 1, 64, 65, 300])
    q, k, v, dout = _inputs(1, int(cu[-1]), 2, 128, 128, torch.bfloat16, 13)
    _check(la, oracle_mod, q, k, v, dout, torch.tensor([0.9, 1.0]), cu=cu)
    _check(la, oracle_mod, q, k, v, dout, torch.tensor([0.99, 0.5]), cu=cu, phi="elu1")


def test_bwd_tc_matches_simt(la):
    q, k, v, dout = _inputs(2, 300, 2, 128, 128, torch.bfloat16, 15)
    dev = torch.device("cuda")
    g = torch.tensor([0.95, 1.0], device=dev)
    args = [x.to(dev) for x in (q, k, v, dout)]
    a = la.la_bwd_chunk(*args, g, phi="elu1")
    b = la.la_bwd_chunk(*args, g, phi="elu1", flags=la.LA_FLAG_SIMT)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert slice_rel_err(to_np(x), to_np(y), seq_slices(2, 300)) < TOL[torch.bfloat16]


def test_bwd_device_error_word_clear(la):
    assert la.device_error(reset=True) == (0, 0)
