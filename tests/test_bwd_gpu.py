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
    dq, dk, dv = la.la_bwd_chunk(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), dout.to(dev), x["gamma"].to(dev))
    torch.cuda.synchronize()
    for b, h in [(0, 0), (7, 15)]:
        sl = lambda t: t[b:b + 1, :, h:h + 1]  # noqa: E731
        rq, rk, rv = oracle_mod.backward(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(dout), [float(x["gamma"][h])])
        for got, ref in ((dq, rq), (dk, rk), (dv, rv)):
            assert slice_rel_err(to_np(sl(got)), ref, seq_slices(1, 2048)) < TOL[torch.bfloat16]
