"""GPU parity of the output RMSNorm with a Swish gate: the standalone kernel
(la_norm_gate) and the forward with the norm fused into its epilogue
(la_fwd_chunk_normgate; fused on the tensor cores at d_k = d_v = 128, a second
pass elsewhere), against the float64 oracle: oracle.norm_gate applied to the
oracle's forward output.
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


def _gate_w(shape, dtype, seed):
    gen = torch.Generator()
    gen.manual_seed(seed)
    gate = (torch.randn(shape, generator=gen) * 2.0).to(dtype)
    w = torch.rand(shape[-1], generator=gen) + 0.5
    return gate, w


@pytest.mark.parametrize("dtype", [torch.float32, BF])
@pytest.mark.parametrize("dv", [16, 64, 128, 256])
def test_norm_gate_standalone(la, oracle_mod, dtype, dv):
    gen = torch.Generator()
    gen.manual_seed(dv)
    o = torch.randn((2, 33, 3, dv), generator=gen).to(dtype)
    gate, w = _gate_w(o.shape, dtype, dv + 1)
    dev = torch.device("cuda")
    y = la.la_norm_gate(o.to(dev), gate.to(dev), w.to(dev), eps=1e-5)
    torch.cuda.synchronize()
    ref = oracle_mod.norm_gate(to_np(o), gate, w.double().numpy(), eps=1e-5)
    assert slice_rel_err(to_np(y), ref, seq_slices(2, 33)) < TOL[dtype]
    # in place
    od = o.to(dev)
    la.la_norm_gate(od, gate.to(dev), w.to(dev), eps=1e-5, y=od)
    torch.cuda.synchronize()
    assert slice_rel_err(to_np(od), ref, seq_slices(2, 33)) < TOL[dtype]


@pytest.mark.parametrize("dk,dv", [(128, 128), (128, 256), (256, 256)])
@pytest.mark.parametrize("phi,normalize", [("identity", False), ("elu1", True)])
@pytest.mark.parametrize("T", [1, 65, 300])
def test_fwd_normgate(la, oracle_mod, dk, dv, phi, normalize, T):
    """Fused on the tensor cores for d_k = d_v = 128; a second pass otherwise."""
    from chunkwise_causal_linear_la_b200.workloads import make_qkv

    q, k, v = make_qkv(2, T, 2, dk, dv, BF, dk ** -0.5, seed=T + dv)
    gate, w = _gate_w(v.shape, BF, T)
    gam = torch.tensor([0.97, 0.3])
    dev = torch.device("cuda")
    out, fs = la.la_fwd_chunk_normgate(q.to(dev), k.to(dev), v.to(dev), gam.to(dev), gate.to(dev), w.to(dev),
                                       eps=1e-5, phi=phi, normalize=normalize)
    torch.cuda.synchronize()
    ref, fref = oracle_mod.recurrent(q, k, v, gam.double().numpy(), phi=phi, normalize=normalize)
    yref = oracle_mod.norm_gate(ref, gate, w.double().numpy(), eps=1e-5)
    assert np.isfinite(to_np(out)).all()
    assert slice_rel_err(to_np(out), yref, seq_slices(2, T)) < TOL[BF]
    assert state_rel_err(to_np(fs), fref) < TOL[BF]


def test_fwd_normgate_varlen(la, oracle_mod):
    from chunkwise_causal_linear_la_b200.workloads import cu_seqlens_from_lengths, make_qkv

    cu = cu_seqlens_from_lengths([130, 0, 1, 64, 65, 300])
    q, k, v = make_qkv(1, int(cu[-1]), 2, 128, 128, BF, 128 ** -0.5, seed=3)
    gate, w = _gate_w(v.shape, BF, 4)
    gam = torch.tensor([1.0, 0.9])
    dev = torch.device("cuda")
    out, _ = la.la_fwd_chunk_normgate(q.to(dev), k.to(dev), v.to(dev), gam.to(dev), gate.to(dev), w.to(dev),
                                      cu_seqlens=cu.to(dev), phi="elu1", normalize=True)
    torch.cuda.synchronize()
    ref, _ = oracle_mod.recurrent(q, k, v, gam.double().numpy(), cu_seqlens=cu.numpy(), phi="elu1", normalize=True)
    yref = oracle_mod.norm_gate(ref, gate, w.double().numpy(), eps=1e-5)
    assert slice_rel_err(to_np(out), yref, seq_slices(1, 0, cu.tolist())) < TOL[BF]


def test_device_error_word_clear_after_norm_gate(la):
    assert la.device_error(reset=True) == (0, 0)
