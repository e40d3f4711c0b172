"""GPU parity of 64-wide heads on the tensor-core kernel against the float64 oracle.

d_k = 64 runs in the d_k = 128 layout with the key and query columns 64 .. 127
read as TMA zero fill (and kept out of the feature map, since elu(0) + 1 = 1);
d_v = 64 runs in a 128-wide value slice whose extra columns are never written.
Cases: every head-dim pairing of 64 with {64, 128, 256}, both feature maps with
and without the normaliser, decays on both of the kernel's decay paths, packed
batches with empty sequences, a long sequence split into segments, the final z
handed to the normalised decode, the per-token decay and the backward pass.
la_fwd_chunk_path must report the tensor cores for each of these shapes, and
the CUDA-core kernel for the shapes that stay there.
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


def _inputs(B, T, H, dk, dv, seed):
    from chunkwise_causal_linear_la_b200.workloads import make_qkv

    return make_qkv(B, T, H, dk, dv, BF, dk ** -0.5, seed=seed)


def _check(la, oracle_mod, q, k, v, gamma, cu=None, phi="identity", normalize=False):
    dev = torch.device("cuda")
    B, T, H, dk = q.shape
    dv = v.shape[3]
    assert la.fwd_chunk_path(dk, dv, T, H, 64, BF) == la.LA_PATH_TENSOR_CORE
    out, fs = la.la_fwd_chunk(q.to(dev), k.to(dev), v.to(dev), gamma.to(dev),
                              cu_seqlens=None if cu is None else cu.to(dev), chunk=64, phi=phi,
                              normalize=normalize)
    torch.cuda.synchronize()
    ref, fref = oracle_mod.recurrent(q, k, v, gamma.double().numpy(), cu_seqlens=None if cu is None else cu.numpy(),
                                     phi=phi, normalize=normalize)
    assert np.isfinite(to_np(out)).all()
    e1 = slice_rel_err(to_np(out), ref, seq_slices(B, T, None if cu is None else cu.tolist()))
    e2 = state_rel_err(to_np(fs), fref)
    assert e1 < TOL[BF] and e2 < TOL[BF], (e1, e2)


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64), (64, 256)])
@pytest.mark.parametrize("phi,normalize", [("identity", False), ("elu1", True), ("elu1", False)])
def test_d64_shapes(la, oracle_mod, dk, dv, phi, normalize):
    q, k, v = _inputs(2, 4 * 64 + 17, 2, dk, dv, seed=dk + dv)
    gamma = torch.tensor([1.0, 1.0] if normalize else [0.95, 1.0])
    _check(la, oracle_mod, q, k, v, gamma, phi=phi, normalize=normalize)


@pytest.mark.parametrize("gamma", [0.0, 0.3, 0.9, 0.999])
@pytest.mark.parametrize("T", [1, 64, 65, 200])
def test_d64_decays_and_lengths(la, oracle_mod, gamma, T):
    """gamma <= 0.3 takes the value-decay path, the others the decayed-key path."""
    q, k, v = _inputs(1, T, 2, 64, 64, seed=T)
    _check(la, oracle_mod, q, k, v, torch.tensor([gamma, 1.0]), phi="elu1")


def test_d64_packed_batch(la, oracle_mod):
    from chunkwise_causal_linear_la_b200.workloads import cu_seqlens_from_lengths

    cu = cu_seqlens_from_lengths([130, 0, 1, 64, 65, 300, 17, 128])
    q, k, v = _inputs(1, int(cu[-1]), 3, 64, 64, seed=5)
    _check(la, oracle_mod, q, k, v, torch.tensor([1.0, 0.97, 0.5]), cu=cu, phi="elu1", normalize=False)
    _check(la, oracle_mod, q, k, v, torch.ones(3), cu=cu, phi="elu1", normalize=True)


@pytest.mark.parametrize("phi,normalize", [("identity", False), ("elu1", True)])
def test_d64_segmented_long_sequence(la, oracle_mod, phi, normalize):
    """One sequence per head on few units: split into segments (state pass, scan, output pass)."""
    T, H = 5000, 2
    assert la.workspace_size(1, T, H, 64, 64, 1, False, 64) > 0
    q, k, v = _inputs(1, T, H, 64, 64, seed=17)
    gamma = torch.ones(H) if normalize else torch.tensor([0.995, 1.0])
    _check(la, oracle_mod, q, k, v, gamma, phi=phi, normalize=normalize)


def test_d64_final_z(la, oracle_mod):
    """z after the last token (la_fwd_chunk_z) for the normalised decode: only d_k = 64 entries."""
    dev = torch.device("cuda")
    q, k, v = _inputs(2, 150, 2, 64, 128, seed=19)
    gamma = torch.tensor([0.98, 1.0])
    out, fs, fz = la.la_fwd_chunk_z(q.to(dev), k.to(dev), v.to(dev), gamma.to(dev), phi="elu1")
    torch.cuda.synchronize()
    zref = oracle_mod.final_z(k, gamma.double().numpy(), phi="elu1")
    assert tuple(fz.shape) == (2, 2, 64)
    assert state_rel_err(to_np(fz)[..., None], zref[..., None]) < 1e-4


def test_d64_per_token_decay(la, oracle_mod):
    from chunkwise_causal_linear_la_b200.workloads import make_log_decay

    dev = torch.device("cuda")
    q, k, v = _inputs(2, 200, 2, 64, 64, seed=23)
    gen = torch.Generator()
    gen.manual_seed(24)
    g = make_log_decay(2, 200, 2, 0.9, 0.999, gen)
    out, fs, _ = la.la_fwd_chunk_gated(q.to(dev), k.to(dev), v.to(dev), g.to(dev), phi="elu1", normalize=False)
    torch.cuda.synchronize()
    ref, fref, _ = oracle_mod.recurrent_gated(q, k, v, g.double().numpy(), phi="elu1", normalize=False)
    assert slice_rel_err(to_np(out), ref, seq_slices(2, 200)) < TOL[BF]
    assert state_rel_err(to_np(fs), fref) < TOL[BF]


@pytest.mark.parametrize("phi", ["identity", "elu1"])
def test_d64_backward(la, oracle_mod, phi):
    from chunkwise_causal_linear_la_b200.workloads import make_dout

    dev = torch.device("cuda")
    q, k, v = _inputs(2, 200, 2, 64, 64, seed=29)
    dout = make_dout(v, seed=29)
    gamma = torch.tensor([0.97, 1.0])
    grads = la.la_bwd_chunk(q.to(dev), k.to(dev), v.to(dev), dout.to(dev), gamma.to(dev), phi=phi)
    torch.cuda.synchronize()
    refs = oracle_mod.backward(q, k, v, dout, gamma.double().numpy(), phi=phi)
    for got, ref in zip(grads, refs):
        assert slice_rel_err(to_np(got), ref, seq_slices(2, 200)) < TOL[BF]


def test_path_query(la):
    tc, cc = la.LA_PATH_TENSOR_CORE, la.LA_PATH_CUDA_CORE
    for dk, dv in [(64, 64), (64, 128), (128, 64), (128, 128), (128, 256), (256, 64), (256, 256)]:
        assert la.fwd_chunk_path(dk, dv, 1000, 4, 64, BF) == tc, (dk, dv)
    assert la.fwd_chunk_path(128, 128, 1000, 4, 64, torch.float32) == cc
    assert la.fwd_chunk_path(128, 128, 1000, 4, 64, BF, la.LA_FLAG_SIMT) == cc
    for chunk in (16, 32, 128):
        assert la.fwd_chunk_path(128, 128, 1000, 4, chunk, BF) == cc
    assert la.fwd_chunk_path(32, 32, 1000, 4, 64, BF) == cc
    assert la.fwd_chunk_path(128, 128, 1000, 4, 48, BF) == -1
    assert la.device_error(reset=True) == (0, 0)
