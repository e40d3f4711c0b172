"""GPU parity of the normaliser state: la_fwd_chunk_z's final z and the
normalised decode step la_step_norm, against the float64 oracle.

z_t = gamma z_{t-1} + phi(k_t) is accumulated in fp32 from exact inputs, so
final z is checked at 1e-4 on both kernels; outputs and states keep the
tolerances of their dtype (2e-2 bf16, 1e-4 f32).
"""
import numpy as np
import pytest
import torch

from parity_util import TOL, seq_slices, slice_rel_err, state_rel_err, to_np

pytestmark = pytest.mark.gpu

BF = torch.bfloat16
Z_TOL = 1e-4


@pytest.fixture(scope="module")
def la():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import chunkwise_causal_linear_la_b200 as la

    la.load_library()
    return la


def _inputs(B, T, H, dk, dv, dtype, scale, seed):
    from chunkwise_causal_linear_la_b200.workloads import make_qkv

    return make_qkv(B, T, H, dk, dv, dtype, scale, seed=seed)


def _z_err(z, ref):
    return state_rel_err(to_np(z)[..., None], np.asarray(ref)[..., None])


@pytest.mark.parametrize("dtype,flags", [(BF, 0), (torch.float32, 1)])
@pytest.mark.parametrize("dk", [128, 256])
@pytest.mark.parametrize("T,gammas", [(200, (1.0, 0.9)), (65, (0.3, 0.99)), (5000, (0.995, 1.0))])
def test_final_z_dense(la, oracle_mod, dtype, flags, dk, T, gammas):
    """Tensor-core (bf16) and CUDA-core (f32) kernels; T = 5000 with few units is
    segmented on the tensor-core path."""
    if dtype == torch.float32 and T == 5000:
        pytest.skip("the f32 kernel has no segmented path; covered by T = 200")
    q, k, v = _inputs(1, T, 2, dk, dk, dtype, dk ** -0.5, seed=T + dk)
    g = torch.tensor(gammas)
    dev = torch.device("cuda")
    out, fs, z = la.la_fwd_chunk_z(q.to(dev), k.to(dev), v.to(dev), g.to(dev), flags=flags)
    torch.cuda.synchronize()
    ref, fref = oracle_mod.recurrent(q, k, v, g.double().numpy(), phi="elu1", normalize=True)
    zref = oracle_mod.final_z(k, g.double().numpy(), phi="elu1")
    assert _z_err(z, zref) < Z_TOL
    assert slice_rel_err(to_np(out), ref, seq_slices(1, T)) < TOL[dtype]
    assert state_rel_err(to_np(fs), fref) < TOL[dtype]


def test_final_z_varlen(la, oracle_mod):
    from chunkwise_causal_linear_la_b200.workloads import cu_seqlens_from_lengths

    cu = cu_seqlens_from_lengths([130, 0, 1, 64, 65, 300])
    q, k, v = _inputs(1, int(cu[-1]), 3, 128, 128, BF, 128 ** -0.5, seed=7)
    g = torch.tensor([1.0, 0.9, 0.2])
    dev = torch.device("cuda")
    out, fs, z = la.la_fwd_chunk_z(q.to(dev), k.to(dev), v.to(dev), g.to(dev), cu_seqlens=cu.to(dev))
    torch.cuda.synchronize()
    zref = oracle_mod.final_z(k, g.double().numpy(), cu_seqlens=cu.numpy(), phi="elu1")
    assert _z_err(z, zref) < Z_TOL
    assert torch.count_nonzero(z[1]) == 0  # zero-length sequence


@pytest.mark.parametrize("dtype", [torch.float32, BF])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 32), (256, 256)])
def test_step_norm_against_oracle(la, oracle_mod, dtype, dk, dv):
    from chunkwise_causal_linear_la_b200.workloads import make_decode_inputs

    gam = (0.99, 0.9, 1.0, 0.5)
    x = make_decode_inputs(37, 4, dk, dv, dk ** -0.5, 0.01, gam, seed=3, dtype=dtype)
    rng = np.random.default_rng(5)
    z0 = torch.from_numpy(np.abs(rng.standard_normal((37, 4, dk))).astype(np.float32))
    dev = torch.device("cuda")
    state, z = x["state"].to(dev), z0.to(dev)
    o = la.la_step_norm(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), x["gamma"].to(dev), state, z, phi="elu1")
    torch.cuda.synchronize()
    ref_o, ref_s, ref_z = oracle_mod.step_norm(x["q"], x["k"], x["v"], x["gamma"].double().numpy(),
                                               x["state"].double().numpy(), z0.double().numpy(), phi="elu1")
    assert state_rel_err(to_np(state), ref_s) < 1e-6
    assert _z_err(z, ref_z) < 1e-6
    err = max(float(np.max(np.abs(to_np(o)[n, h] - ref_o[n, h])) / np.max(np.abs(ref_o[n, h])))
              for n in range(37) for h in range(4))
    assert err < TOL[dtype], err


def test_prefill_then_normalised_decode(la, oracle_mod):
    """la_fwd_chunk_z over T tokens, then la_step_norm on token T, equals the
    normalised recurrence over T + 1 tokens at its last position."""
    B, T, H, d = 3, 333, 2, 128
    q, k, v = _inputs(B, T + 1, H, d, d, BF, d ** -0.5, seed=11)
    g = torch.tensor([0.97, 1.0])
    dev = torch.device("cuda")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    _, fs, z = la.la_fwd_chunk_z(qd[:, :T].contiguous(), kd[:, :T].contiguous(), vd[:, :T].contiguous(),
                                 g.to(dev))
    o = la.la_step_norm(qd[:, T], kd[:, T], vd[:, T], g.to(dev), fs, z, phi="elu1")
    torch.cuda.synchronize()
    ref, _ = oracle_mod.recurrent(q, k, v, g.double().numpy(), phi="elu1", normalize=True)
    for b in range(B):
        for h in range(H):
            r = ref[b, T, h]
            assert float(np.max(np.abs(to_np(o)[b, h] - r)) / np.max(np.abs(r))) < TOL[BF]


def test_device_error_word_clear_after_norm_state(la):
    assert la.device_error(reset=True) == (0, 0)
