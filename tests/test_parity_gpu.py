"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Inputs come from the seeded generators in chunkwise_causal_linear_la_b200.workloads
and are handed unchanged to both sides.  Sizes are small enough for the oracle
to finish in seconds but span several chunks and a ragged last chunk.  The
tolerances are the target's: 1e-4 for fp32 inputs, 2e-2 for bf16 inputs (fp32
accumulation), for the outputs and for the final states, with the error
metric of parity_util.
"""
import numpy as np
import pytest
import torch

from parity_util import TOL, seq_slices, slice_rel_err, state_rel_err, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def la():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import chunkwise_causal_linear_la_b200 as la

    la.load_library()
    return la


def _run_pair(la, oracle_mod, q, k, v, gamma, cu=None, chunk=64, phi="identity", normalize=False, flags=0):
    dev = torch.device("cuda")
    qd, kd, vd, gd = (x.to(dev) for x in (q, k, v, gamma))
    cud = None if cu is None else cu.to(dev)
    out, fs = la.la_fwd_chunk(qd, kd, vd, gd, cu_seqlens=cud, chunk=chunk, phi=phi, normalize=normalize,
                              flags=flags)
    torch.cuda.synchronize()
    ref, fref = oracle_mod.recurrent(q, k, v, gamma.double().numpy(), cu_seqlens=None if cu is None else cu.numpy(),
                                     phi=phi, normalize=normalize)
    B, T = q.shape[:2]
    e_out = slice_rel_err(to_np(out), ref, seq_slices(B, T, None if cu is None else cu.tolist()))
    e_fs = state_rel_err(to_np(fs), fref)
    return e_out, e_fs, out, fs


def _inputs(B, T, H, dk, dv, dtype, scale, seed=0):
    from chunkwise_causal_linear_la_b200.workloads import make_qkv

    return make_qkv(B, T, H, dk, dv, dtype, scale, seed=seed)


def test_tiny_f32_config(la, oracle_mod):
    """B=1, H=2, T=256, d=64, chunk=64, elu+1 with normaliser, gamma=1, N(0,1), fp32."""
    from chunkwise_causal_linear_la_b200.workloads import WORKLOADS, make_inputs

    w = WORKLOADS["tiny_f32"]
    x = make_inputs(w, seed=0)
    e_out, e_fs, _, _ = _run_pair(la, oracle_mod, x["q"], x["k"], x["v"], x["gamma"], chunk=w.chunk,
                                  phi=w.phi, normalize=w.normalize)
    assert e_out < TOL[torch.float32] and e_fs < TOL[torch.float32], (e_out, e_fs)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("chunk", [16, 32, 64, 128])
@pytest.mark.parametrize("phi,normalize", [("identity", False), ("elu1", True), ("elu1", False)])
def test_simt_kernel_shapes(la, oracle_mod, dtype, chunk, phi, normalize):
    # T = 3*chunk + 5: several chunks and a ragged tail
    B, H, d = 2, 3, 64
    T = 3 * chunk + 5
    q, k, v = _inputs(B, T, H, d, d, dtype, 1.0 / 8, seed=chunk)
    gamma = torch.tensor([1.0, 0.95, 0.5], dtype=torch.float32)
    e_out, e_fs, _, _ = _run_pair(la, oracle_mod, q, k, v, gamma, chunk=chunk, phi=phi, normalize=normalize,
                                  flags=la.LA_FLAG_SIMT)
    assert e_out < TOL[dtype] and e_fs < TOL[dtype], (e_out, e_fs)


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (128, 128), (256, 256), (128, 32)])
def test_simt_head_dims(la, oracle_mod, dk, dv):
    q, k, v = _inputs(1, 150, 2, dk, dv, torch.float32, dk ** -0.5, seed=dk + dv)
    gamma = torch.tensor([0.99, 1.0])
    e_out, e_fs, _, _ = _run_pair(la, oracle_mod, q, k, v, gamma, chunk=64, flags=la.LA_FLAG_SIMT)
    assert e_out < TOL[torch.float32] and e_fs < TOL[torch.float32], (e_out, e_fs)


def test_simt_varlen(la, oracle_mod):
    from chunkwise_causal_linear_la_b200.workloads import cu_seqlens_from_lengths

    lengths = [100, 0, 1, 64, 65, 200, 17]
    cu = cu_seqlens_from_lengths(lengths)
    q, k, v = _inputs(1, int(cu[-1]), 4, 64, 64, torch.bfloat16, 0.125, seed=5)
    gamma = torch.tensor([1.0, 0.9, 0.99, 0.0])
    e_out, e_fs, out, fs = _run_pair(la, oracle_mod, q, k, v, gamma, cu=cu, chunk=64, phi="elu1", normalize=True,
                                     flags=la.LA_FLAG_SIMT)
    assert e_out < TOL[torch.bfloat16] and e_fs < TOL[torch.bfloat16], (e_out, e_fs)
    assert torch.count_nonzero(fs[1]) == 0  # zero-length sequence -> zero state


def test_empty_inputs(la):
    dev = torch.device("cuda")
    q = torch.zeros((2, 0, 2, 64), device=dev, dtype=torch.bfloat16)
    gamma = torch.ones(2, device=dev)
    out, fs = la.la_fwd_chunk(q, q, q, gamma)
    torch.cuda.synchronize()
    assert out.shape == (2, 0, 2, 64) and fs.shape == (2, 2, 64, 64)
    assert torch.count_nonzero(fs) == 0


def test_strided_inputs(la, oracle_mod):
    """q, k, v as views into one [B, T, H, 3*d] projection output (non-contiguous token stride)."""
    B, T, H, d = 2, 130, 2, 64
    base = torch.randn((B, T, H, 3 * d), dtype=torch.float32) * 0.2
    q, k, v = base[..., :d], base[..., d:2 * d], base[..., 2 * d:]
    gamma = torch.tensor([0.97, 1.0])
    dev = torch.device("cuda")
    based = base.to(dev)
    qd, kd, vd = based[..., :d], based[..., d:2 * d], based[..., 2 * d:]
    out, fs = la.la_fwd_chunk(qd, kd, vd, gamma.to(dev), chunk=32)
    torch.cuda.synchronize()
    ref, fref = oracle_mod.recurrent(q.contiguous().numpy(), k.contiguous().numpy(), v.contiguous().numpy(),
                                     gamma.double().numpy())
    assert slice_rel_err(to_np(out), ref, seq_slices(B, T)) < 1e-4
    assert state_rel_err(to_np(fs), fref) < 1e-4


# ---------------------------------------------------------------- decode
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("phi", ["identity", "elu1"])
def test_step_against_oracle(la, oracle_mod, dtype, phi):
    from chunkwise_causal_linear_la_b200.workloads import make_decode_inputs

    x = make_decode_inputs(37, 4, 128, 128, 128 ** -0.5, 0.01, (0.99, 0.9, 1.0, 0.5), seed=3, dtype=dtype)
    dev = torch.device("cuda")
    state = x["state"].to(dev)
    o = la.la_step(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), x["gamma"].to(dev), state, phi=phi)
    torch.cuda.synchronize()
    ref_o, ref_s = oracle_mod.step(x["q"], x["k"], x["v"], x["gamma"].double().numpy(), x["state"].double().numpy(),
                                   phi=phi)
    tol = TOL[dtype]
    assert state_rel_err(to_np(state), ref_s) < 1e-6
    err = max(float(np.max(np.abs(to_np(o)[n, h] - ref_o[n, h])) / np.max(np.abs(ref_o[n, h])))
              for n in range(37) for h in range(4))
    assert err < tol, err


@pytest.mark.parametrize("dk,dv", [(64, 64), (256, 256), (128, 32), (32, 4)])
def test_step_head_dims(la, oracle_mod, dk, dv):
    from chunkwise_causal_linear_la_b200.workloads import make_decode_inputs

    x = make_decode_inputs(5, 3, dk, dv, dk ** -0.5, 0.1, (0.9, 1.0, 0.0), seed=dk)
    dev = torch.device("cuda")
    state = x["state"].to(dev)
    o = la.la_step(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), x["gamma"].to(dev), state)
    torch.cuda.synchronize()
    ref_o, ref_s = oracle_mod.step(x["q"], x["k"], x["v"], x["gamma"].double().numpy(), x["state"].double().numpy())
    assert state_rel_err(to_np(state), ref_s) < 1e-6
    assert float(np.max(np.abs(to_np(o) - ref_o)) / np.max(np.abs(ref_o))) < 1e-5


@pytest.mark.parametrize("flags", [0, 1])
def test_prefill_then_step_equals_longer_prefill(la, oracle_mod, flags):
    """la_fwd_chunk on T tokens, then la_step on token T+1, matches the oracle on T+1 tokens."""
    B, T, H, d = 3, 200, 2, 128
    q, k, v = _inputs(B, T + 1, H, d, d, torch.float32, d ** -0.5, seed=11)
    gamma = torch.tensor([0.98, 1.0])
    dev = torch.device("cuda")
    _, fs = la.la_fwd_chunk(q[:, :T].contiguous().to(dev), k[:, :T].contiguous().to(dev),
                            v[:, :T].contiguous().to(dev), gamma.to(dev), chunk=64, flags=flags)
    o = la.la_step(q[:, T].contiguous().to(dev), k[:, T].contiguous().to(dev), v[:, T].contiguous().to(dev),
                   gamma.to(dev), fs)
    torch.cuda.synchronize()
    ref, fref = oracle_mod.recurrent(q, k, v, gamma.double().numpy())
    assert float(np.max(np.abs(to_np(o) - ref[:, T])) / np.max(np.abs(ref[:, T]))) < 1e-4
    assert state_rel_err(to_np(fs), fref) < 1e-4
