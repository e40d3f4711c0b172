"""The autograd wrappers: gradients through torch.autograd equal the backward entry
points' and match the float64 oracle's adjoints (plain, normalised, per-token decay)."""
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


def _leaf(x, dev):
    return x.to(dev).requires_grad_(True)


def _inputs(B, T, H, d, seed):
    from chunkwise_causal_linear_la_b200.workloads import make_qkv

    q, k, v = make_qkv(B, T, H, d, d, torch.bfloat16, d ** -0.5, seed=seed)
    gen = torch.Generator()
    gen.manual_seed(seed + 1)
    return q, k, v, torch.randn((B, T, H, d), generator=gen).to(torch.bfloat16)


@pytest.mark.parametrize("phi,normalize", [("identity", False), ("elu1", False), ("elu1", True)])
def test_autograd_matches_entry_points_and_oracle(la, oracle_mod, phi, normalize):
    from chunkwise_causal_linear_la_b200.autograd import chunk_linear_attention

    dev = torch.device("cuda")
    q, k, v, dout = _inputs(2, 150, 2, 64, 31)
    gamma = torch.tensor([1.0, 0.9] if not normalize else [1.0, 1.0])
    ql, kl, vl = (_leaf(x, dev) for x in (q, k, v))
    o = chunk_linear_attention(ql, kl, vl, gamma.to(dev), phi=phi, normalize=normalize)
    o.backward(dout.to(dev))
    torch.cuda.synchronize()
    ref_o, _ = la.la_fwd_chunk(q.to(dev), k.to(dev), v.to(dev), gamma.to(dev), phi=phi, normalize=normalize)
    bwd = la.la_bwd_chunk_norm if normalize else la.la_bwd_chunk
    grads = bwd(q.to(dev), k.to(dev), v.to(dev), dout.to(dev), gamma.to(dev), phi=phi)
    torch.cuda.synchronize()
    assert torch.equal(o.detach(), ref_o)
    for x, g in zip((ql, kl, vl), grads):
        assert torch.equal(x.grad, g)
    if not normalize:  # against the oracle (the normalised one has its own metric in test_bwd_gpu.py)
        refs = oracle_mod.backward(q, k, v, dout, gamma.double().numpy(), phi=phi)
        sl = seq_slices(2, 150)
        assert max(slice_rel_err(to_np(x.grad), r, sl) for x, r in zip((ql, kl, vl), refs)) < TOL[torch.bfloat16]


def test_autograd_gated_reaches_log_decays(la, oracle_mod):
    from chunkwise_causal_linear_la_b200.autograd import chunk_gated_linear_attention
    from chunkwise_causal_linear_la_b200.workloads import make_log_decay

    dev = torch.device("cuda")
    q, k, v, dout = _inputs(1, 200, 2, 128, 37)
    gen = torch.Generator()
    gen.manual_seed(38)
    g = make_log_decay(1, 200, 2, 0.9, 0.999, gen)
    ql, kl, vl, gl = _leaf(q, dev), _leaf(k, dev), _leaf(v, dev), g.to(dev).requires_grad_(True)
    o = chunk_gated_linear_attention(ql, kl, vl, gl, phi="elu1")
    o.backward(dout.to(dev))
    torch.cuda.synchronize()
    dq, dk, dv, dg = la.la_bwd_chunk_gated(q.to(dev), k.to(dev), v.to(dev), dout.to(dev), g.to(dev), phi="elu1")
    torch.cuda.synchronize()
    for x, r in zip((ql, kl, vl), (dq, dk, dv)):
        assert torch.equal(x.grad, r)
    # dg sums row terms with float atomics: equal up to the order of the additions
    assert torch.allclose(gl.grad, dg, rtol=1e-5, atol=1e-6 * dg.abs().max().item())
    refs = oracle_mod.backward_gated(q, k, v, dout, g.double().numpy(), phi="elu1")
    sl = seq_slices(1, 200)
    assert max(slice_rel_err(to_np(x.grad), r, sl) for x, r in zip((ql, kl, vl), refs[:3])) < TOL[torch.bfloat16]
    assert np.isfinite(to_np(gl.grad)).all()


def test_autograd_packed_batch_f32(la, oracle_mod):
    """Packed batch in f32 (CUDA-core kernels), normalised: gradients are the entry point's."""
    from chunkwise_causal_linear_la_b200.autograd import chunk_linear_attention
    from chunkwise_causal_linear_la_b200.workloads import cu_seqlens_from_lengths, make_qkv

    dev = torch.device("cuda")
    cu = cu_seqlens_from_lengths([70, 0, 1, 64, 33])
    q, k, v = make_qkv(1, int(cu[-1]), 2, 64, 64, torch.float32, 0.125, seed=41)
    dout = torch.randn(v.shape, generator=torch.Generator().manual_seed(42))
    gamma = torch.tensor([1.0, 0.95])
    ql, kl, vl = (_leaf(x, dev) for x in (q, k, v))
    o = chunk_linear_attention(ql, kl, vl, gamma.to(dev), cu_seqlens=cu.to(dev), phi="elu1", normalize=True)
    o.backward(dout.to(dev))
    grads = la.la_bwd_chunk_norm(q.to(dev), k.to(dev), v.to(dev), dout.to(dev), gamma.to(dev), cu_seqlens=cu.to(dev),
                                 phi="elu1")
    torch.cuda.synchronize()
    for x, g in zip((ql, kl, vl), grads):
        assert torch.equal(x.grad, g)


def test_entry_points_from_a_fresh_thread(la):
    """The first call of a thread that has made no CUDA call yet (torch's autograd worker,
    a serving thread): each TMA entry point binds the device's context before encoding
    its tensor maps, so the results equal the main thread's."""
    import threading

    from chunkwise_causal_linear_la_b200.workloads import make_log_decay

    dev = torch.device("cuda")
    q, k, v, dout = (x.to(dev) for x in _inputs(1, 200, 2, 128, 43))
    gamma = torch.tensor([0.97, 1.0], device=dev)
    gen = torch.Generator()
    gen.manual_seed(44)
    g = make_log_decay(1, 200, 2, 0.8, 1.0, gen).to(dev)
    beta = (torch.rand((1, 200, 2), generator=gen) * 0.9 + 0.1).to(dev)
    calls = {
        "fwd": lambda: la.la_fwd_chunk(q, k, v, gamma)[0],
        "bwd": lambda: la.la_bwd_chunk(q, k, v, dout, gamma)[0],
        "bwd_norm": lambda: la.la_bwd_chunk_norm(q, k, v, dout, torch.ones(2, device=dev))[1],
        "gated_delta": lambda: la.la_fwd_gated_delta_chunk(q, k, v, g, beta)[0],
    }
    for name, fn in calls.items():
        want = fn()
        torch.cuda.synchronize()
        got = {}

        def work():
            try:
                got["x"] = fn()
                torch.cuda.synchronize()
            except Exception as e:  # reported below on the test's thread
                got["e"] = e
        t = threading.Thread(target=work)
        t.start()
        t.join()
        assert "e" not in got, (name, got.get("e"))
        assert torch.equal(got["x"], want), name


def test_autograd_gated_normalised(la, oracle_mod):
    from chunkwise_causal_linear_la_b200.autograd import chunk_gated_linear_attention
    from chunkwise_causal_linear_la_b200.workloads import make_log_decay

    dev = torch.device("cuda")
    q, k, v, dout = _inputs(1, 150, 2, 64, 47)
    gen = torch.Generator()
    gen.manual_seed(48)
    g = make_log_decay(1, 150, 2, 0.9, 0.999, gen)
    ql, kl, vl, gl = _leaf(q, dev), _leaf(k, dev), _leaf(v, dev), g.to(dev).requires_grad_(True)
    o = chunk_gated_linear_attention(ql, kl, vl, gl, phi="elu1", normalize=True)
    o.backward(dout.to(dev))
    want = la.la_bwd_chunk_gated_norm(q.to(dev), k.to(dev), v.to(dev), dout.to(dev), g.to(dev), phi="elu1")
    torch.cuda.synchronize()
    for x, r in zip((ql, kl, vl), want[:3]):
        assert torch.equal(x.grad, r)
    assert torch.allclose(gl.grad, want[3], rtol=1e-5, atol=1e-6 * want[3].abs().max().item())
