"""GPU parity of the gated delta rule (la_fwd_gated_delta) against the float64
oracle (oracle.gated_delta): head dims 16 .. 256 (d_k = 256 splits each value
column's state over two threads), f32 and bf16 inputs, strong and mild
decays and write strengths, packed batches with empty sequences, an initial
state, and a decode step updating the state in place.
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


def _inputs(B, T, H, dk, dv, dtype, seed, alo=0.8, blo=0.1):
    from chunkwise_causal_linear_la_b200.workloads import make_log_decay, make_qkv

    q, k, v = make_qkv(B, T, H, dk, dv, dtype, dk ** -0.5, seed=seed)
    gen = torch.Generator()
    gen.manual_seed(seed + 1)
    g = make_log_decay(B, T, H, alo, 1.0, gen)
    beta = torch.rand((B, T, H), generator=gen) * (1.0 - blo) + blo
    return q, k, v, g, beta


def _check(la, oracle_mod, q, k, v, g, beta, cu=None, init=None):
    dev = torch.device("cuda")
    out, fs = la.la_fwd_gated_delta(q.to(dev), k.to(dev), v.to(dev), g.to(dev), beta.to(dev),
                                    cu_seqlens=None if cu is None else cu.to(dev),
                                    initial_state=None if init is None else init.to(dev))
    torch.cuda.synchronize()
    ref, fref = oracle_mod.gated_delta(q, k, v, g.double().numpy(), beta.double().numpy(),
                                       cu_seqlens=None if cu is None else cu.numpy(),
                                       init=None if init is None else init.double().numpy())
    B, T = q.shape[:2]
    tol = TOL[q.dtype]
    e1 = slice_rel_err(to_np(out), ref, seq_slices(B, T, None if cu is None else cu.tolist()))
    e2 = state_rel_err(to_np(fs), fref)
    assert np.isfinite(to_np(out)).all()
    assert e1 < tol and e2 < tol, (e1, e2)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dk,dv", [(16, 16), (64, 64), (128, 128), (256, 256), (64, 128), (128, 32), (256, 64)])
def test_gated_delta_shapes(la, oracle_mod, dtype, dk, dv):
    q, k, v, g, beta = _inputs(2, 150, 2, dk, dv, dtype, dk + dv)
    _check(la, oracle_mod, q, k, v, g, beta)


@pytest.mark.parametrize("T", [1, 64, 65, 300])
@pytest.mark.parametrize("alo,blo", [(0.05, 0.01), (0.99, 0.9)])
def test_gated_delta_lengths_and_gates(la, oracle_mod, T, alo, blo):
    q, k, v, g, beta = _inputs(1, T, 3, 128, 128, torch.bfloat16, T, alo, blo)
    _check(la, oracle_mod, q, k, v, g, beta)


def test_gated_delta_varlen_and_initial_state(la, oracle_mod):
    from chunkwise_causal_linear_la_b200.workloads import cu_seqlens_from_lengths

    cu = cu_seqlens_from_lengths([130, 0, 1, 64, 65, 300])
    q, k, v, g, beta = _inputs(1, int(cu[-1]), 2, 64, 64, torch.float32, 5)
    _check(la, oracle_mod, q, k, v, g, beta, cu=cu)
    init = torch.randn((6, 2, 64, 64)) * 0.1
    _check(la, oracle_mod, q, k, v, g, beta, cu=cu, init=init)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (256, 256), (128, 32), (64, 256)])
def test_gated_delta_one_token_decode_kernel(la, oracle_mod, dtype, dk, dv):
    """T = 1 takes the decode kernel (coalesced state, reductions across warps):
    with and without an initial state, value slices narrower than 128 columns."""
    q, k, v, g, beta = _inputs(5, 1, 3, dk, dv, dtype, dk + 7 * dv)
    init = torch.randn((5, 3, dk, dv)) * 0.3
    _check(la, oracle_mod, q, k, v, g, beta)
    _check(la, oracle_mod, q, k, v, g, beta, init=init)


def test_gated_delta_decode_in_place(la, oracle_mod):
    """Prefill T tokens, then one token at a time with the state updated in place,
    equals the oracle over all tokens."""
    B, T, H, d = 2, 100, 2, 128
    q, k, v, g, beta = _inputs(B, T + 3, H, d, d, torch.float32, 9)
    dev = torch.device("cuda")
    qd, kd, vd, gd, bd = (x.to(dev) for x in (q, k, v, g, beta))
    _, state = la.la_fwd_gated_delta(qd[:, :T].contiguous(), kd[:, :T].contiguous(), vd[:, :T].contiguous(),
                                     gd[:, :T].contiguous(), bd[:, :T].contiguous())
    outs = []
    for t in range(T, T + 3):
        o, _ = la.la_fwd_gated_delta(qd[:, t:t + 1].contiguous(), kd[:, t:t + 1].contiguous(),
                                     vd[:, t:t + 1].contiguous(), gd[:, t:t + 1].contiguous(),
                                     bd[:, t:t + 1].contiguous(), initial_state=state, final_state=state)
        outs.append(o)
    torch.cuda.synchronize()
    ref, fref = oracle_mod.gated_delta(q, k, v, g.double().numpy(), beta.double().numpy())
    for j, o in enumerate(outs):
        assert slice_rel_err(to_np(o), ref[:, T + j:T + j + 1], seq_slices(B, 1)) < 1e-4
    assert state_rel_err(to_np(state), fref) < 1e-4


# ---------------------------------------------------------------- chunked (tensor-core) path
def _check_chunk(la, oracle_mod, q, k, v, g, beta, cu=None, init=None, flags=0, garbage=False):
    """la_fwd_gated_delta_chunk against the token-by-token oracle.  garbage: the
    workspace starts filled with NaN bit patterns (nothing may read unwritten rows)."""
    dev = torch.device("cuda")
    B, T, H, dk = q.shape
    dv = v.shape[3]
    n = B if cu is None else cu.numel() - 1
    ws = None
    need = la.gated_delta_workspace_size(B, T, H, dk, dv, n, cu is not None, q.dtype, flags)
    if need:
        ws = torch.full((need,), 0xFF if garbage else 0, dtype=torch.uint8, device=dev)
    out, fs = la.la_fwd_gated_delta_chunk(q.to(dev), k.to(dev), v.to(dev), g.to(dev), beta.to(dev),
                                          cu_seqlens=None if cu is None else cu.to(dev),
                                          initial_state=None if init is None else init.to(dev), flags=flags,
                                          workspace=ws)
    torch.cuda.synchronize()
    assert la.device_error(reset=True) == (0, 0)
    ref, fref = oracle_mod.gated_delta(q, k, v, g.double().numpy(), beta.double().numpy(),
                                       cu_seqlens=None if cu is None else cu.numpy(),
                                       init=None if init is None else init.double().numpy())
    tol = TOL[q.dtype]
    e1 = slice_rel_err(to_np(out), ref, seq_slices(B, T, None if cu is None else cu.tolist()))
    e2 = state_rel_err(to_np(fs), fref)
    assert e1 < tol and e2 < tol, (e1, e2)
    return out, fs


@pytest.mark.parametrize("T", [1, 63, 64, 65, 200, 1000])
@pytest.mark.parametrize("alo,blo", [(0.05, 0.01), (0.9, 0.5), (0.999, 0.99)])
def test_gated_delta_chunk_lengths_and_gates(la, oracle_mod, T, alo, blo):
    """Tensor-core path (bf16, d = 128): partial last chunks, strong and mild decay,
    weak and full-strength writes."""
    q, k, v, g, beta = _inputs(2, T, 3, 128, 128, torch.bfloat16, 1000 + T, alo, blo)
    _check_chunk(la, oracle_mod, q, k, v, g, beta)


def test_gated_delta_chunk_zero_and_tiny_keys(la, oracle_mod):
    """Keys that are exactly zero or far below the 1e-12 norm floor: the chunk kernel
    reads the raw keys and takes 1/max(|k|, 1e-12) through the decay exponents, so
    such rows must give what the unit-key definition gives (a zero or tiny kt)."""
    q, k, v, g, beta = _inputs(2, 200, 3, 128, 128, torch.bfloat16, 31)
    k[0, 5] = 0                       # every head of token 5
    k[1, 64:70, 1] = 0                # the start of the second chunk, one head
    k[0, 100:140, 2] = (k[0, 100:140, 2].float() * 1e-20).to(torch.bfloat16)  # |k| ~ 1e-20
    k[1, 199] = 0                     # the last token of a partial chunk
    _check_chunk(la, oracle_mod, q, k, v, g, beta)


def test_gated_delta_chunk_wait_timeout_is_reported(la, oracle_mod):
    """Failure detection without a GPU fault: with LA_FLAG_TEST_WAIT_TIMEOUT the WY pass
    issues no tile load, so its first wait (bounded, about two seconds) runs out; the
    CTA raises its abort flag, drains (again bounded), frees its tensor memory and
    returns, and la_device_error reports the timeout and the barrier.  One CTA (one
    chunk, one head) keeps the test short.  The next call on the same context is
    correct again."""
    q, k, v, g, beta = _inputs(1, 64, 1, 128, 128, torch.bfloat16, 5)
    dev = torch.device("cuda")
    assert la.device_error(reset=True) == (0, 0)
    la.la_fwd_gated_delta_chunk(q.to(dev), k.to(dev), v.to(dev), g.to(dev), beta.to(dev),
                                flags=la.LA_FLAG_TEST_WAIT_TIMEOUT)
    torch.cuda.synchronize()
    flags, where = la.device_error(reset=True)
    assert flags & 1, (flags, hex(where))          # a wait ran out
    assert where == 0x80000000, hex(where)         # chunk 0, barrier 0: the tile load
    assert la.device_error(reset=True) == (0, 0)
    _check_chunk(la, oracle_mod, q, k, v, g, beta)


def test_gated_delta_chunk_many_heads(la, oracle_mod):
    """More (sequence, head) units than SMs in the sequential pass, and thousands of
    chunk CTAs in the WY pass; only a few slices are compared in full."""
    q, k, v, g, beta = _inputs(4, 700, 40, 128, 128, torch.bfloat16, 77)
    dev = torch.device("cuda")
    out, fs = la.la_fwd_gated_delta_chunk(q.to(dev), k.to(dev), v.to(dev), g.to(dev), beta.to(dev))
    torch.cuda.synchronize()
    pick = [(0, 0), (1, 17), (3, 39)]
    for b, h in pick:
        sl = (slice(b, b + 1), slice(None), slice(h, h + 1))
        ref, fref = oracle_mod.gated_delta(q[sl], k[sl], v[sl], g[sl].double().numpy(), beta[sl].double().numpy())
        assert slice_rel_err(to_np(out[sl]), ref, seq_slices(1, 700)) < TOL[torch.bfloat16]
        assert state_rel_err(to_np(fs[b:b + 1, h:h + 1]), fref) < TOL[torch.bfloat16]


@pytest.mark.parametrize("garbage", [False, True])
def test_gated_delta_chunk_varlen_and_initial_state(la, oracle_mod, garbage):
    from chunkwise_causal_linear_la_b200.workloads import cu_seqlens_from_lengths

    cu = cu_seqlens_from_lengths([130, 0, 1, 64, 65, 300, 7])
    q, k, v, g, beta = _inputs(1, int(cu[-1]) + 5, 2, 128, 128, torch.bfloat16, 6)  # 5 rows after the last sequence
    _check_chunk(la, oracle_mod, q, k, v, g, beta, cu=cu, garbage=garbage)
    init = torch.randn((7, 2, 128, 128)) * 0.1
    _, fs = _check_chunk(la, oracle_mod, q, k, v, g, beta, cu=cu, init=init, garbage=garbage)
    assert torch.equal(fs[1].cpu(), init[1])  # an empty sequence hands its initial state through


def test_gated_delta_chunk_prefill_then_decode(la, oracle_mod):
    """Chunked prefill, then token steps on the state in place (la_fwd_gated_delta),
    equals the oracle over all tokens."""
    B, T, H, d = 2, 333, 2, 128
    q, k, v, g, beta = _inputs(B, T + 2, H, d, d, torch.bfloat16, 13)
    dev = torch.device("cuda")
    qd, kd, vd, gd, bd = (x.to(dev) for x in (q, k, v, g, beta))
    _, state = la.la_fwd_gated_delta_chunk(qd[:, :T].contiguous(), kd[:, :T].contiguous(), vd[:, :T].contiguous(),
                                           gd[:, :T].contiguous(), bd[:, :T].contiguous())
    outs = []
    for t in range(T, T + 2):
        o, _ = la.la_fwd_gated_delta(qd[:, t:t + 1].contiguous(), kd[:, t:t + 1].contiguous(),
                                     vd[:, t:t + 1].contiguous(), gd[:, t:t + 1].contiguous(),
                                     bd[:, t:t + 1].contiguous(), initial_state=state, final_state=state)
        outs.append(o)
    torch.cuda.synchronize()
    ref, fref = oracle_mod.gated_delta(q, k, v, g.double().numpy(), beta.double().numpy())
    for j, o in enumerate(outs):
        assert slice_rel_err(to_np(o), ref[:, T + j:T + j + 1], seq_slices(B, 1)) < TOL[torch.bfloat16]
    assert state_rel_err(to_np(state), fref) < TOL[torch.bfloat16]


def test_gated_delta_chunk_state_in_place_and_fallbacks(la, oracle_mod):
    """initial_state and final_state one buffer (chunked continuation); f32 and
    LA_FLAG_SIMT take the token-by-token kernel through the same entry point."""
    q, k, v, g, beta = _inputs(2, 260, 2, 128, 128, torch.bfloat16, 21)
    dev = torch.device("cuda")
    qd, kd, vd, gd, bd = (x.to(dev) for x in (q, k, v, g, beta))
    _, st = la.la_fwd_gated_delta_chunk(qd[:, :100].contiguous(), kd[:, :100].contiguous(),
                                        vd[:, :100].contiguous(), gd[:, :100].contiguous(), bd[:, :100].contiguous())
    o2, _ = la.la_fwd_gated_delta_chunk(qd[:, 100:].contiguous(), kd[:, 100:].contiguous(), vd[:, 100:].contiguous(),
                                        gd[:, 100:].contiguous(), bd[:, 100:].contiguous(), initial_state=st,
                                        final_state=st)
    torch.cuda.synchronize()
    ref, fref = oracle_mod.gated_delta(q, k, v, g.double().numpy(), beta.double().numpy())
    assert slice_rel_err(to_np(o2), ref[:, 100:], seq_slices(2, 160)) < TOL[torch.bfloat16]
    assert state_rel_err(to_np(st), fref) < TOL[torch.bfloat16]
    assert la.gated_delta_workspace_size(2, 260, 2, 128, 128, 2, False, torch.float32) == 0
    _check_chunk(la, oracle_mod, q.float(), k.float(), v.float(), g, beta)
    _check_chunk(la, oracle_mod, q, k, v, g, beta, flags=1)
    q2, k2, v2, g2, b2 = _inputs(1, 90, 2, 64, 64, torch.bfloat16, 22)
    _check_chunk(la, oracle_mod, q2, k2, v2, g2, b2)


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
@pytest.mark.parametrize("T", [1, 65, 300])
def test_gated_delta_chunk_d64(la, oracle_mod, dk, dv, T):
    """64-wide heads on the tensor-core path: the d = 128 layout with the extra key,
    query and value columns read as TMA zero fill (zero rows and columns of the
    state, outputs and final state clipped to d_v), with and without an initial state."""
    assert la.gated_delta_workspace_size(2, T, 2, dk, dv, 2, False, torch.bfloat16) > 0
    q, k, v, g, beta = _inputs(2, T, 2, dk, dv, torch.bfloat16, 40 + dk + dv + T)
    _check_chunk(la, oracle_mod, q, k, v, g, beta)
    init = torch.randn((2, 2, dk, dv)) * 0.2
    _check_chunk(la, oracle_mod, q, k, v, g, beta, init=init)


def test_gated_delta_chunk_d64_varlen(la, oracle_mod):
    from chunkwise_causal_linear_la_b200.workloads import cu_seqlens_from_lengths

    cu = cu_seqlens_from_lengths([130, 0, 1, 64, 65, 300, 7])
    q, k, v, g, beta = _inputs(1, int(cu[-1]), 2, 64, 64, torch.bfloat16, 61)
    _check_chunk(la, oracle_mod, q, k, v, g, beta, cu=cu, garbage=True)
