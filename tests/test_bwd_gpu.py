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


# ---------------------------------------------------------------- per-token decay backward
# la_bwd_chunk_gated against oracle.backward_gated (dq, dk, dv and dg, the gradient of
# the log decays): bf16 on the tensor cores, three passes with the per-token decay
# (the two reverse-time ones taking each position's following decay), then dg from
# the row dot products and a reverse cumulative sum per sequence and head.
def _check_gated(la, oracle_mod, q, k, v, dout, g, cu=None, phi="identity", chunk=64, flags=0):
    dev = torch.device("cuda")
    dq, dk, dv, dg = la.la_bwd_chunk_gated(q.to(dev), k.to(dev), v.to(dev), dout.to(dev), g.to(dev),
                                           cu_seqlens=None if cu is None else cu.to(dev), phi=phi, chunk=chunk,
                                           flags=flags)
    torch.cuda.synchronize()
    assert la.device_error(reset=True) == (0, 0)
    rq, rk, rv, rg = oracle_mod.backward_gated(q, k, v, dout, g.double().numpy(),
                                               cu_seqlens=None if cu is None else cu.numpy(), phi=phi)
    B, T = q.shape[:2]
    sl = seq_slices(B, T, None if cu is None else cu.tolist())
    errs = [slice_rel_err(to_np(x), r, sl) for x, r in ((dq, rq), (dk, rk), (dv, rv))]
    errs.append(_dg_err(to_np(dg), rg, q, k, rq, rk, phi, sl))
    assert all(np.isfinite(to_np(x)).all() for x in (dq, dk, dv, dg))
    assert max(errs) < TOL[q.dtype], errs
    return errs


def _dg_err(dg, rg, q, k, rq, rk, phi, slices):
    """dg_t is a reverse cumulative sum of the row terms phi(q_s) . dphi(q)_s - phi(k_s) . dphi(k)_s,
    and is exactly 0 at a sequence's first token (its decay multiplies the zero initial state), so
    a slice can be all zero (one token), and a single term can cancel to far below its parts.  Per
    (sequence, head) slice the error is taken relative to the larger of max |dg_ref| and the largest
    single-token absolute sum sum_c |phi(q)_c dphi(q)_c| + |phi(k)_c dphi(k)_c| (the scale of a dot
    product's rounding error), rebuilt in float64 from the oracle's dq, dk (dphi(x) = dx / phi'(x),
    phi' > 0).  On sequences longer than a few tokens max |dg_ref| is the larger."""
    qf, kf = q.double().numpy(), k.double().numpy()
    if phi == "elu1":
        fq, fk = np.where(qf > 0, qf + 1, np.exp(np.minimum(qf, 0))), np.where(kf > 0, kf + 1, np.exp(np.minimum(kf, 0)))
        dfq, dfk = rq / np.where(qf > 0, 1.0, np.exp(np.minimum(qf, 0))), rk / np.where(kf > 0, 1.0, np.exp(np.minimum(kf, 0)))
    else:
        fq, fk, dfq, dfk = qf, kf, rq, rk
    term = np.sum(np.abs(fq * dfq), -1) + np.sum(np.abs(fk * dfk), -1)  # [B, T, H]
    worst = 0.0
    for b, s0, e0 in slices:
        if e0 <= s0:
            continue
        for h in range(rg.shape[2]):
            scale = max(np.max(np.abs(rg[b, s0:e0, h])), np.max(term[b, s0:e0, h]))
            worst = max(worst, float(np.max(np.abs(dg[b, s0:e0, h] - rg[b, s0:e0, h])) / scale))
    return worst


def _log_decay(B, T, H, lo, hi, seed):
    from chunkwise_causal_linear_la_b200.workloads import make_log_decay

    gen = torch.Generator()
    gen.manual_seed(seed)
    return make_log_decay(B, T, H, lo, hi, gen)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("T", [1, 65, 300])
@pytest.mark.parametrize("phi", ["identity", "elu1"])
def test_bwd_gated_shapes(la, oracle_mod, d, T, phi):
    q, k, v, dout = _inputs(2, T, 2, d, d, torch.bfloat16, 500 + T + d)
    g = _log_decay(2, T, 2, 0.9, 0.999, 600 + T)
    _check_gated(la, oracle_mod, q, k, v, dout, g, phi=phi)


@pytest.mark.parametrize("lo,hi", [(0.05, 0.5), (0.5, 0.99), (0.999, 1.0)])
def test_bwd_gated_decay_ranges(la, oracle_mod, lo, hi):
    """Strong decays (a 64-token chunk's decay underflows), mild ones and none at all."""
    q, k, v, dout = _inputs(1, 400, 3, 128, 128, torch.bfloat16, 31)
    g = _log_decay(1, 400, 3, lo, hi, 32)
    _check_gated(la, oracle_mod, q, k, v, dout, g, phi="elu1")


def test_bwd_gated_varlen(la, oracle_mod):
    from chunkwise_causal_linear_la_b200.workloads import cu_seqlens_from_lengths

    cu = cu_seqlens_from_lengths([130, 0, 1, 64, 65, 300])
    q, k, v, dout = _inputs(1, int(cu[-1]), 2, 128, 128, torch.bfloat16, 33)
    g = _log_decay(1, int(cu[-1]), 2, 0.8, 0.999, 34)
    _check_gated(la, oracle_mod, q, k, v, dout, g, cu=cu)
    _check_gated(la, oracle_mod, q, k, v, dout, g, cu=cu, phi="elu1")


def test_bwd_gated_long_sequence_dg(la, oracle_mod):
    """A 4000-token sequence: dg sums up to 4000 row terms per head in fp32."""
    q, k, v, dout = _inputs(1, 4000, 2, 128, 128, torch.bfloat16, 35)
    g = _log_decay(1, 4000, 2, 0.95, 0.999, 36)
    _check_gated(la, oracle_mod, q, k, v, dout, g)


def test_bwd_gated_constant_decay_equals_per_head_backward(la):
    """A per-token decay constant in time gives la_bwd_chunk's dq, dk, dv for gamma = exp(g)."""
    dev = torch.device("cuda")
    q, k, v, dout = (x.to(dev) for x in _inputs(2, 300, 2, 128, 128, torch.bfloat16, 37))
    lg = torch.log(torch.tensor([0.97, 0.999]))
    g = lg.reshape(1, 1, 2).expand(2, 300, 2).contiguous().to(dev)
    a = la.la_bwd_chunk_gated(q, k, v, dout, g, phi="elu1")[:3]
    b = la.la_bwd_chunk(q, k, v, dout, torch.exp(lg).to(dev), phi="elu1")
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert slice_rel_err(to_np(x), to_np(y), seq_slices(2, 300)) < TOL[torch.bfloat16]


@pytest.mark.parametrize("T", [1, 37, 200])
@pytest.mark.parametrize("phi", ["identity", "elu1"])
def test_bwd_gated_f32_cuda_cores(la, oracle_mod, T, phi):
    """f32 runs the CUDA-core backward with the per-token decay (fp32 throughout)."""
    q, k, v, dout = _inputs(2, T, 2, 64, 64, torch.float32, 79 + T)
    g = _log_decay(2, T, 2, 0.5, 0.999, 80 + T)
    _check_gated(la, oracle_mod, q, k, v, dout, g, phi=phi)


@pytest.mark.parametrize("chunk", [16, 32, 128])
def test_bwd_gated_other_chunks(la, oracle_mod, chunk):
    q, k, v, dout = _inputs(1, 2 * chunk + 9, 2, 64, 64, torch.bfloat16, 83 + chunk)
    g = _log_decay(1, 2 * chunk + 9, 2, 0.8, 0.999, 84 + chunk)
    _check_gated(la, oracle_mod, q, k, v, dout, g, phi="elu1", chunk=chunk)


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (128, 64)])
def test_bwd_gated_cuda_core_shapes(la, oracle_mod, dk, dv):
    """Shapes off the tensor cores, LA_FLAG_SIMT, and a packed batch in f32."""
    from chunkwise_causal_linear_la_b200.workloads import cu_seqlens_from_lengths

    q, k, v, dout = _inputs(1, 130, 2, dk, dv, torch.bfloat16, dk + 3 * dv)
    g = _log_decay(1, 130, 2, 0.9, 0.99, dk + dv)
    _check_gated(la, oracle_mod, q, k, v, dout, g, flags=la.LA_FLAG_SIMT)
    cu = cu_seqlens_from_lengths([70, 0, 1, 33, 64])
    q, k, v, dout = _inputs(1, int(cu[-1]), 2, dk, dv, torch.float32, 2 * dk + dv)
    g = _log_decay(1, int(cu[-1]), 2, 0.7, 0.999, dk * dv)
    _check_gated(la, oracle_mod, q, k, v, dout, g, cu=cu, phi="elu1")


def test_bwd_gated_simt_matches_tc(la):
    """The CUDA-core and tensor-core backward of the same bf16 problem agree to bf16 rounding."""
    dev = torch.device("cuda")
    q, k, v, dout = (x.to(dev) for x in _inputs(1, 300, 2, 128, 128, torch.bfloat16, 89))
    g = _log_decay(1, 300, 2, 0.9, 0.999, 90).to(dev)
    a = la.la_bwd_chunk_gated(q, k, v, dout, g, phi="elu1")
    b = la.la_bwd_chunk_gated(q, k, v, dout, g, phi="elu1", flags=la.LA_FLAG_SIMT)
    torch.cuda.synchronize()
    for x, y in zip(a[:3], b[:3]):
        assert (x.float() - y.float()).abs().max() <= 2e-2 * y.float().abs().max()


# ---- backward of the normalised forward (la_bwd_chunk_norm) ----

def _norm_bwd_scales(oracle_mod, q, k, v, dout, gamma, cu, phi, slices):
    """Error scales for dq and dk of the normalised backward (from the oracle).

    With u = dout / den and e_t = -(dout_t . o_t) / den_t the denominator's adjoint,
        dphi(q)_t = sum_{j<=t} w_tj (u_t . v_j) phi(k_j) + e_t sum_{j<=t} w_tj phi(k_j) = A + B
    (dphi(k) likewise): two sums that cancel, the more so as the sequence grows,
    since a normalised average does not move with the part of phi(k) common to all
    tokens.  In bf16 each of A and B carries its own rounding (the inter-chunk
    state enters the tensor cores in bf16), so the error is measured against
    max(|dq|, |A|, |B|) per slice.  A one-token sequence cancels inside the dot
    products themselves (o_1 = v_1 whatever q and k: exact dq = dk = 0); there the
    scale is the same sums with every term by its absolute value."""
    q64, k64, v64 = q.double(), k.double(), v.double()
    ones = torch.ones(v.shape[:3] + (1,), dtype=torch.float64)
    den, _ = oracle_mod.recurrent(q64, k64, ones, gamma, cu_seqlens=cu, phi=phi, normalize=False)
    o, _ = oracle_mod.recurrent(q64, k64, v64, gamma, cu_seqlens=cu, phi=phi, normalize=True)
    den, o, do = torch.from_numpy(den), torch.from_numpy(o), dout.double()
    u = do / den
    e = -(do * o).sum(-1, keepdim=True) / den
    aq, ak, _ = oracle_mod.backward(q64, k64, v64, u, gamma, cu_seqlens=cu, phi=phi)
    bq, bk, _ = oracle_mod.backward(q64, k64, ones, e, gamma, cu_seqlens=cu, phi=phi)
    xq, xk, _ = oracle_mod.backward(q64, k64, torch.cat([v64.abs(), ones], -1), torch.cat([u.abs(), e.abs()], -1),
                                    gamma, cu_seqlens=cu, phi=phi)
    scales = []
    for a, b, x in ((aq, bq, xq), (ak, bk, xk)):
        sc = np.maximum(np.abs(a), np.abs(b))
        for bb, s0, e0 in slices:
            if e0 - s0 == 1:
                sc[bb, s0:e0] = np.abs(x[bb, s0:e0])
        scales.append(sc)
    return scales


def _check_norm(la, oracle_mod, q, k, v, dout, gamma, cu=None, phi="elu1", chunk=64, flags=0):
    dev = torch.device("cuda")
    dq, dk, dv = la.la_bwd_chunk_norm(q.to(dev), k.to(dev), v.to(dev), dout.to(dev), gamma.to(dev),
                                      cu_seqlens=None if cu is None else cu.to(dev), phi=phi, chunk=chunk,
                                      flags=flags)
    torch.cuda.synchronize()
    g64, cu_np = gamma.double().numpy(), None if cu is None else cu.numpy()
    refs = oracle_mod.backward_norm(q, k, v, dout, g64, cu_seqlens=cu_np, phi=phi)
    B, T = q.shape[:2]
    sl = seq_slices(B, T, None if cu is None else cu.tolist())
    sq, sk = _norm_bwd_scales(oracle_mod, q, k, v, dout, g64, cu_np, phi, sl)
    assert all(np.isfinite(to_np(x)).all() for x in (dq, dk, dv))
    errs = [slice_rel_err(to_np(x), r, sl, scale=s) for x, r, s in zip((dq, dk, dv), refs, (sq, sk, None))]
    assert max(errs) < TOL[q.dtype], errs


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64), (256, 128)])
@pytest.mark.parametrize("T", [1, 65, 300])
def test_bwd_norm_shapes(la, oracle_mod, dk, dv, T):
    q, k, v, dout = _inputs(2, T, 2, dk, dv, torch.bfloat16, dk + dv + T)
    _check_norm(la, oracle_mod, q, k, v, dout, torch.tensor([1.0, 0.9]))


@pytest.mark.parametrize("gamma", [0.0, 0.3, 0.9, 0.999, 1.0])
def test_bwd_norm_gammas(la, oracle_mod, gamma):
    """gamma <= 0.3 takes the value-decay path of each pass, the others the decayed-key path."""
    q, k, v, dout = _inputs(1, 200, 2, 128, 128, torch.bfloat16, 41)
    _check_norm(la, oracle_mod, q, k, v, dout, torch.tensor([gamma, 1.0]))


def test_bwd_norm_identity_positive_features(la, oracle_mod):
    """The identity feature map with positive q, k (den > 0), as the normalised form asks."""
    q, k, v, dout = _inputs(2, 150, 2, 64, 64, torch.bfloat16, 43)
    _check_norm(la, oracle_mod, q.abs(), k.abs(), v, dout, torch.tensor([1.0, 0.95]), phi="identity")


def test_bwd_norm_varlen(la, oracle_mod):
    from chunkwise_causal_linear_la_b200.workloads import cu_seqlens_from_lengths

    cu = cu_seqlens_from_lengths([130, 0, 1, 64, 65, 300, 17])
    q, k, v, dout = _inputs(1, int(cu[-1]), 3, 128, 128, torch.bfloat16, 47)
    _check_norm(la, oracle_mod, q, k, v, dout, torch.tensor([1.0, 0.97, 0.5]), cu=cu)


def test_bwd_norm_long_sequence(la, oracle_mod):
    q, k, v, dout = _inputs(1, 4096, 2, 128, 128, torch.bfloat16, 53)
    _check_norm(la, oracle_mod, q, k, v, dout, torch.tensor([1.0, 0.999]))


def test_bwd_norm_caller_workspace_reused(la, oracle_mod):
    """A caller-owned workspace left dirty by an earlier call gives the same gradients."""
    dev = torch.device("cuda")
    q, k, v, dout = _inputs(1, 257, 2, 128, 128, torch.bfloat16, 59)
    gamma = torch.tensor([1.0, 0.9])
    need = la.bwd_norm_workspace_size(1, 257, 2, 128, 128)
    ws = torch.full((need,), 0x7F, dtype=torch.uint8, device=dev)
    args = [x.to(dev) for x in (q, k, v, dout, gamma)]
    a = la.la_bwd_chunk_norm(*args, workspace=ws)
    b = la.la_bwd_chunk_norm(*args, workspace=ws)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    refs = oracle_mod.backward_norm(q, k, v, dout, gamma.double().numpy())
    sl = seq_slices(1, 257)
    scales = _norm_bwd_scales(oracle_mod, q, k, v, dout, gamma.double().numpy(), None, "elu1", sl) + [None]
    assert max(slice_rel_err(to_np(x), r, sl, scale=sc) for x, r, sc in zip(a, refs, scales)) < TOL[torch.bfloat16]


@pytest.mark.parametrize("T", [1, 100, 256])
def test_bwd_norm_f32_cuda_cores(la, oracle_mod, T):
    """f32 (the tiny workload's dtype: d = 64, elu + 1, normaliser, gamma = 1) runs on
    the CUDA-core kernels in fp32."""
    q, k, v, dout = _inputs(1, T, 2, 64, 64, torch.float32, 67 + T)
    _check_norm(la, oracle_mod, q, k, v, dout, torch.tensor([1.0, 0.9]))


@pytest.mark.parametrize("chunk", [16, 32, 128])
def test_bwd_norm_other_chunks(la, oracle_mod, chunk):
    """bf16 with a chunk other than 64 takes the CUDA-core route."""
    q, k, v, dout = _inputs(2, 3 * chunk + 5, 2, 64, 64, torch.bfloat16, 71 + chunk)
    _check_norm(la, oracle_mod, q, k, v, dout, torch.tensor([1.0, 0.95]), chunk=chunk)


@pytest.mark.parametrize("dk,dv", [(32, 16), (64, 32), (128, 64)])
def test_bwd_norm_cuda_core_shapes(la, oracle_mod, dk, dv):
    """Small heads (no tensor-core shape) and LA_FLAG_SIMT; packed batch with f32."""
    q, k, v, dout = _inputs(1, 150, 2, dk, dv, torch.bfloat16, dk + dv)
    _check_norm(la, oracle_mod, q, k, v, dout, torch.tensor([1.0, 0.8]), flags=la.LA_FLAG_SIMT)
    from chunkwise_causal_linear_la_b200.workloads import cu_seqlens_from_lengths

    cu = cu_seqlens_from_lengths([70, 0, 1, 64, 15])
    q, k, v, dout = _inputs(1, int(cu[-1]), 2, dk, dv, torch.float32, dk * dv)
    _check_norm(la, oracle_mod, q, k, v, dout, torch.tensor([1.0, 0.9]), cu=cu)


def test_bwd_norm_unsupported(la):
    dev = torch.device("cuda")
    assert la.bwd_norm_workspace_size(1, 64, 2, 128, 256) == -1
    assert la.bwd_norm_workspace_size(1, 64, 2, 128, 128, chunk=48) == -1
    q, k, v, dout = _inputs(1, 64, 2, 128, 256, torch.bfloat16, 61)
    with pytest.raises(la.LaError) as e:
        la.la_bwd_chunk_norm(q.to(dev), k.to(dev), v.to(dev), dout.to(dev), torch.ones(2, device=dev))
    assert e.value.status == la.binding.LA_ERR_UNSUPPORTED
    assert la.device_error(reset=True) == (0, 0)


# ---- backward of the normalised per-token-decay forward (la_bwd_chunk_gated_norm) ----

def _gated_norm_scales(oracle_mod, q, k, v, dout, g, cu, phi, slices):
    """Error scales for dq, dk and dg (from the oracle), as _norm_bwd_scales with the
    per-token decay: dq and dk against max(|dq|, |A|, |B|) (numerator and denominator
    terms; one-token sequences: the same sums by absolute value); dg, a reverse
    cumulative sum of the row terms phi(q_s) . dphi(q)_s - phi(k_s) . dphi(k)_s whose
    numerator and denominator parts cancel (the q part exactly: a normalised row
    does not move with the scale of phi(q_s)), against the larger of max|dg| and the
    largest single-token sum of those parts' sizes |phi(x) . A_x| + |phi(x) . B_x|."""
    q64, k64, v64 = q.double(), k.double(), v.double()
    ones = torch.ones(v.shape[:3] + (1,), dtype=torch.float64)
    den, _, _ = oracle_mod.recurrent_gated(q64, k64, ones, g, cu_seqlens=cu, phi=phi, normalize=False)
    o, _, _ = oracle_mod.recurrent_gated(q64, k64, v64, g, cu_seqlens=cu, phi=phi, normalize=True)
    den, o, do = torch.from_numpy(den), torch.from_numpy(o), dout.double()
    u = do / den
    e = -(do * o).sum(-1, keepdim=True) / den
    aq, ak, _, _ = oracle_mod.backward_gated(q64, k64, v64, u, g, cu_seqlens=cu, phi=phi)
    bq, bk, _, _ = oracle_mod.backward_gated(q64, k64, ones, e, g, cu_seqlens=cu, phi=phi)
    xq, xk, _, _ = oracle_mod.backward_gated(q64, k64, torch.cat([v64.abs(), ones], -1),
                                             torch.cat([u.abs(), e.abs()], -1), g, cu_seqlens=cu, phi=phi)
    sq, sk = np.maximum(np.abs(aq), np.abs(bq)), np.maximum(np.abs(ak), np.abs(bk))
    for bb, s0, e0 in slices:
        if e0 - s0 == 1:
            sq[bb, s0:e0], sk[bb, s0:e0] = np.abs(xq[bb, s0:e0]), np.abs(xk[bb, s0:e0])
    qf, kf = q64.numpy(), k64.numpy()
    if phi == "elu1":
        fq, fk = np.where(qf > 0, qf + 1, np.exp(np.minimum(qf, 0))), np.where(kf > 0, kf + 1, np.exp(np.minimum(kf, 0)))
        pq, pk = np.where(qf > 0, 1.0, np.exp(np.minimum(qf, 0))), np.where(kf > 0, 1.0, np.exp(np.minimum(kf, 0)))
    else:
        fq, fk, pq, pk = qf, kf, np.ones_like(qf), np.ones_like(kf)
    row = (np.abs(np.sum(fq * aq / pq, -1)) + np.abs(np.sum(fq * bq / pq, -1)) +
           np.abs(np.sum(fk * ak / pk, -1)) + np.abs(np.sum(fk * bk / pk, -1)))  # [B, T, H]
    return sq, sk, row


def _check_gated_norm(la, oracle_mod, q, k, v, dout, g, cu=None, phi="elu1", chunk=64, flags=0):
    dev = torch.device("cuda")
    dq, dk, dv, dg = la.la_bwd_chunk_gated_norm(q.to(dev), k.to(dev), v.to(dev), dout.to(dev), g.to(dev),
                                                cu_seqlens=None if cu is None else cu.to(dev), phi=phi, chunk=chunk,
                                                flags=flags)
    torch.cuda.synchronize()
    assert la.device_error(reset=True) == (0, 0)
    g64, cu_np = g.double().numpy(), None if cu is None else cu.numpy()
    refs = oracle_mod.backward_gated_norm(q, k, v, dout, g64, cu_seqlens=cu_np, phi=phi)
    B, T = q.shape[:2]
    sl = seq_slices(B, T, None if cu is None else cu.tolist())
    sq, sk, sg = _gated_norm_scales(oracle_mod, q, k, v, dout, g64, cu_np, phi, sl)
    assert all(np.isfinite(to_np(x)).all() for x in (dq, dk, dv, dg))
    errs = [slice_rel_err(to_np(x), r, sl, scale=s) for x, r, s in zip((dq, dk, dv), refs[:3], (sq, sk, None))]
    errs.append(slice_rel_err(to_np(dg)[..., None], refs[3][..., None], sl, scale=sg[..., None]))
    assert max(errs) < TOL[q.dtype], errs
    return errs


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T", [1, 65, 300])
def test_bwd_gated_norm_shapes(la, oracle_mod, d, T):
    q, k, v, dout = _inputs(2, T, 2, d, d, torch.bfloat16, 3 * d + T)
    g = _log_decay(2, T, 2, 0.8, 0.999, 5 * d + T)
    _check_gated_norm(la, oracle_mod, q, k, v, dout, g)


def test_bwd_gated_norm_varlen_and_identity(la, oracle_mod):
    from chunkwise_causal_linear_la_b200.workloads import cu_seqlens_from_lengths

    cu = cu_seqlens_from_lengths([130, 0, 1, 64, 65, 17])
    q, k, v, dout = _inputs(1, int(cu[-1]), 2, 128, 128, torch.bfloat16, 61)
    g = _log_decay(1, int(cu[-1]), 2, 0.7, 0.999, 62)
    _check_gated_norm(la, oracle_mod, q, k, v, dout, g, cu=cu)
    q, k, v, dout = _inputs(1, 150, 2, 64, 64, torch.bfloat16, 63)
    _check_gated_norm(la, oracle_mod, q.abs(), k.abs(), v, dout, _log_decay(1, 150, 2, 0.9, 0.99, 64), phi="identity")


@pytest.mark.parametrize("T", [1, 100])
def test_bwd_gated_norm_f32_and_simt(la, oracle_mod, T):
    """f32 (fp32 CUDA-core kernels, 1e-4) and bf16 with LA_FLAG_SIMT or another chunk."""
    q, k, v, dout = _inputs(2, T, 2, 64, 64, torch.float32, 65 + T)
    g = _log_decay(2, T, 2, 0.6, 0.999, 66 + T)
    _check_gated_norm(la, oracle_mod, q, k, v, dout, g)
    q, k, v, dout = _inputs(1, T + 37, 2, 64, 32, torch.bfloat16, 67 + T)
    g = _log_decay(1, T + 37, 2, 0.8, 0.999, 68 + T)
    _check_gated_norm(la, oracle_mod, q, k, v, dout, g, flags=la.LA_FLAG_SIMT)
    _check_gated_norm(la, oracle_mod, q, k, v, dout, g, chunk=32)


def test_bwd_empty_inputs(la):
    """No token to process: every backward returns without error (T = 0, B = 0, and a
    packed batch of empty sequences), and with a per-token decay dg stays zero."""
    from chunkwise_causal_linear_la_b200.workloads import cu_seqlens_from_lengths

    dev = torch.device("cuda")
    for B, T in ((1, 0), (0, 5)):
        q, k, v, dout = (torch.zeros((B, T, 2, 64), dtype=torch.bfloat16, device=dev) for _ in range(4))
        g = torch.zeros((B, T, 2), device=dev)
        la.la_bwd_chunk(q, k, v, dout, torch.ones(2, device=dev))
        la.la_bwd_chunk_norm(q, k, v, dout, torch.ones(2, device=dev))
        la.la_bwd_chunk_gated(q, k, v, dout, g)
        la.la_bwd_chunk_gated_norm(q, k, v, dout, g)
    cu = cu_seqlens_from_lengths([0, 0, 0]).to(dev)
    q, k, v, dout = (torch.randn((1, 4, 2, 64), device=dev).to(torch.bfloat16) for _ in range(4))
    g = torch.zeros((1, 4, 2), device=dev)
    dq, dk, dv, dg = la.la_bwd_chunk_gated_norm(q, k, v, dout, g, cu_seqlens=cu)
    dq2, dk2, dv2 = la.la_bwd_chunk_norm(q, k, v, dout, torch.ones(2, device=dev), cu_seqlens=cu)
    torch.cuda.synchronize()
    assert la.device_error(reset=True) == (0, 0)
