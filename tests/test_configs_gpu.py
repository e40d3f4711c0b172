"""GPU parity at the full sizes of the standard workloads, in the launch configuration
bench.py times.

Each test draws the workload's inputs on the GPU (workloads.make_inputs, seed 0),
runs the C-ABI forward once over the whole batch exactly as bench.py does (same
shape, chunk, feature map, normaliser, workspace), and checks sampled
(sequence, head) slices of the outputs and final states against the float64
oracle's token-by-token recurrence over their full length.  The error metric
and the 2e-2 bound for bf16 inputs are parity_util's.

Workloads: the long-sequence sweep B=8, H=16, d=128 at T = 4096, 8192, 16384;
the RetNet-style batch B=32, H=4, T=2048, d=256 with gamma_h = 1 - 2^(-5-h);
the 1M-token sequence B=1, H=4, T=2^20 with gamma_h = 1 - 2^(-8-h) (the
segmented path: state pass, scan, output pass); and the decode step on a
[256, 4, 128, 128] fp32 state (all three decode kernels, every (sequence, head)).
"""
import numpy as np
import pytest
import torch

from parity_util import TOL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def la():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import chunkwise_causal_linear_la_b200 as la

    la.load_library()
    return la


def _err(got, ref):
    d = float(np.max(np.abs(ref)))
    return float(np.max(np.abs(got - ref))) / d if d > 0 else float(np.max(np.abs(got - ref)))


def _full_size(la, oracle_mod, name, slices):
    from chunkwise_causal_linear_la_b200.workloads import WORKLOADS, make_inputs

    w = WORKLOADS[name]
    dev = torch.device("cuda")
    x = make_inputs(w, seed=0, device=dev)
    q, k, v, g = x["q"], x["k"], x["v"], x["gamma"]
    B, T = q.shape[:2]
    ws = la.workspace_size(B, T, w.H, w.d_k, w.d_v, B, False, w.chunk, q.dtype)
    wsbuf = torch.empty(max(ws, 1), dtype=torch.uint8, device=dev)
    out, fs = la.la_fwd_chunk(q, k, v, g, chunk=w.chunk, phi=w.phi, normalize=w.normalize, workspace=wsbuf)[:2]
    torch.cuda.synchronize()
    assert la.device_error(reset=True) == (0, 0)
    worst = 0.0
    for b, h in slices:
        cut = lambda t: t[b:b + 1, :, h:h + 1].cpu()  # noqa: E731
        ref, fref = oracle_mod.recurrent(cut(q), cut(k), cut(v), [float(g[h])], phi=w.phi, normalize=w.normalize)
        e_o = _err(cut(out).double().numpy(), ref)
        e_s = _err(fs[b:b + 1, h:h + 1].double().cpu().numpy(), fref)
        worst = max(worst, e_o, e_s)
        assert e_o < TOL[torch.bfloat16] and e_s < TOL[torch.bfloat16], (name, b, h, e_o, e_s)
    return worst, ws


def test_sweep_T16384_full_size(la, oracle_mod):
    """The headline batch: B=8, H=16, d=128, T=16384, gamma evenly spaced in [0.9, 0.999]."""
    _full_size(la, oracle_mod, "sweep_T16384", [(0, 0), (3, 7), (7, 15)])


@pytest.mark.parametrize("name", ["sweep_T4096", "sweep_T8192"])
def test_sweep_full_size(la, oracle_mod, name):
    _full_size(la, oracle_mod, name, [(0, 0), (7, 15)])


def test_retnet_d256_full_size(la, oracle_mod):
    """B=32, H=4, T=2048, d_k=d_v=256: the 64-wide value slices of the d_k=256 instantiation."""
    _full_size(la, oracle_mod, "retnet_d256", [(0, 0), (17, 2), (31, 3)])


def test_1m_token_sequence(la, oracle_mod):
    """B=1, H=4, T=2^20: one sequence per head, split into segments (state pass, scan, output
    pass); heads 0 and 3 (gamma = 1 - 2^-8 and 1 - 2^-11) over all 1,048,576 tokens."""
    _, ws = _full_size(la, oracle_mod, "long_1m", [(0, 0), (0, 3)])
    assert ws > 0  # the segmented path ran


@pytest.mark.parametrize("kind", ["step", "step_norm", "gated_delta"])
def test_decode_full_size(la, oracle_mod, kind):
    """One decode token on the [256, 4, 128, 128] fp32 state (gamma_h = 1 - 2^(-8-h)),
    every (sequence, head) of the output and of the updated state, fp32 bound 1e-4."""
    from chunkwise_causal_linear_la_b200.workloads import DECODE, make_decode_inputs

    dev = torch.device("cuda")
    d = make_decode_inputs(DECODE["N"], DECODE["H"], DECODE["d_k"], DECODE["d_v"], DECODE["scale"],
                           DECODE["state_std"], DECODE["gamma"], seed=0, device=dev)
    q, k, v, gam, st = d["q"], d["k"], d["v"], d["gamma"], d["state"]
    st0 = st.double().cpu().numpy()
    gnp = gam.double().cpu().numpy()
    if kind == "step":
        out = la.la_step(q, k, v, gam, st, phi="identity")
        ref, fref = oracle_mod.step(q.cpu(), k.cpu(), v.cpu(), gnp, st0, phi="identity")
    elif kind == "step_norm":
        z = torch.ones(st.shape[:3], dtype=torch.float32, device=dev)
        z0 = z.double().cpu().numpy()
        out = la.la_step_norm(q, k, v, gam, st, z, phi="elu1")
        ref, fref, zref = oracle_mod.step_norm(q.cpu(), k.cpu(), v.cpu(), gnp, st0, z0, phi="elu1")
        torch.cuda.synchronize()
        assert _err(z.double().cpu().numpy(), zref) < TOL[torch.float32]
    else:
        N, H = q.shape[:2]
        lg = torch.log(gam).reshape(1, 1, -1).expand(N, 1, -1).contiguous()
        bt = torch.full_like(lg, 0.5)
        o4 = torch.empty_like(v.unsqueeze(1))
        la.la_fwd_gated_delta(q.unsqueeze(1), k.unsqueeze(1), v.unsqueeze(1), lg, bt, initial_state=st, out=o4,
                              final_state=st)
        out = o4[:, 0]
        ref, fref = oracle_mod.gated_delta(q.unsqueeze(1).cpu(), k.unsqueeze(1).cpu(), v.unsqueeze(1).cpu(),
                                           lg.double().cpu().numpy(), bt.double().cpu().numpy(), init=st0)
        ref = ref[:, 0]
    torch.cuda.synchronize()
    got_o, got_s = out.double().cpu().numpy(), st.double().cpu().numpy()
    e_o = max(_err(got_o[n, h], ref[n, h]) for n in range(ref.shape[0]) for h in range(ref.shape[1]))
    e_s = max(_err(got_s[n, h], fref[n, h]) for n in range(ref.shape[0]) for h in range(ref.shape[1]))
    assert e_o < TOL[torch.float32] and e_s < TOL[torch.float32], (kind, e_o, e_s)
