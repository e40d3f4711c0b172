"""la_fwd_chunk_noalloc: the chunked forward for callers that cannot allocate.

Some callers may not allocate device memory while they run (a plugin inside a
framework that owns all device memory, a serving loop where cudaMalloc could
synchronise the device).  For them the library keeps one scratch array of
LA_NOALLOC_SCRATCH_BYTES per device, and la_fwd_chunk_noalloc uses it in place
of the caller's workspace.  This test calls it through the C ABI on a problem
that needs scratch (a long sequence split into segments) and on one that does
not, twice in a row, and compares each result with la_fwd_chunk's and with the
float64 oracle's recurrence.  The file is named so that pytest collects it last.
"""
import ctypes

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


def _noalloc(la, q, k, v, gamma, phi, normalize, chunk=64):
    from chunkwise_causal_linear_la_b200 import binding as b

    lib = b.load_library()
    B, T, H, dk = q.shape
    dv = v.shape[3]
    out = torch.full((B, T, H, dv), float("nan"), dtype=q.dtype, device=q.device)
    fs = torch.full((B, H, dk, dv), float("nan"), dtype=torch.float32, device=q.device)
    tq, tk, tv, to = b.describe(q), b.describe(k), b.describe(v), b.describe(out)
    st = lib.la_fwd_chunk_noalloc(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv), gamma.data_ptr(), None, B,
                                  chunk, b._PHI[phi], int(normalize), ctypes.byref(to), fs.data_ptr(), 0,
                                  torch.cuda.current_stream().cuda_stream)
    assert st == b.LA_OK, lib.la_last_error()
    return out, fs


@pytest.mark.parametrize("phi,normalize", [("identity", False), ("elu1", True)])
@pytest.mark.parametrize("T,H", [(5000, 2), (300, 4)])
def test_noalloc_matches_la_fwd_chunk_twice(la, oracle_mod, phi, normalize, T, H):
    from chunkwise_causal_linear_la_b200.workloads import make_qkv

    dev = torch.device("cuda")
    qc, kc, vc = make_qkv(1, T, H, 128, 128, torch.bfloat16, 128 ** -0.5, seed=T + H)
    q, k, v = (x.to(dev) for x in (qc, kc, vc))
    gamma = torch.linspace(0.95, 1.0, H, device=dev)
    needs_scratch = la.workspace_size(1, T, H, 128, 128, 1, False, 64) > 0
    assert needs_scratch == (T == 5000)
    ref_out, ref_fs = la.la_fwd_chunk(q, k, v, gamma, chunk=64, phi=phi, normalize=normalize)[:2]
    o_ref, f_ref = oracle_mod.recurrent(qc, kc, vc, gamma.double().cpu().numpy(), phi=phi, normalize=normalize)
    for _ in range(2):  # the second call sees the scratch as the first call left it
        out, fs = _noalloc(la, q, k, v, gamma, phi, normalize)
        torch.cuda.synchronize()
        assert slice_rel_err(to_np(out), to_np(ref_out), seq_slices(1, T)) < TOL[torch.bfloat16]
        assert state_rel_err(to_np(fs), to_np(ref_fs)) < TOL[torch.bfloat16]
        assert slice_rel_err(to_np(out), o_ref, seq_slices(1, T)) < TOL[torch.bfloat16]
        assert state_rel_err(to_np(fs), f_ref) < TOL[torch.bfloat16]
    assert la.device_error(reset=True) == (0, 0)
