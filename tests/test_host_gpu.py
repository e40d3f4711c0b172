"""la_fwd_chunk_host: the forward on host buffers (copies in, forward, copies out on
one stream) against la_fwd_chunk on device buffers and against the float64 oracle,
for a dense and a packed batch, with page-locked and with pageable host memory."""
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


@pytest.mark.parametrize("pinned", [True, False])
@pytest.mark.parametrize("packed", [False, True])
def test_host_buffers_match_device_call_and_oracle(la, oracle_mod, pinned, packed):
    from chunkwise_causal_linear_la_b200.workloads import cu_seqlens_from_lengths, make_qkv

    cu = cu_seqlens_from_lengths([300, 0, 65, 1, 200]) if packed else None
    B, T = (1, int(cu[-1])) if packed else (2, 333)
    H = 3
    q, k, v = make_qkv(B, T, H, 128, 128, torch.bfloat16, 128 ** -0.5, seed=31)
    gamma = torch.tensor([0.9, 0.99, 1.0])
    if pinned:
        q, k, v, gamma = (t.pin_memory() for t in (q, k, v, gamma))
    out, fs = la.la_fwd_chunk_host(q, k, v, gamma, cu_seqlens=cu, phi="elu1")
    torch.cuda.synchronize()
    dev = torch.device("cuda")
    ref_out, ref_fs = la.la_fwd_chunk(q.to(dev), k.to(dev), v.to(dev), gamma.to(dev),
                                      cu_seqlens=None if cu is None else cu.to(dev), phi="elu1")
    torch.cuda.synchronize()
    sl = seq_slices(B, T, None if cu is None else cu.tolist())
    assert torch.equal(out, ref_out.cpu()) and torch.equal(fs, ref_fs.cpu())  # the same kernels on the same data
    o_ref, f_ref = oracle_mod.recurrent(q, k, v, gamma.double().numpy(), cu_seqlens=None if cu is None else cu.numpy(),
                                        phi="elu1")
    assert slice_rel_err(to_np(out), o_ref, sl) < TOL[torch.bfloat16]
    assert state_rel_err(to_np(fs), f_ref) < TOL[torch.bfloat16]
