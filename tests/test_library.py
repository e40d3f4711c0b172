"""CPU checks of the C-ABI library: it loads, exports every symbol the public
header declares, and its host-side logic (validation, workspace sizing, status
strings) behaves as documented.  No compute call is made here."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from chunkwise_causal_linear_la_b200 import build, binding

    build.build()
    return binding.load_library()


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"^LA_API\s+[\w\s\*]+?\b(la_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_api():
    names = declared_functions()
    for n in ("la_fwd_chunk", "la_step", "la_fwd_chunk_workspace_size", "la_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    from chunkwise_causal_linear_la_b200 import binding

    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in binding.EXPORTS, name


def test_library_exports_nothing_else():
    import subprocess

    from chunkwise_causal_linear_la_b200 import binding

    out = subprocess.check_output(["nm", "-D", "--defined-only", binding.LIB_PATH]).decode()
    exported = sorted(l.split()[-1] for l in out.splitlines() if l.split()[1] == "T")
    assert exported == declared_functions()


def test_status_strings_and_version(lib):
    for s in range(5):
        assert lib.la_status_string(s).startswith(b"LA_")
    assert lib.la_status_string(99) == b"unknown la_status"
    assert lib.la_version() >= 10000


def test_workspace_size_host_logic(lib):
    ws = lib.la_fwd_chunk_workspace_size
    bad = ctypes.c_size_t(-1).value
    assert ws(8, 128, 16, 128, 128, 8, 0, 63, 1, 0) == bad  # chunk not supported
    assert ws(8, 128, 16, 96, 128, 8, 0, 64, 1, 0) == bad  # head dim not supported
    assert ws(8, 128, 0, 128, 128, 8, 0, 64, 1, 0) == bad  # H = 0
    assert ws(1, 256, 2, 64, 64, 1, 0, 64, 0, 0) == 0  # f32 runs on CUDA cores, no workspace
    assert ws(8, 128, 16, 128, 128, 8, 0, 64, 1, 1) == 0  # forced SIMT


def test_gated_delta_workspace_size(lib):
    """The chunked gated delta rule keeps W and T diag(beta) V, bf16 [B, T, H, 128]
    each, the 64 prefix sums b_i and key norms 1/|k_i| of every (chunk slot, head) in fp32, and
    n_seqs + 1 chunk offsets for a packed batch, whose slot count is bounded by
    ceil(T / 64) + n_seqs (each region 256-byte aligned); head dims of 64 use the
    same 128-wide layout; shapes that take the token-by-token kernel need nothing."""
    ws = lib.la_fwd_gated_delta_workspace_size
    bad = ctypes.c_size_t(-1).value
    wu = 8 * 4096 * 16 * 128 * 2
    assert ws(8, 4096, 16, 128, 128, 8, 0, 1, 0) == 2 * wu + (8 * 64) * 16 * 512
    assert ws(1, 1000, 3, 128, 128, 5, 1, 1, 0) == 2 * 768000 + (16 + 5) * 3 * 512 + 256
    assert ws(1, 3, 1, 128, 128, 100, 1, 1, 0) == 2 * 768 + 101 * 512 + 512
    assert ws(8, 4096, 16, 64, 64, 8, 0, 1, 0) == 2 * wu + (8 * 64) * 16 * 512  # d = 64: the 128 layout
    assert ws(8, 4096, 16, 256, 256, 8, 0, 1, 0) == 0    # d = 256: token-by-token kernel
    assert ws(8, 4096, 16, 128, 128, 8, 0, 0, 0) == 0    # f32
    assert ws(8, 4096, 16, 128, 128, 8, 0, 1, 1) == 0    # LA_FLAG_SIMT
    assert ws(8, 4096, 16, 96, 128, 8, 0, 1, 0) == bad   # head dim
    assert ws(8, 4096, 0, 128, 128, 8, 0, 1, 0) == bad   # H = 0
    assert ws(8, 4096, 16, 128, 128, 8, 0, 2, 0) == bad  # dtype
    assert ws(8, 4096, 16, 128, 128, 8, 0, 1, 4) == bad  # flags
    assert ws(8, 4096, 16, 128, 128, 8, 0, 1, 0x100) == 2 * wu + (8 * 64) * 16 * 512  # the test flag


def test_workspace_size_segment_plan(lib):
    """Segment states (S^T, the normaliser sum and the log decay of a
    data-dependent decay) are kept for all but the last segment of each unit,
    one unit per (sequence, head, value slice); value slices are 128 columns
    wide at d_k <= 128 and 64 at d_k = 256."""
    ws = lib.la_fwd_chunk_workspace_size
    # d_k = 128: 2 units, 79 chunks -> G = min(148 // 2, 79 // 16) = 4 segments of 20 chunks
    assert ws(1, 5000, 2, 128, 128, 1, 0, 64, 1, 0) == 2 * 3 * (128 * 128 + 128 + 1) * 4
    # d_k = 256, d_v = 256: 8 units -> G = min(148 // 8, 4) = 4
    assert ws(1, 5000, 2, 256, 256, 1, 0, 64, 1, 0) == 8 * 3 * (256 * 64 + 256 + 1) * 4
    # enough units to fill the GPU (RetNet-style batch: 32 x 4 heads x 4 slices): none
    assert ws(32, 2048, 4, 256, 256, 32, 0, 64, 1, 0) == 0
    # packed batches are not segmented; nor are shapes the tensor cores do not run
    assert ws(1, 5000, 2, 128, 128, 1, 1, 64, 1, 0) == 0
    # packed batches of 2 .. 4096 sequences keep their longest-first order (int32 each, 256-byte blocks)
    assert ws(1, 77431, 8, 128, 128, 64, 1, 64, 1, 0) == 256
    assert ws(1, 77431, 8, 128, 128, 65, 1, 64, 1, 0) == 512
    assert ws(1, 77431, 8, 128, 128, 5000, 1, 64, 1, 0) == 0
    # d_k = d_v = 64 runs in the d_k = 128 layout (zero-padded keys, a 128-wide value slice)
    assert ws(1, 5000, 2, 64, 64, 1, 0, 64, 1, 0) == 2 * 3 * (128 * 128 + 128 + 1) * 4
    assert ws(1, 5000, 2, 32, 32, 1, 0, 64, 1, 0) == 0  # CUDA-core kernel: no workspace


def _t(B=1, T=4, H=2, D=64, dtype=1, ptr=0x1000):
    from chunkwise_causal_linear_la_b200.binding import LaTensor

    return LaTensor(ptr, dtype, B, T, H, D, T * H * D, H * D, D)


def _call(lib, q=None, k=None, v=None, out=None, gamma=0x2000, cu=None, n=1, chunk=64, phi=0, flags=0):
    q = q or _t()
    k = k or _t()
    v = v or _t()
    out = out or _t()
    return lib.la_fwd_chunk(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), gamma, cu, n, chunk, phi, 0,
                            ctypes.byref(out), None, flags, None, 0, None)


def test_validation_rejects_bad_arguments_before_any_device_call(lib):
    from chunkwise_causal_linear_la_b200 import binding as b

    assert _call(lib, gamma=None) == b.LA_ERR_INVALID_ARG
    assert _call(lib, k=_t(dtype=0)) == b.LA_ERR_INVALID_ARG  # dtype mismatch
    assert _call(lib, v=_t(T=5)) == b.LA_ERR_INVALID_ARG  # shape mismatch
    assert _call(lib, q=_t(ptr=0x1004)) == b.LA_ERR_INVALID_ARG  # misaligned
    assert _call(lib, phi=7) == b.LA_ERR_INVALID_ARG
    assert _call(lib, flags=4) == b.LA_ERR_INVALID_ARG
    assert _call(lib, n=2) == b.LA_ERR_INVALID_ARG  # n_seqs != B without cu_seqlens
    assert _call(lib, q=_t(B=2), k=_t(B=2), v=_t(B=2), out=_t(B=2), cu=0x3000, n=1) == b.LA_ERR_INVALID_ARG
    assert _call(lib, chunk=48) == b.LA_ERR_UNSUPPORTED
    assert _call(lib, q=_t(D=96), k=_t(D=96)) == b.LA_ERR_UNSUPPORTED
    assert b"chunk" in lib.la_last_error() or b"head dims" in lib.la_last_error()
    null = _t(ptr=0)
    assert _call(lib, q=null) == b.LA_ERR_INVALID_ARG


def test_gated_delta_chunk_arguments_validated_on_host(lib):
    """la_fwd_gated_delta_chunk rejects bad arguments, unknown flags and a short or
    misaligned workspace before any device call (d = 128 bf16 takes the tensor cores)."""
    from chunkwise_causal_linear_la_b200 import binding as b

    q, k, v, o = _t(D=128), _t(D=128), _t(D=128), _t(D=128)
    need = lib.la_fwd_gated_delta_workspace_size(1, 4, 2, 128, 128, 1, 0, 1, 0)
    assert need > 0

    def call(g=0x2000, beta=0x3000, n=1, flags=0, ws=0x100000, ws_bytes=None, qq=None):
        return lib.la_fwd_gated_delta_chunk(ctypes.byref(qq or q), ctypes.byref(k), ctypes.byref(v), g, beta, None,
                                            n, None, ctypes.byref(o), None, flags, ws,
                                            need if ws_bytes is None else ws_bytes, None)
    assert call(g=None) == b.LA_ERR_INVALID_ARG and b"beta" in lib.la_last_error()
    assert call(beta=0x3002) == b.LA_ERR_INVALID_ARG and b"aligned" in lib.la_last_error()
    assert call(n=2) == b.LA_ERR_INVALID_ARG
    assert call(flags=2) == b.LA_ERR_INVALID_ARG and b"flags" in lib.la_last_error()
    assert call(flags=0x200) == b.LA_ERR_INVALID_ARG and b"flags" in lib.la_last_error()
    assert call(flags=b.LA_FLAG_TEST_WAIT_TIMEOUT, ws_bytes=need - 1) == b.LA_ERR_WORKSPACE  # flag accepted
    assert call(ws_bytes=need - 1) == b.LA_ERR_WORKSPACE
    assert call(ws=None) == b.LA_ERR_WORKSPACE
    assert call(ws=0x100010) == b.LA_ERR_INVALID_ARG and b"256" in lib.la_last_error()
    assert call(qq=_t(D=96)) == b.LA_ERR_INVALID_ARG  # q and k head dims disagree


def test_normaliser_state_arguments_validated_on_host(lib):
    """la_fwd_chunk_z needs normalize for final_z and a 16-byte aligned final_z;
    la_step_norm needs a z pointer.  All rejected before any device call."""
    from chunkwise_causal_linear_la_b200 import binding as b

    q, k, v, o = _t(), _t(), _t(), _t()
    def fz(normalize, final_z):
        return lib.la_fwd_chunk_z(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), 0x2000, None, 1, 64, 1,
                                  normalize, ctypes.byref(o), None, final_z, 0, None, 0, None)
    assert fz(0, 0x4000) == b.LA_ERR_INVALID_ARG and b"normalize" in lib.la_last_error()
    assert fz(1, 0x4004) == b.LA_ERR_INVALID_ARG and b"aligned" in lib.la_last_error()
    one = lambda D: _t(T=1, D=D)  # noqa: E731
    q1, k1, v1, o1 = one(64), one(64), one(64), one(64)
    st = lib.la_step_norm(ctypes.byref(q1), ctypes.byref(k1), ctypes.byref(v1), 0x2000, 0x5000, None,
                          ctypes.byref(o1), 1, None)
    assert st == b.LA_ERR_INVALID_ARG and b"z" in lib.la_last_error()
    st = lib.la_step_norm(ctypes.byref(q1), ctypes.byref(k1), ctypes.byref(v1), 0x2000, 0x5000, 0x6008,
                          ctypes.byref(o1), 1, None)
    assert st == b.LA_ERR_INVALID_ARG and b"aligned" in lib.la_last_error()


def test_path_query_host_logic(lib):
    """la_fwd_chunk_path: -1 where la_fwd_chunk rejects the arguments, the CUDA-core
    kernel for f32, LA_FLAG_SIMT and bf16 shapes the tensor cores do not take (the
    tensor-core answer itself needs a GPU driver; tests/test_tc_d64_gpu.py checks it)."""
    from chunkwise_causal_linear_la_b200 import binding as b

    path = lib.la_fwd_chunk_path
    assert path(96, 128, 100, 4, 64, b.LA_BF16, 0) == -1  # head dim
    assert path(128, 128, 100, 4, 48, b.LA_BF16, 0) == -1  # chunk
    assert path(128, 128, 100, 0, 64, b.LA_BF16, 0) == -1  # heads
    assert path(128, 128, -1, 4, 64, b.LA_BF16, 0) == -1  # length
    assert path(128, 128, 100, 4, 64, 7, 0) == -1  # dtype
    assert path(128, 128, 100, 4, 64, b.LA_BF16, 4) == -1  # flags
    assert path(128, 128, 100, 4, 64, b.LA_F32, 0) == 2
    assert path(128, 128, 100, 4, 64, b.LA_BF16, b.LA_FLAG_SIMT) == 2
    for chunk in (16, 32, 128):
        assert path(128, 128, 100, 4, chunk, b.LA_BF16, 0) == 2
    assert path(32, 32, 100, 4, 64, b.LA_BF16, 0) == 2
    assert path(128, 128, 100, 4, 64, b.LA_BF16, 0) in (1, 2)


def test_host_arena_size_and_validation(lib):
    """la_fwd_chunk_host_arena_size lays out q, k, v, out, the final state, gamma,
    cu_seqlens and the workspace at 256-byte boundaries; la_fwd_chunk_host rejects
    non-contiguous host tensors and a missing arena before touching a device."""
    from chunkwise_causal_linear_la_b200 import binding as b

    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    B, T, H, dk, dv = 2, 100, 3, 128, 64
    tok = B * T * H
    want = up(tok * dk * 2) * 2 + up(tok * dv * 2) * 2 + up(B * H * dk * dv * 4) + up(H * 4)
    assert lib.la_fwd_chunk_host_arena_size(B, T, H, dk, dv, B, 0, 64, b.LA_BF16, 0, 1) == want
    assert lib.la_fwd_chunk_host_arena_size(B, T, H, dk, dv, B, 0, 64, b.LA_BF16, 0, 0) == want - up(B * H * dk * dv * 4)
    # a packed batch adds cu_seqlens (and its longest-first order in the workspace)
    packed = lib.la_fwd_chunk_host_arena_size(1, 500, H, dk, dv, 5, 1, 64, b.LA_BF16, 0, 0)
    assert packed == (up(500 * H * dk * 2) * 2 + up(500 * H * dv * 2) * 2 + up(H * 4) + up(6 * 4)
                      + lib.la_fwd_chunk_workspace_size(1, 500, H, dk, dv, 5, 1, 64, b.LA_BF16, 0))
    assert lib.la_fwd_chunk_host_arena_size(B, T, H, 96, dv, B, 0, 64, b.LA_BF16, 0, 1) == ctypes.c_size_t(-1).value
    t = _t(B=1, T=4, H=2, D=64)
    strided = b.LaTensor(0x1000, 1, 1, 4, 2, 64, 4 * 2 * 128, 2 * 128, 128)
    call = lambda q, arena, nbytes: lib.la_fwd_chunk_host(  # noqa: E731
        ctypes.byref(q), ctypes.byref(t), ctypes.byref(t), 0x2000, None, 1, 64, 0, 0, ctypes.byref(t), None, 0,
        arena, nbytes, None)
    assert call(strided, 0x4000, 1 << 20) == b.LA_ERR_INVALID_ARG
    assert call(t, None, 0) == b.LA_ERR_WORKSPACE
    assert call(t, 0x4010, 1 << 20) == b.LA_ERR_INVALID_ARG  # arena not 256-byte aligned


def test_bwd_norm_workspace_and_validation_on_host(lib):
    """la_bwd_chunk_norm_workspace_size, each region at a 256-byte boundary: on the
    tensor-core route (bf16, chunk 64, d_v in {64, 128}) the augmented rows ([v, 1, 1]
    rounded up to 2 d_v columns) twice, the forward's o (bf16) and den (fp32), and
    phi(k); on the CUDA-core route (f32, other chunks, LA_FLAG_SIMT, d_v of 16 or 32)
    the augmented rows three times (v', u', dv'); -1 for what la_bwd_chunk_norm
    rejects.  Bad arguments and a short or misaligned workspace are rejected before
    any device call."""
    from chunkwise_causal_linear_la_b200 import binding as b

    ws = lib.la_bwd_chunk_norm_workspace_size
    bad = ctypes.c_size_t(-1).value
    rows = 3 * 100 * 5
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731

    def tc(dk, dv):
        return 2 * up(rows * 2 * dv * 2) + up(rows * dv * 2) + up(rows * 4) + up(rows * dk * 2)

    def cc(dv, es):
        return 3 * up(rows * 2 * dv * es)
    assert ws(3, 100, 5, 128, 128, 64, 1, 0) == tc(128, 128)
    assert ws(3, 100, 5, 64, 64, 64, 1, 0) == tc(64, 64)
    assert ws(3, 100, 5, 256, 128, 64, 1, 0) == tc(256, 128)
    assert ws(3, 100, 5, 128, 64, 64, 1, 0) == tc(128, 64)
    assert ws(3, 100, 5, 128, 128, 32, 1, 0) == cc(128, 2)  # chunk 32: CUDA cores
    assert ws(3, 100, 5, 128, 128, 64, 1, 1) == cc(128, 2)  # LA_FLAG_SIMT
    assert ws(3, 100, 5, 64, 64, 64, 0, 0) == cc(64, 4)  # f32
    assert ws(3, 100, 5, 32, 32, 16, 0, 0) == cc(32, 4)
    assert ws(3, 100, 5, 64, 16, 64, 1, 0) == cc(16, 2)  # d_v = 16: widened to 32, no tensor-core shape
    assert ws(3, 100, 5, 128, 256, 64, 1, 0) == bad  # d_v + 2 does not fit 256 columns
    assert ws(3, 100, 5, 128, 128, 48, 1, 0) == bad  # chunk
    assert ws(3, 100, 5, 96, 128, 64, 1, 0) == bad  # d_k
    assert ws(3, 100, 5, 128, 128, 64, 1, 4) == bad  # unknown flag
    assert ws(3, 100, 0, 128, 128, 64, 1, 0) == bad  # H = 0

    need = ws(1, 4, 2, 128, 128, 64, 1, 0)
    q, k, v, do, dq, dk, dv = (_t(D=128) for _ in range(7))

    def call(gamma=0x2000, phi=1, ws_ptr=0x100000, ws_bytes=None, qq=None, vv=None, flags=0, chunk=64):
        return lib.la_bwd_chunk_norm(ctypes.byref(qq or q), ctypes.byref(k), ctypes.byref(vv or v), ctypes.byref(do),
                                     gamma, None, 1, chunk, phi, ctypes.byref(dq), ctypes.byref(dk), ctypes.byref(dv),
                                     flags, ws_ptr, need if ws_bytes is None else ws_bytes, None)
    assert call(gamma=None) == b.LA_ERR_INVALID_ARG and b"gamma" in lib.la_last_error()
    assert call(phi=5) == b.LA_ERR_INVALID_ARG
    assert call(flags=8) == b.LA_ERR_INVALID_ARG and b"flags" in lib.la_last_error()
    assert call(qq=_t(D=64)) == b.LA_ERR_INVALID_ARG  # q and k disagree
    assert call(qq=_t(D=128, ptr=0x1008)) == b.LA_ERR_INVALID_ARG  # misaligned
    assert call(ws_bytes=need - 1) == b.LA_ERR_WORKSPACE
    assert call(ws_ptr=None) == b.LA_ERR_WORKSPACE
    assert call(ws_ptr=0x100010) == b.LA_ERR_INVALID_ARG and b"256" in lib.la_last_error()
    assert call(chunk=48) == b.LA_ERR_UNSUPPORTED and b"chunk" in lib.la_last_error()
    assert call(flags=1, ws_bytes=ws(1, 4, 2, 128, 128, 64, 1, 1) - 1) == b.LA_ERR_WORKSPACE  # CUDA-core route
    big = [_t(D=128), _t(D=128), _t(D=256), _t(D=256), _t(D=128), _t(D=128), _t(D=256)]
    st = lib.la_bwd_chunk_norm(*[ctypes.byref(x) for x in big[:4]], 0x2000, None, 1, 64, 1,
                               *[ctypes.byref(x) for x in big[4:]], 0, 0x100000, 1 << 30, None)
    assert st == b.LA_ERR_UNSUPPORTED


def test_bwd_gated_norm_host_logic(lib):
    """la_bwd_chunk_gated_norm takes la_bwd_chunk_norm's workspace; NULL or misaligned
    decays and gradients are rejected before any device call when there are tokens."""
    from chunkwise_causal_linear_la_b200 import binding as b

    for args in ((3, 100, 5, 128, 128, 64, 1, 0), (3, 100, 5, 64, 32, 32, 0, 0), (3, 100, 5, 128, 256, 64, 1, 0)):
        assert lib.la_bwd_chunk_gated_norm_workspace_size(*args) == lib.la_bwd_chunk_norm_workspace_size(*args)
    need = lib.la_bwd_chunk_norm_workspace_size(1, 4, 2, 128, 128, 64, 1, 0)
    t = [_t(D=128) for _ in range(7)]

    def call(g=0x2000, dg=0x3000):
        return lib.la_bwd_chunk_gated_norm(*[ctypes.byref(x) for x in t[:4]], g, None, 1, 64, 1,
                                           *[ctypes.byref(x) for x in t[4:]], dg, 0, 0x100000, need, None)
    assert call(g=None) == b.LA_ERR_INVALID_ARG and b"g is NULL" in lib.la_last_error()
    assert call(dg=None) == b.LA_ERR_INVALID_ARG and b"dg" in lib.la_last_error()
    assert call(g=0x2002) == b.LA_ERR_INVALID_ARG and b"aligned" in lib.la_last_error()
    st = lib.la_bwd_chunk_gated(*[ctypes.byref(x) for x in t[:4]], None, None, 1, 64, 1,
                                *[ctypes.byref(x) for x in t[4:]], 0x3000, 0, None)
    assert st == b.LA_ERR_INVALID_ARG and b"g is NULL" in lib.la_last_error()
