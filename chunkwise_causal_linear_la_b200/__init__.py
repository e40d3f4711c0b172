"""Chunkwise causal linear attention on NVIDIA B200 (sm_100a).

The compute lives in the C-ABI library libla_b200.so (include/la_b200.h);
this package is its Python binding:

    from chunkwise_causal_linear_la_b200 import la_fwd_chunk, la_step
    out, final_state = la_fwd_chunk(q, k, v, gamma, chunk=64, phi="identity")
    o = la_step(q1, k1, v1, gamma, final_state)   # decode one more token

    # normalised: the prefill also hands over z
    out, final_state, z = la_fwd_chunk_z(q, k, v, gamma, phi="elu1")
    o = la_step_norm(q1, k1, v1, gamma, final_state, z, phi="elu1")

    # training: the forward and its backward as one differentiable call
    from chunkwise_causal_linear_la_b200.autograd import chunk_linear_attention
    o = chunk_linear_attention(q, k, v, gamma, phi="elu1", normalize=True)

``workloads`` draws the seeded synthetic inputs of the standard workloads.
"""
from .binding import (  # noqa: F401
    LA_FLAG_NONE,
    LA_FLAG_SIMT,
    LA_FLAG_TEST_WAIT_TIMEOUT,
    LaError,
    LA_PATH_CUDA_CORE,
    LA_PATH_TENSOR_CORE,
    device_error,
    fwd_chunk_path,
    host_arena_size,
    la_fwd_chunk_host,
    la_bwd_chunk,
    la_bwd_chunk_gated,
    la_bwd_chunk_norm,
    la_bwd_chunk_gated_norm,
    bwd_norm_workspace_size,
    la_fwd_chunk,
    la_fwd_chunk_gated,
    la_fwd_chunk_normgate,
    la_fwd_chunk_z,
    la_fwd_gated_delta,
    la_fwd_gated_delta_chunk,
    gated_delta_workspace_size,
    la_norm_gate,
    la_step,
    la_step_gated,
    la_step_norm,
    load_library,
    workspace_size,
)
