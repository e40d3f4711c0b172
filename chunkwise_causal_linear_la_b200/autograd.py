"""torch.autograd wrappers over the C ABI: the chunked forward and its backward as one
differentiable call, for training.

    from chunkwise_causal_linear_la_b200.autograd import chunk_linear_attention
    o = chunk_linear_attention(q, k, v, gamma, phi="elu1", normalize=True)
    o.backward(dout)          # q.grad, k.grad, v.grad from la_bwd_chunk_norm

Each wrapper only marshals: the forward runs la_fwd_chunk (or la_fwd_chunk_gated),
the backward la_bwd_chunk, la_bwd_chunk_norm or la_bwd_chunk_gated on the saved
inputs (nothing of the forward is kept but q, k, v and the decays).  gamma is not
differentiated (a constant of the layer); the per-token log decays g are.
"""
import torch

from . import binding


class _ChunkLinearAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, gamma, cu_seqlens, chunk, phi, normalize):
        out, _ = binding.la_fwd_chunk(q, k, v, gamma, cu_seqlens=cu_seqlens, chunk=chunk, phi=phi,
                                      normalize=normalize, return_final_state=False)
        ctx.save_for_backward(q, k, v, gamma, cu_seqlens)
        ctx.chunk, ctx.phi, ctx.normalize = chunk, phi, normalize
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, gamma, cu = ctx.saved_tensors
        dout = dout.contiguous()
        if ctx.normalize:
            dq, dk, dv = binding.la_bwd_chunk_norm(q, k, v, dout, gamma, cu_seqlens=cu, chunk=ctx.chunk,
                                                   phi=ctx.phi)
        else:
            dq, dk, dv = binding.la_bwd_chunk(q, k, v, dout, gamma, cu_seqlens=cu, chunk=ctx.chunk, phi=ctx.phi)
        return dq, dk, dv, None, None, None, None, None


class _ChunkGatedLinearAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, g, cu_seqlens, chunk, phi, normalize):
        out, _, _ = binding.la_fwd_chunk_gated(q, k, v, g, cu_seqlens=cu_seqlens, chunk=chunk, phi=phi,
                                               normalize=normalize)
        ctx.save_for_backward(q, k, v, g, cu_seqlens)
        ctx.chunk, ctx.phi, ctx.normalize = chunk, phi, normalize
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, g, cu = ctx.saved_tensors
        bwd = binding.la_bwd_chunk_gated_norm if ctx.normalize else binding.la_bwd_chunk_gated
        dq, dk, dv, dg = bwd(q, k, v, dout.contiguous(), g, cu_seqlens=cu, chunk=ctx.chunk, phi=ctx.phi)
        return dq, dk, dv, dg, None, None, None, None


def chunk_linear_attention(q, k, v, gamma, cu_seqlens=None, chunk=64, phi="identity", normalize=False):
    """Differentiable la_fwd_chunk: o_t = S_t phi(q_t) [/ z_t . phi(q_t)] with
    S_t = gamma S_{t-1} + v_t phi(k_t)^T; gradients reach q, k and v."""
    return _ChunkLinearAttention.apply(q, k, v, gamma, cu_seqlens, chunk, phi, normalize)


def chunk_gated_linear_attention(q, k, v, g, cu_seqlens=None, chunk=64, phi="identity", normalize=False):
    """Differentiable la_fwd_chunk_gated: the decay exp(g[b, t, h]) per token and head,
    optionally normalised; gradients reach q, k, v and the log decays g."""
    return _ChunkGatedLinearAttention.apply(q, k, v, g, cu_seqlens, chunk, phi, normalize)
