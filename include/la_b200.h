/*
 * la_b200.h -- causal linear attention on NVIDIA B200 (sm_100a): C ABI.
 *
 * The method.  "1.6 长上下文与高效注意力" (long context and efficient
 * attention), section 线性注意力 (linear attention), displayed equation:
 * causal attention with sim(q, k) = phi(q)^T phi(k) collapses into a state
 * S_t (d_v x d_k) and a normaliser z_t (d_k) updated once per token,
 *     S_t = gamma S_{t-1} + v_t phi(k_t)^T,     z_t = gamma z_{t-1} + phi(k_t),
 *     o_t = S_t phi(q_t)        or, normalised,  o_t = S_t phi(q_t) / (z_t^T phi(q_t)),
 * with S_0 = 0, z_0 = 0.  phi is elu(x)+1 (the page's positive feature map)
 * or the identity.  gamma is a constant decay per head (gamma = 1 is the
 * page's equation; gamma < 1 is the decay-masked form the same chapter
 * describes under 状态空间模型与 Mamba as linear attention with a decay mask).
 * The same section notes that training runs in parallel or in chunks and that
 * inference keeps O(1) state per token; "Triton fused linear attention
 * kernels" (hotdry blog, 2025-09-14) names the chunk mode.  la_fwd_chunk is the
 * chunk-mode prefill and la_step the one-token recurrent update.
 *
 * Conventions shared by every call.
 *   Memory.  Every pointer given to a compute call is DEVICE memory on the
 *     current CUDA device, owned by the caller.  The library allocates and
 *     frees no device memory; scratch space is passed in as `workspace`.
 *   Streams.  `stream` is a cudaStream_t passed as void* (NULL = legacy
 *     default stream).  Calls enqueue work and return without synchronising;
 *     a returned LA_OK means the arguments were valid and the launches were
 *     accepted, not that the kernels have finished.
 *   Errors.  Every call returns an la_status; nothing aborts, throws or exits
 *     across this interface.  On an error no kernel has been launched (for
 *     LA_ERR_CUDA, a launch itself failed).  la_last_error() gives a message
 *     for the calling thread's last failure.
 *   Thread safety.  Calls may come from several host threads; the only state
 *     kept between calls is a per-thread error message and per-device
 *     attribute caches.
 */
#ifndef LA_B200_H
#define LA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported entry points (the library is built with hidden default visibility). */
#if defined(__GNUC__)
#define LA_API __attribute__((visibility("default")))
#else
#define LA_API
#endif

typedef enum {
  LA_OK = 0,
  LA_ERR_INVALID_ARG = 1, /* a pointer, size, stride or value is invalid */
  LA_ERR_UNSUPPORTED = 2, /* valid, but outside what the kernels implement */
  LA_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required */
  LA_ERR_CUDA = 4         /* a CUDA runtime/driver call or launch failed */
} la_status;

typedef enum { LA_PHI_IDENTITY = 0, LA_PHI_ELU1 = 1 } la_phi;

typedef enum { LA_F32 = 0, LA_BF16 = 1 } la_dtype;

/* Flags for la_fwd_chunk. */
#define LA_FLAG_NONE 0
/* Run the CUDA-core (SIMT, fp32 arithmetic) chunk kernel even where the
 * tensor-core kernel applies.  Both are CUDA kernels; there is no CPU path. */
#define LA_FLAG_SIMT 1
/* Testing the failure path, la_fwd_gated_delta_chunk on the tensor cores only:
 * the WY pass issues no tile load, so its first wait runs out (bounded: about
 * two seconds per CTA, plus as long again to drain), its CTAs raise their
 * abort flags, free their tensor memory and return; la_device_error then
 * reports the timeout (flags bit 0) and where it happened.  The call's
 * outputs are undefined; the CUDA context stays usable. */
#define LA_FLAG_TEST_WAIT_TIMEOUT 0x100

/*
 * A strided 4-D activation tensor [B, T, H, D] in device memory.
 *   data      pointer to element [0,0,0,0]; 16-byte aligned
 *   dtype     la_dtype of every element
 *   B,T,H,D   logical shape (batch, tokens, heads, head dim)
 *   stride_*  element strides of the B, T and H axes; the D axis is
 *             contiguous (stride 1).  Strides must be >= 0.
 * [B, T, hidden] activations with hidden = H*D are this layout with
 * stride_h = D, stride_t = H*D, stride_b = T*H*D.
 */
typedef struct {
  void *data;
  int32_t dtype;
  int64_t B, T, H, D;
  int64_t stride_b, stride_t, stride_h;
} la_tensor;

/*
 * la_fwd_chunk -- chunkwise-parallel causal linear attention forward
 * (prefill) over a dense batch or a packed variable-length batch.
 *
 *   q, k        [B, T, H, d_k]; v [B, T, H, d_v]; one dtype for all three.
 *   gamma       device float[H]: the decay of each head, 0 <= gamma <= 1.
 *   cu_seqlens  NULL for a dense batch (n_seqs = B sequences of T tokens), or
 *               device int32[n_seqs + 1] for a packed batch: B must be 1,
 *               sequence n is tokens cu_seqlens[n] .. cu_seqlens[n+1]-1,
 *               cu_seqlens[0] = 0, entries non-decreasing, last entry <= T.
 *               The state and normaliser restart at zero for each sequence;
 *               a zero-length sequence yields a zero final state.  The entries
 *               are read on the device only; violating these rules gives
 *               undefined results (the call cannot check them without a
 *               device-to-host copy).
 *   n_seqs      number of sequences (B when cu_seqlens is NULL).
 *   chunk       tile length along T: 16, 32, 64 or 128.  The result does not
 *               depend on it beyond floating-point rounding.
 *   phi         la_phi applied to q and k (never to v).
 *   normalize   nonzero: divide each output row by z_t^T phi(q_t).  No epsilon
 *               is added; with phi = identity the denominator can vanish.
 *   out         [B, T, H, d_v], same dtype as q; written for every token that
 *               belongs to a sequence (others are left untouched).
 *   final_state NULL, or device float[n_seqs, H, d_k, d_v] receiving S^T of
 *               each sequence after its last token, row-major: entry
 *               [n][h][c][r] = S[r][c].  This is the `state` la_step takes.
 *   flags       LA_FLAG_NONE or LA_FLAG_SIMT.
 *   workspace   device scratch of at least la_fwd_chunk_workspace_size(...)
 *               bytes (NULL allowed when that size is 0), 256-byte aligned.
 *               Its contents need not be initialised and are undefined after.
 *   stream      cudaStream_t as void*.
 *
 * Kernels: bf16 with chunk 64 and d_k in {64, 128} (d_v = 64, 128 or 256) or
 * d_k = 256 (d_v = 64, 128 or 256) runs on the tensor cores; every other valid
 * shape, f32, and LA_FLAG_SIMT run on the CUDA-core kernel, which computes in
 * fp32 and is roughly ten times slower.  la_fwd_chunk_path tells which one a
 * shape takes.
 *
 * Arithmetic: bf16 inputs are read as bf16, phi is evaluated in fp32 and the
 * tensor-core operands (phi(q), phi(k), decayed phi(k) or decayed v, the masked
 * score tile and the carried state) are rounded to bf16; all accumulation, the
 * carried state and the normaliser are fp32; `out` is rounded to its dtype once.
 * f32 inputs run entirely in fp32 on CUDA cores (no TF32).
 *
 * Errors: LA_ERR_INVALID_ARG for NULL required pointers, inconsistent shapes,
 * dtype mismatch, negative sizes, a bad phi, misaligned pointers;
 * LA_ERR_UNSUPPORTED for a chunk outside {16,32,64,128} or head dims outside
 * {16, 32, 64, 128, 256}; LA_ERR_WORKSPACE when the workspace is too small.
 */
LA_API la_status la_fwd_chunk(const la_tensor *q, const la_tensor *k, const la_tensor *v,
                       const float *gamma, const int32_t *cu_seqlens, int64_t n_seqs,
                       int32_t chunk, int32_t phi, int32_t normalize, const la_tensor *out,
                       float *final_state, int32_t flags, void *workspace,
                       size_t workspace_bytes, void *stream);

/*
 * la_fwd_chunk_z -- la_fwd_chunk that also returns the normaliser's state.
 * "1.6 长上下文与高效注意力", section 线性注意力: the normalised output divides
 * by z_t^T phi(q_t), where z_t = gamma z_{t-1} + phi(k_t) is carried beside S.
 * A normalised decode (la_step_norm) continues from S and z, so a prefill that
 * hands over to it needs z after the last token too.
 *
 *   final_z  NULL, or device float[n_seqs, H, d_k]: z of each sequence after
 *            its last token (zero for a zero-length sequence).  Requires
 *            normalize != 0 (LA_ERR_INVALID_ARG otherwise); 16-byte aligned.
 *   Every other argument, layout, result and error is that of la_fwd_chunk,
 *   which is this call with final_z = NULL.
 */
LA_API la_status la_fwd_chunk_z(const la_tensor *q, const la_tensor *k, const la_tensor *v,
                                const float *gamma, const int32_t *cu_seqlens, int64_t n_seqs,
                                int32_t chunk, int32_t phi, int32_t normalize, const la_tensor *out,
                                float *final_state, float *final_z, int32_t flags, void *workspace,
                                size_t workspace_bytes, void *stream);

/*
 * la_fwd_chunk_gated -- la_fwd_chunk_z with a data-dependent decay.
 * "1.6 长上下文与高效注意力", section 状态空间模型与 Mamba: the decay of the state
 * becomes a function of the input token (Mamba-2: a scalar per step, which is
 * linear attention with a decay mask).  Here the decay of token t in head h is
 * alpha = exp(g[t][h]):
 *     S_t = alpha_t S_{t-1} + v_t phi(k_t)^T,   z_t = alpha_t z_{t-1} + phi(k_t).
 *   g        device float[B, T, H], contiguous (token rows of the q layout; a
 *            packed batch has B = 1): the log decay, finite and <= 0 (alpha in
 *            (0, 1]); it takes the place of gamma.  4-byte aligned.
 *   Every other argument, layout, result and error is that of la_fwd_chunk_z
 *   (final_z may be NULL; it needs normalize).  The workspace size is
 *   la_fwd_chunk_workspace_size's for the same shape.
 */
LA_API la_status la_fwd_chunk_gated(const la_tensor *q, const la_tensor *k, const la_tensor *v, const float *g,
                                    const int32_t *cu_seqlens, int64_t n_seqs, int32_t chunk, int32_t phi,
                                    int32_t normalize, const la_tensor *out, float *final_state, float *final_z,
                                    int32_t flags, void *workspace, size_t workspace_bytes, void *stream);

/*
 * la_fwd_gated_delta -- the gated delta rule ("1.6 长上下文与高效注意力", section
 * Gated delta rule, and its listing), token by token:
 *     kt  = k_t / max(|k_t|, 1e-12)                       (unit key)
 *     S_t = alpha_t S_{t-1} (I - beta_t kt kt^T) + beta_t v_t kt^T,   o_t = S_t q_t
 * with alpha_t = exp(g_t), per (sequence, head); no feature map, no
 * normaliser (as in the section).  One call covers prefill and decode (T = 1
 * with the state passed in and out).
 *   q, k [B, T, H, d_k]; v [B, T, H, d_v]; out [B, T, H, d_v]; one dtype.
 *   g, beta     device float[B, T, H], contiguous: log decay (<= 0) and write
 *               strength (in (0, 1]) of each token.
 *   cu_seqlens, n_seqs  as for la_fwd_chunk.
 *   initial_state  NULL (zero) or device float[n_seqs, H, d_k, d_v] holding S^T.
 *   final_state    NULL or device float[n_seqs, H, d_k, d_v]: S^T after the last
 *               token; may be the same buffer as initial_state (updated in place).
 * CUDA cores, fp32 state and arithmetic: each thread keeps one value column's
 * state in registers and walks the tokens in order (latency-bound, not a
 * chunked kernel).  d_k, d_v in {16, 32, 64, 128, 256}.  Errors as for
 * la_fwd_chunk.
 */
LA_API la_status la_fwd_gated_delta(const la_tensor *q, const la_tensor *k, const la_tensor *v, const float *g,
                                    const float *beta, const int32_t *cu_seqlens, int64_t n_seqs,
                                    const float *initial_state, const la_tensor *out, float *final_state,
                                    void *stream);

/*
 * la_fwd_gated_delta_chunk -- the same rule as la_fwd_gated_delta (same
 * arguments and results), computed in chunks of 64 tokens.  Inside a chunk
 * the writes u_i = beta_i (v_i - alpha_i S_{i-1} kt_i) solve a unit
 * lower-triangular system (the UT / WY form of the delta rule; the pages give
 * the recurrence, the chunk form is its exact regrouping), so
 *     U = T diag(beta) V - T diag(beta e^b) Kt S_0^T,   T = (I + A)^{-1},
 *     A_ij = beta_i e^{b_i - b_j} kt_i . kt_j  (j < i),  b_i = sum of g over the chunk up to i,
 * and outputs and the next chunk's state follow from U with matrix products.
 * Tensor cores (tcgen05) for bf16 with d_k, d_v in {64, 128} and 16-byte aligned
 * initial_state / final_state: a parallel pass over all chunks writes
 * W = T diag(beta e^b) Kt and T diag(beta) V (bf16) and the chunk's b_i and
 * ln(1/|k_i|) - b_i (fp32) to the workspace, then one CTA per (sequence, head)
 * walks its chunks with the fp32 state.  Every other
 * case, and flags = LA_FLAG_SIMT, runs la_fwd_gated_delta's kernel (no
 * workspace needed).
 *   flags       LA_FLAG_NONE or LA_FLAG_SIMT; LA_FLAG_TEST_WAIT_TIMEOUT (tests only).
 *   workspace   device memory of la_fwd_gated_delta_workspace_size bytes,
 *               256-byte aligned, owned by the caller; its contents are
 *               scratch (nothing needs to be zero; nothing is kept).
 * Errors as for la_fwd_chunk (LA_ERR_WORKSPACE when the workspace is short).
 */
LA_API la_status la_fwd_gated_delta_chunk(const la_tensor *q, const la_tensor *k, const la_tensor *v,
                                          const float *g, const float *beta, const int32_t *cu_seqlens,
                                          int64_t n_seqs, const float *initial_state, const la_tensor *out,
                                          float *final_state, int32_t flags, void *workspace,
                                          size_t workspace_bytes, void *stream);

/*
 * Bytes of workspace la_fwd_gated_delta_chunk needs: B, T, H, d_k, d_v,
 * n_seqs, has_cu_seqlens, dtype and flags as they will be passed.  0 when the
 * call needs none (the token-by-token kernel); (size_t)-1 for arguments the
 * call would reject.  Host-only.  On the tensor cores: 2 B T H 128 bf16 values
 * (W, T diag(beta) V), 128 floats per (chunk, head) (b_i, ln(1/|k_i|) - b_i; a packed
 * batch counts ceil(T / 64) + n_seqs chunks) and, for a packed batch,
 * n_seqs + 1 chunk offsets, each region rounded up to 256 bytes.
 */
LA_API size_t la_fwd_gated_delta_workspace_size(int64_t B, int64_t T, int64_t H, int64_t d_k, int64_t d_v,
                                                int64_t n_seqs, int32_t has_cu_seqlens, int32_t dtype,
                                                int32_t flags);

/*
 * la_norm_gate -- the output norm and gate of a retention layer, on its own:
 *     y[r] = o[r] / sqrt(mean_r' o[r']^2 + eps) * w[r] * gate[r] * sigmoid(gate[r])
 * per (token, head) over the d_v values ("使用 FlashAttention 内核实现最先进的线性注意力":
 * RMSNorm fused with a Swish gate; the formula is the plain reading of those
 * two names).  o, gate, y [B, T, H, d_v], one dtype; y may alias o.  w device
 * float[d_v], shared by all heads; eps >= 0.  fp32 arithmetic.
 */
LA_API la_status la_norm_gate(const la_tensor *o, const la_tensor *gate, const float *w, float eps,
                              const la_tensor *y, void *stream);

/*
 * la_fwd_chunk_normgate -- la_fwd_chunk whose `out` receives la_norm_gate of
 * the attention output (gate, w, eps as there).  On the tensor cores with
 * d_k = d_v = 128 the norm and gate run in the kernel's epilogue (the output is
 * written once); otherwise a second pass normalises `out` in place, and then
 * rows of a packed batch outside every sequence are written too.  Other
 * arguments, results and errors as for la_fwd_chunk.
 */
LA_API la_status la_fwd_chunk_normgate(const la_tensor *q, const la_tensor *k, const la_tensor *v,
                                       const float *gamma, const int32_t *cu_seqlens, int64_t n_seqs,
                                       int32_t chunk, int32_t phi, int32_t normalize, const la_tensor *gate,
                                       const float *w, float eps, const la_tensor *out, float *final_state,
                                       int32_t flags, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Bytes of workspace la_fwd_chunk needs for this problem: B, T, H, d_k, d_v
 * and n_seqs as they will be passed, has_cu_seqlens nonzero for a packed
 * batch.  Returns 0 when no workspace is needed and (size_t)-1 for arguments
 * la_fwd_chunk would reject.  Host-only; touches no device.  On the tensor-core
 * path the workspace holds the segment states of long sequences in batches too
 * small to fill the GPU (each sequence then runs as several segments), and the
 * longest-first order of a packed batch of 2 .. 4096 sequences.
 */
LA_API size_t la_fwd_chunk_workspace_size(int64_t B, int64_t T, int64_t H, int64_t d_k, int64_t d_v,
                                   int64_t n_seqs, int32_t has_cu_seqlens, int32_t chunk,
                                   int32_t dtype, int32_t flags);

/*
 * la_fwd_chunk_path -- which kernel la_fwd_chunk (and la_fwd_chunk_z,
 * la_fwd_chunk_gated, la_fwd_chunk_normgate, the noalloc variant) runs for a
 * problem with these head dims, length, heads, chunk, dtype and flags on the
 * current device: LA_PATH_TENSOR_CORE (the tcgen05 kernel) or
 * LA_PATH_CUDA_CORE (fp32 CUDA-core kernel: every other valid shape, much
 * slower); -1 for arguments la_fwd_chunk rejects (LA_ERR_INVALID_ARG or
 * LA_ERR_UNSUPPORTED).  An addition of this library (the pages have no
 * counterpart): it lets a caller see a fall back to the slow kernel before
 * timing it.  Host-only; reads device attributes but launches nothing.
 */
typedef enum { LA_PATH_TENSOR_CORE = 1, LA_PATH_CUDA_CORE = 2 } la_path;
LA_API int32_t la_fwd_chunk_path(int64_t d_k, int64_t d_v, int64_t T, int64_t H, int32_t chunk, int32_t dtype,
                                 int32_t flags);

/*
 * la_fwd_chunk_host -- la_fwd_chunk on host buffers, end to end: the inputs
 * are copied into a device arena, the forward runs there, and the output and
 * final state are copied back, all enqueued on `stream` in that order (one
 * cudaMemcpyAsync per buffer); the call returns before they complete, so
 * synchronise the stream before reading `out` or `final_state`.  An addition
 * of this library (the pages have no counterpart): for callers whose
 * activations are in host memory and who want the whole round trip measured
 * or scheduled as one call.
 *
 *   q, k, v, out  la_tensors whose data pointers are HOST memory, each
 *                 contiguous [B, T, H, D] (stride_h = D, stride_t = H D,
 *                 stride_b = T H D).  Page-locked memory lets the copies run
 *                 asynchronously; pageable memory works, but then each copy
 *                 waits for the host.
 *   gamma         host float[H]; cu_seqlens host int32[n_seqs + 1] or NULL;
 *   final_state   host float[n_seqs, H, d_k, d_v] or NULL.
 *   arena         device memory the caller owns, 256-byte aligned, of at
 *                 least la_fwd_chunk_host_arena_size(...) bytes (with
 *                 has_final_state = final_state != NULL): it receives the device
 *                 copies of every buffer and la_fwd_chunk's workspace.  Its
 *                 contents are undefined after the call.
 *   Every other argument, the results and the arithmetic are la_fwd_chunk's.
 * Errors: LA_ERR_INVALID_ARG for a non-contiguous host tensor, a NULL pointer
 * or a misaligned arena; LA_ERR_UNSUPPORTED for a shape la_fwd_chunk rejects;
 * LA_ERR_WORKSPACE for a missing or short arena; LA_ERR_CUDA if a copy cannot
 * be enqueued; la_fwd_chunk's own errors otherwise.  Nothing is allocated.
 */
LA_API size_t la_fwd_chunk_host_arena_size(int64_t B, int64_t T, int64_t H, int64_t d_k, int64_t d_v,
                                           int64_t n_seqs, int32_t has_cu_seqlens, int32_t chunk, int32_t dtype,
                                           int32_t flags, int32_t has_final_state);
LA_API la_status la_fwd_chunk_host(const la_tensor *q, const la_tensor *k, const la_tensor *v, const float *gamma,
                                   const int32_t *cu_seqlens, int64_t n_seqs, int32_t chunk, int32_t phi,
                                   int32_t normalize, const la_tensor *out, float *final_state, int32_t flags,
                                   void *arena, size_t arena_bytes, void *stream);

/*
 * la_step -- one decode token per sequence: the recurrence applied once.
 *   q, k   [N, 1, H, d_k]; v [N, 1, H, d_v] (la_tensor with T = 1); f32 or
 *          bf16, one dtype for all three.
 *   gamma  device float[H].
 *   state  device float[N, H, d_k, d_v], S^T as la_fwd_chunk writes it,
 *          updated in place:  S^T[c][r] <- gamma S^T[c][r] + phi(k)_c v_r.
 *   out    [N, 1, H, d_v], q's dtype:  o_r = sum_c S^T[c][r] phi(q)_c,
 *          read after the update (the token sees itself, as in prefill).
 *   phi    la_phi.  No normaliser: the state carries no z.
 * The state is read and written exactly once (fp32 arithmetic); the kernel is
 * bound by HBM bandwidth.  Errors as for la_fwd_chunk; LA_ERR_UNSUPPORTED
 * unless d_k <= 256 and d_v is a power of two in [4, 256]; state must be
 * 16-byte aligned.
 */
LA_API la_status la_step(const la_tensor *q, const la_tensor *k, const la_tensor *v, const float *gamma,
                  float *state, const la_tensor *out, int32_t phi, void *stream);

/*
 * la_step_norm -- one normalised decode token per sequence: the displayed
 * equation of "1.6 长上下文与高效注意力", section 线性注意力, applied once with
 * the per-head decay:
 *     z[c]      <- gamma z[c] + phi(k)_c
 *     S^T[c][r] <- gamma S^T[c][r] + phi(k)_c v_r
 *     o_r        = (sum_c S^T[c][r] phi(q)_c) / (sum_c z[c] phi(q)_c)
 * (both sums after the update, as in prefill; no epsilon).
 *   q, k, v, gamma, state, out, phi  as for la_step.
 *   z      device float[N, H, d_k], updated in place; 16-byte aligned.  It
 *          continues from la_fwd_chunk_z's final_z.
 * The state and z are read and written once (fp32); HBM-bound.  Errors and
 * supported sizes as for la_step.
 */
LA_API la_status la_step_norm(const la_tensor *q, const la_tensor *k, const la_tensor *v, const float *gamma,
                              float *state, float *z, const la_tensor *out, int32_t phi, void *stream);

/*
 * la_step_gated -- one decode token with a data-dependent decay: la_step
 * (z == NULL) or la_step_norm (z != NULL) with the decay of sequence n, head h
 * equal to exp(g[n][h]) instead of gamma[h].
 *   g  device float[N, H], contiguous: the log decay of this step, <= 0.
 * Other arguments, sizes and errors as for la_step / la_step_norm.
 */
LA_API la_status la_step_gated(const la_tensor *q, const la_tensor *k, const la_tensor *v, const float *g,
                               float *state, float *z, const la_tensor *out, int32_t phi, void *stream);

/*
 * la_bwd_chunk -- backward of the unnormalised chunked forward: the gradients
 * of a loss with respect to q, k, v, given its gradient dout at the output.
 * The forward is the recurrence of "1.6 长上下文与高效注意力", section 线性注意力,
 * with the per-head decay, S_t = gamma S_{t-1} + v_t phi(k_t)^T, o_t = S_t phi(q_t);
 * its adjoint is
 *     dphi(q)_t = S_t^T dout_t,   G_t = dout_t phi(q_t)^T + gamma G_{t+1},
 *     dphi(k)_t = G_t^T v_t,      dv_t = G_t phi(k_t),
 * and dq = dphi(q) * phi'(q), dk = dphi(k) * phi'(k) (phi' = 1, or 1 / e^x for
 * elu + 1 at x > 0 / x <= 0).
 *   q, k, v, gamma, cu_seqlens, n_seqs, chunk, phi  as for la_fwd_chunk (the
 *               forward's inputs; states start at zero, gamma is not differentiated).
 *   dout        [B, T, H, d_v], q's dtype: the gradient at `out`.
 *   dq, dk      [B, T, H, d_k]; dv [B, T, H, d_v]; q's dtype; written for every
 *               token that belongs to a sequence.
 *   flags       LA_FLAG_NONE or LA_FLAG_SIMT (force the CUDA-core kernel).
 * Kernels: bf16 with chunk 64 and tensor-core head dims (as for la_fwd_chunk;
 * with elu + 1 also d_k == d_v) runs as three tensor-core forward passes on
 * rearranged operands:
 *     dphi(q) = forward(q' = dout, k' = v, v' = phi(k))
 *     dphi(k) = forward in reverse time (q' = v, k' = dout, v' = phi(q))
 *     dv      = forward in reverse time (q' = phi(k), k' = phi(q), v' = dout)
 * (each sum above has exactly that form; reverse time turns sum_{i>=j} into
 * the forward's sum_{j<=i}); bf16 operands and fp32 accumulation as in the
 * forward.  Every other shape, f32, and LA_FLAG_SIMT run one CUDA-core kernel
 * in fp32; it needs the d_k x d_v fp32 state and one chunk's tiles to fit in
 * shared memory (d_k = d_v = 128 fits; 256 does not: LA_ERR_UNSUPPORTED).
 * Tokens outside every sequence of a packed batch may be overwritten in dq,
 * dk, dv.  The normalised forward's backward is la_bwd_chunk_norm, the per-token
 * decay's la_bwd_chunk_gated (la_bwd_chunk_gated_norm when normalised).  Other
 * errors as for la_fwd_chunk.
 */
LA_API la_status la_bwd_chunk(const la_tensor *q, const la_tensor *k, const la_tensor *v, const la_tensor *dout,
                              const float *gamma, const int32_t *cu_seqlens, int64_t n_seqs, int32_t chunk,
                              int32_t phi, const la_tensor *dq, const la_tensor *dk, const la_tensor *dv,
                              int32_t flags, void *stream);

/*
 * la_bwd_chunk_gated -- backward of la_fwd_chunk_gated's unnormalised forward
 * (the data-dependent decay of "1.6 长上下文与高效注意力", section 状态空间模型与
 * Mamba: alpha_t = exp(g_t) per token and head), including the gradient of the
 * log decays.  With b the prefix sum of g over each sequence,
 *     o_i = sum_{j<=i} exp(b_i - b_j) (phi(q_i) . phi(k_j)) v_j,
 * so the gradients of phi(q), phi(k), v have la_bwd_chunk's three sums with
 * exp(b_i - b_j) in place of gamma^(i-j), and, because the loss sees b_s only
 * through those weights,
 *     dg_t = sum_{s >= t} (phi(q_s) . dphi(q)_s - phi(k_s) . dphi(k)_s).
 *   q, k, v, cu_seqlens, n_seqs, chunk, phi  as for la_fwd_chunk_gated.
 *   g           device float[B, T, H], the forward's log decays (<= 0).
 *   dout        [B, T, H, d_v], q's dtype: the gradient at `out`.
 *   dq, dk, dv  as for la_bwd_chunk.
 *   dg          device float[B, T, H]: the gradient with respect to g (fp32
 *               arithmetic: row dot products, then a reverse cumulative sum per
 *               sequence and head); 4-byte aligned.
 * Kernels: bf16 with chunk 64 and head dims for which la_fwd_chunk_path
 * reports LA_PATH_TENSOR_CORE (with elu + 1 also d_k == d_v) run on the
 * tensor cores; the two reverse-time passes take, at each reversed position,
 * the decay of the token after it.  f32, other chunks and shapes and
 * LA_FLAG_SIMT run la_bwd_chunk's CUDA-core kernel with the per-token decay
 * (fp32; LA_ERR_UNSUPPORTED where its shared memory does not fit).  Other
 * errors as for la_bwd_chunk.
 */
LA_API la_status la_bwd_chunk_gated(const la_tensor *q, const la_tensor *k, const la_tensor *v,
                                    const la_tensor *dout, const float *g, const int32_t *cu_seqlens,
                                    int64_t n_seqs, int32_t chunk, int32_t phi, const la_tensor *dq,
                                    const la_tensor *dk, const la_tensor *dv, float *dg, int32_t flags,
                                    void *stream);

/*
 * la_bwd_chunk_norm -- backward of la_fwd_chunk with normalize = 1, the
 * normalised linear attention of "1.6 长上下文与高效注意力", section 线性注意力:
 *     o_t = num_t / den_t,  num_t = sum_{j<=t} gamma^(t-j) (phi(q_t) . phi(k_j)) v_j,
 *                           den_t = sum_{j<=t} gamma^(t-j)  phi(q_t) . phi(k_j).
 * With L = sum_t dout_t . o_t, the gradient reaching num_t is u_t = dout_t / den_t
 * and the one reaching den_t is e_t = -(dout_t . num_t) / den_t^2; so
 *     dphi(q)_t = sum_{j<=t} gamma^(t-j) (u_t . v_j + e_t) phi(k_j),
 *     dphi(k)_j = sum_{t>=j} gamma^(t-j) (u_t . v_j + e_t) phi(q_t),
 *     dv_j      = sum_{t>=j} gamma^(t-j) (phi(q_t) . phi(k_j)) u_t,
 * which are la_bwd_chunk's three sums for the values [v_j, 1] and the output
 * gradient [u_t, e_t]; dq and dk then take phi' (elu + 1) as in la_bwd_chunk.
 *   q, k, v, gamma, cu_seqlens, n_seqs, chunk, phi  as for la_fwd_chunk.
 *   dout, dq, dk, dv  as for la_bwd_chunk.
 *   workspace   device memory of la_bwd_chunk_norm_workspace_size bytes,
 *               256-byte aligned, owned by the caller; it holds [v, 1, 1, 0...]
 *               and [u, e_hi, e_lo, 0...] (q's dtype, 2 d_v columns) and, on
 *               the tensor cores, the forward's o and den (fp32) and, with
 *               elu + 1, phi(k); on the CUDA cores the widened dv as well.
 *               Nothing in it need start at zero.
 * Kernels: bf16 with chunk 64, d_v in {64, 128} and d_k in {64, 128, 256} run
 * on the tensor cores: the normalised forward (which also writes den_t), two
 * row passes ([v, 1, 1] and [u, e]), then the three backward passes (plus two
 * feature-map copies with elu + 1).  f32, the other chunks, d_v in {16, 32}
 * and LA_FLAG_SIMT run on the CUDA-core kernels in fp32: the unnormalised
 * forward of (q, k, [v, 1, 1]) gives [num, den], a row pass turns it into
 * [u, e], the backward kernel runs on the widened values, and a copy takes dv;
 * shapes whose widened rows do not fit that kernel's shared memory (d_k = 128
 * with d_v = 128, say) return LA_ERR_UNSUPPORTED.  Rounding: the sums
 * u_t . v_j + e_t cancel (for a one-token sequence exactly, since o_1 = v_1),
 * so e_t = -(u_t . o_t) is taken from u_t as stored (the exact gradient for an
 * output gradient within one rounding of dout) and kept as a pair
 * e_hi + e_lo.  d_v = 256 (widened past 256 columns), other chunks and head
 * dims return LA_ERR_UNSUPPORTED.  den_t = 0 gives non-finite gradients, as
 * it gives a non-finite forward output.
 * LA_ERR_WORKSPACE if workspace is NULL or short.  Other errors as for
 * la_bwd_chunk.  la_bwd_chunk_norm_workspace_size returns (size_t)-1 for
 * shapes, chunks, dtypes or flags that la_bwd_chunk_norm rejects.
 */
LA_API size_t la_bwd_chunk_norm_workspace_size(int64_t B, int64_t T, int64_t H, int64_t d_k, int64_t d_v,
                                               int32_t chunk, int32_t dtype, int32_t flags);
LA_API la_status la_bwd_chunk_norm(const la_tensor *q, const la_tensor *k, const la_tensor *v,
                                   const la_tensor *dout, const float *gamma, const int32_t *cu_seqlens,
                                   int64_t n_seqs, int32_t chunk, int32_t phi, const la_tensor *dq,
                                   const la_tensor *dk, const la_tensor *dv, int32_t flags, void *workspace,
                                   size_t workspace_bytes, void *stream);

/*
 * la_bwd_chunk_gated_norm -- backward of la_fwd_chunk_gated with normalize = 1
 * (the data-dependent decay of "1.6 长上下文与高效注意力", section 状态空间模型与
 * Mamba, with the normaliser of section 线性注意力): with b the prefix sums of g,
 *     o_t = num_t / den_t,  num_t = sum_{j<=t} exp(b_t - b_j) (phi(q_t) . phi(k_j)) v_j,
 *                           den_t = sum_{j<=t} exp(b_t - b_j)  phi(q_t) . phi(k_j).
 * The same widening as la_bwd_chunk_norm ([v, 1] values, [u, e] output
 * gradient) turns it into la_bwd_chunk_gated's problem, whose dg is this one's:
 * the loss sees g only through the weights of num and den, both outputs of the
 * widened problem.
 *   q, k, v, g, cu_seqlens, n_seqs, chunk, phi  as for la_fwd_chunk_gated.
 *   dout, dq, dk, dv  as for la_bwd_chunk; dg as for la_bwd_chunk_gated.
 *   workspace   as for la_bwd_chunk_norm (la_bwd_chunk_gated_norm_workspace_size
 *               returns the same size).
 * Kernels: as for la_bwd_chunk_norm, with the per-token decay in every pass
 * (the tensor-core route's forward is the normalised la_fwd_chunk_gated
 * kernel, which also writes den_t).  Errors as for la_bwd_chunk_norm; g or dg
 * NULL (with tokens to process) or not 4-byte aligned: LA_ERR_INVALID_ARG.
 * A problem without tokens needs no workspace and returns LA_OK.
 */
LA_API size_t la_bwd_chunk_gated_norm_workspace_size(int64_t B, int64_t T, int64_t H, int64_t d_k, int64_t d_v,
                                                     int32_t chunk, int32_t dtype, int32_t flags);
LA_API la_status la_bwd_chunk_gated_norm(const la_tensor *q, const la_tensor *k, const la_tensor *v,
                                         const la_tensor *dout, const float *g, const int32_t *cu_seqlens,
                                         int64_t n_seqs, int32_t chunk, int32_t phi, const la_tensor *dq,
                                         const la_tensor *dk, const la_tensor *dv, float *dg, int32_t flags,
                                         void *workspace, size_t workspace_bytes, void *stream);

/*
 * la_fwd_chunk_noalloc -- la_fwd_chunk for callers that cannot allocate device
 * memory.  (An addition of this library; the pages have no counterpart.)
 *
 * Some callers may not allocate: a plugin running inside a framework that owns
 * all device memory and hands out none at execution time, or a latency-bound
 * serving loop in which cudaMalloc could synchronise the device.  la_fwd_chunk
 * needs scratch memory for long sequences (the segment states); this variant
 * takes no workspace and uses instead one array of LA_NOALLOC_SCRATCH_BYTES
 * that the library keeps in the memory of every device it is loaded on, until
 * the process exits.  It allocates nothing and frees nothing.
 *
 *   Arguments, layouts, results and errors are those of la_fwd_chunk without
 *   `workspace` / `workspace_bytes`.  LA_ERR_WORKSPACE if the problem needs more
 *   than LA_NOALLOC_SCRATCH_BYTES of scratch (la_fwd_chunk_workspace_size tells;
 *   every problem the current kernels segment fits).
 *   Set-up: the first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current) and caches it together
 *   with the device's current context; a call made in another context of that
 *   device (after cudaDeviceReset, say) looks the address up again.  Make the
 *   first call in each context before any stream capture.
 *   Sharing: all calls on a device use the same array and it keeps the previous
 *   call's contents (nothing in it needs to start at zero).  Calls whose work
 *   overlaps on the GPU (different streams, or several host threads on one
 *   device) race on it: order them.
 */
#define LA_NOALLOC_SCRATCH_BYTES (10u << 20)
LA_API la_status la_fwd_chunk_noalloc(const la_tensor *q, const la_tensor *k, const la_tensor *v,
                                      const float *gamma, const int32_t *cu_seqlens, int64_t n_seqs,
                                      int32_t chunk, int32_t phi, int32_t normalize, const la_tensor *out,
                                      float *final_state, int32_t flags, void *stream);

/*
 * la_device_error -- read the device-side error word of the tensor-core
 * kernel.  Every wait inside that kernel is bounded (about two seconds); a
 * wait that runs out makes the CTA give up, drain its asynchronous copies, free
 * its tensor memory and return, and records the failure here instead of
 * hanging or trapping.
 *   flags   receives a bit set: 1 = a wait timed out, 2 = draining timed out
 *           (0 = no failure since the last reset)
 *   detail  receives the first failed wait: bit 31 set, chunk index << 8,
 *           barrier index in the low 8 bits (0 if none)
 *   reset   nonzero: clear both words after reading
 * Synchronous: waits for all work on the current device to finish (it copies
 * from a device symbol).  Host pointers.  Errors: LA_ERR_INVALID_ARG for NULL
 * pointers, LA_ERR_CUDA if the copy fails.
 */
LA_API la_status la_device_error(uint32_t *flags, uint32_t *detail, int32_t reset);

/* Static description of a status code. */
LA_API const char *la_status_string(int32_t status);

/* Message describing the calling thread's most recent failed call ("" if none). */
LA_API const char *la_last_error(void);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
LA_API int32_t la_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LA_B200_H */
