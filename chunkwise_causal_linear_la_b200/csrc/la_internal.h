// la_internal.h -- host-side interface between the C-ABI layer (la_api.cu)
// and the kernel files.  Not installed; not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "la_b200.h"

namespace la {

// Device-side view of one strided activation tensor [B, T, H, D] (D contiguous).
struct TensorView {
  const void *data;
  int64_t sb, st, sh;  // element strides of B, T, H
};

// Everything a chunked-prefill kernel needs.  Sequence n covers tokens
// [start, start + len) of batch row b:  dense  -> b = n, start = 0, len = T;
// packed (cu_seqlens) -> b = 0, start = cu[n], len = cu[n+1] - cu[n].
struct ChunkArgs {
  TensorView q, k, v;
  void *out;
  int64_t o_sb, o_st, o_sh;
  const float *gamma;         // per-head decay [H] (ignored when g is set)
  const float *g;             // NULL, or data-dependent log decay [B * T][H]
  const int32_t *cu_seqlens;  // NULL for dense batches
  float *final_state;         // NULL allowed
  float *final_z;             // NULL allowed; only with normalize
  int64_t B, T, n_seqs;
  int H, dk, dv, chunk, phi, normalize;
  int dtype;  // la_dtype of q, k, v, out
  // Output norm and gate fused into the epilogue (tensor-core kernel, d_v equal
  // to its value slice): out = RMSNorm(o) * ng_w * swish(gate); NULL ng_w: none
  const float *ng_w;
  TensorView ng_gate;
  float ng_eps;
  int rev;    // 1: reverse time (tensor-core kernel only; used by the backward pass)
  int noseg;  // 1: never split sequences into segments (no workspace)
  // Backward-pass epilogue (tensor-core kernel): with ex.data set, each output row o
  // (fp32, before rounding) meets the row x of ex at the same token, head and
  // columns (q's dtype): edg[row] += esign * phi(x) . o when edg is set (phi =
  // ephi), and with edphi the row written is o * phi'(x) (elu + 1).  ex.data NULL: off.
  TensorView ex;
  float *edg;
  float esign;
  int ephi, edphi;
  // Normalised forward on the tensor cores: den_t per (token, head), [B * T][H] fp32
  // (the backward of the normalised form reads it).  NULL: not written.
  float *den_out;
};

struct StepArgs {
  TensorView q, k, v;
  void *out;
  int64_t o_sb, o_sh;
  const float *gamma;
  const float *g;  // NULL, or per-(sequence, head) log decay [N, H] replacing gamma
  float *state;
  float *z;  // normaliser state [N, H, d_k] (la_step_norm); NULL for la_step
  int64_t N;
  int H, dk, dv, phi, dtype;
};

struct BwdArgs {
  TensorView q, k, v, dout, dq, dk_, dv_;
  const float *gamma;
  // per-token decay (NULL: gamma): log decays [B * T][H]; dg receives the row terms
  // of the log decays' gradient (zeroed by the caller; a reverse cumulative sum
  // per sequence finishes it)
  const float *g;
  float *dg;
  const int32_t *cu_seqlens;  // NULL for dense batches
  int64_t T, n_seqs;
  int H, dk, dv, chunk, phi, dtype;
};

struct DeltaArgs {
  TensorView q, k, v;
  void *out;
  int64_t o_sb, o_st, o_sh;
  const float *g, *beta;      // [B * T][H] log decay and write strength
  const float *init;          // NULL or [n_seqs, H, d_k, d_v] (S^T)
  float *final_state;         // NULL or [n_seqs, H, d_k, d_v]; may alias init
  const int32_t *cu_seqlens;  // NULL for dense batches
  int64_t T, n_seqs;
  int H, dk, dv, dtype;
  bool test_wait_timeout = false;  // LA_FLAG_TEST_WAIT_TIMEOUT (chunked path)
};

// Sets the calling thread's la_last_error() message and returns `status`.
la_status report_error(la_status status, const char *msg);

// The current device, with its primary context made current on the calling thread
// (cudaSetDevice): the driver's tensor-map encoder works in the thread's current
// context, which a thread that has made no call binding one yet (torch's autograd
// worker thread, say) lacks.  Every entry point that launches a TMA kernel calls it.
cudaError_t bind_device(int *device);

// Per-device properties, cached on first use.
int sm_count(int device);
int max_smem_optin(int device);

// SIMT (CUDA-core, fp32 arithmetic) chunked forward.
bool simt_supported(const ChunkArgs &a, int device);
bool bwd_supported(const BwdArgs &a, int device);
cudaError_t launch_phi_copy(TensorView src, TensorView dst, int64_t B, int64_t T, int64_t H, int64_t D, int phi,
                            int dtype, cudaStream_t stream);
cudaError_t launch_aug_v(TensorView v, void *vp, int64_t B, int64_t T, int64_t H, int dv, int dvp, int dtype,
                         cudaStream_t stream);
cudaError_t launch_norm_grad_num(TensorView dout, void *up, int64_t B, int64_t T, int64_t H, int dv, int dvp,
                                 int dtype, cudaStream_t stream);
cudaError_t launch_norm_grad_out(TensorView dout, const void *o, const float *den, void *up, int64_t B, int64_t T,
                                 int64_t H, int dv, int dvp, cudaStream_t stream);
cudaError_t launch_dg_rev_cumsum(float *dg, const int32_t *cu_seqlens, int64_t n_seqs, int64_t T, int64_t H,
                                 cudaStream_t stream);
cudaError_t launch_norm_gate(TensorView o, TensorView g, TensorView y, const float *w, float eps, int64_t B,
                             int64_t T, int64_t H, int dv, int dtype, cudaStream_t stream);
cudaError_t launch_bwd(const BwdArgs &a, cudaStream_t stream);
cudaError_t launch_delta(const DeltaArgs &a, cudaStream_t stream);
cudaError_t launch_chunk_simt(const ChunkArgs &a, cudaStream_t stream);

// One-token decode step.
bool step_supported(const StepArgs &a);
cudaError_t launch_step(const StepArgs &a, cudaStream_t stream);

// Tensor-core (tcgen05 / TMA / TMEM) chunked forward for bf16.
bool tc_supported(const ChunkArgs &a);
bool tc_can_fuse_norm_gate(const ChunkArgs &a);
bool tc_shape(int dk, int dv);  // head dims the tensor-core kernel takes
size_t tc_workspace_bytes(int64_t B, int64_t T, int64_t H, int dk, int dv, int64_t n_seqs,
                          bool varlen, int chunk);
cudaError_t launch_chunk_tc(const ChunkArgs &a, void *workspace, size_t workspace_bytes,
                            cudaStream_t stream, const char **why);
// Device error words of the tensor-core kernel (timeouts of bounded waits).
cudaError_t tc_device_error(unsigned int *flags, unsigned int *where, bool reset);

// [B, T, H, D] bf16 view as a 4-D TMA map with dims (D, H, T, B) and a
// (64, 1, C, 1) box, 128-byte swizzle: one box is a [C rows x 64 cols] slab.
bool make_map(CUtensorMap *m, const TensorView &t, int64_t B, int64_t T, int64_t H, int64_t D, int C);

// Chunked gated delta rule on the tensor cores (bf16, d_k = d_v = 128): a
// per-chunk WY pass into the workspace, then one sequential pass per
// (sequence, head).
bool gdn_tc_supported(const DeltaArgs &a);
size_t gdn_workspace_bytes(int64_t B, int64_t T, int64_t H, int dk, int dv, int64_t n_seqs, bool varlen);
cudaError_t launch_gdn_chunk(const DeltaArgs &a, void *workspace, size_t workspace_bytes, cudaStream_t stream,
                             const char **why);
cudaError_t gdn_device_error(unsigned int *flags, unsigned int *where, bool reset);

}  // namespace la
