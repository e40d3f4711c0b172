// la_host.cu -- la_fwd_chunk_host: the chunked forward on host buffers.
//
// A caller whose activations live in host memory (a CPU-side pipeline, a
// serving front end) hands them over as they are: the call copies q, k, v,
// gamma and cu_seqlens into a device arena the caller owns, runs la_fwd_chunk
// on the copies, and copies the output and the final state back, every step
// enqueued on the caller's stream in that order (one cudaMemcpyAsync per
// buffer).  It allocates nothing: the arena's layout is fixed by the problem
// shape (la_fwd_chunk_host_arena_size), with each buffer at a 256-byte
// boundary so the device copies meet the tensor-core path's alignment rules.
#include <cuda_runtime.h>

#include "la_internal.h"

namespace {

constexpr size_t kAlign = 256;

size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

int esize(int32_t dtype) { return dtype == LA_F32 ? 4 : 2; }

// Byte offsets of the device copies inside the arena.
struct Arena {
  size_t q, k, v, out, fs, gamma, cu, ws, total;
};

bool plan(int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv, int64_t n_seqs, int32_t has_cu, int32_t chunk,
          int32_t dtype, int32_t flags, int32_t has_final_state, Arena *a) {
  const size_t ws = la_fwd_chunk_workspace_size(B, T, H, dk, dv, n_seqs, has_cu, chunk, dtype, flags);
  if (ws == (size_t)-1) return false;
  const size_t e = (size_t)esize(dtype), tok = (size_t)(B * T * H);
  size_t o = 0;
  a->q = o;
  o += up(tok * dk * e);
  a->k = o;
  o += up(tok * dk * e);
  a->v = o;
  o += up(tok * dv * e);
  a->out = o;
  o += up(tok * dv * e);
  a->fs = o;
  o += has_final_state ? up((size_t)(n_seqs * H * dk * dv) * sizeof(float)) : 0;
  a->gamma = o;
  o += up((size_t)H * sizeof(float));
  a->cu = o;
  o += has_cu ? up((size_t)(n_seqs + 1) * sizeof(int32_t)) : 0;
  a->ws = o;
  o += up(ws);
  a->total = o;
  return true;
}

bool contiguous(const la_tensor *t) {
  return t && t->stride_h == t->D && t->stride_t == t->H * t->D && t->stride_b == t->T * t->H * t->D;
}

}  // namespace

extern "C" size_t la_fwd_chunk_host_arena_size(int64_t B, int64_t T, int64_t H, int64_t d_k, int64_t d_v,
                                               int64_t n_seqs, int32_t has_cu_seqlens, int32_t chunk,
                                               int32_t dtype, int32_t flags, int32_t has_final_state) {
  Arena a;
  if (!plan(B, T, H, d_k, d_v, n_seqs, has_cu_seqlens, chunk, dtype, flags, has_final_state, &a)) return (size_t)-1;
  return a.total;
}

extern "C" la_status la_fwd_chunk_host(const la_tensor *q, const la_tensor *k, const la_tensor *v,
                                       const float *gamma, const int32_t *cu_seqlens, int64_t n_seqs,
                                       int32_t chunk, int32_t phi, int32_t normalize, const la_tensor *out,
                                       float *final_state, int32_t flags, void *arena, size_t arena_bytes,
                                       void *stream) {
  using la::report_error;
  if (!q || !k || !v || !out) return report_error(LA_ERR_INVALID_ARG, "la_fwd_chunk_host: NULL tensor descriptor");
  if (!contiguous(q) || !contiguous(k) || !contiguous(v) || !contiguous(out))
    return report_error(LA_ERR_INVALID_ARG, "la_fwd_chunk_host: host tensors must be contiguous [B, T, H, D]");
  if (!gamma) return report_error(LA_ERR_INVALID_ARG, "la_fwd_chunk_host: gamma is NULL");
  Arena a;
  if (!plan(q->B, q->T, q->H, q->D, v->D, n_seqs, cu_seqlens != nullptr, chunk, q->dtype, flags,
            final_state != nullptr, &a))
    return report_error(LA_ERR_UNSUPPORTED, "la_fwd_chunk_host: la_fwd_chunk rejects this shape, chunk or dtype");
  if (!arena || arena_bytes < a.total)
    return report_error(LA_ERR_WORKSPACE, "la_fwd_chunk_host: arena missing or smaller than "
                                          "la_fwd_chunk_host_arena_size");
  if (((uintptr_t)arena) % kAlign) return report_error(LA_ERR_INVALID_ARG, "la_fwd_chunk_host: arena not 256-byte aligned");
  uint8_t *base = static_cast<uint8_t *>(arena);
  // device views: the same shapes, contiguous, in the arena
  auto dev = [&](const la_tensor *t, size_t off) {
    la_tensor d = *t;
    d.data = base + off;
    return d;
  };
  const la_tensor dq = dev(q, a.q), dk = dev(k, a.k), dv = dev(v, a.v), dout = dev(out, a.out);
  const size_t e = (size_t)esize(q->dtype), tok = (size_t)(q->B * q->T * q->H);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  struct Copy {
    void *dst;
    const void *src;
    size_t bytes;
  };
  const Copy in[5] = {{dq.data, q->data, tok * q->D * e},
                      {dk.data, k->data, tok * k->D * e},
                      {dv.data, v->data, tok * v->D * e},
                      {base + a.gamma, gamma, (size_t)q->H * sizeof(float)},
                      {base + a.cu, cu_seqlens, cu_seqlens ? (size_t)(n_seqs + 1) * sizeof(int32_t) : 0}};
  for (const Copy &c : in) {
    if (!c.bytes) continue;
    if (!c.src) return report_error(LA_ERR_INVALID_ARG, "la_fwd_chunk_host: NULL host data pointer");
    const cudaError_t err = cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyHostToDevice, st);
    if (err != cudaSuccess) return report_error(LA_ERR_CUDA, "la_fwd_chunk_host: host-to-device copy failed");
  }
  const la_status s = la_fwd_chunk(&dq, &dk, &dv, reinterpret_cast<const float *>(base + a.gamma),
                                   cu_seqlens ? reinterpret_cast<const int32_t *>(base + a.cu) : nullptr, n_seqs,
                                   chunk, phi, normalize, &dout,
                                   final_state ? reinterpret_cast<float *>(base + a.fs) : nullptr, flags,
                                   base + a.ws, a.total - a.ws, stream);
  if (s != LA_OK) return s;  // la_fwd_chunk's message stays in la_last_error
  const Copy back[2] = {{out->data, dout.data, tok * out->D * e},
                        {final_state, base + a.fs,
                         final_state ? (size_t)(n_seqs * q->H * q->D * v->D) * sizeof(float) : 0}};
  for (const Copy &c : back) {
    if (!c.bytes) continue;
    if (!c.dst) return report_error(LA_ERR_INVALID_ARG, "la_fwd_chunk_host: NULL host data pointer");
    const cudaError_t err = cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyDeviceToHost, st);
    if (err != cudaSuccess) return report_error(LA_ERR_CUDA, "la_fwd_chunk_host: device-to-host copy failed");
  }
  return LA_OK;
}
