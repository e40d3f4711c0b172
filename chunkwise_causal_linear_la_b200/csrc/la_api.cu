// la_api.cu -- the C ABI of include/la_b200.h: argument validation, kernel
// selection and launch.  No allocation, no synchronisation, no exceptions.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>

#include "la_internal.h"

namespace la {
namespace {

thread_local char g_msg[512];

la_status fail(la_status s, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof g_msg, fmt, ap);
  va_end(ap);
  return s;
}

la_status ok() {
  g_msg[0] = 0;
  return LA_OK;
}

constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];
std::atomic<int> g_smem_optin[kMaxDevices];

int elem_size(int dtype) { return dtype == LA_F32 ? 4 : 2; }

bool head_dim_ok(int64_t d) { return d == 16 || d == 32 || d == 64 || d == 128 || d == 256; }

// Shape, stride and alignment checks common to every tensor argument.
la_status check_tensor(const la_tensor *t, const char *name) {
  if (!t) return fail(LA_ERR_INVALID_ARG, "%s: NULL tensor descriptor", name);
  if (t->dtype != LA_F32 && t->dtype != LA_BF16)
    return fail(LA_ERR_INVALID_ARG, "%s: dtype %d is not LA_F32 or LA_BF16", name, t->dtype);
  if (t->B < 0 || t->T < 0 || t->H < 0 || t->D <= 0)
    return fail(LA_ERR_INVALID_ARG, "%s: negative or zero size", name);
  if (t->stride_b < 0 || t->stride_t < 0 || t->stride_h < 0)
    return fail(LA_ERR_INVALID_ARG, "%s: negative stride", name);
  const int64_t numel = t->B * t->T * t->H;
  if (numel > 0 && !t->data) return fail(LA_ERR_INVALID_ARG, "%s: NULL data pointer", name);
  const int es = elem_size(t->dtype);
  if (((uintptr_t)t->data) % 16 != 0)
    return fail(LA_ERR_INVALID_ARG, "%s: data pointer not 16-byte aligned", name);
  if ((t->stride_b * es) % 16 || (t->stride_t * es) % 16 || (t->stride_h * es) % 16)
    return fail(LA_ERR_INVALID_ARG, "%s: strides must be multiples of 16 bytes", name);
  return LA_OK;
}

TensorView view(const la_tensor *t) { return TensorView{t->data, t->stride_b, t->stride_t, t->stride_h}; }

}  // namespace

la_status report_error(la_status status, const char *msg) {
  snprintf(g_msg, sizeof g_msg, "%s", msg);
  return status;
}

int sm_count(int device) {
  if (device < 0 || device >= kMaxDevices) return 148;
  int v = g_sm_count[device].load(std::memory_order_relaxed);
  if (v <= 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || v <= 0) v = 148;
    g_sm_count[device].store(v, std::memory_order_relaxed);
  }
  return v;
}

cudaError_t bind_device(int *device) {
  cudaError_t e = cudaGetDevice(device);
  if (e == cudaSuccess) e = cudaSetDevice(*device);
  return e;
}

int max_smem_optin(int device) {
  if (device < 0 || device >= kMaxDevices) return 232448;
  int v = g_smem_optin[device].load(std::memory_order_relaxed);
  if (v <= 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, device) != cudaSuccess || v <= 0)
      v = 232448;
    g_smem_optin[device].store(v, std::memory_order_relaxed);
  }
  return v;
}

}  // namespace la

using namespace la;

namespace {

// Output norm and gate requested by la_fwd_chunk_normgate (NULL w: none).
struct NormGate {
  const la_tensor *gate = nullptr;
  const float *w = nullptr;
  float eps = 0.f;
};

la_status fwd_common(const la_tensor *q, const la_tensor *k, const la_tensor *v, const float *gamma,
                     const float *g, const int32_t *cu_seqlens, int64_t n_seqs, int32_t chunk, int32_t phi,
                     int32_t normalize, const la_tensor *out, float *final_state, float *final_z,
                     int32_t flags, void *workspace, size_t workspace_bytes, void *stream,
                     const NormGate &ng = NormGate()) {
  la_status s;
  if ((s = check_tensor(q, "q")) != LA_OK) return s;
  if ((s = check_tensor(k, "k")) != LA_OK) return s;
  if ((s = check_tensor(v, "v")) != LA_OK) return s;
  if ((s = check_tensor(out, "out")) != LA_OK) return s;
  if (k->dtype != q->dtype || v->dtype != q->dtype || out->dtype != q->dtype)
    return fail(LA_ERR_INVALID_ARG, "q, k, v and out must share one dtype");
  if (k->B != q->B || v->B != q->B || out->B != q->B || k->T != q->T || v->T != q->T ||
      out->T != q->T || k->H != q->H || v->H != q->H || out->H != q->H)
    return fail(LA_ERR_INVALID_ARG, "q, k, v, out disagree on B, T or H");
  if (k->D != q->D) return fail(LA_ERR_INVALID_ARG, "q and k must have the same head dim d_k");
  if (out->D != v->D) return fail(LA_ERR_INVALID_ARG, "out and v must have the same head dim d_v");
  if (q->H <= 0) return fail(LA_ERR_INVALID_ARG, "H must be positive");
  if (phi != LA_PHI_IDENTITY && phi != LA_PHI_ELU1) return fail(LA_ERR_INVALID_ARG, "phi %d unknown", phi);
  if (flags & ~LA_FLAG_SIMT) return fail(LA_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  if (cu_seqlens) {
    if (q->B != 1) return fail(LA_ERR_INVALID_ARG, "packed batches (cu_seqlens) need B == 1");
    if (n_seqs < 0) return fail(LA_ERR_INVALID_ARG, "n_seqs is negative");
  } else if (n_seqs != q->B) {
    return fail(LA_ERR_INVALID_ARG, "n_seqs must equal B when cu_seqlens is NULL");
  }
  if (((uintptr_t)final_state) % 16 != 0) return fail(LA_ERR_INVALID_ARG, "final_state not 16-byte aligned");
  if (((uintptr_t)final_z) % 16 != 0) return fail(LA_ERR_INVALID_ARG, "final_z not 16-byte aligned");
  if (final_z && !normalize) return fail(LA_ERR_INVALID_ARG, "final_z needs normalize");
  if (chunk != 16 && chunk != 32 && chunk != 64 && chunk != 128)
    return fail(LA_ERR_UNSUPPORTED, "chunk %d not in {16, 32, 64, 128}", chunk);
  if (!head_dim_ok(q->D) || !head_dim_ok(v->D))
    return fail(LA_ERR_UNSUPPORTED, "head dims (%lld, %lld) not in {16, 32, 64, 128, 256}",
                (long long)q->D, (long long)v->D);

  ChunkArgs a;
  a.q = view(q);
  a.k = view(k);
  a.v = view(v);
  a.out = out->data;
  a.o_sb = out->stride_b;
  a.o_st = out->stride_t;
  a.o_sh = out->stride_h;
  a.gamma = gamma;
  a.g = g;
  a.cu_seqlens = cu_seqlens;
  a.final_state = final_state;
  a.final_z = final_z;
  a.B = q->B;
  a.T = q->T;
  a.n_seqs = n_seqs;
  a.H = (int)q->H;
  a.dk = (int)q->D;
  a.dv = (int)v->D;
  a.chunk = chunk;
  a.phi = phi;
  a.normalize = normalize ? 1 : 0;
  a.dtype = q->dtype;
  a.rev = 0;
  a.noseg = 0;
  a.ex = TensorView{nullptr, 0, 0, 0};
  a.edg = nullptr;
  a.esign = 0.f;
  a.ephi = a.edphi = 0;
  a.den_out = nullptr;
  a.ng_w = nullptr;
  a.ng_gate = TensorView{nullptr, 0, 0, 0};
  a.ng_eps = 0.f;
  if (ng.w) {
    if ((s = check_tensor(ng.gate, "gate")) != LA_OK) return s;
    if (ng.gate->dtype != q->dtype || ng.gate->B != out->B || ng.gate->T != out->T || ng.gate->H != out->H ||
        ng.gate->D != out->D)
      return fail(LA_ERR_INVALID_ARG, "gate must have out's shape and dtype");
    if (!(ng.eps >= 0.f)) return fail(LA_ERR_INVALID_ARG, "eps must be >= 0");
  }

  const size_t need = la_fwd_chunk_workspace_size(a.B, a.T, a.H, a.dk, a.dv, n_seqs, cu_seqlens != nullptr,
                                                  chunk, a.dtype, flags);
  if (need > 0 && (workspace_bytes < need || !workspace))
    return fail(LA_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace_bytes);
  if (workspace && ((uintptr_t)workspace) % 256 != 0)
    return fail(LA_ERR_INVALID_ARG, "workspace not 256-byte aligned");

  cudaStream_t st = (cudaStream_t)stream;
  int device = 0;
  cudaError_t err = bind_device(&device);
  if (err != cudaSuccess) return fail(LA_ERR_CUDA, "cudaGetDevice / cudaSetDevice: %s", cudaGetErrorString(err));

  // No token to process: only the final states (all zero) remain to be written.
  if (a.n_seqs == 0) return ok();
  if (a.T == 0 || a.B == 0) {
    if (final_state) {
      err = cudaMemsetAsync(final_state, 0, (size_t)a.n_seqs * a.H * a.dk * a.dv * sizeof(float), st);
      if (err != cudaSuccess) return fail(LA_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(err));
    }
    if (final_z) {
      err = cudaMemsetAsync(final_z, 0, (size_t)a.n_seqs * a.H * a.dk * sizeof(float), st);
      if (err != cudaSuccess) return fail(LA_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(err));
    }
    return ok();
  }

  const bool use_tc = a.dtype == LA_BF16 && !(flags & LA_FLAG_SIMT) && tc_supported(a);
  const bool fuse_ng = ng.w && use_tc && tc_can_fuse_norm_gate(a);
  if (fuse_ng) {
    a.ng_w = ng.w;
    a.ng_gate = view(ng.gate);
    a.ng_eps = ng.eps;
  }
  if (use_tc) {
    const char *why = nullptr;
    err = launch_chunk_tc(a, workspace, workspace_bytes, st, &why);
    if (err != cudaSuccess)
      return fail(LA_ERR_CUDA, "tensor-core chunk kernel: %s%s%s", cudaGetErrorString(err), why ? ": " : "",
                  why ? why : "");
  } else {
    if (!simt_supported(a, device))
      return fail(LA_ERR_UNSUPPORTED, "chunk %d with d_k %d does not fit the CUDA-core kernel's shared memory",
                  chunk, a.dk);
    err = launch_chunk_simt(a, st);
    if (err != cudaSuccess) return fail(LA_ERR_CUDA, "CUDA-core chunk kernel: %s", cudaGetErrorString(err));
  }
  if (ng.w && !fuse_ng) {  // the norm and gate as a second pass over out, in place
    err = launch_norm_gate(view(out), view(ng.gate), view(out), ng.w, ng.eps, out->B, out->T, out->H,
                           (int)out->D, q->dtype, st);
    if (err != cudaSuccess) return fail(LA_ERR_CUDA, "output norm kernel: %s", cudaGetErrorString(err));
  }
  return ok();
}

// Shared by la_step and la_step_norm (z == NULL: no normaliser).
la_status step_common(const char *name, const la_tensor *q, const la_tensor *k, const la_tensor *v,
                      const float *gamma, const float *g, float *state, float *z, const la_tensor *out,
                      int32_t phi, void *stream) {
  la_status s;
  if ((s = check_tensor(q, "q")) != LA_OK) return s;
  if ((s = check_tensor(k, "k")) != LA_OK) return s;
  if ((s = check_tensor(v, "v")) != LA_OK) return s;
  if ((s = check_tensor(out, "out")) != LA_OK) return s;
  if (k->dtype != q->dtype || v->dtype != q->dtype || out->dtype != q->dtype)
    return fail(LA_ERR_INVALID_ARG, "q, k, v and out must share one dtype");
  if (q->T != 1 || k->T != 1 || v->T != 1 || out->T != 1)
    return fail(LA_ERR_INVALID_ARG, "%s takes exactly one token (T == 1)", name);
  if (k->B != q->B || v->B != q->B || out->B != q->B || k->H != q->H || v->H != q->H || out->H != q->H)
    return fail(LA_ERR_INVALID_ARG, "q, k, v, out disagree on N or H");
  if (k->D != q->D || out->D != v->D) return fail(LA_ERR_INVALID_ARG, "head dims disagree");
  if (!gamma && !g) return fail(LA_ERR_INVALID_ARG, "%s is NULL", g ? "g" : "gamma");
  if (((uintptr_t)g) % 4 != 0) return fail(LA_ERR_INVALID_ARG, "g not 4-byte aligned");
  if (q->B * q->H > 0 && !state) return fail(LA_ERR_INVALID_ARG, "state is NULL");
  if (((uintptr_t)state) % 16 != 0) return fail(LA_ERR_INVALID_ARG, "state not 16-byte aligned");
  if (((uintptr_t)z) % 16 != 0) return fail(LA_ERR_INVALID_ARG, "z not 16-byte aligned");
  if (phi != LA_PHI_IDENTITY && phi != LA_PHI_ELU1) return fail(LA_ERR_INVALID_ARG, "phi %d unknown", phi);

  StepArgs a;
  a.q = view(q);
  a.k = view(k);
  a.v = view(v);
  a.out = out->data;
  a.o_sb = out->stride_b;
  a.o_sh = out->stride_h;
  a.gamma = gamma;
  a.g = g;
  a.state = state;
  a.z = z;
  a.N = q->B;
  a.H = (int)q->H;
  a.dk = (int)q->D;
  a.dv = (int)v->D;
  a.phi = phi;
  a.dtype = q->dtype;
  if (a.dk > 256 || a.dv > 256 || !step_supported(a))
    return fail(LA_ERR_UNSUPPORTED, "%s needs d_k <= 256 and d_v a power of two in [4, 256]", name);
  cudaError_t err = launch_step(a, (cudaStream_t)stream);
  if (err != cudaSuccess) return fail(LA_ERR_CUDA, "decode kernel: %s", cudaGetErrorString(err));
  return ok();
}

}  // namespace

extern "C" {

const char *la_status_string(int32_t status) {
  switch (status) {
    case LA_OK: return "LA_OK";
    case LA_ERR_INVALID_ARG: return "LA_ERR_INVALID_ARG: invalid argument";
    case LA_ERR_UNSUPPORTED: return "LA_ERR_UNSUPPORTED: valid but not implemented";
    case LA_ERR_WORKSPACE: return "LA_ERR_WORKSPACE: workspace missing or too small";
    case LA_ERR_CUDA: return "LA_ERR_CUDA: CUDA call or launch failed";
    default: return "unknown la_status";
  }
}

const char *la_last_error(void) { return g_msg; }

int32_t la_version(void) { return 1 * 10000 + 0 * 100 + 0; }

la_status la_device_error(uint32_t *flags, uint32_t *detail, int32_t reset) {
  if (!flags || !detail) return fail(LA_ERR_INVALID_ARG, "flags and detail must not be NULL");
  unsigned int f = 0, w = 0, f2 = 0, w2 = 0;
  cudaError_t err = tc_device_error(&f, &w, reset != 0);
  if (err == cudaSuccess) err = gdn_device_error(&f2, &w2, reset != 0);
  if (err != cudaSuccess) return fail(LA_ERR_CUDA, "reading the device error word: %s", cudaGetErrorString(err));
  *flags = f | f2;
  *detail = w ? w : w2;
  return ok();
}

size_t la_fwd_chunk_workspace_size(int64_t B, int64_t T, int64_t H, int64_t d_k, int64_t d_v,
                                   int64_t n_seqs, int32_t has_cu_seqlens, int32_t chunk,
                                   int32_t dtype, int32_t flags) {
  if (B < 0 || T < 0 || H <= 0 || n_seqs < 0 || !head_dim_ok(d_k) || !head_dim_ok(d_v))
    return (size_t)-1;
  if (chunk != 16 && chunk != 32 && chunk != 64 && chunk != 128) return (size_t)-1;
  if (dtype != LA_F32 && dtype != LA_BF16) return (size_t)-1;
  if (dtype == LA_F32 || (flags & LA_FLAG_SIMT)) return 0;
  return tc_workspace_bytes(B, T, H, (int)d_k, (int)d_v, n_seqs, has_cu_seqlens != 0, chunk);
}

int32_t la_fwd_chunk_path(int64_t d_k, int64_t d_v, int64_t T, int64_t H, int32_t chunk, int32_t dtype,
                          int32_t flags) {
  if (!head_dim_ok(d_k) || !head_dim_ok(d_v) || T < 0 || H <= 0) return -1;
  if (chunk != 16 && chunk != 32 && chunk != 64 && chunk != 128) return -1;
  if ((dtype != LA_F32 && dtype != LA_BF16) || (flags & ~LA_FLAG_SIMT)) return -1;
  ChunkArgs a{};
  a.dtype = dtype;
  a.chunk = chunk;
  a.dk = (int)d_k;
  a.dv = (int)d_v;
  a.T = T;
  a.H = (int)H;
  if (dtype == LA_BF16 && !(flags & LA_FLAG_SIMT) && tc_supported(a)) return LA_PATH_TENSOR_CORE;
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) device = 0;
  return simt_supported(a, device) ? LA_PATH_CUDA_CORE : -1;
}

la_status la_fwd_chunk(const la_tensor *q, const la_tensor *k, const la_tensor *v, const float *gamma,
                       const int32_t *cu_seqlens, int64_t n_seqs, int32_t chunk, int32_t phi,
                       int32_t normalize, const la_tensor *out, float *final_state, int32_t flags,
                       void *workspace, size_t workspace_bytes, void *stream) {
  return la_fwd_chunk_z(q, k, v, gamma, cu_seqlens, n_seqs, chunk, phi, normalize, out, final_state, nullptr,
                        flags, workspace, workspace_bytes, stream);
}

la_status la_fwd_chunk_z(const la_tensor *q, const la_tensor *k, const la_tensor *v, const float *gamma,
                         const int32_t *cu_seqlens, int64_t n_seqs, int32_t chunk, int32_t phi,
                         int32_t normalize, const la_tensor *out, float *final_state, float *final_z,
                         int32_t flags, void *workspace, size_t workspace_bytes, void *stream) {
  if (!gamma) return fail(LA_ERR_INVALID_ARG, "gamma is NULL");
  return fwd_common(q, k, v, gamma, nullptr, cu_seqlens, n_seqs, chunk, phi, normalize, out, final_state, final_z,
                    flags, workspace, workspace_bytes, stream);
}

la_status la_fwd_chunk_gated(const la_tensor *q, const la_tensor *k, const la_tensor *v, const float *g,
                             const int32_t *cu_seqlens, int64_t n_seqs, int32_t chunk, int32_t phi,
                             int32_t normalize, const la_tensor *out, float *final_state, float *final_z,
                             int32_t flags, void *workspace, size_t workspace_bytes, void *stream) {
  if (!g && q && q->B * q->T * q->H > 0) return fail(LA_ERR_INVALID_ARG, "g is NULL");
  if (((uintptr_t)g) % 4 != 0) return fail(LA_ERR_INVALID_ARG, "g not 4-byte aligned");
  return fwd_common(q, k, v, nullptr, g, cu_seqlens, n_seqs, chunk, phi, normalize, out, final_state, final_z,
                    flags, workspace, workspace_bytes, stream);
}

la_status la_fwd_chunk_normgate(const la_tensor *q, const la_tensor *k, const la_tensor *v, const float *gamma,
                                const int32_t *cu_seqlens, int64_t n_seqs, int32_t chunk, int32_t phi,
                                int32_t normalize, const la_tensor *gate, const float *w, float eps,
                                const la_tensor *out, float *final_state, int32_t flags, void *workspace,
                                size_t workspace_bytes, void *stream) {
  if (!gamma) return fail(LA_ERR_INVALID_ARG, "gamma is NULL");
  if (!w) return fail(LA_ERR_INVALID_ARG, "w is NULL");
  if (!gate) return fail(LA_ERR_INVALID_ARG, "gate: NULL tensor descriptor");
  NormGate ng;
  ng.gate = gate;
  ng.w = w;
  ng.eps = eps;
  return fwd_common(q, k, v, gamma, nullptr, cu_seqlens, n_seqs, chunk, phi, normalize, out, final_state, nullptr,
                    flags, workspace, workspace_bytes, stream, ng);
}

}  // extern "C"

namespace {

// Validation shared by the two gated-delta entry points; fills `a`.
la_status delta_setup(const la_tensor *q, const la_tensor *k, const la_tensor *v, const float *g,
                      const float *beta, const int32_t *cu_seqlens, int64_t n_seqs, const float *initial_state,
                      const la_tensor *out, float *final_state, DeltaArgs &a) {
  la_status s;
  const la_tensor *ts[4] = {q, k, v, out};
  const char *names[4] = {"q", "k", "v", "out"};
  for (int i = 0; i < 4; ++i)
    if ((s = check_tensor(ts[i], names[i])) != LA_OK) return s;
  for (int i = 1; i < 4; ++i) {
    if (ts[i]->dtype != q->dtype) return fail(LA_ERR_INVALID_ARG, "%s must have q's dtype", names[i]);
    if (ts[i]->B != q->B || ts[i]->T != q->T || ts[i]->H != q->H)
      return fail(LA_ERR_INVALID_ARG, "%s disagrees with q on B, T or H", names[i]);
  }
  if (k->D != q->D || out->D != v->D) return fail(LA_ERR_INVALID_ARG, "head dims disagree");
  if (q->H <= 0) return fail(LA_ERR_INVALID_ARG, "H must be positive");
  const int64_t rows = q->B * q->T * q->H;
  if (rows > 0 && (!g || !beta)) return fail(LA_ERR_INVALID_ARG, "g or beta is NULL");
  if (((uintptr_t)g) % 4 || ((uintptr_t)beta) % 4 || ((uintptr_t)initial_state) % 4 || ((uintptr_t)final_state) % 4)
    return fail(LA_ERR_INVALID_ARG, "g, beta, initial_state and final_state must be 4-byte aligned");
  if (cu_seqlens) {
    if (q->B != 1) return fail(LA_ERR_INVALID_ARG, "packed batches (cu_seqlens) need B == 1");
    if (n_seqs < 0) return fail(LA_ERR_INVALID_ARG, "n_seqs is negative");
  } else if (n_seqs != q->B) {
    return fail(LA_ERR_INVALID_ARG, "n_seqs must equal B when cu_seqlens is NULL");
  }
  if (!head_dim_ok(q->D) || !head_dim_ok(v->D))
    return fail(LA_ERR_UNSUPPORTED, "head dims (%lld, %lld) not in {16, 32, 64, 128, 256}",
                (long long)q->D, (long long)v->D);
  a.q = view(q);
  a.k = view(k);
  a.v = view(v);
  a.out = out->data;
  a.o_sb = out->stride_b;
  a.o_st = out->stride_t;
  a.o_sh = out->stride_h;
  a.g = g;
  a.beta = beta;
  a.init = initial_state;
  a.final_state = final_state;
  a.cu_seqlens = cu_seqlens;
  a.T = q->T;
  a.n_seqs = n_seqs;
  a.H = (int)q->H;
  a.dk = (int)q->D;
  a.dv = (int)v->D;
  a.dtype = q->dtype;
  return LA_OK;
}

}  // namespace

extern "C" {

la_status la_fwd_gated_delta(const la_tensor *q, const la_tensor *k, const la_tensor *v, const float *g,
                             const float *beta, const int32_t *cu_seqlens, int64_t n_seqs,
                             const float *initial_state, const la_tensor *out, float *final_state, void *stream) {
  DeltaArgs a;
  la_status s = delta_setup(q, k, v, g, beta, cu_seqlens, n_seqs, initial_state, out, final_state, a);
  if (s != LA_OK) return s;
  if (n_seqs == 0) return ok();
  const cudaError_t err = launch_delta(a, (cudaStream_t)stream);
  if (err != cudaSuccess) return fail(LA_ERR_CUDA, "gated delta kernel: %s", cudaGetErrorString(err));
  return ok();
}

la_status la_fwd_gated_delta_chunk(const la_tensor *q, const la_tensor *k, const la_tensor *v, const float *g,
                                   const float *beta, const int32_t *cu_seqlens, int64_t n_seqs,
                                   const float *initial_state, const la_tensor *out, float *final_state,
                                   int32_t flags, void *workspace, size_t workspace_bytes, void *stream) {
  DeltaArgs a;
  la_status s = delta_setup(q, k, v, g, beta, cu_seqlens, n_seqs, initial_state, out, final_state, a);
  if (s != LA_OK) return s;
  if (flags & ~(LA_FLAG_SIMT | LA_FLAG_TEST_WAIT_TIMEOUT))
    return fail(LA_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  a.test_wait_timeout = (flags & LA_FLAG_TEST_WAIT_TIMEOUT) != 0;
  if (n_seqs == 0) return ok();
  cudaError_t err;
  const bool states16 = ((uintptr_t)initial_state) % 16 == 0 && ((uintptr_t)final_state) % 16 == 0;
  if (!(flags & LA_FLAG_SIMT) && gdn_tc_supported(a) && states16) {
    const size_t need = gdn_workspace_bytes(q->B, q->T, q->H, a.dk, a.dv, n_seqs, cu_seqlens != nullptr);
    if (workspace_bytes < need || (need > 0 && !workspace))
      return fail(LA_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed (la_fwd_gated_delta_workspace_size)",
                  workspace_bytes, need);
    if (((uintptr_t)workspace) % 256) return fail(LA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    int device = 0;
    if ((err = bind_device(&device)) != cudaSuccess)
      return fail(LA_ERR_CUDA, "cudaGetDevice / cudaSetDevice: %s", cudaGetErrorString(err));
    const char *why = nullptr;
    err = launch_gdn_chunk(a, workspace, workspace_bytes, (cudaStream_t)stream, &why);
    if (err != cudaSuccess)
      return fail(LA_ERR_CUDA, "chunked gated delta: %s%s%s", cudaGetErrorString(err), why ? ": " : "",
                  why ? why : "");
    return ok();
  }
  err = launch_delta(a, (cudaStream_t)stream);
  if (err != cudaSuccess) return fail(LA_ERR_CUDA, "gated delta kernel: %s", cudaGetErrorString(err));
  return ok();
}

size_t la_fwd_gated_delta_workspace_size(int64_t B, int64_t T, int64_t H, int64_t d_k, int64_t d_v,
                                         int64_t n_seqs, int32_t has_cu_seqlens, int32_t dtype, int32_t flags) {
  if (B < 0 || T < 0 || H <= 0 || n_seqs < 0 || !head_dim_ok(d_k) || !head_dim_ok(d_v)) return (size_t)-1;
  if (dtype != LA_F32 && dtype != LA_BF16) return (size_t)-1;
  if (flags & ~(LA_FLAG_SIMT | LA_FLAG_TEST_WAIT_TIMEOUT)) return (size_t)-1;
  if (dtype == LA_F32 || (flags & LA_FLAG_SIMT)) return 0;
  return gdn_workspace_bytes(B, T, H, (int)d_k, (int)d_v, n_seqs, has_cu_seqlens != 0);
}

la_status la_norm_gate(const la_tensor *o, const la_tensor *gate, const float *w, float eps, const la_tensor *y,
                       void *stream) {
  la_status s;
  if ((s = check_tensor(o, "o")) != LA_OK) return s;
  if ((s = check_tensor(gate, "gate")) != LA_OK) return s;
  if ((s = check_tensor(y, "y")) != LA_OK) return s;
  for (const la_tensor *t : {gate, y})
    if (t->dtype != o->dtype || t->B != o->B || t->T != o->T || t->H != o->H || t->D != o->D)
      return fail(LA_ERR_INVALID_ARG, "gate and y must have o's shape and dtype");
  if (!w) return fail(LA_ERR_INVALID_ARG, "w is NULL");
  if (!(eps >= 0.f)) return fail(LA_ERR_INVALID_ARG, "eps must be >= 0");
  const cudaError_t err = launch_norm_gate(view(o), view(gate), view(y), w, eps, o->B, o->T, o->H, (int)o->D,
                                           o->dtype, (cudaStream_t)stream);
  if (err != cudaSuccess) return fail(LA_ERR_CUDA, "output norm kernel: %s", cudaGetErrorString(err));
  return ok();
}

// The backward of la_fwd_chunk (g == NULL: per-head decay gamma) or of
// la_fwd_chunk_gated's unnormalised form (g: per-token log decay; dg receives
// its gradient).
static la_status bwd_common(const la_tensor *q, const la_tensor *k, const la_tensor *v, const la_tensor *dout,
                            const float *gamma, const float *g, float *dg, const int32_t *cu_seqlens, int64_t n_seqs,
                            int32_t chunk, int32_t phi, const la_tensor *dq, const la_tensor *dk, const la_tensor *dv,
                            int32_t flags, void *stream) {
  la_status s;
  const la_tensor *ts[7] = {q, k, v, dout, dq, dk, dv};
  const char *names[7] = {"q", "k", "v", "dout", "dq", "dk", "dv"};
  for (int i = 0; i < 7; ++i)
    if ((s = check_tensor(ts[i], names[i])) != LA_OK) return s;
  for (int i = 1; i < 7; ++i) {
    if (ts[i]->dtype != q->dtype) return fail(LA_ERR_INVALID_ARG, "%s must have q's dtype", names[i]);
    if (ts[i]->B != q->B || ts[i]->T != q->T || ts[i]->H != q->H)
      return fail(LA_ERR_INVALID_ARG, "%s disagrees with q on B, T or H", names[i]);
  }
  if (k->D != q->D || dq->D != q->D || dk->D != q->D) return fail(LA_ERR_INVALID_ARG, "d_k disagrees");
  if (dout->D != v->D || dv->D != v->D) return fail(LA_ERR_INVALID_ARG, "d_v disagrees");
  if (q->H <= 0) return fail(LA_ERR_INVALID_ARG, "H must be positive");
  if (!gamma && !g && q->B * q->T * q->H > 0) return fail(LA_ERR_INVALID_ARG, "gamma is NULL");
  if (g && (!dg || ((uintptr_t)g) % 4 || ((uintptr_t)dg) % 4))
    return fail(LA_ERR_INVALID_ARG, "g and dg must be non-NULL, 4-byte aligned [B, T, H] float arrays");
  if (phi != LA_PHI_IDENTITY && phi != LA_PHI_ELU1) return fail(LA_ERR_INVALID_ARG, "phi %d unknown", phi);
  if (flags & ~LA_FLAG_SIMT) return fail(LA_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  if (cu_seqlens) {
    if (q->B != 1) return fail(LA_ERR_INVALID_ARG, "packed batches (cu_seqlens) need B == 1");
    if (n_seqs < 0) return fail(LA_ERR_INVALID_ARG, "n_seqs is negative");
  } else if (n_seqs != q->B) {
    return fail(LA_ERR_INVALID_ARG, "n_seqs must equal B when cu_seqlens is NULL");
  }
  if (chunk != 16 && chunk != 32 && chunk != 64 && chunk != 128)
    return fail(LA_ERR_UNSUPPORTED, "chunk %d not in {16, 32, 64, 128}", chunk);
  if (!head_dim_ok(q->D) || !head_dim_ok(v->D))
    return fail(LA_ERR_UNSUPPORTED, "head dims (%lld, %lld) not in {16, 32, 64, 128, 256}",
                (long long)q->D, (long long)v->D);
  BwdArgs a;
  a.q = view(q);
  a.k = view(k);
  a.v = view(v);
  a.dout = view(dout);
  a.dq = view(dq);
  a.dk_ = view(dk);
  a.dv_ = view(dv);
  a.gamma = gamma;
  a.g = g;
  a.dg = g ? dg : nullptr;
  a.cu_seqlens = cu_seqlens;
  a.T = q->T;
  a.n_seqs = n_seqs;
  a.H = (int)q->H;
  a.dk = (int)q->D;
  a.dv = (int)v->D;
  a.chunk = chunk;
  a.phi = phi;
  a.dtype = q->dtype;
  int device = 0;
  cudaError_t err = bind_device(&device);
  if (err != cudaSuccess) return fail(LA_ERR_CUDA, "cudaGetDevice / cudaSetDevice: %s", cudaGetErrorString(err));
  if (a.n_seqs == 0 || a.T == 0 || q->B == 0) return ok();
  cudaStream_t st = (cudaStream_t)stream;

  // Tensor cores: the backward is three forward passes on rearranged operands
  // (each a sum of the forward's form, two of them anti-causal, run in reverse
  // time):  dphi(q) = fwd(dout, v, phi(k));  dphi(k) = rev(v, dout, phi(q));
  // dv = rev(phi(k), phi(q), dout).  With elu + 1 the operands the forward
  // reads untransformed are made phi(x) first (in dq / dv, which are written
  // after they are read), and phi' scales the q and k gradients.
  const bool elu = phi == LA_PHI_ELU1;
  ChunkArgs f;
  f.gamma = gamma;
  f.g = g;
  f.cu_seqlens = cu_seqlens;
  f.final_state = nullptr;
  f.final_z = nullptr;
  f.B = q->B;
  f.T = q->T;
  f.n_seqs = n_seqs;
  f.H = (int)q->H;
  f.chunk = 64;
  f.normalize = 0;
  f.dtype = q->dtype;
  f.noseg = 1;
  f.ng_w = nullptr;
  f.ng_gate = TensorView{nullptr, 0, 0, 0};
  f.ng_eps = 0.f;
  f.ex = TensorView{nullptr, 0, 0, 0};
  f.edg = nullptr;
  f.esign = 0.f;
  f.ephi = f.edphi = 0;
  f.den_out = nullptr;
  auto setup = [&](const la_tensor *qq, const la_tensor *kk, const la_tensor *vv, const la_tensor *oo, int ph,
                   int rev) {
    f.q = view(qq);
    f.k = view(kk);
    f.v = view(vv);
    f.out = oo->data;
    f.o_sb = oo->stride_b;
    f.o_st = oo->stride_t;
    f.o_sh = oo->stride_h;
    f.dk = (int)qq->D;
    f.dv = (int)vv->D;
    f.phi = ph;
    f.rev = rev;
    return tc_supported(f);
  };
  bool tc = q->dtype == LA_BF16 && chunk == 64 && !(flags & LA_FLAG_SIMT) && (!elu || q->D == v->D);
  if (tc) tc = setup(v, dout, q, dk, 0, 1) && setup(dout, v, k, dq, 0, 0) && setup(k, q, dout, dv, 1, 1);
  if (tc) {
    const char *why = nullptr;
    // x: the forward input whose gradient this pass produces (k for dphi(k), q for dphi(q)); the
    // pass's epilogue then scales by phi'(x) (elu + 1) and, with a per-token decay, adds the row
    // term of dg_t = sum_{s>=t} (phi(q_s) . dphi(q)_s - phi(k_s) . dphi(k)_s), both from the fp32
    // accumulators before rounding
    auto run = [&](const la_tensor *qq, const la_tensor *kk, const la_tensor *vv, const la_tensor *oo, int ph,
                   int rev, const la_tensor *x = nullptr, float sign = 0.f) -> cudaError_t {
      setup(qq, kk, vv, oo, ph, rev);
      f.ex = x ? view(x) : TensorView{nullptr, 0, 0, 0};
      f.edg = x && g ? dg : nullptr;
      f.esign = sign;
      f.ephi = phi;
      f.edphi = elu ? 1 : 0;
      const cudaError_t e = launch_chunk_tc(f, nullptr, 0, st, &why);
      f.ex = TensorView{nullptr, 0, 0, 0};
      f.edg = nullptr;
      return e;
    };
    const int64_t B = q->B, T = q->T, H = q->H, Dk = q->D;
    const bool epi = g || elu;  // the dk and dq passes need x in their epilogue
    if (g && (err = cudaMemsetAsync(dg, 0, (size_t)(B * T * H) * sizeof(float), st)) != cudaSuccess)
      return fail(LA_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(err));
    if (elu) {
      if ((err = launch_phi_copy(view(q), view(dq), B, T, H, Dk, 1, q->dtype, st)) != cudaSuccess ||
          (err = run(v, dout, dq, dk, 0, 1, k, -1.f)) != cudaSuccess ||
          (err = launch_phi_copy(view(k), view(dv), B, T, H, Dk, 1, q->dtype, st)) != cudaSuccess ||
          (err = run(dout, v, dv, dq, 0, 0, q, 1.f)) != cudaSuccess ||
          (err = run(k, q, dout, dv, 1, 1)) != cudaSuccess)
        return fail(LA_ERR_CUDA, "backward (tensor cores): %s%s%s", cudaGetErrorString(err), why ? ": " : "",
                    why ? why : "");
    } else {
      if ((err = run(v, dout, q, dk, 0, 1, epi ? k : nullptr, -1.f)) != cudaSuccess ||
          (err = run(dout, v, k, dq, 0, 0, epi ? q : nullptr, 1.f)) != cudaSuccess ||
          (err = run(k, q, dout, dv, 0, 1)) != cudaSuccess)
        return fail(LA_ERR_CUDA, "backward (tensor cores): %s%s%s", cudaGetErrorString(err), why ? ": " : "",
                    why ? why : "");
    }
    if (g && (err = launch_dg_rev_cumsum(dg, cu_seqlens, n_seqs, T, H, st)) != cudaSuccess)
      return fail(LA_ERR_CUDA, "backward (log decay gradient): %s", cudaGetErrorString(err));
    return ok();
  }
  if (!bwd_supported(a, device))
    return fail(LA_ERR_UNSUPPORTED, "d_k %d x d_v %d does not fit the backward kernel's shared memory", a.dk,
                a.dv);
  if (g && (err = cudaMemsetAsync(dg, 0, (size_t)(q->B * q->T * q->H) * sizeof(float), st)) != cudaSuccess)
    return fail(LA_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(err));
  err = launch_bwd(a, st);
  if (err != cudaSuccess) return fail(LA_ERR_CUDA, "backward kernel: %s", cudaGetErrorString(err));
  if (g && (err = launch_dg_rev_cumsum(dg, cu_seqlens, n_seqs, q->T, q->H, st)) != cudaSuccess)
    return fail(LA_ERR_CUDA, "backward (log decay gradient): %s", cudaGetErrorString(err));
  return ok();
}

la_status la_bwd_chunk(const la_tensor *q, const la_tensor *k, const la_tensor *v, const la_tensor *dout,
                       const float *gamma, const int32_t *cu_seqlens, int64_t n_seqs, int32_t chunk, int32_t phi,
                       const la_tensor *dq, const la_tensor *dk, const la_tensor *dv, int32_t flags,
                       void *stream) {
  return bwd_common(q, k, v, dout, gamma, nullptr, nullptr, cu_seqlens, n_seqs, chunk, phi, dq, dk, dv, flags,
                    stream);
}

la_status la_bwd_chunk_gated(const la_tensor *q, const la_tensor *k, const la_tensor *v, const la_tensor *dout,
                             const float *g, const int32_t *cu_seqlens, int64_t n_seqs, int32_t chunk, int32_t phi,
                             const la_tensor *dq, const la_tensor *dk, const la_tensor *dv, float *dg, int32_t flags,
                             void *stream) {
  if (!g && q && q->B * q->T * q->H > 0) return fail(LA_ERR_INVALID_ARG, "g is NULL");
  return bwd_common(q, k, v, dout, nullptr, g, dg, cu_seqlens, n_seqs, chunk, phi, dq, dk, dv, flags, stream);
}

// The backward of la_fwd_chunk's normalised form (o_t = num_t / den_t) through the
// unnormalised backward of an augmented problem.  With the value rows widened to
// v'_t = [v_t, 1, 1, 0...] and the output gradient to u'_t = [u_t, e_t, 0...],
// u_t = dout_t / den_t and e_t = -(u_t . o_t) (the denominator's adjoint, carried
// as a pair e_hi + e_lo over the two columns of ones), the unnormalised backward
// of (q, k, v', u') gives dq and dk of the normalised recurrence, and dv as the
// first d_v columns of dv'.
//   Tensor cores (bf16, chunk 64): the normalised forward (o, and den_t from its
//   epilogue), v' and u' (row passes), then the three passes of la_bwd_chunk with
//   u' as the output gradient; the dv pass reads only u''s first d_v columns.
//   CUDA cores (f32, other chunks, LA_FLAG_SIMT): the unnormalised forward of
//   (q, k, v') gives [num, den, den, 0...], turned into u' in place; the backward
//   kernel on (q, k, v', u') writes dv' to the workspace, and a copy takes dv.
namespace {

// Widths of the augmented value rows: d_v + 2 rounded up to a head dim the
// kernels take (tensor cores: 128 or 256 as the key width of the widened passes).
int64_t norm_aug_width(int64_t dv) { return dv >= 16 && dv <= 128 && (dv & (dv - 1)) == 0 ? 2 * dv : -1; }

struct NormBwdWs {
  bool tc;  // the tensor-core route
  // byte offsets: v', u' (both routes); o, den, phi(k) (tensor cores); dv' (CUDA cores); total size
  size_t vp, up, o, den, kh, dvw, total;
};

bool norm_bwd_plan(int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv, int32_t chunk, int32_t dtype,
                   int32_t flags, NormBwdWs *w) {
  const int64_t dvp = norm_aug_width(dv);
  if ((dtype != LA_BF16 && dtype != LA_F32) || dvp < 0 || B < 0 || T < 0 || H <= 0 || (flags & ~LA_FLAG_SIMT))
    return false;
  if (chunk != 16 && chunk != 32 && chunk != 64 && chunk != 128) return false;
  if (!head_dim_ok(dk) || !head_dim_ok(dvp)) return false;
  w->tc = dtype == LA_BF16 && chunk == 64 && !(flags & LA_FLAG_SIMT) && tc_shape((int)dvp, (int)dk) &&
          tc_shape((int)dk, (int)dv);
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t rows = (size_t)(B * T * H), es = dtype == LA_F32 ? 4 : 2;
  w->vp = 0;
  w->up = up(rows * dvp * es);
  const size_t end = w->up + up(rows * dvp * es);
  if (w->tc) {
    w->o = end;
    w->den = w->o + up(rows * dv * es);
    w->kh = w->den + up(rows * 4);
    w->total = w->kh + up(rows * dk * es);
    w->dvw = 0;
  } else {
    w->dvw = end;
    w->total = w->dvw + up(rows * dvp * es);
    w->o = w->den = w->kh = 0;
  }
  return true;
}

}  // namespace

size_t la_bwd_chunk_norm_workspace_size(int64_t B, int64_t T, int64_t H, int64_t d_k, int64_t d_v, int32_t chunk,
                                        int32_t dtype, int32_t flags) {
  NormBwdWs w;
  return norm_bwd_plan(B, T, H, d_k, d_v, chunk, dtype, flags, &w) ? w.total : (size_t)-1;
}

// Shared by la_bwd_chunk_norm (g == NULL: per-head decay gamma) and
// la_bwd_chunk_gated_norm (g: per-token log decays; dg receives their gradient,
// which the widened backward passes give as for la_bwd_chunk_gated: the loss sees
// g only through the weights of num and den, both outputs of the widened problem).
static la_status norm_bwd_common(const la_tensor *q, const la_tensor *k, const la_tensor *v, const la_tensor *dout,
                                 const float *gamma, const float *g, float *dg, const int32_t *cu_seqlens,
                                 int64_t n_seqs, int32_t chunk, int32_t phi, const la_tensor *dq, const la_tensor *dk,
                                 const la_tensor *dv, int32_t flags, void *workspace, size_t workspace_bytes,
                                 void *stream) {
  la_status s;
  const la_tensor *ts[7] = {q, k, v, dout, dq, dk, dv};
  const char *names[7] = {"q", "k", "v", "dout", "dq", "dk", "dv"};
  for (int i = 0; i < 7; ++i)
    if ((s = check_tensor(ts[i], names[i])) != LA_OK) return s;
  for (int i = 1; i < 7; ++i) {
    if (ts[i]->dtype != q->dtype) return fail(LA_ERR_INVALID_ARG, "%s must have q's dtype", names[i]);
    if (ts[i]->B != q->B || ts[i]->T != q->T || ts[i]->H != q->H)
      return fail(LA_ERR_INVALID_ARG, "%s disagrees with q on B, T or H", names[i]);
  }
  if (k->D != q->D || dq->D != q->D || dk->D != q->D) return fail(LA_ERR_INVALID_ARG, "d_k disagrees");
  if (dout->D != v->D || dv->D != v->D) return fail(LA_ERR_INVALID_ARG, "d_v disagrees");
  if (q->H <= 0) return fail(LA_ERR_INVALID_ARG, "H must be positive");
  if (!gamma && !g && q->B * q->T * q->H > 0) return fail(LA_ERR_INVALID_ARG, "gamma is NULL");
  if (g && (!dg || ((uintptr_t)g) % 4 || ((uintptr_t)dg) % 4))
    return fail(LA_ERR_INVALID_ARG, "g and dg must be non-NULL, 4-byte aligned [B, T, H] float arrays");
  if (phi != LA_PHI_IDENTITY && phi != LA_PHI_ELU1) return fail(LA_ERR_INVALID_ARG, "phi %d unknown", phi);
  if (flags & ~LA_FLAG_SIMT) return fail(LA_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  if (cu_seqlens) {
    if (q->B != 1) return fail(LA_ERR_INVALID_ARG, "packed batches (cu_seqlens) need B == 1");
    if (n_seqs < 0) return fail(LA_ERR_INVALID_ARG, "n_seqs is negative");
  } else if (n_seqs != q->B) {
    return fail(LA_ERR_INVALID_ARG, "n_seqs must equal B when cu_seqlens is NULL");
  }
  NormBwdWs w;
  if (!norm_bwd_plan(q->B, q->T, q->H, q->D, v->D, chunk, q->dtype, flags, &w))
    return fail(LA_ERR_UNSUPPORTED, "the normalised backward takes d_v in {16, 32, 64, 128}, d_k in "
                "{16, 32, 64, 128, 256} and chunk in {16, 32, 64, 128}");
  if (w.total > 0 && (!workspace || workspace_bytes < w.total))  // an empty problem needs none
    return fail(LA_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", w.total, workspace_bytes);
  if (((uintptr_t)workspace) % 256 != 0) return fail(LA_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  int device = 0;
  cudaError_t err = bind_device(&device);
  if (err != cudaSuccess) return fail(LA_ERR_CUDA, "cudaGetDevice / cudaSetDevice: %s", cudaGetErrorString(err));
  if (n_seqs == 0 || q->T == 0 || q->B == 0) return ok();

  const int64_t B = q->B, T = q->T, H = q->H, Dk = q->D, Dv = v->D, Dvp = norm_aug_width(Dv);
  uint8_t *base = static_cast<uint8_t *>(workspace);
  // contiguous [B, T, H, D] buffers of q's dtype in the workspace
  auto buf = [&](size_t off, int64_t D) {
    la_tensor t;
    t.data = base + off;
    t.dtype = q->dtype;
    t.B = B;
    t.T = T;
    t.H = H;
    t.D = D;
    t.stride_h = D;
    t.stride_t = H * D;
    t.stride_b = T * H * D;
    return t;
  };
  const la_tensor vp = buf(w.vp, Dvp), up = buf(w.up, Dvp);
  const bool elu = phi == LA_PHI_ELU1;
  cudaStream_t st = (cudaStream_t)stream;

  ChunkArgs f;
  f.gamma = gamma;
  f.g = g;
  f.cu_seqlens = cu_seqlens;
  f.final_state = nullptr;
  f.final_z = nullptr;
  f.B = B;
  f.T = T;
  f.n_seqs = n_seqs;
  f.H = (int)H;
  f.chunk = chunk;
  f.normalize = 0;
  f.dtype = q->dtype;
  f.rev = 0;
  f.noseg = 1;
  f.ng_w = nullptr;
  f.ng_gate = TensorView{nullptr, 0, 0, 0};
  f.ng_eps = 0.f;
  f.ex = TensorView{nullptr, 0, 0, 0};
  f.edg = nullptr;
  f.esign = 0.f;
  f.ephi = f.edphi = 0;
  f.den_out = nullptr;
  auto set_io = [&](const la_tensor *qq, const la_tensor *kk, const la_tensor *vv, const la_tensor *oo) {
    f.q = view(qq);
    f.k = view(kk);
    f.v = view(vv);
    f.out = oo->data;
    f.o_sb = oo->stride_b;
    f.o_st = oo->stride_t;
    f.o_sh = oo->stride_h;
    f.dk = (int)qq->D;
    f.dv = (int)vv->D;
  };

  if (!w.tc) {  // ---- CUDA cores
    const la_tensor dvw = buf(w.dvw, Dvp);
    set_io(q, k, &vp, &up);
    f.phi = phi;
    BwdArgs b;
    b.q = view(q);
    b.k = view(k);
    b.v = view(&vp);
    b.dout = view(&up);
    b.dq = view(dq);
    b.dk_ = view(dk);
    b.dv_ = view(&dvw);
    b.gamma = gamma;
    b.cu_seqlens = cu_seqlens;
    b.T = T;
    b.n_seqs = n_seqs;
    b.H = (int)H;
    b.dk = (int)Dk;
    b.dv = (int)Dvp;
    b.chunk = chunk;
    b.phi = phi;
    b.dtype = q->dtype;
    b.g = g;
    b.dg = g ? dg : nullptr;
    if (!simt_supported(f, device) || !bwd_supported(b, device))
      return fail(LA_ERR_UNSUPPORTED, "d_k %lld x widened d_v %lld does not fit the CUDA-core kernels' shared "
                  "memory", (long long)Dk, (long long)Dvp);
    la_tensor dv_head = dvw;  // dv' seen as its first d_v columns
    dv_head.D = Dv;
    if ((err = launch_aug_v(view(v), vp.data, B, T, H, (int)Dv, (int)Dvp, q->dtype, st)) != cudaSuccess ||
        (err = launch_chunk_simt(f, st)) != cudaSuccess ||
        (err = launch_norm_grad_num(view(dout), up.data, B, T, H, (int)Dv, (int)Dvp, q->dtype, st)) !=
            cudaSuccess ||
        (g && (err = cudaMemsetAsync(dg, 0, (size_t)(B * T * H) * sizeof(float), st)) != cudaSuccess) ||
        (err = launch_bwd(b, st)) != cudaSuccess ||
        (err = launch_phi_copy(view(&dv_head), view(dv), B, T, H, Dv, LA_PHI_IDENTITY, q->dtype, st)) !=
            cudaSuccess ||
        (g && (err = launch_dg_rev_cumsum(dg, cu_seqlens, n_seqs, T, H, st)) != cudaSuccess))
      return fail(LA_ERR_CUDA, "normalised backward (CUDA cores): %s", cudaGetErrorString(err));
    return ok();
  }

  // ---- tensor cores
  const la_tensor o = buf(w.o, Dv), kh = buf(w.kh, Dk);
  float *den = reinterpret_cast<float *>(base + w.den);
  la_tensor u_head = up;  // u' seen as its first d_v columns: dout / den
  u_head.D = Dv;
  const char *why = nullptr;
  // one tensor-core pass: out = fwd or rev(qq, kk, vv) with feature map ph on qq and kk; x (the
  // input whose gradient this pass produces) makes the epilogue scale by phi'(x)
  auto run = [&](const la_tensor *qq, const la_tensor *kk, const la_tensor *vv, const la_tensor *oo, int ph,
                 int rev, const la_tensor *x) -> cudaError_t {
    set_io(qq, kk, vv, oo);
    f.phi = ph;
    f.rev = rev;
    // x: the input whose gradient this pass produces; the epilogue scales by phi'(x) (elu + 1)
    // and, with a per-token decay, adds the row term sign * phi(x) . dphi(x) to dg
    f.ex = x && (elu || g) ? view(x) : TensorView{nullptr, 0, 0, 0};
    f.edg = x && g ? dg : nullptr;
    f.esign = x == k ? -1.f : 1.f;
    f.ephi = phi;
    f.edphi = x && elu ? 1 : 0;
    if (!tc_supported(f)) return cudaErrorInvalidValue;
    const cudaError_t e = launch_chunk_tc(f, nullptr, 0, st, &why);
    f.ex = TensorView{nullptr, 0, 0, 0};
    f.edg = nullptr;
    return e;
  };
  // the normalised forward (o, and den_t from its epilogue), then u'
  f.normalize = 1;
  f.den_out = den;
  err = run(q, k, v, &o, phi, 0, nullptr);
  f.normalize = 0;
  f.den_out = nullptr;
  if (err != cudaSuccess ||
      (err = launch_aug_v(view(v), vp.data, B, T, H, (int)Dv, (int)Dvp, q->dtype, st)) != cudaSuccess ||
      (err = launch_norm_grad_out(view(dout), o.data, den, up.data, B, T, H, (int)Dv, (int)Dvp, st)) !=
          cudaSuccess)
    return fail(LA_ERR_CUDA, "normalised backward (forward and output gradient): %s%s%s", cudaGetErrorString(err),
                why ? ": " : "", why ? why : "");
  // dphi(k) = rev(v', u', phi(q)); dphi(q) = fwd(u', v', phi(k)); dv = rev(phi(k), phi(q), u'[:d_v]).
  // With elu + 1, phi(q) is staged in dq (written after it is read) and phi(k) in the workspace.
  const la_tensor *qh = elu ? dq : q, *khp = elu ? &kh : k;
  if ((g && (err = cudaMemsetAsync(dg, 0, (size_t)(B * T * H) * sizeof(float), st)) != cudaSuccess) ||
      (elu && (err = launch_phi_copy(view(q), view(dq), B, T, H, Dk, 1, q->dtype, st)) != cudaSuccess) ||
      (err = run(&vp, &up, qh, dk, 0, 1, k)) != cudaSuccess ||
      (elu && (err = launch_phi_copy(view(k), view(&kh), B, T, H, Dk, 1, q->dtype, st)) != cudaSuccess) ||
      (err = run(&up, &vp, khp, dq, 0, 0, q)) != cudaSuccess ||
      (err = run(k, q, &u_head, dv, phi, 1, nullptr)) != cudaSuccess ||
      (g && (err = launch_dg_rev_cumsum(dg, cu_seqlens, n_seqs, T, H, st)) != cudaSuccess))
    return fail(LA_ERR_CUDA, "normalised backward (tensor cores): %s%s%s", cudaGetErrorString(err),
                why ? ": " : "", why ? why : "");
  return ok();
}

la_status la_bwd_chunk_norm(const la_tensor *q, const la_tensor *k, const la_tensor *v, const la_tensor *dout,
                            const float *gamma, const int32_t *cu_seqlens, int64_t n_seqs, int32_t chunk, int32_t phi,
                            const la_tensor *dq, const la_tensor *dk, const la_tensor *dv, int32_t flags,
                            void *workspace, size_t workspace_bytes, void *stream) {
  return norm_bwd_common(q, k, v, dout, gamma, nullptr, nullptr, cu_seqlens, n_seqs, chunk, phi, dq, dk, dv, flags,
                         workspace, workspace_bytes, stream);
}

la_status la_bwd_chunk_gated_norm(const la_tensor *q, const la_tensor *k, const la_tensor *v, const la_tensor *dout,
                                  const float *g, const int32_t *cu_seqlens, int64_t n_seqs, int32_t chunk,
                                  int32_t phi, const la_tensor *dq, const la_tensor *dk, const la_tensor *dv, float *dg,
                                  int32_t flags, void *workspace, size_t workspace_bytes, void *stream) {
  if (!g && q && q->B * q->T * q->H > 0) return fail(LA_ERR_INVALID_ARG, "g is NULL");
  return norm_bwd_common(q, k, v, dout, nullptr, g, dg, cu_seqlens, n_seqs, chunk, phi, dq, dk, dv, flags,
                         workspace, workspace_bytes, stream);
}

size_t la_bwd_chunk_gated_norm_workspace_size(int64_t B, int64_t T, int64_t H, int64_t d_k, int64_t d_v,
                                              int32_t chunk, int32_t dtype, int32_t flags) {
  return la_bwd_chunk_norm_workspace_size(B, T, H, d_k, d_v, chunk, dtype, flags);
}

la_status la_step(const la_tensor *q, const la_tensor *k, const la_tensor *v, const float *gamma, float *state,
                  const la_tensor *out, int32_t phi, void *stream) {
  return step_common("la_step", q, k, v, gamma, nullptr, state, nullptr, out, phi, stream);
}

la_status la_step_norm(const la_tensor *q, const la_tensor *k, const la_tensor *v, const float *gamma,
                       float *state, float *z, const la_tensor *out, int32_t phi, void *stream) {
  if (q && k && q->B * q->H > 0 && !z) return fail(LA_ERR_INVALID_ARG, "z is NULL");
  return step_common("la_step_norm", q, k, v, gamma, nullptr, state, z, out, phi, stream);
}

la_status la_step_gated(const la_tensor *q, const la_tensor *k, const la_tensor *v, const float *g, float *state,
                        float *z, const la_tensor *out, int32_t phi, void *stream) {
  if (!g && q && q->B * q->H > 0) return fail(LA_ERR_INVALID_ARG, "g is NULL");
  return step_common("la_step_gated", q, k, v, nullptr, g, state, z, out, phi, stream);
}

}  // extern "C"
