// la_noalloc.cu -- la_fwd_chunk_noalloc: the chunked forward for callers that
// cannot allocate device memory.
//
// Some callers run where allocating is not allowed or not affordable: a plugin
// executing inside a framework that owns every byte of device memory and hands
// out none at execution time, or a latency-critical serving loop where
// cudaMalloc may synchronise the device.  la_fwd_chunk needs scratch memory
// (the segment states of long sequences) that its caller normally allocates;
// this entry point instead uses one statically sized array that the library
// places in device memory when it is loaded.
//
// The array is shared by every call on a device and keeps the previous call's
// contents.  Nothing in it has to start at zero: the state pass writes every
// slot the scan and the output pass read.  Two calls whose work overlaps on
// the GPU (different streams, or different host threads on one device) race on
// the array; callers must order them.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "la_internal.h"

namespace {

static_assert(LA_NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch size");

// The scratch itself: every GPU that loads the library holds it until exit.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LA_NOALLOC_SCRATCH_BYTES];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

// cuCtxGetCurrent from the driver, looked up once through the runtime (no -lcuda).
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
// Device address of g_noalloc_scratch per device, with the context it was looked up
// in: the array is placed anew whenever the device's context is recreated (after
// cudaDeviceReset, for one), so an address is reused only in the context it came from.
void *g_scratch_addr[kMaxDevices];
CUcontext g_scratch_ctx[kMaxDevices];

// In host code g_noalloc_scratch names a host-side stand-in, not device memory:
// the device address is looked up with that device current, once per device and
// context (the first call on a device, or the first after its context changed).
cudaError_t scratch_address(int device, void **out) {
  if (device < 0 || device >= kMaxDevices) return cudaErrorInvalidDevice;
  CtxGetCurrentFn get = ctx_get_current();
  if (!get) return cudaErrorInitializationError;
  CUcontext ctx = nullptr;  // NULL until the runtime has made a context current on this thread
  if (get(&ctx) != CUDA_SUCCESS) return cudaErrorInitializationError;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!ctx || !g_scratch_addr[device] || g_scratch_ctx[device] != ctx) {
    void *p = nullptr;
    const cudaError_t err = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // sets the context up if needed
    if (err != cudaSuccess) return err;
    if (!ctx && (get(&ctx) != CUDA_SUCCESS || !ctx)) return cudaErrorInitializationError;
    g_scratch_addr[device] = p;
    g_scratch_ctx[device] = ctx;
  }
  *out = g_scratch_addr[device];
  return cudaSuccess;
}

}  // namespace

extern "C" la_status la_fwd_chunk_noalloc(const la_tensor *q, const la_tensor *k, const la_tensor *v,
                                          const float *gamma, const int32_t *cu_seqlens, int64_t n_seqs,
                                          int32_t chunk, int32_t phi, int32_t normalize, const la_tensor *out,
                                          float *final_state, int32_t flags, void *stream) {
  if (!q || !k || !v || !out) return la_fwd_chunk(q, k, v, gamma, cu_seqlens, n_seqs, chunk, phi, normalize, out,
                                                  final_state, flags, nullptr, 0, stream);
  const size_t need = la_fwd_chunk_workspace_size(q->B, q->T, q->H, q->D, v->D, n_seqs, cu_seqlens != nullptr,
                                                  chunk, q->dtype, flags);
  if (need == (size_t)-1 || need == 0)  // rejected or no scratch needed: the ordinary call reports / runs it
    return la_fwd_chunk(q, k, v, gamma, cu_seqlens, n_seqs, chunk, phi, normalize, out, final_state, flags,
                        nullptr, 0, stream);
  if (need > LA_NOALLOC_SCRATCH_BYTES)
    return la::report_error(LA_ERR_WORKSPACE,
                            "la_fwd_chunk_noalloc: this problem needs more scratch than the built-in "
                            "LA_NOALLOC_SCRATCH_BYTES; call la_fwd_chunk with a workspace instead");
  int device = 0;
  void *scratch = nullptr;
  if (cudaGetDevice(&device) != cudaSuccess)
    return la::report_error(LA_ERR_CUDA, "la_fwd_chunk_noalloc: cudaGetDevice failed");
  if (scratch_address(device, &scratch) != cudaSuccess)
    return la::report_error(LA_ERR_CUDA, "la_fwd_chunk_noalloc: cudaGetSymbolAddress of the scratch array failed");
  return la_fwd_chunk(q, k, v, gamma, cu_seqlens, n_seqs, chunk, phi, normalize, out, final_state, flags, scratch,
                      LA_NOALLOC_SCRATCH_BYTES, stream);
}
