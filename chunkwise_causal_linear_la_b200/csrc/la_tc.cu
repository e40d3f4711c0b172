// la_tc.cu -- tensor-core chunk kernel (placeholder until the tcgen05 path lands).
#include "la_internal.h"

namespace la {
bool tc_supported(const ChunkArgs &) { return false; }
size_t tc_workspace_bytes(int64_t, int64_t, int64_t, int, int, int64_t, bool, int) { return 0; }
cudaError_t launch_chunk_tc(const ChunkArgs &, void *, size_t, cudaStream_t, const char **) {
  return cudaErrorNotSupported;
}
}  // namespace la
