// Fused tensor-core prefill (placeholder until the sm_100a kernel lands).
#include "kda_internal.h"

namespace kda {

bool fused_supported(const ChunkArgs&) { return false; }
size_t fused_workspace_bytes(const ChunkArgs&) { return 0; }
int fused_kernel_count(const ChunkArgs&) { return 0; }
cudaError_t launch_fused(const ChunkArgs&, void*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace kda
