// Placeholder until the tcgen05 prefill kernel lands: every call takes the SIMT kernel.
#include "internal.h"

namespace sdpa {

bool prefill_supported(const Problem&, const void*, const void*, const void*, const void*) {
  return false;
}
size_t prefill_workspace_bytes(const Problem&) { return 0; }
cudaError_t launch_prefill(const Problem&, const void*, const void*, const void*, void*, void*,
                           cudaStream_t, const char** msg) {
  if (msg) *msg = "prefill kernel not built";
  return cudaErrorNotSupported;
}

}  // namespace sdpa
