// tcgen05 path (bf16).  Not yet enabled: every bf16 call takes the FFMA path.
#include "gdn_tc.h"

namespace gdn {

bool tc_supported(const gdn_dims&) { return false; }
size_t tc_workspace_bytes(const gdn_dims&, size_t, int) { return 0; }
cudaError_t tc_forward(const Problem&, const Args&, const Work&, void*, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t tc_backward(const Problem&, const Args&, const Work&, void*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace gdn
