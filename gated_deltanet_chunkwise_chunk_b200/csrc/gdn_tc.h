// tcgen05 (5th-generation tensor core) path for bf16 tensors.
#pragma once

#include <cuda_runtime.h>

#include "gdn.h"
#include "gdn_common.cuh"

namespace gdn {

// True when the tcgen05 kernels cover these dimensions (bf16, K = V = 128).
bool tc_supported(const gdn_dims& d);
// True when the tcgen05 backward kernels cover them as well.
bool tc_bwd_supported(const gdn_dims& d);
// True when the driver's tensor-map encoder is available.  Shapes the tcgen05 path covers
// never fall back to the CUDA-core kernels: without the encoder their calls fail with
// GDN_ERR_UNSUPPORTED.
bool tc_ready();
// Bytes of the tcgen05 path's own workspace region for NC chunks.
size_t tc_workspace_bytes(const gdn_dims& d, size_t NC, int pass);
cudaError_t tc_forward(const Problem& p, const Args& a, const Work& w, void* tc_ws, cudaStream_t s);
// reuse_fwd: the tcgen05 region still holds the forward's intermediates for these inputs.
cudaError_t tc_backward(const Problem& p, const Args& a, const Work& w, void* tc_ws,
                        bool reuse_fwd, cudaStream_t s);

}  // namespace gdn
