// Host-side launcher declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>

#include "gdn_common.cuh"

namespace gdn {

// Counts a launch and, while profiling is on, brackets it with CUDA events on `s`.
class ProfScope {
 public:
  ProfScope(const char* name, cudaStream_t s);
  ~ProfScope();
  ProfScope(const ProfScope&) = delete;
  ProfScope& operator=(const ProfScope&) = delete;

 private:
  const char* name_;
  cudaStream_t s_;
  cudaEvent_t a_{}, b_{};
  bool active_ = false;
};

cudaError_t launch_chunk_table(const Problem& p, const int64_t* cu, const Work& w, cudaStream_t s);
cudaError_t launch_chunk_table_only(const Problem& p, const int64_t* cu, int4* table, int* count,
                                    cudaStream_t s);
cudaError_t launch_gate_cumsum(const Problem& p, const Args& a, const Work& w, cudaStream_t s);
// dg and dbeta per token, the parameter gradients and (group_sum) dq, dk from per-value-head
// shares; the tensor-core path writes dq and dk itself and passes group_sum = false.
cudaError_t launch_bwd_tokens(const Problem& p, const Args& a, const Work& w, bool bf16,
                              cudaStream_t s, bool group_sum = true);

// fp32 CUDA-core path (FFMA tiles): used for fp32 tensors.
// KDA gate (per-channel gate) forward and backward; dtypes are gdn_dtype codes.
size_t kda_gate_workspace_bytes(int64_t H, int64_t D);
cudaError_t kda_gate_forward(int64_t T, int H, int D, int in_dtype, const void* g, const float* A_log,
                             const float* dt_bias, int out_dtype, void* yg, cudaStream_t s);
cudaError_t kda_gate_backward(int64_t T, int H, int D, int in_dtype, const void* g, const float* A_log,
                              const float* dt_bias, int dy_dtype, const void* dyg, void* dg,
                              float* dA_log, float* ddt_bias, float* part, cudaStream_t s);
// Token-by-token forward (decoding, short prefills); status: device status word.
cudaError_t state_affine(int64_t count, int K, int V, const float* A, bool transA, const float* X,
                         const float* Bm, float* out, cudaStream_t s);
cudaError_t launch_dqdk_group_sum(const Problem& p, const Args& a, const Work& w, bool bf16, cudaStream_t s);
cudaError_t kda_chunk_backward(const Problem& p, const Args& a, const KdaWork& w, bool bf16, cudaStream_t s);
cudaError_t kda_chunk_forward(const Problem& p, const Args& a, const KdaWork& w, bool bf16, cudaStream_t s);
cudaError_t recurrent_forward(const Problem& p, const Args& a, int* status, bool bf16, cudaStream_t s,
                              bool kda = false);
cudaError_t ffma_forward(const Problem& p, const Args& a, const Work& w, bool bf16, bool bwd_prep,
                         cudaStream_t s);
cudaError_t ffma_backward(const Problem& p, const Args& a, const Work& w, bool bf16,
                          cudaStream_t s);

}  // namespace gdn
