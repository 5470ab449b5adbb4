// Affine maps of states, the arithmetic of the context-parallel exchange.  A segment of a
// sequence maps the state entering it to the state leaving it affinely: in the stored layout
// h[k][v] (K x V), h_end = Mt h_start + Bh, where Mt (K x K) is the state a forward of the
// segment returns from h_start = I with v = 0, and Bh the one it returns from h_start = 0.
// The backward maps the gradient leaving the segment to the one entering it with Mt^T.
// k_state_affine: out[n] = op(A[n]) X[n] + B[n] for count independent (K x K, K x V) pairs,
// op = identity or transpose; one CTA per (pair, 32 columns of X).
#include "gdn_common.cuh"
#include "gdn_launch.h"

namespace gdn {
namespace {

__global__ void __launch_bounds__(256) k_state_affine(int K, int V, const float* __restrict__ A, int transA,
                                                      const float* X, const float* Bm, float* out) {
  const size_t n = blockIdx.x;
  const int v0 = 32 * blockIdx.y, tid = threadIdx.x;
  extern __shared__ float sm[];
  float* sA = sm;                // [K][K+1]  op(A)
  float* sX = sA + K * (K + 1);  // [K][32]   columns v0.. of X
  const float* a = A + n * K * K;
  for (int x = tid; x < K * K; x += blockDim.x) {
    const int r = x / K, c = x % K;  // element (r, c) of A, read in order
    if (transA)
      sA[c * (K + 1) + r] = a[x];
    else
      sA[r * (K + 1) + c] = a[x];
  }
  const float* xs = X + n * K * V;
  for (int x = tid; x < K * 32; x += blockDim.x) sX[x] = xs[(size_t)(x / 32) * V + v0 + x % 32];
  __syncthreads();  // X is read in full before any output is written (out may be X)
  for (int x = tid; x < K * 32; x += blockDim.x) {
    const int r = x / 32, vv = x % 32;
    const size_t o = n * K * V + (size_t)r * V + v0 + vv;
    float acc = Bm ? Bm[o] : 0.f;
    for (int j = 0; j < K; ++j) acc = fmaf(sA[r * (K + 1) + j], sX[j * 32 + vv], acc);
    out[o] = acc;
  }
}

}  // namespace

cudaError_t state_affine(int64_t count, int K, int V, const float* A, bool transA, const float* X,
                         const float* Bm, float* out, cudaStream_t s) {
  if (count == 0) return cudaSuccess;
  const size_t smem = (size_t)(K * (K + 1) + K * 32) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(k_state_affine, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ProfScope ps("state_affine", s);
  k_state_affine<<<dim3((unsigned)count, V / 32), 256, smem, s>>>(K, V, A, transA ? 1 : 0, X, Bm, out);
  return cudaGetLastError();
}

}  // namespace gdn
