// Register-blocked fp32 tile products and tile loads shared by the CUDA-core (FFMA) kernels.
#pragma once

#include "gdn_common.cuh"

namespace gdn {

// C(m,n) = (acc ? C(m,n) : 0) + alpha * sum_kk A(m,kk) B(kk,n)
// A(m,kk) = A[m*am + kk*ak], B(kk,n) = B[kk*bk + n*bn], C(m,n) = C[m*ldc + n].
// M and N multiples of 4.  Each thread owns 4x4 outputs: rows 4*tm.., columns tn + j*N/4.
// Ownership depends only on (M, N, blockDim), so back-to-back calls with the same shape
// may accumulate into the same C without a barrier.
__device__ __forceinline__ void mm(int M, int N, int Kd, float* C, int ldc, float alpha, bool acc,
                                   const float* A, int am, int ak, const float* B, int bk, int bn) {
  const int nct = N / 4;
  const int ntile = (M / 4) * nct;
  for (int ti = threadIdx.x; ti < ntile; ti += blockDim.x) {
    const int tm = ti / nct, tn = ti % nct;
    float r[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) r[i][j] = 0.f;
    const float* a0 = A + (size_t)(tm * 4) * am;
    const float* b0 = B + (size_t)tn * bn;
#pragma unroll 4
    for (int kk = 0; kk < Kd; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = a0[(size_t)i * am + (size_t)kk * ak];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = b0[(size_t)(j * nct) * bn + (size_t)kk * bk];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) r[i][j] = fmaf(av[i], bv[j], r[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float* c = C + (size_t)(tm * 4 + i) * ldc + tn + j * nct;
        *c = (acc ? *c : 0.f) + alpha * r[i][j];
      }
  }
}

// Rows [0, L) of a token tile from global (row stride rs), zero rows [L, 64).
template <typename T>
__device__ __forceinline__ void load_rows(float* dst, const T* src, size_t rs, int L, int D,
                                          const float* rowscale = nullptr) {
  for (int i = threadIdx.x; i < CH * D; i += blockDim.x) {
    const int t = i / D, c = i % D;
    float x = t < L ? to_f<T>(src[(size_t)t * rs + c]) : 0.f;
    if (rowscale) x *= rowscale[t];
    dst[i] = x;
  }
}

__device__ __forceinline__ void copy_f(float* dst, const float* src, int n) {
  for (int i = threadIdx.x; i < n; i += blockDim.x) dst[i] = src[i];
}

}  // namespace gdn
