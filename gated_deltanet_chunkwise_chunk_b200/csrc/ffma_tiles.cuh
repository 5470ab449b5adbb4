// Register-blocked fp32 tile products and tile loads shared by the CUDA-core (FFMA) kernels.
#pragma once

#include "gdn_common.cuh"

namespace gdn {

// C(m,n) = (acc ? C(m,n) : 0) + alpha * sum_kk A(m,kk) B(kk,n)
// A(m,kk) = A[m*am + kk*ak], B(kk,n) = B[kk*bk + n*bn], C(m,n) = C[m*ldc + n].
// M and N multiples of 4.  Each thread owns 4x4 outputs: rows 4*tm.., columns tn + j*N/4.
// Ownership depends only on (M, N, blockDim), so back-to-back calls with the same shape
// may accumulate into the same C without a barrier.  tri = 1: A is lower triangular (A(m,kk) = 0
// for kk > m), tri = 2: upper (A(m,kk) = 0 for kk < m); the loop skips those exact zeros.
__device__ __forceinline__ void mm(int M, int N, int Kd, float* C, int ldc, float alpha, bool acc,
                                   const float* A, int am, int ak, const float* B, int bk, int bn,
                                   int tri = 0) {
  const int nct = N / 4;
  const int ntile = (M / 4) * nct;
  for (int ti = threadIdx.x; ti < ntile; ti += blockDim.x) {
    const int tm = ti / nct, tn = ti % nct;
    const int k0 = tri == 2 ? min(Kd, 4 * tm) : 0, k1 = tri == 1 ? min(Kd, 4 * tm + 4) : Kd;
    float r[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) r[i][j] = 0.f;
    const float* a0 = A + (size_t)(tm * 4) * am;
    const float* b0 = B + (size_t)tn * bn;
#pragma unroll 4
    for (int kk = k0; kk < k1; ++kk) {
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

// 16-byte global -> shared copies (cp.async), all in flight until cp_async_wait_all.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;\n" ::: "memory");
}
// n floats (n % 4 == 0, both ends 16-byte aligned), issued by every thread, not waited for
__device__ __forceinline__ void copy_async(float* dst, const float* src, int n) {
  for (int i = threadIdx.x; i < n / 4; i += blockDim.x) cp_async16(dst + 4 * i, src + 4 * i);
}

// Rows [0, L) of a 64 x D token tile (row stride rs elements, D % 8 == 0, 16-byte aligned rows)
// into fp32 shared memory with row stride ldd, rows past L zero.  16-byte loads, all of a
// thread's loads issued before any is used; 256 threads, D <= 128.
template <typename T>
__device__ __forceinline__ void load_tile(float* dst, int ldd, const T* src, size_t rs, int L, int D) {
  constexpr int E = 16 / sizeof(T);       // elements per 16-byte vector
  constexpr int NV = CH * 128 / E / 256;  // vectors per thread at D = 128
  const int nvec = CH * D / E;
  uint4 r[NV];
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int vi = threadIdx.x + 256 * k, t = vi * E / D, c = vi * E % D;
    r[k] = make_uint4(0u, 0u, 0u, 0u);
    if (vi < nvec && t < L) r[k] = __ldg(reinterpret_cast<const uint4*>(src + (size_t)t * rs + c));
  }
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int vi = threadIdx.x + 256 * k;
    if (vi >= nvec) continue;
    float f[E];
    if constexpr (E == 4) {
      const float4 v4 = *reinterpret_cast<const float4*>(&r[k]);
      f[0] = v4.x; f[1] = v4.y; f[2] = v4.z; f[3] = v4.w;
    } else {
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&r[k]);
#pragma unroll
      for (int j = 0; j < E / 2; ++j) {
        const float2 t2 = __bfloat1622float2(h2[j]);
        f[2 * j] = t2.x;
        f[2 * j + 1] = t2.y;
      }
    }
    const int t = vi * E / D, c = vi * E % D;
    float* d = dst + t * ldd + c;
    if (ldd % 4 == 0) {
#pragma unroll
      for (int j = 0; j < E; j += 4) *reinterpret_cast<float4*>(d + j) = make_float4(f[j], f[j + 1], f[j + 2], f[j + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < E; ++j) d[j] = f[j];
    }
  }
}

}  // namespace gdn
