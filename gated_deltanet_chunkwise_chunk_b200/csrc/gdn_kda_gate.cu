// KDA gate (per-channel gate of Kimi-style delta attention): for g [T, H, D],
//   yg[t,h,d] = -exp(A_log[h]) * softplus(g[t,h,d] + dt_bias[h*D + d]),
//   softplus(x) = x for x > 20, else log(1 + e^x),
// computed in fp32 and written in the output dtype (MindSpeed-Ops issue 9, "KDA gate",
// sections on the formula and the computation flow).  Its backward for a loss L(yg):
//   dg[t,h,d]       = dyg * (-exp(A_log[h])) * (x > 20 ? 1 : sigmoid(x))
//   dA_log[h]       = sum_{t,d} dyg * yg
//   d dt_bias[h*D+d] = sum_t dg[t,h,d]
// Element-wise and HBM-bound.  The two reductions are deterministic: KG_BLOCKS row blocks
// write per-column partial sums, then one CTA per head adds them in block order and reduces
// its columns by a fixed tree.
#include <cuda_fp16.h>

#include "gdn_common.cuh"
#include "gdn_launch.h"

namespace gdn {
namespace {

constexpr int KG_BLOCKS = 128;  // row blocks of the backward reduction

template <typename T>
__device__ __forceinline__ float ld_any(const void* p, size_t i) {
  return to_f<T>(static_cast<const T*>(p)[i]);
}
template <>
__device__ __forceinline__ float ld_any<__half>(const void* p, size_t i) {
  return __half2float(static_cast<const __half*>(p)[i]);
}
template <typename T>
__device__ __forceinline__ void st_any(void* p, size_t i, float x) {
  static_cast<T*>(p)[i] = from_f<T>(x);
}
template <>
__device__ __forceinline__ void st_any<__half>(void* p, size_t i, float x) {
  static_cast<__half*>(p)[i] = __float2half_rn(x);
}

__device__ __forceinline__ float softplus20(float x) { return x > 20.f ? x : log1pf(expf(x)); }

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256) k_kda_gate_fwd(int64_t n, int H, int D, const void* g,
                                                      const float* A_log, const float* dt_bias,
                                                      void* yg) {
  const int64_t HD = (int64_t)H * D;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c = i % HD;
    const int h = (int)(c / D);
    const float x = ld_any<Tin>(g, i) + (dt_bias ? dt_bias[c] : 0.f);
    st_any<Tout>(yg, i, -expf(A_log[h]) * softplus20(x));
  }
}

// Pass 1: rows [b*rows, (b+1)*rows) of block b; thread column c = threadIdx.x + 256 j.
// dg written per element; per-column partial sums of dyg*yg and of dg to part[b][2][HD].
template <typename Tin, typename Tdy>
__global__ void __launch_bounds__(256) k_kda_gate_bwd_rows(int64_t T, int H, int D,
                                                           const void* __restrict__ g,
                                                           const float* __restrict__ A_log,
                                                           const float* __restrict__ dt_bias,
                                                           const void* __restrict__ dyg,
                                                           void* __restrict__ dg,
                                                           float* __restrict__ part) {
  const int64_t HD = (int64_t)H * D;
  const int64_t rows = (T + KG_BLOCKS - 1) / KG_BLOCKS;
  const int64_t t0 = blockIdx.x * rows, t1 = min(T, t0 + rows);
  for (int64_t c = threadIdx.x; c < HD; c += blockDim.x) {
    const int h = (int)(c / D);
    const float nexp = -expf(A_log[h]), bias = dt_bias ? dt_bias[c] : 0.f;
    float sa = 0.f, sb = 0.f;
    for (int64_t t = t0; t < t1; t += 4) {  // four rows per step: their loads are in flight together
      float x[4], dy[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const bool in = t + r < t1;
        const int64_t i = (t + r) * HD + c;
        x[r] = in ? ld_any<Tin>(g, i) + bias : 0.f;
        dy[r] = in ? ld_any<Tdy>(dyg, i) : 0.f;
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        if (t + r >= t1) break;
        const float dx = dy[r] * nexp * (x[r] > 20.f ? 1.f : 1.f / (1.f + expf(-x[r])));
        st_any<Tin>(dg, (t + r) * HD + c, dx);
        sa += dy[r] * nexp * softplus20(x[r]);  // dyg * yg
        sb += dx;
      }
    }
    part[((int64_t)blockIdx.x * 2) * HD + c] = sa;
    part[((int64_t)blockIdx.x * 2 + 1) * HD + c] = sb;
  }
}

// Pass 2: one CTA per head; column sums over the blocks in order, then a fixed tree over d.
__global__ void __launch_bounds__(256) k_kda_gate_bwd_reduce(int H, int D, const float* part,
                                                             float* dA_log, float* ddt_bias) {
  const int h = blockIdx.x;
  const int64_t HD = (int64_t)H * D;
  __shared__ float red[256];
  float acc = 0.f;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    const int64_t c = (int64_t)h * D + d;
    float sa = 0.f, sb = 0.f;
    for (int b = 0; b < KG_BLOCKS; ++b) {
      sa += part[((int64_t)b * 2) * HD + c];
      sb += part[((int64_t)b * 2 + 1) * HD + c];
    }
    if (ddt_bias) ddt_bias[c] = sb;
    acc += sa;
  }
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int s = 128; s > 0; s >>= 1) {
    if (threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0 && dA_log) dA_log[h] = red[0];
}

template <typename Tin>
cudaError_t fwd_out(int64_t n, int H, int D, const void* g, const float* A_log, const float* dt_bias,
                    int out_dtype, void* yg, cudaStream_t s) {
  const int grid = (int)std::min<int64_t>((n + 255) / 256, 148 * 16);
  if (out_dtype == GDN_DTYPE_FP32)
    k_kda_gate_fwd<Tin, float><<<grid, 256, 0, s>>>(n, H, D, g, A_log, dt_bias, yg);
  else if (out_dtype == GDN_DTYPE_BF16)
    k_kda_gate_fwd<Tin, __nv_bfloat16><<<grid, 256, 0, s>>>(n, H, D, g, A_log, dt_bias, yg);
  else
    k_kda_gate_fwd<Tin, __half><<<grid, 256, 0, s>>>(n, H, D, g, A_log, dt_bias, yg);
  return cudaGetLastError();
}

template <typename Tin>
cudaError_t bwd_dy(int64_t T, int H, int D, const void* g, const float* A_log, const float* dt_bias,
                   int dy_dtype, const void* dyg, void* dg, float* part, cudaStream_t s) {
  if (dy_dtype == GDN_DTYPE_FP32)
    k_kda_gate_bwd_rows<Tin, float><<<KG_BLOCKS, 256, 0, s>>>(T, H, D, g, A_log, dt_bias, dyg, dg, part);
  else if (dy_dtype == GDN_DTYPE_BF16)
    k_kda_gate_bwd_rows<Tin, __nv_bfloat16><<<KG_BLOCKS, 256, 0, s>>>(T, H, D, g, A_log, dt_bias, dyg, dg, part);
  else
    k_kda_gate_bwd_rows<Tin, __half><<<KG_BLOCKS, 256, 0, s>>>(T, H, D, g, A_log, dt_bias, dyg, dg, part);
  return cudaGetLastError();
}

}  // namespace

size_t kda_gate_workspace_bytes(int64_t H, int64_t D) {
  return (size_t)KG_BLOCKS * 2 * (size_t)(H * D) * sizeof(float);
}

cudaError_t kda_gate_forward(int64_t T, int H, int D, int in_dtype, const void* g, const float* A_log,
                             const float* dt_bias, int out_dtype, void* yg, cudaStream_t s) {
  const int64_t n = T * H * D;
  if (n == 0) return cudaSuccess;
  ProfScope ps("kda_gate_fwd", s);
  if (in_dtype == GDN_DTYPE_FP32) return fwd_out<float>(n, H, D, g, A_log, dt_bias, out_dtype, yg, s);
  if (in_dtype == GDN_DTYPE_BF16) return fwd_out<__nv_bfloat16>(n, H, D, g, A_log, dt_bias, out_dtype, yg, s);
  return fwd_out<__half>(n, H, D, g, A_log, dt_bias, out_dtype, yg, s);
}

cudaError_t kda_gate_backward(int64_t T, int H, int D, int in_dtype, const void* g, const float* A_log,
                              const float* dt_bias, int dy_dtype, const void* dyg, void* dg,
                              float* dA_log, float* ddt_bias, float* part, cudaStream_t s) {
  cudaError_t e;
  {
    ProfScope ps("kda_gate_bwd", s);
    if (in_dtype == GDN_DTYPE_FP32)
      e = bwd_dy<float>(T, H, D, g, A_log, dt_bias, dy_dtype, dyg, dg, part, s);
    else if (in_dtype == GDN_DTYPE_BF16)
      e = bwd_dy<__nv_bfloat16>(T, H, D, g, A_log, dt_bias, dy_dtype, dyg, dg, part, s);
    else
      e = bwd_dy<__half>(T, H, D, g, A_log, dt_bias, dy_dtype, dyg, dg, part, s);
  }
  if (e != cudaSuccess) return e;
  ProfScope ps("kda_gate_bwd_reduce", s);
  k_kda_gate_bwd_reduce<<<H, 256, 0, s>>>(H, D, part, dA_log, ddt_bias);
  return cudaGetLastError();
}

}  // namespace gdn
