// KDA gate (per-channel gate of Kimi-style delta attention): for g [T, H, D],
//   yg[t,h,d] = -exp(A_log[h]) * softplus(g[t,h,d] + dt_bias[h*D + d]),
//   softplus(x) = x for x > 20, else log(1 + e^x),
// computed in fp32 and written in the output dtype (MindSpeed-Ops issue 9, "KDA gate",
// sections on the formula and the computation flow).  Its backward for a loss L(yg):
//   dg[t,h,d]       = dyg * (-exp(A_log[h])) * (x > 20 ? 1 : sigmoid(x))
//   dA_log[h]       = sum_{t,d} dyg * yg
//   d dt_bias[h*D+d] = sum_t dg[t,h,d]
//
// Element-wise and HBM-bound.  The [T, H*D] matrix is walked in VEC-wide column vectors (16-byte
// loads for 16-bit inputs when D % 8 == 0): a block holds CV column vectors x RP row lanes and
// strides over rows, so every thread keeps one column vector (its head, A_log and dt_bias) for
// the whole launch and no index is divided per element.  softplus and sigmoid share one fast
// exponential e = exp(-|x|):
//   softplus(x) = max(x, 0) + log(1 + e),   sigmoid(x) = x >= 0 ? 1/(1+e) : e/(1+e),
// with log(1 + e), e in [0, 1], from the artanh series (log1p_unit below).
//
// The two backward sums are deterministic: a fixed number of row blocks write per-column
// partial sums, the column sums add them in block order, and one CTA per head reduces its
// columns by a fixed tree.
#include <cuda_fp16.h>

#include <algorithm>
#include <type_traits>

#include "gdn_common.cuh"
#include "kda_gate_math.cuh"
#include "gdn_launch.h"

namespace gdn {
namespace {

constexpr int KG_ROWBLOCKS = 296;  // most row blocks of the backward (2 per SM)
constexpr int KG_THREADS = 256;

// ---- VEC-wide loads and stores (VEC = 8 or 1), widened to / rounded from fp32
template <typename T, int VEC>
__device__ __forceinline__ void ldv(const T* p, float (&x)[VEC]) {
  if constexpr (VEC == 1) {
    if constexpr (std::is_same<T, float>::value) x[0] = p[0];
    else if constexpr (std::is_same<T, __half>::value) x[0] = __half2float(p[0]);
    else x[0] = __bfloat162float(p[0]);
  } else if constexpr (std::is_same<T, float>::value) {
    const float4 a = __ldcs(reinterpret_cast<const float4*>(p));
    const float4 b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  } else {
    const uint4 u = __ldcs(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 f;
      if constexpr (std::is_same<T, __half>::value)
        f = __half22float2(*reinterpret_cast<const __half2*>(&w[j]));
      else
        f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
      x[2 * j] = f.x;
      x[2 * j + 1] = f.y;
    }
  }
}

template <typename T, int VEC>
__device__ __forceinline__ void stv(T* p, const float (&x)[VEC]) {
  if constexpr (VEC == 1) {
    if constexpr (std::is_same<T, float>::value) p[0] = x[0];
    else if constexpr (std::is_same<T, __half>::value) p[0] = __float2half_rn(x[0]);
    else p[0] = __float2bfloat16_rn(x[0]);
  } else if constexpr (std::is_same<T, float>::value) {
    __stcs(reinterpret_cast<float4*>(p), make_float4(x[0], x[1], x[2], x[3]));
    __stcs(reinterpret_cast<float4*>(p) + 1, make_float4(x[4], x[5], x[6], x[7]));
  } else {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if constexpr (std::is_same<T, __half>::value) {
        const __half2 h2 = __floats2half2_rn(x[2 * j], x[2 * j + 1]);
        w[j] = *reinterpret_cast<const uint32_t*>(&h2);
      } else {
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(x[2 * j], x[2 * j + 1]);
        w[j] = *reinterpret_cast<const uint32_t*>(&h2);
      }
    }
    __stcs(reinterpret_cast<uint4*>(p), make_uint4(w[0], w[1], w[2], w[3]));
  }
}

struct Map {  // thread mapping of [T, HD] in VEC-wide column vectors
  int vec, NV, CV, RP;
  int gy() const { return (NV + CV - 1) / CV; }
};

Map make_map(int HD, int D) {
  Map m;
  m.vec = D % 8 == 0 ? 8 : 1;
  m.NV = HD / m.vec;
  m.CV = std::min(m.NV, KG_THREADS);
  m.RP = std::max(1, KG_THREADS / m.CV);
  return m;
}

template <typename Tin, typename Tout, int VEC>
__global__ void __launch_bounds__(KG_THREADS) k_kda_gate_fwd(int64_t T, int HD, int D, int CV, int RP,
                                                             const Tin* __restrict__ g,
                                                             const float* __restrict__ A_log,
                                                             const float* __restrict__ dt_bias,
                                                             Tout* __restrict__ yg) {
  const int cv = blockIdx.y * CV + (int)threadIdx.x % CV;
  if (cv * VEC >= HD) return;
  const int c0 = cv * VEC;
  const float nexp = -expf(A_log[c0 / D]);
  float bias[VEC];
#pragma unroll
  for (int j = 0; j < VEC; ++j) bias[j] = dt_bias ? dt_bias[c0 + j] : 0.f;
  const int64_t stride = (int64_t)gridDim.x * RP;
  for (int64_t t = (int64_t)blockIdx.x * RP + threadIdx.x / CV; t < T; t += 2 * stride) {
    const bool two = t + stride < T;  // two rows per step: both loads in flight together
    float x0[VEC], x1[VEC];
    ldv<Tin, VEC>(g + t * HD + c0, x0);
    if (two) ldv<Tin, VEC>(g + (t + stride) * HD + c0, x1);
#pragma unroll
    for (int j = 0; j < VEC; ++j) x0[j] = nexp * softplus20(x0[j] + bias[j]);
    stv<Tout, VEC>(yg + t * HD + c0, x0);
    if (two) {
#pragma unroll
      for (int j = 0; j < VEC; ++j) x1[j] = nexp * softplus20(x1[j] + bias[j]);
      stv<Tout, VEC>(yg + (t + stride) * HD + c0, x1);
    }
  }
}

// Pass 1: row block blockIdx.x takes rows blockIdx.x*RP + lane + k*gridDim.x*RP; dg is written
// per element, and the block's per-column sums of dyg*yg and of dg go to part[bx][0|1][HD]
// (row lanes added in lane order).
template <typename Tin, typename Tdy, int VEC>
__global__ void __launch_bounds__(KG_THREADS) k_kda_gate_bwd_rows(
    int64_t T, int HD, int D, int CV, int RP, const Tin* __restrict__ g,
    const float* __restrict__ A_log, const float* __restrict__ dt_bias, const Tdy* __restrict__ dyg,
    Tin* __restrict__ dg, float* __restrict__ part) {
  __shared__ float red[2][KG_THREADS * VEC];
  const int lane = threadIdx.x / CV;
  const int cv = blockIdx.y * CV + (int)threadIdx.x % CV;
  const bool live = cv * VEC < HD;
  const int c0 = live ? cv * VEC : 0;
  const float nexp = -expf(A_log[c0 / D]);
  float bias[VEC], sa[VEC], sb[VEC];
#pragma unroll
  for (int j = 0; j < VEC; ++j) {
    bias[j] = dt_bias ? dt_bias[c0 + j] : 0.f;
    sa[j] = 0.f;
    sb[j] = 0.f;
  }
  constexpr int U = 4;  // rows per step, their loads in flight together
  const int64_t stride = (int64_t)gridDim.x * RP;
  if (live) {
    for (int64_t t = (int64_t)blockIdx.x * RP + lane; t < T; t += U * stride) {
      float x[U][VEC], dy[U][VEC];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (t + u * stride < T) {
          ldv<Tin, VEC>(g + (t + u * stride) * HD + c0, x[u]);
          ldv<Tdy, VEC>(dyg + (t + u * stride) * HD + c0, dy[u]);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (t + u * stride >= T) break;
        float o[VEC];
#pragma unroll
        for (int j = 0; j < VEC; ++j) {
          float sp, sig;
          softplus_sigmoid(x[u][j] + bias[j], sp, sig);
          const float dyn = dy[u][j] * nexp;
          o[j] = dyn * sig;
          sa[j] += dyn * sp;  // dyg * yg
          sb[j] += o[j];
        }
        stv<Tin, VEC>(dg + (t + u * stride) * HD + c0, o);
      }
    }
  }
  float* pa = part + (int64_t)blockIdx.x * 2 * HD;
  if (RP == 1) {
    if (live) {
#pragma unroll
      for (int j = 0; j < VEC; ++j) {
        pa[c0 + j] = sa[j];
        pa[HD + c0 + j] = sb[j];
      }
    }
    return;
  }
  const int slot = ((int)threadIdx.x % CV) * VEC;
#pragma unroll
  for (int j = 0; j < VEC; ++j) {
    red[0][lane * CV * VEC + slot + j] = sa[j];
    red[1][lane * CV * VEC + slot + j] = sb[j];
  }
  __syncthreads();
  if (lane == 0 && live) {
#pragma unroll
    for (int j = 0; j < VEC; ++j) {
      float a = 0.f, b = 0.f;
      for (int l = 0; l < RP; ++l) {
        a += red[0][l * CV * VEC + slot + j];
        b += red[1][l * CV * VEC + slot + j];
      }
      pa[c0 + j] = a;
      pa[HD + c0 + j] = b;
    }
  }
}

// Pass 2: column sums over the nbx row blocks (8 strands, each in block order, then the strands
// in order); ddt_bias[c] and the dA column sums colA[c].
__global__ void __launch_bounds__(256) k_kda_gate_bwd_cols(int HD, int nbx, const float* __restrict__ part,
                                                           float* __restrict__ colA,
                                                           float* __restrict__ ddt_bias) {
  __shared__ float s[2][8][32];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int c = blockIdx.x * 32 + tx;
  float a = 0.f, b = 0.f;
  if (c < HD) {
    for (int bx = ty; bx < nbx; bx += 8) {
      a += part[(int64_t)bx * 2 * HD + c];
      b += part[(int64_t)bx * 2 * HD + HD + c];
    }
  }
  s[0][ty][tx] = a;
  s[1][ty][tx] = b;
  __syncthreads();
  if (ty == 0 && c < HD) {
    float A = 0.f, Bs = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      A += s[0][k][tx];
      Bs += s[1][k][tx];
    }
    colA[c] = A;
    if (ddt_bias) ddt_bias[c] = Bs;
  }
}

// Pass 3: one CTA per head, a fixed tree over its D column sums.
__global__ void __launch_bounds__(256) k_kda_gate_bwd_heads(int D, const float* __restrict__ colA,
                                                            float* __restrict__ dA_log) {
  __shared__ float red[256];
  const int h = blockIdx.x;
  float acc = 0.f;
  for (int d = threadIdx.x; d < D; d += blockDim.x) acc += colA[(int64_t)h * D + d];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int s = 128; s > 0; s >>= 1) {
    if ((int)threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) dA_log[h] = red[0];
}

int fwd_grid_x(int64_t T, const Map& m) {
  const int64_t rows = (T + m.RP - 1) / m.RP;
  const int64_t want = std::max<int64_t>(1, (int64_t)num_sms() * (2048 / (m.CV * m.RP)) / m.gy());
  return (int)std::max<int64_t>(1, std::min<int64_t>(rows, want));
}

int bwd_grid_x(int64_t T, const Map& m) {  // a function of the sizes only (deterministic sums)
  const int64_t rows = (T + m.RP - 1) / m.RP;
  return (int)std::min<int64_t>(rows, std::max(1, KG_ROWBLOCKS / m.gy()));
}

template <typename Tin, typename Tout>
cudaError_t fwd_t(int64_t T, int H, int D, const void* g, const float* A_log, const float* dt_bias,
                  void* yg, cudaStream_t s) {
  const int HD = H * D;
  const Map m = make_map(HD, D);
  const dim3 grid(fwd_grid_x(T, m), m.gy());
  if (m.vec == 8)
    k_kda_gate_fwd<Tin, Tout, 8><<<grid, m.CV * m.RP, 0, s>>>(
        T, HD, D, m.CV, m.RP, static_cast<const Tin*>(g), A_log, dt_bias, static_cast<Tout*>(yg));
  else
    k_kda_gate_fwd<Tin, Tout, 1><<<grid, m.CV * m.RP, 0, s>>>(
        T, HD, D, m.CV, m.RP, static_cast<const Tin*>(g), A_log, dt_bias, static_cast<Tout*>(yg));
  return cudaGetLastError();
}

template <typename Tin>
cudaError_t fwd_out(int64_t T, int H, int D, const void* g, const float* A_log, const float* dt_bias,
                    int out_dtype, void* yg, cudaStream_t s) {
  if (out_dtype == GDN_DTYPE_FP32) return fwd_t<Tin, float>(T, H, D, g, A_log, dt_bias, yg, s);
  if (out_dtype == GDN_DTYPE_BF16) return fwd_t<Tin, __nv_bfloat16>(T, H, D, g, A_log, dt_bias, yg, s);
  return fwd_t<Tin, __half>(T, H, D, g, A_log, dt_bias, yg, s);
}

template <typename Tin, typename Tdy>
cudaError_t bwd_t(int64_t T, int H, int D, const void* g, const float* A_log, const float* dt_bias,
                  const void* dyg, void* dg, float* part, int nbx, cudaStream_t s) {
  const int HD = H * D;
  const Map m = make_map(HD, D);
  const dim3 grid(nbx, m.gy());
  if (m.vec == 8)
    k_kda_gate_bwd_rows<Tin, Tdy, 8><<<grid, m.CV * m.RP, 0, s>>>(
        T, HD, D, m.CV, m.RP, static_cast<const Tin*>(g), A_log, dt_bias, static_cast<const Tdy*>(dyg),
        static_cast<Tin*>(dg), part);
  else
    k_kda_gate_bwd_rows<Tin, Tdy, 1><<<grid, m.CV * m.RP, 0, s>>>(
        T, HD, D, m.CV, m.RP, static_cast<const Tin*>(g), A_log, dt_bias, static_cast<const Tdy*>(dyg),
        static_cast<Tin*>(dg), part);
  return cudaGetLastError();
}

template <typename Tin>
cudaError_t bwd_dy(int64_t T, int H, int D, const void* g, const float* A_log, const float* dt_bias,
                   int dy_dtype, const void* dyg, void* dg, float* part, int nbx, cudaStream_t s) {
  if (dy_dtype == GDN_DTYPE_FP32) return bwd_t<Tin, float>(T, H, D, g, A_log, dt_bias, dyg, dg, part, nbx, s);
  if (dy_dtype == GDN_DTYPE_BF16)
    return bwd_t<Tin, __nv_bfloat16>(T, H, D, g, A_log, dt_bias, dyg, dg, part, nbx, s);
  return bwd_t<Tin, __half>(T, H, D, g, A_log, dt_bias, dyg, dg, part, nbx, s);
}

}  // namespace

size_t kda_gate_workspace_bytes(int64_t H, int64_t D) {
  return ((size_t)KG_ROWBLOCKS * 2 + 1) * (size_t)(H * D) * sizeof(float);
}

cudaError_t kda_gate_forward(int64_t T, int H, int D, int in_dtype, const void* g, const float* A_log,
                             const float* dt_bias, int out_dtype, void* yg, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  ProfScope ps("kda_gate_fwd", s);
  if (in_dtype == GDN_DTYPE_FP32) return fwd_out<float>(T, H, D, g, A_log, dt_bias, out_dtype, yg, s);
  if (in_dtype == GDN_DTYPE_BF16) return fwd_out<__nv_bfloat16>(T, H, D, g, A_log, dt_bias, out_dtype, yg, s);
  return fwd_out<__half>(T, H, D, g, A_log, dt_bias, out_dtype, yg, s);
}

cudaError_t kda_gate_backward(int64_t T, int H, int D, int in_dtype, const void* g, const float* A_log,
                              const float* dt_bias, int dy_dtype, const void* dyg, void* dg,
                              float* dA_log, float* ddt_bias, float* work, cudaStream_t s) {
  const int HD = H * D;
  const Map m = make_map(HD, D);
  const int nbx = bwd_grid_x(T, m);  // 0 when T == 0: the sums come out as zeros
  float* part = work;
  float* colA = work + (size_t)KG_ROWBLOCKS * 2 * HD;
  cudaError_t e = cudaSuccess;
  if (nbx > 0) {
    ProfScope ps("kda_gate_bwd", s);
    if (in_dtype == GDN_DTYPE_FP32)
      e = bwd_dy<float>(T, H, D, g, A_log, dt_bias, dy_dtype, dyg, dg, part, nbx, s);
    else if (in_dtype == GDN_DTYPE_BF16)
      e = bwd_dy<__nv_bfloat16>(T, H, D, g, A_log, dt_bias, dy_dtype, dyg, dg, part, nbx, s);
    else
      e = bwd_dy<__half>(T, H, D, g, A_log, dt_bias, dy_dtype, dyg, dg, part, nbx, s);
  }
  if (e != cudaSuccess) return e;
  if (!dA_log && !ddt_bias) return cudaSuccess;
  ProfScope ps("kda_gate_bwd_sums", s);
  k_kda_gate_bwd_cols<<<(HD + 31) / 32, 256, 0, s>>>(HD, nbx, part, colA, ddt_bias);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (dA_log) k_kda_gate_bwd_heads<<<H, 256, 0, s>>>(D, colA, dA_log);
  return cudaGetLastError();
}

}  // namespace gdn
