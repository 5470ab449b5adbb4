// The KDA gate's element math, shared by the gate kernels and the chunkwise KDA kernels that fuse
// the gate: softplus and its derivative (sigmoid) from one fast exponential, with log(1 + e) from
// the artanh series (MindSpeed-Ops KDA gate task: yg = -exp(A_log) softplus(g + dt_bias), softplus
// passing x > 20 through).
#pragma once

#include <cuda_runtime.h>

namespace gdn {

// log(1 + e) for e in [0, 1].  With s = e / (2 + e) in [0, 1/3], 1 + e = (1 + s) / (1 - s), so
// log(1 + e) = 2 artanh(s) = 2 s sum_k s^{2k} / (2k + 1).  s^2 <= 1/9, so the eight terms kept
// leave a relative truncation below (1/9)^8 / 17 < 2^-27; the approximate division costs 2 ulp.
__device__ __forceinline__ float log1p_unit(float e) {
  const float s = __fdividef(e, 2.f + e);
  const float z = s * s;
  float p = 1.f / 15.f;
  p = fmaf(p, z, 1.f / 13.f);
  p = fmaf(p, z, 1.f / 11.f);
  p = fmaf(p, z, 1.f / 9.f);
  p = fmaf(p, z, 1.f / 7.f);
  p = fmaf(p, z, 1.f / 5.f);
  p = fmaf(p, z, 1.f / 3.f);
  p = fmaf(p, z, 1.f);
  return 2.f * s * p;
}

__device__ __forceinline__ float softplus20(float x) {
  return x > 20.f ? x : fmaxf(x, 0.f) + log1p_unit(__expf(-fabsf(x)));
}

// softplus(x) and its derivative sigmoid(x) (1 on the x > 20 pass-through) from one exponential
__device__ __forceinline__ void softplus_sigmoid(float x, float& sp, float& sig) {
  const float e = __expf(-fabsf(x));
  const float r = __fdividef(1.f, 1.f + e);
  sp = x > 20.f ? x : fmaxf(x, 0.f) + log1p_unit(e);
  sig = x > 20.f ? 1.f : (x >= 0.f ? r : e * r);
}

}  // namespace gdn
