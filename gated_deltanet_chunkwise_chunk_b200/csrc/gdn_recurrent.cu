// Token-by-token (recurrent) form of the gated delta rule, for decoding and short prefills:
// the state of each (sequence, value head) is read from HBM once, carried through the
// sequence's tokens in registers, and written back once.  Per token t (S: V x K):
//   g_t = -exp(A_log) softplus(a_t + dt_bias)        (the same gate as the chunk path)
//   S  <- e^{g_t} S;   e = S k_t;   S <- S + beta_t (v_t - e) k_t^T;   o_t = scale S q_t
// (the decay applies before the erase, as in the chunkwise algebra).  HBM-bound at T = 1:
// 2 x 4KV bytes of state per (sequence, value head) plus the token vectors.
//
// CTA (sequence, value head, z) holds rows v0 = 32z .. v0+31 of S; thread (v, kq) keeps
// S[v0+v][kq*K/4 .. (kq+1)*K/4) in fp32 registers, the four kq threads of a row being adjacent
// lanes (row sums by two shuffles).
#include "gdn_common.cuh"
#include "gdn_launch.h"

namespace gdn {
namespace {

constexpr int RV = 32;  // state rows per CTA

template <typename T, int K>
__global__ void __launch_bounds__(128) k_recurrent_fwd(Problem p, Args a, int* status) {
  constexpr int KQ = K / 4;  // state columns per thread
  const int n = blockIdx.x, hv = blockIdx.y, hk = hv / p.G, v0 = RV * blockIdx.z;
  const int tid = threadIdx.x, vl = tid >> 2, kq = tid & 3;
  __shared__ float sk[K], sq[K], sv[RV], sdec, sbeta;
  int bos, eos;
  if (p.varlen) {
    bos = (int)a.cu[n];
    eos = (int)a.cu[n + 1];
    const bool bad = bos < 0 || eos < bos || eos > p.T || (n == 0 && bos != 0) ||
                     (n == p.Nst - 1 && eos != p.T);
    if (bad) {  // not a partition of [0, T): report and leave this sequence alone
      if (tid == 0) atomicExch(status, (int)GDN_ERR_INVALID_ARG);
      return;
    }
  } else {
    bos = n * p.T;
    eos = bos + p.T;
  }
  // state: h[k][v] = S[v][k], fp32 [Nst][HV][K][V]
  const size_t st = ((size_t)n * p.HV + hv) * K * p.V + v0 + vl;
  float S[KQ];
#pragma unroll
  for (int i = 0; i < KQ; ++i) S[i] = a.h0 ? a.h0[st + (size_t)(kq * KQ + i) * p.V] : 0.f;
  const T* q = static_cast<const T*>(a.q);
  const T* k = static_cast<const T*>(a.k);
  const T* v = static_cast<const T*>(a.v);
  T* o = static_cast<T*>(a.o);
  const float nexp = -expf(a.A_log[hv]), dtb = a.dt_bias[hv];
  for (int t = bos; t < eos; ++t) {
    __syncthreads();  // the previous token's vectors are no longer read
    const size_t qk0 = ((size_t)t * p.H + hk) * K, v_0 = ((size_t)t * p.HV + hv) * p.V + v0;
    for (int i = tid; i < K; i += 128) {
      sk[i] = to_f<T>(k[qk0 + i]);
      sq[i] = to_f<T>(q[qk0 + i]);
    }
    if (tid < RV) sv[tid] = to_f<T>(v[v_0 + tid]);
    if (tid == 0) {
      const size_t gi = (size_t)t * p.HV + hv;
      const float x = a.g_raw[gi] + dtb;
      sdec = expf(nexp * (x > 20.f ? x : log1pf(expf(x))));
      sbeta = a.beta[gi];
    }
    __syncthreads();
    const float dec = sdec, b = sbeta;
    float e = 0.f;
#pragma unroll
    for (int i = 0; i < KQ; ++i) {
      S[i] *= dec;
      e += S[i] * sk[kq * KQ + i];
    }
    e += __shfl_xor_sync(0xffffffffu, e, 1);
    e += __shfl_xor_sync(0xffffffffu, e, 2);
    const float dl = b * (sv[vl] - e);
    float y = 0.f;
#pragma unroll
    for (int i = 0; i < KQ; ++i) {
      S[i] += dl * sk[kq * KQ + i];
      y += S[i] * sq[kq * KQ + i];
    }
    y += __shfl_xor_sync(0xffffffffu, y, 1);
    y += __shfl_xor_sync(0xffffffffu, y, 2);
    if (kq == 0) o[v_0 + vl] = from_f<T>(p.scale * y);
  }
  if (a.ht) {
#pragma unroll
    for (int i = 0; i < KQ; ++i) a.ht[st + (size_t)(kq * KQ + i) * p.V] = S[i];
  }
}

template <typename T>
cudaError_t launch_t(const Problem& p, const Args& a, int* status, cudaStream_t s) {
  const dim3 grid(p.Nst, p.HV, p.V / RV);
  if (p.K == 128)
    k_recurrent_fwd<T, 128><<<grid, 128, 0, s>>>(p, a, status);
  else
    k_recurrent_fwd<T, 64><<<grid, 128, 0, s>>>(p, a, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t recurrent_forward(const Problem& p, const Args& a, int* status, bool bf16, cudaStream_t s) {
  if (p.Nst == 0) return cudaSuccess;
  ProfScope ps("recurrent_fwd", s);
  return bf16 ? launch_t<__nv_bfloat16>(p, a, status, s) : launch_t<float>(p, a, status, s);
}

}  // namespace gdn
