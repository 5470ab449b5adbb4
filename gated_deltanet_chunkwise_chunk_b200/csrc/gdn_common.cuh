// Shared device-side definitions of the chunkwise Gated DeltaNet library (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "gdn.h"

namespace gdn {

constexpr int CH = 64;         // tokens per chunk
constexpr int PG_BLOCKS = 128;  // token blocks of the gate-parameter gradient reduction

// Launch-wide problem description (passed by value to every kernel).
struct Problem {
  int B, T, H, HV, K, V;
  int Nst;      // number of independent state sequences (N when varlen, else B)
  int G;        // value heads per k-head (HV / H)
  int varlen;   // 1 when cu_seqlens is used
  int NCmax;    // grid bound on the number of chunks
  float scale;
  int test_timeout;  // GDN_FLAG_TEST_WAIT_TIMEOUT: the forward pass withholds one arrive (tests only)
  int share_ld;      // row stride of the per-value-head dq/dk shares (K, or 128 on the tcgen05 path)
};

// Workspace carve-up (device pointers into the caller's workspace).  Intermediates are
// indexed per chunk gc in [0, NCmax) and value head hv.
struct Work {
  int* status;        // [0] device status word, [1] chunk count
  int4* seq_tab;      // [Nst]   {first chunk, number of chunks, flat bos, length}
  int4* chunk_tab;    // [NCmax] {sequence, chunk in sequence, tokens L, flat token of row 0}
  float* G;           // [HV][NCmax][64]   in-chunk inclusive cumsum of g, padded with G[L-1]
  float* beta_p;      // [HV][NCmax][64]   beta, zero past the chunk's last token
  float* Dec;         // [HV][NCmax][64]   e^{G_63 - G_i}  (decay from token i to the chunk end)
  float* EG;          // [HV][NCmax][64]   e^{G_i}
  // fp32 intermediates of the FFMA path
  float* W;           // [NCmax][HV][64][K]
  float* Ut;          // [NCmax][HV][64][V]
  float* Tm;          // [NCmax][HV][64][64]   (I + A)^-1
  float* h;           // [NCmax][HV][V][K]     state entering the chunk (S orientation)
  float* U;           // [NCmax][HV][64][V]    v_new = U~ - W S^T
  float* dU;          // [NCmax][HV][64][V]    dU_loc, then the full dU
  float* dh;          // [NCmax][HV][V][K]     dL/dS leaving the chunk
  float* dW;          // [NCmax][HV][64][K]
  float* dqp;         // [NCmax][HV][64][K]    per-value-head dq share
  float* dkp;         // [NCmax][HV][64][K]    per-value-head dk share
  float* dG;          // [HV][NCmax][64]       dL/dG (before the reverse cumsum)
  float* dkp2;        // [NCmax][HV][64][K]    a second dk share summed by the assembly (or null)
  float* dG2;         // [HV][NCmax][64]       tcgen05 path: the WY backward's dG part (or null)
  float* tmp;         // [NCmax][HV][64][128]  per-unit scratch
  float* pgp;         // [PG_BLOCKS][HV][2]    partial sums of the gate-parameter gradients
};

// Workspace of the chunkwise KDA forward (fp32, per chunk gc and value head hv).
struct KdaWork {
  int* status;     // [0] device status word, [1] chunk count
  int4* seq_tab;   // [Nst]
  int4* chunk_tab; // [NCmax]
  float* W;        // [NCmax][HV][64][K]   T diag(beta) (k e^{Gam})
  float* Ut;       // [NCmax][HV][64][V]   T diag(beta) V
  float* Kh;       // [NCmax][HV][64][K]   k e^{Gam_C - Gam}
  float* Qt;       // [NCmax][HV][64][K]   q e^{Gam}
  float* P;        // [NCmax][HV][64][64]  sum_c q_i k_j e^{Gam_i - Gam_j}, lower incl. diagonal
  float* eGC;      // [NCmax][HV][K]       e^{Gam_C}
  float* h;        // [NCmax][HV][V][K]    state entering the chunk (S orientation)
  float* U;        // [NCmax][HV][64][V]   U~ - W S^T
  // kept by a forward whose workspace is sized for the backward, and the backward's own
  float* Gam;      // [NCmax][HV][64][K]   in-chunk cumsum of the log-decay, times log2(e)
  float* Tm;       // [NCmax][HV][64][64]  (I + A)^-1
  float* dU;       // [NCmax][HV][64][V]   dL/dU, then dY = T^T dU
  float* dh;       // [NCmax][HV][V][K]    dL/dS leaving the chunk
  float* dW;       // [NCmax][HV][64][K]   dL/dW, then dX = T^T dW
  float* dGam;     // [NCmax][HV][64][K]   dL/dGam, then dL/dyg
  float* dqp;      // [NCmax][HV][64][K]   per-value-head dq share
  float* dkp;      // [NCmax][HV][64][K]   per-value-head dk share
  float* pgp;      // [NCmax][HV][K+1]     per-chunk sums of dL/d dt_bias (K) and dL/dA_log (1)
};

// Pointers of one call (inputs and outputs as given by the caller).
struct Args {
  const void* q;
  const void* k;
  const void* v;
  const float* g_raw;
  const float* A_log;
  const float* dt_bias;
  const float* beta;
  const int64_t* cu;
  const float* h0;
  void* o;
  float* ht;
  const void* dO;
  const float* dht;
  void* dq;
  void* dk;
  void* dv;
  float* dg;
  float* dbeta;
  float* dh0;
  float* dg_raw;
  float* dA_log;
  float* ddt_bias;
};

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// The gate of one token: g = -exp(A_log) * softplus(x), softplus(x) = x for x > 20.
__device__ __forceinline__ float gate_value(float a, float A_log, float dt_bias) {
  const float x = a + dt_bias;
  const float sp = x > 20.f ? x : log1pf(expf(x));
  return -expf(A_log) * sp;
}

// d softplus / dx with the same branch.
__device__ __forceinline__ float gate_dsoftplus(float x) {
  return x > 20.f ? 1.f : 1.f / (1.f + expf(-x));
}

__device__ __forceinline__ bool call_failed(const Work& w) {
  return *((volatile int*)w.status) != 0;
}

// Streaming multiprocessors of the current device (grid sizes of persistent and streaming kernels).
inline int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

}  // namespace gdn
