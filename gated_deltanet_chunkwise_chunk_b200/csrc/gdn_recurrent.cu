// Token-by-token (recurrent) form of the gated delta rule, for decoding and short prefills:
// the state of each (sequence, value head) is read from HBM once, carried through the
// sequence's tokens in registers, and written back once.  Per token t (S: V x K):
//   g_t = -exp(A_log) softplus(a_t + dt_bias)        (the same gate as the chunk path)
//   S  <- e^{g_t} S;   e = S k_t;   S <- S + beta_t (v_t - e) k_t^T;   o_t = scale S q_t
// (the decay applies before the erase, as in the chunkwise algebra).  HBM-bound at T = 1:
// 2 x 4KV bytes of state per (sequence, value head) plus the token vectors.
//
// KDA variant (template flag KDA): the decay is per key channel c, S <- S Diag(e^{yg_t}) with
// yg_t[c] = -exp(A_log) softplus(g_raw[t, hv, c] + dt_bias[hv*K + c]) (the KDA gate of the
// MindSpeed-Ops "KDA gate" task, fused here); everything else is unchanged.
//
// CTA (sequence, value head, z) holds rows v0 = 32z .. v0+31 of S.  Thread (kg, vg) keeps
// S[v0+4vg .. +3][kg*K/16 .. (kg+1)*K/16) in fp32 registers, so the state moves as 16-byte
// rows of h[k][v]; the 16 k-groups of a column block sit in one warp (lane = kg + 16 (vg%2)),
// so row sums are four shuffles.  With a scalar gate each thread reads its own channels of k
// and q and its rows of v straight from global memory (one vector load each; the 16 k-groups
// of a warp read whole 256-byte rows) and computes the gate itself, so a token needs no shared
// memory and no block barrier; the KDA variant shares its per-channel decays through shared
// memory.
#include <algorithm>
#include <type_traits>

#include "ffma_tiles.cuh"  // cp_async16
#include "gdn_common.cuh"
#include "gdn_launch.h"
#include "kda_gate_math.cuh"

namespace gdn {
namespace {

constexpr int RV = 32;  // state rows per CTA

// N (4 or 8) consecutive elements at p (16-byte aligned for fp32, 8/16-byte for bf16) as floats
template <typename T, int N>
__device__ __forceinline__ void ld_floats(const T* p, float* out) {
  if constexpr (std::is_same<T, float>::value) {
#pragma unroll
    for (int i = 0; i < N; i += 4) {
      const float4 x = *reinterpret_cast<const float4*>(p + i);
      out[i] = x.x; out[i + 1] = x.y; out[i + 2] = x.z; out[i + 3] = x.w;
    }
  } else if constexpr (N == 8) {
    const uint4 x = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
      out[2 * i] = f.x; out[2 * i + 1] = f.y;
    }
  } else {
    const uint2 x = *reinterpret_cast<const uint2*>(p);
    const uint32_t w[2] = {x.x, x.y};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
      out[2 * i] = f.x; out[2 * i + 1] = f.y;
    }
  }
}

template <typename T, int K, bool KDA>
__global__ void __launch_bounds__(128) k_recurrent_fwd(Problem p, Args a, int* status) {
  constexpr int KQ = K / 16;  // state columns per thread
  // blockIdx.x = n * (V / RV) + slice: the slices of one state are neighbours in launch order,
  // so the four 128-byte pieces of each 512-byte state row are fetched together
  const int nz = p.V / RV;
  const int n = blockIdx.x / nz, hv = blockIdx.y, hk = hv / p.G, v0 = RV * (blockIdx.x % nz);
  const int tid = threadIdx.x, lane = tid & 31, kg = lane & 15, vg = 2 * (tid >> 5) + (lane >> 4);
  __shared__ __align__(16) float sk[KDA ? K : 4];
  __shared__ __align__(16) float sq[KDA ? K : 4];
  __shared__ __align__(16) float sdk[KDA ? K : 4];
  __shared__ float sv[RV], sbeta;
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
  // state: h[k][v] = S[v][k], fp32 [Nst][HV][K][V]; S4[i] = S[v0+4vg .. +3][kg*KQ + i]
  const size_t st = ((size_t)n * p.HV + hv) * K * p.V + v0 + 4 * vg;
  float4 S4[KQ];
#pragma unroll
  for (int i = 0; i < KQ; ++i)
    S4[i] = a.h0 ? *reinterpret_cast<const float4*>(a.h0 + st + (size_t)(kg * KQ + i) * p.V)
                 : make_float4(0.f, 0.f, 0.f, 0.f);
  const T* q = static_cast<const T*>(a.q);
  const T* k = static_cast<const T*>(a.k);
  const T* v = static_cast<const T*>(a.v);
  T* o = static_cast<T*>(a.o);
  const float nexp = -expf(a.A_log[hv]), dtb = KDA ? 0.f : a.dt_bias[hv];
  // Sums over the 16 k-groups of this lane half of four values at once: each butterfly step
  // halves the values a lane carries (2 + 1 shuffles), two more steps finish the sum; lane
  // kg = 4j then holds the total of value j (x, y, z, w for j = 0..3).  5 shuffles, not 16.
  const bool b3 = kg & 8, b2 = kg & 4;
  auto rowsum4 = [&](const float4& e) {
    float s0 = b3 ? e.z : e.x, s1 = b3 ? e.w : e.y;
    s0 += __shfl_xor_sync(0xffffffffu, b3 ? e.x : e.z, 8);
    s1 += __shfl_xor_sync(0xffffffffu, b3 ? e.y : e.w, 8);
    float t = b2 ? s1 : s0;
    t += __shfl_xor_sync(0xffffffffu, b2 ? s0 : s1, 4);
    t += __shfl_xor_sync(0xffffffffu, t, 2);
    t += __shfl_xor_sync(0xffffffffu, t, 1);
    return t;
  };
  const int half = lane & 16;
  auto gather4 = [&](float t) {  // the four totals to every lane of the half
    return make_float4(__shfl_sync(0xffffffffu, t, half), __shfl_sync(0xffffffffu, t, half + 4),
                       __shfl_sync(0xffffffffu, t, half + 8), __shfl_sync(0xffffffffu, t, half + 12));
  };
  const size_t dtb_k = (size_t)hv * K;
  for (int t = bos; t < eos; ++t) {
    const size_t qk0 = ((size_t)t * p.H + hk) * K, v_0 = ((size_t)t * p.HV + hv) * p.V + v0;
    const size_t gi = (size_t)t * p.HV + hv;
    float kv[KQ], qv[KQ], dv[KQ], vv[4];  // this thread's channels and rows
    float b;
    if constexpr (!KDA) {
      ld_floats<T, KQ>(k + qk0 + kg * KQ, kv);
      ld_floats<T, KQ>(q + qk0 + kg * KQ, qv);
      ld_floats<T, 4>(v + v_0 + 4 * vg, vv);
      const float gf = a.g_raw[gi] + dtb;
      b = a.beta[gi];
      const float dec = expf(nexp * (gf > 20.f ? gf : log1pf(expf(gf))));
#pragma unroll
      for (int i = 0; i < KQ; ++i) dv[i] = dec;
    } else {
      // every load of this token first (one latency), spread over the threads; then one round
      // of shared-memory stores between two barriers (K <= 128: one channel per thread)
      float kf = 0.f, qf = 0.f, vf = 0.f, gf = 0.f, bf = 0.f;
      if (tid < K) {
        kf = to_f<T>(k[qk0 + tid]);
        qf = to_f<T>(q[qk0 + tid]);
        gf = a.g_raw[gi * K + tid] + (a.dt_bias ? a.dt_bias[dtb_k + tid] : 0.f);
      }
      if (tid < RV) vf = to_f<T>(v[v_0 + tid]);
      if (tid == 96) bf = a.beta[gi];
      __syncthreads();  // the previous token's vectors are no longer read
      if (tid < K) {
        sk[tid] = kf;
        sq[tid] = qf;
        sdk[tid] = expf(nexp * (gf > 20.f ? gf : log1pf(expf(gf))));
      }
      if (tid < RV) sv[tid] = vf;
      if (tid == 96) sbeta = bf;
      __syncthreads();
      b = sbeta;
#pragma unroll
      for (int i = 0; i < KQ; i += 4) {  // read as 16-byte vectors
        const float4 k4 = *reinterpret_cast<const float4*>(sk + kg * KQ + i);
        const float4 q4 = *reinterpret_cast<const float4*>(sq + kg * KQ + i);
        const float4 d4 = *reinterpret_cast<const float4*>(sdk + kg * KQ + i);
        kv[i] = k4.x; kv[i + 1] = k4.y; kv[i + 2] = k4.z; kv[i + 3] = k4.w;
        qv[i] = q4.x; qv[i + 1] = q4.y; qv[i + 2] = q4.z; qv[i + 3] = q4.w;
        dv[i] = d4.x; dv[i + 1] = d4.y; dv[i + 2] = d4.z; dv[i + 3] = d4.w;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) vv[i] = sv[4 * vg + i];
    }
    float4 e = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < KQ; ++i) {
      const float dec = dv[i];
      S4[i].x *= dec; S4[i].y *= dec; S4[i].z *= dec; S4[i].w *= dec;
      e.x += S4[i].x * kv[i]; e.y += S4[i].y * kv[i]; e.z += S4[i].z * kv[i]; e.w += S4[i].w * kv[i];
    }
    e = gather4(rowsum4(e));
    const float dx = b * (vv[0] - e.x), dy = b * (vv[1] - e.y), dz = b * (vv[2] - e.z),
                dw = b * (vv[3] - e.w);
    float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < KQ; ++i) {
      S4[i].x += dx * kv[i]; S4[i].y += dy * kv[i]; S4[i].z += dz * kv[i]; S4[i].w += dw * kv[i];
      y.x += S4[i].x * qv[i]; y.y += S4[i].y * qv[i]; y.z += S4[i].z * qv[i]; y.w += S4[i].w * qv[i];
    }
    const float yt = rowsum4(y);  // lane kg = 4j holds output column j
    if ((kg & 3) == 0) o[v_0 + 4 * vg + (kg >> 2)] = from_f<T>(p.scale * yt);
  }
  if (a.ht) {
#pragma unroll
    for (int i = 0; i < KQ; ++i)
      *reinterpret_cast<float4*>(a.ht + st + (size_t)(kg * KQ + i) * p.V) = S4[i];
  }
}

// Decode steps (one token per sequence, dense, with an entering state): persistent CTAs walk the
// (sequence, value head, 32-row slice) items in order, the four slices of a state neighbours.  A
// two-stage cp.async pipeline in shared memory holds the next item's state slice (K x 32 fp32)
// and token vectors while the current one is updated, so a CTA's loads stay in flight across
// its items (with one pass per CTA they overlapped only across CTAs).  The update is the
// recurrent kernel's, thread (kg, vg) holding the same state piece.
__device__ __forceinline__ void cp_async4(void* smem, const void* gmem) {
  const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(sa), "l"(gmem));
}

// A state slice row kk holds its eight 16-byte pieces j at slots j ^ ((kk / 8) % 8), so that the
// eight rows 8 apart that one load instruction of a warp reads fall on different banks.
__device__ __forceinline__ int slice_slot(int kk, int j) { return j ^ ((kk >> 3) & 7); }

template <typename T, int K, bool KDA>
struct DecodeStage {
  static constexpr int S = K * RV * 4;                       // state slice [K][32] fp32
  static constexpr int TK = S, TQ = TK + K * (int)sizeof(T);  // k, q vectors
  static constexpr int TV = TQ + K * (int)sizeof(T);          // v slice [32]
  static constexpr int TG = TV + RV * (int)sizeof(T);         // gate input(s): K (KDA) or 1
  static constexpr int TB = TG + (KDA ? K * 4 : 16);          // beta
  static constexpr int BYTES = (TB + 16 + 15) / 16 * 16;
};

template <typename T, int K, bool KDA>
__global__ void __launch_bounds__(128, KDA ? 6 : 4) k_decode_pipe(Problem p, Args a, int nitems) {
  using St = DecodeStage<T, K, KDA>;
  constexpr int KQ = K / 16;
  extern __shared__ __align__(16) unsigned char dsm[];
  const int nz = p.V / RV, tid = threadIdx.x, lane = tid & 31, kg = lane & 15;
  const int vg = 2 * (tid >> 5) + (lane >> 4), G = gridDim.x;
  const T* q = static_cast<const T*>(a.q);
  const T* k = static_cast<const T*>(a.k);
  const T* v = static_cast<const T*>(a.v);
  T* o = static_cast<T*>(a.o);
  auto issue = [&](int it, int slot) {  // cp.async of item it into stage slot; one group always
    if (it < nitems) {
      unsigned char* st = dsm + slot * St::BYTES;
      const int z = it % nz, nh = it / nz, n = nh / p.HV, hv = nh % p.HV, hk = hv / p.G, v0 = RV * z;
      const float* h0 = a.h0 + (size_t)nh * K * p.V + v0;
#pragma unroll
      for (int m = 0; m < K * RV / 4 / 128; ++m) {  // 16-byte pieces of the slice's rows
        const int c = tid + 128 * m, kk = c >> 3, j = c & 7;
        cp_async16(st + (kk * RV + 4 * slice_slot(kk, j)) * 4, h0 + (size_t)kk * p.V + 4 * j);
      }
      constexpr int CKQ = K * (int)sizeof(T) / 16, CV = RV * (int)sizeof(T) / 16;
      const size_t qk0 = ((size_t)n * p.H + hk) * K, gi = (size_t)n * p.HV + hv;
      if (tid < CKQ) {
        cp_async16(st + St::TK + 16 * tid, reinterpret_cast<const unsigned char*>(k + qk0) + 16 * tid);
        cp_async16(st + St::TQ + 16 * tid, reinterpret_cast<const unsigned char*>(q + qk0) + 16 * tid);
      }
      if (tid >= 64 && tid < 64 + CV)
        cp_async16(st + St::TV + 16 * (tid - 64),
                   reinterpret_cast<const unsigned char*>(v + gi * p.V + v0) + 16 * (tid - 64));
      if constexpr (KDA) {
        if (tid >= 96 && tid < 96 + K / 4)
          cp_async16(st + St::TG + 16 * (tid - 96), a.g_raw + gi * K + 4 * (tid - 96));
      } else {
        if (tid == 96) cp_async4(st + St::TG, a.g_raw + gi);
      }
      if (tid == 127) cp_async4(st + St::TB, a.beta + gi);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  const int i0 = blockIdx.x;
  issue(i0, 0);
  issue(i0 + G, 1);
  const bool b3 = kg & 8, b2 = kg & 4;
  auto rowsum4 = [&](const float4& e) {
    float s0 = b3 ? e.z : e.x, s1 = b3 ? e.w : e.y;
    s0 += __shfl_xor_sync(0xffffffffu, b3 ? e.x : e.z, 8);
    s1 += __shfl_xor_sync(0xffffffffu, b3 ? e.y : e.w, 8);
    float t = b2 ? s1 : s0;
    t += __shfl_xor_sync(0xffffffffu, b2 ? s0 : s1, 4);
    t += __shfl_xor_sync(0xffffffffu, t, 2);
    t += __shfl_xor_sync(0xffffffffu, t, 1);
    return t;
  };
  const int half = lane & 16;
  auto gather4 = [&](float t) {
    return make_float4(__shfl_sync(0xffffffffu, t, half), __shfl_sync(0xffffffffu, t, half + 4),
                       __shfl_sync(0xffffffffu, t, half + 8), __shfl_sync(0xffffffffu, t, half + 12));
  };
  int slot = 0;
  for (int it = i0; it < nitems; it += G, slot ^= 1) {
    asm volatile("cp.async.wait_group 1;" ::: "memory");
    __syncthreads();  // the item's stage has landed for every thread
    const unsigned char* st = dsm + slot * St::BYTES;
    const int z = it % nz, nh = it / nz, n = nh / p.HV, hv = nh % p.HV, v0 = RV * z;
    float4 S4[KQ];
    float kv[KQ], qv[KQ], dv[KQ], vv[4];
#pragma unroll
    for (int i = 0; i < KQ; ++i)
      S4[i] = *reinterpret_cast<const float4*>(st + ((kg * KQ + i) * RV + 4 * slice_slot(kg * KQ + i, vg)) * 4);
    ld_floats<T, KQ>(reinterpret_cast<const T*>(st + St::TK) + kg * KQ, kv);
    ld_floats<T, KQ>(reinterpret_cast<const T*>(st + St::TQ) + kg * KQ, qv);
    ld_floats<T, 4>(reinterpret_cast<const T*>(st + St::TV) + 4 * vg, vv);
    const float b = *reinterpret_cast<const float*>(st + St::TB);
    const float nexp = -expf(a.A_log[hv]);
    if constexpr (KDA) {
      const float* gk = reinterpret_cast<const float*>(st + St::TG);
#pragma unroll
      for (int i = 0; i < KQ; ++i) {
        const int c = kg * KQ + i;
        const float gf = gk[c] + (a.dt_bias ? a.dt_bias[(size_t)hv * K + c] : 0.f);
        dv[i] = expf(nexp * softplus20(gf));
      }
    } else {
      const float gf = *reinterpret_cast<const float*>(st + St::TG) + a.dt_bias[hv];
      const float dec = expf(nexp * softplus20(gf));
#pragma unroll
      for (int i = 0; i < KQ; ++i) dv[i] = dec;
    }
    __syncthreads();  // every thread has read the stage: it takes the item two ahead
    issue(it + 2 * G, slot);
    float4 e = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < KQ; ++i) {
      const float dec = dv[i];
      S4[i].x *= dec; S4[i].y *= dec; S4[i].z *= dec; S4[i].w *= dec;
      e.x += S4[i].x * kv[i]; e.y += S4[i].y * kv[i]; e.z += S4[i].z * kv[i]; e.w += S4[i].w * kv[i];
    }
    e = gather4(rowsum4(e));
    const float dx = b * (vv[0] - e.x), dy = b * (vv[1] - e.y), dz = b * (vv[2] - e.z),
                dw = b * (vv[3] - e.w);
    float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < KQ; ++i) {
      S4[i].x += dx * kv[i]; S4[i].y += dy * kv[i]; S4[i].z += dz * kv[i]; S4[i].w += dw * kv[i];
      y.x += S4[i].x * qv[i]; y.y += S4[i].y * qv[i]; y.z += S4[i].z * qv[i]; y.w += S4[i].w * qv[i];
    }
    const float yt = rowsum4(y);
    if ((kg & 3) == 0) o[((size_t)n * p.HV + hv) * p.V + v0 + 4 * vg + (kg >> 2)] = from_f<T>(p.scale * yt);
    if (a.ht) {
      float* ht = a.ht + (size_t)nh * K * p.V + v0 + 4 * vg;
#pragma unroll
      for (int i = 0; i < KQ; ++i) *reinterpret_cast<float4*>(ht + (size_t)(kg * KQ + i) * p.V) = S4[i];
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

template <typename T, int K, bool KDA>
cudaError_t launch_decode(const Problem& p, const Args& a, cudaStream_t s) {
  using St = DecodeStage<T, K, KDA>;
  const int nitems = p.Nst * p.HV * (p.V / RV);
  int dev = 0, sms = 0, per_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_decode_pipe<T, K, KDA>, 128, 2 * St::BYTES);
  if (e != cudaSuccess) return e;
  const int grid = std::min(nitems, std::max(1, sms * per_sm));
  k_decode_pipe<T, K, KDA><<<grid, 128, 2 * St::BYTES, s>>>(p, a, nitems);
  return cudaGetLastError();
}

template <typename T, bool KDA>
cudaError_t launch_t(const Problem& p, const Args& a, int* status, cudaStream_t s) {
  // a decode step (one token per sequence, an entering state): the pipelined persistent kernel
  if (!p.varlen && p.T == 1 && a.h0 && p.Nst * p.HV * (p.V / RV) >= 1024)
    return p.K == 128 ? launch_decode<T, 128, KDA>(p, a, s) : launch_decode<T, 64, KDA>(p, a, s);
  const dim3 grid((unsigned)p.Nst * (unsigned)(p.V / RV), p.HV);
  if (p.K == 128)
    k_recurrent_fwd<T, 128, KDA><<<grid, 128, 0, s>>>(p, a, status);
  else
    k_recurrent_fwd<T, 64, KDA><<<grid, 128, 0, s>>>(p, a, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t recurrent_forward(const Problem& p, const Args& a, int* status, bool bf16, cudaStream_t s,
                              bool kda) {
  if (p.Nst == 0) return cudaSuccess;
  ProfScope ps(kda ? "kda_recurrent_fwd" : "recurrent_fwd", s);
  if (kda)
    return bf16 ? launch_t<__nv_bfloat16, true>(p, a, status, s) : launch_t<float, true>(p, a, status, s);
  return bf16 ? launch_t<__nv_bfloat16, false>(p, a, status, s) : launch_t<float, false>(p, a, status, s);
}

}  // namespace gdn
