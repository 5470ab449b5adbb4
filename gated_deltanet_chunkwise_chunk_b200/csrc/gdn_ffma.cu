// fp32 CUDA-core (FFMA) kernels of the chunkwise gated delta rule.
//
// One block per (chunk, value head) for the chunk-parallel steps and one block per
// (sequence, value head) for the two sequential state scans.  Products are small
// register-blocked fp32 tile GEMMs over shared/global tiles.  This path serves fp32
// tensors (exact to ~1e-6 relative), where tensor-core tf32 would not meet the fp32
// tolerance; bf16 tensors take the tcgen05 path.
//
// Per chunk (64 tokens, zero-padded past the sequence end, G padded with G[L-1]):
//   A  = strict_lower(diag(beta) (K K^T * Gam)),  Gam_ij = exp(G_i - G_j) (i >= j)
//   T  = (I + A)^-1,   W = T diag(beta e^G) K,   U~ = T diag(beta) V
//   U  = U~ - W S^T                          (S: state entering the chunk, V x K)
//   O  = scale (diag(e^G) Q S^T + (Q K^T * Gam) U)
//   S' = e^{G_C} S + U^T diag(e^{G_C - G}) K
// and the backward terms of each product (see the kernels below).
#include "ffma_tiles.cuh"
#include "gdn_common.cuh"
#include "gdn_launch.h"

namespace gdn {
namespace {

__device__ __forceinline__ float warp_sum(float x) {
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

struct Unit {
  int gc, hv, hk, L, tok0;
};

__device__ __forceinline__ bool unit_begin(const Problem& p, const Work& w, Unit& u) {
  if (call_failed(w)) return false;
  u.gc = blockIdx.x;
  u.hv = blockIdx.y;
  const int4 e = w.chunk_tab[u.gc];
  if (e.x < 0) return false;
  u.hk = u.hv / p.G;
  u.L = e.z;
  u.tok0 = e.w;
  return true;
}

__device__ __forceinline__ size_t unit_off(const Problem& p, const Unit& u, int rows, int cols) {
  return ((size_t)u.gc * p.HV + u.hv) * rows * cols;
}

template <typename T>
__device__ __forceinline__ const T* q_rows(const Problem& p, const void* base, const Unit& u) {
  return static_cast<const T*>(base) + ((size_t)u.tok0 * p.H + u.hk) * p.K;
}
template <typename T>
__device__ __forceinline__ const T* v_rows(const Problem& p, const void* base, const Unit& u) {
  return static_cast<const T*>(base) + ((size_t)u.tok0 * p.HV + u.hv) * p.V;
}

__device__ __forceinline__ void load_gb(const Problem& p, const Work& w, int gc, int hv, float* sG,
                                        float* sb) {
  if (threadIdx.x < CH) {
    const size_t o = ((size_t)hv * p.NCmax + gc) * CH + threadIdx.x;
    sG[threadIdx.x] = w.G[o];
    if (sb) sb[threadIdx.x] = w.beta_p[o];
  }
}

// ------------------------------------------------------------------ forward
// WY representation: A, T = (I+A)^-1, W, U~ (and T itself for the backward).
template <typename T>
__global__ void __launch_bounds__(256) k_ffma_wy(Problem p, Args a, Work w, int store_T) {
  Unit u;
  if (!unit_begin(p, w, u)) return;
  const int K = p.K, V = p.V;
  extern __shared__ float sm[];
  float* sK = sm;
  float* sV = sK + CH * K;
  float* sA = sV + CH * V;
  float* sT = sA + CH * CH;
  float* sG = sT + CH * CH;
  float* sb = sG + CH;
  load_rows<T>(sK, q_rows<T>(p, a.k, u), (size_t)p.H * K, u.L, K);
  load_rows<T>(sV, v_rows<T>(p, a.v, u), (size_t)p.HV * V, u.L, V);
  load_gb(p, w, u.gc, u.hv, sG, sb);
  __syncthreads();
  mm(CH, CH, K, sA, CH, 1.f, false, sK, K, 1, sK, 1, K);  // K K^T
  __syncthreads();
  for (int i = threadIdx.x; i < CH * CH; i += blockDim.x) {
    const int r = i / CH, c = i % CH;
    sA[i] = c < r ? sb[r] * sA[i] * expf(sG[r] - sG[c]) : 0.f;
  }
  __syncthreads();
  // forward substitution, one column of T per thread: T[r][n] = d_rn - sum_{n<=j<r} A[r][j] T[j][n]
  if (threadIdx.x < CH) {
    const int n = threadIdx.x;
    for (int r = 0; r < CH; ++r) {
      float s = 0.f;
      if (r == n) s = 1.f;
      if (r > n) {
        for (int j = n; j < r; ++j) s -= sA[r * CH + j] * sT[j * CH + n];
      }
      sT[r * CH + n] = s;
    }
  }
  for (int i = threadIdx.x; i < CH * K; i += blockDim.x) sK[i] *= sb[i / K] * expf(sG[i / K]);
  for (int i = threadIdx.x; i < CH * V; i += blockDim.x) sV[i] *= sb[i / V];
  __syncthreads();
  mm(CH, K, CH, w.W + unit_off(p, u, CH, K), K, 1.f, false, sT, CH, 1, sK, K, 1);
  mm(CH, V, CH, w.Ut + unit_off(p, u, CH, V), V, 1.f, false, sT, CH, 1, sV, V, 1);
  if (store_T) copy_f(w.Tm + unit_off(p, u, CH, CH), sT, CH * CH);
}

// Sequential state scan over the chunks of one (sequence, value head):
// stores S entering each chunk and U = U~ - W S^T; returns the final state.
template <typename T>
__global__ void __launch_bounds__(256) k_ffma_scan_fwd(Problem p, Args a, Work w) {
  if (call_failed(w)) return;
  const int n = blockIdx.x, hv = blockIdx.y, hk = hv / p.G, K = p.K, V = p.V;
  const int4 sq = w.seq_tab[n];
  extern __shared__ float sm[];
  float* sS = sm;             // [V][K]
  float* sU = sS + V * K;     // [64][V]  U~, then U, then diag(e^{G_C - G}) U
  float* sK = sU + CH * V;    // [64][K]
  float* sW = sK + CH * K;    // [64][K]
  float* sG = sW + CH * K;    // [64]
  for (int i = threadIdx.x; i < V * K; i += blockDim.x) {
    const int vv = i / K, kk = i % K;
    sS[i] = a.h0 ? a.h0[(((size_t)n * p.HV + hv) * K + kk) * V + vv] : 0.f;
  }
  __syncthreads();
  for (int c = 0; c < sq.y; ++c) {
    const int gc = sq.x + c;
    const int4 e = w.chunk_tab[gc];
    const size_t uo = (size_t)gc * p.HV + hv;
    copy_async(sW, w.W + uo * CH * K, CH * K);
    copy_async(sU, w.Ut + uo * CH * V, CH * V);
    load_rows<T>(sK, static_cast<const T*>(a.k) + ((size_t)e.w * p.H + hk) * K, (size_t)p.H * K,
                 e.z, K);
    load_gb(p, w, gc, hv, sG, nullptr);
    float* U = w.U + uo * CH * V;
    copy_f(w.h + uo * V * K, sS, V * K);
    cp_async_wait_all();
    __syncthreads();
    mm(CH, V, K, sU, V, -1.f, true, sW, K, 1, sS, 1, K);  // U = U~ - W S^T
    __syncthreads();
    const float GC = sG[CH - 1];
    for (int i = threadIdx.x; i < CH * V; i += blockDim.x) {
      U[i] = sU[i];
      sU[i] *= expf(GC - sG[i / V]);
    }
    const float eg = expf(GC);
    for (int i = threadIdx.x; i < V * K; i += blockDim.x) sS[i] *= eg;
    __syncthreads();
    mm(V, K, CH, sS, K, 1.f, true, sU, 1, V, sK, K, 1);
    __syncthreads();
  }
  if (a.ht)
    for (int i = threadIdx.x; i < V * K; i += blockDim.x) {
      const int vv = i / K, kk = i % K;
      a.ht[(((size_t)n * p.HV + hv) * K + kk) * V + vv] = sS[i];
    }
}

// P = (Q K^T) * Gam (lower triangle incl. diagonal) into sP.
__device__ __forceinline__ void build_P(int K, const float* sQ, const float* sK, const float* sG,
                                        float* sP) {
  mm(CH, CH, K, sP, CH, 1.f, false, sQ, K, 1, sK, 1, K);
  __syncthreads();
  for (int i = threadIdx.x; i < CH * CH; i += blockDim.x) {
    const int r = i / CH, c = i % CH;
    sP[i] = c <= r ? sP[i] * expf(sG[r] - sG[c]) : 0.f;
  }
  __syncthreads();
}

// chunk_fwd_o: O = scale (diag(e^G) Q S^T + P U)
template <typename T>
__global__ void __launch_bounds__(256) k_ffma_out(Problem p, Args a, Work w) {
  Unit u;
  if (!unit_begin(p, w, u)) return;
  const int K = p.K, V = p.V;
  extern __shared__ float sm[];
  float* sQ = sm;
  float* sK = sQ + CH * K;
  float* sP = sK + CH * K;
  float* sO = sP + CH * CH;
  float* sG = sO + CH * V;
  load_rows<T>(sQ, q_rows<T>(p, a.q, u), (size_t)p.H * K, u.L, K);
  load_rows<T>(sK, q_rows<T>(p, a.k, u), (size_t)p.H * K, u.L, K);
  load_gb(p, w, u.gc, u.hv, sG, nullptr);
  __syncthreads();
  build_P(K, sQ, sK, sG, sP);
  mm(CH, V, CH, sO, V, 1.f, false, sP, CH, 1, w.U + unit_off(p, u, CH, V), V, 1);
  for (int i = threadIdx.x; i < CH * K; i += blockDim.x) sQ[i] *= expf(sG[i / K]);
  __syncthreads();
  mm(CH, V, K, sO, V, 1.f, true, sQ, K, 1, w.h + unit_off(p, u, V, K), 1, K);
  __syncthreads();
  T* o = static_cast<T*>(a.o) + ((size_t)u.tok0 * p.HV + u.hv) * V;
  for (int i = threadIdx.x; i < u.L * V; i += blockDim.x) {
    const int t = i / V, c = i % V;
    o[(size_t)t * p.HV * V + c] = from_f<T>(p.scale * sO[i]);
  }
}

// ------------------------------------------------------------------ backward
// dv_local: dU_loc = scale P^T dO
template <typename T>
__global__ void __launch_bounds__(256) k_ffma_dvlocal(Problem p, Args a, Work w) {
  Unit u;
  if (!unit_begin(p, w, u)) return;
  const int K = p.K, V = p.V;
  extern __shared__ float sm[];
  float* sQ = sm;
  float* sK = sQ + CH * K;
  float* sP = sK + CH * K;
  float* sdO = sP + CH * CH;
  float* sG = sdO + CH * V;
  load_rows<T>(sQ, q_rows<T>(p, a.q, u), (size_t)p.H * K, u.L, K);
  load_rows<T>(sK, q_rows<T>(p, a.k, u), (size_t)p.H * K, u.L, K);
  load_rows<T>(sdO, v_rows<T>(p, a.dO, u), (size_t)p.HV * V, u.L, V);
  load_gb(p, w, u.gc, u.hv, sG, nullptr);
  __syncthreads();
  build_P(K, sQ, sK, sG, sP);
  mm(CH, V, CH, w.dU + unit_off(p, u, CH, V), V, p.scale, false, sP, 1, CH, sdO, V, 1);
}

// Reverse scan: dU = dU_loc + diag(e^{G_C-G}) K dS'^T ;
// dS = e^{G_C} dS' + scale (diag(e^G) dO)^T Q - dU^T W.  Stores dS' (leaving) per chunk.
template <typename T>
__global__ void __launch_bounds__(256) k_ffma_scan_bwd(Problem p, Args a, Work w) {
  if (call_failed(w)) return;
  const int n = blockIdx.x, hv = blockIdx.y, hk = hv / p.G, K = p.K, V = p.V;
  const int4 sq = w.seq_tab[n];
  extern __shared__ float sm[];
  float* sdS = sm;             // [V][K]
  float* sX = sdS + V * K;     // [64][K]: K * D, then Q
  float* sdO = sX + CH * K;    // [64][V]
  float* sdU = sdO + CH * V;   // [64][V]  dU_loc, then dU
  float* sW = sdU + CH * V;    // [64][K]
  float* sG = sW + CH * K;
  float* sD = sG + CH;
  for (int i = threadIdx.x; i < V * K; i += blockDim.x) {
    const int vv = i / K, kk = i % K;
    sdS[i] = a.dht ? a.dht[(((size_t)n * p.HV + hv) * K + kk) * V + vv] : 0.f;
  }
  __syncthreads();
  for (int c = sq.y - 1; c >= 0; --c) {
    const int gc = sq.x + c;
    const int4 e = w.chunk_tab[gc];
    const size_t uo = (size_t)gc * p.HV + hv;
    load_gb(p, w, gc, hv, sG, nullptr);
    __syncthreads();
    const float GC = sG[CH - 1];
    if (threadIdx.x < CH) sD[threadIdx.x] = expf(GC - sG[threadIdx.x]);
    __syncthreads();
    float* dU = w.dU + uo * CH * V;
    copy_async(sdU, dU, CH * V);
    copy_async(sW, w.W + uo * CH * K, CH * K);
    load_rows<T>(sX, static_cast<const T*>(a.k) + ((size_t)e.w * p.H + hk) * K, (size_t)p.H * K,
                 e.z, K, sD);
    copy_f(w.dh + uo * V * K, sdS, V * K);
    cp_async_wait_all();
    __syncthreads();
    mm(CH, V, K, sdU, V, 1.f, true, sX, K, 1, sdS, 1, K);  // dU = dU_loc + (D K) dS'^T
    __syncthreads();
    const float eg = expf(GC);
    for (int i = threadIdx.x; i < CH * V; i += blockDim.x) dU[i] = sdU[i];
    for (int i = threadIdx.x; i < V * K; i += blockDim.x) sdS[i] *= eg;
    if (threadIdx.x < CH) sD[threadIdx.x] = p.scale * expf(sG[threadIdx.x]);
    __syncthreads();
    load_rows<T>(sX, static_cast<const T*>(a.q) + ((size_t)e.w * p.H + hk) * K, (size_t)p.H * K,
                 e.z, K);
    load_rows<T>(sdO, static_cast<const T*>(a.dO) + ((size_t)e.w * p.HV + hv) * V,
                 (size_t)p.HV * V, e.z, V, sD);
    __syncthreads();
    mm(V, K, CH, sdS, K, 1.f, true, sdO, 1, V, sX, K, 1);
    mm(V, K, CH, sdS, K, -1.f, true, sdU, 1, V, sW, K, 1);
    __syncthreads();
  }
  if (a.dh0)
    for (int i = threadIdx.x; i < V * K; i += blockDim.x) {
      const int vv = i / K, kk = i % K;
      a.dh0[(((size_t)n * p.HV + hv) * K + kk) * V + vv] = sdS[i];
    }
}

// dq/dk shares from the output path and the state terms, dW = -dU S, and the dG terms
// rowsum(dP.P) - colsum(dP.P) + scale e^G <dO, S q> - D u^T dS' k (+ the G_C terms).
template <typename T>
__global__ void __launch_bounds__(256) k_ffma_dqkwg(Problem p, Args a, Work w) {
  Unit u;
  if (!unit_begin(p, w, u)) return;
  const int K = p.K, V = p.V;
  extern __shared__ float sm[];
  float* sQ = sm;
  float* sK = sQ + CH * K;
  float* sdO = sK + CH * K;
  float* sP = sdO + CH * V;
  float* sdP = sP + CH * CH;
  float* sG = sdP + CH * CH;
  float* sdG = sG + CH;
  float* sred = sdG + CH;  // [8]
  const float* U = w.U + unit_off(p, u, CH, V);
  const float* dU = w.dU + unit_off(p, u, CH, V);
  const float* S = w.h + unit_off(p, u, V, K);
  const float* dSn = w.dh + unit_off(p, u, V, K);
  float* dW = w.dW + unit_off(p, u, CH, K);
  float* dqp = w.dqp + unit_off(p, u, CH, K);
  float* dkp = w.dkp + unit_off(p, u, CH, K);
  float* Y = w.tmp + unit_off(p, u, CH, 128);
  load_rows<T>(sQ, q_rows<T>(p, a.q, u), (size_t)p.H * K, u.L, K);
  load_rows<T>(sK, q_rows<T>(p, a.k, u), (size_t)p.H * K, u.L, K);
  load_rows<T>(sdO, v_rows<T>(p, a.dO, u), (size_t)p.HV * V, u.L, V);
  load_gb(p, w, u.gc, u.hv, sG, nullptr);
  __syncthreads();
  mm(CH, CH, K, sP, CH, 1.f, false, sQ, K, 1, sK, 1, K);
  mm(CH, CH, V, sdP, CH, p.scale, false, sdO, V, 1, U, 1, V);
  __syncthreads();
  for (int i = threadIdx.x; i < CH * CH; i += blockDim.x) {
    const int r = i / CH, c = i % CH;
    if (c <= r) {
      sP[i] *= expf(sG[r] - sG[c]);
    } else {
      sP[i] = 0.f;
      sdP[i] = 0.f;
    }
  }
  __syncthreads();
  if (threadIdx.x < CH) {
    const int r = threadIdx.x;
    float s = 0.f;
    for (int c = 0; c < CH; ++c) s += sdP[r * CH + c] * sP[r * CH + c] - sdP[c * CH + r] * sP[c * CH + r];
    sdG[r] = s;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < CH * CH; i += blockDim.x) {
    const int r = i / CH, c = i % CH;
    sdP[i] = c <= r ? sdP[i] * expf(sG[r] - sG[c]) : 0.f;
  }
  __syncthreads();
  mm(CH, K, CH, dqp, K, 1.f, false, sdP, CH, 1, sK, K, 1);
  mm(CH, K, CH, dkp, K, 1.f, false, sdP, 1, CH, sQ, K, 1);
  for (int i = threadIdx.x; i < CH * V; i += blockDim.x) sdO[i] *= p.scale * expf(sG[i / V]);
  __syncthreads();
  // dQ1 = scale diag(e^G) dO S (staged in dW), dG += rowsum(dQ1 * Q), dq += dQ1
  mm(CH, K, V, dW, K, 1.f, false, sdO, V, 1, S, K, 1);
  __syncthreads();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, nw = blockDim.x / 32;
  for (int r = warp; r < CH; r += nw) {
    float s = 0.f;
    for (int c = lane; c < K; c += 32) {
      const float x = dW[r * K + c];
      dqp[r * K + c] += x;
      s += x * sQ[r * K + c];
    }
    s = warp_sum(s);
    if (lane == 0) sdG[r] += s;
  }
  __syncthreads();
  mm(CH, K, V, dW, K, -1.f, false, dU, V, 1, S, K, 1);
  mm(CH, K, V, Y, K, 1.f, false, U, V, 1, dSn, K, 1);
  __syncthreads();
  const float GC = sG[CH - 1];
  float racc = 0.f;
  for (int r = warp; r < CH; r += nw) {
    const float D = expf(GC - sG[r]);
    float s = 0.f;
    for (int c = lane; c < K; c += 32) {
      const float y = Y[r * K + c];
      dkp[r * K + c] += D * y;
      s += y * sK[r * K + c];
    }
    s = warp_sum(s) * D;
    if (lane == 0) sdG[r] -= s;
    racc += s;
  }
  float dot = 0.f;
  for (int i = threadIdx.x; i < V * K; i += blockDim.x) dot += dSn[i] * S[i];
  dot = warp_sum(dot);
  if (lane == 0) sred[warp] = dot * expf(GC) + racc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
    for (int i = 0; i < nw; ++i) s += sred[i];
    sdG[CH - 1] += s;
  }
  __syncthreads();
  if (threadIdx.x < CH) w.dG[((size_t)u.hv * p.NCmax + u.gc) * CH + threadIdx.x] = sdG[threadIdx.x];
}

// WY backward: dT = dU Y^T + dW X^T, dX = T^T dW, dY = T^T dU, dA = -(T^T dT T^T) strict
// lower; dv = beta dY; dbeta; dk += diag(beta e^G) dX + dAs K + dAs^T K; dG terms.
template <typename T>
__global__ void __launch_bounds__(256) k_ffma_wy_bwd(Problem p, Args a, Work w) {
  Unit u;
  if (!unit_begin(p, w, u)) return;
  const int K = p.K, V = p.V;
  extern __shared__ float sm[];
  float* sK = sm;
  float* sV = sK + CH * K;
  float* sT = sV + CH * V;
  float* sdT = sT + CH * CH;
  float* sdT2 = sdT + CH * CH;
  float* sKK = sdT2 + CH * CH;
  float* sZ = sKK + CH * CH;
  float* sG = sZ + CH * CH;
  float* sb = sG + CH;
  float* sdb = sb + CH;
  float* sdG = sdb + CH;
  const float* dU = w.dU + unit_off(p, u, CH, V);
  const float* dW = w.dW + unit_off(p, u, CH, K);
  float* dkp = w.dkp + unit_off(p, u, CH, K);
  float* X = w.tmp + unit_off(p, u, CH, 128);
  load_rows<T>(sK, q_rows<T>(p, a.k, u), (size_t)p.H * K, u.L, K);
  load_rows<T>(sV, v_rows<T>(p, a.v, u), (size_t)p.HV * V, u.L, V);
  copy_f(sT, w.Tm + unit_off(p, u, CH, CH), CH * CH);
  load_gb(p, w, u.gc, u.hv, sG, sb);
  __syncthreads();
  mm(CH, CH, V, sdT, CH, 1.f, false, dU, V, 1, sV, 1, V);
  mm(CH, CH, K, sdT2, CH, 1.f, false, dW, K, 1, sK, 1, K);
  mm(CH, CH, K, sKK, CH, 1.f, false, sK, K, 1, sK, 1, K);
  __syncthreads();
  for (int i = threadIdx.x; i < CH * CH; i += blockDim.x) {
    const int c = i % CH;
    sdT[i] = sb[c] * (sdT[i] + expf(sG[c]) * sdT2[i]);
  }
  __syncthreads();
  mm(CH, CH, CH, sZ, CH, 1.f, false, sT, 1, CH, sdT, CH, 1);      // T^T dT
  __syncthreads();
  mm(CH, CH, CH, sdT2, CH, -1.f, false, sZ, CH, 1, sT, 1, CH);    // -(T^T dT) T^T
  __syncthreads();
  for (int i = threadIdx.x; i < CH * CH; i += blockDim.x) {
    const int r = i / CH, c = i % CH;
    if (c < r) {
      const float gam = expf(sG[r] - sG[c]);
      const float dA = sdT2[i];
      const float Av = sb[r] * gam * sKK[i];
      sZ[i] = dA * Av;
      sdT[i] = dA * gam * sb[r];
      sKK[i] = dA * gam * sKK[i];
    } else {
      sZ[i] = 0.f;
      sdT[i] = 0.f;
      sKK[i] = 0.f;
    }
  }
  __syncthreads();
  if (threadIdx.x < CH) {
    const int r = threadIdx.x;
    float db = 0.f, dg = 0.f;
    for (int c = 0; c < CH; ++c) {
      db += sKK[r * CH + c];
      dg += sZ[r * CH + c] - sZ[c * CH + r];
    }
    sdb[r] = db;
    sdG[r] = dg;
  }
  mm(CH, K, CH, dkp, K, 1.f, true, sdT, CH, 1, sK, K, 1);
  mm(CH, K, CH, dkp, K, 1.f, true, sdT, 1, CH, sK, K, 1);
  mm(CH, K, CH, X, K, 1.f, false, sT, 1, CH, dW, K, 1);           // dX = T^T dW
  __syncthreads();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, nw = blockDim.x / 32;
  for (int r = warp; r < CH; r += nw) {
    const float eg = expf(sG[r]);
    float s = 0.f;
    for (int c = lane; c < K; c += 32) {
      const float x = X[r * K + c];
      dkp[r * K + c] += sb[r] * eg * x;
      s += x * sK[r * K + c];
    }
    s = warp_sum(s);
    if (lane == 0) {
      sdb[r] += eg * s;
      sdG[r] += sb[r] * eg * s;
    }
  }
  __syncthreads();
  mm(CH, V, CH, X, V, 1.f, false, sT, 1, CH, dU, V, 1);           // dY = T^T dU
  __syncthreads();
  T* dv = static_cast<T*>(a.dv) + ((size_t)u.tok0 * p.HV + u.hv) * V;
  for (int r = warp; r < CH; r += nw) {
    float s = 0.f;
    for (int c = lane; c < V; c += 32) {
      const float y = X[r * V + c];
      if (r < u.L) dv[(size_t)r * p.HV * V + c] = from_f<T>(sb[r] * y);
      s += y * sV[r * V + c];
    }
    s = warp_sum(s);
    if (lane == 0) sdb[r] += s;
  }
  __syncthreads();
  if (threadIdx.x < CH) {
    const int r = threadIdx.x;
    if (r < u.L) a.dbeta[(size_t)(u.tok0 + r) * p.HV + u.hv] = sdb[r];
    w.dG[((size_t)u.hv * p.NCmax + u.gc) * CH + r] += sdG[r];
  }
}

template <typename Kern>
cudaError_t launch(const char* name, Kern k, dim3 grid, size_t smem, cudaStream_t s,
                   const Problem& p, const Args& a, const Work& w) {
  if (grid.x == 0 || grid.y == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ProfScope ps(name, s);
  k<<<grid, 256, smem, s>>>(p, a, w);
  return cudaGetLastError();
}

template <typename T>
cudaError_t forward_t(const Problem& p, const Args& a, const Work& w, bool bwd_prep, cudaStream_t s) {
  const int K = p.K, V = p.V;
  const dim3 gu(p.NCmax, p.HV), gs(p.Nst, p.HV);
  size_t smem = sizeof(float) * (CH * K + CH * V + 2 * CH * CH + 2 * CH);
  cudaError_t e = cudaFuncSetAttribute(k_ffma_wy<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  if (p.NCmax > 0) {
    ProfScope ps("ffma_wy", s);
    k_ffma_wy<T><<<gu, 256, smem, s>>>(p, a, w, bwd_prep ? 1 : 0);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  Args a2 = a;
  if (bwd_prep) a2.ht = nullptr;
  smem = sizeof(float) * (V * K + CH * V + 2 * CH * K + CH);
  if ((e = launch("ffma_scan_fwd", k_ffma_scan_fwd<T>, gs, smem, s, p, a2, w)) != cudaSuccess) return e;
  if (!bwd_prep) {
    smem = sizeof(float) * (2 * CH * K + CH * CH + CH * V + CH);
    if ((e = launch("ffma_out", k_ffma_out<T>, gu, smem, s, p, a, w)) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <typename T>
cudaError_t backward_t(const Problem& p, const Args& a, const Work& w, cudaStream_t s) {
  const int K = p.K, V = p.V;
  const dim3 gu(p.NCmax, p.HV), gs(p.Nst, p.HV);
  cudaError_t e;
  size_t smem = sizeof(float) * (2 * CH * K + CH * CH + CH * V + CH);
  if ((e = launch("ffma_dvlocal", k_ffma_dvlocal<T>, gu, smem, s, p, a, w)) != cudaSuccess) return e;
  smem = sizeof(float) * (V * K + 2 * CH * K + 2 * CH * V + 2 * CH);
  if ((e = launch("ffma_scan_bwd", k_ffma_scan_bwd<T>, gs, smem, s, p, a, w)) != cudaSuccess) return e;
  smem = sizeof(float) * (2 * CH * K + CH * V + 2 * CH * CH + 2 * CH + 8);
  if ((e = launch("ffma_dqkwg", k_ffma_dqkwg<T>, gu, smem, s, p, a, w)) != cudaSuccess) return e;
  smem = sizeof(float) * (CH * K + CH * V + 5 * CH * CH + 4 * CH);
  if ((e = launch("ffma_wy_bwd", k_ffma_wy_bwd<T>, gu, smem, s, p, a, w)) != cudaSuccess) return e;
  return cudaSuccess;
}

}  // namespace

cudaError_t ffma_forward(const Problem& p, const Args& a, const Work& w, bool bf16, bool bwd_prep,
                         cudaStream_t s) {
  return bf16 ? forward_t<__nv_bfloat16>(p, a, w, bwd_prep, s) : forward_t<float>(p, a, w, bwd_prep, s);
}

cudaError_t ffma_backward(const Problem& p, const Args& a, const Work& w, bool bf16, cudaStream_t s) {
  return bf16 ? backward_t<__nv_bfloat16>(p, a, w, s) : backward_t<float>(p, a, w, s);
}

}  // namespace gdn
