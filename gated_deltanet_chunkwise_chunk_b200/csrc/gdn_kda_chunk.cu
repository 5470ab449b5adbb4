// Chunkwise forward of the KDA delta rule (a decay per key channel) on CUDA cores (fp32).
//
// Recurrence (state S: V x K per value head, h[k][v] = S[v][k] in memory):
//   S_t = S_{t-1} Diag(e^{yg_t}) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = scale S_t q_t,
//   yg_t[c] = -exp(A_log[hv]) softplus(g_raw[t, hv, c] + dt_bias[hv*K + c])  (the KDA gate of the
//   MindSpeed-Ops "KDA gate" task, fused here), i.e. the Gated DeltaNet recurrence with the scalar
//   decay replaced by one per key channel; the pages name the KDA chunk kernels beside the Gated
//   DeltaNet ones (G_T_CONTIG article).
//
// Per 64-token chunk (rows past the sequence end: yg = 0, beta = 0, zero tokens), with
// Gam_i = inclusive cumsum of yg over the chunk (a K-vector per token):
//   A_ij = beta_i sum_c k_i[c] k_j[c] e^{Gam_i[c] - Gam_j[c]} (j < i),   T = (I + A)^-1
//   P_ij =        sum_c q_i[c] k_j[c] e^{Gam_i[c] - Gam_j[c]} (j <= i)
//   W = T diag(beta) (k e^{Gam}),  U~ = T diag(beta) V,  U = U~ - W S^T
//   O = scale ((q e^{Gam}) S^T + P U),  S' = S Diag(e^{Gam_C}) + U^T (k e^{Gam_C - Gam})
// A and P are built in 16-token sub-chunks: across sub-chunks, e^{Gam_i - Gam_j} =
// e^{Gam_i - Gam_r} e^{Gam_r - Gam_j} with r the last token before i's sub-chunk (both factors
// <= 1), so each block is a tile product of rescaled keys and queries; inside a sub-chunk the
// per-channel terms are summed directly (a factored e^{-Gam_j} overflows fp32 within a few
// tokens at strong decay).  Every exponent is <= 0, so nothing overflows.
//
// Three kernels: k_kda_wy per (chunk, value head) builds everything chunk-local; k_kda_scan per
// (sequence, value head, 32-row slice of S) carries the state through the chunks; k_kda_out per
// (chunk, value head) forms the output.
#include "ffma_tiles.cuh"
#include "gdn_common.cuh"
#include "gdn_launch.h"
#include "gdn_tc_common.cuh"  // unit_lower_inverse64, LDA

namespace gdn {
namespace {

constexpr int SUB = 16;  // sub-chunk length
constexpr int RS = 52;   // row stride of the transposed key tile R^T (16-byte rows for float4 reads)
constexpr float LOG2E = 1.4426950408889634f;
using tcx::LDA;          // row stride of A, T and the inverse's scratch

__device__ __forceinline__ bool kda_failed(const KdaWork& w) { return *((volatile int*)w.status) != 0; }

__device__ __forceinline__ float warp_total(float x) {
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

__host__ __device__ constexpr int wy_scratch(int K) {
  return 2 * SUB * (K + 1) + RS * K > 2 * CH * LDA ? 2 * SUB * (K + 1) + RS * K : 2 * CH * LDA;
}
size_t wy_smem(int K, int V) {
  return (size_t)(3 * CH * K + CH * V + CH * LDA + CH * CH + wy_scratch(K) + CH) * sizeof(float);
}
size_t scan_smem(int K) { return (size_t)(32 * (K + 1) + CH * (K + 1) + CH * K + CH * 32 + K) * sizeof(float); }
size_t out_smem(int K, int V) { return (size_t)(CH * K + CH * CH + K * (V + 1) + 2 * CH * V) * sizeof(float); }

template <typename T>
__global__ void __launch_bounds__(256) k_kda_wy(Problem p, Args a, KdaWork w) {
  if (kda_failed(w)) return;
  const int gc = blockIdx.x, hv = blockIdx.y;
  const int4 e = w.chunk_tab[gc];
  if (e.x < 0) return;
  const int K = p.K, V = p.V, L = e.z, tok0 = e.w, hk = hv / p.G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarp = blockDim.x >> 5;
  extern __shared__ float sm[];
  float* sK = sm;             // [64][K] keys; later beta e^{Gam} k
  float* sQ = sK + CH * K;    // [64][K] queries
  float* sG = sQ + CH * K;    // [64][K] Gam * log2(e)
  float* sV = sG + CH * K;    // [64][V]
  float* sA = sV + CH * V;    // [64][LDA]
  float* sP = sA + CH * LDA;  // [64][64]
  float* sX = sP + CH * CH;   // scratch: Lk [16][K+1], Lq [16][K+1], R^T [K][RS]; later T, X [64][LDA]
  float* sb = sX + wy_scratch(K);  // [64] beta, 0 past L
  const size_t rs = (size_t)p.H * K;
  load_tile<T>(sK, K, static_cast<const T*>(a.k) + ((size_t)tok0 * p.H + hk) * K, rs, L, K);
  load_tile<T>(sQ, K, static_cast<const T*>(a.q) + ((size_t)tok0 * p.H + hk) * K, rs, L, K);
  load_tile<T>(sV, V, static_cast<const T*>(a.v) + ((size_t)tok0 * p.HV + hv) * V, (size_t)p.HV * V, L, V);
  load_tile<float>(sG, K, a.g_raw + ((size_t)tok0 * p.HV + hv) * K, (size_t)p.HV * K, L, K);
  if (tid < CH) sb[tid] = tid < L ? a.beta[(size_t)(tok0 + tid) * p.HV + hv] : 0.f;
  __syncthreads();
  {  // the gate of every (token, channel), rows past L zero; then the cumsum per channel
    const float nexp = -expf(a.A_log[hv]);
    for (int x = tid; x < CH * K; x += blockDim.x) {
      const int i = x / K, c = x % K;
      float yg = 0.f;
      if (i < L) {
        const float z = sG[x] + (a.dt_bias ? a.dt_bias[(size_t)hv * K + c] : 0.f);
        yg = nexp * (z > 20.f ? z : log1pf(expf(z)));
      }
      sG[x] = yg;
    }
    __syncthreads();
    for (int c = tid; c < K; c += blockDim.x) {
      float acc = 0.f;
      for (int i = 0; i < CH; ++i) {
        acc += sG[i * K + c];
        sG[i * K + c] = acc * LOG2E;
      }
    }
  }
  for (int x = tid; x < CH * LDA; x += blockDim.x) sA[x] = 0.f;
  for (int x = tid; x < CH * CH; x += blockDim.x) sP[x] = 0.f;
  __syncthreads();
  // diagonal sub-blocks, one warp per pair (i, j), j <= i in one sub-chunk, lanes over channels
  constexpr int PAIRS = SUB * (SUB + 1) / 2;
  for (int pr = warp; pr < (CH / SUB) * PAIRS; pr += nwarp) {
    const int blk = pr / PAIRS;
    int q = pr % PAIRS, ii = 0;
    while (q > ii) q -= ++ii;  // q in [0, ii]
    const int i = blk * SUB + ii, j = blk * SUB + q;
    float sa = 0.f, sp = 0.f;
    for (int c = lane; c < K; c += 32) {
      const float kj = sK[j * K + c] * exp2f(sG[i * K + c] - sG[j * K + c]);
      sa = fmaf(sK[i * K + c], kj, sa);
      sp = fmaf(sQ[i * K + c], kj, sp);
    }
    sa = warp_total(sa);
    sp = warp_total(sp);
    if (lane == 0) {
      if (j < i) sA[i * LDA + j] = sb[i] * sa;
      sP[i * CH + j] = sp;
    }
  }
  // blocks below the diagonal, through the reference token r = last token before sub-chunk blk
  float* Lk = sX;                    // [16][K+1]
  float* Lq = sX + SUB * (K + 1);    // [16][K+1]
  float* RT = sX + 2 * SUB * (K + 1);  // [K][RS]: RT[c][j] = k_j[c] e^{Gam_r[c] - Gam_j[c]}
  for (int blk = 1; blk < CH / SUB; ++blk) {
    const int r = blk * SUB - 1, nj = blk * SUB;
    __syncthreads();  // the previous block's products are done with the scratch
    for (int x = tid; x < SUB * K; x += blockDim.x) {
      const int ii = x / K, c = x % K, i = blk * SUB + ii;
      const float ex = exp2f(sG[i * K + c] - sG[r * K + c]);
      Lk[ii * (K + 1) + c] = sK[i * K + c] * ex;
      Lq[ii * (K + 1) + c] = sQ[i * K + c] * ex;
    }
    for (int x = tid; x < nj * K; x += blockDim.x) {
      const int j = x / K, c = x % K;
      RT[c * RS + j] = sK[x] * exp2f(sG[r * K + c] - sG[x]);
    }
    __syncthreads();
    // one 1 x 4 strip of A (times beta_i) or P per task: all threads busy for every block
    const int ns = nj / 4, per = SUB * ns;
    for (int tk = tid; tk < 2 * per; tk += blockDim.x) {
      const int mat = tk / per, ii = (tk % per) / ns, j4 = 4 * (tk % ns), i = blk * SUB + ii;
      const float* lrow = (mat ? Lq : Lk) + ii * (K + 1);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
      for (int c = 0; c < K; ++c) {
        const float l = lrow[c];
        const float4 rt = *reinterpret_cast<const float4*>(RT + c * RS + j4);
        acc.x = fmaf(l, rt.x, acc.x);
        acc.y = fmaf(l, rt.y, acc.y);
        acc.z = fmaf(l, rt.z, acc.z);
        acc.w = fmaf(l, rt.w, acc.w);
      }
      if (mat) {
        *reinterpret_cast<float4*>(sP + i * CH + j4) = acc;
      } else {
        const float b = sb[i];
        *reinterpret_cast<float4*>(sA + i * LDA + j4) = make_float4(b * acc.x, b * acc.y, b * acc.z, b * acc.w);
      }
    }
  }
  __syncthreads();
  const size_t u = (size_t)gc * p.HV + hv;
  float* gP = w.P + u * CH * CH;
  for (int x = tid; x < CH * CH; x += blockDim.x) gP[x] = sP[x];
  if (w.Gam)
    for (int x = tid; x < CH * K; x += blockDim.x) w.Gam[u * CH * K + x] = sG[x];
  float* sT = sX;
  tcx::unit_lower_inverse64(sA, sT, sX + CH * LDA, tid);  // T = (I + A)^-1 (ends with a barrier)
  if (w.Tm)
    for (int x = tid; x < CH * CH; x += blockDim.x) w.Tm[u * CH * CH + x] = sT[(x / CH) * LDA + x % CH];
  // K^ = k e^{Gam_C - Gam}, Q~ = q e^{Gam}, e^{Gam_C}; then beta e^{Gam} k in place for W
  const size_t uk = u * CH * K;
  for (int x = tid; x < CH * K; x += blockDim.x) {
    const int i = x / K, c = x % K;
    const float g = sG[x], gC = sG[(CH - 1) * K + c];
    w.Kh[uk + x] = sK[x] * exp2f(gC - g);
    w.Qt[uk + x] = sQ[x] * exp2f(g);
    sK[x] *= sb[i] * exp2f(g);
  }
  for (int c = tid; c < K; c += blockDim.x) w.eGC[u * K + c] = exp2f(sG[(CH - 1) * K + c]);
  for (int x = tid; x < CH * V; x += blockDim.x) sV[x] *= sb[x / V];
  __syncthreads();
  mm(CH, K, CH, w.W + uk, K, 1.f, false, sT, LDA, 1, sK, K, 1, 1);  // T lower triangular
  mm(CH, V, CH, w.Ut + u * CH * V, V, 1.f, false, sT, LDA, 1, sV, V, 1, 1);
}

// Sequential scan of one (sequence, value head, rows v0..v0+31 of S): stores the state entering
// each chunk (rows v of S, [V][K]) and U = U~ - W S^T for those rows, returns the final state.
// The next chunk's W, K^, U~ slice and e^{Gam_C} are loaded into registers while the current
// chunk's products run.
__global__ void __launch_bounds__(256) k_kda_scan(Problem p, Args a, KdaWork w) {
  if (kda_failed(w)) return;
  const int n = blockIdx.x, hv = blockIdx.y, v0 = 32 * blockIdx.z, K = p.K, V = p.V, tid = threadIdx.x;
  const int4 sq = w.seq_tab[n];
  extern __shared__ float sm[];
  float* sS = sm;                  // [32][K+1]
  float* sW = sS + 32 * (K + 1);   // [64][K+1]
  float* sKh = sW + CH * (K + 1);  // [64][K]
  float* sU = sKh + CH * K;        // [64][32]
  float* sE = sU + CH * 32;        // [K] e^{Gam_C}
  for (int x = tid; x < 32 * K; x += blockDim.x) {  // lanes along v: coalesced h0 reads
    const int vv = x % 32, c = x / 32;
    sS[vv * (K + 1) + c] = a.h0 ? a.h0[(((size_t)n * p.HV + hv) * K + c) * V + v0 + vv] : 0.f;
  }
  constexpr int NW = CH * 128 / 4 / 256;  // float4 of a [64][128] tile per thread
  const int nw = CH * K / 4 / 256;        // 8 (K = 128) or 4 (K = 64)
  float4 rW[NW], rK[NW];
  float rU[CH * 32 / 256], rE = 0.f;
  auto fetch = [&](size_t u) {
    const float4* gw = reinterpret_cast<const float4*>(w.W + u * CH * K);
    const float4* gk = reinterpret_cast<const float4*>(w.Kh + u * CH * K);
#pragma unroll
    for (int r = 0; r < NW; ++r)
      if (r < nw) {
        rW[r] = gw[tid + 256 * r];
        rK[r] = gk[tid + 256 * r];
      }
#pragma unroll
    for (int r = 0; r < CH * 32 / 256; ++r) {
      const int x = tid + 256 * r;
      rU[r] = w.Ut[u * CH * V + (x / 32) * V + v0 + x % 32];
    }
    if (tid < K) rE = w.eGC[u * K + tid];
  };
  auto stash = [&]() {
#pragma unroll
    for (int r = 0; r < NW; ++r)
      if (r < nw) {
        const int x = 4 * (tid + 256 * r), i = x / K, c = x % K;
        float* d = sW + i * (K + 1) + c;
        d[0] = rW[r].x; d[1] = rW[r].y; d[2] = rW[r].z; d[3] = rW[r].w;
        *reinterpret_cast<float4*>(sKh + x) = rK[r];
      }
#pragma unroll
    for (int r = 0; r < CH * 32 / 256; ++r) sU[tid + 256 * r] = rU[r];
    if (tid < K) sE[tid] = rE;
  };
  if (sq.y > 0) fetch((size_t)sq.x * p.HV + hv);
  for (int ci = 0; ci < sq.y; ++ci) {
    const size_t u = (size_t)(sq.x + ci) * p.HV + hv;
    __syncthreads();  // the previous chunk is done with every buffer
    stash();
    float* h = w.h + u * V * K + (size_t)v0 * K;  // rows v0.. of the state entering the chunk
    for (int x = tid; x < 32 * K; x += blockDim.x) h[x] = sS[(x / K) * (K + 1) + x % K];
    __syncthreads();
    if (ci + 1 < sq.y) fetch(u + p.HV);
    mm(CH, 32, K, sU, 32, -1.f, true, sW, K + 1, 1, sS, 1, K + 1);  // U = U~ - W S^T
    __syncthreads();
    float* U = w.U + u * CH * V;
    for (int x = tid; x < CH * 32; x += blockDim.x) U[(x / 32) * V + v0 + x % 32] = sU[x];
    for (int x = tid; x < 32 * K; x += blockDim.x) {
      const int vv = x / K, c = x % K;
      sS[vv * (K + 1) + c] *= sE[c];
    }
    __syncthreads();
    mm(32, K, CH, sS, K + 1, 1.f, true, sU, 1, 32, sKh, K, 1);  // S' = S Diag(e^{Gam_C}) + U^T K^
  }
  __syncthreads();
  if (a.ht)
    for (int x = tid; x < 32 * K; x += blockDim.x) {
      const int vv = x % 32, c = x / 32;
      a.ht[(((size_t)n * p.HV + hv) * K + c) * V + v0 + vv] = sS[vv * (K + 1) + c];
    }
}

// O = scale (Q~ S^T + P U) for one (chunk, value head)
template <typename T>
__global__ void __launch_bounds__(256) k_kda_out(Problem p, Args a, KdaWork w) {
  if (kda_failed(w)) return;
  const int gc = blockIdx.x, hv = blockIdx.y;
  const int4 e = w.chunk_tab[gc];
  if (e.x < 0) return;
  const int K = p.K, V = p.V, L = e.z, tok0 = e.w;
  extern __shared__ float sm[];
  float* sQt = sm;                 // [64][K]
  float* sP = sQt + CH * K;        // [64][64]
  float* sH = sP + CH * CH;        // [K][V+1]  h[k][v] = S[v][k] of the state entering the chunk
  float* sU = sH + K * (V + 1);    // [64][V]
  float* sO = sU + CH * V;         // [64][V]
  const size_t u = (size_t)gc * p.HV + hv;
  copy_async(sQt, w.Qt + u * CH * K, CH * K);
  copy_async(sP, w.P + u * CH * CH, CH * CH);
  copy_async(sU, w.U + u * CH * V, CH * V);
  {  // S ([V][K] in memory) transposed into h[k][v]
    const float4* S4 = reinterpret_cast<const float4*>(w.h + u * V * K);
    for (int x = threadIdx.x; x < V * K / 4; x += blockDim.x) {
      const float4 f = S4[x];
      const int v = x / (K / 4), c = 4 * (x % (K / 4));
      sH[c * (V + 1) + v] = f.x;
      sH[(c + 1) * (V + 1) + v] = f.y;
      sH[(c + 2) * (V + 1) + v] = f.z;
      sH[(c + 3) * (V + 1) + v] = f.w;
    }
  }
  cp_async_wait_all();
  __syncthreads();
  mm(CH, V, CH, sO, V, 1.f, false, sP, CH, 1, sU, V, 1, 1);  // P lower triangular
  mm(CH, V, K, sO, V, 1.f, true, sQt, K, 1, sH, V + 1, 1);
  __syncthreads();
  T* o = static_cast<T*>(a.o) + ((size_t)tok0 * p.HV + hv) * V;
  for (int x = threadIdx.x; x < L * V; x += blockDim.x)
    o[(size_t)(x / V) * p.HV * V + x % V] = from_f<T>(p.scale * sO[x]);
}

template <typename Kern>
cudaError_t go(const char* name, Kern kern, dim3 grid, size_t smem, cudaStream_t s, const Problem& p,
               const Args& a, const KdaWork& w) {
  if (grid.x == 0 || grid.y == 0 || grid.z == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ProfScope ps(name, s);
  kern<<<grid, 256, smem, s>>>(p, a, w);
  return cudaGetLastError();
}

template <typename T>
cudaError_t forward_t(const Problem& p, const Args& a, const KdaWork& w, cudaStream_t s) {
  cudaError_t e = go("kda_wy", k_kda_wy<T>, dim3(p.NCmax, p.HV), wy_smem(p.K, p.V), s, p, a, w);
  if (e == cudaSuccess)
    e = go("kda_scan", k_kda_scan, dim3(p.Nst, p.HV, p.V / 32), scan_smem(p.K), s, p, a, w);
  if (e == cudaSuccess) e = go("kda_out", k_kda_out<T>, dim3(p.NCmax, p.HV), out_smem(p.K, p.V), s, p, a, w);
  return e;
}

}  // namespace

cudaError_t kda_chunk_forward(const Problem& p, const Args& a, const KdaWork& w, bool bf16, cudaStream_t s) {
  return bf16 ? forward_t<__nv_bfloat16>(p, a, w, s) : forward_t<float>(p, a, w, s);
}

}  // namespace gdn
