// Chunkwise backward of the KDA delta rule (a decay per key channel), fp32 on CUDA cores, for
// L = sum(dO * o) + sum(dht * h_final).  It reads the intermediates a forward kept in the same
// workspace (W, K^, Q~, P, e^{Gam_C}, the entering states S, U, Gam, T).  Per 64-token chunk,
// with dS' = dL/dS leaving the chunk, X = diag(beta) (k e^{Gam}), Y = diag(beta) V:
//   dU = scale P^T dO + K^ dS'^T,            dS = dS' Diag(e^{Gam_C}) + scale dO^T Q~ - dU^T W
//   dQ~ = scale dO S,  dP = scale dO U^T (lower incl. diagonal),  dK^ = U dS',  dW = -dU S
//   dT = dW X^T + dU Y^T,  dX = T^T dW,  dY = T^T dU,  dA = -T^T dT T^T (strictly lower)
//   dv = beta dY,  dbeta = rowsum(dY * V) + rowsum(dX * k e^{Gam}) + rowsum(k * F1)
//   dq = dQ~ e^{Gam} + F2,   dk = dK^ e^{Gam_C - Gam} + beta dX e^{Gam} + G2 + beta F1 + G1
//   dGam = dQ~ Q~ - dK^ K^ + beta dX (k e^{Gam}) + q F2 - k G2 + beta k F1 - k G1,
//   dGam_C += colsum(dK^ K^) + e^{Gam_C} colsum(dS' * S)
// where F_i = sum_{j<=i} Wt_ij R_j e^{Gam_i - Gam_j} and G_j = sum_{i>=j} Wt_ij L_i e^{Gam_i - Gam_j}
// are per-channel gated products (F2, G2: Wt = dP, R = k, L = q; F1: Wt = dA, R = k; G1: Wt =
// diag(beta) dA, L = k), taken in 16-token sub-chunks as in the forward.  dyg is the reverse
// in-chunk cumsum of dGam; the KDA gate's chain gives dg_raw, dA_log and ddt_bias.
//
// Kernels: k_kda_bwd_scan (sequence, value head, 32-row slice of S; reverse over the chunks),
// k_kda_bwd_dqk and k_kda_bwd_wy per (chunk, value head), then the group sum of the dq/dk
// shares and a fixed-order sum of the gate-parameter gradients.
#include <type_traits>

#include "ffma_tiles.cuh"
#include "gdn_common.cuh"
#include "gdn_launch.h"
#include "gdn_tc_common.cuh"  // LDA
#include "kda_gate_math.cuh"

namespace gdn {
namespace {

constexpr int SUB = 16;
constexpr int LDP = CH + 1;  // row stride of the 64 x 64 gradient matrices
using tcx::LDA;

__device__ __forceinline__ bool kda_failed(const KdaWork& w) { return *((volatile int*)w.status) != 0; }

// Per-channel gated products of a 64 x 64 weight Wt (lower triangle used, ldw) with row
// operand R and column operand Lm ([64][K], row stride K), Gam2 = Gam * log2(e) ([64][K]):
//   F_i = sum_{j<=i} Wt_ij R_j e^{Gam_i - Gam_j},   G_j = sum_{i>=j} colw_i Wt_ij Lm_i e^{Gam_i - Gam_j}
// (colw = per-row weights of the column product, or null; R and Lm fp32 or bf16).  Each result
// element is handed to
// sink(i, c, F) / sinkG(j, c, G) once per phase; phases are separated by barriers.
// scratch: [64][K] floats.  Ends with a barrier.
__device__ __forceinline__ float ldf(const float* p) { return *p; }
__device__ __forceinline__ float ldf(const __nv_bfloat16* p) { return __bfloat162float(*p); }

template <typename TR, typename SinkF, typename SinkG>
__device__ void gated_products(const float* Wt, int ldw, const TR* R, const TR* Lm,
                               const float* colw, const float* G2, int K, float* scratch,
                               SinkF sinkF, SinkG sinkG) {
  const int tid = threadIdx.x;
  // diagonal sub-blocks, one (row, channel) per thread
  for (int x = tid; x < CH * K; x += blockDim.x) {
    const int i = x / K, c = x % K, b0 = (i / SUB) * SUB;
    const float gi = G2[x];
    float f = 0.f, g = 0.f;
    for (int j = b0; j <= i; ++j) f += Wt[i * ldw + j] * ldf(R + j * K + c) * exp2f(gi - G2[j * K + c]);
    for (int r = i; r < b0 + SUB; ++r) {  // this row as the column index j = i
      const float wr = Wt[r * ldw + i] * (colw ? colw[r] : 1.f);
      g += wr * ldf(Lm + r * K + c) * exp2f(G2[r * K + c] - gi);
    }
    sinkF(i, c, f);
    sinkG(i, c, g);
  }
  __syncthreads();
  float* RT = scratch;                 // [48][K]: R_j e^{Gam_r - Gam_j}, j < 16 a
  float* Ls = scratch + 3 * SUB * K;   // [16][K]: colw_i Lm_i e^{Gam_i - Gam_r}, i in sub-chunk a
  for (int a = 1; a < CH / SUB; ++a) {
    const int r = a * SUB - 1, nj = a * SUB;
    for (int x = tid; x < nj * K; x += blockDim.x) {
      const int c = x % K;
      RT[x] = ldf(R + x) * exp2f(G2[r * K + c] - G2[x]);
    }
    for (int x = tid; x < SUB * K; x += blockDim.x) {
      const int i = a * SUB + x / K, c = x % K;
      Ls[x] = (colw ? colw[i] : 1.f) * ldf(Lm + i * K + c) * exp2f(G2[i * K + c] - G2[r * K + c]);
    }
    __syncthreads();
    for (int x = tid; x < SUB * K; x += blockDim.x) {  // rows i of sub-chunk a
      const int i = a * SUB + x / K, c = x % K;
      float acc = 0.f;
      for (int j = 0; j < nj; ++j) acc += Wt[i * ldw + j] * RT[j * K + c];
      sinkF(i, c, acc * exp2f(G2[i * K + c] - G2[r * K + c]));
    }
    for (int x = tid; x < nj * K; x += blockDim.x) {  // columns j before sub-chunk a
      const int j = x / K, c = x % K;
      float acc = 0.f;
      for (int ii = 0; ii < SUB; ++ii) acc += Wt[(a * SUB + ii) * ldw + j] * Ls[ii * K + c];
      sinkG(j, c, acc * exp2f(G2[r * K + c] - G2[j * K + c]));
    }
    __syncthreads();
  }
}

// The same products for K = 128 and 512 threads, by channel, with the weights stored transposed
// (WtT[j * LDT + i] = Wt_ij, rows 16-byte aligned, so that the weights of a column j within a
// sub-chunk are 128-bit loads): thread t owns channel c = t % 128 and role t / 128, its operands
// in registers.  The diagonal sub-blocks: role = the sub-chunk, one exponential per pair (i, j)
// serving both F and G.  Below the diagonal, for each sub-chunk a (through r = 16 a - 1): roles 0
// and 1 form F of a's rows 16a + 8 role .. + 7 (independent accumulators, one pass over the
// columns j), roles 2 and 3 G of the columns j = role - 2, role, .. before a; F and G write
// disjoint rows of each channel.  The loops over j stay rolled (a fully unrolled form overflows
// the instruction cache).  Results go to the sinks as above; ends with a barrier.
constexpr int LDT = CH + 4;

__device__ __forceinline__ void ld16(const float* p, float* w) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float4 x = reinterpret_cast<const float4*>(p)[q];
    w[4 * q] = x.x;
    w[4 * q + 1] = x.y;
    w[4 * q + 2] = x.z;
    w[4 * q + 3] = x.w;
  }
}

template <typename TR, typename SinkF, typename SinkG>
__device__ void gated_products_k128x4(const float* WtT, const TR* R, const TR* Lm, const float* colw,
                                      const float* G2, SinkF sinkF, SinkG sinkG) {
  constexpr int K = 128;
  const int c = threadIdx.x & 127, role = threadIdx.x >> 7;
  {
    const int b0 = SUB * role;
    float g[SUB], r[SUB], l[SUB], F[SUB], G[SUB];
#pragma unroll
    for (int j = 0; j < SUB; ++j) {
      g[j] = G2[(b0 + j) * K + c];
      r[j] = ldf(R + (b0 + j) * K + c);
      l[j] = (colw ? colw[b0 + j] : 1.f) * ldf(Lm + (b0 + j) * K + c);
      F[j] = G[j] = 0.f;
    }
#pragma unroll
    for (int j = 0; j < SUB; ++j) {
      float wv[SUB];
      ld16(WtT + (b0 + j) * LDT + b0, wv);
#pragma unroll
      for (int i = j; i < SUB; ++i) {
        const float wt = wv[i] * exp2f(g[i] - g[j]);
        F[i] = fmaf(wt, r[j], F[i]);
        G[j] = fmaf(wt, l[i], G[j]);
      }
    }
#pragma unroll
    for (int i = 0; i < SUB; ++i) {
      sinkF(b0 + i, c, F[i]);
      sinkG(b0 + i, c, G[i]);
    }
  }
#pragma unroll 1
  for (int A = 1; A < CH / SUB; ++A) {
    __syncthreads();
    const int I0 = SUB * A, NJ = SUB * A;
    const float gr = G2[(I0 - 1) * K + c];
    if (role < 2) {  // F_i, i = I0 + 8 role .. + 7
      const int i0 = I0 + 8 * role;
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll 2
      for (int j = 0; j < NJ; ++j) {
        const float rt = ldf(R + j * K + c) * exp2f(gr - G2[j * K + c]);
        const float4 w0 = reinterpret_cast<const float4*>(WtT + j * LDT + i0)[0];
        const float4 w1 = reinterpret_cast<const float4*>(WtT + j * LDT + i0)[1];
        const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(wv[i], rt, acc[i]);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) sinkF(i0 + i, c, acc[i] * exp2f(G2[(i0 + i) * K + c] - gr));
    } else {         // G_j, j = role - 2, role, .. < 16 A
      float ls[SUB];
#pragma unroll
      for (int i = 0; i < SUB; ++i)
        ls[i] = (colw ? colw[I0 + i] : 1.f) * ldf(Lm + (I0 + i) * K + c) * exp2f(G2[(I0 + i) * K + c] - gr);
#pragma unroll 2
      for (int j = role - 2; j < NJ; j += 2) {
        float wv[SUB];
        ld16(WtT + j * LDT + I0, wv);
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
        for (int i = 0; i < SUB; i += 4) {
          a0 = fmaf(wv[i], ls[i], a0);
          a1 = fmaf(wv[i + 1], ls[i + 1], a1);
          a2 = fmaf(wv[i + 2], ls[i + 2], a2);
          a3 = fmaf(wv[i + 3], ls[i + 3], a3);
        }
        sinkG(j, c, ((a0 + a1) + (a2 + a3)) * exp2f(gr - G2[j * K + c]));
      }
    }
  }
  __syncthreads();
}

// ---------------------------------------------------------------- reverse state scan
template <typename T>
__global__ void __launch_bounds__(256) k_kda_bwd_scan(Problem p, Args a, KdaWork w) {
  if (kda_failed(w)) return;
  const int n = blockIdx.x, hv = blockIdx.y, v0 = 32 * blockIdx.z, K = p.K, V = p.V, tid = threadIdx.x;
  const int4 sq = w.seq_tab[n];
  extern __shared__ float sm[];
  float* sdS = sm;                 // [32][K+1]  rows v0.. of dS
  float* sP = sdS + 32 * (K + 1);  // [64][64]
  float* sKh = sP + CH * CH;       // [64][K]
  float* sQt = sKh + CH * K;       // [64][K]
  float* sW = sQt + CH * K;        // [64][K]
  float* sdO = sW + CH * K;        // [64][32]
  float* sdU = sdO + CH * 32;      // [64][32]
  float* sE = sdU + CH * 32;       // [K]
  for (int x = tid; x < 32 * K; x += blockDim.x) {
    const int vv = x % 32, c = x / 32;
    sdS[vv * (K + 1) + c] = a.dht ? a.dht[(((size_t)n * p.HV + hv) * K + c) * V + v0 + vv] : 0.f;
  }
  const T* dO = static_cast<const T*>(a.dO);
  for (int ci = sq.y - 1; ci >= 0; --ci) {
    const int gc = sq.x + ci;
    const int4 e = w.chunk_tab[gc];
    const size_t u = (size_t)gc * p.HV + hv;
    __syncthreads();  // the previous chunk is done with every buffer
    copy_async(sP, w.P + u * CH * CH, CH * CH);
    copy_async(sKh, w.Kh + u * CH * K, CH * K);
    copy_async(sQt, w.Qt + u * CH * K, CH * K);
    copy_async(sW, w.W + u * CH * K, CH * K);
    copy_async(sE, w.eGC + u * K, K);
    for (int x = tid; x < CH * 32; x += blockDim.x) {
      const int i = x / 32, vv = x % 32;
      sdO[x] = i < e.z ? to_f<T>(dO[((size_t)(e.w + i) * p.HV + hv) * V + v0 + vv]) : 0.f;
    }
    float* dh = w.dh + u * V * K + (size_t)v0 * K;  // dS' (leaving the chunk), rows v0..
    for (int x = tid; x < 32 * K; x += blockDim.x) dh[x] = sdS[(x / K) * (K + 1) + x % K];
    cp_async_wait_all();
    __syncthreads();
    mm(CH, 32, CH, sdU, 32, p.scale, false, sP, 1, CH, sdO, 32, 1, 2);  // scale P^T dO (P^T upper)
    mm(CH, 32, K, sdU, 32, 1.f, true, sKh, K, 1, sdS, 1, K + 1);      // + K^ dS'^T
    __syncthreads();
    float* dU = w.dU + u * CH * V;
    for (int x = tid; x < CH * 32; x += blockDim.x) dU[(x / 32) * V + v0 + x % 32] = sdU[x];
    for (int x = tid; x < 32 * K; x += blockDim.x) sdS[(x / K) * (K + 1) + x % K] *= sE[x % K];
    __syncthreads();
    mm(32, K, CH, sdS, K + 1, p.scale, true, sdO, 1, 32, sQt, K, 1);  // + scale dO^T Q~
    mm(32, K, CH, sdS, K + 1, -1.f, true, sdU, 1, 32, sW, K, 1);      // - dU^T W
  }
  __syncthreads();
  if (a.dh0)
    for (int x = tid; x < 32 * K; x += blockDim.x) {
      const int vv = x % 32, c = x / 32;
      a.dh0[(((size_t)n * p.HV + hv) * K + c) * V + v0 + vv] = sdS[vv * (K + 1) + c];
    }
}

// ---------------------------------------------------------------- reverse state scan, tcgen05
// k_kda_bwd_scan for bf16 with K = V = 128: two CTAs per (sequence, value head), each holding half
// of dS's rows (v in [64 z, 64 z + 64)) in fp32 registers in the layout of an M = 64 accumulator,
// both products of a chunk on the tensor cores (compensated bf16 pairs; dO is bf16 already):
//   dU[:, z] = (scale P)^T dO[:, z] + K^ dS'_z^T                  (M = 64 tokens, N = 64)  TMEM [0, 64)
//   dS_z = dS'_z Diag(e^{Gam_C}) + dO[:, z]^T (scale Q~) + dU[:, z]^T (-W)   (M = 64, N = K)  TMEM [128, 256)
namespace kb {
using namespace tcx;
constexpr int NT = 512;  // threads: four warps per TMEM sub-partition, a quarter of the columns each
constexpr int TT = 64 * 128;
constexpr int O_PH = 0, O_PL = 8192, O_DO = 16384, O_KH = 24576, O_KL = 40960, O_QH = 57344;
constexpr int O_QL = 73728, O_WH = 90112, O_WL = 106496, O_UH = 122880, O_UL = 131072;
constexpr int O_SH = 139264, O_SL = 155648, O_E = 172032;
constexpr int BSCAN_BYTES = O_E + 512;
static_assert(1024 + BSCAN_BYTES <= 227 * 1024, "kda backward scan shared memory");
}  // namespace kb

__global__ void __launch_bounds__(kb::NT, 1) k_kda_tc_bwd_scan(Problem p, Args a, KdaWork w) {
  using namespace kb;
  if (kda_failed(w)) return;
  const int n = blockIdx.x, hv = blockIdx.y, z = blockIdx.z;
  const int4 sq = w.seq_tab[n];
  constexpr int K = 128, V = 128;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qt = warp >> 2, sub = 32 * (warp & 3);  // quarter of the columns, sub-partition
  const int r0 = 16 * (warp & 3) + (lane >> 2), cq = 2 * (lane & 3);
  const int v0 = 64 * z;
  extern __shared__ unsigned char smraw[];
  unsigned char* sm = align1k(smraw);
  float* sE = reinterpret_cast<float*>(sm + O_E);
  __shared__ uint64_t bar[2];
  __shared__ uint32_t tslot;
  int* err = w.status;
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (warp == 0) {
    tmem_alloc(&tslot, 256);
    tmem_relinquish();
  }
  // S[4j + q]: dS at row v0 + r0 + 8 (q >> 1), column 32 qt + 8j + cq + (q & 1)
  float S[16];
  {
    const float* dht = a.dht ? a.dht + ((size_t)n * p.HV + hv) * K * V : nullptr;
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int r = v0 + r0 + 8 * (q >> 1), c = 32 * qt + 8 * j + cq + (q & 1);
        S[4 * j + q] = dht ? dht[(size_t)c * V + r] : 0.f;
      }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tslot;
  const bf16* dO = static_cast<const bf16*>(a.dO);
  bool ok = true;
  for (int k = 0; k < sq.y && ok; ++k) {
    const int ci = sq.y - 1 - k, gc = sq.x + ci;
    const int4 e = w.chunk_tab[gc];
    const size_t u = (size_t)gc * p.HV + hv;
    {  // this half of dS' (leaving the chunk): stored, and as a hi/lo tile [64 v][128 k]
      float* dh = w.dh + u * V * K + (size_t)v0 * K;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = 32 * qt + 8 * j + cq;
        *reinterpret_cast<float2*>(dh + r0 * K + c) = make_float2(S[4 * j], S[4 * j + 1]);
        *reinterpret_cast<float2*>(dh + (r0 + 8) * K + c) = make_float2(S[4 * j + 2], S[4 * j + 3]);
        st_pair_split(sm + O_SH, sm + O_SL, r0, c, TT, S[4 * j], S[4 * j + 1]);
        st_pair_split(sm + O_SH, sm + O_SL, r0 + 8, c, TT, S[4 * j + 2], S[4 * j + 3]);
      }
    }
    {  // scale P, K^ as hi/lo tiles; this half's dO columns (bf16, rows past L zero)
      const float* gK = w.Kh + u * CH * K;
      const float* gP = w.P + u * CH * CH;
      float4 rk[4], rp[2];
      uint4 rd[1];
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int x = tid + NT * m, row = x >> 4, j = x & 15;
        const float4* pk = reinterpret_cast<const float4*>(gK + row * K + 8 * j);
        rk[2 * m] = __ldg(pk);
        rk[2 * m + 1] = __ldg(pk + 1);
      }
#pragma unroll
      for (int m = 0; m < 1; ++m) {
        const int x = tid + NT * m, row = x >> 3, j = x & 7;
        rd[m] = row < e.z ? __ldg(reinterpret_cast<const uint4*>(dO + ((size_t)(e.w + row) * p.HV + hv) * V + v0 + 8 * j))
                          : make_uint4(0u, 0u, 0u, 0u);
        const float4* pp = reinterpret_cast<const float4*>(gP + row * CH + 8 * j);
        rp[2 * m] = __ldg(pp);
        rp[2 * m + 1] = __ldg(pp + 1);
      }
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int x = tid + NT * m, row = x >> 4, j = x & 15;
        const float fk[8] = {rk[2 * m].x, rk[2 * m].y, rk[2 * m].z, rk[2 * m].w,
                             rk[2 * m + 1].x, rk[2 * m + 1].y, rk[2 * m + 1].z, rk[2 * m + 1].w};
        st_chunk_split(sm + O_KH, sm + O_KL, row, j, TT, fk);
      }
      const float sc = p.scale;
#pragma unroll
      for (int m = 0; m < 1; ++m) {
        const int x = tid + NT * m, row = x >> 3, j = x & 7;
        *reinterpret_cast<uint4*>(sm + O_DO + sw128_chunk(row, j, TT)) = rd[m];
        const float f[8] = {sc * rp[2 * m].x, sc * rp[2 * m].y, sc * rp[2 * m].z, sc * rp[2 * m].w,
                            sc * rp[2 * m + 1].x, sc * rp[2 * m + 1].y, sc * rp[2 * m + 1].z, sc * rp[2 * m + 1].w};
        st_chunk_split(sm + O_PH, sm + O_PL, row, j, TT, f);
      }
    }
    const float egc = tid < K ? w.eGC[u * K + tid] : 0.f;
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {  // dU[:, z] = (scale P)^T dO[:, z] + K^ dS'_z^T
      const uint32_t ph = smem_u32(sm + O_PH), pl = smem_u32(sm + O_PL), d = smem_u32(sm + O_DO);
      const uint32_t kh = smem_u32(sm + O_KH), kl = smem_u32(sm + O_KL);
      const uint32_t sh = smem_u32(sm + O_SH), sl = smem_u32(sm + O_SL);
      constexpr uint32_t i_pd = idesc_bf16(64, 64, true, true), i_ks = idesc_bf16(64, 64, false, false);
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const uint64_t bd = desc_mnmajor(d, s, TT);
        mma_bf16(taddr(tb, 0, 0), desc_mnmajor(ph, s, TT), bd, i_pd, s > 0);
        mma_bf16(taddr(tb, 0, 0), desc_mnmajor(pl, s, TT), bd, i_pd, 1);
      }
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const uint64_t ak = desc_kmajor(kh, s, TT), bs = desc_kmajor(sh, s, TT);
        mma_bf16(taddr(tb, 0, 0), ak, bs, i_ks, 1);
        mma_bf16(taddr(tb, 0, 0), ak, desc_kmajor(sl, s, TT), i_ks, 1);
        mma_bf16(taddr(tb, 0, 0), desc_kmajor(kl, s, TT), bs, i_ks, 1);
      }
      mma_commit(&bar[0]);
    }
    {  // while they run: scale Q~ and -W as hi/lo tiles (read by the second products only)
      const float* gQ = w.Qt + u * CH * K;
      const float* gW = w.W + u * CH * K;
      float4 rq[4], rw[4];
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int x = tid + NT * m, row = x >> 4, j = x & 15;
        const float4* pq = reinterpret_cast<const float4*>(gQ + row * K + 8 * j);
        const float4* pw = reinterpret_cast<const float4*>(gW + row * K + 8 * j);
        rq[2 * m] = __ldg(pq);
        rq[2 * m + 1] = __ldg(pq + 1);
        rw[2 * m] = __ldg(pw);
        rw[2 * m + 1] = __ldg(pw + 1);
      }
      const float sc = p.scale;
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int x = tid + NT * m, row = x >> 4, j = x & 15;
        const float fq[8] = {sc * rq[2 * m].x, sc * rq[2 * m].y, sc * rq[2 * m].z, sc * rq[2 * m].w,
                             sc * rq[2 * m + 1].x, sc * rq[2 * m + 1].y, sc * rq[2 * m + 1].z, sc * rq[2 * m + 1].w};
        const float fw[8] = {-rw[2 * m].x, -rw[2 * m].y, -rw[2 * m].z, -rw[2 * m].w,
                             -rw[2 * m + 1].x, -rw[2 * m + 1].y, -rw[2 * m + 1].z, -rw[2 * m + 1].w};
        st_chunk_split(sm + O_QH, sm + O_QL, row, j, TT, fq);
        st_chunk_split(sm + O_WH, sm + O_WL, row, j, TT, fw);
      }
    }
    ok = __syncthreads_and(mbar_wait(&bar[0], k & 1, err));
    tc_fence_after();
    if (tid < K) sE[tid] = egc;
    if (ok) {  // dU for this half's values: stored, and as a hi/lo tile [64 tok][64 v]
      float x[8];
      tmem_ld16dp_x2(taddr(tb, sub, 16 * qt), x);
      tmem_wait_ld();
      float* gU = w.dU + u * CH * V + v0;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int c = 16 * qt + 8 * j + cq;
        *reinterpret_cast<float2*>(gU + r0 * V + c) = make_float2(x[4 * j], x[4 * j + 1]);
        *reinterpret_cast<float2*>(gU + (r0 + 8) * V + c) = make_float2(x[4 * j + 2], x[4 * j + 3]);
        st_pair_split(sm + O_UH, sm + O_UL, r0, c, TT, x[4 * j], x[4 * j + 1]);
        st_pair_split(sm + O_UH, sm + O_UL, r0 + 8, c, TT, x[4 * j + 2], x[4 * j + 3]);
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (ok && tid == 0) {  // dO[:, z]^T (scale Q~) + dU[:, z]^T (-W)
      const uint32_t d = smem_u32(sm + O_DO), qh = smem_u32(sm + O_QH), ql = smem_u32(sm + O_QL);
      const uint32_t uh = smem_u32(sm + O_UH), ul = smem_u32(sm + O_UL);
      const uint32_t wh = smem_u32(sm + O_WH), wl = smem_u32(sm + O_WL);
      constexpr uint32_t id = idesc_bf16(64, 128, true, true);
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const uint64_t ad = desc_mnmajor(d, s, TT);
        mma_bf16(taddr(tb, 0, 128), ad, desc_mnmajor(qh, s, TT), id, s > 0);
        mma_bf16(taddr(tb, 0, 128), ad, desc_mnmajor(ql, s, TT), id, 1);
        const uint64_t au = desc_mnmajor(uh, s, TT), bw = desc_mnmajor(wh, s, TT);
        mma_bf16(taddr(tb, 0, 128), au, bw, id, 1);
        mma_bf16(taddr(tb, 0, 128), au, desc_mnmajor(wl, s, TT), id, 1);
        mma_bf16(taddr(tb, 0, 128), desc_mnmajor(ul, s, TT), bw, id, 1);
      }
      mma_commit(&bar[1]);
    }
    ok = __syncthreads_and(ok && mbar_wait(&bar[1], k & 1, err));
    tc_fence_after();
    if (ok) {  // dS = dS' Diag(e^{Gam_C}) + the products
      float x[16];
      tmem_ld16dp_x4(taddr(tb, sub, 128 + 32 * qt), x);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int q = 0; q < 4; ++q)
          S[4 * j + q] = fmaf(S[4 * j + q], sE[32 * qt + 8 * j + cq + (q & 1)], x[4 * j + q]);
    }
  }
  if (ok && a.dh0) {
    float* dh0 = a.dh0 + ((size_t)n * p.HV + hv) * K * V;
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int r = v0 + r0 + 8 * (q >> 1), c = 32 * qt + 8 * j + cq + (q & 1);
        dh0[(size_t)c * V + r] = S[4 * j + q];
      }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, 256);
}

// ---------------------------------------------------------------- output-side terms
// dP, dQ~, dW = -dU S, dK^ (with the Gam_C column terms) and the dP gated products.  Writes the
// unit's dq and dk shares, dGam and dW.  Every product reads both operands from shared memory:
// a 64 KB region holds S, then dS', then q and k.
__host__ __device__ constexpr int dqk_x1(int K, int V) { return V * K > 2 * CH * K ? V * K : 2 * CH * K; }

template <typename T>
__global__ void __launch_bounds__(256) k_kda_bwd_dqk(Problem p, Args a, KdaWork w) {
  if (kda_failed(w)) return;
  const int gc = blockIdx.x, hv = blockIdx.y;
  const int4 e = w.chunk_tab[gc];
  if (e.x < 0) return;
  const int K = p.K, V = p.V, L = e.z, tok0 = e.w, hk = hv / p.G, tid = threadIdx.x;
  const int NP = blockDim.x / K, part = tid / K, cc = tid % K;  // column-sum parts (2 or 4)
  extern __shared__ float sm[];
  float* sX1 = sm;                  // S [V][K], then dS' [V][K], then q [64][K] | k [64][K]
  float* sG = sX1 + dqk_x1(K, V);   // [64][K]  Gam * log2(e)
  float* sR1 = sG + CH * K;         // [64][max(V, K)]  dO, then dU, then scratch
  float* sR2 = sR1 + CH * (V > K ? V : K);  // [64][V+1]  U
  float* sdP = sR2 + CH * (V + 1);  // [64][65]
  float* sred = sdP + CH * LDP;     // [NP][K] partial column sums
  float* sGC = sred + 4 * K;        // [K]  dL/dGam_C
  const size_t u = (size_t)gc * p.HV + hv, uk = u * CH * K;
  float* dqp = w.dqp + uk;
  float* dkp = w.dkp + uk;
  float* dG = w.dGam + uk;
  copy_async(sX1, w.h + u * V * K, V * K);
  copy_async(sG, w.Gam + uk, CH * K);
  load_tile<T>(sR1, V, static_cast<const T*>(a.dO) + ((size_t)tok0 * p.HV + hv) * V, (size_t)p.HV * V, L, V);
  for (int x = tid; x < CH * V; x += blockDim.x) sR2[(x / V) * (V + 1) + x % V] = w.U[u * CH * V + x];
  cp_async_wait_all();
  __syncthreads();
  mm(CH, CH, V, sdP, LDP, p.scale, false, sR1, V, 1, sR2, 1, V + 1);  // dP = scale dO U^T
  mm(CH, K, V, dqp, K, p.scale, false, sR1, V, 1, sX1, K, 1);         // dQ~ = scale dO S (raw)
  {  // e^{Gam_C} colsum(dS' * S), part of dL/dGam_C
    const float* dSn = w.dh + u * V * K;
    float t = 0.f;
    for (int v = part; v < V; v += NP) t += dSn[(size_t)v * K + cc] * sX1[v * K + cc];
    sred[part * K + cc] = t;
  }
  __syncthreads();
  if (tid < K) {
    float t = 0.f;
    for (int q = 0; q < NP; ++q) t += sred[q * K + tid];
    sGC[tid] = exp2f(sG[(CH - 1) * K + tid]) * t;
  }
  for (int x = tid; x < CH * CH; x += blockDim.x)
    if (x % CH > x / CH) sdP[(x / CH) * LDP + x % CH] = 0.f;
  copy_async(sR1, w.dU + u * CH * V, CH * V);  // dO is done
  cp_async_wait_all();
  __syncthreads();
  mm(CH, K, V, w.dW + uk, K, -1.f, false, sR1, V, 1, sX1, K, 1);  // dW = -dU S
  __syncthreads();
  copy_async(sX1, w.dh + u * V * K, V * K);  // S is done
  cp_async_wait_all();
  __syncthreads();
  mm(CH, K, V, dkp, K, 1.f, false, sR2, V + 1, 1, sX1, K, 1);  // dK^ = U dS' (raw)
  __syncthreads();
  float* sQ = sX1;
  float* sK = sX1 + CH * K;
  const size_t rs = (size_t)p.H * K;
  load_tile<T>(sQ, K, static_cast<const T*>(a.q) + ((size_t)tok0 * p.H + hk) * K, rs, L, K);
  load_tile<T>(sK, K, static_cast<const T*>(a.k) + ((size_t)tok0 * p.H + hk) * K, rs, L, K);
  __syncthreads();
  {  // colsum(dK^ * K^), the rest of dL/dGam_C
    const float gC = sG[(CH - 1) * K + cc];
    float t = 0.f;
    for (int i = part; i < CH; i += NP) t += dkp[i * K + cc] * sK[i * K + cc] * exp2f(gC - sG[i * K + cc]);
    sred[part * K + cc] = t;
  }
  __syncthreads();
  if (tid < K) {
    float t = 0.f;
    for (int q = 0; q < NP; ++q) t += sred[q * K + tid];
    sGC[tid] += t;
  }
  __syncthreads();
  for (int x = tid; x < CH * K; x += blockDim.x) {
    const int i = x / K, c = x % K;
    const float g = sG[x], eg = exp2f(g), kh = exp2f(sG[(CH - 1) * K + c] - g);
    const float dkh = dkp[x], dqt = dqp[x];
    dkp[x] = dkh * kh;
    dqp[x] = dqt * eg;
    dG[x] = dqt * sQ[x] * eg - dkh * sK[x] * kh + (i == CH - 1 ? sGC[c] : 0.f);
  }
  __syncthreads();
  // P_ij = sum_c q_i k_j e^{Gam_i - Gam_j}: dq += F2, dk += G2, dGam += q F2 - k G2
  gated_products(sdP, LDP, sK, sQ, nullptr, sG, K, sR1,
                 [&](int i, int c, float f) {
                   dqp[i * K + c] += f;
                   dG[i * K + c] += sQ[i * K + c] * f;
                 },
                 [&](int j, int c, float g) {
                   dkp[j * K + c] += g;
                   dG[j * K + c] -= sK[j * K + c] * g;
                 });
}

// ---------------------------------------------------------------- output-side terms, tcgen05
// The same unit's work with the four state-sized products on the tensor cores (bf16 inputs,
// K = V = 128).  Operands are staged from the fp32 workspace as compensated bf16 pairs
// (hi = bf16(x), lo = bf16(x - hi)) in 128-byte-swizzled tiles; dO is bf16 already and goes in
// as one part.  Accumulators (TMEM, M = 64 tokens):
//   [0, 64)    dP   = dO U^T         (dO.U_hi + dO.U_lo)
//   [64, 192)  dQ~' = dO S           (dO.S_hi + dO.S_lo)           (before scale and e^{Gam})
//   [192, 320) dW'  = dU S           (three of the four hi/lo products)
//   [320, 448) dK^' = U dS'          (same)
// dS' takes S's tiles once the first three products are done; the dP gated products and the
// per-channel terms then run on CUDA cores as in k_kda_bwd_dqk, with dq, dk and dGam accumulated
// in shared memory.  512 threads: four warps per TMEM sub-partition, a quarter of the columns each.
namespace kt {
using namespace tcx;
constexpr int NT = 512;           // threads of the output-side kernel
constexpr int TILE_T = 64 * 128;  // a [64 rows][64 bf16] block
constexpr int TILE_S = 128 * 128; // a [128 rows][64 bf16] block
constexpr int O_DO = 0, O_UH = 16384, O_UL = 32768, O_DUH = 49152, O_DUL = 65536;
constexpr int O_SH = 81920, O_SL = 114688;                  // S, then dS' (hi, lo)
// after the last product, over the tiles: the unit's dq, dk and dGam (fp32 [64][128] each,
// accumulated in shared memory and written out once), q and k (bf16 [64][128], rows past the
// chunk zero) and the gated products' scratch (fp32 [64][128])
constexpr int O_ACQ = 0, O_ACK = 32768, O_ACG = 65536, O_QB = 98304, O_KB = 114688, O_SCR = 131072;
constexpr int O_DP = 163840;                                // fp32 dP^T [64][LDT]
constexpr int O_G = O_DP + CH * LDT * 4;                    // fp32 [64][128] Gam * log2(e)
constexpr int O_RED = O_G + CH * 128 * 4;                   // fp32 [16][128]
constexpr int O_GC = O_RED + 16 * 128 * 4;                  // fp32 [128]
constexpr int DQK_BYTES = O_GC + 128 * 4;
static_assert(O_SL + 32768 <= O_DP && O_SCR + 32768 <= O_DP, "tiles overlap the fp32 area");
static_assert(1024 + DQK_BYTES <= 227 * 1024, "dqk shared memory");

// rows [0, R) of an fp32 [R][128] matrix (row stride ld floats) as a hi/lo pair of sw128 tiles
// (NT threads)
template <int R, int NT = 256>
__device__ __forceinline__ void stage_split(unsigned char* hi, unsigned char* lo, const float* src, size_t ld) {
  constexpr int N = R * 16 / NT;  // 16-byte chunks of 8 floats per thread
  float4 r[2 * N];
#pragma unroll
  for (int m = 0; m < N; ++m) {
    const int x = threadIdx.x + NT * m, row = x >> 4, j = x & 15;
    const float4* p = reinterpret_cast<const float4*>(src + row * ld + 8 * j);
    r[2 * m] = __ldg(p);
    r[2 * m + 1] = __ldg(p + 1);
  }
#pragma unroll
  for (int m = 0; m < N; ++m) {
    const int x = threadIdx.x + NT * m, row = x >> 4, j = x & 15;
    const float f[8] = {r[2 * m].x, r[2 * m].y, r[2 * m].z, r[2 * m].w,
                        r[2 * m + 1].x, r[2 * m + 1].y, r[2 * m + 1].z, r[2 * m + 1].w};
    st_chunk_split(hi, lo, row, j, R * 128, f);
  }
}
// two such matrices with all loads issued before the first store
template <int R, int NT = 256>
__device__ __forceinline__ void stage_split2(unsigned char* hi0, unsigned char* lo0, const float* src0,
                                             unsigned char* hi1, unsigned char* lo1, const float* src1, size_t ld) {
  constexpr int N = R * 16 / NT;
  float4 r[4 * N];
#pragma unroll
  for (int m = 0; m < N; ++m) {
    const int x = threadIdx.x + NT * m, row = x >> 4, j = x & 15;
    const float4* p0 = reinterpret_cast<const float4*>(src0 + row * ld + 8 * j);
    const float4* p1 = reinterpret_cast<const float4*>(src1 + row * ld + 8 * j);
    r[4 * m] = __ldg(p0);
    r[4 * m + 1] = __ldg(p0 + 1);
    r[4 * m + 2] = __ldg(p1);
    r[4 * m + 3] = __ldg(p1 + 1);
  }
#pragma unroll
  for (int m = 0; m < N; ++m) {
    const int x = threadIdx.x + NT * m, row = x >> 4, j = x & 15;
    const float f0[8] = {r[4 * m].x, r[4 * m].y, r[4 * m].z, r[4 * m].w,
                         r[4 * m + 1].x, r[4 * m + 1].y, r[4 * m + 1].z, r[4 * m + 1].w};
    const float f1[8] = {r[4 * m + 2].x, r[4 * m + 2].y, r[4 * m + 2].z, r[4 * m + 2].w,
                         r[4 * m + 3].x, r[4 * m + 3].y, r[4 * m + 3].z, r[4 * m + 3].w};
    st_chunk_split(hi0, lo0, row, j, R * 128, f0);
    st_chunk_split(hi1, lo1, row, j, R * 128, f1);
  }
}
}  // namespace kt

__global__ void __launch_bounds__(kt::NT, 1) k_kda_tc_bwd_dqk(Problem p, Args a, KdaWork w) {
  using namespace kt;
  if (kda_failed(w)) return;
  const int gc = blockIdx.x, hv = blockIdx.y;
  const int4 e = w.chunk_tab[gc];
  if (e.x < 0) return;
  constexpr int K = 128, V = 128;
  const int L = e.z, tok0 = e.w, hk = hv / p.G, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  extern __shared__ unsigned char smraw[];
  unsigned char* sm = align1k(smraw);
  float* sdP = reinterpret_cast<float*>(sm + O_DP);
  float* sG = reinterpret_cast<float*>(sm + O_G);
  float* sred = reinterpret_cast<float*>(sm + O_RED);
  float* sGC = reinterpret_cast<float*>(sm + O_GC);
  __shared__ uint64_t bar[2];
  __shared__ uint32_t tslot;
  int* err = w.status;
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (warp == 0) {
    tmem_alloc(&tslot, 512);
    tmem_relinquish();
  }
  const size_t u = (size_t)gc * p.HV + hv, uk = u * CH * K;
  {  // dO rows [0, L) (bf16, zero past L), U, dU, S; Gam
    const bf16* dO = static_cast<const bf16*>(a.dO) + ((size_t)tok0 * p.HV + hv) * V;
    uint4 r[2];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int x = tid + NT * m, row = x >> 4, j = x & 15;
      r[m] = row < L ? __ldg(reinterpret_cast<const uint4*>(dO + (size_t)row * p.HV * V + 8 * j))
                     : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int x = tid + NT * m, row = x >> 4, j = x & 15;
      *reinterpret_cast<uint4*>(sm + O_DO + sw128_chunk(row, j, TILE_T)) = r[m];
    }
  }
  stage_split2<CH, NT>(sm + O_UH, sm + O_UL, w.U + u * CH * V, sm + O_DUH, sm + O_DUL, w.dU + u * CH * V, V);
  stage_split<128, NT>(sm + O_SH, sm + O_SL, w.h + u * V * K, K);
  copy_async(sG, w.Gam + uk, CH * K);
  cp_async_wait_all();
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tslot;
  const uint32_t aDO = smem_u32(sm + O_DO), aUH = smem_u32(sm + O_UH), aUL = smem_u32(sm + O_UL);
  const uint32_t aDUH = smem_u32(sm + O_DUH), aDUL = smem_u32(sm + O_DUL);
  const uint32_t aSH = smem_u32(sm + O_SH), aSL = smem_u32(sm + O_SL);
  if (tid == 0) {
    constexpr uint32_t i64 = idesc_bf16(64, 64, false, false), i128 = idesc_bf16(64, 128, false, true);
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const uint64_t dO_ = desc_kmajor(aDO, s, TILE_T);
      mma_bf16(taddr(tb, 0, 0), dO_, desc_kmajor(aUH, s, TILE_T), i64, s > 0);
      mma_bf16(taddr(tb, 0, 0), dO_, desc_kmajor(aUL, s, TILE_T), i64, 1);
      const uint64_t sh = desc_mnmajor(aSH, s, TILE_S), sl = desc_mnmajor(aSL, s, TILE_S);
      mma_bf16(taddr(tb, 0, 64), dO_, sh, i128, s > 0);
      mma_bf16(taddr(tb, 0, 64), dO_, sl, i128, 1);
      const uint64_t duh = desc_kmajor(aDUH, s, TILE_T);
      mma_bf16(taddr(tb, 0, 192), duh, sh, i128, s > 0);
      mma_bf16(taddr(tb, 0, 192), duh, sl, i128, 1);
      mma_bf16(taddr(tb, 0, 192), desc_kmajor(aDUL, s, TILE_T), sh, i128, 1);
    }
    mma_commit(&bar[0]);
  }
  // dS' (leaving the chunk) into registers while the products run
  const float* dSn = w.dh + u * V * K;
  float4 rd[8];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int x = tid + NT * m, row = x >> 4, j = x & 15;
    const float4* p4 = reinterpret_cast<const float4*>(dSn + (size_t)row * K + 8 * j);
    rd[2 * m] = __ldg(p4);
    rd[2 * m + 1] = __ldg(p4 + 1);
  }
  bool ok = __syncthreads_and(mbar_wait(&bar[0], 0, err));
  tc_fence_after();
  {  // colsum(dS' * S) (S = hi + lo) over this thread's rows, then dS' over S's tiles
    float cs[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const int j = tid & 15;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int row = (tid >> 4) + 32 * m;
      float h[8], l[8];
      ld_chunk_f(sm + O_SH, row, j, TILE_S, h);
      ld_chunk_f(sm + O_SL, row, j, TILE_S, l);
      const float f[8] = {rd[2 * m].x, rd[2 * m].y, rd[2 * m].z, rd[2 * m].w,
                          rd[2 * m + 1].x, rd[2 * m + 1].y, rd[2 * m + 1].z, rd[2 * m + 1].w};
#pragma unroll
      for (int q = 0; q < 8; ++q) cs[q] = fmaf(f[q], h[q] + l[q], cs[q]);
      st_chunk_split(sm + O_SH, sm + O_SL, row, j, TILE_S, f);
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) cs[q] += __shfl_xor_sync(0xffffffffu, cs[q], 16);  // same j
    if (lane < 16)
#pragma unroll
      for (int q = 0; q < 8; ++q) sred[warp * 128 + 8 * j + q] = cs[q];
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (ok && tid == 0) {
    constexpr uint32_t i128 = idesc_bf16(64, 128, false, true);
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const uint64_t uh = desc_kmajor(aUH, s, TILE_T);
      const uint64_t sh = desc_mnmajor(aSH, s, TILE_S);
      mma_bf16(taddr(tb, 0, 320), uh, sh, i128, s > 0);
      mma_bf16(taddr(tb, 0, 320), uh, desc_mnmajor(aSL, s, TILE_S), i128, 1);
      mma_bf16(taddr(tb, 0, 320), desc_kmajor(aUL, s, TILE_T), sh, i128, 1);
    }
    mma_commit(&bar[1]);
  }
  if (tid < K) {  // e^{Gam_C} colsum(dS' * S), part of dL/dGam_C
    float t = 0.f;
    for (int q = 0; q < 16; ++q) t += sred[q * 128 + tid];
    sGC[tid] = exp2f(sG[(CH - 1) * K + tid]) * t;
  }
  // M = 64 accumulators, 16-lane loads: warp (sub-partition warp % 4, quarter warp / 4), rows r0
  // and r0 + 8, columns 8j + cq + {0, 1} of this warp's quarter of the accumulator
  const int qt = warp >> 2, sub = 32 * (warp & 3), r0 = 16 * (warp & 3) + (lane >> 2), cq = 2 * (lane & 3);
  if (ok) {
    float d[8];
    tmem_ld16dp_x2(taddr(tb, sub, 16 * qt), d);  // dP, columns [16 qt, +16)
    float x[16];
    tmem_ld16dp_x4(taddr(tb, sub, 192 + 32 * qt), x);  // dW', columns [32 qt, +32)
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = r0 + 8 * (q >> 1), c = 16 * qt + 8 * j + cq + (q & 1);
        sdP[c * LDT + i] = c <= i ? p.scale * d[4 * j + q] : 0.f;
      }
    float* dW = w.dW + uk;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = 32 * qt + 8 * j + cq;
      *reinterpret_cast<float2*>(dW + r0 * K + c) = make_float2(-x[4 * j], -x[4 * j + 1]);
      *reinterpret_cast<float2*>(dW + (r0 + 8) * K + c) = make_float2(-x[4 * j + 2], -x[4 * j + 3]);
    }
  }
  ok = __syncthreads_and(ok && mbar_wait(&bar[1], 0, err));
  tc_fence_after();
  bf16* sQ = reinterpret_cast<bf16*>(sm + O_QB);
  bf16* sK = reinterpret_cast<bf16*>(sm + O_KB);
  float* acq = reinterpret_cast<float*>(sm + O_ACQ);
  float* ack = reinterpret_cast<float*>(sm + O_ACK);
  float* acg = reinterpret_cast<float*>(sm + O_ACG);
  {  // q and k rows [0, L) as bf16, zero past L
    const size_t rs = (size_t)p.H * K;
    const bf16* gq = static_cast<const bf16*>(a.q) + ((size_t)tok0 * p.H + hk) * K;
    const bf16* gk = static_cast<const bf16*>(a.k) + ((size_t)tok0 * p.H + hk) * K;
    uint4 rq[2], rk[2];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int x = tid + NT * m, row = x >> 4, j = x & 15;
      rq[m] = rk[m] = make_uint4(0u, 0u, 0u, 0u);
      if (row < L) {
        rq[m] = __ldg(reinterpret_cast<const uint4*>(gq + row * rs + 8 * j));
        rk[m] = __ldg(reinterpret_cast<const uint4*>(gk + row * rs + 8 * j));
      }
    }
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int x = tid + NT * m;
      reinterpret_cast<uint4*>(sQ)[x] = rq[m];
      reinterpret_cast<uint4*>(sK)[x] = rk[m];
    }
  }
  __syncthreads();
  if (ok) {  // dQ~ e^{Gam}, dK^ e^{Gam_C - Gam}, dGam; colsum(dK^ * K^) per column
    float x[16], y[16];
    tmem_ld16dp_x4(taddr(tb, sub, 64 + 32 * qt), x);
    tmem_ld16dp_x4(taddr(tb, sub, 320 + 32 * qt), y);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float cs[2];
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const int c = 32 * qt + 8 * j + cq + b;
        const float gC = sG[(CH - 1) * K + c];
        float t = 0.f;
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const int i = r0 + 8 * hr, o = i * K + c;
          const float g = sG[o], eg = exp2f(g), kh = exp2f(gC - g);
          const float dqt = p.scale * x[4 * j + 2 * hr + b], dkh = y[4 * j + 2 * hr + b];
          const float kk = __bfloat162float(sK[o]);
          acq[o] = dqt * eg;
          ack[o] = dkh * kh;
          acg[o] = dqt * __bfloat162float(sQ[o]) * eg - dkh * kk * kh;
          t = fmaf(dkh * kk, kh, t);
        }
        t += __shfl_xor_sync(0xffffffffu, t, 4);
        t += __shfl_xor_sync(0xffffffffu, t, 8);
        t += __shfl_xor_sync(0xffffffffu, t, 16);
        cs[b] = t;
      }
      if (lane < 4) {
        const int c = 32 * qt + 8 * j + cq;
        sred[(warp & 3) * 128 + c] = cs[0];
        sred[(warp & 3) * 128 + c + 1] = cs[1];
      }
    }
  }
  __syncthreads();
  if (ok && tid < K)  // the last row collects dL/dGam_C
    acg[(CH - 1) * K + tid] += sGC[tid] + sred[tid] + sred[128 + tid] + sred[256 + tid] + sred[384 + tid];
  __syncthreads();
  if (ok)  // P_ij = sum_c q_i k_j e^{Gam_i - Gam_j}: dq += F2, dk += G2, dGam += q F2 - k G2
    gated_products_k128x4(sdP, sK, sQ, nullptr, sG,
                   [&](int i, int c, float f) {
                     acq[i * K + c] += f;
                     acg[i * K + c] += __bfloat162float(sQ[i * K + c]) * f;
                   },
                   [&](int j, int c, float g) {
                     ack[j * K + c] += g;
                     acg[j * K + c] -= __bfloat162float(sK[j * K + c]) * g;
                   });
  if (ok) {  // the unit's dq and dk shares and dGam (gated_products ends with a barrier)
    float4* dq4 = reinterpret_cast<float4*>(w.dqp + uk);
    float4* dk4 = reinterpret_cast<float4*>(w.dkp + uk);
    float4* dg4 = reinterpret_cast<float4*>(w.dGam + uk);
    for (int x = tid; x < CH * K / 4; x += NT) {
      dq4[x] = reinterpret_cast<const float4*>(acq)[x];
      dk4[x] = reinterpret_cast<const float4*>(ack)[x];
      dg4[x] = reinterpret_cast<const float4*>(acg)[x];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, 512);
}

// ---------------------------------------------------------------- WY backward, gate chain
template <typename T>
__global__ void __launch_bounds__(256) k_kda_bwd_wy(Problem p, Args a, KdaWork w) {
  if (kda_failed(w)) return;
  const int gc = blockIdx.x, hv = blockIdx.y;
  const int4 e = w.chunk_tab[gc];
  if (e.x < 0) return;
  const int K = p.K, V = p.V, L = e.z, tok0 = e.w, hk = hv / p.G, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5, nwarp = blockDim.x >> 5;
  const int big = (V > K ? V : K) * CH > CH * LDP ? (V > K ? V : K) * CH : CH * LDP;
  extern __shared__ float sm[];
  float* sK = sm;                  // [64][K]
  float* sG = sK + CH * K;         // [64][K]
  float* sX = sG + CH * K;         // [64][K+1]  beta k e^{Gam}, then F1
  float* sY = sX + CH * (K + 1);   // [64][V+1]  beta V
  float* sdW = sY + CH * (V + 1);  // [big]  dW [64][K], then Z [64][65]
  float* sdU = sdW + big;          // [big]  dU [64][V], then scratch, then g_raw [64][K]
  float* sT = sdU + big;           // [64][LDA]
  float* sdT = sT + CH * LDA;      // [64][65]  dT, then dA
  float* sb = sdT + CH * LDP;      // [64]
  float* sdb = sb + CH;            // [64]
  const size_t u = (size_t)gc * p.HV + hv, uk = u * CH * K;
  const size_t rs = (size_t)p.H * K;
  load_tile<T>(sK, K, static_cast<const T*>(a.k) + ((size_t)tok0 * p.H + hk) * K, rs, L, K);
  load_tile<T>(sY, V + 1, static_cast<const T*>(a.v) + ((size_t)tok0 * p.HV + hv) * V, (size_t)p.HV * V, L, V);
  copy_async(sG, w.Gam + uk, CH * K);
  copy_async(sdW, w.dW + uk, CH * K);
  copy_async(sdU, w.dU + u * CH * V, CH * V);
  if (tid < CH) sb[tid] = tid < L ? a.beta[(size_t)(tok0 + tid) * p.HV + hv] : 0.f;
  for (int x = tid; x < CH * CH; x += blockDim.x)
    sT[(x / CH) * LDA + x % CH] = w.Tm[u * CH * CH + x];
  cp_async_wait_all();
  __syncthreads();
  for (int x = tid; x < CH * K; x += blockDim.x) {
    const int i = x / K, c = x % K;
    sX[i * (K + 1) + c] = sb[i] * sK[x] * exp2f(sG[x]);
  }
  for (int x = tid; x < CH * V; x += blockDim.x) sY[(x / V) * (V + 1) + x % V] *= sb[x / V];
  __syncthreads();
  // dT = dW X^T + dU Y^T
  mm(CH, CH, K, sdT, LDP, 1.f, false, sdW, K, 1, sX, 1, K + 1);
  mm(CH, CH, V, sdT, LDP, 1.f, true, sdU, V, 1, sY, 1, V + 1);
  // dX = T^T dW, dY = T^T dU (into the global dW and dU of this unit)
  float* dX = w.dW + uk;
  float* dY = w.dU + u * CH * V;
  mm(CH, K, CH, dX, K, 1.f, false, sT, 1, LDA, sdW, K, 1, 2);  // T^T upper triangular
  mm(CH, V, CH, dY, V, 1.f, false, sT, 1, LDA, sdU, V, 1, 2);
  __syncthreads();
  float* dkp = w.dkp + uk;
  float* dG = w.dGam + uk;
  // dv = beta dY; dbeta = rowsum(dY V) + rowsum(dX k e^{Gam}); dk += beta dX e^{Gam}
  T* dv = static_cast<T*>(a.dv);
  const T* vin = static_cast<const T*>(a.v);
  for (int i = warp; i < CH; i += nwarp) {
    float s = 0.f;
    for (int v = lane; v < V; v += 32) {
      const float y = dY[i * V + v];
      if (i < L) {
        const size_t o = ((size_t)(tok0 + i) * p.HV + hv) * V + v;
        s += y * to_f<T>(vin[o]);
        dv[o] = from_f<T>(sb[i] * y);
      }
    }
    for (int c = lane; c < K; c += 32) {
      const float eg = exp2f(sG[i * K + c]), dx = dX[i * K + c], kt = sK[i * K + c] * eg;
      s += dx * kt;
      dkp[i * K + c] += sb[i] * dx * eg;
      dG[i * K + c] += sb[i] * dx * kt;
    }
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) sdb[i] = s;
  }
  // dA = -T^T (dT T^T), strictly lower
  float* sZ = sdW;
  mm(CH, CH, CH, sZ, LDP, 1.f, false, sdT, LDP, 1, sT, 1, LDA);
  __syncthreads();
  mm(CH, CH, CH, sdT, LDP, -1.f, false, sT, 1, LDA, sZ, LDP, 1, 2);
  __syncthreads();
  for (int x = tid; x < CH * CH; x += blockDim.x)
    if (x % CH >= x / CH) sdT[(x / CH) * LDP + x % CH] = 0.f;
  for (int x = tid; x < CH * (K + 1); x += blockDim.x) sX[x] = 0.f;  // F1 accumulator
  __syncthreads();
  // A_ij = beta_i sum_c k_i k_j e^{Gam_i - Gam_j}: F1 (rows, weights dA), G1 (columns, beta_i dA)
  gated_products(sdT, LDP, sK, sK, sb, sG, K, sdU,
                 [&](int i, int c, float f) { sX[i * (K + 1) + c] += f; },
                 [&](int j, int c, float g) {
                   dkp[j * K + c] += g;
                   dG[j * K + c] -= sK[j * K + c] * g;
                 });
  // F1 terms: dk += beta F1, dGam += beta k F1, dbeta += rowsum(k F1)
  for (int i = warp; i < CH; i += nwarp) {
    float s = 0.f;
    for (int c = lane; c < K; c += 32) {
      const float f = sX[i * (K + 1) + c], kk = sK[i * K + c];
      s += kk * f;
      dkp[i * K + c] += sb[i] * f;
      dG[i * K + c] += sb[i] * kk * f;
    }
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0 && i < L) a.dbeta[(size_t)(tok0 + i) * p.HV + hv] = sdb[i] + s;
  }
  __syncthreads();
  // the unit's dGam and raw gate inputs in shared memory (the F1 terms above are in dGam)
  float* sdG = sdW;  // Z is done
  float* sg = sdU;   // the scratch is done
  copy_async(sdG, dG, CH * K);
  load_tile<float>(sg, K, a.g_raw + ((size_t)tok0 * p.HV + hv) * K, (size_t)p.HV * K, L, K);
  cp_async_wait_all();
  __syncthreads();
  // dyg = reverse in-chunk cumsum of dGam: NP row parts, each offset by the parts below it
  const int NP = blockDim.x / K, part = tid / K, cc = tid % K, rows = CH / NP;
  float* sred = sT;  // [NP][K]; T is done
  {
    float t = 0.f;
    for (int i = part * rows; i < (part + 1) * rows; ++i) t += sdG[i * K + cc];
    sred[part * K + cc] = t;
  }
  __syncthreads();
  const float nexp = -expf(a.A_log[hv]);
  const float bias = a.dt_bias ? a.dt_bias[(size_t)hv * K + cc] : 0.f;
  float acc = 0.f, pA = 0.f, pB = 0.f;
  for (int q = part + 1; q < NP; ++q) acc += sred[q * K + cc];
  for (int i = (part + 1) * rows - 1; i >= part * rows; --i) {
    acc += sdG[i * K + cc];
    if (i < L) {
      const size_t o = ((size_t)(tok0 + i) * p.HV + hv) * K + cc;
      const float x = sg[i * K + cc] + bias;
      const float sp = x > 20.f ? x : log1pf(expf(x));
      const float sig = x > 20.f ? 1.f : 1.f / (1.f + expf(-x));
      const float dgr = acc * nexp * sig;
      a.dg[o] = acc;
      if (a.dg_raw) a.dg_raw[o] = dgr;
      pA += acc * nexp * sp;
      pB += dgr;
    }
  }
  __syncthreads();
  sred[part * K + cc] = pB;
  for (int off = 16; off > 0; off >>= 1) pA += __shfl_xor_sync(0xffffffffu, pA, off);
  if (lane == 0) sdb[warp] = pA;
  __syncthreads();
  float* pg = w.pgp + u * (K + 1);
  if (tid < K) {
    float t = 0.f;
    for (int q = 0; q < NP; ++q) t += sred[q * K + tid];
    pg[tid] = t;
  }
  if (tid == 0) {
    float t = 0.f;
    for (int q = 0; q < nwarp; ++q) t += sdb[q];
    pg[K] = t;
  }
}

// ---------------------------------------------------------------- WY backward, tcgen05
// k_kda_bwd_wy's work for bf16 with K = V = 128, the five products on the tensor cores from
// compensated bf16 pairs (V is bf16 already), 512 threads (16 warps: four per TMEM
// sub-partition, each taking a quarter of an accumulator's columns).  With X' = k e^{Gam}
// (X = diag(beta) X'):
//   [0, 64)    dT = (dW X'^T + dU V^T) diag(beta)     (beta applied to the columns on the way out)
//   [64, 192)  dX = T^T dW,   [192, 320) dY = T^T dU
//   [320, 384) Z = dT T^T,    [384, 448) -dA = T^T Z
// The dk share and dGam of the unit (from k_kda_tc_bwd_dqk) are read into shared memory,
// collect this kernel's terms there, and dGam goes through the reverse cumsum and the gate
// chain from there; the dA gated products run by channel.
namespace kw {
using namespace tcx;
constexpr int NT = 512;
constexpr int TT = 64 * 128;                          // [64 rows][64 bf16] block
// fixed: Gam (fp32), k (bf16 row-major), V (bf16 tile), small vectors (4 KB)
constexpr int O_G = 0, O_K = 32768, O_V = 49152, O_VEC = 65536;
// region A: dW, dU, X' (hi, lo); after the first products: dk, dGam, F1 (fp32 [64][128] each),
// F1 giving way to the raw gate inputs once its terms are in
constexpr int O_A = 69632;
constexpr int O_DWH = O_A, O_DWL = O_A + 16384, O_DUH = O_A + 32768, O_DUL = O_A + 49152;
constexpr int O_XH = O_A + 65536, O_XL = O_A + 81920;
constexpr int O_ACK = O_A, O_ACG = O_A + 32768, O_F1 = O_A + 65536;
// region B: T, dT, Z (hi, lo [64][64] each); after the last product: dA^T (fp32 [64][LDT])
constexpr int O_B = O_A + 98304;
constexpr int O_TH = O_B, O_TL = O_B + 8192, O_DTH = O_B + 16384, O_DTL = O_B + 24576;
constexpr int O_ZH = O_B + 32768, O_ZL = O_B + 40960;
constexpr int O_DA = O_B;
constexpr int WY_BYTES = O_B + 49152;
static_assert(CH * LDT * 4 <= 49152, "dA fits region B");
static_assert(1024 + WY_BYTES <= 227 * 1024, "wy_bwd shared memory");
static_assert(O_A % 1024 == 0 && O_B % 1024 == 0, "tile alignment");
}  // namespace kw

__global__ void __launch_bounds__(kw::NT, 1) k_kda_tc_bwd_wy(Problem p, Args a, KdaWork w) {
  using namespace kw;
  if (kda_failed(w)) return;
  const int gc = blockIdx.x, hv = blockIdx.y;
  const int4 e = w.chunk_tab[gc];
  if (e.x < 0) return;
  constexpr int K = 128, V = 128, NW = NT / 32;
  const int L = e.z, tok0 = e.w, hk = hv / p.G, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  extern __shared__ unsigned char smraw[];
  unsigned char* sm = align1k(smraw);
  float* sG = reinterpret_cast<float*>(sm + O_G);
  bf16* sK = reinterpret_cast<bf16*>(sm + O_K);
  float* sb = reinterpret_cast<float*>(sm + O_VEC);   // [64] beta, 0 past L
  float* sdb = sb + 64;                                // [64] dbeta; later [16] warp sums
  float* sdbp = sb + 128;                              // [4][64] dbeta by column quarter
  float* sred = sb + 384;                              // [4][128]
  float* ack = reinterpret_cast<float*>(sm + O_ACK);
  float* acg = reinterpret_cast<float*>(sm + O_ACG);
  float* sF1 = reinterpret_cast<float*>(sm + O_F1);
  float* sdA = reinterpret_cast<float*>(sm + O_DA);
  __shared__ uint64_t bar[3];
  __shared__ uint32_t tslot;
  int* err = w.status;
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    mbar_init(&bar[2], 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (warp == 0) {
    tmem_alloc(&tslot, 512);
    tmem_relinquish();
  }
  const size_t u = (size_t)gc * p.HV + hv, uk = u * CH * K;
  {  // k (row-major) and V (swizzled tile), rows past L zero; beta; dW, dU, T (fp32) loads
    const bf16* gk = static_cast<const bf16*>(a.k) + ((size_t)tok0 * p.H + hk) * K;
    const bf16* gv = static_cast<const bf16*>(a.v) + ((size_t)tok0 * p.HV + hv) * V;
    uint4 rk[2], rv[2];
    float4 rw[4], ru[4], rt[2];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int x = tid + NT * m, row = x >> 4, j = x & 15;
      rk[m] = rv[m] = make_uint4(0u, 0u, 0u, 0u);
      if (row < L) {
        rk[m] = __ldg(reinterpret_cast<const uint4*>(gk + (size_t)row * p.H * K + 8 * j));
        rv[m] = __ldg(reinterpret_cast<const uint4*>(gv + (size_t)row * p.HV * V + 8 * j));
      }
      const float4* pw = reinterpret_cast<const float4*>(w.dW + uk + row * K + 8 * j);
      const float4* pu = reinterpret_cast<const float4*>(w.dU + u * CH * V + row * V + 8 * j);
      rw[2 * m] = __ldg(pw);
      rw[2 * m + 1] = __ldg(pw + 1);
      ru[2 * m] = __ldg(pu);
      ru[2 * m + 1] = __ldg(pu + 1);
    }
    {
      const int row = tid >> 3, j = tid & 7;
      const float4* pt = reinterpret_cast<const float4*>(w.Tm + u * CH * CH + row * CH + 8 * j);
      rt[0] = __ldg(pt);
      rt[1] = __ldg(pt + 1);
    }
    if (tid < CH) sb[tid] = tid < L ? a.beta[(size_t)(tok0 + tid) * p.HV + hv] : 0.f;
    copy_async(sG, w.Gam + uk, CH * K);
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int x = tid + NT * m, row = x >> 4, j = x & 15;
      reinterpret_cast<uint4*>(sK)[x] = rk[m];
      *reinterpret_cast<uint4*>(sm + O_V + sw128_chunk(row, j, TT)) = rv[m];
      const float fw[8] = {rw[2 * m].x, rw[2 * m].y, rw[2 * m].z, rw[2 * m].w,
                           rw[2 * m + 1].x, rw[2 * m + 1].y, rw[2 * m + 1].z, rw[2 * m + 1].w};
      const float fu[8] = {ru[2 * m].x, ru[2 * m].y, ru[2 * m].z, ru[2 * m].w,
                           ru[2 * m + 1].x, ru[2 * m + 1].y, ru[2 * m + 1].z, ru[2 * m + 1].w};
      st_chunk_split(sm + O_DWH, sm + O_DWL, row, j, TT, fw);
      st_chunk_split(sm + O_DUH, sm + O_DUL, row, j, TT, fu);
    }
    {
      const int row = tid >> 3, j = tid & 7;
      const float f[8] = {rt[0].x, rt[0].y, rt[0].z, rt[0].w, rt[1].x, rt[1].y, rt[1].z, rt[1].w};
      st_chunk_split(sm + O_TH, sm + O_TL, row, j, TT, f);
    }
  }
  cp_async_wait_all();
  __syncthreads();
#pragma unroll
  for (int m = 0; m < 2; ++m) {  // X' = k e^{Gam}
    const int x = tid + NT * m, row = x >> 4, j = x & 15;
    float f[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int o = row * K + 8 * j + q;
      f[q] = __bfloat162float(sK[o]) * exp2f(sG[o]);
    }
    st_chunk_split(sm + O_XH, sm + O_XL, row, j, TT, f);
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tslot;
  const uint32_t aDWH = smem_u32(sm + O_DWH), aDWL = smem_u32(sm + O_DWL), aDUH = smem_u32(sm + O_DUH);
  const uint32_t aDUL = smem_u32(sm + O_DUL), aXH = smem_u32(sm + O_XH), aXL = smem_u32(sm + O_XL);
  const uint32_t aV = smem_u32(sm + O_V), aTH = smem_u32(sm + O_TH), aTL = smem_u32(sm + O_TL);
  if (tid == 0) {
    constexpr uint32_t i64 = idesc_bf16(64, 64, false, false), i128 = idesc_bf16(64, 128, true, true);
#pragma unroll
    for (int s = 0; s < 8; ++s) {  // dT (before beta)
      const uint64_t dwh = desc_kmajor(aDWH, s, TT), xh = desc_kmajor(aXH, s, TT);
      mma_bf16(taddr(tb, 0, 0), dwh, xh, i64, s > 0);
      mma_bf16(taddr(tb, 0, 0), dwh, desc_kmajor(aXL, s, TT), i64, 1);
      mma_bf16(taddr(tb, 0, 0), desc_kmajor(aDWL, s, TT), xh, i64, 1);
      const uint64_t vv = desc_kmajor(aV, s, TT);
      mma_bf16(taddr(tb, 0, 0), desc_kmajor(aDUH, s, TT), vv, i64, 1);
      mma_bf16(taddr(tb, 0, 0), desc_kmajor(aDUL, s, TT), vv, i64, 1);
    }
#pragma unroll
    for (int s = 0; s < 4; ++s) {  // dX = T^T dW, dY = T^T dU
      const uint64_t th = desc_mnmajor(aTH, s, TT), tl = desc_mnmajor(aTL, s, TT);
      const uint64_t dwh = desc_mnmajor(aDWH, s, TT), duh = desc_mnmajor(aDUH, s, TT);
      mma_bf16(taddr(tb, 0, 64), th, dwh, i128, s > 0);
      mma_bf16(taddr(tb, 0, 64), th, desc_mnmajor(aDWL, s, TT), i128, 1);
      mma_bf16(taddr(tb, 0, 64), tl, dwh, i128, 1);
      mma_bf16(taddr(tb, 0, 192), th, duh, i128, s > 0);
      mma_bf16(taddr(tb, 0, 192), th, desc_mnmajor(aDUL, s, TT), i128, 1);
      mma_bf16(taddr(tb, 0, 192), tl, duh, i128, 1);
    }
    mma_commit(&bar[0]);
  }
  // M = 64 accumulators, 16-lane loads: warp (sub-partition warp % 4, quarter warp / 4), rows r0
  // and r0 + 8, columns (quarter of the accumulator) 8j + cq + {0, 1}
  const int qt = warp >> 2, sub = 32 * (warp & 3), r0 = 16 * (warp & 3) + (lane >> 2), cq = 2 * (lane & 3);
  bool ok = __syncthreads_and(mbar_wait(&bar[0], 0, err));
  tc_fence_after();
  if (ok) {  // dT diag(beta) as a hi/lo tile (columns [16 qt, +16))
    float d[8];
    tmem_ld16dp_x2(taddr(tb, sub, 16 * qt), d);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int c = 16 * qt + 8 * j + cq;
      const float b0 = sb[c], b1 = sb[c + 1];
      st_pair_split(sm + O_DTH, sm + O_DTL, r0, c, TT, d[4 * j] * b0, d[4 * j + 1] * b1);
      st_pair_split(sm + O_DTH, sm + O_DTL, r0 + 8, c, TT, d[4 * j + 2] * b0, d[4 * j + 3] * b1);
    }
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t aDTH = smem_u32(sm + O_DTH), aDTL = smem_u32(sm + O_DTL);
  if (ok && tid == 0) {  // Z = dT T^T
    constexpr uint32_t i64 = idesc_bf16(64, 64, false, false);
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const uint64_t dth = desc_kmajor(aDTH, s, TT), th = desc_kmajor(aTH, s, TT);
      mma_bf16(taddr(tb, 0, 320), dth, th, i64, s > 0);
      mma_bf16(taddr(tb, 0, 320), dth, desc_kmajor(aTL, s, TT), i64, 1);
      mma_bf16(taddr(tb, 0, 320), desc_kmajor(aDTL, s, TT), th, i64, 1);
    }
    mma_commit(&bar[1]);
  }
  // region A is free: the unit's dk share and dGam from the output-side kernel
  {
    const float4* k4 = reinterpret_cast<const float4*>(w.dkp + uk);
    const float4* g4 = reinterpret_cast<const float4*>(w.dGam + uk);
    for (int x = tid; x < CH * K / 4; x += NT) {
      reinterpret_cast<float4*>(ack)[x] = __ldg(k4 + x);
      reinterpret_cast<float4*>(acg)[x] = __ldg(g4 + x);
      reinterpret_cast<float4*>(sF1)[x] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  __syncthreads();
  if (ok) {  // dv = beta dY; dbeta = rowsum(dY V) + rowsum(dX k e^{Gam}); dk, dGam += beta dX e^{Gam} (1, k)
    float x[16], y[16];
    tmem_ld16dp_x4(taddr(tb, sub, 64 + 32 * qt), x);
    tmem_ld16dp_x4(taddr(tb, sub, 192 + 32 * qt), y);
    tmem_wait_ld();
    bf16* dv = static_cast<bf16*>(a.dv) + ((size_t)tok0 * p.HV + hv) * V;
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int i = r0 + 8 * hr;
      const float bi = sb[i];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = 32 * qt + 8 * j + cq;
        const float y0 = y[4 * j + 2 * hr], y1 = y[4 * j + 2 * hr + 1];
        const float2 vv = ld_pair(sm + O_V, i, c, TT);
        rs[hr] += y0 * vv.x + y1 * vv.y;
        if (i < L) *reinterpret_cast<uint32_t*>(dv + (size_t)i * p.HV * V + c) = pack_bf16(bi * y0, bi * y1);
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          const int o = i * K + c + b;
          const float eg = exp2f(sG[o]), dx = x[4 * j + 2 * hr + b], kt = __bfloat162float(sK[o]) * eg;
          rs[hr] = fmaf(dx, kt, rs[hr]);
          ack[o] = fmaf(bi * dx, eg, ack[o]);
          acg[o] = fmaf(bi * dx, kt, acg[o]);
        }
      }
    }
    rs[0] = quad_sum(rs[0]);
    rs[1] = quad_sum(rs[1]);
    if ((lane & 3) == 0) {
      sdbp[qt * 64 + r0] = rs[0];
      sdbp[qt * 64 + r0 + 8] = rs[1];
    }
  }
  ok = __syncthreads_and(ok && mbar_wait(&bar[1], 0, err));
  tc_fence_after();
  if (tid < CH) sdb[tid] = (sdbp[tid] + sdbp[64 + tid]) + (sdbp[128 + tid] + sdbp[192 + tid]);
  if (ok) {  // Z as a hi/lo tile
    float d[8];
    tmem_ld16dp_x2(taddr(tb, sub, 320 + 16 * qt), d);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int c = 16 * qt + 8 * j + cq;
      st_pair_split(sm + O_ZH, sm + O_ZL, r0, c, TT, d[4 * j], d[4 * j + 1]);
      st_pair_split(sm + O_ZH, sm + O_ZL, r0 + 8, c, TT, d[4 * j + 2], d[4 * j + 3]);
    }
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (ok && tid == 0) {  // T^T Z
    constexpr uint32_t i64 = idesc_bf16(64, 64, true, true);
    const uint32_t aZH = smem_u32(sm + O_ZH), aZL = smem_u32(sm + O_ZL);
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const uint64_t th = desc_mnmajor(aTH, s, TT), zh = desc_mnmajor(aZH, s, TT);
      mma_bf16(taddr(tb, 0, 384), th, zh, i64, s > 0);
      mma_bf16(taddr(tb, 0, 384), th, desc_mnmajor(aZL, s, TT), i64, 1);
      mma_bf16(taddr(tb, 0, 384), desc_mnmajor(aTL, s, TT), zh, i64, 1);
    }
    mma_commit(&bar[2]);
  }
  ok = __syncthreads_and(ok && mbar_wait(&bar[2], 0, err));
  tc_fence_after();
  if (ok) {  // dA = -T^T Z, strictly lower, transposed over region B
    float d[8];
    tmem_ld16dp_x2(taddr(tb, sub, 384 + 16 * qt), d);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = r0 + 8 * (q >> 1), c = 16 * qt + 8 * j + cq + (q & 1);
        sdA[c * LDT + i] = c < i ? -d[4 * j + q] : 0.f;
      }
  }
  __syncthreads();
  // A_ij = beta_i sum_c k_i k_j e^{Gam_i - Gam_j}: F1 (rows, weights dA), G1 (columns, beta_i dA)
  if (ok)
    gated_products_k128x4(sdA, sK, sK, sb, sG,
                          [&](int i, int c, float f) { sF1[i * K + c] += f; },
                          [&](int j, int c, float g) {
                            ack[j * K + c] += g;
                            acg[j * K + c] -= __bfloat162float(sK[j * K + c]) * g;
                          });
  // F1 terms: dk += beta F1, dGam += beta k F1, dbeta += rowsum(k F1)
  for (int i = warp; i < CH; i += NW) {
    float sacc = 0.f;
    for (int c = lane; c < K; c += 32) {
      const int o = i * K + c;
      const float f = sF1[o], kk = __bfloat162float(sK[o]);
      sacc += kk * f;
      ack[o] += sb[i] * f;
      acg[o] += sb[i] * kk * f;
    }
    for (int off = 16; off > 0; off >>= 1) sacc += __shfl_xor_sync(0xffffffffu, sacc, off);
    if (ok && lane == 0 && i < L) a.dbeta[(size_t)(tok0 + i) * p.HV + hv] = sdb[i] + sacc;
  }
  __syncthreads();
  float* sg = sF1;  // F1 is done: the raw gate inputs (rows past L zero)
  {
    const float* gsrc = a.g_raw + ((size_t)tok0 * p.HV + hv) * K;
    for (int x = tid; x < CH * K / 4; x += NT) {
      const int row = x >> 5, c4 = x & 31;
      reinterpret_cast<float4*>(sg)[x] = row < L ? __ldg(reinterpret_cast<const float4*>(gsrc + (size_t)row * p.HV * K) + c4)
                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float4* dk4 = reinterpret_cast<float4*>(w.dkp + uk);
    for (int x = tid; x < CH * K / 4; x += NT) dk4[x] = reinterpret_cast<const float4*>(ack)[x];
  }
  __syncthreads();
  // dyg = reverse in-chunk cumsum of dGam: four row parts, each offset by the parts below it
  constexpr int NP = NT / K, rows = CH / NP;
  const int part = tid / K, cc = tid % K;
  {
    float t = 0.f;
    for (int i = part * rows; i < (part + 1) * rows; ++i) t += acg[i * K + cc];
    sred[part * K + cc] = t;
  }
  __syncthreads();
  const float nexp = -expf(a.A_log[hv]);
  const float bias = a.dt_bias ? a.dt_bias[(size_t)hv * K + cc] : 0.f;
  float acc = 0.f, pA = 0.f, pB = 0.f;
  for (int q = part + 1; q < NP; ++q) acc += sred[q * K + cc];
  for (int i = (part + 1) * rows - 1; i >= part * rows; --i) {
    acc += acg[i * K + cc];
    if (i < L) {
      const size_t o = ((size_t)(tok0 + i) * p.HV + hv) * K + cc;
      const float xg = sg[i * K + cc] + bias;
      float sp, sig;
      softplus_sigmoid(xg, sp, sig);
      const float dgr = acc * nexp * sig;
      a.dg[o] = acc;
      if (a.dg_raw) a.dg_raw[o] = dgr;
      pA += acc * nexp * sp;
      pB += dgr;
    }
  }
  __syncthreads();
  sred[part * K + cc] = pB;
  for (int off = 16; off > 0; off >>= 1) pA += __shfl_xor_sync(0xffffffffu, pA, off);
  if (lane == 0) sdb[warp] = pA;
  __syncthreads();
  float* pg = w.pgp + u * (K + 1);
  if (tid < K) {
    float t = 0.f;
    for (int q = 0; q < NP; ++q) t += sred[q * K + tid];
    pg[tid] = t;
  }
  if (tid == 0) {
    float t = 0.f;
    for (int q = 0; q < NW; ++q) t += sdb[q];
    pg[K] = t;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, 512);
}

// dA_log[hv] and ddt_bias[hv*K + c]: the per-chunk sums of the head's chunks (their count from
// the chunk table), eight interleaved partial sums added in a fixed order, so the result is the
// same on every run and the loads of eight chunks are in flight at once.
__global__ void __launch_bounds__(256) k_kda_param_grads(Problem p, Args a, KdaWork w) {
  if (kda_failed(w)) return;
  const int hv = blockIdx.x, K = p.K;
  const int nc = max(0, min(w.status[1], p.NCmax));
  const size_t stride = (size_t)p.HV * (K + 1);
  for (int c = threadIdx.x; c <= K; c += blockDim.x) {
    const float* src = w.pgp + (size_t)hv * (K + 1) + c;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    int gc = 0;
    for (; gc + 8 <= nc; gc += 8)
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] += src[(size_t)(gc + q) * stride];
    for (int q = 0; gc < nc; ++gc, ++q) acc[q] += src[(size_t)gc * stride];
    const float s = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
    if (c < K && a.ddt_bias) a.ddt_bias[(size_t)hv * K + c] = s;
    if (c == K && a.dA_log) a.dA_log[hv] = s;
  }
}

size_t scan_smem(int K) { return (size_t)(32 * (K + 1) + CH * CH + 3 * CH * K + 2 * CH * 32 + K) * sizeof(float); }
size_t dqk_smem(int K, int V) {
  return (size_t)(dqk_x1(K, V) + CH * K + CH * (V > K ? V : K) + CH * (V + 1) + CH * LDP + 5 * K) *
         sizeof(float);
}
size_t wy_smem(int K, int V) {
  const int big = (V > K ? V : K) * CH > CH * LDP ? (V > K ? V : K) * CH : CH * LDP;
  return (size_t)(2 * CH * K + CH * (K + 1) + CH * (V + 1) + 2 * big + CH * LDA + CH * LDP + 2 * CH) *
         sizeof(float);
}

template <typename Kern>
cudaError_t go(const char* name, Kern kern, dim3 grid, size_t smem, cudaStream_t s, const Problem& p,
               const Args& a, const KdaWork& w, int threads = 256) {
  if (grid.x == 0 || grid.y == 0 || grid.z == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ProfScope ps(name, s);
  kern<<<grid, threads, smem, s>>>(p, a, w);
  return cudaGetLastError();
}

// bf16 with 128-wide key and value heads runs the tensor-core kernels
template <typename T>
bool kda_tc(const Problem& p) {
  return std::is_same<T, __nv_bfloat16>::value && p.K == 128 && p.V == 128;
}

template <typename T>
cudaError_t backward_t(const Problem& p, const Args& a, const KdaWork& w, cudaStream_t s) {
  cudaError_t e = kda_tc<T>(p)
      ? go("kda_tc_bwd_scan", k_kda_tc_bwd_scan, dim3(p.Nst, p.HV, 2), 1024 + kb::BSCAN_BYTES, s, p, a, w, kb::NT)
      : go("kda_bwd_scan", k_kda_bwd_scan<T>, dim3(p.Nst, p.HV, p.V / 32), scan_smem(p.K), s, p, a, w);
  if (e == cudaSuccess)
    e = kda_tc<T>(p) ? go("kda_tc_bwd_dqk", k_kda_tc_bwd_dqk, dim3(p.NCmax, p.HV), 1024 + kt::DQK_BYTES, s, p, a, w, kt::NT)
                     : go("kda_bwd_dqk", k_kda_bwd_dqk<T>, dim3(p.NCmax, p.HV), dqk_smem(p.K, p.V), s, p, a, w);
  if (e == cudaSuccess)
    e = kda_tc<T>(p) ? go("kda_tc_bwd_wy", k_kda_tc_bwd_wy, dim3(p.NCmax, p.HV), 1024 + kw::WY_BYTES, s, p, a, w, kw::NT)
                     : go("kda_bwd_wy", k_kda_bwd_wy<T>, dim3(p.NCmax, p.HV), wy_smem(p.K, p.V), s, p, a, w);
  if (e != cudaSuccess) return e;
  Work gw{};  // the group sum's view of the shares
  gw.status = w.status;
  gw.chunk_tab = w.chunk_tab;
  gw.dqp = w.dqp;
  gw.dkp = w.dkp;
  e = launch_dqdk_group_sum(p, a, gw, std::is_same<T, __nv_bfloat16>::value, s);
  if (e == cudaSuccess && (a.dA_log || a.ddt_bias)) {  // zeros when there are no chunks
    ProfScope ps("kda_param_grads", s);
    k_kda_param_grads<<<p.HV, 256, 0, s>>>(p, a, w);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace

cudaError_t kda_chunk_backward(const Problem& p, const Args& a, const KdaWork& w, bool bf16, cudaStream_t s) {
  return bf16 ? backward_t<__nv_bfloat16>(p, a, w, s) : backward_t<float>(p, a, w, s);
}

}  // namespace gdn
