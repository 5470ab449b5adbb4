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
#include <type_traits>

#include "ffma_tiles.cuh"
#include "gdn_common.cuh"
#include "gdn_launch.h"
#include "gdn_tc_common.cuh"  // unit_lower_inverse64, LDA
#include "kda_gate_math.cuh"

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

// k_kda_wy for bf16 with K = V = 128, its products on the tensor cores from compensated bf16
// pairs.  The blocks of A and P below the diagonal, for each sub-chunk a (through r = 16 a - 1):
// one M = 64 tile L holds, in every row i >= 16, k_i e^{Gam_i - Gam_r(i)} (Lq the same with
// q_i), and R_a the rows k_j e^{Gam_r - Gam_j}, j < 16 a; the product L R_a^T holds sub-chunk a's
// block in rows 16a..16a+15 (the other rows are not read).  The diagonal blocks are summed on
// CUDA cores meanwhile (a warp per row, lanes over channels, one butterfly reduce-scatter of the
// row's 32 sums).  After the blocked inverse: W = T' X' and U~ = T' V with
// T' = T diag(beta), X' = k e^{Gam}.  TMEM columns: A_a at 0, 16, 48; P_a at 96, 112, 144;
// W at 256, U~ at 384.
namespace kf {
using namespace tcx;
constexpr int NT = 512;  // threads (16 warps; the blocked inverse runs on the first 256)
constexpr int TT = 64 * 128;
constexpr int O_V = 0, O_KB = 16384, O_QB = 32768, O_G = 49152, O_DD = 81920, O_B = 90112;
constexpr int O_R = 91136;  // region: the A/P operand tiles, then the inverse and the W/U~ operands
constexpr int O_LKH = O_R, O_LKL = O_R + 16384, O_LQH = O_R + 32768, O_LQL = O_R + 49152;
constexpr int O_R1 = O_R + 65536, O_R2 = O_R + 73728, O_R3 = O_R + 90112;  // hi then lo, 16a rows each
constexpr int O_SA = O_R, O_ST = O_R + 17408, O_SX = O_R + 34816, O_SP = O_R + 52224;
constexpr int O_TPH = O_R + 53248, O_TPL = O_R + 61440, O_XH = O_R + 69632, O_XL = O_R + 86016;
constexpr int WYF_BYTES = O_R + 114688;
static_assert(O_SP + CH * CH * 4 <= O_R + 114688 && O_XL + 16384 <= O_R + 114688, "region");
static_assert(1024 + WYF_BYTES <= 227 * 1024, "kda wy shared memory");
static_assert(O_R % 1024 == 0 && O_TPH % 1024 == 0 && O_XH % 1024 == 0, "tile alignment");
}  // namespace kf

// Rows [0, R) of one or two fp32 [R][128] matrices (contiguous rows) as hi/lo pairs of sw128
// tiles, all of a thread's loads issued before its first store (256 threads).
template <int R>
__device__ __forceinline__ void kt_split_rows(unsigned char* hi0, unsigned char* lo0, const float* src0,
                                              unsigned char* hi1, unsigned char* lo1, const float* src1) {
  constexpr int N = R * 16 / 256;
  float4 r[4 * N];
#pragma unroll
  for (int m = 0; m < N; ++m) {
    const int x = threadIdx.x + 256 * m, row = x >> 4, j = x & 15;
    const float4* p0 = reinterpret_cast<const float4*>(src0 + row * 128 + 8 * j);
    r[4 * m] = __ldg(p0);
    r[4 * m + 1] = __ldg(p0 + 1);
    if (src1) {
      const float4* p1 = reinterpret_cast<const float4*>(src1 + row * 128 + 8 * j);
      r[4 * m + 2] = __ldg(p1);
      r[4 * m + 3] = __ldg(p1 + 1);
    }
  }
#pragma unroll
  for (int m = 0; m < N; ++m) {
    const int x = threadIdx.x + 256 * m, row = x >> 4, j = x & 15;
    const float f0[8] = {r[4 * m].x, r[4 * m].y, r[4 * m].z, r[4 * m].w,
                         r[4 * m + 1].x, r[4 * m + 1].y, r[4 * m + 1].z, r[4 * m + 1].w};
    tcx::st_chunk_split(hi0, lo0, row, j, R * 128, f0);
    if (src1) {
      const float f1[8] = {r[4 * m + 2].x, r[4 * m + 2].y, r[4 * m + 2].z, r[4 * m + 2].w,
                           r[4 * m + 3].x, r[4 * m + 3].y, r[4 * m + 3].z, r[4 * m + 3].w};
      tcx::st_chunk_split(hi1, lo1, row, j, R * 128, f1);
    }
  }
}

__global__ void __launch_bounds__(kf::NT, 1) k_kda_tc_wy(Problem p, Args a, KdaWork w) {
  using namespace kf;
  if (kda_failed(w)) return;
  const int gc = blockIdx.x, hv = blockIdx.y;
  const int4 e = w.chunk_tab[gc];
  if (e.x < 0) return;
  constexpr int K = 128, V = 128;
  const int L = e.z, tok0 = e.w, hk = hv / p.G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = NT / 32;
  extern __shared__ unsigned char smraw[];
  unsigned char* sm = align1k(smraw);
  bf16* sK = reinterpret_cast<bf16*>(sm + O_KB);
  bf16* sQ = reinterpret_cast<bf16*>(sm + O_QB);
  float* sG = reinterpret_cast<float*>(sm + O_G);
  float* sDA = reinterpret_cast<float*>(sm + O_DD);  // [4][16][16] diagonal blocks of A (times beta_i)
  float* sDP = sDA + 1024;                           // [4][16][16] of P
  float* sb = reinterpret_cast<float*>(sm + O_B);
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
  {  // k, q (row-major bf16), V (swizzled tile), rows past L zero; beta
    const size_t rs = (size_t)p.H * K;
    const bf16* gk = static_cast<const bf16*>(a.k) + ((size_t)tok0 * p.H + hk) * K;
    const bf16* gq = static_cast<const bf16*>(a.q) + ((size_t)tok0 * p.H + hk) * K;
    const bf16* gv = static_cast<const bf16*>(a.v) + ((size_t)tok0 * p.HV + hv) * V;
    uint4 rk[2], rq[2], rv[2];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int x = tid + NT * m, row = x >> 4, j = x & 15;
      rk[m] = rq[m] = rv[m] = make_uint4(0u, 0u, 0u, 0u);
      if (row < L) {
        rk[m] = __ldg(reinterpret_cast<const uint4*>(gk + row * rs + 8 * j));
        rq[m] = __ldg(reinterpret_cast<const uint4*>(gq + row * rs + 8 * j));
        rv[m] = __ldg(reinterpret_cast<const uint4*>(gv + (size_t)row * p.HV * V + 8 * j));
      }
    }
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int x = tid + NT * m, row = x >> 4, j = x & 15;
      reinterpret_cast<uint4*>(sK)[x] = rk[m];
      reinterpret_cast<uint4*>(sQ)[x] = rq[m];
      *reinterpret_cast<uint4*>(sm + O_V + sw128_chunk(row, j, TT)) = rv[m];
    }
    if (tid < CH) sb[tid] = tid < L ? a.beta[(size_t)(tok0 + tid) * p.HV + hv] : 0.f;
  }
  {  // raw gate inputs, rows past L zero
    const float* gsrc = a.g_raw + ((size_t)tok0 * p.HV + hv) * K;
    for (int x = tid; x < CH * K / 4; x += NT) {
      const int row = x >> 5, c4 = x & 31;
      reinterpret_cast<float4*>(sG)[x] = row < L ? __ldg(reinterpret_cast<const float4*>(gsrc + (size_t)row * p.HV * K) + c4)
                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  __syncthreads();
  {  // the gate of every (token, channel), rows past L zero; then the cumsum per channel
    const float nexp = -expf(a.A_log[hv]);
    for (int x = tid; x < CH * K; x += NT) {
      const int i = x / K, c = x % K;
      float yg = 0.f;
      if (i < L) {
        const float z = sG[x] + (a.dt_bias ? a.dt_bias[(size_t)hv * K + c] : 0.f);
        yg = nexp * softplus20(z);
      }
      sG[x] = yg;
    }
    __syncthreads();
    if (tid < K) {
      float acc = 0.f;
      for (int i = 0; i < CH; ++i) {
        acc += sG[i * K + tid];
        sG[i * K + tid] = acc * LOG2E;
      }
    }
    __syncthreads();
  }
  // L tiles (rows >= 16) and R_a (a = 1, 2, 3) as hi/lo pairs
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    const int x = tid + NT * m, row = x >> 4, j = x & 15;
    float fk[8], fq[8];
    const int r = row >= 16 ? 16 * (row >> 4) - 1 : 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int c = 8 * j + q;
      const float ex = row >= 16 ? exp2f(sG[row * K + c] - sG[r * K + c]) : 0.f;
      fk[q] = __bfloat162float(sK[row * K + c]) * ex;
      fq[q] = __bfloat162float(sQ[row * K + c]) * ex;
    }
    st_chunk_split(sm + O_LKH, sm + O_LKL, row, j, TT, fk);
    st_chunk_split(sm + O_LQH, sm + O_LQL, row, j, TT, fq);
  }
  for (int x = tid; x < 96 * 16; x += NT) {  // 16 + 32 + 48 rows of 16 chunks
    const int ra = x >> 4, j = x & 15;
    const int A = ra < 16 ? 1 : (ra < 48 ? 2 : 3), row = ra - (A == 1 ? 0 : (A == 2 ? 16 : 48));
    const int r = 16 * A - 1, off = A == 1 ? O_R1 : (A == 2 ? O_R2 : O_R3), bb = 16 * A * 128;
    float f[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int c = 8 * j + q;
      f[q] = __bfloat162float(sK[row * K + c]) * exp2f(sG[r * K + c] - sG[row * K + c]);
    }
    st_chunk_split(sm + off, sm + off + 2 * bb, row, j, bb, f);
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tslot;
  if (tid == 0) {
    const uint32_t lkh = smem_u32(sm + O_LKH), lkl = smem_u32(sm + O_LKL);
    const uint32_t lqh = smem_u32(sm + O_LQH), lql = smem_u32(sm + O_LQL);
#pragma unroll
    for (int A = 1; A <= 3; ++A) {
      const int bb = 16 * A * 128;
      const uint32_t rh = smem_u32(sm + (A == 1 ? O_R1 : (A == 2 ? O_R2 : O_R3))), rl = rh + 2 * bb;
      const uint32_t id = idesc_bf16(64, 16 * A, false, false);
      const int ca = A == 1 ? 0 : (A == 2 ? 16 : 48);
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const uint64_t bh = desc_kmajor(rh, s, bb), bl = desc_kmajor(rl, s, bb);
        const uint64_t akh = desc_kmajor(lkh, s, TT), aqh = desc_kmajor(lqh, s, TT);
        mma_bf16(taddr(tb, 0, ca), akh, bh, id, s > 0);
        mma_bf16(taddr(tb, 0, ca), akh, bl, id, 1);
        mma_bf16(taddr(tb, 0, ca), desc_kmajor(lkl, s, TT), bh, id, 1);
        mma_bf16(taddr(tb, 0, 96 + ca), aqh, bh, id, s > 0);
        mma_bf16(taddr(tb, 0, 96 + ca), aqh, bl, id, 1);
        mma_bf16(taddr(tb, 0, 96 + ca), desc_kmajor(lql, s, TT), bh, id, 1);
      }
    }
    mma_commit(&bar[0]);
  }
  // diagonal sub-blocks by row: warp w takes rows w, w + 8, ..; lane l the channels 4l..4l+3.  A
  // row's 16 A and 16 P partial sums (columns j of its sub-chunk, zero for j > i) are summed over
  // the lanes by one butterfly reduce-scatter (31 shuffles), after which lane l holds column l
  // of A (l < 16) or l - 16 of P.
  for (int i = warp; i < CH; i += NW) {
    const int b0 = i & ~(SUB - 1), c = 4 * lane;
    float ki[4], qi[4], gi[4];
    {
      const float4 g4 = *reinterpret_cast<const float4*>(sG + i * K + c);
      const uint2 k2 = *reinterpret_cast<const uint2*>(sK + i * K + c);
      const uint2 q2 = *reinterpret_cast<const uint2*>(sQ + i * K + c);
      const float2 k01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&k2.x));
      const float2 k23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&k2.y));
      const float2 q01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q2.x));
      const float2 q23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q2.y));
      ki[0] = k01.x; ki[1] = k01.y; ki[2] = k23.x; ki[3] = k23.y;
      qi[0] = q01.x; qi[1] = q01.y; qi[2] = q23.x; qi[3] = q23.y;
      gi[0] = g4.x; gi[1] = g4.y; gi[2] = g4.z; gi[3] = g4.w;
    }
    float v[2 * SUB];
#pragma unroll
    for (int jj = 0; jj < SUB; ++jj) {
      const int j = b0 + jj;
      float sa = 0.f, sp = 0.f;
      if (j <= i) {
        const float4 g4 = *reinterpret_cast<const float4*>(sG + j * K + c);
        const uint2 k2 = *reinterpret_cast<const uint2*>(sK + j * K + c);
        const float2 k01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&k2.x));
        const float2 k23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&k2.y));
        const float kj[4] = {k01.x, k01.y, k23.x, k23.y}, gj[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float kk = kj[q] * exp2f(gi[q] - gj[q]);
          sa = fmaf(ki[q], kk, sa);
          sp = fmaf(qi[q], kk, sp);
        }
      }
      v[jj] = sa;
      v[SUB + jj] = sp;
    }
#pragma unroll
    for (int off = 16, n = 2 * SUB; off > 0; off >>= 1, n >>= 1) {
      const bool up = (lane & off) != 0;
#pragma unroll
      for (int x = 0; x < n / 2; ++x) {
        const float keep = up ? v[x + n / 2] : v[x], give = up ? v[x] : v[x + n / 2];
        v[x] = keep + __shfl_xor_sync(0xffffffffu, give, off);
      }
    }
    const int jj = lane & (SUB - 1), j = b0 + jj;
    if (lane < SUB) {
      if (j <= i) sDA[i * SUB + jj] = j < i ? sb[i] * v[0] : 0.f;
    } else if (j <= i) {
      sDP[i * SUB + jj] = v[0];
    }
  }
  bool ok = __syncthreads_and(mbar_wait(&bar[0], 0, err));
  tc_fence_after();
  float* sA = reinterpret_cast<float*>(sm + O_SA);
  float* sT = reinterpret_cast<float*>(sm + O_ST);
  float* sX = reinterpret_cast<float*>(sm + O_SX);
  float* sP = reinterpret_cast<float*>(sm + O_SP);
  // A (times beta_i, strictly lower) and P (lower incl. the diagonal): diagonal blocks and zeros
  for (int x = tid; x < CH * CH; x += NT) {
    const int i = x >> 6, j = x & 63;
    float va = 0.f, vp = 0.f;
    if ((i >> 4) == (j >> 4) && j <= i) {
      va = sDA[(i & ~15) * SUB + (i & 15) * SUB + (j & 15)];
      vp = sDP[(i & ~15) * SUB + (i & 15) * SUB + (j & 15)];
    }
    sA[i * LDA + j] = va;
    sP[x] = vp;
  }
  __syncthreads();
  {  // the blocks below the diagonal from TMEM: warps of sub-partition a = warp % 4 (a >= 1);
     // (warp / 4) % 2 = 0 reads A, 1 reads P; the two warp sets warp / 8 split the 16-column pieces
    const int A = warp & 3, half = (warp >> 2) & 1, set = warp >> 3;
    if (ok && A > 0) {
      const int ca = (half ? 96 : 0) + (A == 1 ? 0 : (A == 2 ? 16 : 48));
      const int ib = 16 * A + (lane >> 2), cq = 2 * (lane & 3);
      for (int t = set; t < A; t += 2) {
        float v[8];
        tmem_ld16dp_x2(taddr(tb, 32 * A, ca + 16 * t), v);
        tmem_wait_ld();
#pragma unroll
        for (int jj = 0; jj < 2; ++jj)
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            const int i = ib + 8 * (qq >> 1), j = 16 * t + 8 * jj + cq + (qq & 1);
            const float val = v[4 * jj + qq];
            if (half) sP[i * CH + j] = val;
            else sA[i * LDA + j] = sb[i] * val;
          }
      }
    }
  }
  __syncthreads();
  const size_t u = (size_t)gc * p.HV + hv, uk = u * CH * K;
  {
    float4* gP = reinterpret_cast<float4*>(w.P + u * CH * CH);
    for (int x = tid; x < CH * CH / 4; x += NT) gP[x] = reinterpret_cast<const float4*>(sP)[x];
    if (w.Gam) {
      float4* gG = reinterpret_cast<float4*>(w.Gam + uk);
      for (int x = tid; x < CH * K / 4; x += NT) gG[x] = reinterpret_cast<const float4*>(sG)[x];
    }
  }
  if (tid < 256) tcx::unit_lower_inverse64<2>(sA, sT, sX, tid);  // T = (I + A)^-1 (threads 0..255)
  __syncthreads();
  if (w.Tm)
    for (int x = tid; x < CH * CH; x += NT) w.Tm[u * CH * CH + x] = sT[(x / CH) * LDA + x % CH];
  // K^ = k e^{Gam_C - Gam}, Q~ = q e^{Gam}, e^{Gam_C}; X' = k e^{Gam} and T' = T diag(beta) as tiles
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    const int x = tid + NT * m, row = x >> 4, j = x & 15;
    float fx[8], fh[8], fq[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int c = 8 * j + q, o = row * K + c;
      const float g = sG[o], kk = __bfloat162float(sK[o]);
      fx[q] = kk * exp2f(g);
      fh[q] = kk * exp2f(sG[(CH - 1) * K + c] - g);
      fq[q] = __bfloat162float(sQ[o]) * exp2f(g);
    }
    float4* kh = reinterpret_cast<float4*>(w.Kh + uk + row * K + 8 * j);
    float4* qt = reinterpret_cast<float4*>(w.Qt + uk + row * K + 8 * j);
    kh[0] = make_float4(fh[0], fh[1], fh[2], fh[3]);
    kh[1] = make_float4(fh[4], fh[5], fh[6], fh[7]);
    qt[0] = make_float4(fq[0], fq[1], fq[2], fq[3]);
    qt[1] = make_float4(fq[4], fq[5], fq[6], fq[7]);
    st_chunk_split(sm + O_XH, sm + O_XL, row, j, TT, fx);
  }
  for (int c = tid; c < K; c += NT) w.eGC[u * K + c] = exp2f(sG[(CH - 1) * K + c]);
  {
    const int row = tid >> 3, j = tid & 7;
    float f[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) f[q] = sT[row * LDA + 8 * j + q] * sb[8 * j + q];
    st_chunk_split(sm + O_TPH, sm + O_TPL, row, j, TT, f);
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (ok && tid == 0) {
    const uint32_t th = smem_u32(sm + O_TPH), tl = smem_u32(sm + O_TPL);
    const uint32_t xh = smem_u32(sm + O_XH), xl = smem_u32(sm + O_XL), vv = smem_u32(sm + O_V);
    constexpr uint32_t id = idesc_bf16(64, 128, false, true);
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const uint64_t ah = desc_kmajor(th, s, TT), al = desc_kmajor(tl, s, TT);
      const uint64_t bx = desc_mnmajor(xh, s, TT), bv = desc_mnmajor(vv, s, TT);
      mma_bf16(taddr(tb, 0, 256), ah, bx, id, s > 0);
      mma_bf16(taddr(tb, 0, 256), ah, desc_mnmajor(xl, s, TT), id, 1);
      mma_bf16(taddr(tb, 0, 256), al, bx, id, 1);
      mma_bf16(taddr(tb, 0, 384), ah, bv, id, s > 0);
      mma_bf16(taddr(tb, 0, 384), al, bv, id, 1);
    }
    mma_commit(&bar[1]);
  }
  ok = __syncthreads_and(ok && mbar_wait(&bar[1], 0, err));
  tc_fence_after();
  if (ok) {  // W and U~, M = 64 accumulators (rows r0, r0 + 8; this warp's quarter of the columns)
    const int qt = warp >> 2, sub = 32 * (warp & 3), r0 = 16 * (warp & 3) + (lane >> 2), cq = 2 * (lane & 3);
    float x[16], y[16];
    tmem_ld16dp_x4(taddr(tb, sub, 256 + 32 * qt), x);
    tmem_ld16dp_x4(taddr(tb, sub, 384 + 32 * qt), y);
    tmem_wait_ld();
    float* gW = w.W + uk;
    float* gU = w.Ut + u * CH * V;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = 32 * qt + 8 * j + cq;
      *reinterpret_cast<float2*>(gW + r0 * K + c) = make_float2(x[4 * j], x[4 * j + 1]);
      *reinterpret_cast<float2*>(gW + (r0 + 8) * K + c) = make_float2(x[4 * j + 2], x[4 * j + 3]);
      *reinterpret_cast<float2*>(gU + r0 * V + c) = make_float2(y[4 * j], y[4 * j + 1]);
      *reinterpret_cast<float2*>(gU + (r0 + 8) * V + c) = make_float2(y[4 * j + 2], y[4 * j + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, 512);
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

// k_kda_scan for bf16 with K = V = 128: two CTAs per (sequence, value head), each holding half of
// the state's rows (v in [64 z, 64 z + 64), z = blockIdx.z) in fp32 registers in the layout of an
// M = 64 accumulator (512 threads; thread: rows r0 and r0 + 8 of its sub-partition, columns
// 8j + cq + {0, 1} of its warp's quarter), both products of a chunk on the tensor cores from
// compensated bf16 pairs:
//   U[:, z] = U~[:, z] - W S_z^T        (M = 64 tokens, N = 64;  A = W, B = S_z, K-major)   TMEM [0, 64)
//   S_z' = S_z Diag(e^{Gam_C}) + U[:, z]^T K^   (M = 64, N = K;  A = U^T, B = K^, MN-major) TMEM [128, 256)
// It stores the state entering every chunk and U, as k_kda_scan does.  The next chunk's W, K^, U~
// and e^{Gam_C} are bulk-copied into an fp32 buffer while a chunk's products run, so a chunk reads
// no global memory on its critical path.
namespace ks {
using namespace tcx;
constexpr int NT = 512;  // threads: four warps per TMEM sub-partition, a quarter of the columns each
constexpr int TT = 64 * 128;
constexpr int O_WH = 0, O_WL = 16384, O_KH = 32768, O_KL = 49152, O_UH = 65536, O_UL = 73728;
constexpr int O_SH = 81920, O_SL = 98304, O_E = 114688;
// fp32 W [64][128], K^ [64][128], U~ [64][128] and e^{Gam_C} [128] of the next chunk (bulk copies)
constexpr int O_F = 115200;
constexpr int F_BYTES = 3 * 64 * 128 * 4 + 128 * 4;
constexpr int SCAN_BYTES = O_F + F_BYTES;
static_assert(1024 + SCAN_BYTES <= 227 * 1024, "kda scan shared memory");
}  // namespace ks

__global__ void __launch_bounds__(ks::NT, 1) k_kda_tc_scan(Problem p, Args a, KdaWork w) {
  using namespace ks;
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
  __shared__ uint64_t bar[3];
  __shared__ uint32_t tslot;
  int* err = w.status;
  float* sF = reinterpret_cast<float*>(sm + O_F);
  auto fetch = [&](size_t uu) {  // thread 0: the chunk's W, K^, U~ and e^{Gam_C} into sF
    mbar_expect_tx(&bar[2], F_BYTES);
    bulk_load(sF, w.W + uu * CH * 128, CH * 128 * 4, &bar[2]);
    bulk_load(sF + CH * 128, w.Kh + uu * CH * 128, CH * 128 * 4, &bar[2]);
    bulk_load(sF + 2 * CH * 128, w.Ut + uu * CH * 128, CH * 128 * 4, &bar[2]);
    bulk_load(sF + 3 * CH * 128, w.eGC + uu * 128, 128 * 4, &bar[2]);
  };
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    mbar_init(&bar[2], 1);
    mbar_fence_init();
    if (sq.y > 0) fetch((size_t)sq.x * p.HV + hv);
  }
  __syncthreads();
  if (warp == 0) {
    tmem_alloc(&tslot, 256);
    tmem_relinquish();
  }
  // S[4j + q]: row v0 + r0 + 8 (q >> 1), column 32 qt + 8j + cq + (q & 1)
  float S[16];
  {
    const float* h0 = a.h0 ? a.h0 + ((size_t)n * p.HV + hv) * K * V : nullptr;
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int r = v0 + r0 + 8 * (q >> 1), c = 32 * qt + 8 * j + cq + (q & 1);
        S[4 * j + q] = h0 ? h0[(size_t)c * V + r] : 0.f;
      }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tslot;
  const uint32_t aWH = smem_u32(sm + O_WH), aWL = smem_u32(sm + O_WL), aKH = smem_u32(sm + O_KH);
  const uint32_t aKL = smem_u32(sm + O_KL), aUH = smem_u32(sm + O_UH), aUL = smem_u32(sm + O_UL);
  const uint32_t aSH = smem_u32(sm + O_SH), aSL = smem_u32(sm + O_SL);
  bool ok = true;
  int pend = sq.y > 0 ? 0 : -1;  // parity of the bulk copy in flight (thread 0's view)
  for (int ci = 0; ci < sq.y && ok; ++ci) {
    const size_t u = (size_t)(sq.x + ci) * p.HV + hv;
    {  // this half of the state entering the chunk: stored, and as a hi/lo tile [64 v][128 k]
      float* h = w.h + u * V * K + (size_t)v0 * K;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = 32 * qt + 8 * j + cq;
        *reinterpret_cast<float2*>(h + r0 * K + c) = make_float2(S[4 * j], S[4 * j + 1]);
        *reinterpret_cast<float2*>(h + (r0 + 8) * K + c) = make_float2(S[4 * j + 2], S[4 * j + 3]);
        st_pair_split(sm + O_SH, sm + O_SL, r0, c, TT, S[4 * j], S[4 * j + 1]);
        st_pair_split(sm + O_SH, sm + O_SL, r0 + 8, c, TT, S[4 * j + 2], S[4 * j + 3]);
      }
    }
    ok = __syncthreads_and(mbar_wait(&bar[2], ci & 1, err));
    if (tid == 0 && ok) pend = -1;
    if (!ok) break;
#pragma unroll
    for (int m = 0; m < 2; ++m) {  // W and K^ as hi/lo tiles
      const int x = tid + NT * m, row = x >> 4, j = x & 15;
      const float4* pw = reinterpret_cast<const float4*>(sF + row * K + 8 * j);
      const float4* pk = reinterpret_cast<const float4*>(sF + CH * K + row * K + 8 * j);
      const float4 w0 = pw[0], w1 = pw[1], k0 = pk[0], k1 = pk[1];
      const float fw[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
      const float fk[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
      st_chunk_split(sm + O_WH, sm + O_WL, row, j, TT, fw);
      st_chunk_split(sm + O_KH, sm + O_KL, row, j, TT, fk);
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {  // W S_z^T
      constexpr uint32_t id = idesc_bf16(64, 64, false, false);
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const uint64_t wh = desc_kmajor(aWH, s, TT), sh = desc_kmajor(aSH, s, TT);
        mma_bf16(taddr(tb, 0, 0), wh, sh, id, s > 0);
        mma_bf16(taddr(tb, 0, 0), wh, desc_kmajor(aSL, s, TT), id, 1);
        mma_bf16(taddr(tb, 0, 0), desc_kmajor(aWL, s, TT), sh, id, 1);
      }
      mma_commit(&bar[0]);
    }
    // e^{Gam_C} for the state update (into shared memory once every thread is past the last
    // chunk's update) and U~ at this thread's (token, value) pairs of the M = 64, N = 64
    // accumulator, from the staging buffer
    const float egc = tid < K ? sF[3 * CH * 128 + tid] : 0.f;
    float ut[8];
    {
      const float* gU = sF + 2 * CH * 128 + v0;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int c = 16 * qt + 8 * j + cq;
        const float2 a0 = *reinterpret_cast<const float2*>(gU + r0 * V + c);
        const float2 a1 = *reinterpret_cast<const float2*>(gU + (r0 + 8) * V + c);
        ut[4 * j] = a0.x;
        ut[4 * j + 1] = a0.y;
        ut[4 * j + 2] = a1.x;
        ut[4 * j + 3] = a1.y;
      }
    }
    ok = __syncthreads_and(mbar_wait(&bar[0], ci & 1, err));
    tc_fence_after();
    if (tid < K) sE[tid] = egc;
    if (tid == 0 && ok && ci + 1 < sq.y) {  // every thread has read sF (the barrier above)
      fence_proxy_async();
      fetch(u + p.HV);
      pend = (ci + 1) & 1;
    }
    if (ok) {  // U = U~ - W S^T for this half's values: stored, and as a hi/lo tile [64 tok][64 v]
      float x[8];
      tmem_ld16dp_x2(taddr(tb, sub, 16 * qt), x);
      tmem_wait_ld();
      float* gU = w.U + u * CH * V + v0;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int c = 16 * qt + 8 * j + cq;
        const float u0 = ut[4 * j] - x[4 * j], u1 = ut[4 * j + 1] - x[4 * j + 1];
        const float u2 = ut[4 * j + 2] - x[4 * j + 2], u3 = ut[4 * j + 3] - x[4 * j + 3];
        *reinterpret_cast<float2*>(gU + r0 * V + c) = make_float2(u0, u1);
        *reinterpret_cast<float2*>(gU + (r0 + 8) * V + c) = make_float2(u2, u3);
        st_pair_split(sm + O_UH, sm + O_UL, r0, c, TT, u0, u1);
        st_pair_split(sm + O_UH, sm + O_UL, r0 + 8, c, TT, u2, u3);
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (ok && tid == 0) {  // U[:, z]^T K^
      constexpr uint32_t id = idesc_bf16(64, 128, true, true);
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const uint64_t uh = desc_mnmajor(aUH, s, TT), kh = desc_mnmajor(aKH, s, TT);
        mma_bf16(taddr(tb, 0, 128), uh, kh, id, s > 0);
        mma_bf16(taddr(tb, 0, 128), uh, desc_mnmajor(aKL, s, TT), id, 1);
        mma_bf16(taddr(tb, 0, 128), desc_mnmajor(aUL, s, TT), kh, id, 1);
      }
      mma_commit(&bar[1]);
    }
    ok = __syncthreads_and(ok && mbar_wait(&bar[1], ci & 1, err));
    tc_fence_after();
    if (ok) {  // S = S Diag(e^{Gam_C}) + U^T K^
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
  if (ok && a.ht) {
    float* ht = a.ht + ((size_t)n * p.HV + hv) * K * V;
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int r = v0 + r0 + 8 * (q >> 1), c = 32 * qt + 8 * j + cq + (q & 1);
        ht[(size_t)c * V + r] = S[4 * j + q];
      }
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && pend >= 0) mbar_wait(&bar[2], (uint32_t)pend, err);  // a copy still in flight lands
  if (warp == 0) tmem_dealloc(tb, 256);
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

// k_kda_out for bf16 with K = V = 128: O = scale (Q~ S^T + P U) on the tensor cores from
// compensated bf16 pairs, one CTA per (chunk, value head); M = 64 tokens, N = V, TMEM [0, 128).
namespace ko {
using namespace tcx;
constexpr int TT = 64 * 128, TS = 128 * 128;
constexpr int O_QH = 0, O_QL = 16384, O_SH = 32768, O_SL = 65536, O_PH = 98304, O_PL = 106496;
constexpr int O_UH = 114688, O_UL = 131072;
constexpr int OUT_BYTES = O_UL + 16384;
static_assert(1024 + OUT_BYTES <= 227 * 1024, "kda output shared memory");
}  // namespace ko

__global__ void __launch_bounds__(256, 1) k_kda_tc_out(Problem p, Args a, KdaWork w) {
  using namespace ko;
  if (kda_failed(w)) return;
  const int gc = blockIdx.x, hv = blockIdx.y;
  const int4 e = w.chunk_tab[gc];
  if (e.x < 0) return;
  constexpr int K = 128, V = 128;
  const int L = e.z, tok0 = e.w, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  extern __shared__ unsigned char smraw[];
  unsigned char* sm = align1k(smraw);
  __shared__ uint64_t bar[1];
  __shared__ uint32_t tslot;
  int* err = w.status;
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (warp == 0) {
    tmem_alloc(&tslot, 128);
    tmem_relinquish();
  }
  const size_t u = (size_t)gc * p.HV + hv;
  kt_split_rows<CH>(sm + O_QH, sm + O_QL, w.Qt + u * CH * K, sm + O_UH, sm + O_UL, w.U + u * CH * V);
  kt_split_rows<128>(sm + O_SH, sm + O_SL, w.h + u * V * K, nullptr, nullptr, nullptr);
  {  // P [64][64]
    float4 r[4];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int x = tid + 256 * m, row = x >> 3, j = x & 7;
      const float4* pp = reinterpret_cast<const float4*>(w.P + u * CH * CH + row * CH + 8 * j);
      r[2 * m] = __ldg(pp);
      r[2 * m + 1] = __ldg(pp + 1);
    }
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int x = tid + 256 * m, row = x >> 3, j = x & 7;
      const float f[8] = {r[2 * m].x, r[2 * m].y, r[2 * m].z, r[2 * m].w,
                          r[2 * m + 1].x, r[2 * m + 1].y, r[2 * m + 1].z, r[2 * m + 1].w};
      st_chunk_split(sm + O_PH, sm + O_PL, row, j, TT, f);
    }
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tslot;
  if (tid == 0) {
    const uint32_t qh = smem_u32(sm + O_QH), ql = smem_u32(sm + O_QL), sh = smem_u32(sm + O_SH);
    const uint32_t sl = smem_u32(sm + O_SL), ph = smem_u32(sm + O_PH), pl = smem_u32(sm + O_PL);
    const uint32_t uh = smem_u32(sm + O_UH), ul = smem_u32(sm + O_UL);
    constexpr uint32_t i_qs = idesc_bf16(64, 128, false, false), i_pu = idesc_bf16(64, 128, false, true);
#pragma unroll
    for (int s = 0; s < 8; ++s) {  // Q~ S^T
      const uint64_t aq = desc_kmajor(qh, s, TT), bs = desc_kmajor(sh, s, TS);
      mma_bf16(taddr(tb, 0, 0), aq, bs, i_qs, s > 0);
      mma_bf16(taddr(tb, 0, 0), aq, desc_kmajor(sl, s, TS), i_qs, 1);
      mma_bf16(taddr(tb, 0, 0), desc_kmajor(ql, s, TT), bs, i_qs, 1);
    }
#pragma unroll
    for (int s = 0; s < 4; ++s) {  // + P U
      const uint64_t ap = desc_kmajor(ph, s, TT), bu = desc_mnmajor(uh, s, TT);
      mma_bf16(taddr(tb, 0, 0), ap, bu, i_pu, 1);
      mma_bf16(taddr(tb, 0, 0), ap, desc_mnmajor(ul, s, TT), i_pu, 1);
      mma_bf16(taddr(tb, 0, 0), desc_kmajor(pl, s, TT), bu, i_pu, 1);
    }
    mma_commit(&bar[0]);
  }
  const bool ok = __syncthreads_and(mbar_wait(&bar[0], 0, err));
  tc_fence_after();
  if (ok) {
    const int half = warp >> 2, r0 = 16 * (warp & 3) + (lane >> 2), cq = 2 * (lane & 3);
    float x[32];
    tmem_ld16dp_x8(taddr(tb, 32 * (warp & 3), 64 * half), x);
    tmem_wait_ld();
    bf16* o = static_cast<bf16*>(a.o) + ((size_t)tok0 * p.HV + hv) * V;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = 64 * half + 8 * j + cq;
      if (r0 < L)
        *reinterpret_cast<uint32_t*>(o + (size_t)r0 * p.HV * V + c) = pack_bf16(p.scale * x[4 * j], p.scale * x[4 * j + 1]);
      if (r0 + 8 < L)
        *reinterpret_cast<uint32_t*>(o + (size_t)(r0 + 8) * p.HV * V + c) =
            pack_bf16(p.scale * x[4 * j + 2], p.scale * x[4 * j + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, 128);
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

template <typename T>
cudaError_t forward_t(const Problem& p, const Args& a, const KdaWork& w, cudaStream_t s) {
  const bool tc = std::is_same<T, __nv_bfloat16>::value && p.K == 128 && p.V == 128;
  cudaError_t e = tc ? go("kda_tc_wy", k_kda_tc_wy, dim3(p.NCmax, p.HV), 1024 + kf::WYF_BYTES, s, p, a, w, kf::NT)
                     : go("kda_wy", k_kda_wy<T>, dim3(p.NCmax, p.HV), wy_smem(p.K, p.V), s, p, a, w);
  if (e == cudaSuccess)
    e = tc ? go("kda_tc_scan", k_kda_tc_scan, dim3(p.Nst, p.HV, 2), 1024 + ks::SCAN_BYTES, s, p, a, w, ks::NT)
           : go("kda_scan", k_kda_scan, dim3(p.Nst, p.HV, p.V / 32), scan_smem(p.K), s, p, a, w);
  if (e == cudaSuccess)
    e = tc ? go("kda_tc_out", k_kda_tc_out, dim3(p.NCmax, p.HV), 1024 + ko::OUT_BYTES, s, p, a, w)
           : go("kda_out", k_kda_out<T>, dim3(p.NCmax, p.HV), out_smem(p.K, p.V), s, p, a, w);
  return e;
}

}  // namespace

cudaError_t kda_chunk_forward(const Problem& p, const Args& a, const KdaWork& w, bool bf16, cudaStream_t s) {
  return bf16 ? forward_t<__nv_bfloat16>(p, a, w, s) : forward_t<float>(p, a, w, s);
}

}  // namespace gdn
