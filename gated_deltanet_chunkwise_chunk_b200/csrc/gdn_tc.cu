// tcgen05 path for bf16 tensors with K = V = 128: chunk products on the 5th-generation tensor
// cores (operands in 128-byte-swizzled shared memory, fed by TMA; fp32 accumulators in TMEM).
//
// Per chunk (64 tokens) and value head, with S the state entering the chunk (V x K):
//   A  = strict_lower(diag(beta) (K K^T * Gam)),  T = (I + A)^-1          (CUDA cores, fp32)
//   W^T = K^T diag(beta e^G) T^T,   U~^T = V^T diag(beta) T^T              (tensor cores)
//   U^T = U~^T - S W^T;   S' = e^{G_C} S + (U^T diag(e^{G_C-G})) K         (sequential scan)
//   O   = scale (diag(e^G) Q S^T + (Q K^T * Gam) U)                        (chunk_fwd_o)
// Intermediates between kernels are bf16 tiles in HBM, laid out so that one TMA box loads
// each as a tensor-core operand:  W^T, U~^T, U^T: [unit][128][64];  S (h): [unit][128][128].
#include <cstdio>
#include <vector>

#include "gdn_tc_common.cuh"

namespace gdn {

using namespace tcx;

namespace {

// ======================================================================================
// WY representation.  One CTA (256 threads) per (chunk, value head).
//   KK^T (M=64) -> A, T = (I+A)^-1 (fp32, 16x16 blocks) ->
//   W^T = K^T (T diag(beta e^G))^T,  U~^T = V^T (T diag(beta))^T   (M=128, N=64, K=64)
// The fp32 A and the solve's scratch share shared memory with the bf16 T tiles written
// after the solve, so two CTAs fit on an SM.
// ======================================================================================
struct WySmem {
  static constexpr int K = 0, V = 2 * TILE64;
  static constexpr int R1 = 4 * TILE64;                  // {A, X} during the solve, then TX/TY
  static constexpr int TX = R1, TY = R1 + TILE64, TXL = R1 + 2 * TILE64, TYL = R1 + 3 * TILE64;
  static constexpr int A = R1, X = R1 + 64 * LDA * 4;    // fp32 [64][LDA] each
  static constexpr int T = R1 + 34 * 1024;              // fp32 [64][LDA]
  static constexpr int G = T + 64 * LDA * 4, B = G + 256, EG = B + 256, DEC = EG + 256;
  static constexpr int TOTAL = DEC + 256;
  static constexpr int NB1 = R1 + 2 * TILE128;           // second -N^T box (solve scratch)
  static_assert(NB1 + TILE128 <= G, "-N^T staging overlaps the per-token vectors");
};

__global__ void __launch_bounds__(256) k_tc_wy(Problem p, Work w, TcWork t,
                                               const __grid_constant__ CUtensorMap mk,
                                               const __grid_constant__ CUtensorMap mv,
                                               const __grid_constant__ CUtensorMap mWT,
                                               const __grid_constant__ CUtensorMap mUtT,
                                               const __grid_constant__ CUtensorMap mDK,
                                               const __grid_constant__ CUtensorMap mNT, int store_T,
                                               int gc0) {
  if (failed(w)) return;
  const int gc = gc0 + blockIdx.x, hv = blockIdx.y, hk = hv / p.G;
  const int4 e = w.chunk_tab[gc];
  if (e.x < 0) return;
  const int L = e.z, tok0 = e.w, tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int sub = 32 * (warp & 3), half = warp >> 2;
  extern __shared__ unsigned char smraw[];
  unsigned char* sm = align1k(smraw);
  unsigned char* sK = sm + WySmem::K;
  unsigned char* sV = sm + WySmem::V;
  unsigned char* sTX = sm + WySmem::TX;
  unsigned char* sTY = sm + WySmem::TY;
  unsigned char* sTXl = sm + WySmem::TXL;
  unsigned char* sTYl = sm + WySmem::TYL;
  float* sA = reinterpret_cast<float*>(sm + WySmem::A);
  float* sX = reinterpret_cast<float*>(sm + WySmem::X);
  float* sT = reinterpret_cast<float*>(sm + WySmem::T);
  float* sG = reinterpret_cast<float*>(sm + WySmem::G);
  float* sb = reinterpret_cast<float*>(sm + WySmem::B);
  float* sEG = reinterpret_cast<float*>(sm + WySmem::EG);   // beta_j e^{G_j}
  float* sDec = reinterpret_cast<float*>(sm + WySmem::DEC); // e^{G_C - G_j}, zero past the end
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
  if (tid == 0) {
    mbar_expect_tx(&bar[0], 4 * TILE64);
    tma_load_3d(sK, &mk, 0, hk, tok0, &bar[0]);
    tma_load_3d(sK + TILE64, &mk, 64, hk, tok0, &bar[0]);
    tma_load_3d(sV, &mv, 0, hv, tok0, &bar[0]);
    tma_load_3d(sV + TILE64, &mv, 64, hv, tok0, &bar[0]);
  }
  if (tid < 64) {
    const size_t o = ((size_t)hv * p.NCmax + gc) * 64 + tid;
    const float g = w.G[o], bb = w.beta_p[o];
    sG[tid] = g;
    sb[tid] = bb;
    sEG[tid] = bb * expf(g);
    sDec[tid] = tid < L ? w.Dec[o] : 0.f;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tslot;
  bool ok = __syncthreads_and(mbar_wait(&bar[0], 0, err));
  if (L < 64) {
    zero_tail_rows(sK, L, tid, 256);
    zero_tail_rows(sV, L, tid, 256);
  }
  fence_proxy_async();
  __syncthreads();
  // KK^T: M=64, N=64, K=128 (both K-major) -> TMEM cols [0,64)
  if (ok && tid == 0) {
    const uint32_t k = smem_u32(sK);
#pragma unroll
    for (int s = 0; s < 8; ++s)
      mma_bf16(taddr(tb, 0, 0), desc_kmajor(k, s, TILE64), desc_kmajor(k, s, TILE64),
               idesc_bf16(64, 64, false, false), s > 0);
    mma_commit(&bar[1]);
  }
  ok = __syncthreads_and(ok && mbar_wait(&bar[1], 0, err));
  tc_fence_after();
  if (ok) {
    // M=64 accumulator read with 16-lane loads: rows r0 = 16 (warp%4) + lane/4 and r0 + 8,
    // columns 32 half + 8j + 2 (lane%4) + {0,1}
    float v[16];
    tmem_ld16dp_x4(taddr(tb, sub, 32 * half), v);
    tmem_wait_ld();
    const int r0 = 16 * (warp & 3) + (lane >> 2);
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int r = r0 + 8 * (q >> 1), cc = 32 * half + 8 * j + 2 * (lane & 3) + (q & 1);
        sA[r * LDA + cc] = cc < r ? sb[r] * v[4 * j + q] * __expf(sG[r] - sG[cc]) : 0.f;
      }
  }
  __syncthreads();
  unit_lower_inverse64(sA, sT, sX, tid);   // T = (I + A)^-1 (ends with a barrier)
  // bf16 operand tiles TX[i][j] = T[i][j] beta_j e^{G_j}, TY[i][j] = T[i][j] beta_j (hi + lo)
  bf16* tbase = t.Tm + ((size_t)gc * p.HV + hv) * 128 * 64;
  for (int idx = tid; idx < 64 * 8; idx += 256) {
    const int i = idx / 8, jc = idx % 8;
    float fx[8], fy[8], ft[8], fl[8];
    for (int q = 0; q < 8; ++q) {
      const int j = jc * 8 + q;
      ft[q] = sT[i * LDA + j];
      fy[q] = ft[q] * sb[j];
      fx[q] = ft[q] * sEG[j];
      fl[q] = ft[q] - __bfloat162float(__float2bfloat16_rn(ft[q]));
    }
    st_chunk_split(sTX, sTXl, i, jc, TILE64, fx);
    st_chunk_split(sTY, sTYl, i, jc, TILE64, fy);
    if (store_T) {  // T as a compensated pair: rows [0,64) hi, [64,128) lo of the unit
      uint4 pk;
      pk.x = pack_bf16(ft[0], ft[1]);
      pk.y = pack_bf16(ft[2], ft[3]);
      pk.z = pack_bf16(ft[4], ft[5]);
      pk.w = pack_bf16(ft[6], ft[7]);
      *reinterpret_cast<uint4*>(tbase + i * 64 + jc * 8) = pk;
      pk.x = pack_bf16(fl[0], fl[1]);
      pk.y = pack_bf16(fl[2], fl[3]);
      pk.z = pack_bf16(fl[4], fl[5]);
      pk.w = pack_bf16(fl[6], fl[7]);
      *reinterpret_cast<uint4*>(tbase + (64 + i) * 64 + jc * 8) = pk;
    }
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // W^T = K^T TX^T, U~^T = V^T TY^T: M=128 (A MN-major), N=64, K=64 (B K-major)
  if (ok && tid == 0) {
    const uint32_t k = smem_u32(sK), vv = smem_u32(sV), tx = smem_u32(sTX), ty = smem_u32(sTY),
                   txl = smem_u32(sTXl), tyl = smem_u32(sTYl);
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      mma_bf16(taddr(tb, 0, 64), desc_mnmajor(k, s, TILE64), desc_kmajor(tx, s, TILE64),
               idesc_bf16(128, 64, true, false), s > 0);
      mma_bf16(taddr(tb, 0, 128), desc_mnmajor(vv, s, TILE64), desc_kmajor(ty, s, TILE64),
               idesc_bf16(128, 64, true, false), s > 0);
    }
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      mma_bf16(taddr(tb, 0, 64), desc_mnmajor(k, s, TILE64), desc_kmajor(txl, s, TILE64),
               idesc_bf16(128, 64, true, false), 1);
      mma_bf16(taddr(tb, 0, 128), desc_mnmajor(vv, s, TILE64), desc_kmajor(tyl, s, TILE64),
               idesc_bf16(128, 64, true, false), 1);
    }
    mma_commit(&bar[1]);
  }
  ok = __syncthreads_and(ok && mbar_wait(&bar[1], 1, err));
  tc_fence_after();
  if (ok) {
    // row = feature index (k for W^T, v for U~^T), this thread's 32 token columns; staged
    // as [128][64] bf16 tiles in the (now free) TX/TY region and stored by TMA
    const int r = sub + lane;
    unsigned char* sWst = sm + WySmem::R1;
    unsigned char* sUst = sWst + TILE128;
    float x[32], y[32];
    tmem_ld16(taddr(tb, sub, 64 + 32 * half), x);
    tmem_ld16(taddr(tb, sub, 64 + 32 * half + 16), x + 16);
    tmem_ld16(taddr(tb, sub, 128 + 32 * half), y);
    tmem_ld16(taddr(tb, sub, 128 + 32 * half + 16), y + 16);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      st_chunk_f(sWst, r, 4 * half + j, TILE128, x + 8 * j);
      st_chunk_f(sUst, r, 4 * half + j, TILE128, y + 8 * j);
    }
    // the products are done with K: it becomes D K (read by both sequential passes)
    for (int idx = tid; idx < 64 * 16; idx += 256) {
      const int rr = idx >> 4, jj = idx & 15;
      float f[8];
      ld_chunk_f(sK, rr, jj, TILE64, f);
      const float d = sDec[rr];
#pragma unroll
      for (int q = 0; q < 8; ++q) f[q] *= d;
      st_chunk_f(sK, rr, jj, TILE64, f);
    }
    fence_proxy_async();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int row = (gc * p.HV + hv) * D;
  if (ok && tid == 0) {
    tma_store_3d(&mWT, sm + WySmem::R1, 0, row, 0);
    tma_store_3d(&mUtT, sm + WySmem::R1 + TILE128, 0, row, 0);
    tma_store_3d(&mDK, sK, 0, (gc * p.HV + hv) * 64, 0);
    tma_store_3d(&mDK, sK + TILE64, 64, (gc * p.HV + hv) * 64, 0);
    tma_store_commit();
    // N^T = (D K)^T W, the state-free factor of the chunk's affine state map (M=128 k',
    // N=128 k, K=64 i; A = D K MN-major, B = W^T K-major), into TMEM columns [128, 256)
    const uint64_t dk = desc_mnmajor(smem_u32(sK), 0, TILE64);
    const uint64_t dw = desc_kmajor(smem_u32(sm + WySmem::R1), 0, TILE128);
#pragma unroll
    for (int s = 0; s < 4; ++s)
      mma_bf16(taddr(tb, 0, 128), dk + mnstep_off(s), dw + kstep_off(s, TILE128),
               idesc_bf16(128, 128, true, false), s > 0);
    mma_commit(&bar[1]);
  }
  ok = __syncthreads_and(ok && mbar_wait(&bar[1], 0, err));
  tc_fence_after();
  if (ok) {
    // -N^T as a bf16 [128 k'][128 k] K-major tile (two 64-column boxes: V's space and a free
    // part of the solve's scratch), the A operand of both sequential passes' chain products
    const int r = sub + lane;
    unsigned char* sNst = sm + (half ? WySmem::NB1 : WySmem::V);
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      float x[32];
      tmem_ld16(taddr(tb, sub, 128 + 64 * half + 32 * part), x);
      tmem_ld16(taddr(tb, sub, 128 + 64 * half + 32 * part + 16), x + 16);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 32; ++q) x[q] = -x[q];
#pragma unroll
      for (int j = 0; j < 4; ++j) st_chunk_f(sNst, r, 4 * part + j, TILE128, x + 8 * j);
    }
    fence_proxy_async();
  }
  __syncthreads();
  if (tid == 0) {
    if (ok) {
      tma_store_3d(&mNT, sm + WySmem::V, 0, row, 0);
      tma_store_3d(&mNT, sm + WySmem::NB1, 64, row, 0);
      tma_store_commit();
    }
    tma_store_wait_read0();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, 256);
}

// ======================================================================================
// chunk_fwd_o.  One CTA (256 threads) per (chunk, value head), S the state entering the chunk:
//   X = Q S^T (M=64, N=128), QK = Q K^T (M=64, N=64), Uc = S W^T (M=128 v, N=64 i)
//   U^T = U~^T - Uc (v_new; also stored for the backward), P = QK * Gam (bf16 hi/lo tile)
//   Y = P U (M=64, N=128, B = U^T K-major);  O = scale (e^{G_i} X + Y)
// With o = NULL (the backward's recompute) only U^T is produced.
// ======================================================================================
__global__ void __launch_bounds__(256) k_tc_out(Problem p, Args a, Work w, TcWork t,
                                                const __grid_constant__ CUtensorMap mq,
                                                const __grid_constant__ CUtensorMap mk,
                                                const __grid_constant__ CUtensorMap mUtT,
                                                const __grid_constant__ CUtensorMap mWT,
                                                const __grid_constant__ CUtensorMap mUT,
                                                const __grid_constant__ CUtensorMap mh, int gc0) {
  if (failed(w)) return;
  const int gc = gc0 + blockIdx.x, hv = blockIdx.y, hk = hv / p.G;
  const int4 e = w.chunk_tab[gc];
  if (e.x < 0) return;
  const int L = e.z, tok0 = e.w, tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  extern __shared__ unsigned char smraw[];
  unsigned char* sm = align1k(smraw);
  unsigned char* sQ = sm;                    // [64][128]
  unsigned char* sK = sQ + 2 * TILE64;       // [64][128]
  unsigned char* sH = sK + 2 * TILE64;       // S^T [128 k][128 v]
  unsigned char* sU = sH + 2 * TILE128;      // U~^T [128][64], then U^T in place
  unsigned char* sW = sU + TILE128;          // W^T [128][64]
  // P (hi, lo [64][64] each) is written once the first products have read K: it takes K's
  // place, so that two CTAs fit on an SM
  unsigned char* sP = sK;
  unsigned char* sPl = sK + TILE64;
  float* sG = reinterpret_cast<float*>(sW + TILE128);
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
  const int row = (gc * p.HV + hv) * D;
  if (tid == 0) {
    mbar_expect_tx(&bar[0], 4 * TILE64 + 4 * TILE128);
    tma_load_3d(sQ, &mq, 0, hk, tok0, &bar[0]);
    tma_load_3d(sQ + TILE64, &mq, 64, hk, tok0, &bar[0]);
    tma_load_3d(sK, &mk, 0, hk, tok0, &bar[0]);
    tma_load_3d(sK + TILE64, &mk, 64, hk, tok0, &bar[0]);
    tma_load_3d(sH, &mh, 0, row, 0, &bar[0]);
    tma_load_3d(sH + TILE128, &mh, 64, row, 0, &bar[0]);
    tma_load_3d(sU, &mUtT, 0, row, 0, &bar[0]);
    tma_load_3d(sW, &mWT, 0, row, 0, &bar[0]);
  }
  if (tid < 64) sG[tid] = w.G[((size_t)hv * p.NCmax + gc) * 64 + tid];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tslot;
  bool ok = __syncthreads_and(mbar_wait(&bar[0], 0, err));
  if (ok && tid == 0) {
    const uint32_t q = smem_u32(sQ), k = smem_u32(sK), h = smem_u32(sH), wt = smem_u32(sW);
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      // S is stored transposed ([k][v]): an MN-major B operand here, an MN-major A below
      mma_bf16(taddr(tb, 0, 0), desc_kmajor(q, s, TILE64), desc_mnmajor(h, s, TILE128),
               idesc_bf16(64, 128, false, true), s > 0);
      mma_bf16(taddr(tb, 0, 128), desc_kmajor(q, s, TILE64), desc_kmajor(k, s, TILE64),
               idesc_bf16(64, 64, false, false), s > 0);
      mma_bf16(taddr(tb, 0, 192), desc_mnmajor(h, s, TILE128), desc_mnmajor(wt, s, TILE128),
               idesc_bf16(128, 64, true, true), s > 0);
    }
    mma_commit(&bar[1]);
  }
  ok = __syncthreads_and(ok && mbar_wait(&bar[1], 0, err));
  tc_fence_after();
  // M=64 accumulators read with 16-lane loads: rows r0 = 16 (warp%4) + lane/4 and r0 + 8,
  // this warp half's columns 8j + 2(lane%4) + {0,1}
  const int half = warp >> 2, r0 = 16 * (warp & 3) + (lane >> 2), cq = 2 * (lane & 3);
  const float g0 = sG[r0], g1 = sG[r0 + 8];
  if (ok) {  // P = QK * Gam (lower incl. diagonal), columns [32 half, +32), as a hi/lo pair
    float d[16];
    tmem_ld16dp_x4(taddr(tb, 32 * (warp & 3), 128 + 32 * half), d);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = 32 * half + 8 * j + cq;
      float f[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = r0 + 8 * (q >> 1), col = c + (q & 1);
        f[q] = col <= i ? d[4 * j + q] * __expf((q < 2 ? g0 : g1) - sG[col]) : 0.f;
      }
      st_pair_split(sP, sPl, r0, c, TILE64, f[0], f[1]);
      st_pair_split(sP, sPl, r0 + 8, c, TILE64, f[2], f[3]);
    }
    // U^T = U~^T - S W^T (M=128 accumulator: lane = value row v), columns [32 half, +32), in place
    float x[32];
    const int v = 32 * (warp & 3) + lane;
    tmem_ld16(taddr(tb, 32 * (warp & 3), 192 + 32 * half), x);
    tmem_ld16(taddr(tb, 32 * (warp & 3), 192 + 32 * half + 16), x + 16);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float f[8];
      ld_chunk_f(sU, v, 4 * half + j, TILE128, f);
#pragma unroll
      for (int q = 0; q < 8; ++q) f[q] -= x[8 * j + q];
      st_chunk_f(sU, v, 4 * half + j, TILE128, f);
    }
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (ok && tid == 0) {
    tma_store_3d(&mUT, sU, 0, row, 0);  // v_new for the backward
    tma_store_commit();
    const uint32_t pp = smem_u32(sP), pl = smem_u32(sPl), u = smem_u32(sU);
#pragma unroll
    for (int s = 0; s < 4; ++s)
      mma_bf16(taddr(tb, 0, 128), desc_kmajor(pp, s, TILE64), desc_kmajor(u, s, TILE128),
               idesc_bf16(64, 128, false, false), s > 0);
#pragma unroll
    for (int s = 0; s < 4; ++s)
      mma_bf16(taddr(tb, 0, 128), desc_kmajor(pl, s, TILE64), desc_kmajor(u, s, TILE128),
               idesc_bf16(64, 128, false, false), 1);
    mma_commit(&bar[1]);
  }
  ok = __syncthreads_and(ok && mbar_wait(&bar[1], 1, err));
  tc_fence_after();
  if (ok && a.o) {  // O = scale (e^{G_i} X + Y), columns [64 half, +64)
    float x[32], y[32];
    tmem_ld16dp_x8(taddr(tb, 32 * (warp & 3), 64 * half), x);
    tmem_ld16dp_x8(taddr(tb, 32 * (warp & 3), 128 + 64 * half), y);
    tmem_wait_ld();
    const float e0 = __expf(g0) * p.scale, e1 = __expf(g1) * p.scale;
    bf16* o0 = static_cast<bf16*>(a.o) + ((size_t)(tok0 + r0) * p.HV + hv) * p.V + 64 * half + cq;
    bf16* o1 = o0 + (size_t)8 * p.HV * p.V;
    const bool live = 64 * half < p.V;  // columns past a 64-wide value head are padding
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (live && r0 < L)
        *reinterpret_cast<uint32_t*>(o0 + 8 * j) =
            pack_bf16(e0 * x[4 * j] + p.scale * y[4 * j], e0 * x[4 * j + 1] + p.scale * y[4 * j + 1]);
      if (live && r0 + 8 < L)
        *reinterpret_cast<uint32_t*>(o1 + 8 * j) =
            pack_bf16(e1 * x[4 * j + 2] + p.scale * y[4 * j + 2], e1 * x[4 * j + 3] + p.scale * y[4 * j + 3]);
    }
  }
  if (tid == 0) tma_store_wait0();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, 256);
}

// ------------------------------------------------------------------ host side
struct Launch {
  TcMaps m;
  TcWork t;
  bool ok = true;
};

Launch setup(const Problem& p, const Args& a, void* tc_ws, int pass) {
  Launch L;
  const int ntok = p.B * p.T;
  L.t = carve_tc(tc_ws, (size_t)p.NCmax, (size_t)p.HV, pass);
  const uint64_t urows = (uint64_t)p.NCmax * p.HV * D;
  L.ok &= map_tokens(&L.m.q, a.q, ntok, p.H, p.K);
  L.ok &= map_tokens(&L.m.k, a.k, ntok, p.H, p.K);
  L.ok &= map_tokens(&L.m.v, a.v, ntok, p.HV, p.V);
  if (a.dO) L.ok &= map_tokens(&L.m.dO, a.dO, ntok, p.HV, p.V);
  L.ok &= map_rows(&L.m.WT, L.t.WT, urows, 64, 128);
  L.ok &= map_rows(&L.m.UtT, L.t.UtT, urows, 64, 128);
  L.ok &= map_rows(&L.m.UT, L.t.UT, urows, 64, 128);
  L.ok &= map_rows(&L.m.h, L.t.h, urows, 128, 128);
  L.ok &= map_rows(&L.m.DK, L.t.DK, (uint64_t)p.NCmax * p.HV * 64, 128, 64);
  L.ok &= map_rows(&L.m.NT, L.t.NT, urows, 128, 128);
  if (pass == 1) {
    const uint64_t trows = (uint64_t)p.NCmax * p.HV * 64;
    L.ok &= map_rows(&L.m.dUlT, L.t.dUlT, urows, 64, 128);
    L.ok &= map_rows(&L.m.dUT, L.t.dUT, urows, 64, 128);
    L.ok &= map_rows(&L.m.dUTl, L.t.dUTl, urows, 64, 128);
    L.ok &= map_rows(&L.m.dh, L.t.dh, urows, 128, 128);
    L.ok &= map_rows(&L.m.dW, L.t.dW, trows, 128, 64);
    L.ok &= map_rows(&L.m.Op, L.t.Op, trows, 128, 64);
    L.ok &= map_rows(&L.m.Tm, L.t.Tm, 2 * trows, 64, 64);
  }
  return L;
}

cudaError_t forward_impl(const Problem& p, const Args& a, const Work& w, const Launch& L,
                         bool bwd_prep, cudaStream_t s) {
  if (!L.ok) return cudaErrorInvalidValue;
  const size_t out_smem = 1024 + 4 * TILE64 + 4 * TILE128 + 256;
  Args ao = a;
  if (bwd_prep) ao.o = nullptr;  // the backward's recompute only needs v_new from the output kernel
  auto wy = [&](int c0, int c1, cudaStream_t st) {
    return tgo("tc_wy", k_tc_wy, dim3(c1 - c0, p.HV), 256, (size_t)1024 + WySmem::TOTAL, st, p, w,
               L.t, L.m.k, L.m.v, L.m.WT, L.m.UtT, L.m.DK, L.m.NT, 1, c0);
  };
  auto out = [&](int c0, int c1, cudaStream_t st) {
    return tgo("tc_out", k_tc_out, dim3(c1 - c0, p.HV), 256, out_smem, st, p, ao, w, L.t, L.m.q,
               L.m.k, L.m.UtT, L.m.WT, L.m.UT, L.m.h, c0);
  };
  float* ht = bwd_prep ? nullptr : a.ht;
  const Segments sg = segments(p, kFwdSeg);
  cudaError_t e;
  if (sg.n == 1) {
    if ((e = wy(0, p.NCmax, s))) return e;
    if ((e = tc_scan_fwd(p, a, w, L.t, L.m, ScanRange{0, p.NCmax, a.h0, ht}, s))) return e;
    return out(0, p.NCmax, s);
  }
  // Segments of the sequence's chunks: the pass over segment i (on the side stream) runs
  // while the WY kernels of later segments and the outputs of earlier ones run on `s`.
  SideLock side;
  if (!side.ok()) return cudaErrorInvalidResourceHandle;
  cudaStream_t hs = side.stream();
  if ((e = side.fork(s))) return e;
  std::vector<cudaEvent_t> wy_done(sg.n), scan_done(sg.n);
  for (int i = 0; i < sg.n; ++i) {
    if ((e = wy(sg.c[i], sg.c[i + 1], s))) return e;
    if ((e = side.record(s, &wy_done[i]))) return e;
  }
  for (int i = 0; i < sg.n; ++i) {
    if ((e = cudaStreamWaitEvent(hs, wy_done[i], 0))) return e;
    const ScanRange r{sg.c[i], sg.c[i + 1], i == 0 ? a.h0 : L.t.hand,
                      i + 1 == sg.n ? ht : L.t.hand};
    if ((e = tc_scan_fwd(p, a, w, L.t, L.m, r, hs))) return e;
    if ((e = side.record(hs, &scan_done[i]))) return e;
  }
  for (int i = 0; i < sg.n; ++i) {
    if ((e = cudaStreamWaitEvent(s, scan_done[i], 0))) return e;
    if ((e = out(sg.c[i], sg.c[i + 1], s))) return e;
  }
  return cudaSuccess;
}

}  // namespace

bool tc_supported(const gdn_dims& d) {
  // 64-wide heads run on the same 128-wide tiles: their token maps are 64 columns wide, so the
  // second 64-column box of every token tile reads as zeros and adds nothing to any product
  return d.dtype == GDN_DTYPE_BF16 && (d.K == 64 || d.K == 128) && (d.V == 64 || d.V == 128) &&
         d.B * d.T > 0;
}

bool tc_bwd_supported(const gdn_dims& d) { return tc_supported(d); }

bool tc_ready() { return encoder() != nullptr; }

size_t tc_workspace_bytes(const gdn_dims& d, size_t NC, int pass) {
  return tc_bytes(NC, (size_t)d.HV, pass);
}

cudaError_t tc_forward(const Problem& p, const Args& a, const Work& w, void* tc_ws, cudaStream_t s) {
  Launch L = setup(p, a, tc_ws, 0);
  return forward_impl(p, a, w, L, false, s);
}

cudaError_t tc_backward(const Problem& p, const Args& a, const Work& w, void* tc_ws, bool reuse_fwd,
                        cudaStream_t s) {
  Launch L = setup(p, a, tc_ws, 1);
  cudaError_t e = cudaSuccess;
  if (!reuse_fwd && (e = forward_impl(p, a, w, L, true, s)) != cudaSuccess) return e;
  if (!L.ok) return cudaErrorInvalidValue;
  if ((e = tc_backward_kernels(p, a, w, L.t, L.m, s)) != cudaSuccess) return e;
  return launch_bwd_tokens(p, a, w, true, s, false);  // dqkwg and wy_bwd write dq, dk
}

}  // namespace gdn
