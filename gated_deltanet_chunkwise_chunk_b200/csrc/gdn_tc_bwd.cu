// tcgen05 backward kernels (bf16, K = V = 128; the reverse state pass is in gdn_tc_scan.cu).  Per chunk (64 tokens) and value head, with
// S the state entering the chunk, dS' = dL/dS leaving it, P = (Q K^T) * Gam (lower incl.
// diagonal), D_j = e^{G_C - G_j}:
//   dv_local  dU_loc = scale P^T dO
//   scan      dU = dU_loc + diag(D) K dS'^T;  dS = e^{G_C} dS' + scale (diag(e^G) dO)^T Q - dU^T W
//   dqkwg     dP = scale dO U^T (masked);  dQ = scale diag(e^G) dO S + (dP*Gam) K;
//             dK = (dP*Gam)^T Q + diag(D) U dS';  dW = -dU S;  dG terms
//   wy_bwd    dT = dU Y^T + dW X^T;  dX = T^T dW;  dY = T^T dU;  dA = -(T^T dT T^T) strict lower;
//             dv = beta dY;  dbeta;  dk += diag(beta e^G) dX + dAs K + dAs^T K;  dG terms
// (X = diag(beta e^G) K, Y = diag(beta) V, dAs = dA * Gam * beta_i).  Column sums go through
// shared memory in a fixed order, so results are bitwise reproducible.
#include <vector>

#include "gdn_tc_common.cuh"

namespace gdn {
namespace tcx {

namespace {

__device__ __forceinline__ float warp_sum(float x) {
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// ======================================================================================
// dv_local: dU_loc^T = scale dO^T P  (M=128 v, N=64 j, K=64 i), after QK^T (M=64).  P takes
// K's place once QK^T has read it, and dU_loc^T K's place again once P has been read, so that
// four CTAs fit on an SM; both outputs leave by bulk stores.
// ======================================================================================
__global__ void __launch_bounds__(128) k_tc_dvlocal(Problem p, Work w, TcWork t,
                                                    const __grid_constant__ CUtensorMap mq,
                                                    const __grid_constant__ CUtensorMap mk,
                                                    const __grid_constant__ CUtensorMap mdO,
                                                    const __grid_constant__ CUtensorMap mOp,
                                                    const __grid_constant__ CUtensorMap mdUlT, int gc0) {
  if (failed(w)) return;
  const int gc = gc0 + blockIdx.x, hv = blockIdx.y, hk = hv / p.G;
  const int4 e = w.chunk_tab[gc];
  if (e.x < 0) return;
  const int L = e.z, tok0 = e.w, tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  extern __shared__ unsigned char smraw[];
  unsigned char* sm = align1k(smraw);
  unsigned char* sQ = sm;
  unsigned char* sK = sQ + 2 * TILE64;
  unsigned char* sO = sK + 2 * TILE64;
  unsigned char* sP = sK;                   // P hi, then dU_loc^T [128][64] over both halves
  unsigned char* sPl = sK + TILE64;         // P lo
  float* sG = reinterpret_cast<float*>(sO + 2 * TILE64);
  float* sEo = sG + 64;                     // -scale e^{G_i}, zero past the chunk end
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
    tmem_alloc(&tslot, 128);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_expect_tx(&bar[0], 6 * TILE64);
    tma_load_3d(sQ, &mq, 0, hk, tok0, &bar[0]);
    tma_load_3d(sQ + TILE64, &mq, 64, hk, tok0, &bar[0]);
    tma_load_3d(sK, &mk, 0, hk, tok0, &bar[0]);
    tma_load_3d(sK + TILE64, &mk, 64, hk, tok0, &bar[0]);
    tma_load_3d(sO, &mdO, 0, hv, tok0, &bar[0]);
    tma_load_3d(sO + TILE64, &mdO, 64, hv, tok0, &bar[0]);
  }
  if (tid < 64) {
    const size_t o = ((size_t)hv * p.NCmax + gc) * 64 + tid;
    sG[tid] = w.G[o];
    sEo[tid] = tid < L ? -p.scale * w.EG[o] : 0.f;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tslot;
  bool ok = __syncthreads_and(mbar_wait(&bar[0], 0, err));
  if (ok && tid == 0) {
    const uint32_t q = smem_u32(sQ), k = smem_u32(sK);
#pragma unroll
    for (int s = 0; s < 8; ++s)
      mma_bf16(taddr(tb, 0, 0), desc_kmajor(q, s, TILE64), desc_kmajor(k, s, TILE64),
               idesc_bf16(64, 64, false, false), s > 0);
    mma_commit(&bar[1]);
  }
  ok = __syncthreads_and(ok && mbar_wait(&bar[1], 0, err));
  tc_fence_after();
  if (ok) {
    // M=64 accumulator with 16-lane loads: rows r0 = 16 warp + lane/4 and r0 + 8,
    // columns 8j + 2(lane%4) + {0,1}
    float d[32];
    tmem_ld16dp_x8(taddr(tb, 32 * warp, 0), d);
    tmem_wait_ld();
    const int r0 = 16 * warp + (lane >> 2), cq = 2 * (lane & 3);
    const float g0 = sG[r0], g1 = sG[r0 + 8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = 8 * j + cq;
      float f[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = r0 + 8 * (q >> 1), col = c + (q & 1);
        f[q] = (col <= i && i < L) ? d[4 * j + q] * __expf((q < 2 ? g0 : g1) - sG[col]) : 0.f;
      }
      st_pair_split(sP, sPl, r0, c, TILE64, f[0], f[1]);
      st_pair_split(sP, sPl, r0 + 8, c, TILE64, f[2], f[3]);
    }
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (ok && tid == 0) {
    const uint32_t o = smem_u32(sO), pp = smem_u32(sP), pl = smem_u32(sPl);
#pragma unroll
    for (int s = 0; s < 4; ++s)
      mma_bf16(taddr(tb, 0, 64), desc_mnmajor(o, s, TILE64), desc_mnmajor(pp, s, TILE64),
               idesc_bf16(128, 64, true, true), s > 0);
#pragma unroll
    for (int s = 0; s < 4; ++s)
      mma_bf16(taddr(tb, 0, 64), desc_mnmajor(o, s, TILE64), desc_mnmajor(pl, s, TILE64),
               idesc_bf16(128, 64, true, true), 1);
    mma_commit(&bar[1]);
  }
  ok = __syncthreads_and(ok && mbar_wait(&bar[1], 1, err));
  tc_fence_after();
  if (ok) {  // dU_loc^T row v (TMEM lane), staged as a [128][64] tile where P was
    const int v = 32 * warp + lane;
#pragma unroll
    for (int c = 0; c < 64; c += 16) {
      float d[16];
      tmem_ld16(taddr(tb, 32 * warp, 64 + c), d);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 16; ++q) d[q] *= p.scale;
      st_chunk_f(sP, v, c / 8, TILE128, d);
      st_chunk_f(sP, v, c / 8 + 1, TILE128, d + 8);
    }
    // the products are done with dO: it becomes O' = -scale e^G dO for the reverse pass
    for (int idx = tid; idx < 64 * 16; idx += 128) {
      const int r = idx >> 4, j = idx & 15;
      float f[8];
      ld_chunk_f(sO, r, j, TILE64, f);
      const float sc = sEo[r];
#pragma unroll
      for (int q = 0; q < 8; ++q) f[q] *= sc;
      st_chunk_f(sO, r, j, TILE64, f);
    }
    fence_proxy_async();
  }
  __syncthreads();
  if (ok && tid == 0) {
    const int orow = (gc * p.HV + hv) * 64;
    tma_store_3d(&mOp, sO, 0, orow, 0);
    tma_store_3d(&mOp, sO + TILE64, 64, orow, 0);
    tma_store_3d(&mdUlT, sP, 0, (gc * p.HV + hv) * D, 0);
    tma_store_commit();
    tma_store_wait_read0();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, 128);
}

// ======================================================================================
// dqkwg.  One CTA (256 threads) per (chunk, value head).  TMEM columns:
//   [0,64) Q K^T   [64,128) dO U^T   [128,256) dO S -> dQ   [256,384) U dS' -> dK   [384,512) dU S
// M=64 accumulators are read with 16-lane loads: warp w covers rows 16(w%4) .. +15, thread t
// rows r0 = 16(w%4) + t/4 and r0 + 8, and the two warps of a sub-partition split columns.
// ======================================================================================
struct DqkSmem {
  static constexpr int Q = 0, K = 2 * TILE64, O = 4 * TILE64, UT = 6 * TILE64,
                       DUT = 6 * TILE64 + TILE128, H = 6 * TILE64 + 2 * TILE128,
                       DH = 6 * TILE64 + 4 * TILE128, PG = 6 * TILE64 + 6 * TILE128,
                       PGL = PG + TILE64, DUTL = PGL + TILE64,
                       M = DUTL + TILE128;                   // fp32 [64][65] dP*P
  static constexpr int G = M + 64 * 65 * 4;
  static constexpr int ROW = G + 256;                        // [3][2][64] per-row partials
  static constexpr int RED = ROW + 3 * 2 * 64 * 4;           // [8]
  static constexpr int TOTAL = RED + 64;
};

__global__ void __launch_bounds__(256) k_tc_dqkwg(Problem p, Args a, Work w, TcWork t,
                                                  const __grid_constant__ CUtensorMap mq,
                                                  const __grid_constant__ CUtensorMap mk,
                                                  const __grid_constant__ CUtensorMap mdO,
                                                  const __grid_constant__ CUtensorMap mUT,
                                                  const __grid_constant__ CUtensorMap mdUT,
                                                  const __grid_constant__ CUtensorMap mdUTl,
                                                  const __grid_constant__ CUtensorMap mh,
                                                  const __grid_constant__ CUtensorMap mdh,
                                                  const __grid_constant__ CUtensorMap mdW,
                                                  UnitRange ur) {
  if (failed(w)) return;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int half = warp >> 2, sub = 32 * (warp & 3);
  const int r0 = 16 * (warp & 3) + lane / 4, r1 = r0 + 8, cq = 2 * (lane & 3);
  extern __shared__ unsigned char smraw[];
  unsigned char* sm = align1k(smraw);
  unsigned char* sQ = sm + DqkSmem::Q;
  unsigned char* sK = sm + DqkSmem::K;
  unsigned char* sO = sm + DqkSmem::O;
  unsigned char* sUT = sm + DqkSmem::UT;     // later: dW staging [64][128]
  unsigned char* sdUT = sm + DqkSmem::DUT;
  unsigned char* sH = sm + DqkSmem::H;
  unsigned char* sdH = sm + DqkSmem::DH;
  unsigned char* sPG = sm + DqkSmem::PG;
  unsigned char* sPGl = sm + DqkSmem::PGL;
  unsigned char* sdUTl = sm + DqkSmem::DUTL;
  float* sM = reinterpret_cast<float*>(sm + DqkSmem::M);
  float* sG = reinterpret_cast<float*>(sm + DqkSmem::G);
  float* sRow = reinterpret_cast<float*>(sm + DqkSmem::ROW);  // [kind][half][64]
  float* sRed = reinterpret_cast<float*>(sm + DqkSmem::RED);
  // barA: Q, K, U^T of a unit;  barB: dO, dU^T (hi, lo), S, dS';  barM: MMA batches
  __shared__ uint64_t barA, barB, barM;
  __shared__ uint32_t tslot;
  int* err = w.status;
  if (tid == 0) {
    mbar_init(&barA, 1);
    mbar_init(&barB, 1);
    mbar_init(&barM, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (warp == 0) {
    tmem_alloc(&tslot, 512);
    tmem_relinquish();
  }
  // Units u = chunk * HV + hv in [u0, u1), handed out in k-head groups (chunk, hk) by an atomic
  // counter: a CTA runs the G value heads of a group back to back (their dq and dk shares go
  // to the k-head's fp32 tiles in a fixed order).  Thread 0 takes the next unit a unit ahead;
  // -1 marks the end of the work (past the range, or a chunk-table entry past the chunk count).
  auto next_of = [&](int u) {
    if (u >= 0 && (u % p.HV) % p.G + 1 < p.G) return u + 1;
    const int kk = ur.u0 / p.G + atomicAdd(ur.ctr, 1);
    if (kk >= ur.u1 / p.G) return -1;
    const int gc = kk / p.H;
    return w.chunk_tab[gc].x >= 0 ? gc * p.HV + (kk % p.H) * p.G : -1;
  };
  auto valid = [](int u) { return u >= 0; };
  auto load_A = [&](int u) {
    const int gc = u / p.HV, hk = (u % p.HV) / p.G, tok0 = w.chunk_tab[gc].w;
    mbar_expect_tx(&barA, 4 * TILE64 + TILE128);
    tma_load_3d(sQ, &mq, 0, hk, tok0, &barA);
    tma_load_3d(sQ + TILE64, &mq, 64, hk, tok0, &barA);
    tma_load_3d(sK, &mk, 0, hk, tok0, &barA);
    tma_load_3d(sK + TILE64, &mk, 64, hk, tok0, &barA);
    tma_load_3d(sUT, &mUT, 0, u * D, 0, &barA);
  };
  auto load_B = [&](int u) {
    const int gc = u / p.HV, hv = u % p.HV, tok0 = w.chunk_tab[gc].w;
    mbar_expect_tx(&barB, 2 * TILE64 + 6 * TILE128);
    tma_load_3d(sO, &mdO, 0, hv, tok0, &barB);
    tma_load_3d(sO + TILE64, &mdO, 64, hv, tok0, &barB);
    tma_load_3d(sdUT, &mdUT, 0, u * D, 0, &barB);
    tma_load_3d(sdUTl, &mdUTl, 0, u * D, 0, &barB);
    tma_load_3d(sH, &mh, 0, u * D, 0, &barB);
    tma_load_3d(sH + TILE128, &mh, 64, u * D, 0, &barB);
    tma_load_3d(sdH, &mdh, 0, u * D, 0, &barB);
    tma_load_3d(sdH + TILE128, &mdh, 64, u * D, 0, &barB);
  };
  // units are handed out in order by an atomic counter (a CTA that starts late, behind other
  // work on its SM, simply takes fewer); thread 0 takes the next one a unit ahead
  __shared__ int s_unit[2];
  int u = -1;
  if (tid == 0) {
    u = next_of(-1);
    s_unit[0] = u;
  }
  // parity of a load group issued and not yet waited on, or -1 (thread 0 issues all loads)
  int pendA = -1, pendB = -1;
  if (tid == 0 && valid(u)) {
    load_A(u);
    load_B(u);
    pendA = pendB = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  u = s_unit[0];
  const uint32_t tb = tslot;
  bool ok = true;
  int nu = -1;
  // the unit's in-chunk gate sums, read into a register a unit ahead (their load latency
  // then overlaps the previous unit instead of stalling this one)
  auto g_of = [&](int uu) {
    return (tid < 64 && valid(uu)) ? w.G[((size_t)(uu % p.HV) * p.NCmax + uu / p.HV) * 64 + tid] : 0.f;
  };
  float g_next = g_of(u);
  for (uint32_t it = 0; valid(u); ++it, u = nu) {
    const int gc = u / p.HV, hv = u % p.HV;
    const int4 e = w.chunk_tab[gc];
    const int L = e.z;
    const size_t unit = (size_t)u;
    if (tid == 0) s_unit[(it + 1) & 1] = next_of(u);
    const uint32_t ph = it & 1;
    if (tid < 64) sG[tid] = g_next;
    const bool got = mbar_wait(&barA, ph, err) && mbar_wait(&barB, ph, err);
    if (tid == 0) pendA = pendB = got ? -1 : (int)ph;
    ok = __syncthreads_and(ok && got);
    if (!ok) break;
    nu = s_unit[(it + 1) & 1];
    const bool nvalid = valid(nu);
    if (L < 64) {
      zero_tail_rows(sQ, L, tid, 256);
      zero_tail_rows(sK, L, tid, 256);
      zero_tail_rows(sO, L, tid, 256);
    }
    fence_proxy_async();
    __syncthreads();
    g_next = g_of(nu);  // after the barrier: its latency hides behind this unit's products
    if (tid == 0) {
      const uint32_t q = smem_u32(sQ), k = smem_u32(sK), o = smem_u32(sO), ut = smem_u32(sUT),
                     dut = smem_u32(sdUT), dutl = smem_u32(sdUTl), h = smem_u32(sH), dh = smem_u32(sdH);
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const uint32_t acc = s > 0;
        mma_bf16(taddr(tb, 0, 0), desc_kmajor(q, s, TILE64), desc_kmajor(k, s, TILE64),
                 idesc_bf16(64, 64, false, false), acc);
        mma_bf16(taddr(tb, 0, 64), desc_kmajor(o, s, TILE64), desc_mnmajor(ut, s, TILE128),
                 idesc_bf16(64, 64, false, true), acc);
        // S and dS' tiles are stored transposed ([k][v]): K-major B operands here
        mma_bf16(taddr(tb, 0, 128), desc_kmajor(o, s, TILE64), desc_kmajor(h, s, TILE128),
                 idesc_bf16(64, 128, false, false), acc);
        mma_bf16(taddr(tb, 0, 256), desc_mnmajor(ut, s, TILE128), desc_kmajor(dh, s, TILE128),
                 idesc_bf16(64, 128, true, false), acc);
        mma_bf16(taddr(tb, 0, 384), desc_mnmajor(dut, s, TILE128), desc_kmajor(h, s, TILE128),
                 idesc_bf16(64, 128, true, false), acc);
      }
#pragma unroll
      for (int s = 0; s < 8; ++s)
        mma_bf16(taddr(tb, 0, 384), desc_mnmajor(dutl, s, TILE128), desc_kmajor(h, s, TILE128),
                 idesc_bf16(64, 128, true, false), 1);
      mma_commit(&barM);
    }
    // <dS', S> over the two bf16 state tiles (while the MMAs run)
    {
      float dot = 0.f;
      for (int c = tid; c < 128 * 16; c += 256) {
        const int rr = c / 16, j = c % 16;
        float a8[8], b8[8];
        ld_chunk_f(sH, rr, j, TILE128, a8);
        ld_chunk_f(sdH, rr, j, TILE128, b8);
        for (int q = 0; q < 8; ++q) dot += a8[q] * b8[q];
      }
      dot = warp_sum(dot);
      if (lane == 0) sRed[warp] = dot;
    }
    fence_proxy_async();
    ok = __syncthreads_and(ok && mbar_wait(&barM, 0, err));
    tc_fence_after();
    if (!ok) break;
    // dO, dU^T, S and dS' are no longer read: the next unit's copies stream in from here
    if (tid == 0 && nvalid) {
      load_B(nu);
      pendB = (int)(ph ^ 1);
    }
    const float G0 = sG[r0], G1 = sG[r1], GC = sG[63];
    {
      // P = QK * Gam, dP = scale dO U^T (lower incl. diagonal), columns [32*half, +32)
      float qk[16], dp[16];
      tmem_ld16dp_x4(taddr(tb, sub, 32 * half), qk);
      tmem_ld16dp_x4(taddr(tb, sub, 64 + 32 * half), dp);
      tmem_wait_ld();
      float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = 32 * half + 8 * j + cq;
        float g[4], m[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int row = q < 2 ? r0 : r1, col = c + (q & 1);
          const float Gi = q < 2 ? G0 : G1;
          float dpp = 0.f, gg = 0.f;
          if (col <= row) {
            const float gam = __expf(Gi - sG[col]);
            const float dpv = p.scale * dp[4 * j + q];
            dpp = dpv * qk[4 * j + q] * gam;
            gg = dpv * gam;
          }
          g[q] = gg;
          m[q] = dpp;
        }
        sM[r0 * 65 + c] = m[0];
        sM[r0 * 65 + c + 1] = m[1];
        sM[r1 * 65 + c] = m[2];
        sM[r1 * 65 + c + 1] = m[3];
        rs0 += m[0] + m[1];
        rs1 += m[2] + m[3];
        st_pair_split(sPG, sPGl, r0, c, TILE64, g[0], g[1]);
        st_pair_split(sPG, sPGl, r1, c, TILE64, g[2], g[3]);
      }
      rs0 = quad_sum(rs0);
      rs1 = quad_sum(rs1);
      // dQ part 1: scale e^{G_i} dO S back into TMEM; dG2 = sum_k (.) Q[i,k]
      float x[32], y[32], z[32];
      tmem_ld16dp_x8(taddr(tb, sub, 128 + 64 * half), x);
      tmem_ld16dp_x8(taddr(tb, sub, 256 + 64 * half), y);
      tmem_ld16dp_x8(taddr(tb, sub, 384 + 64 * half), z);
      tmem_wait_ld();
      const float e0 = p.scale * __expf(G0), e1 = p.scale * __expf(G1);
      const float D0 = __expf(GC - G0), D1 = __expf(GC - G1);
      float x0 = 0.f, x1 = 0.f, y0 = 0.f, y1 = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int c = 64 * half + 8 * j + cq;
        const float2 q0 = ld_pair(sQ, r0, c, TILE64), q1 = ld_pair(sQ, r1, c, TILE64);
        const float2 k0 = ld_pair(sK, r0, c, TILE64), k1 = ld_pair(sK, r1, c, TILE64);
        x[4 * j] *= e0; x[4 * j + 1] *= e0; x[4 * j + 2] *= e1; x[4 * j + 3] *= e1;
        x0 += x[4 * j] * q0.x + x[4 * j + 1] * q0.y;
        x1 += x[4 * j + 2] * q1.x + x[4 * j + 3] * q1.y;
        y[4 * j] *= D0; y[4 * j + 1] *= D0; y[4 * j + 2] *= D1; y[4 * j + 3] *= D1;
        y0 += y[4 * j] * k0.x + y[4 * j + 1] * k0.y;
        y1 += y[4 * j + 2] * k1.x + y[4 * j + 3] * k1.y;
        // dW = -dU S, staged as a bf16 [64][128] tile in the (now free) U^T buffer
        st_pair(sUT, r0, c, TILE64, -z[4 * j], -z[4 * j + 1]);
        st_pair(sUT, r1, c, TILE64, -z[4 * j + 2], -z[4 * j + 3]);
      }
      tmem_st16dp_x8(taddr(tb, sub, 128 + 64 * half), x);
      tmem_st16dp_x8(taddr(tb, sub, 256 + 64 * half), y);
      x0 = quad_sum(x0);
      x1 = quad_sum(x1);
      y0 = quad_sum(y0);
      y1 = quad_sum(y1);
      if ((lane & 3) == 0) {
        sRow[(0 * 2 + half) * 64 + r0] = rs0;
        sRow[(0 * 2 + half) * 64 + r1] = rs1;
        sRow[(1 * 2 + half) * 64 + r0] = x0;
        sRow[(1 * 2 + half) * 64 + r1] = x1;
        sRow[(2 * 2 + half) * 64 + r0] = y0;  // D_i sum_k Y K (y already carries D_i)
        sRow[(2 * 2 + half) * 64 + r1] = y1;
      }
      tmem_wait_st();
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      tma_store_3d(&mdW, sUT, 0, (int)unit * 64, 0);
      tma_store_3d(&mdW, sUT + TILE64, 64, (int)unit * 64, 0);
      tma_store_commit();
      const uint32_t k = smem_u32(sK), q = smem_u32(sQ);
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const uint32_t pg = smem_u32(part ? sPGl : sPG);
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          mma_bf16(taddr(tb, 0, 128), desc_kmajor(pg, s, TILE64), desc_mnmajor(k, s, TILE64),
                   idesc_bf16(64, 128, false, true), 1);
          mma_bf16(taddr(tb, 0, 256), desc_mnmajor(pg, s, TILE64), desc_mnmajor(q, s, TILE64),
                   idesc_bf16(64, 128, true, true), 1);
        }
      }
      mma_commit(&barM);
    }
    // dG for this chunk (rows j = tid < 64), deterministic column sums
    if (tid < 64) {
      const int j = tid;
      float cs = 0.f;
      for (int ii = 0; ii < 64; ++ii) cs += sM[ii * 65 + j];
      float g = sRow[0 * 64 + j] + sRow[1 * 64 + j] - cs + sRow[2 * 64 + j] + sRow[3 * 64 + j] -
                (sRow[4 * 64 + j] + sRow[5 * 64 + j]);
      if (j == 63) {
        float d8 = 0.f, rsum = 0.f;
        for (int q = 0; q < 8; ++q) d8 += sRed[q];
        for (int q = 0; q < 64; ++q) rsum += sRow[4 * 64 + q] + sRow[5 * 64 + q];
        g += __expf(GC) * d8 + rsum;
      }
      w.dG[((size_t)hv * p.NCmax + gc) * 64 + j] = g;
    }
    ok = __syncthreads_and(ok && mbar_wait(&barM, 1, err));
    tc_fence_after();
    if (!ok) break;
    // Q, K no longer read; U^T (the dW staging) once the dW store has read it
    if (tid == 0 && nvalid) {
      tma_store_wait_read0();
      load_A(nu);
      pendA = (int)(ph ^ 1);
    }
    {
      // dq, dk of this value head into the k-head's fp32 tiles: the group's first value head
      // stores, the others add (L2 reductions; one thread's operations on an address stay in
      // order, so every sum is taken in the same order on every run)
      float x[32], y[32];
      tmem_ld16dp_x8(taddr(tb, sub, 128 + 64 * half), x);
      tmem_ld16dp_x8(taddr(tb, sub, 256 + 64 * half), y);
      tmem_wait_ld();
      const size_t kk = (size_t)gc * p.H + hv / p.G;
      float* dq0 = w.dqp + (kk * 64 + r0) * D + 64 * half + cq;
      float* dk0 = w.dkp + (kk * 64 + r0) * D + 64 * half + cq;
      if (hv % p.G == 0) {
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          *reinterpret_cast<float2*>(dq0 + 8 * jj) = make_float2(x[4 * jj], x[4 * jj + 1]);
          *reinterpret_cast<float2*>(dq0 + 8 * D + 8 * jj) = make_float2(x[4 * jj + 2], x[4 * jj + 3]);
          *reinterpret_cast<float2*>(dk0 + 8 * jj) = make_float2(y[4 * jj], y[4 * jj + 1]);
          *reinterpret_cast<float2*>(dk0 + 8 * D + 8 * jj) = make_float2(y[4 * jj + 2], y[4 * jj + 3]);
        }
      } else {
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          atomicAdd(reinterpret_cast<float2*>(dq0 + 8 * jj), make_float2(x[4 * jj], x[4 * jj + 1]));
          atomicAdd(reinterpret_cast<float2*>(dq0 + 8 * D + 8 * jj), make_float2(x[4 * jj + 2], x[4 * jj + 3]));
          atomicAdd(reinterpret_cast<float2*>(dk0 + 8 * jj), make_float2(y[4 * jj], y[4 * jj + 1]));
          atomicAdd(reinterpret_cast<float2*>(dk0 + 8 * D + 8 * jj), make_float2(y[4 * jj + 2], y[4 * jj + 3]));
        }
      }
    }
    // the next unit's first MMAs overwrite every TMEM column read above
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  if (tid == 0) {
    // after an error: let copies still in flight land before the shared memory is released
    if (pendA >= 0) mbar_wait(&barA, (uint32_t)pendA, err);
    if (pendB >= 0) mbar_wait(&barB, (uint32_t)pendB, err);
    tma_store_wait0();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, 512);
}

// ======================================================================================
// WY backward.  One CTA (256 threads) per (chunk, value head).  TMEM columns:
//   [0,64) dU V^T, then T^T dT   [64,128) dW K^T, then Z T^T   [128,192) K K^T
//   [256,384) T^T dW -> dk       [384,512) T^T dU
// 16-lane TMEM loads as in dqkwg: thread rows r0 = 16(w%4) + t/4 and r0 + 8.
// ======================================================================================
struct WyBwdSmem {
  static constexpr int K = 0;                                    // 2 x [64][128] (double buffer)
  static constexpr int V = 4 * TILE64, T = 6 * TILE64, TL = 7 * TILE64, DW = 8 * TILE64,
                       DUT = 10 * TILE64, DT = 10 * TILE64 + TILE128, DTL = DT + TILE64,
                       Z = DTL + TILE64, ZL = Z + TILE64, AS = ZL + TILE64, ASL = AS + TILE64,
                       DUTL = ASL + TILE64, F = DUTL + TILE128;
  static constexpr int KKG = F, AA = KKG + 64 * 65 * 4;        // fp32 [64][65] each
  static constexpr int G = AA + 64 * 65 * 4, B = G + 256, EG = B + 256, ROW = EG + 256;
  static constexpr int TOTAL = ROW + 4 * 2 * 64 * 4;            // ROW [4][2][64]
};

__global__ void __launch_bounds__(256) k_tc_wy_bwd(Problem p, Args a, Work w, TcWork t,
                                                   const __grid_constant__ CUtensorMap mk,
                                                   const __grid_constant__ CUtensorMap mv,
                                                   const __grid_constant__ CUtensorMap mTm,
                                                   const __grid_constant__ CUtensorMap mdW,
                                                   const __grid_constant__ CUtensorMap mdUT,
                                                   const __grid_constant__ CUtensorMap mdUTl,
                                                   UnitRange ur) {
  if (failed(w)) return;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int half = warp >> 2, sub = 32 * (warp & 3);
  const int r0 = 16 * (warp & 3) + lane / 4, r1 = r0 + 8, cq = 2 * (lane & 3);
  extern __shared__ unsigned char smraw[];
  unsigned char* sm = align1k(smraw);
  unsigned char* sKb = sm + WyBwdSmem::K;   // 2 x [64][128]: K of this unit and of the next
  unsigned char* sV = sm + WyBwdSmem::V;
  unsigned char* sT = sm + WyBwdSmem::T;
  unsigned char* sTl = sm + WyBwdSmem::TL;
  unsigned char* sdW = sm + WyBwdSmem::DW;
  unsigned char* sdUT = sm + WyBwdSmem::DUT;
  unsigned char* sdT = sm + WyBwdSmem::DT;
  unsigned char* sdTl = sm + WyBwdSmem::DTL;
  unsigned char* sZ = sm + WyBwdSmem::Z;
  unsigned char* sZl = sm + WyBwdSmem::ZL;
  unsigned char* sAs = sm + WyBwdSmem::AS;
  unsigned char* sAsl = sm + WyBwdSmem::ASL;
  unsigned char* sdUTl = sm + WyBwdSmem::DUTL;
  float* sKKG = reinterpret_cast<float*>(sm + WyBwdSmem::KKG);
  float* sAA = reinterpret_cast<float*>(sm + WyBwdSmem::AA);
  float* sG = reinterpret_cast<float*>(sm + WyBwdSmem::G);
  float* sb = reinterpret_cast<float*>(sm + WyBwdSmem::B);
  float* sEG = reinterpret_cast<float*>(sm + WyBwdSmem::EG);   // e^{G_j}
  float* sRow = reinterpret_cast<float*>(sm + WyBwdSmem::ROW);  // [kind][half][64]
  // barA: K (double-buffered);  barB: dW, dU^T (hi, lo);  barC: V, T (hi, lo);
  // barM: MMA batches (4 per unit)
  __shared__ uint64_t barA, barB, barC, barM;
  __shared__ uint32_t tslot;
  int* err = w.status;
  if (tid == 0) {
    mbar_init(&barA, 1);
    mbar_init(&barB, 1);
    mbar_init(&barC, 1);
    mbar_init(&barM, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (warp == 0) {
    tmem_alloc(&tslot, 512);
    tmem_relinquish();
  }
  // Units u = chunk * HV + hv in [u0, u1), handed out in k-head groups (chunk, hk) by an atomic
  // counter: a CTA runs the G value heads of a group back to back (their dq and dk shares go
  // to the k-head's fp32 tiles in a fixed order).  Thread 0 takes the next unit a unit ahead;
  // -1 marks the end of the work (past the range, or a chunk-table entry past the chunk count).
  auto next_of = [&](int u) {
    if (u >= 0 && (u % p.HV) % p.G + 1 < p.G) return u + 1;
    const int kk = ur.u0 / p.G + atomicAdd(ur.ctr, 1);
    if (kk >= ur.u1 / p.G) return -1;
    const int gc = kk / p.H;
    return w.chunk_tab[gc].x >= 0 ? gc * p.HV + (kk % p.H) * p.G : -1;
  };
  auto valid = [](int u) { return u >= 0; };
  auto load_A = [&](int u, int buf) {
    const int hk = (u % p.HV) / p.G, tok0 = w.chunk_tab[u / p.HV].w;
    unsigned char* dst = sKb + buf * 2 * TILE64;
    mbar_expect_tx(&barA, 2 * TILE64);
    tma_load_3d(dst, &mk, 0, hk, tok0, &barA);
    tma_load_3d(dst + TILE64, &mk, 64, hk, tok0, &barA);
  };
  auto load_B = [&](int u) {
    mbar_expect_tx(&barB, 2 * TILE64 + 2 * TILE128);
    tma_load_3d(sdW, &mdW, 0, u * 64, 0, &barB);
    tma_load_3d(sdW + TILE64, &mdW, 64, u * 64, 0, &barB);
    tma_load_3d(sdUT, &mdUT, 0, u * D, 0, &barB);
    tma_load_3d(sdUTl, &mdUTl, 0, u * D, 0, &barB);
  };
  auto load_C = [&](int u) {
    const int hv = u % p.HV, tok0 = w.chunk_tab[u / p.HV].w;
    mbar_expect_tx(&barC, 4 * TILE64);
    tma_load_3d(sV, &mv, 0, hv, tok0, &barC);
    tma_load_3d(sV + TILE64, &mv, 64, hv, tok0, &barC);
    tma_load_3d(sT, &mTm, 0, u * 128, 0, &barC);
    tma_load_3d(sTl, &mTm, 0, u * 128 + 64, 0, &barC);
  };
  // units handed out in order by an atomic counter, the next one taken a unit ahead
  __shared__ int s_unit[2];
  int u = -1;
  if (tid == 0) {
    u = next_of(-1);
    s_unit[0] = u;
  }
  int pendA = -1, pendB = -1, pendC = -1;  // parity of a load group in flight (thread 0)
  if (tid == 0 && valid(u)) {
    load_A(u, 0);
    load_B(u);
    load_C(u);
    pendA = pendB = pendC = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  u = s_unit[0];
  const uint32_t tb = tslot;
  bool ok = true;
  int nu = -1;
  // the unit's gate sums and beta, read into registers a unit ahead (see dqkwg)
  float g_next = 0.f, b_next = 0.f;
  auto vec_of = [&](int uu) {
    if (tid < 64 && valid(uu)) {
      const size_t o = ((size_t)(uu % p.HV) * p.NCmax + uu / p.HV) * 64 + tid;
      g_next = w.G[o];
      b_next = w.beta_p[o];
    }
  };
  vec_of(u);
  for (uint32_t it = 0; valid(u); ++it, u = nu) {
    const int gc = u / p.HV, hv = u % p.HV;
    const int4 e = w.chunk_tab[gc];
    const int L = e.z, tok0 = e.w;
    if (tid == 0) s_unit[(it + 1) & 1] = next_of(u);
    const uint32_t ph = it & 1;
    if (tid < 64) {
      sG[tid] = g_next;
      sb[tid] = b_next;
      sEG[tid] = __expf(g_next);
    }
    const bool got = mbar_wait(&barA, ph, err) && mbar_wait(&barB, ph, err) && mbar_wait(&barC, ph, err);
    if (tid == 0) pendA = pendB = pendC = got ? -1 : (int)ph;
    ok = __syncthreads_and(ok && got);
    if (!ok) break;
    nu = s_unit[(it + 1) & 1];
    const bool nvalid = valid(nu);
    unsigned char* sK = sKb + (it & 1) * 2 * TILE64;
    if (tid == 0 && nvalid) {  // the other K buffer was last read by the previous unit
      load_A(nu, (int)(ph ^ 1));
      pendA = (int)(ph ^ 1);
    }
    if (L < 64) {
      zero_tail_rows(sK, L, tid, 256);
      zero_tail_rows(sV, L, tid, 256);
    }
    fence_proxy_async();
    __syncthreads();
    vec_of(nu);  // after the barrier: its latency hides behind this unit's products
    const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aT = smem_u32(sT), aTl = smem_u32(sTl),
                   aW = smem_u32(sdW), aU = smem_u32(sdUT), aUl = smem_u32(sdUTl);
    if (tid == 0) {
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const uint32_t acc = s > 0;
        mma_bf16(taddr(tb, 0, 0), desc_mnmajor(aU, s, TILE128), desc_kmajor(aV, s, TILE64),
                 idesc_bf16(64, 64, true, false), acc);
        mma_bf16(taddr(tb, 0, 0), desc_mnmajor(aUl, s, TILE128), desc_kmajor(aV, s, TILE64),
                 idesc_bf16(64, 64, true, false), 1);
        mma_bf16(taddr(tb, 0, 64), desc_kmajor(aW, s, TILE64), desc_kmajor(aK, s, TILE64),
                 idesc_bf16(64, 64, false, false), acc);
        mma_bf16(taddr(tb, 0, 128), desc_kmajor(aK, s, TILE64), desc_kmajor(aK, s, TILE64),
                 idesc_bf16(64, 64, false, false), acc);
      }
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const uint32_t tt = part ? aTl : aT;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint32_t acc = part > 0 || s > 0;
          mma_bf16(taddr(tb, 0, 256), desc_mnmajor(tt, s, TILE64), desc_mnmajor(aW, s, TILE64),
                   idesc_bf16(64, 128, true, true), acc);
          mma_bf16(taddr(tb, 0, 384), desc_mnmajor(tt, s, TILE64), desc_kmajor(aU, s, TILE128),
                   idesc_bf16(64, 128, true, false), acc);
          if (part == 0)
            mma_bf16(taddr(tb, 0, 384), desc_mnmajor(tt, s, TILE64), desc_kmajor(aUl, s, TILE128),
                     idesc_bf16(64, 128, true, false), 1);
        }
      }
      mma_commit(&barM);
    }
    ok = __syncthreads_and(ok && mbar_wait(&barM, 0, err));
    tc_fence_after();
    if (!ok) break;
    if (tid == 0 && nvalid) {  // dW, dU^T are read by the first MMA batch only
      load_B(nu);
      pendB = (int)(ph ^ 1);
    }
    const float G0 = sG[r0], G1 = sG[r1], b0 = sb[r0], b1 = sb[r1];
    {
      float r1v[16], r2v[16], kk[16];
      tmem_ld16dp_x4(taddr(tb, sub, 32 * half), r1v);
      tmem_ld16dp_x4(taddr(tb, sub, 64 + 32 * half), r2v);
      tmem_ld16dp_x4(taddr(tb, sub, 128 + 32 * half), kk);
      tmem_wait_ld();
  #pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = 32 * half + 8 * j + cq;
        const float bc0 = sb[c], bc1 = sb[c + 1], ec0 = sEG[c], ec1 = sEG[c + 1];
        st_pair_split(sdT, sdTl, r0, c, TILE64, bc0 * (r1v[4 * j] + ec0 * r2v[4 * j]),
                      bc1 * (r1v[4 * j + 1] + ec1 * r2v[4 * j + 1]));
        st_pair_split(sdT, sdTl, r1, c, TILE64, bc0 * (r1v[4 * j + 2] + ec0 * r2v[4 * j + 2]),
                      bc1 * (r1v[4 * j + 3] + ec1 * r2v[4 * j + 3]));
        sKKG[r0 * 65 + c] = c < r0 ? __expf(G0 - sG[c]) * kk[4 * j] : 0.f;
        sKKG[r0 * 65 + c + 1] = c + 1 < r0 ? __expf(G0 - sG[c + 1]) * kk[4 * j + 1] : 0.f;
        sKKG[r1 * 65 + c] = c < r1 ? __expf(G1 - sG[c]) * kk[4 * j + 2] : 0.f;
        sKKG[r1 * 65 + c + 1] = c + 1 < r1 ? __expf(G1 - sG[c + 1]) * kk[4 * j + 3] : 0.f;
      }
      // dX: dbeta/dG parts, then beta_i e^{G_i} dX back into TMEM; dY: dv = beta dY, dbeta part
      float x[32], y[32];
      tmem_ld16dp_x8(taddr(tb, sub, 256 + 64 * half), x);
      tmem_ld16dp_x8(taddr(tb, sub, 384 + 64 * half), y);
      tmem_wait_ld();
      const float s0 = b0 * sEG[r0], s1 = b1 * sEG[r1];
      float px0 = 0.f, px1 = 0.f, py0 = 0.f, py1 = 0.f;
      bf16* dv0 = static_cast<bf16*>(a.dv) + ((size_t)(tok0 + r0) * p.HV + hv) * p.V + 64 * half + cq;
      bf16* dv1 = dv0 + (size_t)8 * p.HV * p.V;
      const bool live = 64 * half < p.V;  // columns past a 64-wide value head are padding
  #pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int c = 64 * half + 8 * j + cq;
        const float2 k0 = ld_pair(sK, r0, c, TILE64), k1 = ld_pair(sK, r1, c, TILE64);
        const float2 v0 = ld_pair(sV, r0, c, TILE64), v1 = ld_pair(sV, r1, c, TILE64);
        px0 += x[4 * j] * k0.x + x[4 * j + 1] * k0.y;
        px1 += x[4 * j + 2] * k1.x + x[4 * j + 3] * k1.y;
        x[4 * j] *= s0; x[4 * j + 1] *= s0; x[4 * j + 2] *= s1; x[4 * j + 3] *= s1;
        py0 += y[4 * j] * v0.x + y[4 * j + 1] * v0.y;
        py1 += y[4 * j + 2] * v1.x + y[4 * j + 3] * v1.y;
        if (live && r0 < L)
          *reinterpret_cast<uint32_t*>(dv0 + 8 * j) = pack_bf16(b0 * y[4 * j], b0 * y[4 * j + 1]);
        if (live && r1 < L)
          *reinterpret_cast<uint32_t*>(dv1 + 8 * j) = pack_bf16(b1 * y[4 * j + 2], b1 * y[4 * j + 3]);
      }
      tmem_st16dp_x8(taddr(tb, sub, 256 + 64 * half), x);
      px0 = quad_sum(px0);
      px1 = quad_sum(px1);
      py0 = quad_sum(py0);
      py1 = quad_sum(py1);
      if ((lane & 3) == 0) {
        sRow[(0 * 2 + half) * 64 + r0] = px0;
        sRow[(0 * 2 + half) * 64 + r1] = px1;
        sRow[(1 * 2 + half) * 64 + r0] = py0;
        sRow[(1 * 2 + half) * 64 + r1] = py1;
      }
      tmem_wait_st();
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // Z = T^T dT, dropping lo*lo
    if (tid == 0) {
      const uint32_t dt = smem_u32(sdT), dtl = smem_u32(sdTl);
      const uint32_t pa[3] = {aT, aT, aTl}, pb[3] = {dt, dtl, dt};
#pragma unroll
      for (int part = 0; part < 3; ++part)
#pragma unroll
        for (int s = 0; s < 4; ++s)
          mma_bf16(taddr(tb, 0, 0), desc_mnmajor(pa[part], s, TILE64), desc_mnmajor(pb[part], s, TILE64),
                   idesc_bf16(64, 64, true, true), part > 0 || s > 0);
      mma_commit(&barM);
    }
    ok = __syncthreads_and(ok && mbar_wait(&barM, 1, err));
    tc_fence_after();
    if (!ok) break;
    {
      float z[16];
      tmem_ld16dp_x4(taddr(tb, sub, 32 * half), z);
      tmem_wait_ld();
  #pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = 32 * half + 8 * j + cq;
        st_pair_split(sZ, sZl, r0, c, TILE64, z[4 * j], z[4 * j + 1]);
        st_pair_split(sZ, sZl, r1, c, TILE64, z[4 * j + 2], z[4 * j + 3]);
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // dA' = Z T^T
    if (tid == 0) {
      const uint32_t zz = smem_u32(sZ), zl = smem_u32(sZl);
      const uint32_t pa[3] = {zz, zz, zl}, pb[3] = {aT, aTl, aT};
#pragma unroll
      for (int part = 0; part < 3; ++part)
#pragma unroll
        for (int s = 0; s < 4; ++s)
          mma_bf16(taddr(tb, 0, 64), desc_kmajor(pa[part], s, TILE64), desc_kmajor(pb[part], s, TILE64),
                   idesc_bf16(64, 64, false, false), part > 0 || s > 0);
      mma_commit(&barM);
    }
    ok = __syncthreads_and(ok && mbar_wait(&barM, 0, err));
    tc_fence_after();
    if (!ok) break;
    if (tid == 0 && nvalid) {  // V (last read in the first epilogue) and T (by the MMAs above)
      load_C(nu);
      pendC = (int)(ph ^ 1);
    }
    {
      float da[16];
      tmem_ld16dp_x4(taddr(tb, sub, 64 + 32 * half), da);
      tmem_wait_ld();
      float pa0 = 0.f, pa1 = 0.f, paa0 = 0.f, paa1 = 0.f;
  #pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = 32 * half + 8 * j + cq;
        float as[4];
  #pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int row = q < 2 ? r0 : r1, col = c + (q & 1);
          const float Gi = q < 2 ? G0 : G1, bi = q < 2 ? b0 : b1;
          float dAs = 0.f, aa = 0.f;
          if (col < row) {
            const float dA = -da[4 * j + q];
            const float kkg = sKKG[row * 65 + col];
            if (q < 2) pa0 += dA * kkg; else pa1 += dA * kkg;
            aa = dA * bi * kkg;
            dAs = dA * __expf(Gi - sG[col]) * bi;
          }
          sAA[row * 65 + col] = aa;
          if (q < 2) paa0 += aa; else paa1 += aa;
          as[q] = dAs;
        }
        st_pair_split(sAs, sAsl, r0, c, TILE64, as[0], as[1]);
        st_pair_split(sAs, sAsl, r1, c, TILE64, as[2], as[3]);
      }
      pa0 = quad_sum(pa0);
      pa1 = quad_sum(pa1);
      paa0 = quad_sum(paa0);
      paa1 = quad_sum(paa1);
      if ((lane & 3) == 0) {
        sRow[(2 * 2 + half) * 64 + r0] = pa0;
        sRow[(2 * 2 + half) * 64 + r1] = pa1;
        sRow[(3 * 2 + half) * 64 + r0] = paa0;
        sRow[(3 * 2 + half) * 64 + r1] = paa1;
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // dk += dAs K + dAs^T K onto beta e^G dX
    if (tid == 0) {
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const uint32_t as = smem_u32(part ? sAsl : sAs);
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          mma_bf16(taddr(tb, 0, 256), desc_kmajor(as, s, TILE64), desc_mnmajor(aK, s, TILE64),
                   idesc_bf16(64, 128, false, true), 1);
          mma_bf16(taddr(tb, 0, 256), desc_mnmajor(as, s, TILE64), desc_mnmajor(aK, s, TILE64),
                   idesc_bf16(64, 128, true, true), 1);
        }
      }
      mma_commit(&barM);
    }
    {  // column j = tid/4 of the dAs*beta*KKG products, four threads per column
      const int j = tid >> 2, part = tid & 3;
      float cs = 0.f;
  #pragma unroll
      for (int i = 0; i < 16; ++i) cs += sAA[(part + 4 * i) * 65 + j];
      cs = quad_sum(cs);
      if (part == 0) {
        const float eg = sEG[j], bj = sb[j];
        const float px = sRow[0 * 64 + j] + sRow[1 * 64 + j];
        const float py = sRow[2 * 64 + j] + sRow[3 * 64 + j];
        const float pa = sRow[4 * 64 + j] + sRow[5 * 64 + j];
        const float paa = sRow[6 * 64 + j] + sRow[7 * 64 + j];
        if (j < L) a.dbeta[(size_t)(tok0 + j) * p.HV + hv] = eg * px + py + pa;
        w.dG2[((size_t)hv * p.NCmax + gc) * 64 + j] = bj * eg * px + paa - cs;
      }
    }
    ok = __syncthreads_and(ok && mbar_wait(&barM, 1, err));
    tc_fence_after();
    if (!ok) break;
    {  // this kernel's dk share, added onto dqkwg's k-head tile (value heads in order)
      float x[32];
      tmem_ld16dp_x8(taddr(tb, sub, 256 + 64 * half), x);
      tmem_wait_ld();
      float* dk0 = w.dkp + (((size_t)gc * p.H + hv / p.G) * 64 + r0) * D + 64 * half + cq;
  #pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        atomicAdd(reinterpret_cast<float2*>(dk0 + 8 * jj), make_float2(x[4 * jj], x[4 * jj + 1]));
        atomicAdd(reinterpret_cast<float2*>(dk0 + 8 * D + 8 * jj), make_float2(x[4 * jj + 2], x[4 * jj + 3]));
      }
    }
    // the next unit's first MMAs overwrite every TMEM column read above
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  if (tid == 0) {  // after an error: let copies still in flight land first
    if (pendA >= 0) mbar_wait(&barA, (uint32_t)pendA, err);
    if (pendB >= 0) mbar_wait(&barB, (uint32_t)pendB, err);
    if (pendC >= 0) mbar_wait(&barC, (uint32_t)pendC, err);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tb, 512);
}

// dq, dk of one chunk and k-head from their fp32 tiles (the sums dqkwg and wy_bwd formed) to the
// caller's bf16 [token][head][K] tensors: rows past the chunk's end and columns past a 64-wide
// head are skipped.  Four columns per thread and step.
__global__ void __launch_bounds__(256) k_tc_dqdk_out(Problem p, Args a, Work w, int gc0) {
  if (failed(w)) return;
  const int gc = gc0 + blockIdx.x, hk = blockIdx.y;
  const int4 e = w.chunk_tab[gc];
  if (e.x < 0) return;
  const int L = e.z, tok0 = e.w, K = p.K;
  const size_t base = ((size_t)gc * p.H + hk) * 64 * D;
  for (int i = 4 * threadIdx.x; i < L * K; i += 4 * blockDim.x) {
    const int t = i / K, c = i % K;
    const float4 q = *reinterpret_cast<const float4*>(w.dqp + base + (size_t)t * D + c);
    const float4 k = *reinterpret_cast<const float4*>(w.dkp + base + (size_t)t * D + c);
    const size_t o = ((size_t)(tok0 + t) * p.H + hk) * K + c;
    *reinterpret_cast<uint2*>(static_cast<bf16*>(a.dq) + o) = make_uint2(pack_bf16(q.x, q.y), pack_bf16(q.z, q.w));
    *reinterpret_cast<uint2*>(static_cast<bf16*>(a.dk) + o) = make_uint2(pack_bf16(k.x, k.y), pack_bf16(k.z, k.w));
  }
}

}  // namespace

cudaError_t tc_backward_kernels(const Problem& p, const Args& a, const Work& w, const TcWork& t,
                                const TcMaps& m, cudaStream_t s) {
  const Segments sg = segments(p, kBwdSeg);
  cudaError_t e;
  // one work counter per persistent launch, zero before any of them starts
  if ((e = cudaMemsetAsync(t.ctr, 0, kCounters * sizeof(int), s))) return e;
  auto dvlocal = [&](int c0, int c1, cudaStream_t st) {
    return tgo("tc_dvlocal", k_tc_dvlocal, dim3(c1 - c0, p.HV), 128, 1024 + 6 * TILE64 + 512, st, p, w,
               t, m.q, m.k, m.dO, m.Op, m.dUlT, c0);
  };
  auto chunk_kernels = [&](int i, int c0, int c1, cudaStream_t st) {
    // persistent CTAs over k-head groups
    const int groups = (c1 - c0) * p.H;
    const dim3 gp((unsigned)std::min(groups, num_sms()));
    if ((e = tgo("tc_dqkwg", k_tc_dqkwg, gp, 256, 1024 + DqkSmem::TOTAL, st, p, a, w, t, m.q, m.k, m.dO,
                 m.UT, m.dUT, m.dUTl, m.h, m.dh, m.dW, UnitRange{c0 * p.HV, c1 * p.HV, t.ctr + 2 * i})))
      return e;
    if ((e = tgo("tc_wy_bwd", k_tc_wy_bwd, gp, 256, 1024 + WyBwdSmem::TOTAL, st, p, a, w, t, m.k, m.v,
                 m.Tm, m.dW, m.dUT, m.dUTl, UnitRange{c0 * p.HV, c1 * p.HV, t.ctr + 2 * i + 1})))
      return e;
    return tgo("tc_dqdk_out", k_tc_dqdk_out, dim3(c1 - c0, p.H), 256, 0, st, p, a, w, c0);
  };
  if (sg.n == 1) {
    if ((e = dvlocal(0, p.NCmax, s))) return e;
    if ((e = tc_scan_bwd(p, a, w, t, m, ScanRange{0, p.NCmax, a.dht, a.dh0}, s))) return e;
    return chunk_kernels(0, 0, p.NCmax, s);
  }
  // Segments in reverse: the reverse pass over segment i (side stream) runs while dv_local of
  // earlier segments and dqkwg / wy_bwd of later (already passed) segments run on `s`.
  SideLock side;
  if (!side.ok()) return cudaErrorInvalidResourceHandle;
  cudaStream_t hs = side.stream();
  if ((e = side.fork(s))) return e;
  std::vector<cudaEvent_t> dv_done(sg.n), scan_done(sg.n);
  for (int i = sg.n - 1; i >= 0; --i) {
    if ((e = dvlocal(sg.c[i], sg.c[i + 1], s))) return e;
    if ((e = side.record(s, &dv_done[i]))) return e;
  }
  for (int i = sg.n - 1; i >= 0; --i) {
    if ((e = cudaStreamWaitEvent(hs, dv_done[i], 0))) return e;
    const ScanRange r{sg.c[i], sg.c[i + 1], i + 1 == sg.n ? a.dht : t.hand, i == 0 ? a.dh0 : t.hand};
    if ((e = tc_scan_bwd(p, a, w, t, m, r, hs))) return e;
    if ((e = side.record(hs, &scan_done[i]))) return e;
  }
  for (int i = sg.n - 1; i >= 0; --i) {
    if ((e = cudaStreamWaitEvent(s, scan_done[i], 0))) return e;
    if ((e = chunk_kernels(i, sg.c[i], sg.c[i + 1], s))) return e;
  }
  return cudaSuccess;
}

}  // namespace tcx
}  // namespace gdn
