// Sequential state passes over the chunks (chunk_delta_h forward and the backward dhu pass of
// the G_T_CONTIG page), one CTA per (sequence, value head) carrying the whole 128 x 128 state.
//
// The chunk step is affine in the state.  With D = diag(e^{G_C - G_i}) (zero past the chunk's
// last token), W and U~ the chunk's WY factors and K its keys:
//   forward    S' = e^{G_C} S + U^T D K,  U = U~ - W S^T
//              = e^{G_C} S + B - S N,     N = W^T D K (K x K),  B = U~^T D K (V x K)
//   backward   dS = e^{G_C} dS' + scale (e^G dO)^T Q - dU^T W,  dU = dU_loc + D K dS'^T
//              = e^{G_C} dS' - (F + dS' N^T),  F = W^T... (below, transposed)
// N and B (F) do not depend on the state, so they are built off the chain, one chunk ahead;
// the chain itself is one tensor-core product per chunk (S N), instead of two dependent ones
// (W S^T, then U^T D K).  Everything is kept transposed so that TMEM lane = key index k':
// thread k' of the chain warps holds row k' of S^T (128 fp32 values, one per value index) in
// registers, and the bf16 copy of S^T that feeds the next product is written row by row.
#include "gdn_tc_common.cuh"

namespace gdn {
namespace tcx {

namespace {

// Named barrier of the four "side" warps (4..7) only.
__device__ __forceinline__ void bar_sync_side() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// ======================================================================================
// Forward.  256 threads: warps 0-3 ("chain") own TMEM lanes = rows k' of S^T; warps 4-7
// ("side") scale K, read N and U out of TMEM.  Thread 0 issues the MMAs, thread 32 the TMA
// loads.  Per chunk c, in tensor-pipe order:
//   chain(c)  ACC[c&1] += (-N_c^T) S_c^T            M=128 k', N=128 v, K=128 k   (8 instr)
//   U(c)      UREG      = S_c W_c^T                 M=128 v,  N=64 i,  K=128 k   (8)
//   N(c+1)    NT        = (D K)^T W                 M=128 k', N=128 k, K=64 i    (4)
//   B(c+1)    ACC[~]    = (D K)^T U~                M=128 k', N=128 v, K=64 i    (4)
// Shared memory: three input stages {U~^T [128][64], W^T [128][64], K [64][128]} (the chunk
// two ahead streams in while one is consumed), S^T bf16 [128 k][128 v] (MN-major B operand of
// the chain and MN-major A operand of U), -N^T bf16 [128 k'][128 k] (K-major A of the chain).
// Outputs: h[c] = S_c^T ([k][v] bf16, from registers), U^T ([v][i] bf16, from registers), and
// the final state [k][v] fp32.
// ======================================================================================
struct Fwd2Smem {
  static constexpr int STAGE = 3 * TILE128;                 // U~^T, W^T, K (2 x TILE64)
  static constexpr int S = 3 * STAGE;                       // S^T bf16, 2 blocks [128][64]
  static constexpr int N = S + 2 * TILE128;                 // -N^T bf16, 2 blocks [128][64]
  static constexpr int VEC = N + 2 * TILE128;               // 3 x {D[64], e^{G_C}}
  static constexpr int TOTAL = VEC + 3 * 272;
};

__global__ void __launch_bounds__(256, 1) k_tc_scan_fwd2(Problem p, Args a, Work w, TcWork t,
                                                         const __grid_constant__ CUtensorMap mk,
                                                         const __grid_constant__ CUtensorMap mWT,
                                                         const __grid_constant__ CUtensorMap mUtT,
                                                         ScanRange sr) {
  // one read of the status word decides for the whole CTA (barriers below need every thread)
  __shared__ int s_fail;
  if (threadIdx.x == 0) s_fail = failed(w);
  __syncthreads();
  if (s_fail) return;
  const int n = blockIdx.x, hv = blockIdx.y, hk = hv / p.G;
  const int4 sq0 = w.seq_tab[n];
  // this launch's chunks of the sequence: [cb, cb + nc); sq = the sequence table entry with
  // its first chunk and token moved to cb
  const int cb = min(max(sr.c0, 0), sq0.y), nc = max(min(sr.c1, sq0.y) - cb, 0);
  const int4 sq = make_int4(sq0.x + cb, nc, sq0.z + 64 * cb, sq0.w - 64 * cb);
  const int tid = threadIdx.x, warp = tid / 32;
  const bool chain = tid < 128;
  const int row = tid & 127;  // TMEM lane of this thread's warp quarter: k' (chain) or v / k' (side)
  extern __shared__ unsigned char smraw[];
  unsigned char* sm = align1k(smraw);
  unsigned char* sS = sm + Fwd2Smem::S;
  unsigned char* sN = sm + Fwd2Smem::N;
  auto stage = [&](int c) { return sm + (c % 3) * Fwd2Smem::STAGE; };
  auto vec = [&](int c) { return reinterpret_cast<float*>(sm + Fwd2Smem::VEC + (c % 3) * 272); };
  __shared__ uint64_t barL[3], barC, barU, barN, barE;
  __shared__ uint32_t tslot;
  int* err = w.status;
  // the test flag withholds the first chain product; its wait then runs out quickly
  const long long wait_limit = p.test_timeout ? (1ll << 20) : (1ll << 31);
  if (tid == 0) {
    for (int i = 0; i < 3; ++i) mbar_init(&barL[i], 1);
    mbar_init(&barC, 1);
    mbar_init(&barU, 1);
    mbar_init(&barN, 1);
    mbar_init(&barE, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (warp == 0) {
    tmem_alloc(&tslot, 512);
    tmem_relinquish();
  }
  auto unit_row = [&](int c) { return ((sq.x + c) * p.HV + hv) * D; };
  auto chunk_len = [&](int c) { return min(64, sq.w - 64 * c); };
  auto issue_load = [&](int c) {  // thread 32
    unsigned char* b = stage(c);
    uint64_t* bar = &barL[c % 3];
    const int tok = sq.z + 64 * c, r = unit_row(c);
    mbar_expect_tx(bar, 2 * TILE128 + 2 * TILE64);
    tma_load_3d(b, &mUtT, 0, r, 0, bar);
    tma_load_3d(b + TILE128, &mWT, 0, r, 0, bar);
    tma_load_3d(b + 2 * TILE128, &mk, 0, hk, tok, bar);
    tma_load_3d(b + 2 * TILE128 + TILE64, &mk, 64, hk, tok, bar);
  };
  auto load_vec = [&](int c) {  // side threads 0..63 of the side group
    const int i = tid - 128;
    const size_t o = ((size_t)hv * p.NCmax + sq.x + c) * 64;
    float* v = vec(c);
    v[i] = i < chunk_len(c) ? w.Dec[o + i] : 0.f;
    if (i == 63) v[64] = w.EG[o + 63];
  };
  // side group: K <- D K in place (rows past the chunk end get D = 0)
  auto scale_k = [&](int c) {
    unsigned char* k = stage(c) + 2 * TILE128;
    const float* d = vec(c);
    for (int idx = tid - 128; idx < 64 * 16; idx += 128) {
      const int r = idx >> 4, j = idx & 15;
      float f[8];
      ld_chunk_f(k, r, j, TILE64, f);
      const float s = d[r];
#pragma unroll
      for (int q = 0; q < 8; ++q) f[q] *= s;
      st_chunk_f(k, r, j, TILE64, f);
    }
  };
  // chunk c is the (c/3)-th load into stage c%3: its barrier phase has parity (c/3)&1
  auto load_par = [](int c) { return (uint32_t)((c / 3) & 1); };
  int loaded = min(3, nc);  // chunks whose loads were issued (the same count in every thread)
  int confirmed = 0;        // chunks whose loads every thread saw complete
  if (tid == 32)
    for (int c = 0; c < loaded; ++c) issue_load(c);
  // thread k' = row (chain warps) holds S^T[k'][0..127] (the entering state, [k][v] layout)
  float S[D];
  const size_t st_off = ((size_t)n * p.HV + hv) * D * D + (size_t)row * D;
  if (chain) {
#pragma unroll
    for (int v = 0; v < D; v += 4) {
      const float4 x = sr.s_in ? *reinterpret_cast<const float4*>(sr.s_in + st_off + v) : make_float4(0, 0, 0, 0);
      S[v] = x.x; S[v + 1] = x.y; S[v + 2] = x.z; S[v + 3] = x.w;
    }
  }
  // bf16 S^T rows: the chain operand in shared memory, and h[c] in the workspace
  auto put_state = [&](int c, bool smem) {
    bf16* hrow = t.h + ((size_t)unit_row(c) + row) * D;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      uint4 pk;
      pk.x = pack_bf16(S[8 * j], S[8 * j + 1]);
      pk.y = pack_bf16(S[8 * j + 2], S[8 * j + 3]);
      pk.z = pack_bf16(S[8 * j + 4], S[8 * j + 5]);
      pk.w = pack_bf16(S[8 * j + 6], S[8 * j + 7]);
      if (c < nc) *reinterpret_cast<uint4*>(hrow + 8 * j) = pk;
      if (smem) *reinterpret_cast<uint4*>(sS + sw128_chunk(row, j, TILE128)) = pk;
    }
  };
  if (chain && nc > 0) put_state(0, true);
  if (!chain && tid - 128 < 64 && nc > 0) load_vec(0);
  if (!chain && tid - 128 < 64 && nc > 1) load_vec(1);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tslot;
  const uint32_t tACC0 = taddr(tb, 0, 0), tNT = taddr(tb, 0, 256), tU = taddr(tb, 0, 384);
  bool ok = true;
  // issue N(c) and B(c) (K of chunk c already scaled)
  auto issue_nb = [&](int c) {
    unsigned char* b = stage(c);
    const uint64_t dk = desc_mnmajor(smem_u32(b + 2 * TILE128), 0, TILE64);
    const uint64_t dw = desc_kmajor(smem_u32(b + TILE128), 0, TILE128);
    const uint64_t du = desc_kmajor(smem_u32(b), 0, TILE128);
    constexpr uint32_t id = idesc_bf16(128, 128, true, false);
#pragma unroll
    for (int s = 0; s < 4; ++s)
      mma_bf16(tNT, dk + mnstep_off(s), dw + kstep_off(s, TILE128), id, s > 0);
    mma_commit(&barN);
    const uint32_t tacc = tACC0 + (uint32_t)(128 * (c & 1));
#pragma unroll
    for (int s = 0; s < 4; ++s)
      mma_bf16(tacc, dk + mnstep_off(s), du + kstep_off(s, TILE128), id, s > 0);
  };
  // side group: -N^T (TMEM lanes k', columns k) -> bf16 K-major rows of sN
  auto n_epilogue = [&]() {
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      float x[32];
      tmem_ld16(taddr(tb, 32 * (warp - 4), 256 + 32 * cc), x);
      tmem_ld16(taddr(tb, 32 * (warp - 4), 256 + 32 * cc + 16), x + 16);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 32; ++q) x[q] = -x[q];
#pragma unroll
      for (int j = 0; j < 4; ++j) st_chunk_f(sN, row, 4 * cc + j, TILE128, x + 8 * j);
    }
  };
  // prologue: N(0), B(0), then -N_0^T in shared memory
  if (nc > 0) {
    bool okp = true;
    if (!chain) {
      okp = mbar_wait(&barL[0], load_par(0), err);
      if (okp) scale_k(0);
      fence_proxy_async();
    }
    tc_fence_before();
    ok = __syncthreads_and(okp);
    tc_fence_after();
    if (ok) confirmed = 1;
    if (ok && tid == 0) issue_nb(0);
    if (ok && !chain) {
      okp = mbar_wait(&barN, 0, err);
      tc_fence_after();
      if (okp) n_epilogue();
      fence_proxy_async();
    }
    tc_fence_before();
    ok = __syncthreads_and(ok && okp);
    tc_fence_after();
  }
  for (int c = 0; ok && c < nc; ++c) {
    const bool more = c + 1 < nc;
    const float egc = vec(c)[64];
    bool okt = true;
    if (tid == 0) {
      const uint64_t da = desc_kmajor(smem_u32(sN), 0, TILE128);
      const uint64_t dsB = desc_mnmajor(smem_u32(sS), 0, TILE128);
      const uint32_t tacc = tACC0 + (uint32_t)(128 * (c & 1));
      if (!(p.test_timeout && c == 0)) {
#pragma unroll
        for (int s = 0; s < 8; ++s)  // chain: ACC += (-N^T) S^T
          mma_bf16(tacc, da + kstep_off(s, TILE128), dsB + mnstep_off(s), idesc_bf16(128, 128, false, true), 1);
        mma_commit(&barC);
      }
      const uint64_t dsA = desc_mnmajor(smem_u32(sS), 0, TILE128);
      const uint64_t dw = desc_mnmajor(smem_u32(stage(c) + TILE128), 0, TILE128);
#pragma unroll
      for (int s = 0; s < 8; ++s)  // U: S W^T
        mma_bf16(tU, dsA + mnstep_off(s), dw + mnstep_off(s), idesc_bf16(128, 64, true, true), s > 0);
      mma_commit(&barU);
    }
    if (chain) {
      // S_{c+1}^T = e^{G_C} S_c^T + ACC
      okt = mbar_wait_for(&barC, c & 1, err, wait_limit);
      tc_fence_after();
      if (okt) {
        const uint32_t tacc = 128 * (c & 1);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          float x[32];
          tmem_ld16(taddr(tb, 32 * warp, tacc + 32 * cc), x);
          tmem_ld16(taddr(tb, 32 * warp, tacc + 32 * cc + 16), x + 16);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 32; ++q) S[32 * cc + q] = egc * S[32 * cc + q] + x[q];
        }
      }
      // the U product must be done reading S_c^T before it is overwritten
      okt = okt && mbar_wait(&barU, c & 1, err);
      if (okt) put_state(c + 1, more);
      fence_proxy_async();
    } else {
      // side: the next chunk's K is scaled before N(c+1), B(c+1) are issued
      if (more) {
        okt = mbar_wait(&barL[(c + 1) % 3], load_par(c + 1), err);
        if (okt) scale_k(c + 1);
        fence_proxy_async();
      }
      if (tid - 128 < 64 && c + 2 < nc) load_vec(c + 2);
      // U^T = U~^T - S W^T for this chunk, straight to the workspace
      okt = okt && mbar_wait(&barU, c & 1, err);
      tc_fence_after();
      if (okt) {
        const unsigned char* ut = stage(c);
        bf16* urow = t.UT + ((size_t)unit_row(c) + row) * 64;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          float x[32];
          tmem_ld16(taddr(tb, 32 * (warp - 4), 384 + 32 * h2), x);
          tmem_ld16(taddr(tb, 32 * (warp - 4), 384 + 32 * h2 + 16), x + 16);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float f[8];
            ld_chunk_f(ut, row, 4 * h2 + j, TILE128, f);
            uint4 pk;
            pk.x = pack_bf16(f[0] - x[8 * j], f[1] - x[8 * j + 1]);
            pk.y = pack_bf16(f[2] - x[8 * j + 2], f[3] - x[8 * j + 3]);
            pk.z = pack_bf16(f[4] - x[8 * j + 4], f[5] - x[8 * j + 5]);
            pk.w = pack_bf16(f[6] - x[8 * j + 6], f[7] - x[8 * j + 7]);
            *reinterpret_cast<uint4*>(urow + 8 * (4 * h2 + j)) = pk;
          }
        }
      }
    }
    tc_fence_before();
    ok = __syncthreads_and(ok && okt);
    tc_fence_after();
    if (!ok) break;
    if (more) confirmed = c + 2;
    // stage c%3 is free (U(c) and the U epilogue are done): chunk c+3 streams into it
    if (loaded < nc) {
      if (tid == 32) issue_load(loaded);
      ++loaded;
    }
    if (more) {
      if (tid == 0) issue_nb(c + 1);
      if (!chain) {
        okt = mbar_wait(&barN, (c + 1) & 1, err);
        tc_fence_after();
        if (okt) n_epilogue();
        fence_proxy_async();
      }
      tc_fence_before();
      ok = __syncthreads_and(ok && okt);
      tc_fence_after();
    }
  }
  if (ok && chain && sr.s_out) {  // the final state, or the state handed to the next launch
#pragma unroll
    for (int v = 0; v < D; v += 4)
      *reinterpret_cast<float4*>(sr.s_out + st_off + v) = make_float4(S[v], S[v + 1], S[v + 2], S[v + 3]);
  }
  // on an error exit, let the loads that were issued land and the MMAs finish before the
  // CTA frees its tensor memory and leaves
  if (!ok && tid == 32)
    for (int c = confirmed; c < loaded; ++c) mbar_wait(&barL[c % 3], load_par(c), nullptr);
  if (tid == 0) {
    mma_commit(&barE);
    mbar_wait(&barE, 0, nullptr);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tslot, 512);
}

// ======================================================================================
// Backward (reverse over the chunks).  With dS' the gradient of the state leaving chunk c and
// everything transposed (TMEM lane = key index k):
//   dS_c^T = e^{G_C} dS'^T - ACC,   ACC = W^T dU_loc + Q^T (-scale e^G dO) + N dS'^T
//   dU_c^T = dU_loc^T + dS' K^T D                      (written out as a bf16 hi/lo pair)
// Per chunk, in tensor-pipe order:
//   N(c)     NT   = W^T (D K)                 M=128 k, N=128 k'', K=64 i   (4 instr)
//   dU(c)    DU   = dS' (D K)^T, hi + lo      M=128 v, N=64 i,   K=128 k   (16)
//   F(c)     ACC  = W^T dU_loc + Q^T O'       M=128 k, N=128 v,  K=64 i    (8)
//   chain(c) ACC += N (dS'^T hi + lo)         M=128 k, N=128 v,  K=128 k'' (16)
// The chain operand dS'^T is kept as a compensated bf16 pair (hi + lo) in shared memory.
// Shared memory: two slots of {K [64][128], W^T [128][64]} (the next chunk's loaded while this
// one is used), one of {Q [64][128], dO [64][128] (scaled to O' = -scale e^G dO in place),
// dU_loc^T [128][64]}, N bf16 [128 k][128 k''] (K-major A), dS'^T hi and lo [128 k''][128 v].
// Outputs: dh[c] = dS'^T ([k][v] bf16), dU^T hi/lo ([v][i] bf16), dh0 ([k][v] fp32).
// ======================================================================================
struct Bwd2Smem {
  static constexpr int KW = 0;                              // 2 x {K (2 x TILE64), W^T}
  static constexpr int KW_BYTES = 2 * TILE128;
  static constexpr int Q = 2 * KW_BYTES;                    // Q [64][128]
  static constexpr int O = Q + TILE128;                     // dO [64][128] -> O'
  static constexpr int UL = O + TILE128;                    // dU_loc^T [128][64]
  static constexpr int N = UL + TILE128;                    // N bf16 [128][128]
  static constexpr int DSH = N + 2 * TILE128;               // dS'^T hi [128][128]
  static constexpr int DSL = DSH + 2 * TILE128;             // dS'^T lo
  static constexpr int VEC = DSL + 2 * TILE128;             // 2 x {D[64], O' scale[64], e^{G_C}}
  static constexpr int TOTAL = VEC + 2 * 528;
};

__global__ void __launch_bounds__(256, 1) k_tc_scan_bwd2(Problem p, Args a, Work w, TcWork t,
                                                         const __grid_constant__ CUtensorMap mq,
                                                         const __grid_constant__ CUtensorMap mk,
                                                         const __grid_constant__ CUtensorMap mdO,
                                                         const __grid_constant__ CUtensorMap mWT,
                                                         const __grid_constant__ CUtensorMap mdUlT,
                                                         ScanRange sr) {
  // one read of the status word decides for the whole CTA (barriers below need every thread)
  __shared__ int s_fail;
  if (threadIdx.x == 0) s_fail = failed(w);
  __syncthreads();
  if (s_fail) return;
  const int n = blockIdx.x, hv = blockIdx.y, hk = hv / p.G;
  const int4 sq0 = w.seq_tab[n];
  // this launch's chunks of the sequence: [cb, cb + nc); sq = the sequence table entry with
  // its first chunk and token moved to cb
  const int cb = min(max(sr.c0, 0), sq0.y), nc = max(min(sr.c1, sq0.y) - cb, 0);
  const int4 sq = make_int4(sq0.x + cb, nc, sq0.z + 64 * cb, sq0.w - 64 * cb);
  const int tid = threadIdx.x, warp = tid / 32;
  const bool chain = tid < 128;
  const int row = tid & 127;  // TMEM lane of this thread's warp quarter: k' (chain) or v / k' (side)
  extern __shared__ unsigned char smraw[];
  unsigned char* sm = align1k(smraw);
  unsigned char* sQ = sm + Bwd2Smem::Q;
  unsigned char* sO = sm + Bwd2Smem::O;
  unsigned char* sUl = sm + Bwd2Smem::UL;
  unsigned char* sN = sm + Bwd2Smem::N;
  unsigned char* sDH = sm + Bwd2Smem::DSH;
  unsigned char* sDL = sm + Bwd2Smem::DSL;
  auto sK = [&](int c) { return sm + Bwd2Smem::KW + (c & 1) * Bwd2Smem::KW_BYTES; };
  auto sW = [&](int c) { return sK(c) + TILE128; };
  auto vec = [&](int c) { return reinterpret_cast<float*>(sm + Bwd2Smem::VEC + (c & 1) * 528); };
  __shared__ uint64_t barKW[2], barQOU, barN, barDU, barC, barE;
  __shared__ uint32_t tslot;
  int* err = w.status;
  if (tid == 0) {
    mbar_init(&barKW[0], 1);
    mbar_init(&barKW[1], 1);
    mbar_init(&barQOU, 1);
    mbar_init(&barN, 1);
    mbar_init(&barDU, 1);
    mbar_init(&barC, 1);
    mbar_init(&barE, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (warp == 0) {
    tmem_alloc(&tslot, 512);
    tmem_relinquish();
  }
  auto unit_row = [&](int c) { return ((sq.x + c) * p.HV + hv) * D; };
  auto chunk_len = [&](int c) { return min(64, sq.w - 64 * c); };
  auto tok_of = [&](int c) { return sq.z + 64 * c; };
  // chunk c is loaded in iteration order nc-1, nc-2, ...: its {K, W} are the j-th load into
  // slot c&1 with j = (nc-1-c)/2, and its {Q, dO, dU_loc} the (nc-1-c)-th into their slot
  auto kw_par = [&](int c) { return (uint32_t)(((nc - 1 - c) >> 1) & 1); };
  auto qou_par = [&](int c) { return (uint32_t)((nc - 1 - c) & 1); };
  auto issue_kw = [&](int c) {  // thread 32
    uint64_t* bar = &barKW[c & 1];
    mbar_expect_tx(bar, 2 * TILE128);
    tma_load_3d(sK(c), &mk, 0, hk, tok_of(c), bar);
    tma_load_3d(sK(c) + TILE64, &mk, 64, hk, tok_of(c), bar);
    tma_load_3d(sW(c), &mWT, 0, unit_row(c), 0, bar);
  };
  auto issue_qou = [&](int c) {  // thread 32
    mbar_expect_tx(&barQOU, 3 * TILE128);
    tma_load_3d(sQ, &mq, 0, hk, tok_of(c), &barQOU);
    tma_load_3d(sQ + TILE64, &mq, 64, hk, tok_of(c), &barQOU);
    tma_load_3d(sO, &mdO, 0, hv, tok_of(c), &barQOU);
    tma_load_3d(sO + TILE64, &mdO, 64, hv, tok_of(c), &barQOU);
    tma_load_3d(sUl, &mdUlT, 0, unit_row(c), 0, &barQOU);
  };
  auto load_vec = [&](int c) {  // side threads 0..63
    const int i = tid - 128, L = chunk_len(c);
    const size_t o = ((size_t)hv * p.NCmax + sq.x + c) * 64;
    float* v = vec(c);
    v[i] = i < L ? w.Dec[o + i] : 0.f;
    const float eg = w.EG[o + i];
    v[64 + i] = i < L ? -p.scale * eg : 0.f;
    if (i == 63) v[128] = eg;
  };
  // side group: rows of a [64][128] token tile (2 column blocks) times a per-row factor
  auto scale_rows = [&](unsigned char* tile, const float* f) {
    for (int idx = tid - 128; idx < 64 * 16; idx += 128) {
      const int r = idx >> 4, j = idx & 15;
      float x[8];
      ld_chunk_f(tile, r, j, TILE64, x);
      const float s = f[r];
#pragma unroll
      for (int q = 0; q < 8; ++q) x[q] *= s;
      st_chunk_f(tile, r, j, TILE64, x);
    }
  };
  int kw_issued = 0, qou_issued = 0;  // loads issued, in iteration order (same count in every thread)
  int kw_seen = 0, qou_seen = 0;      // loads every thread saw complete
  if (tid == 32 && nc > 0) {
    issue_kw(nc - 1);
    issue_qou(nc - 1);
  }
  if (nc > 0) kw_issued = qou_issued = 1;
  // thread k = row (chain warps) holds dS'^T[k][0..127] (the gradient leaving the range)
  float S[D];
  const size_t st_off = ((size_t)n * p.HV + hv) * D * D + (size_t)row * D;
  if (chain) {
#pragma unroll
    for (int v = 0; v < D; v += 4) {
      const float4 x = sr.s_in ? *reinterpret_cast<const float4*>(sr.s_in + st_off + v) : make_float4(0, 0, 0, 0);
      S[v] = x.x; S[v + 1] = x.y; S[v + 2] = x.z; S[v + 3] = x.w;
    }
  }
  // dS'^T rows as a compensated bf16 pair in shared memory; for a chunk of the sequence
  // (local index c >= -cb) also its dh (hi part)
  auto put_state = [&](int c) {
    bf16* hrow = c + cb >= 0 ? t.dh + ((size_t)unit_row(c) + row) * D : nullptr;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      float hi[8], lo[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        hi[q] = __bfloat162float(__float2bfloat16_rn(S[8 * j + q]));
        lo[q] = S[8 * j + q] - hi[q];
      }
      uint4 ph, pl;
      ph.x = pack_bf16(hi[0], hi[1]); ph.y = pack_bf16(hi[2], hi[3]);
      ph.z = pack_bf16(hi[4], hi[5]); ph.w = pack_bf16(hi[6], hi[7]);
      pl.x = pack_bf16(lo[0], lo[1]); pl.y = pack_bf16(lo[2], lo[3]);
      pl.z = pack_bf16(lo[4], lo[5]); pl.w = pack_bf16(lo[6], lo[7]);
      *reinterpret_cast<uint4*>(sDH + sw128_chunk(row, j, TILE128)) = ph;
      *reinterpret_cast<uint4*>(sDL + sw128_chunk(row, j, TILE128)) = pl;
      if (hrow) *reinterpret_cast<uint4*>(hrow + 8 * j) = ph;
    }
  };
  if (chain && nc > 0) put_state(nc - 1);
  if (!chain && tid - 128 < 64 && nc > 0) load_vec(nc - 1);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tslot;
  const uint32_t tACC = taddr(tb, 0, 0), tNT = taddr(tb, 0, 128), tDU = taddr(tb, 0, 256);
  bool ok = true;
  // prologue: the first chunk's K scaled by D
  if (nc > 0) {
    bool okp = true;
    if (!chain) {
      okp = mbar_wait(&barKW[(nc - 1) & 1], kw_par(nc - 1), err);
      if (okp) scale_rows(sK(nc - 1), vec(nc - 1));
      fence_proxy_async();
    }
    tc_fence_before();
    ok = __syncthreads_and(okp);
    tc_fence_after();
    if (ok) kw_seen = 1;
  }
  for (int idx = 0; ok && idx < nc; ++idx) {
    const int c = nc - 1 - idx;
    const bool more = c > 0;
    const float* vc = vec(c);
    bool okt = true;
    // A: N(c), dU(c); the next chunk's K and W stream into the other slot
    if (tid == 0) {
      const uint64_t dw = desc_kmajor(smem_u32(sW(c)), 0, TILE128);
      const uint64_t dkB = desc_mnmajor(smem_u32(sK(c)), 0, TILE64);
      constexpr uint32_t idN = idesc_bf16(128, 128, false, true);
#pragma unroll
      for (int s = 0; s < 4; ++s)  // N = W^T (D K)
        mma_bf16(tNT, dw + kstep_off(s, TILE128), dkB + mnstep_off(s), idN, s > 0);
      mma_commit(&barN);
      const uint64_t dkK = desc_kmajor(smem_u32(sK(c)), 0, TILE64);
      constexpr uint32_t idU = idesc_bf16(128, 64, true, false);
      for (int part = 0; part < 2; ++part) {
        const uint64_t da = desc_mnmajor(smem_u32(part ? sDL : sDH), 0, TILE128);
#pragma unroll
        for (int s = 0; s < 8; ++s)  // dU^T = dS' (D K)^T, hi then lo
          mma_bf16(tDU, da + mnstep_off(s), dkK + kstep_off(s, TILE64), idU, (part | s) > 0);
      }
      mma_commit(&barDU);
    }
    if (tid == 32 && more) issue_kw(c - 1);
    if (more) ++kw_issued;
    // B: O' = -scale e^G dO (side), -N in shared memory... N as the K-major A operand
    if (!chain) {
      okt = mbar_wait(&barQOU, qou_par(c), err);
      if (okt) scale_rows(sO, vc + 64);
      okt = okt && mbar_wait(&barN, idx & 1, err);
      tc_fence_after();
      if (okt) {
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          float x[32];
          tmem_ld16(taddr(tb, 32 * (warp - 4), 128 + 32 * cc), x);
          tmem_ld16(taddr(tb, 32 * (warp - 4), 128 + 32 * cc + 16), x + 16);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 4; ++j) st_chunk_f(sN, row, 4 * cc + j, TILE128, x + 8 * j);
        }
      }
      fence_proxy_async();
    }
    tc_fence_before();
    ok = __syncthreads_and(ok && okt);
    tc_fence_after();
    if (!ok) break;
    qou_seen = idx + 1;
    // C: F(c) then the chain product
    if (tid == 0) {
      const uint64_t dwA = desc_kmajor(smem_u32(sW(c)), 0, TILE128);
      const uint64_t dul = desc_kmajor(smem_u32(sUl), 0, TILE128);
      const uint64_t dq = desc_mnmajor(smem_u32(sQ), 0, TILE64);
      const uint64_t dO_ = desc_mnmajor(smem_u32(sO), 0, TILE64);
#pragma unroll
      for (int s = 0; s < 4; ++s)  // W^T dU_loc
        mma_bf16(tACC, dwA + kstep_off(s, TILE128), dul + kstep_off(s, TILE128),
                 idesc_bf16(128, 128, false, false), s > 0);
#pragma unroll
      for (int s = 0; s < 4; ++s)  // + Q^T O'
        mma_bf16(tACC, dq + mnstep_off(s), dO_ + mnstep_off(s), idesc_bf16(128, 128, true, true), 1);
      const uint64_t dn = desc_kmajor(smem_u32(sN), 0, TILE128);
      for (int part = 0; part < 2; ++part) {
        const uint64_t db = desc_mnmajor(smem_u32(part ? sDL : sDH), 0, TILE128);
#pragma unroll
        for (int s = 0; s < 8; ++s)  // + N dS'^T, hi then lo
          mma_bf16(tACC, dn + kstep_off(s, TILE128), db + mnstep_off(s), idesc_bf16(128, 128, false, true), 1);
      }
      mma_commit(&barC);
    }
    if (chain) {
      // E: dS_c^T = e^{G_C} dS'^T - ACC
      okt = mbar_wait(&barC, idx & 1, err);
      tc_fence_after();
      if (okt) {
        const float egc = vc[128];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          float x[32];
          tmem_ld16(taddr(tb, 32 * warp, 32 * cc), x);
          tmem_ld16(taddr(tb, 32 * warp, 32 * cc + 16), x + 16);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 32; ++q) S[32 * cc + q] = egc * S[32 * cc + q] - x[q];
        }
        put_state(c - 1);  // dh[c-1] = the state gradient leaving chunk c-1 (none before the sequence)
      }
      fence_proxy_async();
    } else {
      // D: dU^T = dU_loc^T + DU as a hi/lo pair (rows v), straight to the workspace
      okt = mbar_wait(&barDU, idx & 1, err);
      tc_fence_after();
      if (okt) {
        bf16* hrow = t.dUT + ((size_t)unit_row(c) + row) * 64;
        bf16* lrow = t.dUTl + ((size_t)unit_row(c) + row) * 64;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          float x[32];
          tmem_ld16(taddr(tb, 32 * (warp - 4), 256 + 32 * h2), x);
          tmem_ld16(taddr(tb, 32 * (warp - 4), 256 + 32 * h2 + 16), x + 16);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float f[8], hi[8], lo[8];
            ld_chunk_f(sUl, row, 4 * h2 + j, TILE128, f);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float y = f[q] + x[8 * j + q];
              hi[q] = __bfloat162float(__float2bfloat16_rn(y));
              lo[q] = y - hi[q];
            }
            uint4 ph, pl;
            ph.x = pack_bf16(hi[0], hi[1]); ph.y = pack_bf16(hi[2], hi[3]);
            ph.z = pack_bf16(hi[4], hi[5]); ph.w = pack_bf16(hi[6], hi[7]);
            pl.x = pack_bf16(lo[0], lo[1]); pl.y = pack_bf16(lo[2], lo[3]);
            pl.z = pack_bf16(lo[4], lo[5]); pl.w = pack_bf16(lo[6], lo[7]);
            *reinterpret_cast<uint4*>(hrow + 8 * (4 * h2 + j)) = ph;
            *reinterpret_cast<uint4*>(lrow + 8 * (4 * h2 + j)) = pl;
          }
        }
      }
      if (more) {
        if (tid - 128 < 64) load_vec(c - 1);
        bar_sync_side();
        okt = okt && mbar_wait(&barKW[(c - 1) & 1], kw_par(c - 1), err);
        if (okt) scale_rows(sK(c - 1), vec(c - 1));
        fence_proxy_async();
      }
    }
    tc_fence_before();
    ok = __syncthreads_and(ok && okt);
    tc_fence_after();
    if (!ok) break;
    if (more) kw_seen = idx + 2;
    // F: Q, dO and dU_loc of this chunk are no longer read
    if (more) {
      if (tid == 32) issue_qou(c - 1);
      ++qou_issued;
    }
  }
  if (ok && chain && sr.s_out) {  // dh0, or the gradient handed to the launch of earlier chunks
#pragma unroll
    for (int v = 0; v < D; v += 4)
      *reinterpret_cast<float4*>(sr.s_out + st_off + v) = make_float4(S[v], S[v + 1], S[v + 2], S[v + 3]);
  }
  if (!ok && tid == 32) {  // let issued loads land before the CTA leaves
    for (int j = kw_seen; j < kw_issued; ++j) mbar_wait(&barKW[(nc - 1 - j) & 1], kw_par(nc - 1 - j), nullptr);
    for (int j = qou_seen; j < qou_issued; ++j) mbar_wait(&barQOU, qou_par(nc - 1 - j), nullptr);
  }
  if (tid == 0) {
    mma_commit(&barE);
    mbar_wait(&barE, 0, nullptr);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tslot, 512);
}

}  // namespace

cudaError_t tc_scan_fwd(const Problem& p, const Args& a, const Work& w, const TcWork& t,
                        const TcMaps& m, const ScanRange& sr, cudaStream_t s) {
  const dim3 grid(p.Nst, p.HV);
  return tgo("tc_scan_fwd", k_tc_scan_fwd2, grid, 256, (size_t)1024 + Fwd2Smem::TOTAL, s, p, a, w, t,
             m.k, m.WT, m.UtT, sr);
}

cudaError_t tc_scan_bwd(const Problem& p, const Args& a, const Work& w, const TcWork& t,
                        const TcMaps& m, const ScanRange& sr, cudaStream_t s) {
  const dim3 grid(p.Nst, p.HV);
  return tgo("tc_scan_bwd", k_tc_scan_bwd2, grid, 256, (size_t)1024 + Bwd2Smem::TOTAL, s, p, a, w, t,
             m.q, m.k, m.dO, m.WT, m.dUlT, sr);
}

}  // namespace tcx
}  // namespace gdn
