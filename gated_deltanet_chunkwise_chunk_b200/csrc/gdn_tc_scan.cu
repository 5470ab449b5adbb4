// Sequential state passes over the chunks (chunk_delta_h forward and the backward dhu pass of
// the G_T_CONTIG page), one CTA per (sequence, value head) carrying the whole 128 x 128 state.
//
// The chunk step is affine in the state.  With D = diag(e^{G_C - G_i}) (zero past the chunk's
// last token), W and U~ the chunk's WY factors and K its keys:
//   forward    S' = e^{G_C} S + U^T D K,  U = U~ - W S^T
//              = e^{G_C} S + B - S N,     N = W^T D K (K x K),  B = U~^T D K (V x K)
//   backward   dS = e^{G_C} dS' + scale (e^G dO)^T Q - dU^T W,  dU = dU_loc + D K dS'^T
//              = e^{G_C} dS' - (W^T dU_loc - scale Q^T e^G dO + N dS'^T)^T
// N and B (and the backward's state-free terms) do not depend on the state, so they are built
// off the chain (N by the WY kernel); the chain itself is one tensor-core product per chunk
// (S N) instead of two dependent ones (W S^T, then U^T D K).  Everything is kept transposed so
// that TMEM lane = key index k: the state S^T [k][v] is held in fp32 registers by 16 state
// warps, four threads per row k (32 values each), and its bf16 copy that feeds the next product
// is written row by row; a 17th warp issues the MMAs, the loads and the bulk stores.
#include "gdn_tc_common.cuh"

namespace gdn {
namespace tcx {

namespace {

// ======================================================================================
// Forward.  Warps 0..15 hold the state: warp w, lane l has TMEM lane quarter q = w & 3,
// row = 32q + l, column group cg = w >> 2 (32 state columns).  Warp 16 is the control warp:
// its lane 0 issues every MMA, load and bulk store, so that a thread blocked in issuing
// tensor-core instructions never delays the state update.  -N^T comes ready from the WY kernel, so per chunk c the tensor pipe runs
//   chain(c)  ACC[c&1] += (-N_c^T) S_c^T       M=128 k', N=128 v, K=128 k   (8 instr)
//   B(c+1)    ACC[~]    = (D K)^T U~           M=128 k', N=128 v, K=64 i    (4)
// State warps: wait for chain(c), update S, write its bf16 copy (the next chain operand) and sync
// on named barrier 1 with the control warp, which then issues the next chain product and stores
// the tile as h with a bulk copy (per-thread stores of rows 256 bytes apart cost more than the
// whole chain product).
// Every thread of the CTA takes part in every round of that barrier (a blocking sync, also on
// the error path), so no warp can reach a round early.
// (v_new = U~ - W S^T is left to the output kernel, which reads S anyway.)
// Shared memory: three input stages {U~^T [128][64], -N^T [128][128], D K [64][128]} with
// e^{G_i}, and S^T bf16 [128 k][128 v] (MN-major B of the chain).
// ======================================================================================
constexpr int kStateThreads = 512;
constexpr int kScanThreadsWS = kStateThreads + 32;

struct Fwd2Smem {
  static constexpr int UT = 0, NT = TILE128, DK = 3 * TILE128;   // within a stage
  static constexpr int STAGE = 4 * TILE128;
  static constexpr int S = 3 * STAGE;
  static constexpr int VEC = S + 2 * TILE128;               // 3 x {(unused)[64], e^G[64]}
  static constexpr int TOTAL = VEC + 3 * 512;
};
static_assert(1024 + Fwd2Smem::TOTAL + 256 <= 227 * 1024, "forward pass shared memory");

__global__ void __launch_bounds__(kScanThreadsWS, 1) k_tc_scan_fwd2(
    Problem p, Args a, Work w, TcWork t, const __grid_constant__ CUtensorMap mDK,
    const __grid_constant__ CUtensorMap mNT, const __grid_constant__ CUtensorMap mUtT,
    const __grid_constant__ CUtensorMap mh, ScanRange sr) {
  // one read of the status word decides for the whole CTA (barriers below need every thread)
  __shared__ int s_fail;
  if (threadIdx.x == 0) s_fail = failed(w);
  __syncthreads();
  if (s_fail) return;
  const int n = blockIdx.x, hv = blockIdx.y;
  const int4 sq0 = w.seq_tab[n];
  // this launch's chunks of the sequence: [cb, cb + nc); sq = the sequence table entry with
  // its first chunk and token moved to cb
  const int cb = min(max(sr.c0, 0), sq0.y), nc = max(min(sr.c1, sq0.y) - cb, 0);
  const int4 sq = make_int4(sq0.x + cb, nc, sq0.z + 64 * cb, sq0.w - 64 * cb);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const bool ctl = warp == kStateThreads / 32;
  const int qd = warp & 3, cg = (warp >> 2) & 3, row = 32 * qd + lane;
  extern __shared__ unsigned char smraw[];
  unsigned char* sm = align1k(smraw);
  unsigned char* sS = sm + Fwd2Smem::S;
  auto stage = [&](int c) { return sm + (c % 3) * Fwd2Smem::STAGE; };
  auto vecp = [&](int c) { return reinterpret_cast<float*>(sm + Fwd2Smem::VEC + (c % 3) * 512); };
  // barH: the bulk store of h[c] has read the S^T tile (the state warps may rewrite it)
  __shared__ uint64_t barL[3], barC, barH, barE;
  __shared__ uint32_t tslot;
  __shared__ volatile int s_abort;
  int* err = w.status;
  // the test flag withholds the first chain product; its wait then runs out quickly
  const long long wait_limit = p.test_timeout ? (1ll << 20) : (1ll << 31);
  if (tid == 0) {
    for (int i = 0; i < 3; ++i) mbar_init(&barL[i], 1);
    mbar_init(&barC, 1);
    mbar_init(&barH, 1);
    mbar_init(&barE, 1);
    s_abort = 0;
    mbar_fence_init();
  }
  __syncthreads();
  if (warp == 0) {
    tmem_alloc(&tslot, 512);
    tmem_relinquish();
  }
  auto unit_row = [&](int c) { return ((sq.x + c) * p.HV + hv) * D; };
  // control lane: chunk c's tiles (U~^T, -N^T and D K, written by the WY kernel) and e^{G_i}
  int loaded = 0;  // chunks whose loads were issued, in order 0, 1, 2, ... (control lane)
  auto issue_load = [&](int c) {
    unsigned char* b = stage(c);
    uint64_t* bar = &barL[c % 3];
    const int r = unit_row(c);
    const size_t o = ((size_t)hv * p.NCmax + sq.x + c) * 64;
    mbar_expect_tx(bar, 4 * TILE128 + 256);
    tma_load_3d(b + Fwd2Smem::UT, &mUtT, 0, r, 0, bar);
    tma_load_3d(b + Fwd2Smem::NT, &mNT, 0, r, 0, bar);
    tma_load_3d(b + Fwd2Smem::NT + TILE128, &mNT, 64, r, 0, bar);
    tma_load_3d(b + Fwd2Smem::DK, &mDK, 0, r / 2, 0, bar);
    tma_load_3d(b + Fwd2Smem::DK + TILE64, &mDK, 64, r / 2, 0, bar);
    bulk_load(vecp(c) + 64, w.EG + o, 256, bar);
    ++loaded;
  };
  // chunk c is the (c/3)-th load into stage c%3: its barrier phase has parity (c/3)&1
  auto load_par = [](int c) { return (uint32_t)((c / 3) & 1); };
  const bool issuer = tid == kStateThreads;
  if (issuer)
    for (int c = 0; c < min(3, nc); ++c) issue_load(c);
  // this thread's part of S^T: row `row`, columns 32 cg .. 32 cg + 31
  float S[32];
  // states are [Nst][HV][K][V]; rows k >= K and columns v >= V of a narrower head are padding
  const bool st_live = !ctl && row < p.K && 32 * cg < p.V;
  const size_t st_off = (((size_t)n * p.HV + hv) * p.K + row) * p.V + 32 * cg;
#pragma unroll
  for (int v = 0; v < 32; v += 4) {
    const float4 x = (sr.s_in && st_live) ? *reinterpret_cast<const float4*>(sr.s_in + st_off + v)
                                          : make_float4(0, 0, 0, 0);
    S[v] = x.x; S[v + 1] = x.y; S[v + 2] = x.z; S[v + 3] = x.w;
  }
  // S^T entering a chunk (this thread's row part) as bf16: the chain operand tile (stored as h)
  auto put_state = [&]() {
#pragma unroll
    for (int j = 0; j < 4; ++j) st_chunk_f(sS, row, 4 * cg + j, TILE128, S + 8 * j);
  };
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tslot;
  const uint32_t tACC0 = taddr(tb, 0, 0);
  if (ctl) {
    // B(c) = (D K)^T U~ into ACC[c&1] (K of chunk c already scaled by D)
    auto issue_b = [&](int c) {
      unsigned char* b = stage(c);
      const uint64_t dk = desc_mnmajor(smem_u32(b + Fwd2Smem::DK), 0, TILE64);
      const uint64_t du = desc_kmajor(smem_u32(b + Fwd2Smem::UT), 0, TILE128);
      const uint32_t tacc = tACC0 + (uint32_t)(128 * (c & 1));
#pragma unroll
      for (int s = 0; s < 4; ++s)
        mma_bf16(tacc, dk + mnstep_off(s), du + kstep_off(s, TILE128), idesc_bf16(128, 128, true, false), s > 0);
    };
    if (issuer && nc > 0 && mbar_wait_abort(&barL[0], load_par(0), err, &s_abort)) issue_b(0);
    for (int c = 0; c < nc; ++c) {
      nbar_sync(1, kScanThreadsWS);  // S_c^T is in shared memory (the whole warp syncs)
      if (issuer && !s_abort) {
        tc_fence_after();
        tma_store_3d(&mh, sS, 0, unit_row(c), 0);  // h[c]
        tma_store_3d(&mh, sS + TILE128, 64, unit_row(c), 0);
        tma_store_commit();
        if (!(p.test_timeout && c == 0)) {  // the test flag withholds the first chain product
          const uint64_t da = desc_kmajor(smem_u32(stage(c) + Fwd2Smem::NT), 0, TILE128);
          const uint64_t dsB = desc_mnmajor(smem_u32(sS), 0, TILE128);
          const uint32_t tacc = tACC0 + (uint32_t)(128 * (c & 1));
#pragma unroll
          for (int s = 0; s < 8; ++s)  // chain: ACC += (-N^T) S^T
            mma_bf16(tacc, da + kstep_off(s, TILE128), dsB + mnstep_off(s), idesc_bf16(128, 128, false, true), 1);
          mma_commit(&barC);
        }
        if (c + 1 < nc) {  // the S^T tile is free once the store has read it
          tma_store_wait_read0();
          mbar_arrive(&barH);
        }
        if (c + 1 < nc && mbar_wait_abort(&barL[(c + 1) % 3], load_par(c + 1), err, &s_abort)) issue_b(c + 1);
        // stage c%3 (read by B(c) and chain(c)) refills with chunk c+3
        if (c + 3 < nc && mbar_wait_abort(&barC, c & 1, err, &s_abort)) issue_load(c + 3);
      }
    }
  } else if (nc > 0) {
    // state warps: e^{G_C} of the next chunk is read before the barrier round (its stage is
    // refilled only after the chain product that round releases)
    float egc = 0.f;
    if (mbar_wait_abort(&barL[0], load_par(0), err, &s_abort)) egc = vecp(0)[64 + 63];
    put_state();
    fence_proxy_async();
    tc_fence_before();
    nbar_sync(1, kScanThreadsWS);
    for (int c = 0; c < nc; ++c) {
      // S_{c+1}^T = e^{G_C} S_c^T + ACC
      bool okt = !s_abort && mbar_wait_abort(&barC, c & 1, err, &s_abort, wait_limit);
      tc_fence_after();
      if (okt) {
        float x[32];
        tmem_ld16(taddr(tb, 32 * qd, 128 * (c & 1) + 32 * cg), x);
        tmem_ld16(taddr(tb, 32 * qd, 128 * (c & 1) + 32 * cg + 16), x + 16);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 32; ++q) S[q] = egc * S[q] + x[q];
      }
      if (c + 1 < nc) {
        okt = okt && mbar_wait_abort(&barL[(c + 1) % 3], load_par(c + 1), err, &s_abort);
        if (okt) egc = vecp(c + 1)[64 + 63];
        okt = okt && mbar_wait_abort(&barH, c & 1, err, &s_abort);
        if (okt) put_state();
        fence_proxy_async();
        tc_fence_before();
        nbar_sync(1, kScanThreadsWS);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  const bool ok = !s_abort;
  if (ok && sr.s_out && st_live) {  // the final state, or the state handed to the next launch
#pragma unroll
    for (int v = 0; v < 32; v += 4)
      *reinterpret_cast<float4*>(sr.s_out + st_off + v) = make_float4(S[v], S[v + 1], S[v + 2], S[v + 3]);
  }
  // before the CTA leaves (after an error too): the last load into each stage has landed, so
  // every earlier one has; every MMA issued has finished
  if (issuer) {
    for (int b = 0; b < 3; ++b)  // stage b's last load was its ((loaded - 1 - b) / 3)-th
      if (loaded > b) mbar_wait(&barL[b], (uint32_t)(((loaded - 1 - b) / 3) & 1), nullptr);
    tma_store_wait0();
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
//   dS_c^T = e^{G_C} dS'^T - ACC,   ACC = W^T dU_loc + Q^T O' + N dS'^T,  O' = -scale e^G dO
//   dU_c^T = dU_loc^T + dS' K^T D                      (written out as a bf16 hi/lo pair)
// -N^T comes ready from the WY kernel (read here as an MN-major A operand with the negate bit
// set), O' from dv_local.  Roles as in the forward pass: warps 0..15 hold dS', warp 16's lane 0
// issues every MMA and load.  Per chunk, in tensor-pipe order:
//   chain(c)  ACC[c&1] += N (dS'^T hi + lo)       M=128 k, N=128 v, K=128 k''  (16 instr)
//   dU(c)     DU[c&1]  += dS' (D K)^T, hi + lo    M=128 v, N=64 i,  K=128 k    (16)
//   I(c-1)    DU[~]     = dU_loc^T I              M=128 v, N=64 i,  K=64 i'    (4)
//   F(c-1)    ACC[~]    = W^T dU_loc + Q^T O'     M=128 k, N=128 v, K=64 i     (8)
// The state-free products of the next chunk go in behind this chunk's, into the other
// accumulators, so the pipe keeps working while the state is updated and written back.  dh
// (the hi tile of dS') and dU^T (staged by the state warps in the -N^T slot its chain product
// has finished with) leave by bulk copies the control lane issues after the barrier.
// Shared memory: two slots of -N^T [128][128] with e^{G_i}; one of D K [64][128]; one of
// {Q [64][128], O' [64][128], W^T [128][64], dU_loc^T [128][64]}; dS'^T hi and lo [128][128];
// the 64 x 64 identity.
// ======================================================================================
struct Bwd2Smem {
  static constexpr int NS = 0;                              // 2 x -N^T (two 64-column boxes)
  static constexpr int DK = 4 * TILE128;
  static constexpr int Q = DK + TILE128;
  static constexpr int O = Q + TILE128;
  static constexpr int W = O + TILE128;
  static constexpr int UL = W + TILE128;
  static constexpr int DSH = UL + TILE128;
  static constexpr int DSL = DSH + 2 * TILE128;
  static constexpr int ID = DSL + 2 * TILE128;              // identity [64][64] bf16
  static constexpr int VEC = ID + TILE64;                   // 2 x e^G[64]
  static constexpr int TOTAL = VEC + 2 * 256;
};
static_assert(1024 + Bwd2Smem::TOTAL + 256 <= 227 * 1024, "backward pass shared memory");

__global__ void __launch_bounds__(kScanThreadsWS, 1) k_tc_scan_bwd2(
    Problem p, Args a, Work w, TcWork t, const __grid_constant__ CUtensorMap mq,
    const __grid_constant__ CUtensorMap mDK, const __grid_constant__ CUtensorMap mOp,
    const __grid_constant__ CUtensorMap mWT, const __grid_constant__ CUtensorMap mdUlT,
    const __grid_constant__ CUtensorMap mNT, const __grid_constant__ CUtensorMap mdh,
    const __grid_constant__ CUtensorMap mdUT, const __grid_constant__ CUtensorMap mdUTl, ScanRange sr) {
  __shared__ int s_fail;
  if (threadIdx.x == 0) s_fail = failed(w);
  __syncthreads();
  if (s_fail) return;
  const int n = blockIdx.x, hv = blockIdx.y, hk = hv / p.G;
  const int4 sq0 = w.seq_tab[n];
  const int cb = min(max(sr.c0, 0), sq0.y), nc = max(min(sr.c1, sq0.y) - cb, 0);
  const int4 sq = make_int4(sq0.x + cb, nc, sq0.z + 64 * cb, sq0.w - 64 * cb);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const bool ctl = warp == kStateThreads / 32, issuer = tid == kStateThreads;
  const int qd = warp & 3, cg = (warp >> 2) & 3, row = 32 * qd + lane;
  extern __shared__ unsigned char smraw[];
  unsigned char* sm = align1k(smraw);
  unsigned char* sDKt = sm + Bwd2Smem::DK;
  unsigned char* sQ = sm + Bwd2Smem::Q;
  unsigned char* sO = sm + Bwd2Smem::O;
  unsigned char* sW = sm + Bwd2Smem::W;
  unsigned char* sUl = sm + Bwd2Smem::UL;
  unsigned char* sDH = sm + Bwd2Smem::DSH;
  unsigned char* sDL = sm + Bwd2Smem::DSL;
  unsigned char* sI = sm + Bwd2Smem::ID;
  auto sN = [&](int c) { return sm + Bwd2Smem::NS + (c & 1) * 2 * TILE128; };
  auto vecp = [&](int c) { return reinterpret_cast<float*>(sm + Bwd2Smem::VEC + (c & 1) * 256); };
  // barH: the bulk stores issued after a barrier round have read dS'^T hi and the dU^T staging
  __shared__ uint64_t barN[2], barDK, barQ, barF, barC, barDU, barH, barE;
  __shared__ uint32_t tslot;
  __shared__ volatile int s_abort;
  int* err = w.status;
  if (tid == 0) {
    mbar_init(&barH, 1);
    mbar_init(&barN[0], 1);
    mbar_init(&barN[1], 1);
    mbar_init(&barDK, 1);
    mbar_init(&barQ, 1);
    mbar_init(&barF, 1);
    mbar_init(&barC, 1);
    mbar_init(&barDU, 1);
    mbar_init(&barE, 1);
    s_abort = 0;
    mbar_fence_init();
  }
  __syncthreads();
  if (warp == 0) {
    tmem_alloc(&tslot, 512);
    tmem_relinquish();
  }
  auto unit_row = [&](int c) { return ((sq.x + c) * p.HV + hv) * D; };
  auto tok_of = [&](int c) { return sq.z + 64 * c; };
  // Chunks go in iteration order nc-1, nc-2, ...  A single-slot barrier (D K; Q, O', W, dU_loc;
  // and the commit barriers) completes its j-th phase for chunk nc-1-j; the -N^T slot c&1
  // completes its j-th phase for chunk nc-1-2j-((nc-1-c)&1).
  auto par = [&](int c) { return (uint32_t)((nc - 1 - c) & 1); };
  auto npar = [&](int c) { return (uint32_t)(((nc - 1 - c) >> 1) & 1); };
  // loads issued per barrier (control lane): on the way out it waits for the last one of each
  int n_iss0 = 0, n_iss1 = 0, dk_iss = 0, q_iss = 0;
  auto issue_n = [&](int c) {  // chunk c's -N^T and e^{G_i}
    uint64_t* bar = &barN[c & 1];
    const size_t o = ((size_t)hv * p.NCmax + sq.x + c) * 64;
    mbar_expect_tx(bar, 2 * TILE128 + 256);
    tma_load_3d(sN(c), &mNT, 0, unit_row(c), 0, bar);
    tma_load_3d(sN(c) + TILE128, &mNT, 64, unit_row(c), 0, bar);
    bulk_load(vecp(c), w.EG + o, 256, bar);
    if (c & 1) ++n_iss1; else ++n_iss0;
  };
  auto issue_dk = [&](int c) {
    mbar_expect_tx(&barDK, TILE128);
    tma_load_3d(sDKt, &mDK, 0, unit_row(c) / 2, 0, &barDK);
    tma_load_3d(sDKt + TILE64, &mDK, 64, unit_row(c) / 2, 0, &barDK);
    ++dk_iss;
  };
  // chunk c's Q, O' = -scale e^G dO (the dv_local kernel's), W^T and dU_loc^T
  auto issue_q = [&](int c) {
    mbar_expect_tx(&barQ, 4 * TILE128);
    tma_load_3d(sQ, &mq, 0, hk, tok_of(c), &barQ);
    tma_load_3d(sQ + TILE64, &mq, 64, hk, tok_of(c), &barQ);
    tma_load_3d(sO, &mOp, 0, unit_row(c) / 2, 0, &barQ);
    tma_load_3d(sO + TILE64, &mOp, 64, unit_row(c) / 2, 0, &barQ);
    tma_load_3d(sW, &mWT, 0, unit_row(c), 0, &barQ);
    tma_load_3d(sUl, &mdUlT, 0, unit_row(c), 0, &barQ);
    ++q_iss;
  };
  if (issuer && nc > 0) {
    issue_n(nc - 1);
    issue_dk(nc - 1);
    issue_q(nc - 1);
  }
  // this thread's part of dS'^T: row `row`, columns 32 cg .. 32 cg + 31
  float S[32];
  // states are [Nst][HV][K][V]; rows k >= K and columns v >= V of a narrower head are padding
  const bool st_live = !ctl && row < p.K && 32 * cg < p.V;
  const size_t st_off = (((size_t)n * p.HV + hv) * p.K + row) * p.V + 32 * cg;
#pragma unroll
  for (int v = 0; v < 32; v += 4) {
    const float4 x = (sr.s_in && st_live) ? *reinterpret_cast<const float4*>(sr.s_in + st_off + v)
                                          : make_float4(0, 0, 0, 0);
    S[v] = x.x; S[v + 1] = x.y; S[v + 2] = x.z; S[v + 3] = x.w;
  }
  if (!ctl) {  // the 64 x 64 identity (bf16), one 16-byte chunk per state thread
    const int r = tid >> 3, j = tid & 7;
    float f[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) f[q] = (8 * j + q == r) ? 1.f : 0.f;
    st_chunk_f(sI, r, j, TILE64, f);
  }
  // dS'^T leaving a chunk (this thread's row part) as a compensated bf16 pair for the next
  // products; the hi tile is also dh
  auto put_state = [&]() {
#pragma unroll
    for (int j = 0; j < 4; ++j) st_chunk_split(sDH, sDL, row, 4 * cg + j, TILE128, S + 8 * j);
  };
  fence_proxy_async();  // the identity, before any product reads it
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tslot;
  auto tACC = [&](int c) { return taddr(tb, 0, 128 * (c & 1)); };
  auto tDU = [&](int c) { return taddr(tb, 0, 256 + 64 * (c & 1)); };
  if (ctl) {
    // I(c) and F(c): the state-free products of chunk c
    auto issue_if = [&](int c) {
      const uint64_t dul = desc_kmajor(smem_u32(sUl), 0, TILE128);
      const uint64_t di = desc_kmajor(smem_u32(sI), 0, TILE64);
      const uint64_t dwA = desc_kmajor(smem_u32(sW), 0, TILE128);
      const uint64_t dq = desc_mnmajor(smem_u32(sQ), 0, TILE64);
      const uint64_t dO_ = desc_mnmajor(smem_u32(sO), 0, TILE64);
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        mma_bf16(tDU(c), dul + kstep_off(s, TILE128), di + kstep_off(s, TILE64), idesc_bf16(128, 64, false, false), s > 0);
        mma_bf16(tACC(c), dwA + kstep_off(s, TILE128), dul + kstep_off(s, TILE128),
                 idesc_bf16(128, 128, false, false), s > 0);
      }
#pragma unroll
      for (int s = 0; s < 4; ++s)
        mma_bf16(tACC(c), dq + mnstep_off(s), dO_ + mnstep_off(s), idesc_bf16(128, 128, true, true), 1);
      mma_commit(&barF);
    };
    if (issuer && nc > 0 && mbar_wait_abort(&barQ, par(nc - 1), err, &s_abort)) issue_if(nc - 1);
    // the chain's A operand: -N^T read MN-major is -N; the negate bit makes it N
    constexpr uint32_t kNegA = 1u << 13;
    for (int idx = 0; idx < nc; ++idx) {
      const int c = nc - 1 - idx;
      nbar_sync(1, kScanThreadsWS);  // dS'_c^T is in shared memory (the whole warp syncs)
      if (!issuer || s_abort) continue;
      tc_fence_after();
      const uint64_t dah = desc_mnmajor(smem_u32(sDH), 0, TILE128);
      const uint64_t dal = desc_mnmajor(smem_u32(sDL), 0, TILE128);
      // dh[c] = the hi tile; dU^T of chunk c+1, staged in its -N^T slot
      tma_store_3d(&mdh, sDH, 0, unit_row(c), 0);
      tma_store_3d(&mdh, sDH + TILE128, 64, unit_row(c), 0);
      if (c + 1 < nc) {
        tma_store_3d(&mdUT, sN(c + 1), 0, unit_row(c + 1), 0);
        tma_store_3d(&mdUTl, sN(c + 1) + TILE128, 0, unit_row(c + 1), 0);
      }
      tma_store_commit();
      if (!mbar_wait_abort(&barN[c & 1], npar(c), err, &s_abort)) continue;
      {
        const uint64_t dn = desc_mnmajor(smem_u32(sN(c)), 0, TILE128);
        constexpr uint32_t idC = idesc_bf16(128, 128, true, true) | kNegA;
#pragma unroll
        for (int s = 0; s < 8; ++s) mma_bf16(tACC(c), dn + mnstep_off(s), dah + mnstep_off(s), idC, 1);
#pragma unroll
        for (int s = 0; s < 8; ++s) mma_bf16(tACC(c), dn + mnstep_off(s), dal + mnstep_off(s), idC, 1);
        mma_commit(&barC);
      }
      // chunk c's F and I have run: chunk c-1's Q, O', W, dU_loc replace theirs
      if (c > 0) {
        if (!mbar_wait_abort(&barF, par(c), err, &s_abort)) continue;
        issue_q(c - 1);
      }
      if (!mbar_wait_abort(&barDK, par(c), err, &s_abort)) continue;
      {
        const uint64_t dkK = desc_kmajor(smem_u32(sDKt), 0, TILE64);
        constexpr uint32_t idU = idesc_bf16(128, 64, true, false);
#pragma unroll
        for (int s = 0; s < 8; ++s) mma_bf16(tDU(c), dah + mnstep_off(s), dkK + kstep_off(s, TILE64), idU, 1);
#pragma unroll
        for (int s = 0; s < 8; ++s) mma_bf16(tDU(c), dal + mnstep_off(s), dkK + kstep_off(s, TILE64), idU, 1);
        mma_commit(&barDU);
      }
      // once the stores have read them: dS'^T may be rewritten, and the slot of chunk c+1 (its
      // chain product finished before the state warps released dS'_c) takes chunk c-1's -N^T
      tma_store_wait_read0();
      mbar_arrive(&barH);
      if (c == 0) continue;
      issue_n(c - 1);
      // the previous chunk's state-free products go in behind this chunk's; D K is replaced
      // once dU(c) has read it
      if (!mbar_wait_abort(&barQ, par(c - 1), err, &s_abort)) continue;
      issue_if(c - 1);
      if (mbar_wait_abort(&barDU, par(c), err, &s_abort)) issue_dk(c - 1);
    }
  } else if (nc > 0) {
    // state warps: e^{G_C} of a chunk is read before the barrier round that releases its chain
    // product (its -N^T slot is refilled only after that product)
    float egc = 0.f;
    if (mbar_wait_abort(&barN[(nc - 1) & 1], npar(nc - 1), err, &s_abort)) egc = vecp(nc - 1)[63];
    put_state();
    fence_proxy_async();
    tc_fence_before();
    nbar_sync(1, kScanThreadsWS);
    for (int idx = 0; idx < nc; ++idx) {
      const int c = nc - 1 - idx;
      const bool more = c > 0;
      // (1) dS_c^T = e^{G_C} dS'^T - ACC
      bool okt = !s_abort && mbar_wait_abort(&barC, par(c), err, &s_abort);
      tc_fence_after();
      if (okt) {
        float x[32];
        tmem_ld16(taddr(tb, 32 * qd, 128 * (c & 1) + 32 * cg), x);
        tmem_ld16(taddr(tb, 32 * qd, 128 * (c & 1) + 32 * cg + 16), x + 16);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 32; ++q) S[q] = egc * S[q] - x[q];
      }
      // (2) dU^T = DU as a hi/lo pair (rows v, 16 columns per thread), straight to the workspace
      okt = okt && mbar_wait_abort(&barDU, par(c), err, &s_abort);
      tc_fence_after();
      if (okt) {  // staged as two [128 v][64 i] tiles in chunk c's -N^T slot (chain(c) is done)
        float x[16];
        tmem_ld16(taddr(tb, 32 * qd, 256 + 64 * (c & 1) + 16 * cg), x);
        tmem_wait_ld();
        st_chunk_split(sN(c), sN(c) + TILE128, row, 2 * cg, TILE128, x);
        st_chunk_split(sN(c), sN(c) + TILE128, row, 2 * cg + 1, TILE128, x + 8);
      }
      if (more) {
        // (3) both products of chunk c have read dS'^T: the next one (and dh[c-1]) replaces it
        okt = okt && mbar_wait_abort(&barN[(c - 1) & 1], npar(c - 1), err, &s_abort);
        if (okt) egc = vecp(c - 1)[63];
        okt = okt && mbar_wait_abort(&barH, par(c), err, &s_abort);
        if (okt) put_state();
        fence_proxy_async();
        tc_fence_before();
        nbar_sync(1, kScanThreadsWS);
      } else {
        fence_proxy_async();  // the last dU^T staging, stored after the final barrier
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (!s_abort && sr.s_out && st_live) {  // dh0, or the gradient handed to the launch of earlier chunks
#pragma unroll
    for (int v = 0; v < 32; v += 4)
      *reinterpret_cast<float4*>(sr.s_out + st_off + v) = make_float4(S[v], S[v + 1], S[v + 2], S[v + 3]);
  }
  // before the CTA leaves (after an error too): the first chunk's dU^T is stored, the last load
  // on each barrier has landed (so every earlier one has), every MMA issued has finished
  if (issuer) {
    if (nc > 0 && !s_abort) {
      tma_store_3d(&mdUT, sN(0), 0, unit_row(0), 0);
      tma_store_3d(&mdUTl, sN(0) + TILE128, 0, unit_row(0), 0);
      tma_store_commit();
    }
    tma_store_wait0();
    if (n_iss0 > 0) mbar_wait(&barN[0], (uint32_t)((n_iss0 - 1) & 1), nullptr);
    if (n_iss1 > 0) mbar_wait(&barN[1], (uint32_t)((n_iss1 - 1) & 1), nullptr);
    if (dk_iss > 0) mbar_wait(&barDK, (uint32_t)((dk_iss - 1) & 1), nullptr);
    if (q_iss > 0) mbar_wait(&barQ, (uint32_t)((q_iss - 1) & 1), nullptr);
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
  return tgo("tc_scan_fwd", k_tc_scan_fwd2, grid, kScanThreadsWS, (size_t)1024 + Fwd2Smem::TOTAL, s, p, a,
             w, t, m.DK, m.NT, m.UtT, m.h, sr);
}

cudaError_t tc_scan_bwd(const Problem& p, const Args& a, const Work& w, const TcWork& t,
                        const TcMaps& m, const ScanRange& sr, cudaStream_t s) {
  const dim3 grid(p.Nst, p.HV);
  return tgo("tc_scan_bwd", k_tc_scan_bwd2, grid, kScanThreadsWS, (size_t)1024 + Bwd2Smem::TOTAL, s, p, a,
             w, t, m.q, m.DK, m.Op, m.WT, m.dUlT, m.NT, m.dh, m.dUT, m.dUTl, sr);
}

}  // namespace tcx
}  // namespace gdn
