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
// off the chain; the chain itself is one tensor-core product per chunk (S N) instead of two
// dependent ones (W S^T, then U^T D K).  Everything is kept transposed so that TMEM lane = key
// index k: the state S^T [k][v] is held in fp32 registers, four threads per row k (512 threads,
// 32 values each), and its bf16 copy that feeds the next product is written row by row.
#include "gdn_tc_common.cuh"

namespace gdn {
namespace tcx {

namespace {

constexpr int kScanThreads = 512;

// One 32-byte (256-bit) global store: a whole sector per thread.
__device__ __forceinline__ void st_global_32B(void* p, const uint32_t* v) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(v[0]), "r"(v[1]),
               "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

// ======================================================================================
// Forward.  Thread (warp w, lane l): TMEM lane quarter q = w & 3, row = 32q + l, column group
// cg = w >> 2 (32 state columns).  Thread 0 issues the MMAs, thread 64 the h stores, thread 96
// the loads.  Per chunk c, in tensor-pipe order:
//   chain(c)  ACC[c&1] += (-N_c^T) S_c^T       M=128 k', N=128 v, K=128 k   (8 instr)
//   N(c+1)    NT        = (D K)^T W            M=128 k', N=128 k, K=64 i    (4)
//   B(c+1)    ACC[~]    = (D K)^T U~           M=128 k', N=128 v, K=64 i    (4)
// all issued together; the next chain product waits only for the state update and -N^T.
// (v_new = U~ - W S^T is left to the output kernel, which reads S anyway: on the sequential
// pass every tensor-core instruction counts, at roughly 60-130 cycles each.)
// Shared memory: three input stages {U~^T [128][64], W^T [128][64], D K [64][128]} with e^{G_i},
// S^T bf16 [128 k][128 v] (MN-major B of the chain), -N^T bf16 [128 k'][128 k].
// ======================================================================================
struct Fwd2Smem {
  static constexpr int STAGE = 3 * TILE128;
  static constexpr int S = 3 * STAGE;
  static constexpr int N = S + 2 * TILE128;
  static constexpr int VEC = N + 2 * TILE128;               // 3 x {(unused)[64], e^G[64]}
  static constexpr int TOTAL = VEC + 3 * 512;
};

__global__ void __launch_bounds__(kScanThreads, 1) k_tc_scan_fwd2(
    Problem p, Args a, Work w, TcWork t, const __grid_constant__ CUtensorMap mDK,
    const __grid_constant__ CUtensorMap mWT, const __grid_constant__ CUtensorMap mUtT,
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
  const int qd = warp & 3, cg = warp >> 2, row = 32 * qd + lane;
  extern __shared__ unsigned char smraw[];
  unsigned char* sm = align1k(smraw);
  unsigned char* sS = sm + Fwd2Smem::S;
  unsigned char* sN = sm + Fwd2Smem::N;
  auto stage = [&](int c) { return sm + (c % 3) * Fwd2Smem::STAGE; };
  auto vecp = [&](int c) { return reinterpret_cast<float*>(sm + Fwd2Smem::VEC + (c % 3) * 512); };
  __shared__ uint64_t barL[3], barC, barN, barE;
  __shared__ uint32_t tslot;
  int* err = w.status;
  // the test flag withholds the first chain product; its wait then runs out quickly
  const long long wait_limit = p.test_timeout ? (1ll << 20) : (1ll << 31);
  if (tid == 0) {
    for (int i = 0; i < 3; ++i) mbar_init(&barL[i], 1);
    mbar_init(&barC, 1);
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
  // thread 96: chunk c's tiles (U~^T, W^T and D K, written by the WY kernel) and its e^{G_i}
  auto issue_load = [&](int c) {
    unsigned char* b = stage(c);
    uint64_t* bar = &barL[c % 3];
    const int r = unit_row(c);
    const size_t o = ((size_t)hv * p.NCmax + sq.x + c) * 64;
    mbar_expect_tx(bar, 2 * TILE128 + 2 * TILE64 + 256);
    tma_load_3d(b, &mUtT, 0, r, 0, bar);
    tma_load_3d(b + TILE128, &mWT, 0, r, 0, bar);
    tma_load_3d(b + 2 * TILE128, &mDK, 0, r / 2, 0, bar);
    tma_load_3d(b + 2 * TILE128 + TILE64, &mDK, 64, r / 2, 0, bar);
    bulk_load(vecp(c) + 64, w.EG + o, 256, bar);
  };
  // chunk c is the (c/3)-th load into stage c%3: its barrier phase has parity (c/3)&1
  auto load_par = [](int c) { return (uint32_t)((c / 3) & 1); };
  int loaded = min(3, nc);  // chunks whose loads were issued (the same count in every thread)
  int confirmed = 0;        // chunks whose loads every thread saw complete
  if (tid == 96)
    for (int c = 0; c < loaded; ++c) issue_load(c);
  // this thread's part of S^T: row `row`, columns 32 cg .. 32 cg + 31
  float S[32];
  // states are [Nst][HV][K][V]; rows k >= K and columns v >= V of a narrower head are padding
  const bool st_live = row < p.K && 32 * cg < p.V;
  const size_t st_off = (((size_t)n * p.HV + hv) * p.K + row) * p.V + 32 * cg;
#pragma unroll
  for (int v = 0; v < 32; v += 4) {
    const float4 x = (sr.s_in && st_live) ? *reinterpret_cast<const float4*>(sr.s_in + st_off + v)
                                          : make_float4(0, 0, 0, 0);
    S[v] = x.x; S[v + 1] = x.y; S[v + 2] = x.z; S[v + 3] = x.w;
  }
  auto put_state = [&]() {  // bf16 S^T row part -> the chain operand tile
#pragma unroll
    for (int j = 0; j < 4; ++j) st_chunk_f(sS, row, 4 * cg + j, TILE128, S + 8 * j);
  };
  auto store_h = [&](int c) {  // thread 64: h[c] <- the S^T tile
    tma_store_3d(&mh, sS, 0, unit_row(c), 0);
    tma_store_3d(&mh, sS + TILE128, 64, unit_row(c), 0);
    tma_store_commit();
  };
  if (nc > 0) put_state();
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tslot;
  const uint32_t tACC0 = taddr(tb, 0, 0), tNT = taddr(tb, 0, 256);
  if (tid == 64 && nc > 0) store_h(0);
  // N(c) into NT and B(c) into ACC[c&1] (K of chunk c already scaled)
  auto issue_nb = [&](int c) {
    unsigned char* b = stage(c);
    const uint64_t dk = desc_mnmajor(smem_u32(b + 2 * TILE128), 0, TILE64);
    const uint64_t dw = desc_kmajor(smem_u32(b + TILE128), 0, TILE128);
    const uint64_t du = desc_kmajor(smem_u32(b), 0, TILE128);
    constexpr uint32_t id = idesc_bf16(128, 128, true, false);
    const uint32_t tacc = tACC0 + (uint32_t)(128 * (c & 1));
#pragma unroll
    for (int s = 0; s < 4; ++s) {  // N and B interleaved (independent accumulators)
      mma_bf16(tNT, dk + mnstep_off(s), dw + kstep_off(s, TILE128), id, s > 0);
      mma_bf16(tacc, dk + mnstep_off(s), du + kstep_off(s, TILE128), id, s > 0);
    }
    mma_commit(&barN);
  };
  // -N^T (TMEM lanes k', columns k) -> bf16 K-major rows of sN; 32 columns per thread
  auto n_epilogue = [&]() {
    float x[32];
    tmem_ld16(taddr(tb, 32 * qd, 256 + 32 * cg), x);
    tmem_ld16(taddr(tb, 32 * qd, 256 + 32 * cg + 16), x + 16);
    tmem_wait_ld();
#pragma unroll
    for (int q = 0; q < 32; ++q) x[q] = -x[q];
#pragma unroll
    for (int j = 0; j < 4; ++j) st_chunk_f(sN, row, 4 * cg + j, TILE128, x + 8 * j);
  };
  bool ok = true;
  // prologue: the first two chunks' tiles, N(0) and B(0), -N_0^T in shared memory
  if (nc > 0) {
    bool okp = true;
    for (int c = 0; c < min(2, nc); ++c) okp = okp && mbar_wait(&barL[c], load_par(c), err);
    tc_fence_before();
    ok = __syncthreads_and(okp);
    tc_fence_after();
    if (ok) confirmed = min(2, nc);
    if (ok && tid == 0) issue_nb(0);
    okp = ok && mbar_wait(&barN, 0, err);
    tc_fence_after();
    if (okp) n_epilogue();
    fence_proxy_async();
    tc_fence_before();
    ok = __syncthreads_and(ok && okp);
    tc_fence_after();
  }
  for (int c = 0; ok && c < nc; ++c) {
    const bool more = c + 1 < nc;
    const float egc = vecp(c)[64 + 63];
    // (1) every product of this step at once
    if (tid == 0) {
      const uint64_t da = desc_kmajor(smem_u32(sN), 0, TILE128);
      const uint64_t dsB = desc_mnmajor(smem_u32(sS), 0, TILE128);
      const uint32_t tacc = tACC0 + (uint32_t)(128 * (c & 1));
      if (!(p.test_timeout && c == 0)) {  // the test flag withholds the first chain product
#pragma unroll
        for (int s = 0; s < 8; ++s)  // chain: ACC += (-N^T) S^T
          mma_bf16(tacc, da + kstep_off(s, TILE128), dsB + mnstep_off(s), idesc_bf16(128, 128, false, true), 1);
        mma_commit(&barC);
      }
      if (more) issue_nb(c + 1);
    }
    // (2) S_{c+1}^T = e^{G_C} S_c^T + ACC
    bool okt = mbar_wait_for(&barC, c & 1, err, wait_limit);
    tc_fence_after();
    if (okt) {
      float x[32];
      tmem_ld16(taddr(tb, 32 * qd, 128 * (c & 1) + 32 * cg), x);
      tmem_ld16(taddr(tb, 32 * qd, 128 * (c & 1) + 32 * cg + 16), x + 16);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 32; ++q) S[q] = egc * S[q] + x[q];
    }
    // (4) the tiles of the chunk two ahead have landed
    if (c + 2 < nc) okt = okt && mbar_wait(&barL[(c + 2) % 3], load_par(c + 2), err);
    if (tid == 64) tma_store_wait_read0();  // h[c] has been read out of the S^T tile
    tc_fence_before();
    ok = __syncthreads_and(ok && okt);
    tc_fence_after();
    if (!ok) break;
    confirmed = min(c + 3, nc);
    // (5) stage c%3 (its products N(c), B(c) finished before chain(c)) refills with chunk c+3
    if (loaded < nc) {
      if (tid == 96) issue_load(loaded);
      ++loaded;
    }
    // (6) the next step's operands: S_{c+1}^T and -N_{c+1}^T
    if (more) {
      put_state();
      okt = mbar_wait(&barN, (c + 1) & 1, err);
      tc_fence_after();
      if (okt) n_epilogue();
      fence_proxy_async();
      tc_fence_before();
      ok = __syncthreads_and(ok && okt);
      tc_fence_after();
      if (ok && tid == 64) store_h(c + 1);
    }
  }
  if (ok && sr.s_out && st_live) {  // the final state, or the state handed to the next launch
#pragma unroll
    for (int v = 0; v < 32; v += 4)
      *reinterpret_cast<float4*>(sr.s_out + st_off + v) = make_float4(S[v], S[v + 1], S[v + 2], S[v + 3]);
  }
  // on an error exit, let the loads that were issued land and the MMAs finish before the
  // CTA frees its tensor memory and leaves
  if (!ok && tid == 96)
    for (int c = confirmed; c < loaded; ++c) mbar_wait(&barL[c % 3], load_par(c), nullptr);
  if (tid == 64) tma_store_wait0();
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
//   dS_c^T = e^{G_C} dS'^T - ACC,   ACC = W^T dU_loc + Q^T O' + N dS'^T,  O' = -scale e^G dO
//   dU_c^T = dU_loc^T + dS' K^T D                      (written out as a bf16 hi/lo pair)
// Per chunk, in tensor-pipe order:
//   N(c)     NT   = W^T (D K)                 M=128 k, N=128 k'', K=64 i   (4 instr)
//   dU(c)    DU   = dS' (D K)^T, hi + lo      M=128 v, N=64 i,   K=128 k   (16)
//   ... O' scaled, N copied to shared memory ...
//   I(c)     DU  += dU_loc^T I                M=128 v, N=64 i,   K=64 i'   (4)
//   F(c)     ACC  = W^T dU_loc + Q^T O'       M=128 k, N=128 v,  K=64 i    (8)
//   chain(c) ACC += N (dS'^T hi + lo)         M=128 k, N=128 v,  K=128 k'' (16)
// dU_loc enters dU through the identity product, so once F(c) has run, the slot of Q, dO and
// dU_loc is free and the previous chunk's tiles stream in while the chain product runs.
// Shared memory: two slots of {D K [64][128], W^T [128][64]} with e^{G_i}, one of {Q [64][128],
// O' [64][128], dU_loc^T [128][64]}, N bf16 [128][128] (K-major A), dS'^T hi and lo
// [128 k''][128 v], the 64 x 64 identity.  D K comes from the WY kernel and O' from dv_local.
// ======================================================================================
struct Bwd2Smem {
  static constexpr int KW = 0;                              // 2 x {K (2 x TILE64), W^T}
  static constexpr int KW_BYTES = 2 * TILE128;
  static constexpr int Q = 2 * KW_BYTES;
  static constexpr int O = Q + TILE128;
  static constexpr int UL = O + TILE128;
  static constexpr int N = UL + TILE128;
  static constexpr int DSH = N + 2 * TILE128;
  static constexpr int DSL = DSH + 2 * TILE128;
  static constexpr int ID = DSL + 2 * TILE128;              // identity [64][64] bf16
  static constexpr int VEC = ID + TILE64;                   // 2 x {D[64], e^G[64]} (raw)
  static constexpr int TOTAL = VEC + 2 * 512;
};

__global__ void __launch_bounds__(kScanThreads, 1) k_tc_scan_bwd2(
    Problem p, Args a, Work w, TcWork t, const __grid_constant__ CUtensorMap mq,
    const __grid_constant__ CUtensorMap mDK, const __grid_constant__ CUtensorMap mOp,
    const __grid_constant__ CUtensorMap mWT, const __grid_constant__ CUtensorMap mdUlT,
    const __grid_constant__ CUtensorMap mdh, ScanRange sr) {
  __shared__ int s_fail;
  if (threadIdx.x == 0) s_fail = failed(w);
  __syncthreads();
  if (s_fail) return;
  const int n = blockIdx.x, hv = blockIdx.y, hk = hv / p.G;
  const int4 sq0 = w.seq_tab[n];
  const int cb = min(max(sr.c0, 0), sq0.y), nc = max(min(sr.c1, sq0.y) - cb, 0);
  const int4 sq = make_int4(sq0.x + cb, nc, sq0.z + 64 * cb, sq0.w - 64 * cb);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int qd = warp & 3, cg = warp >> 2, row = 32 * qd + lane;
  extern __shared__ unsigned char smraw[];
  unsigned char* sm = align1k(smraw);
  unsigned char* sQ = sm + Bwd2Smem::Q;
  unsigned char* sO = sm + Bwd2Smem::O;
  unsigned char* sUl = sm + Bwd2Smem::UL;
  unsigned char* sN = sm + Bwd2Smem::N;
  unsigned char* sDH = sm + Bwd2Smem::DSH;
  unsigned char* sDL = sm + Bwd2Smem::DSL;
  unsigned char* sI = sm + Bwd2Smem::ID;
  auto sK = [&](int c) { return sm + Bwd2Smem::KW + (c & 1) * Bwd2Smem::KW_BYTES; };
  auto sW = [&](int c) { return sK(c) + TILE128; };
  auto vecp = [&](int c) { return reinterpret_cast<float*>(sm + Bwd2Smem::VEC + (c & 1) * 512); };
  __shared__ uint64_t barKW[2], barQOU, barN, barDU, barF, barC, barE;
  __shared__ uint32_t tslot;
  int* err = w.status;
  if (tid == 0) {
    mbar_init(&barKW[0], 1);
    mbar_init(&barKW[1], 1);
    mbar_init(&barQOU, 1);
    mbar_init(&barN, 1);
    mbar_init(&barDU, 1);
    mbar_init(&barF, 1);
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
  auto tok_of = [&](int c) { return sq.z + 64 * c; };
  // chunks are loaded in iteration order nc-1, nc-2, ...: chunk c's {K, W} is the j-th load
  // into slot c&1 with j = (nc-1-c)/2, its {Q, dO, dU_loc} the (nc-1-c)-th into their slot
  auto kw_par = [&](int c) { return (uint32_t)(((nc - 1 - c) >> 1) & 1); };
  auto qou_par = [&](int c) { return (uint32_t)((nc - 1 - c) & 1); };
  // thread 32: chunk c's D K (the WY kernel's) and W^T, and its e^{G_i}
  auto issue_kw = [&](int c) {
    uint64_t* bar = &barKW[c & 1];
    const size_t o = ((size_t)hv * p.NCmax + sq.x + c) * 64;
    mbar_expect_tx(bar, 2 * TILE128 + 256);
    tma_load_3d(sK(c), &mDK, 0, unit_row(c) / 2, 0, bar);
    tma_load_3d(sK(c) + TILE64, &mDK, 64, unit_row(c) / 2, 0, bar);
    tma_load_3d(sW(c), &mWT, 0, unit_row(c), 0, bar);
    bulk_load(vecp(c) + 64, w.EG + o, 256, bar);
  };
  // thread 96: chunk c's Q, O' = -scale e^G dO (the dv_local kernel's) and dU_loc^T
  auto issue_qou = [&](int c) {
    mbar_expect_tx(&barQOU, 3 * TILE128);
    tma_load_3d(sQ, &mq, 0, hk, tok_of(c), &barQOU);
    tma_load_3d(sQ + TILE64, &mq, 64, hk, tok_of(c), &barQOU);
    tma_load_3d(sO, &mOp, 0, unit_row(c) / 2, 0, &barQOU);
    tma_load_3d(sO + TILE64, &mOp, 64, unit_row(c) / 2, 0, &barQOU);
    tma_load_3d(sUl, &mdUlT, 0, unit_row(c), 0, &barQOU);
  };
  int kw_issued = 0, qou_issued = 0;  // loads issued, in iteration order (same count in every thread)
  int kw_seen = 0, qou_seen = 0;      // loads every thread saw complete
  if (tid == 32 && nc > 0) issue_kw(nc - 1);
  if (tid == 96 && nc > 0) issue_qou(nc - 1);
  if (nc > 0) kw_issued = qou_issued = 1;
  // this thread's part of dS'^T: row `row`, columns 32 cg .. 32 cg + 31
  float S[32];
  // states are [Nst][HV][K][V]; rows k >= K and columns v >= V of a narrower head are padding
  const bool st_live = row < p.K && 32 * cg < p.V;
  const size_t st_off = (((size_t)n * p.HV + hv) * p.K + row) * p.V + 32 * cg;
#pragma unroll
  for (int v = 0; v < 32; v += 4) {
    const float4 x = (sr.s_in && st_live) ? *reinterpret_cast<const float4*>(sr.s_in + st_off + v)
                                          : make_float4(0, 0, 0, 0);
    S[v] = x.x; S[v + 1] = x.y; S[v + 2] = x.z; S[v + 3] = x.w;
  }
  {  // the 64 x 64 identity (bf16), one 16-byte chunk per thread
    const int r = tid >> 3, j = tid & 7;
    float f[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) f[q] = (8 * j + q == r) ? 1.f : 0.f;
    st_chunk_f(sI, r, j, TILE64, f);
  }
  auto put_state = [&]() {  // dS'^T row part as a compensated bf16 pair
#pragma unroll
    for (int j = 0; j < 4; ++j) st_chunk_split(sDH, sDL, row, 4 * cg + j, TILE128, S + 8 * j);
  };
  auto store_dh = [&](int c) {  // thread 64: dh[c] <- the hi tile
    tma_store_3d(&mdh, sDH, 0, unit_row(c), 0);
    tma_store_3d(&mdh, sDH + TILE128, 64, unit_row(c), 0);
    tma_store_commit();
  };
  if (nc > 0) put_state();
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tslot;
  const uint32_t tACC = taddr(tb, 0, 0), tNT = taddr(tb, 0, 128), tDU = taddr(tb, 0, 256);
  if (tid == 64 && nc > 0) store_dh(nc - 1);
  bool ok = true;
  if (nc > 0) {  // the first chunk's D K and W^T
    bool okp = mbar_wait(&barKW[(nc - 1) & 1], kw_par(nc - 1), err);
    tc_fence_before();
    ok = __syncthreads_and(okp);
    tc_fence_after();
    if (ok) kw_seen = 1;
  }
  for (int idx = 0; ok && idx < nc; ++idx) {
    const int c = nc - 1 - idx;
    const bool more = c > 0;
    const float* vc = vecp(c);
    // (1) N(c), dU(c) (state and K only); the previous chunk's K and W stream into the other slot
    if (tid == 0) {
      const uint64_t dw = desc_kmajor(smem_u32(sW(c)), 0, TILE128);
      const uint64_t dkB = desc_mnmajor(smem_u32(sK(c)), 0, TILE64);
      constexpr uint32_t idN = idesc_bf16(128, 128, false, true);
      const uint64_t dkK = desc_kmajor(smem_u32(sK(c)), 0, TILE64);
      constexpr uint32_t idU = idesc_bf16(128, 64, true, false);
      const uint64_t dah = desc_mnmajor(smem_u32(sDH), 0, TILE128);
      const uint64_t dal = desc_mnmajor(smem_u32(sDL), 0, TILE128);
      // N = W^T (D K) interleaved with dU^T = dS' (D K)^T (hi, then lo): independent accumulators
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        if (s < 4) mma_bf16(tNT, dw + kstep_off(s, TILE128), dkB + mnstep_off(s), idN, s > 0);
        mma_bf16(tDU, dah + mnstep_off(s), dkK + kstep_off(s, TILE64), idU, s > 0);
      }
      mma_commit(&barN);
#pragma unroll
      for (int s = 0; s < 8; ++s) mma_bf16(tDU, dal + mnstep_off(s), dkK + kstep_off(s, TILE64), idU, 1);
    }
    if (tid == 32 && more) issue_kw(c - 1);
    if (more) ++kw_issued;
    if (tid == 64) tma_store_wait_read0();  // the last dh store has read the hi tile
    // (2) this chunk's Q, O', dU_loc; N -> shared memory
    bool okt = mbar_wait(&barQOU, qou_par(c), err);
    okt = okt && mbar_wait(&barN, idx & 1, err);
    tc_fence_after();
    if (okt) {
      float x[32];
      tmem_ld16(taddr(tb, 32 * qd, 128 + 32 * cg), x);
      tmem_ld16(taddr(tb, 32 * qd, 128 + 32 * cg + 16), x + 16);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 4; ++j) st_chunk_f(sN, row, 4 * cg + j, TILE128, x + 8 * j);
    }
    fence_proxy_async();
    tc_fence_before();
    ok = __syncthreads_and(ok && okt);
    tc_fence_after();
    if (!ok) break;
    qou_seen = idx + 1;
    // (3) dU_loc into dU, F, then the chain product
    if (tid == 0) {
      const uint64_t dul = desc_kmajor(smem_u32(sUl), 0, TILE128);
      const uint64_t di = desc_kmajor(smem_u32(sI), 0, TILE64);
      const uint64_t dwA = desc_kmajor(smem_u32(sW(c)), 0, TILE128);
      const uint64_t dq = desc_mnmajor(smem_u32(sQ), 0, TILE64);
      const uint64_t dO_ = desc_mnmajor(smem_u32(sO), 0, TILE64);
      // dU^T += dU_loc^T I interleaved with F = W^T dU_loc + Q^T O'
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        mma_bf16(tDU, dul + kstep_off(s, TILE128), di + kstep_off(s, TILE64), idesc_bf16(128, 64, false, false), 1);
        mma_bf16(tACC, dwA + kstep_off(s, TILE128), dul + kstep_off(s, TILE128),
                 idesc_bf16(128, 128, false, false), s > 0);
      }
      mma_commit(&barDU);
#pragma unroll
      for (int s = 0; s < 4; ++s)
        mma_bf16(tACC, dq + mnstep_off(s), dO_ + mnstep_off(s), idesc_bf16(128, 128, true, true), 1);
      mma_commit(&barF);
      const uint64_t dn = desc_kmajor(smem_u32(sN), 0, TILE128);
      for (int part = 0; part < 2; ++part) {
        const uint64_t db = desc_mnmajor(smem_u32(part ? sDL : sDH), 0, TILE128);
#pragma unroll
        for (int s = 0; s < 8; ++s)  // + N dS'^T, hi then lo
          mma_bf16(tACC, dn + kstep_off(s, TILE128), db + mnstep_off(s), idesc_bf16(128, 128, false, true), 1);
      }
      mma_commit(&barC);
    }
    // (4) the previous chunk's Q, dO, dU_loc once F has read this chunk's
    if (tid == 96 && more) {
      if (mbar_wait(&barF, idx & 1, err)) issue_qou(c - 1);
    }
    if (more) ++qou_issued;
    // dU^T = DU as a hi/lo pair (rows v, 16 columns per thread), straight to the workspace
    okt = mbar_wait(&barDU, idx & 1, err);
    tc_fence_after();
    if (okt) {
      float x[16];
      tmem_ld16(taddr(tb, 32 * qd, 256 + 16 * cg), x);
      tmem_wait_ld();
      bf16* hrow = t.dUT + ((size_t)unit_row(c) + row) * 64 + 16 * cg;
      bf16* lrow = t.dUTl + ((size_t)unit_row(c) + row) * 64 + 16 * cg;
      uint32_t ph[8], pl[8];
#pragma unroll
      for (int q = 0; q < 16; q += 2) {
        const float h0 = __bfloat162float(__float2bfloat16_rn(x[q]));
        const float h1 = __bfloat162float(__float2bfloat16_rn(x[q + 1]));
        ph[q / 2] = pack_bf16(h0, h1);
        pl[q / 2] = pack_bf16(x[q] - h0, x[q + 1] - h1);
      }
      st_global_32B(hrow, ph);  // 16 columns = one full 32-byte sector per row and part
      st_global_32B(lrow, pl);
    }
    // the previous chunk's D K and W^T have landed
    if (more) okt = okt && mbar_wait(&barKW[(c - 1) & 1], kw_par(c - 1), err);
    // dS_c^T = e^{G_C} dS'^T - ACC, then its hi/lo copy for the next step
    okt = okt && mbar_wait(&barC, idx & 1, err);
    tc_fence_after();
    if (okt) {
      const float egc = vc[64 + 63];
      float x[32];
      tmem_ld16(taddr(tb, 32 * qd, 32 * cg), x);
      tmem_ld16(taddr(tb, 32 * qd, 32 * cg + 16), x + 16);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 32; ++q) S[q] = egc * S[q] - x[q];
      if (more) put_state();
    }
    fence_proxy_async();
    tc_fence_before();
    ok = __syncthreads_and(ok && okt);
    tc_fence_after();
    if (!ok) break;
    if (more) kw_seen = idx + 2;
    // (5) dh of chunk c-1: the gradient leaving it (a launch over earlier chunks writes the one
    // leaving chunk cb-1 itself, from the state this launch hands on)
    if (tid == 64 && more) store_dh(c - 1);
  }
  if (ok && sr.s_out && st_live) {  // dh0, or the gradient handed to the launch of earlier chunks
#pragma unroll
    for (int v = 0; v < 32; v += 4)
      *reinterpret_cast<float4*>(sr.s_out + st_off + v) = make_float4(S[v], S[v + 1], S[v + 2], S[v + 3]);
  }
  if (!ok && tid == 32)  // let issued loads land before the CTA leaves
    for (int j = kw_seen; j < kw_issued; ++j) mbar_wait(&barKW[(nc - 1 - j) & 1], kw_par(nc - 1 - j), nullptr);
  if (!ok && tid == 96)
    for (int j = qou_seen; j < qou_issued; ++j) mbar_wait(&barQOU, qou_par(nc - 1 - j), nullptr);
  if (tid == 64) tma_store_wait0();
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
  return tgo("tc_scan_fwd", k_tc_scan_fwd2, grid, kScanThreads, (size_t)1024 + Fwd2Smem::TOTAL, s, p, a,
             w, t, m.DK, m.WT, m.UtT, m.h, sr);
}

cudaError_t tc_scan_bwd(const Problem& p, const Args& a, const Work& w, const TcWork& t,
                        const TcMaps& m, const ScanRange& sr, cudaStream_t s) {
  const dim3 grid(p.Nst, p.HV);
  return tgo("tc_scan_bwd", k_tc_scan_bwd2, grid, kScanThreads, (size_t)1024 + Bwd2Smem::TOTAL, s, p, a,
             w, t, m.q, m.DK, m.Op, m.WT, m.dUlT, m.dh, sr);
}

}  // namespace tcx
}  // namespace gdn
