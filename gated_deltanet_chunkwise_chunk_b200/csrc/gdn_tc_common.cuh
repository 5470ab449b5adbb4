// Shared pieces of the tcgen05 kernels: constants, workspace views, tensor maps and the
// swizzled-tile helpers.
#pragma once

#include <algorithm>
#include <mutex>

#include "gdn_launch.h"
#include "gdn_tc.h"
#include "tc_prims.cuh"

namespace gdn {

using bf16 = __nv_bfloat16;

namespace tcx {
using namespace tc;
constexpr int D = 128;                 // head dimension (K = V = 128 on this path)
constexpr int TILE64 = 64 * 128;       // bytes of a [64 rows x 64 bf16] block
constexpr int TILE128 = 128 * 128;     // bytes of a [128 rows x 64 bf16] block

// ------------------------------------------------------------------ tensor maps (host)
typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                             const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                             CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                             CUtensorMapFloatOOBfill);

inline EncodeFn encoder() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  });
  return fn;
}

// bf16 tensor viewed as [outer][rows][cols] (cols contiguous) with box {64, box_rows, 1}
// (128-byte swizzle, out-of-bounds rows read as zero).
inline bool map3(CUtensorMap* m, const void* base, uint64_t cols, uint64_t mid, uint64_t outer,
          uint64_t mid_stride_elems, uint64_t outer_stride_elems, uint32_t box_mid, uint32_t box_outer) {
  EncodeFn enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {cols, mid, outer};
  cuuint64_t strides[2] = {mid_stride_elems * 2, outer_stride_elems * 2};
  cuuint32_t box[3] = {64, box_mid, box_outer};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// token tensor [ntok][heads][dim] -> 3D map (col, head, token), box = 64 cols x 1 head x 64
// tokens.  With dim = 64 the box at column 64 lies past the tensor and reads as zeros, which is
// how 64-wide heads run on the 128-wide tiles.
inline bool map_tokens(CUtensorMap* m, const void* base, int ntok, int heads, int dim) {
  return map3(m, base, (uint64_t)dim, heads, ntok, (uint64_t)dim, (uint64_t)heads * dim, 1, 64);
}
// 2D row-major [rows][cols] bf16, box = 64 cols x box_rows rows (as a 3D map with outer = 1)
inline bool map_rows(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  return map3(m, base, cols, rows, 1, cols, rows * cols, box_rows, 1);
}

struct TcMaps {
  CUtensorMap q, k, v, dO;            // token tensors
  CUtensorMap WT, UtT, UT;            // [unit*128][64]
  CUtensorMap h;                      // [unit*128][128]
  CUtensorMap dUlT, dUT, dUTl;        // [unit*128][64]      (backward)
  CUtensorMap dh;                     // [unit*128][128]     (backward)
  CUtensorMap dW;                     // [unit*64][128]      (backward)
  CUtensorMap Tm;                     // [unit*64][64]       (backward)
  CUtensorMap DK;                     // [unit*64][128]      keys scaled by e^{G_C - G_i}
  CUtensorMap NT;                     // [unit*128][128]     -N^T of the chunk's state map
  CUtensorMap Op;                     // [unit*64][128]      -scale e^{G_i} dO   (backward)
};

struct TcWork {
  bf16* WT;     // [NC*HV][128][64]
  bf16* UtT;    // [NC*HV][128][64]
  bf16* UT;     // [NC*HV][128][64]
  bf16* h;      // [NC*HV][128 k][128 v]  state entering the chunk, transposed (S^T)
  bf16* Tm;     // [NC*HV][2][64][64] (backward only) (I + A)^-1 as hi, lo bf16 parts
  bf16* dUlT;   // [NC*HV][128][64]  dv_local^T = scale (P^T dO)^T
  bf16* dh;     // [NC*HV][128 k][128 v] dL/dS leaving the chunk, transposed (dS^T)
  bf16* dUT;    // [NC*HV][128][64]  dU^T (full), hi part
  bf16* dUTl;   // [NC*HV][128][64]  dU^T lo part (dU^T - hi)
  bf16* dW;     // [NC*HV][64][128]  dL/dW
  bf16* DK;     // [NC*HV][64][128]  D K = e^{G_C - G_i} k_i (zero past the chunk end), per value head
  bf16* NT;     // [NC*HV][128 k'][128 k]  -N^T, N = W^T D K (the state map's K x K factor)
  bf16* Op;     // [NC*HV][64][128]  O' = -scale e^{G_i} dO_i (zero past the chunk end)  (backward)
  float* hand;  // [HV][128][128] fp32: the state passed between launches of a segmented pass
  int* ctr;     // [kCounters] work counters of the persistent backward kernels
};

// A single sequence's chunks are split into segments so that the sequential pass over one
// segment (one CTA per value head, few SMs) overlaps the chunk-parallel kernels of others.
constexpr int kMaxSeg = 8;          // segments of a pass (at most)
// Segments of the forward and of the backward (measured at 512 chunks x 32 value heads: the
// forward's pass is short next to its chunk kernels, so fewer, longer launches pay; the
// backward's longer pass wants finer overlap)
constexpr int kFwdSeg = 3;
constexpr int kBwdSeg = 8;
constexpr int kSegChunks = 32;      // at least this many chunks per segment
constexpr int kCounters = 2 * kMaxSeg;

struct Segments {
  int n;                  // number of segments (1 = one launch per kernel over all chunks)
  int c[kMaxSeg + 1];     // segment i covers chunks [c[i], c[i+1])
};

inline Segments segments(const Problem& p, int max_seg) {
  Segments sg{};
  sg.n = 1;
  sg.c[0] = 0;
  sg.c[1] = p.NCmax;
  // only one sequence (chunks of one segment are contiguous in the chunk table), and only
  // when the pass leaves most SMs to the other kernels
  if (p.Nst != 1 || 2 * p.HV > num_sms()) return sg;
  const int n = std::min(std::min(max_seg, kMaxSeg), p.NCmax / kSegChunks);
  if (n < 2) return sg;
  sg.n = n;
  for (int i = 0; i <= n; ++i) sg.c[i] = (int)((long long)p.NCmax * i / n);
  return sg;
}

// The library's side stream on the current device (highest priority, so the sequential pass's
// CTAs are placed first when SMs free up) and a pool of events, held under a per-device lock
// while one call queues its work (concurrent calls from several host threads take turns).
class SideLock {
 public:
  SideLock();
  ~SideLock();
  SideLock(const SideLock&) = delete;
  SideLock& operator=(const SideLock&) = delete;
  bool ok() const { return ok_; }
  cudaStream_t stream() const;
  // the side stream waits for the work queued on s so far
  cudaError_t fork(cudaStream_t s);
  // records the next pool event on st
  cudaError_t record(cudaStream_t st, cudaEvent_t* ev);

 private:
  void* dev_ = nullptr;
  int next_ = 0;
  bool ok_ = false;
};

inline size_t align_up(size_t x) { return (x + 1023) / 1024 * 1024; }

// Chunks [c0, c1) of every sequence (clamped to its length) for one launch of a sequential
// pass, with the state it enters with and the state it leaves ([Nst][HV][K][V] fp32 in the
// [k][v] layout; NULL = zero / not written).
struct ScanRange {
  int c0, c1;
  const float* s_in;
  float* s_out;
};

// Units u = chunk * HV + value head in [u0, u1) for one launch of a persistent kernel, handed
// out in order by the atomic counter *ctr (zero before the launch).
struct UnitRange {
  int u0, u1;
  int* ctr;
};

inline TcWork carve_tc(void* base, size_t NC, size_t HV, int pass) {
  char* b = static_cast<char*>(base);
  TcWork t{};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    char* p = b + o;
    o += align_up(bytes);
    return p;
  };
  const size_t units = NC * HV;
  t.WT = reinterpret_cast<bf16*>(take(units * D * 64 * 2));
  t.UtT = reinterpret_cast<bf16*>(take(units * D * 64 * 2));
  t.UT = reinterpret_cast<bf16*>(take(units * D * 64 * 2));
  t.h = reinterpret_cast<bf16*>(take(units * D * D * 2));
  t.Tm = reinterpret_cast<bf16*>(take(units * 2 * 64 * 64 * 2));  // written by every forward
  t.DK = reinterpret_cast<bf16*>(take(units * 64 * D * 2));
  t.NT = reinterpret_cast<bf16*>(take(units * D * D * 2));
  t.hand = reinterpret_cast<float*>(take(HV * D * D * 4));
  t.ctr = reinterpret_cast<int*>(take(kCounters * sizeof(int)));
  if (pass == 1) {
    t.dUlT = reinterpret_cast<bf16*>(take(units * D * 64 * 2));
    t.dh = reinterpret_cast<bf16*>(take(units * D * D * 2));
    t.dUT = reinterpret_cast<bf16*>(take(units * D * 64 * 2));
    t.dUTl = reinterpret_cast<bf16*>(take(units * D * 64 * 2));
    t.dW = reinterpret_cast<bf16*>(take(units * 64 * D * 2));
    t.Op = reinterpret_cast<bf16*>(take(units * 64 * D * 2));
  }
  return t;
}

inline size_t tc_bytes(size_t NC, size_t HV, int pass) {
  const size_t units = NC * HV;
  size_t o = 3 * align_up(units * D * 64 * 2) + 2 * align_up(units * D * D * 2);
  o += align_up(units * 2 * 64 * 64 * 2);
  o += align_up(units * 64 * D * 2);
  o += align_up(HV * D * D * 4) + align_up(kCounters * sizeof(int));
  if (pass == 1)
    o += 3 * align_up(units * D * 64 * 2) +
         align_up(units * D * D * 2) + 2 * align_up(units * 64 * D * 2);
  return o;
}

// ------------------------------------------------------------------ device helpers
__device__ __forceinline__ unsigned char* align1k(unsigned char* p) {
  return reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Zero rows [L, 64) of a [64 x 128] bf16 token tile (two 8 KB column blocks).
__device__ __forceinline__ void zero_tail_rows(unsigned char* tile, int L, int tid, int nthr) {
  const int n = (64 - L) * 16;  // 16-byte chunks per row (2 blocks x 8)
  for (int i = tid; i < n; i += nthr) {
    const int r = L + i / 16, j = i % 16;
    *reinterpret_cast<uint4*>(tile + sw128_chunk(r, j, TILE64)) = make_uint4(0, 0, 0, 0);
  }
}

// One bf16 element of a tile at byte offset off (from sw128).
__device__ __forceinline__ void st_bf16(unsigned char* tile, uint32_t off, float x) {
  *reinterpret_cast<bf16*>(tile + off) = __float2bfloat16_rn(x);
}
__device__ __forceinline__ void st_bf16_raw(unsigned char* tile, uint32_t off, bf16 x) {
  *reinterpret_cast<bf16*>(tile + off) = x;
}
__device__ __forceinline__ float ld_bf16(const unsigned char* tile, uint32_t off) {
  return __bfloat162float(*reinterpret_cast<const bf16*>(tile + off));
}

// Reads 8 bf16 (one 16-byte swizzled chunk) as floats.
__device__ __forceinline__ void ld_chunk_f(const unsigned char* tile, int r, int j, int block_bytes,
                                           float* f) {
  const uint4 v = *reinterpret_cast<const uint4*>(tile + sw128_chunk(r, j, block_bytes));
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x = __bfloat1622float2(h[i]);
    f[2 * i] = x.x;
    f[2 * i + 1] = x.y;
  }
}
__device__ __forceinline__ void st_chunk_f(unsigned char* tile, int r, int j, int block_bytes,
                                           const float* f) {
  uint4 v;
  v.x = pack_bf16(f[0], f[1]);
  v.y = pack_bf16(f[2], f[3]);
  v.z = pack_bf16(f[4], f[5]);
  v.w = pack_bf16(f[6], f[7]);
  *reinterpret_cast<uint4*>(tile + sw128_chunk(r, j, block_bytes)) = v;
}

// Stores 8 floats as a compensated bf16 pair: hi = bf16(f), lo = bf16(f - hi), so that
// A = A_hi + A_lo carries ~16 mantissa bits through two tensor-core products.
__device__ __forceinline__ void st_chunk_split(unsigned char* hi, unsigned char* lo, int r, int j,
                                               int block_bytes, const float* f) {
  float h[8], l[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    h[q] = __bfloat162float(__float2bfloat16_rn(f[q]));
    l[q] = f[q] - h[q];
  }
  st_chunk_f(hi, r, j, block_bytes, h);
  st_chunk_f(lo, r, j, block_bytes, l);
}

// Row stride (floats) of the fp32 64x64 scratch matrices of the triangular inverse: rows are
// 16-byte aligned for 128-bit loads, and 68 = 4 (mod 32) spreads consecutive rows over banks.
constexpr int LDA = 68;

// T = (I + A)^-1 for a strictly lower-triangular 64x64 fp32 A (row stride LDA), 256 threads.
// The four diagonal 16x16 blocks by forward substitution (warps 0..3, one column per lane)
// while warps 4..7 zero the strictly upper 16-blocks; then the blocks below the diagonal by
// block back-substitution, using [[L00, 0], [A10, L11]]^-1 = [[T00, 0], [-T11 A10 T00, T11]]:
//   16-blocks of each 32x32 half:  T10 = -T11 (A10 T00)        (both halves at once)
//   32-blocks:                     T[32:,:32] = -T[32:,32:] (A[32:,:32] T[:32,:32])
// Each thread owns 4 consecutive columns of one output row of a product; operands are read
// as float4 (a row of A four k at a time, a row of T four columns at a time).  sX: [64][LDA].
// Threads 0..255 take part (kBar: see sync256).
// The inverse's barrier: the whole CTA (kBar = 0, a 256-thread CTA), or named barrier kBar over
// threads 0..255 of a larger CTA (the others skip the inverse).
template <int kBar>
__device__ __forceinline__ void sync256() {
  if constexpr (kBar == 0) __syncthreads();
  else nbar_sync(kBar, 256);
}

template <int kBar = 0>
__device__ __forceinline__ void unit_lower_inverse64(const float* sA, float* sT, float* sX, int tid) {
  const int w = tid >> 5, lane = tid & 31;
  if (w < 4) {
    if (lane < 16) {
      const int b0 = 16 * w, c = lane;
      float col[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float s = (r == c) ? 1.f : 0.f;
#pragma unroll
        for (int j = 0; j < r; ++j) s -= sA[(b0 + r) * LDA + b0 + j] * col[j];
        col[r] = (r >= c) ? s : 0.f;
      }
#pragma unroll
      for (int r = 0; r < 16; ++r) sT[(b0 + r) * LDA + b0 + c] = col[r];
    }
  } else {
    for (int i = tid - 128; i < 6 * 64; i += 128) {  // blocks (0,1) (0,2) (0,3) (1,2) (1,3) (2,3)
      const int blk = i >> 6, r = (i >> 2) & 15, c4 = i & 3;
      const int br = blk < 3 ? 0 : (blk < 5 ? 1 : 2), bc = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
      *reinterpret_cast<float4*>(sT + (16 * br + r) * LDA + 16 * bc + 4 * c4) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  sync256<kBar>();
  auto fma4 = [](float4& acc, float a, const float4& b) {
    acc.x += a * b.x; acc.y += a * b.y; acc.z += a * b.z; acc.w += a * b.w;
  };
  // X = A10 T00 in each half p: row 16(2p+1)+r, columns 32p + 4c4 .. +3 (threads 0..127)
  const int p1 = (tid >> 6) & 1, r1 = (tid >> 2) & 15, c41 = tid & 3;
  const int R1 = 16 * (2 * p1 + 1) + r1, C1 = 32 * p1 + 4 * c41;
  if (tid < 128) {
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j4 = 0; j4 < 4; ++j4) {
      const float4 a = *reinterpret_cast<const float4*>(sA + R1 * LDA + 32 * p1 + 4 * j4);
      const float* t = sT + (32 * p1 + 4 * j4) * LDA + C1;
      fma4(x, a.x, *reinterpret_cast<const float4*>(t));
      fma4(x, a.y, *reinterpret_cast<const float4*>(t + LDA));
      fma4(x, a.z, *reinterpret_cast<const float4*>(t + 2 * LDA));
      fma4(x, a.w, *reinterpret_cast<const float4*>(t + 3 * LDA));
    }
    *reinterpret_cast<float4*>(sX + R1 * LDA + C1) = x;
  }
  sync256<kBar>();
  if (tid < 128) {  // T10 = -T11 X
    const int D0 = 16 * (2 * p1 + 1);
    float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int m4 = 0; m4 < 4; ++m4) {
      const float4 tt = *reinterpret_cast<const float4*>(sT + R1 * LDA + D0 + 4 * m4);
      const float* x = sX + (D0 + 4 * m4) * LDA + C1;
      fma4(y, tt.x, *reinterpret_cast<const float4*>(x));
      fma4(y, tt.y, *reinterpret_cast<const float4*>(x + LDA));
      fma4(y, tt.z, *reinterpret_cast<const float4*>(x + 2 * LDA));
      fma4(y, tt.w, *reinterpret_cast<const float4*>(x + 3 * LDA));
    }
    *reinterpret_cast<float4*>(sT + R1 * LDA + C1) = make_float4(-y.x, -y.y, -y.z, -y.w);
  }
  sync256<kBar>();
  // rows 32 + r2, columns 4c4 .. +3 (all 256 threads)
  const int r2 = tid >> 3, C2 = 4 * (tid & 7), R2 = 32 + r2;
  {  // X = A[32:,:32] T[:32,:32]
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j4 = 0; j4 < 8; ++j4) {
      const float4 a = *reinterpret_cast<const float4*>(sA + R2 * LDA + 4 * j4);
      const float* t = sT + (4 * j4) * LDA + C2;
      fma4(x, a.x, *reinterpret_cast<const float4*>(t));
      fma4(x, a.y, *reinterpret_cast<const float4*>(t + LDA));
      fma4(x, a.z, *reinterpret_cast<const float4*>(t + 2 * LDA));
      fma4(x, a.w, *reinterpret_cast<const float4*>(t + 3 * LDA));
    }
    *reinterpret_cast<float4*>(sX + R2 * LDA + C2) = x;
  }
  sync256<kBar>();
  {  // T[32:,:32] = -T[32:,32:] X
    float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int m4 = 0; m4 < 8; ++m4) {
      const float4 tt = *reinterpret_cast<const float4*>(sT + R2 * LDA + 32 + 4 * m4);
      const float* x = sX + (32 + 4 * m4) * LDA + C2;
      fma4(y, tt.x, *reinterpret_cast<const float4*>(x));
      fma4(y, tt.y, *reinterpret_cast<const float4*>(x + LDA));
      fma4(y, tt.z, *reinterpret_cast<const float4*>(x + 2 * LDA));
      fma4(y, tt.w, *reinterpret_cast<const float4*>(x + 3 * LDA));
    }
    *reinterpret_cast<float4*>(sT + R2 * LDA + C2) = make_float4(-y.x, -y.y, -y.z, -y.w);
  }
  sync256<kBar>();
}

// Two adjacent bf16 columns (c even) of row r as one 32-bit store, hi and lo parts.
__device__ __forceinline__ void st_pair_split(unsigned char* hi, unsigned char* lo, int r, int c,
                                              int block_bytes, float a, float b) {
  const float ha = __bfloat162float(__float2bfloat16_rn(a));
  const float hb = __bfloat162float(__float2bfloat16_rn(b));
  *reinterpret_cast<uint32_t*>(hi + sw128(r, c, block_bytes)) = pack_bf16(ha, hb);
  *reinterpret_cast<uint32_t*>(lo + sw128(r, c, block_bytes)) = pack_bf16(a - ha, b - hb);
}
__device__ __forceinline__ void st_pair(unsigned char* tile, int r, int c, int block_bytes, float a,
                                        float b) {
  *reinterpret_cast<uint32_t*>(tile + sw128(r, c, block_bytes)) = pack_bf16(a, b);
}
__device__ __forceinline__ float2 ld_pair(const unsigned char* tile, int r, int c, int block_bytes) {
  const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(tile + sw128(r, c, block_bytes));
  return __bfloat1622float2(h);
}
// Sum over the 4 lanes (t, t^1, t^2, t^3) that hold the same 16dp row.
__device__ __forceinline__ float quad_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  return x;
}

__device__ __forceinline__ bool failed(const Work& w) { return *((volatile int*)w.status) != 0; }


// Launch helper: raises the dynamic shared-memory limit, counts/brackets the launch.
template <typename Kern, typename... A>
cudaError_t tgo(const char* name, Kern kern, dim3 grid, int threads, size_t smem, cudaStream_t s,
                A... args) {
  if (grid.x == 0 || grid.y == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ProfScope ps(name, s);
  kern<<<grid, threads, smem, s>>>(args...);
  return cudaGetLastError();
}

cudaError_t tc_backward_kernels(const Problem& p, const Args& a, const Work& w, const TcWork& t,
                                const TcMaps& m, cudaStream_t s);
// The sequential passes over the chunks (gdn_tc_scan.cu): one CTA per (sequence, value head).
cudaError_t tc_scan_fwd(const Problem& p, const Args& a, const Work& w, const TcWork& t,
                        const TcMaps& m, const ScanRange& sr, cudaStream_t s);
cudaError_t tc_scan_bwd(const Problem& p, const Args& a, const Work& w, const TcWork& t,
                        const TcMaps& m, const ScanRange& sr, cudaStream_t s);

}  // namespace tcx
}  // namespace gdn
