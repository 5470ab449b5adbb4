// Chunk tables, the gate prologue fused with the in-chunk cumsum, and the backward's final
// per-token assembly (reverse in-chunk cumsum of dG, gate chain, group sums of dq/dk).
#include "gdn_common.cuh"
#include "gdn_launch.h"

namespace gdn {

// ---------------------------------------------------------------------------------------
// Chunk table.  One block of 1024 threads: per sequence n its chunk count ceil(len/64), an
// exclusive scan over sequences, then one entry per chunk.  Validates cu_seqlens (cu[0]=0,
// non-decreasing, cu[N]=T) and records the chunk count in status[1].
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) k_chunk_table(Problem p, const int64_t* __restrict__ cu,
                                                      int4* __restrict__ seq_tab,
                                                      int4* __restrict__ chunk_tab,
                                                      int* __restrict__ status,
                                                      int* __restrict__ count, int cap) {
  __shared__ int s_scan[1024];
  __shared__ int s_base, s_bad;
  const int tid = threadIdx.x;
  if (tid == 0) {
    s_base = 0;
    s_bad = 0;
  }
  __syncthreads();
  for (int n0 = 0; n0 < p.Nst; n0 += 1024) {
    const int n = n0 + tid;
    int bos = 0, len = 0, nch = 0;
    if (n < p.Nst) {
      if (cu) {
        const int64_t a = cu[n], b = cu[n + 1];
        if (a < 0 || b < a || b > (int64_t)p.T || (n == 0 && a != 0) ||
            (n == p.Nst - 1 && b != (int64_t)p.T))
          s_bad = 1;
        else {
          bos = (int)a;
          len = (int)(b - a);
        }
      } else {
        bos = n * p.T;
        len = p.T;
      }
      nch = (len + CH - 1) / CH;
    }
    s_scan[tid] = nch;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {
      const int x = tid >= off ? s_scan[tid - off] : 0;
      __syncthreads();
      s_scan[tid] += x;
      __syncthreads();
    }
    const int first = s_base + s_scan[tid] - nch;
    if (n < p.Nst) {
      if (seq_tab) seq_tab[n] = make_int4(first, nch, bos, len);
      for (int c = 0; c < nch; ++c) {
        const int gc = first + c;
        if (gc < cap)
          chunk_tab[gc] = make_int4(n, c, min(CH, len - c * CH), bos + c * CH);
        else
          s_bad = 1;
      }
    }
    __syncthreads();
    if (tid == 0) s_base += s_scan[1023];
    __syncthreads();
  }
  const int total = s_base;
  for (int gc = total + tid; gc < cap; gc += 1024) chunk_tab[gc] = make_int4(-1, -1, 0, 0);
  if (tid == 0) {
    if (status) status[0] = s_bad ? (int)GDN_ERR_INVALID_ARG : 0;
    if (count) count[0] = (s_bad && !status) ? -1 : total;
  }
}

// ---------------------------------------------------------------------------------------
// Gate prologue fused with the in-chunk cumsum.  One block per chunk: reads the chunk's
// [L x HV] slab of g_raw (contiguous), computes g, and per value head writes the inclusive
// cumsum G[hv][gc][0..63] (stride 1 along tokens, padded with G[L-1]) and beta padded
// with zeros.  This is the B200 form of the pages' "transpose g to [B,HV,T] so the time
// axis is stride 1" change, fused into the producer instead of a separate host pass.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_gate_cumsum(Problem p, Args a, Work w) {
  if (call_failed(w)) return;
  const int gc = blockIdx.x;
  const int4 e = w.chunk_tab[gc];
  if (e.x < 0) return;
  const int L = e.z, tok0 = e.w, HV = p.HV;
  extern __shared__ float s_g[];  // [64][HV] gate, then [64][HV] beta
  float* s_b = s_g + CH * HV;
  for (int i = threadIdx.x; i < CH * HV; i += blockDim.x) {
    const int t = i / HV, hv = i % HV;
    float gv = 0.f, bv = 0.f;
    if (t < L) {
      const size_t off = (size_t)(tok0 + t) * HV + hv;
      gv = gate_value(a.g_raw[off], a.A_log[hv], a.dt_bias[hv]);
      bv = a.beta[off];
    }
    s_g[i] = gv;
    s_b[i] = bv;
  }
  __syncthreads();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int hv = warp; hv < HV; hv += blockDim.x / 32) {
    // lane owns tokens 2*lane and 2*lane+1
    const float g0 = s_g[(2 * lane) * HV + hv], g1 = s_g[(2 * lane + 1) * HV + hv];
    float s = g0 + g1;
    for (int off = 1; off < 32; off <<= 1) {
      const float x = __shfl_up_sync(0xffffffffu, s, off);
      if (lane >= off) s += x;
    }
    const float incl1 = s, incl0 = s - g1;
    float2* Gp = reinterpret_cast<float2*>(w.G + ((size_t)hv * p.NCmax + gc) * CH);
    float2* Bp = reinterpret_cast<float2*>(w.beta_p + ((size_t)hv * p.NCmax + gc) * CH);
    Gp[lane] = make_float2(incl0, incl1);
    Bp[lane] = make_float2(s_b[(2 * lane) * HV + hv], s_b[(2 * lane + 1) * HV + hv]);
    // decay vectors of the chunk: e^{G_63 - G_i} (G_63 = the last lane's inclusive sum) and e^{G_i}
    const float gl = __shfl_sync(0xffffffffu, incl1, 31);
    float2* Dp = reinterpret_cast<float2*>(w.Dec + ((size_t)hv * p.NCmax + gc) * CH);
    float2* Ep = reinterpret_cast<float2*>(w.EG + ((size_t)hv * p.NCmax + gc) * CH);
    Dp[lane] = make_float2(expf(gl - incl0), expf(gl - incl1));
    Ep[lane] = make_float2(expf(incl0), expf(incl1));
  }
}

// ---------------------------------------------------------------------------------------
// Backward assembly per chunk: dg = reverse in-chunk cumsum of dG (the gradient of
// G = cumsum g) and the optional d g_raw through the gate (one warp per value head); then
// dq/dk as the sum of the value heads' shares over each k-head's group.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_bwd_tokens(Problem p, Args a, Work w) {
  if (call_failed(w)) return;
  const int gc = blockIdx.x;
  const int4 e = w.chunk_tab[gc];
  if (e.x < 0) return;
  const int L = e.z, tok0 = e.w;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int hv = warp; hv < p.HV; hv += blockDim.x / 32) {
    const float* dGp = w.dG + ((size_t)hv * p.NCmax + gc) * CH;
    // suffix sums: lane owns positions 2*lane, 2*lane+1; scan from the top lane down
    float d0 = dGp[2 * lane], d1 = dGp[2 * lane + 1];
    if (w.dG2) {
      const float* dG2p = w.dG2 + ((size_t)hv * p.NCmax + gc) * CH;
      d0 += dG2p[2 * lane];
      d1 += dG2p[2 * lane + 1];
    }
    float s = d0 + d1;
    for (int off = 1; off < 32; off <<= 1) {
      const float x = __shfl_down_sync(0xffffffffu, s, off);
      if (lane + off < 32) s += x;
    }
    const float suf0 = s, suf1 = s - d0;
    for (int j = 0; j < 2; ++j) {
      const int t = 2 * lane + j;
      if (t < L) {
        const size_t off = (size_t)(tok0 + t) * p.HV + hv;
        const float dgv = j ? suf1 : suf0;
        a.dg[off] = dgv;
        if (a.dg_raw) {
          const float x = a.g_raw[off] + a.dt_bias[hv];
          a.dg_raw[off] = dgv * (-expf(a.A_log[hv])) * gate_dsoftplus(x);
        }
      }
    }
  }
}

// dq, dk of k-head h for one chunk: sums of the per-value-head shares over the G value heads
// of the group (fp32 [chunk][hv][64][K] -> [token][h][K]), four columns per thread and step.
template <typename T>
__global__ void __launch_bounds__(256) k_dqdk_group_sum(Problem p, Args a, Work w) {
  if (call_failed(w)) return;
  const int gc = blockIdx.x, h = blockIdx.y;
  const int4 e = w.chunk_tab[gc];
  if (e.x < 0) return;
  const int L = e.z, tok0 = e.w, K = p.K, ld = p.share_ld;
  T* dq = static_cast<T*>(a.dq);
  T* dk = static_cast<T*>(a.dk);
  const size_t base = ((size_t)gc * p.HV + (size_t)h * p.G) * CH * ld;  // value head h*G, row 0
  for (int i = 4 * threadIdx.x; i < L * K; i += 4 * blockDim.x) {
    float4 sq = make_float4(0.f, 0.f, 0.f, 0.f), sk = sq;
    for (int j = 0; j < p.G; ++j) {
      const size_t o = base + (size_t)j * CH * ld + (size_t)(i / K) * ld + i % K;
      const float4 x = *reinterpret_cast<const float4*>(w.dqp + o);
      const float4 y = *reinterpret_cast<const float4*>(w.dkp + o);
      sq.x += x.x; sq.y += x.y; sq.z += x.z; sq.w += x.w;
      sk.x += y.x; sk.y += y.y; sk.z += y.z; sk.w += y.w;
      if (w.dkp2) {
        const float4 z = *reinterpret_cast<const float4*>(w.dkp2 + o);
        sk.x += z.x; sk.y += z.y; sk.z += z.z; sk.w += z.w;
      }
    }
    const int t = i / K, c = i % K;
    T* q4 = dq + ((size_t)(tok0 + t) * p.H + h) * K + c;
    T* k4 = dk + ((size_t)(tok0 + t) * p.H + h) * K + c;
    q4[0] = from_f<T>(sq.x); q4[1] = from_f<T>(sq.y); q4[2] = from_f<T>(sq.z); q4[3] = from_f<T>(sq.w);
    k4[0] = from_f<T>(sk.x); k4[1] = from_f<T>(sk.y); k4[2] = from_f<T>(sk.z); k4[3] = from_f<T>(sk.w);
  }
}

// dA_log[hv] = sum_t dg_t g_t ;  ddt_bias[hv] = sum_t dL/dx_t.  One block per value head,
// deterministic order.
// dA_log = sum_t dg_t g_t and ddt_bias = sum_t dg_t (-e^{A_log}) softplus'(x_t) per value head,
// in two deterministic passes: PG_BLOCKS token blocks each write per-head partial sums
// (threads read [token][head] rows contiguously; 256 % HV == 0 keeps a thread on one head),
// then one thread per head adds the partials in block order.
__global__ void __launch_bounds__(256) k_param_grads_partial(Problem p, Args a, Work w) {
  if (call_failed(w)) return;
  const int HV = p.HV, tid = threadIdx.x, h = tid % HV, lanes = 256 / HV, l = tid / HV;
  const int ntok = p.B * p.T;
  const int per = (ntok + PG_BLOCKS - 1) / PG_BLOCKS;
  const int t0 = blockIdx.x * per, t1 = min(ntok, t0 + per);
  const float Al = a.A_log[h], db = a.dt_bias[h], nexp = -expf(Al);
  float s1 = 0.f, s2 = 0.f;
  for (int t = t0 + l; t < t1; t += lanes) {
    const size_t off = (size_t)t * HV + h;
    const float dgv = a.dg[off], x = a.g_raw[off] + db;
    s1 += dgv * gate_value(a.g_raw[off], Al, db);
    s2 += dgv * nexp * gate_dsoftplus(x);
  }
  __shared__ float r1[256], r2[256];
  r1[tid] = s1;
  r2[tid] = s2;
  __syncthreads();
  if (tid < HV) {
    float u1 = 0.f, u2 = 0.f;
    for (int j = 0; j < lanes; ++j) {
      u1 += r1[j * HV + tid];
      u2 += r2[j * HV + tid];
    }
    w.pgp[((size_t)blockIdx.x * HV + tid) * 2] = u1;
    w.pgp[((size_t)blockIdx.x * HV + tid) * 2 + 1] = u2;
  }
}

__global__ void k_param_grads_final(Problem p, Args a, Work w) {
  if (call_failed(w)) return;
  for (int h = blockIdx.x * blockDim.x + threadIdx.x; h < p.HV; h += gridDim.x * blockDim.x) {
    float u1 = 0.f, u2 = 0.f;
    for (int b = 0; b < PG_BLOCKS; ++b) {
      u1 += w.pgp[((size_t)b * p.HV + h) * 2];
      u2 += w.pgp[((size_t)b * p.HV + h) * 2 + 1];
    }
    if (a.dA_log) a.dA_log[h] = u1;
    if (a.ddt_bias) a.ddt_bias[h] = u2;
  }
}

// One CTA per value head (any HV): the reduction when 256 % HV != 0.
__global__ void __launch_bounds__(256) k_param_grads(Problem p, Args a, Work w) {
  if (call_failed(w)) return;
  const int hv = blockIdx.x;
  const float Al = a.A_log[hv], db = a.dt_bias[hv];
  float s1 = 0.f, s2 = 0.f;
  const int ntok = p.B * p.T;
  for (int t = threadIdx.x; t < ntok; t += blockDim.x) {
    const size_t off = (size_t)t * p.HV + hv;
    const float dgv = a.dg[off];
    const float x = a.g_raw[off] + db;
    s1 += dgv * gate_value(a.g_raw[off], Al, db);
    s2 += dgv * (-expf(Al)) * gate_dsoftplus(x);
  }
  __shared__ float r1[256], r2[256];
  r1[threadIdx.x] = s1;
  r2[threadIdx.x] = s2;
  __syncthreads();
  for (int off = 128; off > 0; off >>= 1) {
    if (threadIdx.x < off) {
      r1[threadIdx.x] += r1[threadIdx.x + off];
      r2[threadIdx.x] += r2[threadIdx.x + off];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    if (a.dA_log) a.dA_log[hv] = r1[0];
    if (a.ddt_bias) a.ddt_bias[hv] = r2[0];
  }
}

// ------------------------------------------------------------------- launchers
cudaError_t launch_chunk_table(const Problem& p, const int64_t* cu, const Work& w,
                               cudaStream_t s) {
  ProfScope ps("chunk_table", s);
  k_chunk_table<<<1, 1024, 0, s>>>(p, cu, w.seq_tab, w.chunk_tab, w.status, w.status + 1, p.NCmax);
  return cudaGetLastError();
}

cudaError_t launch_chunk_table_only(const Problem& p, const int64_t* cu, int4* table, int* count,
                                    cudaStream_t s) {
  ProfScope ps("chunk_table", s);
  k_chunk_table<<<1, 1024, 0, s>>>(p, cu, nullptr, table, nullptr, count, p.NCmax);
  return cudaGetLastError();
}

cudaError_t launch_gate_cumsum(const Problem& p, const Args& a, const Work& w, cudaStream_t s) {
  if (p.NCmax == 0) return cudaSuccess;
  const size_t smem = (size_t)2 * CH * p.HV * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k_gate_cumsum, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  ProfScope ps("gate_cumsum", s);
  k_gate_cumsum<<<p.NCmax, 256, smem, s>>>(p, a, w);
  return cudaGetLastError();
}

cudaError_t launch_param_grads(const Problem& p, const Args& a, const Work& w, cudaStream_t s) {
  if (!(a.dA_log || a.ddt_bias)) return cudaSuccess;
  if (256 % p.HV == 0 && w.pgp) {
    {
      ProfScope ps("param_grads", s);
      k_param_grads_partial<<<PG_BLOCKS, 256, 0, s>>>(p, a, w);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    ProfScope ps("param_grads_final", s);
    k_param_grads_final<<<(p.HV + 255) / 256, 256, 0, s>>>(p, a, w);
  } else {
    ProfScope ps("param_grads", s);
    k_param_grads<<<p.HV, 256, 0, s>>>(p, a, w);
  }
  return cudaGetLastError();
}

cudaError_t launch_bwd_tokens(const Problem& p, const Args& a, const Work& w, bool bf16,
                              cudaStream_t s, bool group_sum) {
  if (p.NCmax == 0 && !(a.dA_log || a.ddt_bias)) return cudaSuccess;
  if (p.NCmax == 0) return launch_param_grads(p, a, w, s);
  {
    ProfScope ps("bwd_tokens", s);
    k_bwd_tokens<<<p.NCmax, 256, 0, s>>>(p, a, w);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (group_sum && (e = launch_dqdk_group_sum(p, a, w, bf16, s)) != cudaSuccess) return e;
  if (a.dA_log || a.ddt_bias) e = launch_param_grads(p, a, w, s);
  return e;
}

cudaError_t launch_dqdk_group_sum(const Problem& p, const Args& a, const Work& w, bool bf16, cudaStream_t s) {
  if (p.NCmax == 0) return cudaSuccess;
  ProfScope ps("dqdk_group_sum", s);
  const dim3 g(p.NCmax, p.H);
  if (bf16)
    k_dqdk_group_sum<__nv_bfloat16><<<g, 256, 0, s>>>(p, a, w);
  else
    k_dqdk_group_sum<float><<<g, 256, 0, s>>>(p, a, w);
  return cudaGetLastError();
}

}  // namespace gdn
