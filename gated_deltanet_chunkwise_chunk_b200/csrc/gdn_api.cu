// C-ABI entry points: argument validation, workspace carve-up and the launch sequences.
#include <cmath>
#include <cstdint>
#include <cstring>

#include "gdn.h"
#include "gdn_common.cuh"
#include "gdn_launch.h"
#include "gdn_tc.h"

namespace gdn {
namespace {

constexpr size_t kAlign = 256;

inline size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t max_chunks(const gdn_dims& d, bool varlen) {
  if (varlen) return (d.T + 63 * d.N) / CH;
  return d.B * ((d.T + CH - 1) / CH);
}

// Validates dims; 0 on success.
int check_dims(const gdn_dims* d, bool varlen) {
  if (!d) return GDN_ERR_INVALID_ARG;
  if (d->B <= 0 || d->T < 0 || d->H <= 0 || d->HV <= 0 || d->K <= 0 || d->V <= 0)
    return GDN_ERR_INVALID_ARG;
  if (d->HV % d->H) return GDN_ERR_INVALID_ARG;
  if (varlen && (d->B != 1 || d->N <= 0)) return GDN_ERR_INVALID_ARG;
  if ((d->K != 64 && d->K != 128) || (d->V != 64 && d->V != 128)) return GDN_ERR_UNSUPPORTED;
  if (d->dtype != GDN_DTYPE_FP32 && d->dtype != GDN_DTYPE_BF16) return GDN_ERR_UNSUPPORTED;
  if (d->B * d->T >= (int64_t)1 << 31 || d->HV > 65535) return GDN_ERR_INVALID_ARG;
  if (max_chunks(*d, varlen) >= (int64_t)1 << 30) return GDN_ERR_INVALID_ARG;
  // per-(chunk, value head) tiles are addressed by 32-bit TMA row coordinates (unit x 128)
  if (max_chunks(*d, varlen) * d->HV * 128 >= (int64_t)1 << 31) return GDN_ERR_INVALID_ARG;
  if (!(d->scale >= 0.f) || std::isinf(d->scale)) return GDN_ERR_INVALID_ARG;
  return GDN_OK;
}

// Byte offsets of the workspace regions (FFMA path layout; the tcgen05 path appends its
// own regions after the common ones).
struct Plan {
  size_t status, seq_tab, chunk_tab, G, beta_p, Dec, EG;
  size_t W, Ut, Tm, h, U, dU, dh, dW, dqp, dkp, dG, dkp2, dG2, tmp, pgp;
  size_t tc;     // start of the tcgen05 path's region
  size_t total;
};

Plan make_plan(const gdn_dims& d, bool varlen, int pass) {
  Plan pl{};
  const size_t NC = (size_t)max_chunks(d, varlen);
  const size_t Nst = varlen ? (size_t)d.N : (size_t)d.B;
  const size_t HV = d.HV, K = d.K, V = d.V, f = sizeof(float);
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += up(bytes);
    return at;
  };
  pl.status = take(64);
  pl.seq_tab = take(Nst * sizeof(int4));
  pl.chunk_tab = take(NC * sizeof(int4));
  pl.G = take(HV * NC * CH * f);
  pl.beta_p = take(HV * NC * CH * f);
  pl.Dec = take(HV * NC * CH * f);
  pl.EG = take(HV * NC * CH * f);
  const bool ffma = pass == 0 ? !(d.dtype == GDN_DTYPE_BF16 && tc_supported(d))
                              : !(d.dtype == GDN_DTYPE_BF16 && tc_bwd_supported(d));
  if (ffma) {
    pl.W = take(NC * HV * CH * K * f);
    pl.Ut = take(NC * HV * CH * V * f);
    pl.h = take(NC * HV * V * K * f);
    pl.U = take(NC * HV * CH * V * f);
    if (pass == 1) {
      pl.Tm = take(NC * HV * CH * CH * f);
      pl.dU = take(NC * HV * CH * V * f);
      pl.dh = take(NC * HV * V * K * f);
      pl.dW = take(NC * HV * CH * K * f);
      pl.dqp = take(NC * HV * CH * K * f);
      pl.dkp = take(NC * HV * CH * K * f);
      pl.dG = take(HV * NC * CH * f);
      pl.tmp = take(NC * HV * CH * 128 * f);
    }
  } else {
    // the tcgen05 region starts at the same offset for both passes, so a backward can read
    // what the forward left in the same workspace
    pl.tc = take(tc_workspace_bytes(d, NC, pass));
    if (pass == 1) {  // fp32 per-value-head dq/dk shares (128 wide) and dG parts, read by the final assembly
      pl.dqp = take(NC * HV * CH * 128 * f);
      pl.dkp = take(NC * HV * CH * 128 * f);
      pl.dG = take(HV * NC * CH * f);
      pl.dG2 = take(HV * NC * CH * f);
    }
  }
  if (pass == 1) pl.pgp = take((size_t)PG_BLOCKS * HV * 2 * f);
  pl.total = o;
  return pl;
}

Work carve(const Plan& pl, void* ws) {
  char* b = static_cast<char*>(ws);
  Work w{};
  w.status = reinterpret_cast<int*>(b + pl.status);
  w.seq_tab = reinterpret_cast<int4*>(b + pl.seq_tab);
  w.chunk_tab = reinterpret_cast<int4*>(b + pl.chunk_tab);
  w.G = reinterpret_cast<float*>(b + pl.G);
  w.beta_p = reinterpret_cast<float*>(b + pl.beta_p);
  w.Dec = reinterpret_cast<float*>(b + pl.Dec);
  w.EG = reinterpret_cast<float*>(b + pl.EG);
  auto fp = [&](size_t off) { return off ? reinterpret_cast<float*>(b + off) : nullptr; };
  w.W = fp(pl.W);
  w.Ut = fp(pl.Ut);
  w.Tm = fp(pl.Tm);
  w.h = fp(pl.h);
  w.U = fp(pl.U);
  w.dU = fp(pl.dU);
  w.dh = fp(pl.dh);
  w.dW = fp(pl.dW);
  w.dqp = fp(pl.dqp);
  w.dkp = fp(pl.dkp);
  w.dG = fp(pl.dG);
  w.dkp2 = fp(pl.dkp2);
  w.dG2 = fp(pl.dG2);
  w.tmp = fp(pl.tmp);
  w.pgp = fp(pl.pgp);
  return w;
}

Problem make_problem(const gdn_dims& d, bool varlen) {
  Problem p{};
  p.B = (int)d.B;
  p.T = (int)d.T;
  p.H = (int)d.H;
  p.HV = (int)d.HV;
  p.K = (int)d.K;
  p.V = (int)d.V;
  p.Nst = varlen ? (int)d.N : (int)d.B;
  p.G = (int)(d.HV / d.H);
  p.varlen = varlen ? 1 : 0;
  p.NCmax = (int)max_chunks(d, varlen);
  p.scale = d.scale > 0.f ? d.scale : 1.f / std::sqrt((float)d.K);
  p.test_timeout = (d.flags & GDN_FLAG_TEST_WAIT_TIMEOUT) ? 1 : 0;
  p.share_ld = (int)d.K;
  return p;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA; }

// Workspace of the chunkwise KDA forward.
struct KdaPlan {
  size_t status, seq_tab, chunk_tab, W, Ut, Kh, Qt, P, eGC, h, U;
  size_t Gam, Tm, dU, dh, dW, dGam, dqp, dkp, pgp;  // pass 1 only
  size_t total;
};

KdaPlan make_kda_plan(const gdn_dims& d, bool varlen, int pass) {
  KdaPlan pl{};
  const size_t NC = (size_t)max_chunks(d, varlen), Nst = varlen ? (size_t)d.N : (size_t)d.B;
  const size_t HV = d.HV, K = d.K, V = d.V, f = sizeof(float);
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += up(bytes);
    return at;
  };
  pl.status = take(64);
  pl.seq_tab = take(Nst * sizeof(int4));
  pl.chunk_tab = take(NC * sizeof(int4));
  pl.W = take(NC * HV * CH * K * f);
  pl.Ut = take(NC * HV * CH * V * f);
  pl.Kh = take(NC * HV * CH * K * f);
  pl.Qt = take(NC * HV * CH * K * f);
  pl.P = take(NC * HV * CH * CH * f);
  pl.eGC = take(NC * HV * K * f);
  pl.h = take(NC * HV * V * K * f);
  pl.U = take(NC * HV * CH * V * f);
  if (pass == 1) {
    pl.Gam = take(NC * HV * CH * K * f);
    pl.Tm = take(NC * HV * CH * CH * f);
    pl.dU = take(NC * HV * CH * V * f);
    pl.dh = take(NC * HV * V * K * f);
    pl.dW = take(NC * HV * CH * K * f);
    pl.dGam = take(NC * HV * CH * K * f);
    pl.dqp = take(NC * HV * CH * K * f);
    pl.dkp = take(NC * HV * CH * K * f);
    pl.pgp = take(NC * HV * (K + 1) * f);
  }
  pl.total = o;
  return pl;
}

KdaWork carve_kda(const KdaPlan& pl, void* ws) {
  char* b = static_cast<char*>(ws);
  KdaWork w{};
  w.status = reinterpret_cast<int*>(b + pl.status);
  w.seq_tab = reinterpret_cast<int4*>(b + pl.seq_tab);
  w.chunk_tab = reinterpret_cast<int4*>(b + pl.chunk_tab);
  auto fp = [&](size_t off) { return off ? reinterpret_cast<float*>(b + off) : nullptr; };
  w.W = fp(pl.W);
  w.Ut = fp(pl.Ut);
  w.Kh = fp(pl.Kh);
  w.Qt = fp(pl.Qt);
  w.P = fp(pl.P);
  w.eGC = fp(pl.eGC);
  w.h = fp(pl.h);
  w.U = fp(pl.U);
  w.Gam = fp(pl.Gam);
  w.Tm = fp(pl.Tm);
  w.dU = fp(pl.dU);
  w.dh = fp(pl.dh);
  w.dW = fp(pl.dW);
  w.dGam = fp(pl.dGam);
  w.dqp = fp(pl.dqp);
  w.dkp = fp(pl.dkp);
  w.pgp = fp(pl.pgp);
  return w;
}

// Steps shared by the forward and the backward: chunk table, gate + in-chunk cumsum.
cudaError_t prologue(const Problem& p, const Args& a, const Work& w, cudaStream_t s) {
  cudaError_t e = launch_chunk_table(p, a.cu, w, s);
  if (e != cudaSuccess) return e;
  return launch_gate_cumsum(p, a, w, s);
}

}  // namespace
}  // namespace gdn

using namespace gdn;

extern "C" {

size_t gdn_workspace_bytes(const gdn_dims* d, int varlen, int pass) {
  if (check_dims(d, varlen != 0) != GDN_OK || (pass != 0 && pass != 1)) return 0;
  return make_plan(*d, varlen != 0, pass).total;
}

int64_t gdn_max_chunks(const gdn_dims* d, int varlen) {
  if (check_dims(d, varlen != 0) != GDN_OK) return -GDN_ERR_INVALID_ARG;
  return max_chunks(*d, varlen != 0);
}

int gdn_chunk_fwd(const gdn_dims* d, const void* q, const void* k, const void* v,
                  const float* g_raw, const float* A_log, const float* dt_bias, const float* beta,
                  const int64_t* cu_seqlens, const float* initial_state, void* o, float* final_state,
                  void* workspace, size_t workspace_bytes, void* stream) {
  const bool varlen = cu_seqlens != nullptr;
  int rc = check_dims(d, varlen);
  if (rc) return rc;
  // per-token tensors may be null when there are no tokens (B*T == 0)
  const bool empty = d->B * d->T == 0;
  const void* tok[] = {q, k, v, g_raw, beta, o};
  for (const void* x : tok)
    if ((!x && !empty) || !aligned16(x)) return GDN_ERR_INVALID_ARG;
  if (!A_log || !dt_bias || !aligned16(A_log) || !aligned16(dt_bias)) return GDN_ERR_INVALID_ARG;
  if (!aligned16(cu_seqlens) || !aligned16(initial_state) || !aligned16(final_state))
    return GDN_ERR_INVALID_ARG;
  const Plan pl = make_plan(*d, varlen, 0);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) || workspace_bytes < pl.total)
    return GDN_ERR_WORKSPACE;
  // shapes the tcgen05 path covers never run on the CUDA-core kernels instead
  if (tc_supported(*d) && !tc_ready()) return GDN_ERR_UNSUPPORTED;
  const Problem p = make_problem(*d, varlen);
  Args a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.g_raw = g_raw;
  a.A_log = A_log;
  a.dt_bias = dt_bias;
  a.beta = beta;
  a.cu = cu_seqlens;
  a.h0 = initial_state;
  a.o = o;
  a.ht = final_state;
  const Work w = carve(pl, workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = prologue(p, a, w, s);
  if (e != cudaSuccess) return cuda_status(e);
  const bool bf16 = d->dtype == GDN_DTYPE_BF16;
  if (bf16 && tc_supported(*d))
    e = tc_forward(p, a, w, static_cast<char*>(workspace) + pl.tc, s);
  else
    e = ffma_forward(p, a, w, bf16, false, s);
  return cuda_status(e);
}

int gdn_chunk_bwd(const gdn_dims* d, const void* q, const void* k, const void* v,
                  const float* g_raw, const float* A_log, const float* dt_bias, const float* beta,
                  const int64_t* cu_seqlens, const float* initial_state, const void* d_o,
                  const float* dht, void* dq, void* dk, void* dv, float* dg, float* dbeta,
                  float* dh0, float* dg_raw, float* dA_log, float* ddt_bias, void* workspace,
                  size_t workspace_bytes, void* stream) {
  const bool varlen = cu_seqlens != nullptr;
  int rc = check_dims(d, varlen);
  if (rc) return rc;
  const bool empty = d->B * d->T == 0;
  const void* tok[] = {q, k, v, g_raw, beta, d_o, dq, dk, dv, dg, dbeta};
  for (const void* x : tok)
    if ((!x && !empty) || !aligned16(x)) return GDN_ERR_INVALID_ARG;
  if (!A_log || !dt_bias || !aligned16(A_log) || !aligned16(dt_bias)) return GDN_ERR_INVALID_ARG;
  const void* opt[] = {cu_seqlens, initial_state, dht, dh0, dg_raw, dA_log, ddt_bias};
  for (const void* x : opt)
    if (!aligned16(x)) return GDN_ERR_INVALID_ARG;
  const Plan pl = make_plan(*d, varlen, 1);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) || workspace_bytes < pl.total)
    return GDN_ERR_WORKSPACE;
  // shapes the tcgen05 path covers never run on the CUDA-core kernels instead
  if (tc_bwd_supported(*d) && !tc_ready()) return GDN_ERR_UNSUPPORTED;
  Problem p = make_problem(*d, varlen);
  if (tc_bwd_supported(*d)) p.share_ld = 128;  // the tcgen05 kernels' shares are 128 wide
  Args a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.g_raw = g_raw;
  a.A_log = A_log;
  a.dt_bias = dt_bias;
  a.beta = beta;
  a.cu = cu_seqlens;
  a.h0 = initial_state;
  a.dO = d_o;
  a.dht = dht;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.dg = dg;
  a.dbeta = dbeta;
  a.dh0 = dh0;
  a.dg_raw = dg_raw;
  a.dA_log = dA_log;
  a.ddt_bias = ddt_bias;
  const Work w = carve(pl, workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool bf16 = d->dtype == GDN_DTYPE_BF16;
  const bool tc = bf16 && tc_bwd_supported(*d);
  // with the forward's workspace reused, its chunk tables, gates and status word are kept
  const bool reuse = tc && (d->flags & GDN_FLAG_BWD_REUSE_FWD) != 0;
  cudaError_t e = reuse ? cudaSuccess : prologue(p, a, w, s);
  if (e != cudaSuccess) return cuda_status(e);
  if (tc) {
    e = tc_backward(p, a, w, static_cast<char*>(workspace) + pl.tc,
                    (d->flags & GDN_FLAG_BWD_REUSE_FWD) != 0, s);
    if (e != cudaSuccess) return cuda_status(e);
  } else {
    e = ffma_forward(p, a, w, bf16, true, s);
    if (e != cudaSuccess) return cuda_status(e);
    e = ffma_backward(p, a, w, bf16, s);
    if (e != cudaSuccess) return cuda_status(e);
    e = launch_bwd_tokens(p, a, w, bf16, s);
  }
  return cuda_status(e);
}

int64_t gdn_build_chunk_indices(const gdn_dims* d, const int64_t* cu_host, int32_t* out_host,
                                int64_t cap) {
  const bool varlen = cu_host != nullptr;
  if (check_dims(d, varlen) != GDN_OK) return -GDN_ERR_INVALID_ARG;
  if (cap > 0 && !out_host) return -GDN_ERR_INVALID_ARG;
  const int64_t Nst = varlen ? d->N : d->B;
  if (varlen) {
    if (cu_host[0] != 0 || cu_host[Nst] != d->T) return -GDN_ERR_INVALID_ARG;
    for (int64_t n = 0; n < Nst; ++n)
      if (cu_host[n + 1] < cu_host[n]) return -GDN_ERR_INVALID_ARG;
  }
  int64_t count = 0;
  for (int64_t n = 0; n < Nst; ++n) {
    const int64_t bos = varlen ? cu_host[n] : n * d->T;
    const int64_t len = varlen ? cu_host[n + 1] - cu_host[n] : d->T;
    for (int64_t c = 0; c * CH < len; ++c, ++count) {
      if (count < cap) {
        out_host[4 * count + 0] = (int32_t)n;
        out_host[4 * count + 1] = (int32_t)c;
        out_host[4 * count + 2] = (int32_t)(len - c * CH < CH ? len - c * CH : CH);
        out_host[4 * count + 3] = (int32_t)(bos + c * CH);
      }
    }
  }
  return count;
}

int gdn_chunk_table_device(const gdn_dims* d, const int64_t* cu_seqlens, int32_t* table,
                           int64_t cap, int32_t* count_dev, void* stream) {
  const bool varlen = cu_seqlens != nullptr;
  int rc = check_dims(d, varlen);
  if (rc) return rc;
  if (!table || !count_dev || cap <= 0 || cap >= ((int64_t)1 << 30) || !aligned16(table))
    return GDN_ERR_INVALID_ARG;
  Problem p = make_problem(*d, varlen);
  p.NCmax = (int)cap;
  return cuda_status(launch_chunk_table_only(p, cu_seqlens, reinterpret_cast<int4*>(table),
                                             count_dev, static_cast<cudaStream_t>(stream)));
}

size_t gdn_recurrent_workspace_bytes(void) { return GDN_RECURRENT_WORKSPACE_BYTES; }

static int recurrent_common(const gdn_dims* d, const void* q, const void* k, const void* v,
                            const float* g_raw, const float* A_log, const float* dt_bias,
                            const float* beta, const int64_t* cu_seqlens, const float* initial_state,
                            void* o, float* final_state, void* workspace, size_t workspace_bytes,
                            void* stream, bool kda) {
  const bool varlen = cu_seqlens != nullptr;
  int rc = check_dims(d, varlen);
  if (rc) return rc;
  const bool empty = d->B * d->T == 0;
  if ((varlen ? d->N : d->B) * (d->V / 32) > (int64_t)INT32_MAX) return GDN_ERR_INVALID_ARG;  // grid.x
  const void* tok[] = {q, k, v, g_raw, beta, o};
  for (const void* x : tok)
    if ((!x && !empty) || !aligned16(x)) return GDN_ERR_INVALID_ARG;
  if (!A_log || (!dt_bias && !kda) || !aligned16(A_log) || !aligned16(dt_bias)) return GDN_ERR_INVALID_ARG;
  if (!aligned16(cu_seqlens) || !aligned16(initial_state) || !aligned16(final_state))
    return GDN_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) ||
      workspace_bytes < GDN_RECURRENT_WORKSPACE_BYTES)
    return GDN_ERR_WORKSPACE;
  const Problem p = make_problem(*d, varlen);
  Args a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.g_raw = g_raw;
  a.A_log = A_log;
  a.dt_bias = dt_bias;
  a.beta = beta;
  a.cu = cu_seqlens;
  a.h0 = initial_state;
  a.o = o;
  a.ht = final_state;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, 64, s);  // the device status word
  if (e == cudaSuccess)
    e = recurrent_forward(p, a, static_cast<int*>(workspace), d->dtype == GDN_DTYPE_BF16, s, kda);
  return cuda_status(e);
}

int gdn_recurrent_fwd(const gdn_dims* d, const void* q, const void* k, const void* v,
                      const float* g_raw, const float* A_log, const float* dt_bias, const float* beta,
                      const int64_t* cu_seqlens, const float* initial_state, void* o,
                      float* final_state, void* workspace, size_t workspace_bytes, void* stream) {
  return recurrent_common(d, q, k, v, g_raw, A_log, dt_bias, beta, cu_seqlens, initial_state, o,
                          final_state, workspace, workspace_bytes, stream, false);
}

int gdn_kda_recurrent_fwd(const gdn_dims* d, const void* q, const void* k, const void* v,
                          const float* g_raw, const float* A_log, const float* dt_bias,
                          const float* beta, const int64_t* cu_seqlens, const float* initial_state,
                          void* o, float* final_state, void* workspace, size_t workspace_bytes,
                          void* stream) {
  return recurrent_common(d, q, k, v, g_raw, A_log, dt_bias, beta, cu_seqlens, initial_state, o,
                          final_state, workspace, workspace_bytes, stream, true);
}

size_t gdn_kda_chunk_workspace_bytes(const gdn_dims* d, int varlen, int pass) {
  if (check_dims(d, varlen != 0) != GDN_OK || (pass != 0 && pass != 1)) return 0;
  return make_kda_plan(*d, varlen != 0, pass).total;
}

int gdn_kda_chunk_fwd(const gdn_dims* d, const void* q, const void* k, const void* v,
                      const float* g_raw, const float* A_log, const float* dt_bias, const float* beta,
                      const int64_t* cu_seqlens, const float* initial_state, void* o,
                      float* final_state, void* workspace, size_t workspace_bytes, void* stream) {
  const bool varlen = cu_seqlens != nullptr;
  int rc = check_dims(d, varlen);
  if (rc) return rc;
  const bool empty = d->B * d->T == 0;
  const void* tok[] = {q, k, v, g_raw, beta, o};
  for (const void* x : tok)
    if ((!x && !empty) || !aligned16(x)) return GDN_ERR_INVALID_ARG;
  if (!A_log || !aligned16(A_log) || !aligned16(dt_bias)) return GDN_ERR_INVALID_ARG;
  if (!aligned16(cu_seqlens) || !aligned16(initial_state) || !aligned16(final_state))
    return GDN_ERR_INVALID_ARG;
  const KdaPlan pl0 = make_kda_plan(*d, varlen, 0), pl1 = make_kda_plan(*d, varlen, 1);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) || workspace_bytes < pl0.total)
    return GDN_ERR_WORKSPACE;
  // a workspace sized for the backward also keeps what the backward reads
  const KdaPlan& pl = workspace_bytes >= pl1.total ? pl1 : pl0;
  const Problem p = make_problem(*d, varlen);
  Args a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.g_raw = g_raw;
  a.A_log = A_log;
  a.dt_bias = dt_bias;
  a.beta = beta;
  a.cu = cu_seqlens;
  a.h0 = initial_state;
  a.o = o;
  a.ht = final_state;
  const KdaWork w = carve_kda(pl, workspace);
  Work cw{};  // the chunk table kernel's view of the same status word and tables
  cw.status = w.status;
  cw.seq_tab = w.seq_tab;
  cw.chunk_tab = w.chunk_tab;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_chunk_table(p, cu_seqlens, cw, s);
  if (e == cudaSuccess) e = kda_chunk_forward(p, a, w, d->dtype == GDN_DTYPE_BF16, s);
  return cuda_status(e);
}

int gdn_kda_chunk_bwd(const gdn_dims* d, const void* q, const void* k, const void* v,
                      const float* g_raw, const float* A_log, const float* dt_bias, const float* beta,
                      const int64_t* cu_seqlens, const void* d_o, const float* dht, void* dq, void* dk,
                      void* dv, float* dg, float* dbeta, float* dh0, float* dg_raw, float* dA_log,
                      float* ddt_bias, void* workspace, size_t workspace_bytes, void* stream) {
  const bool varlen = cu_seqlens != nullptr;
  int rc = check_dims(d, varlen);
  if (rc) return rc;
  const bool empty = d->B * d->T == 0;
  const void* tok[] = {q, k, v, g_raw, beta, d_o, dq, dk, dv, dg, dbeta};
  for (const void* x : tok)
    if ((!x && !empty) || !aligned16(x)) return GDN_ERR_INVALID_ARG;
  if (!A_log || !aligned16(A_log) || !aligned16(dt_bias)) return GDN_ERR_INVALID_ARG;
  if (ddt_bias && !dt_bias) return GDN_ERR_INVALID_ARG;
  const void* opt[] = {cu_seqlens, dht, dh0, dg_raw, dA_log, ddt_bias};
  for (const void* x : opt)
    if (!aligned16(x)) return GDN_ERR_INVALID_ARG;
  const KdaPlan pl = make_kda_plan(*d, varlen, 1);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) || workspace_bytes < pl.total)
    return GDN_ERR_WORKSPACE;
  const Problem p = make_problem(*d, varlen);
  Args a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.g_raw = g_raw;
  a.A_log = A_log;
  a.dt_bias = dt_bias;
  a.beta = beta;
  a.cu = cu_seqlens;
  a.dO = d_o;
  a.dht = dht;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.dg = dg;
  a.dbeta = dbeta;
  a.dh0 = dh0;
  a.dg_raw = dg_raw;
  a.dA_log = dA_log;
  a.ddt_bias = ddt_bias;
  return cuda_status(kda_chunk_backward(p, a, carve_kda(pl, workspace), d->dtype == GDN_DTYPE_BF16,
                                        static_cast<cudaStream_t>(stream)));
}

int gdn_state_affine(int64_t count, int64_t K, int64_t V, const float* A, int transpose_a, const float* X,
                     const float* B, float* out, void* stream) {
  if (count < 0 || count > INT32_MAX || K < 1 || K > 128 || V < 32 || V % 32 || V / 32 > 65535)
    return GDN_ERR_INVALID_ARG;
  if (count > 0 && (!A || !X || !out)) return GDN_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(X) || !aligned16(B) || !aligned16(out)) return GDN_ERR_INVALID_ARG;
  return cuda_status(state_affine(count, (int)K, (int)V, A, transpose_a != 0, X, B, out,
                                  static_cast<cudaStream_t>(stream)));
}

static int kda_check(int64_t T, int64_t H, int64_t D, int32_t dt1, int32_t dt2) {
  if (T < 0 || H <= 0 || D <= 0 || H > 65535) return GDN_ERR_INVALID_ARG;
  if (H * D > ((int64_t)1 << 24) || T > ((int64_t)1 << 62) / (H * D)) return GDN_ERR_INVALID_ARG;
  auto ok_dt = [](int32_t t) {
    return t == GDN_DTYPE_FP32 || t == GDN_DTYPE_BF16 || t == GDN_DTYPE_FP16;
  };
  return ok_dt(dt1) && ok_dt(dt2) ? GDN_OK : GDN_ERR_UNSUPPORTED;
}

size_t gdn_kda_gate_workspace_bytes(int64_t T, int64_t H, int64_t D) {
  if (kda_check(T, H, D, GDN_DTYPE_FP32, GDN_DTYPE_FP32) != GDN_OK) return 0;
  return kda_gate_workspace_bytes(H, D);
}

int gdn_kda_gate_fwd(int64_t T, int64_t H, int64_t D, int32_t in_dtype, const void* g,
                     const float* A_log, const float* dt_bias, int32_t out_dtype, void* yg,
                     void* stream) {
  int rc = kda_check(T, H, D, in_dtype, out_dtype);
  if (rc) return rc;
  const bool empty = T == 0;
  if ((!g && !empty) || (!yg && !empty) || !A_log) return GDN_ERR_INVALID_ARG;
  if (!aligned16(g) || !aligned16(yg) || !aligned16(A_log) || !aligned16(dt_bias))
    return GDN_ERR_INVALID_ARG;
  return cuda_status(kda_gate_forward(T, (int)H, (int)D, in_dtype, g, A_log, dt_bias, out_dtype, yg,
                                      static_cast<cudaStream_t>(stream)));
}

int gdn_kda_gate_bwd(int64_t T, int64_t H, int64_t D, int32_t in_dtype, const void* g,
                     const float* A_log, const float* dt_bias, int32_t dy_dtype, const void* dyg,
                     void* dg, float* dA_log, float* ddt_bias, void* workspace,
                     size_t workspace_bytes, void* stream) {
  int rc = kda_check(T, H, D, in_dtype, dy_dtype);
  if (rc) return rc;
  const bool empty = T == 0;
  if ((!g && !empty) || (!dyg && !empty) || (!dg && !empty) || !A_log) return GDN_ERR_INVALID_ARG;
  const void* ptrs[] = {g, A_log, dt_bias, dyg, dg, dA_log, ddt_bias};
  for (const void* x : ptrs)
    if (!aligned16(x)) return GDN_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) ||
      workspace_bytes < kda_gate_workspace_bytes(H, D))
    return GDN_ERR_WORKSPACE;
  return cuda_status(kda_gate_backward(T, (int)H, (int)D, in_dtype, g, A_log, dt_bias, dy_dtype, dyg, dg,
                                       dA_log, ddt_bias, static_cast<float*>(workspace),
                                       static_cast<cudaStream_t>(stream)));
}

int gdn_device_status(const void* workspace, void* stream) {
  if (!workspace) return GDN_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int st = 0;
  cudaError_t e = cudaMemcpyAsync(&st, workspace, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return GDN_ERR_CUDA;
  return st;
}

const char* gdn_status_string(int status) {
  switch (status) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
    case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
    case GDN_ERR_WORKSPACE: return "GDN_ERR_WORKSPACE";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
    case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
    default: return "GDN_ERR_UNKNOWN";
  }
}

const char* gdn_version(void) { return "gdn-b200 0.1 sm_100a"; }

}  // extern "C"
