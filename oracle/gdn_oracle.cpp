// Gated DeltaNet oracle: plain, slow, fp64, token-by-token CPU reference.
//
// TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
// this file: only the tests, the smoke check and the bench's CPU-baseline leg do.
// It shares no code, header, table or helper with the CUDA library.
//
// What it computes (one independent problem per (sequence, value head)):
//
//   gate   (MindSpeed-Ops issue 9, "KDA gate" write-up, section "核心计算逻辑 / 数学公式"):
//            x   = a_t + dt_bias[hv]
//            sp  = x            if x > 20      (the page's stable softplus)
//                = log(1 + e^x) otherwise
//            g_t = -exp(A_log[hv]) * sp
//   recurrence (gated delta rule; the pages name it and its kernels but never write
//   it, so its plain form is taken:  S_t = e^{g_t} S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T,
//   o_t = scale * S_t q_t), evaluated literally, one token at a time:
//            S <- e^{g_t} S
//            e  = S k_t
//            S <- S + b_t (v_t - e) k_t^T
//            o_t = scale * S q_t
//   with S in R^{V x K} and the state stored as h[k][v] = S[v][k]  (layout [N,HV,K,V]).
//   Value head hv reads the q/k of k-head hv / (HV/H)  (grouped value heads:
//   "flash-linear-attention ... G_T_CONTIG" page, workload B=2,T=2048,H=4,HV=8).
//   Varlen packing: cu_seqlens (int64, N+1 entries) marks sequence n as tokens
//   [cu[n], cu[n+1]) of batch row 0; each sequence starts from its own initial state
//   ("G_T_CONTIG" page, section "Varlen 场景的三条检查清单").
//
// Backward: a hand-derived reverse-time recurrence on the same token-level definition
// (loss L = sum dO.o + sum dht.h_final), with S re-computed from checkpoints kept every
// 64 tokens.  For t = T..1, with a_t = e^{g_t}, P_t = I - b_t k_t k_t^T and D = dL/dS_t:
//            D    += scale do_t q_t^T
//            dq_t += scale S_t^T do_t
//            dv_t  = b_t D k_t
//            db_t  = (v_t - a_t S_{t-1} k_t)^T D k_t
//            dg_t  = a_t <D, S_{t-1} P_t>
//            dk_t += b_t (D^T v_t - a_t (S_{t-1}^T D k_t + D^T S_{t-1} k_t))
//            D     = a_t D P_t
//   dh0 = D at the start.  Gate chain: da_t = dg_t * (-exp(A_log)) * (x > 20 ? 1 : sigmoid(x)),
//   dA_log = sum_t dg_t g_t, ddt_bias = sum_t da_t.  dq/dk sum over the value heads of a
//   k-head.
//
// Build: g++ -O2 -std=c++17 -shared -fPIC -pthread gdn_oracle.cpp -o liboracle.so
// (oracle/oracle.py does this on first use).

#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>
#include <atomic>
#include <algorithm>

namespace {

struct Dims {
  int64_t B, T, H, HV, K, V;
  int64_t N;          // number of packed sequences when cu != nullptr
  double scale;
};

enum : int {
  FLAG_NO_ERASE = 1,  // test-only: drop the -b k k^T erase term (plain gated linear attention)
};

// One (sequence, value-head) problem: where its tokens live.
struct Unit {
  int64_t b;      // batch row
  int64_t bos;    // first token (within the row)
  int64_t len;    // number of tokens
  int64_t n;      // state index (sequence index in varlen mode, else b)
  int64_t hv;
};

inline double softplus_page(double x) { return x > 20.0 ? x : std::log1p(std::exp(x)); }
inline double dsoftplus_page(double x) { return x > 20.0 ? 1.0 : 1.0 / (1.0 + std::exp(-x)); }

std::vector<Unit> make_units(const Dims& d, const int64_t* cu) {
  std::vector<Unit> u;
  if (cu) {
    for (int64_t n = 0; n < d.N; ++n)
      for (int64_t hv = 0; hv < d.HV; ++hv) u.push_back({0, cu[n], cu[n + 1] - cu[n], n, hv});
  } else {
    for (int64_t b = 0; b < d.B; ++b)
      for (int64_t hv = 0; hv < d.HV; ++hv) u.push_back({b, 0, d.T, b, hv});
  }
  return u;
}

template <class F>
void parallel_for(int64_t n, int nthreads, F f) {
  if (nthreads <= 0) nthreads = (int)std::max(1u, std::thread::hardware_concurrency());
  nthreads = (int)std::min<int64_t>(nthreads, std::max<int64_t>(n, 1));
  std::atomic<int64_t> next{0};
  std::vector<std::thread> th;
  for (int i = 0; i < nthreads; ++i)
    th.emplace_back([&] {
      for (int64_t j; (j = next.fetch_add(1)) < n;) f(j);
    });
  for (auto& t : th) t.join();
}

// Index helpers for the documented layouts.
struct Ix {
  const Dims& d;
  int64_t qk(int64_t b, int64_t t, int64_t h) const { return ((b * d.T + t) * d.H + h) * d.K; }
  int64_t vv(int64_t b, int64_t t, int64_t hv) const { return ((b * d.T + t) * d.HV + hv) * d.V; }
  int64_t sc(int64_t b, int64_t t, int64_t hv) const { return (b * d.T + t) * d.HV + hv; }
  int64_t st(int64_t n, int64_t hv) const { return (n * d.HV + hv) * d.K * d.V; }
};

// Gate for one token of one value head.
inline double gate_g(double a, double A_log, double dt_bias) {
  return -std::exp(A_log) * softplus_page(a + dt_bias);
}

// S is V x K, row-major (S[v*K + k]).  One token step; returns nothing, updates S in place.
inline void token_step(const Dims& d, double* S, const double* k, const double* v, double beta,
                       double g, int flags, double* e /*scratch V*/) {
  const int64_t K = d.K, V = d.V;
  const double a = std::exp(g);
  for (int64_t i = 0; i < V * K; ++i) S[i] *= a;
  for (int64_t r = 0; r < V; ++r) {
    double s = 0;
    for (int64_t c = 0; c < K; ++c) s += S[r * K + c] * k[c];
    e[r] = (flags & FLAG_NO_ERASE) ? 0.0 : s;
  }
  for (int64_t r = 0; r < V; ++r) {
    const double w = beta * (v[r] - e[r]);
    for (int64_t c = 0; c < K; ++c) S[r * K + c] += w * k[c];
  }
}

}  // namespace

extern "C" {

// Gate alone, elementwise over [n] values of one head: g = -exp(A_log) * softplus(a + dt_bias).
void oracle_gate(const double* a, int64_t n, double A_log, double dt_bias, double* g) {
  for (int64_t i = 0; i < n; ++i) g[i] = gate_g(a[i], A_log, dt_bias);
}

// Forward.  All arrays fp64 in the documented layouts:
//   q,k [B,T,H,K]; v,o [B,T,HV,V]; a (raw gate input), beta [B,T,HV]; A_log, dt_bias [HV];
//   h0, ht [Nst,HV,K,V] with Nst = N (varlen) or B; h0 may be null (zero state), ht may be null.
//   g_out [B,T,HV] may be null (receives the gate values).
// Returns 0 on success, -1 on bad arguments.
int oracle_gdn_fwd(int64_t B, int64_t T, int64_t H, int64_t HV, int64_t K, int64_t V, int64_t N,
                   double scale, const double* q, const double* k, const double* v, const double* a,
                   const double* A_log, const double* dt_bias, const double* beta,
                   const int64_t* cu, const double* h0, double* o, double* ht, double* g_out,
                   int flags, int nthreads) {
  if (B <= 0 || T < 0 || H <= 0 || HV <= 0 || K <= 0 || V <= 0 || HV % H) return -1;
  if (cu && B != 1) return -1;
  Dims d{B, T, H, HV, K, V, N, scale};
  Ix ix{d};
  auto units = make_units(d, cu);
  const int64_t G = HV / H;
  parallel_for((int64_t)units.size(), nthreads, [&](int64_t ui) {
    const Unit u = units[ui];
    std::vector<double> S(V * K, 0.0), e(V);
    if (h0)
      for (int64_t kk = 0; kk < K; ++kk)
        for (int64_t vv = 0; vv < V; ++vv) S[vv * K + kk] = h0[ix.st(u.n, u.hv) + kk * V + vv];
    const int64_t hk = u.hv / G;
    for (int64_t t = u.bos; t < u.bos + u.len; ++t) {
      const double g = gate_g(a[ix.sc(u.b, t, u.hv)], A_log[u.hv], dt_bias[u.hv]);
      if (g_out) g_out[ix.sc(u.b, t, u.hv)] = g;
      const double* kt = k + ix.qk(u.b, t, hk);
      const double* qt = q + ix.qk(u.b, t, hk);
      const double* vt = v + ix.vv(u.b, t, u.hv);
      token_step(d, S.data(), kt, vt, beta[ix.sc(u.b, t, u.hv)], g, flags, e.data());
      double* ot = o + ix.vv(u.b, t, u.hv);
      for (int64_t r = 0; r < V; ++r) {
        double s = 0;
        for (int64_t c = 0; c < K; ++c) s += S[r * K + c] * qt[c];
        ot[r] = scale * s;
      }
    }
    if (ht)
      for (int64_t kk = 0; kk < K; ++kk)
        for (int64_t vv = 0; vv < V; ++vv) ht[ix.st(u.n, u.hv) + kk * V + vv] = S[vv * K + kk];
  });
  return 0;
}

// Backward of the forward above for L = sum(dO*o) + sum(dht*h_final).
//   dO [B,T,HV,V]; dht [Nst,HV,K,V] or null (zero).
//   Outputs (all required unless noted): dq,dk [B,T,H,K]; dv [B,T,HV,V]; dg, dbeta, da [B,T,HV]
//   (dg = dL/dg_t, da = dL/da_t); dh0 [Nst,HV,K,V] (null to skip); dA_log, ddt_bias [HV].
int oracle_gdn_bwd(int64_t B, int64_t T, int64_t H, int64_t HV, int64_t K, int64_t V, int64_t N,
                   double scale, const double* q, const double* k, const double* v, const double* a,
                   const double* A_log, const double* dt_bias, const double* beta,
                   const int64_t* cu, const double* h0, const double* dO, const double* dht,
                   double* dq, double* dk, double* dv, double* dg, double* dbeta, double* da,
                   double* dh0, double* dA_log, double* ddt_bias, int flags, int nthreads) {
  if (B <= 0 || T < 0 || H <= 0 || HV <= 0 || K <= 0 || V <= 0 || HV % H) return -1;
  if (cu && B != 1) return -1;
  Dims d{B, T, H, HV, K, V, N, scale};
  Ix ix{d};
  auto units = make_units(d, cu);
  const int64_t G = HV / H;
  const int64_t CK = 64;  // checkpoint spacing
  // per-value-head partials of dq/dk, summed over each k-head's group afterwards
  std::vector<double> dq_hv(B * T * HV * K, 0.0), dk_hv(B * T * HV * K, 0.0);
  std::vector<double> dA_part(units.size(), 0.0), ddt_part(units.size(), 0.0);
  auto qkv_ix = [&](int64_t b, int64_t t, int64_t hv) { return ((b * T + t) * HV + hv) * K; };

  parallel_for((int64_t)units.size(), nthreads, [&](int64_t ui) {
    const Unit u = units[ui];
    const int64_t hk = u.hv / G, L = u.len;
    const double Alog = A_log[u.hv], dtb = dt_bias[u.hv];
    std::vector<double> S(V * K, 0.0), e(V), gl(std::max<int64_t>(L, 1));
    if (h0)
      for (int64_t kk = 0; kk < K; ++kk)
        for (int64_t vv = 0; vv < V; ++vv) S[vv * K + kk] = h0[ix.st(u.n, u.hv) + kk * V + vv];
    // forward sweep: gates and checkpoints; ck[c] = S before token c*CK (local index)
    const int64_t NCk = (L + CK - 1) / CK;
    std::vector<double> ck((size_t)std::max<int64_t>(NCk, 1) * V * K);
    for (int64_t t = 0; t < L; ++t) {
      const int64_t tt = u.bos + t;
      gl[t] = gate_g(a[ix.sc(u.b, tt, u.hv)], Alog, dtb);
      if (t % CK == 0) std::copy(S.begin(), S.end(), ck.begin() + (t / CK) * V * K);
      token_step(d, S.data(), k + ix.qk(u.b, tt, hk), v + ix.vv(u.b, tt, u.hv),
                 beta[ix.sc(u.b, tt, u.hv)], gl[t], flags, e.data());
    }
    // D = dL/dS_T  (S orientation V x K)
    std::vector<double> D(V * K, 0.0);
    if (dht)
      for (int64_t kk = 0; kk < K; ++kk)
        for (int64_t vv = 0; vv < V; ++vv) D[vv * K + kk] = dht[ix.st(u.n, u.hv) + kk * V + vv];
    // segment buffer: states S_{t-1} for the tokens of one checkpoint segment
    std::vector<double> seg((size_t)(CK + 1) * V * K);
    std::vector<double> Sk(V), Dk(V), DTv(K), STDk(K), DTSk(K), tmp(K);
    double dA_acc = 0.0, ddt_acc = 0.0;
    for (int64_t c = NCk - 1; c >= 0; --c) {
      const int64_t t0 = c * CK, t1 = std::min(L, t0 + CK);
      // recompute states: seg[j] = S before token t0+j, seg[t1-t0] = S after token t1-1
      std::copy(ck.begin() + c * V * K, ck.begin() + (c + 1) * V * K, seg.begin());
      for (int64_t t = t0; t < t1; ++t) {
        const int64_t j = t - t0, tt = u.bos + t;
        std::copy(seg.begin() + j * V * K, seg.begin() + (j + 1) * V * K, seg.begin() + (j + 1) * V * K);
        token_step(d, seg.data() + (j + 1) * V * K, k + ix.qk(u.b, tt, hk), v + ix.vv(u.b, tt, u.hv),
                   beta[ix.sc(u.b, tt, u.hv)], gl[t], flags, e.data());
      }
      for (int64_t t = t1 - 1; t >= t0; --t) {
        const int64_t j = t - t0, tt = u.bos + t;
        const double* Sprev = seg.data() + j * V * K;      // S_{t-1}
        const double* Scur = seg.data() + (j + 1) * V * K; // S_t
        const double* kt = k + ix.qk(u.b, tt, hk);
        const double* qt = q + ix.qk(u.b, tt, hk);
        const double* vt = v + ix.vv(u.b, tt, u.hv);
        const double* dot = dO + ix.vv(u.b, tt, u.hv);
        const double bt = beta[ix.sc(u.b, tt, u.hv)];
        const double at = std::exp(gl[t]);
        const double erase = (flags & FLAG_NO_ERASE) ? 0.0 : 1.0;
        // D += scale do q^T
        for (int64_t r = 0; r < V; ++r)
          for (int64_t cc = 0; cc < K; ++cc) D[r * K + cc] += scale * dot[r] * qt[cc];
        // dq_t (this value head's share) = scale S_t^T do
        double* dqt = dq_hv.data() + qkv_ix(u.b, tt, u.hv);
        for (int64_t cc = 0; cc < K; ++cc) {
          double s = 0;
          for (int64_t r = 0; r < V; ++r) s += Scur[r * K + cc] * dot[r];
          dqt[cc] += scale * s;
        }
        // Sk = S_{t-1} k, Dk = D k
        for (int64_t r = 0; r < V; ++r) {
          double s1 = 0, s2 = 0;
          for (int64_t cc = 0; cc < K; ++cc) {
            s1 += Sprev[r * K + cc] * kt[cc];
            s2 += D[r * K + cc] * kt[cc];
          }
          Sk[r] = s1;
          Dk[r] = s2;
        }
        // dv, dbeta
        double db = 0;
        double* dvt = dv + ix.vv(u.b, tt, u.hv);
        for (int64_t r = 0; r < V; ++r) {
          dvt[r] = bt * Dk[r];
          db += (vt[r] - erase * at * Sk[r]) * Dk[r];
        }
        dbeta[ix.sc(u.b, tt, u.hv)] = db;
        // dg = a <D, S_{t-1} P> = a (<D, S_{t-1}> - b (Dk . Sk))   [P = I - b k k^T]
        double dS = 0, dkS = 0;
        for (int64_t i = 0; i < V * K; ++i) dS += D[i] * Sprev[i];
        for (int64_t r = 0; r < V; ++r) dkS += Dk[r] * Sk[r];
        const double dgt = at * (dS - erase * bt * dkS);
        dg[ix.sc(u.b, tt, u.hv)] = dgt;
        // dk = b (D^T v - a (S_{t-1}^T D k + D^T S_{t-1} k))
        for (int64_t cc = 0; cc < K; ++cc) {
          double s1 = 0, s2 = 0, s3 = 0;
          for (int64_t r = 0; r < V; ++r) {
            s1 += D[r * K + cc] * vt[r];
            s2 += Sprev[r * K + cc] * Dk[r];
            s3 += D[r * K + cc] * Sk[r];
          }
          dk_hv[qkv_ix(u.b, tt, u.hv) + cc] += bt * (s1 - erase * at * (s2 + s3));
        }
        // gate chain
        const double x = a[ix.sc(u.b, tt, u.hv)] + dtb;
        const double dat = dgt * (-std::exp(Alog)) * dsoftplus_page(x);
        da[ix.sc(u.b, tt, u.hv)] = dat;
        dA_acc += dgt * gl[t];
        ddt_acc += dat;
        // D = a D P = a (D - b (D k) k^T)
        for (int64_t r = 0; r < V; ++r)
          for (int64_t cc = 0; cc < K; ++cc)
            D[r * K + cc] = at * (D[r * K + cc] - erase * bt * Dk[r] * kt[cc]);
      }
    }
    if (dh0)
      for (int64_t kk = 0; kk < K; ++kk)
        for (int64_t vv = 0; vv < V; ++vv) dh0[ix.st(u.n, u.hv) + kk * V + vv] = D[vv * K + kk];
    dA_part[ui] = dA_acc;
    ddt_part[ui] = ddt_acc;
  });

  // group sums for dq, dk; zero outside covered tokens
  for (int64_t b = 0; b < B; ++b)
    for (int64_t t = 0; t < T; ++t)
      for (int64_t h = 0; h < H; ++h)
        for (int64_t cc = 0; cc < K; ++cc) {
          double sq = 0, sk = 0;
          for (int64_t j = 0; j < G; ++j) {
            sq += dq_hv[qkv_ix(b, t, h * G + j) + cc];
            sk += dk_hv[qkv_ix(b, t, h * G + j) + cc];
          }
          dq[ix.qk(b, t, h) + cc] = sq;
          dk[ix.qk(b, t, h) + cc] = sk;
        }
  for (int64_t hv = 0; hv < HV; ++hv) {
    dA_log[hv] = 0;
    ddt_bias[hv] = 0;
  }
  for (size_t ui = 0; ui < units.size(); ++ui) {
    dA_log[units[ui].hv] += dA_part[ui];
    ddt_bias[units[ui].hv] += ddt_part[ui];
  }
  return 0;
}

}  // extern "C"
