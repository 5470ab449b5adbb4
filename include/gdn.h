/*
 * gdn.h — C ABI of the B200 (sm_100a) chunkwise Gated DeltaNet library.
 *
 * The operation (per sequence and value head; gated delta rule as used by Qwen3-Next-style
 * linear-attention layers and by flash-linear-attention's chunk kernels named on the
 * "flash-linear-attention 中的 G_T_CONTIG" page: chunk_fwd_kernel_o, chunk_bwd_kernel_dv_local,
 * chunk_bwd_kernel_dqkwg, chunk_bwd_kernel_dg, wy_fast / prepare_wy_repr_bwd, chunk_delta_h):
 *
 *   gate   x_t = g_raw_t + dt_bias[hv];  g_t = -exp(A_log[hv]) * (x_t > 20 ? x_t : log(1 + e^{x_t}))
 *          (formula and stable softplus: MindSpeed-Ops issue 9, "KDA gate", section "数学公式")
 *   state  S_t = e^{g_t} S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T      (S: V x K)
 *   output o_t = scale * S_t q_t
 *
 * computed in 64-token chunks (the GDN "cv fusion" block size of 64, Ascend GDN blog,
 * section "昇腾亲和的Tiling优化") by an exact reassociation of that recurrence.
 *
 * Layouts (row-major, contiguous, every base 16-byte aligned):
 *   q, k              [B, T, H,  K]    dtype (bf16 or fp32)
 *   v, o, do, dv      [B, T, HV, V]    dtype
 *   dq, dk            [B, T, H,  K]    dtype
 *   g_raw, beta       [B, T, HV]       fp32   (raw gate input a_t and the write strength)
 *   dg, dbeta, dg_raw [B, T, HV]       fp32   (dg = dL/dg_t; dg_raw = dL/d g_raw_t)
 *   A_log, dt_bias    [HV]             fp32
 *   dA_log, ddt_bias  [HV]             fp32
 *   initial_state, final_state, dht, dh0   [Nst, HV, K, V] fp32, h[k][v] = S[v][k],
 *                     Nst = N (varlen) or B.
 * Value head hv reads the q/k of k-head hv / (HV / H) (HV must be a multiple of H).
 * Varlen: cu_seqlens (DEVICE pointer, int64, N+1 entries, cu[0] = 0, non-decreasing,
 * cu[N] = T) packs N sequences into batch row 0 (B must be 1); chunks never cross a
 * sequence boundary and each sequence has its own state ("G_T_CONTIG" page, section
 * "Varlen 场景的三条检查清单": local lengths, offsets relative to bos, int64 cu_seqlens).
 *
 * Per-token buffers may be NULL when B*T == 0 (then only states are read or written).
 *
 * Ownership: the caller owns every buffer, including the workspace (size from
 * gdn_workspace_bytes).  Entry points allocate nothing, launch asynchronously on `stream`
 * (a cudaStream_t passed as void*, NULL = legacy default stream) and return after the
 * launches are queued.  No exception crosses this boundary.
 *
 * Errors: each entry point returns a gdn_status.  Host-detectable problems (null or
 * misaligned pointers, bad sizes, unsupported K/V/dtype, small workspace) return before any
 * launch.  Problems only the device can see (cu_seqlens values that are not a valid
 * partition of [0,T), a bounded wait that ran out) set a status word inside the workspace;
 * every later kernel of the call then skips its work, and gdn_device_status() returns the
 * word (it synchronises the stream).
 */
#ifndef GDN_B200_H
#define GDN_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gdn_status {
  GDN_OK = 0,
  GDN_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, bad cu_seqlens */
  GDN_ERR_UNSUPPORTED = 2,   /* K or V not in {64,128}, unknown dtype; or a bf16 K = V = 128
                                problem (always run on the tcgen05 kernels) while the driver's
                                tensor-map encoder cannot be obtained */
  GDN_ERR_WORKSPACE = 3,     /* workspace null/misaligned or smaller than gdn_workspace_bytes */
  GDN_ERR_CUDA = 4,          /* a CUDA launch or runtime call failed */
  GDN_ERR_TIMEOUT = 5        /* a device-side bounded wait gave up (reported by gdn_device_status) */
} gdn_status;

typedef enum gdn_dtype {
  GDN_DTYPE_FP32 = 0,
  GDN_DTYPE_BF16 = 1,
  GDN_DTYPE_FP16 = 2  /* the KDA gate entry points only */
} gdn_dtype;

typedef struct gdn_dims {
  int64_t B, T, H, HV, K, V;
  int64_t N;       /* number of packed sequences when cu_seqlens != NULL; ignored otherwise */
  int32_t dtype;   /* gdn_dtype of q,k,v,o,do,dq,dk,dv; gates, beta and states are fp32 */
  float scale;     /* output scale; 0 selects 1/sqrt(K) */
  int32_t flags;   /* bitwise OR of gdn_flags (0 = none) */
} gdn_dims;

typedef enum gdn_flags {
  /* gdn_chunk_bwd only: `workspace` still holds what gdn_chunk_fwd wrote for the same
   * dimensions and the same input contents (the caller ran the forward with this workspace
   * and changed neither since), so the backward uses the forward's saved chunk
   * intermediates (chunk table, in-chunk gate sums, W, U~, T, v_new, per-chunk states) and
   * its device status word instead of recomputing them.  The
   * workspace must be sized for the backward (gdn_workspace_bytes(.., 1) >= the forward's)
   * and passed to both calls.  Honoured by the bf16 K = V = 128 path; other paths always
   * recompute, with identical results. */
  GDN_FLAG_BWD_REUSE_FWD = 1,
  /* Tests of the failure path only (no counterpart on the pages): on the bf16 K = V = 128
   * path, the forward's sequential pass over the chunks withholds its first chain product, so
   * the wait for it runs out after ~2^20 cycles (under a millisecond) instead of completing.
   * The pass then stops cleanly: the copies it issued land, the products it issued finish,
   * its tensor memory is freed, later kernels of the call skip their work, and
   * gdn_device_status reports GDN_ERR_TIMEOUT.  Outputs are not written.  Nothing faults
   * and nothing hangs; the next call without the flag runs normally. */
  GDN_FLAG_TEST_WAIT_TIMEOUT = 1 << 30
} gdn_flags;

/* Size limits (GDN_ERR_INVALID_ARG beyond them): B*T < 2^31 tokens, HV <= 65535, and
 * chunks x HV x 128 < 2^31 (the per-chunk tiles are addressed by 32-bit tensor-map rows).
 *
 * Bytes of workspace needed by gdn_chunk_fwd (pass = 0) or gdn_chunk_bwd (pass = 1) for
 * these dimensions, or 0 if the dimensions are invalid.  With cu_seqlens the bound uses
 * at most (T + 63 N) / 64 chunks.  `varlen` is 1 when cu_seqlens will be passed. */
size_t gdn_workspace_bytes(const gdn_dims* d, int varlen, int pass);

/* Forward: o and (optionally) final_state.  initial_state NULL = zero state;
 * final_state NULL = not written.  Output rows of o are all written. */
int gdn_chunk_fwd(const gdn_dims* d, const void* q, const void* k, const void* v,
                  const float* g_raw, const float* A_log, const float* dt_bias, const float* beta,
                  const int64_t* cu_seqlens, const float* initial_state,
                  void* o, float* final_state,
                  void* workspace, size_t workspace_bytes, void* stream);

/* Backward of L = sum(do * o) + sum(dht * final_state).  By default it recomputes the
 * forward's chunk intermediates from the inputs (stateless); with GDN_FLAG_BWD_REUSE_FWD
 * in d->flags it takes them from the workspace the forward filled.  dht NULL = zero.  Required outputs:
 * dq, dk, dv, dg, dbeta.  Optional (NULL = skipped): dh0, dg_raw, dA_log, ddt_bias. */
int gdn_chunk_bwd(const gdn_dims* d, const void* q, const void* k, const void* v,
                  const float* g_raw, const float* A_log, const float* dt_bias, const float* beta,
                  const int64_t* cu_seqlens, const float* initial_state,
                  const void* d_o, const float* dht,
                  void* dq, void* dk, void* dv, float* dg, float* dbeta, float* dh0,
                  float* dg_raw, float* dA_log, float* ddt_bias,
                  void* workspace, size_t workspace_bytes, void* stream);

/* Forward for callers that cannot allocate device memory (no cudaMalloc, no workspace of
 * their own: e.g. code inside someone else's stream capture, or a plugin whose host owns
 * all device memory).  The paper has no counterpart; this is a packaging variant of
 * gdn_chunk_fwd.  Same arguments and results as gdn_chunk_fwd without the workspace: the
 * scratch is a file-scope device array of GDN_NOALLOC_SCRATCH_BYTES (32 MiB) that every
 * GPU which loads the library holds until the process exits.  Calls whose
 * gdn_workspace_bytes(d, varlen, 0) exceeds that size return GDN_ERR_WORKSPACE before any
 * launch.  The entry point allocates nothing (no cudaMalloc/cudaFree, no library
 * allocator).  Every call looks up the array's device address in the current device's
 * context (cudaGetSymbolAddress, a host-side query); the first call on a device also loads
 * the module there, so make that first call before any stream capture.  All calls share the
 * one array and it keeps the last call's contents, so calls that overlap on the GPU
 * (different streams, or host threads) race, on the scratch and on the status word it holds:
 * serialise them.  Problems only the device sees (invalid cu_seqlens, a bounded wait that ran
 * out) are read back with gdn_noalloc_device_status. */
#define GDN_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
int gdn_chunk_fwd_noalloc(const gdn_dims* d, const void* q, const void* k, const void* v,
                          const float* g_raw, const float* A_log, const float* dt_bias,
                          const float* beta, const int64_t* cu_seqlens,
                          const float* initial_state, void* o, float* final_state, void* stream);

/* Size in bytes of the array gdn_chunk_fwd_noalloc uses (GDN_NOALLOC_SCRATCH_BYTES). */
size_t gdn_noalloc_scratch_bytes(void);

/* gdn_device_status for gdn_chunk_fwd_noalloc: synchronises `stream` and returns the status
 * word the last allocation-free call on the current device left in the shared array
 * (GDN_OK, GDN_ERR_INVALID_ARG for invalid cu_seqlens, GDN_ERR_TIMEOUT), or GDN_ERR_CUDA if
 * the array's address cannot be looked up.  No counterpart on the pages (packaging). */
int gdn_noalloc_device_status(void* stream);

/* Token-by-token (recurrent) forward for decoding and short prefills: the same operation and
 * the same arguments as gdn_chunk_fwd (o for every token, final_state after each sequence's
 * last token), computed one token after another as the recurrence at the top of this file is
 * written, with each (sequence, value head) state read once and written once.  This is the
 * form the chunkwise algorithm reassociates (Ascend GDN blog and the G_T_CONTIG page treat
 * the chunk kernels; the decode step is the same recurrence with T = 1 per sequence).  Cost
 * is linear in T per sequence with no parallelism across a sequence's tokens: use it for
 * T = 1 decode steps and prefills of a few tokens, gdn_chunk_fwd for long sequences.
 * final_state may be the same buffer as initial_state (the state is updated in place).
 * workspace: at least GDN_RECURRENT_WORKSPACE_BYTES, 256-byte aligned; it holds the device
 * status word (gdn_device_status reports invalid cu_seqlens as GDN_ERR_INVALID_ARG).
 * Besides the size limits above, (number of sequences) * V / 32 < 2^31 (GDN_ERR_INVALID_ARG). */
#define GDN_RECURRENT_WORKSPACE_BYTES ((size_t)256)
int gdn_recurrent_fwd(const gdn_dims* d, const void* q, const void* k, const void* v,
                      const float* g_raw, const float* A_log, const float* dt_bias,
                      const float* beta, const int64_t* cu_seqlens, const float* initial_state,
                      void* o, float* final_state, void* workspace, size_t workspace_bytes,
                      void* stream);

/* GDN_RECURRENT_WORKSPACE_BYTES. */
size_t gdn_recurrent_workspace_bytes(void);

/* KDA gate: the per-channel gate of Kimi-style delta attention ("KDA gate" task of the
 * MindSpeed-Ops issue tracker, sections on the formula, the computation flow and the API):
 *   yg[t,h,d] = -exp(A_log[h]) * softplus(g[t,h,d] + dt_bias[h*D + d]),
 *   softplus(x) = x if x > 20 else log(1 + e^x), computed in fp32.
 * g, yg: [T, H, D] row-major (any leading dims flattened into T) in in_dtype / out_dtype
 * (gdn_dtype: fp32, bf16 or fp16); A_log [H] fp32; dt_bias [H*D] fp32 or NULL (no bias).
 * All buffers on the device, 16-byte aligned; launches on `stream`; allocates nothing.
 * Returns GDN_ERR_INVALID_ARG for null or misaligned pointers or bad sizes (H <= 65535,
 * H*D <= 2^24), GDN_ERR_UNSUPPORTED for an unknown dtype.  The KDA recurrence and its chunkwise
 * forward and backward are the gdn_kda_* entry points below. */
int gdn_kda_gate_fwd(int64_t T, int64_t H, int64_t D, int32_t in_dtype, const void* g,
                     const float* A_log, const float* dt_bias, int32_t out_dtype, void* yg,
                     void* stream);

/* Backward of the KDA gate for dyg = dL/dyg ([T,H,D] in dy_dtype):
 *   dg = dyg * (-exp(A_log[h])) * (x > 20 ? 1 : sigmoid(x))    ([T,H,D] in in_dtype),
 *   dA_log[h] = sum_{t,d} dyg * yg,   ddt_bias[h*D+d] = sum_t dg   (fp32; either may be NULL).
 * The two sums are deterministic (fixed-order two-pass reduction).  workspace: at least
 * gdn_kda_gate_workspace_bytes(T, H, D) bytes, 256-byte aligned. */
int gdn_kda_gate_bwd(int64_t T, int64_t H, int64_t D, int32_t in_dtype, const void* g,
                     const float* A_log, const float* dt_bias, int32_t dy_dtype, const void* dyg,
                     void* dg, float* dA_log, float* ddt_bias, void* workspace,
                     size_t workspace_bytes, void* stream);

/* KDA (per-channel gated) delta rule, token by token, for decoding and short prefills:
 *   S_t = S_{t-1} Diag(exp(yg_t)) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = scale S_t q_t,
 *   yg_t[c] = -exp(A_log[hv]) * softplus(g_raw[t,hv,c] + dt_bias[hv*K + c])   (the KDA gate),
 * i.e. gdn_recurrent_fwd with the scalar decay of each value head replaced by a decay per key
 * channel (the pages give the KDA gate and name the KDA chunk kernels; the recurrence is the
 * Gated DeltaNet one with that gate).  Arguments as gdn_recurrent_fwd except
 *   g_raw    [B,T,HV,K] fp32 (raw per-channel gate input),
 *   dt_bias  [HV*K] fp32, or NULL for none.
 * Same workspace, status word, in-place state and error behaviour as gdn_recurrent_fwd. */
int gdn_kda_recurrent_fwd(const gdn_dims* d, const void* q, const void* k, const void* v,
                          const float* g_raw, const float* A_log, const float* dt_bias,
                          const float* beta, const int64_t* cu_seqlens, const float* initial_state,
                          void* o, float* final_state, void* workspace, size_t workspace_bytes,
                          void* stream);

/* Chunkwise forward of the same KDA recurrence as gdn_kda_recurrent_fwd, for long sequences:
 * 64-token chunks, the per-channel decay carried through 16-token sub-chunks (every factor an
 * exponential of a non-positive number), a sequential state pass over the chunks.  bf16 with
 * K = V = 128: every product on the tensor cores (operands as compensated bf16 pairs, fp32
 * accumulation); other dtypes and head sizes: fp32 arithmetic on CUDA cores; the same results
 * within the tolerances either way.  Arguments, layouts and results as gdn_kda_recurrent_fwd
 * (g_raw [B,T,HV,K] fp32, dt_bias [HV*K] or NULL; o for every token, final_state after each
 * sequence's last token; final_state may be NULL).  workspace: at least
 * gdn_kda_chunk_workspace_bytes(d, varlen, 0) bytes, 256-byte aligned; it also holds the device
 * status word (gdn_device_status: GDN_ERR_INVALID_ARG for invalid cu_seqlens).  Given at least
 * gdn_kda_chunk_workspace_bytes(d, varlen, 1) bytes, the forward also keeps in it what
 * gdn_kda_chunk_bwd reads.  Same size limits and error returns as gdn_chunk_fwd. */
int gdn_kda_chunk_fwd(const gdn_dims* d, const void* q, const void* k, const void* v,
                      const float* g_raw, const float* A_log, const float* dt_bias, const float* beta,
                      const int64_t* cu_seqlens, const float* initial_state, void* o,
                      float* final_state, void* workspace, size_t workspace_bytes, void* stream);

/* Backward of gdn_kda_chunk_fwd for L = sum(d_o * o) + sum(dht * final_state): reads the
 * intermediates a gdn_kda_chunk_fwd call with the same inputs left in `workspace` (which must
 * then be at least gdn_kda_chunk_workspace_bytes(d, varlen, 1) bytes; the forward's status
 * word is honoured), and writes
 *   dq, dk [B,T,H,K] and dv [B,T,HV,V] (input dtype), dbeta [B,T,HV] fp32,
 *   dg [B,T,HV,K] fp32 = dL/dyg (the per-channel log-decay),
 *   dg_raw [B,T,HV,K] fp32 (may be NULL), dh0 [Nst,HV,K,V] fp32 (may be NULL),
 *   dA_log [HV] fp32 (may be NULL), ddt_bias [HV*K] fp32 (may be NULL; needs dt_bias).
 * dht may be NULL (zero).  The parameter sums are deterministic (fixed chunk order).  Kernels as
 * for gdn_kda_chunk_fwd (tensor cores for bf16 with K = V = 128). */
int gdn_kda_chunk_bwd(const gdn_dims* d, const void* q, const void* k, const void* v,
                      const float* g_raw, const float* A_log, const float* dt_bias, const float* beta,
                      const int64_t* cu_seqlens, const void* d_o, const float* dht, void* dq, void* dk,
                      void* dv, float* dg, float* dbeta, float* dh0, float* dg_raw, float* dA_log,
                      float* ddt_bias, void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes of gdn_kda_chunk_fwd (pass 0) or of a forward + backward pair (pass 1); 0 for
 * invalid dimensions. */
size_t gdn_kda_chunk_workspace_bytes(const gdn_dims* d, int varlen, int pass);

/* Workspace bytes of gdn_kda_gate_bwd (0 for invalid sizes). */
size_t gdn_kda_gate_workspace_bytes(int64_t T, int64_t H, int64_t D);

/* Affine maps of states, for context parallelism over T (a sequence split into segments, one
 * per rank).  A segment maps the state entering it to the state leaving it affinely; in the
 * [K][V] layout of the state arguments above, h_end = Mt h_start + Bh, where Mt (K x K) is the
 * final_state gdn_chunk_fwd returns for the segment from initial_state = I with v = 0 (K = V),
 * and Bh the one it returns from initial_state = 0 (the state after a segment is linear in the
 * state before it, as every step of the recurrence is).  The gradient entering the segment is
 * Mt^T dh_end + D, D the dh0 of gdn_chunk_bwd for the segment with dht = 0.
 *   out[n] = op(A[n]) X[n] + B[n],  n < count,  op(A) = A or A^T (transpose_a != 0),
 * A [count][K][K], X, B, out [count][K][V] fp32 device pointers (B may be NULL; out may be X).
 * 1 <= K <= 128, V a multiple of 32; GDN_ERR_INVALID_ARG otherwise. */
int gdn_state_affine(int64_t count, int64_t K, int64_t V, const float* A, int transpose_a, const float* X,
                     const float* B, float* out, void* stream);

/* Upper bound on the number of 64-token chunks (the grid size used for chunk kernels). */
int64_t gdn_max_chunks(const gdn_dims* d, int varlen);

/* Host-side chunk table: for each chunk in order (sequence-major), 4 int32 values
 * {sequence n, chunk index c within the sequence, tokens L in the chunk (1..64),
 *  flat token index of its first token in [B*T]}.  cu_host is a HOST copy of cu_seqlens
 * (NULL = dense batch).  Writes min(count, cap) entries; returns the chunk count, or a
 * negative gdn_status on invalid input. */
int64_t gdn_build_chunk_indices(const gdn_dims* d, const int64_t* cu_host, int32_t* out_host,
                                int64_t cap);

/* The same table built by the device kernel the forward/backward use (cu_seqlens is a
 * device pointer, table a device buffer of cap*4 int32 written in the same format; entries
 * past the count are {-1,-1,0,0}); count_dev (device int32) receives the chunk count, or -1
 * when cu_seqlens is not a valid partition of [0, T). */
int gdn_chunk_table_device(const gdn_dims* d, const int64_t* cu_seqlens, int32_t* table,
                           int64_t cap, int32_t* count_dev, void* stream);

/* Synchronise `stream` and return the device status word of the last call that used
 * `workspace` (GDN_OK, GDN_ERR_INVALID_ARG for bad cu_seqlens, GDN_ERR_TIMEOUT). */
int gdn_device_status(const void* workspace, void* stream);

/* Number of kernel launches this library has issued since it was loaded (all threads). */
int64_t gdn_launch_count(void);

/* Per-kernel device timing: while enabled, every launch is bracketed by CUDA events
 * recorded on its own stream (adds a little host overhead; for measurement passes only). */
int gdn_profile(int enable);

/* Synchronises the recorded events, writes {"kernel": [launches, total_ms], ...} as a
 * NUL-terminated JSON object into buf (truncated to cap-1 bytes), clears the records and
 * returns the full text length (negative gdn_status on a CUDA error). */
int64_t gdn_profile_read(char* buf, size_t cap);

/* Human-readable name of a status code (static string). */
const char* gdn_status_string(int status);

/* Version and build tag (static string), e.g. "gdn-b200 0.1 sm_100a". */
const char* gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_B200_H */
