// Forward entry point for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc or hand the library a workspace: code running inside
// a CUDA graph being captured by someone else, plugins whose host framework owns every
// device allocation, or tight inference loops that forbid allocator traffic.  For them,
// gdn_chunk_fwd_noalloc runs the same forward as gdn_chunk_fwd with its scratch taken
// from one file-scope device array of fixed size, reserved when the library is loaded on a
// device and held until the process exits.
#include "gdn.h"

namespace {

constexpr size_t kScratchBytes = GDN_NOALLOC_SCRATCH_BYTES;

// The scratch the forward runs in.  Every call on a device shares it.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// Device address of g_scratch in the current device's context.  The array's name is only a
// host-side stand-in in host code; its device address comes from cudaGetSymbolAddress with
// the device current.  It is looked up on every call (a host-side query, no stream work), so
// a context that was reset and recreated, where the module and its array may sit elsewhere,
// is never handed a stale address.
int scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return GDN_ERR_CUDA;
  *out = p;
  return GDN_OK;
}

}  // namespace

extern "C" {

size_t gdn_noalloc_scratch_bytes(void) { return kScratchBytes; }

int gdn_chunk_fwd_noalloc(const gdn_dims* d, const void* q, const void* k, const void* v,
                          const float* g_raw, const float* A_log, const float* dt_bias,
                          const float* beta, const int64_t* cu_seqlens, const float* initial_state,
                          void* o, float* final_state, void* stream) {
  const size_t need = gdn_workspace_bytes(d, cu_seqlens != nullptr, 0);
  if (need == 0) return GDN_ERR_INVALID_ARG;
  if (need > kScratchBytes) return GDN_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != GDN_OK) return rc;
  // Nothing in the scratch has to start at zero: the forward's first kernel rewrites the
  // status word and the chunk tables, and every later region is written before it is read.
  return gdn_chunk_fwd(d, q, k, v, g_raw, A_log, dt_bias, beta, cu_seqlens, initial_state, o,
                       final_state, scratch, kScratchBytes, stream);
}

int gdn_noalloc_device_status(void* stream) {
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != GDN_OK) return rc;
  return gdn_device_status(scratch, stream);
}

}  // extern "C"
