// nsa_noalloc.cu -- nsa_decode_noalloc: decode for callers that cannot
// allocate device memory.
//
// nsa_decode needs a scratch workspace for its intermediate branch outputs,
// block scores and indices, which the caller normally allocates and passes
// in.  Some callers have no way to do that: a plugin that a host framework
// hands only its input and output buffers, or a runtime whose memory is a
// fixed pool with no allocation hook.  This variant takes its scratch from
// a fixed array in the library's own device memory instead, so the caller
// passes inputs and outputs only, and nothing is allocated at call time.
//
// The array (kNoAllocScratchBytes) is a file-scope __device__ object: every
// GPU that loads the library holds it until the process exits.  All calls
// on a device share it and it keeps the previous call's contents; decode
// writes every scratch element it reads in the same call (stale values from
// an earlier call are never read), so nothing needs clearing.  Calls whose
// executions overlap on the GPU (different streams, or different host
// threads without ordering) race on the array.
#include "common.cuh"
#include "internal.h"
#include "nsa.h"

namespace nsa {
nsa_status decode_scratch_bytes(const nsa_params* p, bool idx_given, size_t* bytes);
}

// Fixed scratch for nsa_decode_noalloc: 16 MiB per device.
static constexpr size_t kNoAllocScratchBytes = (size_t)16 << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

// Device address of the scratch array in the current context.  In host code
// the array's name only stands for it: the address is looked up on every
// call, with the caller's device current, so a call never uses an address
// taken in another context (another device, a context the caller made
// current itself, or one created again after a device reset).  Only the
// first lookup in a context does real work (it may load the library's
// device code): make the first call on a device before any stream capture.
nsa_status scratch_ptr(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return NSA_ERR_CUDA;
  *out = p;
  return NSA_OK;
}

}  // namespace

extern "C" {

size_t nsa_decode_noalloc_max_scratch(void) { return kNoAllocScratchBytes; }

nsa_status nsa_decode_noalloc(const nsa_params* p, const void* q, const void* k_cache,
                              const void* v_cache, const void* kc_cache, const void* vc_cache,
                              const float* gates, void* out, int32_t* idx_out, void* stream) {
  size_t need = 0;
  nsa_status st = nsa::decode_scratch_bytes(p, idx_out != nullptr, &need);
  if (st != NSA_OK) return st;
  if (need > kNoAllocScratchBytes) return NSA_ERR_SCRATCH_TOO_SMALL;
  void* scratch = nullptr;
  st = scratch_ptr(&scratch);
  if (st != NSA_OK) return st;
  return nsa_decode(p, q, k_cache, v_cache, kc_cache, vc_cache, gates, out, idx_out, scratch,
                    kNoAllocScratchBytes, stream);
}

}  // extern "C"
