// Forward with its scratch in a static device array, for callers that
// cannot allocate device memory (see lizard_attn_fwd_noalloc in lizard.h).
#include "../../include/lizard.h"

namespace {

// The scratch every call of lizard_attn_fwd_noalloc uses.  A host-side use
// of this name is only a stand-in for the symbol, never a device address:
// the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LIZARD_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch on the current device, looked up on every
// call with that device current (so a context that was torn down and made
// again never sees a stale address).  Null on failure.
void *scratch_address() {
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
  return p;
}

}  // namespace

extern "C" lizard_status lizard_attn_fwd_noalloc(const lizard_fwd_args *args, lizard_stream_t stream) {
  if (!args) return LIZARD_ERR_INVALID_ARG;
  const size_t need = lizard_fwd_workspace_size(args);
  if (need == 0) {
    // invalid arguments: let the regular checks name the error (nothing runs)
    lizard_fwd_args a = *args;
    a.workspace = nullptr;
    a.workspace_bytes = 0;
    return lizard_attn_fwd(&a, stream);
  }
  if (need > LIZARD_NOALLOC_SCRATCH_BYTES) return LIZARD_ERR_UNSUPPORTED;
  void *scratch = scratch_address();
  if (!scratch) return LIZARD_ERR_CUDA;
  // lizard_attn_fwd clears the status word at the start of the scratch
  // itself before its first kernel; every other byte of the scratch is
  // written before it is read.
  lizard_fwd_args a = *args;
  a.workspace = scratch;
  a.workspace_bytes = LIZARD_NOALLOC_SCRATCH_BYTES;
  return lizard_attn_fwd(&a, stream);
}

extern "C" lizard_status lizard_noalloc_status(lizard_stream_t stream) {
  void *scratch = scratch_address();
  if (!scratch) return LIZARD_ERR_CUDA;
  return lizard_workspace_status(scratch, stream);
}
