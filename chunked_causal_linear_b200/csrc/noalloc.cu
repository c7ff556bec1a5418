// lin_attn_prefill_noalloc: the prefill with its scratch in a fixed device array.
//
// Some callers must not allocate device memory while they run: serving processes that
// reserve their whole device-memory budget at start-up and forbid allocations on the
// request path, host frameworks that own every device allocation through their own
// allocator, and code paths that have no way to recover from a failed allocation.  This
// entry point gives them the prefill without any allocation: the chunk summaries and
// scan totals live in the file-scope array below instead of memory from cudaMalloc or
// cudaMallocAsync.  The caller still provides q, k, v, out and the optional final states.
//
// The array (LA_NOALLOC_SCRATCH_BYTES) is part of the library's device image, so every
// GPU that loads the library holds it until the process exits.  All calls share it and
// it keeps whatever the previous call left there; the kernels write every byte of the
// workspace they later read, so nothing needs clearing between calls.  Calls whose work
// overlaps on the GPU (different streams, or different host threads on one device) race
// on the array and must be serialised by the caller.

#include <cuda_runtime.h>

#include "../../include/linattn.h"
#include "launch.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[LA_NOALLOC_SCRATCH_BYTES];

// Device address of the array on the current device.  In host code the array's name is
// only a host-side stand-in, so the address is looked up, on every call: a cached address
// would go stale after cudaDeviceReset, which loads the module again.
int scratch_address(void** out) {
  void* ptr = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
  if (e != cudaSuccess || ptr == nullptr) {
    cudaGetLastError();
    return LA_ERR_CUDA;
  }
  *out = ptr;
  return LA_OK;
}

}  // namespace

extern "C" int lin_attn_prefill_noalloc(const la_prefill_args* args) {
  if (!args) return LA_ERR_INVALID_ARGUMENT;
  const size_t need = lin_attn_prefill_workspace_bytes(args->B, args->H, args->T, args->dk,
                                                       args->dv, args->C, args->normalize);
  if (need > LA_NOALLOC_SCRATCH_BYTES) return LA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (need > 0) {
    const int st = scratch_address(&scratch);
    if (st != LA_OK) return st;
  }
  la_prefill_args a = *args;
  a.workspace = scratch;
  a.workspace_bytes = LA_NOALLOC_SCRATCH_BYTES;
  return la::prefill_with_args(a);
}
