// Backward entry point for callers that cannot allocate device memory.
//
// monarch_bwd needs a caller-provided workspace.  Some callers have no way to
// obtain one: code running where cudaMalloc is not allowed or not wanted (for
// example a host framework that hands over only its own tensors, a process
// whose memory pool is fixed up front, or code that must not touch the CUDA
// allocator while other work is being captured).  For them this file provides
// monarch_bwd_noalloc, which runs exactly the same backward kernels as
// monarch_bwd but takes its scratch from a fixed array in device memory that is
// part of the library itself.
//
// The array lives at file scope as a __device__ variable, so every GPU on which
// the library is loaded holds it until the process exits.  Host code cannot use
// the array's name as a device address, so every call looks the address up with
// cudaGetSymbolAddress in the calling thread's current context.  The lookup is a
// host-side query that allocates nothing; doing it per call (rather than caching
// one address per device) keeps the address right after cudaDeviceReset or when
// the caller runs in a context other than the device's primary one.
#include "common.cuh"

namespace {

// Upper bound of the scratch this entry point can use (32 MiB).
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch in the current context (nullptr on error).
void* scratch_for_current_context() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
  return p;
}

}  // namespace

extern "C" {

int monarch_bwd_noalloc(const void* dY, const void* X, const void* R, const void* L,
                        const monarch_dims* d, void* dX, void* dR, void* dL, void* stream) {
  const int rc = monarch_validate(d);
  if (rc != MONARCH_OK) return rc;
  if (monarch_bwd_workspace_bytes(d) > kNoAllocScratchBytes) return MONARCH_ERR_SCRATCH;
  void* scratch = scratch_for_current_context();
  if (scratch == nullptr) return MONARCH_ERR_CUDA;
  return monarch_bwd(dY, X, R, L, d, dX, dR, dL, scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
