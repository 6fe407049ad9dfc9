// noalloc.cu -- kata_fwd_chunked_noalloc: the chunked-state forward with its
// scratch memory in a fixed, library-owned device array instead of a
// caller-provided workspace.
//
// Some callers cannot allocate device memory themselves: a plain C host
// program linked only against this library with no allocator of its own, or
// a latency-critical loop whose rules forbid cudaMalloc (which can block and
// synchronise the device).  For them this entry point takes only inputs and
// outputs; the state records that the chunked path needs between its launches
// live in the file-scope array below.
//
// The array holds kNoallocScratchBytes (16 MiB) on every GPU that loads the
// library, until the process exits.  Sizes whose workspace would exceed it
// are rejected with KATA_ERR_WORKSPACE.  All calls share the one array: calls
// that overlap on the GPU (different streams, or different host threads on
// the same device) race on it and must be serialised by the caller.  Nothing
// in the array needs to start at zero: every record the path reads was
// written earlier in the same call.
//
// The device address of the array is looked up with that device current by
// the first call made on it (cudaGetSymbolAddress), and again whenever the
// calling thread's CUDA context is no longer the one the address was taken
// in (after a device reset the array can move); make that first call before
// any stream capture.  Host code never uses the array's name as an address.
#include <cuda_runtime.h>

#include "kata_internal.h"

#define KATA_API extern "C" __attribute__((visibility("default")))

namespace kata {
namespace {

constexpr size_t kNoallocScratchBytes = KATA_NOALLOC_SCRATCH_BYTES;
static_assert(kNoallocScratchBytes == (size_t)16 << 20, "the scratch size stated in kata.h");

static __device__ __align__(256) float g_noalloc_scratch[kNoallocScratchBytes / sizeof(float)];

// Device address of g_noalloc_scratch on the current device, or nullptr.
void* scratch_address() {
  static SymbolCache cache;
  return cache.address(&g_noalloc_scratch);
}

}  // namespace
}  // namespace kata

KATA_API kata_status_t kata_fwd_chunked_noalloc(const void* q, const void* k, const void* v, void* o, int B, int H,
                                                int T, int p, int dv, int C, kata_dtype_t dtype, const float* S0,
                                                const float* z0, float* S_out, float* z_out, void* stream) {
  // the argument errors of kata_fwd_chunked, in its order, before the size
  kata_status_t s = kata::check_chunked_args(q, k, v, o, B, H, T, p, dv, C, dtype, S0, z0, S_out, z_out);
  if (s != KATA_OK) return s;
  const size_t need = kata_fwd_chunked_workspace_size(B, H, T, p, dv, C, dtype);
  if (need > kata::kNoallocScratchBytes) return KATA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (need > 0) {
    scratch = kata::scratch_address();
    if (!scratch) return KATA_ERR_CUDA;
  }
  return kata_fwd_chunked(q, k, v, o, B, H, T, p, dv, C, dtype, S0, z0, S_out, z_out, scratch,
                          need > 0 ? kata::kNoallocScratchBytes : 0, stream);
}
