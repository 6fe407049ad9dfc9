// kata_trace.cuh -- optional per-CTA event timestamps for pipeline analysis.
//
// Compiled out unless KATA_ENABLE_TRACE is defined (the product library is
// built without it; `python -m kernelized_feature_map_b200.build --trace`
// builds a separate libkata_trace.so).  When enabled, a kernel records
// clock64() into a caller-provided buffer:
//   buf[((cta * kTraceTiles + tile) * kTraceSlots) + slot]
// for the first kTraceCtas CTAs of a launch (cta = linear block index) and
// the first kTraceTiles pipeline iterations.  The buffer is attached per
// translation unit by kata_trace_attach_<name>() (trace build only).
#pragma once

#include <stdint.h>

namespace kata {
constexpr int kTraceCtas = 8;
constexpr int kTraceTiles = 64;
constexpr int kTraceSlots = 32;
}  // namespace kata

#ifdef KATA_ENABLE_TRACE
#define KATA_TRACE_DECLARE(name)                                                         \
  static __device__ unsigned long long* g_trace_buf_##name;                             \
  extern "C" __attribute__((visibility("default"))) int kata_trace_attach_##name(void* p) { \
    return (int)cudaMemcpyToSymbol(g_trace_buf_##name, &p, sizeof(p));                    \
  }
// Once per kernel, before any KATA_TRACE of `name`: this CTA's slice of the
// buffer (null when the buffer is not attached or the CTA is not traced),
// held in a register so that recording an event is a single store.
#define KATA_TRACE_BEGIN(name)                                                            \
  unsigned long long* const kata_trace_ptr_##name = [] {                                 \
    const unsigned cta_ = blockIdx.y * gridDim.x + blockIdx.x;                           \
    return (g_trace_buf_##name && cta_ < (unsigned)::kata::kTraceCtas)                   \
               ? g_trace_buf_##name + (size_t)cta_ * ::kata::kTraceTiles * ::kata::kTraceSlots \
               : (unsigned long long*)nullptr;                                          \
  }()
// The same with an explicit CTA index (kernels with a 3-D grid).
#define KATA_TRACE_BEGIN_IDX(name, idx)                                                   \
  unsigned long long* const kata_trace_ptr_##name = [&] {                                \
    const unsigned cta_ = (idx);                                                         \
    return (g_trace_buf_##name && cta_ < (unsigned)::kata::kTraceCtas)                   \
               ? g_trace_buf_##name + (size_t)cta_ * ::kata::kTraceTiles * ::kata::kTraceSlots \
               : (unsigned long long*)nullptr;                                          \
  }()
#define KATA_TRACE(name, tile, slot)                                                     \
  do {                                                                                 \
    if (kata_trace_ptr_##name && (tile) < ::kata::kTraceTiles)                           \
      kata_trace_ptr_##name[(tile) * ::kata::kTraceSlots + (slot)] = clock64();          \
  } while (0)
#else
#define KATA_TRACE_DECLARE(name)
#define KATA_TRACE_BEGIN(name) \
  do {                         \
  } while (0)
#define KATA_TRACE_BEGIN_IDX(name, idx) \
  do {                                  \
  } while (0)
#define KATA_TRACE(name, tile, slot) \
  do {                               \
  } while (0)
#endif
