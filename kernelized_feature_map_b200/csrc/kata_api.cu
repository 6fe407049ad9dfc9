// kata_api.cu -- the C ABI of libkata (declared in include/kata.h).
//
// Validates every argument before anything is launched, plans the chunked
// path, and enqueues the kernels on the caller's stream.  Owns the
// device-side status word that kernels use to report a bounded wait that ran
// out.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "kata_internal.h"

#define KATA_API extern "C" __attribute__((visibility("default")))

namespace kata {

__device__ int g_kata_status;

static std::atomic<long long> g_wait_limit{-1};
constexpr long long kDefaultWaitLimit = 1ll << 31;  // SM cycles (about a second)

long long wait_limit() {
  long long v = g_wait_limit.load();
  return v < 0 ? kDefaultWaitLimit : v;
}

// Driver handle of the calling thread's current CUDA context, or nullptr
// when none is current (or the driver entry point is unavailable).
void* current_context() {
  using Fn = CUresult (*)(CUcontext*);
  static const Fn fn = []() -> Fn {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &qr) != cudaSuccess ||
        qr != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<Fn>(f);
  }();
  CUcontext ctx = nullptr;
  if (!fn || fn(&ctx) != CUDA_SUCCESS) return nullptr;
  return ctx;
}

// Device address of a __device__ symbol on the current device, cached per
// device and re-queried whenever the current context differs from the one
// the cached address was taken in (after a device reset the module, and the
// symbol with it, can move).
void* SymbolCache::address(const void* symbol) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return nullptr;
  std::lock_guard<std::mutex> lock(mu_);
  void* ctx = current_context();
  if (dev < kMaxDevices && ctx && ctx_[dev] == ctx && addr_[dev]) return addr_[dev];
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, symbol) != cudaSuccess) return nullptr;
  if (dev < kMaxDevices) {
    ctx_[dev] = current_context();  // the lookup made the device's context current
    addr_[dev] = p;
  }
  return p;
}

static int* status_word() {
  static SymbolCache cache;
  return static_cast<int*>(cache.address(&g_kata_status));
}

WaitCtl wait_ctl() { return WaitCtl{status_word(), wait_limit()}; }

// Super-chunk length.  One CTA handles one (b,h, super-chunk) unit, 148 SMs
// run one unit each per wave, and every unit costs its chunks plus a fixed
// overhead (prologue, state record written, scanned and read back), counted
// as kUnitOverhead chunks.  On the tensor-core path a single super-chunk per
// (b,h) needs one launch instead of three (no state build, no scan), so
// splitting costs a further kSplitOverhead chunks (two launches with their
// prologues, measured at about that much).  The plan takes the multiple of 128
// tokens that minimises  waves * (chunks per unit + kUnitOverhead) [+ split],
// preferring longer super-chunks (fewer records) on ties.  A pure function of
// the sizes, so that the workspace query and the call agree.
constexpr int kSMs = 148;
constexpr int kUnitOverhead = 2;
constexpr int kSplitOverhead = 8;

// Shared by both plans: tensor-core layout when `tc`, `cta_per_unit` CTAs
// per (b,h, super-chunk) unit (a cluster fills whole groups of four SMs).
static ChunkPlan plan_units(int B, int H, int T, int p, int dv, int C, bool tc, int cta_per_unit) {
  ChunkPlan pl{};
  pl.BH = B * H;
  pl.T = T;
  pl.p = p;
  pl.P = p * p;
  pl.dv = dv;
  pl.ld = dv + 4;
  pl.C = C;
  pl.Ls = 128;
  pl.layout = tc ? kRecPackedT : kRecUnpacked;
  const long long tiles = (T + 127) / 128;
  long long best = -1;
  const long long kmax = tiles < 1 ? 1 : (tiles < 512 ? tiles : 512);  // super-chunks up to 64K tokens
  const long long slots = cta_per_unit > 1 ? (kSMs / 4) * 4 : kSMs;
  for (long long k = kmax; k >= 1; --k) {
    const long long per_bh = (tiles + k - 1) / k;
    const long long units = (long long)pl.BH * per_bh * cta_per_unit;
    const long long waves = (units + slots - 1) / slots;
    const long long split = (tc && per_bh > 1) ? kSplitOverhead : 0;
    const long long cost = waves * (k + kUnitOverhead) + split;
    if (best < 0 || cost < best) {
      best = cost;
      pl.Ls = (int)(k * 128);
    }
  }
  if (pl.Ls < C) pl.Ls = C;
  pl.G = T > 0 ? (T + pl.Ls - 1) / pl.Ls : 0;
  pl.record_floats = tc ? (size_t)(dv + 1) * 144 : (size_t)pl.P * pl.ld;
  // the tensor-core path needs no records for a single super-chunk
  const bool no_records = tc && pl.G <= 1;
  pl.workspace_bytes = no_records ? 0 : (size_t)pl.BH * cta_per_unit * pl.G * pl.record_floats * sizeof(float);
  return pl;
}

ChunkPlan make_chunk_plan(int B, int H, int T, int p, int dv, int C, kata_dtype_t dt) {
  const bool tc = chunked_on_tensor_cores(p, dv, dt);
  return plan_units(B, H, T, p, dv, C, tc, tc ? cluster_blocks(p, 1) : 1);
}

ChunkPlan make_linear_plan(int B, int H, int T, int d, int dv, int C) {
  // The first-order kernels are bound by HBM, not by the per-chunk work of
  // the KATA ones: once every SM has a sequence, the readout alone streams
  // at the HBM rate and a split only adds the state pass's k, v reads.  So
  // one super-chunk per (b,h) when the sequences fill the SMs, otherwise
  // enough super-chunks for one wave.  Measured at H16 T131072: B16 one
  // super-chunk 1814 us against 2245 us with the split of plan_units (4);
  // B1 nine super-chunks 163.5 us against 862.5 us for one.  Records in the
  // unpacked layout (d rows of dv + 4 floats: value columns, then z).
  ChunkPlan pl = plan_units(B, H, T, d, dv, C, true, 1);
  const long long tiles = (T + 127) / 128;
  long long G = pl.BH * 10 >= (long long)kSMs * 9 ? 1 : kSMs / pl.BH;
  if (G > tiles) G = tiles;
  if (G < 1) G = 1;
  pl.Ls = (int)(((tiles + G - 1) / G) * 128);
  if (pl.Ls < C) pl.Ls = C;
  pl.G = T > 0 ? (T + pl.Ls - 1) / pl.Ls : 0;
  pl.P = d;
  pl.layout = kRecUnpacked;
  pl.record_floats = (size_t)d * pl.ld;
  pl.workspace_bytes = pl.G <= 1 ? 0 : (size_t)pl.BH * pl.G * pl.record_floats * sizeof(float);
  return pl;
}

ChunkPlan make_cluster_plan(int B, int H, int T, int p, int blocks, int dv, int C) {
  return plan_units(B, H, T, p, dv, C, true, blocks);
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static kata_status_t check_common(int B, int H, int T, int p, int dv, kata_dtype_t dt) {
  if (B < 1 || H < 1 || T < 0) return KATA_ERR_INVALID_ARG;
  if (dt != KATA_F32 && dt != KATA_BF16) return KATA_ERR_INVALID_ARG;
  if (!((p == 16 || p == 32) && (dv == 16 || dv == 64))) return KATA_ERR_UNSUPPORTED;
  // per-(b,h) offsets are kept in 32-bit integers inside the kernels
  if ((long long)T * (dv > p ? dv : p) >= (1ll << 31)) return KATA_ERR_UNSUPPORTED;
  if ((long long)B * H >= (1ll << 31) / 1) return KATA_ERR_UNSUPPORTED;
  return KATA_OK;
}

static kata_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? KATA_OK : KATA_ERR_CUDA; }

}  // namespace kata

using namespace kata;

KATA_API int kata_abi_version(void) { return KATA_ABI_VERSION; }

KATA_API const char* kata_status_string(kata_status_t s) {
  switch (s) {
    case KATA_OK: return "KATA_OK";
    case KATA_ERR_INVALID_ARG: return "KATA_ERR_INVALID_ARG";
    case KATA_ERR_UNSUPPORTED: return "KATA_ERR_UNSUPPORTED";
    case KATA_ERR_MISALIGNED: return "KATA_ERR_MISALIGNED";
    case KATA_ERR_WORKSPACE: return "KATA_ERR_WORKSPACE";
    case KATA_ERR_CUDA: return "KATA_ERR_CUDA";
    case KATA_ERR_TIMEOUT: return "KATA_ERR_TIMEOUT";
  }
  return "KATA_ERR_UNKNOWN";
}

KATA_API void kata_set_wait_limit(long long cycles) { g_wait_limit.store(cycles < 0 ? -1 : cycles); }

KATA_API kata_status_t kata_get_status(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return KATA_ERR_CUDA;
  int* addr = status_word();
  if (!addr) return KATA_ERR_CUDA;
  int h = 0;
  if (cudaMemcpy(&h, addr, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return KATA_ERR_CUDA;
  if (h != 0) {
    const int zero = 0;
    if (cudaMemcpy(addr, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return KATA_ERR_CUDA;
  }
  return static_cast<kata_status_t>(h);
}

KATA_API kata_status_t kata_fwd_quadratic(const void* q, const void* k, const void* v, void* o, int B, int H, int T,
                                          int p, int dv, kata_dtype_t dtype, void* stream) {
  kata_status_t s = check_common(B, H, T, p, dv, dtype);
  if (s != KATA_OK) return s;
  if (T == 0) return KATA_OK;
  if (!q || !k || !v || !o) return KATA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return KATA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == KATA_BF16) return from_cuda(launch_flash_sm100(q, k, v, o, B, H, T, p, dv, false, nullptr, wait_ctl(), st));
  return from_cuda(launch_quadratic_simt(q, k, v, o, B * H, T, p, dv, dtype, st));
}

KATA_API size_t kata_fwd_chunked_workspace_size(int B, int H, int T, int p, int dv, int C, kata_dtype_t dtype) {
  if (check_common(B, H, T, p, dv, dtype) != KATA_OK || !(C == 64 || C == 128) || T == 0) return 0;
  return make_chunk_plan(B, H, T, p, dv, C, dtype).workspace_bytes;
}

namespace kata {
// The chunked path of the cluster kernels (p = 32, KATA-Mg): the block sums
// of super-chunks 0..G-2 and their scan (B H x blocks sequences of records,
// no initial state) exist only when G > 1; the readout adds S0 to every
// prefix and writes the final state itself.
static cudaError_t run_cluster_chunked(const void* q, const void* k, const void* v, void* o, const ChunkPlan& plan,
                                       int H, int groups, bool bthd, const float* S0, const float* z0, float* S_out,
                                       float* z_out, float* ws, const WaitCtl& wc, cudaStream_t st) {
  cudaError_t e = cudaSuccess;
  if (plan.G > 1) {
    e = launch_chunk_state_cluster(k, v, ws, plan, H, groups, bthd, wc, st);
    ChunkPlan blocks = plan;
    blocks.BH = plan.BH * cluster_blocks(plan.p, groups);
    if (e == cudaSuccess) e = launch_state_scan(ws, blocks, plan.G - 1, nullptr, nullptr, nullptr, nullptr, st);
  }
  if (e == cudaSuccess)
    e = launch_chunk_readout_cluster(q, k, v, o, ws, S0, z0, S_out, z_out, plan, H, groups, bthd, wc, st);
  return e;
}

// Every argument check of kata_fwd_chunked except the workspace's, in the
// order that call makes them.
kata_status_t check_chunked_args(const void* q, const void* k, const void* v, const void* o, int B, int H, int T,
                                 int p, int dv, int C, kata_dtype_t dtype, const float* S0, const float* z0,
                                 const float* S_out, const float* z_out) {
  kata_status_t s = check_common(B, H, T, p, dv, dtype);
  if (s != KATA_OK) return s;
  if (!(C == 64 || C == 128)) return KATA_ERR_UNSUPPORTED;
  if ((S0 == nullptr) != (z0 == nullptr)) return KATA_ERR_INVALID_ARG;
  if ((S_out == nullptr) != (z_out == nullptr)) return KATA_ERR_INVALID_ARG;
  for (const void* ptr : {(const void*)S0, (const void*)z0, (const void*)S_out, (const void*)z_out})
    if (ptr && !aligned16(ptr)) return KATA_ERR_MISALIGNED;
  if (T == 0) return KATA_OK;
  if (!q || !k || !v || !o) return KATA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return KATA_ERR_MISALIGNED;
  return KATA_OK;
}
}  // namespace kata

KATA_API kata_status_t kata_fwd_chunked(const void* q, const void* k, const void* v, void* o, int B, int H, int T,
                                        int p, int dv, int C, kata_dtype_t dtype, const float* S0, const float* z0,
                                        float* S_out, float* z_out, void* workspace, size_t workspace_bytes,
                                        void* stream) {
  kata_status_t s = check_chunked_args(q, k, v, o, B, H, T, p, dv, C, dtype, S0, z0, S_out, z_out);
  if (s != KATA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t P = (size_t)p * p, BH = (size_t)B * H;
  if (T == 0) {
    if (!S_out) return KATA_OK;
    if (S0) {
      cudaError_t e = cudaMemcpyAsync(S_out, S0, BH * P * dv * sizeof(float), cudaMemcpyDeviceToDevice, st);
      if (e == cudaSuccess) e = cudaMemcpyAsync(z_out, z0, BH * P * sizeof(float), cudaMemcpyDeviceToDevice, st);
      return from_cuda(e);
    }
    cudaError_t e = cudaMemsetAsync(S_out, 0, BH * P * dv * sizeof(float), st);
    if (e == cudaSuccess) e = cudaMemsetAsync(z_out, 0, BH * P * sizeof(float), st);
    return from_cuda(e);
  }
  const ChunkPlan plan = make_chunk_plan(B, H, T, p, dv, C, dtype);
  if (plan.workspace_bytes > 0) {
    if (!workspace || workspace_bytes < plan.workspace_bytes) return KATA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KATA_ERR_MISALIGNED;
  }
  float* ws = plan.workspace_bytes > 0 ? static_cast<float*>(workspace) : nullptr;
  const WaitCtl wc = wait_ctl();
  if (plan.layout == kRecPackedT && p == 32)
    return from_cuda(run_cluster_chunked(q, k, v, o, plan, H, 1, false, S0, z0, S_out, z_out, ws, wc, st));
  if (plan.layout == kRecPackedT) {
    // bf16 with p = 16, dv = 64 on the tensor cores: the sums of super-chunks
    // 0..G-2 and their scan exist only when G > 1; the readout takes the
    // prefix (or S0 when G == 1) and writes the final state itself
    cudaError_t e = cudaSuccess;
    if (plan.G > 1) {
      e = launch_chunk_state_sm100(k, v, ws, plan, wc, st);
      if (e == cudaSuccess) e = launch_state_scan(ws, plan, plan.G - 1, S0, z0, nullptr, nullptr, st);
    }
    if (e == cudaSuccess)
      e = launch_chunk_readout_sm100(q, k, v, o, ws, plan.G > 1 ? nullptr : S0, plan.G > 1 ? nullptr : z0, S_out,
                                     z_out, plan, wc, st);
    return from_cuda(e);
  }
  // other sizes and fp32 inputs: the same three steps on the CUDA cores
  cudaError_t e = launch_chunk_aggregate_simt(k, v, ws, plan, dtype, st);
  if (e == cudaSuccess) e = launch_state_scan(ws, plan, plan.G, S0, z0, S_out, z_out, st);
  if (e == cudaSuccess) e = launch_chunk_readout_simt(q, k, v, o, ws, plan, dtype, st);
  return from_cuda(e);
}

KATA_API kata_status_t kata_fwd_chunked_sequential(const void* q, const void* k, const void* v, void* o, int B,
                                                   int H, int T, int p, int dv, int C, kata_dtype_t dtype,
                                                   const float* S0, const float* z0, float* S_out, float* z_out,
                                                   void* stream) {
  kata_status_t s = check_common(B, H, T, p, dv, dtype);
  if (s != KATA_OK) return s;
  if (!(C == 64 || C == 128)) return KATA_ERR_UNSUPPORTED;
  if (!chunked_on_tensor_cores(p, dv, dtype) || p != 16) return KATA_ERR_UNSUPPORTED;
  if ((S0 == nullptr) != (z0 == nullptr)) return KATA_ERR_INVALID_ARG;
  if ((S_out == nullptr) != (z_out == nullptr)) return KATA_ERR_INVALID_ARG;
  for (const void* ptr : {(const void*)S0, (const void*)z0, (const void*)S_out, (const void*)z_out})
    if (ptr && !aligned16(ptr)) return KATA_ERR_MISALIGNED;
  if (T == 0) return kata_fwd_chunked(q, k, v, o, B, H, T, p, dv, C, dtype, S0, z0, S_out, z_out, nullptr, 0, stream);
  if (!q || !k || !v || !o) return KATA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return KATA_ERR_MISALIGNED;
  // one super-chunk per (b,h): one CTA walks every chunk of its sequence in
  // order, carrying the state; no state build, no scan, no workspace
  ChunkPlan plan = make_chunk_plan(B, H, T, p, dv, C, dtype);
  plan.Ls = ((T + 127) / 128) * 128;
  plan.G = 1;
  plan.workspace_bytes = 0;
  return from_cuda(launch_chunk_readout_sm100(q, k, v, o, nullptr, S0, z0, S_out, z_out, plan, wait_ctl(),
                                              static_cast<cudaStream_t>(stream)));
}

static kata_status_t check_linear_args(const void* q, const void* k, const void* v, const void* o, int B, int H,
                                       int T, int d, int dv, int C, kata_dtype_t dtype, const float* S0,
                                       const float* z0, const float* S_out, const float* z_out) {
  if (B < 1 || H < 1 || T < 0) return KATA_ERR_INVALID_ARG;
  if (dtype != KATA_F32 && dtype != KATA_BF16) return KATA_ERR_INVALID_ARG;
  if (dtype != KATA_BF16 || d != 16 || dv != 64) return KATA_ERR_UNSUPPORTED;
  if ((long long)T * dv >= (1ll << 31)) return KATA_ERR_UNSUPPORTED;
  if (!(C == 64 || C == 128)) return KATA_ERR_UNSUPPORTED;
  if ((S0 == nullptr) != (z0 == nullptr)) return KATA_ERR_INVALID_ARG;
  if ((S_out == nullptr) != (z_out == nullptr)) return KATA_ERR_INVALID_ARG;
  for (const void* ptr : {(const void*)S0, (const void*)z0, (const void*)S_out, (const void*)z_out})
    if (ptr && !aligned16(ptr)) return KATA_ERR_MISALIGNED;
  if (T == 0) return KATA_OK;
  if (!q || !k || !v || !o) return KATA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return KATA_ERR_MISALIGNED;
  return KATA_OK;
}

// T == 0: the final state is the initial one (or zero)
static kata_status_t linear_empty(int B, int H, int d, int dv, const float* S0, const float* z0, float* S_out,
                                  float* z_out, cudaStream_t st) {
  if (!S_out) return KATA_OK;
  const size_t BH = (size_t)B * H;
  cudaError_t e = S0 ? cudaMemcpyAsync(S_out, S0, BH * d * dv * sizeof(float), cudaMemcpyDeviceToDevice, st)
                     : cudaMemsetAsync(S_out, 0, BH * d * dv * sizeof(float), st);
  if (e == cudaSuccess)
    e = S0 ? cudaMemcpyAsync(z_out, z0, BH * d * sizeof(float), cudaMemcpyDeviceToDevice, st)
           : cudaMemsetAsync(z_out, 0, BH * d * sizeof(float), st);
  return from_cuda(e);
}

KATA_API size_t kata_fwd_linear_chunked_workspace_size(int B, int H, int T, int d, int dv, int C) {
  if (B < 1 || H < 1 || T <= 0 || d != 16 || dv != 64 || !(C == 64 || C == 128)) return 0;
  return make_linear_plan(B, H, T, d, dv, C).workspace_bytes;
}

KATA_API kata_status_t kata_fwd_linear_chunked(const void* q, const void* k, const void* v, void* o, int B, int H,
                                               int T, int d, int dv, int C, kata_dtype_t dtype, const float* S0,
                                               const float* z0, float* S_out, float* z_out, void* workspace,
                                               size_t workspace_bytes, void* stream) {
  kata_status_t s = check_linear_args(q, k, v, o, B, H, T, d, dv, C, dtype, S0, z0, S_out, z_out);
  if (s != KATA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (T == 0) return linear_empty(B, H, d, dv, S0, z0, S_out, z_out, st);
  const ChunkPlan plan = make_linear_plan(B, H, T, d, dv, C);
  if (plan.workspace_bytes > 0) {
    if (!workspace || workspace_bytes < plan.workspace_bytes) return KATA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KATA_ERR_MISALIGNED;
  }
  float* ws = plan.workspace_bytes > 0 ? static_cast<float*>(workspace) : nullptr;
  const WaitCtl wc = wait_ctl();
  // sums of super-chunks 0..G-2, their scan (which adds S0), the readout
  cudaError_t e = cudaSuccess;
  if (plan.G > 1) {
    e = launch_linear_state_sm100(k, v, ws, plan, wc, st);
    if (e == cudaSuccess) e = launch_state_scan(ws, plan, plan.G - 1, S0, z0, nullptr, nullptr, st);
  }
  if (e == cudaSuccess)
    e = launch_linear_readout_sm100(q, k, v, o, ws, plan.G > 1 ? nullptr : S0, plan.G > 1 ? nullptr : z0, S_out,
                                    z_out, plan, wc, st);
  return from_cuda(e);
}

KATA_API kata_status_t kata_fwd_linear_chunked_sequential(const void* q, const void* k, const void* v, void* o,
                                                          int B, int H, int T, int d, int dv, int C,
                                                          kata_dtype_t dtype, const float* S0, const float* z0,
                                                          float* S_out, float* z_out, void* stream) {
  kata_status_t s = check_linear_args(q, k, v, o, B, H, T, d, dv, C, dtype, S0, z0, S_out, z_out);
  if (s != KATA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (T == 0) return linear_empty(B, H, d, dv, S0, z0, S_out, z_out, st);
  // one super-chunk per (b,h): one CTA walks every chunk of its sequence in
  // order, carrying the state; no state build, no scan, no workspace
  ChunkPlan plan = make_linear_plan(B, H, T, d, dv, C);
  plan.Ls = ((T + 127) / 128) * 128;
  plan.G = 1;
  plan.workspace_bytes = 0;
  return from_cuda(launch_linear_readout_sm100(q, k, v, o, nullptr, S0, z0, S_out, z_out, plan, wait_ctl(), st));
}

KATA_API kata_status_t kata_decode_step(const void* q, const void* k, const void* v, void* o, float* S, float* z,
                                        int B, int H, int p, int dv, kata_dtype_t dtype, void* stream) {
  kata_status_t s = check_common(B, H, 1, p, dv, dtype);
  if (s != KATA_OK) return s;
  if (!q || !k || !v || !o || !S || !z) return KATA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(S) || !aligned16(z))
    return KATA_ERR_MISALIGNED;
  return from_cuda(launch_decode(q, k, v, o, S, z, B * H, p, 1, dv, dtype, static_cast<cudaStream_t>(stream)));
}

static kata_status_t check_train(int B, int H, int T, int p, int dv, kata_dtype_t dt) {
  kata_status_t s = check_common(B, H, T, p, dv, dt);
  if (s != KATA_OK) return s;
  if (dt != KATA_BF16 || dv != 64) return KATA_ERR_UNSUPPORTED;
  return KATA_OK;
}

// Training on the chunked path (bf16, p = 16, dv = 64): the forward that
// also writes D, and the O(T) backward.
KATA_API kata_status_t kata_fwd_chunked_train(const void* q, const void* k, const void* v, void* o, float* D, int B,
                                              int H, int T, int p, int dv, int C, kata_dtype_t dtype, void* workspace,
                                              size_t workspace_bytes, void* stream) {
  kata_status_t s = check_chunked_args(q, k, v, o, B, H, T, p, dv, C, dtype, nullptr, nullptr, nullptr, nullptr);
  if (s != KATA_OK) return s;
  if (dtype != KATA_BF16 || p != 16 || dv != 64) return KATA_ERR_UNSUPPORTED;
  if (T == 0) return KATA_OK;
  if (!D) return KATA_ERR_INVALID_ARG;
  if (!aligned16(D)) return KATA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const ChunkPlan plan = make_chunk_plan(B, H, T, p, dv, C, dtype);
  if (plan.workspace_bytes > 0) {
    if (!workspace || workspace_bytes < plan.workspace_bytes) return KATA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KATA_ERR_MISALIGNED;
  }
  float* ws = plan.workspace_bytes > 0 ? static_cast<float*>(workspace) : nullptr;
  const WaitCtl wc = wait_ctl();
  cudaError_t e = cudaSuccess;
  if (plan.G > 1) {
    e = launch_chunk_state_sm100(k, v, ws, plan, wc, st);
    if (e == cudaSuccess) e = launch_state_scan(ws, plan, plan.G - 1, nullptr, nullptr, nullptr, nullptr, st);
  }
  if (e == cudaSuccess)
    e = launch_chunk_readout_sm100(q, k, v, o, ws, nullptr, nullptr, nullptr, nullptr, plan, wc, st, D);
  return from_cuda(e);
}

static size_t round256(size_t x) { return (x + 255) / 256 * 256; }

KATA_API size_t kata_bwd_chunked_workspace_size(int B, int H, int T, int p, int dv, kata_dtype_t dtype) {
  if (B < 1 || H < 1 || T <= 0 || p != 16 || dv != 64 || dtype != KATA_BF16) return 0;
  const int BH = B * H;
  return round256(flash_bwd_workspace_bytes(BH, T, dv)) + chunk_bwd_records_bytes(BH, T);
}

KATA_API kata_status_t kata_bwd_chunked(const void* q, const void* k, const void* v, const void* o, const float* D,
                                        const void* dO, void* dq, void* dk, void* dv, int B, int H, int T, int p,
                                        int dv_width, kata_dtype_t dtype, void* workspace, size_t workspace_bytes,
                                        void* stream) {
  kata_status_t s = check_train(B, H, T, p, dv_width, dtype);
  if (s != KATA_OK) return s;
  if (p != 16) return KATA_ERR_UNSUPPORTED;
  if (T == 0) return KATA_OK;
  for (const void* ptr : {q, k, v, o, (const void*)D, dO, (const void*)dq, (const void*)dk, (const void*)dv})
    if (!ptr) return KATA_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, o, (const void*)D, dO, (const void*)dq, (const void*)dk, (const void*)dv})
    if (!aligned16(ptr)) return KATA_ERR_MISALIGNED;
  const int BH = B * H;
  if (!workspace || workspace_bytes < kata_bwd_chunked_workspace_size(B, H, T, p, dv_width, dtype))
    return KATA_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KATA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const WaitCtl wc = wait_ctl();
  // the per-row constants; the pairs across chunks through the chunk states
  // (written to dq, dk, dv); then the pairs inside each 128-token chunk, the
  // flash backward on its diagonal tiles, added to them
  uint8_t* w8 = static_cast<uint8_t*>(workspace);
  const bool inter = T > 128;  // some pair crosses a chunk boundary
  cudaError_t e = launch_flash_bwd_rows(dO, o, D, w8, BH, T, st);
  if (e == cudaSuccess && inter)
    e = launch_chunk_bwd_inter_sm100(q, k, v, dO, reinterpret_cast<const float2*>(w8),
                                     reinterpret_cast<float*>(w8 + round256(flash_bwd_workspace_bytes(BH, T, dv_width))),
                                     dq, dk, dv, BH, T, wc, st);
  if (e == cudaSuccess)
    e = launch_flash_bwd_sm100(q, k, v, o, D, dO, dq, dk, dv, BH, T, p, p, true, inter, inter, inter, w8, wc, st,
                               true);
  return from_cuda(e);
}


KATA_API kata_status_t kata_fwd_quadratic_train(const void* q, const void* k, const void* v, void* o, float* D,
                                                int B, int H, int T, int p, int dv, kata_dtype_t dtype,
                                                void* stream) {
  kata_status_t s = check_train(B, H, T, p, dv, dtype);
  if (s != KATA_OK) return s;
  if (T == 0) return KATA_OK;
  if (!q || !k || !v || !o || !D) return KATA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(D)) return KATA_ERR_MISALIGNED;
  return from_cuda(
      launch_flash_sm100(q, k, v, o, B, H, T, p, dv, false, D, wait_ctl(), static_cast<cudaStream_t>(stream)));
}

KATA_API size_t kata_bwd_quadratic_workspace_size(int B, int H, int T, int p, int dv, kata_dtype_t dtype) {
  if (check_train(B, H, T, p, dv, dtype) != KATA_OK || T == 0) return 0;
  return flash_bwd_workspace_bytes(B * H, T, dv);
}

KATA_API kata_status_t kata_bwd_quadratic(const void* q, const void* k, const void* v, const void* o, const float* D,
                                          const void* dO, void* dq, void* dk, void* dv, int B, int H, int T, int p,
                                          int dv_width, kata_dtype_t dtype, void* workspace, size_t workspace_bytes,
                                          void* stream) {
  kata_status_t s = check_train(B, H, T, p, dv_width, dtype);
  if (s != KATA_OK) return s;
  if (T == 0) return KATA_OK;
  for (const void* ptr : {q, k, v, o, (const void*)D, dO, (const void*)dq, (const void*)dk, (const void*)dv})
    if (!ptr) return KATA_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, o, (const void*)D, dO, (const void*)dq, (const void*)dk, (const void*)dv})
    if (!aligned16(ptr)) return KATA_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < flash_bwd_workspace_bytes(B * H, T, dv_width)) return KATA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return KATA_ERR_MISALIGNED;
  return from_cuda(launch_flash_bwd_sm100(q, k, v, o, D, dO, dq, dk, dv, B * H, T, p, p, false, false, false, false,
                                          workspace,
                                          wait_ctl(), static_cast<cudaStream_t>(stream)));
}

// Shape checks shared by the KATA-Mg entry points: p = d / groups.
static kata_status_t check_mg(int B, int H, int T, int d, int groups, int dv, kata_dtype_t dt, int* p_out) {
  if (groups < 1 || d < 1 || d % groups != 0) return KATA_ERR_INVALID_ARG;
  const int p = d / groups;
  kata_status_t s = check_common(B, H, T, p, dv, dt);
  if (s != KATA_OK) return s;
  if ((long long)T * d >= (1ll << 31)) return KATA_ERR_UNSUPPORTED;
  if (groups > 1 && !flash_mg_sm100_supports(p, groups, dv)) return KATA_ERR_UNSUPPORTED;
  *p_out = p;
  return KATA_OK;
}

KATA_API kata_status_t kata_fwd_mg_quadratic(const void* q, const void* k, const void* v, void* o, int B, int H,
                                             int T, int d, int groups, int dv, kata_layout_t layout,
                                             kata_dtype_t dtype, void* stream) {
  int p = 0;
  kata_status_t s = check_mg(B, H, T, d, groups, dv, dtype, &p);
  if (s != KATA_OK) return s;
  if (layout != KATA_LAYOUT_BHTD && layout != KATA_LAYOUT_BTHD) return KATA_ERR_INVALID_ARG;
  if (dtype != KATA_BF16) return KATA_ERR_UNSUPPORTED;
  if (T == 0) return KATA_OK;
  if (!q || !k || !v || !o) return KATA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return KATA_ERR_MISALIGNED;
  const bool bthd = layout == KATA_LAYOUT_BTHD;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (flash_mg_sm100_supports(p, groups, dv))
    return from_cuda(launch_flash_mg_sm100(q, k, v, o, nullptr, B, H, T, p, groups, bthd, wait_ctl(), st));
  return from_cuda(launch_flash_sm100(q, k, v, o, B, H, T, p, dv, bthd, nullptr, wait_ctl(), st));
}

// (d, groups) of the chunked KATA-Mg path on the cluster kernels, after the
// shape checks of check_mg.
static bool mg_chunked_on_clusters(int p, int groups, int dv, kata_dtype_t dt) {
  return dt == KATA_BF16 && groups > 1 && cluster_chunked_supports(p, groups, dv);
}

KATA_API size_t kata_fwd_mg_chunked_workspace_size(int B, int H, int T, int d, int groups, int dv, int C,
                                                   kata_dtype_t dtype) {
  int p = 0;
  if (check_mg(B, H, T, d, groups, dv, dtype, &p) != KATA_OK || !(C == 64 || C == 128) || T == 0) return 0;
  if (groups == 1) return kata_fwd_chunked_workspace_size(B, H, T, p, dv, C, dtype);
  if (!mg_chunked_on_clusters(p, groups, dv, dtype)) return 0;
  return make_cluster_plan(B, H, T, p, cluster_blocks(p, groups), dv, C).workspace_bytes;
}

KATA_API kata_status_t kata_fwd_mg_chunked(const void* q, const void* k, const void* v, void* o, int B, int H, int T,
                                           int d, int groups, int dv, int C, kata_layout_t layout,
                                           kata_dtype_t dtype, const float* S0, const float* z0, float* S_out,
                                           float* z_out, void* workspace, size_t workspace_bytes, void* stream) {
  int p = 0;
  kata_status_t s = check_mg(B, H, T, d, groups, dv, dtype, &p);
  if (s != KATA_OK) return s;
  if (layout != KATA_LAYOUT_BHTD && layout != KATA_LAYOUT_BTHD) return KATA_ERR_INVALID_ARG;
  if (!(C == 64 || C == 128)) return KATA_ERR_UNSUPPORTED;
  const bool bthd = layout == KATA_LAYOUT_BTHD;
  if (groups == 1 && !bthd)
    return kata_fwd_chunked(q, k, v, o, B, H, T, p, dv, C, dtype, S0, z0, S_out, z_out, workspace, workspace_bytes,
                            stream);
  const bool single32 = groups == 1 && p == 32 && dtype == KATA_BF16 && dv == 64;
  if (!single32 && !mg_chunked_on_clusters(p, groups, dv, dtype)) return KATA_ERR_UNSUPPORTED;
  if ((S0 == nullptr) != (z0 == nullptr)) return KATA_ERR_INVALID_ARG;
  if ((S_out == nullptr) != (z_out == nullptr)) return KATA_ERR_INVALID_ARG;
  for (const void* ptr : {(const void*)S0, (const void*)z0, (const void*)S_out, (const void*)z_out})
    if (ptr && !aligned16(ptr)) return KATA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t P = (size_t)groups * p * p, BH = (size_t)B * H;
  if (T == 0) {
    if (!S_out) return KATA_OK;
    cudaError_t e;
    if (S0) {
      e = cudaMemcpyAsync(S_out, S0, BH * P * dv * sizeof(float), cudaMemcpyDeviceToDevice, st);
      if (e == cudaSuccess) e = cudaMemcpyAsync(z_out, z0, BH * P * sizeof(float), cudaMemcpyDeviceToDevice, st);
    } else {
      e = cudaMemsetAsync(S_out, 0, BH * P * dv * sizeof(float), st);
      if (e == cudaSuccess) e = cudaMemsetAsync(z_out, 0, BH * P * sizeof(float), st);
    }
    return from_cuda(e);
  }
  if (!q || !k || !v || !o) return KATA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return KATA_ERR_MISALIGNED;
  const ChunkPlan plan = make_cluster_plan(B, H, T, p, cluster_blocks(p, groups), dv, C);
  if (plan.workspace_bytes > 0) {
    if (!workspace || workspace_bytes < plan.workspace_bytes) return KATA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KATA_ERR_MISALIGNED;
  }
  float* ws = plan.workspace_bytes > 0 ? static_cast<float*>(workspace) : nullptr;
  return from_cuda(run_cluster_chunked(q, k, v, o, plan, H, groups, bthd, S0, z0, S_out, z_out, ws, wait_ctl(), st));
}

KATA_API kata_status_t kata_fwd_sg_quadratic(const void* q, const void* k, const void* v, void* o, int B, int H,
                                             int T, int d, int groups, int dv, kata_layout_t layout,
                                             kata_dtype_t dtype, void* stream) {
  int p = 0;
  kata_status_t s = check_mg(B, H, T, d, groups, dv, dtype, &p);
  if (s != KATA_OK) return s;
  if (layout != KATA_LAYOUT_BHTD && layout != KATA_LAYOUT_BTHD) return KATA_ERR_INVALID_ARG;
  if (dtype != KATA_BF16 || groups < 2) return KATA_ERR_UNSUPPORTED;
  if (T == 0) return KATA_OK;
  if (!q || !k || !v || !o) return KATA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return KATA_ERR_MISALIGNED;
  return from_cuda(launch_flash_sg_sm100(q, k, v, o, nullptr, B, H, T, p, groups, layout == KATA_LAYOUT_BTHD, wait_ctl(),
                                         static_cast<cudaStream_t>(stream)));
}

KATA_API kata_status_t kata_fwd_mg_quadratic_train(const void* q, const void* k, const void* v, void* o, float* D,
                                                   int B, int H, int T, int d, int groups, int dv,
                                                   kata_dtype_t dtype, void* stream) {
  int p = 0;
  kata_status_t s = check_mg(B, H, T, d, groups, dv, dtype, &p);
  if (s != KATA_OK) return s;
  if (dtype != KATA_BF16 || groups < 2) return KATA_ERR_UNSUPPORTED;
  if (T == 0) return KATA_OK;
  if (!q || !k || !v || !o || !D) return KATA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(D)) return KATA_ERR_MISALIGNED;
  return from_cuda(launch_flash_mg_sm100(q, k, v, o, D, B, H, T, p, groups, false, wait_ctl(),
                                         static_cast<cudaStream_t>(stream)));
}

KATA_API kata_status_t kata_bwd_mg_quadratic(const void* q, const void* k, const void* v, const void* o,
                                             const float* D, const void* dO, void* dq, void* dk, void* dv, int B,
                                             int H, int T, int d, int groups, int dv_width, kata_dtype_t dtype,
                                             void* workspace, size_t workspace_bytes, void* stream) {
  int p = 0;
  kata_status_t s = check_mg(B, H, T, d, groups, dv_width, dtype, &p);
  if (s != KATA_OK) return s;
  if (dtype != KATA_BF16 || groups < 2) return KATA_ERR_UNSUPPORTED;
  if (T == 0) return KATA_OK;
  for (const void* ptr : {q, k, v, o, (const void*)D, dO, (const void*)dq, (const void*)dk, (const void*)dv})
    if (!ptr) return KATA_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, o, (const void*)D, dO, (const void*)dq, (const void*)dk, (const void*)dv})
    if (!aligned16(ptr)) return KATA_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < flash_bwd_workspace_bytes(B * H, T, dv_width)) return KATA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return KATA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // one pass per group on its columns: dq^j, dk^j from the group's scores,
  // dv summed over the groups; the per-row constants are computed once
  for (int j = 0; j < groups; ++j) {
    const size_t off = (size_t)j * p * 2;  // bytes
    cudaError_t e = launch_flash_bwd_sm100(static_cast<const char*>(q) + off, static_cast<const char*>(k) + off, v, o, D,
                                           dO, static_cast<char*>(dq) + off, static_cast<char*>(dk) + off, dv, B * H,
                                           T, p, d, j > 0, j > 0, false, false, workspace, wait_ctl(), st);
    if (e != cudaSuccess) return from_cuda(e);
  }
  return KATA_OK;
}

KATA_API kata_status_t kata_fwd_sg_quadratic_train(const void* q, const void* k, const void* v, void* o, float* D,
                                                   int B, int H, int T, int d, int groups, int dv,
                                                   kata_dtype_t dtype, void* stream) {
  int p = 0;
  kata_status_t s = check_mg(B, H, T, d, groups, dv, dtype, &p);
  if (s != KATA_OK) return s;
  if (dtype != KATA_BF16 || groups < 2) return KATA_ERR_UNSUPPORTED;
  if (T == 0) return KATA_OK;
  if (!q || !k || !v || !o || !D) return KATA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(D)) return KATA_ERR_MISALIGNED;
  return from_cuda(launch_flash_sg_sm100(q, k, v, o, D, B, H, T, p, groups, false, wait_ctl(),
                                         static_cast<cudaStream_t>(stream)));
}

KATA_API kata_status_t kata_bwd_sg_quadratic(const void* q, const void* k, const void* v, const void* o,
                                             const float* D, const void* dO, void* dq, void* dk, void* dv, int B,
                                             int H, int T, int d, int groups, int dv_width, kata_dtype_t dtype,
                                             void* workspace, size_t workspace_bytes, void* stream) {
  int p = 0;
  kata_status_t s = check_mg(B, H, T, d, groups, dv_width, dtype, &p);
  if (s != KATA_OK) return s;
  if (dtype != KATA_BF16 || groups < 2) return KATA_ERR_UNSUPPORTED;
  if (T == 0) return KATA_OK;
  for (const void* ptr : {q, k, v, o, (const void*)D, dO, (const void*)dq, (const void*)dk, (const void*)dv})
    if (!ptr) return KATA_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, o, (const void*)D, dO, (const void*)dq, (const void*)dk, (const void*)dv})
    if (!aligned16(ptr)) return KATA_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < flash_bwd_workspace_bytes(B * H, T, dv_width)) return KATA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return KATA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // one pass per (query group j, key group l) with that pair's scores
  // q^j . k^l: dq^j sums over l, dk^l over j and dv over every pair (the
  // weight is linear in the pairs' squares); the per-row constants are
  // computed in the first pass
  for (int j = 0; j < groups; ++j) {
    for (int l = 0; l < groups; ++l) {
      const size_t oj = (size_t)j * p * 2, ol = (size_t)l * p * 2;  // bytes
      const bool first = j == 0 && l == 0;
      cudaError_t e = launch_flash_bwd_sm100(static_cast<const char*>(q) + oj, static_cast<const char*>(k) + ol, v, o,
                                             D, dO, static_cast<char*>(dq) + oj, static_cast<char*>(dk) + ol, dv,
                                             B * H, T, p, d, !first, !first, l > 0, j > 0, workspace, wait_ctl(), st);
      if (e != cudaSuccess) return from_cuda(e);
    }
  }
  return KATA_OK;
}

// KATA-Sigma-g on the chunked path: groups of 16 (p = 16), dv = 64, bf16.
static kata_status_t check_sg_chunked(const void* q, const void* k, const void* v, const void* o, int B, int H,
                                      int T, int d, int groups, int dv, int C, kata_dtype_t dtype, const float* S0,
                                      const float* z0, const float* S_out, const float* z_out) {
  if (groups < 1 || d < 1 || d % groups != 0) return KATA_ERR_INVALID_ARG;
  if (dtype != KATA_F32 && dtype != KATA_BF16) return KATA_ERR_INVALID_ARG;
  if (dtype != KATA_BF16 || dv != 64 || d / groups != 16 || !(groups == 2 || groups == 4))
    return KATA_ERR_UNSUPPORTED;
  return check_chunked_args(q, k, v, o, B, H, T, 16, dv, C, dtype, S0, z0, S_out, z_out);
}

KATA_API size_t kata_fwd_sg_chunked_workspace_size(int B, int H, int T, int d, int groups, int dv, int C) {
  if (groups < 1 || d != 16 * groups) return 0;
  return kata_fwd_chunked_workspace_size(B, H, T, 16, dv, C, KATA_BF16);
}

KATA_API kata_status_t kata_fwd_sg_chunked(const void* q, const void* k, const void* v, void* o, int B, int H, int T,
                                           int d, int groups, int dv, int C, kata_dtype_t dtype, const float* S0,
                                           const float* z0, float* S_out, float* z_out, void* workspace,
                                           size_t workspace_bytes, void* stream) {
  kata_status_t s = check_sg_chunked(q, k, v, o, B, H, T, d, groups, dv, C, dtype, S0, z0, S_out, z_out);
  if (s != KATA_OK) return s;
  // T == 0: the state passes through (the p = 16 state of the summed feature)
  if (T == 0) return kata_fwd_chunked(q, k, v, o, B, H, 0, 16, dv, C, dtype, S0, z0, S_out, z_out, nullptr, 0, stream);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const ChunkPlan plan = make_chunk_plan(B, H, T, 16, dv, C, dtype);
  if (plan.workspace_bytes > 0) {
    if (!workspace || workspace_bytes < plan.workspace_bytes) return KATA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KATA_ERR_MISALIGNED;
  }
  float* ws = plan.workspace_bytes > 0 ? static_cast<float*>(workspace) : nullptr;
  const WaitCtl wc = wait_ctl();
  cudaError_t e = cudaSuccess;
  if (plan.G > 1) {
    e = launch_chunk_state_sg(k, v, ws, plan, groups, wc, st);
    if (e == cudaSuccess) e = launch_state_scan(ws, plan, plan.G - 1, S0, z0, nullptr, nullptr, st);
  }
  if (e == cudaSuccess)
    e = launch_chunk_readout_sg(q, k, v, o, ws, plan.G > 1 ? nullptr : S0, plan.G > 1 ? nullptr : z0, S_out, z_out,
                                plan, groups, wc, st);
  return from_cuda(e);
}

KATA_API kata_status_t kata_decode_step_sg(const void* q, const void* k, const void* v, void* o, float* S, float* z,
                                           int B, int H, int d, int groups, int dv, kata_dtype_t dtype,
                                           void* stream) {
  int p = 0;
  kata_status_t s = check_mg(B, H, 1, d, groups, dv, dtype, &p);
  if (s != KATA_OK) return s;
  if (groups == 1) return kata_decode_step(q, k, v, o, S, z, B, H, p, dv, dtype, stream);
  if (!q || !k || !v || !o || !S || !z) return KATA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(S) || !aligned16(z))
    return KATA_ERR_MISALIGNED;
  return from_cuda(
      launch_decode_sg(q, k, v, o, S, z, B * H, p, groups, dv, dtype, static_cast<cudaStream_t>(stream)));
}

KATA_API kata_status_t kata_decode_step_mg(const void* q, const void* k, const void* v, void* o, float* S, float* z,
                                           int B, int H, int d, int groups, int dv, kata_dtype_t dtype,
                                           void* stream) {
  int p = 0;
  kata_status_t s = check_mg(B, H, 1, d, groups, dv, dtype, &p);
  if (s != KATA_OK) return s;
  if (!q || !k || !v || !o || !S || !z) return KATA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(S) || !aligned16(z))
    return KATA_ERR_MISALIGNED;
  return from_cuda(launch_decode(q, k, v, o, S, z, B * H, p, groups, dv, dtype, static_cast<cudaStream_t>(stream)));
}
