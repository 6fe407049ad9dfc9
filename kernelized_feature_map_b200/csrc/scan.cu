// scan.cu -- inter-chunk state propagation as a work-efficient associative
// scan (parallel prefix sum).
//
// The chunk states combine by plain addition (the state update is
// commutative and additive: ai.info summary, Main Findings "The readout gate
// is free"), so the state entering super-chunk g is the exclusive prefix sum
// S0 + sum_{g' < g} A_{g'} of the per-super-chunk sums A_{g'}.  A sequential
// pass over the G records would have depth O(G); this kernel runs the
// up-sweep / down-sweep prefix scan (Blelloch) over them instead, depth
// O(log G) (gist.science technical summary, sec. 2.3 "Chunked Parallelism" /
// "Complexiteitsreductie": recurrence depth O(N_C) -> O(log N_C)).
//
// Work decomposition: one CTA per (b,h) and strip of 32 state entries; lane
// = entry, the 8 warps share the tree levels.  The [G x 32] strip sits in
// shared memory (at most 1024 records per pass; longer sequences are scanned
// in blocks of 1024 with a running carry).  The kernel streams each record
// once in and once out, so it is bound by HBM.
//
// Record layout (per (b,h), per super-chunk g): P rows x ld floats; columns
// 0..dv-1 hold the sum of psi(k) v^T, column dv the sum of psi(k) (the
// normaliser), columns dv+1..ld-1 are padding and are not touched here.
#include "kata_common.cuh"
#include "kata_internal.h"

namespace kata {

constexpr int kScanBlock = 1024;  // records per shared-memory pass
constexpr int kScanThreads = 256;

__global__ void __launch_bounds__(kScanThreads) state_scan_kernel(float* __restrict__ ws, int G, int P, int dv,
                                                                   int ld, long long record_floats,
                                                                   const float* __restrict__ S0,
                                                                   const float* __restrict__ z0,
                                                                   float* __restrict__ S_out,
                                                                   float* __restrict__ z_out) {
  extern __shared__ float tile[];  // [Gp][32]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = kScanThreads / 32;
  const long long bh = blockIdx.y;
  const int E = P * (dv + 1);
  const int e = blockIdx.x * 32 + lane;
  const bool active = e < E;
  const int r = active ? e / (dv + 1) : 0;
  const int c = active ? e % (dv + 1) : 0;
  const long long off = (long long)r * ld + c;
  float* base = ws + bh * (long long)G * record_floats + off;

  float carry = 0.f;
  if (active && S0) carry = (c < dv) ? S0[(bh * P + r) * dv + c] : z0[bh * P + r];

  for (int g0 = 0; g0 < G; g0 += kScanBlock) {
    const int n = min(kScanBlock, G - g0);
    int Gp = 1;
    while (Gp < n) Gp <<= 1;
    for (int g = warp; g < Gp; g += nwarps)
      tile[g * 32 + lane] = (active && g < n) ? base[(long long)(g0 + g) * record_floats] : 0.f;
    __syncthreads();
    // up-sweep: tile[k*2d + 2d - 1] += tile[k*2d + d - 1]
    for (int d = 1; d < Gp; d <<= 1) {
      const int pairs = Gp / (2 * d);
      for (int i = warp; i < pairs; i += nwarps) {
        const int hi = (2 * i + 2) * d - 1, lo = (2 * i + 1) * d - 1;
        tile[hi * 32 + lane] += tile[lo * 32 + lane];
      }
      __syncthreads();
    }
    const float total = tile[(Gp - 1) * 32 + lane];
    __syncthreads();
    if (warp == 0) tile[(Gp - 1) * 32 + lane] = 0.f;
    __syncthreads();
    // down-sweep
    for (int d = Gp >> 1; d >= 1; d >>= 1) {
      const int pairs = Gp / (2 * d);
      for (int i = warp; i < pairs; i += nwarps) {
        const int hi = (2 * i + 2) * d - 1, lo = (2 * i + 1) * d - 1;
        const float t = tile[lo * 32 + lane];
        tile[lo * 32 + lane] = tile[hi * 32 + lane];
        tile[hi * 32 + lane] += t;
      }
      __syncthreads();
    }
    if (active)
      for (int g = warp; g < n; g += nwarps) base[(long long)(g0 + g) * record_floats] = carry + tile[g * 32 + lane];
    carry += total;
    __syncthreads();
  }
  if (active && warp == 0) {
    if (c < dv) {
      if (S_out) S_out[(bh * P + r) * dv + c] = carry;
    } else {
      if (z_out) z_out[bh * P + r] = carry;
    }
  }
}

cudaError_t launch_state_scan(float* ws, const ChunkPlan& plan, const float* S0, const float* z0, float* S_out,
                              float* z_out, cudaStream_t st) {
  int Gp = 1;
  while (Gp < plan.G && Gp < kScanBlock) Gp <<= 1;
  const size_t smem = (size_t)Gp * 32 * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(state_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const int E = plan.P * (plan.dv + 1);
  dim3 grid(ceil_div(E, 32), plan.BH);
  state_scan_kernel<<<grid, kScanThreads, smem, st>>>(ws, plan.G, plan.P, plan.dv, plan.ld,
                                                      (long long)plan.record_floats, S0, z0, S_out, z_out);
  return cudaGetLastError();
}

}  // namespace kata
