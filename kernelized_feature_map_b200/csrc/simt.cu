// simt.cu -- CUDA-core kernels for fp32 inputs.
//
// Tensor cores on sm_100a take fp32 operands only as TF32 (10-bit mantissa),
// which cannot meet a 1e-4 relative error bound for fp32 inputs; these
// kernels do the same computation with exact fp32 FMA on the CUDA cores.
// They follow the same decomposition as the tensor-core path:
//
//   quadratic  causal squared-score attention, thread per query row, key and
//              value tiles staged in shared memory;
//   chunked    (1) per-super-chunk state sums psi(K)^T [V | 1],
//              (2) the shared associative scan (scan.cu),
//              (3) per chunk of C tokens: readout psi(Q_c) . S_prefix plus
//                  intra-chunk squared-score attention, then the state is
//                  advanced by the chunk's psi(K_c)^T [V_c | 1].
#include "kata_common.cuh"
#include "kata_internal.h"

namespace kata {

// ---------------------------------------------------------------------------
// quadratic form
// ---------------------------------------------------------------------------
constexpr int kQTile = 128;  // queries per CTA (one per thread)
constexpr int kKTile = 64;   // keys staged per step

template <typename Tin, int p, int DV>
__global__ void __launch_bounds__(kQTile) quadratic_simt_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                                                                const Tin* __restrict__ v, Tin* __restrict__ o,
                                                                int T) {
  __shared__ float sk[kKTile][p];
  __shared__ float sv[kKTile][DV];
  const long long bh = blockIdx.y;
  const int t = blockIdx.x * kQTile + threadIdx.x;
  const bool valid = t < T;
  const Tin* qb = q + bh * T * p;
  const Tin* kb = k + bh * T * p;
  const Tin* vb = v + bh * T * DV;

  float qr[p];
#pragma unroll
  for (int i = 0; i < p; ++i) qr[i] = valid ? Elem<Tin>::load(qb + (long long)t * p + i) : 0.f;
  float num[DV];
#pragma unroll
  for (int e = 0; e < DV; ++e) num[e] = 0.f;
  float den = 0.f;

  const int last = min(T, (int)(blockIdx.x + 1) * kQTile) - 1;
  for (int s0 = 0; s0 <= last; s0 += kKTile) {
    const int n = min(kKTile, T - s0);
    __syncthreads();
    for (int x = threadIdx.x; x < n * p; x += kQTile) sk[x / p][x % p] = Elem<Tin>::load(kb + (long long)s0 * p + x);
    for (int x = threadIdx.x; x < n * DV; x += kQTile)
      sv[x / DV][x % DV] = Elem<Tin>::load(vb + (long long)s0 * DV + x);
    __syncthreads();
    const int jmax = min(n, t - s0 + 1);  // causal: s <= t
    for (int j = 0; j < jmax; ++j) {
      float dot = 0.f;
#pragma unroll
      for (int i = 0; i < p; ++i) dot = fmaf(qr[i], sk[j][i], dot);
      const float w = dot * dot;
      den += w;
#pragma unroll
      for (int e = 0; e < DV; ++e) num[e] = fmaf(w, sv[j][e], num[e]);
    }
  }
  if (valid) {
    Tin* ob = o + (bh * T + t) * DV;
#pragma unroll
    for (int e = 0; e < DV; ++e) Elem<Tin>::store(ob + e, den > 0.f ? num[e] / den : 0.f);
  }
}

template <typename Tin, int p, int DV>
static cudaError_t launch_quad_t(const void* q, const void* k, const void* v, void* o, int BH, int T,
                                 cudaStream_t st) {
  dim3 grid(ceil_div(T, kQTile), BH);
  quadratic_simt_kernel<Tin, p, DV><<<grid, kQTile, 0, st>>>((const Tin*)q, (const Tin*)k, (const Tin*)v, (Tin*)o, T);
  return cudaGetLastError();
}

template <typename Tin>
static cudaError_t launch_quad_dt(const void* q, const void* k, const void* v, void* o, int BH, int T, int p, int dv,
                                  cudaStream_t st) {
  if (p == 16 && dv == 64) return launch_quad_t<Tin, 16, 64>(q, k, v, o, BH, T, st);
  if (p == 16 && dv == 16) return launch_quad_t<Tin, 16, 16>(q, k, v, o, BH, T, st);
  if (p == 32 && dv == 64) return launch_quad_t<Tin, 32, 64>(q, k, v, o, BH, T, st);
  if (p == 32 && dv == 16) return launch_quad_t<Tin, 32, 16>(q, k, v, o, BH, T, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_quadratic_simt(const void* q, const void* k, const void* v, void* o, int BH, int T, int p, int dv,
                                  kata_dtype_t dt, cudaStream_t st) {
  if (dt == KATA_BF16) return launch_quad_dt<__nv_bfloat16>(q, k, v, o, BH, T, p, dv, st);
  return launch_quad_dt<float>(q, k, v, o, BH, T, p, dv, st);
}

// ---------------------------------------------------------------------------
// chunked form, step 1: per-super-chunk state sums
// ---------------------------------------------------------------------------
constexpr int kAggThreads = 256;
constexpr int kAggPer = 16;      // state entries per thread per pass
constexpr int kAggTok = 64;      // tokens staged per step

template <typename Tin, int p, int DV>
__global__ void __launch_bounds__(kAggThreads) chunk_aggregate_simt_kernel(const Tin* __restrict__ k,
                                                                           const Tin* __restrict__ v,
                                                                           float* __restrict__ ws, int T, int Ls,
                                                                           int G, int ld, long long record_floats) {
  constexpr int P = p * p;
  constexpr int E = P * (DV + 1);
  __shared__ float sk[kAggTok][p];
  __shared__ float sv[kAggTok][DV + 1];
  const long long bh = blockIdx.y;
  const int g = blockIdx.x;
  const int t0 = g * Ls, t1 = min(T, t0 + Ls);
  const Tin* kb = k + bh * T * p;
  const Tin* vb = v + bh * T * DV;
  float* rec = ws + (bh * G + g) * record_floats;

  for (int e0 = 0; e0 < E; e0 += kAggThreads * kAggPer) {
    float acc[kAggPer];
#pragma unroll
    for (int i = 0; i < kAggPer; ++i) acc[i] = 0.f;
    for (int s0 = t0; s0 < t1; s0 += kAggTok) {
      const int n = min(kAggTok, t1 - s0);
      __syncthreads();
      for (int x = threadIdx.x; x < n * p; x += kAggThreads) sk[x / p][x % p] = Elem<Tin>::load(kb + (long long)s0 * p + x);
      for (int x = threadIdx.x; x < n * DV; x += kAggThreads)
        sv[x / DV][x % DV] = Elem<Tin>::load(vb + (long long)s0 * DV + x);
      for (int x = threadIdx.x; x < n; x += kAggThreads) sv[x][DV] = 1.f;
      __syncthreads();
#pragma unroll
      for (int i = 0; i < kAggPer; ++i) {
        const int e = e0 + i * kAggThreads + threadIdx.x;
        if (e < E) {
          const int r = e / (DV + 1), c = e % (DV + 1);
          const int ii = r / p, jj = r % p;
          float a = acc[i];
          for (int j = 0; j < n; ++j) a = fmaf(sk[j][ii] * sk[j][jj], sv[j][c], a);
          acc[i] = a;
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kAggPer; ++i) {
      const int e = e0 + i * kAggThreads + threadIdx.x;
      if (e < E) rec[(e / (DV + 1)) * ld + e % (DV + 1)] = acc[i];
    }
  }
}

template <typename Tin, int p, int DV>
static cudaError_t launch_agg_t(const void* k, const void* v, float* ws, const ChunkPlan& pl, cudaStream_t st) {
  dim3 grid(pl.G, pl.BH);
  chunk_aggregate_simt_kernel<Tin, p, DV><<<grid, kAggThreads, 0, st>>>(
      (const Tin*)k, (const Tin*)v, ws, pl.T, pl.Ls, pl.G, pl.ld, (long long)pl.record_floats);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// chunked form, step 3: readout and intra-chunk attention
// ---------------------------------------------------------------------------
constexpr int kRdThreads = 256;

template <typename Tin, int p, int DV>
__global__ void __launch_bounds__(kRdThreads) chunk_readout_simt_kernel(const Tin* __restrict__ q,
                                                                        const Tin* __restrict__ k,
                                                                        const Tin* __restrict__ v,
                                                                        Tin* __restrict__ o, float* __restrict__ ws,
                                                                        int T, int C, int Ls, int G, int ld,
                                                                        long long record_floats) {
  constexpr int P = p * p;
  constexpr int NC = DV + 1;
  extern __shared__ float smem[];
  float* sq = smem;                 // [C][p]
  float* sk = sq + C * p;           // [C][p]
  float* sv = sk + C * p;           // [C][NC], column DV = 1
  float* so = sv + C * NC;          // [C][NC]
  const long long bh = blockIdx.y;
  const int g = blockIdx.x;
  const int t0 = g * Ls, t1 = min(T, t0 + Ls);
  const Tin* qb = q + bh * T * p;
  const Tin* kb = k + bh * T * p;
  const Tin* vb = v + bh * T * DV;
  float* rec = ws + (bh * G + g) * record_floats;  // state entering this super-chunk, advanced in place

  for (int c0 = t0; c0 < t1; c0 += C) {
    const int n = min(C, t1 - c0);
    __syncthreads();
    for (int x = threadIdx.x; x < n * p; x += kRdThreads) {
      sq[x] = Elem<Tin>::load(qb + (long long)c0 * p + x);
      sk[x] = Elem<Tin>::load(kb + (long long)c0 * p + x);
    }
    for (int x = threadIdx.x; x < n * DV; x += kRdThreads) sv[(x / DV) * NC + x % DV] = Elem<Tin>::load(vb + (long long)c0 * DV + x);
    for (int x = threadIdx.x; x < n; x += kRdThreads) sv[x * NC + DV] = 1.f;
    __syncthreads();
    // readout against the state entering the chunk, plus intra-chunk terms
    for (int x = threadIdx.x; x < n * NC; x += kRdThreads) {
      const int t = x / NC, c = x % NC;
      const float* qt = sq + t * p;
      float acc = 0.f;
      for (int ii = 0; ii < p; ++ii) {
        float part = 0.f;
        for (int jj = 0; jj < p; ++jj) part = fmaf(qt[jj], rec[(ii * p + jj) * ld + c], part);
        acc = fmaf(qt[ii], part, acc);
      }
      for (int s = 0; s <= t; ++s) {
        float dot = 0.f;
#pragma unroll
        for (int i = 0; i < p; ++i) dot = fmaf(qt[i], sk[s * p + i], dot);
        acc = fmaf(dot * dot, sv[s * NC + c], acc);
      }
      so[x] = acc;
    }
    __syncthreads();
    for (int x = threadIdx.x; x < n * DV; x += kRdThreads) {
      const int t = x / DV, c = x % DV;
      const float D = so[t * NC + DV];
      Elem<Tin>::store(o + (bh * T + c0 + t) * DV + c, D > 0.f ? so[t * NC + c] / D : 0.f);
    }
    // advance the state by this chunk: S += psi(K_c)^T [V_c | 1]
    for (int e = threadIdx.x; e < P * NC; e += kRdThreads) {
      const int r = e / NC, c = e % NC;
      const int ii = r / p, jj = r % p;
      float a = 0.f;
      for (int s = 0; s < n; ++s) a = fmaf(sk[s * p + ii] * sk[s * p + jj], sv[s * NC + c], a);
      rec[r * ld + c] += a;
    }
  }
}

template <typename Tin, int p, int DV>
static cudaError_t launch_rd_t(const void* q, const void* k, const void* v, void* o, float* ws, const ChunkPlan& pl,
                               cudaStream_t st) {
  const size_t smem = sizeof(float) * ((size_t)pl.C * p * 2 + (size_t)pl.C * (DV + 1) * 2);
  auto kern = chunk_readout_simt_kernel<Tin, p, DV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(pl.G, pl.BH);
  kern<<<grid, kRdThreads, smem, st>>>((const Tin*)q, (const Tin*)k, (const Tin*)v, (Tin*)o, ws, pl.T, pl.C, pl.Ls,
                                       pl.G, pl.ld, (long long)pl.record_floats);
  return cudaGetLastError();
}

#define KATA_DISPATCH_PDV(FN, ...)                                              \
  do {                                                                          \
    if (pl.p == 16 && pl.dv == 64) return FN<Tin, 16, 64>(__VA_ARGS__);         \
    if (pl.p == 16 && pl.dv == 16) return FN<Tin, 16, 16>(__VA_ARGS__);         \
    if (pl.p == 32 && pl.dv == 64) return FN<Tin, 32, 64>(__VA_ARGS__);         \
    if (pl.p == 32 && pl.dv == 16) return FN<Tin, 32, 16>(__VA_ARGS__);         \
    return cudaErrorInvalidValue;                                               \
  } while (0)

template <typename Tin>
static cudaError_t agg_dt(const void* k, const void* v, float* ws, const ChunkPlan& pl, cudaStream_t st) {
  KATA_DISPATCH_PDV(launch_agg_t, k, v, ws, pl, st);
}
template <typename Tin>
static cudaError_t rd_dt(const void* q, const void* k, const void* v, void* o, float* ws, const ChunkPlan& pl,
                         cudaStream_t st) {
  KATA_DISPATCH_PDV(launch_rd_t, q, k, v, o, ws, pl, st);
}

cudaError_t launch_chunk_aggregate_simt(const void* k, const void* v, float* ws, const ChunkPlan& plan,
                                        kata_dtype_t dt, cudaStream_t st) {
  if (dt == KATA_BF16) return agg_dt<__nv_bfloat16>(k, v, ws, plan, st);
  return agg_dt<float>(k, v, ws, plan, st);
}

cudaError_t launch_chunk_readout_simt(const void* q, const void* k, const void* v, void* o, float* ws,
                                      const ChunkPlan& plan, kata_dtype_t dt, cudaStream_t st) {
  if (dt == KATA_BF16) return rd_dt<__nv_bfloat16>(q, k, v, o, ws, plan, st);
  return rd_dt<float>(q, k, v, o, ws, plan, st);
}

}  // namespace kata
