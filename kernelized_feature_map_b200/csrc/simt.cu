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
// acc[x][y] += a[x] * b[y] (fp32 FMA)
__device__ __forceinline__ void fma4x4(float (&acc)[4][4], const float4 a, const float4 b) {
  const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
  for (int x = 0; x < 4; ++x)
#pragma unroll
    for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(av[x], bv[y], acc[x][y]);
}

// Per super-chunk: A[r] = sum_t psi_r(k_t) [v_t | 1] over its tokens, as an
// fp32 record of P rows x LD columns ([S row | z | pad]).  A pass covers
// NB blocks of 64 state rows; a thread owns 4 rows x 4 record columns in each
// block (16 NB accumulators).  Tokens stream through shared memory AT at a
// time together with their psi values for the pass's rows, read as float4.
template <int p, int DV>
struct SimtAggLayout {
  static constexpr int LD = DV + 4;
  static constexpr int RB = 64;                          // rows per block
  static constexpr int NB = (p * p) / RB < 4 ? (p * p) / RB : 4;  // blocks per pass
  static constexpr int AT = 64;                          // tokens staged at a time
  static constexpr int offV = 0;                         // [AT][LD]
  static constexpr int offPsi = offV + AT * LD;          // [AT][NB * RB]
  static constexpr int offK = offPsi + AT * NB * RB;     // [AT][p+1]
  static constexpr int kFloats = offK + AT * (p + 1);
  static constexpr int NCG = LD / 4;
  static constexpr int kThreads = (RB / 4) * NCG;
};

template <typename Tin, int p, int DV>
__global__ void __launch_bounds__(SimtAggLayout<p, DV>::kThreads)
    chunk_aggregate_simt_kernel(const Tin* __restrict__ k, const Tin* __restrict__ v, float* __restrict__ ws, int T,
                                int Ls, int G, long long record_floats) {
  using L = SimtAggLayout<p, DV>;
  constexpr int P = p * p, LD = L::LD, RB = L::RB, NB = L::NB, AT = L::AT, NT = L::kThreads, NCG = L::NCG;
  constexpr int PQ = p + 1, ROWS = NB * RB;
  extern __shared__ __align__(16) float smem[];
  float* sv = smem + L::offV;
  float* sPsi = smem + L::offPsi;
  float* sk = smem + L::offK;
  const int tid = threadIdx.x;
  const int rr = 4 * (tid / NCG), c0 = 4 * (tid % NCG);
  const long long bh = blockIdx.y;
  const int g = blockIdx.x;
  const int ts = g * Ls, te = min(T, ts + Ls);
  const Tin* kb = k + bh * T * p;
  const Tin* vb = v + bh * T * DV;
  float* rec = ws + (bh * G + g) * record_floats;

  for (int r0 = 0; r0 < P; r0 += ROWS) {
    float acc[NB][4][4];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[b][x][y] = 0.f;
    for (int cs = ts; cs < te; cs += AT) {
      const int n = min(AT, te - cs);
      __syncthreads();
      for (int x = tid; x < AT * p; x += NT) {
        const int t = x / p, i = x % p;
        sk[t * PQ + i] = t < n ? Elem<Tin>::load(kb + (long long)(cs + t) * p + i) : 0.f;
      }
      for (int x = tid; x < AT * LD; x += NT) {
        const int t = x / LD, c = x % LD;
        float val = 0.f;
        if (t < n) val = c < DV ? Elem<Tin>::load(vb + (long long)(cs + t) * DV + c) : (c == DV ? 1.f : 0.f);
        sv[x] = val;
      }
      __syncthreads();
      for (int x = tid; x < AT * ROWS; x += NT) {
        const int t = x / ROWS, r = r0 + x % ROWS;
        sPsi[x] = sk[t * PQ + r / p] * sk[t * PQ + r % p];
      }
      __syncthreads();
      for (int t = 0; t < AT; ++t) {
        const float4 v4 = *reinterpret_cast<const float4*>(sv + t * LD + c0);
#pragma unroll
        for (int b = 0; b < NB; ++b)
          fma4x4(acc[b], *reinterpret_cast<const float4*>(sPsi + t * ROWS + b * RB + rr), v4);
      }
    }
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int x = 0; x < 4; ++x)
        *reinterpret_cast<float4*>(rec + (long long)(r0 + b * RB + rr + x) * LD + c0) =
            make_float4(acc[b][x][0], acc[b][x][1], acc[b][x][2], acc[b][x][3]);
  }
}

template <typename Tin, int p, int DV>
static cudaError_t launch_agg_t(const void* k, const void* v, float* ws, const ChunkPlan& pl, cudaStream_t st) {
  using L = SimtAggLayout<p, DV>;
  if (pl.ld != L::LD) return cudaErrorInvalidValue;
  const size_t smem = sizeof(float) * (size_t)L::kFloats;
  auto kern = chunk_aggregate_simt_kernel<Tin, p, DV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(pl.G, pl.BH);
  kern<<<grid, L::kThreads, smem, st>>>((const Tin*)k, (const Tin*)v, ws, pl.T, pl.Ls, pl.G,
                                        (long long)pl.record_floats);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// chunked form, step 3: readout and intra-chunk attention
// ---------------------------------------------------------------------------
// Shared-memory layout of the readout kernel (floats).  The arrays read as
// float4 come first, so that each starts on a 16-byte boundary.
template <int p, int DV, int C>
struct SimtRdLayout {
  static constexpr int LD = DV + 4;                 // record row stride: [S row | z | pad]
  static constexpr int RB = 64;                     // state rows per block
  static constexpr int offV = 0;                    // [C][LD]   v | 1 | 0
  static constexpr int offW = offV + C * LD;        // [C][C]    w(t, s) at [s][t]
  static constexpr int offPsi = offW + C * C;       // [RB][C] psi_r(q_t), or [C][RB] psi_r(k_s)
  static constexpr int offS = offPsi + RB * C;      // [RB][LD]  state block
  static constexpr int offO = offS + RB * LD;       // [C][LD]   [numerator | denominator]
  static constexpr int offQ = offO + C * LD;        // [C][p+1]  (row padding: no bank conflicts)
  static constexpr int offK = offQ + C * (p + 1);   // [C][p+1]
  static constexpr int kFloats = offK + C * (p + 1);
  static constexpr int NCG = LD / 4;                // 4-column groups per row
  static constexpr int kThreads = (C / 4) * NCG;    // one 4-token x 4-column tile per thread
};

// Per chunk of C tokens:
//   [O | D](t) = sum_{s <= t in the chunk} (q_t . k_s)^2 [v_s | 1]
//              + sum_r psi_r(q_t) S[r]                       (state entering the chunk)
//   o_t        = O / D
//   S[r]      += sum_s psi_r(k_s) [v_s | 1]                  (unless it is the last chunk)
// with S the fp32 record in the workspace (ABI psi index r = i*p + j).  Each
// thread owns a tile of 4 tokens x 4 record columns; the weights and psi
// values it needs are staged in shared memory and read as float4, so the
// inner loops do 16 FMA per two 16-byte shared loads.
template <typename Tin, int p, int DV, int C>
__global__ void __launch_bounds__(SimtRdLayout<p, DV, C>::kThreads)
    chunk_readout_simt_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                              Tin* __restrict__ o, float* __restrict__ ws, int T, int Ls, int G,
                              long long record_floats) {
  using L = SimtRdLayout<p, DV, C>;
  constexpr int P = p * p, LD = L::LD, RB = L::RB, NT = L::kThreads, NCG = L::NCG, PQ = p + 1;
  extern __shared__ __align__(16) float smem[];
  float* sv = smem + L::offV;
  float* sW = smem + L::offW;
  float* sPsi = smem + L::offPsi;
  float* sS = smem + L::offS;
  float* sO = smem + L::offO;
  float* sq = smem + L::offQ;
  float* sk = smem + L::offK;
  const int tid = threadIdx.x;
  const int t0 = 4 * (tid / NCG), c0 = 4 * (tid % NCG);
  const long long bh = blockIdx.y;
  const int g = blockIdx.x;
  const int ts = g * Ls, te = min(T, ts + Ls);
  const Tin* qb = q + bh * T * p;
  const Tin* kb = k + bh * T * p;
  const Tin* vb = v + bh * T * DV;
  float* rec = ws + (bh * G + g) * record_floats;  // state entering this super-chunk, advanced in place

  for (int cs = ts; cs < te; cs += C) {
    const int n = min(C, te - cs);
    __syncthreads();
    for (int x = tid; x < C * p; x += NT) {
      const int t = x / p, i = x % p;
      sq[t * PQ + i] = t < n ? Elem<Tin>::load(qb + (long long)(cs + t) * p + i) : 0.f;
      sk[t * PQ + i] = t < n ? Elem<Tin>::load(kb + (long long)(cs + t) * p + i) : 0.f;
    }
    for (int x = tid; x < C * LD; x += NT) {
      const int t = x / LD, c = x % LD;
      float val = 0.f;
      if (t < n) val = c < DV ? Elem<Tin>::load(vb + (long long)(cs + t) * DV + c) : (c == DV ? 1.f : 0.f);
      sv[x] = val;
    }
    __syncthreads();
    // intra-chunk weights w(t, s) = (q_t . k_s)^2 for s <= t, stored at [s][t]
    for (int x = tid; x < C * C; x += NT) {
      const int s = x / C, t = x % C;
      float w = 0.f;
      if (s <= t && t < n) {
        float dot = 0.f;
#pragma unroll
        for (int i = 0; i < p; ++i) dot = fmaf(sq[t * PQ + i], sk[s * PQ + i], dot);
        w = dot * dot;
      }
      sW[x] = w;
    }
    __syncthreads();
    float acc[4][4];
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int y = 0; y < 4; ++y) acc[x][y] = 0.f;
    for (int s = 0; s < C; ++s)
      fma4x4(acc, *reinterpret_cast<const float4*>(sW + s * C + t0), *reinterpret_cast<const float4*>(sv + s * LD + c0));
    // readout against the state entering the chunk, RB rows at a time
    for (int r0 = 0; r0 < P; r0 += RB) {
      __syncthreads();
      for (int x = tid; x < RB * C; x += NT) {
        const int r = r0 + x / C, t = x % C;
        sPsi[x] = sq[t * PQ + r / p] * sq[t * PQ + r % p];
      }
      for (int x = tid; x < RB * LD; x += NT) sS[x] = rec[(long long)(r0 + x / LD) * LD + x % LD];
      __syncthreads();
#pragma unroll 4
      for (int r = 0; r < RB; ++r)
        fma4x4(acc, *reinterpret_cast<const float4*>(sPsi + r * C + t0), *reinterpret_cast<const float4*>(sS + r * LD + c0));
    }
#pragma unroll
    for (int x = 0; x < 4; ++x)
      *reinterpret_cast<float4*>(sO + (t0 + x) * LD + c0) = make_float4(acc[x][0], acc[x][1], acc[x][2], acc[x][3]);
    __syncthreads();
    for (int x = tid; x < n * DV; x += NT) {
      const int t = x / DV, c = x % DV;
      const float D = sO[t * LD + DV];
      Elem<Tin>::store(o + (bh * T + cs + t) * DV + c, D > 0.f ? sO[t * LD + c] / D : 0.f);
    }
    if (cs + C >= te) break;  // the state after the last chunk is not needed
    // advance the state: S[r] += sum_s psi_r(k_s) [v_s | 1], RB rows at a time;
    // a thread owns 4 rows x 4 record columns of the block
    for (int r0 = 0; r0 < P; r0 += RB) {
      __syncthreads();
      for (int x = tid; x < C * RB; x += NT) {
        const int s = x / RB, r = r0 + x % RB;
        sPsi[x] = sk[s * PQ + r / p] * sk[s * PQ + r % p];
      }
      __syncthreads();
      if (tid < (RB / 4) * NCG) {
        const int rr = 4 * (tid / NCG);
        float a2[4][4];
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) a2[x][y] = 0.f;
        for (int s = 0; s < C; ++s)
          fma4x4(a2, *reinterpret_cast<const float4*>(sPsi + s * RB + rr), *reinterpret_cast<const float4*>(sv + s * LD + c0));
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          float4* dst = reinterpret_cast<float4*>(rec + (long long)(r0 + rr + x) * LD + c0);
          float4 cur = *dst;
          cur.x += a2[x][0];
          cur.y += a2[x][1];
          cur.z += a2[x][2];
          cur.w += a2[x][3];
          *dst = cur;
        }
      }
    }
  }
}

template <typename Tin, int p, int DV, int C>
static cudaError_t launch_rd_tc(const void* q, const void* k, const void* v, void* o, float* ws, const ChunkPlan& pl,
                                cudaStream_t st) {
  using L = SimtRdLayout<p, DV, C>;
  if (pl.ld != L::LD) return cudaErrorInvalidValue;
  const size_t smem = sizeof(float) * (size_t)L::kFloats;
  auto kern = chunk_readout_simt_kernel<Tin, p, DV, C>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(pl.G, pl.BH);
  kern<<<grid, L::kThreads, smem, st>>>((const Tin*)q, (const Tin*)k, (const Tin*)v, (Tin*)o, ws, pl.T, pl.Ls, pl.G,
                                        (long long)pl.record_floats);
  return cudaGetLastError();
}

template <typename Tin, int p, int DV>
static cudaError_t launch_rd_t(const void* q, const void* k, const void* v, void* o, float* ws, const ChunkPlan& pl,
                               cudaStream_t st) {
  if (pl.C == 64) return launch_rd_tc<Tin, p, DV, 64>(q, k, v, o, ws, pl, st);
  if (pl.C == 128) return launch_rd_tc<Tin, p, DV, 128>(q, k, v, o, ws, pl, st);
  return cudaErrorInvalidValue;
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
