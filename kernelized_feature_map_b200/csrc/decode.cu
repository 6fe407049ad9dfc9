// decode.cu -- one recurrent decode step on the fixed-size state.
//
//   S <- S + psi(k) v^T,  z <- z + psi(k),  o = psi(q)^T S / psi(q)^T z
//
// (constant-time recurrent inference on the state, arXiv abstract; the
// state recurrence of the ai.info summary, Methodology in Plain English.)
//
// The step is bound by HBM: every (b,h) streams its p^2 x dv fp32 state in
// and out once (2 * 64 KiB at p = 16, dv = 64).  One CTA per (b,h) (128 or
// 256 threads, see DecodeCfg).  Thread layout: DV/4 consecutive threads
// cover one state row with 16-byte vectors, so each pass of the CTA reads
// one 16-byte vector per thread, contiguous across the CTA; all of a batch's loads are issued before any use so that enough
// bytes are in flight per SM.  The first batch of state rows and the
// normaliser entries are requested before q, k and v are staged, since they
// do not depend on them, so their latency overlaps.  Loads and stores carry
// the streaming hint (the state is touched once per step).  psi(k)_r and psi(q)_r for the row
// r = i*p + j are formed on the fly from the p values staged in shared
// memory.  The numerator is reduced over rows through shared memory.
//
// KATA-Mg (G factors of width p per head, q and k rows of d = G*p values):
// the feature is the concatenation of the G group maps, so the state has
// G*p*p rows and row r = g*p*p + i*p + j holds the products of coordinates
// g*p + i and g*p + j; G = 1 is the single-factor step above.
// KATA-Sigma-g (SUM): the feature is the sum of the G group maps, so the
// state has the single factor's p*p rows and row r = i*p + j holds
// sum_g u_{g*p+i} u_{g*p+j} (gist.science sec. 2.3 "Varianten"; ai.info Main
// Findings, the Sigma-g state (d/g)(d/g+1)/2 * dv, here unpacked).
#include "kata_common.cuh"
#include "kata_internal.h"

namespace kata {

// Threads per CTA, batch of state loads per thread, and CTAs per SM.  A
// small state (64 KiB per stream for the p = 16 single factor) runs on
// 128-thread CTAs in batches of 8 loads per thread, seven CTAs per SM: the
// 1024 streams of a B = 64, H = 16 step are then resident in one wave, each
// SM keeping ~110 KiB of loads in flight, instead of three and a half waves
// of two 256-thread CTAs with a tail.  Larger states (p = 32, KATA-Mg)
// stream long enough per CTA with 256 threads and 16-deep batches.
// Measured at B = 64, H = 16 (p = 16, dv = 64): 33 us with 256-thread CTAs
// and 16-deep batches, 28.8 us in this configuration; double-buffering the
// batches (next batch's loads issued before the current one is stored)
// measured 29.7 us and is not used.
template <int P, int DV>
struct DecodeCfg {
  static constexpr bool kSmall = P * DV <= 256 * 64;
  static constexpr int kThreads = kSmall ? 128 : 256;
  static constexpr int kBatchMax = kSmall ? 8 : 16;
  static constexpr bool kPipe = false;
  static constexpr int kMinBlocks = kSmall ? 7 : 1;
};

template <int p, int G, bool SUM>
constexpr int decode_rows() { return SUM ? p * p : G * p * p; }

// psi_r(u) for state row r of the concatenated (Mg) or summed (Sigma-g)
// feature, from the row u staged in shared memory
template <int p, int G, bool SUM>
__device__ __forceinline__ float decode_feature(const float* u, int r) {
  if constexpr (SUM) {
    const int i = r / p, j = r % p;
    float f = 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g) f = fmaf(u[g * p + i], u[g * p + j], f);
    return f;
  } else {
    const int gp = (r / (p * p)) * p, ii = gp + (r % (p * p)) / p, jj = gp + r % p;
    return u[ii] * u[jj];
  }
}

template <typename Tin, int p, int DV, int G, bool SUM>
__global__ void __launch_bounds__((DecodeCfg<decode_rows<p, G, SUM>(), DV>::kThreads),
                                  (DecodeCfg<decode_rows<p, G, SUM>(), DV>::kMinBlocks))
    decode_step_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                       Tin* __restrict__ o, float* __restrict__ S, float* __restrict__ z) {
  constexpr int D = G * p;                       // q/k row width
  constexpr int P = decode_rows<p, G, SUM>();    // state rows
  constexpr int NT = DecodeCfg<P, DV>::kThreads;
  constexpr int CG = DV / 4;        // 16-byte column groups per state row
  constexpr int RPP = NT / CG;      // rows covered by one pass of the CTA
  constexpr int PASSES = P / RPP;   // passes over the state
  constexpr int BMAX = DecodeCfg<P, DV>::kBatchMax;
  constexpr int BATCH = PASSES < BMAX ? PASSES : BMAX;
  static_assert(PASSES % BATCH == 0, "pass batching");
  static_assert(D <= NT && DV <= NT, "q, k and v are staged by one thread per value");

  __shared__ float sq[D], sk[D], sv[DV];
  __shared__ float4 red[NT];
  __shared__ float sden[NT / 32];

  constexpr int ZPT = (P + NT - 1) / NT;  // normaliser entries per thread
  const int tid = threadIdx.x;
  const long long bh = blockIdx.x;
  const int cg = tid % CG;
  const int r0 = tid / CG;
  float4* Sb = reinterpret_cast<float4*>(S + bh * (long long)P * DV);
  float* zb = z + bh * P;
  float4 s[BATCH];
#pragma unroll
  for (int i = 0; i < BATCH; ++i) s[i] = __ldcs(Sb + (r0 + i * RPP) * CG + cg);
  float zz[ZPT];
#pragma unroll
  for (int u = 0; u < ZPT; ++u) zz[u] = (tid + NT * u < P) ? __ldcs(zb + tid + NT * u) : 0.f;
  if (tid < D) {
    sq[tid] = Elem<Tin>::load(q + bh * D + tid);
    sk[tid] = Elem<Tin>::load(k + bh * D + tid);
  }
  if (tid < DV) sv[tid] = Elem<Tin>::load(v + bh * DV + tid);
  __syncthreads();

  const float4 vv = make_float4(sv[4 * cg], sv[4 * cg + 1], sv[4 * cg + 2], sv[4 * cg + 3]);

  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
  for (int b0 = 0; b0 < PASSES; b0 += BATCH) {
    float4 nx[DecodeCfg<P, DV>::kPipe ? BATCH : 1];
    if constexpr (DecodeCfg<P, DV>::kPipe) {
      if (b0 + BATCH < PASSES) {
#pragma unroll
        for (int i = 0; i < BATCH; ++i) nx[i] = __ldcs(Sb + (r0 + (b0 + BATCH + i) * RPP) * CG + cg);
      }
    } else if (b0 > 0) {
#pragma unroll
      for (int i = 0; i < BATCH; ++i) s[i] = __ldcs(Sb + (r0 + (b0 + i) * RPP) * CG + cg);
    }
#pragma unroll
    for (int i = 0; i < BATCH; ++i) {
      const int r = r0 + (b0 + i) * RPP;
      const float pk = decode_feature<p, G, SUM>(sk, r);
      const float pq = decode_feature<p, G, SUM>(sq, r);
      s[i].x = fmaf(pk, vv.x, s[i].x);
      s[i].y = fmaf(pk, vv.y, s[i].y);
      s[i].z = fmaf(pk, vv.z, s[i].z);
      s[i].w = fmaf(pk, vv.w, s[i].w);
      __stcs(Sb + r * CG + cg, s[i]);
      acc.x = fmaf(pq, s[i].x, acc.x);
      acc.y = fmaf(pq, s[i].y, acc.y);
      acc.z = fmaf(pq, s[i].z, acc.z);
      acc.w = fmaf(pq, s[i].w, acc.w);
    }
    if constexpr (DecodeCfg<P, DV>::kPipe) {
#pragma unroll
      for (int i = 0; i < BATCH; ++i) s[i] = nx[i];
    }
  }

  // normaliser z and the denominator psi(q)^T z
  float den = 0.f;
#pragma unroll
  for (int u = 0; u < ZPT; ++u) {
    const int r = tid + NT * u;
    if (r < P) {
      const float zn = zz[u] + decode_feature<p, G, SUM>(sk, r);
      __stcs(zb + r, zn);
      den = fmaf(decode_feature<p, G, SUM>(sq, r), zn, den);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
  if ((tid & 31) == 0) sden[tid >> 5] = den;
  red[tid] = acc;
  __syncthreads();

  if (tid < DV) {
    float D = 0.f;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) D += sden[w];
    const int c4 = tid / 4, comp = tid % 4;
    float num = 0.f;
#pragma unroll 4
    for (int j = 0; j < RPP; ++j) {
      const float4 x = red[j * CG + c4];
      num += comp == 0 ? x.x : comp == 1 ? x.y : comp == 2 ? x.z : x.w;
    }
    Elem<Tin>::store(o + bh * DV + tid, D > 0.f ? num / D : 0.f);
  }
}

template <typename Tin, int p, int DV, int G, bool SUM = false>
static cudaError_t launch_decode_t(const void* q, const void* k, const void* v, void* o, float* S, float* z,
                                   int BH, cudaStream_t st) {
  decode_step_kernel<Tin, p, DV, G, SUM><<<BH, DecodeCfg<decode_rows<p, G, SUM>(), DV>::kThreads, 0, st>>>(
      (const Tin*)q, (const Tin*)k, (const Tin*)v, (Tin*)o, S, z);
  return cudaGetLastError();
}

template <typename Tin>
static cudaError_t launch_decode_dt(const void* q, const void* k, const void* v, void* o, float* S, float* z,
                                    int BH, int p, int groups, int dv, cudaStream_t st) {
  if (groups == 1) {
    if (p == 16 && dv == 64) return launch_decode_t<Tin, 16, 64, 1>(q, k, v, o, S, z, BH, st);
    if (p == 16 && dv == 16) return launch_decode_t<Tin, 16, 16, 1>(q, k, v, o, S, z, BH, st);
    if (p == 32 && dv == 64) return launch_decode_t<Tin, 32, 64, 1>(q, k, v, o, S, z, BH, st);
    if (p == 32 && dv == 16) return launch_decode_t<Tin, 32, 16, 1>(q, k, v, o, S, z, BH, st);
  } else if (dv == 64) {
    if (p == 16 && groups == 2) return launch_decode_t<Tin, 16, 64, 2>(q, k, v, o, S, z, BH, st);
    if (p == 16 && groups == 4) return launch_decode_t<Tin, 16, 64, 4>(q, k, v, o, S, z, BH, st);
    if (p == 32 && groups == 2) return launch_decode_t<Tin, 32, 64, 2>(q, k, v, o, S, z, BH, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode(const void* q, const void* k, const void* v, void* o, float* S, float* z, int BH,
                          int p, int groups, int dv, kata_dtype_t dt, cudaStream_t st) {
  if (dt == KATA_BF16) return launch_decode_dt<__nv_bfloat16>(q, k, v, o, S, z, BH, p, groups, dv, st);
  return launch_decode_dt<float>(q, k, v, o, S, z, BH, p, groups, dv, st);
}

template <typename Tin>
static cudaError_t launch_decode_sg_dt(const void* q, const void* k, const void* v, void* o, float* S, float* z,
                                       int BH, int p, int groups, int dv, cudaStream_t st) {
  if (dv == 64) {
    if (p == 16 && groups == 2) return launch_decode_t<Tin, 16, 64, 2, true>(q, k, v, o, S, z, BH, st);
    if (p == 16 && groups == 4) return launch_decode_t<Tin, 16, 64, 4, true>(q, k, v, o, S, z, BH, st);
    if (p == 32 && groups == 2) return launch_decode_t<Tin, 32, 64, 2, true>(q, k, v, o, S, z, BH, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode_sg(const void* q, const void* k, const void* v, void* o, float* S, float* z, int BH,
                             int p, int groups, int dv, kata_dtype_t dt, cudaStream_t st) {
  if (dt == KATA_BF16) return launch_decode_sg_dt<__nv_bfloat16>(q, k, v, o, S, z, BH, p, groups, dv, st);
  return launch_decode_sg_dt<float>(q, k, v, o, S, z, BH, p, groups, dv, st);
}

}  // namespace kata
