// flash_bwd_sm100.cu -- backward pass of the quadratic (flash-style) KATA
// forward on tcgen05 / TMEM (bf16 inputs, fp32 accumulation, dv = 64).
//
// For one (b,h): S_ts = q_t . k_s, w_ts = S_ts^2 (s <= t), o_t = N_t / D_t
// with N_t = sum_s w_ts v_s and D_t = sum_s w_ts (gist.science technical
// summary, sec. 2.1 "Output Gating" and sec. 2.2 "PSD Kegel (Rank-One)").
// Given dO, the chain rule through o = N / D gives
//   dN_t  = dO_t / D_t,   dD_t = -(dO_t . o_t) / D_t    (0 where D_t = 0)
//   dS_ts = 2 S_ts (dN_t . v_s + dD_t)                    (s <= t)
//   dv_s  = sum_{t>=s} w_ts dN_t
//   dq_t  = sum_{s<=t} dS_ts k_s,   dk_s = sum_{t>=s} dS_ts q_t
// evaluated as dS_ts = (S_ts r_t) (dO_t . v_s - delta_t) and
// dv_s = 1/2 sum_t (S_ts^2 r_t) dO_t with r_t = 2 / D_t and delta_t = dO_t . o_t:
// the tensor core multiplies dO itself (exact bf16 input), and the
// difference dO.v - dO.o, which cancels when the row's weight sits on few
// keys, is taken in fp32 before the 1 / D scaling.  (Rounding dN = dO / D to
// bf16 first turns that cancellation into errors of order 2^-9 |dO||v| / D,
// which dominate the gradient when some D_t is small.)
// (the pages print no backward pass; they say the kernels are competitive
// on the training step, arXiv abstract).  D comes from the forward
// (kata_fwd_quadratic_train).  Three launches:
//   1. bwd_rows_kernel   (-delta_t, r_t) per row, eight lanes per row;
//   2. bwd_dq_kernel     persistent, items of one 128-row query tile: per key tile j,
//                        S = Q K_j^T and dP = dO V_j^T on the tensor core,
//                        dS in the weight warps, then
//                        dQ += dS K_j with dS read from TMEM;
//   3. bwd_dkdv_kernel   persistent, items of one 128-row key tile: per query tile i,
//                        S^T = K Q_i^T and dP^T = V dO_i^T, W^T = (S^T)^2 r / 2 and
//                        dS^T in the weight warps, then dV += W^T dO_i and
//                        dK += dS^T Q_i.
// Both main kernels keep the products in TMEM with keys (dQ) or queries
// (dK, dV) along the reduction dimension, so every MMA's A operand comes
// from TMEM in the K-major form tcgen05 requires and every B operand is a
// TMA tile read K-major or MN-major as loaded.  The next tile's S and dP are
// issued as soon as the weight warps have loaded the current ones.
// Warps: 0 TMA, 1 MMA (converged, elected lane), 2-17 sixteen weight warps
// (TMEM lane quarter x 32-column quarter).  Every wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>

#include "kata_internal.h"
#include "kata_trace.cuh"
#include "sm100.cuh"

KATA_TRACE_DECLARE(bwd)

namespace kata {

bool make_tmap_bf16(CUtensorMap* map, const void* base, int inner, int T, int BH, int rows);

// 3-D bf16 tensor map over rows of `inner` values that start ld values apart
// ([B*H][T][ld], e.g. one group's columns of a [B*H, T, d] tensor), box
// {inner, rows, 1}, swizzled over the box row.
static bool make_tmap_bf16_ld(CUtensorMap* map, const void* base, int inner, int ld, int T, int BH, int rows) {
  typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                               const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                               CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
  static EncodeFn enc = nullptr;
  if (!enc) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qr) != cudaSuccess ||
        qr != cudaDriverEntryPointSuccess)
      return false;
    enc = reinterpret_cast<EncodeFn>(fn);
  }
  const int box_bytes = inner * 2;
  const CUtensorMapSwizzle sw = box_bytes == 32   ? CU_TENSOR_MAP_SWIZZLE_32B
                                : box_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                  : CU_TENSOR_MAP_SWIZZLE_128B;
  const cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)T, (cuuint64_t)BH};
  const cuuint64_t strides[2] = {(cuuint64_t)ld * 2, (cuuint64_t)ld * 2 * (cuuint64_t)T};
  const cuuint32_t box[3] = {(cuuint32_t)inner, (cuuint32_t)rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

using namespace sm100;

constexpr int kBw = 128;          // rows per tile (queries or keys)
constexpr int kBwDV = 64;
constexpr int kBwThreads = 576;
constexpr int kBwStages = 4;
constexpr uint32_t kBwTmemCols = 512;

// ---------------------------------------------------------------------------
// 1. Per row: (-delta_t, r_t) with delta_t = dO_t . o_t and r_t = 2 / D_t, both
//    fp32 (the factor 2 of dS is folded into r; the dV accumulator, which
//    gets it too, is halved in its epilogue -- exact); a row with D_t = 0
//    (output constant 0) gets r_t = 0, so it passes no gradient.  Eight
//    lanes per row of 64 values (16 bytes of dO and of o each), 16 rows per
//    warp with all their loads issued before the first use, so that enough
//    bytes are in flight to stream dO and o at the HBM rate (one warp per
//    row, two values a lane: 290 us for B1 H16 T131072 under ncu).
// ---------------------------------------------------------------------------
constexpr int kRowsPerWarp = 16;
constexpr int kRowsPerBlock = 8 * kRowsPerWarp;

__global__ void __launch_bounds__(256) bwd_rows_kernel(const __nv_bfloat16* __restrict__ dO,
                                                       const __nv_bfloat16* __restrict__ o,
                                                       const float* __restrict__ D, float2* __restrict__ rowc,
                                                       long long rows) {
  const int lane = threadIdx.x & 31, part = lane & 7, sub = lane >> 3;
  const long long base = (long long)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5) * kRowsPerWarp + sub;
  constexpr int kPass = kRowsPerWarp / 4;
  uint4 a[kPass], b[kPass];
#pragma unroll
  for (int j = 0; j < kPass; ++j) {
    const long long row = base + 4 * j;
    a[j] = b[j] = make_uint4(0u, 0u, 0u, 0u);
    if (row < rows) {
      a[j] = __ldcs(reinterpret_cast<const uint4*>(dO + row * kBwDV) + part);
      b[j] = __ldcs(reinterpret_cast<const uint4*>(o + row * kBwDV) + part);
    }
  }
#pragma unroll
  for (int j = 0; j < kPass; ++j) {
    const long long row = base + 4 * j;
    const uint32_t* x = reinterpret_cast<const uint32_t*>(&a[j]);
    const uint32_t* y = reinterpret_cast<const uint32_t*>(&b[j]);
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      dot = fmaf(__uint_as_float(x[e] << 16), __uint_as_float(y[e] << 16), dot);
      dot = fmaf(__uint_as_float(x[e] & 0xffff0000u), __uint_as_float(y[e] & 0xffff0000u), dot);
    }
    // the 8 lanes of the row (xor offsets below 8 stay inside the group)
#pragma unroll
    for (int off = 4; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
    if (part == 0 && row < rows) {
      const float d = D[row];
      rowc[row] = make_float2(-dot, d > 0.f ? 2.f / d : 0.f);
    }
  }
}

template <int p>
struct BwCfg {
  static constexpr int kQKBytes = kBw * p * 2;         // a Q or K tile
  static constexpr int kVBytes = kBw * kBwDV * 2;      // a V or dO tile
  static constexpr Swizzle kQKSw = p == 16 ? kSw32 : kSw64;
  // 8-row group stride: K-major rows of the Q/K tile, or 8 reduction rows
  // when the same tile is read MN-major
  static constexpr uint32_t kQKSbo = 8 * p * 2;
  static constexpr uint32_t kVSbo = 8 * kBwDV * 2;
  static constexpr uint32_t kQKKStep = 16 * p * 2;     // 16 rows of a Q/K tile read MN-major
  static constexpr uint32_t kVKStep = 16 * kBwDV * 2;  // 16 rows of a V/dO tile read MN-major
  // TMEM columns
  static constexpr uint32_t colS = 0;                  // S or S^T, fp32
  static constexpr uint32_t colP = 128;                // dP or dP^T, fp32
  static constexpr uint32_t colA(int b) { return 256u + 64u * (uint32_t)b; }  // bf16 operands (2 x 64)
  static constexpr uint32_t colAcc = 384;              // dQ (p) or dV (64) then dK (p)
};

// Gradient weights (and, with kW, scaled squares) of 16 columns of one row,
// half HF of the row's 32, on fp32 pairs: s, d are the 16 scores and dP
// values; the row constants (-delta, r) of column c are rc for every column,
// or, with kCol, cc[x] = (-delta, r of column 2x, -delta, r of column 2x + 1).
// g[8 HF + x] receives the bf16 pair of dS = (s r) (dP - delta) for
// columns 2x, 2x + 1, w[8 HF + x] that of s (s r) (with r = 2 / D: twice the
// weight the dV product needs).  With kMask, column c
// (0..31 in the row's 32) is kept only when kGE ? c >= lane : c <= lane.
template <int HF, bool kW, bool kCol, bool kMask, bool kGE>
__device__ __forceinline__ void grad_pairs(const uint32_t (&s)[16], const uint32_t (&d)[16], const float4* cc,
                                           float2 rc, int lane, uint32_t (&g)[16], uint32_t (&w)[16]) {
#pragma unroll
  for (int x = 0; x < 8; ++x) {
    const float4 e = kCol ? cc[x] : make_float4(rc.x, rc.y, rc.x, rc.y);
    const uint64_t s2 = f32x2(s[2 * x], s[2 * x + 1]);
    const uint64_t t = f32x2_add(f32x2(d[2 * x], d[2 * x + 1]), f32x2(__float_as_uint(e.x), __float_as_uint(e.z)));
    const uint64_t u = f32x2_mul(s2, f32x2(__float_as_uint(e.y), __float_as_uint(e.w)));
    const uint64_t gg = f32x2_mul(u, t);
    float g0 = f32x2_lo(gg), g1 = f32x2_hi(gg);
    if (kMask) {
      const int c = 16 * HF + 2 * x;
      if (kGE ? c < lane : c > lane) g0 = 0.f;
      if (kGE ? c + 1 < lane : c + 1 > lane) g1 = 0.f;
    }
    g[8 * HF + x] = pack_bf16x2(g0, g1);
    if (kW) {
      const uint64_t ww = f32x2_mul(s2, u);
      float w0 = f32x2_lo(ww), w1 = f32x2_hi(ww);
      if (kMask) {
        const int c = 16 * HF + 2 * x;
        if (kGE ? c < lane : c > lane) w0 = 0.f;
        if (kGE ? c + 1 < lane : c + 1 > lane) w1 = 0.f;
      }
      w[8 * HF + x] = pack_bf16x2(w0, w1);
    }
  }
}

// 16 fp32 values -> 16 bf16 at dst (32 bytes, 16-byte aligned)
// The 16 bf16 values at src_row added into the fp32 row r (bf16 -> fp32 is
// a 16-bit shift, exact): for a gradient another pass has already written
// part of (KATA-Mg's dV; KATA-Sigma-g's dQ, dK and dV).
__device__ __forceinline__ void add_row16(const __nv_bfloat16* src_row, uint32_t (&r)[16]) {
  const uint4* old = reinterpret_cast<const uint4*>(src_row);
  const uint4 a = old[0], b = old[1];
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int x = 0; x < 8; ++x) {
    r[2 * x] = __float_as_uint(__uint_as_float(r[2 * x]) + __uint_as_float(w[x] << 16));
    r[2 * x + 1] = __float_as_uint(__uint_as_float(r[2 * x + 1]) + __uint_as_float(w[x] & 0xffff0000u));
  }
}

// The same, from the two 16-byte words of the row loaded earlier.
__device__ __forceinline__ void add_row16_words(const uint4 (&old)[2], uint32_t (&r)[16]) {
  const uint32_t w[8] = {old[0].x, old[0].y, old[0].z, old[0].w, old[1].x, old[1].y, old[1].z, old[1].w};
#pragma unroll
  for (int x = 0; x < 8; ++x) {
    r[2 * x] = __float_as_uint(__uint_as_float(r[2 * x]) + __uint_as_float(w[x] << 16));
    r[2 * x + 1] = __float_as_uint(__uint_as_float(r[2 * x + 1]) + __uint_as_float(w[x] & 0xffff0000u));
  }
}

__device__ __forceinline__ void load_row16_words(const __nv_bfloat16* src_row, uint4 (&old)[2]) {
  const uint4* src = reinterpret_cast<const uint4*>(src_row);
  old[0] = src[0];
  old[1] = src[1];
}

__device__ __forceinline__ void store_row16(__nv_bfloat16* dst_row, const uint32_t (&r)[16]) {
  uint4* dst = reinterpret_cast<uint4*>(dst_row);
  dst[0] = make_uint4(pack_bf16x2(__uint_as_float(r[0]), __uint_as_float(r[1])),
                      pack_bf16x2(__uint_as_float(r[2]), __uint_as_float(r[3])),
                      pack_bf16x2(__uint_as_float(r[4]), __uint_as_float(r[5])),
                      pack_bf16x2(__uint_as_float(r[6]), __uint_as_float(r[7])));
  dst[1] = make_uint4(pack_bf16x2(__uint_as_float(r[8]), __uint_as_float(r[9])),
                      pack_bf16x2(__uint_as_float(r[10]), __uint_as_float(r[11])),
                      pack_bf16x2(__uint_as_float(r[12]), __uint_as_float(r[13])),
                      pack_bf16x2(__uint_as_float(r[14]), __uint_as_float(r[15])));
}

// ---------------------------------------------------------------------------
// 2. dQ: persistent CTAs over items (query tile i, head bh), heaviest first;
//    per item, key tiles j = 0..i
// ---------------------------------------------------------------------------
template <int p>
struct DqSmem {
  using C = BwCfg<p>;
  static constexpr int offDO = 0;                                       // 2 buffers of dO_i (SW128)
  static constexpr int offQ = offDO + 2 * C::kVBytes;                   // 2 buffers of Q_i
  static constexpr int offK = (offQ + 2 * C::kQKBytes + 1023) / 1024 * 1024;  // ring of K_j
  static constexpr int offV = (offK + kBwStages * C::kQKBytes + 1023) / 1024 * 1024;  // ring of V_j
  static constexpr int offBar = offV + kBwStages * C::kVBytes;
  static constexpr int kBars = 4 + 2 * kBwStages + 7;
  static constexpr int offMisc = offBar + kBars * 8;
  static constexpr int kBytes = offMisc + 16 + 1024;
};

template <int p>
__global__ void __launch_bounds__(kBwThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const float2* __restrict__ rowc, __nv_bfloat16* __restrict__ dq, int T, int BH, int ld,
                  int dq_accumulate, int diag_only, WaitCtl wc) {
  using C = BwCfg<p>;
  using L = DqSmem<p>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::offBar);
  uint64_t* q_full = bars;                      // [2] Q_i and dO_i landed
  uint64_t* q_empty = q_full + 2;               // [2]
  uint64_t* kv_full = q_empty + 2;              // [kBwStages]
  uint64_t* kv_empty = kv_full + kBwStages;     // [kBwStages]
  uint64_t* s_full = kv_empty + kBwStages;      // S and dP of a key tile in TMEM
  uint64_t* s_read = s_full + 1;                // ... loaded by the weight warps (512)
  uint64_t* p_full = s_read + 1;                // [2] dS buffer written (512)
  uint64_t* acc_full = p_full + 2;              // an item's dQ complete
  uint64_t* acc_free = acc_full + 1;            // ... read by the epilogue (512)
  uint64_t* done = acc_free + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::offMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::offMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = (T + kBw - 1) / kBw;
  const int n_items = n_tiles * BH;
  auto item_tile = [&](int it) { return n_tiles - 1 - it / BH; };  // heaviest first
  auto my_item = [&](int r) {
    const int it = r * (int)gridDim.x + ((r & 1) ? (int)gridDim.x - 1 - (int)blockIdx.x : (int)blockIdx.x);
    return it < n_items ? it : -1;
  };

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(q_full + b, 1);
      mbar_init(q_empty + b, 1);
      mbar_init(p_full + b, 512);
    }
    for (int s = 0; s < kBwStages; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_read, 512);
    mbar_init(acc_full, 1);
    mbar_init(acc_free, 512);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_holder, kBwTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitEnv env{wc.status, abort_flag, wc.limit};

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      prefetch_tmap(&tm_do);
      int nq = 0;
      long rg = 0;  // key tiles loaded (ring position)
      bool ok = true;
      for (int it = my_item(nq); ok && it >= 0; it = my_item(++nq)) {
        const int tile = item_tile(it), bh = it % BH, qb = nq & 1;
        if (!mbar_wait(q_empty + qb, ((nq >> 1) & 1) ^ 1, env)) break;
        mbar_arrive_expect_tx(q_full + qb, C::kVBytes + C::kQKBytes);
        tma_load_3d(smem + L::offDO + qb * C::kVBytes, &tm_do, q_full + qb, 0, tile * kBw, bh);
        tma_load_3d(smem + L::offQ + qb * C::kQKBytes, &tm_q, q_full + qb, 0, tile * kBw, bh);
        for (int j = diag_only ? tile : 0; j <= tile; ++j, ++rg) {
          const int st = (int)(rg % kBwStages);
          if (!mbar_wait(kv_empty + st, (int)((rg / kBwStages) & 1) ^ 1, env)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(kv_full + st, C::kQKBytes + C::kVBytes);
          tma_load_3d(smem + L::offK + st * C::kQKBytes, &tm_k, kv_full + st, 0, j * kBw, bh);
          tma_load_3d(smem + L::offV + st * C::kVBytes, &tm_v, kv_full + st, 0, j * kBw, bh);
        }
      }
      for (int n = nq - 2 < 0 ? 0 : nq - 2; n < nq; ++n) mbar_wait_drain(q_full + (n & 1), (n >> 1) & 1);
      for (long n = rg - kBwStages < 0 ? 0 : rg - kBwStages; n < rg; ++n)
        mbar_wait_drain(kv_full + n % kBwStages, (int)((n / kBwStages) & 1));
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    constexpr uint32_t id_s = idesc_bf16(kBw, kBw, false, false);  // both operands K-major
    constexpr uint32_t id_dq = idesc_bf16(kBw, p, false, true);    // A = dS (TMEM), B = K_j MN-major
    const uint64_t dq0 = smem_desc(smem_u32(smem + L::offQ), 16, C::kQKSbo, C::kQKSw);
    const uint64_t ddn0 = smem_desc(smem_u32(smem + L::offDO), 16, C::kVSbo, kSw128);
    const uint64_t dk0 = smem_desc(smem_u32(smem + L::offK), 16, C::kQKSbo, C::kQKSw);
    const uint64_t dv0 = smem_desc(smem_u32(smem + L::offV), 16, C::kVSbo, kSw128);
    // S = Q K_j^T (K = p) and dP = dO V_j^T (K = dv): query buffer qb, key stage st
    auto issue_sdp = [&](int qb, int st) {
#pragma unroll
      for (int ks = 0; ks < p / 16; ++ks)
        mma_ss_w(tmem + C::colS, desc_add(dq0, qb * C::kQKBytes + ks * 32), desc_add(dk0, st * C::kQKBytes + ks * 32),
                 id_s, ks > 0);
#pragma unroll
      for (int ks = 0; ks < kBwDV / 16; ++ks)
        mma_ss_w(tmem + C::colP, desc_add(ddn0, qb * C::kVBytes + ks * 32), desc_add(dv0, st * C::kVBytes + ks * 32),
                 id_s, ks > 0);
      mma_commit_w(s_full);
    };
    int gs = 0;       // key tiles processed by this CTA (global step)
    int nq = 0, acc_cnt = 0;
    bool ok = true;
    for (int it = my_item(nq); ok && it >= 0; it = my_item(++nq)) {
      const int qb = nq & 1, nkv = diag_only ? 1 : item_tile(it) + 1;
      if (!mbar_wait_w(q_full + qb, (nq >> 1) & 1, env) ||
          !mbar_wait_w(kv_full + gs % kBwStages, (gs / kBwStages) & 1, env) ||
          (gs > 0 && !mbar_wait_w(s_read, (gs - 1) & 1, env))) {
        ok = false;
        break;
      }
      tc_fence_after();
      issue_sdp(qb, gs % kBwStages);
      for (int j = 0; j < nkv; ++j) {
        const int g = gs + j, st = g % kBwStages;
        if (j + 1 < nkv) {
          // the next tile's S and dP overwrite the current ones: wait until loaded
          if (!mbar_wait_w(kv_full + (g + 1) % kBwStages, ((g + 1) / kBwStages) & 1, env) ||
              !mbar_wait_w(s_read, g & 1, env)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_sdp(qb, (g + 1) % kBwStages);
        }
        if (!mbar_wait_w(p_full + (g & 1), (g >> 1) & 1, env)) {
          ok = false;
          break;
        }
        // the item's first dQ MMA overwrites the accumulator: the previous
        // item's epilogue must have read it
        if (j == 0 && acc_cnt > 0 && !mbar_wait_w(acc_free, (acc_cnt - 1) & 1, env)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < kBw / 16; ++ks)  // keys 16ks..: dS columns 8ks.. of the buffer
          mma_ts_w(tmem + C::colAcc, tmem + C::colA(g & 1) + 8 * ks,
                   desc_add(dk0, st * C::kQKBytes + ks * C::kQKKStep), id_dq, (j > 0 || ks > 0) ? 1u : 0u);
        mma_commit_w(kv_empty + st);
      }
      if (!ok) break;
      mma_commit_w(acc_full);
      ++acc_cnt;
      mma_commit_w(q_empty + qb);
      gs += nkv;
    }
    mma_commit_w(done);
    mbar_wait_drain(done, 0);
  } else {
    // ------------------------------------------------------------- weight warps + epilogue
    const int quarter = warp % 4;                 // rows (queries) 32 quarter ..
    const int kq = (warp - 2) / 4;                // keys 32 kq .. of the key tile
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    int gs = 0;
    int nq = 0, acc_cnt = 0;
    bool ok = true;
    for (int it = my_item(nq); ok && it >= 0; it = my_item(++nq)) {
      const int tile = item_tile(it), bh = it % BH, nkv = diag_only ? 1 : tile + 1;
      const int row = tile * kBw + quarter * 32 + lane;
      const float2 rc = row < T ? rowc[(size_t)bh * T + row] : make_float2(0.f, 0.f);  // (-delta, 1/D)
      for (int j = 0; j < nkv; ++j) {
        const int g = gs + j;
        if (!mbar_wait_w(s_full, g & 1, env)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // causal mask on the diagonal tile: key 32 kq + c <= query 32 quarter + lane
        const bool diag = (j == nkv - 1);
        const bool skip = diag && kq > quarter;
        const bool part = diag && kq == quarter;
        uint32_t gr[16], unused[16];
        if (skip) {
#pragma unroll
          for (int x = 0; x < 16; ++x) gr[x] = 0u;
        } else {
          uint32_t s[16], d[16];
          tmem_ld16(lane_base + C::colS + 32 * kq, s);
          tmem_ld16(lane_base + C::colP + 32 * kq, d);
          tmem_wait_ld();
          if (part)
            grad_pairs<0, false, false, true, false>(s, d, nullptr, rc, lane, gr, unused);
          else
            grad_pairs<0, false, false, false, false>(s, d, nullptr, rc, lane, gr, unused);
          tmem_ld16(lane_base + C::colS + 32 * kq + 16, s);
          tmem_ld16(lane_base + C::colP + 32 * kq + 16, d);
          tmem_wait_ld();
          if (part)
            grad_pairs<1, false, false, true, false>(s, d, nullptr, rc, lane, gr, unused);
          else
            grad_pairs<1, false, false, false, false>(s, d, nullptr, rc, lane, gr, unused);
        }
        // S and dP are in registers: the next key tile's may overwrite them
        tc_fence_before();
        mbar_arrive(s_read);
        // dS buffer g % 2 was last read by the dQ MMAs of step g - 2, which
        // completed before S(g) did
        tmem_st16(lane_base + C::colA(g & 1) + 16 * kq, gr);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full + (g & 1));
      }
      // the rows another pass wrote, loaded before the accumulator is
      // complete so that their latency overlaps the item's last MMAs
      // (p = 16 only: at p = 32 the registers held across the wait spill)
      uint4 old0[2];
      if constexpr (p == 16)
        if (dq_accumulate && kq == 0 && row < T) load_row16_words(dq + ((size_t)bh * T + row) * ld, old0);
      if (!ok || !mbar_wait_w(acc_full, acc_cnt & 1, env)) break;
      ++acc_cnt;
      tc_fence_after();
      // epilogue: dQ (p fp32 columns) -> registers (warps of key quarter 0),
      // then free the accumulator; bf16 rows < T
      uint32_t r0[16], r1[16];
      if (kq == 0) {
        tmem_ld16(lane_base + C::colAcc, r0);
        if constexpr (p == 32) tmem_ld16(lane_base + C::colAcc + 16, r1);
        tmem_wait_ld();
      }
      tc_fence_before();
      mbar_arrive(acc_free);
      if (kq == 0 && row < T) {
        __nv_bfloat16* dqr = dq + ((size_t)bh * T + row) * ld;
        if (dq_accumulate) {
          if constexpr (p == 16) {
            add_row16_words(old0, r0);
          } else {
            add_row16(dqr, r0);
            add_row16(dqr + 16, r1);
          }
        }
        store_row16(dqr, r0);
        if constexpr (p == 32) store_row16(dqr + 16, r1);
      }
      gs += nkv;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kBwTmemCols);
  }
}

template <int p>
struct DkvSmem {
  using C = BwCfg<p>;
  static constexpr int offV = 0;                                        // 2 buffers of V_j (SW128)
  static constexpr int offK = offV + 2 * C::kVBytes;                    // 2 buffers of K_j
  static constexpr int offDO = (offK + 2 * C::kQKBytes + 1023) / 1024 * 1024;  // ring of dO_i
  static constexpr int offQ = offDO + kBwStages * C::kVBytes;           // ring of Q_i
  static constexpr int offDD = offQ + kBwStages * C::kQKBytes;          // (-delta, 1/D) of 32 queries per weight warp
  static constexpr int offBar = (offDD + 16 * 32 * 8 + 1023) / 1024 * 1024;
  static constexpr int kBars = 4 + 2 * kBwStages + 7;
  static constexpr int offMisc = offBar + kBars * 8;
  static constexpr int kBytes = offMisc + 16 + 1024;
};

template <int p>
__global__ void __launch_bounds__(kBwThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const float2* __restrict__ rowc, __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv,
                    int T, int BH, int ld, int dv_accumulate, int dk_accumulate, int diag_only, WaitCtl wc) {
  using C = BwCfg<p>;
  using L = DkvSmem<p>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::offBar);
  uint64_t* kv_full = bars;                     // [2] K_j and V_j landed
  uint64_t* kv_empty = kv_full + 2;             // [2]
  uint64_t* q_full = kv_empty + 2;              // [kBwStages] Q_i and dO_i
  uint64_t* q_empty = q_full + kBwStages;       // [kBwStages]
  uint64_t* s_full = q_empty + kBwStages;       // S^T and dP^T of a query tile in TMEM
  uint64_t* s_read = s_full + 1;                // ... loaded by the weight warps (512)
  uint64_t* p_full = s_read + 1;                // W^T and dS^T written (512)
  uint64_t* w_free = p_full + 1;                // ... read by the dV / dK MMAs
  uint64_t* acc_full = w_free + 1;              // an item's dV, dK complete
  uint64_t* acc_free = acc_full + 1;            // ... read by the epilogue (512)
  uint64_t* done = acc_free + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::offMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::offMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  KATA_TRACE_BEGIN(bwd);
  const int n_tiles = (T + kBw - 1) / kBw;
  const int n_items = n_tiles * BH;
  // item it: key tile it / BH (tile 0 has the most query tiles), head it % BH;
  // the r-th item of this CTA in snake order over the CTAs
  auto my_item = [&](int r) {
    const int it = r * (int)gridDim.x + ((r & 1) ? (int)gridDim.x - 1 - (int)blockIdx.x : (int)blockIdx.x);
    return it < n_items ? it : -1;
  };

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(kv_full + b, 1);
      mbar_init(kv_empty + b, 1);
    }
    for (int s = 0; s < kBwStages; ++s) {
      mbar_init(q_full + s, 1);
      mbar_init(q_empty + s, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_read, 512);
    mbar_init(p_full, 512);
    mbar_init(w_free, 1);
    mbar_init(acc_full, 1);
    mbar_init(acc_free, 512);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_holder, kBwTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitEnv env{wc.status, abort_flag, wc.limit};

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      prefetch_tmap(&tm_do);
      int nq = 0;
      long rg = 0;  // query tiles loaded (ring position)
      bool ok = true;
      for (int it = my_item(nq); ok && it >= 0; it = my_item(++nq)) {
        const int tile = it / BH, bh = it % BH, kb = nq & 1;
        if (!mbar_wait(kv_empty + kb, ((nq >> 1) & 1) ^ 1, env)) break;
        mbar_arrive_expect_tx(kv_full + kb, C::kVBytes + C::kQKBytes);
        tma_load_3d(smem + L::offV + kb * C::kVBytes, &tm_v, kv_full + kb, 0, tile * kBw, bh);
        tma_load_3d(smem + L::offK + kb * C::kQKBytes, &tm_k, kv_full + kb, 0, tile * kBw, bh);
        for (int i = tile; i < (diag_only ? tile + 1 : n_tiles); ++i, ++rg) {
          const int st = (int)(rg % kBwStages);
          if (!mbar_wait(q_empty + st, (int)((rg / kBwStages) & 1) ^ 1, env)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(q_full + st, C::kVBytes + C::kQKBytes);
          tma_load_3d(smem + L::offDO + st * C::kVBytes, &tm_do, q_full + st, 0, i * kBw, bh);
          tma_load_3d(smem + L::offQ + st * C::kQKBytes, &tm_q, q_full + st, 0, i * kBw, bh);
        }
      }
      for (int n = nq - 2 < 0 ? 0 : nq - 2; n < nq; ++n) mbar_wait_drain(kv_full + (n & 1), (n >> 1) & 1);
      for (long n = rg - kBwStages < 0 ? 0 : rg - kBwStages; n < rg; ++n)
        mbar_wait_drain(q_full + n % kBwStages, (int)((n / kBwStages) & 1));
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    constexpr uint32_t id_s = idesc_bf16(kBw, kBw, false, false);
    constexpr uint32_t id_dv = idesc_bf16(kBw, kBwDV, false, true);  // A = W^T (TMEM), B = dO_i MN-major
    constexpr uint32_t id_dk = idesc_bf16(kBw, p, false, true);      // A = dS^T (TMEM), B = Q_i MN-major
    const uint64_t dk0 = smem_desc(smem_u32(smem + L::offK), 16, C::kQKSbo, C::kQKSw);
    const uint64_t dv0 = smem_desc(smem_u32(smem + L::offV), 16, C::kVSbo, kSw128);
    const uint64_t dq0 = smem_desc(smem_u32(smem + L::offQ), 16, C::kQKSbo, C::kQKSw);
    const uint64_t ddn0 = smem_desc(smem_u32(smem + L::offDO), 16, C::kVSbo, kSw128);
    // S^T = K Q_i^T (K = p) and dP^T = V dO_i^T (K = dv): key buffer kb, query stage st
    auto issue_sdp = [&](int kb, int st) {
#pragma unroll
      for (int ks = 0; ks < p / 16; ++ks)
        mma_ss_w(tmem + C::colS, desc_add(dk0, kb * C::kQKBytes + ks * 32), desc_add(dq0, st * C::kQKBytes + ks * 32),
                 id_s, ks > 0);
#pragma unroll
      for (int ks = 0; ks < kBwDV / 16; ++ks)
        mma_ss_w(tmem + C::colP, desc_add(dv0, kb * C::kVBytes + ks * 32), desc_add(ddn0, st * C::kVBytes + ks * 32),
                 id_s, ks > 0);
      mma_commit_w(s_full);
    };
    int gs = 0;       // query tiles processed by this CTA (global step)
    int nq = 0, acc_cnt = 0;
    bool ok = true;
    for (int it = my_item(nq); ok && it >= 0; it = my_item(++nq)) {
      const int tile = it / BH, kb = nq & 1, cnt = diag_only ? 1 : n_tiles - tile;
      if (!mbar_wait_w(kv_full + kb, (nq >> 1) & 1, env) ||
          !mbar_wait_w(q_full + gs % kBwStages, (int)((gs / kBwStages) & 1), env) ||
          (gs > 0 && !mbar_wait_w(s_read, (int)((gs - 1) & 1), env))) {
        ok = false;
        break;
      }
      tc_fence_after();
      issue_sdp(kb, (int)(gs % kBwStages));
      KATA_TRACE(bwd, gs, 0);
      for (int n = 0; n < cnt; ++n) {
        const int g = gs + n;
        const int st = g % kBwStages;
        if (n + 1 < cnt) {
          // the next tile's S^T and dP^T overwrite the current ones: wait until loaded
          if (!mbar_wait_w(q_full + (g + 1) % kBwStages, (int)(((g + 1) / kBwStages) & 1), env) ||
              !mbar_wait_w(s_read, (int)(g & 1), env)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_sdp(kb, (int)((g + 1) % kBwStages));
          KATA_TRACE(bwd, g + 1, 0);
        }
        if (!mbar_wait_w(p_full, (int)(g & 1), env)) {
          ok = false;
          break;
        }
        KATA_TRACE(bwd, g, 1);
        // the item's first dV / dK overwrite the accumulators: the previous
        // item's epilogue must have read them
        if (n == 0 && acc_cnt > 0 && !mbar_wait_w(acc_free, (acc_cnt - 1) & 1, env)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < kBw / 16; ++ks)  // queries 16ks..: operand columns 8ks..
          mma_ts_w(tmem + C::colAcc, tmem + C::colA(0) + 8 * ks, desc_add(ddn0, st * C::kVBytes + ks * C::kVKStep),
                   id_dv, (n > 0 || ks > 0) ? 1u : 0u);
#pragma unroll
        for (int ks = 0; ks < kBw / 16; ++ks)
          mma_ts_w(tmem + C::colAcc + kBwDV, tmem + C::colA(1) + 8 * ks,
                   desc_add(dq0, st * C::kQKBytes + ks * C::kQKKStep), id_dk, (n > 0 || ks > 0) ? 1u : 0u);
        mma_commit_w(w_free);
        mma_commit_w(q_empty + st);
        KATA_TRACE(bwd, g, 2);
      }
      if (!ok) break;
      mma_commit_w(acc_full);
      ++acc_cnt;
      mma_commit_w(kv_empty + kb);
      gs += cnt;
    }
    mma_commit_w(done);
    mbar_wait_drain(done, 0);
  } else {
    // ------------------------------------------------------------- weight warps + epilogue
    const int quarter = warp % 4;                 // rows (keys) 32 quarter ..
    const int kq = (warp - 2) / 4;                // queries 32 kq .. of the query tile
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    float2* dd_slot = reinterpret_cast<float2*>(smem + L::offDD) + (warp - 2) * 32;
    const int tslot = (warp == 2 && lane == 0) ? 5 : (warp == 17 && lane == 0) ? 9 : -1;  // traced warps
    const float4* dd_pairs = reinterpret_cast<const float4*>(dd_slot);
    int gs = 0;
    int nq = 0, acc_cnt = 0;
    bool ok = true;
    for (int it = my_item(nq); ok && it >= 0; it = my_item(++nq)) {
      const int tile = it / BH, bh = it % BH, cnt = diag_only ? 1 : n_tiles - tile;
      for (int n = 0; n < cnt; ++n) {
        const int g = gs + n;
        // (-delta, 1/D) of this warp's 32 queries, one per lane (0 past T)
        const int qrow = (tile + n) * kBw + 32 * kq + lane;
        const float2 rcl = qrow < T ? rowc[(size_t)bh * T + qrow] : make_float2(0.f, 0.f);
        if (!mbar_wait_w(s_full, (int)(g & 1), env)) {
          ok = false;
          break;
        }
        if (tslot >= 0) KATA_TRACE(bwd, g, tslot);
        tc_fence_after();
        // causal mask on the diagonal tile: query 32 kq + c >= key 32 quarter + lane
        const bool diag = (n == 0);
        const bool skip = diag && kq < quarter;
        const bool part = diag && kq == quarter;
        uint32_t gr[16], w[16];
        if (skip) {
#pragma unroll
          for (int x = 0; x < 16; ++x) gr[x] = w[x] = 0u;
        } else {
          // the 32 queries' constants, read back as column pairs (a broadcast per pair)
          __syncwarp();
          dd_slot[lane] = rcl;
          __syncwarp();
          uint32_t s[16], d[16];
          tmem_ld16(lane_base + C::colS + 32 * kq, s);
          tmem_ld16(lane_base + C::colP + 32 * kq, d);
          tmem_wait_ld();
          if (part)
            grad_pairs<0, true, true, true, true>(s, d, dd_pairs, make_float2(0.f, 0.f), lane, gr, w);
          else
            grad_pairs<0, true, true, false, true>(s, d, dd_pairs, make_float2(0.f, 0.f), lane, gr, w);
          tmem_ld16(lane_base + C::colS + 32 * kq + 16, s);
          tmem_ld16(lane_base + C::colP + 32 * kq + 16, d);
          tmem_wait_ld();
          if (part)
            grad_pairs<1, true, true, true, true>(s, d, dd_pairs + 8, make_float2(0.f, 0.f), lane, gr, w);
          else
            grad_pairs<1, true, true, false, true>(s, d, dd_pairs + 8, make_float2(0.f, 0.f), lane, gr, w);
        }
        tc_fence_before();
        mbar_arrive(s_read);
        if (tslot >= 0) KATA_TRACE(bwd, g, tslot + 1);
        // the operand buffers are read by the previous query tile's MMAs
        if (g > 0 && !mbar_wait_w(w_free, (int)((g - 1) & 1), env)) {
          ok = false;
          break;
        }
        if (tslot >= 0) KATA_TRACE(bwd, g, tslot + 2);
        tc_fence_after();
        tmem_st16(lane_base + C::colA(0) + 16 * kq, w);
        tmem_st16(lane_base + C::colA(1) + 16 * kq, gr);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full);
        if (tslot >= 0) KATA_TRACE(bwd, g, tslot + 3);
      }
      // rows another pass wrote, loaded before the accumulators are complete
      // so that their latency overlaps the item's last MMAs
      const int row = tile * kBw + quarter * 32 + lane;  // this thread's key
      const size_t r0 = (size_t)bh * T + (row < T ? row : 0);
      // (p = 16 only: at p = 32 the registers held across the wait spill)
      uint4 old_v[2], old_k0[2];
      if constexpr (p == 16) {
        if (dv_accumulate && row < T) load_row16_words(dv + r0 * kBwDV + 16 * kq, old_v);
        if (dk_accumulate && kq == 0 && row < T) load_row16_words(dk + r0 * ld, old_k0);
      }
      if (!ok || !mbar_wait_w(acc_full, acc_cnt & 1, env)) break;
      ++acc_cnt;
      tc_fence_after();
      // epilogue: dV (16 columns per key-quarter warp) and dK (p columns,
      // warps of key quarter 0) -> registers, then free the accumulators
      uint32_t rv[16], rk0[16], rk1[16];
      tmem_ld16(lane_base + C::colAcc + 16 * kq, rv);
      if (kq == 0) {
        tmem_ld16(lane_base + C::colAcc + kBwDV, rk0);
        if constexpr (p == 32) tmem_ld16(lane_base + C::colAcc + kBwDV + 16, rk1);
      }
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(acc_free);
      // dV was accumulated with r = 2 / D: halve it (exact)
#pragma unroll
      for (int x = 0; x < 16; ++x) rv[x] = __float_as_uint(0.5f * __uint_as_float(rv[x]));
      if (row < T) {
        __nv_bfloat16* dvr = dv + r0 * kBwDV + 16 * kq;
        if (dv_accumulate) {  // another pass's dV is already there
          if constexpr (p == 16) add_row16_words(old_v, rv);
          else add_row16(dvr, rv);
        }
        store_row16(dvr, rv);
        if (kq == 0) {
          if (dk_accumulate) {
            if constexpr (p == 16) {
              add_row16_words(old_k0, rk0);
            } else {
              add_row16(dk + r0 * ld, rk0);
              add_row16(dk + r0 * ld + 16, rk1);
            }
          }
          store_row16(dk + r0 * ld, rk0);
          if constexpr (p == 32) store_row16(dk + r0 * ld + 16, rk1);
        }
      }
      gs += cnt;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kBwTmemCols);
  }
}

template <int p>
static cudaError_t launch_bwd_t(const void* q, const void* k, const void* v, const void* o, const float* D,
                                const void* dO, void* dq, void* dk, void* dv, int BH, int T, int ld, bool rows_ready,
                                bool dv_accumulate, bool dq_accumulate, bool dk_accumulate, bool diag_only,
                                void* ws, const WaitCtl& wc, cudaStream_t st) {
  float2* rowc = static_cast<float2*>(ws);
  const long long rows = (long long)BH * T;
  cudaError_t e = cudaSuccess;
  if (!rows_ready) {
    bwd_rows_kernel<<<(unsigned)((rows + kRowsPerBlock - 1) / kRowsPerBlock), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(dO), static_cast<const __nv_bfloat16*>(o), D, rowc, rows);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  CUtensorMap tq, tk, tv, tdo;
  if (!make_tmap_bf16_ld(&tq, q, p, ld, T, BH, kBw) || !make_tmap_bf16_ld(&tk, k, p, ld, T, BH, kBw) ||
      !make_tmap_bf16(&tv, v, kBwDV, T, BH, kBw) || !make_tmap_bf16(&tdo, dO, kBwDV, T, BH, kBw))
    return cudaErrorInvalidValue;
  const dim3 grid((T + kBw - 1) / kBw, BH);
  auto kq = bwd_dq_kernel<p>;
  auto kkv = bwd_dkdv_kernel<p>;
  if ((e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, DqSmem<p>::kBytes)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(kkv, cudaFuncAttributeMaxDynamicSharedMemorySize, DkvSmem<p>::kBytes)) != cudaSuccess)
    return e;
  static int num_sms = 0;
  if (num_sms == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || num_sms <= 0)
      num_sms = 148;
  }
  const long items = (long)grid.x * BH;
  const int pgrid = (int)(items < num_sms ? items : num_sms);
  kq<<<pgrid, kBwThreads, DqSmem<p>::kBytes, st>>>(tq, tk, tv, tdo, rowc, static_cast<__nv_bfloat16*>(dq), T, BH, ld,
                                                    dq_accumulate ? 1 : 0, diag_only ? 1 : 0, wc);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  kkv<<<pgrid, kBwThreads, DkvSmem<p>::kBytes, st>>>(tq, tk, tv, tdo, rowc, static_cast<__nv_bfloat16*>(dk),
                                                      static_cast<__nv_bfloat16*>(dv), T, BH, ld, dv_accumulate ? 1 : 0,
                                                      dk_accumulate ? 1 : 0, diag_only ? 1 : 0, wc);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_flash_bwd_rows(const void* dO, const void* o, const float* D, void* ws, int BH, int T,
                                  cudaStream_t st) {
  const long long rows = (long long)BH * T;
  if (rows == 0) return cudaSuccess;
  bwd_rows_kernel<<<(unsigned)((rows + kRowsPerBlock - 1) / kRowsPerBlock), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(dO), static_cast<const __nv_bfloat16*>(o), D, static_cast<float2*>(ws), rows);
  return cudaGetLastError();
}

size_t flash_bwd_workspace_bytes(int BH, int T, int dv) {
  (void)dv;
  return (size_t)BH * T * sizeof(float2);  // (-delta, 1/D) per row
}

cudaError_t launch_flash_bwd_sm100(const void* q, const void* k, const void* v, const void* o, const float* D,
                                   const void* dO, void* dq, void* dk, void* dv, int BH, int T, int p, int ld,
                                   bool rows_ready, bool dv_accumulate, bool dq_accumulate, bool dk_accumulate,
                                   void* ws, const WaitCtl& wc, cudaStream_t st, bool diag_only) {
  if (p == 16)
    return launch_bwd_t<16>(q, k, v, o, D, dO, dq, dk, dv, BH, T, ld, rows_ready, dv_accumulate, dq_accumulate,
                            dk_accumulate, diag_only, ws, wc, st);
  if (p == 32)
    return launch_bwd_t<32>(q, k, v, o, D, dO, dq, dk, dv, BH, T, ld, rows_ready, dv_accumulate, dq_accumulate,
                            dk_accumulate, diag_only, ws, wc, st);
  return cudaErrorInvalidValue;
}

}  // namespace kata
