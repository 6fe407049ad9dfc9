// chunk_bwd_sm100.cu -- the inter-chunk part of the O(T) backward pass of the
// chunked KATA forward on tcgen05 / TMEM (bf16 inputs, p = 16, dv = 64).
//
// With the notation of flash_bwd_sm100.cu (dN_t = dO_t / D_t,
// dD_t = -(dO_t . o_t) / D_t, 0 where D_t = 0) the gradients of
// o_t = psi(q_t)^T S_t / psi(q_t)^T z_t are
//   dpsi(q_t) = S_t dN_t + z_t dD_t          S_t = sum_{s<=t} psi(k_s) v_s^T
//   dpsi(k_s) = G_s v_s + g_s                G_s = sum_{t>=s} psi(q_t) dN_t^T,
//   dv_s      = G_s^T psi(k_s)               g_s = sum_{t>=s} psi(q_t) dD_t
// and dq_t = 2 dPsi(q_t) q_t, dk_s = 2 dPsi(k_s) k_s for the symmetric p x p
// forms dPsi of dpsi (the derivative of vec(u u^T)).  Split at the 128-token
// chunks: the pairs of a chunk with itself are the flash backward kernels'
// diagonal tiles (launched with diag_only); this file adds the pairs of a
// token with the chunks before it (dq) or after it (dk, dv) through the
// chunk states:
//   1. chunk_grad_sums_kernel: per chunk c the sums
//        dS~_c^T = [V_c | 1]^T psi~(K_c)     (the forward's state update)
//        dG~_c^T = [dN_c | dD_c]^T psi~(Q_c)
//      written as records (dG in reverse chunk order);
//   2. the scan (scan.cu) over each: record c becomes the state before
//      chunk c, S_{c-1}, and the reverse one the state after it, G_{c+1};
//   3. chunk_grad_inter_kernel: per chunk
//        X = [dN | dD] S~        -> dq_t += 2 dPsi_X q_t
//        Y = [V | 1]  G~         -> dk_s += 2 dPsi_Y k_s
//        Z = psi~(K) G~^T        -> dv_s += Z[:, 0:64]
//      added to the rows the diagonal pass wrote.
// Packed coordinates as in chunk_common.cuh: the key side of S~ carries the
// factor 2 off the diagonal, the query side of G~ does not.  Every chunk is
// independent once the scans are done, so one CTA handles one chunk.
#include <cuda.h>

#include "chunk_common.cuh"
#include "kata_internal.h"

namespace kata {

bool make_tmap_bf16(CUtensorMap* map, const void* base, int inner, int T, int BH, int rows);

namespace {

using namespace sm100;
using namespace chunk;

constexpr int kGThreads = 320;  // warp 0 TMA, warp 1 MMA, warps 2-9 operands and epilogue

// ---------------------------------------------------------------------------
// 1. per-chunk sums
// ---------------------------------------------------------------------------
struct SumSmem {
  static constexpr int offV = 0;                      // V tile, 128B swizzle
  static constexpr int offDN = offV + kVBytes;        // dO tile, scaled to dN in place
  static constexpr int offOnes = offDN + kVBytes;     // block of ones
  static constexpr int offAux = offOnes + kOnesBytes; // block of dD (every column of row t)
  static constexpr int offQ = offAux + kOnesBytes;    // Q tile, 32B swizzle
  static constexpr int offK = offQ + kQKBytes;        // K tile
  static constexpr int offPsiK = offK + kQKBytes;     // psi~(K), key side
  static constexpr int offPsiQ = offPsiK + kPsiBytes; // psi~(Q), query side
  static constexpr int offBar = offPsiQ + kPsiBytes;
  static constexpr int offMisc = offBar + 4 * 8;
  static constexpr int kBytes = offMisc + 16 + 1024;
};

// Scales the dO row t of a 128B-swizzled [128 x 64] tile by s in place (the
// swizzle only permutes the row's 16-byte chunks).
__device__ __forceinline__ void scale_row_sw128(uint8_t* tile, int t, float s) {
  uint4* row = reinterpret_cast<uint4*>(tile + t * 128);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint4 a = row[c];
    uint32_t* w = reinterpret_cast<uint32_t*>(&a);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float lo = __uint_as_float(w[e] << 16) * s, hi = __uint_as_float(w[e] & 0xffff0000u) * s;
      w[e] = pack_bf16x2(lo, hi);
    }
    row[c] = a;
  }
}

// Row t of a [128 x 64] 128B-swizzled block: every value = x (bf16).
__device__ __forceinline__ void fill_row_sw128(uint8_t* tile, int t, float x) {
  const uint32_t w = pack_bf16x2(x, x);
  uint4* row = reinterpret_cast<uint4*>(tile + t * 128);
#pragma unroll
  for (int c = 0; c < 8; ++c) row[c] = make_uint4(w, w, w, w);
}

__global__ void __launch_bounds__(kGThreads, 1)
    chunk_grad_sums_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                           const float2* __restrict__ rowc, float* __restrict__ wsS, float* __restrict__ wsG, int T,
                           int n_chunks, long long record_floats, WaitCtl wc) {
  using L = SumSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::offBar);
  uint64_t* tiles_full = bars;
  uint64_t* ops_ready = bars + 1;  // operands formed (256)
  uint64_t* acc_done = bars + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::offMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::offMisc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x, bh = blockIdx.y;
  const int row0 = c * kTile;

  if (threadIdx.x == 0) {
    mbar_init(tiles_full, 1);
    mbar_init(ops_ready, 256);
    mbar_init(acc_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  fill_ones(smem + L::offOnes, threadIdx.x, kGThreads);
  if (warp == 1) tmem_alloc(tmem_holder, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitEnv env{wc.status, abort_flag, wc.limit};
  constexpr uint32_t colS = 0, colG = 256;

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(tiles_full, 2 * kVBytes + 2 * kQKBytes);
      tma_load_3d(smem + L::offV, &tm_v, tiles_full, 0, row0, bh);
      tma_load_3d(smem + L::offDN, &tm_do, tiles_full, 0, row0, bh);
      tma_load_3d(smem + L::offQ, &tm_q, tiles_full, 0, row0, bh);
      tma_load_3d(smem + L::offK, &tm_k, tiles_full, 0, row0, bh);
      mbar_wait_drain(tiles_full, 0);
    }
  } else if (warp == 1) {
    // whole warp; one elected lane issues
    bool issued = false;
    if (mbar_wait_w(ops_ready, 0, env)) {
      tc_fence_after();
      constexpr uint32_t id_u = idesc_bf16(128, kNP, true, true);  // A = [X | w]^T (MN-major), B = psi~ (N-major)
      const uint64_t dvo = desc_vones(smem_u32(smem + L::offV), smem_u32(smem + L::offOnes));
      const uint64_t dna = desc_vones(smem_u32(smem + L::offDN), smem_u32(smem + L::offAux));
      const uint64_t dpk = smem_desc(smem_u32(smem + L::offPsiK), kPsiAtom, 256, kSw32);
      const uint64_t dpq = smem_desc(smem_u32(smem + L::offPsiQ), kPsiAtom, 256, kSw32);
#pragma unroll
      for (int ks = 0; ks < kTile / 16; ++ks)
        mma_ss_w(tmem + colS, desc_add(dvo, ks * 2048), desc_add(dpk, ks * 512), id_u, ks > 0);
#pragma unroll
      for (int ks = 0; ks < kTile / 16; ++ks)
        mma_ss_w(tmem + colG, desc_add(dna, ks * 2048), desc_add(dpq, ks * 512), id_u, ks > 0);
      mma_commit_w(acc_done);
      issued = true;
    }
    if (issued) mbar_wait_drain(acc_done, 0);
  } else {
    // warps 2-9: token m of the chunk; warps 2-5 psi~(k_m) and dN_m, warps
    // 6-9 psi~(q_m) and the dD block
    const int quarter = warp % 4;
    const int m = quarter * 32 + lane;
    const bool kside = warp < 6;
    bool ok = mbar_wait_w(tiles_full, 0, env);
    if (ok) {
      const int t = row0 + m;
      const float2 rc = t < T ? rowc[(size_t)bh * T + t] : make_float2(0.f, 0.f);  // (-delta, 2/D)
      __nv_bfloat162 u[8];
      uint32_t w[kNPW];
      if (kside) {
        load_row_sw<1>(smem + L::offK, m, u);
        packed_psi<true>(u, w);
        store_psi_k(smem + L::offPsiK, m, w);
        scale_row_sw128(smem + L::offDN, m, 0.5f * rc.y);  // dN = dO / D
      } else {
        load_row_sw<1>(smem + L::offQ, m, u);
        packed_psi<false>(u, w);
        store_psi_k(smem + L::offPsiQ, m, w);
        fill_row_sw128(smem + L::offAux, m, 0.5f * rc.x * rc.y);  // dD = -delta / D
      }
      fence_proxy_async_smem();
      mbar_arrive(ops_ready);
    }
    // records: TMEM lanes 0..64 of both sums (quarters 0-2, one warp each)
    const bool writer = (warp == 2 || warp == 4 || warp == 5 || warp == 6 || warp == 8 || warp == 9);
    if (ok && writer && mbar_wait_w(acc_done, 0, env)) {
      tc_fence_after();
      const int d = quarter * 32 + lane;
      const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
      if (kside) {
        float* row = wsS + ((size_t)bh * n_chunks + c) * record_floats + (size_t)min(d, kRecRows - 1) * kNP;
        state_lane_to_global(lane_base + colS, row, d < kRecRows);
      } else {
        float* row = wsG + ((size_t)bh * n_chunks + (n_chunks - 1 - c)) * record_floats +
                     (size_t)min(d, kRecRows - 1) * kNP;
        state_lane_to_global(lane_base + colG, row, d < kRecRows);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// 3. inter-chunk gradients
// ---------------------------------------------------------------------------
constexpr int kTAtom = kNP * 32;  // one K step (16 values) of a [144 coordinates x 80] K-major copy

struct InterSmem {
  static constexpr int offV = 0;
  static constexpr int offDN = offV + kVBytes;
  static constexpr int offOnes = offDN + kVBytes;
  static constexpr int offAux = offOnes + kOnesBytes;
  static constexpr int offQ = offAux + kOnesBytes;
  static constexpr int offK = offQ + kQKBytes;
  static constexpr int offPsiK = offK + kQKBytes;       // psi~(K), key side (K-major A operand)
  static constexpr int offST = offPsiK + kPsiBytes;     // S~ as [144 x 80] K-major (5 atoms)
  static constexpr int offGT = offST + 5 * kTAtom;      // G~ as [144 x 80] K-major
  static constexpr int offG = offGT + 5 * kTAtom;       // G~ as [80 x 144] K-major (the forward's copy layout)
  static constexpr int offBar = offG + kSBBytes;
  static constexpr int offMisc = offBar + 4 * 8;
  static constexpr int kBytes = offMisc + 16 + 1024;
  // TMEM columns
  static constexpr uint32_t colX = 0;    // [dN | dD] S~, 144
  static constexpr uint32_t colY = 160;  // [V | 1] G~, 144
  static constexpr uint32_t colZ = 320;  // psi~(K) G~^T, 80
};

// Element (n, e) of a [144 x 80] K-major bf16 copy (K steps of 16 as 32B-
// swizzled atoms of [144 rows x 32 B]).
__device__ __forceinline__ uint32_t tcopy_offset(int n, int e) {
  return (uint32_t)((e >> 4) * kTAtom + n * 32 + ((((e >> 3) & 1) ^ ((n >> 2) & 1)) << 4) + (e & 7) * 2);
}
// Element (e, w) of the forward's [80 x 144] copy layout.
__device__ __forceinline__ uint32_t copy_offset(int e, int w) {
  return (uint32_t)((w >> 4) * kSBAtom + e * 32 + ((((w >> 3) & 1) ^ ((e >> 2) & 1)) << 4) + (w & 7) * 2);
}

// 2 dPsi(u) u for the symmetric p x p form of a packed gradient row held in
// TMEM columns [taddr, taddr + 144) of this lane: off-diagonal packed entries
// count f_off times (the entry of one triangle), diagonal ones f_diag times.
// Warp-collective (the loads).
template <int kFDiag, int kFOff>
__device__ __forceinline__ void packed_grad_times_u(uint32_t taddr, const float (&u)[16], float (&out)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) out[i] = 0.f;
#pragma unroll
  for (int b = 0; b < 9; ++b) {
    uint32_t r[16];
    tmem_ld16(taddr + 16 * b, r);
    tmem_wait_ld();
#pragma unroll
    for (int x = 0; x < 16; ++x) {
      const int w = 16 * b + x;
      const int i = packed_i(w), j = packed_j(w);
      if (i < 0) continue;
      const float g = __uint_as_float(r[x]);
      if (i == j) {
        out[i] = fmaf((float)kFDiag * g, u[i], out[i]);
      } else {
        out[i] = fmaf((float)kFOff * g, u[j], out[i]);
        out[j] = fmaf((float)kFOff * g, u[i], out[j]);
      }
    }
  }
}

// the N bf16 values at row, plus the fp32 values in add, written back
template <int N>
__device__ __forceinline__ void add_to_bf16_row(__nv_bfloat16* row, const float (&add)[N]) {
#pragma unroll
  for (int e = 0; e < N; e += 8) {
    uint4* p4 = reinterpret_cast<uint4*>(row + e);
    uint4 a = *p4;
    uint32_t* w = reinterpret_cast<uint32_t*>(&a);
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const float lo = __uint_as_float(w[x] << 16) + add[e + 2 * x];
      const float hi = __uint_as_float(w[x] & 0xffff0000u) + add[e + 2 * x + 1];
      w[x] = pack_bf16x2(lo, hi);
    }
    *p4 = a;
  }
}

__global__ void __launch_bounds__(kGThreads, 1)
    chunk_grad_inter_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                            const float2* __restrict__ rowc, const float* __restrict__ wsS,
                            const float* __restrict__ wsG, __nv_bfloat16* __restrict__ dq,
                            __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv, int T, int n_chunks,
                            long long record_floats, WaitCtl wc) {
  using L = InterSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::offBar);
  uint64_t* tiles_full = bars;
  uint64_t* ops_ready = bars + 1;  // operands formed (256)
  uint64_t* acc_done = bars + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::offMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::offMisc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x, bh = blockIdx.y;
  const int row0 = c * kTile;

  if (threadIdx.x == 0) {
    mbar_init(tiles_full, 1);
    mbar_init(ops_ready, 256);
    mbar_init(acc_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  fill_ones(smem + L::offOnes, threadIdx.x, kGThreads);
  if (warp == 1) tmem_alloc(tmem_holder, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitEnv env{wc.status, abort_flag, wc.limit};

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(tiles_full, 2 * kVBytes + 2 * kQKBytes);
      tma_load_3d(smem + L::offV, &tm_v, tiles_full, 0, row0, bh);
      tma_load_3d(smem + L::offDN, &tm_do, tiles_full, 0, row0, bh);
      tma_load_3d(smem + L::offQ, &tm_q, tiles_full, 0, row0, bh);
      tma_load_3d(smem + L::offK, &tm_k, tiles_full, 0, row0, bh);
      mbar_wait_drain(tiles_full, 0);
    }
  } else if (warp == 1) {
    bool issued = false;
    if (mbar_wait_w(ops_ready, 0, env)) {
      tc_fence_after();
      constexpr uint32_t id_xy = idesc_bf16(128, kNP, false, false);  // A [128 x 80] K-major, B [144 x 80] K-major
      constexpr uint32_t id_z = idesc_bf16(128, 80, false, false);    // A psi~(K) K-major, B [80 x 144] K-major
      const uint64_t dV = smem_desc(smem_u32(smem + L::offV), 16, 1024, kSw128);
      const uint64_t dOnes = smem_desc(smem_u32(smem + L::offOnes), 16, 1024, kSw128);
      const uint64_t dN = smem_desc(smem_u32(smem + L::offDN), 16, 1024, kSw128);
      const uint64_t dAux = smem_desc(smem_u32(smem + L::offAux), 16, 1024, kSw128);
      const uint64_t dST = smem_desc(smem_u32(smem + L::offST), 16, 256, kSw32);
      const uint64_t dGT = smem_desc(smem_u32(smem + L::offGT), 16, 256, kSw32);
      const uint64_t dG = smem_desc(smem_u32(smem + L::offG), 16, 256, kSw32);
      const uint64_t dPK = smem_desc(smem_u32(smem + L::offPsiK), 16, 256, kSw32);
      // X = [dN | dD] S~ and Y = [V | 1] G~: K = 80 in 5 steps, the fifth
      // from the dD / ones block
#pragma unroll
      for (int ks = 0; ks < 5; ++ks) {
        const uint64_t a = ks < 4 ? desc_add(dN, ks * 32) : dAux;
        mma_ss_w(tmem + L::colX, a, desc_add(dST, ks * kTAtom), id_xy, ks > 0);
      }
#pragma unroll
      for (int ks = 0; ks < 5; ++ks) {
        const uint64_t a = ks < 4 ? desc_add(dV, ks * 32) : dOnes;
        mma_ss_w(tmem + L::colY, a, desc_add(dGT, ks * kTAtom), id_xy, ks > 0);
      }
      // Z = psi~(K) G~^T: K = 144 in 9 steps
#pragma unroll
      for (int ks = 0; ks < kNP / 16; ++ks)
        mma_ss_w(tmem + L::colZ, desc_add(dPK, ks * kPsiAtom), desc_add(dG, ks * kSBAtom), id_z, ks > 0);
      mma_commit_w(acc_done);
      issued = true;
    }
    if (issued) mbar_wait_drain(acc_done, 0);
  } else {
    const int quarter = warp % 4;
    const int m = quarter * 32 + lane;
    const int wt = threadIdx.x - 64;  // 0..255
    // the state before the chunk (record c of wsS) and the state after it
    // (record n_chunks - 1 - c of wsG) -> bf16 copies, rows past the
    // normaliser (65..79) zero.  Consecutive threads take consecutive rows of
    // a copy (16-byte stores 32 bytes apart, conflict-free under the 32-byte
    // swizzle) and read consecutive record columns.
    const float* recS = wsS + ((size_t)bh * n_chunks + c) * record_floats;
    const float* recG = wsG + ((size_t)bh * n_chunks + (n_chunks - 1 - c)) * record_floats;
    for (int x = wt; x < kNP * 10; x += 256) {  // [144 x 80] copies: row n, values e0..e0+7
      const int n = x % kNP, e0 = 8 * (x / kNP);
      float sv[8], gv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const bool live = e0 + u < kRecRows;
        sv[u] = live ? __ldcg(recS + (size_t)(e0 + u) * kNP + n) : 0.f;
        gv[u] = live ? __ldcg(recG + (size_t)(e0 + u) * kNP + n) : 0.f;
      }
      *reinterpret_cast<uint4*>(smem + L::offST + tcopy_offset(n, e0)) =
          make_uint4(pack_bf16x2(sv[0], sv[1]), pack_bf16x2(sv[2], sv[3]), pack_bf16x2(sv[4], sv[5]),
                     pack_bf16x2(sv[6], sv[7]));
      *reinterpret_cast<uint4*>(smem + L::offGT + tcopy_offset(n, e0)) =
          make_uint4(pack_bf16x2(gv[0], gv[1]), pack_bf16x2(gv[2], gv[3]), pack_bf16x2(gv[4], gv[5]),
                     pack_bf16x2(gv[6], gv[7]));
    }
    for (int x = wt; x < kSBRows * (kNP / 8); x += 256) {  // [80 x 144] copy: row e, values w0..w0+7
      const int e = x % kSBRows, w0 = 8 * (x / kSBRows);
      uint4 val = make_uint4(0, 0, 0, 0);
      if (e < kRecRows) {
        const float4 a = __ldcg(reinterpret_cast<const float4*>(recG + (size_t)e * kNP + w0));
        const float4 b = __ldcg(reinterpret_cast<const float4*>(recG + (size_t)e * kNP + w0 + 4));
        val = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
      }
      *reinterpret_cast<uint4*>(smem + L::offG + copy_offset(e, w0)) = val;
    }
    bool ok = mbar_wait_w(tiles_full, 0, env);
    const int t = row0 + m;
    const float2 rc = t < T ? rowc[(size_t)bh * T + t] : make_float2(0.f, 0.f);  // (-delta, 2/D)
    if (ok) {
      if (warp < 6) {
        __nv_bfloat162 u[8];
        uint32_t w[kNPW];
        load_row_sw<1>(smem + L::offK, m, u);
        packed_psi<true>(u, w);
        store_psi_k(smem + L::offPsiK, m, w);
      } else {
        scale_row_sw128(smem + L::offDN, m, 0.5f * rc.y);         // dN = dO / D
        fill_row_sw128(smem + L::offAux, m, 0.5f * rc.x * rc.y);  // dD = -delta / D
      }
      fence_proxy_async_smem();
      mbar_arrive(ops_ready);
    }
    if (ok && mbar_wait_w(acc_done, 0, env)) {
      tc_fence_after();
      const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
      if (warp < 6) {
        // dq_t += 2 dPsi_X q_t (X from the key-side S~: off-diagonal entries
        // already count both triangles)
        __nv_bfloat162 u2[8];
        load_row_sw<1>(smem + L::offQ, m, u2);
        float u[16], g[16];
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          u[2 * x] = __low2float(u2[x]);
          u[2 * x + 1] = __high2float(u2[x]);
        }
        packed_grad_times_u<2, 1>(lane_base + L::colX, u, g);
        if (t < T) add_to_bf16_row<16>(dq + ((size_t)bh * T + t) * 16, g);
      } else {
        // dk_s += 2 dPsi_Y k_s (Y from the query-side G~: one triangle's
        // entries) and dv_s += Z[:, 0:64]
        __nv_bfloat162 u2[8];
        load_row_sw<1>(smem + L::offK, m, u2);
        float u[16], g[16];
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          u[2 * x] = __low2float(u2[x]);
          u[2 * x + 1] = __high2float(u2[x]);
        }
        packed_grad_times_u<2, 2>(lane_base + L::colY, u, g);
        if (t < T) add_to_bf16_row<16>(dk + ((size_t)bh * T + t) * 16, g);
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          uint32_t r[32];
          tmem_ld32(lane_base + L::colZ + 32 * b, r);
          tmem_wait_ld();
          float z[32];
#pragma unroll
          for (int x = 0; x < 32; ++x) z[x] = __uint_as_float(r[x]);
          if (t < T) add_to_bf16_row<32>(dv + ((size_t)bh * T + t) * kDV + 32 * b, z);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

size_t chunk_bwd_records_bytes(int BH, int T) {
  const size_t n_chunks = (size_t)(T + kTile - 1) / kTile;
  return 2 * (size_t)BH * n_chunks * kRecRows * kNP * sizeof(float);
}

cudaError_t launch_chunk_bwd_inter_sm100(const void* q, const void* k, const void* v, const void* dO,
                                         const float2* rowc, float* records, void* dq, void* dk, void* dv, int BH,
                                         int T, const WaitCtl& wc, cudaStream_t st) {
  const int n_chunks = (T + kTile - 1) / kTile;
  if (n_chunks < 2) return cudaSuccess;  // no pair crosses a chunk boundary
  CUtensorMap tq, tk, tv, tdo;
  if (!make_tmap_bf16(&tq, q, 16, T, BH, kTile) || !make_tmap_bf16(&tk, k, 16, T, BH, kTile) ||
      !make_tmap_bf16(&tv, v, kDV, T, BH, kTile) || !make_tmap_bf16(&tdo, dO, kDV, T, BH, kTile))
    return cudaErrorInvalidValue;
  const long long rf = (long long)kRecRows * kNP;
  float* wsS = records;
  float* wsG = records + (size_t)BH * n_chunks * rf;
  cudaError_t e =
      cudaFuncSetAttribute(chunk_grad_sums_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SumSmem::kBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(chunk_grad_inter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             InterSmem::kBytes);
  if (e != cudaSuccess) return e;
  const dim3 grid(n_chunks, BH);
  chunk_grad_sums_kernel<<<grid, kGThreads, SumSmem::kBytes, st>>>(tq, tk, tv, tdo, rowc, wsS, wsG, T, n_chunks, rf,
                                                                    wc);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // exclusive prefix over the chunks of each (b,h): S before chunk c, and
  // (records in reverse order) G after chunk c
  ChunkPlan pl{};
  pl.BH = BH;
  pl.T = T;
  pl.p = 16;
  pl.P = 256;
  pl.dv = kDV;
  pl.ld = kDV + 4;
  pl.C = kTile;
  pl.Ls = kTile;
  pl.G = n_chunks;
  pl.layout = kRecPackedT;
  pl.record_floats = (size_t)rf;
  if ((e = launch_state_scan(wsS, pl, n_chunks, nullptr, nullptr, nullptr, nullptr, st)) != cudaSuccess) return e;
  if ((e = launch_state_scan(wsG, pl, n_chunks, nullptr, nullptr, nullptr, nullptr, st)) != cudaSuccess) return e;
  chunk_grad_inter_kernel<<<grid, kGThreads, InterSmem::kBytes, st>>>(
      tq, tk, tv, tdo, rowc, wsS, wsG, static_cast<__nv_bfloat16*>(dq), static_cast<__nv_bfloat16*>(dk),
      static_cast<__nv_bfloat16*>(dv), T, n_chunks, rf, wc);
  return cudaGetLastError();
}

}  // namespace kata
