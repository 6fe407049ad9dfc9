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
// token with the chunks before it (dq) or after it (dk, dv) through two
// running states, walked the way the forward's readout walks S~:
//   1. chunk_grad_sums_kernel (G > 1 super-chunks): per super-chunk the sums
//        S~^T = sum_c [V_c | 1]^T psi~(K_c)        (the forward's state)
//        G~^T = sum_c [dN_c | dD_c]^T psi~(Q_c)
//      over its chunks, written as records (the G~ ones in reverse order);
//   2. the scan (scan.cu) over both record sequences: the state entering
//      each super-chunk, S~ from the left and G~ from the right;
//   3. chunk_grad_walk_kernel: one CTA per (super-chunk, head, direction).
//      The S walk goes forward through the chunks; per chunk c, against the
//      bf16 copy of S~ entering it,
//        X = dN_c S~                   -> dq_t += 2 dPsi(X_t + dD_t z~) q_t
//      then S~ takes in chunk c.  The G walk goes backward; per chunk c,
//      against the copy of G~ leaving it,
//        Y = V_c G~                    -> dk_s += 2 dPsi(Y_s + g~) k_s
//        Z = psi~(K_c) G~^T            -> dv_s += Z_s
//      then G~ takes in chunk c.  The walks write dq, dk, dv; the diagonal
//      pass adds the pairs inside each chunk to them afterwards.
// Packed coordinates as in chunk_common.cuh: the key side of S~ carries the
// factor 2 off the diagonal, the query side of G~ does not.  Row 64 of each
// state (z~ or g~) is kept in fp32 beside the bf16 copy and added in the
// epilogue, so no product needs a block of dD or ones for it.
//
// The bf16 copy [80 x 144] of a state is the forward's layout: K-major for
// Z's B operand (K = 144 packed coordinates, N = 64 value rows) and, read
// with its atoms along N, MN-major for the B operand of X and Y (K = 64 value
// rows, N = 144), the way psi~ is read as the update's B operand.
#include <cuda.h>

#include "chunk_common.cuh"
#include "kata_internal.h"

namespace kata {

bool make_tmap_bf16(CUtensorMap* map, const void* base, int inner, int T, int BH, int rows);

namespace {

using namespace sm100;
using namespace chunk;

constexpr int kSMCount = 148;

// Scales the bf16 row t of a 128B-swizzled [128 x 64] tile by s in place:
// n of its physical 16-byte chunks, c0, c0 + step, ... (the swizzle only
// permutes a row's chunks, and the scale is the same for the whole row).
// Rows are 128 bytes apart, so the threads of a warp (consecutive rows) start
// at different chunks (rotated by t): with the same chunk in every row all 32
// accesses of an instruction fell into the same four banks.
__device__ __forceinline__ void scale_row_chunks_sw128(uint8_t* tile, int t, float s, int c0, int n, int step) {
  uint4* row = reinterpret_cast<uint4*>(tile + t * 128);
#pragma unroll
  for (int j = 0; j < n; ++j) {
    const int c = (c0 + step * (j + t)) & 7;
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

// Column 0 of row t of a zeroed 128B-swizzled [128 x 64] block := x (bf16);
// the rest of the row stays zero.  As the second M atom of the MN-major A
// operand [dN | block]^T it makes row 64 of the update dD^T psi~(Q).
__device__ __forceinline__ void set_col0_sw128(uint8_t* blk, int t, float x) {
  *reinterpret_cast<uint4*>(blk + t * 128 + ((t & 7) << 4)) = make_uint4(pack_bf16x2(x, 0.f), 0u, 0u, 0u);
}

__device__ __forceinline__ void zero_block(uint8_t* blk, int tid, int nthreads) {
  uint4* w = reinterpret_cast<uint4*>(blk);
  for (int x = tid; x < kOnesBytes / 16; x += nthreads) w[x] = make_uint4(0u, 0u, 0u, 0u);
}

// (-delta, 2/D) of token t of head bh; zero past T
__device__ __forceinline__ float2 load_rowc(const float2* rowc, int bh, int T, int t) {
  return t < T ? rowc[(size_t)bh * T + t] : make_float2(0.f, 0.f);
}

// ---------------------------------------------------------------------------
// 1. per-super-chunk sums of both states
// ---------------------------------------------------------------------------
constexpr int kSumThreads = 320;  // warp 0 TMA, warp 1 MMA, warps 2-9 operands (two threads a token)
constexpr int kSumStages = 5;

struct SumSmem {
  static constexpr int kStage = kVBytes + kQKBytes;                 // [V | K] or [dO | Q]
  static constexpr int offStage = 0;
  static constexpr int offBlk = offStage + kSumStages * kStage;      // ones, or a dD block per psi~ buffer
  static constexpr int offPsi = offBlk + 2 * kOnesBytes;             // 2 psi~ buffers
  static constexpr int offBar = offPsi + 2 * kPsiBytes;
  static constexpr int kBars = 2 * kSumStages + 4 + 1;
  static constexpr int offMisc = offBar + kBars * 8;
  static constexpr int kBytes = offMisc + 16 + 1024;
};

// blockIdx.z = 0: super-chunk g = blockIdx.x (0 .. G-2), its S~ sum into
// record (bh, g); blockIdx.z = 1: super-chunk g = blockIdx.x + 1 (1 .. G-1),
// its G~ sum into record (BH + bh, G - 1 - g).  The last super-chunk's S~ sum
// and the first one's G~ sum enter no other super-chunk and are not formed.
__global__ void __launch_bounds__(kSumThreads, 1)
    chunk_grad_sums_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                           const float2* __restrict__ rowc, float* __restrict__ ws, int T, int Ls, int G,
                           long long record_floats, WaitCtl wc) {
  using L = SumSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::offBar);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + kSumStages;
  uint64_t* psi_full = kv_empty + kSumStages;  // [2]
  uint64_t* psi_empty = psi_full + 2;          // [2]
  uint64_t* acc_done = psi_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::offMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::offMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool grad = blockIdx.z == 1;
  const int g = grad ? (int)blockIdx.x + 1 : (int)blockIdx.x, bh = blockIdx.y, BH = gridDim.y;
  const int t0 = g * Ls;
  const int n_chunks = (min(T, t0 + Ls) - t0 + kTile - 1) / kTile;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSumStages; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(psi_full + b, 256);
      mbar_init(psi_empty + b, 1);
    }
    mbar_init(acc_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (grad) {
    zero_block(smem + L::offBlk, threadIdx.x, kSumThreads);
    zero_block(smem + L::offBlk + kOnesBytes, threadIdx.x, kSumThreads);
  } else {
    fill_ones(smem + L::offBlk, threadIdx.x, kSumThreads);
  }
  fence_proxy_async_smem();
  if (warp == 1) tmem_alloc(tmem_holder, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitEnv env{wc.status, abort_flag, wc.limit};

  if (warp == 0) {
    if (lane == 0) {
      const CUtensorMap* big = grad ? &tm_do : &tm_v;
      const CUtensorMap* small = grad ? &tm_q : &tm_k;
      prefetch_tmap(big);
      prefetch_tmap(small);
      int issued = 0;
      for (int c = 0; c < n_chunks; ++c) {
        const int st = c % kSumStages;
        if (!mbar_wait(kv_empty + st, ((c / kSumStages) & 1) ^ 1, env)) break;
        uint8_t* base = smem + L::offStage + st * L::kStage;
        mbar_arrive_expect_tx(kv_full + st, L::kStage);
        tma_load_3d(base, big, kv_full + st, 0, t0 + c * kTile, bh);
        tma_load_3d(base + kVBytes, small, kv_full + st, 0, t0 + c * kTile, bh);
        ++issued;
      }
      for (int c = issued - kSumStages < 0 ? 0 : issued - kSumStages; c < issued; ++c)
        mbar_wait_drain(kv_full + c % kSumStages, (c / kSumStages) & 1);
    }
  } else if (warp == 1) {
    // whole warp; one elected lane issues
    constexpr uint32_t id_u = idesc_bf16(128, kNP, true, true);  // A = [X | w]^T (MN-major), B = psi~ (N-major)
    const uint32_t sStage = smem_u32(smem + L::offStage), sBlk = smem_u32(smem + L::offBlk);
    const uint64_t dpsi = smem_desc(smem_u32(smem + L::offPsi), kPsiAtom, 256, kSw32);
    for (int c = 0; c < n_chunks; ++c) {
      const int st = c % kSumStages, pb = c & 1;
      if (!mbar_wait_w(kv_full + st, (c / kSumStages) & 1, env)) break;
      if (!mbar_wait_w(psi_full + pb, (c >> 1) & 1, env)) break;
      tc_fence_after();
      const uint64_t da = desc_vones(sStage + st * L::kStage, sBlk + (grad ? pb * kOnesBytes : 0));
      const uint64_t db = desc_add(dpsi, pb * kPsiBytes);
#pragma unroll
      for (int ks = 0; ks < kTile / 16; ++ks)
        mma_ss_w(tmem, desc_add(da, ks * 2048), desc_add(db, ks * 512), id_u, (c > 0 || ks > 0) ? 1u : 0u);
      mma_commit_w(psi_empty + pb);
      mma_commit_w(kv_empty + st);
    }
    mma_commit_w(acc_done);
    mbar_wait_drain(acc_done, 0);
  } else {
    // warps 2-9: token (warp - 2) % 4 * 32 + lane, half (warp - 2) / 4 of its
    // packed psi~ (and, for G~, of its dO row)
    const int tid = ((warp - 2) & 3) * 32 + lane;
    const int half = (warp - 2) >> 2;
    const int quarter = warp % 4;
    const int d = quarter * 32 + lane;  // TMEM lane = record row
    bool ok = true;
    float2 rc_next = grad && n_chunks > 0 ? load_rowc(rowc, bh, T, t0 + tid) : make_float2(0.f, 0.f);
    for (int c = 0; c < n_chunks; ++c) {
      const int st = c % kSumStages, pb = c & 1;
      const float2 rc = rc_next;
      if (grad && c + 1 < n_chunks) rc_next = load_rowc(rowc, bh, T, t0 + (c + 1) * kTile + tid);
      if (!mbar_wait_w(kv_full + st, (c / kSumStages) & 1, env)) {
        ok = false;
        break;
      }
      if (c >= 2 && !mbar_wait_w(psi_empty + pb, ((c >> 1) - 1) & 1, env)) {
        ok = false;
        break;
      }
      uint8_t* stage = smem + L::offStage + st * L::kStage;
      __nv_bfloat162 u[8];
      load_row_sw<1>(stage + kVBytes, tid, u);
      uint32_t w[kNPW / 2];
      uint8_t* dst = smem + L::offPsi + pb * kPsiBytes;
      if (half == 0) {
        if (grad) packed_psi_half<false, 0>(u, w);
        else packed_psi_half<true, 0>(u, w);
        store_psi_k_half<0>(dst, tid, w);
      } else {
        if (grad) packed_psi_half<false, 1>(u, w);
        else packed_psi_half<true, 1>(u, w);
        store_psi_k_half<1>(dst, tid, w);
      }
      if (grad) {
        // dN = dO / D in place (this thread's half of the row); dD into
        // column 0 of the block that follows dN in the A operand
        scale_row_chunks_sw128(stage, tid, 0.5f * rc.y, half, 4, 2);  // chunks of parity `half`
        if (half == 0) set_col0_sw128(smem + L::offBlk + pb * kOnesBytes, tid, 0.5f * rc.x * rc.y);
      }
      fence_proxy_async_smem();
      mbar_arrive(psi_full + pb);
    }
    // record rows 0..64 live in TMEM lanes 0..64: warps of lane quarters 0-2
    // load (the load is warp-collective), lanes below 65 store
    if (ok && warp < 6 && quarter < 3 && n_chunks > 0 && mbar_wait_w(acc_done, 0, env)) {
      tc_fence_after();
      const size_t seq = grad ? (size_t)BH + bh : (size_t)bh;
      const int rec = grad ? G - 1 - g : g;
      float* row = ws + (seq * G + rec) * record_floats + (size_t)min(d, kRecRows - 1) * kNP;
      state_lane_to_global(tmem + ((uint32_t)(quarter * 32) << 16), row, d < kRecRows);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ---------------------------------------------------------------------------
// 3. the walks
// ---------------------------------------------------------------------------
// Warp roles (448 threads):
//   warp 0       TMA: [dO | V | K | Q] tiles of each chunk into a 2-stage ring
//   warp 1       TMEM allocator; MMA issue (the whole warp, one elected lane)
//   warps 2-5    epilogue: token m = lane quarter * 32 + lane of the chunk
//   warps 6-9    S walk: psi~(K); G walk: psi~(Q), formed and stored once
//                the update by the chunk before has read the buffer; then
//                half 0 of the state copy
//   warps 10-13  dN in place (and for the G walk dD, and psi~(K) into TMEM);
//                then half 1 of the state copy
// MMA order per chunk: the products against the copy of the state entering
// the chunk (X, or Y and Z), then the state update by the chunk.  The copy
// for the next chunk is refreshed in place once the update has landed (the
// products, issued before it, have then read it).  Row 64 of the state goes
// to one of two fp32 vectors, each with its own barrier for the epilogue.
// TMEM is handed over a chunk at a time: the operand warps read the state
// (and the G walk stores psi~(K)) only after the epilogue has released the
// products of the chunk before (acc_free).  With those accesses overlapping
// the epilogue's reads of the same lane quarter, the epilogue read wrong
// products for whole lane quarters in some runs (B4 H8 T1000, one
// super-chunk of 8 chunks per walk); with this hand-over every run is
// bitwise the same.
constexpr int kWalkThreads = 448;
// Three stages of the ring, so that the next chunks' loads are in flight
// while a chunk is worked on; that leaves room for one psi~ buffer, which the
// operand warps fill once the update by the chunk before has read it.  Measured at B1 H16 T131072 (backward): 2 stages and 2 psi~
// buffers 1.99 ms.
constexpr int kWalkStages = 3;

struct WalkSmem {
  static constexpr int kStage = 2 * kVBytes + 2 * kQKBytes;  // [dO | V | K | Q]
  static constexpr int offStage = 0;
  static constexpr int offBlk = offStage + kWalkStages * kStage;  // ones (S walk) or 2 dD blocks (G walk)
  static constexpr int offPsi = offBlk + 2 * kOnesBytes;          // psi~ buffer
  static constexpr int offSB = offPsi + kPsiBytes;                // bf16 copy of the state
  static constexpr int offZ = offSB + kSBBytes;                   // 2 x 144 fp32: row 64 of the state
  static constexpr int offBar = offZ + 2 * kNP * 4;
  static constexpr int kBars = 2 * kWalkStages + 8;
  static constexpr int offMisc = offBar + kBars * 8;
  static constexpr int kBytes = offMisc + 16 + 1024;
  // TMEM columns (512 allocated)
  static constexpr uint32_t colState = 0;  // S~^T or G~^T, 144
  static constexpr uint32_t colAcc = 160;  // X or Y, 144
  static constexpr uint32_t colZ = 320;    // Z, 64
  static constexpr uint32_t colPK = 384;   // psi~(K) of the G walk, 72
};

// Half `half` of record row `row` (zeros when row is null) -> TMEM lane; also
// into bf16 copy row n when `copy`, and as fp32 into zb when zb is not null.
// Warp-collective (the TMEM stores).
__device__ __forceinline__ void init_state_half(const float* row, uint32_t taddr, uint8_t* sb, int n, bool copy,
                                                float* zb, int half) {
  auto ld4 = [&](int col, uint32_t* r) {
    float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row) v4 = *reinterpret_cast<const float4*>(row + col);
    r[0] = __float_as_uint(v4.x);
    r[1] = __float_as_uint(v4.y);
    r[2] = __float_as_uint(v4.z);
    r[3] = __float_as_uint(v4.w);
    if (zb) *reinterpret_cast<float4*>(zb + col) = v4;
  };
  const int a0 = half == 0 ? 0 : 5;  // first whole atom of the half
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    uint32_t r[16];
#pragma unroll
    for (int e = 0; e < 16; e += 4) ld4(16 * (a0 + a) + e, r + e);
    tmem_st16(taddr + 16 * (a0 + a), r);
    if (copy) store_state_bf16_atom(sb, n, a0 + a, r);
  }
  uint32_t r[8];
  const int col = half == 0 ? 64 : 72;
  ld4(col, r);
  ld4(col + 4, r + 4);
  tmem_st8(taddr + col, r);
  if (copy) store_state_bf16_chunk(sb, n, 4, half, r);
}

// Half `half` of a TMEM lane of the state as fp32 into zb (when `active`).
// Warp-collective.
__device__ __forceinline__ void state_half_to_f32(uint32_t taddr, float* zb, bool active, int half) {
  uint32_t a[32], b[32], c[8];
  if (half == 0) {
    tmem_ld32(taddr, a);
    tmem_ld32(taddr + 32, b);
    tmem_ld8(taddr + 64, c);
  } else {
    tmem_ld8(taddr + 72, c);
    tmem_ld32(taddr + 80, a);
    tmem_ld32(taddr + 112, b);
  }
  tmem_wait_ld();
  if (!active) return;
  auto st4 = [&](int col, const uint32_t* r) {
    *reinterpret_cast<float4*>(zb + col) =
        make_float4(__uint_as_float(r[0]), __uint_as_float(r[1]), __uint_as_float(r[2]), __uint_as_float(r[3]));
  };
  const int ca = half == 0 ? 0 : 80, cc = half == 0 ? 64 : 72;
#pragma unroll
  for (int e = 0; e < 32; e += 4) {
    st4(ca + e, a + e);
    st4(ca + 32 + e, b + e);
  }
  st4(cc, c);
  st4(cc + 4, c + 4);
}

// 2 dPsi(u) u for the symmetric p x p form of the packed gradient row
// r_w + coef * zb[w], r in TMEM columns [taddr, taddr + 144) of this lane:
// off-diagonal packed entries count kFOff times (the entry of one triangle),
// diagonal ones kFDiag times.  Warp-collective (the loads).
template <int kFDiag, int kFOff>
__device__ __forceinline__ void packed_grad_times_u(uint32_t taddr, const float* zb, float coef,
                                                    const float (&u)[16], float (&out)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) out[i] = 0.f;
  // two TMEM loads (32 columns) in flight per wait
#pragma unroll
  for (int b0 = 0; b0 < 9; b0 += 2) {
    uint32_t r[2][16];
#pragma unroll
    for (int bb = 0; bb < 2; ++bb)
      if (b0 + bb < 9) tmem_ld16(taddr + 16 * (b0 + bb), r[bb]);
    tmem_wait_ld();
#pragma unroll
    for (int bb = 0; bb < 2; ++bb) {
      const int b = b0 + bb;
      if (b >= 9) continue;
#pragma unroll
      for (int x = 0; x < 16; x += 4) {
        const float4 z4 = *reinterpret_cast<const float4*>(zb + 16 * b + x);
        const float zv[4] = {z4.x, z4.y, z4.z, z4.w};
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          const int w = 16 * b + x + y;
          const int i = packed_i(w), j = packed_j(w);
          if (i < 0) continue;
          const float gr = fmaf(coef, zv[y], __uint_as_float(r[bb][x + y]));
          if (i == j) {
            out[i] = fmaf((float)kFDiag * gr, u[i], out[i]);
          } else {
            out[i] = fmaf((float)kFOff * gr, u[j], out[i]);
            out[j] = fmaf((float)kFOff * gr, u[i], out[j]);
          }
        }
      }
    }
  }
}

// 16 fp32 values rounded to bf16 and stored at row (32 bytes)
__device__ __forceinline__ void store_bf16_row16(__nv_bfloat16* row, const float (&v)[16]) {
  uint4* p4 = reinterpret_cast<uint4*>(row);
#pragma unroll
  for (int q = 0; q < 2; ++q)
    p4[q] = make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                       pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
}

// blockIdx.z = 0: the S walk of super-chunk blockIdx.x (dq); 1: its G walk
// (dk, dv).  ws holds the scanned records ([2 BH] sequences of G), null when
// G = 1 (both walks then start from zero).
__global__ void __launch_bounds__(kWalkThreads, 1)
    chunk_grad_walk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                           const float2* __restrict__ rowc, const float* __restrict__ ws,
                           __nv_bfloat16* __restrict__ dq, __nv_bfloat16* __restrict__ dk,
                           __nv_bfloat16* __restrict__ dv, int T, int Ls, int G, long long record_floats,
                           WaitCtl wc) {
  using L = WalkSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::offBar);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + kWalkStages;   // MMA commit + 128 epilogue threads
  uint64_t* ops_full = kv_empty + kWalkStages;  // operands and state copy of the chunk (256)
  uint64_t* acc_full = ops_full + 1;            // X, or Y and Z, in TMEM
  uint64_t* acc_free = acc_full + 1;            // the epilogue has read them (128)
  uint64_t* upd_done = acc_free + 1;            // state updated by the chunk
  uint64_t* z_ready = upd_done + 1;             // [2] fp32 row 64 of the state (the 64 threads of quarter 2)
  uint64_t* mma_done = z_ready + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::offMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::offMisc + 4);
  float* zbuf = reinterpret_cast<float*>(smem + L::offZ);  // [2][144]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool gw = blockIdx.z == 1;  // the G walk
  const int g = blockIdx.x, bh = blockIdx.y, BH = gridDim.y;
  const int t0 = g * Ls;
  const int n_chunks = (min(T, t0 + Ls) - t0 + kTile - 1) / kTile;
  // the i-th chunk of the walk
  auto chunk_of = [&](int i) { return gw ? n_chunks - 1 - i : i; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kWalkStages; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1 + 128);
    }
    mbar_init(ops_full, 256);
    mbar_init(acc_full, 1);
    mbar_init(acc_free, 128);
    mbar_init(upd_done, 1);
    for (int b = 0; b < 2; ++b) mbar_init(z_ready + b, 64);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (gw) {
    zero_block(smem + L::offBlk, threadIdx.x, kWalkThreads);
    zero_block(smem + L::offBlk + kOnesBytes, threadIdx.x, kWalkThreads);
  } else {
    fill_ones(smem + L::offBlk, threadIdx.x, kWalkThreads);
  }
  fence_proxy_async_smem();
  if (warp == 1) tmem_alloc(tmem_holder, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitEnv env{wc.status, abort_flag, wc.limit};

  if (warp == 0) {
    // ------------------------------------------------------------- TMA
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      prefetch_tmap(&tm_do);
      int issued = 0;
      for (int i = 0; i < n_chunks; ++i) {
        const int st = i % kWalkStages;
        if (!mbar_wait(kv_empty + st, ((i / kWalkStages) & 1) ^ 1, env)) break;
        uint8_t* base = smem + L::offStage + st * L::kStage;
        mbar_arrive_expect_tx(kv_full + st, L::kStage);
        const int row = t0 + chunk_of(i) * kTile;
        tma_load_3d(base, &tm_do, kv_full + st, 0, row, bh);
        tma_load_3d(base + kVBytes, &tm_v, kv_full + st, 0, row, bh);
        tma_load_3d(base + 2 * kVBytes, &tm_k, kv_full + st, 0, row, bh);
        tma_load_3d(base + 2 * kVBytes + kQKBytes, &tm_q, kv_full + st, 0, row, bh);
        ++issued;
      }
      for (int i = issued - kWalkStages < 0 ? 0 : issued - kWalkStages; i < issued; ++i)
        mbar_wait_drain(kv_full + i % kWalkStages, (i / kWalkStages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA
    constexpr uint32_t id_xy = idesc_bf16(128, kNP, false, true);  // A [128 x 64] K-major, B copy MN-major
    constexpr uint32_t id_z = idesc_bf16(128, kDV, false, false);  // A psi~(K) (TMEM), B copy K-major
    constexpr uint32_t id_u = idesc_bf16(128, kNP, true, true);    // A [X | w]^T MN-major, B psi~ N-major
    const uint32_t sStage = smem_u32(smem + L::offStage), sBlk = smem_u32(smem + L::offBlk);
    const uint32_t sSB = smem_u32(smem + L::offSB);
    const uint64_t dsb_mn = smem_desc(sSB, kSBAtom, 256, kSw32);  // copy as [K = 64 rows x N = 144]
    const uint64_t dsb_k = smem_desc(sSB, 16, 256, kSw32);        // copy as [N = 64 rows x K = 144]
    const uint64_t dpsi = smem_desc(smem_u32(smem + L::offPsi), kPsiAtom, 256, kSw32);
    for (int i = 0; i < n_chunks; ++i) {
      const int st = i % kWalkStages, pb = i & 1;
      const uint32_t sDO = sStage + st * L::kStage, sV = sDO + kVBytes;
      if (!mbar_wait_w(ops_full, i & 1, env)) break;
      if (i > 0 && !mbar_wait_w(acc_free, (i - 1) & 1, env)) break;
      tc_fence_after();
      // products against the copy of the state entering the chunk
      const uint64_t da = smem_desc(gw ? sV : sDO, 16, 1024, kSw128);  // V or dN, K-major
#pragma unroll
      for (int ks = 0; ks < kDV / 16; ++ks)
        mma_ss_w(tmem + L::colAcc, desc_add(da, ks * 32), desc_add(dsb_mn, ks * 512), id_xy, ks > 0);
      if (gw) {
#pragma unroll
        for (int ks = 0; ks < kNP / 16; ++ks)
          mma_ts_w(tmem + L::colZ, tmem + L::colPK + ks * 8, desc_add(dsb_k, ks * kSBAtom), id_z, ks > 0);
      }
      mma_commit_w(acc_full);
      // the state takes in the chunk: S~^T += [V | 1]^T psi~(K), or
      // G~^T += [dN | dD]^T psi~(Q)
      const uint64_t du = gw ? desc_vones(sDO, sBlk + pb * kOnesBytes) : desc_vones(sV, sBlk);
      const uint64_t db = dpsi;
#pragma unroll
      for (int ks = 0; ks < kTile / 16; ++ks)
        mma_ss_w(tmem + L::colState, desc_add(du, ks * 2048), desc_add(db, ks * 512), id_u, 1);
      mma_commit_w(upd_done);
      mma_commit_w(kv_empty + st);
    }
    mma_commit_w(mma_done);
    mbar_wait_drain(mma_done, 0);
  } else if (warp < 6) {
    // ------------------------------------------------------------- epilogue
    // writes every row of its walk (the diagonal pass adds to them later);
    // the S walk's per-row constants are loaded a chunk ahead
    const int quarter = warp % 4;
    const int m = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    float2 rc_next = !gw && n_chunks > 0 ? load_rowc(rowc, bh, T, t0 + chunk_of(0) * kTile + m) : make_float2(0.f, 0.f);
    for (int i = 0; i < n_chunks; ++i) {
      const int st = i % kWalkStages;
      const int t = t0 + chunk_of(i) * kTile + m;
      const float2 rc = rc_next;
      if (!gw && i + 1 < n_chunks) rc_next = load_rowc(rowc, bh, T, t0 + chunk_of(i + 1) * kTile + m);
      if (!mbar_wait_w(kv_full + st, (i / kWalkStages) & 1, env)) break;
      // this token's q (S walk) or k (G walk) row, then the stage may go
      const uint8_t* tile = smem + L::offStage + st * L::kStage + 2 * kVBytes + (gw ? 0 : kQKBytes);
      __nv_bfloat162 u2[8];
      load_row_sw<1>(tile, m, u2);
      mbar_arrive(kv_empty + st);
      float u[16];
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        u[2 * x] = __low2float(u2[x]);
        u[2 * x + 1] = __high2float(u2[x]);
      }
      const bool live = t < T;
      const size_t r = (size_t)bh * T + (live ? t : 0);
      const float* zb = zbuf + (i & 1) * kNP;
      if (!mbar_wait_w(z_ready + (i & 1), (i >> 1) & 1, env) || !mbar_wait_w(acc_full, i & 1, env)) break;
      tc_fence_after();
      float gr[16];
      if (!gw) {
        packed_grad_times_u<2, 1>(lane_base + L::colAcc, zb, 0.5f * rc.x * rc.y, u, gr);
        tc_fence_before();
        mbar_arrive(acc_free);
        if (live) store_bf16_row16(dq + r * 16, gr);
      } else {
        packed_grad_times_u<2, 2>(lane_base + L::colAcc, zb, 1.f, u, gr);
        // Z, 32 columns at a time, packed to bf16 before the accumulators
        // are released
        uint4 zv[8];
#pragma unroll
        for (int hb = 0; hb < 2; ++hb) {
          uint32_t za[32];
          tmem_ld32(lane_base + L::colZ + 32 * hb, za);
          tmem_wait_ld();
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const uint32_t* e = za + 8 * q4;
            zv[4 * hb + q4] = make_uint4(pack_bf16x2(__uint_as_float(e[0]), __uint_as_float(e[1])),
                                         pack_bf16x2(__uint_as_float(e[2]), __uint_as_float(e[3])),
                                         pack_bf16x2(__uint_as_float(e[4]), __uint_as_float(e[5])),
                                         pack_bf16x2(__uint_as_float(e[6]), __uint_as_float(e[7])));
          }
        }
        tc_fence_before();
        mbar_arrive(acc_free);
        if (live) {
          store_bf16_row16(dk + r * 16, gr);
          uint4* dvr = reinterpret_cast<uint4*>(dv + r * kDV);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) dvr[q4] = zv[q4];
        }
      }
    }
  } else {
    // ------------------------------------------------------------- operands and state copies
    const bool groupA = warp < 10;
    const int half = groupA ? 0 : 1;
    const int quarter = warp % 4;
    const int m = quarter * 32 + lane;  // token of the chunk / TMEM lane = state row
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    uint8_t* sb = smem + L::offSB;
    // group A: the row of the i-th chunk of the walk that psi~ is formed from
    // (k for the S walk, key side; q for the G walk, query side), read from
    // its landed stage; psi~ is formed and stored once the update by the
    // chunk before has read the buffer (holding the 72 words across the waits
    // would spill)
    __nv_bfloat162 u_psi[8];
    auto load_psi_row = [&](int i) {
      const uint8_t* ktile = smem + L::offStage + (i % kWalkStages) * L::kStage + 2 * kVBytes;
      load_row_sw<1>(gw ? ktile + kQKBytes : ktile, m, u_psi);
    };
    auto store_psi = [&]() {
      uint32_t w[kNPW];
      if (gw) packed_psi<false>(u_psi, w);
      else packed_psi<true>(u_psi, w);
      store_psi_k(smem + L::offPsi, m, w);
    };
    // group B: the other operands of the i-th chunk; false if a wait gave up
    auto operands_b = [&](int i, float2 rc) -> bool {
      const int st = i % kWalkStages, pb = i & 1;
      uint8_t* stage = smem + L::offStage + st * L::kStage;
      scale_row_chunks_sw128(stage, m, 0.5f * rc.y, 0, 8, 1);  // dN = dO / D
      if (!gw) return true;
      set_col0_sw128(smem + L::offBlk + pb * kOnesBytes, m, 0.5f * rc.x * rc.y);  // dD
      // psi~(K) into TMEM once the Z of chunk i-1 has read the previous one
      // and the epilogue has read the products of chunk i-1
      __nv_bfloat162 u[8];
      uint32_t w[kNPW];
      load_row_sw<1>(stage + 2 * kVBytes, m, u);
      packed_psi<true>(u, w);
      if (i > 0) {
        if (!mbar_wait_w(acc_free, (i - 1) & 1, env)) return false;
        tc_fence_after();
      }
      store_psi_q_tmem(lane_base + L::colPK, w);
      tmem_wait_st();
      return true;
    };
    // the state entering the walk: the scanned record (rows 0..64) or zero;
    // rows 0..63 also into the bf16 copy, row 64 (z~ or g~) into zbuf[0].
    // After the scan this kernel is its programmatic dependent.
    griddep_wait();
    if (quarter < 3) {
      const int d = min(m, kRecRows - 1);
      const float* row = nullptr;
      if (ws) {
        const size_t seq = gw ? (size_t)BH + bh : (size_t)bh;
        const int rec = gw ? G - 1 - g : g;
        row = ws + (seq * G + rec) * record_floats + (size_t)d * kNP;
      }
      init_state_half(row, lane_base + L::colState, sb, m, m < kDV, m == kDV ? zbuf : nullptr, half);
    }
    if (quarter == 2) mbar_arrive(z_ready);
    // group B's per-row constants, loaded a chunk ahead
    auto rc_of = [&](int i) {
      return !groupA && i < n_chunks ? load_rowc(rowc, bh, T, t0 + chunk_of(i) * kTile + m) : make_float2(0.f, 0.f);
    };
    float2 rc_cur = rc_of(0), rc_nxt = rc_of(1);
    bool ok = n_chunks > 0 && mbar_wait_w(kv_full, 0, env);
    if (ok && groupA) {
      load_psi_row(0);
      store_psi();
    }
    if (ok && !groupA) ok = operands_b(0, rc_cur);
    tmem_wait_st();  // the state's TMEM stores land before the first update reads them
    fence_proxy_async_smem();
    tc_fence_before();
    if (ok) mbar_arrive(ops_full);
    for (int i = 0; ok && i + 1 < n_chunks; ++i) {
      const int st1 = (i + 1) % kWalkStages;
      rc_cur = rc_nxt;
      rc_nxt = rc_of(i + 2);
      if (!mbar_wait_w(kv_full + st1, ((i + 1) / kWalkStages) & 1, env)) break;
      if (groupA) load_psi_row(i + 1);
      else if (!operands_b(i + 1, rc_cur)) break;
      // the state after chunk i: this group's half of the copy (rows 0..63)
      // and of row 64 in fp32, for chunk i+1, once the epilogue has read the
      // products of chunk i out of TMEM (see the class comment); group A's
      // psi~ into the buffer the update by chunk i has read
      if (!mbar_wait_w(upd_done, i & 1, env) || !mbar_wait_w(acc_free, i & 1, env)) break;
      tc_fence_after();
      if (groupA) store_psi();
      if (quarter < 2) {
        state_half_to_bf16(lane_base + L::colState, sb, m, true, half);
      } else if (quarter == 2) {
        state_half_to_f32(lane_base + L::colState, zbuf + ((i + 1) & 1) * kNP, lane == 0, half);
        mbar_arrive(z_ready + ((i + 1) & 1));
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(ops_full);
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

ChunkPlan chunk_bwd_plan(int BH, int T) {
  // Both walks of every super-chunk run at once, 2 BH G CTAs, one per SM at a
  // time.  G (at most 16, so that the records scan in registers) is chosen by
  // a cost in chunk steps on the busiest SM: waves x (chunks per walk + 2 for
  // a CTA's set-up and drain), plus for G > 1 the sums pass (a sums step costs
  // about half a walk step) and the scan.
  ChunkPlan pl{};
  pl.BH = BH;
  pl.T = T;
  pl.p = 16;
  pl.P = 256;
  pl.dv = kDV;
  pl.ld = kDV + 4;
  pl.C = kTile;
  pl.layout = kRecPackedT;
  pl.record_floats = (size_t)kRecRows * kNP;
  const long long tiles = (T + kTile - 1) / kTile;
  auto waves = [](long long units) { return (units + kSMCount - 1) / kSMCount; };
  long long best = -1, bestG = 1;
  for (long long Gc = 1; Gc <= 16 && Gc <= (tiles > 0 ? tiles : 1); ++Gc) {
    const long long per = (tiles + Gc - 1) / Gc;
    const long long Geff = (tiles + per - 1) / per;
    long long cost = 2 * waves(2 * (long long)BH * Geff) * (per + 2);  // in half steps
    if (Geff > 1) cost += waves(2 * (long long)BH * (Geff - 1)) * (per + 4) + 4;
    if (best < 0 || cost < best) {
      best = cost;
      bestG = Gc;
    }
  }
  const long long per = tiles > 0 ? (tiles + bestG - 1) / bestG : 1;
  pl.Ls = (int)(per * kTile);
  pl.G = T > 0 ? (T + pl.Ls - 1) / pl.Ls : 0;
  pl.workspace_bytes = pl.G > 1 ? 2 * (size_t)BH * pl.G * pl.record_floats * sizeof(float) : 0;
  return pl;
}

size_t chunk_bwd_records_bytes(int BH, int T) { return chunk_bwd_plan(BH, T).workspace_bytes; }

cudaError_t launch_chunk_bwd_inter_sm100(const void* q, const void* k, const void* v, const void* dO,
                                         const float2* rowc, float* records, void* dq, void* dk, void* dv, int BH,
                                         int T, const WaitCtl& wc, cudaStream_t st) {
  const int n_chunks = (T + kTile - 1) / kTile;
  if (n_chunks < 2) return cudaSuccess;  // no pair crosses a chunk boundary
  const ChunkPlan pl = chunk_bwd_plan(BH, T);
  CUtensorMap tq, tk, tv, tdo;
  if (!make_tmap_bf16(&tq, q, 16, T, BH, kTile) || !make_tmap_bf16(&tk, k, 16, T, BH, kTile) ||
      !make_tmap_bf16(&tv, v, kDV, T, BH, kTile) || !make_tmap_bf16(&tdo, dO, kDV, T, BH, kTile))
    return cudaErrorInvalidValue;
  cudaError_t e =
      cudaFuncSetAttribute(chunk_grad_sums_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SumSmem::kBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(chunk_grad_walk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, WalkSmem::kBytes);
  if (e != cudaSuccess) return e;
  const long long rf = (long long)pl.record_floats;
  const dim3 wgrid(pl.G, BH, 2);
  auto* dqb = static_cast<__nv_bfloat16*>(dq);
  auto* dkb = static_cast<__nv_bfloat16*>(dk);
  auto* dvb = static_cast<__nv_bfloat16*>(dv);
  if (pl.G > 1) {
    if (!records) return cudaErrorInvalidValue;
    chunk_grad_sums_kernel<<<dim3(pl.G - 1, BH, 2), kSumThreads, SumSmem::kBytes, st>>>(tq, tk, tv, tdo, rowc,
                                                                                          records, T, pl.Ls, pl.G,
                                                                                          rf, wc);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // exclusive prefix over the super-chunks of each of the 2 BH sequences:
    // S~ entering super-chunk g, and (records in reverse order) G~ leaving it
    ChunkPlan both = pl;
    both.BH = 2 * BH;
    if ((e = launch_state_scan(records, both, pl.G - 1, nullptr, nullptr, nullptr, nullptr, st)) != cudaSuccess)
      return e;
    return launch_pdl(chunk_grad_walk_kernel, wgrid, dim3(kWalkThreads), (size_t)WalkSmem::kBytes, st, tq, tk, tv,
                      tdo, rowc, (const float*)records, dqb, dkb, dvb, T, pl.Ls, pl.G, rf, wc);
  }
  chunk_grad_walk_kernel<<<wgrid, kWalkThreads, WalkSmem::kBytes, st>>>(tq, tk, tv, tdo, rowc, nullptr, dqb, dkb,
                                                                        dvb, T, pl.Ls, pl.G, rf, wc);
  return cudaGetLastError();
}

}  // namespace kata
