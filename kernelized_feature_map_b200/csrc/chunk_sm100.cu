// chunk_sm100.cu -- exact O(T) chunked-state KATA forward on tcgen05 / TMEM
// (bf16 inputs, p = 16), the second operating point of the gist.science
// technical summary, sec. 2.3 ("Chunked Parallelism": intra-chunk attention
// on tensor cores, inter-chunk state propagation by an associative scan).
//
// The sequence of every (b,h) is cut into super-chunks of Ls tokens (a
// multiple of the 128-token chunk).  Three launches:
//
//  1. chunk_state_kernel     per super-chunk g: A_g = sum_t psi(k_t) [v_t | 1]^T
//                            (P = 256 state rows x (dv + 1) columns, fp32),
//                            accumulated chunk by chunk in TMEM by tcgen05.mma
//                            with A = psi(K_c)^T formed in shared memory;
//  2. state_scan_kernel      (scan.cu) exclusive prefix over g, depth O(log G);
//  3. chunk_readout_kernel   per super-chunk, per 128-token chunk c:
//                              O_c  = psi(Q_c) . S_run          (readout)
//                                   + W_c [V_c | 1],  W = (Q_c K_c^T)^2 masked
//                              S_run += psi(K_c)^T [V_c | 1]     (advance)
//                              o_c = O_c[:, :dv] / O_c[:, dv]
//                            with S_run starting at the scanned prefix.  S_run
//                            lives in TMEM in fp32; a bf16 copy in shared
//                            memory is the B operand of the next readout.
//
// psi(u) = vec(u u^T) is formed on chip only: psi(q) rows go straight into
// TMEM as the A operand of the readout, psi(k) rows into shared memory as the
// (M-major) A operand of the state update.  Products of two bf16 values are
// exact in fp32, so forming them with bf16x2 multiplies rounds each entry
// once, exactly as rounding the fp32 product would.
//
// The denominator shares every MMA with the numerator: the value operand is
// extended by a block of ones ([V | 1]), so z = sum psi(k) is accumulated in
// 16 identical TMEM columns next to the state, and D_t = psi(q_t)^T z plus
// the intra-chunk weights lands next to the numerator.
#include <cuda.h>

#include "kata_internal.h"
#include "sm100.cuh"

namespace kata {

bool make_tmap_bf16(CUtensorMap* map, const void* base, int inner, int T, int BH, int rows);

namespace {

using namespace sm100;

constexpr int kTile = 128;     // tokens per chunk / MMA M
constexpr int kP = 256;        // psi width for p = 16
constexpr int kPsiBytes = kP * kTile * 2;  // psi(K_c) tile in shared memory: 64 KiB

// psi(K_c)^T as an M-major (state index contiguous) operand with 128-byte
// swizzle: [atom a = state rows 64a..64a+63][token][64 x bf16].
constexpr uint32_t kPsiLbo = kTile * 128;  // between 64-row atoms
constexpr uint32_t kPsiSbo = 1024;         // between 8-token groups

__device__ __forceinline__ uint32_t psi_store_offset(int token, int atom, int chunk) {
  return (uint32_t)atom * kPsiLbo + (uint32_t)token * 128u + (uint32_t)((chunk ^ (token & 7)) << 4);
}

// Load one 16-element bf16 row (32 bytes) as 8 bf16x2 words; zeros if !valid.
__device__ __forceinline__ void load_row16(const __nv_bfloat16* src, bool valid, __nv_bfloat162 (&u)[8]) {
  uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
  if (valid) {
    a = __ldg(reinterpret_cast<const uint4*>(src));
    b = __ldg(reinterpret_cast<const uint4*>(src) + 1);
  }
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int x = 0; x < 8; ++x) u[x] = *reinterpret_cast<const __nv_bfloat162*>(&w[x]);
}

__device__ __forceinline__ uint32_t as_u32(__nv_bfloat162 h) { return *reinterpret_cast<uint32_t*>(&h); }

// psi(k) of one token into the psi(K_c) tile (row = token).
__device__ __forceinline__ void write_psi_k(uint8_t* psi, int token, const __nv_bfloat162 (&u)[8]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const __nv_bfloat16 ui = (i & 1) ? u[i >> 1].y : u[i >> 1].x;
    const __nv_bfloat162 b2 = __halves2bfloat162(ui, ui);
#pragma unroll
    for (int h = 0; h < 2; ++h) {  // j = 8h .. 8h+7
      uint4 v;
      v.x = as_u32(__hmul2(b2, u[4 * h + 0]));
      v.y = as_u32(__hmul2(b2, u[4 * h + 1]));
      v.z = as_u32(__hmul2(b2, u[4 * h + 2]));
      v.w = as_u32(__hmul2(b2, u[4 * h + 3]));
      const int atom = i >> 2, chunk = (i & 3) * 2 + h;
      *reinterpret_cast<uint4*>(psi + psi_store_offset(token, atom, chunk)) = v;
    }
  }
}

// psi(q) of one query row into TMEM columns [col, col+128) of this thread's lane.
__device__ __forceinline__ void write_psi_q_tmem(uint32_t taddr, const __nv_bfloat162 (&u)[8]) {
#pragma unroll
  for (int i2 = 0; i2 < 8; ++i2) {  // two psi rows (i = 2*i2, 2*i2+1) per 16-column store
    uint32_t w[16];
#pragma unroll
    for (int ii = 0; ii < 2; ++ii) {
      const __nv_bfloat16 ui = ii ? u[i2].y : u[i2].x;
      const __nv_bfloat162 b2 = __halves2bfloat162(ui, ui);
#pragma unroll
      for (int x = 0; x < 8; ++x) w[8 * ii + x] = as_u32(__hmul2(b2, u[x]));
    }
    tmem_st16(taddr + 16 * i2, w);
  }
}

template <int DV>
struct ChunkCfg {
  static constexpr int kSRW = DV + 16;                 // TMEM columns per 128-row state block
  static constexpr int kVBytes = kTile * DV * 2;
  static constexpr int kQKBytes = kTile * 16 * 2;
  static constexpr Swizzle kVSw = (DV == 64) ? kSw128 : kSw32;
  static constexpr uint32_t kVSbo = 8 * DV * 2;
  static constexpr uint32_t kVKStep = 16 * DV * 2;     // 16 tokens
  // bf16 copy of the state: SV [256 rows x DV] and SZ [256 rows x 16], both
  // N-major (columns contiguous) B operands of the readout
  static constexpr int kSVBytes = kP * DV * 2;
  static constexpr int kSZBytes = kP * 16 * 2;
  static constexpr uint32_t kSVSbo = 8 * DV * 2;
  static constexpr uint32_t kSVKStep = 16 * DV * 2;    // 16 state rows
};

// Store one state row (DV values + z) as bf16 into SV / SZ.
template <int DV>
__device__ __forceinline__ void store_state_row_bf16(uint8_t* sv, uint8_t* sz, int r, const float* vals, float zval) {
  if constexpr (DV == 64) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint4 w;
      w.x = pack_bf16x2(vals[8 * c + 0], vals[8 * c + 1]);
      w.y = pack_bf16x2(vals[8 * c + 2], vals[8 * c + 3]);
      w.z = pack_bf16x2(vals[8 * c + 4], vals[8 * c + 5]);
      w.w = pack_bf16x2(vals[8 * c + 6], vals[8 * c + 7]);
      *reinterpret_cast<uint4*>(sv + r * 128 + ((c ^ (r & 7)) << 4)) = w;
    }
  } else {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      uint4 w;
      w.x = pack_bf16x2(vals[8 * c + 0], vals[8 * c + 1]);
      w.y = pack_bf16x2(vals[8 * c + 2], vals[8 * c + 3]);
      w.z = pack_bf16x2(vals[8 * c + 4], vals[8 * c + 5]);
      w.w = pack_bf16x2(vals[8 * c + 6], vals[8 * c + 7]);
      *reinterpret_cast<uint4*>(sv + r * 32 + ((c ^ ((r >> 2) & 1)) << 4)) = w;
    }
  }
  const uint32_t zz = pack_bf16x2(zval, zval);
  const uint4 w = make_uint4(zz, zz, zz, zz);
#pragma unroll
  for (int c = 0; c < 2; ++c) *reinterpret_cast<uint4*>(sz + r * 32 + ((c ^ ((r >> 2) & 1)) << 4)) = w;
}

// Read DV + 1 state columns of this thread's TMEM lane at column `col`.
template <int DV>
__device__ __forceinline__ void load_state_row_tmem(uint32_t taddr, float* vals, float& zval) {
  uint32_t zb;
  if constexpr (DV == 64) {
    uint32_t r0[32], r1[32];
    tmem_ld32(taddr, r0);
    tmem_ld32(taddr + 32, r1);
    tmem_ld1(taddr + 64, zb);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      vals[e] = __uint_as_float(r0[e]);
      vals[32 + e] = __uint_as_float(r1[e]);
    }
  } else {
    uint32_t r0[16];
    tmem_ld16(taddr, r0);
    tmem_ld1(taddr + 16, zb);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 16; ++e) vals[e] = __uint_as_float(r0[e]);
  }
  zval = __uint_as_float(zb);
}

// Write DV state columns then 16 copies of z into this thread's TMEM lane.
template <int DV>
__device__ __forceinline__ void store_state_row_tmem(uint32_t taddr, const float* vals, float zval) {
#pragma unroll
  for (int c = 0; c < DV / 16; ++c) {
    uint32_t w[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) w[e] = __float_as_uint(vals[16 * c + e]);
    tmem_st16(taddr + 16 * c, w);
  }
  uint32_t w[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) w[e] = __float_as_uint(zval);
  tmem_st16(taddr + DV, w);
}

// ===========================================================================
// 1. per-super-chunk state sums
// ===========================================================================
constexpr int kStateThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 psi(k)
constexpr int kStateStages = 2;

template <int DV>
struct StateSmem {
  using Cfg = ChunkCfg<DV>;
  static constexpr int offPsi = 0;                                   // 2 x 64 KiB
  static constexpr int offV = offPsi + 2 * kPsiBytes;                // stages x V tile
  static constexpr int offOnes = offV + kStateStages * Cfg::kVBytes;
  static constexpr int offBar = offOnes + 512;
  static constexpr int kBars = 2 * kStateStages + 4 + 1;
  static constexpr int offMisc = offBar + kBars * 8;
  static constexpr int kBytes = offMisc + 16 + 1024;
};

template <int DV>
__global__ void __launch_bounds__(kStateThreads, 1)
    chunk_state_kernel(const __grid_constant__ CUtensorMap tm_v, const __nv_bfloat16* __restrict__ k,
                       float* __restrict__ ws, int T, int Ls, int G, int ld, long long record_floats, WaitCtl wc) {
  using Cfg = ChunkCfg<DV>;
  using L = StateSmem<DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::offBar);
  uint64_t* v_full = bars;
  uint64_t* v_empty = v_full + kStateStages;
  uint64_t* psi_full = v_empty + kStateStages;  // [2]
  uint64_t* psi_empty = psi_full + 2;           // [2]
  uint64_t* acc_done = psi_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::offMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::offMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x, bh = blockIdx.y;
  const int t0 = g * Ls;
  const int t1 = min(T, t0 + Ls);
  const int n_chunks = (t1 - t0 + kTile - 1) / kTile;
  constexpr uint32_t kCols = (2 * Cfg::kSRW <= 64) ? 64 : (2 * Cfg::kSRW <= 128 ? 128 : 256);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStateStages; ++s) {
      mbar_init(v_full + s, 1);
      mbar_init(v_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(psi_full + s, 128);
      mbar_init(psi_empty + s, 1);
    }
    mbar_init(acc_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  {
    uint32_t* ones = reinterpret_cast<uint32_t*>(smem + L::offOnes);
    for (int x = threadIdx.x; x < 128; x += kStateThreads) ones[x] = 0x3F803F80u;
    fence_proxy_async_smem();
  }
  if (warp == 1) tmem_alloc(tmem_holder, kCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitEnv env{wc.status, abort_flag, wc.limit};

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tm_v);
      int issued = 0;
      for (int c = 0; c < n_chunks; ++c) {
        const int st = c % kStateStages;
        if (!mbar_wait(v_empty + st, ((c / kStateStages) & 1) ^ 1, env)) break;
        mbar_arrive_expect_tx(v_full + st, Cfg::kVBytes);
        tma_load_3d(smem + L::offV + st * Cfg::kVBytes, &tm_v, v_full + st, 0, t0 + c * kTile, bh);
        ++issued;
      }
      for (int c = issued - kStateStages < 0 ? 0 : issued - kStateStages; c < issued; ++c)
        mbar_wait_drain(v_full + c % kStateStages, (c / kStateStages) & 1, wc.limit);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t id_v = idesc_bf16(128, DV, true, true);
      constexpr uint32_t id_z = idesc_bf16(128, 16, true, false);
      const uint32_t sPsi = smem_u32(smem + L::offPsi), sV = smem_u32(smem + L::offV);
      const uint64_t ones_desc = smem_desc(smem_u32(smem + L::offOnes), 256, 128, kSwNone);
      for (int c = 0; c < n_chunks; ++c) {
        const int st = c % kStateStages, pb = c & 1;
        if (!mbar_wait(v_full + st, (c / kStateStages) & 1, env)) break;
        if (!mbar_wait(psi_full + pb, (c >> 1) & 1, env)) break;
        tc_fence_after();
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
#pragma unroll
          for (int ks = 0; ks < kTile / 16; ++ks) {
            const uint64_t a = smem_desc(sPsi + pb * kPsiBytes + blk * 2 * kPsiLbo + ks * 2048, kPsiLbo, kPsiSbo,
                                         kSw128);
            const uint64_t b = smem_desc(sV + st * Cfg::kVBytes + ks * Cfg::kVKStep, Cfg::kVBytes, Cfg::kVSbo,
                                         Cfg::kVSw);
            const uint32_t acc = (c > 0 || ks > 0) ? 1u : 0u;
            mma_ss(tmem + blk * Cfg::kSRW, a, b, id_v, acc);
            mma_ss(tmem + blk * Cfg::kSRW + DV, a, ones_desc, id_z, acc);
          }
        }
        mma_commit(psi_empty + pb);
        mma_commit(v_empty + st);
      }
      mma_commit(acc_done);
      mbar_wait_drain(acc_done, 0, wc.limit);
    }
  } else {
    // psi(k) producers: thread = token of the chunk, then TMEM lane for the store
    const int tid = threadIdx.x - 64;           // 0..127
    const int quarter = warp % 4;
    const int m = quarter * 32 + lane;          // TMEM lane this thread may read
    const __nv_bfloat16* kb = k + (size_t)bh * T * 16;
    bool ok = true;
    for (int c = 0; c < n_chunks; ++c) {
      const int pb = c & 1;
      if (c >= 2 && !mbar_wait(psi_empty + pb, ((c >> 1) - 1) & 1, env)) {
        ok = false;
        break;
      }
      const int t = t0 + c * kTile + tid;
      __nv_bfloat162 u[8];
      load_row16(kb + (size_t)t * 16, t < t1, u);
      write_psi_k(smem + L::offPsi + pb * kPsiBytes, tid, u);
      fence_proxy_async_smem();
      mbar_arrive(psi_full + pb);
    }
    if (ok && mbar_wait(acc_done, 0, env)) {
      tc_fence_after();
      float* rec = ws + ((size_t)bh * G + g) * record_floats;
#pragma unroll 1
      for (int blk = 0; blk < 2; ++blk) {
        float vals[DV];
        float zval;
        load_state_row_tmem<DV>(tmem + ((uint32_t)(quarter * 32) << 16) + blk * Cfg::kSRW, vals, zval);
        float* row = rec + (size_t)(blk * 128 + m) * ld;
#pragma unroll
        for (int e = 0; e < DV; e += 4) *reinterpret_cast<float4*>(row + e) = make_float4(vals[e], vals[e + 1], vals[e + 2], vals[e + 3]);
        row[DV] = zval;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

// ===========================================================================
// 3. readout
// ===========================================================================
constexpr int kReadThreads = 320;  // warp 0 TMA, 1 MMA, 2-5 weights + output, 6-9 psi + state
constexpr int kReadStages = 2;

template <int DV>
struct ReadSmem {
  using Cfg = ChunkCfg<DV>;
  static constexpr int kStageBytes = 2 * Cfg::kQKBytes + Cfg::kVBytes;
  static constexpr int offPsi = 0;                               // 64 KiB
  static constexpr int offSV = offPsi + kPsiBytes;               // bf16 state, N-major
  static constexpr int offSZ = offSV + Cfg::kSVBytes;
  static constexpr int offStage = (offSZ + Cfg::kSZBytes + 1023) / 1024 * 1024;  // [Q | K | V] per stage
  static constexpr int offOnes = offStage + kReadStages * kStageBytes;
  static constexpr int offBar = offOnes + 512;
  static constexpr int kBars = 2 * kReadStages + 8;
  static constexpr int offMisc = offBar + kBars * 8;
  static constexpr int kBytes = offMisc + 16 + 1024;
  // TMEM columns
  static constexpr uint32_t colRun(int blk) { return (uint32_t)blk * Cfg::kSRW; }
  static constexpr uint32_t colO = 2 * Cfg::kSRW;
  static constexpr uint32_t colD = colO + DV;
  static constexpr uint32_t colS = 256;
  static constexpr uint32_t colPQ = 384;
};

template <int DV>
__global__ void __launch_bounds__(kReadThreads, 1)
    chunk_readout_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const __nv_bfloat16* __restrict__ q,
                         const __nv_bfloat16* __restrict__ k, __nv_bfloat16* __restrict__ o,
                         const float* __restrict__ ws, int T, int Ls, int G, int ld, long long record_floats,
                         WaitCtl wc) {
  using Cfg = ChunkCfg<DV>;
  using L = ReadSmem<DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::offBar);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + kReadStages;
  uint64_t* s_full = kv_empty + kReadStages;  // QK^T in TMEM
  uint64_t* p_full = s_full + 1;              // W written (128 arrivals)
  uint64_t* feat_full = p_full + 1;           // psi(Q) in TMEM, psi(K) in smem (128)
  uint64_t* state_full = feat_full + 1;       // bf16 state in smem (128)
  uint64_t* upd_done = state_full + 1;        // readout + update of the chunk done
  uint64_t* o_full = upd_done + 1;            // O complete
  uint64_t* o_free = o_full + 1;              // O read by the epilogue (128)
  uint64_t* mma_done = o_free + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::offMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::offMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x, bh = blockIdx.y;
  const int t0 = g * Ls;
  const int t1 = min(T, t0 + Ls);
  const int n_chunks = (t1 - t0 + kTile - 1) / kTile;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kReadStages; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(feat_full, 128);
    mbar_init(state_full, 128);
    mbar_init(upd_done, 1);
    mbar_init(o_full, 1);
    mbar_init(o_free, 128);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  {
    uint32_t* ones = reinterpret_cast<uint32_t*>(smem + L::offOnes);
    for (int x = threadIdx.x; x < 128; x += kReadThreads) ones[x] = 0x3F803F80u;
    fence_proxy_async_smem();
  }
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
      int issued = 0;
      for (int c = 0; c < n_chunks; ++c) {
        const int st = c % kReadStages;
        if (!mbar_wait(kv_empty + st, ((c / kReadStages) & 1) ^ 1, env)) break;
        uint8_t* base = smem + L::offStage + st * L::kStageBytes;
        mbar_arrive_expect_tx(kv_full + st, L::kStageBytes);
        const int row = t0 + c * kTile;
        tma_load_3d(base, &tm_q, kv_full + st, 0, row, bh);
        tma_load_3d(base + Cfg::kQKBytes, &tm_k, kv_full + st, 0, row, bh);
        tma_load_3d(base + 2 * Cfg::kQKBytes, &tm_v, kv_full + st, 0, row, bh);
        ++issued;
      }
      for (int c = issued - kReadStages < 0 ? 0 : issued - kReadStages; c < issued; ++c)
        mbar_wait_drain(kv_full + c % kReadStages, (c / kReadStages) & 1, wc.limit);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t id_qk = idesc_bf16(128, 128, false, false);
      constexpr uint32_t id_ov = idesc_bf16(128, DV, false, true);   // A from TMEM (K-major), B N-major
      constexpr uint32_t id_oz = idesc_bf16(128, 16, false, true);   // against SZ
      constexpr uint32_t id_o1 = idesc_bf16(128, 16, false, false);  // against the ones block
      constexpr uint32_t id_uv = idesc_bf16(128, DV, true, true);    // A = psi(K)^T M-major
      constexpr uint32_t id_u1 = idesc_bf16(128, 16, true, false);
      const uint32_t sPsi = smem_u32(smem + L::offPsi), sSV = smem_u32(smem + L::offSV);
      const uint32_t sSZ = smem_u32(smem + L::offSZ), sStage = smem_u32(smem + L::offStage);
      const uint64_t ones_desc = smem_desc(smem_u32(smem + L::offOnes), 256, 128, kSwNone);
      for (int c = 0; c < n_chunks; ++c) {
        const int st = c % kReadStages;
        const uint32_t sQ = sStage + st * L::kStageBytes, sK = sQ + Cfg::kQKBytes, sV = sK + Cfg::kQKBytes;
        if (!mbar_wait(kv_full + st, (c / kReadStages) & 1, env)) break;
        tc_fence_after();
        // intra-chunk scores S = Q_c K_c^T (K = p = 16: one MMA)
        mma_ss(tmem + L::colS, smem_desc(sQ, 16, 256, kSw32), smem_desc(sK, 16, 256, kSw32), id_qk, 0);
        mma_commit(s_full);
        // readout against the state entering the chunk
        if (!mbar_wait(feat_full, c & 1, env)) break;
        if (!mbar_wait(state_full, c & 1, env)) break;
        if (c > 0 && !mbar_wait(o_free, (c - 1) & 1, env)) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < kP / 16; ++ks) {
          const uint32_t a = tmem + L::colPQ + ks * 8;
          mma_ts(tmem + L::colO, a, smem_desc(sSV + ks * Cfg::kSVKStep, Cfg::kSVBytes, Cfg::kSVSbo, Cfg::kVSw), id_ov,
                 ks > 0);
          mma_ts(tmem + L::colD, a, smem_desc(sSZ + ks * 512, Cfg::kSZBytes, 256, kSw32), id_oz, ks > 0);
        }
        // advance the running state by the chunk
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
#pragma unroll
          for (int ks = 0; ks < kTile / 16; ++ks) {
            const uint64_t a = smem_desc(sPsi + blk * 2 * kPsiLbo + ks * 2048, kPsiLbo, kPsiSbo, kSw128);
            const uint64_t b = smem_desc(sV + ks * Cfg::kVKStep, Cfg::kVBytes, Cfg::kVSbo, Cfg::kVSw);
            mma_ss(tmem + L::colRun(blk), a, b, id_uv, 1);
            mma_ss(tmem + L::colRun(blk) + DV, a, ones_desc, id_u1, 1);
          }
        }
        mma_commit(upd_done);
        // intra-chunk weights against [V_c | 1]
        if (!mbar_wait(p_full, c & 1, env)) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < kTile / 16; ++ks) {
          const uint32_t a = tmem + L::colS + ks * 8;
          mma_ts(tmem + L::colO, a, smem_desc(sV + ks * Cfg::kVKStep, Cfg::kVBytes, Cfg::kVSbo, Cfg::kVSw), id_ov, 1);
          mma_ts(tmem + L::colD, a, ones_desc, id_o1, 1);
        }
        mma_commit(o_full);
        mma_commit(kv_empty + st);
      }
      mma_commit(mma_done);
      mbar_wait_drain(mma_done, 0, wc.limit);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------- weights + output
    const int quarter = warp % 4;
    const int m = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    for (int c = 0; c < n_chunks; ++c) {
      if (!mbar_wait(s_full, c & 1, env)) break;
      tc_fence_after();
#pragma unroll
      for (int b = 0; b < kTile / 32; ++b) {
        uint32_t r[32];
        tmem_ld32(lane_base + L::colS + 32 * b, r);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          const float s0 = __uint_as_float(r[2 * x]), s1 = __uint_as_float(r[2 * x + 1]);
          const int col = 32 * b + 2 * x;
          w[x] = pack_bf16x2(col > m ? 0.f : s0 * s0, col + 1 > m ? 0.f : s1 * s1);
        }
        tmem_st16(lane_base + L::colS + 16 * b, w);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full);
      // output of the chunk
      if (!mbar_wait(o_full, c & 1, env)) break;
      tc_fence_after();
      float ov[DV];
      float D;
      load_state_row_tmem<DV>(lane_base + L::colO, ov, D);
      tc_fence_before();
      mbar_arrive(o_free);
      const int t = t0 + c * kTile + m;
      if (t < t1) {
        const float inv = D > 0.f ? 1.f / D : 0.f;
        uint4* dst = reinterpret_cast<uint4*>(o + ((size_t)bh * T + t) * DV);
#pragma unroll
        for (int e = 0; e < DV / 8; ++e) {
          uint4 u;
          u.x = pack_bf16x2(ov[8 * e + 0] * inv, ov[8 * e + 1] * inv);
          u.y = pack_bf16x2(ov[8 * e + 2] * inv, ov[8 * e + 3] * inv);
          u.z = pack_bf16x2(ov[8 * e + 4] * inv, ov[8 * e + 5] * inv);
          u.w = pack_bf16x2(ov[8 * e + 6] * inv, ov[8 * e + 7] * inv);
          dst[e] = u;
        }
      }
    }
  } else {
    // ------------------------------------------------------------- psi + state
    const int quarter = warp % 4;
    const int m = quarter * 32 + lane;  // token row / TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    uint8_t* sv = smem + L::offSV;
    uint8_t* sz = smem + L::offSZ;
    const __nv_bfloat16* qb = q + (size_t)bh * T * 16;
    const __nv_bfloat16* kb = k + (size_t)bh * T * 16;
    // running state <- scanned prefix (fp32 into TMEM, bf16 into shared memory)
    {
      const float* rec = ws + ((size_t)bh * G + g) * record_floats;
#pragma unroll 1
      for (int blk = 0; blk < 2; ++blk) {
        const int r = blk * 128 + m;
        const float* row = rec + (size_t)r * ld;
        float vals[DV];
#pragma unroll
        for (int e = 0; e < DV; e += 4) {
          const float4 x = *reinterpret_cast<const float4*>(row + e);
          vals[e] = x.x; vals[e + 1] = x.y; vals[e + 2] = x.z; vals[e + 3] = x.w;
        }
        const float zval = row[DV];
        store_state_row_tmem<DV>(lane_base + L::colRun(blk), vals, zval);
        store_state_row_bf16<DV>(sv, sz, r, vals, zval);
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(state_full);
    }
    for (int c = 0; c < n_chunks; ++c) {
      const int t = t0 + c * kTile + m;
      __nv_bfloat162 uq[8], uk[8];
      load_row16(qb + (size_t)t * 16, t < t1, uq);
      load_row16(kb + (size_t)t * 16, t < t1, uk);
      write_psi_q_tmem(lane_base + L::colPQ, uq);
      write_psi_k(smem + L::offPsi, m, uk);
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(feat_full);
      if (!mbar_wait(upd_done, c & 1, env)) break;
      tc_fence_after();
      if (c + 1 < n_chunks) {
#pragma unroll 1
        for (int blk = 0; blk < 2; ++blk) {
          float vals[DV];
          float zval;
          load_state_row_tmem<DV>(lane_base + L::colRun(blk), vals, zval);
          store_state_row_bf16<DV>(sv, sz, blk * 128 + m, vals, zval);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(state_full);
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

template <int DV>
static cudaError_t launch_state_t(const void* k, const void* v, float* ws, const ChunkPlan& pl, const WaitCtl& wc,
                                  cudaStream_t st) {
  using L = StateSmem<DV>;
  CUtensorMap tv;
  if (!make_tmap_bf16(&tv, v, DV, pl.T, pl.BH, kTile)) return cudaErrorInvalidValue;
  auto kern = chunk_state_kernel<DV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(pl.G, pl.BH);
  kern<<<grid, kStateThreads, L::kBytes, st>>>(tv, static_cast<const __nv_bfloat16*>(k), ws, pl.T, pl.Ls, pl.G,
                                               pl.ld, (long long)pl.record_floats, wc);
  return cudaGetLastError();
}

template <int DV>
static cudaError_t launch_read_t(const void* q, const void* k, const void* v, void* o, const float* ws,
                                 const ChunkPlan& pl, const WaitCtl& wc, cudaStream_t st) {
  using L = ReadSmem<DV>;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_bf16(&tq, q, 16, pl.T, pl.BH, kTile) || !make_tmap_bf16(&tk, k, 16, pl.T, pl.BH, kTile) ||
      !make_tmap_bf16(&tv, v, DV, pl.T, pl.BH, kTile))
    return cudaErrorInvalidValue;
  auto kern = chunk_readout_kernel<DV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(pl.G, pl.BH);
  kern<<<grid, kReadThreads, L::kBytes, st>>>(tq, tk, tv, static_cast<const __nv_bfloat16*>(q),
                                              static_cast<const __nv_bfloat16*>(k), static_cast<__nv_bfloat16*>(o),
                                              ws, pl.T, pl.Ls, pl.G, pl.ld, (long long)pl.record_floats, wc);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_state_sm100(const void* k, const void* v, float* ws, const ChunkPlan& pl, const WaitCtl& wc,
                                     cudaStream_t st) {
  if (pl.p != 16) return cudaErrorInvalidValue;
  if (pl.dv == 64) return launch_state_t<64>(k, v, ws, pl, wc, st);
  if (pl.dv == 16) return launch_state_t<16>(k, v, ws, pl, wc, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_chunk_readout_sm100(const void* q, const void* k, const void* v, void* o, const float* ws,
                                       const ChunkPlan& pl, const WaitCtl& wc, cudaStream_t st) {
  if (pl.p != 16) return cudaErrorInvalidValue;
  if (pl.dv == 64) return launch_read_t<64>(q, k, v, o, ws, pl, wc, st);
  if (pl.dv == 16) return launch_read_t<16>(q, k, v, o, ws, pl, wc, st);
  return cudaErrorInvalidValue;
}

}  // namespace kata
