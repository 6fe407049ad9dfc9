// chunk_linear_sm100.cu -- the chunked-state forward of first-order (linear)
// attention on tcgen05 / TMEM (bf16 inputs, d = 16, dv = 64):
//
//   o_t = sum_{s<=t} (q_t . k_s) v_s / sum_{s<=t} q_t . k_s
//
// i.e. the KATA recurrence with the identity feature psi(u) = u in place of
// vec(u u^T).  It is the comparator of the pages' scan-versus-sequential
// claim: an associative scan of the first-order feature lowers the
// inter-chunk recurrence depth to O(log(T/C)) and averages ~2.4x the
// throughput of a matched sequential linear-attention baseline (arXiv
// abstract; review page, Figure 3 caption; gist.science technical summary,
// sec. 2.3).  Both forms are built here from the same kernels: the scan form
// (state build, scan.cu, readout over super-chunks in parallel) and the
// sequential form (one readout CTA per (b,h) walking every chunk).
//
// The feature is the input itself, so nothing is formed: the key tile, as
// loaded by TMA ([128 tokens x 16] bf16, 32-byte swizzle), is directly the
// N-major B operand of the state update, and the query tile the K-major A
// operand of the readout.  The state is held transposed, S^T: TMEM lanes =
// value rows (lanes 64..127 the normaliser z, through a block of ones
// appended to V as in chunk_sm100.cu), 16 columns = feature coordinates:
//   S^T += [V_c | 1]^T K_c                  M = 128, N = 16, K = 16 tokens
//   [O | D] = Q_c S  + W_c [V_c | 1]        W = Q_c K_c^T, causal, in bf16
// The workspace record of a super-chunk uses scan.cu's unpacked layout
// (16 rows = coordinates, columns 0..63 = value, column 64 = z), so the scan
// also converts the caller's S0/z0 ([d, dv] / [d]) and nothing here is
// specific to it.
//
// The denominator of the first-order feature can be negative or zero:
// o = O / D when D != 0 and 0 when D == 0 (the D = 0 rule of the KATA paths).
#include <cuda.h>

#include "chunk_common.cuh"
#include "kata_internal.h"

namespace kata {

bool make_tmap_bf16(CUtensorMap* map, const void* base, int inner, int T, int BH, int rows);
bool make_tmap_bf16_box(CUtensorMap* map, const void* base, int inner, int T, int BH, int box_inner, int rows);

namespace {

using namespace sm100;
using namespace chunk;

constexpr int kLD = 16;                 // feature width d
constexpr int kLinLd = kDV + 4;         // unpacked record row stride (scan.cu)

// ===========================================================================
// 1. per-super-chunk state sums
// ===========================================================================
// warp 0 TMA ([V | K] ring), warp 1 MMA; afterwards warps 4, 5 and 2 (TMEM
// lane quarters 0, 1, 2) write the record.
constexpr int kLinStateThreads = 192;
constexpr int kLinStateStages = 8;

struct LinStateSmem {
  static constexpr int kStage = kVBytes + kQKBytes;  // [V | K]
  static constexpr int offStage = 0;
  static constexpr int offOnes = offStage + kLinStateStages * kStage;  // 1024-aligned
  static constexpr int offBar = offOnes + kOnesBytes;
  static constexpr int kBars = 2 * kLinStateStages + 1;
  static constexpr int offMisc = offBar + kBars * 8;
  static constexpr int kBytes = offMisc + 16 + 1024;
};

__global__ void __launch_bounds__(kLinStateThreads, 1)
    linear_state_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        float* __restrict__ ws, int T, int Ls, int G, long long record_floats, WaitCtl wc) {
  using L = LinStateSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::offBar);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + kLinStateStages;
  uint64_t* acc_done = kv_empty + kLinStateStages;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::offMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::offMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x, bh = blockIdx.y;
  const int t0 = g * Ls;
  const int n_chunks = (min(T, t0 + Ls) - t0 + kTile - 1) / kTile;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kLinStateStages; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    mbar_init(acc_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  fill_ones(smem + L::offOnes, threadIdx.x, kLinStateThreads);
  fence_proxy_async_smem();
  if (warp == 1) tmem_alloc(tmem_holder, 32);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitEnv env{wc.status, abort_flag, wc.limit};
  bool ok = true;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      int issued = 0;
      for (int c = 0; c < n_chunks; ++c) {
        const int st = c % kLinStateStages;
        if (!mbar_wait(kv_empty + st, ((c / kLinStateStages) & 1) ^ 1, env)) break;
        uint8_t* base = smem + L::offStage + st * L::kStage;
        mbar_arrive_expect_tx(kv_full + st, L::kStage);
        tma_load_3d(base, &tm_v, kv_full + st, 0, t0 + c * kTile, bh);
        tma_load_3d(base + kVBytes, &tm_k, kv_full + st, 0, t0 + c * kTile, bh);
        ++issued;
      }
      for (int c = issued - kLinStateStages < 0 ? 0 : issued - kLinStateStages; c < issued; ++c)
        mbar_wait_drain(kv_full + c % kLinStateStages, (c / kLinStateStages) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // whole warp; one elected lane issues
    constexpr uint32_t id_u = idesc_bf16(128, kLD, true, true);  // A = [V | 1]^T, B = K (N-major)
    const uint32_t sStage = smem_u32(smem + L::offStage), sOnes = smem_u32(smem + L::offOnes);
    int c = 0;
    for (; c < n_chunks; ++c) {
      const int st = c % kLinStateStages;
      if (!mbar_wait_w(kv_full + st, (c / kLinStateStages) & 1, env)) break;
      tc_fence_after();
      const uint32_t sV = sStage + st * L::kStage;
      const uint64_t da = desc_vones(sV, sOnes), db = smem_desc(sV + kVBytes, kPsiAtom, 256, kSw32);
#pragma unroll
      for (int ks = 0; ks < kTile / 16; ++ks)
        mma_ss_w(tmem, desc_add(da, ks * 2048), desc_add(db, ks * 512), id_u, (c > 0 || ks > 0) ? 1u : 0u);
      mma_commit_w(kv_empty + st);
    }
    mma_commit_w(acc_done);
    mbar_wait_drain(acc_done, 0);
  }
  // record rows: TMEM lane d (value d < 64, z at 64) and column i become the
  // unpacked record's entry [i][d] (z in column dv)
  const int quarter = warp % 4;
  const int d = quarter * 32 + lane;
  if (ok && (warp == 2 || warp == 4 || warp == 5) && mbar_wait_w(acc_done, 0, env)) {
    tc_fence_after();
    uint32_t r[16];
    tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16), r);
    tmem_wait_ld();
    if (d <= kDV) {
      float* rec = ws + ((size_t)bh * G + g) * record_floats;
#pragma unroll
      for (int i = 0; i < kLD; ++i) rec[i * kLinLd + d] = __uint_as_float(r[i]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 32);
  }
}

// ===========================================================================
// 2. readout
// ===========================================================================
// Warp roles (448 threads):
//   warp 0       TMA: [V | Q | K] tiles of each chunk into a ring
//   warp 1       TMEM allocator; MMA issue (the whole warp, one elected lane)
//   warps 2-5,   weights W = Q K^T (causal, bf16) into TMEM; output o = O / D;
//   6-9          the two warps on a TMEM lane quarter split the key columns
//                of the weights and the value columns of the output
//   warps 10-13  the state entering the super-chunk in; the bf16 copy of the
//                state after each chunk; the final state
// MMA order per chunk c: scores of c, readout of c against the bf16 copy of
// S made before c, advance S by c, intra-chunk weights; the copy is
// refreshed in place once the advance lands (the readout, issued before it,
// has read it by then).  The MMA warp waits on two barriers per chunk:
// state_full(c), arrived on by warps 10-13 once the copy is refreshed and
// chunk c's tiles have landed, and by warps 2-9 once they have read the
// output of chunk c-2 out of the [O | D] buffer the readout of c reuses; and
// p_full(c), by warps 2-9 after the weights of c.
constexpr int kLinReadThreads = 448;
constexpr int kLinReadStages = 6;

struct LinReadSmem {
  static constexpr int kStage = kVBytes + 2 * kQKBytes;  // [V | Q | K]
  static constexpr int offStage = 0;
  static constexpr int offOnes = offStage + kLinReadStages * kStage;  // 1024-aligned
  static constexpr int offSB = offOnes + kOnesBytes;                  // bf16 copy: [80 rows x 32 B]
  static constexpr int offOut = offSB + kSBAtom;                      // output staging: 8 boxes [32 x 32]
  static constexpr int offBar = offOut + kVBytes;
  static constexpr int kBars = 2 * kLinReadStages + 7;
  static constexpr int offMisc = offBar + kBars * 8;
  static constexpr int kBytes = offMisc + 16 + 1024;
  // TMEM columns
  static constexpr uint32_t colRun = 0;                                   // S^T, 16
  static constexpr uint32_t colO(int b) { return 32u + 80u * (uint32_t)b; }  // [O | D] x 2
  static constexpr uint32_t colS = 256;                                   // scores / weights, 128
};

__global__ void __launch_bounds__(kLinReadThreads, 1)
    linear_readout_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                          const float* __restrict__ ws, const float* __restrict__ S0, const float* __restrict__ z0,
                          float* __restrict__ S_out, float* __restrict__ z_out, int T, int Ls, int G,
                          long long record_floats, WaitCtl wc) {
  using L = LinReadSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::offBar);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + kLinReadStages;
  uint64_t* s_full = kv_empty + kLinReadStages;  // scores in TMEM
  uint64_t* p_full = s_full + 1;                 // weights written (256)
  uint64_t* state_full = p_full + 1;             // copy refreshed, tiles in, [O | D] buffer free (384)
  uint64_t* upd_done = state_full + 1;           // state advanced by the chunk
  uint64_t* o_full = upd_done + 1;               // [2] [O | D] complete
  uint64_t* mma_done = o_full + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::offMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::offMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // super-chunks in reverse order of the state kernel (its last key/value
  // tiles are then still in L2)
  const int g = gridDim.x - 1 - blockIdx.x, bh = blockIdx.y;
  const int t0 = g * Ls;
  const int t1 = min(T, t0 + Ls);
  const int n_chunks = (t1 - t0 + kTile - 1) / kTile;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kLinReadStages; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 256);
    mbar_init(state_full, 384);
    mbar_init(upd_done, 1);
    for (int b = 0; b < 2; ++b) mbar_init(o_full + b, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  fill_ones(smem + L::offOnes, threadIdx.x, kLinReadThreads);
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
      int issued = 0;
      for (int c = 0; c < n_chunks; ++c) {
        const int st = c % kLinReadStages;
        if (!mbar_wait(kv_empty + st, ((c / kLinReadStages) & 1) ^ 1, env)) break;
        uint8_t* base = smem + L::offStage + st * L::kStage;
        mbar_arrive_expect_tx(kv_full + st, L::kStage);
        const int row = t0 + c * kTile;
        tma_load_3d(base, &tm_v, kv_full + st, 0, row, bh);
        tma_load_3d(base + kVBytes, &tm_q, kv_full + st, 0, row, bh);
        tma_load_3d(base + kVBytes + kQKBytes, &tm_k, kv_full + st, 0, row, bh);
        ++issued;
      }
      for (int c = issued - kLinReadStages < 0 ? 0 : issued - kLinReadStages; c < issued; ++c)
        mbar_wait_drain(kv_full + c % kLinReadStages, (c / kLinReadStages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA
    constexpr uint32_t id_qk = idesc_bf16(128, 128, false, false);  // A = Q, B = K, both K-major
    constexpr uint32_t id_rd = idesc_bf16(128, 80, false, false);   // A = Q, B = bf16 copy of S (K-major)
    constexpr uint32_t id_wv = idesc_bf16(128, 80, false, true);    // A = W (TMEM), B = [V | 1]
    constexpr uint32_t id_u = idesc_bf16(128, kLD, true, true);     // A = [V | 1]^T, B = K (N-major)
    const uint32_t sStage = smem_u32(smem + L::offStage), sOnes = smem_u32(smem + L::offOnes);
    const uint64_t dq0 = smem_desc(sStage + kVBytes, 16, 256, kSw32);
    const uint64_t dk0 = smem_desc(sStage + kVBytes + kQKBytes, 16, 256, kSw32);
    const uint64_t dkn0 = smem_desc(sStage + kVBytes + kQKBytes, kPsiAtom, 256, kSw32);
    const uint64_t dsb = smem_desc(smem_u32(smem + L::offSB), 16, 256, kSw32);
    for (int c = 0; c < n_chunks; ++c) {
      const int st = c % kLinReadStages, ob = c & 1;
      const uint32_t sV = sStage + st * L::kStage;
      if (!mbar_wait_w(state_full, c & 1, env)) break;
      tc_fence_after();
      // scores of chunk c (over the weights of chunk c-1 only after the
      // intra-chunk MMAs of c-1, issued before them)
      mma_ss_w(tmem + L::colS, desc_add(dq0, st * L::kStage), desc_add(dk0, st * L::kStage), id_qk, 0);
      mma_commit_w(s_full);
      // readout against the copy of the state entering the chunk
      const uint32_t dO = tmem + L::colO(ob);
      mma_ss_w(dO, desc_add(dq0, st * L::kStage), dsb, id_rd, 0);
      // advance the state by the chunk
      const uint64_t dvo = desc_vones(sV, sOnes);
#pragma unroll
      for (int ks = 0; ks < kTile / 16; ++ks)
        mma_ss_w(tmem + L::colRun, desc_add(dvo, ks * 2048), desc_add(dkn0, st * L::kStage + ks * 512), id_u, 1);
      mma_commit_w(upd_done);
      // intra-chunk weights against [V_c | 1]
      if (!mbar_wait_w(p_full, c & 1, env)) break;
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < kTile / 16; ++ks)
        mma_ts_w(dO, tmem + L::colS + (ks >> 2) * 64 + (ks & 3) * 8, desc_add(dvo, ks * 2048), id_wv, 1);
      mma_commit_w(o_full + ob);
      mma_commit_w(kv_empty + st);
    }
    mma_commit_w(mma_done);
    mbar_wait_drain(mma_done, 0);
  } else if (warp < 10) {
    // ------------------------------------------------------------- weights + output
    const int quarter = warp % 4;
    const int h = warp >= 6 ? 1 : 0;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    uint8_t* slab = smem + L::offOut + (quarter * 2 + h) * (32 * 64);  // this warp's [32 x 32] output box
    // output of chunk co: read [O | D] out of TMEM, then arrive on
    // state_full(co + 2) when that chunk exists (its readout reuses the
    // buffer); o = O / D (0 where D == 0) rounded to bf16, staged as this
    // warp's 64B-swizzled [32 x 32] box of the o tensor map and written by
    // one TMA store (rows past T are not written)
    auto output = [&](int co) -> bool {
      const int ob = co & 1;
      if (!mbar_wait_w(o_full + ob, (co >> 1) & 1, env)) return false;
      tc_fence_after();
      uint32_t r[32], db;
      tmem_ld32(lane_base + L::colO(ob) + 32 * h, r);
      tmem_ld1(lane_base + L::colO(ob) + 64, db);
      tmem_wait_ld();
      tc_fence_before();
      if (co + 2 < n_chunks) mbar_arrive(state_full);
      const float D = __uint_as_float(db);
      const float inv = D != 0.f ? 1.f / D : 0.f;
      const uint64_t inv2 = f32x2(__float_as_uint(inv), __float_as_uint(inv));
      auto scaled = [&](int k) {
        const uint64_t v = f32x2_mul(f32x2(r[k], r[k + 1]), inv2);
        return pack_bf16x2(f32x2_lo(v), f32x2_hi(v));
      };
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
      uint8_t* orow = slab + lane * 64;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        *reinterpret_cast<uint4*>(orow + ((e ^ ((lane >> 1) & 3)) << 4)) =
            make_uint4(scaled(8 * e), scaled(8 * e + 2), scaled(8 * e + 4), scaled(8 * e + 6));
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_3d(&tm_o, slab, 32 * h, t0 + co * kTile + quarter * 32, bh);
        bulk_commit_group();
      }
      return true;
    };
    // the readouts of chunks 0 and 1 write fresh [O | D] buffers; the
    // arrival for chunk 1 is made once state_full(0) has completed (the
    // scores of chunk 0 are issued after it)
    if (n_chunks > 0) mbar_arrive(state_full);
    bool ok = true;
    for (int c = 0; ok && c < n_chunks; ++c) {
      if (!mbar_wait_w(s_full, c & 1, env)) break;
      if (c == 0 && n_chunks > 1) mbar_arrive(state_full);
      tc_fence_after();
      // causal within the chunk: 32-column block bb of row m is fully kept
      // for bb < quarter, diagonal for bb == quarter, zero for bb > quarter.
      // Block bb's 16 bf16x2 words go to columns 64 (bb / 2) + 16 (bb % 2).
#pragma unroll
      for (int b2 = 0; b2 < 2; ++b2) {
        const int bb = 2 * h + b2;
        uint32_t w[16];
        if (bb > quarter) {
#pragma unroll
          for (int x = 0; x < 16; ++x) w[x] = 0u;
        } else {
          uint32_t r[32];
          tmem_ld32(lane_base + L::colS + 32 * bb, r);
          tmem_wait_ld();
          if (bb < quarter) {
#pragma unroll
            for (int x = 0; x < 16; ++x) w[x] = pack_bf16x2(__uint_as_float(r[2 * x]), __uint_as_float(r[2 * x + 1]));
          } else {
#pragma unroll
            for (int x = 0; x < 16; ++x) {
              const float a = 2 * x > lane ? 0.f : __uint_as_float(r[2 * x]);
              const float b = 2 * x + 1 > lane ? 0.f : __uint_as_float(r[2 * x + 1]);
              w[x] = pack_bf16x2(a, b);
            }
          }
        }
        tmem_st16(lane_base + L::colS + 64 * h + 16 * b2, w);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full);
      if (c > 0) ok = output(c - 1);
    }
    if (ok && n_chunks > 0) output(n_chunks - 1);
    if (lane == 0) bulk_wait_all();
  } else {
    // ------------------------------------------------------------- state rows
    const int quarter = warp % 4;
    const int m = quarter * 32 + lane;  // TMEM lane: value row (64..127: z)
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    uint8_t* sb = smem + L::offSB;
    const bool active = m < kSBRows;  // rows 0..63 values, 64..79 copies of z
    const int dz = min(m, kDV);       // record column of this lane
    // the state entering the super-chunk: the scanned record g, or with a
    // single super-chunk the caller's initial state (or zero).  After a scan
    // this kernel is its programmatic dependent: wait for the records.
    griddep_wait();
    {
      uint32_t r[16];
      if (ws) {
        const float* rec = ws + ((size_t)bh * G + g) * record_floats;
#pragma unroll
        for (int i = 0; i < kLD; ++i) r[i] = __float_as_uint(rec[i * kLinLd + dz]);
      } else {
#pragma unroll
        for (int i = 0; i < kLD; ++i)
          r[i] = __float_as_uint(!S0 ? 0.f : m < kDV ? S0[((size_t)bh * kLD + i) * kDV + m] : z0[(size_t)bh * kLD + i]);
      }
      tmem_st16(lane_base + L::colRun, r);
      if (active) store_state_bf16_atom(sb, m, 0, r);
    }
    tmem_wait_st();
    fence_proxy_async_smem();
    tc_fence_before();
    bool ok = n_chunks > 0 && mbar_wait_w(kv_full, 0, env);
    if (ok) mbar_arrive(state_full);
    for (int c = 0; ok && c + 1 < n_chunks; ++c) {
      // the state after chunk c: the copy for the readout of chunk c+1 (the
      // readout of chunk c, issued before this advance, has read the copy)
      if (!mbar_wait_w(upd_done, c & 1, env)) break;
      tc_fence_after();
      uint32_t r[16];
      tmem_ld16(lane_base + L::colRun, r);
      tmem_wait_ld();
      if (active) store_state_bf16_atom(sb, m, 0, r);
      fence_proxy_async_smem();
      tc_fence_before();
      const int st1 = (c + 1) % kLinReadStages;
      if (!mbar_wait_w(kv_full + st1, ((c + 1) / kLinReadStages) & 1, env)) break;
      mbar_arrive(state_full);
    }
    // the last super-chunk ends at token T: its running state, once the
    // advance by its last chunk has landed, is the final state
    if (S_out && g == G - 1 && n_chunks > 0 && quarter < 3 && mbar_wait_w(upd_done, (n_chunks - 1) & 1, env)) {
      tc_fence_after();
      uint32_t r[16];
      tmem_ld16(lane_base + L::colRun, r);  // warp-collective
      tmem_wait_ld();
      if (m <= kDV) {
#pragma unroll
        for (int i = 0; i < kLD; ++i) {
          if (m < kDV) S_out[((size_t)bh * kLD + i) * kDV + m] = __uint_as_float(r[i]);
          else z_out[(size_t)bh * kLD + i] = __uint_as_float(r[i]);
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

cudaError_t launch_linear_state_sm100(const void* k, const void* v, float* ws, const ChunkPlan& pl, const WaitCtl& wc,
                                      cudaStream_t st) {
  if (pl.p != kLD || pl.dv != kDV || pl.ld != kLinLd) return cudaErrorInvalidValue;
  CUtensorMap tk, tv;
  if (!make_tmap_bf16(&tk, k, kLD, pl.T, pl.BH, kTile) || !make_tmap_bf16(&tv, v, kDV, pl.T, pl.BH, kTile))
    return cudaErrorInvalidValue;
  cudaError_t e =
      cudaFuncSetAttribute(linear_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, LinStateSmem::kBytes);
  if (e != cudaSuccess) return e;
  if (pl.G < 2) return cudaSuccess;  // the last super-chunk's sum is never needed
  linear_state_kernel<<<dim3(pl.G - 1, pl.BH), kLinStateThreads, LinStateSmem::kBytes, st>>>(
      tk, tv, ws, pl.T, pl.Ls, pl.G, (long long)pl.record_floats, wc);
  return cudaGetLastError();
}

cudaError_t launch_linear_readout_sm100(const void* q, const void* k, const void* v, void* o, const float* ws,
                                        const float* S0, const float* z0, float* S_out, float* z_out,
                                        const ChunkPlan& pl, const WaitCtl& wc, cudaStream_t st) {
  if (pl.p != kLD || pl.dv != kDV || pl.ld != kLinLd) return cudaErrorInvalidValue;
  if (!ws && pl.G != 1) return cudaErrorInvalidValue;
  CUtensorMap tq, tk, tv, to;
  if (!make_tmap_bf16(&tq, q, kLD, pl.T, pl.BH, kTile) || !make_tmap_bf16(&tk, k, kLD, pl.T, pl.BH, kTile) ||
      !make_tmap_bf16(&tv, v, kDV, pl.T, pl.BH, kTile) || !make_tmap_bf16_box(&to, o, kDV, pl.T, pl.BH, 32, 32))
    return cudaErrorInvalidValue;
  cudaError_t e =
      cudaFuncSetAttribute(linear_readout_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, LinReadSmem::kBytes);
  if (e != cudaSuccess) return e;
  const dim3 grid(pl.G, pl.BH), block(kLinReadThreads);
  if (ws)  // after the state build and scan of this call
    return launch_pdl(linear_readout_kernel, grid, block, (size_t)LinReadSmem::kBytes, st, tq, tk, tv, to,
                      (const float*)ws, S0, z0, S_out, z_out, pl.T, pl.Ls, pl.G, (long long)pl.record_floats, wc);
  linear_readout_kernel<<<grid, block, LinReadSmem::kBytes, st>>>(tq, tk, tv, to, ws, S0, z0, S_out, z_out, pl.T,
                                                                   pl.Ls, pl.G, (long long)pl.record_floats, wc);
  return cudaGetLastError();
}

}  // namespace kata
