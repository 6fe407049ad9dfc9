// chunk_sm100.cu -- exact O(T) chunked-state KATA forward on tcgen05 / TMEM
// (bf16 inputs, p = 16, dv = 64): the second operating point of the
// gist.science technical summary, sec. 2.3 ("Chunked Parallelism":
// intra-chunk attention on tensor cores, inter-chunk state propagation by an
// associative scan).
//
// Packed feature map.  psi(u) = vec(u u^T) is symmetric, so the state only
// needs the n = p(p+1)/2 = 136 unique coordinates (ai.info summary, Main
// Findings, "State size, not just feature width, dominates memory").  The
// packed coordinates are ordered by runs: for i = 0..15 the entries (i, j),
// j = i..15, each run padded with one zero to even length, which gives
// exactly 144 = 9 x 16 coordinates and lets every bf16 pair come from one
// bf16x2 multiply.  The query side holds q_i q_j; the key side holds
// k_i^2 on the diagonal and 2 k_i k_j off it (the factor 2 is exact), so
//   <psi~(q), psi~(k)> = sum_i q_i^2 k_i^2 + 2 sum_{i<j} q_i q_j k_i k_j
//                      = (q . k)^2.
//
// State layout.  The state is held transposed, S~^T: 128 TMEM lanes (row d
// = value column, rows 64..127 = the normaliser z) x 144 columns (packed psi
// index), fp32.  It is the accumulator of
//   S~^T += [V_c | 1]^T psi~(K_c)        M = 128, N = 144, K = 16 tokens
// where the A operand is the TMA-loaded V tile followed, one swizzle atom
// further, by a block of ones, and the B operand psi~(K_c) is formed in
// shared memory.  The workspace record of a super-chunk is rows 0..64 of it
// (65 x 144 fp32).
//
// Launches per call, with G super-chunks per (b,h):
//  1. chunk_state_kernel    (G > 1) per super-chunk g < G-1: A_g = sum over
//                           its chunks (nothing reads the last one's sum);
//  2. state_scan            (G > 1, scan.cu) exclusive prefix over g, depth
//                           O(log G);
//  3. chunk_readout_kernel  per super-chunk, per 128-token chunk c:
//        [O | D] = psi~(Q_c) S~          readout, K = 144, B = bf16 copy of S~
//                + W_c [V_c | 1]         W = (Q_c K_c^T)^2, causal
//        S~^T   += [V_c | 1]^T psi~(K_c) advance
//        o_c     = O / D
//     with S~ starting at the scanned prefix (G = 1: at the caller's initial
//     state, or zero); the CTA of the last super-chunk writes the final state.
#include <cuda.h>

#include "chunk_common.cuh"
#include "kata_internal.h"
#include "kata_trace.cuh"

KATA_TRACE_DECLARE(chunk)
KATA_TRACE_DECLARE(chunkstate)

namespace kata {

bool make_tmap_bf16(CUtensorMap* map, const void* base, int inner, int T, int BH, int rows);
bool make_tmap_bf16_box(CUtensorMap* map, const void* base, int inner, int T, int BH, int box_inner, int rows);

namespace {

using namespace sm100;
using namespace chunk;

// G = 1: the single factor psi(u) = vec(u u^T) with p = 16.  G = 2 or 4:
// KATA-Sigma-g with G groups of 16 (d = 16 G), the summed feature
// psi_S(u) = sum_j vec(u^j u^j^T) on the same 16 x 16 state (gist.science
// sec. 2.3 "Varianten"; ai.info Main Findings: state (d/g)(d/g+1)/2 * dv).
// Its packed entries are summed over the groups in fp32 and rounded to bf16
// once, and the intra-chunk weights sum_{j,l} (q^j . k^l)^2 are the inner
// products psi~_S(Q) psi~_S(K)^T (9 MMAs over the 144 packed coordinates)
// instead of squared Q K^T scores.  The wider Q and K tiles leave room for
// fewer ring stages.
template <int G>
struct ChunkCfg {
  static constexpr int kD = 16 * G;                    // q, k row width
  static constexpr int kQKB = kTile * kD * 2;          // one Q or K tile
  static constexpr int kStateStages = G == 1 ? 6 : 4;
  static constexpr int kReadStages = G == 4 ? 2 : 3;
};

// ===========================================================================
// 1. per-super-chunk state sums
// ===========================================================================
constexpr int kStateThreads = 320;  // warp 0 TMA, warp 1 MMA, warps 2-9 psi~(k), warps 2-5 record
// psi~(K) buffers.  Measured at B1 H16 T131072: 6 stages with 2 buffers
// 243 us for the whole chunked call, 4 with 3 buffers 252 us, 3 with 4
// buffers 259 us -- the deeper TMA ring matters more than forming psi~(K)
// further ahead
constexpr int kStatePsiBufs = 2;

template <int G>
struct StateSmem {
  static constexpr int kStages = ChunkCfg<G>::kStateStages;
  static constexpr int kStage = kVBytes + ChunkCfg<G>::kQKB;  // [V | K]
  static constexpr int offStage = 0;
  static constexpr int offOnes = offStage + kStages * kStage;  // 1024-aligned
  static constexpr int offPsi = offOnes + kOnesBytes;                 // kStatePsiBufs buffers
  static constexpr int offBar = offPsi + kStatePsiBufs * kPsiBytes;
  static constexpr int kBars = 2 * kStages + 2 * kStatePsiBufs + 1;
  static constexpr int offMisc = offBar + kBars * 8;
  static constexpr int kBytes = offMisc + 16 + 1024;
};

template <int NG>
__global__ void __launch_bounds__(kStateThreads, 1)
    chunk_state_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       float* __restrict__ ws, int T, int Ls, int G, long long record_floats, WaitCtl wc) {
  using L = StateSmem<NG>;
  constexpr int kStateStages = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::offBar);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + kStateStages;
  uint64_t* psi_full = kv_empty + kStateStages;  // [kStatePsiBufs]
  uint64_t* psi_empty = psi_full + kStatePsiBufs;
  uint64_t* acc_done = psi_empty + kStatePsiBufs;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::offMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::offMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  KATA_TRACE_BEGIN(chunkstate);
  const int g = blockIdx.x, bh = blockIdx.y;
  const int t0 = g * Ls;
  const int n_chunks = (min(T, t0 + Ls) - t0 + kTile - 1) / kTile;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStateStages; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    for (int s = 0; s < kStatePsiBufs; ++s) {
      mbar_init(psi_full + s, 256);
      mbar_init(psi_empty + s, 1);
    }
    mbar_init(acc_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  fill_ones(smem + L::offOnes, threadIdx.x, kStateThreads);
  fence_proxy_async_smem();
  if (warp == 1) tmem_alloc(tmem_holder, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitEnv env{wc.status, abort_flag, wc.limit};

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      int issued = 0;
      for (int c = 0; c < n_chunks; ++c) {
        const int st = c % kStateStages;
        if (!mbar_wait(kv_empty + st, ((c / kStateStages) & 1) ^ 1, env)) break;
        uint8_t* base = smem + L::offStage + st * L::kStage;
        KATA_TRACE(chunkstate, c, 5);
        mbar_arrive_expect_tx(kv_full + st, L::kStage);
        tma_load_3d(base, &tm_v, kv_full + st, 0, t0 + c * kTile, bh);
        tma_load_3d(base + kVBytes, &tm_k, kv_full + st, 0, t0 + c * kTile, bh);
        ++issued;
      }
      for (int c = issued - kStateStages < 0 ? 0 : issued - kStateStages; c < issued; ++c)
        mbar_wait_drain(kv_full + c % kStateStages, (c / kStateStages) & 1);
    }
  } else if (warp == 1) {
    {  // whole warp; one elected lane issues
      constexpr uint32_t id_u = idesc_bf16(128, kNP, true, true);
      const uint32_t sStage = smem_u32(smem + L::offStage), sOnes = smem_u32(smem + L::offOnes);
      const uint32_t sPsi = smem_u32(smem + L::offPsi);
      const uint64_t dpsi = smem_desc(sPsi, kPsiAtom, 256, kSw32);
      for (int c = 0; c < n_chunks; ++c) {
        const int st = c % kStateStages, pb = c % kStatePsiBufs;
        if (!mbar_wait_w(kv_full + st, (c / kStateStages) & 1, env)) break;
        if (!mbar_wait_w(psi_full + pb, (c / kStatePsiBufs) & 1, env)) break;
        KATA_TRACE(chunkstate, c, 0);
        tc_fence_after();
        const uint32_t sV = sStage + st * L::kStage;
        const uint64_t da = desc_vones(sV, sOnes), db = desc_add(dpsi, pb * kPsiBytes);
#pragma unroll
        for (int ks = 0; ks < kTile / 16; ++ks)
          mma_ss_w(tmem, desc_add(da, ks * 2048), desc_add(db, ks * 512), id_u, (c > 0 || ks > 0) ? 1u : 0u);
        KATA_TRACE(chunkstate, c, 1);
        mma_commit_w(psi_empty + pb);
        mma_commit_w(kv_empty + st);
      }
      mma_commit_w(acc_done);
      mbar_wait_drain(acc_done, 0);
    }
  } else {
    // warps 2-9: token (warp - 2) % 4 * 32 + lane, half (warp - 2) / 4 of its packed psi
    const int tid = ((warp - 2) & 3) * 32 + lane;
    const int half = (warp - 2) >> 2;
    const int quarter = warp % 4;
    const int d = quarter * 32 + lane;  // TMEM lane = record row
    bool ok = true;
    for (int c = 0; c < n_chunks; ++c) {
      const int st = c % kStateStages, pb = c % kStatePsiBufs;
      if (!mbar_wait_w(kv_full + st, (c / kStateStages) & 1, env)) {
        ok = false;
        break;
      }
      if (tid == 0) KATA_TRACE(chunkstate, c, 2);
      if (c >= kStatePsiBufs && !mbar_wait_w(psi_empty + pb, ((c / kStatePsiBufs) - 1) & 1, env)) {
        ok = false;
        break;
      }
      if (tid == 0) KATA_TRACE(chunkstate, c, 3);
      __nv_bfloat162 u[8 * NG];
      load_row_sw<NG>(smem + L::offStage + st * L::kStage + kVBytes, tid, u);
      uint32_t w[kNPW / 2];
      if (half == 0) {
        if constexpr (NG == 1) packed_psi_half<true, 0>(u, w);
        else packed_psi_sum_half<true, 0, NG>(u, w);
        store_psi_k_half<0>(smem + L::offPsi + pb * kPsiBytes, tid, w);
      } else {
        if constexpr (NG == 1) packed_psi_half<true, 1>(u, w);
        else packed_psi_sum_half<true, 1, NG>(u, w);
        store_psi_k_half<1>(smem + L::offPsi + pb * kPsiBytes, tid, w);
      }
      fence_proxy_async_smem();
      mbar_arrive(psi_full + pb);
      if (tid == 0) KATA_TRACE(chunkstate, c, 4);
    }
    // record rows 0..64 live in TMEM lanes 0..64: warps of lane quarters 0-2
    // load (the load is warp-collective), lanes below 65 store
    if (ok && warp < 6 && quarter < 3 && mbar_wait_w(acc_done, 0, env)) {
      tc_fence_after();
      float* row = ws + ((size_t)bh * G + g) * record_floats + (size_t)min(d, kRecRows - 1) * kNP;
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

// ===========================================================================
// 3. readout
// ===========================================================================
// Warp roles (576 threads):
//   warp 0       TMA: [V | Q | K] tiles of each chunk into a 3-stage ring
//   warp 1       TMEM allocator; MMA issue (the whole warp, one elected lane)
//   warps 2-5,   weights W = (Q K^T)^2 (causal) into TMEM; output o = O / D;
//   14-17        each pair of warps on a TMEM lane quarter splits the columns
//   warps 6-9    psi~(k_{c+1}) into shared memory (two buffers); bf16 copy of
//                packed coordinates 0..71 of the state after chunk c
//   warps 10-13  prefix state in; psi~(q_{c+1}) into TMEM once the readout of
//                chunk c has read psi~(q_c); then the bf16 copy of coordinates
//                72..143
// MMA order per chunk c: scores of chunk c, readout of chunk c against the
// bf16 copy of S~ made before chunk c, advance S~ by chunk c, intra-chunk
// weights.  The readout reads only the bf16 copy, and comes first so that
// psi~(q_c) is released early; the copy for chunk c+1 is refreshed in place
// once the advance lands (the readout, issued before it, has then read the
// copy), while the intra-chunk MMAs of chunk c run.  One copy instead of two
// frees 22.5 KiB of shared memory: 246.8 -> 242.7 us at B1 H16 T131072.
// The MMA warp waits on two barriers per chunk.  state_full(c) is arrived on
// by warps 6-13 after everything chunk c needs from them (its psi~(k), its
// psi~(q), the bf16 copy; each of them waited for chunk c's tiles to land
// first) and by warps 2-5 and 14-17 once they have read the output of chunk
// c-2 out of the [O | D] buffer the readout of chunk c reuses; p_full(c) by
// warps 2-5 and 14-17 after the weights of chunk c.  Each wait in the
// issuing warp costs ~100 cycles in which the tensor pipe drains, so the
// implied ones are not waited for separately.
constexpr int kReadThreads = 576;

template <int G>
struct ReadSmem {
  static constexpr int kStages = ChunkCfg<G>::kReadStages;
  static constexpr int kQKB = ChunkCfg<G>::kQKB;
  static constexpr int kStage = kVBytes + 2 * kQKB;  // [V | Q | K]
  static constexpr int offStage = 0;
  static constexpr int offOnes = offStage + kStages * kStage;  // 1024-aligned
  static constexpr int offPsi = offOnes + kOnesBytes;  // 2 buffers
  static constexpr int offSB = offPsi + 2 * kPsiBytes;  // one buffer
  static constexpr int offOut = offSB + kSBBytes;      // output staging: 8 boxes [32 x 32], 64B swizzle
  static constexpr int offBar = offOut + kVBytes;
  static constexpr int kBars = 2 * kStages + 8;
  static constexpr int offMisc = offBar + kBars * 8;
  static constexpr int kBytes = offMisc + 16 + 1024;
  // TMEM columns (multiples of 16, 512 in total)
  static constexpr uint32_t colRun = 0;                                    // S~^T, 144
  static constexpr uint32_t colO(int b) { return 144u + 80u * (uint32_t)b; }  // [O | D] x 2
  static constexpr uint32_t colPQ = 304;                                   // psi~(Q_c), 72
  static constexpr uint32_t colS = 384;                                    // scores / weights, 128
};

template <int NG>
__global__ void __launch_bounds__(kReadThreads, 1)
    chunk_readout_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                         const float* __restrict__ ws, const float* __restrict__ S0, const float* __restrict__ z0,
                         float* __restrict__ S_out, float* __restrict__ z_out, float* __restrict__ D_out, int T,
                         int Ls, int G, long long record_floats, WaitCtl wc) {
  using L = ReadSmem<NG>;
  constexpr int kReadStages = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::offBar);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + kReadStages;
  uint64_t* s_full = kv_empty + kReadStages;  // scores in TMEM
  uint64_t* p_full = s_full + 1;              // weights written (256)
  uint64_t* state_full = p_full + 1;          // chunk c's operands ready and its [O | D] buffer free (512)
  uint64_t* rd_done = state_full + 1;         // readout of the chunk done
  uint64_t* upd_done = rd_done + 1;           // state advanced by the chunk
  uint64_t* o_full = upd_done + 1;            // [2] [O | D] complete
  uint64_t* mma_done = o_full + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::offMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::offMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  KATA_TRACE_BEGIN(chunk);
  // super-chunks in reverse order of the state kernel, so the key/value tiles
  // it touched last are still in L2 when they are read here first
  const int g = gridDim.x - 1 - blockIdx.x, bh = blockIdx.y;
  const int t0 = g * Ls;
  const int t1 = min(T, t0 + Ls);
  const int n_chunks = (t1 - t0 + kTile - 1) / kTile;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kReadStages; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 256);
    mbar_init(state_full, 512);
    mbar_init(rd_done, 1);
    mbar_init(upd_done, 1);
    for (int b = 0; b < 2; ++b) mbar_init(o_full + b, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  fill_ones(smem + L::offOnes, threadIdx.x, kReadThreads);
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
        const int st = c % kReadStages;
        if (!mbar_wait(kv_empty + st, ((c / kReadStages) & 1) ^ 1, env)) break;
        uint8_t* base = smem + L::offStage + st * L::kStage;
        mbar_arrive_expect_tx(kv_full + st, L::kStage);
        const int row = t0 + c * kTile;
        tma_load_3d(base, &tm_v, kv_full + st, 0, row, bh);
        tma_load_3d(base + kVBytes, &tm_q, kv_full + st, 0, row, bh);
        tma_load_3d(base + kVBytes + L::kQKB, &tm_k, kv_full + st, 0, row, bh);
        ++issued;
      }
      for (int c = issued - kReadStages < 0 ? 0 : issued - kReadStages; c < issued; ++c)
        mbar_wait_drain(kv_full + c % kReadStages, (c / kReadStages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA
    // the whole warp runs this loop; one elected lane issues (see mma_ts_w)
    {
      constexpr uint32_t id_qk = idesc_bf16(128, 128, false, false);  // also psi~_S(Q) (TMEM) psi~_S(K)^T
      constexpr uint32_t id_rd = idesc_bf16(128, 80, false, false);  // A = psi~(Q) (TMEM), B = S~ K-major
      constexpr uint32_t id_wv = idesc_bf16(128, 80, false, true);   // A = W (TMEM), B = [V | 1]
      constexpr uint32_t id_u = idesc_bf16(128, kNP, true, true);    // A = [V | 1]^T, B = psi~(K)
      const uint32_t sStage = smem_u32(smem + L::offStage), sOnes = smem_u32(smem + L::offOnes);
      const uint32_t sPsi = smem_u32(smem + L::offPsi), sSB = smem_u32(smem + L::offSB);
      // descriptors built once; stages and K steps are constant offsets
      const uint64_t dq0 = smem_desc(sStage + kVBytes, 16, 256, kSw32);
      const uint64_t dk0 = smem_desc(sStage + kVBytes + L::kQKB, 16, 256, kSw32);
      const uint64_t dpsi = smem_desc(sPsi, kPsiAtom, 256, kSw32);
      const uint64_t dpsik = smem_desc(sPsi, 16, 256, kSw32);  // psi~_S(K) as a K-major B operand
      const uint64_t dsb0 = smem_desc(sSB, 16, 256, kSw32);
      for (int c = 0; c < n_chunks; ++c) {
        const int st = c % kReadStages, ob = c & 1;
        const uint32_t sV = sStage + st * L::kStage;
        // everything chunk c needs from warps 6-13; its tiles have landed
        KATA_TRACE(chunk, c, 0);
        if (!mbar_wait_w(state_full, c & 1, env)) break;
        KATA_TRACE(chunk, c, 1);
        tc_fence_after();
        // scores of chunk c (overwrite the weights of chunk c-1 only after
        // the intra-chunk MMAs of c-1 issued before them)
        if constexpr (NG == 1) {
          mma_ss_w(tmem + L::colS, desc_add(dq0, st * L::kStage), desc_add(dk0, st * L::kStage), id_qk, 0);
        } else {
          // the Sigma-g weights directly: psi~_S(Q_c) psi~_S(K_c)^T
#pragma unroll
          for (int ks = 0; ks < kNP / 16; ++ks)
            mma_ts_w(tmem + L::colS, tmem + L::colPQ + ks * 8, desc_add(dpsik, (c & 1) * kPsiBytes + ks * kPsiAtom),
                     id_qk, ks > 0);
        }
        mma_commit_w(s_full);
        // readout against the bf16 copy of the state entering the chunk (the
        // [O | D] buffer is free: see state_full); first, so that psi~(q_c)
        // is released early for psi~(q_{c+1})
        const uint64_t dsb = dsb0;
        const uint32_t dO = tmem + L::colO(ob);
#pragma unroll
        for (int ks = 0; ks < kNP / 16; ++ks)
          mma_ts_w(dO, tmem + L::colPQ + ks * 8, desc_add(dsb, ks * kSBAtom), id_rd, ks > 0);
        mma_commit_w(rd_done);
        KATA_TRACE(chunk, c, 2);
        // advance the state by the chunk
        const uint64_t dvo = desc_vones(sV, sOnes);
#pragma unroll
        for (int ks = 0; ks < kTile / 16; ++ks)
          mma_ss_w(tmem + L::colRun, desc_add(dvo, ks * 2048), desc_add(dpsi, (c & 1) * kPsiBytes + ks * 512), id_u, 1);
        mma_commit_w(upd_done);
        // intra-chunk weights against [V_c | 1]
        KATA_TRACE(chunk, c, 4);
        if (!mbar_wait_w(p_full, c & 1, env)) break;
        KATA_TRACE(chunk, c, 5);
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < kTile / 16; ++ks)
          mma_ts_w(dO, tmem + L::colS + (ks >> 2) * 64 + (ks & 3) * 8, desc_add(dvo, ks * 2048), id_wv, 1);
        mma_commit_w(o_full + ob);
        mma_commit_w(kv_empty + st);
        KATA_TRACE(chunk, c, 6);
      }
      mma_commit_w(mma_done);
      mbar_wait_drain(mma_done, 0);
    }
  } else if (warp < 6 || warp >= 14) {
    // ------------------------------------------------------------- weights + output
    // warps 2-5 take key columns 0..63 of the weights and value columns
    // 0..31 of the output, warps 14-17 the other halves; both warps of a
    // pair read the same TMEM lane quarter (rows 32 * quarter ..)
    const int quarter = warp % 4;
    const int h = warp >= 14 ? 1 : 0;
    const int m = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    uint8_t* slab = smem + L::offOut + (quarter * 2 + h) * (32 * 64);  // this warp's [32 x 32] output box
    // output of chunk co: read [O | D] out of TMEM, then (once the read is
    // done) arrive on state_full(co + 2) when that chunk exists, since the
    // readout of chunk co + 2 reuses this [O | D] buffer; then o = O / D
    // rounded to bf16, staged as this warp's 64B-swizzled [32 x 32] box of
    // the o tensor map (16-byte chunk j of row r at chunk j ^ ((r / 2) % 4))
    // and written by one TMA store (rows past T are not written)
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
      if (m == 0) KATA_TRACE(chunk, co, 14);
      const float D = __uint_as_float(db);
      if (D_out != nullptr && h == 0 && t0 + co * kTile + m < T) D_out[(size_t)bh * T + t0 + co * kTile + m] = D;
      const float inv = D > 0.f ? 1.f / D : 0.f;
      const uint64_t inv2 = f32x2(__float_as_uint(inv), __float_as_uint(inv));
      auto scaled = [&](int k) {
        const uint64_t v = f32x2_mul(f32x2(r[k], r[k + 1]), inv2);
        return pack_bf16x2(f32x2_lo(v), f32x2_hi(v));
      };
      // the warp's staging slab is free once its previous store has read it
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
    // the readouts of chunks 0 and 1 write fresh [O | D] buffers; an arrival
    // for state_full(c) is made only once state_full(c-1) has completed
    // (for c = 1: once the scores of chunk 0, issued after it, are in)
    if (n_chunks > 0) mbar_arrive(state_full);
    bool ok = true;
    for (int c = 0; ok && c < n_chunks; ++c) {
      if (!mbar_wait_w(s_full, c & 1, env)) break;
      if (c == 0 && n_chunks > 1) mbar_arrive(state_full);
      if (m == 0) KATA_TRACE(chunk, c, 8);
      tc_fence_after();
      // causal within the chunk: 32-column block bb of row m is fully kept
      // for bb < quarter, diagonal for bb == quarter, zero for bb > quarter.
      // Block bb's 16 bf16x2 words go to columns 64 (bb / 2) + 16 (bb % 2),
      // inside the half's own score columns and over scores already read.
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
          if constexpr (NG == 1) {
            // squares on fp32 pairs (each rounded as a scalar multiply)
            if (bb < quarter) {
#pragma unroll
              for (int x = 0; x < 16; ++x) {
                const uint64_t sq = f32x2_mul(f32x2(r[2 * x], r[2 * x + 1]), f32x2(r[2 * x], r[2 * x + 1]));
                w[x] = pack_bf16x2(f32x2_lo(sq), f32x2_hi(sq));
              }
            } else {
#pragma unroll
              for (int x = 0; x < 16; ++x) {
                const uint32_t a = 2 * x > lane ? 0u : r[2 * x], b = 2 * x + 1 > lane ? 0u : r[2 * x + 1];
                const uint64_t sq = f32x2_mul(f32x2(a, b), f32x2(a, b));
                w[x] = pack_bf16x2(f32x2_lo(sq), f32x2_hi(sq));
              }
            }
          } else {
            // the Sigma-g weights are the scores themselves
#pragma unroll
            for (int x = 0; x < 16; ++x) {
              const float a = bb == quarter && 2 * x > lane ? 0.f : __uint_as_float(r[2 * x]);
              const float b = bb == quarter && 2 * x + 1 > lane ? 0.f : __uint_as_float(r[2 * x + 1]);
              w[x] = pack_bf16x2(a, b);
            }
          }
        }
        tmem_st16(lane_base + L::colS + 64 * h + 16 * b2, w);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full);
      if (m == 0) KATA_TRACE(chunk, c, 9);
      // the output of the previous chunk, after these weights so that the
      // weights are never held up by it
      if (c > 0) ok = output(c - 1);
    }
    if (ok && n_chunks > 0) output(n_chunks - 1);
    if (lane == 0) bulk_wait_all();
  } else {
    // ------------------------------------------------------------- psi~ and state copies
    const bool psi_group = warp < 10;   // warps 6-9: psi~(k) + half 0; warps 10-13: half 1 + psi~(q)
    const int half = psi_group ? 0 : 1;
    const int quarter = warp % 4;
    const int m = quarter * 32 + lane;  // token of the chunk / TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    uint8_t* sb = smem + L::offSB;
    const bool active = m < kSBRows;    // rows 0..63 values, 64..79 copies of z
    // psi~(k) of chunk cc into shared-memory buffer cc % 2, or psi~(q) of
    // chunk cc into TMEM, from the chunk's landed stage
    auto psi_k = [&](int cc) {
      const uint8_t* tile = smem + L::offStage + (cc % kReadStages) * L::kStage + kVBytes + L::kQKB;
      uint8_t* dst = smem + L::offPsi + (cc & 1) * kPsiBytes;
      if constexpr (NG == 1) {
        __nv_bfloat162 u[8];
        uint32_t w[kNPW];
        load_row_sw<1>(tile, m, u);
        packed_psi<true>(u, w);
        store_psi_k(dst, m, w);
      } else {
        __nv_bfloat162 u[8 * NG];
        uint32_t w[kNPW / 2];
        load_row_sw<NG>(tile, m, u);
        packed_psi_sum_half<true, 0, NG>(u, w);
        store_psi_k_half<0>(dst, m, w);
        packed_psi_sum_half<true, 1, NG>(u, w);
        store_psi_k_half<1>(dst, m, w);
      }
    };
    auto psi_q_formed = [&](int cc, uint32_t (&w)[kNPW]) {
      __nv_bfloat162 u[8];
      load_row_sw<1>(smem + L::offStage + (cc % kReadStages) * L::kStage + kVBytes, m, u);
      packed_psi<false>(u, w);
    };
    // Sigma-g: psi~_S(q) of chunk cc into TMEM one half at a time (the
    // groups' values and a whole row do not fit in registers together);
    // `before` runs between forming the first half and storing it
    auto psi_q_sum_to_tmem = [&](int cc, auto&& before) -> bool {
      __nv_bfloat162 u[8 * NG];
      uint32_t w[kNPW / 2];
      load_row_sw<NG>(smem + L::offStage + (cc % kReadStages) * L::kStage + kVBytes, m, u);
      packed_psi_sum_half<false, 0, NG>(u, w);
      if (!before()) return false;
      store_psi_q_tmem_half<0>(lane_base + L::colPQ, w);
      packed_psi_sum_half<false, 1, NG>(u, w);
      store_psi_q_tmem_half<1>(lane_base + L::colPQ, w);
      return true;
    };
    // running state <- scanned prefix (fp32 into TMEM, bf16 into shared
    // memory); with a single super-chunk there is no workspace and the
    // prefix is the caller's initial state (or zero).  After a scan this
    // kernel is its programmatic dependent: wait for the scanned records.
    const int d = min(m, kRecRows - 1);  // record row of this lane
    griddep_wait();
    if (quarter < 3) {
      if (ws) {
        const float* row = ws + ((size_t)bh * G + g) * record_floats + (size_t)d * kNP;
        global_half_to_state(row, lane_base + L::colRun, sb, m, active, half);
      } else {
        const float* S = S0 ? S0 + (size_t)bh * 256 * kDV : nullptr;
        const float* z = z0 ? z0 + (size_t)bh * 256 : nullptr;
        if (half == 0) abi_half_to_state<0>(S, z, d, lane_base + L::colRun, sb, m, active);
        else abi_half_to_state<1>(S, z, d, lane_base + L::colRun, sb, m, active);
      }
    }
    // chunk 0's psi~(k) or psi~(q): they need nothing but its stage
    bool ok = n_chunks > 0 && mbar_wait_w(kv_full, 0, env);
    if (ok) {
      if (psi_group) {
        psi_k(0);
      } else if constexpr (NG == 1) {
        uint32_t w[kNPW];
        psi_q_formed(0, w);
        store_psi_q_tmem(lane_base + L::colPQ, w);
      } else {
        psi_q_sum_to_tmem(0, [] { return true; });
      }
    }
    tmem_wait_st();
    fence_proxy_async_smem();
    tc_fence_before();
    if (ok) mbar_arrive(state_full);
    for (int c = 0; ok && c + 1 < n_chunks; ++c) {
      // operands of chunk c+1, whose tiles land in stage (c+1) % kReadStages
      const int st1 = (c + 1) % kReadStages;
      if (!mbar_wait_w(kv_full + st1, ((c + 1) / kReadStages) & 1, env)) break;
      if (psi_group) {
        // psi~(k_{c+1}) into the buffer last read by the advance by chunk
        // c-1, which this group saw complete in the previous iteration
        psi_k(c + 1);
        if (m == 0) KATA_TRACE(chunk, c, 11);
      } else if constexpr (NG == 1) {
        // psi~(q_{c+1}) into TMEM once the readout of chunk c (the first MMAs
        // of the chunk) has read psi~(q_c)
        uint32_t wq[kNPW];
        psi_q_formed(c + 1, wq);
        if (!mbar_wait_w(rd_done, c & 1, env)) break;
        if (m == 0) KATA_TRACE(chunk, c, 19);
        tc_fence_after();
        store_psi_q_tmem(lane_base + L::colPQ, wq);
        tmem_wait_st();
      } else {
        // the same; the readout of chunk c also ends the scores' use of
        // psi~_S(q_c), issued before it
        if (!psi_q_sum_to_tmem(c + 1, [&] {
              if (!mbar_wait_w(rd_done, c & 1, env)) return false;
              tc_fence_after();
              return true;
            }))
          break;
        tmem_wait_st();
      }
      // the state after chunk c is complete: this group's half of the bf16
      // copy for the readout of chunk c+1 (the copy was last read by the
      // readout of chunk c, which completed before this advance did)
      if (!mbar_wait_w(upd_done, c & 1, env)) break;
      if (m == 0) KATA_TRACE(chunk, c, psi_group ? 15 : 16);
      tc_fence_after();
      if (quarter < 3) state_half_to_bf16(lane_base + L::colRun, sb, m, active, half);
      if (m == 0) KATA_TRACE(chunk, c, psi_group ? 17 : 18);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(state_full);
      if (m == 0) KATA_TRACE(chunk, c, psi_group ? 12 : 13);
    }
    // the last super-chunk ends at token T: its running state, once the
    // advance by its last chunk has landed, is the final state
    if (S_out && g == G - 1 && n_chunks > 0 && mbar_wait_w(upd_done, (n_chunks - 1) & 1, env) &&
        quarter < 3) {
      tc_fence_after();
      float* S = S_out + (size_t)bh * 256 * kDV;
      float* z = z_out + (size_t)bh * 256;
      if (half == 0) state_half_to_abi<0>(lane_base + L::colRun, S, z, m, m < kRecRows);
      else state_half_to_abi<1>(lane_base + L::colRun, S, z, m, m < kRecRows);
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

size_t chunk_record_floats_sm100() { return (size_t)kRecRows * kNP; }

namespace {

template <int NG>
cudaError_t launch_state_t(const void* k, const void* v, float* ws, const ChunkPlan& pl, const WaitCtl& wc,
                           cudaStream_t st) {
  using L = StateSmem<NG>;
  if (pl.p != 16 || pl.dv != kDV) return cudaErrorInvalidValue;
  CUtensorMap tk, tv;
  if (!make_tmap_bf16(&tk, k, ChunkCfg<NG>::kD, pl.T, pl.BH, kTile) ||
      !make_tmap_bf16(&tv, v, kDV, pl.T, pl.BH, kTile))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(chunk_state_kernel<NG>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
  if (e != cudaSuccess) return e;
  if (pl.G < 2) return cudaSuccess;  // the last super-chunk's sum is never needed
  dim3 grid(pl.G - 1, pl.BH);
  chunk_state_kernel<NG><<<grid, kStateThreads, L::kBytes, st>>>(tk, tv, ws, pl.T, pl.Ls, pl.G,
                                                                  (long long)pl.record_floats, wc);
  return cudaGetLastError();
}

template <int NG>
cudaError_t launch_readout_t(const void* q, const void* k, const void* v, void* o, const float* ws, const float* S0,
                             const float* z0, float* S_out, float* z_out, const ChunkPlan& pl, const WaitCtl& wc,
                             cudaStream_t st, float* D_out = nullptr) {
  using L = ReadSmem<NG>;
  if (pl.p != 16 || pl.dv != kDV) return cudaErrorInvalidValue;
  if (!ws && pl.G != 1) return cudaErrorInvalidValue;
  constexpr int kD = ChunkCfg<NG>::kD;
  CUtensorMap tq, tk, tv, to;
  if (!make_tmap_bf16(&tq, q, kD, pl.T, pl.BH, kTile) || !make_tmap_bf16(&tk, k, kD, pl.T, pl.BH, kTile) ||
      !make_tmap_bf16(&tv, v, kDV, pl.T, pl.BH, kTile) || !make_tmap_bf16_box(&to, o, kDV, pl.T, pl.BH, 32, 32))
    return cudaErrorInvalidValue;
  cudaError_t e =
      cudaFuncSetAttribute(chunk_readout_kernel<NG>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
  if (e != cudaSuccess) return e;
  const dim3 grid(pl.G, pl.BH), block(kReadThreads);
  if (ws)  // after the state build and scan of this call: launched as the scan's programmatic dependent
    return launch_pdl(chunk_readout_kernel<NG>, grid, block, (size_t)L::kBytes, st, tq, tk, tv, to,
                      (const float*)ws, S0, z0, S_out, z_out, D_out, pl.T, pl.Ls, pl.G, (long long)pl.record_floats,
                      wc);
  chunk_readout_kernel<NG><<<grid, block, L::kBytes, st>>>(tq, tk, tv, to, ws, S0, z0, S_out, z_out, D_out, pl.T,
                                                           pl.Ls, pl.G, (long long)pl.record_floats, wc);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_state_sm100(const void* k, const void* v, float* ws, const ChunkPlan& pl, const WaitCtl& wc,
                                     cudaStream_t st) {
  return launch_state_t<1>(k, v, ws, pl, wc, st);
}

cudaError_t launch_chunk_readout_sm100(const void* q, const void* k, const void* v, void* o, const float* ws,
                                       const float* S0, const float* z0, float* S_out, float* z_out,
                                       const ChunkPlan& pl, const WaitCtl& wc, cudaStream_t st, float* D_out) {
  return launch_readout_t<1>(q, k, v, o, ws, S0, z0, S_out, z_out, pl, wc, st, D_out);
}

cudaError_t launch_chunk_state_sg(const void* k, const void* v, float* ws, const ChunkPlan& pl, int groups,
                                  const WaitCtl& wc, cudaStream_t st) {
  if (groups == 2) return launch_state_t<2>(k, v, ws, pl, wc, st);
  if (groups == 4) return launch_state_t<4>(k, v, ws, pl, wc, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_chunk_readout_sg(const void* q, const void* k, const void* v, void* o, const float* ws,
                                    const float* S0, const float* z0, float* S_out, float* z_out,
                                    const ChunkPlan& pl, int groups, const WaitCtl& wc, cudaStream_t st) {
  if (groups == 2) return launch_readout_t<2>(q, k, v, o, ws, S0, z0, S_out, z_out, pl, wc, st);
  if (groups == 4) return launch_readout_t<4>(q, k, v, o, ws, S0, z0, S_out, z_out, pl, wc, st);
  return cudaErrorInvalidValue;
}

}  // namespace kata
