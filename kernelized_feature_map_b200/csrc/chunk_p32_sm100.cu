// chunk_p32_sm100.cu -- exact O(T) chunked-state KATA forward for p = 32
// (bf16 inputs, dv = 64) on tcgen05 / TMEM, with the state split over a
// cluster of four CTAs.
//
// State size.  For p = 32 the packed feature has n = p(p+1)/2 = 528
// coordinates (ai.info summary, Main Findings, "State size, not just feature
// width, dominates memory"); the transposed fp32 state would need 544 TMEM
// columns of the 512 an SM has.  Writing u = [a | b] with a, b the two
// halves of 16 coordinates,
//
//   (q . k)^2 = (q_a . k_a)^2 + (q_b . k_b)^2 + 2 (q_a . k_a)(q_b . k_b),
//
// so the feature splits into four blocks of at most 144 coordinates:
//   block 0   psi~(a): the packed p = 16 feature of the first half (136 + 8 pads)
//   block 1   psi~(b): the same for the second half
//   block 2   a_i b_j for i = 0..7,  j = 0..15 (128 + 16 pads), key side x 2
//   block 3   a_i b_j for i = 8..15, j = 0..15
// with <psi~_0(q), psi~_0(k)> + ... + <psi~_3(q), psi~_3(k)> = (q . k)^2.
// Each block is the size of the p = 16 state, so each CTA of a cluster of
// four holds one block's transposed state S~_b^T in the TMEM layout of the
// p = 16 kernel and computes, per 128-token chunk c,
//   [O | D]_b = psi~_b(Q_c) S~_b        (readout against the state entering c)
//   S~_b^T  += [V_c | 1]^T psi~_b(K_c)  (advance)
// and CTA 0 adds the intra-chunk squared-score attention W_c [V_c | 1].  The
// numerator and denominator of a token are sums over the four blocks: the
// warps of TMEM lane quarter q in every CTA send their rows of [O | D]_b to
// CTA q through distributed shared memory, and two warps of CTA q add the
// four partial rows, form o = O / D and store rows 32q .. 32q+31 of the
// chunk.
//
// Launches per call, as on the p = 16 path (G super-chunks per (b,h)):
//  1. chunk_state_p32_kernel (G > 1) per super-chunk g < G-1 and block:
//                            A_{g,b} = sum over its chunks;
//  2. state_scan             (G > 1, scan.cu) exclusive prefix over g of the
//                            4 B H block sequences;
//  3. chunk_readout_p32_kernel, clusters of four CTAs (one per block) per
//                            (b,h, super-chunk), starting from the scanned
//                            prefix plus the caller's initial state; the
//                            cluster of the last super-chunk writes the final
//                            state.
#include <cuda.h>

#include "chunk_common.cuh"
#include "kata_internal.h"

namespace kata {

bool make_tmap_bf16(CUtensorMap* map, const void* base, int inner, int T, int BH, int rows);
bool make_tmap_bf16_box(CUtensorMap* map, const void* base, int inner, int T, int BH, int box_inner, int rows);

namespace {

using namespace sm100;
using namespace chunk;

constexpr int kBlocks = 4;                  // cluster size: one CTA per coordinate block
constexpr int kQK32Bytes = kTile * 32 * 2;  // Q or K tile: 64-byte rows, 64B swizzle

// ---------------------------------------------------------------------------
// cluster primitives (distributed shared memory)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the variable at local shared address `a` in CTA `rank`
__device__ __forceinline__ uint32_t map_rank(uint32_t a, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_cluster_v4(uint32_t a, float x, float y, float z, float w) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(x), "f"(y), "f"(z), "f"(w)
               : "memory");
}
__device__ __forceinline__ void st_cluster_f32(uint32_t a, float x) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(a), "f"(x) : "memory");
}
// arrive on an mbarrier of a CTA of the cluster, releasing this thread's
// earlier writes at cluster scope
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait, with acquire at cluster scope, on a local mbarrier that other
// CTAs of the cluster arrive on (same contract as mbar_wait); warp-uniform.
__device__ __forceinline__ bool mbar_wait_cluster_w(uint64_t* bar, uint32_t parity, const WaitEnv& env) {
  bool ok = true;
  if (env.limit == 0) {
    ok = mbar_try_wait_cluster(bar, parity);
  } else if (!mbar_try_wait_cluster(bar, parity)) {
    const long long t0 = clock64();
    while (true) {
      if (*env.abort_flag) {
        ok = false;
        break;
      }
      if (clock64() - t0 >= env.limit) {
        *env.abort_flag = 1;
        report_status(env.status, kErrTimeout);
        ok = false;
        break;
      }
      if (mbar_try_wait_cluster(bar, parity)) break;
    }
  }
  if (!ok && env.limit == 0) {
    *env.abort_flag = 1;
    report_status(env.status, kErrTimeout);
  }
  return __all_sync(0xffffffffu, ok);
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// block psi~ formation from a row of 32 bf16 values
// ---------------------------------------------------------------------------
// Row r of a 64B-swizzled [128 x 32] bf16 tile (16-byte chunk c of row r at
// chunk c ^ ((r >> 1) & 3)) -> a = u[0..7], b = u[8..15] (bf16 pairs).
__device__ __forceinline__ void load_row_sw64(const uint8_t* tile, int r, __nv_bfloat162 (&u)[16]) {
  const uint8_t* row = tile + r * 64;
  const int x = (r >> 1) & 3;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 a = *reinterpret_cast<const uint4*>(row + ((c ^ x) << 4));
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) u[4 * c + e] = *reinterpret_cast<const __nv_bfloat162*>(&w[e]);
  }
}

// Block 2 or 3: word il*8 + jp = (a_i b_{2jp}, a_i b_{2jp+1}) for the eight
// a_i of the block (x 2 on the key side, exact), then 8 zero words (pads).
template <bool key>
__device__ __forceinline__ void cross_psi(const __nv_bfloat162 (&a4)[4], const __nv_bfloat162 (&b)[8],
                                          uint32_t (&out)[kNPW]) {
#pragma unroll
  for (int il = 0; il < 8; ++il) {
    const __nv_bfloat16 ai = (il & 1) ? a4[il >> 1].y : a4[il >> 1].x;
    const __nv_bfloat16 f = key ? __hmul(ai, __float2bfloat16_rn(2.f)) : ai;
    const __nv_bfloat162 f2 = __halves2bfloat162(f, f);
#pragma unroll
    for (int jp = 0; jp < 8; ++jp) out[il * 8 + jp] = as_u32(__hmul2(f2, b[jp]));
  }
#pragma unroll
  for (int w = 64; w < kNPW; ++w) out[w] = 0u;
}

// The 72 words of block `blk`'s psi~ of one token (blk is uniform per CTA).
template <bool key>
__device__ __forceinline__ void block_psi(const __nv_bfloat162 (&u)[16], int blk, uint32_t (&out)[kNPW]) {
  if (blk < 2) {
    __nv_bfloat162 h[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) h[e] = blk == 0 ? u[e] : u[8 + e];
    packed_psi<key>(h, out);
  } else {
    __nv_bfloat162 a4[4], b[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) a4[e] = blk == 2 ? u[e] : u[4 + e];
#pragma unroll
    for (int e = 0; e < 8; ++e) b[e] = u[8 + e];
    cross_psi<key>(a4, b, out);
  }
}

// ---------------------------------------------------------------------------
// block coordinates <-> the ABI state layout (S [p*p, dv], z [p*p], p = 32,
// psi index r = i*32 + j)
// ---------------------------------------------------------------------------
// Packed coordinate w of block blk -> ABI rows r1 and r2 (r2 = -1 on the
// diagonal; r1 = -1 for a pad).  The packed value is the sum of both rows.
__device__ __forceinline__ void block_coord(int blk, int w, int& r1, int& r2) {
  if (blk < 2) {
    const int i = packed_i(w), j = packed_j(w), o = 16 * blk;
    r1 = i < 0 ? -1 : (i + o) * 32 + (j + o);
    r2 = (i < 0 || i == j) ? -1 : (j + o) * 32 + (i + o);
  } else {
    const int il = w >> 4, j = w & 15, i = 8 * (blk - 2) + il;
    r1 = w < 128 ? i * 32 + 16 + j : -1;
    r2 = w < 128 ? (16 + j) * 32 + i : -1;
  }
}

// Initial value of word w (packed coordinate) of row d (<= 64) of block blk:
// the scanned record's entry (when `rec`) plus the caller's initial state
// (when S).
__device__ __forceinline__ float prefix_entry(const float* rec, const float* S, const float* z, int blk, int d,
                                              int w) {
  float v = rec ? rec[w] : 0.f;
  if (S) {
    int r1, r2;
    block_coord(blk, w, r1, r2);
    if (r1 >= 0) {
      if (d < kDV) v += S[r1 * kDV + d] + (r2 >= 0 ? S[r2 * kDV + d] : 0.f);
      else v += z[r1] + (r2 >= 0 ? z[r2] : 0.f);
    }
  }
  return v;
}

// Half `half` of the prefix row d into the TMEM lane and the bf16 copy row n.
// Warp-collective.
template <int half>
__device__ __forceinline__ void prefix_half_to_state(const float* rec, const float* S, const float* z, int blk, int d,
                                                     uint32_t taddr, uint8_t* sb, int n, bool active) {
  uint32_t r[72];
#pragma unroll
  for (int e = 0; e < 72; ++e) r[e] = __float_as_uint(active ? prefix_entry(rec, S, z, blk, d, 72 * half + e) : 0.f);
  if (half == 0) {
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      tmem_st16(taddr + 16 * a, *reinterpret_cast<const uint32_t(*)[16]>(r + 16 * a));
      if (active) store_state_bf16_atom(sb, n, a, r + 16 * a);
    }
    tmem_st8(taddr + 64, *reinterpret_cast<const uint32_t(*)[8]>(r + 64));
    if (active) store_state_bf16_chunk(sb, n, 4, 0, r + 64);
  } else {
    tmem_st8(taddr + 72, *reinterpret_cast<const uint32_t(*)[8]>(r));
    if (active) store_state_bf16_chunk(sb, n, 4, 1, r);
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      tmem_st16(taddr + 80 + 16 * a, *reinterpret_cast<const uint32_t(*)[16]>(r + 8 + 16 * a));
      if (active) store_state_bf16_atom(sb, n, 5 + a, r + 8 + 16 * a);
    }
  }
}

// Half `half` of TMEM lane d (<= 64) of block blk's final state -> the ABI
// layout (an off-diagonal packed entry is halved into its two rows, exactly).
// Warp-collective.
template <int half>
__device__ __forceinline__ void block_state_to_abi(uint32_t taddr, float* S, float* z, int blk, int d, bool active) {
  uint32_t r[72];
  if (half == 0) {
    tmem_ld32(taddr, *reinterpret_cast<uint32_t(*)[32]>(r));
    tmem_ld32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(r + 32));
    tmem_ld8(taddr + 64, *reinterpret_cast<uint32_t(*)[8]>(r + 64));
  } else {
    tmem_ld8(taddr + 72, *reinterpret_cast<uint32_t(*)[8]>(r));
    tmem_ld32(taddr + 80, *reinterpret_cast<uint32_t(*)[32]>(r + 8));
    tmem_ld32(taddr + 112, *reinterpret_cast<uint32_t(*)[32]>(r + 40));
  }
  tmem_wait_ld();
  if (!active) return;
#pragma unroll
  for (int e = 0; e < 72; ++e) {
    int r1, r2;
    block_coord(blk, 72 * half + e, r1, r2);
    if (r1 < 0) continue;
    const float val = __uint_as_float(r[e]);
    const float hv = r2 < 0 ? val : 0.5f * val;
    if (d < kDV) {
      S[r1 * kDV + d] = hv;
      if (r2 >= 0) S[r2 * kDV + d] = hv;
    } else {
      z[r1] = hv;
      if (r2 >= 0) z[r2] = hv;
    }
  }
}

// ===========================================================================
// 1. per-super-chunk block state sums
// ===========================================================================
constexpr int kStateThreads = 320;  // warp 0 TMA, warp 1 MMA, warps 2-9 psi~(k), warps 2-5 record
constexpr int kStateStages = 5;

struct State32Smem {
  static constexpr int kStage = kVBytes + kQK32Bytes;  // [V | K]
  static constexpr int offStage = 0;
  static constexpr int offOnes = offStage + kStateStages * kStage;  // 1024-aligned
  static constexpr int offPsi = offOnes + kOnesBytes;                 // 2 buffers
  static constexpr int offBar = offPsi + 2 * kPsiBytes;
  static constexpr int kBars = 2 * kStateStages + 4 + 1;
  static constexpr int offMisc = offBar + kBars * 8;
  static constexpr int kBytes = offMisc + 16 + 1024;
};

// grid (G - 1, BH, 4): super-chunk g, sequence bh, block blockIdx.z; record
// ((bh * 4 + blk) * G + g) of the workspace.
__global__ void __launch_bounds__(kStateThreads, 1)
    chunk_state_p32_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                           float* __restrict__ ws, int T, int Ls, int G, long long record_floats, WaitCtl wc) {
  using L = State32Smem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::offBar);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + kStateStages;
  uint64_t* psi_full = kv_empty + kStateStages;  // [2]
  uint64_t* psi_empty = psi_full + 2;            // [2]
  uint64_t* acc_done = psi_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::offMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::offMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x, bh = blockIdx.y, blk = blockIdx.z;
  const int t0 = g * Ls;
  const int n_chunks = (min(T, t0 + Ls) - t0 + kTile - 1) / kTile;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStateStages; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
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
        mbar_arrive_expect_tx(kv_full + st, L::kStage);
        tma_load_3d(base, &tm_v, kv_full + st, 0, t0 + c * kTile, bh);
        tma_load_3d(base + kVBytes, &tm_k, kv_full + st, 0, t0 + c * kTile, bh);
        ++issued;
      }
      for (int c = issued - kStateStages < 0 ? 0 : issued - kStateStages; c < issued; ++c)
        mbar_wait_drain(kv_full + c % kStateStages, (c / kStateStages) & 1);
    }
  } else if (warp == 1) {
    constexpr uint32_t id_u = idesc_bf16(128, kNP, true, true);
    const uint32_t sStage = smem_u32(smem + L::offStage), sOnes = smem_u32(smem + L::offOnes);
    const uint64_t dpsi = smem_desc(smem_u32(smem + L::offPsi), kPsiAtom, 256, kSw32);
    for (int c = 0; c < n_chunks; ++c) {
      const int st = c % kStateStages, pb = c & 1;
      if (!mbar_wait_w(kv_full + st, (c / kStateStages) & 1, env)) break;
      if (!mbar_wait_w(psi_full + pb, (c >> 1) & 1, env)) break;
      tc_fence_after();
      const uint64_t da = desc_vones(sStage + st * L::kStage, sOnes), db = desc_add(dpsi, pb * kPsiBytes);
#pragma unroll
      for (int ks = 0; ks < kTile / 16; ++ks)
        mma_ss_w(tmem, desc_add(da, ks * 2048), desc_add(db, ks * 512), id_u, (c > 0 || ks > 0) ? 1u : 0u);
      mma_commit_w(psi_empty + pb);
      mma_commit_w(kv_empty + st);
    }
    mma_commit_w(acc_done);
    mbar_wait_drain(acc_done, 0);
  } else {
    // warps 2-9: token (warp - 2) % 4 * 32 + lane, half (warp - 2) / 4 of its words
    const int tid = ((warp - 2) & 3) * 32 + lane;
    const int half = (warp - 2) >> 2;
    const int quarter = warp % 4;
    const int d = quarter * 32 + lane;  // TMEM lane = record row
    bool ok = true;
    for (int c = 0; c < n_chunks; ++c) {
      const int st = c % kStateStages, pb = c & 1;
      if (!mbar_wait_w(kv_full + st, (c / kStateStages) & 1, env)) {
        ok = false;
        break;
      }
      if (c >= 2 && !mbar_wait_w(psi_empty + pb, ((c >> 1) - 1) & 1, env)) {
        ok = false;
        break;
      }
      __nv_bfloat162 u[16];
      load_row_sw64(smem + L::offStage + st * L::kStage + kVBytes, tid, u);
      uint32_t w[kNPW];
      block_psi<true>(u, blk, w);
      uint32_t wh[kNPW / 2];
#pragma unroll
      for (int e = 0; e < kNPW / 2; ++e) wh[e] = half == 0 ? w[e] : w[kNPW / 2 + e];
      if (half == 0) store_psi_k_half<0>(smem + L::offPsi + pb * kPsiBytes, tid, wh);
      else store_psi_k_half<1>(smem + L::offPsi + pb * kPsiBytes, tid, wh);
      fence_proxy_async_smem();
      mbar_arrive(psi_full + pb);
    }
    // record rows 0..64 live in TMEM lanes 0..64: warps of lane quarters 0-2
    // load (the load is warp-collective), lanes below 65 store
    if (ok && warp < 6 && quarter < 3 && mbar_wait_w(acc_done, 0, env)) {
      tc_fence_after();
      float* row = ws + (((size_t)bh * kBlocks + blk) * G + g) * record_floats + (size_t)min(d, kRecRows - 1) * kNP;
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
// 3. readout, one cluster of four CTAs (blocks) per (b,h, super-chunk)
// ===========================================================================
// Warp roles (640 threads):
//   warp 0       TMA: [V | Q | K] tiles of each chunk into a 2-stage ring
//   warp 1       TMEM allocator; MMA issue (the whole warp, one elected lane)
//   warps 2-5,   block 0: weights W = (Q K^T)^2 (causal) into TMEM; every
//   14-17        block: the rows of [O | D]_b of lane quarter q (columns
//                split between the two warps of a quarter) sent to CTA q
//   warps 6-9    psi~_b(k_{c+1}) into shared memory (two buffers); bf16 copy
//                of packed coordinates 0..71 of S~_b after chunk c
//   warps 10-13  prefix in; psi~_b(q_{c+1}) into TMEM once the readout of
//                chunk c has read psi~_b(q_c); bf16 copy of coordinates 72..143
//   warps 18-19  the four partial rows of this CTA's 32 output rows summed,
//                o = O / D, stored (columns 0..31 and 32..63)
// MMA order per chunk: [block 0: scores], readout, advance, [block 0:
// intra-chunk weights].  The bf16 copy of S~_b has one buffer: it is
// refreshed once the advance by chunk c has landed, and the readout of chunk
// c, issued before that advance, has then completed.
// Cluster exchange per chunk: slot[src][row][68 floats] in the receiving CTA
// (O columns 0..63, D at 64); recv_full (256 arrivals: 4 CTAs x 2 warps x 32
// lanes) completes when all four blocks' rows of the chunk are in;
// recv_empty[q] in the sending CTA (64 arrivals from CTA q's two adding
// warps) completes when CTA q has read them, so the slot may be reused.
constexpr int kRead32Threads = 640;
constexpr int kRead32Stages = 2;
constexpr int kSlotFloats = 68;                       // per row: O (64), D, pad
constexpr int kSlotBytes = 32 * kSlotFloats * 4;      // one source's 32 rows

struct Read32Smem {
  static constexpr int kStage = kVBytes + 2 * kQK32Bytes;  // [V | Q | K]
  static constexpr int offStage = 0;
  static constexpr int offOnes = offStage + kRead32Stages * kStage;  // 1024-aligned
  static constexpr int offPsi = offOnes + kOnesBytes;                  // 2 buffers
  static constexpr int offSB = offPsi + 2 * kPsiBytes;                 // 1 buffer
  static constexpr int offSlot = offSB + kSBBytes;                     // [4 sources]
  static constexpr int offOut = (offSlot + kBlocks * kSlotBytes + 1023) / 1024 * 1024;  // 2 boxes [32 x 32] bf16, 64B swizzle
  static constexpr int offBar = offOut + 2 * 32 * 64;
  static constexpr int kBars = 2 * kRead32Stages + 9 + kBlocks;
  static constexpr int offMisc = offBar + kBars * 8;
  static constexpr int kBytes = offMisc + 16 + 1024;
  static constexpr uint32_t colRun = 0;                                    // S~_b^T, 144
  static constexpr uint32_t colO(int b) { return 144u + 80u * (uint32_t)b; }  // [O | D] x 2
  static constexpr uint32_t colPQ = 304;                                   // psi~_b(Q_c), 72
  static constexpr uint32_t colS = 384;                                    // scores / weights, 128
};
static_assert(Read32Smem::offSlot % 16 == 0 && Read32Smem::offOut % 1024 == 0 && Read32Smem::offSB % 1024 == 0 &&
                  Read32Smem::kBytes <= 232448,
              "shared-memory layout");

__global__ void __cluster_dims__(1, 1, kBlocks) __launch_bounds__(kRead32Threads, 1)
    chunk_readout_p32_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                             const float* __restrict__ ws, const float* __restrict__ S0, const float* __restrict__ z0,
                             float* __restrict__ S_out, float* __restrict__ z_out, int T, int Ls, int G,
                             long long record_floats, WaitCtl wc) {
  using L = Read32Smem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::offBar);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + kRead32Stages;
  uint64_t* s_full = kv_empty + kRead32Stages;  // scores in TMEM (block 0)
  uint64_t* p_full = s_full + 1;                // weights written (block 0, 256)
  uint64_t* state_full = p_full + 1;            // chunk c's operands ready, its [O | D] buffer free (512)
  uint64_t* rd_done = state_full + 1;           // readout of the chunk done
  uint64_t* upd_done = rd_done + 1;             // state advanced by the chunk
  uint64_t* o_full = upd_done + 1;              // [2] [O | D] complete
  uint64_t* mma_done = o_full + 2;
  uint64_t* recv_full = mma_done + 1;           // all four blocks' rows of the chunk received (256)
  uint64_t* recv_empty = recv_full + 1;         // [4] CTA q has read this CTA's rows (64)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::offMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::offMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int blk = (int)cluster_rank();
  const bool intra = blk == 0;
  const int g = blockIdx.x, bh = blockIdx.y;
  const int t0 = g * Ls;
  const int t1 = min(T, t0 + Ls);
  const int n_chunks = (t1 - t0 + kTile - 1) / kTile;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRead32Stages; ++s) {
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
    mbar_init(recv_full, 256);
    for (int b = 0; b < kBlocks; ++b) mbar_init(recv_empty + b, 64);
    *abort_flag = 0;
    fence_barrier_init();
  }
  fill_ones(smem + L::offOnes, threadIdx.x, kRead32Threads);
  fence_proxy_async_smem();
  if (warp == 1) tmem_alloc(tmem_holder, 512);
  tc_fence_before();
  __syncthreads();
  // every CTA's barriers are initialised before any CTA arrives on them remotely
  cluster_sync_all();
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
        const int st = c % kRead32Stages;
        if (!mbar_wait(kv_empty + st, ((c / kRead32Stages) & 1) ^ 1, env)) break;
        uint8_t* base = smem + L::offStage + st * L::kStage;
        mbar_arrive_expect_tx(kv_full + st, L::kStage);
        const int row = t0 + c * kTile;
        tma_load_3d(base, &tm_v, kv_full + st, 0, row, bh);
        tma_load_3d(base + kVBytes, &tm_q, kv_full + st, 0, row, bh);
        tma_load_3d(base + kVBytes + kQK32Bytes, &tm_k, kv_full + st, 0, row, bh);
        ++issued;
      }
      for (int c = issued - kRead32Stages < 0 ? 0 : issued - kRead32Stages; c < issued; ++c)
        mbar_wait_drain(kv_full + c % kRead32Stages, (c / kRead32Stages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA
    constexpr uint32_t id_qk = idesc_bf16(128, 128, false, false);
    constexpr uint32_t id_rd = idesc_bf16(128, 80, false, false);  // A = psi~(Q) (TMEM), B = S~ K-major
    constexpr uint32_t id_wv = idesc_bf16(128, 80, false, true);   // A = W (TMEM), B = [V | 1]
    constexpr uint32_t id_u = idesc_bf16(128, kNP, true, true);    // A = [V | 1]^T, B = psi~(K)
    const uint32_t sStage = smem_u32(smem + L::offStage), sOnes = smem_u32(smem + L::offOnes);
    const uint32_t sPsi = smem_u32(smem + L::offPsi), sSB = smem_u32(smem + L::offSB);
    // Q and K tiles: K-major, 64-byte rows, 64B swizzle (8-row groups 512 B
    // apart); the second 16-element K step starts 32 bytes into the rows
    const uint64_t dq0 = smem_desc(sStage + kVBytes, 16, 512, kSw64);
    const uint64_t dk0 = smem_desc(sStage + kVBytes + kQK32Bytes, 16, 512, kSw64);
    const uint64_t dpsi = smem_desc(sPsi, kPsiAtom, 256, kSw32);
    const uint64_t dsb = smem_desc(sSB, 16, 256, kSw32);
    for (int c = 0; c < n_chunks; ++c) {
      const int st = c % kRead32Stages, ob = c & 1;
      const uint32_t sV = sStage + st * L::kStage;
      if (!mbar_wait_w(state_full, c & 1, env)) break;
      tc_fence_after();
      if (intra) {
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
          mma_ss_w(tmem + L::colS, desc_add(dq0, st * L::kStage + ks * 32), desc_add(dk0, st * L::kStage + ks * 32),
                   id_qk, ks);
        mma_commit_w(s_full);
      }
      const uint32_t dO = tmem + L::colO(ob);
#pragma unroll
      for (int ks = 0; ks < kNP / 16; ++ks)
        mma_ts_w(dO, tmem + L::colPQ + ks * 8, desc_add(dsb, ks * kSBAtom), id_rd, ks > 0);
      mma_commit_w(rd_done);
      if (!intra) mma_commit_w(o_full + ob);
      const uint64_t dvo = desc_vones(sV, sOnes);
#pragma unroll
      for (int ks = 0; ks < kTile / 16; ++ks)
        mma_ss_w(tmem + L::colRun, desc_add(dvo, ks * 2048), desc_add(dpsi, (c & 1) * kPsiBytes + ks * 512), id_u, 1);
      mma_commit_w(upd_done);
      if (intra) {
        if (!mbar_wait_w(p_full, c & 1, env)) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < kTile / 16; ++ks)
          mma_ts_w(dO, tmem + L::colS + (ks >> 2) * 64 + (ks & 3) * 8, desc_add(dvo, ks * 2048), id_wv, 1);
        mma_commit_w(o_full + ob);
      }
      mma_commit_w(kv_empty + st);
    }
    mma_commit_w(mma_done);
    mbar_wait_drain(mma_done, 0);
  } else if (warp < 6 || (warp >= 14 && warp < 18)) {
    // ------------------------------------------------------------- weights (block 0) + partial rows out
    const int quarter = warp % 4;
    const int h = warp >= 14 ? 1 : 0;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    // this warp's 32 rows go to CTA `quarter`, into its slot of source blk
    const uint32_t slot_local = smem_u32(smem + L::offSlot + blk * kSlotBytes + lane * kSlotFloats * 4);
    const uint32_t slot_remote = map_rank(slot_local, (uint32_t)quarter);
    const uint32_t full_remote = map_rank(smem_u32(recv_full), (uint32_t)quarter);
    auto send = [&](int co) -> bool {
      const int ob = co & 1;
      if (!mbar_wait_w(o_full + ob, (co >> 1) & 1, env)) return false;
      tc_fence_after();
      uint32_t r[32], db;
      tmem_ld32(lane_base + L::colO(ob) + 32 * h, r);
      tmem_ld1(lane_base + L::colO(ob) + 64, db);
      tmem_wait_ld();
      tc_fence_before();
      // the readout of chunk co+2 reuses this [O | D] buffer.  An arrival on
      // state_full for chunk co+2 must come after its phase for chunk co+1
      // has completed, or it would count towards that phase: in CTA 0 the
      // weights of chunk co+1, which wait for its scores, come first; the
      // other CTAs have no weights and wait for the phase here
      if (co + 2 < n_chunks) {
        if (!intra && !mbar_wait_w(state_full, (co + 1) & 1, env)) return false;
        mbar_arrive(state_full);
      }
      // CTA `quarter` has read what this warp sent for chunk co-1
      if (co > 0 && !mbar_wait_cluster_w(recv_empty + quarter, (co - 1) & 1, env)) return false;
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        st_cluster_v4(slot_remote + (32 * h + e) * 4, __uint_as_float(r[e]), __uint_as_float(r[e + 1]),
                      __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
      if (h == 0) st_cluster_f32(slot_remote + 64 * 4, __uint_as_float(db));
      mbar_arrive_cluster(full_remote);
      return true;
    };
    bool ok = true;
    if (n_chunks > 0) mbar_arrive(state_full);
    if (n_chunks > 1) {
      // the readout of chunk 1 writes a fresh [O | D] buffer too; arrive for
      // it once state_full(0) has completed
      ok = mbar_wait_w(state_full, 0, env);
      if (ok) mbar_arrive(state_full);
    }
    for (int c = 0; ok && c < n_chunks; ++c) {
      if (intra) {
        if (!mbar_wait_w(s_full, c & 1, env)) break;
        tc_fence_after();
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
          }
          tmem_st16(lane_base + L::colS + 64 * h + 16 * b2, w);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full);
        if (c > 0) ok = send(c - 1);
      } else {
        ok = send(c);
      }
    }
    if (ok && intra && n_chunks > 0) send(n_chunks - 1);
  } else if (warp >= 18) {
    // ------------------------------------------------------------- add the four blocks, o = O / D
    const int h = warp - 18;  // output columns 32h .. 32h+31
    uint8_t* slab = smem + L::offOut + h * (32 * 64);
    const float* slot = reinterpret_cast<const float*>(smem + L::offSlot) + lane * kSlotFloats;
    uint32_t empty_remote[kBlocks];
#pragma unroll
    for (int s = 0; s < kBlocks; ++s) empty_remote[s] = map_rank(smem_u32(recv_empty + blk), (uint32_t)s);
    for (int c = 0; c < n_chunks; ++c) {
      if (!mbar_wait_cluster_w(recv_full, c & 1, env)) break;
      float acc[32], D = 0.f;
#pragma unroll
      for (int e = 0; e < 32; ++e) acc[e] = 0.f;
#pragma unroll
      for (int s = 0; s < kBlocks; ++s) {
        const float* row = slot + s * (kSlotBytes / 4);
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 x = *reinterpret_cast<const float4*>(row + 32 * h + e);
          acc[e] += x.x;
          acc[e + 1] += x.y;
          acc[e + 2] += x.z;
          acc[e + 3] += x.w;
        }
        D += row[64];
      }
      // the slots may be refilled
#pragma unroll
      for (int s = 0; s < kBlocks; ++s) mbar_arrive_cluster(empty_remote[s]);
      const float inv = D > 0.f ? 1.f / D : 0.f;
      // this warp's staging box is free once its previous store has read it
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
      uint8_t* orow = slab + lane * 64;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        *reinterpret_cast<uint4*>(orow + ((e ^ ((lane >> 1) & 3)) << 4)) =
            make_uint4(pack_bf16x2(acc[8 * e] * inv, acc[8 * e + 1] * inv),
                       pack_bf16x2(acc[8 * e + 2] * inv, acc[8 * e + 3] * inv),
                       pack_bf16x2(acc[8 * e + 4] * inv, acc[8 * e + 5] * inv),
                       pack_bf16x2(acc[8 * e + 6] * inv, acc[8 * e + 7] * inv));
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_3d(&tm_o, slab, 32 * h, t0 + c * kTile + 32 * blk, bh);
        bulk_commit_group();
      }
    }
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
    auto psi_k = [&](int cc) {
      __nv_bfloat162 u[16];
      uint32_t w[kNPW];
      load_row_sw64(smem + L::offStage + (cc % kRead32Stages) * L::kStage + kVBytes + kQK32Bytes, m, u);
      block_psi<true>(u, blk, w);
      store_psi_k(smem + L::offPsi + (cc & 1) * kPsiBytes, m, w);
    };
    auto psi_q_formed = [&](int cc, uint32_t (&w)[kNPW]) {
      __nv_bfloat162 u[16];
      load_row_sw64(smem + L::offStage + (cc % kRead32Stages) * L::kStage + kVBytes, m, u);
      block_psi<false>(u, blk, w);
    };
    // running state <- scanned prefix (none for super-chunk 0) plus the
    // caller's initial state; after a scan this kernel is its programmatic
    // dependent: wait for the scanned records
    const int d = min(m, kRecRows - 1);  // record row of this lane
    griddep_wait();
    if (quarter < 3) {
      const float* rec =
          (ws && g > 0) ? ws + (((size_t)bh * kBlocks + blk) * G + g) * record_floats + (size_t)d * kNP : nullptr;
      const float* S = S0 ? S0 + (size_t)bh * 1024 * kDV : nullptr;
      const float* z = z0 ? z0 + (size_t)bh * 1024 : nullptr;
      if (half == 0) prefix_half_to_state<0>(rec, S, z, blk, d, lane_base + L::colRun, sb, m, active);
      else prefix_half_to_state<1>(rec, S, z, blk, d, lane_base + L::colRun, sb, m, active);
    }
    bool ok = n_chunks > 0 && mbar_wait_w(kv_full, 0, env);
    if (ok) {
      if (psi_group) {
        psi_k(0);
      } else {
        uint32_t w[kNPW];
        psi_q_formed(0, w);
        store_psi_q_tmem(lane_base + L::colPQ, w);
      }
    }
    tmem_wait_st();
    fence_proxy_async_smem();
    tc_fence_before();
    if (ok) mbar_arrive(state_full);
    for (int c = 0; ok && c + 1 < n_chunks; ++c) {
      const int st1 = (c + 1) % kRead32Stages;
      if (!mbar_wait_w(kv_full + st1, ((c + 1) / kRead32Stages) & 1, env)) break;
      if (psi_group) {
        // psi~(k_{c+1}) into the buffer last read by the advance by chunk
        // c-1, which this group saw complete in the previous iteration
        psi_k(c + 1);
      } else {
        uint32_t wq[kNPW];
        psi_q_formed(c + 1, wq);
        if (!mbar_wait_w(rd_done, c & 1, env)) break;
        tc_fence_after();
        store_psi_q_tmem(lane_base + L::colPQ, wq);
        tmem_wait_st();
      }
      // the state after chunk c is complete; the readout of chunk c, issued
      // before that advance, has read the single bf16 copy
      if (!mbar_wait_w(upd_done, c & 1, env)) break;
      tc_fence_after();
      if (quarter < 3) state_half_to_bf16(lane_base + L::colRun, sb, m, active, half);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(state_full);
    }
    // the last super-chunk ends at token T: its running state, once the
    // advance by its last chunk has landed, is this block's part of the
    // final state
    if (S_out && g == G - 1 && n_chunks > 0 && mbar_wait_w(upd_done, (n_chunks - 1) & 1, env) && quarter < 3) {
      tc_fence_after();
      float* S = S_out + (size_t)bh * 1024 * kDV;
      float* z = z_out + (size_t)bh * 1024;
      if (half == 0) block_state_to_abi<0>(lane_base + L::colRun, S, z, blk, m, m < kRecRows);
      else block_state_to_abi<1>(lane_base + L::colRun, S, z, blk, m, m < kRecRows);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  // no CTA leaves while another may still write into its shared memory
  cluster_sync_all();
}

}  // namespace

cudaError_t launch_chunk_state_p32(const void* k, const void* v, float* ws, const ChunkPlan& pl, const WaitCtl& wc,
                                   cudaStream_t st) {
  if (pl.p != 32 || pl.dv != kDV) return cudaErrorInvalidValue;
  CUtensorMap tk, tv;
  if (!make_tmap_bf16(&tk, k, 32, pl.T, pl.BH, kTile) || !make_tmap_bf16(&tv, v, kDV, pl.T, pl.BH, kTile))
    return cudaErrorInvalidValue;
  cudaError_t e =
      cudaFuncSetAttribute(chunk_state_p32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, State32Smem::kBytes);
  if (e != cudaSuccess) return e;
  if (pl.G < 2) return cudaSuccess;
  dim3 grid(pl.G - 1, pl.BH, kBlocks);
  chunk_state_p32_kernel<<<grid, kStateThreads, State32Smem::kBytes, st>>>(tk, tv, ws, pl.T, pl.Ls, pl.G,
                                                                            (long long)pl.record_floats, wc);
  return cudaGetLastError();
}

cudaError_t launch_chunk_readout_p32(const void* q, const void* k, const void* v, void* o, const float* ws,
                                     const float* S0, const float* z0, float* S_out, float* z_out,
                                     const ChunkPlan& pl, const WaitCtl& wc, cudaStream_t st) {
  if (pl.p != 32 || pl.dv != kDV) return cudaErrorInvalidValue;
  if (!ws && pl.G != 1) return cudaErrorInvalidValue;
  CUtensorMap tq, tk, tv, to;
  if (!make_tmap_bf16(&tq, q, 32, pl.T, pl.BH, kTile) || !make_tmap_bf16(&tk, k, 32, pl.T, pl.BH, kTile) ||
      !make_tmap_bf16(&tv, v, kDV, pl.T, pl.BH, kTile) || !make_tmap_bf16_box(&to, o, kDV, pl.T, pl.BH, 32, 32))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(chunk_readout_p32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Read32Smem::kBytes);
  if (e != cudaSuccess) return e;
  const dim3 grid(pl.G, pl.BH, kBlocks), block(kRead32Threads);
  if (ws)  // after the state build and scan of this call: launched as the scan's programmatic dependent
    return launch_pdl(chunk_readout_p32_kernel, grid, block, (size_t)Read32Smem::kBytes, st, tq, tk, tv, to,
                      (const float*)ws, S0, z0, S_out, z_out, pl.T, pl.Ls, pl.G, (long long)pl.record_floats, wc);
  chunk_readout_p32_kernel<<<grid, block, Read32Smem::kBytes, st>>>(tq, tk, tv, to, ws, S0, z0, S_out, z_out, pl.T,
                                                                    pl.Ls, pl.G, (long long)pl.record_floats, wc);
  return cudaGetLastError();
}

}  // namespace kata
