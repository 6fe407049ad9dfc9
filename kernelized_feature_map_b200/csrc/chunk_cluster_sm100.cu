// chunk_cluster_sm100.cu -- exact O(T) chunked-state KATA forward on
// tcgen05 / TMEM with the packed state split over the CTAs of a cluster:
// the single factor with p = 32, and KATA-Mg with 2 or 4 groups over a head
// of width d = 64 (bf16 inputs, dv = 64).
//
// Coordinate blocks.  Each CTA holds one block of at most 144 packed
// coordinates -- the size of the p = 16 state -- as its transposed state
// S~_b^T in TMEM.
//  * A factor of width 16 is one block: psi~(u), its 136 packed coordinates
//    (ai.info summary, Main Findings, "State size, not just feature width,
//    dominates memory") in runs, with 8 pads.
//  * A factor of width 32 (p = 32: n = 528 packed coordinates, 544 TMEM
//    columns for one CTA, more than the 512 there are) is four blocks.  With
//    u = [a | b], a and b its two halves of 16,
//      (q . k)^2 = (q_a . k_a)^2 + (q_b . k_b)^2 + 2 (q_a . k_a)(q_b . k_b),
//    so the blocks are psi~(a), psi~(b), and a_i b_j for i = 0..7 and for
//    i = 8..15 (j = 0..15; 128 coordinates and 16 pads each, key side x 2).
//  * KATA-Mg concatenates the groups' features (KATA repository README,
//    "concat-SPD"; ai.info, Main Findings: state d(d/g+1)/2 * dv packed), so
//    g groups of width 16 are g blocks and g groups of width 32 are 4g
//    blocks.
// Per 128-token chunk c every CTA computes
//   [O | D]_b = psi~_b(Q_c) S~_b            (readout against the state entering c)
//   S~_b^T  += [V_c | 1]^T psi~_b(K_c)      (advance)
// and the first CTA of each group adds that group's intra-chunk part
// W_j [V_c | 1] with W_j = (Q_c^j K_c^j^T)^2 (causal): the weight of a pair
// is the sum over the groups of their squared scores, sum_j (q^j . k^j)^2, so
// the intra-chunk part splits by group (for one factor of width 32 it is a
// single block, in CTA 0).  Numerator and denominator are sums over the
// CTAs: each CTA owns 128 / cluster-size rows of every chunk; the warps that
// read [O | D]_b out of TMEM send each row to its owner through distributed
// shared memory, and two warps of the owner add the partial rows, form
// o = O / D and store them.
//
// Launches per call (G super-chunks per (b,h), as on the p = 16 path):
//  1. chunk_state_cluster_kernel (G > 1) per super-chunk g < G-1 and block:
//                                A_{g,b} = sum over its chunks;
//  2. state_scan                 (G > 1, scan.cu) exclusive prefix over g of
//                                the B H x (blocks) sequences;
//  3. chunk_readout_cluster_kernel, one cluster per (b,h, super-chunk),
//                                starting from the scanned prefix plus the
//                                caller's initial state; the cluster of the
//                                last super-chunk writes the final state.
// q, k, v and o are read and written through 4-D tensor maps in either the
// [B,H,T,*] or the [B,T,H,*] layout.
#include <cuda.h>

#include "chunk_common.cuh"
#include "kata_internal.h"
#include "kata_trace.cuh"

KATA_TRACE_DECLARE(cluster)

namespace kata {

bool make_tmap_bf16_4d(CUtensorMap* map, const void* base, int inner, int T, int H, int B, bool bthd, int box_inner,
                       int rows);

namespace {

using namespace sm100;
using namespace chunk;

// ---------------------------------------------------------------------------
// configuration: P = width of a factor (16 or 32), NG = factors per head
// ---------------------------------------------------------------------------
template <int P, int NG>
struct CCfg {
  static_assert((P == 16 && NG == 4) || (P == 32 && (NG == 1 || NG == 2)), "supported cluster configurations");
  static constexpr int kBPG = P == 32 ? 4 : 1;         // blocks per factor
  static constexpr int kCS = NG * kBPG;                 // CTAs per cluster
  static constexpr int kRows = kTile / kCS;             // output rows each CTA owns (32 or 16)
  static constexpr int kD = NG * P;                     // q/k row width
  static constexpr int kStateRows = NG * P * P;         // ABI state rows per (b,h)
  static constexpr int kQKBytes = kTile * P * 2;        // one factor's columns of a Q or K tile
  static constexpr Swizzle kQKSw = P == 16 ? kSw32 : kSw64;
  static constexpr uint32_t kQKSbo = 8 * P * 2;         // 8-row group stride of that tile
  static constexpr int kStages = P == 16 ? 3 : 2;       // [V | Q | K] ring of the readout
  static constexpr int kStateStages = P == 16 ? 6 : 5;  // [V | K] ring of the state kernel
};

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
// Asynchronous stores into another CTA's shared memory that report their
// bytes to an mbarrier of that CTA on completion (the issuing thread does
// not wait; the receiver's barrier counts the bytes).
__device__ __forceinline__ void st_async_v4(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w,
                                            uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(a),
               "r"(x), "r"(y), "r"(z), "r"(w), "r"(bar)
               : "memory");
}
__device__ __forceinline__ void st_async_b32(uint32_t a, uint32_t x, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(a), "r"(x), "r"(bar)
               : "memory");
}
// Arrive on an mbarrier of a CTA of the cluster without ordering this
// thread's earlier memory accesses (a release arrival waits for them at
// cluster scope, ~1000 cycles per arrival measured).
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t bar_cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait, with acquire at cluster scope, on a local mbarrier (shared
// address `bar`, may differ between lanes) that other CTAs of the cluster
// arrive on; same contract as mbar_wait, warp-uniform result.
__device__ __forceinline__ bool mbar_wait_cluster_w(uint32_t bar, uint32_t parity, const WaitEnv& env) {
  bool ok = mbar_try_wait_cluster(bar, parity);
  if (!ok && env.limit != 0) {
    const long long t0 = clock64();
    while (!(ok = mbar_try_wait_cluster(bar, parity))) {
      if (*env.abort_flag) break;
      if (clock64() - t0 >= env.limit) break;
    }
  }
  if (!ok && !*env.abort_flag) {
    *env.abort_flag = 1;
    report_status(env.status, kErrTimeout);
  }
  return __all_sync(0xffffffffu, ok);
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// block psi~ formation
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

// Blocks 2 and 3 of a width-32 factor: word il*8 + jp = (a_i b_{2jp},
// a_i b_{2jp+1}) for the eight a_i of the block (x 2 on the key side,
// exact), then 8 zero words (pads).
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

// The 72 words of block bb (of its factor) of one token, from the factor's
// row in the stage tile.
template <int P, bool key>
__device__ __forceinline__ void block_psi_row(const uint8_t* tile, int r, int bb, uint32_t (&out)[kNPW]) {
  if constexpr (P == 16) {
    __nv_bfloat162 u[8];
    load_row_sw32(tile, r, u);
    packed_psi<key>(u, out);
  } else {
    __nv_bfloat162 u[16];
    load_row_sw64(tile, r, u);
    if (bb < 2) {
      __nv_bfloat162 h[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) h[e] = bb == 0 ? u[e] : u[8 + e];
      packed_psi<key>(h, out);
    } else {
      __nv_bfloat162 a4[4], b[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) a4[e] = bb == 2 ? u[e] : u[4 + e];
#pragma unroll
      for (int e = 0; e < 8; ++e) b[e] = u[8 + e];
      cross_psi<key>(a4, b, out);
    }
  }
}

// ---------------------------------------------------------------------------
// block coordinates <-> the ABI state layout ([NG * P * P, dv] and
// [NG * P * P] per (b,h); row grp * P^2 + i * P + j of factor grp holds the
// products of its coordinates i and j)
// ---------------------------------------------------------------------------
// Packed coordinate w of block bb of factor grp -> ABI rows r1 and r2 (r2 =
// -1 on the diagonal; r1 = -1 for a pad).  The packed value is the sum of
// both rows.
template <int P>
__device__ __forceinline__ void block_coord(int grp, int bb, int w, int& r1, int& r2) {
  const int base = grp * P * P;
  if (P == 16 || bb < 2) {
    const int i = packed_i(w), j = packed_j(w), o = P == 16 ? 0 : 16 * bb;
    r1 = i < 0 ? -1 : base + (i + o) * P + (j + o);
    r2 = (i < 0 || i == j) ? -1 : base + (j + o) * P + (i + o);
  } else {
    const int il = w >> 4, j = w & 15, i = 8 * (bb - 2) + il;
    r1 = w < 128 ? base + i * 32 + 16 + j : -1;
    r2 = w < 128 ? base + (16 + j) * 32 + i : -1;
  }
}

// Initial value of word w of row d (<= 64) of a block: the scanned record's
// entry (when `rec`) plus the caller's initial state (when S).
template <int P>
__device__ __forceinline__ float prefix_entry(const float* rec, const float* S, const float* z, int grp, int bb,
                                              int d, int w) {
  float v = rec ? rec[w] : 0.f;
  if (S) {
    int r1, r2;
    block_coord<P>(grp, bb, w, r1, r2);
    if (r1 >= 0) {
      if (d < kDV) v += S[r1 * kDV + d] + (r2 >= 0 ? S[r2 * kDV + d] : 0.f);
      else v += z[r1] + (r2 >= 0 ? z[r2] : 0.f);
    }
  }
  return v;
}

// Half `half` of the prefix row d into the TMEM lane and the bf16 copy row n.
// Warp-collective.
template <int P, int half>
__device__ __forceinline__ void prefix_half_to_state(const float* rec, const float* S, const float* z, int grp,
                                                     int bb, int d, uint32_t taddr, uint8_t* sb, int n, bool active) {
  uint32_t r[72];
#pragma unroll
  for (int e = 0; e < 72; ++e)
    r[e] = __float_as_uint(active ? prefix_entry<P>(rec, S, z, grp, bb, d, 72 * half + e) : 0.f);
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

// Half `half` of TMEM lane d (<= 64) of a block's final state -> the ABI
// layout (an off-diagonal packed entry is halved into its two rows, exactly).
// Warp-collective.
template <int P, int half>
__device__ __forceinline__ void block_state_to_abi(uint32_t taddr, float* S, float* z, int grp, int bb, int d,
                                                   bool active) {
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
    block_coord<P>(grp, bb, 72 * half + e, r1, r2);
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

// rows [t, t + box) of head bh of a 4-D tensor map ({inner, T, H, B} for the
// [B,H,T,*] layout, {inner, H, T, B} for [B,T,H,*]), from column x
__device__ __forceinline__ void load_tile(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int t, int bh,
                                          int H, bool bthd) {
  const int b = bh / H, hd = bh - b * H;
  if (bthd) tma_load_4d(dst, map, bar, x, hd, t, b);
  else tma_load_4d(dst, map, bar, x, t, hd, b);
}
__device__ __forceinline__ void store_tile(const CUtensorMap* map, const void* src, int x, int t, int bh, int H,
                                           bool bthd) {
  const int b = bh / H, hd = bh - b * H;
  if (bthd) tma_store_4d(map, src, x, hd, t, b);
  else tma_store_4d(map, src, x, t, hd, b);
}

// ===========================================================================
// 1. per-super-chunk block state sums
// ===========================================================================
constexpr int kStateThreads = 320;  // warp 0 TMA, warp 1 MMA, warps 2-9 psi~(k), warps 2-5 record

template <int P, int NG>
struct StateCSmem {
  using C = CCfg<P, NG>;
  static constexpr int kStage = kVBytes + C::kQKBytes;  // [V | K]
  static constexpr int offStage = 0;
  static constexpr int offOnes = offStage + C::kStateStages * kStage;  // 1024-aligned
  static constexpr int offPsi = offOnes + kOnesBytes;                    // 2 buffers
  static constexpr int offBar = offPsi + 2 * kPsiBytes;
  static constexpr int kBars = 2 * C::kStateStages + 4 + 1;
  static constexpr int offMisc = offBar + kBars * 8;
  static constexpr int kBytes = offMisc + 16 + 1024;
  static_assert(kBytes <= 232448, "shared memory");
};

// grid (G - 1, B*H, blocks): super-chunk g, sequence bh, block blockIdx.z;
// record ((bh * blocks + block) * G + g) of the workspace.
template <int P, int NG>
__global__ void __launch_bounds__(kStateThreads, 1)
    chunk_state_cluster_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                               float* __restrict__ ws, int T, int H, int bthd, int Ls, int G, long long record_floats,
                               WaitCtl wc) {
  using C = CCfg<P, NG>;
  using L = StateCSmem<P, NG>;
  constexpr int kSt = C::kStateStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::offBar);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + kSt;
  uint64_t* psi_full = kv_empty + kSt;  // [2]
  uint64_t* psi_empty = psi_full + 2;   // [2]
  uint64_t* acc_done = psi_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::offMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::offMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x, bh = blockIdx.y, blk = blockIdx.z;
  const int grp = blk / C::kBPG, bb = blk % C::kBPG;
  const int t0 = g * Ls;
  const int n_chunks = (min(T, t0 + Ls) - t0 + kTile - 1) / kTile;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSt; ++s) {
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
        const int st = c % kSt;
        if (!mbar_wait(kv_empty + st, ((c / kSt) & 1) ^ 1, env)) break;
        uint8_t* base = smem + L::offStage + st * L::kStage;
        mbar_arrive_expect_tx(kv_full + st, L::kStage);
        load_tile(base, &tm_v, kv_full + st, 0, t0 + c * kTile, bh, H, bthd);
        load_tile(base + kVBytes, &tm_k, kv_full + st, grp * P, t0 + c * kTile, bh, H, bthd);
        ++issued;
      }
      for (int c = issued - kSt < 0 ? 0 : issued - kSt; c < issued; ++c)
        mbar_wait_drain(kv_full + c % kSt, (c / kSt) & 1);
    }
  } else if (warp == 1) {
    constexpr uint32_t id_u = idesc_bf16(128, kNP, true, true);
    const uint32_t sStage = smem_u32(smem + L::offStage), sOnes = smem_u32(smem + L::offOnes);
    const uint64_t dpsi = smem_desc(smem_u32(smem + L::offPsi), kPsiAtom, 256, kSw32);
    for (int c = 0; c < n_chunks; ++c) {
      const int st = c % kSt, pb = c & 1;
      if (!mbar_wait_w(kv_full + st, (c / kSt) & 1, env)) break;
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
      const int st = c % kSt, pb = c & 1;
      if (!mbar_wait_w(kv_full + st, (c / kSt) & 1, env)) {
        ok = false;
        break;
      }
      if (c >= 2 && !mbar_wait_w(psi_empty + pb, ((c >> 1) - 1) & 1, env)) {
        ok = false;
        break;
      }
      uint32_t w[kNPW];
      block_psi_row<P, true>(smem + L::offStage + st * L::kStage + kVBytes, tid, bb, w);
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
      float* row = ws + (((size_t)bh * C::kCS + blk) * G + g) * record_floats + (size_t)min(d, kRecRows - 1) * kNP;
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
// 3. readout, one cluster per (b,h, super-chunk), one CTA per block
// ===========================================================================
// Warp roles (640 threads):
//   warp 0       TMA: [V | Q_j | K_j] tiles of each chunk (the factor's
//                columns of q and k) into a ring
//   warp 1       TMEM allocator; MMA issue (the whole warp, one elected lane)
//   warps 2-5,   first CTA of a factor: weights W_j = (Q_j K_j^T)^2 (causal)
//   14-17        into TMEM; every CTA: the rows of [O | D]_b of lane quarter
//                q (columns split between the two warps of a quarter) sent
//                to the CTAs that own them
//   warps 6-9    psi~_b(k_{c+1}) into shared memory (two buffers); bf16 copy
//                of packed coordinates 0..71 of S~_b after chunk c
//   warps 10-13  prefix in; psi~_b(q_{c+1}) into TMEM once the readout of
//                chunk c has read psi~_b(q_c); bf16 copy of coordinates 72..143
//   warps 18-19  the partial rows of this CTA's own rows summed over the
//                cluster, o = O / D written from registers (columns 0..31
//                and 32..63)
// MMA order per chunk: [first CTA of a factor: scores], readout, advance,
// [first CTA of a factor: intra-chunk weights].  The bf16 copy of S~_b has
// one buffer: it is refreshed once the advance by chunk c has landed, and
// the readout of chunk c, issued before that advance, has then completed.
// Cluster exchange per chunk: slot[src][row][68 floats] in the owning CTA
// (O columns 0..63, D at 64), written with asynchronous remote stores that
// count their bytes on the owner's recv_full, which completes when all
// partial rows of the chunk are in (one arrival per phase, with the byte
// count, from the owner); recv_empty[t] in the sending CTA (one arrival from
// each of CTA t's two adding warps) completes when CTA t has read them, so
// its slot may be reused.
constexpr int kReadCThreads = 640;
constexpr int kSlotFloats = 68;  // per row: O (64), D, pad

template <int P, int NG>
struct ReadCSmem {
  using C = CCfg<P, NG>;
  static constexpr int kSlotBytes = C::kRows * kSlotFloats * 4;        // one source's rows
  static constexpr int kStage = kVBytes + 2 * C::kQKBytes;               // [V | Q | K]
  static constexpr int offStage = 0;
  static constexpr int offOnes = offStage + C::kStages * kStage;         // 1024-aligned
  static constexpr int offPsi = offOnes + kOnesBytes;                      // 2 buffers
  static constexpr int offSB = offPsi + 2 * kPsiBytes;                     // 1 buffer
  static constexpr int offSlot = offSB + kSBBytes;                         // [sources]
  static constexpr int offBar = offSlot + C::kCS * kSlotBytes;
  static constexpr int kBars = 2 * C::kStages + 9 + C::kCS;
  static constexpr int offMisc = offBar + kBars * 8;
  static constexpr int kBytes = offMisc + 16 + 1024;
  static constexpr uint32_t colRun = 0;                                    // S~_b^T, 144
  static constexpr uint32_t colO(int b) { return 144u + 80u * (uint32_t)b; }  // [O | D] x 2
  static constexpr uint32_t colPQ = 304;                                   // psi~_b(Q_c), 72
  static constexpr uint32_t colS = 384;                                    // scores / weights, 128
  static_assert(offSlot % 16 == 0 && offSB % 1024 == 0 && kBytes <= 232448,
                "shared-memory layout");
};

template <int P, int NG>
__global__ void __launch_bounds__(kReadCThreads, 1)
    chunk_readout_cluster_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                                 const __grid_constant__ CUtensorMap tm_v, void* __restrict__ o,
                                 const float* __restrict__ ws, const float* __restrict__ S0,
                                 const float* __restrict__ z0, float* __restrict__ S_out, float* __restrict__ z_out,
                                 int T, int H, int bthd, int Ls, int G, long long record_floats, WaitCtl wc) {
  using C = CCfg<P, NG>;
  using L = ReadCSmem<P, NG>;
  constexpr int kSt = C::kStages;
  constexpr int kRows = C::kRows;
  // bytes an owner receives per chunk: from every CTA, its rows' O (64
  // floats, two 32-column halves) and D
  constexpr uint32_t kRecvBytes = (uint32_t)C::kCS * kRows * 65 * 4;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::offBar);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + kSt;
  uint64_t* s_full = kv_empty + kSt;  // scores in TMEM (first CTA of a factor)
  uint64_t* p_full = s_full + 1;      // weights written (256)
  uint64_t* state_full = p_full + 1;  // chunk c's operands ready, its [O | D] buffer free (512)
  uint64_t* rd_done = state_full + 1; // readout of the chunk done
  uint64_t* upd_done = rd_done + 1;   // state advanced by the chunk
  uint64_t* o_full = upd_done + 1;    // [2] [O | D] complete
  uint64_t* mma_done = o_full + 2;
  uint64_t* recv_full = mma_done + 1; // all partial rows of the chunk received (kRecvBytes)
  uint64_t* recv_empty = recv_full + 1;  // [cluster size] CTA t has read this CTA's rows (its 2 adding warps)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::offMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::offMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int blk = (int)cluster_rank();
  const int grp = blk / C::kBPG, bb = blk % C::kBPG;
  const bool lead = bb == 0;  // computes its factor's intra-chunk part
  KATA_TRACE_BEGIN_IDX(cluster, (blockIdx.y * gridDim.x + blockIdx.x) * gridDim.z + blk);
  const int g = blockIdx.x, bh = blockIdx.y;
  const int t0 = g * Ls;
  const int t1 = min(T, t0 + Ls);
  const int n_chunks = (t1 - t0 + kTile - 1) / kTile;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSt; ++s) {
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
    mbar_init(recv_full, 1);
    for (int b = 0; b < C::kCS; ++b) mbar_init(recv_empty + b, 2);
    *abort_flag = 0;
    fence_barrier_init();
  }
  fill_ones(smem + L::offOnes, threadIdx.x, kReadCThreads);
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
        const int st = c % kSt;
        if (!mbar_wait(kv_empty + st, ((c / kSt) & 1) ^ 1, env)) break;
        uint8_t* base = smem + L::offStage + st * L::kStage;
        mbar_arrive_expect_tx(kv_full + st, L::kStage);
        const int row = t0 + c * kTile;
        load_tile(base, &tm_v, kv_full + st, 0, row, bh, H, bthd);
        load_tile(base + kVBytes, &tm_q, kv_full + st, grp * P, row, bh, H, bthd);
        load_tile(base + kVBytes + C::kQKBytes, &tm_k, kv_full + st, grp * P, row, bh, H, bthd);
        ++issued;
      }
      for (int c = issued - kSt < 0 ? 0 : issued - kSt; c < issued; ++c)
        mbar_wait_drain(kv_full + c % kSt, (c / kSt) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA
    constexpr uint32_t id_qk = idesc_bf16(128, 128, false, false);
    constexpr uint32_t id_rd = idesc_bf16(128, 80, false, false);  // A = psi~(Q) (TMEM), B = S~ K-major
    constexpr uint32_t id_wv = idesc_bf16(128, 80, false, true);   // A = W (TMEM), B = [V | 1]
    constexpr uint32_t id_u = idesc_bf16(128, kNP, true, true);    // A = [V | 1]^T, B = psi~(K)
    const uint32_t sStage = smem_u32(smem + L::offStage), sOnes = smem_u32(smem + L::offOnes);
    const uint32_t sPsi = smem_u32(smem + L::offPsi), sSB = smem_u32(smem + L::offSB);
    // the factor's Q and K tiles: K-major; each further 16 columns start 32
    // bytes further into the swizzled rows
    const uint64_t dq0 = smem_desc(sStage + kVBytes, 16, C::kQKSbo, C::kQKSw);
    const uint64_t dk0 = smem_desc(sStage + kVBytes + C::kQKBytes, 16, C::kQKSbo, C::kQKSw);
    const uint64_t dpsi = smem_desc(sPsi, kPsiAtom, 256, kSw32);
    const uint64_t dsb = smem_desc(sSB, 16, 256, kSw32);
    for (int c = 0; c < n_chunks; ++c) {
      const int st = c % kSt, ob = c & 1;
      const uint32_t sV = sStage + st * L::kStage;
      KATA_TRACE(cluster, c, 0);
      if (!mbar_wait_w(state_full, c & 1, env)) break;
      KATA_TRACE(cluster, c, 1);
      tc_fence_after();
      if (lead) {
#pragma unroll
        for (int ks = 0; ks < P / 16; ++ks)
          mma_ss_w(tmem + L::colS, desc_add(dq0, st * L::kStage + ks * 32), desc_add(dk0, st * L::kStage + ks * 32),
                   id_qk, ks);
        mma_commit_w(s_full);
      }
      const uint32_t dO = tmem + L::colO(ob);
#pragma unroll
      for (int ks = 0; ks < kNP / 16; ++ks)
        mma_ts_w(dO, tmem + L::colPQ + ks * 8, desc_add(dsb, ks * kSBAtom), id_rd, ks > 0);
      mma_commit_w(rd_done);
      if (!lead) mma_commit_w(o_full + ob);
      KATA_TRACE(cluster, c, 2);
      const uint64_t dvo = desc_vones(sV, sOnes);
#pragma unroll
      for (int ks = 0; ks < kTile / 16; ++ks)
        mma_ss_w(tmem + L::colRun, desc_add(dvo, ks * 2048), desc_add(dpsi, (c & 1) * kPsiBytes + ks * 512), id_u, 1);
      mma_commit_w(upd_done);
      KATA_TRACE(cluster, c, 3);
      if (lead) {
        if (!mbar_wait_w(p_full, c & 1, env)) break;
        KATA_TRACE(cluster, c, 4);
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < kTile / 16; ++ks)
          mma_ts_w(dO, tmem + L::colS + (ks >> 2) * 64 + (ks & 3) * 8, desc_add(dvo, ks * 2048), id_wv, 1);
        mma_commit_w(o_full + ob);
      }
      mma_commit_w(kv_empty + st);
      KATA_TRACE(cluster, c, 5);
    }
    mma_commit_w(mma_done);
    mbar_wait_drain(mma_done, 0);
  } else if (warp < 6 || (warp >= 14 && warp < 18)) {
    // ------------------------------------------------------------- weights + partial rows out
    const int quarter = warp % 4;
    const int h = warp >= 14 ? 1 : 0;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    // token row 32 quarter + lane belongs to CTA `owner`, its row orow there
    const int m = quarter * 32 + lane;
    const int owner = m / kRows, orow = m % kRows;
    const uint32_t slot_remote =
        map_rank(smem_u32(smem + L::offSlot + blk * L::kSlotBytes + orow * kSlotFloats * 4), (uint32_t)owner);
    const uint32_t full_remote = map_rank(smem_u32(recv_full), (uint32_t)owner);
    const uint32_t empty_local = smem_u32(recv_empty + owner);
    auto send = [&](int co) -> bool {
      const int ob = co & 1;
      if (!mbar_wait_w(o_full + ob, (co >> 1) & 1, env)) return false;
      if (m == 0 && h == 0) KATA_TRACE(cluster, co, 10);
      tc_fence_after();
      uint32_t r[32], db;
      tmem_ld32(lane_base + L::colO(ob) + 32 * h, r);
      tmem_ld1(lane_base + L::colO(ob) + 64, db);
      tmem_wait_ld();
      tc_fence_before();
      // the readout of chunk co+2 reuses this [O | D] buffer.  An arrival on
      // state_full for chunk co+2 must come after its phase for chunk co+1
      // has completed, or it would count towards that phase: in the first
      // CTA of a factor the weights of chunk co+1, which wait for its
      // scores, come first; the other CTAs wait for the phase here
      if (co + 2 < n_chunks) {
        if (!lead && !mbar_wait_w(state_full, (co + 1) & 1, env)) return false;
        mbar_arrive(state_full);
      }
      // the owner has read what this lane sent for chunk co-1
      if (co > 0 && !mbar_wait_cluster_w(empty_local, (co - 1) & 1, env)) return false;
      if (m == 0 && h == 0) KATA_TRACE(cluster, co, 11);
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        st_async_v4(slot_remote + (32 * h + e) * 4, r[e], r[e + 1], r[e + 2], r[e + 3], full_remote);
      if (h == 0) st_async_b32(slot_remote + 64 * 4, db, full_remote);
      if (m == 0 && h == 0) KATA_TRACE(cluster, co, 26);
      if (m == 0 && h == 0) KATA_TRACE(cluster, co, 12);
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
      if (lead) {
        if (!mbar_wait_w(s_full, c & 1, env)) break;
        if (m == 0 && h == 0) KATA_TRACE(cluster, c, 8);
        tc_fence_after();
#pragma unroll
        for (int b2 = 0; b2 < 2; ++b2) {
          const int bb2 = 2 * h + b2;
          uint32_t w[16];
          if (bb2 > quarter) {
#pragma unroll
            for (int x = 0; x < 16; ++x) w[x] = 0u;
          } else {
            uint32_t r[32];
            tmem_ld32(lane_base + L::colS + 32 * bb2, r);
            tmem_wait_ld();
            if (bb2 < quarter) {
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
        if (m == 0 && h == 0) KATA_TRACE(cluster, c, 9);
        if (c > 0) ok = send(c - 1);
      } else {
        ok = send(c);
      }
    }
    if (ok && lead && n_chunks > 0) send(n_chunks - 1);
  } else if (warp >= 18) {
    // ------------------------------------------------------------- sum over the cluster, o = O / D
    const int h = warp - 18;  // output columns 32h .. 32h+31
    const bool act = lane < kRows;
    const int lr = act ? lane : 0;  // this lane's own row
    // row t of this head of o ([B,H,T,dv] or [B,T,H,dv])
    const int ob = bh / H, oh = bh - ob * H;
    auto out_row = [&](int t) {
      const size_t r = bthd ? ((size_t)ob * T + t) * H + oh : ((size_t)ob * H + oh) * T + t;
      return reinterpret_cast<__nv_bfloat16*>(o) + r * kDV;
    };
    const float* slot = reinterpret_cast<const float*>(smem + L::offSlot) + lr * kSlotFloats;
    const uint32_t full_local = smem_u32(recv_full);
    // the bytes of chunk 0 are expected (one arrival per phase, by one lane)
    if (h == 0 && lane == 0 && n_chunks > 0) mbar_arrive_expect_tx(recv_full, kRecvBytes);
    for (int c = 0; c < n_chunks; ++c) {
      if (!mbar_wait_cluster_w(full_local, c & 1, env)) break;
      if (lane == 0 && h == 0) KATA_TRACE(cluster, c, 14);
      float acc[32], D = 0.f;
#pragma unroll
      for (int e = 0; e < 32; ++e) acc[e] = 0.f;
#pragma unroll
      for (int s = 0; s < C::kCS; ++s) {
        const float* row = slot + s * (L::kSlotBytes / 4);
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
      if (lane == 0 && h == 0) KATA_TRACE(cluster, c, 23);
      // the bytes of chunk c+1 are expected before any source may send
      // them (they wait for this warp's arrival below)
      if (h == 0 && lane == 0 && c + 1 < n_chunks) mbar_arrive_expect_tx(recv_full, kRecvBytes);
      // every source's slot may be refilled: one arrival per warp and
      // source once all its lanes have read (the values are in registers,
      // already added, so no later store into the slot can change them)
      __syncwarp();
      if (lane == 0) {
#pragma unroll
        for (int s = 0; s < C::kCS; ++s)
          mbar_arrive_cluster_relaxed(map_rank(smem_u32(recv_empty + blk), (uint32_t)s));
      }
      if (lane == 0 && h == 0) KATA_TRACE(cluster, c, 24);
      const float inv = D > 0.f ? 1.f / D : 0.f;
      // o = O / D straight from registers: this lane's 32 values of its row
      // (64 bytes; the other warp writes the other half of the row).  A TMA
      // store from shared memory measured ~2300 cycles per chunk here, its
      // proxy fence waiting behind the cluster's incoming traffic.
      const int t = t0 + c * kTile + kRows * blk + lane;
      if (act && t < T) {
        uint4* dst = reinterpret_cast<uint4*>(out_row(t) + 32 * h);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          dst[e] = make_uint4(pack_bf16x2(acc[8 * e] * inv, acc[8 * e + 1] * inv),
                              pack_bf16x2(acc[8 * e + 2] * inv, acc[8 * e + 3] * inv),
                              pack_bf16x2(acc[8 * e + 4] * inv, acc[8 * e + 5] * inv),
                              pack_bf16x2(acc[8 * e + 6] * inv, acc[8 * e + 7] * inv));
      }
      if (lane == 0 && h == 0) KATA_TRACE(cluster, c, 15);
    }
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
      uint32_t w[kNPW];
      block_psi_row<P, true>(smem + L::offStage + (cc % kSt) * L::kStage + kVBytes + C::kQKBytes, m, bb, w);
      store_psi_k(smem + L::offPsi + (cc & 1) * kPsiBytes, m, w);
    };
    auto psi_q_formed = [&](int cc, uint32_t (&w)[kNPW]) {
      block_psi_row<P, false>(smem + L::offStage + (cc % kSt) * L::kStage + kVBytes, m, bb, w);
    };
    // running state <- scanned prefix (none for super-chunk 0) plus the
    // caller's initial state; after a scan this kernel is its programmatic
    // dependent: wait for the scanned records
    const int d = min(m, kRecRows - 1);  // record row of this lane
    griddep_wait();
    if (quarter < 3) {
      const float* rec =
          (ws && g > 0) ? ws + (((size_t)bh * C::kCS + blk) * G + g) * record_floats + (size_t)d * kNP : nullptr;
      const float* S = S0 ? S0 + (size_t)bh * C::kStateRows * kDV : nullptr;
      const float* z = z0 ? z0 + (size_t)bh * C::kStateRows : nullptr;
      if (half == 0) prefix_half_to_state<P, 0>(rec, S, z, grp, bb, d, lane_base + L::colRun, sb, m, active);
      else prefix_half_to_state<P, 1>(rec, S, z, grp, bb, d, lane_base + L::colRun, sb, m, active);
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
      const int st1 = (c + 1) % kSt;
      if (!mbar_wait_w(kv_full + st1, ((c + 1) / kSt) & 1, env)) break;
      if (m == 0) KATA_TRACE(cluster, c, psi_group ? 16 : 21);
      if (psi_group) {
        // psi~(k_{c+1}) into the buffer last read by the advance by chunk
        // c-1, which this group saw complete in the previous iteration
        psi_k(c + 1);
      } else {
        uint32_t wq[kNPW];
        psi_q_formed(c + 1, wq);
        if (!mbar_wait_w(rd_done, c & 1, env)) break;
        if (m == 0) KATA_TRACE(cluster, c, 19);
        tc_fence_after();
        store_psi_q_tmem(lane_base + L::colPQ, wq);
        tmem_wait_st();
      }
      // the state after chunk c is complete; the readout of chunk c, issued
      // before that advance, has read the single bf16 copy
      if (!mbar_wait_w(upd_done, c & 1, env)) break;
      if (m == 0) KATA_TRACE(cluster, c, psi_group ? 17 : 22);
      tc_fence_after();
      if (quarter < 3) state_half_to_bf16(lane_base + L::colRun, sb, m, active, half);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(state_full);
      if (m == 0) KATA_TRACE(cluster, c, psi_group ? 18 : 20);
    }
    // the last super-chunk ends at token T: its running state, once the
    // advance by its last chunk has landed, is this block's part of the
    // final state
    if (S_out && g == G - 1 && n_chunks > 0 && mbar_wait_w(upd_done, (n_chunks - 1) & 1, env) && quarter < 3) {
      tc_fence_after();
      float* S = S_out + (size_t)bh * C::kStateRows * kDV;
      float* z = z_out + (size_t)bh * C::kStateRows;
      if (half == 0) block_state_to_abi<P, 0>(lane_base + L::colRun, S, z, grp, bb, m, m < kRecRows);
      else block_state_to_abi<P, 1>(lane_base + L::colRun, S, z, grp, bb, m, m < kRecRows);
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

template <int P, int NG>
cudaError_t launch_state_t(const void* k, const void* v, float* ws, const ChunkPlan& pl, int H, bool bthd,
                           const WaitCtl& wc, cudaStream_t st) {
  using C = CCfg<P, NG>;
  using L = StateCSmem<P, NG>;
  const int B = pl.BH / H;
  CUtensorMap tk, tv;
  if (!make_tmap_bf16_4d(&tk, k, C::kD, pl.T, H, B, bthd, P, kTile) ||
      !make_tmap_bf16_4d(&tv, v, kDV, pl.T, H, B, bthd, kDV, kTile))
    return cudaErrorInvalidValue;
  cudaError_t e =
      cudaFuncSetAttribute(chunk_state_cluster_kernel<P, NG>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
  if (e != cudaSuccess) return e;
  if (pl.G < 2) return cudaSuccess;
  dim3 grid(pl.G - 1, pl.BH, C::kCS);
  chunk_state_cluster_kernel<P, NG><<<grid, kStateThreads, L::kBytes, st>>>(tk, tv, ws, pl.T, H, bthd ? 1 : 0, pl.Ls,
                                                                            pl.G, (long long)pl.record_floats, wc);
  return cudaGetLastError();
}

template <int P, int NG>
cudaError_t launch_readout_t(const void* q, const void* k, const void* v, void* o, const float* ws, const float* S0,
                             const float* z0, float* S_out, float* z_out, const ChunkPlan& pl, int H, bool bthd,
                             const WaitCtl& wc, cudaStream_t st) {
  using C = CCfg<P, NG>;
  using L = ReadCSmem<P, NG>;
  if (!ws && pl.G != 1) return cudaErrorInvalidValue;
  const int B = pl.BH / H;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_bf16_4d(&tq, q, C::kD, pl.T, H, B, bthd, P, kTile) ||
      !make_tmap_bf16_4d(&tk, k, C::kD, pl.T, H, B, bthd, P, kTile) ||
      !make_tmap_bf16_4d(&tv, v, kDV, pl.T, H, B, bthd, kDV, kTile))
    return cudaErrorInvalidValue;
  auto kern = chunk_readout_cluster_kernel<P, NG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.G, pl.BH, C::kCS);
  cfg.blockDim = dim3(kReadCThreads);
  cfg.dynamicSmemBytes = L::kBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = C::kCS;
  // after the state build and scan of this call: the scan's programmatic dependent
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = ws ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, o, ws, S0, z0, S_out, z_out, pl.T, H, bthd ? 1 : 0, pl.Ls, pl.G,
                            (long long)pl.record_floats, wc);
}

}  // namespace

bool cluster_chunked_supports(int p, int groups, int dv) {
  return dv == kDV && ((p == 32 && (groups == 1 || groups == 2)) || (p == 16 && groups == 4));
}

cudaError_t launch_chunk_state_cluster(const void* k, const void* v, float* ws, const ChunkPlan& pl, int H, int groups,
                                       bool bthd, const WaitCtl& wc, cudaStream_t st) {
  if (pl.p == 32 && groups == 1) return launch_state_t<32, 1>(k, v, ws, pl, H, bthd, wc, st);
  if (pl.p == 32 && groups == 2) return launch_state_t<32, 2>(k, v, ws, pl, H, bthd, wc, st);
  if (pl.p == 16 && groups == 4) return launch_state_t<16, 4>(k, v, ws, pl, H, bthd, wc, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_chunk_readout_cluster(const void* q, const void* k, const void* v, void* o, const float* ws,
                                         const float* S0, const float* z0, float* S_out, float* z_out,
                                         const ChunkPlan& pl, int H, int groups, bool bthd, const WaitCtl& wc,
                                         cudaStream_t st) {
  if (pl.p == 32 && groups == 1) return launch_readout_t<32, 1>(q, k, v, o, ws, S0, z0, S_out, z_out, pl, H, bthd, wc, st);
  if (pl.p == 32 && groups == 2) return launch_readout_t<32, 2>(q, k, v, o, ws, S0, z0, S_out, z_out, pl, H, bthd, wc, st);
  if (pl.p == 16 && groups == 4) return launch_readout_t<16, 4>(q, k, v, o, ws, S0, z0, S_out, z_out, pl, H, bthd, wc, st);
  return cudaErrorInvalidValue;
}

}  // namespace kata
