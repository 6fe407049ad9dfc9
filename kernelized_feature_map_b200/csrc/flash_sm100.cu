// flash_sm100.cu -- quadratic (flash-style) KATA forward on tcgen05 / TMEM.
//
// o_t = sum_{s<=t} (q_t.k_s)^2 v_s / sum_{s<=t} (q_t.k_s)^2 evaluated tile by
// tile without materialising any state: the first operating point of the
// gist.science technical summary, sec. 2.3 (a FlashAttention-style O(T^2)
// forward), for bf16 inputs with fp32 accumulation.
//
// Persistent CTAs (one per SM) walk work items of two 128-row query tiles of
// one (b,h), heaviest first; key/value tiles of 128 rows stream through a
// 4-stage TMA ring that continues across items, and the Q tiles of the next
// item are prefetched into a second buffer.  Warp roles (576 threads):
//   warp 0      TMA producer (one lane): Q tiles once, then K/V tiles;
//   warp 1      TMEM allocator and MMA issuer (one lane);
//   warps 2-17  two "weight" groups of 8 warps, one per query tile; a
//               thread owns one row and one half of the key columns.
// Per key tile j and query tile i:
//   S_i      = Q_i K_j^T                 tcgen05.mma, A,B from shared memory,
//                                         fp32 accumulator in TMEM (128 cols)
//   W_i      = (S_i)^2, causal mask       tcgen05.ld -> registers -> bf16 ->
//                                         tcgen05.st back over S_i in TMEM
//   [O|D]_i += W_i [V_j | 1]              one tcgen05.mma per 16 keys with
//                                         A = W_i from TMEM; the B operand is
//                                         the V tile followed (one swizzle atom
//                                         further) by a block of ones, so the
//                                         denominator D comes out of the same
//                                         MMA, from the identical bf16 weights
// and at the end o = O_i / D_i (D = 0 gives 0), rounded to bf16.
// Causal masking touches only the diagonal tile; tiles above it are skipped.
//
// The MMA issue order alternates between the two query tiles
//   ... [O|D]_0 += W_0 V_j, S_0 = Q_0 K_{j+1}^T, [O|D]_1 += W_1 V_j,
//       S_1 = Q_1 K_{j+1}^T, ...
// so that one warpgroup squares its next tile while the tensor core works
// for the other.
//
// TMEM columns: S_0 [0,128) S_1 [128,256) [O|D]_0, [O|D]_1 (DV + 16 each)
// from 256; 512 columns are allocated.
//
// Every wait is bounded (sm100.cuh): a wait that runs out records
// KATA_ERR_TIMEOUT, the CTA drains its own TMA copies and MMAs, frees TMEM
// and exits.
#include <cuda.h>

#include "kata_internal.h"
#include "kata_trace.cuh"
#include "sm100.cuh"

KATA_TRACE_DECLARE(flash)

namespace kata {
namespace {

using namespace sm100;

constexpr int kBM = 128;       // query rows per tile
constexpr int kBN = 128;       // keys per tile
constexpr int kNQ = 2;         // query tiles per CTA
constexpr int kThreads = 576;  // 18 warps
constexpr uint32_t kTmemCols = 512;

template <int p, int DV>
struct FlashCfg {
  static constexpr int kQKBytes = kBM * p * 2;          // one Q or K tile
  static constexpr int kVBytes = kBN * DV * 2;          // one V tile
  // block of ones read as the second N-atom of the [V | 1] operand
  static constexpr int kOnesBytes = kBN * DV * 2;
  static constexpr int kStages = 4;                     // K/V ring depth
  // K-major Q/K rows are p*2 bytes: 32 B (p=16, 32B swizzle) or 64 B (p=32)
  static constexpr Swizzle kQKSw = (p == 16) ? kSw32 : kSw64;
  static constexpr uint32_t kQKSbo = 8 * p * 2;         // 8-row group stride
  // MN-major V rows are DV*2 bytes: 128 B (DV=64, 128B swizzle) or 32 B
  static constexpr Swizzle kVSw = (DV == 64) ? kSw128 : kSw32;
  static constexpr uint32_t kVSbo = 8 * DV * 2;         // 8-key group stride
  static constexpr uint32_t kVKStep = 16 * DV * 2;      // 16 keys
  // TMEM column map
  static constexpr uint32_t colS(int i) { return (uint32_t)i * 128; }
  static constexpr uint32_t colO(int i) { return 256u + (uint32_t)i * (DV + 16); }
  static constexpr uint32_t colD(int i) { return colO(i) + DV; }
  // shared memory map (offsets from a 1024-aligned base)
  static constexpr int offQ = 0;                        // 2 buffers x kNQ tiles
  static constexpr int offK = offQ + 2 * kNQ * kQKBytes;
  static constexpr int offV = ((offK + kStages * kQKBytes) + 1023) / 1024 * 1024;
  static constexpr int offOnes = offV + kStages * kVBytes;  // 1024-aligned
  // output staging: one [32 rows x DV/2] box per weight warp (row = DV bytes)
  static constexpr int kOutSlab = 32 * DV;
  static constexpr int offOut = offOnes + kOnesBytes;  // 1024-aligned
  static constexpr int offBar = offOut + 16 * kOutSlab;
  static constexpr int kNumBars = 4 + 2 * kStages + 4 * kNQ + 1;
  static constexpr int offMisc = offBar + kNumBars * 8;
  static constexpr int kSmemBytes = offMisc + 16 + 1024;  // + alignment slack
};

template <int p, int DV>
__global__ void __launch_bounds__(kThreads, 1)
    flash_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o, int T, int BH,
                     int H, int bthd, float* __restrict__ D_out, WaitCtl wc) {
  using Cfg = FlashCfg<p, DV>;
  constexpr int kStages = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::offBar);
  uint64_t* q_full = bars;                 // [2] Q buffers
  uint64_t* q_empty = q_full + 2;          // [2]
  uint64_t* kv_full = q_empty + 2;         // [kStages]
  uint64_t* kv_empty = kv_full + kStages;  // [kStages]
  uint64_t* s_full = kv_empty + kStages;   // [kNQ] scores of tile i in TMEM
  uint64_t* p_full = s_full + kNQ;         // [kNQ] weights of tile i written
  uint64_t* o_full = p_full + kNQ;         // [kNQ] [O|D] of tile i complete
  uint64_t* o_free = o_full + kNQ;         // [kNQ] [O|D] of tile i read by the epilogue
  uint64_t* mma_done = o_free + kNQ;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Cfg::offMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::offMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  KATA_TRACE_BEGIN(flash);
  // Persistent CTAs.  A work item is (pair of query tiles ct, head bh); items
  // are ordered heaviest first (largest ct) and dealt over CTAs in snake order.
  const int n_tiles = (T + kBM - 1) / kBM;
  const int n_ct = (n_tiles + kNQ - 1) / kNQ;
  const int n_items = n_ct * BH;
  auto item_ct = [&](int it) { return n_ct - 1 - it / BH; };
  auto item_bh = [&](int it) { return it % BH; };
  auto item_nkv = [&](int it, int i) {
    const int qtile = item_ct(it) * kNQ + i;
    return qtile < n_tiles ? qtile + 1 : 0;
  };
  // the r-th item of this CTA: rounds of gridDim.x items, dealt in a snake
  // order (odd rounds reversed) so that heavy and light items pair up; -1
  // once the items run out
  auto my_item = [&](int r) {
    const int it = r * (int)gridDim.x + ((r & 1) ? (int)gridDim.x - 1 - (int)blockIdx.x : (int)blockIdx.x);
    return it < n_items ? it : -1;
  };

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(q_full + b, 1);
      mbar_init(q_empty + b, 1);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    for (int i = 0; i < kNQ; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(p_full + i, 2 * kBM);
      mbar_init(o_full + i, 1);
      mbar_init(o_free + i, 2 * kBM);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  {  // block of bf16 ones for the denominator MMA
    uint32_t* ones = reinterpret_cast<uint32_t*>(smem + Cfg::offOnes);
    for (int x = threadIdx.x; x < Cfg::kOnesBytes / 4; x += kThreads) ones[x] = 0x3F803F80u;
    fence_proxy_async_smem();
  }
  if (warp == 1) tmem_alloc(tmem_holder, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitEnv env{wc.status, abort_flag, wc.limit};
  // rows [row, row + box) of head bh: the tensor maps are 4-D, {inner, T, H, B}
  // for the [B,H,T,inner] layout and {inner, H, T, B} for [B,T,H,inner]
  auto load_rows = [&](void* dst, const CUtensorMap* map, uint64_t* bar, int row, int bh) {
    const int b = bh / H, hd = bh - b * H;
    if (bthd)
      tma_load_4d(dst, map, bar, 0, hd, row, b);
    else
      tma_load_4d(dst, map, bar, 0, row, hd, b);
  };

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      int nq = 0;    // items whose Q was loaded
      long g = 0;    // key/value tiles loaded so far (ring position)
      bool ok = true;
      for (int it = my_item(nq); ok && it >= 0; it = my_item(++nq)) {
        const int qb = nq & 1, ct = item_ct(it), bh = item_bh(it);
        if (!mbar_wait(q_empty + qb, ((nq >> 1) & 1) ^ 1, env)) break;
        mbar_arrive_expect_tx(q_full + qb, kNQ * Cfg::kQKBytes);
        for (int i = 0; i < kNQ; ++i)
          load_rows(smem + Cfg::offQ + (qb * kNQ + i) * Cfg::kQKBytes, &tm_q, q_full + qb, (ct * kNQ + i) * kBM, bh);
        const int nkv_max = max(item_nkv(it, 0), item_nkv(it, 1));
        for (int j = 0; j < nkv_max; ++j, ++g) {
          const int st = (int)(g % kStages);
          if (!mbar_wait(kv_empty + st, (int)((g / kStages) & 1) ^ 1, env)) {
            ok = false;
            break;
          }
          KATA_TRACE(flash, (int)g, 9);
          mbar_arrive_expect_tx(kv_full + st, Cfg::kQKBytes + Cfg::kVBytes);
          load_rows(smem + Cfg::offK + st * Cfg::kQKBytes, &tm_k, kv_full + st, j * kBN, bh);
          load_rows(smem + Cfg::offV + st * Cfg::kVBytes, &tm_v, kv_full + st, j * kBN, bh);
        }
      }
      // drain: every copy this CTA started must land before it exits
      for (int n = nq - 2 < 0 ? 0 : nq - 2; n < nq; ++n) mbar_wait_drain(q_full + (n & 1), (n >> 1) & 1);
      for (long n = g - kStages < 0 ? 0 : g - kStages; n < g; ++n)
        mbar_wait_drain(kv_full + n % kStages, (int)((n / kStages) & 1));
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    // the whole warp runs this loop; one elected lane issues (see mma_ts_w)
    {
      constexpr uint32_t id_qk = idesc_bf16(kBM, kBN, false, false);
      constexpr uint32_t id_pv = idesc_bf16(kBM, DV + 16, false, true);  // [V | 1]
      const uint32_t sQ = smem_u32(smem + Cfg::offQ), sK = smem_u32(smem + Cfg::offK);
      const uint32_t sV = smem_u32(smem + Cfg::offV), sOnes = smem_u32(smem + Cfg::offOnes);
      // descriptors built once; K steps, Q buffers and stages are constant offsets
      const uint64_t dq0 = smem_desc(sQ, 16, Cfg::kQKSbo, Cfg::kQKSw);
      const uint64_t dk0 = smem_desc(sK, 16, Cfg::kQKSbo, Cfg::kQKSw);
      auto issue_qk = [&](int i, int qb, int st) {
        const uint64_t a = desc_add(dq0, (qb * kNQ + i) * Cfg::kQKBytes), b = desc_add(dk0, st * Cfg::kQKBytes);
#pragma unroll
        for (int ks = 0; ks < p / 16; ++ks) mma_ss_w(tmem + Cfg::colS(i), desc_add(a, ks * 32), desc_add(b, ks * 32), id_qk, ks > 0);
        mma_commit_w(s_full + i);
      };
      int nq = 0;
      long g = 0;                   // ring position of the item's first key tile
      int p_cnt[kNQ] = {0, 0};      // p_full phases consumed per tile
      int o_cnt[kNQ] = {0, 0};      // o_full phases committed per tile
      bool ok = true;
      for (int it = my_item(nq); ok && it >= 0; it = my_item(++nq)) {
        const int qb = nq & 1;
        int nkv[kNQ];
        for (int i = 0; i < kNQ; ++i) nkv[i] = item_nkv(it, i);
        const int nkv_max = max(nkv[0], nkv[1]);
        if (!mbar_wait_w(q_full + qb, (nq >> 1) & 1, env) || !mbar_wait_w(kv_full + g % kStages, (int)((g / kStages) & 1), env)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int i = 0; i < kNQ; ++i)
          if (nkv[i] > 0) issue_qk(i, qb, (int)(g % kStages));
        long kv_ready = g;  // highest ring position whose K/V landed
        for (int j = 0; ok && j < nkv_max; ++j) {
          const long gj = g + j;
          const int st = (int)(gj % kStages);
          const uint32_t sVst = sV + st * Cfg::kVBytes;
          const uint64_t dv = smem_desc(sVst, sOnes - sVst, Cfg::kVSbo, Cfg::kVSw);  // V atom, then ones atom
          for (int i = 0; i < kNQ; ++i) {
            if (j >= nkv[i]) continue;
            KATA_TRACE(flash, (int)gj, 2 * i);
            if (!mbar_wait_w(p_full + i, p_cnt[i] & 1, env)) {
              ok = false;
              break;
            }
            KATA_TRACE(flash, (int)gj, 2 * i + 1);
            ++p_cnt[i];
            // the first P.V of this tile overwrites [O|D]_i: the previous
            // item's epilogue must have read it
            if (j == 0 && o_cnt[i] > 0 && !mbar_wait_w(o_free + i, (o_cnt[i] - 1) & 1, env)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t aw = tmem + Cfg::colS(i), dO = tmem + Cfg::colO(i);
#pragma unroll
            for (int ks = 0; ks < kBN / 16; ++ks)  // keys 16ks..: W columns 64*(ks/4) + 8*(ks%4)
              mma_ts_w(dO, aw + (ks >> 2) * 64 + (ks & 3) * 8, desc_add(dv, ks * Cfg::kVKStep), id_pv,
                     (j > 0 || ks > 0) ? 1u : 0u);
            if (j == nkv[i] - 1) {
              mma_commit_w(o_full + i);
              ++o_cnt[i];
            }
            if (j + 1 < nkv[i]) {
              const long gn = gj + 1;
              if (kv_ready < gn) {
                if (!mbar_wait_w(kv_full + gn % kStages, (int)((gn / kStages) & 1), env)) {
                  ok = false;
                  break;
                }
                tc_fence_after();
                kv_ready = gn;
              }
              issue_qk(i, qb, (int)(gn % kStages));
            }
          }
          if (!ok) break;
          KATA_TRACE(flash, (int)gj, 4);
          mma_commit_w(kv_empty + st);
        }
        mma_commit_w(q_empty + qb);  // the item's Q tiles are free once its MMAs complete
        g += nkv_max;
      }
      mma_commit_w(mma_done);
      mbar_wait_drain(mma_done, 0);
    }
  } else {
    // ------------------------------------------------------------- weights + epilogue
    // warps 2-9 serve query tile 0, warps 10-17 query tile 1; within a tile
    // two warps share each TMEM lane quarter and split the 128 key columns:
    // half h squares keys 64h .. 64h+63 and writes their bf16 weights over
    // its own score columns [64h, 64h+32), so no warp overwrites scores
    // another warp has yet to read.
    const int idx = warp - 2;
    const int i = idx / 8;                 // query tile of this warpgroup
    const int h = (idx & 7) / 4;           // key-column half
    const int quarter = warp % 4;          // TMEM lane quarter this warp may access
    const int m = quarter * 32 + lane;     // row within the tile
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    // the output of a pair is read out of TMEM, scaled and staged in this
    // warp's shared-memory box right after the pair's last weights (which
    // frees the [O|D] buffer for the next pair); its TMA store is issued
    // after the next pair's first weights, so that the weights of the next
    // item never wait for the store
    constexpr int kHalf = DV / 2;          // output columns per thread
    uint8_t* slab = smem + Cfg::offOut + idx * Cfg::kOutSlab;
    bool pend = false;
    int pend_row0 = 0, pend_bh = 0;
    auto flush_out = [&]() {
      if (pend && lane == 0) {
        const int b = pend_bh / H, hd = pend_bh - b * H;
        if (bthd)
          tma_store_4d(&tm_o, slab, kHalf * h, hd, pend_row0, b);
        else
          tma_store_4d(&tm_o, slab, kHalf * h, pend_row0, hd, b);
        bulk_commit_group();
      }
      pend = false;
    };
    int s_cnt = 0, o_cnt = 0;
    bool ok = true;
    int rr = 0;
    for (int it = my_item(rr); ok && it >= 0; it = my_item(++rr)) {
      const int nkv = item_nkv(it, i);
      if (nkv == 0) {
        flush_out();
        continue;
      }
      const int bh = item_bh(it);
      const int row0 = (item_ct(it) * kNQ + i) * kBM + quarter * 32;  // this warp's first row
      for (int j = 0; j < nkv; ++j) {
        if (!mbar_wait_w(s_full + i, s_cnt & 1, env)) {
          ok = false;
          break;
        }
        if (m == 0 && h == 0) KATA_TRACE(flash, s_cnt, 5 + 2 * i);
        ++s_cnt;
        tc_fence_after();
        const bool diag = (j == nkv - 1);
        const uint32_t sa = lane_base + Cfg::colS(i) + 64 * h;
        // on the diagonal tile, 32-column block bb of row m is kept for
        // bb < quarter, masked for bb == quarter and zero for bb > quarter
        const int bb0 = 2 * h;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int bb = bb0 + hh;
          uint32_t w[16];
          if (diag && bb > quarter) {
#pragma unroll
            for (int x = 0; x < 16; ++x) w[x] = 0u;
          } else {
            uint32_t r[32];
            tmem_ld32(sa + 32 * hh, r);
            tmem_wait_ld();
            // squares on fp32 pairs (each rounded as a scalar multiply)
            if (diag && bb == quarter) {
#pragma unroll
              for (int x = 0; x < 16; ++x) {
                const uint32_t a = 2 * x > lane ? 0u : r[2 * x], b = 2 * x + 1 > lane ? 0u : r[2 * x + 1];
                const uint64_t sq = f32x2_mul(f32x2(a, b), f32x2(a, b));
                w[x] = pack_bf16x2(f32x2_lo(sq), f32x2_hi(sq));
              }
            } else {
#pragma unroll
              for (int x = 0; x < 16; ++x) {
                const uint64_t sq = f32x2_mul(f32x2(r[2 * x], r[2 * x + 1]), f32x2(r[2 * x], r[2 * x + 1]));
                w[x] = pack_bf16x2(f32x2_lo(sq), f32x2_hi(sq));
              }
            }
          }
          tmem_st16(sa + 16 * hh, w);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full + i);
        if (m == 0 && h == 0) KATA_TRACE(flash, s_cnt - 1, 6 + 2 * i);
        if (j == 0) flush_out();
      }
      if (!ok || !mbar_wait_w(o_full + i, o_cnt & 1, env)) break;
      ++o_cnt;
      tc_fence_after();
      uint32_t dbits;
      uint32_t ov[kHalf];
      tmem_ld1(lane_base + Cfg::colD(i), dbits);
      if constexpr (DV == 64) {
        tmem_ld32(lane_base + Cfg::colO(i) + kHalf * h, ov);
      } else {
        tmem_ld8(lane_base + Cfg::colO(i) + kHalf * h, ov);
      }
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(o_free + i);
      // o = O / D (D = 0 gives 0) rounded to bf16, staged as row `lane` of
      // the box: for DV = 64 the 64-byte rows are 64B-swizzled (16-byte chunk
      // e at e ^ ((lane / 2) % 4)), for DV = 16 the 16-byte rows are plain
      const float D = __uint_as_float(dbits);
      // the denominator of each row, for the backward pass (optional)
      if (D_out != nullptr && h == 0 && row0 + lane < T) D_out[(size_t)bh * T + row0 + lane] = D;
      const float inv = D > 0.f ? 1.f / D : 0.f;
      const uint64_t inv2 = f32x2(__float_as_uint(inv), __float_as_uint(inv));
      auto scaled = [&](int k) {
        const uint64_t v = f32x2_mul(f32x2(ov[k], ov[k + 1]), inv2);
        return pack_bf16x2(f32x2_lo(v), f32x2_hi(v));
      };
      if (lane == 0) bulk_wait_read_all();  // the previous store has read the box
      __syncwarp();
      uint8_t* orow = slab + lane * DV;
#pragma unroll
      for (int e = 0; e < kHalf / 8; ++e) {
        const int chunk = DV == 64 ? (e ^ ((lane >> 1) & 3)) : e;
        *reinterpret_cast<uint4*>(orow + chunk * 16) =
            make_uint4(scaled(8 * e), scaled(8 * e + 2), scaled(8 * e + 4), scaled(8 * e + 6));
      }
      fence_proxy_async_smem();
      __syncwarp();
      pend = true;
      pend_row0 = row0;
      pend_bh = bh;
    }
    if (ok) flush_out();
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

}  // namespace

EncodeTiledFn get_encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 3-D bf16 tensor map over [BH][T][inner] with a box of {box_inner, rows, 1};
// the swizzle is the one whose span equals the box row (32, 64 or 128 bytes).
bool make_tmap_bf16_box(CUtensorMap* map, const void* base, int inner, int T, int BH, int box_inner, int rows) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  const int row_bytes = inner * 2, box_bytes = box_inner * 2;
  CUtensorMapSwizzle sw = box_bytes == 32    ? CU_TENSOR_MAP_SWIZZLE_32B
                          : box_bytes == 64  ? CU_TENSOR_MAP_SWIZZLE_64B
                          : box_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                             : CU_TENSOR_MAP_SWIZZLE_NONE;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)T, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)row_bytes, (cuuint64_t)row_bytes * (cuuint64_t)T};
  cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 tensor map over [BH][T][inner] with a box of {inner, rows, 1}.
bool make_tmap_bf16(CUtensorMap* map, const void* base, int inner, int T, int BH, int rows) {
  return make_tmap_bf16_box(map, base, inner, T, BH, inner, rows);
}

// 4-D bf16 tensor map over a [B,H,T,inner] tensor (dims {inner, T, H, B}) or,
// with bthd, a [B,T,H,inner] tensor (dims {inner, H, T, B}), so that the
// strides grow with the dimension either way; the box covers box_inner
// values of `rows` consecutive tokens of one head, swizzled over the box row.
bool make_tmap_bf16_4d(CUtensorMap* map, const void* base, int inner, int T, int H, int B, bool bthd, int box_inner,
                       int rows) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  const cuuint64_t row_bytes = (cuuint64_t)inner * 2;
  const int box_bytes = box_inner * 2;
  CUtensorMapSwizzle sw = box_bytes == 32    ? CU_TENSOR_MAP_SWIZZLE_32B
                          : box_bytes == 64  ? CU_TENSOR_MAP_SWIZZLE_64B
                          : box_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                             : CU_TENSOR_MAP_SWIZZLE_NONE;
  cuuint64_t dims[4], strides[3];
  cuuint32_t box[4];
  dims[0] = (cuuint64_t)inner;
  dims[3] = (cuuint64_t)B;
  box[0] = (cuuint32_t)box_inner;
  box[3] = 1;
  if (bthd) {
    dims[1] = (cuuint64_t)H;
    dims[2] = (cuuint64_t)T;
    strides[0] = row_bytes;       // next head
    strides[1] = row_bytes * H;   // next token
    box[1] = 1;
    box[2] = (cuuint32_t)rows;
  } else {
    dims[1] = (cuuint64_t)T;
    dims[2] = (cuuint64_t)H;
    strides[0] = row_bytes;       // next token
    strides[1] = row_bytes * T;   // next head
    box[1] = (cuuint32_t)rows;
    box[2] = 1;
  }
  strides[2] = row_bytes * (cuuint64_t)T * (cuuint64_t)H;  // next batch entry
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int p, int DV>
static cudaError_t launch_flash_t(const void* q, const void* k, const void* v, void* o, int B, int H, int T, bool bthd,
                                  float* D_out, const WaitCtl& wc, cudaStream_t st) {
  using Cfg = FlashCfg<p, DV>;
  const int BH = B * H;
  CUtensorMap tq, tk, tv, to;
  if (!make_tmap_bf16_4d(&tq, q, p, T, H, B, bthd, p, kBM) || !make_tmap_bf16_4d(&tk, k, p, T, H, B, bthd, p, kBN) ||
      !make_tmap_bf16_4d(&tv, v, DV, T, H, B, bthd, DV, kBN) ||
      !make_tmap_bf16_4d(&to, o, DV, T, H, B, bthd, DV / 2, 32))
    return cudaErrorInvalidValue;
  auto kern = flash_fwd_kernel<p, DV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  // persistent: one CTA per SM (or fewer when there are fewer work items)
  static int num_sms = 0;
  if (num_sms == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || num_sms <= 0)
      num_sms = 148;
  }
  const long items = (long)((T + kBM * kNQ - 1) / (kBM * kNQ)) * BH;
  const int grid = (int)(items < num_sms ? items : num_sms);
  kern<<<grid, kThreads, Cfg::kSmemBytes, st>>>(tq, tk, tv, to, T, BH, H, bthd ? 1 : 0, D_out, wc);
  return cudaGetLastError();
}

cudaError_t launch_flash_sm100(const void* q, const void* k, const void* v, void* o, int B, int H, int T, int p, int dv,
                               bool bthd, float* D_out, const WaitCtl& wc, cudaStream_t st) {
  if (p == 16 && dv == 64) return launch_flash_t<16, 64>(q, k, v, o, B, H, T, bthd, D_out, wc, st);
  if (p == 16 && dv == 16) return launch_flash_t<16, 16>(q, k, v, o, B, H, T, bthd, D_out, wc, st);
  if (p == 32 && dv == 64) return launch_flash_t<32, 64>(q, k, v, o, B, H, T, bthd, D_out, wc, st);
  if (p == 32 && dv == 16) return launch_flash_t<32, 16>(q, k, v, o, B, H, T, bthd, D_out, wc, st);
  return cudaErrorInvalidValue;
}

}  // namespace kata
