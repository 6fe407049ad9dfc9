// flash_mg_sm100.cu -- quadratic (flash-style) KATA-Mg forward on tcgen05 / TMEM.
//
// KATA-Mg splits a head's d coordinates into G groups of width p = d / G and
// concatenates the groups' rank-one maps (arXiv abstract and gist.science
// sec. 2.3 "Varianten": several PSD factors; ai.info summary, Main Findings:
// state d(d/G+1)/2 * dv), so that
//   w_ts = sum_g (q_t^g . k_s^g)^2,   o_t = sum_{s<=t} w_ts v_s / sum_{s<=t} w_ts
// with one value vector and one denominator shared by the groups.
//
// Design (G = 2 or 4, dv = 64, bf16 inputs, fp32 accumulation):
//   * Persistent CTAs, one per SM; a work item is ONE 128-row query tile of
//     one (b,h), items heaviest first, dealt in snake order.  Key/value tiles
//     of 128 rows stream through a 4-stage TMA ring that continues across
//     items; the next item's Q tile is prefetched into a second buffer.
//   * The scores of two groups fit TMEM side by side (S_0 and S_1, 128 fp32
//     columns each), so one hand-off between the MMA warp and the weight
//     warps covers two groups: G = 2 needs one round per key tile, G = 4
//     two rounds whose squares are summed in registers.
//   * Sixteen weight warps share the tile: the warp of TMEM lane quarter qr
//     and key quarter kq owns rows 32qr.. and keys 32kq..32kq+31, reads
//     those 32 columns of every group's scores, sums the squares in fp32
//     pairs, applies the causal mask on the diagonal tile, and writes its 32
//     bf16 weights to its 16 columns of a weight buffer.
//   * The weights live apart from the scores, in two alternating TMEM
//     buffers, so the scores of key tile j+1 are computed as soon as the
//     weight warps have loaded those of tile j (barrier s_read), while they
//     square and convert; [O|D] += W_j [V_j | 1] follows once W_j is written
//     (B8 H16 T2048 d64, two groups: 132 -> 115 us against weights written
//     over the scores).  What remains is mostly the tensor pipe: the P.V
//     MMAs, which read their A operand from TMEM, run at about half rate
//     while sixteen warps load scores from TMEM beside them.
//   * [O|D] += W [V | 1] by one tcgen05.mma per 16 keys (A = W from TMEM),
//     the denominator coming out of the same MMA from the identical bf16
//     weights.
//   * Epilogue: each weight warp reads its 32 rows x 16 value columns of
//     [O|D], frees the accumulator, scales by 1/D (D = 0 gives 0), rounds to
//     bf16 and stages them as its own 32B-swizzled box; one TMA store per
//     warp, issued after the next item's first weights.
//   * Layout [B,H,T,*] or [B,T,H,*] through 4-D tensor maps; rows past T are
//     zero-filled on load and clipped on store.
// Every wait is bounded (sm100.cuh): a wait that runs out records
// KATA_ERR_TIMEOUT, the CTA drains its own TMA copies and MMAs, frees TMEM
// and exits.
#include <cuda.h>

#include "kata_internal.h"
#include "kata_trace.cuh"
#include "sm100.cuh"

KATA_TRACE_DECLARE(mg)

namespace kata {

bool make_tmap_bf16_4d(CUtensorMap* map, const void* base, int inner, int T, int H, int B, bool bthd, int box_inner,
                       int rows);

namespace {

using namespace sm100;

constexpr int kMgBM = 128;        // query rows per tile
constexpr int kMgBN = 128;        // keys per tile
constexpr int kMgDV = 64;
constexpr int kMgThreads = 576;   // warp 0 TMA, warp 1 MMA, warps 2-17 weights + epilogue
constexpr int kMgStages = 4;      // K/V ring depth
constexpr uint32_t kMgTmemCols = 512;

// kSum selects KATA-Sigma-g (summed factors, gist.science sec. 2.3
// "Varianten"): the weight is sum_{j,l} (q^j . k^l)^2 over every pair of a
// query group and a key group, so the kernel's score "groups" are the G^2
// pairs (j, l) -- the same pipeline with G^2 instead of G score blocks.
template <int p, int G, bool kSum = false>
struct MgCfg {
  static constexpr int kD = G * p;                      // q/k row width (32 or 64)
  static constexpr int kGR = 2;                         // score blocks per round
  static constexpr int kBlocks = kSum ? G * G : G;      // score blocks per key tile
  static constexpr int kRounds = kBlocks / kGR;
  // column group of the query (key) side of score block v
  static constexpr int q_group(int v) { return kSum ? v / G : v; }
  static constexpr int k_group(int v) { return kSum ? v % G : v; }
  static constexpr int kQKBytes = kMgBM * kD * 2;       // one Q or K tile
  static constexpr int kVBytes = kMgBN * kMgDV * 2;     // one V tile
  static constexpr int kOnesBytes = kMgBN * kMgDV * 2;  // ones block of the [V | 1] operand
  static constexpr Swizzle kQKSw = kD == 32 ? kSw64 : kSw128;
  static constexpr uint32_t kQKSbo = 8 * kD * 2;
  static constexpr uint32_t kVSbo = 8 * kMgDV * 2;
  static constexpr uint32_t kVKStep = 16 * kMgDV * 2;
  // TMEM columns: scores of the round's groups, two weight buffers, [O | D]
  static constexpr uint32_t colS(int gg) { return (uint32_t)gg * 128; }
  static constexpr uint32_t colW(int b) { return 256u + 64u * (uint32_t)b; }
  static constexpr uint32_t colO = 384;
  static constexpr uint32_t colD = colO + kMgDV;
  // shared memory (offsets from a 1024-aligned base)
  static constexpr int offQ = 0;                                   // 2 buffers
  static constexpr int offK = offQ + 2 * kQKBytes;
  static constexpr int offV = offK + kMgStages * kQKBytes;         // 1024-aligned
  static constexpr int offOnes = offV + kMgStages * kVBytes;
  static constexpr int kOutSlab = 32 * 16 * 2;                     // [32 rows x 16 values] per warp
  static constexpr int offOut = offOnes + kOnesBytes;
  static constexpr int offBar = offOut + 16 * kOutSlab;
  static constexpr int kNumBars = 4 + 2 * kMgStages + 7;
  static constexpr int offMisc = offBar + kNumBars * 8;
  static constexpr int kSmemBytes = offMisc + 16 + 1024;
  static_assert(kBlocks % kGR == 0, "score blocks per round");
  static_assert(offV % 1024 == 0 && offOnes % 1024 == 0 && offOut % 1024 == 0, "alignment");
};

template <int p, int G, bool kSum>
__global__ void __launch_bounds__(kMgThreads, 1)
    flash_mg_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o, int T, int BH,
                    int H, int bthd, float* __restrict__ D_out, WaitCtl wc) {
  using Cfg = MgCfg<p, G, kSum>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::offBar);
  uint64_t* q_full = bars;                    // [2]
  uint64_t* q_empty = q_full + 2;             // [2]
  uint64_t* kv_full = q_empty + 2;            // [kMgStages]
  uint64_t* kv_empty = kv_full + kMgStages;   // [kMgStages]
  uint64_t* s_full = kv_empty + kMgStages;    // a round's scores in TMEM
  uint64_t* s_read = s_full + 1;              // a round's scores read (512)
  uint64_t* p_full = s_read + 1;              // [2] weight buffer written (512)
  uint64_t* o_full = p_full + 2;              // [O|D] of the item complete
  uint64_t* o_free = o_full + 1;              // [O|D] read by the epilogue (512)
  uint64_t* mma_done = o_free + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Cfg::offMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::offMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  KATA_TRACE_BEGIN(mg);
  const int n_tiles = (T + kMgBM - 1) / kMgBM;
  const int n_items = n_tiles * BH;
  auto item_tile = [&](int it) { return n_tiles - 1 - it / BH; };  // heaviest first
  auto item_bh = [&](int it) { return it % BH; };
  auto my_item = [&](int r) {
    const int it = r * (int)gridDim.x + ((r & 1) ? (int)gridDim.x - 1 - (int)blockIdx.x : (int)blockIdx.x);
    return it < n_items ? it : -1;
  };

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(q_full + b, 1);
      mbar_init(q_empty + b, 1);
    }
    for (int s = 0; s < kMgStages; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_read, 512);
    mbar_init(p_full, 512);
    mbar_init(p_full + 1, 512);
    mbar_init(o_full, 1);
    mbar_init(o_free, 512);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  {
    uint32_t* ones = reinterpret_cast<uint32_t*>(smem + Cfg::offOnes);
    for (int x = threadIdx.x; x < Cfg::kOnesBytes / 4; x += kMgThreads) ones[x] = 0x3F803F80u;
    fence_proxy_async_smem();
  }
  if (warp == 1) tmem_alloc(tmem_holder, kMgTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const WaitEnv env{wc.status, abort_flag, wc.limit};
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
      int nq = 0;
      long g = 0;
      bool ok = true;
      for (int it = my_item(nq); ok && it >= 0; it = my_item(++nq)) {
        const int qb = nq & 1, tile = item_tile(it), bh = item_bh(it);
        if (!mbar_wait(q_empty + qb, ((nq >> 1) & 1) ^ 1, env)) break;
        mbar_arrive_expect_tx(q_full + qb, Cfg::kQKBytes);
        load_rows(smem + Cfg::offQ + qb * Cfg::kQKBytes, &tm_q, q_full + qb, tile * kMgBM, bh);
        for (int j = 0; j <= tile; ++j, ++g) {
          const int st = (int)(g % kMgStages);
          if (!mbar_wait(kv_empty + st, (int)((g / kMgStages) & 1) ^ 1, env)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(kv_full + st, Cfg::kQKBytes + Cfg::kVBytes);
          load_rows(smem + Cfg::offK + st * Cfg::kQKBytes, &tm_k, kv_full + st, j * kMgBN, bh);
          load_rows(smem + Cfg::offV + st * Cfg::kVBytes, &tm_v, kv_full + st, j * kMgBN, bh);
        }
      }
      for (int n = nq - 2 < 0 ? 0 : nq - 2; n < nq; ++n) mbar_wait_drain(q_full + (n & 1), (n >> 1) & 1);
      for (long n = g - kMgStages < 0 ? 0 : g - kMgStages; n < g; ++n)
        mbar_wait_drain(kv_full + n % kMgStages, (int)((n / kMgStages) & 1));
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    // the whole warp runs this loop; one elected lane issues (see mma_ss_w)
    {
      constexpr uint32_t id_qk = idesc_bf16(kMgBM, kMgBN, false, false);
      constexpr uint32_t id_pv = idesc_bf16(kMgBM, kMgDV + 16, false, true);  // [V | 1]
      const uint32_t sQ = smem_u32(smem + Cfg::offQ), sK = smem_u32(smem + Cfg::offK);
      const uint32_t sV = smem_u32(smem + Cfg::offV), sOnes = smem_u32(smem + Cfg::offOnes);
      const uint64_t dq0 = smem_desc(sQ, 16, Cfg::kQKSbo, Cfg::kQKSw);
      const uint64_t dk0 = smem_desc(sK, 16, Cfg::kQKSbo, Cfg::kQKSw);
      // scores of round r (groups kGR*r ..) of the key tile at stage st
      auto issue_round = [&](int qb, int st, int r) {
#pragma unroll
        for (int gg = 0; gg < Cfg::kGR; ++gg) {
          const int blk = r * Cfg::kGR + gg;
          const uint32_t qoff = (uint32_t)(Cfg::q_group(blk) * p * 2), koff = (uint32_t)(Cfg::k_group(blk) * p * 2);
          const uint64_t a = desc_add(dq0, qb * Cfg::kQKBytes + qoff), b = desc_add(dk0, st * Cfg::kQKBytes + koff);
#pragma unroll
          for (int ks = 0; ks < p / 16; ++ks)
            mma_ss_w(tmem + Cfg::colS(gg), desc_add(a, ks * 32), desc_add(b, ks * 32), id_qk, ks > 0);
        }
        mma_commit_w(s_full);
      };
      // rounds issued so far; round k + 1 overwrites the scores of round k,
      // so it first waits until the weight warps have loaded them (s_read)
      int r_cnt = 0;
      auto issue_tile = [&](int qb, int st) -> bool {
        for (int r = 0; r < Cfg::kRounds; ++r) {
          if (r_cnt > 0) {
            if (!mbar_wait_w(s_read, (r_cnt - 1) & 1, env)) return false;
            tc_fence_after();
          }
          ++r_cnt;
          issue_round(qb, st, r);
        }
        return true;
      };
      int n_step = 0, o_cnt = 0;  // key steps done (weight buffer n_step % 2); items finished
      int nq = 0;
      long g = 0;
      bool ok = true;
      for (int it = my_item(nq); ok && it >= 0; it = my_item(++nq)) {
        const int qb = nq & 1, nkv = item_tile(it) + 1;
        if (!mbar_wait_w(q_full + qb, (nq >> 1) & 1, env) ||
            !mbar_wait_w(kv_full + g % kMgStages, (int)((g / kMgStages) & 1), env)) {
          ok = false;
          break;
        }
        tc_fence_after();
        KATA_TRACE(mg, n_step, 0);
        if (!issue_tile(qb, (int)(g % kMgStages))) {
          ok = false;
          break;
        }
        KATA_TRACE(mg, n_step, 1);
        for (int j = 0; j < nkv; ++j) {
          const long gj = g + j;
          const int st = (int)(gj % kMgStages);
          // scores of key tile j + 1 first: they run while the weight warps
          // square tile j
          if (j + 1 < nkv) {
            const long gn = gj + 1;
            KATA_TRACE(mg, n_step + 1, 0);
            if (!mbar_wait_w(kv_full + gn % kMgStages, (int)((gn / kMgStages) & 1), env)) {
              ok = false;
              break;
            }
            tc_fence_after();
            if (!issue_tile(qb, (int)(gn % kMgStages))) {
              ok = false;
              break;
            }
            KATA_TRACE(mg, n_step + 1, 1);
          }
          const int wb = n_step & 1;
          if (!mbar_wait_w(p_full + wb, (n_step >> 1) & 1, env)) {
            ok = false;
            break;
          }
          KATA_TRACE(mg, n_step, 2);
          ++n_step;
          // the first P.V of the item overwrites [O|D]: the previous item's
          // epilogue must have read it
          if (j == 0 && o_cnt > 0 && !mbar_wait_w(o_free, (o_cnt - 1) & 1, env)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sVst = sV + st * Cfg::kVBytes;
          const uint64_t dv = smem_desc(sVst, sOnes - sVst, Cfg::kVSbo, kSw128);  // V atom, then ones atom
#pragma unroll
          for (int ks = 0; ks < kMgBN / 16; ++ks)  // keys 16ks..: weight buffer columns 8ks..
            mma_ts_w(tmem + Cfg::colO, tmem + Cfg::colW(wb) + 8 * ks, desc_add(dv, ks * Cfg::kVKStep), id_pv,
                     (j > 0 || ks > 0) ? 1u : 0u);
          KATA_TRACE(mg, n_step - 1, 3);
          if (j == nkv - 1) {
            mma_commit_w(o_full);
            ++o_cnt;
          }
          mma_commit_w(kv_empty + st);
        }
        mma_commit_w(q_empty + qb);
        g += nkv;
      }
      mma_commit_w(mma_done);
      mbar_wait_drain(mma_done, 0);
    }
  } else {
    // ------------------------------------------------------------- weights + epilogue
    const int quarter = warp % 4;          // TMEM lane quarter: rows 32 quarter ..
    const int kq = (warp - 2) / 4;         // key quarter: keys 32 kq .. 32 kq + 31
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    uint8_t* slab = smem + Cfg::offOut + (warp - 2) * Cfg::kOutSlab;  // [32 rows x 16 values], 32B rows
    bool pend = false;
    int pend_row0 = 0, pend_bh = 0;
    auto flush_out = [&]() {
      if (pend && lane == 0) {
        const int b = pend_bh / H, hd = pend_bh - b * H;
        if (bthd)
          tma_store_4d(&tm_o, slab, 16 * kq, hd, pend_row0, b);
        else
          tma_store_4d(&tm_o, slab, 16 * kq, pend_row0, hd, b);
        bulk_commit_group();
      }
      pend = false;
    };
    int s_cnt = 0, o_cnt = 0, n_step = 0;
    const int tslot = (warp == 2 && lane == 0) ? 5 : (warp == 17 && lane == 0) ? 8 : -1;  // traced warps
    bool ok = true;
    int rr = 0;
    for (int it = my_item(rr); ok && it >= 0; it = my_item(++rr)) {
      const int tile = item_tile(it), nkv = tile + 1, bh = item_bh(it);
      const int row0 = tile * kMgBM + quarter * 32;
      for (int j = 0; j < nkv; ++j) {
        const bool diag = (j == nkv - 1);
        // on the diagonal tile keys 32 kq + c of row 32 quarter + lane are
        // kept for kq < quarter, for c <= lane when kq == quarter, and are
        // zero (never read) for kq > quarter
        const bool skip = diag && kq > quarter;
        uint64_t acc[16];  // keys 2y, 2y + 1 of this warp's 32, fp32 pairs
        for (int r = 0; r < Cfg::kRounds; ++r) {
          if (!mbar_wait_w(s_full, s_cnt & 1, env)) {
            ok = false;
            break;
          }
          ++s_cnt;
          if (tslot >= 0 && r == 0) KATA_TRACE(mg, n_step, tslot);
          tc_fence_after();
          if (!skip) {
#pragma unroll
            for (int gg = 0; gg < Cfg::kGR; ++gg) {
#pragma unroll
              for (int hf = 0; hf < 2; ++hf) {
                uint32_t sc16[16];
                tmem_ld16(lane_base + Cfg::colS(gg) + 32 * kq + 16 * hf, sc16);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                  const uint64_t sc = f32x2(sc16[2 * x], sc16[2 * x + 1]);
                  uint64_t& a = acc[8 * hf + x];
                  a = (r == 0 && gg == 0) ? f32x2_mul(sc, sc) : f32x2_fma(sc, sc, a);
                }
              }
            }
          }
          // the scores are in registers: the next round or key tile may
          // overwrite them
          tc_fence_before();
          mbar_arrive(s_read);
          if (tslot >= 0 && r == Cfg::kRounds - 1) KATA_TRACE(mg, n_step, tslot + 1);
        }
        if (!ok) break;
        uint32_t w[16];
        if (skip) {
#pragma unroll
          for (int y = 0; y < 16; ++y) w[y] = 0u;
        } else if (diag && kq == quarter) {
#pragma unroll
          for (int y = 0; y < 16; ++y)
            w[y] = pack_bf16x2(2 * y > lane ? 0.f : f32x2_lo(acc[y]), 2 * y + 1 > lane ? 0.f : f32x2_hi(acc[y]));
        } else {
#pragma unroll
          for (int y = 0; y < 16; ++y) w[y] = pack_bf16x2(f32x2_lo(acc[y]), f32x2_hi(acc[y]));
        }
        // weight buffer n_step % 2: the P.V that last read it (two key steps
        // ago) completed before the scores just read were computed
        const int wb = n_step & 1;
        ++n_step;
        tmem_st16(lane_base + Cfg::colW(wb) + 16 * kq, w);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full + wb);
        if (tslot >= 0) KATA_TRACE(mg, n_step - 1, tslot + 2);
        if (j == 0) flush_out();
      }
      if (!ok || !mbar_wait_w(o_full, o_cnt & 1, env)) break;
      ++o_cnt;
      tc_fence_after();
      uint32_t dbits, ov[16];
      tmem_ld1(lane_base + Cfg::colD, dbits);
      tmem_ld16(lane_base + Cfg::colO + 16 * kq, ov);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(o_free);
      const float D = __uint_as_float(dbits);
      // the denominator of each row, for the backward pass (optional)
      if (D_out != nullptr && kq == 0 && row0 + lane < T) D_out[(size_t)bh * T + row0 + lane] = D;
      const float inv = D > 0.f ? 1.f / D : 0.f;
      const uint64_t inv2 = f32x2(__float_as_uint(inv), __float_as_uint(inv));
      auto scaled = [&](int x) {
        const uint64_t v = f32x2_mul(f32x2(ov[x], ov[x + 1]), inv2);
        return pack_bf16x2(f32x2_lo(v), f32x2_hi(v));
      };
      if (lane == 0) bulk_wait_read_all();  // the previous store has read the box
      __syncwarp();
      // row `lane` of the box: two 16-byte chunks, 32B-swizzled (chunk e at
      // e ^ ((lane / 4) % 2))
      uint8_t* orow = slab + lane * 32;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int chunk = e ^ ((lane >> 2) & 1);
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
    tmem_dealloc(tmem, kMgTmemCols);
  }
}

template <int p, int G, bool kSum = false>
static cudaError_t launch_flash_mg_t(const void* q, const void* k, const void* v, void* o, float* D_out, int B, int H,
                                     int T, bool bthd, const WaitCtl& wc, cudaStream_t st) {
  using Cfg = MgCfg<p, G, kSum>;
  CUtensorMap tq, tk, tv, to;
  if (!make_tmap_bf16_4d(&tq, q, Cfg::kD, T, H, B, bthd, Cfg::kD, kMgBM) ||
      !make_tmap_bf16_4d(&tk, k, Cfg::kD, T, H, B, bthd, Cfg::kD, kMgBN) ||
      !make_tmap_bf16_4d(&tv, v, kMgDV, T, H, B, bthd, kMgDV, kMgBN) ||
      !make_tmap_bf16_4d(&to, o, kMgDV, T, H, B, bthd, 16, 32))
    return cudaErrorInvalidValue;
  auto kern = flash_mg_kernel<p, G, kSum>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  static int num_sms = 0;
  if (num_sms == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || num_sms <= 0)
      num_sms = 148;
  }
  const long items = (long)((T + kMgBM - 1) / kMgBM) * B * H;
  const int grid = (int)(items < num_sms ? items : num_sms);
  kern<<<grid, kMgThreads, Cfg::kSmemBytes, st>>>(tq, tk, tv, to, T, B * H, H, bthd ? 1 : 0, D_out, wc);
  return cudaGetLastError();
}

}  // namespace

// One group per head stays on the single-factor kernel (flash_sm100.cu): its
// two query tiles per CTA interleave one tile's weights with the other's
// MMAs, which this kernel's single tile cannot (82 against 104 us at
// B8 H16 T2048 p16, with bitwise identical outputs).
bool flash_mg_sm100_supports(int p, int groups, int dv) {
  return dv == kMgDV && ((p == 16 && (groups == 2 || groups == 4)) || (p == 32 && groups == 2));
}

cudaError_t launch_flash_mg_sm100(const void* q, const void* k, const void* v, void* o, float* D_out, int B, int H, int T,
                                  int p, int groups, bool bthd, const WaitCtl& wc, cudaStream_t st) {
  if (p == 16 && groups == 2) return launch_flash_mg_t<16, 2>(q, k, v, o, D_out, B, H, T, bthd, wc, st);
  if (p == 16 && groups == 4) return launch_flash_mg_t<16, 4>(q, k, v, o, D_out, B, H, T, bthd, wc, st);
  if (p == 32 && groups == 2) return launch_flash_mg_t<32, 2>(q, k, v, o, D_out, B, H, T, bthd, wc, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_flash_sg_sm100(const void* q, const void* k, const void* v, void* o, float* D_out, int B, int H,
                                  int T, int p, int groups, bool bthd, const WaitCtl& wc, cudaStream_t st) {
  if (p == 16 && groups == 2) return launch_flash_mg_t<16, 2, true>(q, k, v, o, D_out, B, H, T, bthd, wc, st);
  if (p == 16 && groups == 4) return launch_flash_mg_t<16, 4, true>(q, k, v, o, D_out, B, H, T, bthd, wc, st);
  if (p == 32 && groups == 2) return launch_flash_mg_t<32, 2, true>(q, k, v, o, D_out, B, H, T, bthd, wc, st);
  return cudaErrorInvalidValue;
}

}  // namespace kata
