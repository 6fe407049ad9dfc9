// chunk_common.cuh -- pieces shared by the tcgen05 chunked-state kernels
// (chunk_sm100.cu for p = 16, chunk_p32_sm100.cu for p = 32): tile sizes,
// packed psi formation from a row of 16 bf16 values, the psi~(K) B-operand
// and psi~(Q) TMEM layouts, and the transposed state S~^T (TMEM) with its
// bf16 shared-memory copy and fp32 workspace record.
//
// Packed feature map.  psi(u) = vec(u u^T) is symmetric, so a factor of 16
// coordinates needs only its n = 136 unique coordinates (ai.info summary,
// Main Findings, "State size, not just feature width, dominates memory").
// They are ordered by runs: for i = 0..15 the entries (i, j), j = i..15, each
// run padded with one zero to even length, 144 = 9 x 16 coordinates in all,
// so that every bf16 pair comes from one bf16x2 multiply.  The query side
// holds u_i u_j; the key side holds u_i^2 on the diagonal and 2 u_i u_j off
// it (the factor 2 is exact), so <psi~(q), psi~(k)> = (q . k)^2.
#pragma once

#include <cuda.h>

#include "sm100.cuh"

namespace kata {
namespace chunk {

using namespace sm100;

constexpr int kTile = 128;          // tokens per chunk = MMA M
constexpr int kDV = 64;
constexpr int kNP = 144;            // packed psi coordinates (with pads)
constexpr int kNPW = kNP / 2;       // bf16x2 words per packed psi row
constexpr int kRecRows = kDV + 1;   // workspace record rows: dv value rows + z
constexpr int kQKBytes = kTile * 16 * 2;   // Q or K tile (32-byte rows, 32B swizzle)
constexpr int kVBytes = kTile * kDV * 2;   // V tile (128-byte rows, 128B swizzle)
constexpr int kOnesBytes = kTile * 64 * 2; // one 128B-swizzle atom of ones
// psi~(K_c): B operand [K = 128 tokens x N = 144], N-major, 32-byte swizzle:
// 9 atoms of 16 coordinates, each [128 tokens x 32 B]
constexpr uint32_t kPsiAtom = kTile * 32;
constexpr int kPsiBytes = 9 * kPsiAtom;    // 36 KiB
// bf16 copy of the state for the readout: B operand [K = 144 x N = 80],
// K-major, 32-byte swizzle: 9 atoms (one per K step) of [80 rows x 32 B]
constexpr int kSBRows = 80;
constexpr uint32_t kSBAtom = kSBRows * 32;
constexpr int kSBBytes = 9 * kSBAtom;      // 22.5 KiB

// --------------------------------------------------------------------------
// packed psi formation
// --------------------------------------------------------------------------
__device__ __forceinline__ uint32_t as_u32(__nv_bfloat162 h) { return *reinterpret_cast<uint32_t*>(&h); }

// Row of 16 bf16 from a 32-byte-swizzled tile (row r at r*32, 16-byte chunk
// c stored at chunk c ^ ((r >> 2) & 1)).
__device__ __forceinline__ void load_row_sw32(const uint8_t* tile, int r, __nv_bfloat162 (&u)[8]) {
  const uint8_t* row = tile + r * 32;
  const int x = (r >> 2) & 1;
  const uint4 a = *reinterpret_cast<const uint4*>(row + ((0 ^ x) << 4));
  const uint4 b = *reinterpret_cast<const uint4*>(row + ((1 ^ x) << 4));
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) u[i] = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
}

// The 72 bf16x2 words of packed psi for one token.  key = true applies the
// factor 2 off the diagonal.
template <bool key>
__device__ __forceinline__ void packed_psi(const __nv_bfloat162 (&u)[8], uint32_t (&out)[kNPW]) {
  // s[y] = (u_{2y+1}, u_{2y+2}), s[7] = (u_15, 0): pairs starting at odd j
  __nv_bfloat162 s[8];
#pragma unroll
  for (int y = 0; y < 7; ++y) s[y] = __halves2bfloat162(u[y].y, u[y + 1].x);
  s[7] = __halves2bfloat162(u[7].y, __float2bfloat16_rn(0.f));
  int w = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const __nv_bfloat16 ui = (i & 1) ? u[i >> 1].y : u[i >> 1].x;
    const __nv_bfloat16 ui2 = key ? __hmul(ui, __float2bfloat16_rn(2.f)) : ui;
    const int npairs = (16 - i + 1) / 2;
#pragma unroll
    for (int x = 0; x < npairs; ++x) {
      const int j0 = i + 2 * x;
      const __nv_bfloat162 pr = (j0 & 1) ? s[j0 >> 1] : u[j0 >> 1];
      const __nv_bfloat162 f = (x == 0) ? __halves2bfloat162(ui, ui2) : __halves2bfloat162(ui2, ui2);
      out[w++] = as_u32(__hmul2(f, pr));
    }
  }
}

// Row r of a [128 x 16G] bf16 tile as loaded by TMA with the swizzle of its
// row width (32, 64 or 128 bytes: 16-byte chunk c of row r stored at chunk
// c ^ ((r >> 2) & 1), c ^ ((r >> 1) & 3) or c ^ (r & 7)); u[8g + e] holds
// values 16g + 2e, 16g + 2e + 1.
template <int G>
__device__ __forceinline__ void load_row_sw(const uint8_t* tile, int r, __nv_bfloat162 (&u)[8 * G]) {
  static_assert(G == 1 || G == 2 || G == 4, "row widths of 32, 64 or 128 bytes");
  const uint8_t* row = tile + r * 32 * G;
  const int x = G == 1 ? (r >> 2) & 1 : G == 2 ? (r >> 1) & 3 : r & 7;
#pragma unroll
  for (int c = 0; c < 2 * G; ++c) {
    const uint4 a = *reinterpret_cast<const uint4*>(row + ((c ^ x) << 4));
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) u[4 * c + e] = *reinterpret_cast<const __nv_bfloat162*>(&w[e]);
  }
}

// Half `half` of the packed summed feature psi~_S(u) = sum_g psi~(u^g) of one
// token with G groups of 16 values (u as from load_row_sw<G>): the words of
// packed_psi_half, each entry sum_g u^g_i u^g_j accumulated over the groups
// in fp32 and rounded to bf16 once; key = true applies the factor 2 off the
// diagonal (exact).
template <bool key, int half, int G>
__device__ __forceinline__ void packed_psi_sum_half(const __nv_bfloat162 (&u)[8 * G], uint32_t (&out)[kNPW / 2]) {
  auto val = [&](int g, int i) {
    return __bfloat162float((i & 1) ? u[8 * g + (i >> 1)].y : u[8 * g + (i >> 1)].x);
  };
  int w = 0;
#pragma unroll
  for (int i = (half == 0 ? 0 : 5); i < (half == 0 ? 5 : 16); ++i) {
    const int npairs = (16 - i + 1) / 2;
#pragma unroll
    for (int x = 0; x < npairs; ++x) {
      const int j0 = i + 2 * x;
      float a = 0.f, b = 0.f;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float ui = val(g, i);
        a = fmaf(ui, val(g, j0), a);
        if (j0 + 1 < 16) b = fmaf(ui, val(g, j0 + 1), b);
      }
      if (key) {
        if (x > 0) a *= 2.f;
        b *= 2.f;
      }
      out[w++] = pack_bf16x2(a, b);
    }
  }
}

// Half of the packed psi words of one token: half 0 = runs i = 0..4 (words
// 0..35), half 1 = runs i = 5..15 (words 36..71); used when two threads
// share a token.
template <bool key, int half>
__device__ __forceinline__ void packed_psi_half(const __nv_bfloat162 (&u)[8], uint32_t (&out)[kNPW / 2]) {
  __nv_bfloat162 s[8];
#pragma unroll
  for (int y = 0; y < 7; ++y) s[y] = __halves2bfloat162(u[y].y, u[y + 1].x);
  s[7] = __halves2bfloat162(u[7].y, __float2bfloat16_rn(0.f));
  int w = 0;
#pragma unroll
  for (int i = (half == 0 ? 0 : 5); i < (half == 0 ? 5 : 16); ++i) {
    const __nv_bfloat16 ui = (i & 1) ? u[i >> 1].y : u[i >> 1].x;
    const __nv_bfloat16 ui2 = key ? __hmul(ui, __float2bfloat16_rn(2.f)) : ui;
    const int npairs = (16 - i + 1) / 2;
#pragma unroll
    for (int x = 0; x < npairs; ++x) {
      const int j0 = i + 2 * x;
      const __nv_bfloat162 pr = (j0 & 1) ? s[j0 >> 1] : u[j0 >> 1];
      const __nv_bfloat162 f = (x == 0) ? __halves2bfloat162(ui, ui2) : __halves2bfloat162(ui2, ui2);
      out[w++] = as_u32(__hmul2(f, pr));
    }
  }
}

// Half `half` (36 words) of psi~(k) of token t into the B tile: word groups
// of 4 are 16-byte chunks, group g -> atom g / 2, chunk g % 2.
template <int half>
__device__ __forceinline__ void store_psi_k_half(uint8_t* psi, int t, const uint32_t (&w)[kNPW / 2]) {
  const int x = (t >> 2) & 1;
#pragma unroll
  for (int q = 0; q < 9; ++q) {
    const int g = half * 9 + q, a = g >> 1, c = g & 1;
    *reinterpret_cast<uint4*>(psi + a * kPsiAtom + t * 32 + ((c ^ x) << 4)) =
        make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  }
}

// psi~(k) of token t into the N-major 32B-swizzled B tile.
__device__ __forceinline__ void store_psi_k(uint8_t* psi, int t, const uint32_t (&w)[kNPW]) {
  const int x = (t >> 2) & 1;
#pragma unroll
  for (int a = 0; a < 9; ++a) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int w0 = a * 8 + c * 4;
      *reinterpret_cast<uint4*>(psi + a * kPsiAtom + t * 32 + ((c ^ x) << 4)) =
          make_uint4(w[w0], w[w0 + 1], w[w0 + 2], w[w0 + 3]);
    }
  }
}

// psi~(q) of one query row into TMEM columns [col, col + 72) of this lane.
__device__ __forceinline__ void store_psi_q_tmem(uint32_t taddr, const uint32_t (&w)[kNPW]) {
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    uint32_t r[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) r[e] = w[16 * b + e];
    tmem_st16(taddr + 16 * b, r);
  }
  uint32_t r[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) r[e] = w[64 + e];
  tmem_st8(taddr + 64, r);
}

// Half `half` (words 36 * half ..) of psi~(q) of one query row into TMEM
// columns [col + 36 * half, col + 36 * half + 36) of this lane; every store
// starts at a column that is a multiple of its width.
template <int half>
__device__ __forceinline__ void store_psi_q_tmem_half(uint32_t taddr, const uint32_t (&w)[kNPW / 2]) {
  if constexpr (half == 0) {
    uint32_t a[16], b[16], c[4];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      a[e] = w[e];
      b[e] = w[16 + e];
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) c[e] = w[32 + e];
    tmem_st16(taddr, a);
    tmem_st16(taddr + 16, b);
    tmem_st4(taddr + 32, c);
  } else {
    uint32_t c[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) c[e] = w[e];
    tmem_st4(taddr + 36, c);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t r[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) r[e] = w[4 + 8 * q + e];
      tmem_st8(taddr + 40 + 8 * q, r);
    }
  }
}

// --------------------------------------------------------------------------
// state rows: TMEM <-> registers <-> bf16 copy, 16 or 32 columns at a time
// --------------------------------------------------------------------------
// 16 consecutive packed coordinates (one K step) of row n of the bf16 state
// copy (K-major, one 32B-swizzled atom of [80 rows x 32 B] per K step).
__device__ __forceinline__ void store_state_bf16_atom(uint8_t* sb, int n, int atom, const uint32_t* bits) {
  const int sw = (n >> 2) & 1;
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const uint32_t* e = bits + 8 * c;
    *reinterpret_cast<uint4*>(sb + atom * kSBAtom + n * 32 + ((c ^ sw) << 4)) = make_uint4(
        pack_bf16x2(__uint_as_float(e[0]), __uint_as_float(e[1])), pack_bf16x2(__uint_as_float(e[2]), __uint_as_float(e[3])),
        pack_bf16x2(__uint_as_float(e[4]), __uint_as_float(e[5])), pack_bf16x2(__uint_as_float(e[6]), __uint_as_float(e[7])));
  }
}

// TMEM lane -> fp32 record row in global memory (when `active`).
// Warp-collective.
__device__ __forceinline__ void state_lane_to_global(uint32_t taddr, float* row, bool active) {
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    uint32_t r[32];
    tmem_ld32(taddr + 32 * b, r);
    tmem_wait_ld();
    if (active)
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        *reinterpret_cast<float4*>(row + 32 * b + e) = make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]),
                                                                   __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
  }
  uint32_t r[16];
  tmem_ld16(taddr + 128, r);
  tmem_wait_ld();
  if (active)
#pragma unroll
    for (int e = 0; e < 16; e += 4)
      *reinterpret_cast<float4*>(row + 128 + e) = make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]),
                                                              __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
}

// One 8-coordinate chunk (c = 0 or 1) of atom `atom` of row n of the bf16 copy.
__device__ __forceinline__ void store_state_bf16_chunk(uint8_t* sb, int n, int atom, int c, const uint32_t* e) {
  const int sw = (n >> 2) & 1;
  *reinterpret_cast<uint4*>(sb + atom * kSBAtom + n * 32 + ((c ^ sw) << 4)) = make_uint4(
      pack_bf16x2(__uint_as_float(e[0]), __uint_as_float(e[1])), pack_bf16x2(__uint_as_float(e[2]), __uint_as_float(e[3])),
      pack_bf16x2(__uint_as_float(e[4]), __uint_as_float(e[5])), pack_bf16x2(__uint_as_float(e[6]), __uint_as_float(e[7])));
}

// Half `half` of a TMEM lane of S~^T (half 0: packed coordinates 0..71,
// half 1: 72..143) -> bf16 copy row n (when `active`).  All loads of the half
// are in flight before a single wait.  Warp-collective.
__device__ __forceinline__ void state_half_to_bf16(uint32_t taddr, uint8_t* sb, int n, bool active, int half) {
  uint32_t a[32], b[32], c[8];
  if (half == 0) {
    tmem_ld32(taddr, a);
    tmem_ld32(taddr + 32, b);
    tmem_ld8(taddr + 64, c);
    tmem_wait_ld();
    if (active) {
      store_state_bf16_atom(sb, n, 0, a);
      store_state_bf16_atom(sb, n, 1, a + 16);
      store_state_bf16_atom(sb, n, 2, b);
      store_state_bf16_atom(sb, n, 3, b + 16);
      store_state_bf16_chunk(sb, n, 4, 0, c);
    }
  } else {
    tmem_ld8(taddr + 72, c);
    tmem_ld32(taddr + 80, a);
    tmem_ld32(taddr + 112, b);
    tmem_wait_ld();
    if (active) {
      store_state_bf16_chunk(sb, n, 4, 1, c);
      store_state_bf16_atom(sb, n, 5, a);
      store_state_bf16_atom(sb, n, 6, a + 16);
      store_state_bf16_atom(sb, n, 7, b);
      store_state_bf16_atom(sb, n, 8, b + 16);
    }
  }
}

// Half of an fp32 record row (or zeros) -> TMEM lane and bf16 copy row n.
// Warp-collective.
__device__ __forceinline__ void global_half_to_state(const float* row, uint32_t taddr, uint8_t* sb, int n,
                                                     bool active, int half) {
  auto ld4 = [&](int col, uint32_t* r) {
    float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (active) v4 = *reinterpret_cast<const float4*>(row + col);
    r[0] = __float_as_uint(v4.x);
    r[1] = __float_as_uint(v4.y);
    r[2] = __float_as_uint(v4.z);
    r[3] = __float_as_uint(v4.w);
  };
  const int a0 = half == 0 ? 0 : 5;  // first whole atom of the half
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    uint32_t r[16];
#pragma unroll
    for (int e = 0; e < 16; e += 4) ld4(16 * (a0 + a) + e, r + e);
    tmem_st16(taddr + 16 * (a0 + a), r);
    if (active) store_state_bf16_atom(sb, n, a0 + a, r);
  }
  uint32_t r[8];
  const int col = half == 0 ? 64 : 72;
  ld4(col, r);
  ld4(col + 4, r + 4);
  tmem_st8(taddr + col, r);
  if (active) store_state_bf16_chunk(sb, n, 4, half, r);
}

// Packed coordinate w -> (i, j) of psi, or i = j = -1 for a pad (runs
// i = 0..15 of (i, j >= i), each padded to even length).  Evaluated at compile
// time inside fully unrolled loops.
__host__ __device__ constexpr int packed_i(int w) {
  int base = 0;
  for (int i = 0; i < 16; ++i) {
    const int len = (16 - i) + ((16 - i) & 1);
    if (w < base + len) return w - base < 16 - i ? i : -1;
    base += len;
  }
  return -1;
}
__host__ __device__ constexpr int packed_j(int w) {
  int base = 0;
  for (int i = 0; i < 16; ++i) {
    const int len = (16 - i) + ((16 - i) & 1);
    if (w < base + len) return w - base < 16 - i ? i + (w - base) : -1;
    base += len;
  }
  return -1;
}
static_assert(packed_i(0) == 0 && packed_j(0) == 0 && packed_j(15) == 15 && packed_i(16) == 1 && packed_j(16) == 1 &&
                  packed_i(31) == -1 && packed_i(32) == 2 && packed_i(143) == -1 && packed_j(142) == 15,
              "packed psi coordinate layout");

// Value of packed coordinate w of row d of the state in the ABI layout
// (S [p*p, dv], z [p*p], psi index r = i*p + j): the sum of the (i, j) and
// (j, i) entries off the diagonal (the packed key side carries the factor 2).
// Called with w known at compile time after unrolling.
__device__ __forceinline__ float abi_packed_entry(const float* S, const float* z, int d, int w) {
  const int i = packed_i(w), j = packed_j(w);
  if (i < 0) return 0.f;
  if (d < kDV) return i == j ? S[(i * 16 + j) * kDV + d] : S[(i * 16 + j) * kDV + d] + S[(j * 16 + i) * kDV + d];
  return i == j ? z[i * 16 + j] : z[i * 16 + j] + z[j * 16 + i];
}

// Half `half` of row d (<= 64) of the state, packed, from the ABI-layout
// initial state (zeros when S is null) -> TMEM lane and bf16 copy row n.
// Warp-collective.
template <int half>
__device__ __forceinline__ void abi_half_to_state(const float* S, const float* z, int d, uint32_t taddr, uint8_t* sb,
                                                  int n, bool active) {
  uint32_t r[72];
#pragma unroll
  for (int e = 0; e < 72; ++e) r[e] = __float_as_uint(S && active ? abi_packed_entry(S, z, d, 72 * half + e) : 0.f);
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

// Half `half` of TMEM lane d (<= 64) of the final state -> the ABI layout
// (an off-diagonal packed entry is halved into (i, j) and (j, i), exactly).
// Warp-collective.
template <int half>
__device__ __forceinline__ void state_half_to_abi(uint32_t taddr, float* S, float* z, int d, bool active) {
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
    const int w = 72 * half + e;
    const int i = packed_i(w), j = packed_j(w);
    if (i < 0) continue;
    const float val = __uint_as_float(r[e]);
    const float hv = i == j ? val : 0.5f * val;
    if (d < kDV) {
      S[(i * 16 + j) * kDV + d] = hv;
      if (i != j) S[(j * 16 + i) * kDV + d] = hv;
    } else {
      z[i * 16 + j] = hv;
      if (i != j) z[j * 16 + i] = hv;
    }
  }
}

__device__ __forceinline__ void fill_ones(uint8_t* ones, int tid, int nthreads) {
  uint32_t* w = reinterpret_cast<uint32_t*>(ones);
  for (int x = tid; x < kOnesBytes / 4; x += nthreads) w[x] = 0x3F803F80u;
}

// [V_c | 1] as an MN-major operand with 128-byte swizzle: the V tile is the
// first atom (columns / rows 0..63), the block of ones the second (64..127).
// Used as the A operand [V_c | 1]^T (M = 128) of the state update and as the
// B operand [V_c | 1] (N = 80) of the intra-chunk product.  K steps of 16
// tokens are +2048 bytes.
__device__ __forceinline__ uint64_t desc_vones(uint32_t sV, uint32_t sOnes) {
  return smem_desc(sV, sOnes - sV, 1024, kSw128);
}

}  // namespace chunk
}  // namespace kata
