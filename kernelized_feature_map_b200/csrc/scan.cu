// scan.cu -- inter-chunk state propagation as a work-efficient associative
// scan (parallel prefix sum).
//
// The chunk states combine by plain addition (the state update is
// commutative and additive: ai.info summary, Main Findings "The readout gate
// is free"), so the state entering super-chunk g is the exclusive prefix sum
// S0 + sum_{g' < g} A_{g'} of the per-super-chunk sums A_{g'}.  A sequential
// pass over the G records would have depth O(G); this kernel runs the
// up-sweep / down-sweep prefix scan (Blelloch) over them instead, depth
// O(log G) (gist.science technical summary, sec. 2.3 "Chunked Parallelism" /
// "Complexiteitsreductie": recurrence depth O(N_C) -> O(log N_C)).
//
// Work decomposition.  Up to 32 records per (b,h): one thread per record
// column runs the tree over that column's records in registers.  More
// records: one CTA per (b,h) and column block of NC record entries; the
// [G x NC] tile sits in shared memory (at most 1024 records per pass; longer
// sequences are scanned in blocks of 1024 with a running carry) and the 256
// threads share every tree level.  NC is chosen so that a tile is about
// 32 KiB.  Either way every record is streamed once in and once out.
//
// Record layouts (per (b,h), per super-chunk g), see kata_internal.h:
//   kRecUnpacked  P rows x ld floats: columns 0..dv-1 = sum psi(k) v^T,
//                 column dv = sum psi(k), the rest padding;
//   kRecPackedT   65 rows x 144 floats: row d < 64 = value column d, row 64 =
//                 normaliser; column = packed psi coordinate (runs i = 0..15
//                 of (i, j >= i), each padded to even length), off-diagonal
//                 coordinates carry the sum of the (i,j) and (j,i) entries.
// S0/z0 (optional initial state) and S_out/z_out (optional final state) use
// the ABI layout [P, dv] / [P] and are converted here.
#include "kata_common.cuh"
#include "kata_internal.h"

namespace kata {

constexpr int kScanBlock = 1024;  // records per shared-memory pass
constexpr int kScanThreads = 256;

// packed coordinate -> (i, j), -1 for a pad (p = 16): runs i = 0..15 of
// (i, j >= i), each padded to even length.  Built at compile time, so no
// upload (and no host-side state) is needed before the first launch.
struct PackTable {
  signed char i[144], j[144];
};
constexpr PackTable make_pack_table() {
  PackTable t{};
  int w = 0;
  for (int a = 0; a < 16; ++a) {
    for (int b = a; b < 16; ++b) {
      t.i[w] = (signed char)a;
      t.j[w] = (signed char)b;
      ++w;
    }
    if ((16 - a) & 1) {
      t.i[w] = -1;
      t.j[w] = -1;
      ++w;
    }
  }
  return t;
}
constexpr PackTable kPackTable = make_pack_table();
static_assert(kPackTable.i[16] == 1 && kPackTable.j[16] == 1 && kPackTable.i[31] == -1 &&
                  kPackTable.j[142] == 15 && kPackTable.i[143] == -1,
              "packed psi coordinate layout");
__constant__ PackTable c_pack = kPackTable;

struct ScanArgs {
  float* ws;
  int G;
  int G_in;       // records holding data (the rest are read as zero)
  int E;          // floats per record
  int NC;         // columns per CTA (power of two)
  int Gp;         // records per shared-memory pass (power of two)
  int layout;     // kRecUnpacked / kRecPackedT
  int p, P, dv, ld;
  const float* S0;
  const float* z0;
  float* S_out;
  float* z_out;
};

// Initial value of record entry e for (b,h) from the ABI-layout S0/z0.
__device__ __forceinline__ float initial_entry(const ScanArgs& a, long long bh, int e) {
  if (a.layout == kRecUnpacked) {
    const int r = e / a.ld, c = e % a.ld;
    if (c < a.dv) return a.S0[(bh * a.P + r) * a.dv + c];
    if (c == a.dv) return a.z0[bh * a.P + r];
    return 0.f;
  }
  const int d = e / 144, w = e % 144;
  const int i = c_pack.i[w], j = c_pack.j[w];
  if (i < 0) return 0.f;
  const int r1 = i * 16 + j, r2 = j * 16 + i;
  if (d < 64) {
    const float* S = a.S0 + bh * a.P * a.dv;
    return i == j ? S[r1 * a.dv + d] : S[r1 * a.dv + d] + S[r2 * a.dv + d];
  }
  const float* z = a.z0 + bh * a.P;
  return i == j ? z[r1] : z[r1] + z[r2];
}

// Write the final value of record entry e into the ABI-layout S_out/z_out.
__device__ __forceinline__ void final_entry(const ScanArgs& a, long long bh, int e, float val) {
  if (a.layout == kRecUnpacked) {
    const int r = e / a.ld, c = e % a.ld;
    if (c < a.dv) a.S_out[(bh * a.P + r) * a.dv + c] = val;
    else if (c == a.dv) a.z_out[bh * a.P + r] = val;
    return;
  }
  const int d = e / 144, w = e % 144;
  const int i = c_pack.i[w], j = c_pack.j[w];
  if (i < 0) return;
  const float h = i == j ? val : 0.5f * val;  // symmetric halves (exact)
  const int r1 = i * 16 + j, r2 = j * 16 + i;
  if (d < 64) {
    float* S = a.S_out + bh * a.P * a.dv;
    S[r1 * a.dv + d] = h;
    if (i != j) S[r2 * a.dv + d] = h;
  } else {
    float* z = a.z_out + bh * a.P;
    z[r1] = h;
    if (i != j) z[r2] = h;
  }
}

__global__ void __launch_bounds__(kScanThreads) state_scan_kernel(ScanArgs a) {
  // launched while the kernel that wrote the records may still run: let the
  // readout after it start launching, then wait for the records
  griddep_launch_dependents();
  griddep_wait();
  extern __shared__ float sm[];
  const int NC = a.NC, Gp_max = a.Gp;
  float* tile = sm;                       // [Gp_max][NC]
  float* carry = tile + Gp_max * NC;      // [NC]
  float* total = carry + NC;              // [NC]
  const int tid = threadIdx.x;
  const long long bh = blockIdx.y;
  const int col0 = blockIdx.x * NC;
  float* base = a.ws + bh * (long long)a.G * a.E + col0;
  int lognc = 0;
  while ((1 << lognc) < NC) ++lognc;

  for (int c = tid; c < NC; c += kScanThreads) {
    const int e = col0 + c;
    carry[c] = (a.S0 && e < a.E) ? initial_entry(a, bh, e) : 0.f;
  }
  for (int g0 = 0; g0 < a.G; g0 += kScanBlock) {
    const int n = min(kScanBlock, a.G - g0);
    int Gp = 1;
    while (Gp < n) Gp <<= 1;
    // loads are batched 32 deep so that many are in flight per thread
    for (int idx0 = 0; idx0 < Gp * NC; idx0 += 32 * kScanThreads) {
      float r[32];
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const int idx = idx0 + u * kScanThreads + tid;
        const int g = idx >> lognc, c = idx & (NC - 1);
        r[u] = (idx < Gp * NC && g < n && g0 + g < a.G_in && col0 + c < a.E)
                   ? __ldcs(base + (long long)(g0 + g) * a.E + c)
                   : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const int idx = idx0 + u * kScanThreads + tid;
        if (idx < Gp * NC) tile[idx] = r[u];
      }
    }
    __syncthreads();
    // up-sweep: tile[(2i+2)d - 1] += tile[(2i+1)d - 1]
    for (int d = 1; d < Gp; d <<= 1) {
      const int pairs = Gp / (2 * d);
      for (int idx = tid; idx < pairs * NC; idx += kScanThreads) {
        const int i = idx >> lognc, c = idx & (NC - 1);
        tile[((2 * i + 2) * d - 1) * NC + c] += tile[((2 * i + 1) * d - 1) * NC + c];
      }
      __syncthreads();
    }
    for (int c = tid; c < NC; c += kScanThreads) {
      total[c] = tile[(Gp - 1) * NC + c];
      tile[(Gp - 1) * NC + c] = 0.f;
    }
    __syncthreads();
    // down-sweep
    for (int d = Gp >> 1; d >= 1; d >>= 1) {
      const int pairs = Gp / (2 * d);
      for (int idx = tid; idx < pairs * NC; idx += kScanThreads) {
        const int i = idx >> lognc, c = idx & (NC - 1);
        float* lo = tile + ((2 * i + 1) * d - 1) * NC + c;
        float* hi = tile + ((2 * i + 2) * d - 1) * NC + c;
        const float t = *lo;
        *lo = *hi;
        *hi += t;
      }
      __syncthreads();
    }
    for (int idx = tid; idx < n * NC; idx += kScanThreads) {
      const int g = idx >> lognc, c = idx & (NC - 1);
      if (col0 + c < a.E) base[(long long)(g0 + g) * a.E + c] = carry[c] + tile[idx];
    }
    __syncthreads();
    for (int c = tid; c < NC; c += kScanThreads) carry[c] += total[c];
    __syncthreads();
  }
  if (a.S_out)
    for (int c = tid; c < NC; c += kScanThreads)
      if (col0 + c < a.E) final_entry(a, bh, col0 + c, carry[c]);
}

// Few records per (b,h): the same up-sweep / down-sweep tree (depth log2 GP),
// over one record column per thread held in registers.  Consecutive threads
// take consecutive columns, so every record row is read and written
// coalesced, and no shared memory or block barrier is needed.
constexpr int kScanRegThreads = 256;

template <int GP>
__global__ void __launch_bounds__(kScanRegThreads) state_scan_reg_kernel(ScanArgs a) {
  griddep_launch_dependents();
  griddep_wait();
  const int col = blockIdx.x * kScanRegThreads + threadIdx.x;
  const long long bh = blockIdx.y;
  if (col >= a.E) return;
  float* base = a.ws + bh * (long long)a.G * a.E + col;
  float x[GP];
#pragma unroll
  for (int g = 0; g < GP; ++g) x[g] = (g < a.G_in) ? __ldcs(base + (long long)g * a.E) : 0.f;
  const float carry = a.S0 ? initial_entry(a, bh, col) : 0.f;
  // up-sweep: x[(2i+2)d - 1] += x[(2i+1)d - 1]
#pragma unroll
  for (int d = 1; d < GP; d <<= 1)
#pragma unroll
    for (int i = 2 * d - 1; i < GP; i += 2 * d) x[i] += x[i - d];
  const float total = x[GP - 1];
  x[GP - 1] = 0.f;
  // down-sweep
#pragma unroll
  for (int d = GP >> 1; d >= 1; d >>= 1)
#pragma unroll
    for (int i = 2 * d - 1; i < GP; i += 2 * d) {
      const float t = x[i - d];
      x[i - d] = x[i];
      x[i] += t;
    }
#pragma unroll
  for (int g = 0; g < GP; ++g)
    if (g < a.G) base[(long long)g * a.E] = carry + x[g];
  if (a.S_out) final_entry(a, bh, col, carry + total);
}

cudaError_t launch_state_scan(float* ws, const ChunkPlan& plan, int G_in, const float* S0, const float* z0,
                              float* S_out, float* z_out, cudaStream_t st) {
  ScanArgs a;
  a.ws = ws;
  a.G = plan.G;
  a.G_in = G_in;
  a.E = (int)plan.record_floats;
  a.Gp = 1;
  while (a.Gp < plan.G && a.Gp < kScanBlock) a.Gp <<= 1;
  a.NC = 8192 / a.Gp;
  if (a.NC < 32) a.NC = 32;
  if (a.NC > 2048) a.NC = 2048;
  a.layout = plan.layout;
  a.p = plan.p;
  a.P = plan.P;
  a.dv = plan.dv;
  a.ld = plan.ld;
  a.S0 = S0;
  a.z0 = z0;
  a.S_out = S_out;
  a.z_out = z_out;
  if (plan.G <= 32) {
    // the scan always follows the kernel of the same call that wrote the
    // records: launched as its programmatic dependent
    const dim3 grid(ceil_div(a.E, kScanRegThreads), plan.BH), block(kScanRegThreads);
    if (plan.G <= 2) return launch_pdl(state_scan_reg_kernel<2>, grid, block, 0, st, a);
    if (plan.G <= 4) return launch_pdl(state_scan_reg_kernel<4>, grid, block, 0, st, a);
    if (plan.G <= 8) return launch_pdl(state_scan_reg_kernel<8>, grid, block, 0, st, a);
    if (plan.G <= 16) return launch_pdl(state_scan_reg_kernel<16>, grid, block, 0, st, a);
    return launch_pdl(state_scan_reg_kernel<32>, grid, block, 0, st, a);
  }
  const size_t smem = ((size_t)a.Gp * a.NC + 2 * (size_t)a.NC) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(state_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(state_scan_kernel, dim3(ceil_div(a.E, a.NC), plan.BH), dim3(kScanThreads), smem, st, a);
}

}  // namespace kata
