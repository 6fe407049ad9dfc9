// kata_internal.h -- host-side interface between the C ABI (kata_api.cu) and
// the kernel translation units.  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <mutex>

#include "../../include/kata.h"

namespace kata {

// Everything a kernel needs to report a bounded wait that ran out.
struct WaitCtl {
  int* status;           // device address of the library's status word
  long long limit;       // cycles before a wait gives up
};

// Layout of a workspace state record (one per (b,h) per super-chunk).
enum RecordLayout {
  kRecUnpacked = 0,  // P rows x ld floats: [sum psi(k) v^T | sum psi(k) | pad]
  kRecPackedT = 1,   // 65 rows x 144 floats: transposed, packed psi (p=16, dv=64; per block for p=32)
};

// Chunked-path plan: how the sequence is grouped for the state scan.
struct ChunkPlan {
  int BH;        // B * H
  int T;
  int p, P;      // psi input width, P = p * p
  int dv;
  int ld;        // row stride (floats) of an unpacked record: dv + 4
  int C;         // chunk length requested by the caller
  int Ls;        // super-chunk length (tokens per state record), multiple of 128 and C
  int G;         // number of super-chunks per (b,h): ceil(T / Ls)
  int layout;    // RecordLayout
  size_t record_floats;
  size_t workspace_bytes;
};

// True when the tensor-core chunked kernels serve these sizes (bf16, dv = 64,
// p = 16 in chunk_sm100.cu or p = 32 in chunk_p32_sm100.cu).
inline bool chunked_on_tensor_cores(int p, int dv, kata_dtype_t dt) {
  return dt == KATA_BF16 && (p == 16 || p == 32) && dv == 64;
}



ChunkPlan make_chunk_plan(int B, int H, int T, int p, int dv, int C, kata_dtype_t dt);
// The plan of the cluster kernels: p = factor width, `blocks` CTAs per unit.
ChunkPlan make_cluster_plan(int B, int H, int T, int p, int blocks, int dv, int C);

// Every argument check of kata_fwd_chunked except the workspace's (kata_api.cu).
kata_status_t check_chunked_args(const void* q, const void* k, const void* v, const void* o, int B, int H, int T,
                                 int p, int dv, int C, kata_dtype_t dtype, const float* S0, const float* z0,
                                 const float* S_out, const float* z_out);

// decode.cu -- `groups` PSD factors of width p per head (1: the single-factor step)
cudaError_t launch_decode(const void* q, const void* k, const void* v, void* o, float* S, float* z,
                          int BH, int p, int groups, int dv, kata_dtype_t dt, cudaStream_t st);
// the same with the summed (KATA-Sigma-g) feature: p*p state rows
cudaError_t launch_decode_sg(const void* q, const void* k, const void* v, void* o, float* S, float* z,
                             int BH, int p, int groups, int dv, kata_dtype_t dt, cudaStream_t st);

// scan.cu -- exclusive prefix over the G records of every (b,h), in place,
// plus S0 and the final state.  Records g >= G_in hold no data (treated as
// zero), so the tensor-core path, whose state kernel skips the last
// super-chunk, passes G_in = G - 1.
cudaError_t launch_state_scan(float* ws, const ChunkPlan& plan, int G_in, const float* S0, const float* z0,
                              float* S_out, float* z_out, cudaStream_t st);

// simt.cu -- CUDA-core kernels (fp32 inputs; exact fp32 arithmetic).
cudaError_t launch_quadratic_simt(const void* q, const void* k, const void* v, void* o, int BH, int T,
                                  int p, int dv, kata_dtype_t dt, cudaStream_t st);
cudaError_t launch_chunk_aggregate_simt(const void* k, const void* v, float* ws, const ChunkPlan& plan,
                                        kata_dtype_t dt, cudaStream_t st);
cudaError_t launch_chunk_readout_simt(const void* q, const void* k, const void* v, void* o, float* ws,
                                      const ChunkPlan& plan, kata_dtype_t dt, cudaStream_t st);

// flash_sm100.cu -- tcgen05 flash-style forward (bf16 inputs), one PSD
// factor of width p per head; bthd selects the [B,T,H,*] layout of q, k, v
// and o instead of [B,H,T,*].  D_out (nullable, fp32 [B*H, T]) receives each
// row's denominator.
cudaError_t launch_flash_sm100(const void* q, const void* k, const void* v, void* o, int B, int H, int T, int p, int dv,
                               bool bthd, float* D_out, const WaitCtl& wc, cudaStream_t st);

// flash_bwd_sm100.cu -- backward pass of the flash-style forward (bf16,
// p in {16, 32}, dv = 64, [B*H, T, *] layouts); D is the forward's
// denominator [B*H, T] fp32; ws holds flash_bwd_workspace_bytes().
// q, k, dq and dk rows are ld elements apart (ld = p for [B*H, T, p]; one
// group of a [B*H, T, d] tensor with ld = d); with rows_ready the per-row
// constants already in ws are reused; with dv_accumulate (dq_accumulate,
// dk_accumulate) the pass's dv (dq, dk) is added to what is there; with
// diag_only only the pairs of each 128-token tile with itself are taken (the
// intra-chunk part of the chunked backward).
size_t flash_bwd_workspace_bytes(int BH, int T, int dv);
// The per-row constants (-delta_t, 2/D_t) of the flash backward alone, into
// the first flash_bwd_workspace_bytes() of ws.
cudaError_t launch_flash_bwd_rows(const void* dO, const void* o, const float* D, void* ws, int BH, int T,
                                  cudaStream_t st);
cudaError_t launch_flash_bwd_sm100(const void* q, const void* k, const void* v, const void* o, const float* D,
                                   const void* dO, void* dq, void* dk, void* dv, int BH, int T, int p, int ld,
                                   bool rows_ready, bool dv_accumulate, bool dq_accumulate, bool dk_accumulate,
                                   void* ws, const WaitCtl& wc, cudaStream_t st, bool diag_only = false);

// flash_mg_sm100.cu -- tcgen05 flash-style KATA-Mg forward (bf16 inputs,
// dv = 64) with `groups` PSD factors of width p per head; D_out (nullable,
// fp32 [B*H, T]) receives each row's denominator.
bool flash_mg_sm100_supports(int p, int groups, int dv);
// KATA-Sigma-g (summed factors): the same kernel over all (query group, key
// group) score pairs; the (p, groups, dv) of flash_mg_sm100_supports.
cudaError_t launch_flash_sg_sm100(const void* q, const void* k, const void* v, void* o, float* D_out, int B, int H,
                                  int T, int p, int groups, bool bthd, const WaitCtl& wc, cudaStream_t st);
cudaError_t launch_flash_mg_sm100(const void* q, const void* k, const void* v, void* o, float* D_out, int B, int H, int T,
                                  int p, int groups, bool bthd, const WaitCtl& wc, cudaStream_t st);

// chunk_sm100.cu -- tcgen05 chunked-state forward (bf16 inputs, p = 16).
// The state kernel sums super-chunks 0..G-2 (the last one's sum is never
// needed); the readout of super-chunk g starts from workspace record g, or,
// when G == 1 (ws == nullptr), from S0/z0 (zero when null), and the readout
// of the last super-chunk writes the final state S_out/z_out when non-null.
cudaError_t launch_chunk_state_sm100(const void* k, const void* v, float* ws, const ChunkPlan& pl, const WaitCtl& wc,
                                     cudaStream_t st);
// D_out, when not null, receives each row's denominator [B*H, T] fp32 (the
// training forward of the chunked path).
cudaError_t launch_chunk_readout_sm100(const void* q, const void* k, const void* v, void* o, const float* ws,
                                       const float* S0, const float* z0, float* S_out, float* z_out,
                                       const ChunkPlan& pl, const WaitCtl& wc, cudaStream_t st,
                                       float* D_out = nullptr);
// The same kernels for KATA-Sigma-g with `groups` (2 or 4) groups of 16
// (d = 16 * groups): the summed feature on the p = 16 state, the same plan
// and record layout.
cudaError_t launch_chunk_state_sg(const void* k, const void* v, float* ws, const ChunkPlan& pl, int groups,
                                  const WaitCtl& wc, cudaStream_t st);
cudaError_t launch_chunk_readout_sg(const void* q, const void* k, const void* v, void* o, const float* ws,
                                    const float* S0, const float* z0, float* S_out, float* z_out,
                                    const ChunkPlan& pl, int groups, const WaitCtl& wc, cudaStream_t st);

// chunk_bwd_sm100.cu -- the inter-chunk part of the chunked backward (bf16,
// p = 16, dv = 64, [B*H, T, *]): per-super-chunk sums of the forward state and
// of the gradient state, their scan, and the two walks through each
// super-chunk's chunks that write the gradient terms to dq, dk, dv (which the
// diagonal-only flash backward adds to afterwards).  rowc is the flash
// backward's per-row (-delta, 2/D); records needs chunk_bwd_records_bytes()
// (0 when a super-chunk spans the whole sequence).
ChunkPlan chunk_bwd_plan(int BH, int T);
size_t chunk_bwd_records_bytes(int BH, int T);
cudaError_t launch_chunk_bwd_inter_sm100(const void* q, const void* k, const void* v, const void* dO,
                                         const float2* rowc, float* records, void* dq, void* dk, void* dv, int BH,
                                         int T, const WaitCtl& wc, cudaStream_t st);

// chunk_linear_sm100.cu -- first-order (linear) attention, psi(u) = u, with
// d = 16 and dv = 64 in bf16: the same three steps with unpacked records
// (make_linear_plan), the state entering each super-chunk from the scan (or
// S0/z0 when G == 1), the final state written by the last readout.
ChunkPlan make_linear_plan(int B, int H, int T, int d, int dv, int C);
cudaError_t launch_linear_state_sm100(const void* k, const void* v, float* ws, const ChunkPlan& pl, const WaitCtl& wc,
                                      cudaStream_t st);
cudaError_t launch_linear_readout_sm100(const void* q, const void* k, const void* v, void* o, const float* ws,
                                        const float* S0, const float* z0, float* S_out, float* z_out,
                                        const ChunkPlan& pl, const WaitCtl& wc, cudaStream_t st);

// chunk_cluster_sm100.cu -- the same with the packed state split over the
// CTAs of a cluster: p = 32 (groups = 1: four blocks) and KATA-Mg over d = 64
// (groups = 2 of p = 32: eight blocks; groups = 4 of p = 16: four blocks);
// q, k, v, o in [B,H,T,*] or, with bthd, [B,T,H,*].  Records
// ((bh * blocks + block) * G + g).  The readout adds S0/z0 (when non-null)
// to the scanned prefix of every super-chunk itself, so the scan runs
// without an initial state.  pl.p is the width of one factor.
bool cluster_chunked_supports(int p, int groups, int dv);
inline int cluster_blocks(int p, int groups) { return groups * (p == 32 ? 4 : 1); }
cudaError_t launch_chunk_state_cluster(const void* k, const void* v, float* ws, const ChunkPlan& pl, int H, int groups,
                                       bool bthd, const WaitCtl& wc, cudaStream_t st);
cudaError_t launch_chunk_readout_cluster(const void* q, const void* k, const void* v, void* o, const float* ws,
                                         const float* S0, const float* z0, float* S_out, float* z_out,
                                         const ChunkPlan& pl, int H, int groups, bool bthd, const WaitCtl& wc,
                                         cudaStream_t st);

// Current bound on in-kernel waits and the status word (kata_api.cu).
WaitCtl wait_ctl();

// Device addresses of file-scope __device__ arrays, for host code (kata_api.cu).
void* current_context();
class SymbolCache {
 public:
  // Address of `symbol` (the host-side name of a __device__ variable) on the
  // current device, or nullptr on failure.  Thread-safe.
  void* address(const void* symbol);

 private:
  static constexpr int kMaxDevices = 64;
  std::mutex mu_;
  void* ctx_[kMaxDevices] = {};
  void* addr_[kMaxDevices] = {};
};

}  // namespace kata
