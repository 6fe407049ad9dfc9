/*
 * kata.h -- C ABI of libkata, the sm_100a (B200) KATA forward library.
 *
 * The operation is causal normalized linear attention with the rank-one PSD
 * feature map psi(u) = vec(u u^T).  For one (batch b, head h) pair, with
 * q_t, k_t in R^p and v_t in R^dv (t = 1..T):
 *
 *   w_{t,s} = <psi(q_t), psi(k_s)> = (q_t . k_s)^2 >= 0
 *   o_t     = sum_{s<=t} w_{t,s} v_s  /  sum_{s<=t} w_{t,s}
 *
 * -- gist.science technical summary of arXiv:2607.17419, sec. 2.2 ("PSD Kegel
 *    (Rank-One)": the map squares the raw inner product) and sec. 2.1
 *    ("Output Gating": the denominator is a parameter-free convex output
 *    gate); ai.info summary, Main Findings ("The readout gate is free").
 *
 * Equivalently, with the fixed-size state S_t = sum_{s<=t} psi(k_s) v_s^T
 * (p^2 x dv) and z_t = sum_{s<=t} psi(k_s) (p^2):
 *   o_t = psi(q_t)^T S_t / psi(q_t)^T z_t
 * (ai.info summary, Methodology in Plain English: a recurrence on a
 * fixed-size state).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout     q, k: [B, H, T, p]; v, o: [B, H, T, dv]; row-major, contiguous.
 *            State S: [B, H, p*p, dv] fp32 with psi index r = i*p + j;
 *            z: [B, H, p*p] fp32.  A state is symmetric in (i, j).
 * Dtypes     q, k, v, o share one dtype: KATA_F32 (fp32) or KATA_BF16
 *            (bfloat16).  Accumulation is fp32.  o is rounded to nearest.
 * Shapes     p in {16, 32}; dv in {16, 64}; B, H >= 1; T >= 0 (T = 0 is a
 *            no-op); C in {64, 128}.  Anything else: KATA_ERR_UNSUPPORTED.
 * Pointers   device pointers, 16-byte aligned (KATA_ERR_MISALIGNED
 *            otherwise); input and output buffers must not overlap.
 * Ownership  the caller owns every buffer; the library never allocates,
 *            frees or retains caller memory.  Workspace is caller-provided.
 * Streams    `stream` is a cudaStream_t passed as void* (NULL = legacy
 *            default stream).  Calls enqueue work and return; they never
 *            synchronise the device.
 * Errors     argument errors are returned before anything is launched;
 *            a failed launch returns KATA_ERR_CUDA.  Waits inside kernels are
 *            bounded: a wait that runs out records KATA_ERR_TIMEOUT in a
 *            device-side status word, the kernel drains its own copies and
 *            returns, and kata_get_status() reports it.  No C++ exception
 *            crosses this boundary.
 * Scaling    no 1/sqrt(p) or temperature factor is applied, and q, k are
 *            used as given (the caller normalises them if wanted).
 * Zero gate  a row whose denominator is exactly 0 (q_t orthogonal to every
 *            key so far) yields o_t = 0.
 */
#ifndef KATA_H_
#define KATA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KATA_OK = 0,
  KATA_ERR_INVALID_ARG = 1,
  KATA_ERR_UNSUPPORTED = 2,
  KATA_ERR_MISALIGNED = 3,
  KATA_ERR_WORKSPACE = 4,
  KATA_ERR_CUDA = 5,
  KATA_ERR_TIMEOUT = 6
} kata_status_t;

typedef enum { KATA_F32 = 0, KATA_BF16 = 1 } kata_dtype_t;

/*
 * Quadratic (flash-style) operating point: o = causal squared-score attention
 * over the whole sequence, O(T^2) work, no state is materialised.
 * (gist.science sec. 2.3, first operating point: a FlashAttention-style
 * kernel that never materialises the full state.)
 *
 * q, k: [B,H,T,p] in; v: [B,H,T,dv] in; o: [B,H,T,dv] out.
 */
kata_status_t kata_fwd_quadratic(const void* q, const void* k, const void* v, void* o,
                                 int B, int H, int T, int p, int dv,
                                 kata_dtype_t dtype, void* stream);

/*
 * Bytes of device workspace kata_fwd_chunked needs for these sizes: 0 when
 * T == 0, and on the tensor-core path (bf16, dv = 64, p = 16 or 32) whenever
 * each (b,h) sequence is handled as a single super-chunk; otherwise one fp32
 * state record per (b,h) per super-chunk (four for p = 32 on the tensor
 * cores).  A pure function of the arguments; the same arguments must be
 * passed to kata_fwd_chunked.  The dtype is an argument because it selects
 * the path and with it the record layout.
 */
size_t kata_fwd_chunked_workspace_size(int B, int H, int T, int p, int dv, int C,
                                       kata_dtype_t dtype);

/*
 * Exact O(T) chunked-state operating point (gist.science sec. 2.3, "Chunked
 * Parallelism" and the second operating point; ai.info Main Findings,
 * "Chunk recurrence avoids the triangular solve"):
 *   1. per-chunk states psi(K_c)^T [V_c | 1], summed over super-chunks of
 *      Ls consecutive tokens,
 *   2. an exclusive associative (parallel prefix) scan of those sums over
 *      the G = ceil(T / Ls) super-chunks of each sequence, depth O(log G)
 *      (gist.science sec. 2.3, "Complexiteitsreductie"),
 *   3. per chunk: intra-chunk squared-score attention plus the readout
 *      psi(Q_c) . S_prefix, then o = numerator / denominator; inside a
 *      super-chunk one CTA (p = 32: one cluster of four) carries the state
 *      from chunk to chunk, Ls/128 steps in sequence.
 * Ls is chosen by the plan (a pure function of the sizes) to fill the GPU:
 * for example Ls = 2048 (G = 1) at B = 8, H = 16, T = 2048 and Ls = 14592
 * (G = 9, 114 steps per CTA) at B = 1, H = 16, T = 131072, both p = 16.
 * Steps 1 and 3 run on the tensor cores (tcgen05) for bf16 inputs with
 * dv = 64 and p = 16 or 32 (p = 32 splits the packed state over four CTAs);
 * fp32 inputs, and bf16 with dv = 16, run the same three steps on the CUDA
 * cores in exact fp32 arithmetic.
 * The result equals kata_fwd_quadratic's up to rounding; C is the chunk
 * length and changes rounding only.
 *
 * S0, z0     optional state before token 1 ([B,H,p*p,dv], [B,H,p*p] fp32);
 *            both NULL means a zero state; exactly one NULL is an error.
 * S_out,z_out optional state after token T (same layouts); both or neither.
 * workspace  device buffer of at least kata_fwd_chunked_workspace_size()
 *            bytes, 256-byte aligned; contents on entry are ignored.  When
 *            that size is 0 (every sequence fits one super-chunk of the
 *            plan, the normal case for short sequences on the tensor-core
 *            path) workspace may be NULL and workspace_bytes 0.
 */
kata_status_t kata_fwd_chunked(const void* q, const void* k, const void* v, void* o,
                               int B, int H, int T, int p, int dv, int C,
                               kata_dtype_t dtype,
                               const float* S0, const float* z0,
                               float* S_out, float* z_out,
                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * kata_fwd_chunked without a caller-provided workspace.  The pages have no
 * counterpart of this call; it exists for callers that cannot allocate
 * device memory themselves (for example a C host program with no allocator
 * of its own, or a loop whose rules forbid cudaMalloc because it can block
 * and synchronise the device).
 *
 * Arguments, layouts, results and errors are those of kata_fwd_chunked.
 * The scratch space lives in one library-owned device array of
 * KATA_NOALLOC_SCRATCH_BYTES (16 MiB) that every GPU which loads the library
 * holds until the process exits; sizes whose
 * kata_fwd_chunked_workspace_size() exceeds it return KATA_ERR_WORKSPACE,
 * after the argument checks of kata_fwd_chunked.  The call allocates nothing.
 * All calls share that array: calls that overlap on the GPU race on it and
 * must be serialised by the caller.  The first call on a device looks up the
 * array's device address (with that device current), and looks it up again
 * when the calling thread's CUDA context has changed since (a device reset);
 * make that first call before any stream capture.
 */
#define KATA_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
kata_status_t kata_fwd_chunked_noalloc(const void* q, const void* k, const void* v, void* o,
                                       int B, int H, int T, int p, int dv, int C,
                                       kata_dtype_t dtype,
                                       const float* S0, const float* z0,
                                       float* S_out, float* z_out, void* stream);

/*
 * Sequential inter-chunk baseline: the chunked forward with every (b,h)
 * sequence handled by one CTA that walks all of its chunks in order,
 * carrying the state from chunk to chunk (a depth-O(T/C) recurrence), with
 * no super-chunk sums and no associative scan.  It exists to measure what
 * the scan of kata_fwd_chunked buys (the pages compare their scan against a
 * sequential linear-attention baseline: gist.science sec. 2.3; KATA
 * repository README, Figure 3).  Results equal kata_fwd_chunked's up to
 * rounding.
 *
 * Arguments, layouts and errors as kata_fwd_chunked, without a workspace.
 * Only the tensor-core configuration (bf16, p = 16, dv = 64) is supported;
 * other sizes return KATA_ERR_UNSUPPORTED.
 */
kata_status_t kata_fwd_chunked_sequential(const void* q, const void* k, const void* v, void* o,
                                          int B, int H, int T, int p, int dv, int C,
                                          kata_dtype_t dtype,
                                          const float* S0, const float* z0,
                                          float* S_out, float* z_out, void* stream);

/*
 * First-order (linear) attention, the feature psi(u) = u: the comparator of
 * the pages' scan claim ("an associative scan of the first-order feature
 * lowers the inter-chunk recurrence depth to O(log(T/C)) and averages ~2.4x
 * the throughput of a matched sequential linear-attention baseline": arXiv
 * abstract; review page, Figure 3 caption; gist.science sec. 2.3).  For
 * every (b,h) and t:
 *   o_t = sum_{s<=t} (q_t . k_s) v_s / sum_{s<=t} (q_t . k_s),
 * o_t = 0 where the denominator is exactly 0 (it may be negative: the
 * feature is not sign-constrained).  State: S = S0 + sum_s k_s v_s^T
 * [d, dv] and z = z0 + sum_s k_s [d].
 *
 * kata_fwd_linear_chunked is the chunked form with the associative scan
 * across super-chunks (state build, scan, readout, as kata_fwd_chunked);
 * kata_fwd_linear_chunked_sequential is the matched sequential baseline: one
 * CTA per (b,h) walks all chunks in order, no workspace.  Both run on the
 * tensor cores and agree up to rounding.
 *
 * q, k: [B, H, T, d]; v, o: [B, H, T, dv]; bf16, row-major, 16-byte aligned.
 * S0/z0 (optional, both or neither) and S_out/z_out (optional, both or
 * neither): fp32 [B, H, d, dv] / [B, H, d], 16-byte aligned; S_out/z_out
 * receive the state after token T.  Only d = 16, dv = 64 and
 * KATA_BF16 are supported (others: KATA_ERR_UNSUPPORTED); C is 64 or 128.
 * workspace: device memory of at least
 * kata_fwd_linear_chunked_workspace_size() bytes, 256-byte aligned
 * (KATA_ERR_WORKSPACE / KATA_ERR_MISALIGNED otherwise; 0 bytes when the
 * whole sequence fits one super-chunk).  All pointers are owned by the
 * caller; the calls are asynchronous on `stream`.
 */
size_t kata_fwd_linear_chunked_workspace_size(int B, int H, int T, int d, int dv, int C);
kata_status_t kata_fwd_linear_chunked(const void* q, const void* k, const void* v, void* o,
                                      int B, int H, int T, int d, int dv, int C,
                                      kata_dtype_t dtype,
                                      const float* S0, const float* z0,
                                      float* S_out, float* z_out,
                                      void* workspace, size_t workspace_bytes, void* stream);
kata_status_t kata_fwd_linear_chunked_sequential(const void* q, const void* k, const void* v, void* o,
                                                 int B, int H, int T, int d, int dv, int C,
                                                 kata_dtype_t dtype,
                                                 const float* S0, const float* z0,
                                                 float* S_out, float* z_out, void* stream);

/*
 * One recurrent decode step for B*H independent streams (constant-time
 * recurrent inference on the fixed-size state; arXiv abstract on aiqbench):
 *   S <- S + psi(k) v^T,  z <- z + psi(k),  o = psi(q)^T S / psi(q)^T z
 * The update comes first, so the current token is included (the same causal
 * convention as the forward entry points).
 *
 * q, k: [B,H,p]; v, o: [B,H,dv] (dtype); S: [B,H,p*p,dv] and z: [B,H,p*p]
 * fp32, read and updated in place.
 */
kata_status_t kata_decode_step(const void* q, const void* k, const void* v, void* o,
                               float* S, float* z, int B, int H, int p, int dv,
                               kata_dtype_t dtype, void* stream);

/*
 * Training: the forward that also saves each row's denominator, and the
 * backward pass (the chain rule through o = N / D with w = (q.k)^2; the
 * pages print no backward pass).  bf16 only, p in {16, 32}, dv = 64, the
 * [B,H,T,*] layouts above; other shapes or fp32: KATA_ERR_UNSUPPORTED.
 *
 * kata_fwd_quadratic_train: as kata_fwd_quadratic, and D: [B,H,T] fp32 out,
 *   D_t = sum_{s<=t} (q_t . k_s)^2.
 * kata_bwd_quadratic: given q, k, v, the forward's o and D, and the upstream
 *   gradient dO ([B,H,T,dv]), writes dq, dk ([B,H,T,p]) and dv ([B,H,T,dv]),
 *   all bf16 (fp32 accumulation).  A row with D_t = 0 (output constant 0)
 *   passes no gradient.  `workspace` (16-byte aligned, at least
 *   kata_bwd_quadratic_workspace_size bytes = 8 per row) holds dO.o and 1/D
 *   per row.
 */
kata_status_t kata_fwd_quadratic_train(const void* q, const void* k, const void* v, void* o, float* D,
                                       int B, int H, int T, int p, int dv,
                                       kata_dtype_t dtype, void* stream);
size_t kata_bwd_quadratic_workspace_size(int B, int H, int T, int p, int dv, kata_dtype_t dtype);
kata_status_t kata_bwd_quadratic(const void* q, const void* k, const void* v, const void* o,
                                 const float* D, const void* dO, void* dq, void* dk, void* dv,
                                 int B, int H, int T, int p, int dv_width, kata_dtype_t dtype,
                                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * Training on the chunked path (bf16, p = 16, dv = 64, [B,H,T,*]): an O(T)
 * forward and backward.  kata_fwd_chunked_train is kata_fwd_chunked (no
 * initial or final state) that also writes each row's denominator D
 * [B,H,T] fp32.  kata_bwd_chunked gives the gradients (dq, dk, dv; layouts
 * of q, k, v; bf16) of the same function as kata_bwd_quadratic, from o, D
 * and dO: the pairs across 128-token chunks through two walks over the
 * chunks of each super-chunk, one carrying the forward state (S before each
 * chunk) for dq, one carrying the gradient state (sum over later tokens of
 * psi(q_t) [dN_t | dD_t]^T) backwards for dk and dv, each entering its
 * super-chunk from a scan of per-super-chunk sums; then the pairs inside each
 * chunk with the flash backward kernels on their diagonal tiles, added to
 * those.  Work and memory are linear in T.  Workspace:
 * kata_bwd_chunked_workspace_size() bytes, 256-byte aligned (8 bytes per row,
 * rounded up to 256, plus, when a sequence is split into G > 1 super-chunks,
 * two 65 x 144 fp32 records per super-chunk of every (b,h)).  Repeated calls
 * give bitwise the same gradients.  Other sizes: KATA_ERR_UNSUPPORTED.
 * Streams and errors as above.
 */
kata_status_t kata_fwd_chunked_train(const void* q, const void* k, const void* v, void* o, float* D,
                                     int B, int H, int T, int p, int dv, int C, kata_dtype_t dtype,
                                     void* workspace, size_t workspace_bytes, void* stream);
size_t kata_bwd_chunked_workspace_size(int B, int H, int T, int p, int dv, kata_dtype_t dtype);
kata_status_t kata_bwd_chunked(const void* q, const void* k, const void* v, const void* o,
                               const float* D, const void* dO, void* dq, void* dk, void* dv,
                               int B, int H, int T, int p, int dv_width, kata_dtype_t dtype,
                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * Training with KATA-Mg ([B,H,T,*] layout, bf16, dv = 64, the (p, groups)
 * of kata_fwd_mg_quadratic with groups > 1): the Mg forward that also saves
 * D [B,H,T] fp32, and its backward pass.  With w = sum_j (q^j . k^j)^2 the
 * gradient of each group's q^j, k^j is the single-factor one taken with the
 * group's own scores and the Mg output's o and D, and dv is the sum over the
 * groups; the backward runs the single-factor kernels once per group on the
 * group's columns (read and written in place) and accumulates dv.  Workspace
 * as kata_bwd_quadratic (8 bytes per row).
 */
kata_status_t kata_fwd_mg_quadratic_train(const void* q, const void* k, const void* v, void* o, float* D,
                                          int B, int H, int T, int d, int groups, int dv,
                                          kata_dtype_t dtype, void* stream);
kata_status_t kata_bwd_mg_quadratic(const void* q, const void* k, const void* v, const void* o,
                                    const float* D, const void* dO, void* dq, void* dk, void* dv,
                                    int B, int H, int T, int d, int groups, int dv_width,
                                    kata_dtype_t dtype, void* workspace, size_t workspace_bytes,
                                    void* stream);

/*
 * KATA-Mg: g PSD factors per head (arXiv abstract and gist.science sec. 2.3
 * "Varianten": several PSD factors; ai.info summary, Main Findings: state
 * d(d/g+1)/2 * dv packed, the full map at g = 1).  The head's d coordinates
 * split into `groups` consecutive groups of width p = d / groups,
 * u = [u^1 | ... | u^g], and the feature is the concatenation of the group
 * maps, psi_Mg(u) = [psi(u^1) | ... | psi(u^g)], so that
 *
 *   w_{t,s} = sum_j (q_t^j . k_s^j)^2,   o_t = sum_{s<=t} w_{t,s} v_s / sum_{s<=t} w_{t,s}
 *
 * with one value vector and one denominator shared by all groups.
 *
 * Layouts of q, k ([.., d]) and v, o ([.., dv]) for the forward call:
 *   KATA_LAYOUT_BHTD  [B, H, T, *] as in the entry points above;
 *   KATA_LAYOUT_BTHD  [B, T, H, *], the layout of the pages' attention call
 *                     (KATA repository README: (B,T,H,D) in and out),
 *                     read and written in place through strided tile copies.
 */
typedef enum { KATA_LAYOUT_BHTD = 0, KATA_LAYOUT_BTHD = 1 } kata_layout_t;

/*
 * Quadratic (flash-style) KATA-Mg forward.  bf16 only; supported
 * (p = d/groups, groups, dv): groups = 1 with p in {16, 32} and dv in
 * {16, 64} (the single-factor kernel of kata_fwd_quadratic), and dv = 64 with
 * (16, 2), (16, 4) or (32, 2).  Other shapes or fp32: KATA_ERR_UNSUPPORTED;
 * groups < 1 or d not a multiple of groups: KATA_ERR_INVALID_ARG.  Pointers,
 * streams, errors and the zero gate as above.
 */
kata_status_t kata_fwd_mg_quadratic(const void* q, const void* k, const void* v, void* o,
                                    int B, int H, int T, int d, int groups, int dv,
                                    kata_layout_t layout, kata_dtype_t dtype, void* stream);

/*
 * Exact O(T) chunked-state KATA-Mg forward (the chunked operating point of
 * kata_fwd_chunked with the concatenated feature psi_Mg): the same
 * arguments as kata_fwd_mg_quadratic plus the chunk length C (64 or 128,
 * rounding only), an optional initial and final state, and a workspace.
 * The state is the concatenation of the groups' states:
 * S [B,H,groups*p*p,dv] and z [B,H,groups*p*p] fp32, row
 * r = j*p*p + a*p + b holding the products of coordinates j*p + a and
 * j*p + b (group j), as for kata_decode_step_mg; S0/z0 and S_out/z_out are
 * both-or-neither, as for kata_fwd_chunked.
 *
 * bf16, dv = 64.  (d, groups) = (64, 4) and (64, 2) run the cluster kernels:
 * each group's packed state in its own CTAs (one for a group of 16, four
 * for a group of 32) with each group's intra-chunk squared scores in the
 * first of them, in either layout.  groups = 1 is kata_fwd_chunked (p = d;
 * [B,T,H,*] only for p = 32).  Other shapes or fp32: KATA_ERR_UNSUPPORTED.
 * workspace: at least kata_fwd_mg_chunked_workspace_size() bytes, 256-byte
 * aligned (NULL when that size is 0).
 */
size_t kata_fwd_mg_chunked_workspace_size(int B, int H, int T, int d, int groups, int dv, int C,
                                          kata_dtype_t dtype);
kata_status_t kata_fwd_mg_chunked(const void* q, const void* k, const void* v, void* o,
                                  int B, int H, int T, int d, int groups, int dv, int C,
                                  kata_layout_t layout, kata_dtype_t dtype,
                                  const float* S0, const float* z0, float* S_out, float* z_out,
                                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * Quadratic (flash-style) KATA-Sigma-g forward: summed PSD factors
 * (gist.science sec. 2.3 "Varianten"; ai.info Main Findings: state
 * (d/g)(d/g+1)/2 * dv).  The feature is the sum of the groups' rank-one maps,
 * psi_S(u) = sum_j vec(u^j u^j^T), so that
 *   w_{t,s} = sum_{j,l} (q_t^j . k_s^l)^2
 * over every pair of a query group and a key group, with one value vector and
 * one denominator.  Arguments, layouts, supported (p, groups, dv) and errors
 * as for kata_fwd_mg_quadratic with groups > 1 (groups = 1 is the single
 * factor: use kata_fwd_mg_quadratic).
 */
kata_status_t kata_fwd_sg_quadratic(const void* q, const void* k, const void* v, void* o,
                                    int B, int H, int T, int d, int groups, int dv,
                                    kata_layout_t layout, kata_dtype_t dtype, void* stream);

/*
 * Training with KATA-Sigma-g ([B,H,T,*] layout, bf16, dv = 64, the
 * (p, groups) of kata_fwd_sg_quadratic with groups > 1): the Sigma-g forward
 * that also saves D [B,H,T] fp32, and its backward pass.  With
 * w = sum_{j,l} (q^j . k^l)^2 the gradient is a sum over the (query group,
 * key group) pairs of the single-factor gradient taken with the pair's
 * scores and the Sigma-g output's o and D: dq^j sums over l, dk^l over j and
 * dv over every pair.  The backward runs the single-factor kernels once per
 * pair on the pair's columns (read and written in place), adding each pass
 * to the rows the earlier passes wrote (in bf16).  Workspace as
 * kata_bwd_quadratic (8 bytes per row).
 */
kata_status_t kata_fwd_sg_quadratic_train(const void* q, const void* k, const void* v, void* o, float* D,
                                          int B, int H, int T, int d, int groups, int dv,
                                          kata_dtype_t dtype, void* stream);
kata_status_t kata_bwd_sg_quadratic(const void* q, const void* k, const void* v, const void* o,
                                    const float* D, const void* dO, void* dq, void* dk, void* dv,
                                    int B, int H, int T, int d, int groups, int dv_width,
                                    kata_dtype_t dtype, void* workspace, size_t workspace_bytes,
                                    void* stream);

/*
 * Exact O(T) chunked-state KATA-Sigma-g forward: the three steps of
 * kata_fwd_chunked on the summed feature psi_S, whose state has the single
 * factor's size: S [B,H,p*p,dv] and z [B,H,p*p] fp32 (p = d/groups), row
 * r = a*p + b holding sum_j u^j_a u^j_b, as for kata_decode_step_sg.
 * q, k: [B,H,T,d]; v, o: [B,H,T,dv] (bf16).  Supported: groups 2 or 4 with
 * p = 16 (d = 32 or 64), dv = 64, bf16; others KATA_ERR_UNSUPPORTED (groups
 * < 1 or d not a multiple of groups: KATA_ERR_INVALID_ARG).  C, S0/z0,
 * S_out/z_out, the workspace (kata_fwd_sg_chunked_workspace_size bytes),
 * streams and errors as for kata_fwd_chunked.
 */
size_t kata_fwd_sg_chunked_workspace_size(int B, int H, int T, int d, int groups, int dv, int C);
kata_status_t kata_fwd_sg_chunked(const void* q, const void* k, const void* v, void* o,
                                  int B, int H, int T, int d, int groups, int dv, int C,
                                  kata_dtype_t dtype,
                                  const float* S0, const float* z0,
                                  float* S_out, float* z_out,
                                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * One KATA-Mg decode step (update with (k, v), then read with q):
 * q, k: [B,H,d]; v, o: [B,H,dv] (fp32 or bf16); S: [B,H,groups*p*p,dv] and
 * z: [B,H,groups*p*p] fp32, read and updated in place, with row
 * r = j*p*p + a*p + b holding the products of coordinates j*p + a and
 * j*p + b (group j).  Supported (p, groups, dv) as for
 * kata_fwd_mg_quadratic, in either dtype.
 */
kata_status_t kata_decode_step_mg(const void* q, const void* k, const void* v, void* o,
                                  float* S, float* z, int B, int H, int d, int groups, int dv,
                                  kata_dtype_t dtype, void* stream);

/*
 * One KATA-Sigma-g decode step (update with (k, v), then read with q) on
 * the summed-feature state: psi_S(u) = sum_j vec(u^j u^j^T), so the state
 * has the single factor's size: S [B,H,p*p,dv] and z [B,H,p*p] fp32
 * (p = d/groups), read and updated in place, row r = a*p + b holding
 * sum_j u^j_a u^j_b.  q, k: [B,H,d]; v, o: [B,H,dv] (fp32 or bf16).
 * Supported (p, groups, dv) as for kata_fwd_sg_quadratic; groups = 1 is
 * kata_decode_step.  Errors as for kata_decode_step_mg.
 */
kata_status_t kata_decode_step_sg(const void* q, const void* k, const void* v, void* o,
                                  float* S, float* z, int B, int H, int d, int groups, int dv,
                                  kata_dtype_t dtype, void* stream);

/*
 * Synchronises `stream`, then returns and clears the device-side status word
 * of the current device (KATA_ERR_TIMEOUT if a bounded wait in a kernel ran
 * out since the last call), or KATA_ERR_CUDA if the stream reports an error.
 */
kata_status_t kata_get_status(void* stream);

/* Static, human-readable name of a status code. */
const char* kata_status_string(kata_status_t status);

/*
 * Upper bound, in SM clock cycles, on every wait inside the library's
 * kernels (default about 2^31, i.e. on the order of a second).  Affects
 * launches made after the call.  Passing 0 makes any wait that is not
 * already satisfied give up at once, which tests use to exercise the timeout
 * path; a negative value restores the default.
 */
void kata_set_wait_limit(long long cycles);

/* ABI version of this header: major * 10000 + minor * 100 + patch. */
int kata_abi_version(void);

#define KATA_ABI_VERSION 10400

#ifdef __cplusplus
}
#endif

#endif /* KATA_H_ */
