/*
 * libtheta -- theta-bundle projections on NVIDIA B200 (sm_100a).
 *
 * A decoder projection weight W [out_dim O, in_dim I] is represented by a
 * theta bundle ("The theta bundle" -- component table and approximation
 * formula):
 *
 *     W  ~  diag(s) . W0[band] + U . V^T
 *
 *   W0 [O, I]  shared block: the mean of the family's weights over a
 *              contiguous band of layers ("Banded sharing");
 *   s  [O]     per-output-row least-squares scale against W0 (fp32 always);
 *   U  [O, r]  left factor of the rank-r residual (absorbs the singular values);
 *   V  [I, r]  right factor (stored [in_dim, rank], not transposed).
 *
 * Conventions for every call
 *   - Matrices are dense, row-major, with no padding: row pitch = columns.
 *     X [M, I], W0 [O, I], U [O, r], V [I, r], Y [M, O].
 *   - Element type: THETA_F32 (fp32 everywhere) or THETA_BF16 (bf16 storage,
 *     fp32 arithmetic and accumulation). s is always fp32.
 *   - "device" pointers point to memory of the current CUDA device; "host"
 *     pointers to host memory. The caller owns every buffer; the library keeps
 *     no pointer after a call returns and allocates no device memory.
 *   - Calls taking a stream are asynchronous: they validate arguments on the
 *     host, enqueue kernels on `stream` (a cudaStream_t; NULL means the legacy
 *     default stream) and return. Errors found on the host are returned before
 *     anything is enqueued; nothing is written in that case.
 *   - THETA_BF16 calls use the Tensor Memory Accelerator and need 16-byte
 *     aligned base pointers and row pitches that are multiples of 16 bytes
 *     (I, O and r multiples of 8); otherwise they return THETA_ERR_ALIGNMENT.
 *   - Kernels bound every wait they make. A wait that runs out records a flag
 *     on the device and the kernel returns early; theta_device_status() reports
 *     it as THETA_ERR_TIMEOUT and clears it. While the flag is set, kernels
 *     with waits skip their work (outputs undefined) so that a fault does not
 *     cost every later CTA its own wait limit.
 *   - theta_last_error() gives a message for the last failing call on the
 *     calling thread.
 */
#ifndef THETA_H
#define THETA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define THETA_VERSION 1
#define THETA_MAX_LAYERS 256 /* layers per call of the band/prelude entry points */
#define THETA_MAX_GROUP 256  /* problems per call of theta_linear_forward_grouped */

typedef enum {
  THETA_OK = 0,
  THETA_ERR_INVALID_ARG = -1, /* bad size, count, pointer or dtype */
  THETA_ERR_UNSUPPORTED = -2, /* valid request this build cannot serve */
  THETA_ERR_ALIGNMENT = -3,   /* TMA alignment rule broken (bf16 paths) */
  THETA_ERR_CUDA = -4,        /* CUDA runtime/driver error; see theta_last_error */
  THETA_ERR_TIMEOUT = -5,     /* a bounded device wait ran out */
  THETA_ERR_WORKSPACE = -6    /* workspace missing or smaller than required */
} theta_status;

typedef enum { THETA_F32 = 0, THETA_BF16 = 1 } theta_dtype;

typedef enum {
  THETA_OP_FROB_ERROR = 0,
  THETA_OP_LINEAR_FORWARD = 1,
  THETA_OP_GATE_UP_FORWARD = 2,
  THETA_OP_RESIDUAL_SVD = 3,
  THETA_OP_NVFP4_QUANTIZE = 4,
  THETA_OP_LINEAR_FORWARD_NVFP4 = 5,
  THETA_OP_LINEAR_FORWARD_GROUPED = 6
} theta_op;

/* How the tensor-core kernels size their grids (see theta_set_policy). */
typedef enum {
  THETA_POLICY_LATENCY = 0,   /* default: split K across a cluster so one call fills the GPU */
  THETA_POLICY_THROUGHPUT = 1 /* one CTA per output tile: many calls run concurrently */
} theta_policy;

/* Library version (THETA_VERSION of the build). */
int theta_version(void);

/* Static name of a status code. */
const char* theta_status_string(int status);

/* Message of the last failing call on this thread ("" if none). The pointer
 * stays valid until the next libtheta call on the same thread. */
const char* theta_last_error(void);

/*
 * theta_band_index -- layer-to-band map ("Banded sharing" -- How layers map
 * to bands): num_layers layers form G contiguous bands, as equal in size as
 * possible, the earlier bands taking the remainder. With q = num_layers / G
 * and m = num_layers % G, band b has q + 1 layers if b < m, else q.
 *
 *   band_of_layer  host int32[num_layers], written: band of each layer.
 *   band_start     host int32[G + 1] or NULL, written: first layer of each
 *                  band, band_start[G] = num_layers.
 * Synchronous and host-only (no CUDA call). Returns THETA_ERR_INVALID_ARG
 * unless 1 <= G <= num_layers and band_of_layer is non-NULL.
 */
int theta_band_index(int num_layers, int G, int32_t* band_of_layer, int32_t* band_start);

/*
 * theta_band_mean -- shared block of one band ("The theta bundle" --
 * Analytic decomposition, Shared block): W0 = (1/n) sum_l W_l over the n
 * given layers. Accumulates in fp32 in layer order, divides once by n and
 * rounds once to dt.
 *
 *   weights  host array of n device pointers, each [O, I] of dt.
 *   W0       device [O, I] of dt, written.
 * 1 <= n <= THETA_MAX_LAYERS; O, I >= 1.
 */
int theta_band_mean(const void* const* weights, int n, int64_t O, int64_t I, theta_dtype dt,
                    void* W0, void* stream);

/*
 * theta_row_scale -- per-row least-squares scale ("The theta bundle" --
 * Per-row scale): s[o] = <W[o,:], W0[o,:]> / <W0[o,:], W0[o,:]>, both dot
 * products in fp32 with the same summation order (so W == W0 gives s == 1
 * exactly). A row with <W0,W0> == 0 gets s = 0.
 *
 *   weight device [O, I] of dt;  W0 device [O, I] of dt;  s device fp32 [O], written.
 */
int theta_row_scale(const void* weight, const void* W0, int64_t O, int64_t I, theta_dtype dt,
                    float* s, void* stream);

/*
 * theta_residual -- residual of the scaled shared block ("The theta bundle" --
 * Low-rank residual): R = W - diag(s) . W0, each element computed as one
 * fused multiply-add fmaf(-s[o], W0[o,i], W[o,i]) and rounded once to dt.
 *
 *   weight, W0  device [O, I] of dt;  s device fp32 [O];  R device [O, I] of dt, written.
 */
int theta_residual(const void* weight, const void* W0, const float* s, int64_t O, int64_t I,
                   theta_dtype dt, void* R, void* stream);

/*
 * theta_decompose_prelude -- the analytic decomposition of one projection
 * family up to the truncated SVD ("The theta bundle" -- Analytic
 * decomposition; "Banded sharing" for the bands): for each of the G bands of
 * num_layers layers, W0[b] = band mean; then for every layer l of band b,
 * s[l] = row scale of W_l against the stored W0[b] and, if residual is
 * non-NULL, residual[l] = W_l - diag(s[l]) . W0[b]. Same arithmetic as the
 * three calls above; the row scale and residual of a band's layers run in
 * one pass that reads each W0[b] row once.
 *
 *   weights   host array of num_layers device pointers, each [O, I] of dt.
 *   W0        host array of G device pointers, each [O, I] of dt, written.
 *   s         host array of num_layers device pointers, each fp32 [O], written.
 *   residual  host array of num_layers device pointers ([O, I] of dt, written),
 *             or NULL to skip the residual.
 * 1 <= G <= num_layers <= THETA_MAX_LAYERS.
 */
int theta_decompose_prelude(const void* const* weights, int num_layers, int G, int64_t O,
                            int64_t I, theta_dtype dt, void* const* W0, float* const* s,
                            void* const* residual, void* stream);

/*
 * theta_residual_svd -- rank-r factors of a residual, U . V^T ~ R, with U
 * absorbing the singular values ("The theta bundle" -- Low-rank residual:
 * a randomized SVD, Halko et al., for large matrices). Steps: range sample
 * Y = R . omega^T; orthonormal basis Q of Y (shifted Cholesky QR, then two
 * plain passes); power_iters rounds of subspace iteration; B = Q^T . R; the
 * eigen-decomposition of B . B^T (Jacobi, fp64) gives B's singular vectors;
 * U = Q . E_r . diag(sigma), V = B^T . E_r . diag(1 / sigma).
 *
 *   R [O, I] (dt); omega fp32 [samples, I], the Gaussian test matrix (the
 *   caller draws it; samples = rank + oversampling); U [O, rank] and
 *   V [I, rank] (dt), written. 1 <= rank <= samples <= min(96, O, I);
 *   0 <= power_iters <= 8; O, I <= 4,194,240 (larger: THETA_ERR_UNSUPPORTED).
 *   workspace  device scratch of theta_workspace_size(THETA_OP_RESIDUAL_SVD,
 *              samples, O, I, rank, dt) bytes (M carries samples).
 * fp32 arithmetic (fp64 for the k x k steps): decomposition work, not the
 * projection's hot path. For a bf16 R with I a multiple of 8 and R 16-byte
 * aligned, the products that stream R (R . omega^T, Q^T . R, R . Z) run on
 * tensor cores with the fp32 factor split exactly into three bf16 parts
 * (sums of the exact products of the fp32 operands, in another order than
 * an fp32 GEMM); every other product, and every product of an fp32 R, runs
 * on CUDA cores. A direction the sample lacks (R of rank below samples)
 * comes out as a zero column of U and V.
 */
int theta_residual_svd(const void* R, int64_t O, int64_t I, theta_dtype dt, int rank, int samples,
                       int power_iters, const float* omega, void* U, void* V, void* workspace,
                       size_t workspace_bytes, void* stream);

/*
 * theta_reconstruct -- reconstruct_weight(s, W0, U, V) = diag(s) . W0 + U . V^T
 * ("The theta bundle" -- approximation formula; reconstruct_weight). fp32
 * accumulation over the rank, one rounding to dt. rank == 0 leaves only the
 * scaled shared block diag(s).W0 and allows U = V = NULL.
 *
 *   s fp32 [O]; W0 [O, I]; U [O, rank]; V [I, rank]; W_out [O, I], written.
 *   All device pointers, dt elements except s.
 */
int theta_reconstruct(const float* s, const void* W0, const void* U, const void* V, int64_t O,
                      int64_t I, int rank, theta_dtype dt, void* W_out, void* stream);

/*
 * theta_reconstruct_band -- theta_reconstruct for the n layers of one band,
 * which share one W0 ("Banded sharing"; "The theta bundle" -- the
 * approximation formula): W_out[l] = diag(s[l]) . W0 + U[l] . V[l]^T.
 *
 *   s, U, V, W_out  host arrays of n device pointers (one per layer), each as
 *                   in theta_reconstruct; U and V may be NULL when rank == 0.
 *   W0       device [O, I], the band's shared block.
 *   1 <= n <= THETA_MAX_LAYERS; other rules as theta_reconstruct.
 * Every output is element for element what theta_reconstruct gives for that
 * layer; the bf16 path reads each 128 x 128 tile of W0 once for all the
 * layers (up to 64 layers per launch, rank <= 128; otherwise one
 * theta_reconstruct per layer), fp32 runs theta_reconstruct per layer.
 */
int theta_reconstruct_band(const float* const* s, const void* W0, const void* const* U, const void* const* V, int n,
                           int64_t O, int64_t I, int rank, theta_dtype dt, void* const* W_out, void* stream);

/*
 * theta_frob_error -- relative_frobenius_error(original, reconstructed)
 * = ||A - B||_F / ||A||_F ("Quality" -- Reconstruction error; "The theta
 * bundle" -- relative_frobenius_error). 0 if both norms are 0, +inf if only
 * ||A|| is. Squares are summed in fp32 over 8-element groups and in fp64
 * beyond; the two-stage reduction has a fixed order (deterministic).
 *
 *   original, reconstructed  device [n] of dt (any shape, flattened).
 *   out        device double[1], written.
 *   workspace  device scratch of at least theta_workspace_size(THETA_OP_FROB_ERROR)
 *              bytes, 16-byte aligned; its contents are overwritten.
 */
int theta_frob_error(const void* original, const void* reconstructed, int64_t n, theta_dtype dt,
                     double* out, void* workspace, size_t workspace_bytes, void* stream);

/*
 * theta_frob_partials -- the two sums behind relative_frobenius_error
 * ("Quality" -- Reconstruction error): out[0] = sum (A - B)^2 and
 * out[1] = sum A^2, with the same kernels, order and precision as
 * theta_frob_error. Both are plain sums, so when the rows of a matrix are
 * split across GPUs (every quantity of "The theta bundle" component table is
 * per output row) each GPU takes the sums of its rows, one all-reduce adds
 * them, and sqrt(out[0]) / sqrt(out[1]) is the error of the whole matrix.
 *
 *   original, reconstructed  device [n] of dt (any shape, flattened).
 *   out        device double[2], 8-byte aligned, written.
 *   workspace  as for theta_frob_error (THETA_OP_FROB_ERROR).
 */
int theta_frob_partials(const void* original, const void* reconstructed, int64_t n, theta_dtype dt,
                        double* out, void* workspace, size_t workspace_bytes, void* stream);

/*
 * theta_linear_forward -- the projection by the rebuilt weight without
 * forming it:  Y = X . (diag(s) . W0 + U . V^T)^T = s (.) (X . W0^T) + (X . V) . U^T
 * (identity from "The theta bundle" approximation formula).
 *
 *   X [M, I]; W0 [O, I] (the band's shared block); s fp32 [O]; U [O, rank];
 *   V [I, rank]; Y [M, O], written. Device pointers, dt elements except s.
 *   workspace  device scratch of theta_workspace_size(THETA_OP_LINEAR_FORWARD)
 *              bytes (holds T = X . V); may be NULL when that size is 0.
 * THETA_BF16: tensor cores (tcgen05) with fp32 accumulation in tensor memory;
 * T = X.V is kept as a bf16 high part plus a bf16 low part, so the rank-r term
 * carries about 16 significand bits. One or two tokens on a W0 of at most 32M
 * elements take a CUDA-core sweep instead (fp32 accumulation, T in fp32).
 * Grid sizing follows theta_set_policy. THETA_F32: fp32 CUDA cores
 * throughout. rank == 0 allows U = V = NULL.
 */
int theta_linear_forward(const void* X, int64_t M, int64_t I, const void* W0, int64_t O,
                         const float* s, const void* U, const void* V, int rank, theta_dtype dt,
                         void* Y, void* workspace, size_t workspace_bytes, void* stream);

/*
 * theta_linear_gate_up_forward -- an MLP's gate and up projections of one
 * layer, fused:  Y = gelu_tanh(G) (.) P  with
 *   G = s_gate (.) (X . W0_gate^T) + (X . V_gate) . U_gate^T   (the gate projection)
 *   P = s_up   (.) (X . W0_up^T)   + (X . V_up)   . U_up^T     (the up projection)
 *   gelu_tanh(x) = 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))),
 * the activation the Gemma models name in their config ("Quality" --
 * Native-equivalent at passthrough: the MLP takes its activation from the
 * config, gelu_tanh for Gemma 3 and 4; the fused MLP of "Quality" -- What
 * quantizing attention costs). Each weight is rebuilt as in
 * theta_linear_forward and never formed; G and P stay in fp32 until the
 * product is rounded once to bf16.
 *
 *   X [M, I]; W0_gate, W0_up [O, I]; s_gate, s_up fp32 [O]; U_gate, U_up
 *   [O, rank]; V_gate, V_up [I, rank]; Y [M, O], written. The two
 *   projections share O, I and rank.
 *   workspace  device scratch of theta_workspace_size(THETA_OP_GATE_UP_FORWARD)
 *              bytes (both T = X . V), NULL when that size is 0 (rank 0).
 * THETA_BF16 only (THETA_ERR_UNSUPPORTED otherwise): one tensor-core kernel
 * streams both W0 tiles against each X tile it loads, with four accumulators
 * in tensor memory (gate and up, main and rank terms) and the activation in
 * its epilogue. Same alignment rules and policy as theta_linear_forward.
 */
int theta_linear_gate_up_forward(const void* X, int64_t M, int64_t I, int64_t O, int rank, theta_dtype dt,
                                 const void* W0_gate, const float* s_gate, const void* U_gate,
                                 const void* V_gate, const void* W0_up, const float* s_up, const void* U_up,
                                 const void* V_up, void* Y, void* workspace, size_t workspace_bytes,
                                 void* stream);

/*
 * theta_nvfp4_quantize -- encodes a shared block W0 in NVFP4, the 4-bit
 * weight format the pages measure ("Quality" -- What NVFP4 quantization
 * costs: 3.18x smaller weights), at 0.5625 bytes per weight: E2M1 elements,
 * one FP8 E4M3 scale per 16 consecutive elements of a row, one FP32 scale per
 * tensor. Every decision in fp32, round-to-nearest-even, saturating:
 *   g = amax|W0| / (6 * 448); per block: sq = E4M3(max|w| / 6 / g);
 *   code = E2M1(w * (1 / (E4M3value(sq) * g))) with the sign of w (+0 for a
 *   value that rounds to zero). The weight it stands for: E2M1 * E4M3 * g.
 *
 *   W0 [O, I] bf16 (I a multiple of 32, 16-byte aligned); codes uint8
 *   [O, I/2] (element 2j in the low nibble of byte j; 16-byte aligned); scales
 *   uint8 [O, I/16] (E4M3 codes; 2-byte aligned); g: device fp32 scalar,
 *   written. workspace: 16 bytes (theta_workspace_size(THETA_OP_NVFP4_QUANTIZE)).
 */
int theta_nvfp4_quantize(const void* W0, int64_t O, int64_t I, void* codes, void* scales, float* g,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * One problem of theta_linear_forward_grouped: the arguments of one bf16
 * theta_linear_forward call (the token count M is shared by the group).
 * 72 bytes, natural alignment; the field order is the ABI.
 */
typedef struct theta_forward_problem {
  const void* X;   /* [M, I] bf16 */
  const void* W0;  /* [O, I] bf16 */
  const float* s;  /* [O] fp32 */
  const void* U;   /* [O, rank] bf16; NULL when rank == 0 */
  const void* V;   /* [I, rank] bf16; NULL when rank == 0 */
  void* Y;         /* [M, O] bf16, written */
  int64_t O;
  int64_t I;
  int64_t rank;
} theta_forward_problem;

/*
 * theta_linear_forward_grouped -- `count` independent bf16 theta forwards of
 * the same one or two tokens count, in one call ("The theta bundle" --
 * approximation formula, applied to every projection of every layer: the
 * decode step of a whole model, whose per-call latency dominates at small
 * sizes). Each Y is what theta_linear_forward would write, up to fp32
 * summation order. Three launches for the whole group: T = X.V of every
 * problem (8 slices of I each), their fixed-order sums, and one CUDA-core
 * sweep over the rows of all problems laid end to end.
 *   problems         host array of `count` descriptors (read during the call
 *                    only: sizes, validation)
 *   problems_device  device copy of the same array (the kernels read it);
 *                    the caller keeps it alive and unchanged until the work
 *                    has run. The two must hold the same contents.
 *   1 <= count <= THETA_MAX_GROUP; 1 <= M <= 2 (else THETA_ERR_UNSUPPORTED).
 *   Per problem: O, I >= 1, 0 <= rank <= 256; I, O, rank multiples of 8 and
 *   X, W0, s, U, V 16-byte aligned (else THETA_ERR_ALIGNMENT).
 *   workspace: theta_workspace_size(THETA_OP_LINEAR_FORWARD_GROUPED, M,
 *   count, 0, max rank over the problems, THETA_BF16) bytes (0 when every
 *   rank is 0).
 */
int theta_linear_forward_grouped(const theta_forward_problem* problems, const theta_forward_problem* problems_device,
                                 int count, int64_t M, void* workspace, size_t workspace_bytes, void* stream);

/*
 * theta_linear_forward_nvfp4 -- theta_linear_forward with the shared block
 * given in NVFP4 (from theta_nvfp4_quantize): Y = s (.) (X . W0q^T) +
 * (X . V) . U^T with W0q the dequantized block, for one or two tokens --
 * the decode case, where the HBM bytes of W0 set the time and NVFP4 cuts
 * them 3.56x. A CUDA-core sweep: each CTA first writes X into shared
 * memory in fp16, scaled by a power of two per group of 1024 values so that
 * |x| <= 2^9 (no block sum can leave fp16's range); each pair of codes is
 * widened to f16x2 by the Blackwell E2M1 conversion; a block's 16 products
 * are summed by packed fp16 FMAs, scaled in fp32 by its E4M3 scale and the
 * group's power of two, and the row sum multiplied by g.
 *   X [M, I], U [O, rank], V [I, rank], Y [M, O] bf16; s fp32 [O]; codes,
 *   scales, g as written by theta_nvfp4_quantize. M <= 2 (else
 *   THETA_ERR_UNSUPPORTED); I a multiple of 32 with M * ceil(I / 1024) <= 99
 *   (X in fp16 must fit in shared memory: I <= 101376 for one token, 50176
 *   for two; else THETA_ERR_UNSUPPORTED); O, rank multiples of 8.
 *   workspace: theta_workspace_size(THETA_OP_LINEAR_FORWARD_NVFP4, M, O, I,
 *   rank, THETA_BF16) bytes (the partial sums of T = X.V; 0 at rank 0).
 */
int theta_linear_forward_nvfp4(const void* X, int64_t M, int64_t I, const void* codes, const void* scales,
                               const float* g, int64_t O, const float* s, const void* U, const void* V, int rank,
                               void* Y, void* workspace, size_t workspace_bytes, void* stream);

/*
 * theta_linear_forward_noalloc -- theta_linear_forward for callers that
 * cannot allocate device memory. (A library convenience: the pages describe
 * no counterpart.)
 *
 * Same arguments, arithmetic, kernels and result as theta_linear_forward,
 * minus the workspace: its scratch (T = X.V) lives in a 4 MiB array built
 * into the library. It is meant for code that must not call cudaMalloc:
 * serving engines whose device memory is all owned by their own fixed pool,
 * with nothing left over for a library, and plugins that are handed only
 * their input and output buffers.
 *
 *   - Capacity: the call needs theta_workspace_size(THETA_OP_LINEAR_FORWARD)
 *     bytes, at most 4 MiB (about M * rank <= 1,048,576). Larger requests
 *     return THETA_ERR_WORKSPACE before anything is enqueued.
 *   - Memory: every GPU that loads the library holds the 4 MiB array until
 *     the process exits. This entry point itself allocates nothing.
 *   - Sharing: all calls on a device use the same array. Calls ordered on one
 *     stream are safe; calls whose kernels may overlap on the GPU (different
 *     streams without ordering between them) race on it and must not be made.
 *     Each call writes the scratch it reads, so leftovers from an earlier call
 *     do not matter.
 *   - Set-up: the first call on each device looks up the array's device
 *     address (cudaGetSymbolAddress, with that device current). Make that
 *     first call before any stream capture begins.
 */
int theta_linear_forward_noalloc(const void* X, int64_t M, int64_t I, const void* W0, int64_t O,
                                 const float* s, const void* U, const void* V, int rank,
                                 theta_dtype dt, void* Y, void* stream);

/*
 * theta_workspace_size -- device scratch bytes a call needs (0 if none).
 * op is a theta_op; the sizes are those the call will receive (unused ones
 * are ignored). Writes *bytes.
 */
int theta_workspace_size(int op, int64_t M, int64_t O, int64_t I, int rank, theta_dtype dt,
                         size_t* bytes);

/*
 * theta_set_policy -- grid sizing of the tensor-core kernels of
 * theta_linear_forward (the T = X.V kernel and the main projection) for the
 * calls that follow, process-wide. Not an operation of the method: a launch
 * choice that does not change any result beyond floating-point summation
 * order.
 *   THETA_POLICY_LATENCY (default): when the output tiles of one call leave
 *     SMs idle, K is split over a thread-block cluster and the partial tiles
 *     are summed through distributed shared memory -- the fastest single call.
 *   THETA_POLICY_THROUGHPUT: no split of the main projection; every CTA
 *     owns a whole output tile. For callers that keep the GPU busy with many
 *     independent calls on several streams, where split-K's extra CTAs,
 *     cluster scheduling and reductions cost more than they gain. (The small
 *     T = X.V kernel in front of it splits K under both policies.)
 * Returns THETA_ERR_INVALID_ARG for any other value. Safe to call from any
 * thread; calls already enqueued keep the policy they were launched with.
 * theta_get_policy returns the current policy.
 */
int theta_set_policy(int policy);
int theta_get_policy(void);

/*
 * theta_selftest_wait_timeout -- exercises the failure path of the bounded
 * device waits (not an operation of the method): enqueues one kernel whose
 * wait on a barrier that nothing completes gives up after limit_ms
 * milliseconds (1..2000) and records the timeout flag, exactly as a kernel
 * whose producer stopped would. The next theta_device_status() on `stream`
 * returns THETA_ERR_TIMEOUT and clears the flag; the CUDA context stays
 * usable. Returns THETA_ERR_INVALID_ARG for a limit outside the range.
 */
int theta_selftest_wait_timeout(unsigned limit_ms, void* stream);

/*
 * theta_device_status -- synchronises `stream`, then reads and clears the
 * current device's error flags. Returns THETA_ERR_TIMEOUT if a kernel's
 * bounded wait ran out since the last check, THETA_ERR_CUDA on a CUDA error,
 * else THETA_OK.
 */
int theta_device_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* THETA_H */
