/*
 * kronq.h -- C ABI of libkronq.so, KronQ's per-layer quantization pass on
 * NVIDIA B200 (sm_100a).
 *
 * The pass (KronQ README intro; KronQ arXiv abstract):
 *   1. accumulate the Kronecker factors of the layer Hessian H ~ H_X (x) H_G,
 *      H_X = sum x x^T over calibration inputs, H_G = sum g g^T over output
 *      gradients                                   -> kronq_accumulate_factors
 *   2. the inter-layer sensitivity tr(H_G) * tr(H_X) -> kronq_sensitivity,
 *      and the bit allocation it drives            -> kronq_allocate_bits*
 *   3. bidirectional incoherence processing (BiIP): rescale + randomized
 *      Hadamard rotation on the input and output side -> kronq_biip_forward,
 *      and its inverse for unrotated export          -> kronq_biip_inverse
 *   4. GPTQ-style blocked column quantization under the K-FAC loss with the
 *      Cholesky factor of the damped inverse H_X, lazy-batch error feedback
 *      and per-group scales at 2/3/4 bits           -> kronq_quantize_layer
 *   5. packed int4/int2 storage (KronQ README "Model zoo") -> kronq_pack
 *
 * Around the pass:
 *   - the Kronecker factor estimators of the "WaterKron and FlipFlop
 *     Hessian" page, Table 1 (input, marginal, Frobenius, FlipFlop)
 *                                                    -> kronq_kron_factors
 *   - the deploy path's matvec from packed codes (KronQ README intro: fused
 *     dequant + BiIP matvec for single-token decode) -> kronq_decode_matvec
 *   - two-sided rounding that uses H_G inside the sweep ("BaKron" abstract:
 *     GPTQ on vec(W) under H_X (x) H_G)            -> kronq_quantize_two_sided
 *
 * Conventions (all calls):
 *   - Matrices are row-major.  W is m x n (out x in), X is T x n, G is T x m.
 *   - Every array argument is DEVICE memory owned by the caller, except where
 *     a comment says "host".  The library allocates no memory: scratch comes
 *     from the caller's workspace (query its size with *_workspace_bytes).
 *   - Calls are asynchronous on the given stream, except kronq_sensitivity
 *     and kronq_device_status, which synchronise that stream.
 *   - Arguments are checked on the host before anything is launched; a bad
 *     argument returns KRONQ_ERR_INVALID_ARG (or KRONQ_ERR_UNSUPPORTED for a
 *     valid but unimplemented combination) and touches no memory.
 *   - A failure inside a kernel never traps: non-positive-definite factors
 *     are reported through *info (LAPACK convention), and any bounded wait
 *     that gives up records KRONQ_ERR_TIMEOUT in the library's device status
 *     word (read it with kronq_device_status).
 *   - kronq_last_error() returns a thread-local message for the last non-OK
 *     status returned on the calling thread.
 */
#ifndef KRONQ_H
#define KRONQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream handle (cudaStream_t / CUstream); NULL is the legacy default stream. */
typedef struct CUstream_st* kronq_stream_t;

typedef enum {
  KRONQ_OK = 0,
  KRONQ_ERR_INVALID_ARG = 1,
  KRONQ_ERR_UNSUPPORTED = 2,
  KRONQ_ERR_CUDA = 3,
  KRONQ_ERR_NOT_PD = 4,
  KRONQ_ERR_TIMEOUT = 5
} kronq_status;

typedef enum { KRONQ_BF16 = 0, KRONQ_F32 = 1 } kronq_dtype;

/* BiIP ablation modes (KronQ README, "Mapping paper results to flags":
 * --incoh_mode {full,no_rescale,su_only,sv_only}).  SU is the output-side
 * (left, m) transform, SV the input-side (right, n) transform. */
typedef enum {
  KRONQ_BIIP_FULL = 0,       /* rescale + rotation on both sides          */
  KRONQ_BIIP_NO_RESCALE = 1, /* rotation on both sides, no rescale        */
  KRONQ_BIIP_SU_ONLY = 2,    /* output side only (U, D_out)               */
  KRONQ_BIIP_SV_ONLY = 3     /* input side only (V, D_in)                 */
} kronq_biip_mode;

/* kronq_quant_params.flags */
#define KRONQ_U_GIVEN      1u /* HX already holds U (upper): skip dead columns, damping, factorisation */
#define KRONQ_ORDERED_FP32 2u /* fixed-order float32 trailing update (bit-exact test mode)             */
#define KRONQ_WRITE_E      4u /* keep the scaled error E (m x n) in the E argument                      */
#define KRONQ_R_FORM       8u /* sweep on R itself (H~ = R R^T); U = R^-1 is never formed               */

/* Quantizer settings (KronQ README, "Reproduce from scratch":
 * --w_bits --w_groupsize --w_asym).
 *   bits     2, 3 or 4.
 *   group    -1 (one group per row) or g > 0 with block % g == 0 or
 *            g % block == 0; a ragged last group is allowed.
 *   asym     1: asymmetric grid, zero = rint(-min/scale); 0: symmetric.
 *   damp_rel damping lambda = damp_rel * mean(diag H~_X) (0.01 typical).
 *   block    lazy-batch width; 128 is the only value implemented.
 *   flags    KRONQ_* flags above. */
typedef struct {
  int bits;
  int group;
  int asym;
  float damp_rel;
  int block;
  unsigned flags;
} kronq_quant_params;

/* ---------------------------------------------------------------------------
 * Step 1 -- factor accumulation.  KronQ README intro (H ~ H_X (x) H_G);
 * "WaterKron and FlipFlop Hessian", Table 1, "Marginal" row (A = E[x x^T],
 * B = E[g g^T]); read here as sums over tokens, not means.
 *
 *   H (d x d, float32, row-major, full symmetric storage) += A^T A
 *   A     T x d token rows, row stride lda elements (lda >= d), dtype dt.
 *         KRONQ_BF16 runs on the tcgen05 tensor cores (bf16 x bf16 -> fp32);
 *         it needs A 16-byte aligned and lda % 8 == 0.  KRONQ_F32 runs an
 *         exact-fp32 SIMT kernel (small layers).
 *   zero_first  nonzero: H is overwritten with A^T A instead of added to.
 *   Call once per token chunk to stream T (pass zero_first only first).
 *   Both triangles of H are kept equal; when adding, H must be symmetric on
 *   input (as every call leaves it): from d = 2048 on only its upper
 *   triangle is read.  T == 0 is allowed (no-op, or a zero fill when
 *   zero_first).
 * ------------------------------------------------------------------------- */
kronq_status kronq_accumulate_factors(const void* A, kronq_dtype dt, int64_t T, int64_t d,
                                      int64_t lda, float* H, int zero_first, kronq_stream_t s);

/* ---------------------------------------------------------------------------
 * Step 2 -- sensitivity.  KronQ abstract point (2); README bullet
 * "Inter-layer mixed precision": s = tr(H_G) * tr(H_X).
 *   HX n x n, HG m x m (device, float32).  out3 (HOST, 3 doubles) receives
 *   { tr(H_X), tr(H_G), tr(H_G) * tr(H_X) }, diagonals summed in float64.
 *   workspace: >= 16 bytes of device memory, 8-byte aligned.
 *   Synchronises the stream.
 * ------------------------------------------------------------------------- */
kronq_status kronq_sensitivity(const float* HX, int64_t n, const float* HG, int64_t m,
                               double* out3, void* workspace, size_t ws_bytes, kronq_stream_t s);

/* The same traces straight from the tokens, without forming the factors:
 * tr(A^T A) = sum_t |a_t|^2 (a first pass over a whole model's sublayers,
 * before any factor is accumulated, so that the bit allocation can run
 * first).  A: T x d token rows, row stride lda (bf16 or float32), device.
 * trace: ONE double of device memory, overwritten (zero_first != 0) or
 * added to, so that token chunks can be streamed; the sum is formed in
 * float64 in a fixed order.  workspace: kronq_trace_tokens_workspace_bytes()
 * bytes of device memory, 256-byte aligned.  Asynchronous on s.
 * kronq_sensitivity_from_traces: traces = two device doubles { tr(H_X),
 * tr(H_G) } (e.g. two kronq_trace_tokens results); out3 (HOST) receives
 * { tr(H_X), tr(H_G), tr(H_G) * tr(H_X) }.  Synchronises the stream. */
size_t kronq_trace_tokens_workspace_bytes(void);
kronq_status kronq_trace_tokens(const void* A, kronq_dtype dt, int64_t T, int64_t d, int64_t lda,
                                double* trace, int zero_first, void* workspace, size_t ws_bytes,
                                kronq_stream_t s);
kronq_status kronq_sensitivity_from_traces(const double* traces, double* out3, kronq_stream_t s);

/* Bit allocation over L sublayers (host only; KronQ README "Mapping paper
 * results to flags", --inter_layer_mp).  Budget mode: start at bmin bits,
 * repeatedly give +1 bit to the sublayer with the largest
 * s_i (4^-b_i - 4^-(b_i+1)) / size_i among those whose upgrade keeps
 * sum b_i size_i <= avg_bits * sum size_i and b_i < bmax; ties to the lower
 * index.  sens, sizes, bits_out are HOST arrays of length L. */
kronq_status kronq_allocate_bits(const double* sens, const int64_t* sizes, int L, double avg_bits,
                                 int bmin, int bmax, int* bits_out);

/* Type-level rule (--inter_layer_mp N): the N sublayer types with the
 * largest summed sensitivity get base_bits + 1, the rest base_bits.
 * type_ids[i] in [0, n_types) names sublayer i's type; ties to the lower
 * type id.  HOST arrays of length L. */
kronq_status kronq_allocate_topn_types(const double* sens, const int* type_ids, int L, int n_types,
                                       int base_bits, int N, int* bits_out);

/* ---------------------------------------------------------------------------
 * Step 3 -- BiIP.  KronQ abstract point (1); README bullet "Bidirectional
 * incoherence processing"; flags --incoh_rotate --incoh_kernel had
 * --incoh_mode --alpha; the incoherence follows QuIP# (README
 * "Acknowledgements").  Reading fixed by this library:
 *   d_in[j]  = (H_X[j,j] / ||W[:,j]||^2)^alpha, d_out[i] = (H_G[i,i] / ||W[i,:]||^2)^alpha,
 *   degenerate (zero) entries 1, each vector scaled to geometric mean 1;
 *   V = (Had_{2^k}/sqrt(2^k) (x) DCT-II_K) diag(s_in) for n = 2^k K, K odd
 *   (K <= 255); U likewise for m with s_out; signs from SplitMix64:
 *   s_side[i] = 1 - 2 * bit63(mix64(2*seed + side + (i+1) * 0x9E3779B97F4A7C15)),
 *   side 0 = input, 1 = output.
 *   W~ = U D_out W D_in V^T,  H~_X = V D_in^-1 H_X D_in^-1 V^T,
 *   H~_G = U D_out^-1 H_G D_out^-1 U^T.
 *
 * kronq_biip_forward
 *   W   m x n, dtype wdt (bf16 or f32), read only.
 *   Wt  m x n float32 out (may not alias W).
 *   HX  n x n float32, transformed in place.
 *   HG  m x m float32, transformed in place; may be NULL in modes
 *       NO_RESCALE and SV_ONLY (then it is left alone).
 *   alpha   rescale exponent (0.25 weight-only).
 *   d_in (n), d_out (m)  float32 out: the rescale vectors (1 where unused).
 *   workspace  >= kronq_biip_workspace_bytes(m, n) bytes, 256-byte aligned.
 * kronq_biip_inverse
 *   W (m x n float32) in place: W <- D_out^-1 U^T W V D_in^-1.
 * ------------------------------------------------------------------------- */
size_t kronq_biip_workspace_bytes(int64_t m, int64_t n);

kronq_status kronq_biip_forward(const void* W, kronq_dtype wdt, float* Wt, int64_t m, int64_t n,
                                float* HX, float* HG, uint64_t seed, float alpha,
                                kronq_biip_mode mode, float* d_in, float* d_out,
                                void* workspace, size_t ws_bytes, kronq_stream_t s);

kronq_status kronq_biip_inverse(float* W, int64_t m, int64_t n, uint64_t seed,
                                kronq_biip_mode mode, const float* d_in, const float* d_out,
                                void* workspace, size_t ws_bytes, kronq_stream_t s);

/* ---------------------------------------------------------------------------
 * Step 4 -- quantization.  KronQ README intro ("extends GPTQ/GPTAQ");
 * "Reproduce from scratch" flags.  Readings fixed by this library:
 *   dead columns (diag 0): H_jj := 1, W[:, j] := 0; lambda = damp_rel *
 *   mean diag; U upper with U^T U = (H~_X + lambda I)^-1, computed as the
 *   upper "reverse" Cholesky factor R of H~_X + lambda I = R R^T followed by
 *   U = R^-1.  For every column j in order: at a group start, per-row grid
 *   from the current values of the group's columns (x_min = min(0, min w),
 *   x_max = max(0, max w), equal -> (-1, 1); scale = (x_max - x_min) /
 *   (2^b - 1), zero = rint(-x_min / scale)); q = clamp(rint(w / scale) +
 *   zero, 0, 2^b - 1) (round half to even); e = (w - scale (q - zero)) /
 *   U_jj; later columns -= e U[j, later], batched per `block` columns.
 *   With KRONQ_R_FORM the same decisions are taken from R (H~_X + lambda I
 *   = R R^T, U = R^-1) and the 128 x 128 diagonal blocks of U only: for the
 *   swept columns S and the rest T, GPTQ's partial state W~_T - E_S U_ST is
 *   W~_T + F U_TT with F = (W~ - Q)_S R_ST (W~ before the sweep), so each
 *   128-column block starts from W~_G + F_G U_GG and is swept as above on
 *   U_GG, and F accumulates (W~ - Q)_G R_G,later.  Not with KRONQ_U_GIVEN
 *   or KRONQ_ORDERED_FP32 (KRONQ_ERR_INVALID_ARG); groups of at most 128
 *   columns or -1 (KRONQ_ERR_UNSUPPORTED otherwise).
 *
 *   Wt     m x n float32: in W~, out the dequantised W~_q.
 *   HX     n x n float32: in H~_X (or U with KRONQ_U_GIVEN), out U (upper
 *          triangle; the strict lower triangle is scratch on return); with
 *          KRONQ_R_FORM out R instead (upper, H~_X + lambda I = R R^T).
 *   codes  m x n uint8 out, values 0 .. 2^bits - 1.
 *   scales, zeros  m x ngroups float32 out, ngroups = 1 if group == -1 else
 *          ceil(n / group); zeros are integer valued.
 *   E      m x n float32 out (scaled errors) with KRONQ_WRITE_E, else NULL.
 *   info   one int (device) out: 0, or 1 + the largest index j for which the
 *          trailing submatrix (H~_X + lambda I)[j:, j:] was found not
 *          positive definite (codes etc. are then unspecified).
 *   workspace >= kronq_quantize_workspace_bytes(m, n, p), 256-byte aligned
 *          (KRONQ_R_FORM adds m n floats for the copy of W~ and 128^2
 *          ceil(n / 128) for U's diagonal blocks).
 * ------------------------------------------------------------------------- */
size_t kronq_quantize_workspace_bytes(int64_t m, int64_t n, const kronq_quant_params* p);

kronq_status kronq_quantize_layer(float* Wt, float* HX, int64_t m, int64_t n,
                                  const kronq_quant_params* p, uint8_t* codes, float* scales,
                                  float* zeros, float* E, int* info, void* workspace,
                                  size_t ws_bytes, kronq_stream_t s);

/* kronq_quantize_layer_static -- the same call for callers that cannot
 * allocate device memory (no counterpart on the pages; the paper has none).
 * Such callers hold only pointers handed to them by another runtime (a
 * plugin inside a framework whose memory pool owns all device memory and
 * exposes no allocator, or a foreign-language caller without a CUDA
 * allocation binding), or run where cudaMalloc is not allowed because it
 * synchronises the device.  Arguments as kronq_quantize_layer, minus the
 * workspace: the scratch is a file-scope static device array of 64 MiB that
 * every GPU loading the library holds until the process exits.
 *   - Layers whose kronq_quantize_workspace_bytes(m, n, p) exceeds 64 MiB
 *     (for example n = 4096 with m above ~6500, or any n above 4096, whose
 *     blocked factorisation needs more scratch) are rejected with
 *     KRONQ_ERR_INVALID_ARG before anything runs.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.
 *   - No cudaMalloc, cudaFree or allocating library routine is called.
 *   - All calls on a device share the array, which keeps the last call's
 *     contents; nothing in it has to start at zero, but calls that overlap
 *     on the GPU (two streams, two threads) race on it. */
kronq_status kronq_quantize_layer_static(float* Wt, float* HX, int64_t m, int64_t n,
                                         const kronq_quant_params* p, uint8_t* codes, float* scales,
                                         float* zeros, float* E, int* info, kronq_stream_t s);

/* kronq_quantize_layer_act_order -- the same pass with the recipe's
 * --act_order (KronQ README, "Reproduce from scratch"; not defined on the
 * pages, read as GPTQ's act-order heuristic): after the dead-column rule
 * the columns are swept in order of decreasing diagonal of H~_X (ties keep
 * the column order), groups are consecutive columns of that order, and the
 * outputs come back in the original column order.
 *   Wt, codes, E   as kronq_quantize_layer, in the ORIGINAL column order.
 *   scales, zeros  m x ngroups, one column per group of the SWEEP order.
 *   g_idx          n ints (device) out: column j uses group g_idx[j]
 *                  (rank of j in the sweep order / group; 0 for group -1).
 *   perm           n ints (device) out, may be NULL: perm[k] = the column
 *                  swept k-th.
 *   HX             in H~_X; out U (R with KRONQ_R_FORM) of the permuted,
 *                  damped factor (upper triangle, sweep order).
 *   flags          KRONQ_WRITE_E, KRONQ_ORDERED_FP32 and KRONQ_R_FORM;
 *                  KRONQ_U_GIVEN is rejected (the order comes from H~_X).
 *   workspace      >= kronq_quantize_act_order_workspace_bytes(m, n, p)
 *                  (holds the permuted copies: n^2 + m n floats and more).
 * Asynchronous on s. */
size_t kronq_quantize_act_order_workspace_bytes(int64_t m, int64_t n, const kronq_quant_params* p);
kronq_status kronq_quantize_layer_act_order(float* Wt, float* HX, int64_t m, int64_t n,
                                            const kronq_quant_params* p, uint8_t* codes, float* scales,
                                            float* zeros, float* E, int* g_idx, int* perm, int* info,
                                            void* workspace, size_t ws_bytes, kronq_stream_t s);

/* kronq_quantize_two_sided -- two-sided rounding that uses H_G inside the
 * sweep ("BaKron: Efficient Quantization with Kronecker-Factored Hessians"
 * page, abstract: GPTQ-style rounding in the vectorised weight domain under
 * the Kronecker-factored Hessian, anti-diagonal parallelism, O(m + n)
 * sequential steps, O(mn(m + n)) work).  The abstract gives no algorithm;
 * the reading implemented is GPTQ on vec(W) with the upper factor
 * U = U_X (x) U_G of the damped inverse Hessian:
 *   - both factors damped by the relative rule (lambda = damp_rel * mean
 *     diagonal; no dead-column rule), U_X^T U_X = (H~_X + lambda_X I)^-1,
 *     U_G^T U_G = (H~_G + lambda_G I)^-1, both upper;
 *   - static per-row group grids taken from W~ before the sweep (the grid
 *     rule of kronq_quantize_layer; a grid taken at a group start would
 *     depend on the processing order);
 *   - element (i, j): q = clamp(rint(w~ / scale) + zero, 0, 2^b - 1),
 *     e_ij = (w~_ij - deq) / (U_X[j, j] U_G[i, i]) (in float32, the
 *     divisions as products with the float32 reciprocals), and
 *     w~_i'j' -= e_ij U_G[i, i'] U_X[j, j'] for every later (i' >= i,
 *     j' >= j) element.  Every order that respects that partial order gives
 *     the same result; the library runs 32 x 128 tiles along anti-diagonals.
 *   Wt     m x n float32: in W~, out the dequantised W~_q.
 *   HX     n x n float32: in H~_X (or U_X with KRONQ_U_GIVEN), out U_X
 *          (upper triangle; the strict lower triangle is scratch).
 *   HG     m x m float32: in H~_G (or U_G with KRONQ_U_GIVEN), out U_G.
 *   codes  m x n uint8 out; scales, zeros m x ngroups float32 out.
 *   E      m x n float32 out (the scaled errors e_ij) with KRONQ_WRITE_E,
 *          else NULL.
 *   info   TWO ints (device) out: info[0] for H~_X, info[1] for H~_G, each
 *          0 or 1 + the largest index whose trailing submatrix was found not
 *          positive definite (the outputs are then unspecified).
 *   flags  KRONQ_U_GIVEN and KRONQ_WRITE_E; KRONQ_R_FORM and
 *          KRONQ_ORDERED_FP32 are rejected (KRONQ_ERR_INVALID_ARG).
 *          block must be 128; groups as kronq_quantize_layer.
 *   workspace >= kronq_quantize_two_sided_workspace_bytes(m, n, p), 256-byte
 *          aligned (2 m n floats plus the factorisation scratch of the larger
 *          factor).
 * Asynchronous on s. */
size_t kronq_quantize_two_sided_workspace_bytes(int64_t m, int64_t n, const kronq_quant_params* p);
kronq_status kronq_quantize_two_sided(float* Wt, float* HX, float* HG, int64_t m, int64_t n,
                                      const kronq_quant_params* p, uint8_t* codes, float* scales,
                                      float* zeros, float* E, int* info, void* workspace, size_t ws_bytes,
                                      kronq_stream_t s);

/* ---------------------------------------------------------------------------
 * Step 5 -- packing.  KronQ README "Model zoo": W4/W2 as packed int4/int2,
 * W3 not bit-packable (bits == 3 -> KRONQ_ERR_INVALID_ARG).  Layout: per
 * row, along n, codes fill uint32 words from the least significant bit up
 * (8 per word at 4 bits, 16 at 2 bits); words per row = ceil(n*bits/32),
 * a ragged last word zero-padded.  codes m x n uint8; words m x wpr uint32.
 * ------------------------------------------------------------------------- */
kronq_status kronq_pack(const uint8_t* codes, int64_t m, int64_t n, int bits, uint32_t* out,
                        kronq_stream_t s);
kronq_status kronq_unpack(const uint32_t* in, int64_t m, int64_t n, int bits, uint8_t* codes,
                          kronq_stream_t s);

/* ---------------------------------------------------------------------------
 * Diagnostics (no counterpart on the pages).
 * kronq_device_status: synchronises the stream, returns in *out (host) the
 *   library's device status word (KRONQ_OK or KRONQ_ERR_TIMEOUT) and clears it.
 * kronq_kfac_loss: out (HOST double) = sum_j e_j^T HG e_j for the columns e_j
 *   of E (m x n), HG m x m -- the K-FAC loss of the sweep,
 *   tr(dW (H~_X + lambda I) dW^T H~_G), because dW = E U.  Workspace of
 *   kronq_kfac_loss_workspace_bytes(m, n) bytes, 256-byte aligned.
 *   Synchronises the stream.
 * ------------------------------------------------------------------------- */
kronq_status kronq_device_status(int* out, kronq_stream_t s);
/* kronq_wait_selftest: launches one CTA whose bounded wait is never
 *   satisfied, so that it gives up after limit_ns (0 < limit_ns <= 1e9)
 *   exactly as a stuck wait inside the pass would: which 0 waits on an
 *   mbarrier phase that nothing completes (the wait of every tensor-core
 *   kernel), which 1 on a step counter that no CTA advances (the cross-CTA
 *   wait of the persistent factorisation, which then raises its abort
 *   flag).  The wait records KRONQ_ERR_TIMEOUT in the device status word
 *   (read and cleared by kronq_device_status) and the kernel returns; the
 *   CUDA context stays usable.  workspace: >= 3 ints of device memory;
 *   on return w[0] = counter (0), w[1] = abort flag (1 for which 1),
 *   w[2] = 1 when the wait gave up.  Asynchronous on s. */
kronq_status kronq_wait_selftest(int which, uint64_t limit_ns, void* workspace, size_t ws_bytes,
                                 kronq_stream_t s);
size_t kronq_kfac_loss_workspace_bytes(int64_t m, int64_t n);
kronq_status kronq_kfac_loss(const float* E, const float* HG, int64_t m, int64_t n, double* out,
                             void* workspace, size_t ws_bytes, kronq_stream_t s);

/* ---------------------------------------------------------------------------
 * Kronecker factor estimators A (x) B ~ H = E[x x^T (x) g g^T]
 * ("WaterKron and FlipFlop Hessian" page, Table 1 and its caption).
 *
 *   KRONQ_EST_INPUT      A = E[x x^T],               B = I
 *   KRONQ_EST_MARGINAL   A = E[x x^T],               B = E[g g^T]
 *   KRONQ_EST_FROBENIUS  A = E[(g^T B g) x x^T] / ||B||_F^2,
 *                        B = E[(x^T A x) g g^T] / ||A||_F^2
 *   KRONQ_EST_FLIPFLOP   A = E[(g^T B^-1 g) x x^T] / m,
 *                        B = E[(x^T A^-1 x) g g^T] / n
 * E is the mean over the T tokens.  Frobenius and FlipFlop start from
 * B = I and run `iters` sweeps (A from B, then B from A); each update is the
 * exact minimiser of the row's target over one factor (||H - A (x) B||_F;
 * for FlipFlop the Gaussian fit tr((A (x) B)^-1 H) + log det(A (x) B)).
 *
 * X: T x n bf16, G: T x m bf16, device, row-major with row strides n and m;
 * n and m multiples of 8 (16-byte rows for the tensor-core loads).  A (n x n)
 * and B (m x m): fp32 device outputs, both triangles written.  info: device
 * int, 0 on success, else the failing pivot + 1 of the Cholesky factor of a
 * FlipFlop factor that is not positive definite (the remaining steps are
 * skipped).  Per-token weights come from a tensor-core product of the tokens
 * with a bf16 hi/lo split of the other factor (or of the Cholesky factor of
 * its inverse), the weighted second moment from the tensor-core SYRK of the
 * sqrt(weight)-scaled tokens rounded to bf16.  Workspace of
 * kronq_kron_factors_workspace_bytes(T, n, m) bytes, 256-byte aligned.
 * Asynchronous on s.
 * ------------------------------------------------------------------------- */
typedef enum {
  KRONQ_EST_INPUT = 0,
  KRONQ_EST_MARGINAL = 1,
  KRONQ_EST_FROBENIUS = 2,
  KRONQ_EST_FLIPFLOP = 3
} kronq_estimator;

size_t kronq_kron_factors_workspace_bytes(int64_t T, int64_t n, int64_t m);
kronq_status kronq_kron_factors(const void* X, const void* G, int64_t T, int64_t n, int64_t m,
                                kronq_estimator est, int iters, float* A, float* B, int* info,
                                void* workspace, size_t ws_bytes, kronq_stream_t s);

/* ---------------------------------------------------------------------------
 * Deploy-path matvec from packed codes (KronQ README intro: packed int4/int2
 * weights, a fused dequant + BiIP matvec for single-token decode):
 *   y = D_o^-1 U^T Q V D_i^-1 x,  Q[i, j] = scales[i, g] (q[i, j] - zeros[i, g]),
 * g = j / group (0 when group == -1), q from `packed` (m x ceil(n bits / 32)
 * uint32 words, least significant bits first along n: kronq_pack's layout).
 * U, V, d_in, d_out, seed and mode are those of kronq_biip_forward.
 *   x: n activations, bf16 or float32 (xdt); y: m float32 out.  All device
 *   memory.  bits 2 or 4.  Workspace of kronq_decode_matvec_workspace_bytes
 *   bytes, 256-byte aligned.  Asynchronous on s.
 * ------------------------------------------------------------------------- */
size_t kronq_decode_matvec_workspace_bytes(int64_t m, int64_t n);
kronq_status kronq_decode_matvec(const uint32_t* packed, const float* scales, const float* zeros,
                                 int64_t m, int64_t n, int bits, int group, uint64_t seed,
                                 kronq_biip_mode mode, const float* d_in, const float* d_out,
                                 const void* x, kronq_dtype xdt, float* y, void* workspace,
                                 size_t ws_bytes, kronq_stream_t s);

/* Number of kernels this library has launched in the process so far (all
 * devices and streams); a host counter, no synchronisation. */
uint64_t kronq_launch_count(void);

const char* kronq_last_error(void);
const char* kronq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KRONQ_H */
