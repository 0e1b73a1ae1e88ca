// Internal launchers of libkronq (C++ linkage, not exported).  Every
// launcher assumes its arguments were validated by the C ABI layer.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/kronq.h"

namespace kq {

// ------------------------------------------------------------ TMA maps (host)
// The driver's cuTensorMapEncodeTiled (nullptr when unavailable) and a 2-D
// tiled map with the 128-byte swizzle: inner x outer elements, row stride
// ld elements, box box_inner x box_outer, zero fill out of bounds.
PFN_cuTensorMapEncodeTiled_v12000 tma_encode_fn();
bool tma_map_2d(CUtensorMap* map, CUtensorMapDataType dt, int esize, const void* base, int64_t inner,
                int64_t outer, int64_t ld, uint32_t box_inner, uint32_t box_outer);

// ------------------------------------------------------------ SIMT GEMM
// C = beta * C + alpha * op(A) op(B), float32, one launch, optional batch.
//   op(A)(i,k) = transA ? A[k*lda + i] : A[i*lda + k]          (M x K)
//   op(B)(k,j) = transB ? B[j*ldb + k] : B[k*ldb + j]          (K x N)
//   a_upper: op(A)(i,k) is taken as 0 for k < i; b_upper: op(B)(k,j) = 0 for k > j
//   c_mode : 0 all entries, 1 only i <= j, 2 i <= j plus the mirror C[j][i] = C[i][j]
//   ordered: every product and sum rounded separately in ascending k and the
//            result applied as C = C - acc (alpha must be -1, beta 1)
//   beta == 0 never reads C.  If info != nullptr and *info != 0, no-op.
struct GemmDesc {
  int64_t M = 0, N = 0, K = 0;
  const float* A = nullptr;
  int64_t lda = 0;
  bool transA = false;
  const float* B = nullptr;
  int64_t ldb = 0;
  bool transB = false;
  float* C = nullptr;
  int64_t ldc = 0;
  float alpha = 1.f, beta = 0.f;
  bool a_upper = false, b_upper = false;
  int c_mode = 0;
  bool ordered = false;
  int batch = 1;
  int64_t strideA = 0, strideB = 0, strideC = 0;
  const int* info = nullptr;
};
cudaError_t gemm_f32(const GemmDesc& g, cudaStream_t s);

// ------------------------------------------------------------ tensor-core triangular GEMM
// C = alpha * A B (row-major fp32, optional batch with element strides) with
// exactly one triangular operand: a_upper (A[i][k] = 0 for k < i) or
// b_upper (B[k][j] = 0 for k > j); the other triangle of its storage is
// never used.  fp32-level accuracy (six bf16 split products).  No-op when
// info != nullptr and *info != 0.
struct TriGemm {
  int64_t M = 0, N = 0, K = 0;
  const float* A = nullptr;
  int64_t lda = 0;
  const float* B = nullptr;
  int64_t ldb = 0;
  float* C = nullptr;
  int64_t ldc = 0;
  float alpha = 1.f;
  bool a_upper = false, b_upper = false;
  int batch = 1;
  int64_t strideA = 0, strideB = 0, strideC = 0;
  const int* info = nullptr;
  // Optional: the whole matrices that hold A and B (row strides lda, ldb),
  // for TMA maps; A and B point inside them.  nullptr: plain loads only.
  const float* holdA = nullptr;
  int64_t holdA_rows = 0, holdA_cols = 0;
  const float* holdB = nullptr;
  int64_t holdB_rows = 0, holdB_cols = 0;
};
kronq_status trigemm_tc(const TriGemm& t, cudaStream_t s);
cudaError_t status_fetch_trigemm(int* out, cudaStream_t s);

// ------------------------------------------------------------ factors
kronq_status syrk_bf16_tc(const void* A, int64_t T, int64_t d, int64_t lda, float* H,
                          bool zero_first, cudaStream_t s);
cudaError_t status_fetch_syrk(int* out, cudaStream_t s);
cudaError_t fill_f32(float* p, int64_t count, float v, cudaStream_t s);

// ------------------------------------------------------------ BiIP
// One pass of the row transform with a transposed store:
//   out[j * ld_out + r] = T(in row r)[j],  r < rows, j < L
// forward: v = in * scale * sign  ->  (Had/sqrt(P) (x) C_K) v
// inverse: v = (Had/sqrt(P) (x) C_K^T) in  ->  v * sign / scale
// scale_mode: 0 none, 1 multiply by scale[j], 2 divide by scale[j].
// rotate == false: only the scaling and the transposed store.
struct RowPass {
  const void* in = nullptr;
  bool in_bf16 = false;
  int64_t ld_in = 0;
  float* out = nullptr;
  int64_t ld_out = 0;
  int64_t rows = 0, L = 0;
  const float* scale = nullptr;
  int scale_mode = 0;
  bool rotate = true;
  bool inverse = false;
  uint64_t sign_state = 0;  // 2 * seed + side
  float* cf = nullptr;      // optional scratch of L floats for the column factors
  // false: out = the transformed rows, transposed (out[j * ld_out + row]);
  // true: stored as rows (out[row * ld_out + j]), for a result that is
  // symmetric anyway (the second pass of V F H F V^T)
  bool rowwise = false;
  // optional scratch of rows x L floats (row stride ld_tmp; it may be `in`
  // itself when that is float32 and may be overwritten): a transposed pass
  // may then run as a row-wise pass into it followed by a transpose
  float* tmp = nullptr;
  int64_t ld_tmp = 0;
};
kronq_status rowpass(const RowPass& p, cudaStream_t s);
// sum of squares along columns (colsq[n]) and rows (rowsq[m]) of W.
kronq_status wnorms(const void* W, bool bf16, int64_t m, int64_t n, float* colsq, float* rowsq,
                    float* partial, cudaStream_t s);
size_t wnorms_partial_floats(int64_t m, int64_t n);
// d[j] = (H[j,j] / nrm[j])^alpha, degenerate -> 1, normalised to geometric mean 1.
kronq_status rescale_vector(const float* H, int64_t ldh, const float* nrm, int64_t len, float alpha,
                            float* d, cudaStream_t s);

// ------------------------------------------------------------ factorisation
// TMA descriptors of the tensor-core Schur update (the three panel splits,
// 128-row boxes, and the fp32 matrix in 32-column boxes).
struct alignas(64) SchurMaps {
  unsigned char raw[4 * 128];
  int tma_c = 0;   // tile of A staged by TMA (needs a 16-byte row stride)
};
kronq_status schur_maps(SchurMaps* sm, const __nv_bfloat16* splits, float* H, int64_t n);
kronq_status schur_update_tc(const SchurMaps* sm, float* H, int64_t n, int64_t j0, const int* info,
                             cudaStream_t s);
cudaError_t status_fetch_schur(int* out, cudaStream_t s);
// In: H (n x n) full symmetric.  Out (upper triangle): U with U^T U =
// (H + lambda I)^-1, or with want_u false the factor R = U^-1 itself
// (H + lambda I = R R^T, R upper); dead-column flags, info.  ws: see
// chol_workspace_bytes.
size_t chol_workspace_bytes(int64_t n);
// Above this order the factorisation is blocked in two levels (chol_blocked).
constexpr int64_t kOuterBlock = 4096;
// The single-level factorisation of a contiguous n x n block (no damping,
// info untouched unless a pivot fails) and its workspace.
size_t chol_core_workspace_bytes(int64_t n);
size_t chol_tbuf_bytes(int64_t n);
// want_u false: R instead of U (the diagonal blocks U_JJ stay staged in ws,
// and chol_core_finish_u then turns R into U in place).
kronq_status chol_core(float* H, int64_t n, int* info, void* ws, cudaStream_t s, bool want_u = true);
kronq_status chol_core_finish_u(float* H, int64_t n, int* info, void* ws, cudaStream_t s);
// U = R^-1 from the diagonal blocks U_JJ of size S0 (aligned from the top)
// and the off-diagonal blocks of R, level by level (tensor-core products).
kronq_status chol_inverse_levels(float* H, int64_t n, int64_t S0, float* Tbuf, const int* info,
                                 cudaStream_t s);
// Two-level blocked factorisation for n > kOuterBlock (after damping).
size_t chol_blocked_workspace_bytes(int64_t n);
kronq_status chol_blocked(float* H, int64_t n, int* info, void* ws, cudaStream_t s, bool want_u = true);
cudaError_t status_fetch_schurk(int* out, cudaStream_t s);
// One CTA whose bounded wait (which 0: mbarrier, 1: cross-CTA counter) is
// never satisfied; gives up after limit_ns.  w: 3 device ints.
kronq_status wait_selftest(int which, unsigned long long limit_ns, int* w, cudaStream_t s);
cudaError_t status_fetch_chol(int* out, cudaStream_t s);
kronq_status chol_upper_inverse(float* H, int64_t n, float damp_rel, bool skip_damp,
                                uint8_t* dead, int* info, void* ws, cudaStream_t s, bool want_u = true);

// ------------------------------------------------------------ sweep
// Storage for the four TMA descriptors of the tensor-core trailing update
// (E hi/lo, U-block hi/lo); filled by trailing_maps on the host.
struct alignas(64) TrailingMaps {
  unsigned char raw[5 * 128];
  int tma_c = 0;   // W tile staged by TMA (needs a 16-byte row stride)
};
// E hi/lo: m x lde bf16 (K-major); U hi/lo: ku x n bf16 (row stride ldu).
kronq_status trailing_maps(TrailingMaps* tm, const void* Eh, const void* El, int64_t m, int64_t lde,
                           const void* Uh, const void* Ul, int64_t ku, int64_t ldu, float* W, int64_t n);
// W[:, c_begin : c_begin + ncols] -= E[:, k0 : k0 + K] U[k0 : k0 + K, same columns]
// (K rounded up to 64; the E and U entries beyond K must be zero).
kronq_status trailing_update_tc(const TrailingMaps* tm, float* W, int64_t m, int64_t n, int64_t c_begin,
                                int64_t ncols, int64_t k0, int64_t K, const int* info, cudaStream_t s);
cudaError_t status_fetch_trailing(int* out, cudaStream_t s);

struct SweepDesc {
  float* W = nullptr;  // m x n, row stride n
  const float* U = nullptr;  // n x n upper
  int64_t m = 0, n = 0;
  int bits = 4, group = 128;
  bool asym = true;
  uint8_t* codes = nullptr;
  float* scales = nullptr;
  float* zeros = nullptr;
  int64_t ngroups = 1;
  float* E = nullptr;  // m x n (caller) or nullptr
  float* Eblk = nullptr;  // m x 128 workspace
  const uint8_t* dead = nullptr;
  const int* info = nullptr;
  bool ordered = false;
  // tensor-core trailing updates (used unless ordered), two-level: bf16
  // hi/lo splits of the scaled errors (m x lde, lde = 128 gblocks) and of the
  // rows of U (128 gblocks x ldu) of the blocks of the current group of
  // gblocks blocks.  After a block, the group's later columns get its update
  // (K = 128); at the group's end the columns past it get the whole group's
  // update at once (K = 128 gblocks).
  __nv_bfloat16* Eh = nullptr;
  __nv_bfloat16* El = nullptr;
  __nv_bfloat16* Uh = nullptr;
  __nv_bfloat16* Ul = nullptr;
  int64_t ldu = 0;
  int64_t lde = 128;
  int gblocks = 1;
  // R form (not with ordered; groups of at most 128 columns, or one per
  // row): U points at R (upper, H~ = R R^T) and U = R^-1 is not formed.
  // W holds the feedback F = (W0 - Q)_done R_done,: (zero at the start),
  // W0 the weights before the sweep, Ublk the 128 x 128 diagonal blocks
  // U_GG = (R_GG)^-1 (block b at rows 128 b .., row stride 128).  A block
  // starts from W0_G + F_G U_GG (GPTQ's partial state of its columns) and is
  // swept on U_GG as in the U form; its later columns then get F += (W0 -
  // Q)_G R_G,later.
  const float* W0 = nullptr;
  const float* Ublk = nullptr;
};
kronq_status gptq_sweep(const SweepDesc& d, cudaStream_t s);
// The 128 x 128 diagonal blocks of U = R^-1 for the R form (ceil(n / 128)
// blocks of 128 x 128 floats, row stride 128).
kronq_status diag_block_inverse(const float* R, int64_t n, float* Ublk, const int* info, cudaStream_t s);

// The body of kronq_quantize_layer after validation.  mode 0: dead columns,
// damping and factorisation of HX; 1: HX holds U already; 2: HX is damped
// already (no dead-column rule), factorisation only.  KRONQ_R_FORM in the
// flags (modes 0 and 2): the factor is left as R and the sweep runs on it.
size_t quantize_core_workspace_bytes(int64_t m, int64_t n, bool rform);
kronq_status check_quant_args(float* Wt, float* HX, int64_t m, int64_t n, const kronq_quant_params* p,
                              uint8_t* codes, float* scales, float* zeros, float* E, int* info,
                              const char* who);
kronq_status quantize_core(float* Wt, float* HX, int64_t m, int64_t n, const kronq_quant_params* p,
                           uint8_t* codes, float* scales, float* zeros, float* E, int* info,
                           void* workspace, cudaStream_t st, int mode);
// Dead-column rule and damping of H in place (dead flags out, info reset).
kronq_status damp_factor(float* H, int64_t n, float damp_rel, uint8_t* dead, int* info, cudaStream_t s);
// Damping alone (zero diagonal entries stay zero before lambda is added),
// info reset.
kronq_status damp_only(float* H, int64_t n, float damp_rel, int* info, cudaStream_t s);

// ------------------------------------------------------------ pack / misc
kronq_status pack_codes(const uint8_t* codes, int64_t m, int64_t n, int bits, uint32_t* out,
                        cudaStream_t s);
kronq_status unpack_codes(const uint32_t* in, int64_t m, int64_t n, int bits, uint8_t* codes,
                          cudaStream_t s);
kronq_status diag_sums(const float* HX, int64_t n, const float* HG, int64_t m, double* dev2,
                       cudaStream_t s);
// out (+)= sum of squares of the T x d token matrix A (float64); partial:
// token_sqsum_partials() doubles of device scratch.
size_t token_sqsum_partials();
kronq_status token_sqsum(const void* A, bool bf16, int64_t T, int64_t d, int64_t lda, double* out,
                         int zero_first, double* partial, cudaStream_t s);
kronq_status dot_sum(const float* a, const float* b, int64_t count, double* dev1, double* partial,
                     cudaStream_t s);

}  // namespace kq
