// Internal launch interfaces between the translation units of the library.
#pragma once

#include "gptq_common.cuh"

namespace gptq {

// Tile-granular triangular structure for launch_gemm (tiles are 128 x 128 and
// a triangular operand must hold zeros below the diagonal inside the tiles on
// its diagonal).
enum GemmFlags {
  GEMM_KMIN_ROW = 1,  // A upper triangular: k starts at the row tile
  GEMM_KMIN_COL = 2,  // op(B) lower (B^T of an upper matrix): k starts at the column tile
  GEMM_KMAX_COL = 4,  // B upper triangular: k ends with the column tile
  GEMM_UPPER_C = 8    // only output tiles on or above the diagonal
};

// C = alpha * A * op(B) + beta * C, all row-major fp32; op(B) = B (K x N) or
// B^T with B stored N x K.  Leading dimensions and column offsets must be
// multiples of 4 floats, K a multiple of 8.
struct GemmArgs {
  int M, N, K;
  const float *A;
  int64_t lda;
  const float *B;
  int64_t ldb;
  float *C;
  int64_t ldc;
  float alpha, beta;
  int flags;
  const int *status;  // skip the launch's work if *status != 0 (may be NULL)
};

int launch_gemm(const GemmArgs &g, bool trans_b, cudaStream_t stream);

int launch_damp(float *H, int64_t ld, int d, float damp, bool add_in_place, float *lambda,
                cudaStream_t stream);
int launch_act_order(const float *H, int64_t ld, int d, int *perm, int *inv, const float *lambda,
                     float *Hp, cudaStream_t stream);
size_t factor_scratch_floats(int64_t d);
// One diagonal block (nb <= 128, nb % 32 == 0) of H_d -> U in place (full block, zeros below).
int launch_leaf(float *A, int64_t ld, int nb, int *status, cudaStream_t stream);
int launch_factor(float *A, int64_t d, float *T1, int *status, cudaStream_t stream);

struct SweepArgs {
  float *Wk;          // working weights r x d (sweep order), row stride ldw
  int64_t ldw;
  const float *U;     // factor (upper triangle), row stride ldu
  int64_t ldu;
  int r, j0, ncols;   // block start column and width (<= block)
  int bits, group;    // group: -1 or the group size
  float *scales;      // r x G
  int32_t *zeros;     // r x G
  int G;
  uint8_t *codes;     // r x d codes in sweep order
  int64_t ldc;
  float *err;         // r x lde; column 0 is the block's first column
  int64_t lde;
  double *loss_rows;  // per-row running sum of e^2 / 2
  const int *status;
};

int launch_gather_w(const float *W, int r, int d, const int *perm, float *Wk, const int *status,
                    cudaStream_t stream);
int launch_row_params(const float *Wk, int r, int d, int bits, float *scales, int32_t *zeros,
                      const int *status, cudaStream_t stream);
int launch_sweep_block(const SweepArgs &a, int block, cudaStream_t stream);

struct FinalizeArgs {
  const float *W;       // original weights r x d
  const float *Wk;      // dequantised weights, sweep order
  const uint8_t *codes_p;
  const int *inv;       // inv[c] = sweep position of column c (NULL: identity)
  int r, d, bits, group;
  float *W_hat;         // may be NULL
  uint8_t *codes;       // may be NULL
  int32_t *qweight;
  int32_t *g_idx;       // may be NULL
  double *dsq_rows;     // per-row ||W - W^||^2
  const int *status;
};
int launch_finalize(const FinalizeArgs &a, cudaStream_t stream);
int launch_loss_reduce(const double *loss_rows, const double *dsq_rows, int r,
                       const float *lambda, double *out, const int *status,
                       cudaStream_t stream);

int launch_pack(const uint8_t *codes, int64_t r, int64_t d, int bits, int32_t *qweight,
                cudaStream_t stream);

}  // namespace gptq
