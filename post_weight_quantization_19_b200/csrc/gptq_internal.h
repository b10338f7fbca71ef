// Internal launch interfaces between the translation units of the library.
#pragma once

#include <utility>

#include "gptq_common.cuh"

namespace gptq {

// ---- programmatic dependent launch ----
// The kernels of the layer sequence are launched with programmatic stream
// serialisation: a kernel may start while its predecessor is still running,
// does only set-up that needs nothing from its predecessor (barriers,
// descriptor prefetch, reads of data its predecessor does not write), then
// waits for the predecessor grid to complete and only after that lets its own
// successor launch.  So when a kernel starts, every grid before its
// predecessor has completed, and at most two grids of the sequence are in
// flight.
__device__ __forceinline__ void pdl_wait_then_release() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Scheduling priority of a launch, by level: 0 = the layer sequence's critical
// path (the device's greatest priority), 1 = work the critical path will wait
// for soon (the factorisation's trailing updates; the middle of the range), 2 =
// work only the end of the factorisation waits for (the merge products that
// assemble U; the least priority).  SMs that free up go to the higher level
// first.
int launch_priority(int level);

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_prio(int level, void (*kernel)(KArgs...), dim3 grid, dim3 block,
                            size_t smem, cudaStream_t stream, Args &&...args) {
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributePriority;
  attr[1].val.priority = launch_priority(level);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args &&...args) {
  return launch_pdl_prio(0, kernel, grid, block, smem, stream, std::forward<Args>(args)...);
}

// The dynamic shared-memory limit of a kernel, raised once per device (the
// attribute belongs to the kernel in the current device's context).
// (Two threads may both set it the first time; setting it twice is harmless.)
template <typename K>
int ensure_smem_attr(K kernel, size_t bytes, std::atomic<bool> (&done)[64]) {
  int dev = 0;
  GPTQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return GPTQ_ERR_INVALID_ARG;
  if (!done[dev].load(std::memory_order_acquire)) {
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)bytes));
    done[dev].store(true, std::memory_order_release);
  }
  return GPTQ_OK;
}

// launch_pdl with the library's launch accounting and error reporting; a
// template kernel name goes in parentheses.
#define GPTQ_LAUNCH_PDL(kernel, grid, block, smem, stream, ...)                          \
  do {                                                                                  \
    ::gptq::count_launch();                                                             \
    cudaError_t e_ = ::gptq::launch_pdl(kernel, grid, block, smem, stream, __VA_ARGS__); \
    if (e_ != cudaSuccess) {                                                            \
      (void)cudaGetLastError();                                                         \
      ::gptq::set_last_error(__FILE__, __LINE__, "kernel launch", e_);                  \
      return GPTQ_ERR_CUDA;                                                             \
    }                                                                                   \
  } while (0)

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
  int prio = 0;              // launch priority level (see launch_priority)
  int stall_after = -1;      // self-test of the timeout path only (see gptq_selftest_timeout)
};

int launch_gemm(const GemmArgs &g, bool trans_b, cudaStream_t stream);
// Whether products with two or more row tiles may use the two-CTA kernel
// (gptq_set_gemm_pair; off by default).
int gemm_pair_enabled();

int launch_damp(float *H, int64_t ld, int d, float damp, bool add_in_place, float *lambda,
                cudaStream_t stream);
int launch_act_order(const float *H, int64_t ld, int d, int *perm, int *inv, const float *lambda,
                     float *Hp, cudaStream_t stream);
// inv[perm[p]] = p after checking that perm is a permutation (status set otherwise).
int launch_check_perm(const int *perm, int d, int *inv, int *status, cudaStream_t stream);
// Scratch floats of the factorisation of a d x d matrix: the merge products of
// non-square merge-tree nodes and, for wide layers, a copy of the outer panel.
size_t factor_scratch_floats(int64_t d);
// One diagonal block (nb <= 128, nb % 32 == 0) of H_d -> U in place (full block, zeros below).
int launch_leaf(float *A, int64_t ld, int nb, int *status, cudaStream_t stream);
// dst[rows x cols] = src[rows x cols] (fp32, row strides ldd / lds; all multiples of 4 floats).
int launch_copy2d(float *dst, int64_t ldd, const float *src, int64_t lds, int64_t rows,
                  int64_t cols, const int *status, cudaStream_t stream);
// use_side: run the work off the critical path (trailing updates, merge
// products) on side streams (created once per device, with their events);
// false keeps everything on `stream`.
int launch_factor(float *A, int64_t d, float *T1, int *status, cudaStream_t stream,
                  bool use_side);

// ---- factorisation plan recording (a host-only diagnostic) ----
// While a PlanRecorder is installed on the calling thread, launch_leaf,
// launch_gemm and launch_copy2d validate their arguments and append one line
// to it instead of launching, and launch_factor records its stream events
// instead of creating them.  Pointers are written as a buffer name and an
// element offset into one of the registered buffers.
struct PlanRecorder {
  char *out = nullptr;     // caller's text buffer (may be NULL: count only)
  size_t cap = 0, used = 0;
  const char *name[4] = {nullptr, nullptr, nullptr, nullptr};
  const float *base[4] = {nullptr, nullptr, nullptr, nullptr};
  size_t len[4] = {0, 0, 0, 0};   // floats
  int nevents = 0;
  void line(const char *fmt, ...);
  // "name+offset" of p (or "?") into buf
  void ref(const float *p, char *buf, size_t n) const;
};
PlanRecorder *plan_recorder();
// stream handle -> index recorded in the plan (fake handles in recording mode)
int plan_stream_index(cudaStream_t s);
// outer block width of the factorisation of a d-wide layer (d: one block)
int64_t factor_outer_cols(int64_t d);
int launch_factor_plan(float *A, int64_t d, int64_t S, float *T1, bool use_side);

// The argument checks of gptq_quantize_layer other than the workspace's.
int check_layer_args(const float *W, int64_t r, int64_t d, const float *H, int bits, int group,
                     int block, float damp, int options, const float *W_hat,
                     const int32_t *qweight, const float *scales, const int32_t *zeros,
                     const int32_t *g_idx, const uint8_t *codes);
// gptq_quantize_layer; plain = true creates nothing (no CUDA graph, no second
// stream or events) and launches every kernel directly on `stream`.
int quantize_layer(const float *W, int64_t r, int64_t d, float *H, int bits, int group, int block,
                   float damp, int options, float *W_hat, int32_t *qweight, float *scales,
                   int32_t *zeros, int32_t *g_idx, uint8_t *codes, double *loss, void *workspace,
                   size_t workspace_bytes, gptq_stream_t stream, bool plain);

// SweepArgs::flags.  (The struct stays at 128 bytes: a larger kernel parameter
// block costs the sweep kernel about 35 registers.)
enum SweepFlags {
  SWEEP_SYM = 1,     // symmetric quantiser
  SWEEP_STATIC = 2   // parameters fixed before the sweep: read, never computed
};

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
  int flags;          // SWEEP_SYM | SWEEP_STATIC
  uint8_t *codes;     // r x d codes in sweep order, row stride ldw
  const int *perm;    // static groups under act-order: column j of the sweep is
                      // original column perm[j], of group perm[j] / group
  float *err;         // r x lde; column 0 is the block's first column
  int64_t lde;
  double *loss_rows;  // per-row running sum of e^2 / 2
  const int *status;
};

int launch_gather_w(const float *W, int r, int d, const int *perm, float *Wk, const int *status,
                    cudaStream_t stream);
// Per-row parameters of groups of g consecutive columns of Wsrc [r x d] (g = d:
// one group per row), G = d / g per row.
int launch_row_params(const float *Wsrc, int r, int d, int g, int bits, int sym, float *scales,
                      int32_t *zeros, const int *status, cudaStream_t stream);
int launch_sweep_block(const SweepArgs &a, int block, cudaStream_t stream);

struct FinalizeArgs {
  const float *W;       // original weights r x d
  const float *Wk;      // dequantised weights, sweep order
  const uint8_t *codes_p;
  const int *inv;       // inv[c] = sweep position of column c (NULL: identity)
  int r, d, bits, group;
  int static_groups;    // g_idx[c] = c / group even under act-order
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
