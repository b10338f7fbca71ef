// Damping, act-order and the inverse-Hessian factor U (U^T U = H_d^-1).
//
// Sources: the GPTQ reading card ("GPTQ: Accurate Post-Training Quantization
// for Generative Pre-trained Transformers", 方法适配) -- a Cholesky kernel
// precomputes the needed rows of H^-1, with mild damping, for numerical
// stability; the "LLM 量化技术" blog §2.3 item 3 -- Cholesky instead of an
// explicit inverse; the reading card's "any fixed order" for act-order.
//
// Route: H_d = R R^T with R upper (a Cholesky taken from the bottom-right
// corner), then U = R^-1, which is upper and satisfies U^T U = H_d^-1, i.e. U
// is exactly the upper Cholesky factor of H_d^-1 that GPTQ needs.  Both are
// computed together by a recursion on 2 x 2 block partitions
//     [A11 A12; . A22]:  A22 -> U22;  R12 = A12 U22^T;  A11 -= R12 R12^T;
//                        A11 -> U11;  U12 = -U11 R12 U22
// whose work is dense GEMMs with triangular operands (tensor cores, 3xTF32,
// gemm_tc.cu), down to 128 x 128 leaves that one CTA factors and inverts in
// registers (fp64).
#include <mutex>
#include <vector>

#include "gptq_common.cuh"
#include "gptq_internal.h"

namespace gptq {
namespace {

constexpr int64_t kLeaf = 128;   // diagonal block handled by one CTA (leaf.cu)

// ---------------------------------------------------------------- damping

// One CTA: lambda = damp * mean(diag H) (fp64 sum in a fixed order); optionally
// add lambda to the diagonal of H in place.
__global__ void __launch_bounds__(1024) damp_kernel(float *H, int64_t ld, int d, float damp,
                                                    int add_in_place, float *lambda_out) {
  __shared__ double red[32];
  pdl_wait_then_release();
  double s = 0.0;
  for (int i = threadIdx.x; i < d; i += blockDim.x) s += (double)H[(size_t)i * ld + i];
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    double v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0;
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float lam = (float)((double)damp * red[0] / (double)d);
  if (threadIdx.x == 0) *lambda_out = lam;
  if (add_in_place)
    for (int i = threadIdx.x; i < d; i += blockDim.x) H[(size_t)i * ld + i] += lam;
}

// ---------------------------------------------------------------- act-order

// Stable descending order of diag(H): rank(i) = #{k : h_k > h_i or (h_k == h_i and k < i)}.
// perm[rank(i)] = i and inv[i] = rank(i).  O(d^2) comparisons, exact and
// deterministic (no tie depends on thread timing).
__global__ void __launch_bounds__(256) rank_kernel(const float *H, int64_t ld, int d, int *perm,
                                                   int *inv) {
  __shared__ float tile[1024];
  pdl_wait_then_release();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const float hi = i < d ? H[(size_t)i * ld + i] : 0.f;
  int rank = 0;
  for (int k0 = 0; k0 < d; k0 += 1024) {
    __syncthreads();
    for (int k = threadIdx.x; k < 1024 && k0 + k < d; k += blockDim.x)
      tile[k] = H[(size_t)(k0 + k) * ld + (k0 + k)];
    __syncthreads();
    const int kn = min(1024, d - k0);
    if (i < d)
      for (int k = 0; k < kn; ++k) {
        const float hk = tile[k];
        rank += (hk > hi) || (hk == hi && k0 + k < i);
      }
  }
  if (i < d) {
    perm[rank] = i;
    inv[i] = rank;
  }
}

// Hp[a][b] = H[perm[a]][perm[b]] (+ lambda on the diagonal).
__global__ void permute_sym_kernel(const float *H, int64_t ld, int d, const int *perm,
                                   const float *lambda, float *Hp) {
  pdl_wait_then_release();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  const int a = blockIdx.y;
  if (b >= d) return;
  const int pa = perm[a], pb = perm[b];
  float v = H[(size_t)pa * ld + pb];
  if (a == b) v += *lambda;
  Hp[(size_t)a * d + b] = v;
}

// dst[i][j] = src[i][j] for a rows x cols block (cols a multiple of 4, rows
// 16-byte aligned).
__global__ void copy_block_kernel(float *dst, int64_t ldd, const float *src, int64_t lds, int rows,
                                  int cols, const int *status) {
  pdl_wait_then_release();
  if (*(volatile const int *)status) return;
  const int q = cols / 4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < (int64_t)rows * q;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / q;
    const int c = (int)(i - r * q) * 4;
    *reinterpret_cast<float4 *>(dst + r * ldd + c) =
        *reinterpret_cast<const float4 *>(src + r * lds + c);
  }
}

}  // namespace

// ---------------------------------------------------------------- host drivers

int launch_damp(float *H, int64_t ld, int d, float damp, bool add_in_place, float *lambda,
                cudaStream_t stream) {
  GPTQ_LAUNCH_PDL(damp_kernel, dim3(1), dim3(1024), 0, stream, H, ld, d, damp,
                  add_in_place ? 1 : 0, lambda);
  return GPTQ_OK;
}

int launch_act_order(const float *H, int64_t ld, int d, int *perm, int *inv, const float *lambda,
                     float *Hp, cudaStream_t stream) {
  GPTQ_LAUNCH_PDL(rank_kernel, dim3((d + 255) / 256), dim3(256), 0, stream, H, ld, d, perm, inv);
  dim3 grid((d + 255) / 256, d);
  GPTQ_LAUNCH_PDL(permute_sym_kernel, grid, dim3(256), 0, stream, H, ld, d, (const int *)perm,
                  lambda, Hp);
  return GPTQ_OK;
}

int launch_priority(bool background) {
  static int least = 0, greatest = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) least = greatest = 0;
  });
  return background ? least : greatest;
}

namespace {

// Node sizes of the recursion: a node of n columns (nblk = ceil(n/128)
// blocks) splits into h = 128 * floor(nblk/2) leading and m = n - h trailing
// columns.  The largest node of each depth is the trailing child of the
// largest node of the depth above.
void split(int64_t n, int64_t *h, int64_t *m) {
  const int64_t nblk = (n + kLeaf - 1) / kLeaf;
  *h = kLeaf * (nblk / 2);
  *m = n - *h;
}

}  // namespace

size_t factor_scratch_floats(int64_t d) {
  size_t total = 0;
  for (int64_t n = d; (n + kLeaf - 1) / kLeaf > 1;) {
    int64_t h, m;
    split(n, &h, &m);
    total += (size_t)h * (size_t)m;
    n = m;
  }
  return total;
}

namespace {

// Per-device stream for the background products, and events to fork and
// join it (two per recursion node).
struct SideStream {
  cudaStream_t s = nullptr;
  std::vector<cudaEvent_t> ev;
};

int side_stream(int64_t d, SideStream **out) {
  static SideStream side[64];
  static std::mutex mu;
  int dev = 0;
  GPTQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return GPTQ_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(mu);
  SideStream &ss = side[dev];
  if (!ss.s) GPTQ_CUDA_TRY(cudaStreamCreateWithPriority(&ss.s, cudaStreamNonBlocking,
                                                        launch_priority(true)));
  const size_t need = 2 * (size_t)((d + kLeaf - 1) / kLeaf);
  while (ss.ev.size() < need) {
    cudaEvent_t e;
    GPTQ_CUDA_TRY(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
    ss.ev.push_back(e);
  }
  *out = &ss;
  return GPTQ_OK;
}

struct FactorRun {
  float *A;
  int64_t ld;
  float *scratch;                  // factor_scratch_floats(d) floats
  std::vector<size_t> depth_off;   // offset of each depth's product in scratch
  int *status;
  cudaStream_t stream;
  SideStream *side;
  size_t next_ev;
};

// Node [off, off+n) of A -> U in place.
//   A22 -> U22 (recursively);  T = A12 U22^T;  A11 -= T T^T;  P = T U22;
//   A11 -> U11 (recursively);  A12 = -U11 P.
// P does not depend on U11, so when the node is square (h == m) it is formed
// on the side stream, at the least priority, while A11 is factored, and it is
// stored in the node's strictly lower block A21 (h x m there, scratch), so
// the last product writes A12 directly.  T lives in its depth's scratch,
// which the A11 subtree (one depth down) does not touch.
int potrf_inv(FactorRun &fr, int64_t off, int64_t n, int depth) {
  const int64_t nblk = (n + kLeaf - 1) / kLeaf;
  float *A = fr.A;
  const int64_t ld = fr.ld;
  if (nblk <= 1) return launch_leaf(A + off * ld + off, ld, (int)n, fr.status, fr.stream);
  int64_t h, m;
  split(n, &h, &m);
  float *A11 = A + off * ld + off;
  float *A12 = A + off * ld + (off + h);
  float *A21 = A + (off + h) * ld + off;
  float *A22 = A + (off + h) * ld + (off + h);
  float *T = fr.scratch + fr.depth_off[depth];
  int *status = fr.status;
  cudaStream_t st = fr.stream;
  int rc;
  if ((rc = potrf_inv(fr, off + h, m, depth + 1)) != GPTQ_OK) return rc;
  // T = A12 U22^T   (U22^T is lower: k >= n)
  GemmArgs g{(int)h, (int)m, (int)m, A12, ld, A22, ld, T, m, 1.f, 0.f, GEMM_KMIN_COL, status};
  if ((rc = launch_gemm(g, true, st)) != GPTQ_OK) return rc;
  // A11 -= T T^T  (upper tiles)
  g = GemmArgs{(int)h, (int)h, (int)m, T, m, T, m, A11, ld, -1.f, 1.f, GEMM_UPPER_C, status};
  if ((rc = launch_gemm(g, true, st)) != GPTQ_OK) return rc;
  if (h == m && fr.side) {
    cudaEvent_t fork = fr.side->ev[fr.next_ev++], join = fr.side->ev[fr.next_ev++];
    GPTQ_CUDA_TRY(cudaEventRecord(fork, st));
    GPTQ_CUDA_TRY(cudaStreamWaitEvent(fr.side->s, fork, 0));
    // P = T U22 into A21   (U22 upper: k <= n)
    g = GemmArgs{(int)h, (int)m, (int)m, T, m, A22, ld, A21, ld, 1.f, 0.f, GEMM_KMAX_COL, status,
                 true};
    if ((rc = launch_gemm(g, false, fr.side->s)) != GPTQ_OK) return rc;
    GPTQ_CUDA_TRY(cudaEventRecord(join, fr.side->s));
    if ((rc = potrf_inv(fr, off, h, depth + 1)) != GPTQ_OK) return rc;
    GPTQ_CUDA_TRY(cudaStreamWaitEvent(st, join, 0));
    // A12 = -U11 P   (U11 upper: k >= m)
    g = GemmArgs{(int)h, (int)m, (int)h, A11, ld, A21, ld, A12, ld, -1.f, 0.f, GEMM_KMIN_ROW,
                 status};
    return launch_gemm(g, false, st);
  }
  // A12 <- T U22
  g = GemmArgs{(int)h, (int)m, (int)m, T, m, A22, ld, A12, ld, 1.f, 0.f, GEMM_KMAX_COL, status};
  if ((rc = launch_gemm(g, false, st)) != GPTQ_OK) return rc;
  if ((rc = potrf_inv(fr, off, h, depth + 1)) != GPTQ_OK) return rc;
  // T = -U11 A12, then A12 <- T
  g = GemmArgs{(int)h, (int)m, (int)h, A11, ld, A12, ld, T, m, -1.f, 0.f, GEMM_KMIN_ROW, status};
  if ((rc = launch_gemm(g, false, st)) != GPTQ_OK) return rc;
  const int64_t pieces = h * (m / 4);
  const int64_t cap = (int64_t)num_sms() * 8;
  const int blocks = (int)((pieces + 255) / 256 < cap ? (pieces + 255) / 256 : cap);
  GPTQ_LAUNCH_PDL(copy_block_kernel, dim3(blocks), dim3(256), 0, st, A12, ld, (const float *)T, m,
                  (int)h, (int)m, (const int *)status);
  return GPTQ_OK;
}

}  // namespace

int launch_factor(float *A, int64_t d, float *T1, int *status, cudaStream_t stream,
                  bool use_side) {
  FactorRun fr{A, d, T1, {}, status, stream, nullptr, 0};
  size_t off = 0;
  for (int64_t n = d; (n + kLeaf - 1) / kLeaf > 1;) {
    int64_t h, m;
    split(n, &h, &m);
    fr.depth_off.push_back(off);
    off += (size_t)h * (size_t)m;
    n = m;
  }
  if (use_side && !fr.depth_off.empty()) {
    const int rc = side_stream(d, &fr.side);
    if (rc != GPTQ_OK) return rc;
  }
  return potrf_inv(fr, 0, d, 0);
}

}  // namespace gptq
