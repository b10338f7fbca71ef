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

size_t factor_scratch_floats(int64_t d) {
  const int64_t nblk = (d + kLeaf - 1) / kLeaf;
  if (nblk <= 1) return 0;
  const int64_t h = kLeaf * (nblk / 2);
  return (size_t)h * (size_t)(d - h);
}

namespace {

// Node [off, off+n) of the matrix A (leading dimension ld) -> U in place.
int potrf_inv(float *A, int64_t ld, int64_t off, int64_t n, float *T1, int *status,
              cudaStream_t stream) {
  const int64_t nblk = (n + kLeaf - 1) / kLeaf;
  if (nblk <= 1) return launch_leaf(A + off * ld + off, ld, (int)n, status, stream);
  const int64_t h = kLeaf * (nblk / 2);
  const int64_t m = n - h;
  float *A11 = A + off * ld + off;
  float *A12 = A + off * ld + (off + h);
  float *A22 = A + (off + h) * ld + (off + h);
  int rc;
  if ((rc = potrf_inv(A, ld, off + h, m, T1, status, stream)) != GPTQ_OK) return rc;
  GemmArgs g{};
  g.status = status;
  // R12 = A12 U22^T   (U22^T is lower: k >= n)
  g = GemmArgs{(int)h, (int)m, (int)m, A12, ld, A22, ld, T1, m, 1.f, 0.f, GEMM_KMIN_COL, status};
  if ((rc = launch_gemm(g, true, stream)) != GPTQ_OK) return rc;
  // A11 -= R12 R12^T  (upper tiles)
  g = GemmArgs{(int)h, (int)h, (int)m, T1, m, T1, m, A11, ld, -1.f, 1.f, GEMM_UPPER_C, status};
  if ((rc = launch_gemm(g, true, stream)) != GPTQ_OK) return rc;
  // A12 <- R12 U22    (U22 upper: k <= n)
  g = GemmArgs{(int)h, (int)m, (int)m, T1, m, A22, ld, A12, ld, 1.f, 0.f, GEMM_KMAX_COL, status};
  if ((rc = launch_gemm(g, false, stream)) != GPTQ_OK) return rc;
  if ((rc = potrf_inv(A, ld, off, h, T1, status, stream)) != GPTQ_OK) return rc;
  // T1 = -U11 (R12 U22)   (U11 upper: k >= m)
  g = GemmArgs{(int)h, (int)m, (int)h, A11, ld, A12, ld, T1, m, -1.f, 0.f, GEMM_KMIN_ROW, status};
  if ((rc = launch_gemm(g, false, stream)) != GPTQ_OK) return rc;
  {
    const int64_t pieces = h * (m / 4);
    const int64_t cap = (int64_t)num_sms() * 8;
    const int blocks = (int)((pieces + 255) / 256 < cap ? (pieces + 255) / 256 : cap);
    GPTQ_LAUNCH_PDL(copy_block_kernel, dim3(blocks), dim3(256), 0, stream, A12, ld,
                    (const float *)T1, m, (int)h, (int)m, (const int *)status);
  }
  return GPTQ_OK;
}

}  // namespace

int launch_factor(float *A, int64_t d, float *T1, int *status, cudaStream_t stream) {
  return potrf_inv(A, d, 0, d, T1, status, stream);
}

}  // namespace gptq
