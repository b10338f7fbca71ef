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
// whose work is dense GEMMs with triangular operands, down to 128 x 128
// leaves that one CTA factors and inverts in shared memory (fp64).
#include "gptq_common.cuh"
#include "gptq_internal.h"

namespace gptq {
namespace {

// ---------------------------------------------------------------- damping

// One CTA: lambda = damp * mean(diag H) (fp64 sum in a fixed order); optionally
// add lambda to the diagonal of H in place.
__global__ void __launch_bounds__(1024) damp_kernel(float *H, int64_t ld, int d, float damp,
                                                    int add_in_place, float *lambda_out) {
  __shared__ double red[32];
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
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  const int a = blockIdx.y;
  if (b >= d) return;
  const int pa = perm[a], pb = perm[b];
  float v = H[(size_t)pa * ld + pb];
  if (a == b) v += *lambda;
  Hp[(size_t)a * d + b] = v;
}

// ---------------------------------------------------------------- leaf

constexpr int LEAF = 128;
constexpr int LEAF_LD = LEAF + 1;
constexpr int LEAF_THREADS = 512;
constexpr size_t LEAF_SMEM = (size_t)LEAF * LEAF_LD * sizeof(double);

// Factor one diagonal block in place: A (upper triangle, nb <= 128) -> U, the
// inverse of its reverse-order Cholesky factor, written as a full nb x nb
// block with zeros below the diagonal.  fp64 in shared memory.
//
// Step k = nb-1 .. 0 does, in order:
//   pivot:    r = sqrt(S[k][k])           (non-positive pivot -> GPTQ_ERR_NOT_PD)
//   column:   col[i] = S[i][k] / r (i < k)       -- column k of R
//             row[c] = S[k][c] / r (c > k), row[k] = 1 / r   -- row k of U
//   update:   S[i][j] -= col[i] col[j]  (i <= j < k)         -- Cholesky Schur update
//             S[m][c]  = (c == k ? 0 : S[m][c]) - col[m] row[c]  (m < k <= c)
//                                                            -- back-substitution of R U = I
//             S[k][c]  = row[c]  (c >= k)
// Columns >= k of rows < k hold the running right-hand sides of R U = I, and
// the Cholesky update only touches columns < k, so one array holds both.
__global__ void __launch_bounds__(LEAF_THREADS) leaf_kernel(float *A, int64_t lda, int nb,
                                                            int *status) {
  extern __shared__ double S[];
  __shared__ double col[LEAF], row[LEAF];
  __shared__ int fail;
  if (*(volatile int *)status) return;
  const int tid = threadIdx.x;
  for (int idx = tid; idx < nb * nb; idx += LEAF_THREADS) {
    const int i = idx / nb, j = idx - i * nb;
    S[i * LEAF_LD + j] = j >= i ? (double)A[(size_t)i * lda + j] : 0.0;
  }
  if (tid == 0) fail = 0;
  __syncthreads();
  const int jc = tid & (LEAF - 1);     // column this thread updates
  const int r0 = tid >> 7;             // first row; rows r0, r0+4, ...
  for (int k = nb - 1; k >= 0; --k) {
    const double p = S[k * LEAF_LD + k];
    if (!(p > 0.0)) {                  // NaN or non-positive pivot
      if (tid == 0) fail = 1;
      break;
    }
    const double r = sqrt(p);
    const double rinv = 1.0 / r;
    for (int i = tid; i < nb; i += LEAF_THREADS) {
      if (i < k) col[i] = S[i * LEAF_LD + k] / r;
      else if (i > k) row[i] = S[k * LEAF_LD + i] * rinv;
      else row[k] = rinv;
    }
    __syncthreads();
    if (jc < k) {
      const double cj = col[jc];
      for (int i = r0; i <= jc; i += 4) S[i * LEAF_LD + jc] -= col[i] * cj;
    } else if (jc < nb) {
      const double rc = row[jc];
      for (int m = r0; m < k; m += 4) {
        const double base = jc == k ? 0.0 : S[m * LEAF_LD + jc];
        S[m * LEAF_LD + jc] = base - col[m] * rc;
      }
      if (r0 == 0) S[k * LEAF_LD + jc] = rc;
    }
    __syncthreads();
  }
  __syncthreads();
  if (fail) {
    if (tid == 0) atomicCAS(status, 0, (int)GPTQ_ERR_NOT_PD);
    return;
  }
  for (int idx = tid; idx < nb * nb; idx += LEAF_THREADS) {
    const int i = idx / nb, j = idx - i * nb;
    A[(size_t)i * lda + j] = (float)S[i * LEAF_LD + j];
  }
}

}  // namespace

// ---------------------------------------------------------------- fp32 GEMM

namespace {

constexpr int GBM = 128, GBN = 128, GBK = 8;

// C = alpha * A * op(B) + beta * C, row-major fp32.  Tile 128 x 128, 256
// threads, 8 x 8 outputs per thread, double-buffered shared-memory K slices.
// Triangular operands are skipped at 128-tile granularity (their sub-diagonal
// blocks inside a tile must hold zeros); see GemmFlags.
template <bool TB>
__global__ void __launch_bounds__(256) sgemm_kernel(GemmArgs g) {
  if (g.status && *(volatile const int *)g.status) return;
  const int bn = blockIdx.x, bm = blockIdx.y;
  if ((g.flags & GEMM_UPPER_C) && bn < bm) return;
  const int m0 = bm * GBM, n0 = bn * GBN;
  int klo = 0, khi = g.K;
  if (g.flags & GEMM_KMIN_ROW) klo = max(klo, m0);
  if (g.flags & GEMM_KMIN_COL) klo = max(klo, n0);
  if (g.flags & GEMM_KMAX_COL) khi = min(khi, n0 + GBN);

  __shared__ __align__(16) float As[2][GBK][GBM];
  __shared__ __align__(16) float Bs[2][GBK][GBN];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  // global -> register staging
  const int a_row = tid >> 1, a_k = (tid & 1) * 4;
  const int b_k = tid >> 5, b_n = (tid & 31) * 4;   // !TB
  const int bt_n = tid >> 1, bt_k = (tid & 1) * 4;  // TB
  float4 ra, rb;

  auto load = [&](int k0) {
    const int gm = m0 + a_row;
    ra = (gm < g.M) ? *reinterpret_cast<const float4 *>(g.A + (size_t)gm * g.lda + k0 + a_k)
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    if (!TB) {
      const int gn = n0 + b_n;
      rb = (gn < g.N) ? *reinterpret_cast<const float4 *>(g.B + (size_t)(k0 + b_k) * g.ldb + gn)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    } else {
      const int gn = n0 + bt_n;
      rb = (gn < g.N) ? *reinterpret_cast<const float4 *>(g.B + (size_t)gn * g.ldb + k0 + bt_k)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  auto store = [&](int buf) {
    As[buf][a_k + 0][a_row] = ra.x;
    As[buf][a_k + 1][a_row] = ra.y;
    As[buf][a_k + 2][a_row] = ra.z;
    As[buf][a_k + 3][a_row] = ra.w;
    if (!TB) {
      *reinterpret_cast<float4 *>(&Bs[buf][b_k][b_n]) = rb;
    } else {
      Bs[buf][bt_k + 0][bt_n] = rb.x;
      Bs[buf][bt_k + 1][bt_n] = rb.y;
      Bs[buf][bt_k + 2][bt_n] = rb.z;
      Bs[buf][bt_k + 3][bt_n] = rb.w;
    }
  };

  if (klo < khi) {
    load(klo);
    store(0);
    __syncthreads();
    int buf = 0;
    for (int k0 = klo; k0 < khi; k0 += GBK) {
      const bool more = k0 + GBK < khi;
      if (more) load(k0 + GBK);
#pragma unroll
      for (int kk = 0; kk < GBK; ++kk) {
        const float4 a0 = *reinterpret_cast<const float4 *>(&As[buf][kk][ty * 4]);
        const float4 a1 = *reinterpret_cast<const float4 *>(&As[buf][kk][64 + ty * 4]);
        const float4 b0 = *reinterpret_cast<const float4 *>(&Bs[buf][kk][tx * 4]);
        const float4 b1 = *reinterpret_cast<const float4 *>(&Bs[buf][kk][64 + tx * 4]);
        const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
      }
      if (more) {
        store(buf ^ 1);
        __syncthreads();
        buf ^= 1;
      }
    }
  }

#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int gm = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
    if (gm >= g.M) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int gn = n0 + h * 64 + tx * 4;
      if (gn >= g.N) continue;
      float4 *cp = reinterpret_cast<float4 *>(g.C + (size_t)gm * g.ldc + gn);
      float4 c = g.beta != 0.f ? *cp : make_float4(0.f, 0.f, 0.f, 0.f);
      c.x = g.alpha * acc[i][h * 4 + 0] + g.beta * c.x;
      c.y = g.alpha * acc[i][h * 4 + 1] + g.beta * c.y;
      c.z = g.alpha * acc[i][h * 4 + 2] + g.beta * c.z;
      c.w = g.alpha * acc[i][h * 4 + 3] + g.beta * c.w;
      *cp = c;
    }
  }
}

}  // namespace

int launch_gemm(const GemmArgs &g, bool trans_b, cudaStream_t stream) {
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return GPTQ_OK;
  dim3 grid((g.N + GBN - 1) / GBN, (g.M + GBM - 1) / GBM);
  if (grid.y > 65535) return GPTQ_ERR_INVALID_ARG;
  if (trans_b)
    sgemm_kernel<true><<<grid, 256, 0, stream>>>(g);
  else
    sgemm_kernel<false><<<grid, 256, 0, stream>>>(g);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

// ---------------------------------------------------------------- host drivers

int launch_damp(float *H, int64_t ld, int d, float damp, bool add_in_place, float *lambda,
                cudaStream_t stream) {
  damp_kernel<<<1, 1024, 0, stream>>>(H, ld, d, damp, add_in_place ? 1 : 0, lambda);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

int launch_act_order(const float *H, int64_t ld, int d, int *perm, int *inv, const float *lambda,
                     float *Hp, cudaStream_t stream) {
  rank_kernel<<<(d + 255) / 256, 256, 0, stream>>>(H, ld, d, perm, inv);
  GPTQ_LAUNCH_CHECK();
  dim3 grid((d + 255) / 256, d);
  permute_sym_kernel<<<grid, 256, 0, stream>>>(H, ld, d, perm, lambda, Hp);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

size_t factor_scratch_floats(int64_t d) {
  const int64_t nblk = (d + LEAF - 1) / LEAF;
  if (nblk <= 1) return 0;
  const int64_t h = LEAF * (nblk / 2);
  return (size_t)h * (size_t)(d - h);
}

namespace {

int leaf(float *A, int64_t ld, int nb, int *status, cudaStream_t stream) {
  static bool attr_set = false;
  if (!attr_set) {
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(leaf_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)LEAF_SMEM));
    attr_set = true;
  }
  leaf_kernel<<<1, LEAF_THREADS, LEAF_SMEM, stream>>>(A, ld, nb, status);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

// Node [off, off+n) of the matrix A (leading dimension ld) -> U in place.
int potrf_inv(float *A, int64_t ld, int64_t off, int64_t n, float *T1, int *status,
              cudaStream_t stream) {
  const int64_t nblk = (n + LEAF - 1) / LEAF;
  if (nblk <= 1) return leaf(A + off * ld + off, ld, (int)n, status, stream);
  const int64_t h = LEAF * (nblk / 2);
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
  GPTQ_CUDA_TRY(cudaMemcpy2DAsync(A12, ld * sizeof(float), T1, m * sizeof(float),
                                  m * sizeof(float), h, cudaMemcpyDeviceToDevice, stream));
  return GPTQ_OK;
}

}  // namespace

int launch_factor(float *A, int64_t d, float *T1, int *status, cudaStream_t stream) {
  return potrf_inv(A, d, 0, d, T1, status, stream);
}

}  // namespace gptq
