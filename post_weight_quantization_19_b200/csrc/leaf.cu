// Diagonal blocks of the inverse-Hessian factor: one CTA turns a <= 128 x 128
// block of H_d into U = R^-1, with H_d = R R^T and R upper (the Cholesky taken
// from the bottom-right corner).
//
// Source: the GPTQ reading card ("GPTQ: Accurate Post-Training Quantization
// for Generative Pre-trained Transformers", 方法适配) -- the needed rows of H^-1
// come from a Cholesky kernel; the "LLM 量化技术" blog §2.3 item 3.
//
// The block lives in shared memory (fp32, like the rest of the solve) and is
// processed by the same 2 x 2
// block recursion as the full matrix,
//     A22 -> U22;  T = A12 U22^T;  A11 -= T T^T;  A12 = T U22;
//     A11 -> U11;  A12 = -U11 A12,
// with register-tiled shared-memory products run by all 256 threads, down to
// 32 x 32 blocks that a single warp factors and inverts in registers (one row
// per lane, every index static, shuffles instead of CTA barriers).  The lower
// triangle is kept at zero throughout, so the triangular operands can be used
// as dense ones.
#include "gptq_internal.h"

namespace gptq {
namespace {

typedef float real;                // leaf arithmetic
constexpr int LB = 128;            // largest block
constexpr int LLD = LB + 1;        // shared-memory leading dimension
constexpr int LT = 256;            // threads (255 registers each for the warp factor)
constexpr size_t LEAF_SMEM = ((size_t)LB * LLD + 64 * 64) * sizeof(real);

// C[M x N] = alpha * A[M x K] * op(B) + beta * C in shared memory, all shapes
// and strides known at compile time; op(B) = B (K x N) or B^T (B stored N x K).
// The M x N outputs are spread over all threads in RM x RN register tiles.
// UPPER: only entries with column >= row are written (C is a diagonal block).
// Ends with a CTA barrier.
template <int M, int N, int K, int LDA, int LDB, int LDC, bool TB, bool UPPER>
__device__ __forceinline__ void smem_gemm(real *C, const real *A, const real *B, real alpha,
                                          real beta) {
  constexpr int RM = (M * N >= 16 * LT) ? 4 : 2;
  constexpr int RN = (M * N >= 8 * LT) ? 4 : 2;
  constexpr int TN = N / RN;
  constexpr int NT = (M / RM) * TN;
  for (int tile = threadIdx.x; tile < NT; tile += LT) {
    const int i0 = (tile / TN) * RM, j0 = (tile % TN) * RN;
    if (UPPER && j0 + RN - 1 < i0) continue;
    real acc[RM][RN];
#pragma unroll
    for (int r = 0; r < RM; ++r)
#pragma unroll
      for (int c = 0; c < RN; ++c) acc[r][c] = 0.f;
#pragma unroll 16
    for (int k = 0; k < K; ++k) {
      real a[RM], b[RN];
#pragma unroll
      for (int r = 0; r < RM; ++r) a[r] = A[(i0 + r) * LDA + k];
#pragma unroll
      for (int c = 0; c < RN; ++c) b[c] = TB ? B[(j0 + c) * LDB + k] : B[k * LDB + j0 + c];
#pragma unroll
      for (int r = 0; r < RM; ++r)
#pragma unroll
        for (int c = 0; c < RN; ++c) acc[r][c] = fmaf(a[r], b[c], acc[r][c]);
    }
#pragma unroll
    for (int r = 0; r < RM; ++r)
#pragma unroll
      for (int c = 0; c < RN; ++c) {
        if (UPPER && j0 + c < i0 + r) continue;
        real *p = C + (i0 + r) * LDC + j0 + c;
        *p = alpha * acc[r][c] + (beta != 0.f ? beta * *p : 0.f);
      }
  }
  __syncthreads();
}

// One warp: 32 x 32 block S (upper triangle, zeros below) -> U = R^-1.
// Lane i holds row i.  Step k = 31..0 with p = S[k][k]:
//   Cholesky update   S[i][j] -= S[i][k] S[j][k] / p          (i <= j < k)
//   right-hand sides  S[i][c]  = (c == k ? 0 : S[i][c]) - S[i][k] (c == k ? 1 : S[k][c]) / p
//                                                              (i < k <= c)
//   row k             S[k][c]  = (c == k ? 1 : S[k][c]) / sqrt(p)   (c >= k)
// Returns false (for every lane) on a non-positive pivot.
__device__ __noinline__ bool warp_factor32(real *S, int ld) {
  // The caller's tile loops may leave the warp split into divergent groups; a
  // split warp would run every shuffle below once per group.
  __syncwarp();
  const int i = threadIdx.x & 31;
  real d[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) d[j] = j >= i ? S[i * ld + j] : 0.f;
  bool bad = false;
#pragma unroll
  for (int k = 31; k >= 0; --k) {
    real p = __shfl_sync(0xffffffffu, d[k], k);
    bad |= !(p > 0.f);
    p = bad ? 1.f : p;
    real ri = rsqrtf(p);
    ri = ri * fmaf(-0.5f * p * ri, ri, 1.5f);   // one Newton step
    const real ri2 = ri * ri;
    const real ck = d[k];
    // Descending j: the next pivot (row k-1, column k-1) is updated first.
#pragma unroll
    for (int j = k - 1; j >= 0; --j) {
      const real cj = __shfl_sync(0xffffffffu, d[k], j);
      if (i <= j) d[j] = fmaf(-ck * ri2, cj, d[j]);
    }
#pragma unroll
    for (int c = k; c < 32; ++c) {
      const real rc = __shfl_sync(0xffffffffu, d[c], k);
      if (i < k) {
        d[c] = fmaf(-ck * ri2, c == k ? 1.f : rc, c == k ? 0.f : d[c]);
      } else if (i == k) {
        d[c] = (c == k ? 1.f : rc) * ri;
      }
    }
  }
#pragma unroll
  for (int j = 0; j < 32; ++j) S[i * ld + j] = d[j];
  return !bad;
}

// Node [off, off + N) of the shared-memory block.  N is a compile-time size
// (32, 64, 96 or 128), so the recursion unfolds at compile time and uses no
// call stack.
template <int N>
__device__ __forceinline__ bool node_factor(real *S, real *T, int off, bool *fail) {
  if constexpr (N == 32) {
    if (threadIdx.x < 32) {
      const bool ok = warp_factor32(S + off * LLD + off, LLD);
      if (threadIdx.x == 0 && !ok) *fail = true;
    }
    __syncthreads();
    return !*fail;
  } else {
    constexpr int h = 32 * ((N / 32) / 2), m = N - h;
    if (!node_factor<m>(S, T, off + h, fail)) return false;
    real *A11 = S + off * LLD + off;
    real *A12 = S + off * LLD + off + h;
    const real *U22 = S + (off + h) * LLD + off + h;
    smem_gemm<h, m, m, LLD, LLD, m, true, false>(T, A12, U22, 1.f, 0.f);      // R12 = A12 U22^T
    smem_gemm<h, h, m, m, m, LLD, true, true>(A11, T, T, -1.f, 1.f);          // A11 -= R12 R12^T
    smem_gemm<h, m, m, m, LLD, LLD, false, false>(A12, T, U22, 1.f, 0.f);     // A12 = R12 U22
    if (!node_factor<h>(S, T, off, fail)) return false;
    smem_gemm<h, m, h, LLD, LLD, m, false, false>(T, A11, A12, -1.f, 0.f);    // T = -U11 A12
    for (int idx = threadIdx.x; idx < h * m; idx += LT) {
      const int r = idx / m, c = idx - r * m;
      A12[r * LLD + c] = T[r * m + c];
    }
    __syncthreads();
    return true;
  }
}

__global__ void __launch_bounds__(LT) leaf_kernel(float *A, int64_t lda, int nb, int *status) {
  extern __shared__ real lsm[];
  __shared__ bool fail;
  if (*(volatile int *)status) return;
  real *S = lsm;
  real *T = lsm + LB * LLD;
  // 16-byte loads, all issued before any is used (nb and lda are multiples of 32).
#pragma unroll 16
  for (int idx = threadIdx.x; idx < LB * (LB / 4); idx += LT) {
    const int i = idx >> 5, j = (idx & 31) * 4;
    if (i < nb && j < nb) {
      const float4 v = *reinterpret_cast<const float4 *>(A + (size_t)i * lda + j);
      real *s = S + i * LLD + j;
      s[0] = j + 0 >= i ? v.x : 0.f;
      s[1] = j + 1 >= i ? v.y : 0.f;
      s[2] = j + 2 >= i ? v.z : 0.f;
      s[3] = j + 3 >= i ? v.w : 0.f;
    }
  }
  if (threadIdx.x == 0) fail = false;
  __syncthreads();
  bool ok;
  switch (nb) {
    case 32: ok = node_factor<32>(S, T, 0, &fail); break;
    case 64: ok = node_factor<64>(S, T, 0, &fail); break;
    case 96: ok = node_factor<96>(S, T, 0, &fail); break;
    default: ok = node_factor<128>(S, T, 0, &fail); break;
  }
  if (!ok) {
    if (threadIdx.x == 0) atomicCAS(status, 0, (int)GPTQ_ERR_NOT_PD);
    return;
  }
#pragma unroll 4
  for (int idx = threadIdx.x; idx < LB * (LB / 4); idx += LT) {
    const int i = idx >> 5, j = (idx & 31) * 4;
    if (i < nb && j < nb) {
      const real *s = S + i * LLD + j;
      *reinterpret_cast<float4 *>(A + (size_t)i * lda + j) = make_float4(s[0], s[1], s[2], s[3]);
    }
  }
}

}  // namespace

int launch_leaf(float *A, int64_t ld, int nb, int *status, cudaStream_t stream) {
  if (nb <= 0 || nb > LB || nb % 32 != 0) return GPTQ_ERR_INVALID_ARG;
  static bool attr = false;
  if (!attr) {
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(leaf_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)LEAF_SMEM));
    attr = true;
  }
  leaf_kernel<<<1, LT, LEAF_SMEM, stream>>>(A, ld, nb, status);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

}  // namespace gptq
