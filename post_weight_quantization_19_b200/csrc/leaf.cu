// Diagonal blocks of the inverse-Hessian factor: one CTA turns a <= 128 x 128
// block of H_d into U = R^-1, with H_d = R R^T and R upper (the Cholesky taken
// from the bottom-right corner).
//
// Source: the GPTQ reading card ("GPTQ: Accurate Post-Training Quantization
// for Generative Pre-trained Transformers", 方法适配) -- the needed rows of H^-1
// come from a Cholesky kernel; the "LLM 量化技术" blog §2.3 item 3.
//
// The block lives in shared memory (fp32, like the rest of the solve) and is
// processed by a 2 x 2 block recursion,
//     A22 -> U22;  T = A12 U22^T;  A11 -= T T^T;  A12 = T U22;
//     A11 -> U11;  A12 = -U11 A12,
// with register-tiled fp32 shared-memory products (all LT threads), down to
// blocks of at most BASE columns that CF_THREADS threads factor and invert one
// column per barrier (each thread keeps a small tile in registers).  The lower
// triangle is kept at zero between steps, so the triangular operands can be
// used as dense ones.  (Tensor-core products and two column steps per barrier
// were measured slower on the 4096-wide layer, by 0.03 ms and 0.25 ms.)  The
// recursion levels, the column factor and the products are separate
// (non-inlined) functions: the fully inlined kernel was four times the code
// and stalled on instruction fetch; sharing one copy of each took the 4096
// layer's factorisation from 2.42 to 2.32 ms.

#include "gptq_internal.h"

namespace gptq {
namespace {

typedef float real;                // leaf arithmetic
constexpr int LB = 128;            // largest block
constexpr int LLD = LB + 4;        // shared-memory leading dimension (16-byte rows)
constexpr int LT = 512;            // threads (the products; more loads in flight)
constexpr int GC = 16;             // column-factor thread grid: (CF_THREADS / GC) x GC tiles
constexpr int CF_THREADS = 256;    // threads of the column factor (a named barrier)
constexpr int BASE = 32;           // blocks up to this size go to the column factor
constexpr size_t LEAF_SMEM = ((size_t)LB * LLD + 64 * 68) * sizeof(real);

// Barrier of the column factor's threads only (warps 0 .. CF_THREADS/32 - 1).
__device__ __forceinline__ void cf_barrier() {
  if constexpr (CF_THREADS == LT)
    __syncthreads();
  else
    asm volatile("bar.sync 1, %0;" ::"n"(CF_THREADS) : "memory");
}


// C[M x N] = alpha * A[M x K] * op(B) + beta * C in shared memory, all shapes
// and strides known at compile time; op(B) = B (K x N) or B^T (B stored N x K).
// The M x N outputs are spread over all threads in RM x RN register tiles; A
// (and B^T) are read 4 k values at a time with 16-byte loads.  A thread's
// columns are interleaved (jt + TN c) when B is read transposed, so the B rows
// of neighbouring threads fall in different banks, and contiguous otherwise,
// for 16-byte loads of a B row.  UPPER: only entries with column >= row are
// written (C is a diagonal block).  Ends with a CTA barrier.
template <int M, int N, int K, int LDA, int LDB, int LDC, bool TB, bool UPPER>
__device__ __noinline__ void smem_gemm(real *C, const real *A, const real *B, real alpha,
                                          real beta) {
  static_assert(K % 4 == 0 && LDA % 4 == 0 && LDB % 4 == 0 && LDC % 4 == 0, "16-byte rows");
  constexpr int RM = (M * N >= 16 * LT) ? 4 : 2;
  constexpr int RN = (M * N >= 8 * LT) ? 4 : 2;
  constexpr int TN = N / RN;
  constexpr int NT = (M / RM) * TN;
  for (int tile = threadIdx.x; tile < NT; tile += LT) {
    const int i0 = (tile / TN) * RM, jt = tile % TN;
    auto col = [&](int c) { return TB ? jt + TN * c : jt * RN + c; };
    if (UPPER && col(RN - 1) < i0) continue;
    real acc[RM][RN];
#pragma unroll
    for (int r = 0; r < RM; ++r)
#pragma unroll
      for (int c = 0; c < RN; ++c) acc[r][c] = 0.f;
#pragma unroll 4
    for (int k = 0; k < K; k += 4) {
      float4 a4[RM];
#pragma unroll
      for (int r = 0; r < RM; ++r) a4[r] = *reinterpret_cast<const float4 *>(A + (i0 + r) * LDA + k);
      real a[RM][4];
#pragma unroll
      for (int r = 0; r < RM; ++r) {
        a[r][0] = a4[r].x;
        a[r][1] = a4[r].y;
        a[r][2] = a4[r].z;
        a[r][3] = a4[r].w;
      }
      real b[4][RN];
      if (TB) {
#pragma unroll
        for (int c = 0; c < RN; ++c) {
          const float4 v = *reinterpret_cast<const float4 *>(B + col(c) * LDB + k);
          b[0][c] = v.x;
          b[1][c] = v.y;
          b[2][c] = v.z;
          b[3][c] = v.w;
        }
      } else {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const real *br = B + (k + kk) * LDB + jt * RN;
          if constexpr (RN == 4) {
            const float4 v = *reinterpret_cast<const float4 *>(br);
            b[kk][0] = v.x;
            b[kk][1] = v.y;
            b[kk][2] = v.z;
            b[kk][3] = v.w;
          } else {
            const float2 v = *reinterpret_cast<const float2 *>(br);
            b[kk][0] = v.x;
            b[kk][1] = v.y;
          }
        }
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
#pragma unroll
        for (int r = 0; r < RM; ++r)
#pragma unroll
          for (int c = 0; c < RN; ++c) acc[r][c] = fmaf(a[r][kk], b[kk][c], acc[r][c]);
    }
#pragma unroll
    for (int r = 0; r < RM; ++r)
#pragma unroll
      for (int c = 0; c < RN; ++c) {
        if (UPPER && col(c) < i0 + r) continue;
        real *p = C + (i0 + r) * LDC + col(c);
        *p = alpha * acc[r][c] + (beta != 0.f ? beta * *p : 0.f);
      }
  }
  __syncthreads();
}

// Column factor of an N x N block at S (leading dimension LLD, N = 32 or 64)
// by CF_THREADS threads: H_d = R R^T with R upper, overwritten by U = R^-1.
// Thread (gr, gc) of a (CF_THREADS / GC) x GC grid keeps the TR x TC tile at rows
// gr * TR, columns gc * TC in registers.  Step k = N-1 .. 0 reads a vector v
// that holds column k above the diagonal (v_j = S[j][k], j < k), the pivot
// p = S[k][k] at index k and row k right of the diagonal (v_j = S[k][j],
// j > k).  With v_k taken as 1,
//   rows i < k:  S[i][j] <- (j == k ? 0 : S[i][j]) - S[i][k] v_j / p
//   row  k:      S[k][j] <- v_j / sqrt(p)
// i.e. the Cholesky update of the leading block together with the
// substitution that turns the finished rows into rows of R^-1.  Rows below k
// are final; entries below the diagonal may pick up junk on the way and are
// zeroed when the tile is written back.  The owners of column k-1 and row k-1
// publish the next vector into the other half of a double buffer, so a step
// costs one CTA barrier.  Returns false (in every thread) on a non-positive
// pivot.
template <int N>
__device__ __noinline__ bool col_factor(real *S, real *vbuf) {
  __shared__ int cf_ok;
  if (threadIdx.x >= CF_THREADS) {   // the other warps wait at the closing barrier
    __syncthreads();
    return cf_ok != 0;
  }
  constexpr int GR = CF_THREADS / GC;
  constexpr int TR = N / GR, TC = N / GC;
  static_assert(TR >= 1 && TC >= 1 && TR * GR == N && TC * GC == N, "tile grid");
  const int gr = threadIdx.x / GC, gc = threadIdx.x % GC;
  const int i0 = gr * TR, j0 = gc * TC;
  const bool owner = j0 + TC - 1 >= i0;   // the tile reaches the upper triangle
  real t[TR][TC];
#pragma unroll
  for (int r = 0; r < TR; ++r)
#pragma unroll
    for (int q = 0; q < TC; ++q) t[r][q] = owner ? S[(i0 + r) * LLD + j0 + q] : 0.f;
  if (owner && j0 + TC == N) {
#pragma unroll
    for (int r = 0; r < TR; ++r) vbuf[((N - 1) & 1) * N + i0 + r] = t[r][TC - 1];
  }
  cf_barrier();
  bool bad = false;
  // Fully unrolled: every comparison with k below becomes static.
#pragma unroll
  for (int k = N - 1; k >= 0; --k) {
    const real *vb = vbuf + (k & 1) * N;
    real p = vb[k];
    bad |= !(p > 0.f);
    p = bad ? 1.f : p;
    real ri = rsqrtf(p);
    ri = ri * fmaf(-0.5f * p * ri, ri, 1.5f);   // one Newton step
    if (owner && i0 <= k) {
      const real mip = -ri * ri;
      real c[TR], v[TC];
#pragma unroll
      for (int r = 0; r < TR; ++r) c[r] = i0 + r < k ? vb[i0 + r] * mip : 0.f;
#pragma unroll
      for (int q = 0; q < TC; ++q) v[q] = j0 + q == k ? 1.f : vb[j0 + q];
#pragma unroll
      for (int r = 0; r < TR; ++r)
#pragma unroll
        for (int q = 0; q < TC; ++q) t[r][q] = fmaf(c[r], v[q], j0 + q == k ? 0.f : t[r][q]);
#pragma unroll
      for (int r = 0; r < TR; ++r)
        if (i0 + r == k) {
#pragma unroll
          for (int q = 0; q < TC; ++q) t[r][q] = v[q] * ri;
        }
      const int kn = k - 1;
      if (kn >= 0) {
        real *nb = vbuf + (kn & 1) * N;
#pragma unroll
        for (int r = 0; r < TR; ++r)
#pragma unroll
          for (int q = 0; q < TC; ++q) {
            if (j0 + q == kn && i0 + r <= kn) nb[i0 + r] = t[r][q];
            if (i0 + r == kn && j0 + q > kn) nb[j0 + q] = t[r][q];
          }
      }
    }
    cf_barrier();
  }
  if (owner) {
#pragma unroll
    for (int r = 0; r < TR; ++r)
#pragma unroll
      for (int q = 0; q < TC; ++q)
        S[(i0 + r) * LLD + j0 + q] = j0 + q >= i0 + r ? t[r][q] : 0.f;
  }
  if (threadIdx.x == 0) cf_ok = !bad;
  __syncthreads();
  return !bad;
}

// Node [off, off + N) of the shared-memory block.  N is a compile-time size
// (32, 64, 96 or 128), so the recursion unfolds at compile time and uses no
// call stack.
template <int N>
__device__ __noinline__ bool node_factor(real *S, real *T, real *vbuf, int off) {
  if constexpr (N <= BASE) {
    return col_factor<N>(S + off * LLD + off, vbuf);
  } else {
    constexpr int h = 32 * ((N / 32) / 2), m = N - h;
    if (!node_factor<m>(S, T, vbuf, off + h)) return false;
    real *A11 = S + off * LLD + off;
    real *A12 = S + off * LLD + off + h;
    const real *U22 = S + (off + h) * LLD + off + h;
    // T (h x m): leading dimension m + 4, so rows stay 16-byte aligned and
    // the rows that neighbouring threads read transposed fall in different banks.
    constexpr int LT_ = m + 4;
      smem_gemm<h, m, m, LLD, LLD, LT_, true, false>(T, A12, U22, 1.f, 0.f);
      smem_gemm<h, h, m, LT_, LT_, LLD, true, true>(A11, T, T, -1.f, 1.f);
      smem_gemm<h, m, m, LT_, LLD, LLD, false, false>(A12, T, U22, 1.f, 0.f);
    if (!node_factor<h>(S, T, vbuf, off)) return false;
      smem_gemm<h, m, h, LLD, LLD, LT_, false, false>(T, A11, A12, -1.f, 0.f);
    for (int idx = threadIdx.x; idx < h * m; idx += LT) {
      const int r = idx / m, c = idx - r * m;
      A12[r * LLD + c] = T[r * LT_ + c];
    }
    __syncthreads();
    return true;
  }
}

__global__ void __launch_bounds__(LT) leaf_kernel(float *A, int64_t lda, int nb, int *status) {
  extern __shared__ real lsm[];
  __shared__ real vbuf[4 * BASE];   // two published pairs of vectors
  pdl_wait_then_release();
  if (*(volatile int *)status) return;
  real *S = lsm;
  real *T = lsm + LB * LLD;
  // 16-byte loads, all issued before any is used (nb and lda are multiples of 32).
#pragma unroll 16
  for (int idx = threadIdx.x; idx < LB * (LB / 4); idx += LT) {
    const int i = idx >> 5, j = (idx & 31) * 4;
    if (i < nb && j < nb) {
      const float4 v = *reinterpret_cast<const float4 *>(A + (size_t)i * lda + j);
      *reinterpret_cast<float4 *>(S + i * LLD + j) =
          make_float4(j + 0 >= i ? v.x : 0.f, j + 1 >= i ? v.y : 0.f, j + 2 >= i ? v.z : 0.f,
                      j + 3 >= i ? v.w : 0.f);
    }
  }
  __syncthreads();
  bool ok;
  switch (nb) {
    case 32: ok = node_factor<32>(S, T, vbuf, 0); break;
    case 64: ok = node_factor<64>(S, T, vbuf, 0); break;
    case 96: ok = node_factor<96>(S, T, vbuf, 0); break;
    default: ok = node_factor<128>(S, T, vbuf, 0); break;
  }
  if (!ok) {
    if (threadIdx.x == 0) atomicCAS(status, 0, (int)GPTQ_ERR_NOT_PD);
    return;
  }
#pragma unroll 4
  for (int idx = threadIdx.x; idx < LB * (LB / 4); idx += LT) {
    const int i = idx >> 5, j = (idx & 31) * 4;
    if (i < nb && j < nb)
      *reinterpret_cast<float4 *>(A + (size_t)i * lda + j) =
          *reinterpret_cast<const float4 *>(S + i * LLD + j);
  }
}

}  // namespace

int launch_leaf(float *A, int64_t ld, int nb, int *status, cudaStream_t stream) {
  if (nb <= 0 || nb > LB || nb % 32 != 0) return GPTQ_ERR_INVALID_ARG;
  if (PlanRecorder *rec = plan_recorder()) {
    char a[64];
    rec->ref(A, a, sizeof a);
    rec->line("L s=%d A=%s ld=%lld nb=%d\n", plan_stream_index(stream), a, (long long)ld, nb);
    return GPTQ_OK;
  }
  static std::atomic<bool> attr[64] = {};
  if (const int rc = ensure_smem_attr(leaf_kernel, LEAF_SMEM, attr)) return rc;
  GPTQ_LAUNCH_PDL(leaf_kernel, dim3(1), dim3(LT), LEAF_SMEM, stream, A, ld, nb, status);
  return GPTQ_OK;
}

}  // namespace gptq
