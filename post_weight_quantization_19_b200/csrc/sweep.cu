// Column sweep of GPTQ: quantise column by column with OBS error compensation.
//
// Sources: "GPTQ：一键量化大模型压缩" §误差补偿 (after a column is rounded the
// not-yet-quantised weights of the row move along the inverse-Hessian
// direction) and §分组方案 (per-group min-max scale and zero); the "LLM 量化技术"
// blog §1.2 (x_q = round(x/s + z), dequantised s (x_q - z)) and §2.3 (fixed
// column order shared by all rows; blocks of B = 128 columns); the GPTQ reading
// card 方法适配 (updates inside a block are exact, the global update is deferred
// to the block's end).
//
// With U the upper Cholesky factor of H_d^-1, column j of every row does
//   q = clamp(rint(w_j / s) + z, 0, 2^b - 1),  w^_j = s (q - z),
//   e_j = (w_j - w^_j) / U_jj,  w_{j+1..} -= e_j U[j, j+1..].
// Rows are independent, so one warp owns one row of the current block: lane l
// holds columns l*V .. l*V+V-1 (V = B/32) in registers, the block of U sits in
// shared memory, and each step is one shuffle (broadcast w_j), the quantiser,
// and V fused multiply-adds per lane.  No inter-warp synchronisation at all.
#include <float.h>

#include "gptq_internal.h"
#include "pack_bits.cuh"

namespace gptq {
namespace {

constexpr int SWEEP_THREADS = 512;
constexpr int SWEEP_WARPS = SWEEP_THREADS / 32;

__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Asymmetric min-max parameters over a range [lo, hi] widened to include 0:
// s = (xmax - xmin)/(2^b - 1) (1 for an empty range), z = rint(-xmin/s).
__device__ __forceinline__ void minmax_params(float lo, float hi, float maxq, float &s, float &z) {
  const float xmin = fminf(lo, 0.f), xmax = fmaxf(hi, 0.f);
  s = (xmax == xmin) ? 1.f : __fdiv_rn(xmax - xmin, maxq);
  z = rintf(__fdiv_rn(-xmin, s));
}

// 1/s rounded to nearest; w * (1/s) is within about one ulp of w / s, which
// moves a code only when w/s sits within that distance of a rounding tie.
__device__ __forceinline__ float recip(float s) { return __frcp_rn(s); }

__global__ void gather_w_kernel(const float *__restrict__ W, int64_t total, int d,
                                const int *__restrict__ perm, float *__restrict__ Wk,
                                const int *status) {
  if (*(volatile const int *)status) return;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / d;
    const int p = (int)(i - row * d);
    const int c = perm ? perm[p] : p;
    Wk[i] = W[row * d + c];
  }
}

// group = -1: one (s, z) per row from the row's original values.
__global__ void row_params_kernel(const float *__restrict__ Wk, int r, int d, int bits,
                                  float *__restrict__ scales, int32_t *__restrict__ zeros,
                                  const int *status) {
  if (*(volatile const int *)status) return;
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= r) return;
  const float *w = Wk + (size_t)row * d;
  float lo = FLT_MAX, hi = -FLT_MAX;
  for (int c = lane; c < d; c += 32) {
    const float x = w[c];
    lo = fminf(lo, x);
    hi = fmaxf(hi, x);
  }
  lo = warp_min(lo);
  hi = warp_max(hi);
  float s, z;
  minmax_params(lo, hi, (float)((1 << bits) - 1), s, z);
  if (lane == 0) {
    scales[row] = s;
    zeros[row] = (int32_t)z;
  }
}

template <int V>
__global__ void __launch_bounds__(SWEEP_THREADS) sweep_block_kernel(SweepArgs a) {
  constexpr int B = 32 * V;
  extern __shared__ __align__(16) float sU[];  // B x B: U[j0+j][j0+c] for c > j, else 0
  __shared__ float sDinv[B];
  if (*(volatile const int *)a.status) return;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nc = a.ncols;
  // U block -> shared memory with 16-byte loads (rows of U are contiguous and
  // the block starts on a multiple of 32 columns); entries on or below the
  // diagonal are zeroed, the diagonal is kept as 1/U_jj.
  constexpr int Q = B / 4;   // float4 per row
#pragma unroll 4
  for (int idx = tid; idx < B * Q; idx += SWEEP_THREADS) {
    const int j = idx / Q, c4 = (idx - j * Q) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (j < nc && c4 < nc)
      v = *reinterpret_cast<const float4 *>(a.U + (size_t)(a.j0 + j) * a.ldu + a.j0 + c4);
    if (j < nc && j >= c4 && j < c4 + 4) {
      const float dj = j == c4 ? v.x : j == c4 + 1 ? v.y : j == c4 + 2 ? v.z : v.w;
      sDinv[j] = 1.f / dj;
    }
    v.x = c4 + 0 > j ? v.x : 0.f;
    v.y = c4 + 1 > j ? v.y : 0.f;
    v.z = c4 + 2 > j ? v.z : 0.f;
    v.w = c4 + 3 > j ? v.w : 0.f;
    *reinterpret_cast<float4 *>(sU + idx * 4) = v;
  }
  for (int j = nc + tid; j < B; j += SWEEP_THREADS) sDinv[j] = 0.f;
  __syncthreads();

  const float maxq = (float)((1 << a.bits) - 1);
  const int g = a.group;
  const int gmask = (g > 0 && g <= B) ? g - 1 : -1;         // group starts inside the block
  const bool start_here = g > B && (a.j0 % g) == 0;         // a long group starts at column 0
  const bool inherit = g < 0 || (g > B && !start_here);     // parameters set before this block
  const int gi0 = g < 0 ? 0 : a.j0 / (g > 0 ? g : 1);

  for (int row = blockIdx.x * SWEEP_WARPS + warp; row < a.r; row += gridDim.x * SWEEP_WARPS) {
    float *wrow = a.Wk + (size_t)row * a.ldw + a.j0;
    float w[V];
    float code[V];   // converted to bytes once, at the store
    float eo[V];
#pragma unroll
    for (int v = 0; v < V; ++v) {
      const int c = lane * V + v;
      w[v] = c < nc ? wrow[c] : 0.f;
      code[v] = 0.f;
      eo[v] = 0.f;
    }
    float s = 1.f, z = 0.f, si = 1.f;
    if (inherit) {
      s = a.scales[(size_t)row * a.G + gi0];
      z = (float)a.zeros[(size_t)row * a.G + gi0];
      si = recip(s);
    }
    float esq = 0.f;
    // Column j = jj*V + v lives in register v of lane jj.  nc is a multiple of
    // 32, so every lane group of V columns is either whole or absent.
    const int njj = nc / V;
    for (int jj = 0; jj < njj; ++jj) {
#pragma unroll
      for (int v = 0; v < V; ++v) {
        const int j = jj * V + v;
        if ((gmask >= 0 && (j & gmask) == 0) || (j == 0 && start_here)) {
          float lo = FLT_MAX, hi = -FLT_MAX;
          const int jend = gmask >= 0 ? j + g : B;
#pragma unroll
          for (int u = 0; u < V; ++u) {
            const int c = lane * V + u;
            if (c >= j && c < jend && c < nc) {
              lo = fminf(lo, w[u]);
              hi = fmaxf(hi, w[u]);
            }
          }
          if (gmask < 0) {
            // A group longer than the block: its remaining columns are already
            // up to date in global memory (every earlier column's update has
            // landed there).
            for (int c = B + lane; c < g; c += 32) {
              const float x = wrow[c];
              lo = fminf(lo, x);
              hi = fmaxf(hi, x);
            }
          }
          lo = warp_min(lo);
          hi = warp_max(hi);
          minmax_params(lo, hi, maxq, s, z);
          si = recip(s);
          if (lane == 0) {
            const int gi = (a.j0 + j) / g;
            a.scales[(size_t)row * a.G + gi] = s;
            a.zeros[(size_t)row * a.G + gi] = (int32_t)z;
          }
        }
        const float wj = __shfl_sync(0xffffffffu, w[v], jj);
        float q = rintf(wj * si) + z;
        q = fminf(fmaxf(q, 0.f), maxq);
        const float wq = s * (q - z);
        const float e = (wj - wq) * sDinv[j];
        if (lane == jj) {
          w[v] = wq;
          code[v] = q;
          eo[v] = e;
        }
        esq = fmaf(e, e, esq);
        const float *urow = sU + j * B + lane * V;
#pragma unroll
        for (int u = 0; u < V; ++u) w[u] = fmaf(-e, urow[u], w[u]);
      }
    }
#pragma unroll
    for (int v = 0; v < V; ++v) {
      const int c = lane * V + v;
      if (c < nc) {
        wrow[c] = w[v];
        a.codes[(size_t)row * a.ldc + a.j0 + c] = (uint8_t)(int)code[v];
        a.err[(size_t)row * a.lde + c] = eo[v];
      }
    }
    if (lane == 0) a.loss_rows[row] += 0.5 * (double)esq;
  }
}

// Unpermute, dequantised output, ||W - W^||^2 per row, codes and packing.
// One CTA per row, in chunks of 1024 columns: each thread handles 4
// consecutive columns (16-byte loads and stores of W, W^), the chunk's codes
// are staged in shared memory, then 32 threads pack them (32 codes -> BITS
// words each).
template <int BITS>
__global__ void __launch_bounds__(256) finalize_kernel(FinalizeArgs a) {
  constexpr int CH = 1024;
  __shared__ uint8_t sc[CH];
  __shared__ double red[8];
  if (*(volatile const int *)a.status) return;
  const int row = blockIdx.x;
  const size_t rb = (size_t)row * a.d;
  const float *w = a.W + rb;
  const float *wk = a.Wk + rb;
  const uint8_t *cp = a.codes_p + rb;
  uint32_t *qrow = reinterpret_cast<uint32_t *>(a.qweight) + (size_t)row * (a.d / 32) * BITS;
  double dsq = 0.0;
  for (int c0 = 0; c0 < a.d; c0 += CH) {
    const int c = c0 + threadIdx.x * 4;
    if (c < a.d) {
      const float4 wo = *reinterpret_cast<const float4 *>(w + c);
      float4 wq;
      uchar4 q;
      if (a.inv) {
        const int4 p = *reinterpret_cast<const int4 *>(a.inv + c);
        wq = make_float4(wk[p.x], wk[p.y], wk[p.z], wk[p.w]);
        q = make_uchar4(cp[p.x], cp[p.y], cp[p.z], cp[p.w]);
        if (row == 0 && a.g_idx) {
          const int g = a.group;
          *reinterpret_cast<int4 *>(a.g_idx + c) =
              g < 0 ? make_int4(0, 0, 0, 0) : make_int4(p.x / g, p.y / g, p.z / g, p.w / g);
        }
      } else {
        wq = *reinterpret_cast<const float4 *>(wk + c);
        q = *reinterpret_cast<const uchar4 *>(cp + c);
        if (row == 0 && a.g_idx) {
          const int g = a.group;
          *reinterpret_cast<int4 *>(a.g_idx + c) =
              g < 0 ? make_int4(0, 0, 0, 0)
                    : make_int4(c / g, (c + 1) / g, (c + 2) / g, (c + 3) / g);
        }
      }
      const double dx = (double)wo.x - wq.x, dy = (double)wo.y - wq.y;
      const double dz = (double)wo.z - wq.z, dw = (double)wo.w - wq.w;
      dsq += dx * dx + dy * dy + dz * dz + dw * dw;
      if (a.W_hat) *reinterpret_cast<float4 *>(a.W_hat + rb + c) = wq;
      if (a.codes) *reinterpret_cast<uchar4 *>(a.codes + rb + c) = q;
      *reinterpret_cast<uchar4 *>(sc + threadIdx.x * 4) = q;
    }
    __syncthreads();
    const int ng = min(CH, a.d - c0) / 32;
    if (threadIdx.x < ng) {
      uint32_t c32[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) c32[k] = sc[threadIdx.x * 32 + k];
      uint32_t words[BITS];
      pack32<BITS>(c32, words);
      uint32_t *qw = qrow + (size_t)(c0 / 32 + threadIdx.x) * BITS;
#pragma unroll
      for (int k = 0; k < BITS; ++k) qw[k] = words[k];
    }
    __syncthreads();
  }
  for (int o = 16; o > 0; o >>= 1) dsq += __shfl_xor_sync(0xffffffffu, dsq, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = dsq;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < 8; ++i) t += red[i];
    a.dsq_rows[row] = t;
  }
}

__global__ void loss_reduce_kernel(const double *loss_rows, const double *dsq_rows, int r,
                                   const float *lambda, double *out, const int *status) {
  if (*(volatile const int *)status) return;
  __shared__ double ra[32], rb[32];
  double sa = 0.0, sb = 0.0;
  for (int i = threadIdx.x; i < r; i += blockDim.x) {
    sa += loss_rows[i];
    sb += dsq_rows[i];
  }
  for (int o = 16; o > 0; o >>= 1) {
    sa += __shfl_xor_sync(0xffffffffu, sa, o);
    sb += __shfl_xor_sync(0xffffffffu, sb, o);
  }
  if ((threadIdx.x & 31) == 0) {
    ra[threadIdx.x >> 5] = sa;
    rb[threadIdx.x >> 5] = sb;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double ta = 0.0, tb = 0.0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) {
      ta += ra[i];
      tb += rb[i];
    }
    out[0] = ta - 0.5 * (double)(*lambda) * tb;  // 1/2 tr(D H D^T) with the undamped H
    out[1] = ta;                                 // sum of e^2/2 (damped objective)
    out[2] = tb;                                 // ||W - W^||_F^2
  }
}

}  // namespace

int launch_gather_w(const float *W, int r, int d, const int *perm, float *Wk, const int *status,
                    cudaStream_t stream) {
  const int64_t total = (int64_t)r * d;
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = (int64_t)num_sms() * 16;
  if (blocks > cap) blocks = cap;
  gather_w_kernel<<<(unsigned)blocks, 256, 0, stream>>>(W, total, d, perm, Wk, status);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

int launch_row_params(const float *Wk, int r, int d, int bits, float *scales, int32_t *zeros,
                      const int *status, cudaStream_t stream) {
  row_params_kernel<<<(r + 7) / 8, 256, 0, stream>>>(Wk, r, d, bits, scales, zeros, status);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

template <int V>
static int sweep_launch(const SweepArgs &a, cudaStream_t stream) {
  constexpr int B = 32 * V;
  const size_t smem = (size_t)B * B * sizeof(float);
  static bool attr = false;
  if (!attr) {
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(sweep_block_kernel<V>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    attr = true;
  }
  // One resident warp per row when the SMs can hold them all (2 CTAs of 16
  // warps per SM), so no CTA runs a sparse second round.
  const int want = (a.r + SWEEP_WARPS - 1) / SWEEP_WARPS;
  const int cap = num_sms() * 2;
  const int grid = want < cap ? want : cap;
  sweep_block_kernel<V><<<grid, SWEEP_THREADS, smem, stream>>>(a);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

int launch_sweep_block(const SweepArgs &a, int block, cudaStream_t stream) {
  switch (block) {
    case 32: return sweep_launch<1>(a, stream);
    case 64: return sweep_launch<2>(a, stream);
    case 128: return sweep_launch<4>(a, stream);
    default: return GPTQ_ERR_INVALID_ARG;
  }
}

int launch_finalize(const FinalizeArgs &a, cudaStream_t stream) {
  switch (a.bits) {
    case 2: finalize_kernel<2><<<a.r, 256, 0, stream>>>(a); break;
    case 3: finalize_kernel<3><<<a.r, 256, 0, stream>>>(a); break;
    case 4: finalize_kernel<4><<<a.r, 256, 0, stream>>>(a); break;
    case 8: finalize_kernel<8><<<a.r, 256, 0, stream>>>(a); break;
    default: return GPTQ_ERR_INVALID_ARG;
  }
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

int launch_loss_reduce(const double *loss_rows, const double *dsq_rows, int r,
                       const float *lambda, double *out, const int *status,
                       cudaStream_t stream) {
  loss_reduce_kernel<<<1, 1024, 0, stream>>>(loss_rows, dsq_rows, r, lambda, out, status);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

}  // namespace gptq
