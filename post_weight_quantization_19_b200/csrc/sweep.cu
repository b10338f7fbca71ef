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
// Rows are independent.  One row of the current block belongs to L = B/CW
// neighbouring lanes of a warp, each holding CW consecutive columns in
// registers (CW = 16 for 128-column blocks: 8 lanes per row; 32 for narrower
// blocks); the block of U sits in shared memory.  Column j is broadcast from
// its lane by one shuffle, every lane of the row runs the quantiser on it
// (the same value, so no divergence) and updates its CW columns with fused
// multiply-adds.  No inter-warp synchronisation at all.
#include <float.h>
#include <stdlib.h>

#include "gptq_internal.h"
#include "pack_bits.cuh"

namespace gptq {
namespace {

constexpr int SWEEP_WARPS = 4;   // warps per CTA (8 for the 16-lane form of the 128-column block)
constexpr int SWEEP_CW = 16;     // columns of a 128-column block held by one lane

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
// Over the L lanes of one row (xor offsets below L stay inside the row's lanes).
template <int L>
__device__ __forceinline__ float row_min(float v) {
#pragma unroll
  for (int o = L / 2; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
template <int L>
__device__ __forceinline__ float row_max(float v) {
#pragma unroll
  for (int o = L / 2; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Parameters of a group whose values span [lo, hi].
// Asymmetric min-max: the range widened to include 0, s = (xmax - xmin)/(2^b - 1)
// (1 for an empty range), z = rint(-xmin/s).
// Symmetric ("LLM 量化技术" §1.2): zero point 0 in the signed code, s = max|x| /
// (2^(b-1) - 1) (1 for an all-zero group); the signed code is stored as code +
// 2^(b-1), i.e. z = 2^(b-1), and the clamp [-z, maxq - z] is then the signed range.
__device__ __forceinline__ void quant_params(float lo, float hi, float maxq, bool sym, float &s,
                                             float &z) {
  if (sym) {
    const float amax = fmaxf(fabsf(lo), fabsf(hi));
    const float half = 0.5f * (maxq + 1.f);
    s = amax == 0.f ? 1.f : __fdiv_rn(amax, half - 1.f);
    z = half;
    return;
  }
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
  pdl_wait_then_release();
  if (*(volatile const int *)status) return;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / d;
    const int p = (int)(i - row * d);
    const int c = perm ? perm[p] : p;
    Wk[i] = W[row * d + c];
  }
}

// Parameters fixed before the sweep, one warp per row, over groups of g
// consecutive columns of Wsrc: g = d for group = -1 (one (s, z) per row, from
// the sweep-order copy: a permutation leaves the minimum and maximum alone),
// g = group for static groups (from the original W, in its own column order).
__global__ void row_params_kernel(const float *__restrict__ Wsrc, int r, int d, int g, int bits,
                                  int sym, float *__restrict__ scales,
                                  int32_t *__restrict__ zeros, const int *status) {
  pdl_wait_then_release();
  if (*(volatile const int *)status) return;
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= r) return;
  const float *w = Wsrc + (size_t)row * d;
  const int G = d / g;
  const float maxq = (float)((1 << bits) - 1);
  for (int k = 0; k < G; ++k) {
    float lo = FLT_MAX, hi = -FLT_MAX;
    for (int c = k * g + lane; c < (k + 1) * g; c += 32) {
      const float x = w[c];
      lo = fminf(lo, x);
      hi = fmaxf(hi, x);
    }
    lo = warp_min(lo);
    hi = warp_max(hi);
    float s, z;
    quant_params(lo, hi, maxq, sym != 0, s, z);
    if (lane == 0) {
      scales[(size_t)row * G + k] = s;
      zeros[(size_t)row * G + k] = (int32_t)z;
    }
  }
}

// Round to nearest even through the float adder: exact for |x| < 2^22.
__device__ __forceinline__ float round_even(float x) {
  const float m = 12582912.f;   // 1.5 * 2^23
  return __fsub_rn(__fadd_rn(x, m), m);
}

// 16-byte global -> shared copy that does not wait (all of a thread's copies
// are in flight together).
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// B = CW * L columns per block: each row is held by L lanes with CW columns each.
// VAR: the quantiser variants of SweepArgs::flags are honoured (the plain
// instantiation compiles them out, leaving its registers and schedule alone).
// With static groups under act-order (perm given) every column reads its own
// group's fixed parameters: the groups of the original columns are scattered
// over the sweep order.
template <int CW, int L, bool VAR, int WARPS>
__global__ void __launch_bounds__(32 * WARPS) sweep_block_kernel(SweepArgs a) {
  constexpr int SWEEP_THREADS = 32 * WARPS;
  constexpr int B = CW * L;
  constexpr int CHUNK = CW + 4;        // stride of one lane's part of a U row in shared
                                       // memory: the L parts start in different banks
  constexpr int RSTRIDE = CHUNK * L;   // floats per U row in shared memory
  constexpr int RPW = 32 / L;          // rows per warp
  // U[j0+j][j0+c] for c > j, else 0; element (j, c) at j * RSTRIDE + (c / CW) * CHUNK + c % CW
  extern __shared__ __align__(16) float sU[];
  __shared__ float sDinv[B];
  __shared__ int sGrp[VAR ? B : 1];   // group of each column of the block (per-column mode)

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nc = a.ncols;
  // U block -> shared memory with 16-byte asynchronous copies, all in flight
  // at once (rows of U are contiguous and the block starts on a multiple of 32
  // columns); then entries on or below the diagonal are zeroed and the
  // diagonal is kept as 1/U_jj.
  constexpr int Q = B / 4;   // 16-byte pieces per row
  for (int idx = tid; idx < B * Q; idx += SWEEP_THREADS) {
    const int j = idx / Q, c4 = (idx - j * Q) * 4;
    float *dst = sU + j * RSTRIDE + (c4 / CW) * CHUNK + c4 % CW;
    if (j < nc && c4 < nc && c4 + 3 >= j)   // pieces wholly below the diagonal stay zero
      cp_async16(dst, a.U + (size_t)(a.j0 + j) * a.ldu + a.j0 + c4);
    else
      *reinterpret_cast<float4 *>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  cp_async_wait_all();
  __syncthreads();
  // The piece holding the diagonal: keep 1/U_jj, zero the entries up to it.
  for (int j = tid; j < B; j += SWEEP_THREADS) {
    const int c4 = j & ~3;
    float *piece = sU + j * RSTRIDE + (c4 / CW) * CHUNK + c4 % CW;
    sDinv[j] = j < nc ? 1.f / piece[j - c4] : 0.f;
    for (int c = c4; c <= j; ++c) piece[c - c4] = 0.f;
  }
  __syncthreads();
  // U was finished by the factorisation, before this kernel's predecessor
  // began; W, the parameters and the outputs belong to the sequence.
  pdl_wait_then_release();
  if (*(volatile const int *)a.status) return;

  const float maxq = (float)((1 << a.bits) - 1);
  const int g = a.group;   // -1 or a multiple of 32
  const int flags = VAR ? a.flags : 0;
  const bool percol = VAR && a.perm != nullptr;   // uniform over the grid
  if (percol) {
    for (int j = tid; j < B; j += SWEEP_THREADS) sGrp[j] = j < nc ? a.perm[a.j0 + j] / g : 0;
    __syncthreads();
  }
  const int gmask = (g > 0 && g <= B) ? g - 1 : -1;         // groups start inside the block
  const bool start_here = g > B && (a.j0 % g) == 0;         // a long group starts at column 0
  const bool inherit = g < 0 || (g > B && !start_here);     // parameters set before this block
  const int gi0 = g < 0 ? 0 : a.j0 / (g > 0 ? g : 1);
  const int ql = lane % L;        // this lane holds columns ql*CW .. ql*CW+CW-1 of the block
  const int base = lane - ql;     // first lane of the row
  const int nsub = nc / CW;       // 32-column parts present in this block
  const bool mine = ql < nsub;

  for (int row0 = (blockIdx.x * WARPS + warp) * RPW; row0 < a.r;
       row0 += gridDim.x * WARPS * RPW) {
    // Lanes of rows past the end keep going (zeros) so the shuffles stay whole.
    const int row = row0 + lane / L;
    const bool valid = row < a.r;
    float *wrow = a.Wk + (size_t)(valid ? row : 0) * a.ldw + a.j0;
    float w[CW];
    float code[CW];   // converted to bytes once, at the store
    float eo[CW];
#pragma unroll
    for (int c = 0; c < CW; c += 4) {
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (valid && mine) v = *reinterpret_cast<const float4 *>(wrow + ql * CW + c);
      w[c] = v.x;
      w[c + 1] = v.y;
      w[c + 2] = v.z;
      w[c + 3] = v.w;
    }
#pragma unroll
    for (int c = 0; c < CW; ++c) {
      code[c] = 0.f;
      eo[c] = 0.f;
    }
    const double loss0 = (ql == 0 && valid) ? a.loss_rows[row] : 0.0;   // needed at the end
    float s = 1.f, z = 0.f, si = 1.f;
    if (inherit && valid) {
      s = a.scales[(size_t)row * a.G + gi0];
      z = (float)a.zeros[(size_t)row * a.G + gi0];
      si = recip(s);
    }
    float esq = 0.f;
    for (int sb = 0; sb < nsub; ++sb) {
      const int jb = sb * CW;
      // Groups are multiples of 32 columns, so they start only at a part's first column.
      if (percol) {
        // parameters are read per column below
      } else if ((flags & SWEEP_STATIC) &&
                 ((gmask >= 0 && (jb & gmask) == 0) || (jb == 0 && start_here))) {
        // fixed before the sweep: read, not computed
        const int gi = (a.j0 + jb) / g;
        s = valid ? a.scales[(size_t)row * a.G + gi] : 1.f;
        z = valid ? (float)a.zeros[(size_t)row * a.G + gi] : 0.f;
        si = recip(s);
      } else if ((gmask >= 0 && (jb & gmask) == 0) || (jb == 0 && start_here)) {
        float lo = FLT_MAX, hi = -FLT_MAX;
        const int jend = gmask >= 0 ? jb + g : B;
        if (mine && ql >= sb && ql * CW < jend) {
#pragma unroll
          for (int c = 0; c < CW; ++c) {
            lo = fminf(lo, w[c]);
            hi = fmaxf(hi, w[c]);
          }
        }
        if (gmask < 0 && valid) {
          // A group longer than the block: its remaining columns are already
          // up to date in global memory (every earlier column's update has
          // landed there).
          for (int c = B + ql; c < g; c += L) {
            const float x = wrow[c];
            lo = fminf(lo, x);
            hi = fmaxf(hi, x);
          }
        }
        lo = row_min<L>(lo);
        hi = row_max<L>(hi);
        quant_params(lo, hi, maxq, (flags & SWEEP_SYM) != 0, s, z);
        si = recip(s);
        if (ql == 0 && valid) {
          const int gi = (a.j0 + jb) / g;
          a.scales[(size_t)row * a.G + gi] = s;
          a.zeros[(size_t)row * a.G + gi] = (int32_t)z;
        }
      }
      const float *ub = sU + jb * RSTRIDE + ql * CHUNK;
      const float *dv = sDinv + jb;
      // clamp(rint(x) + z, 0, maxq) - z == clamp(rint(x), -z, maxq - z) exactly
      // (z is a small integer), which takes two operations off the chain.
      // rint(x) is taken as (x + 1.5 * 2^23) - 1.5 * 2^23 in round-to-nearest-
      // even: exact for |x| < 2^22, and for larger |x| both forms clamp to the
      // same end of [-z, maxq - z].
      float tlo = -z, thi = maxq - z;
      float wj = __shfl_sync(0xffffffffu, w[0], base + sb);
#pragma unroll
      for (int i = 0; i < CW; ++i) {
        if (percol) {
          // the same column for every row: one broadcast read of its group
          const size_t at = (size_t)(valid ? row : 0) * a.G + sGrp[jb + i];
          s = __ldg(a.scales + at);
          z = (float)__ldg(a.zeros + at);
          si = recip(s);
          tlo = -z;
          thi = maxq - z;
        }
        const float t = fminf(fmaxf(round_even(wj * si), tlo), thi);
        const float wq = s * t;
        const float e = (wj - wq) * dv[i];
        if (ql == sb) {
          w[i] = wq;
          code[i] = t + z;
          eo[i] = e;
        }
        esq = fmaf(e, e, esq);
        float u[CW];
        const float4 *u4 = reinterpret_cast<const float4 *>(ub + i * RSTRIDE);
#pragma unroll
        for (int c = 0; c < CW; c += 4) {
          const float4 v = u4[c / 4];
          u[c] = v.x;
          u[c + 1] = v.y;
          u[c + 2] = v.z;
          u[c + 3] = v.w;
        }
        // The next column first: its broadcast is the next step's critical path.
        if (i + 1 < CW) {
          w[i + 1] = fmaf(-e, u[i + 1], w[i + 1]);
          wj = __shfl_sync(0xffffffffu, w[i + 1], base + sb);
        }
#pragma unroll
        for (int c = 0; c < CW; ++c)
          if (c != i + 1) w[c] = fmaf(-e, u[c], w[c]);
      }
    }
    if (valid && mine) {
      float *wp = wrow + ql * CW;
      float *ep = a.err + (size_t)row * a.lde + ql * CW;
      uint8_t *cp = a.codes + (size_t)row * a.ldw + a.j0 + ql * CW;
#pragma unroll
      for (int c = 0; c < CW; c += 4) {
        *reinterpret_cast<float4 *>(wp + c) = make_float4(w[c], w[c + 1], w[c + 2], w[c + 3]);
        *reinterpret_cast<float4 *>(ep + c) = make_float4(eo[c], eo[c + 1], eo[c + 2], eo[c + 3]);
      }
      // 16 codes per 16-byte store (8 per 8-byte store when a lane holds 8 columns)
      constexpr int CS = CW % 16 == 0 ? 16 : 8;
      static_assert(CW % CS == 0, "codes per store");
#pragma unroll
      for (int c = 0; c < CW; c += CS) {
        uint32_t wd[CS / 4];
#pragma unroll
        for (int k = 0; k < CS / 4; ++k)
          wd[k] = (uint32_t)(int)code[c + 4 * k] | ((uint32_t)(int)code[c + 4 * k + 1] << 8) |
                  ((uint32_t)(int)code[c + 4 * k + 2] << 16) |
                  ((uint32_t)(int)code[c + 4 * k + 3] << 24);
        if constexpr (CS == 16)
          *reinterpret_cast<uint4 *>(cp + c) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        else
          *reinterpret_cast<uint2 *>(cp + c) = make_uint2(wd[0], wd[1]);
      }
    }
    if (ql == 0 && valid) a.loss_rows[row] = loss0 + 0.5 * (double)esq;
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
  pdl_wait_then_release();
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
              g < 0              ? make_int4(0, 0, 0, 0)
              : a.static_groups  ? make_int4(c / g, (c + 1) / g, (c + 2) / g, (c + 3) / g)
                                 : make_int4(p.x / g, p.y / g, p.z / g, p.w / g);
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
  pdl_wait_then_release();
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
  GPTQ_LAUNCH_PDL(gather_w_kernel, dim3((unsigned)blocks), dim3(256), 0, stream, W, total, d, perm,
                  Wk, status);
  return GPTQ_OK;
}

int launch_row_params(const float *Wsrc, int r, int d, int g, int bits, int sym, float *scales,
                      int32_t *zeros, const int *status, cudaStream_t stream) {
  if (g <= 0 || g % 32 != 0 || d % g != 0) return GPTQ_ERR_INVALID_ARG;
  GPTQ_LAUNCH_PDL(row_params_kernel, dim3((r + 7) / 8), dim3(256), 0, stream, Wsrc, r, d, g, bits,
                  sym, scales, zeros, status);
  return GPTQ_OK;
}

template <int CW, int L, bool VAR, int WARPS = SWEEP_WARPS>
static int sweep_launch(const SweepArgs &a, cudaStream_t stream) {
  constexpr int B = CW * L;
  const size_t smem = (size_t)B * (CW + 4) * L * sizeof(float);
  static std::atomic<bool> attr[64] = {};
  if (const int rc = ensure_smem_attr(sweep_block_kernel<CW, L, VAR, WARPS>, smem, attr))
    return rc;
  // Every row gets its lanes in one wave when the SMs can hold them (two CTAs
  // per SM: about 180 registers per thread).
  const int rows_per_cta = WARPS * (32 / L);
  const int want = (a.r + rows_per_cta - 1) / rows_per_cta;
  const int cap = num_sms() * 2;
  const int grid = want < cap ? want : cap;
  GPTQ_LAUNCH_PDL((sweep_block_kernel<CW, L, VAR, WARPS>), dim3(grid), dim3(32 * WARPS), smem,
                  stream, a);
  return GPTQ_OK;
}

template <bool VAR>
static int sweep_launch_block(const SweepArgs &a, int block, cudaStream_t stream) {
  switch (block) {
    case 32: return sweep_launch<32, 1, VAR>(a, stream);
    case 64: return sweep_launch<32, 2, VAR>(a, stream);
    case 128: return sweep_launch<SWEEP_CW, 128 / SWEEP_CW, VAR>(a, stream);
    default: return GPTQ_ERR_INVALID_ARG;
  }
}

int launch_sweep_block(const SweepArgs &a, int block, cudaStream_t stream) {
  if (a.perm && !((a.flags & SWEEP_STATIC) && a.group > 0)) return GPTQ_ERR_INVALID_ARG;
  return (a.flags || a.perm) ? sweep_launch_block<true>(a, block, stream)
                             : sweep_launch_block<false>(a, block, stream);
}

int launch_finalize(const FinalizeArgs &a, cudaStream_t stream) {
  switch (a.bits) {
    case 2: GPTQ_LAUNCH_PDL(finalize_kernel<2>, dim3(a.r), dim3(256), 0, stream, a); break;
    case 3: GPTQ_LAUNCH_PDL(finalize_kernel<3>, dim3(a.r), dim3(256), 0, stream, a); break;
    case 4: GPTQ_LAUNCH_PDL(finalize_kernel<4>, dim3(a.r), dim3(256), 0, stream, a); break;
    case 8: GPTQ_LAUNCH_PDL(finalize_kernel<8>, dim3(a.r), dim3(256), 0, stream, a); break;
    default: return GPTQ_ERR_INVALID_ARG;
  }
  return GPTQ_OK;
}

int launch_loss_reduce(const double *loss_rows, const double *dsq_rows, int r,
                       const float *lambda, double *out, const int *status,
                       cudaStream_t stream) {
  GPTQ_LAUNCH_PDL(loss_reduce_kernel, dim3(1), dim3(1024), 0, stream, loss_rows, dsq_rows, r, lambda,
                  out, status);
  return GPTQ_OK;
}

}  // namespace gptq
