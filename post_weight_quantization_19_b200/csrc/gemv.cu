// Dequantising matrix-vector product over a packed layer: y = x W^^T.
//
// Sources: the GPTQ reading card ("GPTQ: Accurate Post-Training Quantization
// for Generative Pre-trained Transformers", 计算设置) -- the quantised layers
// run through a dequantising matrix-vector kernel at inference, which is
// bound by reading the packed weights; "一文读懂GPTQ" §三 -- 3/4-bit codes in
// 32-bit integer arrays, group_size and desc_act (the group index g_idx).
//
// W^[row, c] = s[row, gi(c)] (q[row, c] - z[row, gi(c)]), with q the b-bit code
// of column c in the row's LSB-first stream (the layout gptq_quantize_layer and
// gptq_pack write) and gi(c) = g_idx[c] when given (act-order), else c / group
// (0 for group = -1).  One warp per row: lane l takes the 32-code chunks l,
// l + 32, ... of the row (b consecutive words each, fetched 4 chunks ahead),
// unpacks them with static shifts, and accumulates the m dot products in fp32
// (m rounded up to 1, 2, 4 or 8 accumulators); a shuffle reduction ends the
// row.  Bandwidth bound at small m: r*d*b/8 bytes of codes, 8*r*G bytes of
// scales and zeros, 4*m*(d + r) bytes of x and y.
//
// x is read by every row.  Neighbouring lanes need x 128 bytes apart (one
// chunk each), so a warp's 16-byte load of x straight from global memory
// touches 32 cache lines; each CTA therefore first copies x into shared memory
// with 4 floats of padding after every 32, where the same warp-wide read hits
// every bank exactly four times (the minimum for 512 bytes).  Shapes whose x
// does not fit read it from global memory instead.
#include "gptq_internal.h"

namespace gptq {
namespace {

constexpr int GEMV_WARPS = 8;
constexpr int GEMV_MAX_M = GPTQ_GEMV_MAX_M;

constexpr int XPAD = 36;                         // floats per staged 32-float chunk of x
constexpr size_t GEMV_SMEM_MAX = 200u << 10;     // staged x, bytes

struct GemvArgs {
  const uint32_t *qweight;
  const float *scales;
  const int32_t *zeros;
  const int32_t *g_idx;   // may be NULL
  int64_t r;
  int d, group, G, m;
  const float *x;         // [m x d], 16-byte aligned rows
  float *y;               // [m x r]
  uint32_t magic;         // 0x4B000000, the bits of 2^23, passed at run time (fold_chunk)
};

// One 32-code chunk: unpack with static shifts and accumulate MB dot products.
// SX: x staged in shared memory (sx, XPAD floats per chunk), else read from a.x.
template <int BITS, int MB, bool SX>
__device__ __forceinline__ void gemv_chunk(const uint32_t (&w)[BITS], const GemvArgs &a,
                                           const float *srow, const int32_t *zrow, int k,
                                           const float *sx, float (&acc)[MB]) {
  constexpr uint32_t mask = (1u << BITS) - 1u;
  float s = 0.f, z = 0.f;
  if (!a.g_idx) {   // groups are multiples of 32 columns: one group per chunk
    const int gi = a.group > 0 ? (k * 32) / a.group : 0;
    s = __ldg(srow + gi);
    z = (float)__ldg(zrow + gi);
  }
#pragma unroll
  for (int j4 = 0; j4 < 32; j4 += 4) {
    float4 xv[MB];
#pragma unroll
    for (int i = 0; i < MB; ++i) {
      if (i >= a.m)
        xv[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      else if constexpr (SX)
        xv[i] = *reinterpret_cast<const float4 *>(sx + ((size_t)i * (a.d / 32) + k) * XPAD + j4);
      else
        xv[i] = __ldg(reinterpret_cast<const float4 *>(a.x + (int64_t)i * a.d + k * 32 + j4));
    }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int j = j4 + jj;
      const int pos = j * BITS, wi = pos >> 5, off = pos & 31;
      uint32_t v = w[wi] >> off;
      if (off + BITS > 32) v |= w[wi + 1] << (32 - off);
      const float q = (float)(v & mask);
      if (a.g_idx) {
        int gi = __ldg(a.g_idx + k * 32 + j);
        gi = gi < 0 ? 0 : (gi >= a.G ? a.G - 1 : gi);   // out-of-range entries clamp
        s = __ldg(srow + gi);
        z = (float)__ldg(zrow + gi);
      }
      const float wv = s * (q - z);
#pragma unroll
      for (int i = 0; i < MB; ++i) {
        const float xj = jj == 0 ? xv[i].x : jj == 1 ? xv[i].y : jj == 2 ? xv[i].z : xv[i].w;
        acc[i] = fmaf(wv, xj, acc[i]);
      }
    }
  }
}

// MB accumulators (the batch rounded up to 1, 2, 4 or 8); a lane fetches the
// words of up to PF of its chunks before any arithmetic, so each row waits on
// memory about once.
template <int BITS, int MB, bool SX>
__global__ void __launch_bounds__(32 * GEMV_WARPS) gemv_kernel(GemvArgs a) {
  constexpr int PF = 4;
  extern __shared__ __align__(16) float sx[];   // SX: [m][d/32][XPAD]
  const int lane = threadIdx.x & 31;
  const int nchunk = a.d / 32;
  if constexpr (SX) {
    const int per = nchunk * 8;                  // 16-byte pieces of one vector
    for (int idx = threadIdx.x; idx < a.m * per; idx += blockDim.x) {
      const int i = idx / per, rem = idx - i * per, k = rem >> 3, q = rem & 7;
      *reinterpret_cast<float4 *>(sx + ((size_t)i * nchunk + k) * XPAD + q * 4) =
          __ldg(reinterpret_cast<const float4 *>(a.x + (int64_t)i * a.d + k * 32 + q * 4));
    }
    __syncthreads();
  }
  const int64_t wpr = (int64_t)nchunk * BITS;   // words per row
  for (int64_t row = (int64_t)blockIdx.x * GEMV_WARPS + (threadIdx.x >> 5); row < a.r;
       row += (int64_t)gridDim.x * GEMV_WARPS) {
    float acc[MB];
#pragma unroll
    for (int i = 0; i < MB; ++i) acc[i] = 0.f;
    const uint32_t *qrow = a.qweight + row * wpr;
    const float *srow = a.scales + row * a.G;
    const int32_t *zrow = a.zeros + row * a.G;
    for (int k0 = lane; k0 < nchunk; k0 += 32 * PF) {
      uint32_t w[PF][BITS];
#pragma unroll
      for (int p = 0; p < PF; ++p) {
        const int k = k0 + 32 * p;
#pragma unroll
        for (int t = 0; t < BITS; ++t) w[p][t] = k < nchunk ? __ldg(qrow + (int64_t)k * BITS + t) : 0u;
      }
#pragma unroll
      for (int p = 0; p < PF; ++p)
        if (k0 + 32 * p < nchunk) gemv_chunk<BITS, MB, SX>(w[p], a, srow, zrow, k0 + 32 * p, sx, acc);
    }
#pragma unroll
    for (int i = 0; i < MB; ++i) {
      float v = acc[i];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0 && i < a.m) a.y[(int64_t)i * a.r + row] = v;
    }
  }
}

// ---------------------------------------------------------------- the fold form
// (no g_idx, x staged): per 32-code chunk (one group), with x_j the inputs,
//   sum_j s (q_j - z) x_j = s (sum_j q_j x_j - z sum_j x_j),
// so each code costs one bit operation that places it in the mantissa of
// 2^23 (LOP3: (w & mask << off) | 0x4B000000 is the float 2^23 + q 2^off,
// exact while q 2^off < 2^23), one subtraction of 2^23 and one fused
// multiply-add with x_j 2^-off -- the staged copy of x carries that power of
// two, so the product is exactly q_j x_j.  Codes whose offset is too high for
// the exponent trick are read from the word shifted right once by FSH bits;
// the two 3-bit codes that straddle words come from a funnel shift.  The sums
// of x per chunk are staged too.  A warp takes R rows at once (lane l the
// chunks l, l + 32, ... of each), so every staged x value it reads serves R
// rows; the grid holds one CTA per SM slot with just enough warps that every
// warp takes the same number of row groups.

template <int BITS>
struct CodeAt {
  static constexpr int FSH = BITS == 8 ? 16 : 12;   // shift of the high codes
  static constexpr int TOP = 23 - BITS;              // highest offset the trick takes
  __host__ __device__ static constexpr int pos(int j) { return j * BITS; }
  __host__ __device__ static constexpr int word(int j) { return pos(j) >> 5; }
  __host__ __device__ static constexpr int off(int j) { return pos(j) & 31; }
  __host__ __device__ static constexpr bool straddle(int j) { return off(j) + BITS > 32; }
  // offset of the code in the value it is extracted from
  __host__ __device__ static constexpr int eff(int j) {
    return straddle(j) ? 0 : (off(j) <= TOP ? off(j) : off(j) - FSH);
  }
};

// R rows of one chunk at a time: each staged x value read from shared memory
// serves R rows' codes (read once per row, x alone would cost 4 d bytes of
// shared-memory traffic per row, more than the codes' share of HBM time).
// xk: the staged chunk of vector 0 (XPAD floats per chunk, vectors vstride
// floats apart), read at compile-time offsets.
template <int BITS, int MB, int R>
__device__ __forceinline__ void fold_chunk(const uint32_t (&w)[R][BITS], const float *xk,
                                           size_t vstride, float (&part)[R][MB], int m,
                                           uint32_t magic) {
  using C = CodeAt<BITS>;
  constexpr uint32_t mask = (1u << BITS) - 1u;
  uint32_t wsh[R][BITS];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int t = 0; t < BITS; ++t) wsh[r][t] = w[r][t] >> C::FSH;
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int i = 0; i < MB; ++i) part[r][i] = 0.f;
#pragma unroll
  for (int j4 = 0; j4 < 32; j4 += 4) {
    float4 xv[MB];
#pragma unroll
    for (int i = 0; i < MB; ++i)
      xv[i] = (i == 0 || i < m) ? *reinterpret_cast<const float4 *>(xk + i * vstride + j4)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int j = j4 + jj;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        // (value & mask) | magic: one LOP3, the mask an immediate and magic a
        // register (a run-time value, so it is not folded into a second one)
        uint32_t bits;
        if (C::straddle(j))
          bits = (__funnelshift_r(w[r][C::word(j)], w[r][C::word(j) + 1], C::off(j)) & mask) |
                 magic;
        else if (C::off(j) <= C::TOP)
          bits = (w[r][C::word(j)] & (mask << C::off(j))) | magic;
        else
          bits = (wsh[r][C::word(j)] & (mask << C::eff(j))) | magic;
        const float q = __uint_as_float(bits) - 8388608.f;   // q_j 2^eff, exact
#pragma unroll
        for (int i = 0; i < MB; ++i) {
          const float xj = jj == 0 ? xv[i].x : jj == 1 ? xv[i].y : jj == 2 ? xv[i].z : xv[i].w;
          part[r][i] = fmaf(q, xj, part[r][i]);
        }
      }
    }
  }
}

// Threads per CTA of the fold form: fewer for more vectors (registers).
__host__ __device__ constexpr int fold_threads(int mb) { return mb <= 2 ? 768 : (mb == 4 ? 512 : 256); }

// Chunks a lane fetches before any arithmetic: up to 32 words of codes, at
// most 2 chunks when it takes 4 rows (registers).
__host__ __device__ constexpr int fold_prefetch(int bits, int rows) {
  return 32 / (bits * rows) < 1 ? 1
         : (32 / (bits * rows) > (rows >= 4 ? 2 : 4) ? (rows >= 4 ? 2 : 4) : 32 / (bits * rows));
}

template <int BITS, int MB, int R>
__global__ void __launch_bounds__(fold_threads(MB)) gemv_fold_kernel(GemvArgs a) {
  using C = CodeAt<BITS>;
  constexpr int PF = fold_prefetch(BITS, R);
  extern __shared__ __align__(16) float fsm[];
  const int nchunk = a.d / 32;
  const size_t vstride = (size_t)nchunk * XPAD;      // floats between staged vectors
  float *xs = fsm;                                   // [m][nchunk][XPAD], scaled
  float *xsum = fsm + (size_t)a.m * vstride;         // [m][nchunk]
  // stage x: thread per (vector, chunk)
  for (int idx = threadIdx.x; idx < a.m * nchunk; idx += blockDim.x) {
    const int i = idx / nchunk, k = idx - i * nchunk;
    const float *src = a.x + (int64_t)i * a.d + k * 32;
    float *dst = xs + (size_t)idx * XPAD;
    float sum = 0.f;
#pragma unroll
    for (int j4 = 0; j4 < 32; j4 += 4) {
      const float4 v = __ldg(reinterpret_cast<const float4 *>(src + j4));
      sum += (v.x + v.y) + (v.z + v.w);
      float4 o;
      o.x = ldexpf(v.x, -C::eff(j4 + 0));
      o.y = ldexpf(v.y, -C::eff(j4 + 1));
      o.z = ldexpf(v.z, -C::eff(j4 + 2));
      o.w = ldexpf(v.w, -C::eff(j4 + 3));
      *reinterpret_cast<float4 *>(dst + j4) = o;
    }
    xsum[idx] = sum;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int64_t row0 = (int64_t)blockIdx.x * a.r / gridDim.x;
  const int64_t row1 = (int64_t)(blockIdx.x + 1) * a.r / gridDim.x;
  const int64_t wpr = (int64_t)nchunk * BITS;
  // chunks per group: a power of two in every layout the library writes, else
  // a division per chunk
  const int cpg = a.group > 0 ? a.group / 32 : nchunk;
  const int gshift = (cpg & (cpg - 1)) == 0 ? __ffs(cpg) - 1 : -1;
  for (int64_t rb = row0 + (int64_t)warp * R; rb < row1; rb += (int64_t)nwarps * R) {
    const int nr = row1 - rb < R ? (int)(row1 - rb) : R;   // rows of this group
    // rows past the group's last read the last row again (their sums are dropped)
    const uint32_t *qp[R];
    const float *sp[R];
    const int32_t *zp[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int64_t row = rb + (r < nr ? r : nr - 1);
      qp[r] = a.qweight + row * wpr;
      sp[r] = a.scales + row * a.G;
      zp[r] = a.zeros + row * a.G;
    }
    float acc[R][MB];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int i = 0; i < MB; ++i) acc[r][i] = 0.f;
    for (int k0 = lane; k0 < nchunk; k0 += 32 * PF) {
      // every load of the PF chunks (codes, scale, zero) before any arithmetic
      uint32_t w[PF][R][BITS];
      float sc[PF][R], zr[PF][R];
#pragma unroll
      for (int p = 0; p < PF; ++p) {
        const int k = k0 + 32 * p;
        const bool in = k < nchunk;
        const int gi = !in ? 0 : (gshift >= 0 ? k >> gshift : k / cpg);
#pragma unroll
        for (int r = 0; r < R; ++r) {
#pragma unroll
          for (int t = 0; t < BITS; ++t)
            w[p][r][t] = in ? __ldg(qp[r] + (int64_t)k * BITS + t) : 0u;
          sc[p][r] = in ? __ldg(sp[r] + gi) : 0.f;
          zr[p][r] = in ? (float)__ldg(zp[r] + gi) : 0.f;
        }
      }
#pragma unroll
      for (int p = 0; p < PF; ++p) {
        const int k = k0 + 32 * p;
        if (k < nchunk) {
          float part[R][MB];
          fold_chunk<BITS, MB, R>(w[p], xs + (size_t)k * XPAD, vstride, part, a.m, a.magic);
#pragma unroll
          for (int i = 0; i < MB; ++i) {
            if (i == 0 || i < a.m) {
              const float xk = xsum[i * nchunk + k];
#pragma unroll
              for (int r = 0; r < R; ++r)
                acc[r][i] = fmaf(sc[p][r], fmaf(-zr[p][r], xk, part[r][i]), acc[r][i]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int i = 0; i < MB; ++i) {
        float v = acc[r][i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0 && i < a.m && r < nr) a.y[(int64_t)i * a.r + rb + r] = v;
      }
  }
}

// Shared memory of the fold form: staged x and its chunk sums.
size_t fold_smem(const GemvArgs &a) {
  return (size_t)a.m * (a.d / 32) * (XPAD + 1) * sizeof(float);
}
constexpr size_t FOLD_SMEM_MAX = 227u << 10;   // the per-CTA limit (no static shared memory)

// One CTA per SM slot; rows split evenly over the CTAs, taken R at a time by
// the fewest warps that take every CTA's row groups in whole rounds.
template <int BITS, int MB, int R>
int gemv_launch_fold(const GemvArgs &a, int64_t ctas, cudaStream_t st) {
  static std::atomic<bool> attr[64] = {};
  if (const int rc = ensure_smem_attr(gemv_fold_kernel<BITS, MB, R>, FOLD_SMEM_MAX, attr))
    return rc;
  const int64_t rows = (a.r + ctas - 1) / ctas;
  const int64_t groups = (rows + R - 1) / R;
  const int max_w = fold_threads(MB) / 32;
  const int64_t rounds = (groups + max_w - 1) / max_w;
  const int warps = (int)((groups + rounds - 1) / rounds);
  gemv_fold_kernel<BITS, MB, R><<<(unsigned)ctas, 32 * warps, fold_smem(a), st>>>(a);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

// Rows per warp group: the most (up to 4 for one vector, 2 for two, 1 for
// four or eight: registers) that still leave every SM a dozen warps.
template <int BITS>
int gemv_launch_fold_m(const GemvArgs &a, cudaStream_t st) {
  const size_t smem = fold_smem(a);
  const int sms = num_sms();
  int per_sm = (int)(FOLD_SMEM_MAX / (smem > 0 ? smem : 1));
  const int mb = a.m <= 1 ? 1 : a.m <= 2 ? 2 : a.m <= 4 ? 4 : GEMV_MAX_M;
  const int by_threads = 2048 / fold_threads(mb);
  per_sm = per_sm < 1 ? 1 : (per_sm > by_threads ? by_threads : per_sm);
  int64_t ctas = (int64_t)sms * per_sm;
  if (ctas > a.r) ctas = a.r;
  const int64_t rows_per_sm = (a.r + sms - 1) / sms;
  const int rmax = rows_per_sm >= 4 * 12 ? 4 : rows_per_sm >= 2 * 12 ? 2 : 1;
  if (mb == 1) {
    if (rmax >= 4) return gemv_launch_fold<BITS, 1, 4>(a, ctas, st);
    if (rmax >= 2) return gemv_launch_fold<BITS, 1, 2>(a, ctas, st);
    return gemv_launch_fold<BITS, 1, 1>(a, ctas, st);
  }
  if (mb == 2) {
    if (rmax >= 2) return gemv_launch_fold<BITS, 2, 2>(a, ctas, st);
    return gemv_launch_fold<BITS, 2, 1>(a, ctas, st);
  }
  if (mb == 4) return gemv_launch_fold<BITS, 4, 1>(a, ctas, st);
  return gemv_launch_fold<BITS, GEMV_MAX_M, 1>(a, ctas, st);
}

template <int BITS, int MB, bool SX>
int gemv_launch_mb(const GemvArgs &a, cudaStream_t st) {
  const int64_t want = (a.r + GEMV_WARPS - 1) / GEMV_WARPS;
  size_t smem = 0;
  int64_t cap = (int64_t)num_sms() * 16;
  if constexpr (SX) {
    static std::atomic<bool> attr[64] = {};
    smem = (size_t)a.m * (a.d / 32) * XPAD * sizeof(float);
    if (const int rc = ensure_smem_attr(gemv_kernel<BITS, MB, true>, GEMV_SMEM_MAX, attr))
      return rc;
    // every CTA stages x once: a few CTAs per SM, each looping over rows
    const int64_t per_sm = (int64_t)(GEMV_SMEM_MAX / smem);
    cap = (int64_t)num_sms() * (per_sm < 1 ? 1 : per_sm > 4 ? 4 : per_sm);
  }
  const dim3 grid((unsigned)(want < cap ? want : cap));
  gemv_kernel<BITS, MB, SX><<<grid, 32 * GEMV_WARPS, smem, st>>>(a);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

template <int BITS, bool SX>
int gemv_launch_sx(const GemvArgs &a, cudaStream_t st) {
  if (a.m <= 1) return gemv_launch_mb<BITS, 1, SX>(a, st);
  if (a.m <= 2) return gemv_launch_mb<BITS, 2, SX>(a, st);
  if (a.m <= 4) return gemv_launch_mb<BITS, 4, SX>(a, st);
  return gemv_launch_mb<BITS, GEMV_MAX_M, SX>(a, st);
}

template <int BITS>
int gemv_launch(const GemvArgs &a, cudaStream_t st) {
  if (!a.g_idx && fold_smem(a) <= FOLD_SMEM_MAX) return gemv_launch_fold_m<BITS>(a, st);
  const size_t staged = (size_t)a.m * (a.d / 32) * XPAD * sizeof(float);
  return staged <= GEMV_SMEM_MAX ? gemv_launch_sx<BITS, true>(a, st)
                                 : gemv_launch_sx<BITS, false>(a, st);
}

}  // namespace
}  // namespace gptq

using namespace gptq;

extern "C" int gptq_dequant_gemv(const int32_t *qweight, const float *scales,
                                 const int32_t *zeros, const int32_t *g_idx, int64_t r,
                                 int64_t d, int bits, int group, const float *x, int64_t m,
                                 float *y, gptq_stream_t stream) {
  if (r < 0 || r > (int64_t)INT32_MAX) return GPTQ_ERR_INVALID_ARG;
  if (d <= 0 || d % 32 != 0 || d > 65536) return GPTQ_ERR_INVALID_ARG;
  if (bits != 2 && bits != 3 && bits != 4 && bits != 8) return GPTQ_ERR_INVALID_ARG;
  if (group != -1 && (group < 32 || group % 32 != 0 || d % group != 0))
    return GPTQ_ERR_INVALID_ARG;
  if (m < 0 || m > GEMV_MAX_M) return GPTQ_ERR_INVALID_ARG;
  if (r == 0 || m == 0) return GPTQ_OK;
  if (!qweight || !scales || !zeros || !x || !y) return GPTQ_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(x) % 16 || reinterpret_cast<uintptr_t>(qweight) % 4 ||
      reinterpret_cast<uintptr_t>(scales) % 4 || reinterpret_cast<uintptr_t>(zeros) % 4 ||
      reinterpret_cast<uintptr_t>(y) % 4 || (g_idx && reinterpret_cast<uintptr_t>(g_idx) % 4))
    return GPTQ_ERR_INVALID_ARG;
  GemvArgs a{reinterpret_cast<const uint32_t *>(qweight), scales, zeros, g_idx, r, (int)d,
             group, group < 0 ? 1 : (int)(d / group), (int)m, x, y, 0x4B000000u};
  cudaStream_t st = (cudaStream_t)stream;
  switch (bits) {
    case 2: return gemv_launch<2>(a, st);
    case 3: return gemv_launch<3>(a, st);
    case 4: return gemv_launch<4>(a, st);
    default: return gemv_launch<8>(a, st);
  }
}
