// The quantised layer run forward on calibration tokens: Y = fp16(X W16^T),
// with the dequantised weights W16 = fp16(s (q - z)) built from the packed
// layer first.
//
// Source: the GPTQ reading card ("GPTQ: Accurate Post-Training Quantization
// for Generative Pre-trained Transformers", 计算设置) -- a block is quantised,
// then run to produce the next block's calibration inputs; the "GPTQ" concept
// page (compassingai.com), §3 技術原理 -- at inference the codes are
// dequantised to FP16 and multiplied in floating point.
//
// X [n x d] (tokens x features, fp16) and W16 [r x d] (fp16) are both K-major,
// so one tcgen05.mma.kind::f16 of M = 128, N = 256, K = 16 per 16 features
// reads both from 128-byte-swizzled tiles that TMA loads.  Warp 0 issues TMA
// into a 4-stage ring, warp 1 issues the UMMAs into one of two 256-column TMEM
// accumulators, warps 2..9 drain TMEM.  Accumulation chains are 512 features
// long and are folded into fp32 registers (the tensor core's fp32 accumulation
// is not guaranteed to round to nearest), then each row is rounded once to
// fp16.  Persistent grid; consecutive tiles share their rows of X, so a slab
// of X is read from HBM once and W16 stays in L2.
#include <cuda_fp16.h>

#include <mutex>

#include "gptq_internal.h"

namespace gptq {
namespace {

constexpr int LM = 128;                          // tokens per tile (UMMA M)
constexpr int LN = 256;                          // outputs per tile (UMMA N)
constexpr int LK = 64;                           // features per stage (one 128-byte row)
constexpr int LSTAGES = 4;
constexpr int LFOLD = 8;                         // stages per TMEM chain (512 features)
constexpr int LA_BYTES = LM * LK * 2;            // 16 KB
constexpr int LB_BYTES = LN * LK * 2;            // 32 KB
constexpr int LSTAGE_BYTES = LA_BYTES + LB_BYTES;
constexpr int LEPI_WARPS = 8;
constexpr int LTHREADS = 32 * (2 + LEPI_WARPS);
constexpr uint32_t LTMEM_COLS = 512;             // two 256-column accumulators
constexpr size_t LSMEM_BYTES = (size_t)LSTAGES * LSTAGE_BYTES + 1024;

struct LinShared {
  uint64_t full[LSTAGES];
  uint64_t empty[LSTAGES];
  uint64_t accf[2];
  uint64_t acce[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void lin_timeout(int *status, LinShared &sh) {
  atomicCAS(status, 0, (int)GPTQ_ERR_TIMEOUT);
  *(volatile int *)&sh.abort = 1;
}

__global__ void __launch_bounds__(LTHREADS, 1)
    linear_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     int n, int d, int r, __half *__restrict__ Y, int *__restrict__ status) {
  extern __shared__ uint8_t dyn_smem[];
  __shared__ LinShared sh;
  uint8_t *smem =
      reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nM = (n + LM - 1) / LM, nN = (r + LN - 1) / LN;
  const int T = nM * nN;
  const int nsteps = (d + LK - 1) / LK;
  const int nchunks = (nsteps + LFOLD - 1) / LFOLD;

  if (threadIdx.x == 0) {
    for (int s = 0; s < LSTAGES; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh.accf[b], 1);
      mbar_init(&sh.acce[b], LEPI_WARPS);
    }
    mbar_init(&sh.drain, 1);
    sh.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, LTMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0, issued = 0, issued_par = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < T && ok; t += gridDim.x) {
        const int m0 = (t / nN) * LM, n0 = (t % nN) * LN;
        for (int ks = 0; ks < nsteps; ++ks) {
          if (*(volatile int *)&sh.abort) {
            ok = false;
            break;
          }
          if (!mbar_wait_bounded(&sh.empty[stage], phase ^ 1)) {
            lin_timeout(status, sh);
            ok = false;
            break;
          }
          uint8_t *sA = smem + (size_t)stage * LSTAGE_BYTES;
          mbar_arrive_expect_tx(&sh.full[stage], LSTAGE_BYTES);
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          // x = feature offset (a multiple of 64 fp16 = 128 bytes), y = row
          tma_load_2d(sA, &tmX, ks * LK, m0, &sh.full[stage]);
          tma_load_2d(sA + LA_BYTES, &tmW, ks * LK, n0, &sh.full[stage]);
          if (++stage == LSTAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      for (int s = 0; s < LSTAGES; ++s)
        if (issued & (1u << s)) (void)mbar_wait_bounded(&sh.full[s], (issued_par >> s) & 1u);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- UMMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = instr_desc(0, 0, 0, 0, LM, LN);
      uint32_t stage = 0, phase = 0, abuf = 0, aphase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < T && ok; t += gridDim.x) {
        for (int c = 0; c < nchunks && ok; ++c) {
          if (!mbar_wait_bounded(&sh.acce[abuf], aphase ^ 1)) {
            lin_timeout(status, sh);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t dt = tmem + abuf * LN;
          const int s0 = c * LFOLD, s1 = min(nsteps, s0 + LFOLD);
          for (int ks = s0; ks < s1; ++ks) {
            if (!mbar_wait_bounded(&sh.full[stage], phase)) {
              lin_timeout(status, sh);
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a0 = smem_u32(smem + (size_t)stage * LSTAGE_BYTES);
            const uint32_t b0 = a0 + LA_BYTES;
#pragma unroll
            for (int kk = 0; kk < LK / 16; ++kk) {
              // K-major, 128-byte swizzle: 16 fp16 = 32 bytes per K step inside
              // the 128-byte row; 8-row atoms 1024 bytes apart.
              const uint64_t ad = smem_desc(a0 + kk * 32, 16, 1024, 2);
              const uint64_t bd = smem_desc(b0 + kk * 32, 16, 1024, 2);
              umma_f16_ss(dt, ad, bd, idesc, (ks > s0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(&sh.empty[stage]);
            if (++stage == LSTAGES) {
              stage = 0;
              phase ^= 1;
            }
          }
          if (!ok) break;
          umma_commit(&sh.accf[abuf]);
          abuf ^= 1;
          if (abuf == 0) aphase ^= 1;
        }
      }
      umma_commit(&sh.drain);
      (void)mbar_wait_bounded(&sh.drain, 0);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quarter = warp & 3;             // TMEM lanes this warp may access
    const int half = (warp - 2) >> 2;         // which 128 of the tile's 256 columns
    uint32_t abuf = 0, aphase = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < T && ok; t += gridDim.x) {
      const int m0 = (t / nN) * LM, n0 = (t % nN) * LN;
      float acc[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) acc[i] = 0.f;
      for (int c = 0; c < nchunks; ++c) {
        if (!mbar_wait_bounded(&sh.accf[abuf], aphase)) {
          if (lane == 0) lin_timeout(status, sh);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t base = tmem + ((uint32_t)(quarter * 32) << 16) + abuf * LN + half * 128;
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          float v[16];
          tmem_ld_32x32b_x16(base + p * 16, v);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) acc[p * 16 + i] += v[i];
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.acce[abuf]);
        abuf ^= 1;
        if (abuf == 0) aphase ^= 1;
      }
      if (!ok) break;
      const int row = m0 + quarter * 32 + lane;
      const int cb = n0 + half * 128;
      if (row < n) {
        __half *yrow = Y + (size_t)row * r;
#pragma unroll
        for (int c8 = 0; c8 < 16; ++c8) {
          const int col = cb + c8 * 8;
          if (col < r) {   // r % 8 == 0: a chunk of 8 is wholly in or out
            __align__(16) __half2 h[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
              h[u] = __floats2half2_rn(acc[c8 * 8 + 2 * u], acc[c8 * 8 + 2 * u + 1]);
            *reinterpret_cast<uint4 *>(yrow + col) = *reinterpret_cast<const uint4 *>(h);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, LTMEM_COLS);
  }
}

// W16[row, c] = fp16(s[row, gi(c)] (q[row, c] - z[row, gi(c)])), one thread per
// 32-code chunk (b words), static unpacking of the LSB-first stream.
template <int BITS>
__global__ void dequant_fp16_kernel(const uint32_t *__restrict__ qweight,
                                    const float *__restrict__ scales,
                                    const int32_t *__restrict__ zeros,
                                    const int32_t *__restrict__ g_idx, int64_t r, int d, int group,
                                    int G, __half *__restrict__ W16) {
  constexpr uint32_t mask = (1u << BITS) - 1u;
  const int nchunk = d / 32;
  const int64_t total = r * nchunk;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / nchunk;
    const int k = (int)(i - row * nchunk);
    uint32_t w[BITS];
#pragma unroll
    for (int t = 0; t < BITS; ++t) w[t] = qweight[i * BITS + t];
    const float *srow = scales + row * G;
    const int32_t *zrow = zeros + row * G;
    __align__(16) __half2 out[16];
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      float vv[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int pos = (j + u) * BITS, wi = pos >> 5, off = pos & 31;
        uint32_t v = w[wi] >> off;
        if (off + BITS > 32) v |= w[wi + 1] << (32 - off);
        const int c = k * 32 + j + u;
        int gi = g_idx ? g_idx[c] : (group > 0 ? c / group : 0);
        gi = gi < 0 ? 0 : (gi >= G ? G - 1 : gi);
        vv[u] = srow[gi] * ((float)(v & mask) - (float)zrow[gi]);
      }
      out[j / 2] = __floats2half2_rn(vv[0], vv[1]);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(W16 + row * d + (int64_t)k * 32);
    const uint4 *src = reinterpret_cast<const uint4 *>(out);
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = src[q];
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn lin_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// fp16 row-major [rows x cols] (leading dimension cols), box {64, box_rows}, 128-byte swizzle.
bool lin_map(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, int box_rows) {
  EncodeTiledFn enc = lin_encode_fn();
  if (!enc) return false;
  const cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t gstride[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)LK, (cuuint32_t)box_rows};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), gdim, gstride, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace
}  // namespace gptq

using namespace gptq;

extern "C" int gptq_dequant_fp16(const int32_t *qweight, const float *scales, const int32_t *zeros,
                                 const int32_t *g_idx, int64_t r, int64_t d, int bits, int group,
                                 void *W16, gptq_stream_t stream) {
  if (r < 0 || r > (int64_t)INT32_MAX) return GPTQ_ERR_INVALID_ARG;
  if (d <= 0 || d % 32 != 0 || d > 65536) return GPTQ_ERR_INVALID_ARG;
  if (bits != 2 && bits != 3 && bits != 4 && bits != 8) return GPTQ_ERR_INVALID_ARG;
  if (group != -1 && (group < 32 || group % 32 != 0 || d % group != 0))
    return GPTQ_ERR_INVALID_ARG;
  if (r == 0) return GPTQ_OK;
  if (!qweight || !scales || !zeros || !W16) return GPTQ_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(W16) % 16 || reinterpret_cast<uintptr_t>(qweight) % 4 ||
      reinterpret_cast<uintptr_t>(scales) % 4 || reinterpret_cast<uintptr_t>(zeros) % 4 ||
      (g_idx && reinterpret_cast<uintptr_t>(g_idx) % 4))
    return GPTQ_ERR_INVALID_ARG;
  const int G = group < 0 ? 1 : (int)(d / group);
  const int64_t total = r * (d / 32);
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = (int64_t)num_sms() * 16;
  if (blocks > cap) blocks = cap;
  cudaStream_t st = (cudaStream_t)stream;
  const uint32_t *q = reinterpret_cast<const uint32_t *>(qweight);
  __half *w = static_cast<__half *>(W16);
  switch (bits) {
    case 2: dequant_fp16_kernel<2><<<(unsigned)blocks, 256, 0, st>>>(q, scales, zeros, g_idx, r, (int)d, group, G, w); break;
    case 3: dequant_fp16_kernel<3><<<(unsigned)blocks, 256, 0, st>>>(q, scales, zeros, g_idx, r, (int)d, group, G, w); break;
    case 4: dequant_fp16_kernel<4><<<(unsigned)blocks, 256, 0, st>>>(q, scales, zeros, g_idx, r, (int)d, group, G, w); break;
    default: dequant_fp16_kernel<8><<<(unsigned)blocks, 256, 0, st>>>(q, scales, zeros, g_idx, r, (int)d, group, G, w); break;
  }
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

extern "C" int gptq_linear_fp16(const void *X, int64_t n, int64_t d, const void *W16, int64_t r,
                                void *Y, gptq_stream_t stream) {
  if (n < 0 || n > (int64_t)INT32_MAX || r < 0 || r > 65536) return GPTQ_ERR_INVALID_ARG;
  if (d <= 0 || d % 32 != 0 || d > 65536 || r % 32 != 0) return GPTQ_ERR_INVALID_ARG;
  if (n == 0 || r == 0) return GPTQ_OK;
  if (!X || !W16 || !Y) return GPTQ_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(X) % 16 || reinterpret_cast<uintptr_t>(W16) % 16 ||
      reinterpret_cast<uintptr_t>(Y) % 16)
    return GPTQ_ERR_INVALID_ARG;
  CUtensorMap tx, tw;
  if (!lin_map(&tx, X, n, d, LM) || !lin_map(&tw, W16, r, d, LN)) {
    set_last_error_msg(__FILE__, __LINE__, "cuTensorMapEncodeTiled rejected a forward operand");
    return GPTQ_ERR_CUDA;
  }
  int *status = device_status_word();
  if (!status) return GPTQ_ERR_CUDA;
  static std::atomic<bool> attr[64] = {};
  if (const int rc = ensure_smem_attr(linear_tc_kernel, LSMEM_BYTES, attr)) return rc;
  const int64_t T = ((n + LM - 1) / LM) * ((r + LN - 1) / LN);
  const int grid = (int)(T < num_sms() ? T : num_sms());
  linear_tc_kernel<<<grid, LTHREADS, LSMEM_BYTES, (cudaStream_t)stream>>>(
      tx, tw, (int)n, (int)d, (int)r, static_cast<__half *>(Y), status);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}
