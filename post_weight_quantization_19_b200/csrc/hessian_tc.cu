// H += 2 X^T X on the sm_100a tensor cores (tcgen05 + TMEM, operands by TMA).
//
// Source: "GPTQ：一键量化大模型压缩" §二阶信息 -- the layer Hessian is
// H = 2 sum_i x_i x_i^T over the calibration activations; with X [n x d]
// (tokens x features) that is 2 X^T X.
//
// Design (B200):
//  * H is symmetric, so only output tiles that touch the upper triangle are
//    computed; the epilogue writes each upper element and its mirror once.
//  * CTA pairs (clusters of 2) share each 256 x 256 output tile through one
//    tcgen05.mma.cta_group::2 of M = 256, N = 256, K = 16: each CTA loads its
//    own 128 rows of A and half (128 columns) of B, and the pair's MMA reads
//    both halves of B from both CTAs' shared memory.  Per SM that is 32 KB of
//    X per 64-token stage for a 128 x 256 share of the product (48 KB for a
//    lone CTA), which matters because the operand stream from L2 is what
//    bounds this kernel.  No TMA load is multicast.
//  * X is token-major, so both UMMA operands are MN-major: a TMA box of
//    64 features x 64 tokens (128-byte rows, 128-byte swizzle) is one swizzle
//    atom column; each CTA's A and B halves take two boxes each.
//  * Warp roles: warp 0 issues TMA into a 6-stage ring (both CTAs; the
//    loads complete on the leader CTA's barrier), warp 1 of the leader issues
//    the pair's UMMAs into one of two 256-column TMEM accumulators and
//    commits to barriers in both CTAs, warps 2..9 of each CTA drain its TMEM.
//  * Accuracy: the tensor core's fp32 accumulation is not rounded to nearest,
//    so each TMEM accumulation chain is limited to 128 tokens and then folded
//    into fp32 registers of the epilogue warps (double-buffered TMEM, so the
//    tensor core keeps running while a chain is folded).  Longer chains bias
//    H (about 2e-6 for 512 tokens, 1e-6 for 256), which the ill-conditioned
//    Hessians of calibration sets with few tokens per feature turn into
//    different codes.  Eight epilogue warps (two per TMEM lane quarter, 128
//    columns each) fold a chain with two 32-column TMEM loads in flight per
//    wait (sixteen warps of 64 columns ran out of registers and were slower).
//  * Pacing: X is read once from HBM only while the pairs working on tiles
//    that share panels read the same token slab at about the same time.
//    Every PACE_EVERY stages each pair's leader publishes how many stages it
//    has issued (per device, tagged with the launch) and, if it is more than
//    PACE_LAG stages ahead of the slowest pair still working, waits for it --
//    a bounded wait after which it goes on anyway, so pacing can only cost
//    time, never stall the kernel (pairs not yet resident just are not waited
//    for beyond the bound).
//  * Persistent grid of one cluster per SM pair walking the tile list (in
//    bands of 8 tile rows, column by column; see tile_coords); all clusters
//    sweep the tokens at the same pace, so the current X slab is shared
//    through L2.
#include <mutex>

#include "gptq_common.cuh"

namespace gptq {

__device__ int g_device_status;

// Progress of the Hessian's CTA pairs: (launch tag << 32) | stages issued;
// the low word 0xFFFFFFFF marks a pair that has finished its tiles.
__device__ unsigned long long g_hess_progress[256];

// Per-device lookups are cached so that no runtime query runs inside a
// stream capture of the solve.
// (Atomic slots: host threads driving different devices may fill them at once.)
int *device_status_word() {
  static std::atomic<int *> cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  int *p = cache[dev].load(std::memory_order_acquire);
  if (!p) {
    void *q = nullptr;
    if (cudaGetSymbolAddress(&q, g_device_status) != cudaSuccess) return nullptr;
    p = static_cast<int *>(q);
    cache[dev].store(p, std::memory_order_release);
  }
  return p;
}

int num_sms() {
  static std::atomic<int> cache[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 1;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (!v) {
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    v = v > 0 ? v : 1;
    cache[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

namespace {

constexpr int HM = 128;                          // tile rows per CTA (UMMA M = 256 per pair)
constexpr int HN = 256;                          // tile cols  (UMMA N)
constexpr int HK = 64;                           // tokens per pipeline stage
constexpr int STAGES = 6;
constexpr int FOLD = 2;                          // stages per TMEM chain (128 tokens)
constexpr int PACE_EVERY = 64;                   // stages between progress reports
constexpr int PACE_LAG = 160;                    // stages a pair may run ahead of the slowest
constexpr int PACE_SPINS = 500;                  // bounded wait: about 1 ms, then go on
constexpr int BOXF = 64;                         // features per TMA box (128 bytes)
constexpr int BOX_BYTES = BOXF * HK * 2;         // 8 KB
constexpr int A_BYTES = HM * HK * 2;             // 16 KB: this CTA's 128 rows
constexpr int B_BYTES = (HN / 2) * HK * 2;       // 16 KB: this CTA's half of the columns
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;   // 32 KB
constexpr int NUM_EPI_WARPS = 8;                 // 2 per TMEM lane quarter, 128 columns each
constexpr int EPI_COLS = HN / (NUM_EPI_WARPS / 4);   // accumulator columns per epilogue thread
constexpr int THREADS = 32 * (2 + NUM_EPI_WARPS);
constexpr uint32_t TMEM_COLS = 512;              // two 256-column accumulators
constexpr size_t SMEM_BYTES = (size_t)STAGES * STAGE_BYTES + 1024;

struct HessShared {
  uint64_t full[STAGES];   // leader: both CTAs' loads of a stage have landed
  uint64_t empty[STAGES];  // each CTA: the pair's MMAs are done reading its stage
  uint64_t accf[2];        // each CTA: an accumulator buffer is complete
  uint64_t acce[2];        // leader: both CTAs have folded an accumulator buffer
  uint64_t drain;          // leader: every MMA issued has completed
  uint32_t tmem_base;
  int abort;
};

// Pair tile t -> (P, J): the 256 x 256 output block with rows 256 P .. and
// columns 256 J .., J >= P.  Tiles are ordered in bands of BAND tile rows;
// inside a band column by column (J from the band's first row on), each
// column's rows top to bottom.  The pairs walk the list in lockstep (tile t,
// t + pairs, ...), so the tiles in flight at one time are about pairs / BAND
// consecutive columns of one band: they read about BAND + pairs / BAND
// distinct 256-feature panels of the current token slab between them instead
// of one panel per tile, which keeps the traffic from HBM well below the
// operand stream of the tensor cores on wide layers.
constexpr int BAND = 8;

__device__ __forceinline__ void tile_coords(int t, int nP, int nJ, int &P, int &J) {
  for (int P0 = 0; P0 < nP; P0 += BAND) {
    const int hb = min(BAND, nP - P0);
    // columns P0 .. P0 + hb - 1 hold 1 .. hb tiles, later columns hb each
    const int tri = hb * (hb + 1) / 2;
    const int cnt = tri + hb * (nJ - P0 - hb);
    if (t < cnt) {
      if (t < tri) {
        int c = 0;
        while (t >= c + 1) {
          t -= c + 1;
          ++c;
        }
        J = P0 + c;
        P = P0 + t;
      } else {
        t -= tri;
        J = P0 + hb + t / hb;
        P = P0 + t % hb;
      }
      return;
    }
    t -= cnt;
  }
  P = nP - 1;
  J = nJ - 1;
}

__device__ __forceinline__ void record_timeout(int *status, HessShared &sh) {
  atomicCAS(status, 0, (int)GPTQ_ERR_TIMEOUT);
  *(volatile int *)&sh.abort = 1;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    hessian_tc_kernel(const __grid_constant__ CUtensorMap tmap, int64_t n, int d,
                      float *__restrict__ H, int *__restrict__ status, uint32_t tag) {
  extern __shared__ uint8_t dyn_smem[];
  __shared__ HessShared sh;
  uint8_t *smem =
      reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int nJ = (d + HN - 1) / HN;
  const int nP = nJ;   // row blocks of 256 (two CTAs of 128)
  int T = 0;
  for (int P = 0; P < nP; ++P) T += nJ - P;
  const int nsteps = (int)((n + HK - 1) / HK);
  const int nchunks = (nsteps + FOLD - 1) / FOLD;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh.accf[b], 1);
      mbar_init(&sh.acce[b], 2 * NUM_EPI_WARPS);
    }
    mbar_init(&sh.drain, 1);
    sh.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) prefetch_tmap(&tmap);
  if (warp == 1) {
    tmem_alloc_pair(&sh.tmem_base, TMEM_COLS);
    tmem_relinquish_pair();
  }
  // Both CTAs' barriers are initialised and the pair's TMEM is allocated
  // before either CTA signals the other.
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    // Lane 0 issues the loads; in the leader the whole warp reads the other
    // pairs' progress for pacing.
    const uint32_t full0 = cluster_addr(&sh.full[0], 0);   // the leader's barriers
    uint32_t stage = 0, phase = 0;
    uint32_t issued = 0, issued_par = 0;  // leader: bit s = stage s armed / its parity
    bool ok = true;
    uint32_t done = 0;                    // stages this pair has issued
    bool pacing = true;                   // off once a wait has run out
    const unsigned long long mine = (unsigned long long)tag << 32;
    for (int t = pair; t < T && ok; t += npairs) {
      int P, J;
      tile_coords(t, nP, nJ, P, J);
      const int i0 = P * 2 * HM + (int)rank * HM;      // this CTA's rows
      const int j0 = J * HN + (int)rank * (HN / 2);    // this CTA's half of the columns
      for (int ks = 0; ks < nsteps; ++ks, ++done) {
        if (leader && pacing && done % PACE_EVERY == 0) {
          if (lane == 0) atomicExch(&g_hess_progress[pair], mine | done);
          int spin = 0;
          for (; spin < PACE_SPINS; ++spin) {
            uint32_t slowest = 0xFFFFFFFFu;
            for (int q = lane; q < npairs; q += 32) {
              const unsigned long long v = *(volatile unsigned long long *)&g_hess_progress[q];
              const uint32_t got = (v >> 32) == tag ? (uint32_t)v : 0u;   // not started: 0
              slowest = min(slowest, got);
            }
            for (int o = 16; o > 0; o >>= 1) slowest = min(slowest, __shfl_xor_sync(0xffffffffu, slowest, o));
            if (slowest == 0xFFFFFFFFu || done <= slowest + PACE_LAG) break;
            __nanosleep(2000);
          }
          if (spin == PACE_SPINS) pacing = false;   // a pair is not coming: stop waiting
        }
        if (lane == 0) {
          // A failure in the other CTA surfaces here as a bounded wait running out.
          if (*(volatile int *)&sh.abort) {
            ok = false;
          } else if (!mbar_wait_bounded(&sh.empty[stage], phase ^ 1)) {
            record_timeout(status, sh);
            ok = false;
          } else {
            uint8_t *sA = smem + (size_t)stage * STAGE_BYTES;
            uint8_t *sB = sA + A_BYTES;
            const int y = ks * HK;
            const uint32_t fb = full0 + stage * (uint32_t)sizeof(uint64_t);
            if (leader) {
              mbar_arrive_expect_tx(&sh.full[stage], 2 * STAGE_BYTES);
              issued |= 1u << stage;
              issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
            }
            tma_load_2d_pair(sA, &tmap, i0, y, fb);
            tma_load_2d_pair(sA + BOX_BYTES, &tmap, i0 + BOXF, y, fb);
            tma_load_2d_pair(sB, &tmap, j0, y, fb);
            tma_load_2d_pair(sB + BOX_BYTES, &tmap, j0 + BOXF, y, fb);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    // This pair is done: the others no longer wait for it.
    if (leader && lane == 0) atomicExch(&g_hess_progress[pair], mine | 0xFFFFFFFFull);
    // Let every armed stage land (both CTAs' loads) before the pair can exit.
    if (leader && lane == 0)
      for (int s = 0; s < STAGES; ++s)
        if (issued & (1u << s)) (void)mbar_wait_bounded(&sh.full[s], (issued_par >> s) & 1u);
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer (leader)
    if (leader && lane == 0) {
      constexpr uint32_t idesc = instr_desc(0, 0, 1, 1, 2 * HM, HN);
      uint32_t stage = 0, phase = 0, abuf = 0, aphase = 0;
      bool ok = true;
      for (int t = pair; t < T && ok; t += npairs) {
        for (int c = 0; c < nchunks && ok; ++c) {
          if (!mbar_wait_bounded(&sh.acce[abuf], aphase ^ 1)) {
            record_timeout(status, sh);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t dt = tmem + abuf * HN;
          const int s0 = c * FOLD;
          const int s1 = min(nsteps, s0 + FOLD);
          for (int ks = s0; ks < s1; ++ks) {
            if (!mbar_wait_bounded(&sh.full[stage], phase)) {
              record_timeout(status, sh);
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a0 = smem_u32(smem + (size_t)stage * STAGE_BYTES);
            const uint32_t b0 = a0 + A_BYTES;
#pragma unroll
            for (int kk = 0; kk < HK / 16; ++kk) {
              // 16 tokens = two 8-row groups of the 128-byte swizzle atom.
              const uint64_t ad = smem_desc(a0 + kk * 2048, BOX_BYTES, 1024, 2);
              const uint64_t bd = smem_desc(b0 + kk * 2048, BOX_BYTES, 1024, 2);
              umma_f16_pair(dt, ad, bd, idesc, (ks > s0 || kk > 0) ? 1u : 0u);
            }
            umma_commit_both(&sh.empty[stage]);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1;
            }
          }
          if (!ok) break;
          umma_commit_both(&sh.accf[abuf]);
          abuf ^= 1;
          if (abuf == 0) aphase ^= 1;
        }
      }
      // Every MMA this thread issued has completed once the drain barrier fires.
      umma_commit_pair_local(&sh.drain);
      (void)mbar_wait_bounded(&sh.drain, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int ew = warp - 2;
    const int quarter = warp & 3;       // TMEM lanes this warp may access
    const int half = ew >> 2;           // which EPI_COLS of the 256 tile columns
    uint32_t abuf = 0, aphase = 0;
    bool ok = true;
    for (int t = pair; t < T && ok; t += npairs) {
      int P, J;
      tile_coords(t, nP, nJ, P, J);
      const int i0 = P * 2 * HM + (int)rank * HM, j0 = J * HN;
      float acc[EPI_COLS];
#pragma unroll
      for (int i = 0; i < EPI_COLS; ++i) acc[i] = 0.f;
      for (int c = 0; c < nchunks; ++c) {
        if (!mbar_wait_bounded(&sh.accf[abuf], aphase)) {
          if (lane == 0) record_timeout(status, sh);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t base = tmem + ((uint32_t)(quarter * 32) << 16) + abuf * HN + half * EPI_COLS;
        // two 32-column loads in flight per wait
#pragma unroll
        for (int p = 0; p < EPI_COLS / 64; ++p) {
          float v0[32], v1[32];
          tmem_ld_32x32b_x32(base + p * 64, v0);
          tmem_ld_32x32b_x32(base + p * 64 + 32, v1);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            acc[p * 64 + i] += v0[i];
            acc[p * 64 + 32 + i] += v1[i];
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(cluster_addr(&sh.acce[abuf], 0));   // the leader's
        abuf ^= 1;
        if (abuf == 0) aphase ^= 1;
      }
      if (!ok) break;
      const int row = i0 + quarter * 32 + lane;
      const int cb = j0 + half * EPI_COLS;
      if (row < d) {
#pragma unroll
        for (int i = 0; i < EPI_COLS; ++i) {
          const int col = cb + i;
          if (col < d && col >= row) {
            const float v = 2.f * acc[i];
            H[(size_t)row * d + col] += v;
            if (col > row) H[(size_t)col * d + row] += v;
          }
        }
      }
    }
  }

  // Neither CTA leaves (or frees the pair's TMEM) while the other may still
  // touch its shared memory, barriers or TMEM.
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

}  // namespace

}  // namespace gptq

using namespace gptq;

extern "C" int gptq_hessian_accumulate(const void *X, int64_t n, int64_t d, int64_t ldx, float *H,
                                       gptq_stream_t stream) {
  if (n < 0 || n > (int64_t)INT32_MAX) return GPTQ_ERR_INVALID_ARG;
  if (d <= 0 || d % 32 != 0 || d > 65536) return GPTQ_ERR_INVALID_ARG;
  if (ldx < d || ldx % 8 != 0) return GPTQ_ERR_INVALID_ARG;
  if (n == 0) return GPTQ_OK;  // nothing to add; X may be NULL
  if (!X || !H) return GPTQ_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(X) % 16 != 0 || reinterpret_cast<uintptr_t>(H) % 16 != 0)
    return GPTQ_ERR_INVALID_ARG;

  EncodeTiledFn enc = encode_fn();
  if (!enc) {
    set_last_error_msg(__FILE__, __LINE__, "cuTensorMapEncodeTiled entry point not available");
    return GPTQ_ERR_CUDA;
  }
  CUtensorMap tmap;
  const cuuint64_t gdim[2] = {(cuuint64_t)d, (cuuint64_t)n};
  const cuuint64_t gstride[1] = {(cuuint64_t)ldx * 2};
  const cuuint32_t box[2] = {(cuuint32_t)BOXF, (cuuint32_t)HK};
  const cuuint32_t estride[2] = {1, 1};
  if (enc(&tmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(X), gdim, gstride, box,
          estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
    set_last_error_msg(__FILE__, __LINE__, "cuTensorMapEncodeTiled rejected the X descriptor");
    return GPTQ_ERR_CUDA;
  }

  int *status = device_status_word();
  if (!status) {
    set_last_error_msg(__FILE__, __LINE__, "cudaGetSymbolAddress of the status word failed");
    return GPTQ_ERR_CUDA;
  }
  GPTQ_CUDA_TRY(cudaFuncSetAttribute(hessian_tc_kernel,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES));
  const int nJ = (int)((d + HN - 1) / HN);
  int T = 0;
  for (int P = 0; P < nJ; ++P) T += nJ - P;
  const int max_pairs = num_sms() / 2 > 0 ? num_sms() / 2 : 1;
  const int pairs = T < max_pairs ? T : max_pairs;
  // a tag per launch, so that progress left by an earlier launch is not read as this one's
  static std::atomic<uint32_t> launches{1};
  const uint32_t tag = launches.fetch_add(1, std::memory_order_relaxed);
  hessian_tc_kernel<<<2 * pairs, THREADS, SMEM_BYTES, (cudaStream_t)stream>>>(tmap, n, (int)d, H,
                                                                              status, tag);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}
