// fp32 GEMM on the sm_100a tensor cores with error-compensated TF32 (3xTF32).
//
//   C = alpha * A * op(B) + beta * C     (row-major fp32; op(B) = B or B^T)
//
// Used by the trailing (lazy-batch) updates of the column sweep and by the
// blocked factorisation that forms U -- the dense contractions of the layer solve
// (GPTQ reading card, 方法适配: the deferred global update is a matrix product).
//
// Each fp32 operand is split into two TF32 parts and the product is
// hi*hi + hi*lo + lo*hi: three tcgen05.mma.kind::tf32 per K step.  A's parts are
// rounded to nearest (hi = rna(a), lo = rna(a - hi)); B's hi part is the raw
// tile, which the tensor core reads as its top 19 bits (truncation), and its lo
// part is rna(b - trunc(b)).  So the dropped lo*lo term has a random sign (A's
// lo is rounded to nearest) and every split residual is unbiased: the product
// is good to about 2^-21 relative with no systematic drift.  The tensor core's
// fp32 accumulation is not rounded to nearest, so each K step (12 MMAs) goes
// into one of two TMEM accumulators and is folded into fp32 registers of the
// converter warps one step later, while the next step accumulates in the other
// buffer: the long sums of the trailing updates (K up to 1024) are rounded to
// nearest like plain fp32 sums.  These GEMMs feed the Cholesky updates and the
// sweep's compensation, whose errors the ill-conditioned Hessians of
// calibration sets with few tokens per feature amplify.
//
// Tile 128 x 128 x 32 per stage: a 4-deep TMA ring of raw A/B tiles and a
// 2-deep ring of converted operands (3-deep in the CTA-pair kernel).  A (and B^T) are K-major with a 128-byte
// swizzle; a row-major B is consumed MN-major with the 128-byte swizzle of
// 32-byte atoms (the only MN-major layout for tf32).  The converter warps put
// A's hi and lo parts into tensor memory (tcgen05.st; the MMAs take A from
// TMEM) and B's lo part into shared memory (B's hi part is the raw tile), so
// the three MMAs of a K step read only B from shared memory -- shared-memory
// bandwidth is what bounds this three-pass product.  Warp 0 issues TMA, warp 1
// issues UMMA, warps 2..17 convert each landed stage, fold the previous step's
// accumulator (four warps per TMEM lane quarter, 32 columns each) and end with
// the epilogue (the CTA-pair kernel below has 8 such warps per CTA; with 8,
// the conversion and fold of a step took longer than its MMAs).  The C tile travels by TMA both ways: it is loaded into shared
// memory while the main loop runs (when beta != 0), updated there in place by
// the epilogue warps, and stored with four bulk tensor stores, so every global
// access of the epilogue is a full 128-byte line.
#include <cstdio>
#include <cstring>
#include <mutex>

#include "gptq_internal.h"

namespace gptq {
namespace {

constexpr int TM = 128, TN = 128, TK = 32;
constexpr int RS = 4;                       // TMA ring: raw A, B tiles
constexpr int LS = 3;                       // converted operands: B_lo (shared), A hi/lo (TMEM)
constexpr int TILE_BYTES = 128 * TK * 4;    // 16 KB: 128 rows x 32 fp32
constexpr int PAIR_BYTES = 2 * TILE_BYTES;  // A and B
constexpr int THREADS = 32 * 10;             // CTA-pair kernel: producer, MMA, 8 converter warps
constexpr int CONV_THREADS = 256;
// One-CTA kernel: 4 converter warps (one per TMEM lane quarter) run ahead of
// the MMAs; 8 fold/epilogue warps drain one of three TMEM accumulators while
// the tensor core fills the other two.
constexpr int CONV1_THREADS = 128;
constexpr int FOLD1_THREADS = 256;
constexpr int THREADS1 = 64 + CONV1_THREADS + FOLD1_THREADS;
constexpr int LS1 = 2;                       // converted stages of the one-CTA kernel
constexpr int NACC1 = 3;                     // its accumulators

constexpr int C_BOX_BYTES = 128 * 32 * 4;  // one 32-column box of the C tile
constexpr int C_BYTES = 4 * C_BOX_BYTES;    // 64 KB: the 128 x 128 C tile

constexpr size_t SMEM1_BYTES =
    (size_t)RS * PAIR_BYTES + (size_t)LS1 * TILE_BYTES + C_BYTES + 1024;
// TMEM columns: two 128 x 128 accumulators (K steps alternate), then per
// converted stage t the A hi part (32 columns, one K value each) and the A lo
// part (32 columns).
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_A0 = 2 * TN;
__host__ __device__ constexpr uint32_t tmem_a_hi(int t) { return TMEM_A0 + (uint32_t)t * 2 * TK; }
__host__ __device__ constexpr uint32_t tmem_a_lo(int t) { return tmem_a_hi(t) + TK; }
static_assert(TMEM_A0 + LS * 2 * TK <= TMEM_COLS, "TMEM budget");
constexpr uint32_t TMEM1_A0 = NACC1 * TN;
__host__ __device__ constexpr uint32_t tmem1_a_hi(int t) { return TMEM1_A0 + (uint32_t)t * 2 * TK; }
__host__ __device__ constexpr uint32_t tmem1_a_lo(int t) { return tmem1_a_hi(t) + TK; }
static_assert(TMEM1_A0 + LS1 * 2 * TK <= TMEM_COLS, "TMEM budget (one-CTA kernel)");

struct TcShared {
  uint64_t full[RS];
  uint64_t empty[RS];
  uint64_t conv[LS];
  uint64_t lofree[LS];
  uint64_t accf[NACC1];   // a K step's products are in accumulator b
  uint64_t acce[NACC1];   // accumulator b has been folded (by every fold warp)
  uint64_t drain;
  uint64_t cfull;
  uint32_t tmem_base;
  int abort;
};

struct TcArgs {
  int M, N, K;
  float *C;
  int64_t ldc;
  float alpha, beta;
  int flags;
  int trans_b;
  const int *status;
  int *dev_status;
  int stall_after;   // self-test only: the producer stops after this many K steps (-1: never)
  int probe;         // launch-form probe: the kernel returns at entry
};

// The tensor core reads an fp32 operand in kind::tf32 as its top 19 bits
// (sign, exponent, 10 mantissa bits): the raw tile already is hi = trunc(x).
// The split only has to produce lo = trunc(x - trunc(x)), with integer masks
// (full ALU rate): |x - hi - lo| <= 2^-20 |x|.
__device__ __forceinline__ float tf32_trunc(float x) {
  return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u);
}

// Round to the nearest TF32 value, ties away from zero, with integer ops (full
// ALU rate): add half a TF32 ulp to the magnitude bits and clear the low 13
// (a carry into the exponent is the correct rounding up).
__device__ __forceinline__ float tf32_rna(float x) {
  return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 2-D tiled TMA store shared -> global (bulk-group completion).  Elements of
// the box outside the tensor are not written.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *tmap, const void *smem_src, int x,
                                             int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(tmap)),
               "r"(x), "r"(y), "r"(smem_u32(smem_src))
               : "memory");
}

__device__ __forceinline__ void bulk_commit_and_wait_read() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// 32 lanes x 16 columns of 32-bit TMEM <- 16 registers per thread (thread t <-> lane t).
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const float (&v)[16]) {
  const uint32_t *u = reinterpret_cast<const uint32_t *>(v);
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7]),
      "r"(u[8]), "r"(u[9]), "r"(u[10]), "r"(u[11]), "r"(u[12]), "r"(u[13]), "r"(u[14]),
      "r"(u[15])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// D[tmem] (+)= A[tmem] * B[smem], kind::tf32.
__device__ __forceinline__ void umma_tf32_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Epilogue warps only (warps 2 .. 2 + N/32 - 1).
template <int N = CONV_THREADS>
__device__ __forceinline__ void epilogue_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void fail_timeout(TcShared &sh, int *dev_status) {
  if (dev_status) atomicCAS(dev_status, 0, (int)GPTQ_ERR_TIMEOUT);
  *(volatile int *)&sh.abort = 1;
}

// lo part of one 16 KB B tile: lo = rna(x - trunc(x)), same (swizzled) layout.
template <int N>
__device__ __forceinline__ void split_tile(const uint8_t *tile, uint8_t *lo, int t) {
  const float4 *p = reinterpret_cast<const float4 *>(tile);
  float4 *q = reinterpret_cast<float4 *>(lo);
#pragma unroll 4
  for (int i = t; i < TILE_BYTES / 16; i += N) {
    const float4 v = p[i];
    float4 l;
    l.x = tf32_rna(v.x - tf32_trunc(v.x));
    l.y = tf32_rna(v.y - tf32_trunc(v.y));
    l.z = tf32_rna(v.z - tf32_trunc(v.z));
    l.w = tf32_rna(v.w - tf32_trunc(v.w));
    q[i] = l;
  }
}

__global__ void __launch_bounds__(THREADS1, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, TcArgs g) {
  extern __shared__ uint8_t dyn_smem[];
  __shared__ TcShared sh;
  const int bn = blockIdx.x, bm = blockIdx.y;
  if ((g.flags & GEMM_UPPER_C) && bn < bm) return;
  const int m0 = bm * TM, n0 = bn * TN;
  int klo = 0, khi = g.K;
  if (g.flags & GEMM_KMIN_ROW) klo = max(klo, m0);
  if (g.flags & GEMM_KMIN_COL) klo = max(klo, n0);
  if (g.flags & GEMM_KMAX_COL) khi = min(khi, n0 + TN);
  const int nk = khi > klo ? (khi - klo) / TK : 0;

  uint8_t *smem =
      reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < RS; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], 1);
    }
    for (int t = 0; t < LS1; ++t) {
      mbar_init(&sh.conv[t], CONV1_THREADS / 32);
      mbar_init(&sh.lofree[t], 1);
    }
    for (int b = 0; b < NACC1; ++b) {
      mbar_init(&sh.accf[b], 1);
      mbar_init(&sh.acce[b], FOLD1_THREADS / 32);
    }
    mbar_init(&sh.drain, 1);
    mbar_init(&sh.cfull, 1);
    sh.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmC);
  }
  // Operands and C come from earlier kernels of the sequence.
  pdl_wait_then_release();
  if (threadIdx.x == 0) sh.abort = g.status ? *(volatile const int *)g.status : 0;
  __syncthreads();
  if (sh.abort) return;   // an earlier step failed: the same value in every thread
  uint8_t *loring = smem + (size_t)RS * PAIR_BYTES;       // B lo tiles
  uint8_t *ctile = loring + (size_t)LS1 * TILE_BYTES;
  const bool load_c = g.beta != 0.f;
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t issued = 0, issued_par = 0;
      // C is needed only by the epilogue: request it once the first ring
      // fill (the main loop's critical path) is on its way.
      const int c_after = min(nk, RS) - 1;
      bool c_issued = false;
      auto issue_c = [&]() {
        mbar_arrive_expect_tx(&sh.cfull, C_BYTES);
#pragma unroll
        for (int b = 0; b < 4; ++b) tma_load_2d(ctile + b * C_BOX_BYTES, &tmC, n0 + 32 * b, m0, &sh.cfull);
        c_issued = true;
      };
      if (load_c && c_after < 0) issue_c();
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % RS;
        const uint32_t ph = (kb / RS) & 1;
        if (*(volatile int *)&sh.abort || kb == g.stall_after) break;
        if (!mbar_wait_bounded(&sh.empty[s], ph ^ 1)) {
          fail_timeout(sh, g.dev_status);
          break;
        }
        uint8_t *st = smem + (size_t)s * PAIR_BYTES;
        const int k0 = klo + kb * TK;
        mbar_arrive_expect_tx(&sh.full[s], 2 * TILE_BYTES);
        tma_load_2d(st, &tmA, k0, m0, &sh.full[s]);
        if (g.trans_b) {
          tma_load_2d(st + TILE_BYTES, &tmB, k0, n0, &sh.full[s]);
        } else {
#pragma unroll
          for (int c = 0; c < TN / 32; ++c)
            tma_load_2d(st + TILE_BYTES + c * (TK * 128), &tmB, n0 + 32 * c, k0, &sh.full[s]);
        }
        issued |= 1u << s;
        issued_par = (issued_par & ~(1u << s)) | (ph << s);
        if (load_c && kb == c_after) issue_c();
      }
      for (int s = 0; s < RS; ++s)
        if (issued & (1u << s)) (void)mbar_wait_bounded(&sh.full[s], (issued_par >> s) & 1u);
      if (c_issued) (void)mbar_wait_bounded(&sh.cfull, 0);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = instr_desc(2, 2, 0, g.trans_b ? 0u : 1u, TM, TN);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % RS, t = kb % LS1, ab = kb % NACC1;
        // accumulator ab is free once the step NACC1 before has been folded
        if ((kb >= NACC1 && !mbar_wait_bounded(&sh.acce[ab], (kb / NACC1 - 1) & 1)) ||
            !mbar_wait_bounded(&sh.conv[t], (kb / LS1) & 1)) {
          fail_timeout(sh, g.dev_status);
          break;
        }
        tc_fence_after();
        const uint32_t dacc = tmem + (uint32_t)ab * TN;
        const uint32_t b = smem_u32(smem + (size_t)s * PAIR_BYTES) + TILE_BYTES;
        const uint32_t bl = smem_u32(loring + (size_t)t * TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < TK / 8; ++kk) {
          // A from TMEM: 8 K values = 8 columns per K step.
          // B^T: K-major, 8 tf32 = 32 bytes per K step inside the swizzle atom.
          // B row-major: MN-major, 8 K rows (1024 bytes) per K step.
          const uint32_t ah = tmem + tmem1_a_hi(t) + kk * 8;
          const uint32_t al = tmem + tmem1_a_lo(t) + kk * 8;
          uint64_t bd, bld;
          if (g.trans_b) {
            bd = smem_desc(b + kk * 32, 16, 1024, 2);
            bld = smem_desc(bl + kk * 32, 16, 1024, 2);
          } else {
            // MN-major tf32 uses the 128-byte swizzle with 32-byte atoms: 4-row K
            // groups 512 bytes apart, 32-column boxes 4 KB apart.
            bd = smem_desc(b + kk * 1024, TK * 128, 512, 1);
            bld = smem_desc(bl + kk * 1024, TK * 128, 512, 1);
          }
          const uint32_t acc0 = kk > 0 ? 1u : 0u;   // each K step starts its accumulator
          umma_tf32_ts(dacc, ah, bd, idesc, acc0);
          umma_tf32_ts(dacc, ah, bld, idesc, 1u);
          umma_tf32_ts(dacc, al, bd, idesc, 1u);
        }
        umma_commit(&sh.empty[s]);
        umma_commit(&sh.lofree[t]);
        umma_commit(&sh.accf[ab]);
      }
      umma_commit(&sh.drain);
      (void)mbar_wait_bounded(&sh.drain, 0);
    }
  } else if (warp < 2 + CONV1_THREADS / 32) {
    // ---------------------------------------------------------------- conversion
    // Warps 2..5 (one per TMEM lane quarter): each thread converts its A row
    // (all 32 K values) into TMEM and a quarter of B's lo part, as far ahead
    // of the MMAs as the converted stages allow.
    const int tt = threadIdx.x - 64;
    const int row = (warp & 3) * 32 + lane;   // row of the tile = TMEM lane
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % RS, t = kb % LS1;
      if (!mbar_wait_bounded(&sh.full[s], (kb / RS) & 1) ||
          !mbar_wait_bounded(&sh.lofree[t], ((kb / LS1) & 1) ^ 1)) {
        if (lane == 0) fail_timeout(sh, g.dev_status);
        break;
      }
      uint8_t *st = smem + (size_t)s * PAIR_BYTES;
      split_tile<CONV1_THREADS>(st + TILE_BYTES, loring + (size_t)t * TILE_BYTES, tt);
      // A: the raw tile is K-major with the 128-byte swizzle (16-byte chunk c
      // of row r at chunk position c ^ (r & 7)).
      const uint8_t *rowp = st + row * 128;
      const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float hi[16], lo[16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float4 v =
              *reinterpret_cast<const float4 *>(rowp + (((h * 4 + c) ^ (row & 7)) << 4));
          hi[4 * c + 0] = v.x;
          hi[4 * c + 1] = v.y;
          hi[4 * c + 2] = v.z;
          hi[4 * c + 3] = v.w;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float x = hi[i];
          hi[i] = tf32_rna(x);
          lo[i] = tf32_rna(x - hi[i]);
        }
        tmem_st_32x32b_x16(lane_base + tmem1_a_hi(t) + h * 16, hi);
        tmem_st_32x32b_x16(lane_base + tmem1_a_lo(t) + h * 16, lo);
      }
      tmem_wait_st();
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.conv[t]);
    }
  } else {
    // ---------------------------------------------------------------- fold + epilogue
    // Warps 6..13: two per TMEM lane quarter, 64 accumulator columns each.
    const int ft = threadIdx.x - 64 - CONV1_THREADS;
    const int quarter = warp & 3;
    const int half = (warp - 2 - CONV1_THREADS / 32) >> 2;
    const int row = quarter * 32 + lane;
    bool ok = true;
    float acc[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) acc[i] = 0.f;
    for (int c = 0; c < nk; ++c) {
      const int ab = c % NACC1;
      if (!mbar_wait_bounded(&sh.accf[ab], (c / NACC1) & 1)) {
        if (lane == 0) fail_timeout(sh, g.dev_status);
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t base = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)ab * TN + half * 64;
      float v0[32], v1[32];
      tmem_ld_32x32b_x32(base, v0);
      tmem_ld_32x32b_x32(base + 32, v1);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.acce[ab]);   // the registers hold it now
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        acc[i] += v0[i];
        acc[32 + i] += v1[i];
      }
    }
    if (ok && load_c && !mbar_wait_bounded(&sh.cfull, 0)) {
      if (lane == 0) fail_timeout(sh, g.dev_status);
      ok = false;
    }
    if (ok) {
      // The C tile sits in shared memory as four 128-byte-swizzled boxes of
      // 128 rows x 32 columns: 16-byte chunk c of a row is stored at chunk
      // position c ^ (row & 7), so the 8 rows of each quarter-warp phase hit
      // distinct banks.
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int box = 2 * half + j;
        const float *v = acc + 32 * j;   // compile-time offsets (unrolled): acc stays in registers
        uint8_t *rp = ctile + box * C_BOX_BYTES + row * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float4 *q = reinterpret_cast<float4 *>(rp + ((c ^ (row & 7)) << 4));
          float4 o;
          if (load_c) {
            const float4 cv = *q;
            o.x = fmaf(g.alpha, v[4 * c + 0], g.beta * cv.x);
            o.y = fmaf(g.alpha, v[4 * c + 1], g.beta * cv.y);
            o.z = fmaf(g.alpha, v[4 * c + 2], g.beta * cv.z);
            o.w = fmaf(g.alpha, v[4 * c + 3], g.beta * cv.w);
          } else {
            o = make_float4(g.alpha * v[4 * c], g.alpha * v[4 * c + 1], g.alpha * v[4 * c + 2],
                            g.alpha * v[4 * c + 3]);
          }
          *q = o;
        }
      }
      fence_async_smem();
    }
    // ok is the same in every fold warp unless a wait timed out; the barrier
    // is passed by all of them either way.
    epilogue_bar<FOLD1_THREADS>();
    if (ok && ft == 0 && !*(volatile int *)&sh.abort) {
#pragma unroll
      for (int b = 0; b < 4; ++b)
        if (n0 + 32 * b < g.N) tma_store_2d(&tmC, ctile + b * C_BOX_BYTES, n0 + 32 * b, m0);
      bulk_commit_and_wait_read();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- CTA pairs
// The same product on pairs of CTAs (a cluster of two along M): one
// tcgen05.mma.cta_group::2 of M = 256, N = 128, K = 8 takes A from both CTAs'
// tensor memory (128 rows each) and B from both CTAs' shared memory (64 of the
// 128 columns each).  Each CTA loads, converts and holds only half of B, so
// the shared-memory traffic per K step and CTA falls from about 128 KB to
// about 80 KB -- below what the tensor core needs the step to take -- for the
// same 128 x 128 of output per CTA.  Each CTA's loads complete on its own
// barrier (its converters read them); the converters of both CTAs arrive on
// the leader's barrier, which the leader's MMA thread waits on; the MMA
// commits reach both CTAs.  A K range bounded by the row tile (GEMM_KMIN_ROW)
// is the leader's; the second CTA zeroes the A values of its rows below its
// own bound.  With GEMM_UPPER_C the second CTA of a pair on the diagonal
// computes a tile below it and does not store it.

constexpr int PN = 128;                              // pair tile columns (UMMA N)
constexpr int PB_BYTES = (PN / 2) * TK * 4;          // 8 KB: this CTA's half of B
constexpr int PSTAGE_BYTES = TILE_BYTES + PB_BYTES;  // 24 KB: A rows + B half
constexpr size_t PSMEM_BYTES = (size_t)RS * PSTAGE_BYTES + (size_t)LS * PB_BYTES + C_BYTES + 1024;

__device__ __forceinline__ void split_half(const uint8_t *tile, uint8_t *lo, int t) {
  const float4 *p = reinterpret_cast<const float4 *>(tile);
  float4 *q = reinterpret_cast<float4 *>(lo);
#pragma unroll
  for (int i = t; i < PB_BYTES / 16; i += CONV_THREADS) {
    const float4 v = p[i];
    float4 l;
    l.x = tf32_rna(v.x - tf32_trunc(v.x));
    l.y = tf32_rna(v.y - tf32_trunc(v.y));
    l.z = tf32_rna(v.z - tf32_trunc(v.z));
    l.w = tf32_rna(v.w - tf32_trunc(v.w));
    q[i] = l;
  }
}

// XL: the pair's two CTAs are neighbours along x (row tile from blockIdx.x),
// else along y (row tile from blockIdx.y).
template <bool XL>
__device__ __forceinline__ void gemm_pair_body(const CUtensorMap &tmA, const CUtensorMap &tmB,
                                               const CUtensorMap &tmC, const TcArgs &g) {
  extern __shared__ uint8_t dyn_smem[];
  __shared__ TcShared sh;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int bn = XL ? blockIdx.y : blockIdx.x;
  const int bm = XL ? blockIdx.x : blockIdx.y;      // bm = 2 * pair + rank
  const int bm0 = bm - (int)rank;                   // the leader's row tile
  if ((g.flags & GEMM_UPPER_C) && bn < bm0) return; // both tiles below the diagonal
  const bool store = !((g.flags & GEMM_UPPER_C) && bn < bm);
  const int m0 = bm * TM, n0 = bn * PN;
  int klo = 0, khi = g.K;
  if (g.flags & GEMM_KMIN_ROW) klo = max(klo, bm0 * TM);
  if (g.flags & GEMM_KMIN_COL) klo = max(klo, n0);
  if (g.flags & GEMM_KMAX_COL) khi = min(khi, n0 + PN);
  const int nk = khi > klo ? (khi - klo) / TK : 0;
  const int a_klo = (g.flags & GEMM_KMIN_ROW) ? m0 : 0;   // this CTA's rows are zero below it

  uint8_t *smem =
      reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < RS; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], 1);
    }
    for (int t = 0; t < LS; ++t) {
      mbar_init(&sh.conv[t], 2 * CONV_THREADS / 32);   // leader: both CTAs' converter warps
      mbar_init(&sh.lofree[t], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh.accf[b], 1);
      mbar_init(&sh.acce[b], 2 * CONV_THREADS / 32);   // leader: both CTAs have folded
    }
    mbar_init(&sh.drain, 1);
    mbar_init(&sh.cfull, 1);
    sh.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmC);
  }
  pdl_wait_then_release();
  if (threadIdx.x == 0) sh.abort = g.status ? *(volatile const int *)g.status : 0;
  __syncthreads();
  if (sh.abort) return;   // an earlier step failed: the same value in both CTAs
  uint8_t *loring = smem + (size_t)RS * PSTAGE_BYTES;   // B lo halves
  uint8_t *ctile = loring + (size_t)LS * PB_BYTES;
  const bool load_c = g.beta != 0.f;
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
    if (lane == 0) {
      uint32_t issued = 0, issued_par = 0;
      const int c_after = min(nk, RS) - 1;
      bool c_issued = false;
      auto issue_c = [&]() {
        mbar_arrive_expect_tx(&sh.cfull, C_BYTES);
#pragma unroll
        for (int b = 0; b < 4; ++b) tma_load_2d(ctile + b * C_BOX_BYTES, &tmC, n0 + 32 * b, m0, &sh.cfull);
        c_issued = true;
      };
      if (load_c && c_after < 0) issue_c();
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % RS;
        const uint32_t ph = (kb / RS) & 1;
        if (*(volatile int *)&sh.abort) break;
        if (!mbar_wait_bounded(&sh.empty[s], ph ^ 1)) {
          fail_timeout(sh, g.dev_status);
          break;
        }
        uint8_t *st = smem + (size_t)s * PSTAGE_BYTES;
        const int k0 = klo + kb * TK;
        const int nh = n0 + (int)rank * (PN / 2);   // this CTA's half of the columns
        mbar_arrive_expect_tx(&sh.full[s], PSTAGE_BYTES);
        tma_load_2d(st, &tmA, k0, m0, &sh.full[s]);
        if (g.trans_b) {
          tma_load_2d(st + TILE_BYTES, &tmB, k0, nh, &sh.full[s]);
        } else {
#pragma unroll
          for (int c = 0; c < PN / 2 / 32; ++c)
            tma_load_2d(st + TILE_BYTES + c * (TK * 128), &tmB, nh + 32 * c, k0, &sh.full[s]);
        }
        issued |= 1u << s;
        issued_par = (issued_par & ~(1u << s)) | (ph << s);
        if (load_c && kb == c_after) issue_c();
      }
      for (int s = 0; s < RS; ++s)
        if (issued & (1u << s)) (void)mbar_wait_bounded(&sh.full[s], (issued_par >> s) & 1u);
      if (c_issued) (void)mbar_wait_bounded(&sh.cfull, 0);
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      const uint32_t idesc = instr_desc(2, 2, 0, g.trans_b ? 0u : 1u, 2 * TM, PN);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % RS, t = kb % LS, ab = kb & 1;
        if ((kb >= 2 && !mbar_wait_bounded(&sh.acce[ab], ((kb >> 1) - 1) & 1)) ||
            !mbar_wait_bounded(&sh.conv[t], (kb / LS) & 1)) {
          fail_timeout(sh, g.dev_status);
          break;
        }
        tc_fence_after();
        const uint32_t dacc = tmem + (uint32_t)ab * TN;
        const uint32_t b = smem_u32(smem + (size_t)s * PSTAGE_BYTES) + TILE_BYTES;
        const uint32_t bl = smem_u32(loring + (size_t)t * PB_BYTES);
#pragma unroll
        for (int kk = 0; kk < TK / 8; ++kk) {
          const uint32_t ah = tmem + tmem_a_hi(t) + kk * 8;
          const uint32_t al = tmem + tmem_a_lo(t) + kk * 8;
          uint64_t bd, bld;
          if (g.trans_b) {
            bd = smem_desc(b + kk * 32, 16, 1024, 2);
            bld = smem_desc(bl + kk * 32, 16, 1024, 2);
          } else {
            bd = smem_desc(b + kk * 1024, TK * 128, 512, 1);
            bld = smem_desc(bl + kk * 1024, TK * 128, 512, 1);
          }
          const uint32_t acc0 = kk > 0 ? 1u : 0u;
          umma_tf32_pair_ts(dacc, ah, bd, idesc, acc0);
          umma_tf32_pair_ts(dacc, ah, bld, idesc, 1u);
          umma_tf32_pair_ts(dacc, al, bd, idesc, 1u);
        }
        umma_commit_both(&sh.empty[s]);
        umma_commit_both(&sh.lofree[t]);
        umma_commit_both(&sh.accf[ab]);
      }
      umma_commit_pair_local(&sh.drain);
      (void)mbar_wait_bounded(&sh.drain, 0);
    }
  } else {
    // ---------------------------------------------------------------- split + fold + epilogue
    const int tt = threadIdx.x - 64;
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t conv0 = cluster_addr(&sh.conv[0], 0);   // the leader's barriers
    const uint32_t acce0 = cluster_addr(&sh.acce[0], 0);
    bool ok = true;
    float acc[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) acc[i] = 0.f;
    auto fold = [&](int c) -> bool {
      const int ab = c & 1;
      if (!mbar_wait_bounded(&sh.accf[ab], (c >> 1) & 1)) return false;
      tc_fence_after();
      const uint32_t base = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)ab * TN + half * 64;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float v[32];
        tmem_ld_32x32b_x32(base + 32 * j, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[32 * j + i] += v[i];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acce0 + ab * (uint32_t)sizeof(uint64_t));
      return true;
    };
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % RS, t = kb % LS;
      if (!mbar_wait_bounded(&sh.full[s], (kb / RS) & 1) ||
          !mbar_wait_bounded(&sh.lofree[t], ((kb / LS) & 1) ^ 1)) {
        if (lane == 0) fail_timeout(sh, g.dev_status);
        ok = false;
        break;
      }
      uint8_t *st = smem + (size_t)s * PSTAGE_BYTES;
      split_half(st + TILE_BYTES, loring + (size_t)t * PB_BYTES, tt);
      {
        const int q = warp & 3, hf = (warp - 2) >> 2;
        const int r = q * 32 + lane;
        const uint8_t *rowp = st + r * 128;
        const int kbase = klo + kb * TK + hf * 16;   // K index of this thread's first value
        float hi[16], lo[16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float4 v =
              *reinterpret_cast<const float4 *>(rowp + (((hf * 4 + c) ^ (r & 7)) << 4));
          hi[4 * c + 0] = v.x;
          hi[4 * c + 1] = v.y;
          hi[4 * c + 2] = v.z;
          hi[4 * c + 3] = v.w;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float x = kbase + i < a_klo ? 0.f : hi[i];
          hi[i] = tf32_rna(x);
          lo[i] = tf32_rna(x - hi[i]);
        }
        const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16) + hf * 16;
        tmem_st_32x32b_x16(lane_base + tmem_a_hi(t), hi);
        tmem_st_32x32b_x16(lane_base + tmem_a_lo(t), lo);
        tmem_wait_st();
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(conv0 + t * (uint32_t)sizeof(uint64_t));
      if (kb >= 1 && !fold(kb - 1)) {
        if (lane == 0) fail_timeout(sh, g.dev_status);
        ok = false;
        break;
      }
    }
    if (ok && nk > 0 && !fold(nk - 1)) {
      if (lane == 0) fail_timeout(sh, g.dev_status);
      ok = false;
    }
    if (ok && load_c && !mbar_wait_bounded(&sh.cfull, 0)) {
      if (lane == 0) fail_timeout(sh, g.dev_status);
      ok = false;
    }
    if (ok && store) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int box = 2 * half + j;
        const float *v = acc + 32 * j;
        uint8_t *rp = ctile + box * C_BOX_BYTES + row * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float4 *q = reinterpret_cast<float4 *>(rp + ((c ^ (row & 7)) << 4));
          float4 o;
          if (load_c) {
            const float4 cv = *q;
            o.x = fmaf(g.alpha, v[4 * c + 0], g.beta * cv.x);
            o.y = fmaf(g.alpha, v[4 * c + 1], g.beta * cv.y);
            o.z = fmaf(g.alpha, v[4 * c + 2], g.beta * cv.z);
            o.w = fmaf(g.alpha, v[4 * c + 3], g.beta * cv.w);
          } else {
            o = make_float4(g.alpha * v[4 * c], g.alpha * v[4 * c + 1], g.alpha * v[4 * c + 2],
                            g.alpha * v[4 * c + 3]);
          }
          *q = o;
        }
      }
      fence_async_smem();
    }
    epilogue_bar<CONV_THREADS>();
    if (ok && store && tt == 0 && !*(volatile int *)&sh.abort) {
#pragma unroll
      for (int b = 0; b < 4; ++b)
        if (n0 + 32 * b < g.N) tma_store_2d(&tmC, ctile + b * C_BOX_BYTES, n0 + 32 * b, m0);
      bulk_commit_and_wait_read();
    }
  }

  // Neither CTA frees the pair's TMEM (or leaves) while the other may still
  // use its barriers, shared memory or tensor memory.
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

// The pair kernel in three launch forms: pairs along y or along x with the
// cluster shape given at launch, and pairs along x with a compile-time
// cluster shape.  A probe launch returns at entry.
__global__ void __launch_bounds__(THREADS, 1)
    gemm_pair_y_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmC, TcArgs g) {
  if (g.probe) return;
  gemm_pair_body<false>(tmA, tmB, tmC, g);
}

__global__ void __launch_bounds__(THREADS, 1)
    gemm_pair_x_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmC, TcArgs g) {
  if (g.probe) return;
  gemm_pair_body<true>(tmA, tmB, tmC, g);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    gemm_pair_x2_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmC, TcArgs g) {
  if (g.probe) return;
  gemm_pair_body<true>(tmA, tmB, tmC, g);
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

// fp32 row-major view [rows x cols] with leading dimension ld, box {32, box_rows}.
bool make_map(CUtensorMap *m, const float *base, int64_t rows, int64_t cols, int64_t ld,
              int box_rows, CUtensorMapSwizzle swz) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t gstride[1] = {(cuuint64_t)ld * 4};
  const cuuint32_t box[2] = {32u, (cuuint32_t)box_rows};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(base), gdim, gstride, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

}  // namespace

// Launch forms of the pair GEMM, tried in this order once per device by
// probe launches (which return at entry) before the first pair-sized product:
//   0  pairs along y, cluster shape, priority and programmatic serialisation
//      given at launch;
//   1  pairs along y, cluster shape only;
//   2  pairs along x, cluster shape, priority and programmatic serialisation;
//   3  pairs along x, cluster shape only;
//   4  pairs along x, compile-time cluster shape, priority and programmatic
//      serialisation;
//   5  pairs along x, compile-time cluster shape, plain launch;
//   6  none accepted: every product runs on the single-CTA kernel.
constexpr int kPairForms = 6;
static std::atomic<int> g_pair_enabled{0};  // gptq_set_gemm_pair
static std::atomic<int> g_pair_form[64];   // form + 1 per device, 0 = not probed yet
static std::mutex g_pair_mu;
static char g_pair_log[512];               // the last probe: each form tried and its result

static dim3 pair_grid(int form, int N, int mt) {
  const unsigned cols = (unsigned)((N + PN - 1) / PN), rows = (unsigned)(2 * ((mt + 1) / 2));
  return form <= 1 ? dim3(cols, rows) : dim3(rows, cols);
}

static cudaError_t launch_pair_form(int form, int level, dim3 grid, cudaStream_t stream,
                             const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &tc,
                             const TcArgs &a) {
  if (form == 5) {
    gemm_pair_x2_kernel<<<grid, THREADS, PSMEM_BYTES, stream>>>(ta, tb, tc, a);
    return cudaGetLastError();
  }
  cudaLaunchAttribute attr[3];
  unsigned n = 0;
  if (form <= 3) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = form <= 1 ? 1 : 2;
    attr[n].val.clusterDim.y = form <= 1 ? 2 : 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (form == 0 || form == 2 || form == 4) {
    attr[n].id = cudaLaunchAttributePriority;
    attr[n].val.priority = launch_priority(level);
    ++n;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = PSMEM_BYTES;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  if (form <= 1) return cudaLaunchKernelEx(&cfg, gemm_pair_y_kernel, ta, tb, tc, a);
  if (form <= 3) return cudaLaunchKernelEx(&cfg, gemm_pair_x_kernel, ta, tb, tc, a);
  return cudaLaunchKernelEx(&cfg, gemm_pair_x2_kernel, ta, tb, tc, a);
}

// The accepted form on this device (probing on `stream` the first time, which
// must not be capturing), or -1 when it is not known and cannot be probed now.
static int pair_form(cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return kPairForms;
  const int known = g_pair_form[dev].load(std::memory_order_acquire);
  if (known > 0) return known - 1;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone)
    return -1;
  std::lock_guard<std::mutex> lock(g_pair_mu);
  if (g_pair_form[dev].load(std::memory_order_acquire) > 0)
    return g_pair_form[dev].load() - 1;
  static std::atomic<bool> attr_y[64] = {}, attr_x[64] = {}, attr_x2[64] = {};
  if (ensure_smem_attr(gemm_pair_y_kernel, PSMEM_BYTES, attr_y) ||
      ensure_smem_attr(gemm_pair_x_kernel, PSMEM_BYTES, attr_x) ||
      ensure_smem_attr(gemm_pair_x2_kernel, PSMEM_BYTES, attr_x2)) {
    (void)cudaGetLastError();
    g_pair_form[dev].store(kPairForms + 1, std::memory_order_release);
    return kPairForms;
  }
  CUtensorMap none;
  std::memset(&none, 0, sizeof none);
  TcArgs probe{};
  probe.probe = 1;
  int form = 0;
  size_t used = 0;
  g_pair_log[0] = 0;
  for (; form < kPairForms; ++form) {
    const cudaError_t e = launch_pair_form(form, 0, pair_grid(form, PN, 2), stream, none, none,
                                           none, probe);
    if (used < sizeof g_pair_log)
      used += (size_t)std::snprintf(g_pair_log + used, sizeof g_pair_log - used, "%d:%s ", form,
                                    cudaGetErrorName(e));
    if (e == cudaSuccess) break;
    (void)cudaGetLastError();
  }
  g_pair_form[dev].store(form + 1, std::memory_order_release);
  return form;
}

int gemm_pair_enabled() { return g_pair_enabled.load(std::memory_order_relaxed); }

int launch_gemm(const GemmArgs &g, bool trans_b, cudaStream_t stream) {
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return GPTQ_OK;
  if (g.K % TK != 0 || g.lda % 4 || g.ldb % 4 || g.ldc % 4 ||
      reinterpret_cast<uintptr_t>(g.A) % 16 || reinterpret_cast<uintptr_t>(g.B) % 16 ||
      reinterpret_cast<uintptr_t>(g.C) % 16) {
    set_last_error_msg(__FILE__, __LINE__, "GEMM operands not 16-byte aligned / K % 32 != 0");
    return GPTQ_ERR_INVALID_ARG;
  }
  if (PlanRecorder *rec = plan_recorder()) {
    char a[64], b[64], c[64];
    rec->ref(g.A, a, sizeof a);
    rec->ref(g.B, b, sizeof b);
    rec->ref(g.C, c, sizeof c);
    rec->line("G s=%d M=%d N=%d K=%d A=%s lda=%lld B=%s ldb=%lld C=%s ldc=%lld alpha=%g beta=%g "
              "flags=%d tb=%d prio=%d\n",
              plan_stream_index(stream), g.M, g.N, g.K, a, (long long)g.lda, b, (long long)g.ldb,
              c, (long long)g.ldc, (double)g.alpha, (double)g.beta, g.flags, trans_b ? 1 : 0,
              g.prio);
    return GPTQ_OK;
  }
  // Two or more row tiles: CTA pairs when enabled (the self-test keeps the
  // single-CTA form), in the launch form this device accepts.
  const int mt = (g.M + TM - 1) / TM;
  const int form =
      mt >= 2 && g.stall_after < 0 && g_pair_enabled.load(std::memory_order_relaxed)
          ? pair_form(stream)
          : -1;
  const bool pair = form >= 0 && form < kPairForms;
  CUtensorMap ta, tb, tc;
  const CUtensorMapSwizzle kmaj = CU_TENSOR_MAP_SWIZZLE_128B;
  const CUtensorMapSwizzle mnmaj = CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B;
  const int bt_rows = pair ? PN / 2 : TN;   // rows of a B^T box (this CTA's columns)
  if (!make_map(&ta, g.A, g.M, g.K, g.lda, TM, kmaj) ||
      !(trans_b ? make_map(&tb, g.B, g.N, g.K, g.ldb, bt_rows, kmaj)
                : make_map(&tb, g.B, g.K, g.N, g.ldb, TK, mnmaj)) ||
      !make_map(&tc, g.C, g.M, g.N, g.ldc, TM, kmaj)) {
    set_last_error_msg(__FILE__, __LINE__, "cuTensorMapEncodeTiled rejected a GEMM operand");
    return GPTQ_ERR_CUDA;
  }
  TcArgs a{g.M, g.N, g.K, g.C, g.ldc, g.alpha, g.beta, g.flags, trans_b ? 1 : 0, g.status,
           device_status_word(), g.stall_after, 0};
  cudaError_t e;
  if (pair) {
    const dim3 grid = pair_grid(form, g.N, mt);
    if (grid.y > 65535) return GPTQ_ERR_INVALID_ARG;
    count_launch();
    e = launch_pair_form(form, g.prio, grid, stream, ta, tb, tc, a);
  } else {
    static std::atomic<bool> attr[64] = {};
    if (const int rc = ensure_smem_attr(gemm_tc_kernel, SMEM1_BYTES, attr)) return rc;
    dim3 grid((g.N + TN - 1) / TN, mt);
    if (grid.y > 65535) return GPTQ_ERR_INVALID_ARG;
    count_launch();
    e = launch_pdl_prio(g.prio, gemm_tc_kernel, grid, dim3(THREADS1), SMEM1_BYTES, stream, ta, tb,
                        tc, a);
  }
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    set_last_error(__FILE__, __LINE__, "kernel launch", e);
    return GPTQ_ERR_CUDA;
  }
  return GPTQ_OK;
}

}  // namespace gptq

// ---------------------------------------------------------------- self-test

using namespace gptq;

// A 128 x 128 x 256 product whose operand loads stop after two of its eight K
// steps: the converter warps' and the MMA warp's bounded waits run out, the
// kernel records GPTQ_ERR_TIMEOUT in the status word, frees its tensor memory
// and returns.
extern "C" int gptq_selftest_timeout(float *buf, gptq_stream_t stream) {
  if (!buf || reinterpret_cast<uintptr_t>(buf) % 16) return GPTQ_ERR_INVALID_ARG;
  float *A = buf, *B = buf + 128 * 256, *C = buf + 2 * 128 * 256;
  GemmArgs g{128, 128, 256, A, 256, B, 128, C, 128, 1.f, 0.f, 0, nullptr};
  g.stall_after = 2;
  return launch_gemm(g, false, (cudaStream_t)stream);
}

// The launch form of the two-CTA product accepted on the current device
// (-1 before the first product with two or more row tiles has probed it).
extern "C" int gptq_gemm_pair_form(char *log, size_t log_bytes) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    (void)cudaGetLastError();
    return -1;
  }
  std::lock_guard<std::mutex> lock(g_pair_mu);
  if (log && log_bytes) std::snprintf(log, log_bytes, "%s", g_pair_log);
  return g_pair_form[dev].load() - 1;
}

// Products with two or more row tiles on CTA pairs (nonzero) or on the one-CTA
// kernel (0, the default: measured faster on the 4096- and 49152-wide layers).
extern "C" int gptq_set_gemm_pair(int enable) {
  return g_pair_enabled.exchange(enable ? 1 : 0);
}
