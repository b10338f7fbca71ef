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
// is exactly the upper Cholesky factor of H_d^-1 that GPTQ needs.  R comes
// from a blocked right-looking Cholesky on two levels: outer blocks of 1024
// columns for wide layers (so the updates of the rest of the matrix are
// products with K = 1024), each factored by 128-column steps whose diagonal
// blocks one CTA factors and inverts (leaf.cu, fp32).  U is assembled from R
// and the inverted blocks over a binary merge tree, U12 = -U11 R12 U22.  All
// the remaining work is dense GEMMs with triangular operands on the tensor
// cores (3xTF32, gemm_tc.cu); see factor_impl for the order and the streams.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <vector>

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

// Hp[a][b] = H[perm[a]][perm[b]] (+ lambda on the diagonal); rows a step by
// the grid's height (at most 65535).
__global__ void permute_sym_kernel(const float *H, int64_t ld, int d, const int *perm,
                                   const float *lambda, float *Hp) {
  pdl_wait_then_release();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= d) return;
  const int pb = perm[b];
  for (int a = blockIdx.y; a < d; a += gridDim.y) {
    float v = H[(size_t)perm[a] * ld + pb];
    if (a == b) v += *lambda;
    Hp[(size_t)a * d + b] = v;
  }
}

// inv[perm[p]] = p after checking that perm is a permutation of 0 .. d-1
// (d <= 65536); otherwise the status word is set and the later kernels skip.
__global__ void __launch_bounds__(1024) check_perm_kernel(const int *perm, int d, int *inv,
                                                          int *status) {
  __shared__ unsigned seen[65536 / 32];
  __shared__ int bad;
  pdl_wait_then_release();
  for (int i = threadIdx.x; i < 65536 / 32; i += blockDim.x) seen[i] = 0u;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  for (int p = threadIdx.x; p < d; p += blockDim.x) {
    const int c = perm[p];
    if (c < 0 || c >= d) {
      bad = 1;
      continue;
    }
    const unsigned bit = 1u << (c & 31);
    if (atomicOr(&seen[c >> 5], bit) & bit)
      bad = 1;   // a repeated entry (so another is missing)
    else
      inv[c] = p;
  }
  __syncthreads();
  if (threadIdx.x == 0 && bad) atomicCAS(status, 0, (int)GPTQ_ERR_INVALID_ARG);
}


// dst[rows x cols] = src (float4 granules; rows x cols/4 threads, grid-stride).
__global__ void copy2d_kernel(float *__restrict__ dst, int64_t ldd, const float *__restrict__ src,
                              int64_t lds, int64_t rows, int64_t cols, const int *status) {
  pdl_wait_then_release();
  if (status && *(volatile const int *)status) return;
  const int64_t q = cols / 4, total = rows * q;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / q, c = (i - r * q) * 4;
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
  dim3 grid((d + 255) / 256, d < 65535 ? d : 65535);
  GPTQ_LAUNCH_PDL(permute_sym_kernel, grid, dim3(256), 0, stream, H, ld, d, (const int *)perm,
                  lambda, Hp);
  return GPTQ_OK;
}

int launch_check_perm(const int *perm, int d, int *inv, int *status, cudaStream_t stream) {
  if (d <= 0 || d > 65536) return GPTQ_ERR_INVALID_ARG;
  GPTQ_LAUNCH_PDL(check_perm_kernel, dim3(1), dim3(1024), 0, stream, perm, d, inv, status);
  return GPTQ_OK;
}

int launch_copy2d(float *dst, int64_t ldd, const float *src, int64_t lds, int64_t rows,
                  int64_t cols, const int *status, cudaStream_t stream) {
  if (rows <= 0 || cols <= 0) return GPTQ_OK;
  if (cols % 4 || ldd % 4 || lds % 4 || reinterpret_cast<uintptr_t>(dst) % 16 ||
      reinterpret_cast<uintptr_t>(src) % 16)
    return GPTQ_ERR_INVALID_ARG;
  if (PlanRecorder *rec = plan_recorder()) {
    char a[64], b[64];
    rec->ref(dst, a, sizeof a);
    rec->ref(src, b, sizeof b);
    rec->line("C s=%d dst=%s ldd=%lld src=%s lds=%lld rows=%lld cols=%lld\n",
              plan_stream_index(stream), a, (long long)ldd, b, (long long)lds, (long long)rows,
              (long long)cols);
    return GPTQ_OK;
  }
  const int64_t total = rows * (cols / 4);
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = (int64_t)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  GPTQ_LAUNCH_PDL(copy2d_kernel, dim3((unsigned)blocks), dim3(256), 0, stream, dst, ldd, src, lds,
                  rows, cols, status);
  return GPTQ_OK;
}

int launch_priority(int level) {
  static int least = 0, greatest = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) least = greatest = 0;
  });
  if (level <= 0) return greatest;
  if (level >= 2) return least;
  return (least + greatest) / 2;   // numerically lower is higher priority
}

// ---------------------------------------------------------------- plan recording

namespace {
thread_local PlanRecorder *t_plan = nullptr;
}

PlanRecorder *plan_recorder() { return t_plan; }

int plan_stream_index(cudaStream_t s) {
  // recording mode hands out the handles 1 .. 6 for the six streams
  return (int)(reinterpret_cast<uintptr_t>(s)) - 1;
}

void PlanRecorder::line(const char *fmt, ...) {
  char tmp[512];
  va_list ap;
  va_start(ap, fmt);
  const int k = vsnprintf(tmp, sizeof tmp, fmt, ap);
  va_end(ap);
  if (k <= 0) return;
  const size_t n = (size_t)k < sizeof tmp ? (size_t)k : sizeof tmp - 1;
  if (out && used + n < cap) memcpy(out + used, tmp, n);
  used += n;
}

void PlanRecorder::ref(const float *p, char *buf, size_t n) const {
  for (int i = 0; i < 4; ++i)
    if (name[i] && p >= base[i] && p <= base[i] + len[i]) {
      snprintf(buf, n, "%s+%lld", name[i], (long long)(p - base[i]));
      return;
    }
  snprintf(buf, n, "?");
}

// ---------------------------------------------------------------- merge tree and scratch

namespace {

constexpr int64_t kLeaf = 128;       // diagonal block handled by one CTA (leaf.cu)
constexpr int64_t kOuter = 1024;     // outer block of wide layers (K of their trailing updates)
constexpr int64_t kOuterFrom = 6144; // layers at least this wide use outer blocks

// A node of n columns splits into h leading and m = n - h trailing columns,
// h a multiple of the unit: the outer block S while the node spans several
// outer blocks (so every outer block is a subtree), else the 128-column leaf.
void split(int64_t n, int64_t S, int64_t *h, int64_t *m) {
  const int64_t unit = n > S ? S : kLeaf;
  const int64_t nu = (n + unit - 1) / unit;
  *h = unit * (nu / 2);
  *m = n - *h;
}

// A node of the merge tree: columns [off, off + h + m), split at off + h.
// Outer nodes span several outer blocks; inner nodes lie inside one, with
// depths counted from that block's root.
struct MergeNode {
  int64_t off, h, m;
  int depth;
  bool outer;
};

void merge_nodes(int64_t off, int64_t n, int64_t S, int depth, std::vector<MergeNode> &out) {
  if ((n + kLeaf - 1) / kLeaf <= 1) return;
  int64_t h, m;
  split(n, S, &h, &m);
  const bool outer = n > S;
  auto child_depth = [&](int64_t c) { return (outer && c <= S) ? 0 : depth + 1; };
  merge_nodes(off + h, m, S, child_depth(m), out);
  merge_nodes(off, h, S, child_depth(h), out);
  out.push_back(MergeNode{off, h, m, depth, outer});   // after both children
}

// Scratch (floats): per depth, the largest h x m product of a non-square node
// (square nodes keep theirs in their own free lower block), separately for
// outer and inner nodes (inner merges and outer merges run on different
// streams; nodes of one kind run one at a time), then the panel copy.
struct FactorScratch {
  std::vector<size_t> outer_off, inner_off;
  size_t panel = 0, total = 0;
};

FactorScratch scratch_layout(int64_t d, int64_t S) {
  std::vector<MergeNode> nodes;
  merge_nodes(0, d, S, 0, nodes);
  std::vector<size_t> need_o, need_i;
  for (const MergeNode &nd : nodes) {
    if (nd.h == nd.m) continue;
    std::vector<size_t> &v = nd.outer ? need_o : need_i;
    if (v.size() <= (size_t)nd.depth) v.resize(nd.depth + 1, 0);
    const size_t hm = (size_t)nd.h * (size_t)nd.m;
    if (hm > v[nd.depth]) v[nd.depth] = hm;
  }
  FactorScratch L;
  size_t off = 0;
  for (size_t x : need_o) {
    L.outer_off.push_back(off);
    off += align_up(x, 64);
  }
  for (size_t x : need_i) {
    L.inner_off.push_back(off);
    off += align_up(x, 64);
  }
  L.panel = off;
  if (S < d) off += (size_t)d * (size_t)S;   // rows above an outer block x its columns
  L.total = off;
  return L;
}

}  // namespace

int64_t factor_outer_cols(int64_t d) { return d >= kOuterFrom ? kOuter : d; }

size_t factor_scratch_floats(int64_t d) { return scratch_layout(d, factor_outer_cols(d)).total; }

// ---------------------------------------------------------------- schedule

namespace {

// The streams of the factorisation.  MAIN is the caller's stream (the critical
// path: leaves, panels, the next diagonal block's update); the others are
// per-device side streams.
enum Sid { MAIN = 0, IN_TRAIL, IN_MERGE, OUT_TRAIL, OUT_NEXT, OUT_MERGE, NSID };
constexpr int kPrio[NSID] = {0, 1, 2, 1, 1, 2};

struct SideStreams {
  cudaStream_t s[NSID] = {};
  std::vector<cudaEvent_t> ev;
};

int side_streams(size_t events, SideStreams **out) {
  static SideStreams side[64];
  static std::mutex mu;
  int dev = 0;
  GPTQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return GPTQ_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(mu);
  SideStreams &ss = side[dev];
  for (int i = 1; i < NSID; ++i)
    if (!ss.s[i])
      GPTQ_CUDA_TRY(cudaStreamCreateWithPriority(&ss.s[i], cudaStreamNonBlocking,
                                                 launch_priority(kPrio[i])));
  while (ss.ev.size() < events) {
    cudaEvent_t e;
    GPTQ_CUDA_TRY(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
    ss.ev.push_back(e);
  }
  *out = &ss;
  return GPTQ_OK;
}

// Stream handles and events of one factorisation.  Without side streams every
// id maps to the caller's stream, marks are empty and waits do nothing: the
// program order of the calls below is then itself a valid order.
struct Sched {
  cudaStream_t s[NSID] = {};
  bool side = false;
  SideStreams *ss = nullptr;    // event pool (side streams on a device)
  PlanRecorder *rec = nullptr;  // recording mode: events are numbers
  size_t nev = 0;

  // An event after everything enqueued on stream i so far.
  int mark(int i, cudaEvent_t *e) {
    *e = nullptr;
    if (!side) return GPTQ_OK;
    if (rec) {
      *e = reinterpret_cast<cudaEvent_t>((uintptr_t)(++nev));
      rec->line("E s=%d e=%zu\n", i, nev);
      return GPTQ_OK;
    }
    if (nev >= ss->ev.size()) return GPTQ_ERR_INVALID_ARG;
    *e = ss->ev[nev++];
    GPTQ_CUDA_TRY(cudaEventRecord(*e, s[i]));
    return GPTQ_OK;
  }
  // Stream i waits for event e (nothing if e is empty).
  int wait(int i, cudaEvent_t e) {
    if (!side || !e) return GPTQ_OK;
    if (rec) {
      rec->line("W s=%d e=%zu\n", i, (size_t) reinterpret_cast<uintptr_t>(e));
      return GPTQ_OK;
    }
    GPTQ_CUDA_TRY(cudaStreamWaitEvent(s[i], e, 0));
    return GPTQ_OK;
  }
  // Stream `to` waits for everything enqueued on stream `from` so far.
  int join(int to, int from) {
    cudaEvent_t e;
    int rc = mark(from, &e);
    if (rc == GPTQ_OK) rc = wait(to, e);
    return rc;
  }
};

size_t events_needed(int64_t d, int64_t S) {
  const size_t nb = (size_t)((d + kLeaf - 1) / kLeaf), nS = (size_t)((d + S - 1) / S);
  return 4 * nb + 8 * nS + 4 * NSID;
}

#define FTRY(expr)                      \
  do {                                  \
    const int rc_ = (expr);             \
    if (rc_ != GPTQ_OK) return rc_;     \
  } while (0)

// U12 = -U11 R12 U22 for one node, once U11 and U22 are in place:
//   P = R12 U22  (into the node's strictly lower block when square, else the
//   scratch of its depth);  A12 = -U11 P.
int merge(const Sched &sc, int sid, float *A, int64_t ld, const MergeNode &nd, float *scratch,
          const std::vector<size_t> &depth_off, int *status) {
  const int64_t off = nd.off, h = nd.h, m = nd.m;
  float *A11 = A + off * ld + off;
  float *A12 = A + off * ld + (off + h);
  float *A22 = A + (off + h) * ld + (off + h);
  float *P;
  int64_t ldp;
  if (h == m) {
    P = A + (off + h) * ld + off;
    ldp = ld;
  } else {
    P = scratch + depth_off[nd.depth];
    ldp = m;
  }
  // P = R12 U22   (U22 upper: k <= n)
  GemmArgs g{(int)h, (int)m, (int)m, A12, ld, A22, ld, P, ldp, 1.f, 0.f, GEMM_KMAX_COL, status,
             kPrio[sid]};
  FTRY(launch_gemm(g, false, sc.s[sid]));
  // A12 = -U11 P   (U11 upper: k >= m)
  g = GemmArgs{(int)h, (int)m, (int)h, A11, ld, P, ldp, A12, ld, -1.f, 0.f, GEMM_KMIN_ROW, status,
               kPrio[sid]};
  return launch_gemm(g, false, sc.s[sid]);
}

// One outer block -- columns (and rows) [c, c + n), n <= S -- of H_d -> its U
// in place, assuming every update from the blocks to its right has been
// applied.  Right-looking by 128-column blocks from the last one (block k =
// columns [c0, c0 + ck)):
//   leaf:      A_kk -> U_kk = R_kk^-1                           (one CTA)
//   panel:     R[c:c0, k] = A[c:c0, k] U_kk^T                    (in place)
//   next:      A[c:c0, k-1] -= R[c:c0, k] R[c0-128:c0, k]^T     (the next block column)
//   trailing:  A[c:c0-128, c:c0-128] -= R[.., k] R[.., k]^T     (upper tiles)
// Only leaf -> panel -> next is on the critical path; the trailing update of
// step k runs on IN_TRAIL and must finish before step k-1's "next" (which
// writes a block column it also writes).  The merges of the block's own tree
// run on IN_MERGE as soon as the leaf of their first block has run.  *u_done
// is an event after which the block's U is complete (empty: complete in the
// order of MAIN).
int factor_block(Sched &sc, float *A, int64_t ld, int64_t c, int64_t n,
                 const std::vector<MergeNode> &nodes, float *T1, const std::vector<size_t> &ioff,
                 int *status, cudaEvent_t *u_done) {
  const int64_t nb = (n + kLeaf - 1) / kLeaf;
  std::vector<std::vector<const MergeNode *>> at(nb);
  for (const MergeNode &nd : nodes)
    if (!nd.outer && nd.off >= c && nd.off < c + n) at[(nd.off - c) / kLeaf].push_back(&nd);
  bool merged = false;
  cudaEvent_t trail_done = nullptr;   // trailing update of the step before
  for (int64_t k = nb - 1; k >= 0; --k) {
    const int64_t c0 = c + k * kLeaf;
    const int64_t ck = (c + n - c0) < kLeaf ? (c + n - c0) : kLeaf;
    FTRY(launch_leaf(A + c0 * ld + c0, ld, (int)ck, status, sc.s[MAIN]));
    if (!at[k].empty()) {
      FTRY(sc.join(IN_MERGE, MAIN));
      for (const MergeNode *nd : at[k]) FTRY(merge(sc, IN_MERGE, A, ld, *nd, T1, ioff, status));
      merged = true;
    }
    if (k == 0) break;
    float *colk = A + c * ld + c0;   // block column k, rows c .. c0
    const int64_t rows = c0 - c;
    // panel: R[c:c0, k] = A[c:c0, k] U_kk^T, in place (each tile reads only its own rows)
    GemmArgs g{(int)rows, (int)ck, (int)ck, colk, ld, A + c0 * ld + c0, ld, colk, ld, 1.f, 0.f,
               GEMM_KMIN_COL, status, kPrio[MAIN]};
    FTRY(launch_gemm(g, true, sc.s[MAIN]));
    // trailing: A[c:c0-128, c:c0-128] -= R R^T over the rows above the next block
    cudaEvent_t this_trail = nullptr;
    if (k >= 2) {
      const int64_t mt = rows - kLeaf;
      g = GemmArgs{(int)mt, (int)mt, (int)ck, colk, ld, colk, ld, A + c * ld + c, ld, -1.f, 1.f,
                   GEMM_UPPER_C, status, kPrio[IN_TRAIL]};
      FTRY(sc.join(IN_TRAIL, MAIN));
      FTRY(launch_gemm(g, true, sc.s[IN_TRAIL]));
      FTRY(sc.mark(IN_TRAIL, &this_trail));
    }
    // next: A[c:c0, k-1] -= R[c:c0, k] R[c0-128:c0, k]^T, after the previous
    // step's trailing update (it wrote block column k-1 too)
    FTRY(sc.wait(MAIN, trail_done));
    g = GemmArgs{(int)rows, (int)kLeaf, (int)ck, colk, ld, colk + (rows - kLeaf) * ld, ld,
                 A + c * ld + (c0 - kLeaf), ld, -1.f, 1.f, 0, status, kPrio[MAIN]};
    FTRY(launch_gemm(g, true, sc.s[MAIN]));
    trail_done = this_trail;
  }
  *u_done = nullptr;
  if (merged) FTRY(sc.mark(IN_MERGE, u_done));
  return GPTQ_OK;
}

// H_d = R R^T with R upper (the Cholesky taken from the bottom-right corner),
// then U = R^-1, in place: U in the upper triangle of A.
//
// Outer blocks of S columns from the last one (block K = columns [C0, C1)):
//   block:     A_KK -> U_KK                           (factor_block; 128-column steps)
//   panel:     R[0:C0, K] = A[0:C0, K] U_KK^T           (from a copy of A[0:C0, K])
//   next:      A[0:C0, K-1] -= R[0:C0, K] R[C0-S:C0, K]^T   (its diagonal block on
//              MAIN, the rows above on OUT_NEXT)
//   trailing:  A[0:C0-S, 0:C0-S] -= R[.., K] R[.., K]^T     (upper tiles, OUT_TRAIL)
// so every update of the matrix above and left of a block is a product with
// K = S; with S = d this is factor_block alone.  The trailing update of step K
// must finish before step K-1's "next" (both write block column K-2), and the
// rows-above part of "next" before step K-1's panel.
//
// Inverse: the diagonal blocks hold U_KK; each outer node of the merge tree
// forms U12 = -U11 R12 U22 once both halves are inverted.  A node's merge
// reads and writes only its own rows and columns, which are final once its
// first block's U is complete; after the rows-above part of the step before's
// "next" (the last reader of R in its rows), no later Cholesky step touches
// them (those work on the rows above it), so the outer merges run on
// OUT_MERGE alongside the Cholesky.
int factor_impl(Sched &sc, float *A, int64_t d, int64_t S, float *T1, int *status) {
  const int64_t ld = d;
  const FactorScratch L = scratch_layout(d, S);
  std::vector<MergeNode> nodes;
  merge_nodes(0, d, S, 0, nodes);
  const int64_t nS = (d + S - 1) / S;
  std::vector<std::vector<const MergeNode *>> outer_at(nS);
  for (const MergeNode &nd : nodes)
    if (nd.outer) outer_at[nd.off / S].push_back(&nd);
  float *Tp = T1 + L.panel;

  // The side streams start after everything already on MAIN.
  cudaEvent_t start;
  FTRY(sc.mark(MAIN, &start));
  for (int i = 1; i < NSID; ++i) FTRY(sc.wait(i, start));

  cudaEvent_t trail_prev = nullptr, next_prev = nullptr;
  for (int64_t K = nS - 1; K >= 0; --K) {
    const int64_t C0 = K * S, C1 = (C0 + S) < d ? (C0 + S) : d, sK = C1 - C0;
    cudaEvent_t u_done;
    FTRY(factor_block(sc, A, ld, C0, sK, nodes, T1, L.inner_off, status, &u_done));
    if (!outer_at[K].empty()) {
      // ... after the block's U, and after the previous step's "next" of the
      // rows above, which still reads R in this block's rows
      FTRY(sc.wait(OUT_MERGE, u_done));
      FTRY(sc.wait(OUT_MERGE, next_prev));
      FTRY(sc.join(OUT_MERGE, MAIN));
      for (const MergeNode *nd : outer_at[K])
        FTRY(merge(sc, OUT_MERGE, A, ld, *nd, T1, L.outer_off, status));
    }
    if (K == 0) break;
    // panel: R[0:C0, K] = A[0:C0, K] U_KK^T; block column K (rows above the
    // block) is copied first, since a tile of the in-place product would read
    // columns that other tiles write.
    FTRY(sc.wait(MAIN, u_done));
    FTRY(sc.wait(MAIN, next_prev));
    float *colK = A + C0;
    FTRY(launch_copy2d(Tp, S, colK, ld, C0, sK, status, sc.s[MAIN]));
    GemmArgs g{(int)C0, (int)sK, (int)sK, Tp, S, A + C0 * ld + C0, ld, colK, ld, 1.f, 0.f,
               GEMM_KMIN_COL, status, kPrio[MAIN]};
    FTRY(launch_gemm(g, true, sc.s[MAIN]));
    cudaEvent_t panel_done;
    FTRY(sc.mark(MAIN, &panel_done));
    // trailing (off the critical path)
    cudaEvent_t this_trail = nullptr;
    if (K >= 2) {
      const int64_t mt = C0 - S;
      g = GemmArgs{(int)mt, (int)mt, (int)sK, colK, ld, colK, ld, A, ld, -1.f, 1.f, GEMM_UPPER_C,
                   status, kPrio[OUT_TRAIL]};
      FTRY(sc.wait(OUT_TRAIL, panel_done));
      FTRY(launch_gemm(g, true, sc.s[OUT_TRAIL]));
      FTRY(sc.mark(OUT_TRAIL, &this_trail));
    }
    // next, diagonal block: A[C0-S:C0, C0-S:C0] -= R R^T, after the previous
    // step's trailing update
    FTRY(sc.wait(MAIN, trail_prev));
    cudaEvent_t next_go;
    FTRY(sc.mark(MAIN, &next_go));
    float *Rlast = A + (C0 - S) * ld + C0;   // R[C0-S:C0, K]
    g = GemmArgs{(int)S, (int)S, (int)sK, Rlast, ld, Rlast, ld, A + (C0 - S) * ld + (C0 - S), ld,
                 -1.f, 1.f, GEMM_UPPER_C, status, kPrio[MAIN]};
    FTRY(launch_gemm(g, true, sc.s[MAIN]));
    // next, rows above: A[0:C0-S, K-1] -= R[0:C0-S, K] R[C0-S:C0, K]^T
    next_prev = nullptr;
    if (K >= 2) {
      g = GemmArgs{(int)(C0 - S), (int)S, (int)sK, colK, ld, Rlast, ld, A + (C0 - S), ld, -1.f,
                   1.f, 0, status, kPrio[OUT_NEXT]};
      FTRY(sc.wait(OUT_NEXT, next_go));
      FTRY(launch_gemm(g, true, sc.s[OUT_NEXT]));
      FTRY(sc.mark(OUT_NEXT, &next_prev));
    }
    trail_prev = this_trail;
  }
  // Join: every side stream's last work (the root's merges among them).
  for (int i = 1; i < NSID; ++i) FTRY(sc.join(MAIN, i));
  return GPTQ_OK;
}

}  // namespace

int launch_factor(float *A, int64_t d, float *T1, int *status, cudaStream_t stream,
                  bool use_side) {
  const int64_t S = factor_outer_cols(d);
  Sched sc;
  for (int i = 0; i < NSID; ++i) sc.s[i] = stream;
  if (use_side) {
    FTRY(side_streams(events_needed(d, S), &sc.ss));
    for (int i = 1; i < NSID; ++i) sc.s[i] = sc.ss->s[i];
    sc.side = true;
  }
  return factor_impl(sc, A, d, S, T1, status);
}

// Recording mode (the caller installs the recorder): fake stream handles 1 .. 6.
int launch_factor_plan(float *A, int64_t d, int64_t S, float *T1, bool use_side) {
  PlanRecorder *rec = plan_recorder();
  if (!rec) return GPTQ_ERR_INVALID_ARG;
  Sched sc;
  sc.rec = rec;
  sc.side = use_side;
  for (int i = 0; i < NSID; ++i)
    sc.s[i] = reinterpret_cast<cudaStream_t>((uintptr_t)(use_side ? i + 1 : 1));
  static int dummy_status = 0;
  return factor_impl(sc, A, d, S, T1, &dummy_status);
}

}  // namespace gptq

// ---------------------------------------------------------------- diagnostic entry point

using namespace gptq;

extern "C" size_t gptq_factor_plan(int64_t d, int64_t outer_cols, int side_streams, char *buf,
                                   size_t buf_bytes) {
  if (d <= 0 || d % 32 != 0 || d > 65536) return 0;
  const int64_t S = outer_cols > 0 ? outer_cols : factor_outer_cols(d);
  if (S % kLeaf != 0 && S != d) return 0;
  const FactorScratch L = scratch_layout(d, S);
  // Fake, aligned, non-overlapping device addresses: nothing is dereferenced.
  float *A = reinterpret_cast<float *>((uintptr_t)1 << 40);
  float *T1 = reinterpret_cast<float *>((uintptr_t)1 << 44);
  PlanRecorder rec;
  rec.out = buf;
  rec.cap = buf ? buf_bytes : 0;
  rec.name[0] = "A";
  rec.base[0] = A;
  rec.len[0] = (size_t)d * (size_t)d;
  rec.name[1] = "T";
  rec.base[1] = T1;
  rec.len[1] = L.total;
  rec.line("P d=%lld S=%lld T=%zu side=%d\n", (long long)d, (long long)S, L.total,
           side_streams ? 1 : 0);
  PlanRecorder *prev = t_plan;
  t_plan = &rec;
  const int rc = launch_factor_plan(A, d, S, T1, side_streams != 0);
  t_plan = prev;
  if (rc != GPTQ_OK) return 0;
  if (buf && rec.used < buf_bytes) buf[rec.used] = 0;
  return rec.used + 1;
}
