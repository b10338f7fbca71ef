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
// from a blocked right-looking Cholesky over 128-column blocks whose diagonal
// blocks one CTA factors and inverts (leaf.cu, fp32); U is assembled from R and
// those inverted blocks over a binary merge tree, U12 = -U11 R12 U22.  All the
// remaining work is dense GEMMs with triangular operands on the tensor cores
// (3xTF32, gemm_tc.cu); see launch_factor for the order and the streams.
#include <mutex>
#include <vector>

#include "gptq_common.cuh"
#include "gptq_internal.h"

namespace gptq {
namespace {

constexpr int64_t kLeaf = 128;   // diagonal block handled by one CTA (leaf.cu)

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

int launch_priority(bool background) {
  static int least = 0, greatest = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) least = greatest = 0;
  });
  return background ? least : greatest;
}

namespace {

// Node sizes of the merge tree: a node of n columns (nblk = ceil(n/128)
// blocks) splits into h = 128 * floor(nblk/2) leading and m = n - h trailing
// columns.  The largest node of each depth is the trailing child of the
// largest node of the depth above.
void split(int64_t n, int64_t *h, int64_t *m) {
  const int64_t nblk = (n + kLeaf - 1) / kLeaf;
  *h = kLeaf * (nblk / 2);
  *m = n - *h;
}

}  // namespace

size_t factor_scratch_floats(int64_t d) {
  size_t total = 0;
  for (int64_t n = d; (n + kLeaf - 1) / kLeaf > 1;) {
    int64_t h, m;
    split(n, &h, &m);
    total += (size_t)h * (size_t)m;
    n = m;
  }
  return total;
}

namespace {

// Per-device streams for the work taken off the critical path -- the trailing
// rank-128 updates and the merges that assemble U -- and events to order them.
struct SideStreams {
  cudaStream_t trail = nullptr, merge = nullptr;
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
  if (!ss.trail) {
    GPTQ_CUDA_TRY(cudaStreamCreateWithPriority(&ss.trail, cudaStreamNonBlocking,
                                               launch_priority(true)));
    GPTQ_CUDA_TRY(cudaStreamCreateWithPriority(&ss.merge, cudaStreamNonBlocking,
                                               launch_priority(true)));
  }
  while (ss.ev.size() < events) {
    cudaEvent_t e;
    GPTQ_CUDA_TRY(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
    ss.ev.push_back(e);
  }
  *out = &ss;
  return GPTQ_OK;
}

// A node of the merge tree: columns [off, off + h + m), split at off + h.
struct MergeNode {
  int64_t off, h, m;
  int depth;
};

void merge_nodes(int64_t off, int64_t n, int depth, std::vector<MergeNode> &out) {
  if ((n + kLeaf - 1) / kLeaf <= 1) return;
  int64_t h, m;
  split(n, &h, &m);
  merge_nodes(off + h, m, depth + 1, out);
  merge_nodes(off, h, depth + 1, out);
  out.push_back(MergeNode{off, h, m, depth});   // after both children
}

// U12 = -U11 R12 U22 for one node, once U11 and U22 are in place:
//   P = R12 U22  (into the node's strictly lower block when square, else
//   its depth's scratch);  A12 = -U11 P.
int merge(float *A, int64_t ld, const MergeNode &nd, float *scratch,
          const std::vector<size_t> &depth_off, int *status, bool background,
          cudaStream_t st) {
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
  int rc;
  // P = R12 U22   (U22 upper: k <= n)
  GemmArgs g{(int)h, (int)m, (int)m, A12, ld, A22, ld, P, ldp, 1.f, 0.f, GEMM_KMAX_COL, status,
             background};
  if ((rc = launch_gemm(g, false, st)) != GPTQ_OK) return rc;
  // A12 = -U11 P   (U11 upper: k >= m)
  g = GemmArgs{(int)h, (int)m, (int)h, A11, ld, P, ldp, A12, ld, -1.f, 0.f, GEMM_KMIN_ROW, status,
               background};
  return launch_gemm(g, false, st);
}

}  // namespace

// H_d = R R^T with R upper (the Cholesky taken from the bottom-right corner),
// then U = R^-1, in place: U in the upper triangle of A.
//
// Cholesky, right-looking by 128-column blocks from the last one (block k =
// columns [c0, c0 + ck)):
//   leaf:      A_kk -> U_kk = R_kk^-1                       (one CTA)
//   panel:     R[0:c0, k] = A[0:c0, k] U_kk^T                (k tiles)
//   next:      A[0:c0, k-1] -= R[0:c0, k] R[c0-128:c0, k]^T  (the next block column)
//   trailing:  A[0:c0-128, 0:c0-128] -= R[.., k] R[.., k]^T  (upper tiles)
// Only leaf -> panel -> next is on the critical path; the trailing update of
// step k runs on a least-priority side stream and must finish before step
// k-1's "next" (which writes a block column it also writes).
//
// Inverse: the diagonal blocks already hold U_kk; each node of the merge tree
// forms U12 = -U11 R12 U22 once both halves are inverted.  A node's merge
// reads only R and U in its own columns, which are final as soon as the leaf
// of its first block has run, and nothing the later Cholesky steps touch
// (rows above the node), so merges run on a third stream alongside the
// Cholesky.
int launch_factor(float *A, int64_t d, float *T1, int *status, cudaStream_t stream,
                  bool use_side) {
  const int64_t ld = d;
  const int64_t nb = (d + kLeaf - 1) / kLeaf;
  if (nb <= 1) return launch_leaf(A, ld, (int)d, status, stream);
  std::vector<size_t> depth_off;
  {
    size_t off = 0;
    for (int64_t n = d; (n + kLeaf - 1) / kLeaf > 1;) {
      int64_t h, m;
      split(n, &h, &m);
      depth_off.push_back(off);
      off += (size_t)h * (size_t)m;
      n = m;
    }
  }
  std::vector<MergeNode> nodes;
  merge_nodes(0, d, 0, nodes);
  // Nodes by the block of their first column, children before parents.
  std::vector<std::vector<MergeNode>> at(nb);
  for (const MergeNode &nd : nodes) at[nd.off / kLeaf].push_back(nd);

  SideStreams *ss = nullptr;
  if (use_side) {
    const int rc = side_streams((size_t)(3 * nb + 2), &ss);
    if (rc != GPTQ_OK) return rc;
  }
  size_t nev = 0;
  auto event = [&]() { return ss->ev[nev++]; };
  cudaStream_t st = stream;
  cudaEvent_t trail_done = nullptr;   // trailing update of the step before
  int rc;
  if (ss) {
    // The side streams start after everything already on `stream`.
    cudaEvent_t start = event();
    GPTQ_CUDA_TRY(cudaEventRecord(start, st));
    GPTQ_CUDA_TRY(cudaStreamWaitEvent(ss->trail, start, 0));
    GPTQ_CUDA_TRY(cudaStreamWaitEvent(ss->merge, start, 0));
  }
  for (int64_t k = nb - 1; k >= 0; --k) {
    const int64_t c0 = k * kLeaf;
    const int64_t ck = (d - c0) < kLeaf ? (d - c0) : kLeaf;
    if ((rc = launch_leaf(A + c0 * ld + c0, ld, (int)ck, status, st)) != GPTQ_OK) return rc;
    // Merges whose first block is k: their halves are inverted now.
    if (!at[k].empty()) {
      cudaStream_t ms = st;
      if (ss) {
        cudaEvent_t e = event();
        GPTQ_CUDA_TRY(cudaEventRecord(e, st));
        GPTQ_CUDA_TRY(cudaStreamWaitEvent(ss->merge, e, 0));
        ms = ss->merge;
      }
      for (const MergeNode &nd : at[k])
        if ((rc = merge(A, ld, nd, T1, depth_off, status, ss != nullptr, ms)) != GPTQ_OK)
          return rc;
    }
    if (k == 0) break;
    float *colk = A + c0;   // block column k, rows 0 .. c0
    // panel: R[0:c0, k] = A[0:c0, k] U_kk^T, in place (each tile reads only its own rows)
    GemmArgs g{(int)c0, (int)ck, (int)ck, colk, ld, A + c0 * ld + c0, ld, colk, ld, 1.f, 0.f,
               GEMM_KMIN_COL, status};
    if ((rc = launch_gemm(g, true, st)) != GPTQ_OK) return rc;
    // trailing: A[0:c0-128, 0:c0-128] -= R R^T over the rows above the next block
    cudaEvent_t this_trail = nullptr;
    if (k >= 2) {
      const int64_t mt = c0 - kLeaf;
      g = GemmArgs{(int)mt, (int)mt, (int)ck, colk, ld, colk, ld, A, ld, -1.f, 1.f, GEMM_UPPER_C,
                   status, ss != nullptr};
      if (ss) {
        cudaEvent_t fork = event();
        this_trail = event();
        GPTQ_CUDA_TRY(cudaEventRecord(fork, st));
        GPTQ_CUDA_TRY(cudaStreamWaitEvent(ss->trail, fork, 0));
        if ((rc = launch_gemm(g, true, ss->trail)) != GPTQ_OK) return rc;
        GPTQ_CUDA_TRY(cudaEventRecord(this_trail, ss->trail));
      } else if ((rc = launch_gemm(g, true, st)) != GPTQ_OK) {
        return rc;
      }
    }
    // next: A[0:c0, k-1] -= R[0:c0, k] R[c0-128:c0, k]^T, after the previous
    // step's trailing update (it wrote block column k-1 too)
    if (trail_done) GPTQ_CUDA_TRY(cudaStreamWaitEvent(st, trail_done, 0));
    g = GemmArgs{(int)c0, (int)kLeaf, (int)ck, colk, ld, colk + (c0 - kLeaf) * ld, ld,
                 A + (c0 - kLeaf), ld, -1.f, 1.f, 0, status};
    if ((rc = launch_gemm(g, true, st)) != GPTQ_OK) return rc;
    trail_done = this_trail;
  }
  if (ss) {
    // Join: the last merges (the root's) and any trailing update still running.
    cudaEvent_t e = event();
    GPTQ_CUDA_TRY(cudaEventRecord(e, ss->merge));
    GPTQ_CUDA_TRY(cudaStreamWaitEvent(st, e, 0));
    e = event();
    GPTQ_CUDA_TRY(cudaEventRecord(e, ss->trail));
    GPTQ_CUDA_TRY(cudaStreamWaitEvent(st, e, 0));
  }
  return GPTQ_OK;
}

}  // namespace gptq
