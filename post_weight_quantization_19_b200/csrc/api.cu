// C-ABI entry points of the layer solve: validation, workspace layout, and the
// stream-ordered sequence of kernels (see include/gptq.h for the contract).
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "gptq_internal.h"

namespace gptq {

std::atomic<uint64_t> g_launches{0};

namespace {
thread_local char g_last_error[512] = "";
}

void set_last_error(const char *file, int line, const char *what, cudaError_t e) {
  const char *base = strrchr(file, '/');
  snprintf(g_last_error, sizeof(g_last_error), "%s:%d %s: %s (%s)", base ? base + 1 : file, line,
           what, cudaGetErrorName(e), cudaGetErrorString(e));
}

void set_last_error_msg(const char *file, int line, const char *msg) {
  const char *base = strrchr(file, '/');
  snprintf(g_last_error, sizeof(g_last_error), "%s:%d %s", base ? base + 1 : file, line, msg);
}

namespace {

constexpr int kSuperblock = 1024;  // columns per global (deferred) trailing update

bool valid_bits(int b) { return b == 2 || b == 3 || b == 4 || b == 8; }

bool valid_options(int options) {
  return (options & ~(GPTQ_ACT_ORDER | GPTQ_SYMMETRIC | GPTQ_STATIC_GROUPS)) == 0;
}

bool valid_layer(int64_t r, int64_t d, int bits, int group, int block) {
  if (r < 0 || r > (int64_t)INT32_MAX / 2) return false;
  if (d <= 0 || d % 32 != 0 || d > 65536) return false;
  if (!valid_bits(bits)) return false;
  if (block != 32 && block != 64 && block != 128) return false;
  if (group != -1) {
    if (group < 32 || group % 32 != 0 || d % group != 0) return false;
    if (!(block % group == 0 || group % block == 0)) return false;
  }
  return true;
}

// Columns between global trailing updates: a multiple of the block, and
// aligned so that no quantisation group straddles a superblock end unless it
// also starts at a superblock start (then every column it reads is current).
int superblock(int64_t d, int group, int block) {
  int S = kSuperblock;
  if (group > block && S % group != 0 && group % S != 0) S = group;
  const int64_t dr = (d + block - 1) / block * block;
  if (S > dr) S = (int)dr;
  return S;
}

struct Layout {
  size_t Wk, ErrS, codes_p, perm, inv, Hp, T1, loss_rows, dsq_rows, out, lambda, status, total;
};

Layout layout(int64_t r, int64_t d, int group, int block, int options) {
  Layout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  const int S = superblock(d, group, block);
  L.Wk = take((size_t)r * d * 4);
  L.ErrS = take((size_t)r * S * 4);
  L.codes_p = take((size_t)r * d);
  L.perm = take((size_t)d * 4);
  L.inv = take((size_t)d * 4);
  L.Hp = take((options & GPTQ_ACT_ORDER) ? (size_t)d * d * 4 : 0);
  L.T1 = take(factor_scratch_floats(d) * 4);
  L.loss_rows = take((size_t)r * 8);
  L.dsq_rows = take((size_t)r * 8);
  L.out = take(4 * 8);
  L.lambda = take(4);
  L.status = take(16);
  L.total = off;
  return L;
}

// Phase timing (optional).  The solve replays as four CUDA graphs, one per
// phase, and the phase events are recorded on the solve's stream between them
// (never inside a capture), then read after the call's final synchronisation.
// t_timing is set only around a gptq_quantize_layer call that times its phases
// (not the no-alloc path, which creates nothing).
bool g_timing = false;
float g_phase_ms[4] = {0, 0, 0, 0};
cudaEvent_t g_ev[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};
int g_ev_device = -1;
thread_local bool t_timing = false;

int ensure_phase_events() {
  int dev = 0;
  GPTQ_CUDA_TRY(cudaGetDevice(&dev));
  if (g_ev_device != dev) {
    for (auto &e : g_ev) e = nullptr;   // events of another device's context are not reused
    g_ev_device = dev;
  }
  for (auto &e : g_ev)
    if (!e) GPTQ_CUDA_TRY(cudaEventCreate(&e));
  return GPTQ_OK;
}

int record(int i, cudaStream_t s) {
  if (!t_timing) return GPTQ_OK;
  GPTQ_CUDA_TRY(cudaEventRecord(g_ev[i], s));
  return GPTQ_OK;
}

// ---------------------------------------------------------------- graph cache

struct GraphKey {
  const void *W, *H, *W_hat, *qweight, *scales, *zeros, *g_idx, *codes, *ws;
  size_t ws_bytes;
  cudaStream_t stream;
  int64_t r, d;
  int bits, group, block;
  float damp;
  int options;
  int segment;   // phase of the solve this graph replays
  int device = -1;
  int pair = 0;  // the two-CTA GEMM was enabled when the graph was captured
  bool operator==(const GraphKey &o) const {
    return W == o.W && H == o.H && W_hat == o.W_hat && qweight == o.qweight &&
           scales == o.scales && zeros == o.zeros && g_idx == o.g_idx && codes == o.codes &&
           ws == o.ws && ws_bytes == o.ws_bytes && stream == o.stream && r == o.r &&
           d == o.d && bits == o.bits && group == o.group && block == o.block &&
           memcmp(&damp, &o.damp, sizeof(float)) == 0 && options == o.options &&
           segment == o.segment && device == o.device && pair == o.pair;
  }
};

struct GraphEntry {
  GraphKey key;
  int seen = 0;
  cudaGraphExec_t exec = nullptr;
  uint64_t kernels = 0;
  uint64_t last_use = 0;
};

std::mutex g_graph_mu;
std::vector<GraphEntry> g_graphs;
uint64_t g_graph_clock = 0;
constexpr size_t kMaxGraphs = 32;

template <class F>
int run_graph_cached(GraphKey key, cudaStream_t st, F &&enqueue) {
  GPTQ_CUDA_TRY(cudaGetDevice(&key.device));
  key.pair = gemm_pair_enabled();
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (st == nullptr || cudaStreamIsCapturing(st, &cs) != cudaSuccess ||
      cs != cudaStreamCaptureStatusNone)
    return enqueue();
  std::lock_guard<std::mutex> lock(g_graph_mu);
  GraphEntry *e = nullptr;
  for (auto &x : g_graphs)
    if (x.key == key) e = &x;
  if (!e) {
    if (g_graphs.size() >= kMaxGraphs) {
      auto victim = g_graphs.begin();
      for (auto it = g_graphs.begin(); it != g_graphs.end(); ++it)
        if (it->last_use < victim->last_use) victim = it;
      if (victim->exec) cudaGraphExecDestroy(victim->exec);
      g_graphs.erase(victim);
    }
    g_graphs.push_back(GraphEntry{key});
    e = &g_graphs.back();
  }
  e->last_use = ++g_graph_clock;
  if (!e->exec && e->seen++ == 0) return enqueue();   // first sighting: run directly
  if (!e->exec) {
    const uint64_t before = g_launches.load();
    GPTQ_CUDA_TRY(cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal));
    const int rc = enqueue();
    cudaGraph_t graph = nullptr;
    const cudaError_t ce = cudaStreamEndCapture(st, &graph);
    const uint64_t captured = g_launches.load() - before;
    g_launches.fetch_sub(captured);
    if (rc != GPTQ_OK || ce != cudaSuccess) {
      if (graph) cudaGraphDestroy(graph);
      (void)cudaGetLastError();
      return rc != GPTQ_OK ? rc : GPTQ_ERR_CUDA;
    }
    const cudaError_t ie = cudaGraphInstantiate(&e->exec, graph, 0);
    cudaGraphDestroy(graph);
    if (ie != cudaSuccess) {
      e->exec = nullptr;
      set_last_error(__FILE__, __LINE__, "cudaGraphInstantiate", ie);
      return GPTQ_ERR_CUDA;
    }
    e->kernels = captured;
  }
  GPTQ_CUDA_TRY(cudaGraphLaunch(e->exec, st));
  count_launch(e->kernels);
  return GPTQ_OK;
}

#define GPTQ_TRY(expr)                      \
  do {                                      \
    const int rc_ = (expr);                 \
    if (rc_ != GPTQ_OK) return rc_;         \
  } while (0)

}  // namespace
}  // namespace gptq

using namespace gptq;

extern "C" const char *gptq_status_string(int status) {
  switch (status) {
    case GPTQ_OK: return "ok";
    case GPTQ_ERR_INVALID_ARG: return "invalid argument";
    case GPTQ_ERR_NOT_PD: return "damped Hessian is not positive definite";
    case GPTQ_ERR_CUDA: return "CUDA runtime error";
    case GPTQ_ERR_NO_MEMORY: return "workspace too small";
    case GPTQ_ERR_TIMEOUT: return "bounded in-kernel wait timed out";
    default: return "unknown status";
  }
}

extern "C" uint64_t gptq_launch_count(void) { return g_launches.load(); }

extern "C" const char *gptq_last_error(void) { return g_last_error; }

extern "C" int gptq_set_phase_timing(int enable) {
  g_timing = enable != 0;
  return GPTQ_OK;
}

extern "C" int gptq_last_phase_ms(float *ms, int n) {
  if (!ms || n < 0) return 0;
  const int k = n < 4 ? n : 4;
  for (int i = 0; i < k; ++i) ms[i] = g_phase_ms[i];
  return k;
}

extern "C" int gptq_check_device_status(gptq_stream_t stream) {
  GPTQ_CUDA_TRY(cudaStreamSynchronize((cudaStream_t)stream));
  int *w = device_status_word();
  if (!w) return GPTQ_ERR_CUDA;
  int v = 0;
  GPTQ_CUDA_TRY(cudaMemcpy(&v, w, sizeof(int), cudaMemcpyDeviceToHost));
  if (v != 0) {
    const int zero = 0;
    GPTQ_CUDA_TRY(cudaMemcpy(w, &zero, sizeof(int), cudaMemcpyHostToDevice));
  }
  return v;
}

extern "C" size_t gptq_quantize_workspace_bytes(int64_t r, int64_t d, int bits, int group,
                                                int block, int options) {
  if (!valid_layer(r, d, bits, group, block) || !valid_options(options)) return 0;
  return layout(r, d, group, block, options).total;
}

namespace gptq {
namespace {

// Phases 0-1 on `st`: lambda = damp * mean(diag H), the act-order permutation
// (perm, inv and the permuted H_d in Hp), then U in place of H_d.  *U is set to
// the matrix that holds U (H, or Hp under act-order).
// Phase 0: lambda = damp * mean(diag H) and, under act-order, the permutation
// (perm, inv) and the permuted H_d in Hp.  Returns the matrix to factor (H, or
// Hp under act-order).
float *enqueue_damp(float *H, int64_t d, float damp, bool act_order, int *perm, int *inv,
                    float *lambda, float *Hp, cudaStream_t st, int *rc) {
  const int di = (int)d;
  if (act_order) {
    *rc = launch_damp(H, d, di, damp, false, lambda, st);
    if (*rc == GPTQ_OK) *rc = launch_act_order(H, d, di, perm, inv, lambda, Hp, st);
    return Hp;
  }
  *rc = launch_damp(H, d, di, damp, true, lambda, st);
  return H;
}

// Phases 0-1 on `st`: damping / act-order, then U in place of H_d.  *U is set
// to the matrix that holds U (H, or Hp under act-order).
int enqueue_factor(float *H, int64_t d, float damp, bool act_order, int *perm, int *inv,
                   float *lambda, float *Hp, float *T1, int *status, cudaStream_t st,
                   bool use_side, float **U) {
  int rc = GPTQ_OK;
  float *Hf = enqueue_damp(H, d, damp, act_order, perm, inv, lambda, Hp, st, &rc);
  GPTQ_TRY(rc);
  GPTQ_TRY(launch_factor(Hf, d, T1, status, st, use_side));
  *U = Hf;
  return GPTQ_OK;
}

// Everything the sweep half needs: inputs, outputs and its part of the workspace.
struct SweepPlan {
  const float *W;
  int r, d, bits, group, block, sym, static_groups;
  const float *U;
  const int *perm, *inv;   // act-order only (NULL otherwise)
  const float *lambda;
  float *W_hat;
  int32_t *qweight;
  float *scales;
  int32_t *zeros;
  int32_t *g_idx;
  uint8_t *codes;
  float *Wk, *ErrS;
  uint8_t *codes_p;
  double *loss_rows, *dsq_rows, *out;
  int *status;
};

// Phases 2-3 on `st`: working copy of W, column sweep in blocks with lazy
// trailing updates, then unpermute, loss and packing.  The sweep kernels read
// their U block before waiting for their predecessor, so the kernel just
// before each of them must not write U: the copy of W separates the
// factorisation from the first block.
int enqueue_sweep(const SweepPlan &p, cudaStream_t st) {
  const int ri = p.r, di = p.d, group = p.group, block = p.block;
  const int G = group < 0 ? 1 : di / group;
  const int S = superblock(p.d, group, block);
  GPTQ_TRY(launch_gather_w(p.W, ri, di, p.perm, p.Wk, p.status, st));
  if (group < 0)
    GPTQ_TRY(launch_row_params(p.Wk, ri, di, di, p.bits, p.sym, p.scales, p.zeros, p.status, st));
  if (p.static_groups)
    GPTQ_TRY(launch_row_params(p.W, ri, di, group, p.bits, p.sym, p.scales, p.zeros, p.status, st));
  for (int s0 = 0; s0 < di; s0 += S) {
    const int sEnd = s0 + S < di ? s0 + S : di;
    for (int j0 = s0; j0 < sEnd; j0 += block) {
      const int j1 = j0 + block < sEnd ? j0 + block : sEnd;
      SweepArgs a{};
      a.Wk = p.Wk;
      a.ldw = di;
      a.U = p.U;
      a.ldu = di;
      a.r = ri;
      a.j0 = j0;
      a.ncols = j1 - j0;
      a.bits = p.bits;
      a.group = group;
      a.scales = p.scales;
      a.zeros = p.zeros;
      a.G = G;
      a.flags = (p.sym ? SWEEP_SYM : 0) | (p.static_groups ? SWEEP_STATIC : 0);
      a.codes = p.codes_p;
      a.perm = p.static_groups && p.perm ? p.perm : nullptr;
      a.err = p.ErrS + (j0 - s0);
      a.lde = S;
      a.loss_rows = p.loss_rows;
      a.status = p.status;
      GPTQ_TRY(launch_sweep_block(a, block, st));
      if (j1 < sEnd) {
        // Rest of this superblock: W[:, j1:sEnd] -= E_blk U[j0:j1, j1:sEnd]
        GemmArgs g{ri, sEnd - j1, j1 - j0, p.ErrS + (j0 - s0), S, p.U + (size_t)j0 * di + j1, di,
                   p.Wk + j1, di, -1.f, 1.f, 0, p.status};
        GPTQ_TRY(launch_gemm(g, false, st));
      }
    }
    if (sEnd < di) {
      // Deferred global update: W[:, sEnd:] -= E_S U[s0:sEnd, sEnd:]
      GemmArgs g{ri, di - sEnd, sEnd - s0, p.ErrS, S, p.U + (size_t)s0 * di + sEnd, di,
                 p.Wk + sEnd, di, -1.f, 1.f, 0, p.status};
      GPTQ_TRY(launch_gemm(g, false, st));
    }
  }
  return GPTQ_OK;
}

// Phase 3 on `st`: unpermute, loss and packing.
int enqueue_finalize(const SweepPlan &p, cudaStream_t st) {
  const int ri = p.r, di = p.d, group = p.group;
  FinalizeArgs f{};
  f.W = p.W;
  f.Wk = p.Wk;
  f.codes_p = p.codes_p;
  f.inv = p.inv;
  f.r = ri;
  f.d = di;
  f.bits = p.bits;
  f.group = group;
  f.static_groups = p.static_groups;
  f.W_hat = p.W_hat;
  f.codes = p.codes;
  f.qweight = p.qweight;
  f.g_idx = p.g_idx;
  f.dsq_rows = p.dsq_rows;
  f.status = p.status;
  GPTQ_TRY(launch_finalize(f, st));
  GPTQ_TRY(launch_loss_reduce(p.loss_rows, p.dsq_rows, ri, p.lambda, p.out, p.status, st));
  return GPTQ_OK;
}

}  // namespace

int check_layer_args(const float *W, int64_t r, int64_t d, const float *H, int bits, int group,
                     int block, float damp, int options, const float *W_hat,
                     const int32_t *qweight, const float *scales, const int32_t *zeros,
                     const int32_t *g_idx, const uint8_t *codes) {
  if (!valid_layer(r, d, bits, group, block)) return GPTQ_ERR_INVALID_ARG;
  if (!(damp >= 0.f) || damp > 1e30f) return GPTQ_ERR_INVALID_ARG;
  if (!valid_options(options)) return GPTQ_ERR_INVALID_ARG;
  if (r == 0) return GPTQ_OK;   // nothing is read or written
  if (!W || !H || !qweight || !scales || !zeros) return GPTQ_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(W) % 16 || reinterpret_cast<uintptr_t>(H) % 16 ||
      (W_hat && reinterpret_cast<uintptr_t>(W_hat) % 16) ||
      reinterpret_cast<uintptr_t>(qweight) % 4 || reinterpret_cast<uintptr_t>(scales) % 4 ||
      reinterpret_cast<uintptr_t>(zeros) % 4 || (g_idx && reinterpret_cast<uintptr_t>(g_idx) % 16) ||
      (codes && reinterpret_cast<uintptr_t>(codes) % 4))
    return GPTQ_ERR_INVALID_ARG;
  return GPTQ_OK;
}

int quantize_layer(const float *W, int64_t r, int64_t d, float *H, int bits, int group, int block,
                   float damp, int options, float *W_hat, int32_t *qweight, float *scales,
                   int32_t *zeros, int32_t *g_idx, uint8_t *codes, double *loss, void *workspace,
                   size_t workspace_bytes, gptq_stream_t stream, bool plain) {
  GPTQ_TRY(check_layer_args(W, r, d, H, bits, group, block, damp, options, W_hat, qweight, scales,
                            zeros, g_idx, codes));
  const bool act_order = (options & GPTQ_ACT_ORDER) != 0;
  const int sym = (options & GPTQ_SYMMETRIC) ? 1 : 0;
  // with one group per row both rules take the parameters from the original row
  const int static_groups = (options & GPTQ_STATIC_GROUPS) && group > 0 ? 1 : 0;
  if (r == 0) {
    if (loss) *loss = 0.0;
    return GPTQ_OK;
  }
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256) return GPTQ_ERR_INVALID_ARG;
  const Layout L = layout(r, d, group, block, options);
  if (workspace_bytes < L.total) return GPTQ_ERR_NO_MEMORY;

  cudaStream_t st = (cudaStream_t)stream;
  char *ws = static_cast<char *>(workspace);
  float *Wk = reinterpret_cast<float *>(ws + L.Wk);
  float *ErrS = reinterpret_cast<float *>(ws + L.ErrS);
  uint8_t *codes_p = reinterpret_cast<uint8_t *>(ws + L.codes_p);
  int *perm = reinterpret_cast<int *>(ws + L.perm);
  int *inv = reinterpret_cast<int *>(ws + L.inv);
  float *Hp = reinterpret_cast<float *>(ws + L.Hp);
  float *T1 = reinterpret_cast<float *>(ws + L.T1);
  double *loss_rows = reinterpret_cast<double *>(ws + L.loss_rows);
  double *dsq_rows = reinterpret_cast<double *>(ws + L.dsq_rows);
  double *out = reinterpret_cast<double *>(ws + L.out);
  float *lambda = reinterpret_cast<float *>(ws + L.lambda);
  int *status = reinterpret_cast<int *>(ws + L.status);
  const int ri = (int)r, di = (int)d;

  // The four phases of the solve: damping (and the act-order permutation),
  // the factor U, the sweep, and finalize (unpermute, loss, packing).
  float *U = nullptr;
  auto seg_damp = [&]() -> int {
    GPTQ_CUDA_TRY(cudaMemsetAsync(status, 0, 16, st));
    GPTQ_CUDA_TRY(cudaMemsetAsync(loss_rows, 0, (size_t)r * 8, st));
    int rc = GPTQ_OK;
    U = enqueue_damp(H, d, damp, act_order, perm, inv, lambda, Hp, st, &rc);
    return rc;
  };
  auto seg_factor = [&]() -> int { return launch_factor(U, d, T1, status, st, !plain); };
  auto sweep_plan = [&]() {
    return SweepPlan{W, ri, di, bits, group, block, sym, static_groups, U,
                     act_order ? perm : nullptr, act_order ? inv : nullptr, lambda, W_hat,
                     qweight, scales, zeros, g_idx, codes, Wk, ErrS, codes_p, loss_rows,
                     dsq_rows, out, status};
  };
  auto seg_sweep = [&]() -> int { return enqueue_sweep(sweep_plan(), st); };
  auto seg_final = [&]() -> int { return enqueue_finalize(sweep_plan(), st); };

  // Each phase replays as a CUDA graph when the same call (pointers, sizes,
  // settings, stream) repeats: the phases hold a few hundred short kernels
  // whose launch cost would otherwise pace the GPU.  The first call of a
  // configuration runs directly, the second is captured, later ones replay.
  // Streams that cannot be captured run directly.  The phase events (when
  // timing) are recorded between the phases, outside any capture.
  const bool timing = g_timing && !plain;
  if (timing) GPTQ_TRY(ensure_phase_events());
  t_timing = timing;
  GraphKey key{W, H, W_hat, qweight, scales, zeros, g_idx, codes, workspace,
               workspace_bytes, st, r, d, bits, group, block, damp, options, 0};
  int rc = GPTQ_OK;
  if (plain) {
    rc = seg_damp();
    if (rc == GPTQ_OK) rc = seg_factor();
    if (rc == GPTQ_OK) rc = seg_sweep();
    if (rc == GPTQ_OK) rc = seg_final();
  } else {
    // the matrix to factor is known without running the damping phase
    U = act_order ? Hp : H;
    rc = record(0, st);
    if (rc == GPTQ_OK) rc = run_graph_cached(key, st, seg_damp);
    if (rc == GPTQ_OK) rc = record(1, st);
    key.segment = 1;
    if (rc == GPTQ_OK) rc = run_graph_cached(key, st, seg_factor);
    if (rc == GPTQ_OK) rc = record(2, st);
    key.segment = 2;
    if (rc == GPTQ_OK) rc = run_graph_cached(key, st, seg_sweep);
    if (rc == GPTQ_OK) rc = record(3, st);
    key.segment = 3;
    if (rc == GPTQ_OK) rc = run_graph_cached(key, st, seg_final);
    if (rc == GPTQ_OK) rc = record(4, st);
  }
  t_timing = false;
  if (rc != GPTQ_OK) return rc;

  double host_out[3] = {0, 0, 0};
  int host_status = 0;
  GPTQ_CUDA_TRY(cudaMemcpyAsync(host_out, out, sizeof(host_out), cudaMemcpyDeviceToHost, st));
  GPTQ_CUDA_TRY(cudaMemcpyAsync(&host_status, status, sizeof(int), cudaMemcpyDeviceToHost, st));
  GPTQ_CUDA_TRY(cudaStreamSynchronize(st));
  if (timing)
    for (int i = 0; i < 4; ++i)
      if (cudaEventElapsedTime(&g_phase_ms[i], g_ev[i], g_ev[i + 1]) != cudaSuccess)
        g_phase_ms[i] = -1.f;
  if (host_status != 0) return host_status;
  if (loss) *loss = host_out[0];
  return GPTQ_OK;
}

}  // namespace gptq

extern "C" int gptq_quantize_layer(const float *W, int64_t r, int64_t d, float *H, int bits,
                                   int group, int block, float damp, int options, float *W_hat,
                                   int32_t *qweight, float *scales, int32_t *zeros,
                                   int32_t *g_idx, uint8_t *codes, double *loss, void *workspace,
                                   size_t workspace_bytes, gptq_stream_t stream) {
  return gptq::quantize_layer(W, r, d, H, bits, group, block, damp, options, W_hat, qweight,
                              scales, zeros, g_idx, codes, loss, workspace, workspace_bytes,
                              stream, false);
}

// ------------------------------------------------------- factor once, sweep many

namespace {

struct FactorLayout {
  size_t inv, Hp, T1, status, total;
};

FactorLayout factor_layout(int64_t d, int options) {
  FactorLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  L.inv = take((size_t)d * 4);
  L.Hp = take((options & GPTQ_ACT_ORDER) ? (size_t)d * d * 4 : 0);
  L.T1 = take(factor_scratch_floats(d) * 4);
  L.status = take(16);
  L.total = off;
  return L;
}

struct SweepLayout {
  size_t Wk, ErrS, codes_p, inv, loss_rows, dsq_rows, out, status, total;
};

SweepLayout sweep_layout(int64_t r, int64_t d, int group, int block) {
  SweepLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  const int S = superblock(d, group, block);
  L.Wk = take((size_t)r * d * 4);
  L.ErrS = take((size_t)r * S * 4);
  L.codes_p = take((size_t)r * d);
  L.inv = take((size_t)d * 4);
  L.loss_rows = take((size_t)r * 8);
  L.dsq_rows = take((size_t)r * 8);
  L.out = take(4 * 8);
  L.status = take(16);
  L.total = off;
  return L;
}

bool valid_d(int64_t d) { return d > 0 && d % 32 == 0 && d <= 65536; }

}  // namespace

extern "C" size_t gptq_factor_workspace_bytes(int64_t d, int options) {
  if (!valid_d(d) || !valid_options(options)) return 0;
  return factor_layout(d, options).total;
}

extern "C" int gptq_factor(float *H, int64_t d, float damp, int options, int32_t *perm,
                           float *lambda, void *workspace, size_t workspace_bytes,
                           gptq_stream_t stream) {
  if (!valid_d(d) || !valid_options(options)) return GPTQ_ERR_INVALID_ARG;
  if (!(damp >= 0.f) || damp > 1e30f) return GPTQ_ERR_INVALID_ARG;
  const bool act_order = (options & GPTQ_ACT_ORDER) != 0;
  if (!H || !lambda || !workspace || (act_order && !perm)) return GPTQ_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(H) % 16 || reinterpret_cast<uintptr_t>(lambda) % 4 ||
      reinterpret_cast<uintptr_t>(workspace) % 256 ||
      (perm && reinterpret_cast<uintptr_t>(perm) % 4))
    return GPTQ_ERR_INVALID_ARG;
  const FactorLayout L = factor_layout(d, options);
  if (workspace_bytes < L.total) return GPTQ_ERR_NO_MEMORY;
  cudaStream_t st = (cudaStream_t)stream;
  char *ws = static_cast<char *>(workspace);
  int *inv = reinterpret_cast<int *>(ws + L.inv);
  float *Hp = reinterpret_cast<float *>(ws + L.Hp);
  float *T1 = reinterpret_cast<float *>(ws + L.T1);
  int *status = reinterpret_cast<int *>(ws + L.status);
  GPTQ_CUDA_TRY(cudaMemsetAsync(status, 0, 16, st));
  float *U = nullptr;
  GPTQ_TRY(enqueue_factor(H, d, damp, act_order, perm, inv, lambda, Hp, T1, status, st, true, &U));
  if (U != H)   // act-order: the factor of the permuted H_d goes back into H
    GPTQ_CUDA_TRY(cudaMemcpyAsync(H, U, (size_t)d * d * 4, cudaMemcpyDeviceToDevice, st));
  int host_status = 0;
  GPTQ_CUDA_TRY(cudaMemcpyAsync(&host_status, status, sizeof(int), cudaMemcpyDeviceToHost, st));
  GPTQ_CUDA_TRY(cudaStreamSynchronize(st));
  return host_status;
}

extern "C" size_t gptq_quantize_with_factor_workspace_bytes(int64_t r, int64_t d, int bits,
                                                            int group, int block) {
  if (!valid_layer(r, d, bits, group, block)) return 0;
  return sweep_layout(r, d, group, block).total;
}

extern "C" int gptq_quantize_with_factor(const float *W, int64_t r, int64_t d, const float *U,
                                         const int32_t *perm, const float *lambda, int bits,
                                         int group, int block, int options, float *W_hat,
                                         int32_t *qweight, float *scales, int32_t *zeros,
                                         int32_t *g_idx, uint8_t *codes, double *loss,
                                         void *workspace, size_t workspace_bytes,
                                         gptq_stream_t stream) {
  if (!valid_layer(r, d, bits, group, block) || !valid_options(options))
    return GPTQ_ERR_INVALID_ARG;
  const bool act_order = (options & GPTQ_ACT_ORDER) != 0;
  const int sym = (options & GPTQ_SYMMETRIC) ? 1 : 0;
  const int static_groups = (options & GPTQ_STATIC_GROUPS) && group > 0 ? 1 : 0;
  if (r == 0) {
    if (loss) *loss = 0.0;
    return GPTQ_OK;
  }
  if (!W || !U || !lambda || !qweight || !scales || !zeros || !workspace || (act_order && !perm))
    return GPTQ_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(W) % 16 || reinterpret_cast<uintptr_t>(U) % 16 ||
      reinterpret_cast<uintptr_t>(workspace) % 256 || reinterpret_cast<uintptr_t>(lambda) % 4 ||
      (W_hat && reinterpret_cast<uintptr_t>(W_hat) % 16) ||
      reinterpret_cast<uintptr_t>(qweight) % 4 || reinterpret_cast<uintptr_t>(scales) % 4 ||
      reinterpret_cast<uintptr_t>(zeros) % 4 ||
      (g_idx && reinterpret_cast<uintptr_t>(g_idx) % 16) ||
      (codes && reinterpret_cast<uintptr_t>(codes) % 4) ||
      (perm && reinterpret_cast<uintptr_t>(perm) % 4))
    return GPTQ_ERR_INVALID_ARG;
  const SweepLayout L = sweep_layout(r, d, group, block);
  if (workspace_bytes < L.total) return GPTQ_ERR_NO_MEMORY;
  cudaStream_t st = (cudaStream_t)stream;
  char *ws = static_cast<char *>(workspace);
  int *inv = reinterpret_cast<int *>(ws + L.inv);
  double *loss_rows = reinterpret_cast<double *>(ws + L.loss_rows);
  double *out = reinterpret_cast<double *>(ws + L.out);
  int *status = reinterpret_cast<int *>(ws + L.status);
  GPTQ_CUDA_TRY(cudaMemsetAsync(status, 0, 16, st));
  GPTQ_CUDA_TRY(cudaMemsetAsync(loss_rows, 0, (size_t)r * 8, st));
  // The caller's permutation indexes W: checked on the device before any
  // kernel uses it (a bad one sets the status word and the sweep is skipped).
  if (act_order) GPTQ_TRY(launch_check_perm(perm, (int)d, inv, status, st));
  const SweepPlan sp{W, (int)r, (int)d, bits, group, block, sym, static_groups, U,
                     act_order ? perm : nullptr, act_order ? inv : nullptr, lambda, W_hat,
                     qweight, scales, zeros, g_idx, codes,
                     reinterpret_cast<float *>(ws + L.Wk), reinterpret_cast<float *>(ws + L.ErrS),
                     reinterpret_cast<uint8_t *>(ws + L.codes_p), loss_rows,
                     reinterpret_cast<double *>(ws + L.dsq_rows), out, status};
  GPTQ_TRY(enqueue_sweep(sp, st));
  GPTQ_TRY(enqueue_finalize(sp, st));
  double host_out[3] = {0, 0, 0};
  int host_status = 0;
  GPTQ_CUDA_TRY(cudaMemcpyAsync(host_out, out, sizeof(host_out), cudaMemcpyDeviceToHost, st));
  GPTQ_CUDA_TRY(cudaMemcpyAsync(&host_status, status, sizeof(int), cudaMemcpyDeviceToHost, st));
  GPTQ_CUDA_TRY(cudaStreamSynchronize(st));
  if (host_status != 0) return host_status;
  if (loss) *loss = host_out[0];
  return GPTQ_OK;
}

namespace {

struct HostLayout {
  size_t X, H, W, qw, sc, zr, gi, qws, total;
};

// Per-device stream for the host-to-device copies of the end-to-end entry
// point, and events to hand each copied chunk to the computing stream.
struct CopyStream {
  cudaStream_t s = nullptr;
  std::vector<cudaEvent_t> ev;
};

int copy_stream(size_t events, CopyStream **out) {
  static CopyStream cs[64];
  static std::mutex mu;
  int dev = 0;
  GPTQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return GPTQ_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(mu);
  CopyStream &c = cs[dev];
  if (!c.s) GPTQ_CUDA_TRY(cudaStreamCreateWithFlags(&c.s, cudaStreamNonBlocking));
  while (c.ev.size() < events) {
    cudaEvent_t e;
    GPTQ_CUDA_TRY(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
    c.ev.push_back(e);
  }
  *out = &c;
  return GPTQ_OK;
}

// Tokens per copied chunk of X: at least 32768, at most 64 chunks.
int64_t x_chunk_tokens(int64_t n) {
  const int64_t c = (n + 63) / 64;
  return c > 32768 ? c : 32768;
}

HostLayout host_layout(int64_t r, int64_t d, int64_t n, int bits, int group, int block,
                       int options) {
  HostLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  const int64_t G = group < 0 ? 1 : d / group;
  L.X = take((size_t)n * d * 2);
  L.H = take((size_t)d * d * 4);
  L.W = take((size_t)r * d * 4);
  L.qw = take((size_t)r * (d * bits / 32) * 4);
  L.sc = take((size_t)r * G * 4);
  L.zr = take((size_t)r * G * 4);
  L.gi = take((size_t)d * 4);
  L.qws = take(layout(r, d, group, block, options).total);
  L.total = off;
  return L;
}

}  // namespace

extern "C" size_t gptq_layer_host_workspace_bytes(int64_t r, int64_t d, int64_t n, int bits,
                                                  int group, int block, int options) {
  if (!valid_layer(r, d, bits, group, block) || !valid_options(options) || n < 0 ||
      n > (int64_t)INT32_MAX)
    return 0;
  return host_layout(r, d, n, bits, group, block, options).total;
}

extern "C" int gptq_solve_layer_host(const uint16_t *X_host, int64_t n, const float *W_host,
                                     int64_t r, int64_t d, int bits, int group, int block,
                                     float damp, int options, int32_t *qweight_host,
                                     float *scales_host, int32_t *zeros_host,
                                     int32_t *g_idx_host, double *loss, void *dev_workspace,
                                     size_t dev_workspace_bytes, gptq_stream_t stream) {
  if (!valid_layer(r, d, bits, group, block) || !valid_options(options) || n < 0 ||
      n > (int64_t)INT32_MAX)
    return GPTQ_ERR_INVALID_ARG;
  if ((n > 0 && !X_host) || !W_host || !qweight_host || !scales_host || !zeros_host ||
      !dev_workspace || reinterpret_cast<uintptr_t>(dev_workspace) % 256)
    return GPTQ_ERR_INVALID_ARG;
  if (r == 0) {
    if (loss) *loss = 0.0;
    return GPTQ_OK;
  }
  const HostLayout L = host_layout(r, d, n, bits, group, block, options);
  if (dev_workspace_bytes < L.total) return GPTQ_ERR_NO_MEMORY;
  cudaStream_t st = (cudaStream_t)stream;
  char *ws = static_cast<char *>(dev_workspace);
  uint16_t *X = reinterpret_cast<uint16_t *>(ws + L.X);
  float *H = reinterpret_cast<float *>(ws + L.H);
  float *W = reinterpret_cast<float *>(ws + L.W);
  int32_t *qw = reinterpret_cast<int32_t *>(ws + L.qw);
  float *sc = reinterpret_cast<float *>(ws + L.sc);
  int32_t *zr = reinterpret_cast<int32_t *>(ws + L.zr);
  int32_t *gi = reinterpret_cast<int32_t *>(ws + L.gi);
  const int64_t G = group < 0 ? 1 : d / group;

  // X travels in token chunks on a copy stream; the Hessian of each chunk is
  // accumulated on `stream` as soon as the chunk has landed, so the tensor-core
  // work hides behind the host-to-device copy of the next chunk.
  const int64_t chunk = x_chunk_tokens(n);
  const int64_t nch = n > 0 ? (n + chunk - 1) / chunk : 0;
  CopyStream *cs = nullptr;
  GPTQ_TRY(copy_stream((size_t)nch + 2, &cs));
  GPTQ_CUDA_TRY(cudaEventRecord(cs->ev[0], st));   // the workspace is free on `stream`
  GPTQ_CUDA_TRY(cudaStreamWaitEvent(cs->s, cs->ev[0], 0));
  GPTQ_CUDA_TRY(cudaMemcpyAsync(W, W_host, (size_t)r * d * 4, cudaMemcpyHostToDevice, cs->s));
  GPTQ_CUDA_TRY(cudaMemsetAsync(H, 0, (size_t)d * d * 4, st));
  for (int64_t c = 0; c < nch; ++c) {
    const int64_t t0 = c * chunk, tn = (n - t0) < chunk ? (n - t0) : chunk;
    GPTQ_CUDA_TRY(cudaMemcpyAsync(X + t0 * d, X_host + t0 * d, (size_t)tn * d * 2,
                                  cudaMemcpyHostToDevice, cs->s));
    GPTQ_CUDA_TRY(cudaEventRecord(cs->ev[c + 1], cs->s));
    GPTQ_CUDA_TRY(cudaStreamWaitEvent(st, cs->ev[c + 1], 0));
    GPTQ_TRY(gptq_hessian_accumulate(X + t0 * d, tn, d, d, H, stream));
  }
  GPTQ_CUDA_TRY(cudaEventRecord(cs->ev[nch + 1], cs->s));   // W (copied first) and all of X
  GPTQ_CUDA_TRY(cudaStreamWaitEvent(st, cs->ev[nch + 1], 0));
  GPTQ_TRY(gptq_quantize_layer(W, r, d, H, bits, group, block, damp, options, nullptr, qw, sc,
                               zr, gi, nullptr, loss, ws + L.qws, L.total - L.qws, stream));
  GPTQ_CUDA_TRY(cudaMemcpyAsync(qweight_host, qw, (size_t)r * (d * bits / 32) * 4,
                                cudaMemcpyDeviceToHost, st));
  GPTQ_CUDA_TRY(cudaMemcpyAsync(scales_host, sc, (size_t)r * G * 4, cudaMemcpyDeviceToHost, st));
  GPTQ_CUDA_TRY(cudaMemcpyAsync(zeros_host, zr, (size_t)r * G * 4, cudaMemcpyDeviceToHost, st));
  if (g_idx_host)
    GPTQ_CUDA_TRY(cudaMemcpyAsync(g_idx_host, gi, (size_t)d * 4, cudaMemcpyDeviceToHost, st));
  GPTQ_CUDA_TRY(cudaStreamSynchronize(st));
  return GPTQ_OK;
}
