// gptq_quantize_layer_noalloc: the layer solve for callers that cannot allocate
// device memory.
//
// Some callers cannot call cudaMalloc at all, or cannot do so at the moment they
// need to quantise a layer: code running inside a memory pool whose owner
// forbids side allocations, a runtime that has already reserved every byte of
// the device up front, or a host that hands this library only its inputs and
// outputs and no scratch buffer.  For them this entry point takes its scratch
// from one fixed-size array in the library's own device memory instead of a
// caller-provided workspace.  The array is a file-scope static __device__
// object, so it exists on every GPU that loads this library, for as long as
// the process lives, whether or not this entry point is ever called.
//
// Host code cannot use the array's name as a device address (on the host it
// names a stand-in object), so the device address is looked up once per
// device with cudaGetSymbolAddress and reused.
#include <mutex>

#include "gptq_internal.h"

namespace gptq {
namespace {

constexpr size_t kScratchBytes = GPTQ_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up on the
// first call made with that device current.
int scratch_address(void **out) {
  int dev = 0;
  GPTQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) {
    set_last_error_msg(__FILE__, __LINE__, "device ordinal beyond the scratch table");
    return GPTQ_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    GPTQ_CUDA_TRY(cudaGetSymbolAddress(&p, g_noalloc_scratch));
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return GPTQ_OK;
}

}  // namespace
}  // namespace gptq

extern "C" int gptq_quantize_layer_noalloc(const float *W, int64_t r, int64_t d, float *H,
                                           int bits, int group, int block, float damp,
                                           int options, float *W_hat, int32_t *qweight,
                                           float *scales, int32_t *zeros, int32_t *g_idx,
                                           uint8_t *codes, double *loss, gptq_stream_t stream) {
  // Every argument is checked before the size, so a bad argument reports
  // GPTQ_ERR_INVALID_ARG whatever the layer's size.
  const int bad = gptq::check_layer_args(W, r, d, H, bits, group, block, damp, options, W_hat,
                                         qweight, scales, zeros, g_idx, codes);
  if (bad != GPTQ_OK) return bad;
  const size_t need = gptq_quantize_workspace_bytes(r, d, bits, group, block, options);
  if (need == 0) return GPTQ_ERR_INVALID_ARG;
  if (need > gptq::kScratchBytes) {
    gptq::set_last_error_msg(__FILE__, __LINE__,
                             "layer needs more scratch than GPTQ_NOALLOC_SCRATCH_BYTES");
    return GPTQ_ERR_NO_MEMORY;
  }
  if (r == 0) {
    if (loss) *loss = 0.0;
    return GPTQ_OK;
  }
  void *scratch = nullptr;
  const int rc = gptq::scratch_address(&scratch);
  if (rc != GPTQ_OK) return rc;
  // The solve clears every part of its workspace that must start at zero, so
  // whatever an earlier call left in the array does not leak into this one.
  // The plain form launches the kernels directly: no CUDA graph, stream or
  // event is created on this path (phase timing does not apply to it).
  return gptq::quantize_layer(W, r, d, H, bits, group, block, damp, options, W_hat, qweight,
                              scales, zeros, g_idx, codes, loss, scratch, gptq::kScratchBytes,
                              stream, true);
}
