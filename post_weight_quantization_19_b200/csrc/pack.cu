// gptq_pack: codes [r x d] uint8 -> int32 words [r x d*bits/32].
//
// Source: "一文读懂GPTQ" §三 -- quantised 3/4-bit weights are stored packed in
// 32-bit integer arrays.  One thread packs 32 consecutive codes of a row into
// BITS words (see pack_bits.cuh for the bit layout): two 16-byte loads in, BITS
// consecutive 4-byte stores out, so a warp reads 1 KB and writes BITS*128 bytes
// contiguously.  Purely bandwidth bound: r*d*(1 + bits/8) bytes per call.
#include "gptq_internal.h"
#include "pack_bits.cuh"

namespace gptq {
namespace {

template <int BITS>
__global__ void __launch_bounds__(256) pack_kernel(const uint8_t *__restrict__ codes,
                                                   int64_t ngroups_total,
                                                   uint32_t *__restrict__ out) {
  const int64_t gq = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (gq >= ngroups_total) return;
  const uint4 *src = reinterpret_cast<const uint4 *>(codes + gq * 32);
  const uint4 lo = src[0], hi = src[1];
  const uint32_t raw[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
  uint32_t c[32];
#pragma unroll
  for (int k = 0; k < 32; ++k) c[k] = (raw[k >> 2] >> ((k & 3) * 8)) & 0xFFu;
  uint32_t words[BITS];
  pack32<BITS>(c, words);
  uint32_t *dst = out + gq * BITS;
#pragma unroll
  for (int w = 0; w < BITS; ++w) dst[w] = words[w];
}

}  // namespace

int launch_pack(const uint8_t *codes, int64_t r, int64_t d, int bits, int32_t *qweight,
                cudaStream_t stream) {
  // Rows are contiguous and d % 32 == 0, so the 32-code groups of all rows
  // form one flat sequence whose packed words are also contiguous.
  const int64_t ng = r * (d / 32);
  if (ng == 0) return GPTQ_OK;
  const int64_t blocks = (ng + 255) / 256;
  if (blocks > INT32_MAX) return GPTQ_ERR_INVALID_ARG;
  uint32_t *out = reinterpret_cast<uint32_t *>(qweight);
  switch (bits) {
    case 2: pack_kernel<2><<<(unsigned)blocks, 256, 0, stream>>>(codes, ng, out); break;
    case 3: pack_kernel<3><<<(unsigned)blocks, 256, 0, stream>>>(codes, ng, out); break;
    case 4: pack_kernel<4><<<(unsigned)blocks, 256, 0, stream>>>(codes, ng, out); break;
    case 8: pack_kernel<8><<<(unsigned)blocks, 256, 0, stream>>>(codes, ng, out); break;
    default: return GPTQ_ERR_INVALID_ARG;
  }
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

}  // namespace gptq

extern "C" int gptq_pack(const uint8_t *codes, int64_t r, int64_t d, int bits, int32_t *qweight,
                         gptq_stream_t stream) {
  if (!codes || !qweight) return GPTQ_ERR_INVALID_ARG;
  if (r < 0 || d <= 0 || d % 32 != 0) return GPTQ_ERR_INVALID_ARG;
  if (bits != 2 && bits != 3 && bits != 4 && bits != 8) return GPTQ_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(codes) % 16 != 0 || reinterpret_cast<uintptr_t>(qweight) % 4 != 0)
    return GPTQ_ERR_INVALID_ARG;
  return gptq::launch_pack(codes, r, d, bits, qweight, (cudaStream_t)stream);
}
