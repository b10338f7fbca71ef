// Bit packing of 32 codes into BITS int32 words (LSB-first stream).
//
// Source: "一文读懂GPTQ" §三 -- 3/4-bit codes are stored in 32-bit integer
// arrays.  Layout: per row, code c occupies stream bits [c*BITS, (c+1)*BITS),
// and stream bit k is bit (k mod 32) of word k/32, so 32 codes always fill
// exactly BITS words and 3-bit codes straddle word boundaries.
#pragma once

#include <stdint.h>

namespace gptq {

template <int BITS>
__device__ __forceinline__ void pack32(const uint32_t (&c)[32], uint32_t (&out)[BITS]) {
  constexpr uint32_t mask = (1u << BITS) - 1u;
#pragma unroll
  for (int w = 0; w < BITS; ++w) out[w] = 0u;
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const uint32_t v = c[k] & mask;
    const int pos = k * BITS;
    const int wi = pos >> 5, off = pos & 31;
    out[wi] |= v << off;
    if (off + BITS > 32) out[wi + 1] |= v >> (32 - off);
  }
}

}  // namespace gptq
