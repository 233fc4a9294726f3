// Element arithmetic of the per-token int8 absmax activation quantiser, shared
// by the act-quant kernel and the decode GEMV (which quantises its few token
// rows itself): a' = max(max_k |x|, 1e-5), xq = sign(x) * rne(fl32(127 |x|) / a')
// clamped to [-128, 127].
#pragma once

#include <stdint.h>

namespace sbl {

__device__ __forceinline__ float bf16_abs_value(uint32_t bits16) { return __uint_as_float((bits16 & 0x7FFFu) << 16); }

// 8 bf16 values -> 8 int8 codes (two words).
__device__ __forceinline__ uint2 quantise8(const uint4 v, float ap) {
  const uint32_t words[4] = {v.x, v.y, v.z, v.w};
  uint32_t packed[2] = {0u, 0u};
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const uint32_t b = (words[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
    const float q = __fdiv_rn(__fmul_rn(127.0f, bf16_abs_value(b)), ap);
    const int n = min(__float2int_rn(q), 127);  // nearest, ties to even
    const int code = (b & 0x8000u) ? -n : n;
    packed[e >> 2] |= (static_cast<uint32_t>(code) & 0xFFu) << (8 * (e & 3));
  }
  return make_uint2(packed[0], packed[1]);
}

__device__ __forceinline__ void scan8(const uint4 v, float& amax, uint32_t& bad) {
  const uint32_t words[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t b = (words[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
    bad |= ((b & 0x7F80u) == 0x7F80u);
    amax = fmaxf(amax, bf16_abs_value(b));
  }
}

}  // namespace sbl
