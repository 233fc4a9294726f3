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

// One code back to bf16: xhat = RN_bf16(code * a' / 127), rounded once from
// the exact value.  The fp64 product is exact; the fp64 quotient's rounding
// cannot cross a bf16 rounding boundary (a non-dyadic quotient stays ~2^-32
// relative away from every 9-bit dyadic; a dyadic one is exact in fp64).
// a' >= 1e-5 keeps every non-zero result a normal bf16.
__device__ __forceinline__ uint32_t dequant_bf16(int code, float ap) {
  if (code == 0) return 0u;
  const double d = static_cast<double>(code) * static_cast<double>(ap) / 127.0;
  const uint64_t bits = static_cast<uint64_t>(__double_as_longlong(d));
  const uint32_t sign = static_cast<uint32_t>(bits >> 48) & 0x8000u;
  const uint64_t mag = bits & 0x7FFFFFFFFFFFFFFFull;
  uint64_t top = mag >> 45;                   // 11 exponent bits, 7 mantissa bits
  const uint64_t rest = mag & ((1ull << 45) - 1), half = 1ull << 44;
  top += (rest > half || (rest == half && (top & 1u))) ? 1u : 0u;  // nearest, ties to even
  const int exp = static_cast<int>(top >> 7) - 1023 + 127;
  if (exp >= 255) return sign | 0x7F80u;      // rounds past the bf16 maximum
  return sign | (static_cast<uint32_t>(exp) << 7) | static_cast<uint32_t>(top & 0x7Fu);
}

// 8 bf16 values -> their 8 dequantised values (bf16, one 16-byte vector).
__device__ __forceinline__ uint4 dequantise8(const uint4 v, float ap) {
  const uint2 q = quantise8(v, ap);
  const uint32_t codes[2] = {q.x, q.y};
  uint32_t out[4];
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    const int c0 = static_cast<int8_t>((codes[h >> 1] >> (16 * (h & 1))) & 0xFFu);
    const int c1 = static_cast<int8_t>((codes[h >> 1] >> (16 * (h & 1) + 8)) & 0xFFu);
    out[h] = dequant_bf16(c0, ap) | (dequant_bf16(c1, ap) << 16);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
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
