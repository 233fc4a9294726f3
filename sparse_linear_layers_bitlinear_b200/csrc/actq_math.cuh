// Element arithmetic of the per-token int8 absmax activation quantiser, shared
// by the act-quant kernel and the decode GEMV (which quantises its few token
// rows itself): a' = max(max_k |x|, 1e-5), xq = sign(x) * rne(fl32(127 |x|) / a')
// clamped to [-128, 127].
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace sbl {

__device__ __forceinline__ float bf16_abs_value(uint32_t bits16) { return __uint_as_float((bits16 & 0x7FFFu) << 16); }

// Per-row constants of the quantiser.
//
// The code is rne(Q), Q = 127 |x| / a' (127 |x| is exact in fp32, and the
// oracle's IEEE quotient rounds to the same integer).  When a' is a row
// maximum it is a bf16 value too, and rne(Q) comes from one fused
// multiply-add: the low byte of RN(x * c + 1.5 * 2^23), c = RU(127 / a')
// rounded UP, whose ulp is 1 (quantise8_fma).  Why that is exact, writing
// |x| = X 2^p and a' = A 2^q with X, A odd (at most 8 significant bits):
//   - A quotient that is not a half-integer h lies at least 2^-16 (relative)
//     from every h: Q - h is a non-zero multiple of 1 / (2A) when p >= q,
//     of 2^(p-q) / (2A) otherwise, against Q <= 127.  The product x * c is
//     Q (1 + d) with 0 <= d < 2^-23, so it rounds to the same integer.
//   - A tie 127 X 2^(p-q+1) = (2n + 1) A needs 127 X = (2n + 1) A.  The prime
//     127 then divides A (A = 127: a' is 254/128 times a power of two, so
//     127 / a' is a power of two, c is exact, and the addition rounds the
//     exact tie to even) or 2n + 1 = 127 (Q = 63.5 at |x| = a' / 2: d > 0
//     unless a' is a power of two, so |x c| is just above 63.5 and rounds to
//     the even 64; for a power of two c is exact and the tie rounds to even).
// The clamped a' = 1e-5 is not a bf16 value, and from a' = 2^120 up the
// reciprocal leaves the normal range; those rows take the IEEE division.
struct QScale {
  float ap;    // a'
  float c;     // RU(127 / a'): the multiplier of quantise8_fma
  bool exact;  // a' is the 1e-5 clamp or at least 2^120 (or not finite)
};

__device__ __forceinline__ QScale make_qscale(float ap) {
  return QScale{ap, __fdiv_ru(127.0f, ap), ap == 1e-5f || !(ap < 0x1p120f)};
}

// 8 bf16 values -> 8 int8 codes (two words), for a row with QScale::exact
// false.  A code's byte is the low byte of n + 1.5 * 2^23 (two's complement
// for |n| <= 127).
__device__ __forceinline__ uint2 quantise8_fma(const uint4 v, float c) {
  const uint32_t words[4] = {v.x, v.y, v.z, v.w};
  uint32_t bytes[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const uint32_t w = words[e >> 1];
    const float x = __uint_as_float((e & 1) ? (w & 0xFFFF0000u) : (w << 16));
    bytes[e] = __float_as_uint(__fmaf_rn(x, c, 12582912.0f));
  }
  return make_uint2(__byte_perm(__byte_perm(bytes[0], bytes[1], 0x0040), __byte_perm(bytes[2], bytes[3], 0x0040), 0x5410),
                    __byte_perm(__byte_perm(bytes[4], bytes[5], 0x0040), __byte_perm(bytes[6], bytes[7], 0x0040), 0x5410));
}

// 8 bf16 values -> 8 int8 codes by the IEEE division, for any a':
// sign(x) * min(rne(fl32(127 |x|) / a'), 127).
__device__ __forceinline__ uint2 quantise8_div(const uint4 v, float ap) {
  const uint32_t words[4] = {v.x, v.y, v.z, v.w};
  uint32_t packed[2] = {0u, 0u};
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const uint32_t b = (words[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
    const int n = min(__float2int_rn(__fdiv_rn(__fmul_rn(127.0f, bf16_abs_value(b)), ap)), 127);
    const int code = (b & 0x8000u) ? -n : n;
    packed[e >> 2] |= (static_cast<uint32_t>(code) & 0xFFu) << (8 * (e & 3));
  }
  return make_uint2(packed[0], packed[1]);
}

// 8 codes by whichever form the row allows (uniform over a row).
__device__ __forceinline__ uint2 quantise8(const uint4 v, const QScale& s) {
  return s.exact ? quantise8_div(v, s.ap) : quantise8_fma(v, s.c);
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

// The same value with fp32 arithmetic, for a row whose a' is a bf16 value
// below 2^120 (QScale::exact false), given c = RN(a' / 127): RN(code * c) is
// within ~2^-23 (relative) of Q = code * a' / 127.  A Q that is not dyadic
// lies at least 2^-16 (relative) from every bf16 rounding boundary (N 2^e /
// 127 against a 9-bit dyadic, N = |code| * A < 2^15), so RN_bf16 of the
// estimate is RN_bf16(Q); a dyadic Q (code = +-127, or A = 254) has at most 8
// significant bits, is a bf16 value, and the estimate rounds back onto it.
__device__ __forceinline__ uint32_t dequant_bf16_fast(int code, float a_over_127) {
  const float v = __fmul_rn(static_cast<float>(code), a_over_127);
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v)));
}

// 8 codes (two words) -> their dequantised values (bf16, one 16-byte vector).
__device__ __forceinline__ uint4 dequant8_fast(const uint2 q, float a_over_127) {
  const uint32_t codes[2] = {q.x, q.y};
  uint32_t out[4];
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    const int c0 = static_cast<int8_t>((codes[h >> 1] >> (16 * (h & 1))) & 0xFFu);
    const int c1 = static_cast<int8_t>((codes[h >> 1] >> (16 * (h & 1) + 8)) & 0xFFu);
    out[h] = dequant_bf16_fast(c0, a_over_127) | (dequant_bf16_fast(c1, a_over_127) << 16);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

// 8 bf16 values -> their 8 dequantised values (bf16, one 16-byte vector).
__device__ __forceinline__ uint4 dequantise8(const uint4 v, const QScale& s) {
  const uint2 q = quantise8(v, s);
  const uint32_t codes[2] = {q.x, q.y};
  uint32_t out[4];
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    const int c0 = static_cast<int8_t>((codes[h >> 1] >> (16 * (h & 1))) & 0xFFu);
    const int c1 = static_cast<int8_t>((codes[h >> 1] >> (16 * (h & 1) + 8)) & 0xFFu);
    out[h] = dequant_bf16(c0, s.ap) | (dequant_bf16(c1, s.ap) << 16);
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
