// Per-token int8 absmax activation quantisation (step 4 of the forward pass).
// The Sparse-BitNet pages do not spell out the activation quantiser; this is
// the BitNet b1.58 convention: a' = max(max_k |x|, 1e-5), and
// xq = sign(x) * rne(fl32(127 |x|) / a') clamped to [-128, 127].
#include "sbl_kernels.h"

#include "sbl_device.cuh"

namespace sbl {

constexpr int kActWarps = 8;  // one warp per token row

__device__ __forceinline__ float bf16_abs_value(uint32_t bits16) { return __uint_as_float((bits16 & 0x7FFFu) << 16); }

__global__ void __launch_bounds__(kActWarps * 32)
    k_act_quant(const uint16_t* __restrict__ x, int64_t t, int64_t k, int8_t* __restrict__ xq,
                float* __restrict__ a_prime, uint32_t* status) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t nvec = k / 8;  // 16-byte vectors per row
  for (int64_t row = int64_t(blockIdx.x) * kActWarps + warp; row < t; row += int64_t(gridDim.x) * kActWarps) {
    const uint4* src = reinterpret_cast<const uint4*>(x + row * k);
    float amax = 0.0f;
    uint32_t bad = 0;
    auto scan = [&](const uint4 v) {
      const uint32_t words[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t b = (words[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
        bad |= ((b & 0x7F80u) == 0x7F80u);
        amax = fmaxf(amax, bf16_abs_value(b));
      }
    };
    int64_t i = lane;
    for (; i + 96 < nvec; i += 128) {
      const uint4 v0 = __ldg(src + i), v1 = __ldg(src + i + 32), v2 = __ldg(src + i + 64), v3 = __ldg(src + i + 96);
      scan(v0);
      scan(v1);
      scan(v2);
      scan(v3);
    }
    for (; i < nvec; i += 32) scan(__ldg(src + i));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (__any_sync(0xffffffffu, bad != 0) && lane == 0) raise_status(status, SBL_STATUS_NONFINITE_X);
    const float ap = fmaxf(amax, 1e-5f);
    if (lane == 0) a_prime[row] = ap;

    uint2* dst = reinterpret_cast<uint2*>(xq + row * k);
    for (int64_t j = lane; j < nvec; j += 32) {
      const uint4 v = __ldg(src + j);  // second read hits L1/L2
      const uint32_t words[4] = {v.x, v.y, v.z, v.w};
      uint32_t packed[2] = {0u, 0u};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint32_t b = (words[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
        const float ax = bf16_abs_value(b);
        const float q = __fdiv_rn(__fmul_rn(127.0f, ax), ap);
        int n = __float2int_rn(q);  // nearest, ties to even
        n = min(n, 127);
        const int code = (b & 0x8000u) ? -n : n;
        packed[e >> 2] |= (static_cast<uint32_t>(code) & 0xFFu) << (8 * (e & 3));
      }
      dst[j] = make_uint2(packed[0], packed[1]);
    }
  }
}

cudaError_t launch_act_quant(const uint16_t* x, int64_t t, int64_t k, int8_t* xq, float* a_prime, uint32_t* status,
                             int num_sms, cudaStream_t s) {
  if (t <= 0) return cudaSuccess;
  int64_t blocks = (t + kActWarps - 1) / kActWarps;
  const int64_t cap = int64_t(num_sms) * 16;
  if (blocks > cap) blocks = cap;
  k_act_quant<<<static_cast<unsigned>(blocks), kActWarps * 32, 0, s>>>(x, t, k, xq, a_prime, status);
  return cudaGetLastError();
}

}  // namespace sbl
