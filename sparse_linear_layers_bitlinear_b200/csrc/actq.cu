// Per-token int8 absmax activation quantisation (step 4 of the forward pass).
// The Sparse-BitNet pages do not spell out the activation quantiser; this is
// the BitNet b1.58 convention: a' = max(max_k |x|, 1e-5), and
// xq = sign(x) * rne(fl32(127 |x|) / a') clamped to [-128, 127].
//
// Rows of up to 3072 elements: one warp per token row, the row in registers
// (RW 16-byte vectors a lane), read from memory once.  The absmax is an
// integer max over the bf16 magnitude bits (their order is the order of the
// values, and a non-finite value shows as bits >= 0x7F80), two halves at a
// time, then one warp reduction; no block barrier.  All rows of a
// 4096-token batch are resident at once.  Its codes come without a division:
// one fused multiply-add per element by RU(127 / a'), exact for every row
// whose a' is a bf16 value (quantise8_fma), the IEEE division only for a row
// under the 1e-5 clamp or with a' at or above 2^120.  Longer rows: one block of 128
// threads per row with R vectors a thread (up to 16384 elements), then a
// two-pass, warp-per-row kernel.
//
// Launched with programmatic stream serialisation: its launch overlaps the
// kernel before it, and it waits for that kernel (which may have written x,
// or reset the status word) before it reads anything.  With early_trigger it
// then lets the next kernel (the GEMM or the decode kernel) launch at once.
//
// DEQ = true is the same pass writing the dequantised activations
// xhat = RN_bf16(xq * a' / 127) instead of the codes: the dW operand of the
// detach-form STE (SBL_DW_QUANT_X).
#include "sbl_kernels.h"

#include "sbl_device.cuh"
#include "actq_math.cuh"

namespace sbl {

constexpr int kActThreads = 128;
constexpr int kMaxR = 16;  // rows up to 16384 elements stay in registers

// Stores the quantised (or, with DEQ, dequantised) form of 8 elements.
template <bool DEQ>
__device__ __forceinline__ void store_quantised(void* out, int64_t row, int64_t nvec, int64_t i, const uint4 v,
                                                const QScale& qs) {
  if constexpr (DEQ)
    reinterpret_cast<uint4*>(out)[row * nvec + i] = dequantise8(v, qs);
  else
    reinterpret_cast<uint2*>(out)[row * nvec + i] = quantise8(v, qs);
}

// The codes of one row held in registers (v[r] is vector base + r * stride),
// for a row whose a' is a bf16 value below 2^120: one fused multiply-add per
// element (quantise8_fma).
template <bool DEQ, int R>
__device__ __forceinline__ void emit_codes(const uint4 (&v)[R], void* out, int64_t row, int64_t nvec, int base,
                                           int stride, const QScale& qs) {
  const float a_over_127 = DEQ ? __fdiv_rn(qs.ap, 127.0f) : 0.0f;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int64_t i = int64_t(r) * stride + base;
    const uint2 c = quantise8_fma(v[r], qs.c);
    if (i < nvec) {
      if constexpr (DEQ)
        reinterpret_cast<uint4*>(out)[row * nvec + i] = dequant8_fast(c, a_over_127);
      else
        reinterpret_cast<uint2*>(out)[row * nvec + i] = c;
    }
  }
}

template <int R, bool DEQ>
__global__ void __launch_bounds__(kActThreads, 4)
    k_act_quant_rows(const uint4* __restrict__ x, int64_t t, int64_t nvec, void* __restrict__ out,
                     float* __restrict__ a_prime, uint32_t* status, int early_trigger, int pf_stride) {
  // x may be the output of the kernel before this one: bring it towards L2
  // while that kernel runs, then wait for it.  The first pf_stride blocks
  // prefetch every row between them.
  if (threadIdx.x == 0 && static_cast<int>(blockIdx.x) < pf_stride)
    for (int64_t row = blockIdx.x; row < t; row += pf_stride)
      bulk_prefetch_l2(x + row * nvec, static_cast<uint32_t>(nvec * 16));
  pdl_wait();
  if (early_trigger) pdl_trigger();
  __shared__ uint32_t s_max[kActThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int64_t row = blockIdx.x; row < t; row += gridDim.x) {
    const uint4* src = x + row * nvec;
    uint4 v[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int64_t i = int64_t(r) * kActThreads + tid;
      v[r] = (i < nvec) ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
    }
    // the absmax as an integer max over the magnitude bits, two halves at a
    // time (as in the warp-per-row kernel)
    uint32_t m2 = 0;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      m2 = __vmaxu2(m2, v[r].x & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v[r].y & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v[r].z & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v[r].w & 0x7FFF7FFFu);
    }
    const uint32_t mw = __reduce_max_sync(0xFFFFFFFFu, max(m2 & 0xFFFFu, m2 >> 16));
    if (lane == 0) s_max[warp] = mw;
    __syncthreads();
    uint32_t m = s_max[0];
#pragma unroll
    for (int w = 1; w < kActThreads / 32; ++w) m = max(m, s_max[w]);
    __syncthreads();  // s_max is rewritten by the next row
    const float ap = fmaxf(__uint_as_float(m << 16), 1e-5f);
    if (tid == 0) {
      if (!DEQ) a_prime[row] = ap;
      if (m >= 0x7F80u) raise_status(status, SBL_STATUS_NONFINITE_X);
    }
    const QScale qs = make_qscale(ap);
    if (qs.exact) {  // the clamp or a' >= 2^120: the IEEE division
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int64_t i = int64_t(r) * kActThreads + tid;
        if (i < nvec) store_quantised<DEQ>(out, row, nvec, i, v[r], qs);
      }
    } else {  // the division-free codes
      emit_codes<DEQ>(v, out, row, nvec, tid, kActThreads, qs);
    }
  }
}

// Long rows: one warp per row, absmax pass then a second (L1/L2) pass.
constexpr int kActWarps = 8;

template <bool DEQ>
__global__ void __launch_bounds__(kActWarps * 32)
    k_act_quant_long(const uint4* __restrict__ x, int64_t t, int64_t nvec, void* __restrict__ out,
                     float* __restrict__ a_prime, uint32_t* status, int early_trigger) {
  pdl_wait();  // x may be the output of the kernel before this one
  if (early_trigger) pdl_trigger();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int64_t row = int64_t(blockIdx.x) * kActWarps + warp; row < t; row += int64_t(gridDim.x) * kActWarps) {
    const uint4* src = x + row * nvec;
    float amax = 0.0f;
    uint32_t bad = 0;
    int64_t i = lane;
    for (; i + 96 < nvec; i += 128) {
      const uint4 v0 = __ldg(src + i), v1 = __ldg(src + i + 32), v2 = __ldg(src + i + 64), v3 = __ldg(src + i + 96);
      scan8(v0, amax, bad);
      scan8(v1, amax, bad);
      scan8(v2, amax, bad);
      scan8(v3, amax, bad);
    }
    for (; i < nvec; i += 32) scan8(__ldg(src + i), amax, bad);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (__any_sync(0xffffffffu, bad != 0) && lane == 0) raise_status(status, SBL_STATUS_NONFINITE_X);
    const float ap = fmaxf(amax, 1e-5f);
    if (!DEQ && lane == 0) a_prime[row] = ap;
    const QScale qs = make_qscale(ap);
    for (int64_t j = lane; j < nvec; j += 32) store_quantised<DEQ>(out, row, nvec, j, __ldg(src + j), qs);
  }
}

constexpr int kWarpRowMax = 12;  // 16-byte vectors a lane: rows up to 3072 elements

template <int RW, bool DEQ>
__global__ void __launch_bounds__(kActThreads, DEQ ? 1 : 8)
    k_act_quant_warp(const uint4* __restrict__ x, int64_t t, int64_t nvec, void* __restrict__ out,
                     float* __restrict__ a_prime, uint32_t* status, int early_trigger, int pf_stride) {
  // x may be the output of the kernel before this one: bring it towards L2
  // while that kernel runs, then wait for it.
  if (threadIdx.x == 0 && static_cast<int>(blockIdx.x) < pf_stride)
    for (int64_t row = blockIdx.x; row < t; row += pf_stride)
      bulk_prefetch_l2(x + row * nvec, static_cast<uint32_t>(nvec * 16));
  pdl_wait();
  if (early_trigger) pdl_trigger();
  const int lane = threadIdx.x & 31;
  constexpr int kWarps = kActThreads / 32;
  for (int64_t row = int64_t(blockIdx.x) * kWarps + (threadIdx.x >> 5); row < t;
       row += int64_t(gridDim.x) * kWarps) {
    const uint4* src = x + row * nvec;
    uint4 v[RW];
#pragma unroll
    for (int r = 0; r < RW; ++r) {
      const int64_t i = int64_t(r) * 32 + lane;
      v[r] = (i < nvec) ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
    }
    uint32_t m2 = 0;
#pragma unroll
    for (int r = 0; r < RW; ++r) {
      m2 = __vmaxu2(m2, v[r].x & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v[r].y & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v[r].z & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v[r].w & 0x7FFF7FFFu);
    }
    const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, max(m2 & 0xFFFFu, m2 >> 16));
    const float ap = fmaxf(__uint_as_float(m << 16), 1e-5f);
    if (lane == 0) {
      if (!DEQ) a_prime[row] = ap;
      if (m >= 0x7F80u) raise_status(status, SBL_STATUS_NONFINITE_X);
    }
    const QScale qs = make_qscale(ap);
    if (qs.exact) {  // the clamp or a' >= 2^120: the IEEE division
#pragma unroll
      for (int r = 0; r < RW; ++r) {
        const int64_t i = int64_t(r) * 32 + lane;
        if (i < nvec) store_quantised<DEQ>(out, row, nvec, i, v[r], qs);
      }
    } else {  // the division-free codes
      emit_codes<DEQ>(v, out, row, nvec, lane, 32, qs);
    }
  }
}

template <int RW, bool DEQ>
static cudaError_t launch_warp_rows(const uint4* x, int64_t t, int64_t nvec, void* out, float* ap, uint32_t* status,
                                    int num_sms, cudaStream_t s, int early) {
  constexpr int kWarps = kActThreads / 32;
  int64_t blocks = (t + kWarps - 1) / kWarps;
  const int64_t cap = int64_t(num_sms) * 16;
  if (blocks > cap) blocks = cap;
  return launch_pdl(k_act_quant_warp<RW, DEQ>, dim3(static_cast<unsigned>(blocks)), dim3(kActThreads), 0, s, x, t,
                    nvec, out, ap, status, early, num_sms);
}

template <int R, bool DEQ>
static cudaError_t launch_rows(const uint4* x, int64_t t, int64_t nvec, void* out, float* ap, uint32_t* status,
                               int num_sms, cudaStream_t s, int early) {
  int64_t blocks = t;
  const int64_t cap = int64_t(num_sms) * 64;
  if (blocks > cap) blocks = cap;
  return launch_pdl(k_act_quant_rows<R, DEQ>, dim3(static_cast<unsigned>(blocks)), dim3(kActThreads), 0, s, x, t,
                    nvec, out, ap, status, early, num_sms);
}

template <bool DEQ>
static cudaError_t launch_quant(const uint16_t* x, int64_t t, int64_t k, void* out, float* a_prime, uint32_t* status,
                                int num_sms, cudaStream_t s, int early) {
  if (t <= 0) return cudaSuccess;
  const uint4* xv = reinterpret_cast<const uint4*>(x);
  const int64_t nvec = k / 8;
  const int64_t rw = (nvec + 31) / 32;
  if (rw <= 2) return launch_warp_rows<2, DEQ>(xv, t, nvec, out, a_prime, status, num_sms, s, early);
  if (rw <= 4) return launch_warp_rows<4, DEQ>(xv, t, nvec, out, a_prime, status, num_sms, s, early);
  if (rw <= 6) return launch_warp_rows<6, DEQ>(xv, t, nvec, out, a_prime, status, num_sms, s, early);
  if (rw <= 8) return launch_warp_rows<8, DEQ>(xv, t, nvec, out, a_prime, status, num_sms, s, early);
  if (rw <= 10) return launch_warp_rows<10, DEQ>(xv, t, nvec, out, a_prime, status, num_sms, s, early);
  if (rw <= kWarpRowMax) return launch_warp_rows<kWarpRowMax, DEQ>(xv, t, nvec, out, a_prime, status, num_sms, s, early);
  const int64_t r = (nvec + kActThreads - 1) / kActThreads;  // >= 4 here
  if (r <= 4) return launch_rows<4, DEQ>(xv, t, nvec, out, a_prime, status, num_sms, s, early);
  if (r <= 6) return launch_rows<6, DEQ>(xv, t, nvec, out, a_prime, status, num_sms, s, early);
  if (r <= 8) return launch_rows<8, DEQ>(xv, t, nvec, out, a_prime, status, num_sms, s, early);
  if (r <= 12) return launch_rows<12, DEQ>(xv, t, nvec, out, a_prime, status, num_sms, s, early);
  if (r <= kMaxR) return launch_rows<kMaxR, DEQ>(xv, t, nvec, out, a_prime, status, num_sms, s, early);
  int64_t blocks = (t + kActWarps - 1) / kActWarps;
  const int64_t cap = int64_t(num_sms) * 16;
  if (blocks > cap) blocks = cap;
  return launch_pdl(k_act_quant_long<DEQ>, dim3(static_cast<unsigned>(blocks)), dim3(kActWarps * 32), 0, s, xv, t,
                    nvec, out, a_prime, status, early);
}

cudaError_t launch_act_quant(const uint16_t* x, int64_t t, int64_t k, int8_t* xq, float* a_prime, uint32_t* status,
                             int num_sms, cudaStream_t s, bool early_trigger) {
  return launch_quant<false>(x, t, k, xq, a_prime, status, num_sms, s, early_trigger ? 1 : 0);
}

cudaError_t launch_act_dequant(const uint16_t* x, int64_t t, int64_t k, uint16_t* xhat, uint32_t* status, int num_sms,
                               cudaStream_t s) {
  return launch_quant<true>(x, t, k, xhat, nullptr, status, num_sms, s, 0);
}

}  // namespace sbl
