// Epilogues and parameter blocks of the CTA-pair tensor-core GEMMs
// (gemm_pair.cuh): the accumulator, read from tensor memory by tcgen05.ld,
// is rescaled and stored to global memory.  An epilogue warp reads TMEM lanes
// 32*(w%4) .. +31, i.e. one output row per thread, in 32-column chunks.
#pragma once

#include "actq_math.cuh"
#include "sbl_device.cuh"

namespace sbl {

// ---------------------------------------------------------------------------
// Backward GEMMs: D[M, N] = alpha * sum_k A[m, k] B[n, k], bf16 in, fp32 accumulate.
//   A_MN = false: A stored [M][K] (K contiguous);  true: A stored [K][M].
//   B_MN = false: B stored [N][K];                 true: B stored [K][N].
// Output row-major [M][N], bf16 (RN) or fp32.
// ---------------------------------------------------------------------------
struct Bf16Params {
  int M, N, K;
  const float* alpha;  // device scalar, or nullptr for 1
  void* out;
  int64_t ldo;         // elements
  uint32_t* status;
  const uint8_t* mask;  // optional N:M keep bits [M][N / mask_m]: zero out[r][c] where bit c % mask_m is clear
  int mask_m;
};

// Keep bits of columns col0 .. col0 + 31 of row `row` (col0 a multiple of 32,
// N a multiple of 64), one bit per column, from mask bytes of mask_m bits.
__device__ __forceinline__ uint32_t keep_bits32(const uint8_t* mask, int mask_m, int row, int N, int col0) {
  const uint8_t* src = mask + int64_t(row) * (N / mask_m) + col0 / mask_m;
  uint32_t keep = 0;
  if (mask_m == 8) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(src);
    keep = w;  // four bytes of eight bits: byte i holds columns 8i .. 8i + 7
  } else if (mask_m == 4) {
    const uint2 w = *reinterpret_cast<const uint2*>(src);
#pragma unroll
    for (int i = 0; i < 4; ++i) keep |= ((w.x >> (8 * i)) & 0xFu) << (4 * i);
#pragma unroll
    for (int i = 0; i < 4; ++i) keep |= ((w.y >> (8 * i)) & 0xFu) << (16 + 4 * i);
  } else {  // mask_m == 2
    const uint4 w = *reinterpret_cast<const uint4*>(src);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int i = 0; i < 4; ++i) keep |= ((ws[j] >> (8 * i)) & 0x3u) << (8 * j + 2 * i);
  }
  return keep;
}

// bf16 (or fp32) output of one 256-column accumulator tile:
// out[row][n0 + c] = alpha * acc, with the optional N:M keep bits applied.
template <bool OUT_F32>
__device__ __forceinline__ void bf16_epilogue(const Bf16Params& p, uint32_t t_acc, int row, int n0, int part,
                                            int parts) {
  constexpr int BN = 256;
  const float alpha = p.alpha ? *p.alpha : 1.0f;
#pragma unroll 1
  for (int c = part; c < BN / 32; c += parts) {
    uint32_t r[32];
    __syncwarp();
    tmem_load_32x32b_x32(t_acc + c * 32, r);
    tmem_load_wait();
    const int col0 = n0 + c * 32;
    if (row >= p.M || col0 >= p.N) continue;  // after the warp-wide load: divergence is harmless
    if (p.mask != nullptr) {
      const uint32_t keep = keep_bits32(p.mask, p.mask_m, row, p.N, col0);
#pragma unroll
      for (int e = 0; e < 32; ++e) r[e] = ((keep >> e) & 1u) ? r[e] : 0u;
    }
    if (OUT_F32) {
      float* dst = reinterpret_cast<float*>(p.out) + int64_t(row) * p.ldo + col0;
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        if (col0 + 4 * v < p.N) {
          float4 o;
          o.x = __fmul_rn(alpha, __uint_as_float(r[4 * v + 0]));
          o.y = __fmul_rn(alpha, __uint_as_float(r[4 * v + 1]));
          o.z = __fmul_rn(alpha, __uint_as_float(r[4 * v + 2]));
          o.w = __fmul_rn(alpha, __uint_as_float(r[4 * v + 3]));
          *reinterpret_cast<float4*>(dst + 4 * v) = o;
        }
      }
    } else {
      __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + int64_t(row) * p.ldo + col0;
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        if (col0 + 8 * v < p.N) {
          uint32_t packed[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float lo = __fmul_rn(alpha, __uint_as_float(r[8 * v + 2 * e]));
            const float hi = __fmul_rn(alpha, __uint_as_float(r[8 * v + 2 * e + 1]));
            __nv_bfloat162 h2 = __floats2bfloat162_rn(lo, hi);
            packed[e] = *reinterpret_cast<uint32_t*>(&h2);
          }
          *reinterpret_cast<uint4*>(dst + 8 * v) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Forward: acc[o, t] = sum_k W_eff[o, k] xq[t, k] in int32 on the tensor
// cores (W_eff is the A operand so that the 2:4 sparsity sits on A along K),
// then y[t, o] = (float)acc * ((g * a'_t) / 127).
// ---------------------------------------------------------------------------
struct FwdParams {
  int n_out, T, K;
  const float* g;        // device scalar in the prepared blob
  const float* a_prime;  // [T]
  float* y;              // [T][n_out]
  int32_t* acc_out;      // optional [T][n_out]
  const uint8_t* meta;   // sparse: tensor-core metadata section
  int meta_kblocks;      // 128-wide k blocks per row block in the metadata section
  uint32_t* status;
  // Configurations that quantise the activations in the same launch (QX):
  const uint4* x;        // bf16 [T][K] as 16-byte vectors
  int8_t* xq;            // the codes (the B operand's tensor map covers them)
  float* ap_out;         // a' per token (the array a_prime points to)
  uint32_t* ready;       // per BN-token tile: rows quantised so far, zero at launch
};

// Rows of up to kQxMaxRW * 32 * 8 elements are quantised by one warp, the row
// held in registers.
constexpr int kQxMaxRW = 12;  // 16-byte vectors a lane: K <= 3072

// One token row quantised by one warp: a' = max(max_k |x|, 1e-5) through an
// integer max over the bf16 magnitude bits, then the codes by one fused
// multiply-add each (or the IEEE division for a row under the clamp or at
// 2^120 and above), as the act-quant kernel computes them.
__device__ __forceinline__ void quantise_row_warp(const FwdParams& p, int row, int lane) {
  const int nvec = p.K / 8;
  const uint4* src = p.x + int64_t(row) * nvec;
  uint4 v[kQxMaxRW];
#pragma unroll
  for (int r = 0; r < kQxMaxRW; ++r) {
    const int i = r * 32 + lane;
    v[r] = (i < nvec) ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
  }
  uint32_t m2 = 0;
#pragma unroll
  for (int r = 0; r < kQxMaxRW; ++r) {
    m2 = __vmaxu2(m2, v[r].x & 0x7FFF7FFFu);
    m2 = __vmaxu2(m2, v[r].y & 0x7FFF7FFFu);
    m2 = __vmaxu2(m2, v[r].z & 0x7FFF7FFFu);
    m2 = __vmaxu2(m2, v[r].w & 0x7FFF7FFFu);
  }
  const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, max(m2 & 0xFFFFu, m2 >> 16));
  const float ap = fmaxf(__uint_as_float(m << 16), 1e-5f);
  if (lane == 0) {
    p.ap_out[row] = ap;
    if (m >= 0x7F80u) raise_status(p.status, SBL_STATUS_NONFINITE_X);
  }
  const QScale qs = make_qscale(ap);
  uint2* dst = reinterpret_cast<uint2*>(p.xq + int64_t(row) * p.K);
#pragma unroll
  for (int r = 0; r < kQxMaxRW; ++r) {
    const int i = r * 32 + lane;
    if (i < nvec) dst[i] = qs.exact ? quantise8_div(v[r], qs.ap) : quantise8_fma(v[r], qs.c);
  }
}

// One 32-token chunk of the forward epilogue.  The thread owns output row o
// (a TMEM lane) and holds its 32 int32 accumulators for tokens t0..t0+31;
// lane j computes token t0+j's scale (g * a') / 127 and shares it with a
// shuffle.  For each token the warp stores 32 consecutive floats of y.

template <bool ACC_OUT, int NC = 32>
__device__ __forceinline__ void fwd_epilogue_chunk(const FwdParams& p, const uint32_t (&r)[NC], int o, int t0,
                                                   int lane, float g) {
  const int tl = t0 + lane;
  // a' through L2: in a launch that quantises the activations itself, other
  // CTAs wrote it during this launch
  const float f_mine = (tl < p.T) ? __fdiv_rn(__fmul_rn(g, __ldcg(p.a_prime + tl)), 127.0f) : 0.0f;
  const bool row_ok = o < p.n_out;
  const int64_t ld = p.n_out;
  float* yp = p.y + int64_t(t0) * ld + o;
  int32_t* ap = ACC_OUT ? p.acc_out + int64_t(t0) * ld + o : nullptr;
  if (t0 + NC <= p.T) {  // full chunk: no per-token bound
#pragma unroll
    for (int j = 0; j < NC; ++j) {
      const float f = __shfl_sync(0xffffffffu, f_mine, j);
      const int32_t a = static_cast<int32_t>(r[j]);
      if (row_ok) {
        *yp = __fmul_rn(static_cast<float>(a), f);
        if (ACC_OUT) *ap = a;
      }
      yp += ld;
      if (ACC_OUT) ap += ld;
    }
  } else {
#pragma unroll
    for (int j = 0; j < NC; ++j) {
      const float f = __shfl_sync(0xffffffffu, f_mine, j);
      const int32_t a = static_cast<int32_t>(r[j]);
      if (row_ok && t0 + j < p.T) {
        *yp = __fmul_rn(static_cast<float>(a), f);
        if (ACC_OUT) *ap = a;
      }
      yp += ld;
      if (ACC_OUT) ap += ld;
    }
  }
}

}  // namespace sbl
