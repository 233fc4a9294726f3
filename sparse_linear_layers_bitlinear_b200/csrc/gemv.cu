// Decode-shaped forward (t <= 16 tokens) over the 2-bit weight packing, with
// the per-token activation quantisation fused in.
//
// The weight stream is the whole cost at these token counts: 2 bits per
// weight (one byte per group of four: the metadata nibble i0 | i1 << 2 in the
// high half, the two kept codes in the low half, 01 = +1, 11 = -1).  Each
// block owns a contiguous range of output rows.  Calls are launched with
// programmatic dependent launch: a call starts while the kernel before it
// still runs, prefetches its block's weight rows (and x) into L2 with one bulk
// prefetch, lets the next call launch, and only then waits for its
// predecessor, so in a chain of decode calls each weight stream overlaps the
// call before it.  After the wait eight threads per row load the row's 16-byte
// pieces (L2 hits), the block quantises the t activation rows into shared
// memory (the same arithmetic as the act-quant kernel; block 0 also writes them
// out when the caller asked for them), and a group byte expands through a
// 256-entry table into its four int8 weights that dp4a multiplies with four
// activation codes of each token.
#include <mutex>

#include "sbl_kernels.h"

#include "actq_math.cuh"
#include "sbl_device.cuh"

namespace sbl {

constexpr int kGemvThreads = 512;
constexpr size_t kGemvMaxSmem = 200 * 1024;
constexpr int kLutWords = 256 * 32;
constexpr int kRowThreads = 8;                      // threads sharing one output row
constexpr int kRowSlots = kGemvThreads / kRowThreads;  // rows in flight per block

struct GemvArgs {
  const uint4* gemv;   // [n_out][k/64] 16-byte pieces
  const uint4* x;      // bf16 [t][k/8] 16-byte vectors
  const float* g;
  float* y;
  int32_t* acc_out;
  int8_t* xq_out;      // optional
  float* ap_out;       // optional
  const int8_t* xq_in; // codes written by the act-quant kernel (PREQUANT)
  const float* ap_in;
  uint32_t* status;
  int n_out, t, k;
};

// 16-byte weight pieces each thread keeps in flight (fewer when many tokens'
// accumulators need the registers).
template <int TP>
constexpr int gemv_pieces() {
  return TP >= 8 ? 4 : 8;
}

template <int TP, bool PREQUANT>
__global__ void __launch_bounds__(kGemvThreads) k_gemv(const GemvArgs a) {
  constexpr int kPieces = gemv_pieces<TP>();
  extern __shared__ __align__(16) uint32_t smem_w[];
  uint32_t* lut = smem_w;                    // [256 entries][32 banks]: one copy per bank
  float* s_scale = reinterpret_cast<float*>(smem_w + kLutWords);  // [TP] (g * a') / 127
  float* s_red = s_scale + 16;               // [16 warps] reduction scratch
  uint32_t* xw = smem_w + kLutWords + 32;    // [TP][k/4] int8 codes as words
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int kw = a.k / 4;                    // code words per token row

  // Rows of this block.  The kernel before this one in the stream may still
  // be writing this call's inputs (a prepare writes the weights, the previous
  // layer writes x), so they are only prefetched into L2 before the wait and
  // read after it; the next call may launch at once and do the same, so the
  // weight streams of consecutive calls overlap.
  const int rpb = (a.n_out + gridDim.x - 1) / gridDim.x;
  const int row_begin = blockIdx.x * rpb;
  const int row_end = min(a.n_out, row_begin + rpb);
  const int slot = tid / kRowThreads, sub = tid % kRowThreads;
  const int pieces = a.k / 64;  // 16-byte weight pieces per row
  if (tid == 0 && row_end > row_begin)
    bulk_prefetch_l2(a.gemv + int64_t(row_begin) * pieces, static_cast<uint32_t>(row_end - row_begin) * pieces * 16u);
  if (tid == 32 && blockIdx.x == 0) {
    if (PREQUANT) bulk_prefetch_l2(a.xq_in, static_cast<uint32_t>(a.t) * static_cast<uint32_t>(a.k));
    else bulk_prefetch_l2(a.x, static_cast<uint32_t>(a.t) * static_cast<uint32_t>(a.k) * 2u);
  }
  pdl_trigger();
  // Expansion table: group byte -> four int8 weights, replicated so that
  // lane l always reads bank l (the bytes a warp looks up are random).
  {
    const int i = tid >> 1, half = tid & 1;  // 256 entries x 2 threads, 16 copies each
    const int c0 = (i & 1) ? ((i & 2) ? -1 : 1) : 0;  // 2-bit codes: 01 = +1, 11 = -1, 00 = 0
    const int c1 = (i & 4) ? ((i & 8) ? -1 : 1) : 0;
    const int i0 = (i >> 4) & 3, i1 = (i >> 6) & 3;
    const uint32_t v = ((static_cast<uint32_t>(c0) & 0xFFu) << (8 * i0)) | ((static_cast<uint32_t>(c1) & 0xFFu) << (8 * i1));
    uint4* dst = reinterpret_cast<uint4*>(lut + i * 32 + half * 16);
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = make_uint4(v, v, v, v);
  }
  pdl_wait();
  uint4 wbuf[kPieces];
  {
    const int row = row_begin + slot;
#pragma unroll
    for (int q = 0; q < kPieces; ++q) {
      const int j = sub + kRowThreads * q;
      wbuf[q] = (row < row_end && j < pieces) ? __ldcs(a.gemv + int64_t(row) * pieces + j) : make_uint4(0, 0, 0, 0);
    }
  }

  // This thread's share of the activation rows (fused quantisation) and g.
  constexpr int kXq = 4;  // 16-byte activation vectors kept in registers
  const int nvec = a.k / 8;
  const int wpr = (kGemvThreads / 32) / TP;  // warps per token row
  const int xrow = warp / wpr, xsub = warp % wpr;
  const uint4* xsrc = a.x + int64_t(xrow) * nvec;
  uint4 xbuf[kXq];
  if (!PREQUANT) {
#pragma unroll
    for (int q = 0; q < kXq; ++q) {
      const int i = (xsub + q * wpr) * 32 + lane;
      xbuf[q] = (xrow < a.t && i < nvec) ? __ldg(xsrc + i) : make_uint4(0, 0, 0, 0);
    }
  }
  const float g = __ldg(a.g);

  const uint32_t* my_lut = lut + lane;

  if (!PREQUANT) {
    // Activation quantisation of the t rows into shared memory: the warps
    // split into t groups, one per row; two block barriers in all.
    float amax = 0.0f;
    uint32_t bad = 0;
    if (xrow < a.t) {
#pragma unroll
      for (int q = 0; q < kXq; ++q) scan8(xbuf[q], amax, bad);
      for (int i = (xsub + kXq * wpr) * 32 + lane; i < nvec; i += wpr * 32) scan8(__ldg(xsrc + i), amax, bad);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      bad |= __shfl_xor_sync(0xffffffffu, bad, off);
    }
    if (lane == 0) s_red[warp] = bad ? -1.0f : amax;  // amax >= 0, so -1 flags a non-finite row
    __syncthreads();
    float m = 0.0f;
    bool row_bad = false;
    for (int w = 0; w < wpr; ++w) {
      const float v = s_red[xrow * wpr + w];
      row_bad |= v < 0.0f;
      m = fmaxf(m, v);
    }
    const float ap = fmaxf(m, 1e-5f);
    if (xrow < a.t) {
      if (xsub == 0 && lane == 0) {
        s_scale[xrow] = __fdiv_rn(__fmul_rn(g, ap), 127.0f);
        if (blockIdx.x == 0) {
          if (a.ap_out) a.ap_out[xrow] = ap;
          if (row_bad) raise_status(a.status, SBL_STATUS_NONFINITE_X);
        }
      }
      const QScale qs = make_qscale(ap);
      uint2* dst = reinterpret_cast<uint2*>(xw + xrow * kw);
      uint2* gdst = (blockIdx.x == 0 && a.xq_out) ? reinterpret_cast<uint2*>(a.xq_out + int64_t(xrow) * a.k) : nullptr;
#pragma unroll
      for (int q = 0; q < kXq; ++q) {
        const int i = (xsub + q * wpr) * 32 + lane;
        if (i < nvec) {
          const uint2 c = quantise8(xbuf[q], qs);
          dst[i] = c;
          if (gdst) gdst[i] = c;
        }
      }
      for (int i = (xsub + kXq * wpr) * 32 + lane; i < nvec; i += wpr * 32) {
        const uint2 c = quantise8(__ldg(xsrc + i), qs);
        dst[i] = c;
        if (gdst) gdst[i] = c;
      }
    }
  } else {
    // The act-quant kernel before this one wrote the codes and scales.
    // One bulk copy brings all t rows of codes (t * k bytes, a multiple of 64).
    __shared__ uint64_t bar;
    if (tid == 0) {
      mbar_init(&bar, 1);
      fence_mbar_init();
      fence_proxy_async_smem();
      const uint32_t bytes = static_cast<uint32_t>(a.t) * static_cast<uint32_t>(a.k);
      mbar_arrive_expect_tx(&bar, bytes);
      bulk_load(xw, a.xq_in, bytes, &bar);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&bar, 0)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
          raise_status(a.status, SBL_STATUS_TIMEOUT);
          break;
        }
      }
    }
    if (tid < a.t) s_scale[tid] = __fdiv_rn(__fmul_rn(g, __ldcg(a.ap_in + tid)), 127.0f);
  }
  for (int i = a.t * kw + tid; i < TP * kw; i += kGemvThreads) xw[i] = 0u;  // padding tokens
  __syncthreads();

  // Dot products: eight threads per row, then a reduction inside the group.
  for (int r0 = row_begin; r0 < row_end; r0 += kRowSlots) {
    const int row = r0 + slot;
    // a warp holds 4 rows; it skips the pass when all of them are past the end
    if (r0 + (warp * 32) / kRowThreads >= row_end) continue;
    int acc[TP];
#pragma unroll
    for (int tt = 0; tt < TP; ++tt) acc[tt] = 0;
    for (int j0 = 0; j0 < pieces; j0 += kRowThreads * kPieces) {
      if (r0 != row_begin || j0 != 0) {  // the first batch was loaded up front
#pragma unroll
        for (int q = 0; q < kPieces; ++q) {
          const int j = j0 + sub + kRowThreads * q;
          wbuf[q] = (row < row_end && j < pieces) ? __ldcs(a.gemv + int64_t(row) * pieces + j) : make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll(TP >= 8 ? 1 : kPieces)
      for (int q = 0; q < kPieces; ++q) {
        const int j = j0 + sub + kRowThreads * q;
        if (j >= pieces) break;
        const uint32_t words[4] = {wbuf[q].x, wbuf[q].y, wbuf[q].z, wbuf[q].w};
        // 16 groups = 64 weights = code words 16j .. 16j+15; the rotation by
        // (sub >> 1) keeps the 16-byte shared loads of a row's threads on
        // distinct banks.
#pragma unroll
        for (int i2 = 0; i2 < 4; ++i2) {
          const int i = (i2 + (sub >> 1)) & 3;
          const uint32_t wd = words[i];
          const uint32_t w0 = my_lut[(wd & 0xFFu) << 5], w1 = my_lut[((wd >> 8) & 0xFFu) << 5];
          const uint32_t w2 = my_lut[((wd >> 16) & 0xFFu) << 5], w3 = my_lut[(wd >> 24) << 5];
#pragma unroll
          for (int tt = 0; tt < TP; ++tt) {
            const uint4 xv = *reinterpret_cast<const uint4*>(xw + tt * kw + 16 * j + 4 * i);
            int s = acc[tt];
            s = __dp4a(static_cast<int>(w0), static_cast<int>(xv.x), s);
            s = __dp4a(static_cast<int>(w1), static_cast<int>(xv.y), s);
            s = __dp4a(static_cast<int>(w2), static_cast<int>(xv.z), s);
            s = __dp4a(static_cast<int>(w3), static_cast<int>(xv.w), s);
            acc[tt] = s;
          }
        }
      }
    }
#pragma unroll
    for (int tt = 0; tt < TP; ++tt) {
#pragma unroll
      for (int off = kRowThreads / 2; off > 0; off >>= 1) acc[tt] += __shfl_xor_sync(0xffffffffu, acc[tt], off);
    }
    if (row < row_end) {
#pragma unroll
      for (int tt = 0; tt < TP; ++tt) {
        if (tt % kRowThreads == sub && tt < a.t) {
          a.y[int64_t(tt) * a.n_out + row] = __fmul_rn(static_cast<float>(acc[tt]), s_scale[tt]);
          if (a.acc_out) a.acc_out[int64_t(tt) * a.n_out + row] = acc[tt];
        }
      }
    }
  }
}

template <int TP, bool PREQUANT>
static cudaError_t gemv_tp(const GemvArgs& a, int num_sms, cudaStream_t s) {
  const size_t smem = (kLutWords + 32 + size_t(TP) * size_t(a.k / 4)) * 4;
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    err = cudaFuncSetAttribute(k_gemv<TP, PREQUANT>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemvMaxSmem);
  });
  if (err != cudaSuccess) return err;
  // At most one block per SM, each owning a contiguous range of rows.
  int blocks = (a.n_out < num_sms) ? a.n_out : num_sms;
  return launch_pdl(k_gemv<TP, PREQUANT>, dim3(blocks), dim3(kGemvThreads), smem, s, a);
}

bool gemv_fits(int64_t t, int64_t k) {
  const int64_t tp = t <= 1 ? 1 : t <= 2 ? 2 : t <= 4 ? 4 : t <= 8 ? 8 : 16;
  return t >= 1 && t <= 16 && (kLutWords + 32 + tp * (k / 4)) * 4 <= int64_t(kGemvMaxSmem);
}

// The GEMV's dot products run on the CUDA cores and grow with t * n_out * k,
// while the 2:4 tensor-core GEMM costs about one round of tiles for a handful
// of tokens (measured at k = 2560: ~12 us for t = 4..32 against 6.8-17.5 us
// for the GEMV, which wins up to about 8e7 multiply-adds, e.g. t = 4 at
// n_out = 6912 or t = 8 at n_out = 2560).
constexpr int64_t kGemvMaxMacs = 80000000;

bool gemv_preferred(int64_t t, int64_t n_out, int64_t k) { return t * n_out * k <= kGemvMaxMacs; }

// Token counts up to kFusedMaxT quantise inside the GEMV (every block redoes
// that small amount of work, which saves a launch); larger ones run the
// act-quant kernel first.
constexpr int64_t kFusedMaxT = 4;

bool gemv_fuses_act_quant(int64_t t) { return t <= kFusedMaxT; }

cudaError_t launch_forward_gemv(const uint8_t* gemv, const uint16_t* x, const int8_t* xq_in, const float* ap_in,
                                const float* g, int64_t n_out, int64_t t, int64_t k, float* y, int32_t* acc_out,
                                int8_t* xq_out, float* ap_out, uint32_t* status, int num_sms, cudaStream_t s) {
  GemvArgs a;
  a.gemv = reinterpret_cast<const uint4*>(gemv);
  a.x = reinterpret_cast<const uint4*>(x);
  a.g = g;
  a.y = y;
  a.acc_out = acc_out;
  a.xq_out = xq_out;
  a.ap_out = ap_out;
  a.xq_in = xq_in;
  a.ap_in = ap_in;
  a.status = status;
  a.n_out = static_cast<int>(n_out);
  a.t = static_cast<int>(t);
  a.k = static_cast<int>(k);
  // codes from the caller (x == NULL) or from the act-quant kernel before
  // this one, else quantised here
  const bool pre = x == nullptr || !gemv_fuses_act_quant(t);
  if (t <= 1) return pre ? gemv_tp<1, true>(a, num_sms, s) : gemv_tp<1, false>(a, num_sms, s);
  if (t <= 2) return pre ? gemv_tp<2, true>(a, num_sms, s) : gemv_tp<2, false>(a, num_sms, s);
  if (t <= 4) return pre ? gemv_tp<4, true>(a, num_sms, s) : gemv_tp<4, false>(a, num_sms, s);
  if (t <= 8) return gemv_tp<8, true>(a, num_sms, s);
  return gemv_tp<16, true>(a, num_sms, s);
}

}  // namespace sbl
