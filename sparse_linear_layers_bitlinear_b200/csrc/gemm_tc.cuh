// Persistent, warp-specialised tcgen05 GEMM mainloop for sm_100a.
//
//   warp 0      TMA producer: fills a ring of shared-memory stages
//   warp 1      allocates TMEM; lane 0 issues tcgen05.mma into one of two
//               TMEM accumulators and commits stage / accumulator barriers
//   warps 2..5  epilogue: tcgen05.ld the accumulator (warp w reads TMEM lanes
//               32*(w%4) .. +31), rescale, store to global memory
//
// A configuration class supplies tile sizes, the per-stage loads, the MMA
// issue for one stage and the epilogue.  Every mbarrier wait is bounded: on
// timeout the kernel records SBL_STATUS_TIMEOUT and all roles wind down.
#pragma once

#include "sbl_device.cuh"

namespace sbl {

constexpr int kGemmThreads = 192;

struct GemmSmemTail {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  volatile uint32_t consumed;  // stages the MMA thread has consumed (for abort drain)
};

template <class Cfg>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const typename Cfg::Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms.
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* smA = smem;
  uint8_t* smB = smA + Cfg::STAGES * Cfg::A_BYTES;
  uint8_t* smE = smB + Cfg::STAGES * Cfg::B_BYTES;
  GemmSmemTail* tail = reinterpret_cast<GemmSmemTail*>(smE + Cfg::STAGES * Cfg::E_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint32_t* status = p.status;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::STAGES; ++s) {
      mbar_init(&tail->full[s], 1);
      mbar_init(&tail->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tail->acc_full[b], 1);
      mbar_init(&tail->acc_empty[b], 4);  // one arrive per epilogue warp
    }
    mbar_init(&tail->drain, 1);
    tail->abort_flag = 0;
    tail->consumed = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  if (warp == 1) tmem_alloc(&tail->tmem_base, Cfg::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem_base = tail->tmem_base;
  volatile int* abort_flag = &tail->abort_flag;
  const int m_blocks = (Cfg::rows_M(p) + Cfg::BM - 1) / Cfg::BM;
  const int n_blocks = (Cfg::cols_N(p) + Cfg::BN - 1) / Cfg::BN;
  const int num_tiles = m_blocks * n_blocks;
  const int k_blocks = Cfg::k_blocks(p);

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t stage = 0, phase = 0, issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m0 = (tile % m_blocks) * Cfg::BM;
        const int n0 = (tile / m_blocks) * Cfg::BN;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&tail->empty[stage], phase ^ 1u, abort_flag, status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&tail->full[stage], Cfg::A_BYTES + Cfg::B_BYTES + Cfg::E_BYTES);
          Cfg::load_stage(&tmA, &tmB, p, smA + stage * Cfg::A_BYTES, smB + stage * Cfg::B_BYTES,
                          smE + stage * Cfg::E_BYTES, m0, n0, kb, &tail->full[stage]);
          ++issued;
          if (++stage == Cfg::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // Let the copies already in flight land before the CTA exits.
        for (uint32_t i = tail->consumed; i < issued; ++i) {
          uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(&tail->full[i % Cfg::STAGES], (i / Cfg::STAGES) & 1u)) {
            if (globaltimer_ns() - t0 > 10000000ull) break;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      uint32_t local = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
        const uint32_t ab = local & 1u;
        const uint32_t aphase = (local >> 1) & 1u;
        if (!mbar_wait(&tail->acc_empty[ab], aphase ^ 1u, abort_flag, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + ab * Cfg::ACC_COLS;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&tail->full[stage], phase, abort_flag, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          Cfg::mma_stage(p, d_tmem, tmem_base + Cfg::E_COL0 + (stage & 1u) * Cfg::E_COLS, smA + stage * Cfg::A_BYTES,
                         smB + stage * Cfg::B_BYTES, smE + stage * Cfg::E_BYTES, kb == 0);
          mma_commit(&tail->empty[stage]);  // frees the stage once these MMAs have read it
          tail->consumed = tail->consumed + 1;
          if (++stage == Cfg::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&tail->acc_full[ab]);  // accumulator complete
      }
      // Make sure no MMA is still running when TMEM is released.
      mma_commit(&tail->drain);
      uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&tail->drain, 0)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
          raise_status(status, SBL_STATUS_TIMEOUT);
          break;
        }
      }
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    uint32_t local = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
      const uint32_t ab = local & 1u;
      const uint32_t aphase = (local >> 1) & 1u;
      bool ready = true;
      if (lane == 0) ready = mbar_wait(&tail->acc_full[ab], aphase, abort_flag, status);
      ready = __shfl_sync(0xffffffffu, ready ? 1 : 0, 0) != 0;
      if (!ready) break;
      tc_fence_after();
      const int m0 = (tile % m_blocks) * Cfg::BM;
      const int n0 = (tile / m_blocks) * Cfg::BN;
      const uint32_t t_acc = tmem_base + ab * Cfg::ACC_COLS + (uint32_t(quarter * 32) << 16);
      Cfg::epilogue(p, t_acc, m0 + quarter * 32 + lane, n0, lane);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tail->acc_empty[ab]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

template <class Cfg>
constexpr int gemm_smem_bytes() {
  return 1024 + Cfg::STAGES * (Cfg::A_BYTES + Cfg::B_BYTES + Cfg::E_BYTES) + int(sizeof(GemmSmemTail));
}

// ---------------------------------------------------------------------------
// Backward: D[M, N] = alpha * sum_k A[m, k] B[n, k], bf16 in, fp32 accumulate.
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

template <bool A_MN, bool B_MN, bool OUT_F32>
struct CfgBf16 {
  using Params = Bf16Params;
  static constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
  static constexpr int A_BYTES = BM * BK * 2;  // 16 KB
  static constexpr int B_BYTES = BN * BK * 2;  // 32 KB
  static constexpr int E_BYTES = 0;
  static constexpr int ACC_COLS = BN;
  static constexpr int TMEM_COLS = 512;
  static constexpr int E_COL0 = 0, E_COLS = 0;
  static constexpr uint32_t IDESC = idesc_bf16(128, BN, A_MN, B_MN);

  __device__ static int rows_M(const Params& p) { return p.M; }
  __device__ static int cols_N(const Params& p) { return p.N; }
  __device__ static int k_blocks(const Params& p) { return (p.K + BK - 1) / BK; }

  __device__ static void load_stage(const CUtensorMap* tA, const CUtensorMap* tB, const Params&, uint8_t* sA,
                                    uint8_t* sB, uint8_t*, int m0, int n0, int kb, uint64_t* bar) {
    const int k0 = kb * BK;
    if (A_MN) {  // two boxes of [64 k][64 m]
      tma_load_2d(sA, tA, m0, k0, bar);
      tma_load_2d(sA + 8192, tA, m0 + 64, k0, bar);
    } else {  // one box of [128 m][64 k]
      tma_load_2d(sA, tA, k0, m0, bar);
    }
    if (B_MN) {  // four boxes of [64 k][64 n]
#pragma unroll
      for (int j = 0; j < 4; ++j) tma_load_2d(sB + 8192 * j, tB, n0 + 64 * j, k0, bar);
    } else {  // one box of [256 n][64 k]
      tma_load_2d(sB, tB, k0, n0, bar);
    }
  }

  __device__ static void mma_stage(const Params&, uint32_t d_tmem, uint32_t, uint8_t* sA, uint8_t* sB, uint8_t*,
                                   bool first) {
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
#pragma unroll
    for (int kk = 0; kk < BK / 16; ++kk) {
      const uint64_t ad = A_MN ? smem_desc(a0 + kk * 2048, 8192, 1024, 2) : smem_desc(a0 + kk * 32, 16, 1024, 2);
      const uint64_t bd = B_MN ? smem_desc(b0 + kk * 2048, 8192, 1024, 2) : smem_desc(b0 + kk * 32, 16, 1024, 2);
      mma_bf16(d_tmem, ad, bd, IDESC, (first && kk == 0) ? 0u : 1u);
    }
  }

  __device__ static void epilogue(const Params& p, uint32_t t_acc, int row, int n0, int, int part = 0,
                                  int parts = 1) {
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
};

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
};

// One 32-token chunk of the forward epilogue.  The thread owns output row o
// (a TMEM lane) and holds its 32 int32 accumulators for tokens t0..t0+31;
// lane j computes token t0+j's scale (g * a') / 127 and shares it with a
// shuffle.  For each token the warp stores 32 consecutive floats of y.

template <bool ACC_OUT, int NC = 32>
__device__ __forceinline__ void fwd_epilogue_chunk(const FwdParams& p, const uint32_t (&r)[NC], int o, int t0,
                                                   int lane, float g) {
  const int tl = t0 + lane;
  const float f_mine = (tl < p.T) ? __fdiv_rn(__fmul_rn(g, p.a_prime[tl]), 127.0f) : 0.0f;
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

// Dense int8: A = W_eff codes [n_out][K], B = xq [T][K]; UMMA 128 x 256 x 32.
template <bool ACC_OUT>
struct CfgFwdDense {
  using Params = FwdParams;
  static constexpr int BM = 128, BN = 256, BK = 128, STAGES = 4;
  static constexpr int A_BYTES = BM * BK;  // 16 KB
  static constexpr int B_BYTES = BN * BK;  // 32 KB
  static constexpr int E_BYTES = 0;
  static constexpr int ACC_COLS = BN;
  static constexpr int TMEM_COLS = 512;
  static constexpr int E_COL0 = 0, E_COLS = 0;
  static constexpr uint32_t IDESC = idesc_i8(128, BN, false);

  __device__ static int rows_M(const Params& p) { return p.n_out; }
  __device__ static int cols_N(const Params& p) { return p.T; }
  __device__ static int k_blocks(const Params& p) { return (p.K + BK - 1) / BK; }

  __device__ static void load_stage(const CUtensorMap* tA, const CUtensorMap* tB, const Params&, uint8_t* sA,
                                    uint8_t* sB, uint8_t*, int m0, int n0, int kb, uint64_t* bar) {
    tma_load_2d(sA, tA, kb * BK, m0, bar);  // box [128 rows][128 bytes]
    tma_load_2d(sB, tB, kb * BK, n0, bar);  // box [256 rows][128 bytes]
  }

  __device__ static void mma_stage(const Params&, uint32_t d_tmem, uint32_t, uint8_t* sA, uint8_t* sB, uint8_t*,
                                   bool first) {
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
#pragma unroll
    for (int kk = 0; kk < BK / 32; ++kk) {
      mma_i8(d_tmem, smem_desc(a0 + kk * 32, 16, 1024, 2), smem_desc(b0 + kk * 32, 16, 1024, 2), IDESC,
             (first && kk == 0) ? 0u : 1u);
    }
  }

  __device__ static void epilogue(const Params& p, uint32_t t_acc, int row, int n0, int lane) {
    const float g = *p.g;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      uint32_t r[32];
      __syncwarp();
      tmem_load_32x32b_x32(t_acc + c * 32, r);
      tmem_load_wait();
      if (n0 + c * 32 >= p.T) continue;  // uniform across the warp
      fwd_epilogue_chunk<ACC_OUT>(p, r, row, n0 + c * 32, lane, g);
    }
  }
};

// 2:4 sparse int8: A = kept codes [n_out][K/2] plus metadata, B = xq [T][K].
// One stage covers 256 logical k: A 128 x 128 bytes, B 2 x [128 rows][128
// bytes], metadata 2 blocks of 128 rows x 16 bytes.  UMMA 128 x 128 x 64.
template <bool ACC_OUT>
struct CfgFwdSparse {
  using Params = FwdParams;
  static constexpr int BM = 128, BN = 128, BK = 256, STAGES = 4;
  static constexpr int A_BYTES = BM * BK / 2;  // 16 KB
  static constexpr int B_BYTES = BN * BK;      // 32 KB
  static constexpr int E_BYTES = 2 * 2048;     // 4 KB
  static constexpr int ACC_COLS = BN;
  static constexpr int TMEM_COLS = 512;
  static constexpr int E_COL0 = 2 * BN;        // metadata lives after the two accumulators
  static constexpr int E_COLS = 8;             // 2 blocks x 4 columns
  static constexpr uint32_t IDESC = idesc_i8(128, BN, true);

  __device__ static int rows_M(const Params& p) { return p.n_out; }
  __device__ static int cols_N(const Params& p) { return p.T; }
  __device__ static int k_blocks(const Params& p) { return (p.K + BK - 1) / BK; }

  __device__ static void load_stage(const CUtensorMap* tA, const CUtensorMap* tB, const Params& p, uint8_t* sA,
                                    uint8_t* sB, uint8_t* sE, int m0, int n0, int kb, uint64_t* bar) {
    tma_load_2d(sA, tA, kb * (BK / 2), m0, bar);          // compressed columns
    tma_load_2d(sB, tB, kb * BK, n0, bar);                // logical k 0..127 of the stage
    tma_load_2d(sB + BN * 128, tB, kb * BK + 128, n0, bar);  // logical k 128..255
    const uint8_t* src = p.meta + (int64_t(m0 / 128) * p.meta_kblocks + kb * 2) * 2048;
    bulk_load(sE, src, E_BYTES, bar);
  }

  __device__ static void mma_stage(const Params&, uint32_t d_tmem, uint32_t e_tmem, uint8_t* sA, uint8_t* sB,
                                   uint8_t* sE, bool first) {
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB), e0 = smem_u32(sE);
    // metadata: two 128 x 16-byte blocks -> TMEM columns e_tmem + 0..3, + 4..7
    tmem_copy_128x128b(e_tmem, smem_desc(e0, 2048, 128, 0));
    tmem_copy_128x128b(e_tmem + 4, smem_desc(e0 + 2048, 2048, 128, 0));
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint64_t ad = smem_desc(a0 + kk * 32, 16, 1024, 2);  // 32 compressed bytes = 64 logical k
      const uint32_t bsub = (kk >> 1) * (BN * 128) + (kk & 1) * 64;
      const uint64_t bd = smem_desc(b0 + bsub, 16, 1024, 2);
      mma_sp_i8(d_tmem, ad, bd, e_tmem + 2 * kk, IDESC, (first && kk == 0) ? 0u : 1u);
    }
  }

  __device__ static void epilogue(const Params& p, uint32_t t_acc, int row, int n0, int lane) {
    const float g = *p.g;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      uint32_t r[32];
      __syncwarp();
      tmem_load_32x32b_x32(t_acc + c * 32, r);
      tmem_load_wait();
      if (n0 + c * 32 >= p.T) continue;  // uniform across the warp
      fwd_epilogue_chunk<ACC_OUT>(p, r, row, n0 + c * 32, lane, g);
    }
  }
};

}  // namespace sbl
