// Persistent, warp-specialised tcgen05 GEMM on CTA pairs (sm_100a).
//
// A cluster of two CTAs on two SMs computes one 256-row output tile with the
// 2-SM MMA (tcgen05.mma.cta_group::2): CTA r holds rows 128r..128r+127 of the
// A tile and half of the B tile in its shared memory, and receives its 128
// rows of the accumulator in its own tensor memory.  Per SM that halves the B
// traffic of a 128-row tile with the same N, which is what keeps the tensor
// pipe fed from L2.
//
//   warp 0      TMA producer, in both CTAs: its copies land in its own shared
//               memory and count on the even (leader) CTA's "full" barrier
//   warp 1      allocates tensor memory (both CTAs); in the leader, lane 0
//               issues the MMAs and commits to the "empty" and accumulator
//               barriers of both CTAs at once
//   warps 2..5  epilogue, in both CTAs: drain this CTA's accumulator rows,
//               then arrive on the leader's "accumulator empty" barrier
//
// Every wait is bounded; a CTA whose wait runs out records SBL_STATUS_TIMEOUT
// and winds down, and its partner's waits run out in turn.  Both CTAs always
// reach the final cluster barrier, so neither frees memory the other can
// still signal.
#pragma once

#include "gemm_epilogue.cuh"

namespace sbl {

// One output tile of a pair: problem index (for multi-problem launches),
// 256-row block, BN-column block and its number of k blocks.
struct PairTile {
  int prob, mb, nb, kblocks;
};

// Default schedule: tiles of one problem striped over the pairs, M fastest.
template <class Cfg>
struct StripedTiles {
  __device__ static int count(const typename Cfg::Params& p, int pair, int npairs) {
    const int nt = ((Cfg::rows_M(p) + 255) / 256) * ((Cfg::cols_N(p) + Cfg::BN - 1) / Cfg::BN);
    return pair < nt ? (nt - pair + npairs - 1) / npairs : 0;
  }
  __device__ static PairTile at(const typename Cfg::Params& p, int pair, int npairs, int i) {
    const int mb = (Cfg::rows_M(p) + 255) / 256;
    const int t = pair + i * npairs;
    return PairTile{0, t % mb, t / mb, Cfg::k_blocks(p)};
  }
};

struct PairSmemTail {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <class Cfg>
constexpr int pair_threads() {
  return 64 + 32 * Cfg::EPI_WARPS;
}

template <class Cfg>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pair_threads<Cfg>(), 1)
    k_gemm_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmF,
                const typename Cfg::Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* smA = smem;
  uint8_t* smB = smA + Cfg::STAGES * Cfg::A_BYTES;
  uint8_t* smE = smB + Cfg::STAGES * Cfg::B_BYTES;
  PairSmemTail* tail = reinterpret_cast<PairSmemTail*>(smE + Cfg::STAGES * Cfg::E_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  uint32_t* status = p.status;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::STAGES; ++s) {
      mbar_init(&tail->full[s], 2);   // leader: its expect-tx arrive + the partner's arrive
      mbar_init(&tail->empty[s], 1);  // one MMA commit, sent to both CTAs
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tail->acc_full[b], 1);
      mbar_init(&tail->acc_empty[b], 2 * Cfg::EPI_WARPS);  // every epilogue warp of both CTAs
    }
    mbar_init(&tail->drain, 1);
    tail->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    if (Cfg::MAPS > 2) prefetch_tensormap(&tmE);
    if (Cfg::MAPS > 3) prefetch_tensormap(&tmF);
  }
  cluster_sync_all();  // barriers initialised in both CTAs before any remote use
  if (warp == 1) tmem_alloc_pair(&tail->tmem_base, Cfg::TMEM_COLS);
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();

  const uint32_t tmem_base = tail->tmem_base;
  volatile int* abort_flag = &tail->abort_flag;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int ntiles = Cfg::Tiles::count(p, pair, npairs);

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      // A forward launch may start while the activation quantiser before it
      // still runs (programmatic dependent launch): wait for it before the
      // first load.  A no-op for launches without a programmatic dependency.
      pdl_wait();
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      const uint32_t leader_full0 = map_to_rank(&tail->full[0], 0);
      for (int i = 0; i < ntiles && ok; ++i) {
        const PairTile t = Cfg::Tiles::at(p, pair, npairs, i);
        const int m0 = t.mb * 256 + 128 * int(rank);
        const int n0 = t.nb * Cfg::BN + int(rank) * (Cfg::BN / 2);
        if constexpr (Cfg::QUANT_X) {
          // the tile's token rows are quantised by the epilogue warps of the
          // whole grid: wait for their count, then read the codes by TMA
          if (!wait_count(p.ready + t.nb, Cfg::tile_rows(p, t.nb), abort_flag, status)) break;
          fence_proxy_async_global();
        }
        for (int kb = 0; kb < t.kblocks; ++kb) {
          if (!mbar_wait(&tail->empty[stage], phase ^ 1u, abort_flag, status)) {
            ok = false;
            break;
          }
          Cfg::load_stage(&tmA, &tmB, &tmE, &tmF, p, t.prob, smA + stage * Cfg::A_BYTES, smB + stage * Cfg::B_BYTES,
                          smE + stage * Cfg::E_BYTES, m0, n0, kb, &tail->full[stage]);
          if (leader) {
            mbar_arrive_expect_tx(&tail->full[stage], 2 * (Cfg::A_BYTES + Cfg::B_BYTES + Cfg::E_BYTES));
          } else {
            mbar_arrive_remote(leader_full0 + stage * 8u);
          }
          if (++stage == Cfg::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader only) ----------------
    if (leader && lane == 0) {
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      for (int i = 0; i < ntiles && ok; ++i) {
        const PairTile t = Cfg::Tiles::at(p, pair, npairs, i);
        const uint32_t ab = uint32_t(i) & 1u;
        const uint32_t aphase = (uint32_t(i) >> 1) & 1u;
        if (!mbar_wait(&tail->acc_empty[ab], aphase ^ 1u, abort_flag, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + ab * Cfg::ACC_COLS;
        for (int kb = 0; kb < t.kblocks; ++kb) {
          if (!mbar_wait(&tail->full[stage], phase, abort_flag, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          Cfg::mma_stage(p, t.prob, d_tmem, tmem_base + Cfg::E_COL0 + (stage & 1u) * Cfg::E_COLS,
                         smA + stage * Cfg::A_BYTES, smB + stage * Cfg::B_BYTES, smE + stage * Cfg::E_BYTES, kb == 0);
          mma_commit_pair(&tail->empty[stage]);  // frees the stage in both CTAs once these MMAs have read it
          if (++stage == Cfg::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair(&tail->acc_full[ab]);  // accumulator complete in both CTAs
      }
      // No MMA may still run when tensor memory is released.
      mma_commit_pair(&tail->drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&tail->drain, 0)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
          raise_status(status, SBL_STATUS_TIMEOUT);
          break;
        }
      }
    }
  } else {
    // ---------------- epilogue (warps 2.., both CTAs) ----------------
    // Warp w reads TMEM lanes 32*(w%4)..+31; with 8 epilogue warps two warps
    // share a lane quarter and split its 32-column chunks.
    const int quarter = warp & 3;
    const int part = (warp - 2) >> 2, parts = Cfg::EPI_WARPS / 4;
    const uint32_t leader_acc_empty0 = map_to_rank(&tail->acc_empty[0], 0);
    if constexpr (Cfg::QUANT_X) {
      // Before the first accumulator is ready, the epilogue warps of the grid
      // quantise the token rows, warp by warp in row order (so the first
      // tiles' rows come first), each row counted on its tile once written.
      pdl_wait();  // x may come from the kernel before
      const int nw = int(gridDim.x) * Cfg::EPI_WARPS;
      for (int row = int(blockIdx.x) * Cfg::EPI_WARPS + (warp - 2); row < p.T; row += nw) {
        quantise_row_warp(p, row, lane);
        fence_proxy_async_global();  // the codes are read by TMA
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(p.ready + row / Cfg::BN, 1u);
      }
    }
    for (int i = 0; i < ntiles; ++i) {
      const PairTile t = Cfg::Tiles::at(p, pair, npairs, i);
      const uint32_t ab = uint32_t(i) & 1u;
      const uint32_t aphase = (uint32_t(i) >> 1) & 1u;
      bool ready = true;
      if (lane == 0) ready = mbar_wait(&tail->acc_full[ab], aphase, abort_flag, status);
      ready = __shfl_sync(0xffffffffu, ready ? 1 : 0, 0) != 0;
      if (!ready) break;
      if constexpr (Cfg::QUANT_X) {
        // the tile's a' were written by other CTAs: acquire their count
        // (complete by now: the producer waited for it before the loads)
        if (!__all_sync(0xffffffffu, wait_count(p.ready + t.nb, Cfg::tile_rows(p, t.nb), abort_flag, status))) break;
      }
      tc_fence_after();
      const int m0 = t.mb * 256 + 128 * int(rank);
      const int n0 = t.nb * Cfg::BN;
      const uint32_t t_acc = tmem_base + ab * Cfg::ACC_COLS + (uint32_t(quarter * 32) << 16);
      Cfg::epilogue(p, t.prob, t_acc, m0 + quarter * 32 + lane, n0, lane, part, parts);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(leader_acc_empty0 + ab * 8u);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the partner no longer signals this CTA's barriers
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
  }
}

template <class Cfg>
constexpr int pair_smem_bytes() {
  return 1024 + Cfg::STAGES * (Cfg::A_BYTES + Cfg::B_BYTES + Cfg::E_BYTES) + int(sizeof(PairSmemTail));
}

// ---------------------------------------------------------------------------
// bf16 backward on pairs: tile 256 (M) x 256 (N), K 64 per stage.  Each CTA
// holds A 128 x 64 and B 128 x 64 (its half of N); output by bf16_epilogue.
// ---------------------------------------------------------------------------
template <bool A_MN, bool B_MN, bool OUT_F32>
struct CfgPairBf16 {
  using Params = Bf16Params;
  using Tiles = StripedTiles<CfgPairBf16>;
  static constexpr bool QUANT_X = false;
  static constexpr int MAPS = 2;
  static constexpr int EPI_WARPS = 4;
  static constexpr int BN = 256, BK = 64, STAGES = 6;
  static constexpr int A_BYTES = 128 * BK * 2;        // 16 KB
  static constexpr int B_BYTES = (BN / 2) * BK * 2;   // 16 KB
  static constexpr int E_BYTES = 0;
  static constexpr int ACC_COLS = BN;
  static constexpr int TMEM_COLS = 512;
  static constexpr int E_COL0 = 0, E_COLS = 0;
  static constexpr uint32_t IDESC = idesc_bf16(256, BN, A_MN, B_MN);

  __device__ static int rows_M(const Params& p) { return p.M; }
  __device__ static int cols_N(const Params& p) { return p.N; }
  __device__ static int k_blocks(const Params& p) { return (p.K + BK - 1) / BK; }

  __device__ static void load_stage(const CUtensorMap* tA, const CUtensorMap* tB, const CUtensorMap*,
                                    const CUtensorMap*, const Params&, int, uint8_t* sA, uint8_t* sB, uint8_t*, int m0,
                                    int n0, int kb, uint64_t* bar) {
    const int k0 = kb * BK;
    if (A_MN) {  // two boxes of [64 k][64 m]
      tma_load_2d_pair(sA, tA, m0, k0, bar);
      tma_load_2d_pair(sA + 8192, tA, m0 + 64, k0, bar);
    } else {  // one box of [128 m][64 k]
      tma_load_2d_pair(sA, tA, k0, m0, bar);
    }
    if (B_MN) {  // two boxes of [64 k][64 n]
      tma_load_2d_pair(sB, tB, n0, k0, bar);
      tma_load_2d_pair(sB + 8192, tB, n0 + 64, k0, bar);
    } else {  // one box of [128 n][64 k]
      tma_load_2d_pair(sB, tB, k0, n0, bar);
    }
  }

  __device__ static void mma_stage(const Params&, int, uint32_t d_tmem, uint32_t, uint8_t* sA, uint8_t* sB,
                                   uint8_t*, bool first) {
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
#pragma unroll
    for (int kk = 0; kk < BK / 16; ++kk) {
      const uint64_t ad = A_MN ? smem_desc(a0 + kk * 2048, 8192, 1024, 2) : smem_desc(a0 + kk * 32, 16, 1024, 2);
      const uint64_t bd = B_MN ? smem_desc(b0 + kk * 2048, 8192, 1024, 2) : smem_desc(b0 + kk * 32, 16, 1024, 2);
      mma_bf16_pair(d_tmem, ad, bd, IDESC, (first && kk == 0) ? 0u : 1u);
    }
  }

  __device__ static void epilogue(const Params& p, int, uint32_t t_acc, int row, int n0, int lane, int part,
                                  int parts) {
    bf16_epilogue<OUT_F32>(p, t_acc, row, n0, part, parts);
  }
};

// ---------------------------------------------------------------------------
// Both STE backward products in one launch, tiles of 256 x 256:
//   problem 0 (dX):  out0[M0][N] = alpha0 * A0 . B0,  A0 K-major [M0][K0], B0 MN-major [K0][N]
//   problem 1 (dW):  out1[M1][N] = A1^T . B1,          A1 MN-major [K1][M1], B1 MN-major [K1][N]
// The host orders the tiles of both problems longest first over the pairs
// (the two problems have different depths), so the launch ends with all
// pairs close to even instead of two separate tails.
// ---------------------------------------------------------------------------
constexpr int kDualMaxPairs = 96;
constexpr int kDualMaxTiles = 1280;

struct DualBf16Params {
  int M[2], N, K[2];
  int mblocks[2];           // 256-row blocks per problem
  int tiles0;               // tile ids below this are problem 0
  const float* alpha[2];    // device scalars or nullptr for 1
  void* out[2];
  uint32_t* status;
  const uint8_t* mask1;     // optional keep bits for problem 1 (dW)
  int mask_m;
  uint16_t sched_off[kDualMaxPairs + 1];  // pair p runs sched[sched_off[p] .. sched_off[p+1])
  uint16_t sched[kDualMaxTiles];
};

template <bool OUT_F32>
struct CfgPairDualBf16 {
  using Params = DualBf16Params;
  static constexpr bool QUANT_X = false;
  static constexpr int MAPS = 4;
  static constexpr int EPI_WARPS = 4;
  static constexpr int BN = 256, BK = 64, STAGES = 6;
  static constexpr int A_BYTES = 128 * BK * 2;        // 16 KB
  static constexpr int B_BYTES = (BN / 2) * BK * 2;   // 16 KB
  static constexpr int E_BYTES = 0;
  static constexpr int ACC_COLS = BN;
  static constexpr int TMEM_COLS = 512;
  static constexpr int E_COL0 = 0, E_COLS = 0;
  static constexpr uint32_t IDESC0 = idesc_bf16(256, BN, false, true);
  static constexpr uint32_t IDESC1 = idesc_bf16(256, BN, true, true);

  struct Tiles {
    __device__ static int count(const Params& p, int pair, int) { return p.sched_off[pair + 1] - p.sched_off[pair]; }
    __device__ static PairTile at(const Params& p, int pair, int, int i) {
      const int id = p.sched[p.sched_off[pair] + i];
      const int prob = id >= p.tiles0 ? 1 : 0;
      const int local = id - (prob ? p.tiles0 : 0);
      const int mb = p.mblocks[prob];
      return PairTile{prob, local % mb, local / mb, (p.K[prob] + BK - 1) / BK};
    }
  };

  // Maps: A0, B0, A1, B1.
  __device__ static void load_stage(const CUtensorMap* tA, const CUtensorMap* tB, const CUtensorMap* tA1,
                                    const CUtensorMap* tB1, const Params&, int prob, uint8_t* sA, uint8_t* sB,
                                    uint8_t*, int m0, int n0, int kb, uint64_t* bar) {
    const int k0 = kb * BK;
    if (prob == 0) {
      tma_load_2d_pair(sA, tA, k0, m0, bar);  // [128 m][64 k]
      tma_load_2d_pair(sB, tB, n0, k0, bar);
      tma_load_2d_pair(sB + 8192, tB, n0 + 64, k0, bar);
    } else {
      tma_load_2d_pair(sA, tA1, m0, k0, bar);  // [64 k][64 m] x 2
      tma_load_2d_pair(sA + 8192, tA1, m0 + 64, k0, bar);
      tma_load_2d_pair(sB, tB1, n0, k0, bar);
      tma_load_2d_pair(sB + 8192, tB1, n0 + 64, k0, bar);
    }
  }

  __device__ static void mma_stage(const Params&, int prob, uint32_t d_tmem, uint32_t, uint8_t* sA, uint8_t* sB,
                                   uint8_t*, bool first) {
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
#pragma unroll
    for (int kk = 0; kk < BK / 16; ++kk) {
      const uint64_t ad = prob ? smem_desc(a0 + kk * 2048, 8192, 1024, 2) : smem_desc(a0 + kk * 32, 16, 1024, 2);
      const uint64_t bd = smem_desc(b0 + kk * 2048, 8192, 1024, 2);
      mma_bf16_pair(d_tmem, ad, bd, prob ? IDESC1 : IDESC0, (first && kk == 0) ? 0u : 1u);
    }
  }

  __device__ static void epilogue(const Params& p, int prob, uint32_t t_acc, int row, int n0, int lane, int part,
                                  int parts) {
    Bf16Params q;
    q.M = p.M[prob];
    q.N = p.N;
    q.K = p.K[prob];
    q.alpha = p.alpha[prob];
    q.out = p.out[prob];
    q.ldo = p.N;
    q.status = p.status;
    q.mask = prob ? p.mask1 : nullptr;
    q.mask_m = p.mask_m;
    bf16_epilogue<OUT_F32>(q, t_acc, row, n0, part, parts);
  }
};

// ---------------------------------------------------------------------------
// 2:4 sparse int8 forward on pairs: tile 256 W rows x BN tokens, 256 logical
// k per stage.  Each CTA holds its 128 rows of compressed codes (128 x 128
// bytes), BN/2 tokens of xq (2 boxes of [BN/2 rows][128 bytes]) and its rows'
// metadata (2 blocks of 128 rows x 16 bytes, copied to tensor memory).  A
// stage costs about the same tensor-pipe time from 192 to 240 tokens (the
// sparse MMA has a large fixed cost per instruction), so the tile is 240
// tokens wide, the widest that tensor memory holds twice; it never needs more
// tiles than 224 (the 30-layer training step: 88.1 -> 82.7 ms; the prefill
// step unchanged within 0.2%).  Tensor memory at 240: accumulators at columns
// 0 and 256, the two
// metadata slots in the gap at 240-255 (at 224 tokens: accumulators at 0 and
// 224, metadata after them at 448).
// ---------------------------------------------------------------------------
template <bool ACC_OUT, int BN_ = 240, bool QX = false>
struct CfgPairSparse {
  using Params = FwdParams;
  using Tiles = StripedTiles<CfgPairSparse>;
  static constexpr bool QUANT_X = QX;  // quantise the activations in the same launch
  static constexpr int MAPS = 3;
  static constexpr int EPI_WARPS = 8;  // the fp32 output is the heavy part of this epilogue
  static constexpr int BN = BN_, BK = 256, STAGES = 4;
  static constexpr int A_BYTES = 128 * BK / 2;      // 16 KB
  static constexpr int B_BYTES = (BN / 2) * BK;     // 30 KB at 240 tokens
  static constexpr int E_BYTES = 2 * 2048;          // 4 KB
  static constexpr int ACC_COLS = (BN + 31) / 32 * 32;  // accumulator stride, 32-column aligned
  static constexpr int TMEM_COLS = 512;
  static constexpr int E_COLS = 8;                  // 2 blocks x 4 columns, two slots
  static constexpr int E_COL0 = (ACC_COLS - BN >= 2 * E_COLS) ? BN : 2 * ACC_COLS;
  static constexpr uint32_t IDESC = idesc_i8(256, BN, true);
  static_assert(BN % 16 == 0 && BN <= 256, "2-SM MMA tile width");
  static_assert(ACC_COLS + BN <= TMEM_COLS && E_COL0 + 2 * E_COLS <= TMEM_COLS &&
                    (E_COL0 >= 2 * ACC_COLS || E_COL0 + 2 * E_COLS <= ACC_COLS),
                "tensor memory budget: two accumulators and two metadata slots, disjoint");

  __device__ static int rows_M(const Params& p) { return p.n_out; }
  __device__ static int cols_N(const Params& p) { return p.T; }
  __device__ static int k_blocks(const Params& p) { return (p.K + BK - 1) / BK; }
  __device__ static uint32_t tile_rows(const Params& p, int nb) { return static_cast<uint32_t>(min(BN, p.T - nb * BN)); }

  __device__ static void load_stage(const CUtensorMap* tA, const CUtensorMap* tB, const CUtensorMap* tE,
                                    const CUtensorMap*, const Params& p, int, uint8_t* sA, uint8_t* sB, uint8_t* sE,
                                    int m0, int n0, int kb, uint64_t* bar) {
    tma_load_2d_pair(sA, tA, kb * (BK / 2), m0, bar);              // compressed columns
    tma_load_2d_pair(sB, tB, kb * BK, n0, bar);                    // logical k 0..127 of the stage
    tma_load_2d_pair(sB + (BN / 2) * 128, tB, kb * BK + 128, n0, bar);  // logical k 128..255
    // metadata: 2 consecutive 2 KB blocks = 16 rows of 256 bytes in the section
    const int row = ((m0 / 128) * p.meta_kblocks + kb * 2) * 8;
    tma_load_2d_pair(sE, tE, 0, row, bar);
  }

  __device__ static void mma_stage(const Params&, int, uint32_t d_tmem, uint32_t e_tmem, uint8_t* sA, uint8_t* sB,
                                   uint8_t* sE, bool first) {
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB), e0 = smem_u32(sE);
    tmem_copy_128x128b_pair(e_tmem, smem_desc(e0, 2048, 128, 0));
    tmem_copy_128x128b_pair(e_tmem + 4, smem_desc(e0 + 2048, 2048, 128, 0));
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint64_t ad = smem_desc(a0 + kk * 32, 16, 1024, 2);  // 32 compressed bytes = 64 logical k
      const uint32_t bsub = (kk >> 1) * ((BN / 2) * 128) + (kk & 1) * 64;
      const uint64_t bd = smem_desc(b0 + bsub, 16, 1024, 2);
      mma_sp_i8_pair(d_tmem, ad, bd, e_tmem + 2 * kk, IDESC, (first && kk == 0) ? 0u : 1u);
    }
  }

  __device__ static void epilogue(const Params& p, int, uint32_t t_acc, int row, int n0, int lane, int part,
                                  int parts) {
    const float g = *p.g;
#pragma unroll 1
    for (int c = part; c < BN / 32; c += parts) {
      uint32_t r[32];
      __syncwarp();
      tmem_load_32x32b_x32(t_acc + c * 32, r);
      tmem_load_wait();
      if (n0 + c * 32 >= p.T) continue;  // uniform across the warp
      fwd_epilogue_chunk<ACC_OUT>(p, r, row, n0 + c * 32, lane, g);
    }
    if constexpr (BN % 32 == 16) {  // the last 16 columns
      constexpr int c = BN / 32;
      if (c % parts == part) {
        uint32_t r[16];
        __syncwarp();
        tmem_load_32x32b_x16(t_acc + c * 32, r);
        tmem_load_wait();
        if (n0 + c * 32 < p.T) fwd_epilogue_chunk<ACC_OUT, 16>(p, r, row, n0 + c * 32, lane, g);
      }
    }
  }
};

// ---------------------------------------------------------------------------
// Dense int8 forward on pairs (every N:M pattern other than 2:4): tile 256 W
// rows x BN tokens, 128 k per stage.  Each CTA holds 128 rows of W_eff codes
// (128 x 128 bytes) and BN/2 tokens of xq.
// ---------------------------------------------------------------------------
template <bool ACC_OUT, int BN_, bool QX = false>
struct CfgPairDense {
  using Params = FwdParams;
  using Tiles = StripedTiles<CfgPairDense>;
  static constexpr bool QUANT_X = QX;  // quantise the activations in the same launch
  static constexpr int MAPS = 2;
  static constexpr int EPI_WARPS = 8;
  static constexpr int BN = BN_, BK = 128;
  static constexpr int A_BYTES = 128 * BK;        // 16 KB
  static constexpr int B_BYTES = (BN / 2) * BK;   // 16 KB at BN = 256
  static constexpr int E_BYTES = 0;
  static constexpr int STAGES = (200 * 1024) / (A_BYTES + B_BYTES) < 8 ? (200 * 1024) / (A_BYTES + B_BYTES) : 8;
  static constexpr int ACC_COLS = BN;
  static constexpr int TMEM_COLS = 512;
  static constexpr int E_COL0 = 0, E_COLS = 0;
  static constexpr uint32_t IDESC = idesc_i8(256, BN, false);
  static_assert((BN / 2) % 8 == 0 && 2 * BN <= TMEM_COLS, "tile");

  __device__ static int rows_M(const Params& p) { return p.n_out; }
  __device__ static int cols_N(const Params& p) { return p.T; }
  __device__ static int k_blocks(const Params& p) { return (p.K + BK - 1) / BK; }
  __device__ static uint32_t tile_rows(const Params& p, int nb) { return static_cast<uint32_t>(min(BN, p.T - nb * BN)); }

  __device__ static void load_stage(const CUtensorMap* tA, const CUtensorMap* tB, const CUtensorMap*,
                                    const CUtensorMap*, const Params&, int, uint8_t* sA, uint8_t* sB, uint8_t*, int m0,
                                    int n0, int kb, uint64_t* bar) {
    tma_load_2d_pair(sA, tA, kb * BK, m0, bar);  // [128 rows][128 bytes]
    tma_load_2d_pair(sB, tB, kb * BK, n0, bar);  // [BN/2 rows][128 bytes]
  }

  __device__ static void mma_stage(const Params&, int, uint32_t d_tmem, uint32_t, uint8_t* sA, uint8_t* sB, uint8_t*,
                                   bool first) {
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
#pragma unroll
    for (int kk = 0; kk < BK / 32; ++kk) {
      mma_i8_pair(d_tmem, smem_desc(a0 + kk * 32, 16, 1024, 2), smem_desc(b0 + kk * 32, 16, 1024, 2), IDESC,
                  (first && kk == 0) ? 0u : 1u);
    }
  }

  __device__ static void epilogue(const Params& p, int, uint32_t t_acc, int row, int n0, int lane, int part,
                                  int parts) {
    const float g = *p.g;
#pragma unroll 1
    for (int c = part; c < BN / 32; c += parts) {
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
