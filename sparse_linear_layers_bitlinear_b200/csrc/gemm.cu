// Launchers for the tensor-core GEMMs (forward int8, dense or 2:4 sparse;
// backward bf16), the tensor-map encoder and the bounded-wait self test.
#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "gemm_pair.cuh"
#include "sbl_kernels.h"

namespace sbl {

// ---------------------------------------------------------------------------
// Tensor maps
// ---------------------------------------------------------------------------
using PFN_encodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                     const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                     CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static PFN_encodeTiled get_encoder() {
  static PFN_encodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled>(p);
  });
  return fn;
}

bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  PFN_encodeTiled enc = get_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Pair kernels: grid = two CTAs per concurrently resident cluster, capped by
// the tile count.
template <class Cfg>
static cudaError_t pair_setup(int num_sms, int* max_clusters_out) {
  constexpr int smem = pair_smem_bytes<Cfg>();
  static_assert(smem <= 227 * 1024, "shared memory budget");
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  static int max_clusters = 0;
  std::call_once(once, [num_sms] {
    attr_err = cudaFuncSetAttribute(k_gemm_pair<Cfg>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (attr_err != cudaSuccess) return;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(num_sms & ~1);
    cfg.blockDim = dim3(pair_threads<Cfg>());
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    attr_err = cudaOccupancyMaxActiveClusters(&n, k_gemm_pair<Cfg>, &cfg);
    max_clusters = n;
  });
  if (attr_err != cudaSuccess) return attr_err;
  if (max_clusters <= 0) return cudaErrorInvalidConfiguration;
  *max_clusters_out = max_clusters;
  return cudaSuccess;
}

// pdl: launch with programmatic stream serialisation (the kernel's producer
// waits for the predecessor before its first load).
template <class Cfg>
static cudaError_t launch_pair(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& e,
                               const typename Cfg::Params& p, int m_rows, int n_cols, int num_sms, cudaStream_t s,
                               bool pdl = false) {
  int max_clusters = 0;
  const cudaError_t err = pair_setup<Cfg>(num_sms, &max_clusters);
  if (err != cudaSuccess) return err;
  const int tiles = ((m_rows + 255) / 256) * ((n_cols + Cfg::BN - 1) / Cfg::BN);
  const int pairs = tiles < max_clusters ? tiles : max_clusters;
  if (pairs <= 0) return cudaSuccess;
  if (pdl)
    return launch_pdl(k_gemm_pair<Cfg>, dim3(2 * pairs), dim3(pair_threads<Cfg>()), pair_smem_bytes<Cfg>(), s, a, b,
                      e, e, p);
  k_gemm_pair<Cfg><<<2 * pairs, pair_threads<Cfg>(), pair_smem_bytes<Cfg>(), s>>>(a, b, e, e, p);
  return counted(cudaGetLastError());
}

// ---------------------------------------------------------------------------
// Forward int8 GEMM
// ---------------------------------------------------------------------------
// The forward configuration for (accumulators out, tile width, in-launch
// quantisation), launched by programmatic dependent launch.
template <template <bool, int, bool> class Cfg, int BN>
static cudaError_t launch_fwd(bool acc, bool qx, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& te,
                              const FwdParams& p, int num_sms, cudaStream_t s) {
  if (qx)
    return acc ? launch_pair<Cfg<true, BN, true>>(ta, tb, te, p, p.n_out, p.T, num_sms, s, true)
               : launch_pair<Cfg<false, BN, true>>(ta, tb, te, p, p.n_out, p.T, num_sms, s, true);
  return acc ? launch_pair<Cfg<true, BN, false>>(ta, tb, te, p, p.n_out, p.T, num_sms, s, true)
             : launch_pair<Cfg<false, BN, false>>(ta, tb, te, p, p.n_out, p.T, num_sms, s, true);
}

cudaError_t launch_forward_gemm(bool sparse, const int8_t* codes, const uint8_t* meta, int meta_kblocks,
                                uint64_t meta_bytes, const int8_t* xq, const float* a_prime, const float* g,
                                int64_t n_out, int64_t t, int64_t k, float* y, int32_t* acc_out, uint32_t* status,
                                int num_sms, cudaStream_t s, const uint16_t* x_quantise, uint32_t* ready) {
  FwdParams p;
  p.n_out = static_cast<int>(n_out);
  p.T = static_cast<int>(t);
  p.K = static_cast<int>(k);
  p.g = g;
  p.a_prime = a_prime;
  p.y = y;
  p.acc_out = acc_out;
  p.meta = meta;
  p.meta_kblocks = meta_kblocks;
  p.status = status;
  // In-launch quantisation: the codes and a' go to xq / a_prime, counted per
  // token tile on `ready` (zeroed here, ahead of the launch).
  const bool qx = x_quantise != nullptr;
  p.x = reinterpret_cast<const uint4*>(x_quantise);
  p.xq = const_cast<int8_t*>(xq);
  p.ap_out = const_cast<float*>(a_prime);
  p.ready = ready;
  if (qx) {
    if (k > int64_t(kQxMaxRW) * 256 || ready == nullptr) return cudaErrorInvalidValue;
    const cudaError_t e = cudaMemsetAsync(ready, 0, size_t(forward_tile_counters(t)) * 4, s);
    if (e != cudaSuccess) return e;
  }
  CUtensorMap ta, tb, te;
  const bool acc = acc_out != nullptr;
  if (sparse) {
    // A: compressed codes [n_out][k/2]; B: xq [t][k], 120-token halves; E:
    // the metadata section viewed as rows of 256 bytes.
    if (!encode_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, k / 2, n_out, k / 2, 128, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, k, t, k, 128, CfgPairSparse<false>::BN / 2,
                        CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tmap_2d(&te, CU_TENSOR_MAP_DATA_TYPE_UINT8, meta, 256, meta_bytes / 256, 256, 256, 16,
                        CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
    return launch_fwd<CfgPairSparse, 240>(acc, qx, ta, tb, te, p, num_sms, s);
  }
  // Dense int8 over W_eff codes.  Tile width: 192 tokens when that takes no
  // more rounds of pair tiles than 256, else 256.  A round of 192-token tiles
  // costs 0.91-0.98 of a round of 256-token ones (the mainloop also pays for
  // re-reading W once per token block), so the count of rounds decides.
  int max_clusters = 0;
  cudaError_t err = pair_setup<CfgPairDense<false, 256>>(num_sms, &max_clusters);
  if (err != cudaSuccess) return err;
  auto rounds = [&](int bn) {
    const int tiles = ((p.n_out + 255) / 256) * ((p.T + bn - 1) / bn);
    return (tiles + max_clusters - 1) / max_clusters;
  };
  const bool narrow = rounds(192) <= rounds(256);
  const int bn = narrow ? 192 : 256;
  if (!encode_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, k, n_out, k, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, k, t, k, 128, bn / 2, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (narrow) return launch_fwd<CfgPairDense, 192>(acc, qx, ta, tb, tb, p, num_sms, s);
  return launch_fwd<CfgPairDense, 256>(acc, qx, ta, tb, tb, p, num_sms, s);
}

// Token-tile counters the in-launch quantisation needs: one per 16 tokens
// covers every tile width (192, 240, 256).
int64_t forward_tile_counters(int64_t t) { return (t + 15) / 16; }

// ---------------------------------------------------------------------------
// Backward bf16 GEMM
// ---------------------------------------------------------------------------
template <bool A_MN, bool B_MN, bool F32>
static cudaError_t bf16_dispatch(const uint16_t* A, const uint16_t* B, int64_t M, int64_t N, int64_t K,
                                 const float* alpha, void* out, uint32_t* status, int num_sms, cudaStream_t s,
                                 const uint8_t* mask, int mask_m) {
  using Cfg = CfgPairBf16<A_MN, B_MN, F32>;
  CUtensorMap ta, tb;
  const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  // Per CTA: A 128 rows, B 128 columns (half of the pair's 256).
  const bool ok_a = A_MN ? encode_tmap_2d(&ta, bf, A, M, K, M * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B)
                         : encode_tmap_2d(&ta, bf, A, K, M, K * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  const bool ok_b = B_MN ? encode_tmap_2d(&tb, bf, B, N, K, N * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B)
                         : encode_tmap_2d(&tb, bf, B, K, N, K * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok_a || !ok_b) return cudaErrorInvalidValue;
  Bf16Params p;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.alpha = alpha;
  p.out = out;
  p.ldo = N;
  p.status = status;
  p.mask = mask;
  p.mask_m = mask_m;
  return launch_pair<Cfg>(ta, tb, tb, p, p.M, p.N, num_sms, s, true);  // producer waits before its first load
}

cudaError_t launch_bf16_gemm(bool a_mn, bool b_mn, bool out_f32, const uint16_t* A, const uint16_t* B, int64_t M,
                             int64_t N, int64_t K, const float* alpha, void* out, uint32_t* status, int num_sms,
                             cudaStream_t s, const uint8_t* mask, int mask_m) {
  const int sel = (a_mn ? 4 : 0) | (b_mn ? 2 : 0) | (out_f32 ? 1 : 0);
  switch (sel) {
    case 0: return bf16_dispatch<false, false, false>(A, B, M, N, K, alpha, out, status, num_sms, s, mask, mask_m);
    case 1: return bf16_dispatch<false, false, true>(A, B, M, N, K, alpha, out, status, num_sms, s, mask, mask_m);
    case 2: return bf16_dispatch<false, true, false>(A, B, M, N, K, alpha, out, status, num_sms, s, mask, mask_m);
    case 3: return bf16_dispatch<false, true, true>(A, B, M, N, K, alpha, out, status, num_sms, s, mask, mask_m);
    case 4: return bf16_dispatch<true, false, false>(A, B, M, N, K, alpha, out, status, num_sms, s, mask, mask_m);
    case 5: return bf16_dispatch<true, false, true>(A, B, M, N, K, alpha, out, status, num_sms, s, mask, mask_m);
    case 6: return bf16_dispatch<true, true, false>(A, B, M, N, K, alpha, out, status, num_sms, s, mask, mask_m);
    default: return bf16_dispatch<true, true, true>(A, B, M, N, K, alpha, out, status, num_sms, s, mask, mask_m);
  }
}

// ---------------------------------------------------------------------------
// dX and dW in one launch
// ---------------------------------------------------------------------------
namespace {

struct DualSchedule {
  std::vector<uint16_t> off, ids;
};

// Longest-processing-time-first: tiles by depth (k blocks), deepest first,
// each to the pair with the least work so far.  Cached per shape.
const DualSchedule& dual_schedule(int tiles0, int kb0, int tiles1, int kb1, int npairs) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, int, int, int>, DualSchedule> cache;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_tuple(tiles0, kb0, tiles1, kb1, npairs);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  std::vector<int> order;
  order.reserve(tiles0 + tiles1);
  const bool first0 = kb0 >= kb1;
  for (int pass = 0; pass < 2; ++pass) {
    const bool prob0 = (pass == 0) == first0;
    const int base = prob0 ? 0 : tiles0, n = prob0 ? tiles0 : tiles1;
    for (int i = 0; i < n; ++i) order.push_back(base + i);
  }
  std::vector<std::vector<uint16_t>> per(npairs);
  std::vector<long long> load(npairs, 0);
  for (int id : order) {
    const int cost = id < tiles0 ? kb0 : kb1;
    int best = 0;
    for (int q = 1; q < npairs; ++q)
      if (load[q] < load[best]) best = q;
    per[best].push_back(static_cast<uint16_t>(id));
    load[best] += cost;
  }
  DualSchedule sch;
  sch.off.push_back(0);
  for (int q = 0; q < npairs; ++q) {
    sch.ids.insert(sch.ids.end(), per[q].begin(), per[q].end());
    sch.off.push_back(static_cast<uint16_t>(sch.ids.size()));
  }
  return cache.emplace(key, std::move(sch)).first->second;
}

template <bool F32>
cudaError_t dual_dispatch(const uint16_t* dy, const uint16_t* weff, const uint16_t* x, int64_t t, int64_t n_out,
                          int64_t k, const float* g, void* dx, void* dw, const uint8_t* dw_mask, int mask_m,
                          uint32_t* status, int num_sms, cudaStream_t s, bool* done) {
  using Cfg = CfgPairDualBf16<F32>;
  *done = false;
  int max_clusters = 0;
  cudaError_t err = pair_setup<Cfg>(num_sms, &max_clusters);
  if (err != cudaSuccess) return err;
  const int nb = static_cast<int>((k + 255) / 256);
  const int mb0 = static_cast<int>((t + 255) / 256), mb1 = static_cast<int>((n_out + 255) / 256);
  const int tiles0 = mb0 * nb, tiles1 = mb1 * nb;
  if (tiles0 + tiles1 > kDualMaxTiles) return cudaSuccess;  // caller runs two launches
  int npairs = std::min(std::min(max_clusters, kDualMaxPairs), tiles0 + tiles1);
  const int kb0 = static_cast<int>((n_out + 63) / 64), kb1 = static_cast<int>((t + 63) / 64);
  const DualSchedule& sch = dual_schedule(tiles0, kb0, tiles1, kb1, npairs);

  CUtensorMap a0, b0, a1, b1;
  const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  // dX: A0 = dY [t][n_out] K-major, B0 = W_eff [n_out][k] MN-major
  // dW: A1 = dY [t][n_out] MN-major (M = n_out), B1 = X [t][k] MN-major
  if (!encode_tmap_2d(&a0, bf, dy, n_out, t, n_out * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&b0, bf, weff, k, n_out, k * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&a1, bf, dy, n_out, t, n_out * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&b1, bf, x, k, t, k * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  DualBf16Params p;
  p.M[0] = static_cast<int>(t);
  p.M[1] = static_cast<int>(n_out);
  p.N = static_cast<int>(k);
  p.K[0] = static_cast<int>(n_out);
  p.K[1] = static_cast<int>(t);
  p.mblocks[0] = mb0;
  p.mblocks[1] = mb1;
  p.tiles0 = tiles0;
  p.alpha[0] = g;
  p.alpha[1] = nullptr;
  p.out[0] = dx;
  p.out[1] = dw;
  p.status = status;
  p.mask1 = dw_mask;
  p.mask_m = mask_m;
  std::copy(sch.off.begin(), sch.off.end(), p.sched_off);
  std::copy(sch.ids.begin(), sch.ids.end(), p.sched);
  // Programmatic dependent launch: the CTAs set up (barriers, tensor memory)
  // as SMs free up under the kernel before; the producer waits for that
  // kernel before its first load, and every output write follows the loads.
  err = launch_pdl(k_gemm_pair<Cfg>, dim3(2 * npairs), dim3(pair_threads<Cfg>()), pair_smem_bytes<Cfg>(), s, a0, b0,
                   a1, b1, p);
  *done = err == cudaSuccess;
  return err;
}

}  // namespace

cudaError_t launch_bf16_backward_dual(bool out_f32, const uint16_t* dy, const uint16_t* weff, const uint16_t* x,
                                      int64_t t, int64_t n_out, int64_t k, const float* g, void* dx, void* dw,
                                      const uint8_t* dw_mask, int mask_m, uint32_t* status, int num_sms,
                                      cudaStream_t s, bool* done) {
  return out_f32 ? dual_dispatch<true>(dy, weff, x, t, n_out, k, g, dx, dw, dw_mask, mask_m, status, num_sms, s, done)
                 : dual_dispatch<false>(dy, weff, x, t, n_out, k, g, dx, dw, dw_mask, mask_m, status, num_sms, s, done);
}

// ---------------------------------------------------------------------------
// Tensor-pipe rate with resident operands.  One CTA pair issues a GEMM
// configuration's per-stage instructions (the MMAs, and for 2:4 the copy of
// the stage's metadata into tensor memory) back to back over its shared-
// memory stages, which are filled once: ternary codes for the weights, int8
// activations, valid 2:4 metadata (kept positions 0 and 1), finite bf16
// values for the backward.  No copies, waits or epilogues come in between,
// so the launch time over `pairs` pairs gives the rate those instructions
// reach on their own: the ceiling of the GEMM that issues them.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t rate_hash(uint32_t x) {
  x ^= x >> 16;
  x *= 0x7FEB352Du;
  x ^= x >> 15;
  x *= 0x846CA68Bu;
  x ^= x >> 16;
  return x;
}

template <class Cfg, bool INT8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(128, 1) k_mma_rate(int stages, uint32_t* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* smA = smem;
  uint8_t* smB = smA + Cfg::STAGES * Cfg::A_BYTES;
  uint8_t* smE = smB + Cfg::STAGES * Cfg::B_BYTES;
  PairSmemTail* tail = reinterpret_cast<PairSmemTail*>(smE + Cfg::STAGES * Cfg::E_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool leader = cluster_rank() == 0;

  constexpr int nA = Cfg::STAGES * Cfg::A_BYTES / 4, nB = Cfg::STAGES * Cfg::B_BYTES / 4;
  constexpr int nE = Cfg::STAGES * Cfg::E_BYTES / 4;
  uint32_t* words = reinterpret_cast<uint32_t*>(smem);
  for (int i = threadIdx.x; i < nA + nB + nE; i += blockDim.x) {
    const uint32_t h = rate_hash(static_cast<uint32_t>(i) * 2654435761u + blockIdx.x);
    uint32_t v;
    if (i >= nA + nB) {
      v = 0x44444444u;  // metadata nibbles i0 = 0, i1 = 1
    } else if (!INT8) {
      v = (h & 0x807F807Fu) | 0x3C003C00u;  // two bf16 of magnitude in [2^-7, 2^-6)
    } else if (i < nA) {
      // four ternary codes: byte value h_b mod 3 -> 0, +1, -1
      v = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const uint32_t r = ((h >> (8 * b)) & 0xFFu) % 3u;
        v |= (r == 0u ? 0u : (r == 1u ? 0x01u : 0xFFu)) << (8 * b);
      }
    } else {
      v = h;  // int8 activation codes
    }
    words[i] = v;
  }
  if (threadIdx.x == 0) {
    mbar_init(&tail->drain, 1);
    fence_mbar_init();
  }
  fence_proxy_async_smem();  // the operands written above are read by the tensor pipe
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) tmem_alloc_pair(&tail->tmem_base, Cfg::TMEM_COLS);
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = tail->tmem_base;

  if (warp == 1 && leader && lane == 0) {
    typename Cfg::Params p{};
    for (int i = 0; i < stages; ++i) {
      const uint32_t s = static_cast<uint32_t>(i % Cfg::STAGES);
      Cfg::mma_stage(p, 0, tmem_base, tmem_base + Cfg::E_COL0 + (s & 1u) * Cfg::E_COLS, smA + s * Cfg::A_BYTES,
                     smB + s * Cfg::B_BYTES, smE + s * Cfg::E_BYTES, i == 0);
    }
    mma_commit_pair(&tail->drain);
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(&tail->drain, 0)) {
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        raise_status(status, SBL_STATUS_TIMEOUT);
        break;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the leader's MMAs no longer read the partner's operands
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
  }
}

template <class Cfg, bool INT8>
static cudaError_t mma_rate_launch(int stages, int pairs, uint32_t* status, cudaStream_t s) {
  constexpr int smem = pair_smem_bytes<Cfg>();
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(k_mma_rate<Cfg, INT8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  });
  if (attr_err != cudaSuccess) return attr_err;
  k_mma_rate<Cfg, INT8><<<2 * pairs, 128, smem, s>>>(stages, status);
  return counted(cudaGetLastError());
}

int64_t mma_rate_macs_per_stage(int kind) {
  switch (kind) {
    case 0: return int64_t(256) * CfgPairSparse<false>::BN * CfgPairSparse<false>::BK;  // logical k
    case 1: return int64_t(256) * CfgPairDense<false, 256>::BN * CfgPairDense<false, 256>::BK;
    case 2: return int64_t(256) * CfgPairDualBf16<false>::BN * CfgPairDualBf16<false>::BK;
    default: return 0;
  }
}

cudaError_t launch_mma_rate(int kind, int stages, int pairs, uint32_t* status, cudaStream_t s) {
  switch (kind) {
    case 0: return mma_rate_launch<CfgPairSparse<false>, true>(stages, pairs, status, s);
    case 1: return mma_rate_launch<CfgPairDense<false, 256>, true>(stages, pairs, status, s);
    case 2: return mma_rate_launch<CfgPairDualBf16<false>, false>(stages, pairs, status, s);
    default: return cudaErrorInvalidValue;
  }
}

// ---------------------------------------------------------------------------
// Bounded-wait self test: waits on an mbarrier that nothing arrives on.
// ---------------------------------------------------------------------------
__global__ void k_selftest_wait(uint32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = globaltimer_ns();
    bool done = false;
    while (!(done = mbar_try_wait(&bar, 0))) {
      if (globaltimer_ns() - t0 > limit_ns) break;
    }
    if (!done) atomicOr(status, SBL_STATUS_TIMEOUT);
  }
}

cudaError_t launch_selftest_wait(uint32_t* status, uint64_t limit_ns, cudaStream_t s) {
  k_selftest_wait<<<1, 32, 0, s>>>(status, limit_ns);
  return counted(cudaGetLastError());
}

// ---------------------------------------------------------------------------
// The floor of a chain of dependent launches: a kernel that lets its
// successor launch, waits for its predecessor and exits, launched the way
// every kernel of the library is (programmatic dependent launch).
// ---------------------------------------------------------------------------
__global__ void k_chain_floor() {
  pdl_trigger();
  pdl_wait();
}

cudaError_t launch_chain_floor(int blocks, cudaStream_t s) {
  return launch_pdl(k_chain_floor, dim3(blocks), dim3(256), 0, s);
}

}  // namespace sbl
