// Weight preparation for Sparse-BitLinear: exact absmean scale, N:M mask from
// the master magnitudes, ternary codes with the mask applied after
// quantisation, and the packed forms the GEMM kernels read.
//
// Paper: "Sparse-BitNet: 1.58-bit LLMs are Naturally Friendly to
// Semi-Structured Sparsity" -- gist.science German technical summary §2
// (magnitude mask from the masters, quantise then mask), Korean summary
// §2.1-2.2 (per-step recompute), French summary §2.
//
// Three kernels:
//   k_absmean_partials  streams W once, adds every |w| exactly into per-block
//                       integer bins
//   k_gamma_finalize    one block: folds the bins, rounds the exact mean once to
//                       fp32, writes gamma, g and the header
//   k_prep_pack<M>      re-reads W (from L2), masks, ternarises and writes every
//                       packed section
// The last two are launched with programmatic stream serialisation, so their
// launches overlap the tail of the kernel before them.
#include "sbl_kernels.h"

#include "sbl_device.cuh"

namespace sbl {

// ---------------------------------------------------------------------------
// Exact sum of |w| (absmean numerator).
//
// In units of 2^-133 a bf16 magnitude (biased exponent e, mantissa f) is the
// integer sig << s with sig = (e ? 128 + f : f) and s = max(e, 1) - 1 <= 253,
// i.e. sig - s * 128 = mag - s * 128 with mag = e * 128 + f.  Each lane keeps
// 32 private 32-bit bins in shared memory, bin b = s >> 3 collecting
// sig << (s & 7) (< 2^15 per add).  A round lets each lane add at most 2^16
// weights, so no bin overflows; after each round the block folds its lanes'
// bins into 64-bit totals.  A slot bin b is an integer in units of 2^(8b-133).
// ---------------------------------------------------------------------------
constexpr int kAbsThreads = 1024;
constexpr int kAbsWarps = kAbsThreads / 32;
constexpr int kLaneBins = 32;
constexpr int64_t kRoundVecs = 8192;  // 16-byte vectors per thread per round (8 weights each)

__global__ void __launch_bounds__(kAbsThreads, 1)
    k_absmean_partials(const uint4* __restrict__ w, int64_t nvec, uint64_t* __restrict__ slot_bins,
                       uint32_t* __restrict__ slot_flags) {
  extern __shared__ uint32_t lane_bins[];  // [warp][bin][lane]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t* my = lane_bins + warp * (kLaneBins * 32) + lane;

  uint32_t emax = 0;
  auto consume = [&](const uint4 v) {
    const uint32_t words[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t mag = (words[j >> 1] >> (16 * (j & 1))) & 0x7FFFu;
      const uint32_t e = mag >> 7;
      emax = max(emax, e);
      const uint32_t s = max(e, 1u) - 1u;
      const uint32_t sig = mag - (s << 7);
      my[(s >> 3) * 32] += sig << (s & 7u);
    }
  };

  const int64_t stride = int64_t(gridDim.x) * kAbsThreads;
  const int64_t round = stride * kRoundVecs;
  uint64_t total = 0;  // thread (bin = warp, part = lane) keeps the block total of its bin
  for (int64_t r0 = 0; r0 < nvec; r0 += round) {
#pragma unroll
    for (int b = 0; b < kLaneBins; ++b) my[b * 32] = 0u;
    const int64_t r1 = (nvec - r0 < round) ? nvec : r0 + round;
    int64_t i = r0 + int64_t(blockIdx.x) * kAbsThreads + threadIdx.x;
    // Four independent 16-byte loads in flight per thread (default caching:
    // the pack kernel re-reads W right after this one).
    for (; i + 3 * stride < r1; i += 4 * stride) {
      const uint4 v0 = __ldg(w + i);
      const uint4 v1 = __ldg(w + i + stride);
      const uint4 v2 = __ldg(w + i + 2 * stride);
      const uint4 v3 = __ldg(w + i + 3 * stride);
      consume(v0);
      consume(v1);
      consume(v2);
      consume(v3);
    }
    for (; i < r1; i += stride) consume(__ldg(w + i));
    __syncthreads();
    // Warp `bin` folds bin `bin`: lane p sums the 32 lanes of warp p.
    {
      const int bin = warp, part = lane;
      const uint32_t* src = lane_bins + part * (kLaneBins * 32) + bin * 32;
      uint64_t sum = 0;
#pragma unroll 8
      for (int l = 0; l < 32; ++l) sum += src[(l + lane) & 31];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      total += sum;
    }
    __syncthreads();
  }
  if (lane == 0) slot_bins[int64_t(blockIdx.x) * kExactBins + warp] = total;
  if (threadIdx.x < kExactBins - kLaneBins) slot_bins[int64_t(blockIdx.x) * kExactBins + kLaneBins + threadIdx.x] = 0ull;
  const int bad = __syncthreads_or(emax == 0xFFu);
  if (threadIdx.x == 0) slot_flags[blockIdx.x] = bad ? SBL_STATUS_NONFINITE_W : 0u;
  pdl_trigger();
}

// ---------------------------------------------------------------------------
// gamma = RN_fp32(S * 2^-133 / numel) with S = sum_b bins[b] << 8b exactly.
// S (< 2^310) is assembled in six 64-bit limbs, normalised to a 128-bit
// integer N with its top bit at 127 (bits shifted out only feed the sticky
// bit), one 128/64 division gives a quotient of at least 86 bits, and that
// quotient is rounded to nearest-even at the fp32 precision (24 bits, or the
// 2^-149 step for subnormal results).  Straight-line code on registers.
// ---------------------------------------------------------------------------
constexpr int kLimbs = 6;

__device__ float exact_mean_fp32(const uint64_t* bins, uint64_t numel) {
  unsigned __int128 T[kLimbs];
#pragma unroll
  for (int L = 0; L < kLimbs; ++L) T[L] = 0;
#pragma unroll
  for (int b = 0; b < kExactBins; ++b) {
    const uint64_t v = bins[b];  // < 2^60
    const int sh = 8 * b, L = sh >> 6, off = sh & 63;
    T[L] += static_cast<unsigned __int128>(v << off);
    if (off != 0 && L + 1 < kLimbs) T[L + 1] += static_cast<unsigned __int128>(v >> (64 - off));
  }
  uint64_t S[kLimbs];
#pragma unroll
  for (int L = 0; L < kLimbs; ++L) {
    S[L] = static_cast<uint64_t>(T[L]);
    if (L + 1 < kLimbs) T[L + 1] += T[L] >> 64;
  }
  int topS = -1;
#pragma unroll
  for (int L = kLimbs - 1; L >= 0; --L)
    if (topS < 0 && S[L] != 0ull) topS = 64 * L + 63 - __clzll(static_cast<long long>(S[L]));
  if (topS < 0) return 0.0f;
  // the 64 bits of S starting at bit pos (pos may be negative: zeros below bit 0)
  auto get64 = [&](int pos) -> uint64_t {
    uint64_t r = 0;
#pragma unroll
    for (int L = 0; L < kLimbs; ++L) {
      const int d = 64 * L - pos;
      if (d >= 0 && d < 64) r |= S[L] << d;
      else if (d < 0 && d > -64) r |= S[L] >> (-d);
    }
    return r;
  };
  const int low = topS - 127;  // bit of S that lands at bit 0 of N
  const unsigned __int128 N = (static_cast<unsigned __int128>(get64(low + 64)) << 64) | get64(low);
  bool sticky0 = false;
#pragma unroll
  for (int L = 0; L < kLimbs; ++L) {
    const int lim = low - 64 * L;  // bits of limb L below `low`
    if (lim >= 64) sticky0 |= S[L] != 0ull;
    else if (lim > 0) sticky0 |= (S[L] & ((1ull << lim) - 1ull)) != 0ull;
  }
  const unsigned __int128 q = N / numel;
  const bool rem_nz = (N % numel) != 0;
  // bit j of q has weight 2^(j + topS - 260); q >= 2^86
  const uint64_t q_hi = static_cast<uint64_t>(q >> 64), q_lo = static_cast<uint64_t>(q);
  const int topq = q_hi ? 127 - __clzll(static_cast<long long>(q_hi)) : 63 - __clzll(static_cast<long long>(q_lo));
  const int E = topq + topS - 260;
  const int lsb = (E - 23 > -149) ? E - 23 : -149;
  const int sh = lsb - (topS - 260);  // bit of q that becomes the last mantissa bit; 63 <= sh <= 111
  uint64_t mant = static_cast<uint64_t>(q >> sh);
  const int rpos = sh - 1;
  const uint32_t round_bit = static_cast<uint32_t>((q >> rpos) & 1u);
  const bool below = (q & ((static_cast<unsigned __int128>(1) << rpos) - 1u)) != 0;
  const bool sticky = sticky0 || rem_nz || below;
  if (round_bit && (sticky || (mant & 1ull))) ++mant;
  // value = mant * 2^lsb: the pattern covers subnormals and the rounding carry.
  return __uint_as_float((static_cast<uint32_t>(lsb + 149) << 23) + static_cast<uint32_t>(mant));
}

// ---------------------------------------------------------------------------
// Fold the per-block partial sums, compute gamma and g, write the header.
// One block.  It lets the pack kernel start launching right away (that kernel
// waits for this one to complete before it reads g), then waits for the
// partial sums.
// ---------------------------------------------------------------------------
constexpr int kFinGroups = 25;                       // slot groups
constexpr int kFinThreads = kFinGroups * kExactBins;  // 1000 threads: (group, bin) pairs

__global__ void __launch_bounds__(1024) k_gamma_finalize(const uint64_t* slot_bins, const uint32_t* slot_flags,
                                                         int nslots, BlobHeader* h, int64_t n_out, int64_t k, int n,
                                                         int m, uint32_t layer_flags) {
  __shared__ uint64_t s_part[kFinGroups][kExactBins];
  __shared__ uint64_t s_bins[kExactBins];
  __shared__ uint32_t s_flags;
  pdl_trigger();
  pdl_wait();
  const int tid = threadIdx.x;
  if (tid == 0) s_flags = 0u;
  if (tid < kFinThreads) {
    // Group grp folds slots grp, grp + 25, ...: all its loads are issued before
    // any add, so the fold costs one memory round trip.
    const int bin = tid % kExactBins, grp = tid / kExactBins;
    const int per = (nslots - grp + kFinGroups - 1) / kFinGroups;  // slots of this group
    uint64_t v[8];
    uint64_t a = 0;
    for (int j0 = 0; j0 < per; j0 += 8) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int slot = grp + (j0 + j) * kFinGroups;
        v[j] = (j0 + j < per) ? __ldcg(slot_bins + int64_t(slot) * kExactBins + bin) : 0ull;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) a += v[j];
    }
    s_part[grp][bin] = a;
  }
  __syncthreads();
  uint32_t f = 0;
  for (int i = tid; i < nslots; i += blockDim.x) f |= __ldcg(slot_flags + i);
  if (f) atomicOr(&s_flags, f);
  if (tid < kExactBins) {
    uint64_t t = 0;
#pragma unroll 5
    for (int g2 = 0; g2 < kFinGroups; ++g2) t += s_part[g2][tid];
    s_bins[tid] = t;
  }
  __syncthreads();
  if (tid == 0) {
    const uint32_t flags = s_flags;
    const bool bad = (flags & SBL_STATUS_NONFINITE_W) != 0u;
    const float gamma = bad ? __int_as_float(0x7fc00000) : exact_mean_fp32(s_bins, uint64_t(n_out) * uint64_t(k));
    h->magic = kMagic;
    h->version = 2;
    h->n_out = n_out;
    h->k = k;
    h->n = n;
    h->m = m;
    h->flags = layer_flags;
    h->gamma = gamma;
    h->g = (gamma > 1e-5f) ? gamma : 1e-5f;  // a NaN gamma gives 1e-5; the status word says why
    h->status = flags;                        // a new prepare resets the status word
  }
}

// ---------------------------------------------------------------------------
// Mask, ternarise, pack.  Lane = 8 consecutive weights of a row (one 16-byte
// vector); a warp covers 256 consecutive weights, so every load and most
// stores are contiguous across the warp.  k is a multiple of 64, so a row has
// a multiple of 8 lanes' worth of weights and no group or quad of lanes
// straddles two rows.
//
// Bit tricks (all exact):
//  * code != 0  <=>  2|w| > g  <=>  |w| > g/2 (g/2 is exact)  <=>  the 15-bit
//    magnitude field exceeds bits(g/2) >> 16, compared two at a time with
//    __vcmpgtu2 on the packed bf16 pairs;
//  * W_eff as bf16 is (sign | 0x3F80) masked by (kept & code != 0);
//  * the int8 code byte of a bf16 W_eff value h is (h bit 13) | 0xFE * (h bit 15).
// ---------------------------------------------------------------------------
constexpr int kPackThreads = 256;
constexpr int kPackDepth = 8;  // 16-byte loads in flight per lane

// (i0 | i1 << 2) for each 4-bit kept pattern with exactly two bits set.
constexpr uint64_t kPairNibble = (uint64_t(0x4) << (4 * 0x3)) | (uint64_t(0x8) << (4 * 0x5)) |
                                 (uint64_t(0x9) << (4 * 0x6)) | (uint64_t(0xC) << (4 * 0x9)) |
                                 (uint64_t(0xD) << (4 * 0xA)) | (uint64_t(0xE) << (4 * 0xC));

// Keep-bits of one group of M magnitudes: position a is kept when fewer than
// n positions beat it, where b beats a if |w_b| > |w_a|, or if they are equal
// and b < a.  For b < a that is |w_b| >= |w_a|.
template <int M>
__device__ __forceinline__ uint32_t keep_bits(const uint32_t (&mag)[8], int base, int n) {
  int rank[M];
#pragma unroll
  for (int a = 0; a < M; ++a) rank[a] = 0;
#pragma unroll
  for (int i = 0; i < M; ++i)
#pragma unroll
    for (int j = i + 1; j < M; ++j) {
      const int i_wins = mag[base + i] >= mag[base + j] ? 1 : 0;  // i < j: ties go to i
      rank[j] += i_wins;
      rank[i] += 1 - i_wins;
    }
  uint32_t kept = 0;
#pragma unroll
  for (int a = 0; a < M; ++a) kept |= (rank[a] < n ? 1u : 0u) << a;
  return kept;
}

// Packed bf16 compares: 0xFFFF in each half where a > b (a >= b).  Inputs here
// are magnitudes (sign bits cleared), so the float order is the order of the
// 15-bit magnitude fields.
__device__ __forceinline__ uint32_t bf16x2_gt_mask(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("set.gt.u32.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t bf16x2_ge_mask(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("set.ge.u32.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// The six outcomes c_ij = |w_i| >= |w_j| (i < j) of a group of four held as
// two words of magnitudes (m0 | m1 << 16, m2 | m3 << 16), in the table-index
// bit order c01, c02, c03, c12, c13, c23.
__device__ __forceinline__ uint32_t pair_outcomes4_packed(uint32_t m01, uint32_t m23) {
  const uint32_t rA = bf16x2_ge_mask(__byte_perm(m01, m23, 0x5410), __byte_perm(m01, m23, 0x7632));  // c01 | c23
  const uint32_t rB = bf16x2_ge_mask(m01, m23);                                                       // c02 | c13
  const uint32_t rC = bf16x2_ge_mask(m01, __byte_perm(m23, m23, 0x1032));                             // c03 | c12
  return (rA & 1u) | (rB & 2u) | (rC & 4u) | ((rC >> 13) & 8u) | ((rB >> 12) & 16u) | ((rA >> 11) & 32u);
}

// Groups of four: the six pairwise outcomes c_ij = (|w_i| >= |w_j|), i < j,
// index a 64-entry table whose byte holds the keep pattern (bits 0..3) and,
// for n == 2, the metadata nibble i0 | i1 << 2 (bits 4..7).
__device__ __forceinline__ uint32_t select4_entry(uint32_t cbits, int n) {
  const uint32_t c01 = cbits & 1u, c02 = (cbits >> 1) & 1u, c03 = (cbits >> 2) & 1u;
  const uint32_t c12 = (cbits >> 3) & 1u, c13 = (cbits >> 4) & 1u, c23 = (cbits >> 5) & 1u;
  const uint32_t r0 = 3u - c01 - c02 - c03;
  const uint32_t r1 = c01 + 2u - c12 - c13;
  const uint32_t r2 = c02 + c12 + 1u - c23;
  const uint32_t r3 = c03 + c13 + c23;
  const uint32_t kept = (r0 < uint32_t(n) ? 1u : 0u) | (r1 < uint32_t(n) ? 2u : 0u) | (r2 < uint32_t(n) ? 4u : 0u) |
                        (r3 < uint32_t(n) ? 8u : 0u);
  const uint32_t nib = static_cast<uint32_t>(kPairNibble >> (4 * kept)) & 0xFu;
  return kept | (nib << 4);
}

// int8 codes (+1 = 0x01, -1 = 0xFF, 0) of four bf16 W_eff values held in two
// words: their high bytes are 0x3F, 0xBF or 0x00.
__device__ __forceinline__ uint32_t code_bytes4(uint32_t weff_lo, uint32_t weff_hi) {
  const uint32_t hb = __byte_perm(weff_lo, weff_hi, 0x7531);
  return ((hb >> 5) & 0x01010101u) | (((hb >> 7) & 0x01010101u) * 0xFEu);
}

template <int M>
__global__ void __launch_bounds__(kPackThreads)
    k_prep_pack(const uint4* __restrict__ w, int64_t n_out, int64_t k, int n, const BlobHeader* h, PackOut out) {
  // M == 4: per comparison outcome, the keep masks of the group's two words
  // (0xFFFF per kept weight) and the byte keep pattern | nibble << 4.
  __shared__ uint4 s_sel[64];
  if (M == 4 && threadIdx.x < 64) {
    const uint32_t e = select4_entry(threadIdx.x, n), kp = e & 0xFu;
    const uint32_t km_lo = ((kp & 1u) | ((kp & 2u) << 15)) * 0xFFFFu;
    const uint32_t km_hi = (((kp >> 2) & 1u) | (((kp >> 2) & 2u) << 15)) * 0xFFFFu;
    s_sel[threadIdx.x] = make_uint4(km_lo, km_hi, e, 0u);
  }
  __syncthreads();
  pdl_wait();  // g comes from k_gamma_finalize (a kernel that may overlap this one: coherent load)
  const float g = __ldcg(&h->g);
  // code != 0 <=> 2|w| > g <=> |w| > g/2 (exact) <=> the 15-bit magnitude
  // exceeds bits(g/2) >> 16, i.e. |w| > that bf16 value as a float compare.
  const uint32_t thr = __float_as_uint(__fmul_rn(g, 0.5f)) >> 16;
  const uint32_t thr2 = thr | (thr << 16);
  pdl_trigger();

  const int lane = threadIdx.x & 31;
  const int upr = static_cast<int>(k / 8);  // lanes' worth of weights per row (multiple of 8)
  const int64_t gwarp = int64_t(blockIdx.x) * (kPackThreads / 32) + (threadIdx.x >> 5);
  const int64_t nwarps = int64_t(gridDim.x) * (kPackThreads / 32);
  for (int64_t row = gwarp; row < n_out; row += nwarps) {
    const uint4* wrow = w + row * upr;
    uint4* weff_row = reinterpret_cast<uint4*>(out.weff_bf16) + row * upr;
    // kPackDepth 16-byte loads in flight per lane, then process them one by one.
    for (int c0 = 0; c0 < upr; c0 += kPackDepth * 32) {
      uint4 vbuf[kPackDepth];
#pragma unroll
      for (int q = 0; q < kPackDepth; ++q) {
        const int cq = c0 + 32 * q + lane;
        vbuf[q] = (cq < upr) ? __ldcs(wrow + cq) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int q = 0; q < kPackDepth; ++q) {
        if (c0 + 32 * q >= upr) break;  // uniform across the warp
        const int c = c0 + 32 * q + lane;
        const bool active = c < upr;  // upr is a multiple of 8: quads are all-or-nothing
        const uint32_t wd[4] = {vbuf[q].x, vbuf[q].y, vbuf[q].z, vbuf[q].w};
        uint32_t mw[4];  // magnitudes, two per word
#pragma unroll
        for (int j = 0; j < 4; ++j) mw[j] = wd[j] & 0x7FFF7FFFu;
        uint32_t kept = 0, sel0 = 0, sel1 = 0;
        uint32_t km[4];  // 0xFFFF per kept weight
        if (M == 4) {
          const uint4 e0 = s_sel[pair_outcomes4_packed(mw[0], mw[1])];
          const uint4 e1 = s_sel[pair_outcomes4_packed(mw[2], mw[3])];
          km[0] = e0.x;
          km[1] = e0.y;
          km[2] = e1.x;
          km[3] = e1.y;
          sel0 = e0.z;
          sel1 = e1.z;
          kept = (sel0 & 0xFu) | ((sel1 & 0xFu) << 4);
        } else {
          uint32_t mag[8];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            mag[2 * j] = mw[j] & 0xFFFFu;
            mag[2 * j + 1] = mw[j] >> 16;
          }
#pragma unroll
          for (int gi = 0; gi < 8 / M; ++gi) kept |= keep_bits<M>(mag, gi * M, n) << (gi * M);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t kp = (kept >> (2 * j)) & 3u;
            km[j] = ((kp & 1u) | ((kp & 2u) << 15)) * 0xFFFFu;
          }
        }

        // W_eff in bf16, two weights per word: (sign | 0x3F80) where kept and code != 0.
        uint32_t weff[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t nz = bf16x2_gt_mask(mw[j], thr2);
          weff[j] = ((wd[j] & 0x80008000u) | 0x3F803F80u) & nz & km[j];
        }
        const uint32_t codes_lo = code_bytes4(weff[0], weff[1]);  // weights 0..3
        const uint32_t codes_hi = code_bytes4(weff[2], weff[3]);  // weights 4..7

        if (active) {
          if (M == 2) {
            const uint32_t mw = (kept & 3u) | (((kept >> 2) & 3u) << 8) | (((kept >> 4) & 3u) << 16) |
                                (((kept >> 6) & 3u) << 24);
            reinterpret_cast<uint32_t*>(out.mask + row * (k / 2))[c] = mw;
          } else if (M == 4) {
            const uint32_t mw = (kept & 0xFu) | (((kept >> 4) & 0xFu) << 8);
            reinterpret_cast<uint16_t*>(out.mask + row * (k / 4))[c] = static_cast<uint16_t>(mw);
          } else {
            out.mask[row * (k / 8) + c] = static_cast<uint8_t>(kept);
          }
          weff_row[c] = make_uint4(weff[0], weff[1], weff[2], weff[3]);
          if (out.codes != nullptr) reinterpret_cast<uint2*>(out.codes + row * k)[c] = make_uint2(codes_lo, codes_hi);
        }
        if (M == 4 && out.sp_values != nullptr) {  // 2:4: kept values, metadata, optional GEMV bytes
          const uint32_t nib0 = sel0 >> 4, nib1 = sel1 >> 4;
          // the two kept codes of each group, in index order
          const uint32_t v0 = __byte_perm(codes_lo, 0u, (nib0 & 3u) | ((nib0 >> 2) << 4));
          const uint32_t v1 = __byte_perm(codes_hi, 0u, (nib1 & 3u) | ((nib1 >> 2) << 4));
          const uint32_t vals = (v0 & 0xFFFFu) | (v1 << 16);
          const uint32_t meta = nib0 | (nib1 << 4);
          // tensor-core metadata: [row_block][k_block][128 rows][16 bytes]; this
          // lane's byte is byte (c % 16) of the row's 16 bytes in k block c / 16.
          uint32_t word = meta << (8 * (lane & 3));
          word |= __shfl_xor_sync(0xffffffffu, word, 1);
          word |= __shfl_xor_sync(0xffffffffu, word, 2);
          if (active) {
            reinterpret_cast<uint32_t*>(out.sp_values + row * (k / 2))[c] = vals;
            if ((lane & 3) == 0) {
              uint8_t* mrow = out.sp_meta + ((row >> 7) * out.meta_kblocks * 128 + (row & 127)) * 16;
              *reinterpret_cast<uint32_t*>(mrow + (c >> 4) * 2048 + (c & 15)) = word;
            }
            if (out.gemv != nullptr) {
              const uint32_t g0 = (nib0 << 4) | (v0 & 3u) | (((v0 >> 8) & 3u) << 2);
              const uint32_t g1 = (nib1 << 4) | (v1 & 3u) | (((v1 >> 8) & 3u) << 2);
              reinterpret_cast<uint16_t*>(out.gemv + row * (k / 4))[c] = static_cast<uint16_t>(g0 | (g1 << 8));
            }
          }
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Host launcher
// ---------------------------------------------------------------------------
cudaError_t launch_prepare(const uint16_t* w, int64_t n_out, int64_t k, int n, int m, uint32_t flags,
                           uint8_t* blob, const sbl_blob_layout& L, int num_sms, cudaStream_t s) {
  BlobHeader* h = reinterpret_cast<BlobHeader*>(blob + L.header);
  uint64_t* slot_bins = reinterpret_cast<uint64_t*>(blob + L.scratch);
  uint32_t* slot_flags = reinterpret_cast<uint32_t*>(blob + L.scratch + uint64_t(kPrepSlots) * kExactBins * 8);
  if (L.sp_meta && (n_out % 256 != 0 || k % 256 != 0)) {
    cudaError_t e = cudaMemsetAsync(blob + L.sp_meta, 0x44, L.sp_meta_bytes, s);
    if (e != cudaSuccess) return e;
  }
  const int64_t nvec = n_out * k / 8;
  int slots = num_sms < kPrepSlots ? num_sms : kPrepSlots;
  const int64_t need = (nvec + kAbsThreads - 1) / kAbsThreads;
  if (need < slots) slots = static_cast<int>(need);
  constexpr int abs_smem = kAbsWarps * kLaneBins * 32 * 4;  // 128 KB of lane bins
  static const cudaError_t attr_err =
      cudaFuncSetAttribute(k_absmean_partials, cudaFuncAttributeMaxDynamicSharedMemorySize, abs_smem);
  if (attr_err != cudaSuccess) return attr_err;
  k_absmean_partials<<<slots, kAbsThreads, abs_smem, s>>>(reinterpret_cast<const uint4*>(w), nvec, slot_bins,
                                                          slot_flags);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  PackOut out;
  out.mask = blob + L.mask;
  out.codes = L.codes ? reinterpret_cast<int8_t*>(blob + L.codes) : nullptr;
  out.weff_bf16 = reinterpret_cast<uint16_t*>(blob + L.weff_bf16);
  out.sp_values = L.sp_values ? reinterpret_cast<int8_t*>(blob + L.sp_values) : nullptr;
  out.sp_meta = L.sp_meta ? blob + L.sp_meta : nullptr;
  out.gemv = L.gemv ? blob + L.gemv : nullptr;
  out.meta_kblocks = static_cast<int>(meta_k_padded(k) / 128);
  e = launch_pdl(k_gamma_finalize, dim3(1), dim3(kFinThreads), 0, s, slot_bins, slot_flags, slots, h, n_out, k, n, m, flags);
  if (e != cudaSuccess) return e;
  // Rows are spread over warps; pick the warp count so every warp gets the
  // same number of rows (within one) and the grid stays within three blocks/SM.
  const int64_t max_warps = int64_t(num_sms) * 3 * (kPackThreads / 32);
  const int64_t rounds = (n_out + max_warps - 1) / max_warps;
  const int64_t warps = (n_out + rounds - 1) / rounds;
  const int64_t blocks = (warps + kPackThreads / 32 - 1) / (kPackThreads / 32);
  const dim3 grid(static_cast<unsigned>(blocks)), block(kPackThreads);
  const uint4* wv = reinterpret_cast<const uint4*>(w);
  const BlobHeader* hc = h;
  switch (m) {
    case 2: return launch_pdl(k_prep_pack<2>, grid, block, 0, s, wv, n_out, k, n, hc, out);
    case 4: return launch_pdl(k_prep_pack<4>, grid, block, 0, s, wv, n_out, k, n, hc, out);
    default: return launch_pdl(k_prep_pack<8>, grid, block, 0, s, wv, n_out, k, n, hc, out);
  }
}

}  // namespace sbl
