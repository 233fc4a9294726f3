// Weight preparation for Sparse-BitLinear: exact absmean scale, N:M mask from
// the master magnitudes, ternary codes with the mask applied after
// quantisation, and the packed forms the GEMM kernels read.
//
// Paper: "Sparse-BitNet: 1.58-bit LLMs are Naturally Friendly to
// Semi-Structured Sparsity" -- gist.science German technical summary §2
// (magnitude mask from the masters, quantise then mask), Korean summary
// §2.1-2.2 (per-step recompute), French summary §2.
//
// One cooperative launch, one CTA per SM.  Each CTA owns a contiguous range
// of W (in 16-byte vectors of eight weights) and streams it twice through a
// ring of shared-memory stages filled by bulk copies (one producer warp,
// twenty-four consumer warps):
//   phase 1  from HBM: every |w| is added exactly (below); W stays in L2;
//   barrier  every CTA publishes its partial sum and waits for the others
//            (bounded wait on per-CTA arrival words);
//   phase 2  from L2: every CTA folds all partial sums and rounds the exact
//            mean once to fp32 (so all CTAs hold the same g) while the first
//            stages refill, then masks, ternarises and writes every packed
//            section.
// The kernel lets its successor (the activation quantiser, launched with
// programmatic stream serialisation) start at once, so the two HBM streams
// overlap.
#include "sbl_kernels.h"

#include "sbl_device.cuh"

namespace sbl {

constexpr int kPrepConsumers = 768;                    // 24 consumer warps
constexpr int kPrepConsumerWarps = kPrepConsumers / 32;
constexpr int kPrepThreads = kPrepConsumers + 32;      // + one producer warp
constexpr int kVecsPerThread = 2;                      // 16-byte vectors per consumer per stage
constexpr int kChunkVecs = kVecsPerThread * kPrepConsumers;  // 24 KB per stage
constexpr int kPrepStages = 8;
constexpr size_t kPrepTailBytes = 4096;
constexpr size_t kSelBytes = 64 * 32 * 8;  // 64 entries x 32 lane copies x 8 bytes
constexpr size_t kPrepSmem = size_t(kPrepStages) * kChunkVecs * 16 + kSelBytes + kPrepTailBytes;

// ---------------------------------------------------------------------------
// Exact sum of |w| (absmean numerator).
//
// Fast path, exact by construction: a bf16 magnitude field `mag` (biased
// exponent e, 7-bit fraction f) shifted left by 13 is the high word of the
// fp64 number |w| * 2^-896 (the fp64 exponent field takes e, the top fraction
// bits take f).  For 2^-30 <= |w| < 2^6 every such number
// is an integer multiple of 2^(-37-896) below 2^(6-896), so a sum of up to
// 64 of them stays below 2^49 units and fp64 adds it without rounding.  After
// each stage (16 weights per thread) a thread converts its fp64 sum (scaled by 2^933) to
// an exact integer in units of 2^-37 and adds it to a 128-bit integer.
//
// Slow path, for any vector holding a weight outside that window (below
// 2^-30, zero included, at or above 2^6, Inf or NaN): in units of 2^-133 the magnitude
// is sig << s with sig = (e ? 128 + f : f) and s = max(e, 1) - 1 <= 253;
// shared 64-bit bin b = s >> 3 collects sig << (s & 7).  Bin b is an integer
// in units of 2^(8b - 133); the fast path's units 2^-37 are bin 12.
// ---------------------------------------------------------------------------
constexpr uint32_t kWinLo = 97u << 7;   // magnitude field of 2^-30
constexpr uint32_t kWinSpan = 36u << 7;  // up to, not including, 2^6
constexpr int kFastBin = 12;             // 8 * 12 - 133 = -37
constexpr int kFastBinHi = 19;           // 2^56 units of bin 12

__device__ __forceinline__ double fp64_of_hi_word(uint32_t hi_word) {
  return __hiloint2double(static_cast<int>(hi_word), 0);
}

__device__ __forceinline__ uint32_t bf16x2_max_nan(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t bf16x2_min(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("min.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t bf16x2_lt_mask(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("set.lt.u32.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t bf16x2_ge_mask_(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("set.ge.u32.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// All eight magnitudes (four words of two, sign bits clear) inside the fast
// window: the packed maximum (NaN propagating) below 2^6 and the packed
// minimum at least 2^-30.  Zeros take the slow path too.
__device__ __forceinline__ bool in_window(const uint32_t (&mw)[4]) {
  const uint32_t mx = bf16x2_max_nan(bf16x2_max_nan(mw[0], mw[1]), bf16x2_max_nan(mw[2], mw[3]));
  const uint32_t mn = bf16x2_min(bf16x2_min(mw[0], mw[1]), bf16x2_min(mw[2], mw[3]));
  constexpr uint32_t kHi2 = (kWinLo + kWinSpan) | ((kWinLo + kWinSpan) << 16), kLo2 = kWinLo | (kWinLo << 16);
  return (bf16x2_lt_mask(mx, kHi2) & bf16x2_ge_mask_(mn, kLo2)) == 0xFFFFFFFFu;
}

// A vector with a magnitude outside the fast window: its in-window magnitudes
// are returned as an fp64 sum for the caller's exact accumulator (so a stage
// still adds at most 16 window terms there), the others go to the exact
// 64-bit bins.  Flags: bit 0 a non-finite weight, bit 1 the bins are in use,
// bit 2 a magnitude at or above the window (2^6); *s_tiny counts the non-zero
// magnitudes below it (2^-30), whose total the scale's fast decision bounds.
__device__ __noinline__ double add_slow(uint32_t m0, uint32_t m1, uint32_t m2, uint32_t m3,
                                        unsigned long long* s_bins, uint32_t* s_flags, uint32_t* s_tiny) {
  const uint32_t mw[4] = {m0, m1, m2, m3};
  uint32_t fl = 0, tiny = 0;
  double in_win = 0.0;
#pragma unroll 1
  for (int j = 0; j < 8; ++j) {
    const uint32_t mag = (mw[j >> 1] >> (16 * (j & 1))) & 0x7FFFu;
    if (mag >= kWinLo && mag < kWinLo + kWinSpan) {
      in_win += fp64_of_hi_word(mag << 13);
      continue;
    }
    const uint32_t e = mag >> 7;
    if (e == 0xFFu) {
      fl |= 1u;
      continue;
    }
    if (mag >= kWinLo) fl |= 4u;
    else if (mag != 0u) ++tiny;
    const uint32_t s = max(e, 1u) - 1u;
    const uint32_t sig = mag - (s << 7);
    if (sig != 0u) atomicAdd(&s_bins[s >> 3], static_cast<unsigned long long>(sig << (s & 7u)));
  }
  atomicOr(s_flags, 2u | fl);
  if (tiny) atomicAdd(s_tiny, tiny);
  return in_win;
}

// Correct rounding without a division.  q approximates a positive value v
// within 2^-51 relative, plus (when `extra` > 0) an unknown non-negative
// addend below `extra`.  If q is farther than both from the fp32 rounding
// midpoint on its side of RN_fp32(q), then v lies on the same side and
// RN_fp32(v) = RN_fp32(q).  Returns false when q is too close to decide (an
// exact or near tie) or too small (the fp32 subnormal range is left to the
// exact path).
__device__ __forceinline__ bool round_fp32_if_clear(double q, double extra, float* out) {
  if (!(q > 0x1p-120)) return false;
  const float f = __double2float_rn(q);
  const double fd = static_cast<double>(f);
  const double nb = (q >= fd) ? static_cast<double>(nextafterf(f, 3.0e38f)) : static_cast<double>(nextafterf(f, 0.0f));
  const double mid = 0.5 * (fd + nb);  // exact: both are fp32 values
  if (fabs(q - mid) > q * 0x1p-48 + extra) {
    *out = f;
    return true;
  }
  return false;
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
  {
    // division-free attempt: the top 64 bits of S (truncated) in fp64
    float r;
    const double ds = ldexp(static_cast<double>(get64(topS - 63)), topS - 63 - 133);
    if (round_fp32_if_clear(ds / static_cast<double>(numel), 0.0, &r)) return r;
  }
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


// gamma = RN_fp32((S * 2^-37 + T) / numel) for a sum S held as a 128-bit
// integer (hi, lo), from an fp64 quotient (one rounding of S, one of the
// division), where T is the unknown total of `ntiny` magnitudes below 2^-30
// (so 0 <= T < ntiny * 2^-30).  False when that does not decide the rounding.
__device__ bool mean_fp32_fast(uint64_t lo, uint64_t hi, uint64_t numel, uint64_t ntiny, float* out) {
  const double s = __ull2double_rn(hi) * 0x1p64 + __ull2double_rn(lo);  // hi * 2^64 is exact
  if (s == 0.0) {
    if (ntiny != 0) return false;  // the mean is the tiny magnitudes' alone
    *out = 0.0f;
    return true;
  }
  const double dn = __ull2double_rn(numel);
  const double slack = __ddiv_rn(static_cast<double>(ntiny) * 0x1p-30, dn) * (1.0 + 0x1p-40);
  return round_fp32_if_clear(__ddiv_rn(s, dn) * 0x1p-37, slack, out);
}

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
// two words of magnitudes (m0 | m1 << 16, m2 | m3 << 16), as a 6-bit table
// index: bit 0 c01, bit 1 c02, bit 2 c03, bit 3 c23, bit 4 c13, bit 5 c12.
// Each packed compare gives 0xFFFF per true half, so the low halves supply
// bits 0-2 and the high halves bits 3-5 (taken from bits 19-21).
__device__ __forceinline__ uint32_t outcomes4_index(uint32_t m01, uint32_t m23) {
  const uint32_t rA = bf16x2_ge_mask(__byte_perm(m01, m23, 0x5410), __byte_perm(m01, m23, 0x7632));  // c01 | c23
  const uint32_t rB = bf16x2_ge_mask(m01, m23);                                                       // c02 | c13
  const uint32_t rC = bf16x2_ge_mask(m01, __byte_perm(m23, m23, 0x1032));                             // c03 | c12
  const uint32_t u = (rA & 0x00080001u) | (rB & 0x00100002u) | (rC & 0x00200004u);
  return (u >> 16) | (u & 7u);
}

// Table entry for one outcome index (8 bytes, replicated per lane so that a
// warp's random lookups never share a bank):
//   x  the keep bit of position p in the sign bit of byte p (a byte permute
//      with sign replication turns it into the 0xFFFF-per-kept-weight masks)
//   y  bits 0-3 the kept pattern, bits 4-7 the 2:4 metadata nibble
//      i0 | i1 << 2, bits 8-15 the byte-permute selector nibbles i0, i1 that
//      pick the two kept high bytes (i0 < i1 are the first two kept positions)
__device__ uint2 select4_entry(uint32_t idx, int n) {
  const uint32_t c01 = idx & 1u, c02 = (idx >> 1) & 1u, c03 = (idx >> 2) & 1u;
  const uint32_t c23 = (idx >> 3) & 1u, c13 = (idx >> 4) & 1u, c12 = (idx >> 5) & 1u;
  const uint32_t r0 = 3u - c01 - c02 - c03;  // positions that beat position 0
  const uint32_t r1 = c01 + 2u - c12 - c13;
  const uint32_t r2 = c02 + c12 + 1u - c23;
  const uint32_t r3 = c03 + c13 + c23;
  const uint32_t kept = (r0 < uint32_t(n) ? 1u : 0u) | (r1 < uint32_t(n) ? 2u : 0u) | (r2 < uint32_t(n) ? 4u : 0u) |
                        (r3 < uint32_t(n) ? 8u : 0u);
  uint32_t i0 = 0, i1 = 0;
  {
    int found = 0;
    for (uint32_t p = 0; p < 4; ++p)
      if (kept & (1u << p)) {
        if (found == 0) i0 = p;
        else if (found == 1) i1 = p;
        ++found;
      }
  }
  const uint32_t x = ((kept & 1u) << 7) | ((kept & 2u) << 14) | ((kept & 4u) << 21) | ((kept & 8u) << 28);
  const uint32_t y = kept | ((i0 | (i1 << 2)) << 4) | ((i0 | (i1 << 4)) << 8);
  return make_uint2(x, y);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// int8 codes (+1 = 0x01, -1 = 0xFF, 0) of four W_eff values given by their
// bf16 high bytes (0x3F, 0xBF or 0x00): the sign byte replicated, or bit 5.
__device__ __forceinline__ uint32_t codes_of_high_bytes(uint32_t hb) {
  // prmt with selector bit 3 set replicates the sign bit of the chosen byte
  return prmt(hb, 0u, 0xBA98u) | ((hb >> 5) & 0x01010101u);
}

// ---------------------------------------------------------------------------
// Grid barrier on the blob's scratch: a generation word `gen` and each CTA's
// tagged partial-sum words.  Every CTA reads gen (= G) before it publishes,
// tags its words with G + 1, and waits until all CTAs' words carry G + 1;
// CTA 0 then stores G + 1 to gen (plain stores, so gen wraps like the tags).  Nothing needs initialising: a blob holds
// the tag G + 1 in every word only by accident of its previous contents,
// which a completed launch never leaves behind (it leaves tags equal to gen).
// A wait that gives up raises the timeout bit and stores G + 2 to gen, so
// stale words of that launch cannot satisfy the next one.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void st_release_u64(uint64_t* p, uint64_t v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ void st_relaxed_u64(uint64_t* p, uint64_t v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ ulonglong2 ld_relaxed_v2u64(const ulonglong2* p) {
  ulonglong2 v;
  asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(v.x), "=l"(v.y) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint64_t ld_relaxed_u64(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kPrepConsumers) : "memory"); }

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void bulk_load_hint(void* smem_dst, const void* gmem_src, uint32_t bytes, uint64_t* bar,
                                               uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// What one launch does: the whole preparation; only the exact sum of |w| of
// this (shard of the) matrix, written out as SBL_SUM_WORDS words; or the
// preparation with the scale taken from given sum words (the word-wise sum
// over all shards of a row-sharded matrix) instead of this matrix's own sum.
enum PrepMode : int { kPrepFull = 0, kPrepSumOnly = 1, kPrepFromSum = 2 };

struct PrepArgs {
  const uint4* w;
  int64_t n_out, k;
  int mode;                 // PrepMode
  uint64_t numel;           // weights the mean runs over (all shards' for kPrepFromSum)
  uint64_t* sum_out;        // kPrepSumOnly: SBL_SUM_WORDS words, written by CTA 0
  const uint64_t* sum_in;   // kPrepFromSum: SBL_SUM_WORDS words
  int n, m;
  uint32_t layer_flags;
  BlobHeader* h;
  uint64_t* slot_fast;  // [grid][4]: tagged pieces of the 128-bit fast sum, tagged flags
  uint64_t* slot_bins;  // [grid][kExactBins], written only when the slow path ran
  uint64_t* gen;
  PackOut out;
};

struct PrepTail {
  uint64_t full[kPrepStages];
  uint64_t empty[kPrepStages];
  unsigned long long bins[kExactBins];
  unsigned long long fold_bins[kExactBins];
  uint64_t warp_lo[kPrepConsumerWarps], warp_hi[kPrepConsumerWarps];
  uint64_t gen;
  uint32_t flags;       // bit 0 non-finite, bit 1 slow bins in use, bit 2 a magnitude >= 2^6 (this CTA)
  uint32_t ntiny;       // non-zero magnitudes below 2^-30 in this CTA's bins
  float g;
  int abort_flag;
};
static_assert(sizeof(PrepTail) <= kPrepTailBytes, "prepare kernel's shared tail overflows its slot");

// The exact path of the scale: add the 128-bit fast sum (L, H) to the folded
// slow-path bins of all CTAs, then round the exact mean once.  Kept out of line: it runs only for ties, tiny means or
// magnitudes outside the fast window.
__device__ __noinline__ float gamma_exact(const unsigned long long* slow_bins, uint64_t L, uint64_t H, uint64_t numel) {
  uint64_t bins[kExactBins];
#pragma unroll
  for (int b = 0; b < kExactBins; ++b) bins[b] = slow_bins[b];
  bins[kFastBin] += L & ((1ull << 56) - 1ull);
  bins[kFastBinHi] += (L >> 56) | (H << 8);
  return exact_mean_fp32(bins, numel);
}

// The whole preparation of one matrix by CTA `blk` of the `G` CTAs that
// work on it (a launch of one matrix, or one matrix's share of a grouped
// launch).
template <int M>
__device__ __forceinline__ void prepare_body(const PrepArgs& a, const int G, const int blk) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint4* ring = reinterpret_cast<uint4*>(smem);
  uint2* sel = reinterpret_cast<uint2*>(smem + size_t(kPrepStages) * kChunkVecs * 16);  // [64][32 lanes]
  PrepTail* tail = reinterpret_cast<PrepTail*>(smem + size_t(kPrepStages) * kChunkVecs * 16 + kSelBytes);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t* status = &a.h->status;
  volatile int* abort_flag = &tail->abort_flag;
  // The successor only reads its own inputs before it waits for this kernel.
  pdl_trigger();

  // This CTA's vectors [v0, v1): equal shares rounded to 32 vectors.
  const int64_t nvec = a.n_out * a.k / 8;
  const int64_t share = ((nvec + G - 1) / G + 31) / 32 * 32;
  const int64_t v0 = share * blk < nvec ? share * blk : nvec;
  const int64_t v1 = v0 + share < nvec ? v0 + share : nvec;
  const int nch = static_cast<int>((v1 - v0 + kChunkVecs - 1) / kChunkVecs);

  if (tid < kExactBins) {
    tail->bins[tid] = 0ull;
    tail->fold_bins[tid] = 0ull;
  }
  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < kPrepStages; ++s) {
      mbar_init(&tail->full[s], 1);
      mbar_init(&tail->empty[s], kPrepConsumerWarps);
    }
    fence_mbar_init();
    tail->gen = ld_relaxed_u64(a.gen);
    tail->flags = 0u;
    tail->ntiny = 0u;
    tail->abort_flag = 0;
    if (blk == 0) *status = 0u;  // a new prepare resets the status word
  }
  if (M == 4) {
    for (int i = tid; i < 64 * 32; i += kPrepThreads) sel[i] = select4_entry(static_cast<uint32_t>(i >> 5), a.n);
  }
  __syncthreads();

  if (warp == kPrepConsumerWarps) {
    // ---- producer: phase 1 chunks from HBM, then phase 2 chunks from L2 (W
    // does not depend on the scale, so refills need not wait for the barrier)
    if (lane == 0) {
      const uint64_t keep = l2_policy_evict_last(), drop = l2_policy_evict_first();
      // phase-1 chunks (J < nch) then phase-2 chunks; a launch streams only
      // the phases its mode runs, ring slots counted from its first chunk
      const int J0 = a.mode == kPrepFromSum ? nch : 0, J1 = a.mode == kPrepSumOnly ? nch : 2 * nch;
      for (int J = J0; J < J1; ++J) {
        const int j = J < nch ? J : J - nch;
        const int u = J - J0, s = u % kPrepStages;
        if (u >= kPrepStages && !mbar_wait(&tail->empty[s], ((u / kPrepStages) - 1) & 1, abort_flag, status)) break;
        const int64_t c0 = v0 + int64_t(j) * kChunkVecs;
        const int64_t cnt = (v1 - c0 < kChunkVecs) ? v1 - c0 : kChunkVecs;
        const uint32_t bytes = static_cast<uint32_t>(cnt) * 16u;
        mbar_arrive_expect_tx(&tail->full[s], bytes);
        bulk_load_hint(ring + size_t(s) * kChunkVecs, a.w + c0, bytes, &tail->full[s], J < nch ? keep : drop);
      }
    }
    return;
  }

  // ---- consumers, phase 1: exact sum of |w| ----
  uint64_t lo = 0, hi = 0;
  for (int j = 0; j < (a.mode == kPrepFromSum ? 0 : nch); ++j) {
    const int s = j % kPrepStages;
    if (!mbar_wait(&tail->full[s], (j / kPrepStages) & 1, abort_flag, status)) break;
    const int64_t rem = v1 - v0 - int64_t(j) * kChunkVecs;
    const int cnt = rem < kChunkVecs ? static_cast<int>(rem) : kChunkVecs;
    const uint4* st = ring + size_t(s) * kChunkVecs;
    double acc[kVecsPerThread];
#pragma unroll
    for (int h2 = 0; h2 < kVecsPerThread; ++h2) {
      acc[h2] = 0.0;
      const int e = tid + h2 * kPrepConsumers;
      if (e < cnt) {
        const uint4 v = st[e];
        const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
        const uint32_t mw[4] = {v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu, v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu};
        if (in_window(mw)) {
          // the high words of |w| * 2^-896 in fp64, read straight off the bf16
          // bits (the masks drop the sign and the neighbouring weight)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            acc[h2] += fp64_of_hi_word((wd[q] << 13) & 0x0FFFE000u);
            acc[h2] += fp64_of_hi_word((wd[q] >> 3) & 0x0FFFE000u);
          }
        } else {
          acc[h2] += add_slow(mw[0], mw[1], mw[2], mw[3], tail->bins, &tail->flags, &tail->ntiny);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&tail->empty[s]);
    double tot = acc[0];
#pragma unroll
    for (int h2 = 1; h2 < kVecsPerThread; ++h2) tot += acc[h2];
    const uint64_t units = __double2ull_rn(tot * 0x1p933);  // exact: an integer below 2^48
    lo += units;
    hi += (lo < units) ? 1ull : 0ull;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const uint64_t olo = __shfl_xor_sync(0xffffffffu, lo, off), ohi = __shfl_xor_sync(0xffffffffu, hi, off);
    lo += olo;
    hi += ohi + ((lo < olo) ? 1ull : 0ull);
  }
  if (lane == 0) {
    tail->warp_lo[warp] = lo;
    tail->warp_hi[warp] = hi;
  }
  consumers_sync();

  // ---- grid barrier and fold in one (warp 0) ----
  // Each CTA publishes its partial sum as four 64-bit words, each carrying
  // the generation tag G + 1 in its upper half (a 64-bit store is seen whole
  // or not at all): the 128-bit sum in three 32-bit pieces and the flags.
  // Warp 0 of every CTA polls all CTAs' words until every tag reads G + 1,
  // summing the pieces as it goes, so the wait and the fold cost one pass.
  const uint64_t gen0 = tail->gen;
  if (warp == 0) {
    uint64_t s0 = 0, s1 = 0, s2 = 0, s3 = 0;  // the sum in 32-bit pieces; s3: tiny magnitudes in the bins
    uint32_t fl = 0, slow_r = 0;  // slow_r: bit r set when CTA lane + 32 r used its slow bins
    if (a.mode == kPrepFromSum) {
      // The scale from given sum words (all shards' sums added word by
      // word): every CTA reads them, so no grid barrier is needed.
      s0 = a.sum_in[0];
      s1 = a.sum_in[1];
      s2 = a.sum_in[2];
      for (int b = lane; b < kExactBins; b += 32) {
        const uint64_t v = a.sum_in[3 + b];
        tail->fold_bins[b] = v;
        if (v != 0ull) fl = 2u;
      }
      fl = __ballot_sync(0xffffffffu, fl != 0u) ? 2u : 0u;
      if (a.sum_in[3 + kExactBins] != 0ull) fl |= 1u;
      if (a.sum_in[4 + kExactBins] != 0ull) fl |= 4u;
      s3 = a.sum_in[5 + kExactBins];
      __syncwarp();
    } else {
      uint64_t L = lane < kPrepConsumerWarps ? tail->warp_lo[lane] : 0ull;
      uint64_t H = lane < kPrepConsumerWarps ? tail->warp_hi[lane] : 0ull;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const uint64_t olo = __shfl_xor_sync(0xffffffffu, L, off), ohi = __shfl_xor_sync(0xffffffffu, H, off);
        L += olo;
        H += ohi + ((L < olo) ? 1ull : 0ull);
      }
      // flags in the low byte, the count of tiny magnitudes above it (a count
      // too large to carry forces the exact path, as a huge magnitude does)
      const uint32_t nt = tail->ntiny;
      const uint32_t fl_own = (tail->flags | (nt > 0xFFFFFFu ? 4u : 0u)) | ((nt > 0xFFFFFFu ? 0u : nt) << 8);
      if (fl_own & 2u) {  // slow bins in use: publish them first
        for (int b = lane; b < kExactBins; b += 32) a.slot_bins[int64_t(blk) * kExactBins + b] = tail->bins[b];
        __threadfence();
      }
      __syncwarp();
      const uint32_t tagv = static_cast<uint32_t>(gen0 + 1);
      const uint64_t tag = uint64_t(tagv) << 32;
      if (lane == 0) {  // H < 2^32: a CTA holds at most 2^40 weights below 2^6, i.e. below 2^83 units
        uint64_t* sf = a.slot_fast + int64_t(blk) * 4;
        st_relaxed_u64(sf + 0, tag | (L & 0xFFFFFFFFull));
        st_relaxed_u64(sf + 1, tag | (L >> 32));
        st_relaxed_u64(sf + 2, tag | (H & 0xFFFFFFFFull));
        st_release_u64(sf + 3, tag | fl_own);
      }
      uint64_t t0 = 0;
      for (uint32_t it = 0;; ++it) {
        bool all = true;
        s0 = s1 = s2 = s3 = 0;
        fl = slow_r = 0;
        auto take = [&](int c, int r) {
          const ulonglong2* sf = reinterpret_cast<const ulonglong2*>(a.slot_fast + int64_t(c) * 4);
          const ulonglong2 p01 = ld_relaxed_v2u64(sf), p23 = ld_relaxed_v2u64(sf + 1);
          all &= ((p01.x >> 32) == tagv) & ((p01.y >> 32) == tagv) & ((p23.x >> 32) == tagv) & ((p23.y >> 32) == tagv);
          s0 += p01.x & 0xFFFFFFFFull;
          s1 += p01.y & 0xFFFFFFFFull;
          s2 += p23.x & 0xFFFFFFFFull;
          fl |= static_cast<uint32_t>(p23.y) & 0xFFu;
          s3 += (p23.y >> 8) & 0xFFFFFFull;
          if (r < 32 && (p23.y & 2u)) slow_r |= 1u << r;
        };
#pragma unroll
        for (int r = 0; r < 8; ++r)
          if (lane + 32 * r < G) take(lane + 32 * r, r);
        for (int c = lane + 256, r = 8; c < G; c += 32, ++r) take(c, r);
        if (__all_sync(0xffffffffu, all)) break;
        __nanosleep(128);
        if ((it & 7u) == 7u) {
          const uint64_t now = globaltimer_ns();
          if (t0 == 0) {
            t0 = now;
          } else if (now - t0 > kWaitLimitNs) {
            if (lane == 0) {
              raise_status(status, SBL_STATUS_TIMEOUT);
              st_relaxed_u64(a.gen, gen0 + 2);
            }
            break;
          }
        }
      }
      __threadfence();  // acquire: the slow bins behind the tags are visible from here on
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        s0 += __shfl_xor_sync(0xffffffffu, s0, off);
        s1 += __shfl_xor_sync(0xffffffffu, s1, off);
        s2 += __shfl_xor_sync(0xffffffffu, s2, off);
        s3 += __shfl_xor_sync(0xffffffffu, s3, off);
        fl |= __shfl_xor_sync(0xffffffffu, fl, off);
      }
    }
    // the 128-bit total: s0 + s1 * 2^32 + s2 * 2^64 (each below 2^42)
    const uint64_t t1 = s1 << 32;
    const uint64_t Lt = s0 + t1;
    const uint64_t Ht = s2 + (s1 >> 32) + ((Lt < t1) ? 1ull : 0ull);
    const uint64_t numel = a.numel;
    // The fast sum decides gamma unless a weight is non-finite or at least
    // 2^6, or the rounding is too close to call given the tiny magnitudes'
    // bound; every lane computes the same decision.
    float gamma = 0.0f;
    bool decided = false;
    if (fl & 1u) {
      gamma = __int_as_float(0x7fc00000);
      decided = true;
    } else if (!(fl & 4u)) {
      decided = mean_fp32_fast(Lt, Ht, numel, s3, &gamma);
    }
    // Fold the slow bins of the CTAs that used them, lanes over bins: rarely
    // needed for the scale; always for a sum-only launch, which writes them.
    if (a.mode != kPrepFromSum && (fl & 2u) && (!decided || a.mode == kPrepSumOnly)) {
      for (int r = 0; 32 * r < G && r < 32; ++r) {
        uint32_t slow = __ballot_sync(0xffffffffu, (slow_r >> r) & 1u);
        while (slow) {
          const int c = 32 * r + __ffs(slow) - 1;
          slow &= slow - 1u;
          const unsigned long long* src = reinterpret_cast<const unsigned long long*>(a.slot_bins + int64_t(c) * kExactBins);
          const unsigned long long v0 = __ldcg(src + lane);
          const unsigned long long v1 = (lane + 32 < kExactBins) ? __ldcg(src + lane + 32) : 0ull;
          if (v0) atomicAdd(&tail->fold_bins[lane], v0);
          if (v1) atomicAdd(&tail->fold_bins[lane + 32], v1);
        }
      }
      __syncwarp();
    }
    if (a.mode == kPrepSumOnly) {
      // the sum words: fast sum pieces, slow bins, then counts of non-finite
      // and huge magnitudes (as 0/1) and of tiny ones; words of shards add up
      if (blk == 0) {
        for (int b = lane; b < kExactBins; b += 32) a.sum_out[3 + b] = tail->fold_bins[b];
        if (lane == 0) {
          a.sum_out[0] = s0;
          a.sum_out[1] = s1;
          a.sum_out[2] = s2;
          a.sum_out[3 + kExactBins] = (fl & 1u) ? 1ull : 0ull;
          a.sum_out[4 + kExactBins] = (fl & 4u) ? 1ull : 0ull;
          a.sum_out[5 + kExactBins] = s3;
          st_relaxed_u64(a.gen, gen0 + 1);
          if (fl & 1u) raise_status(status, SBL_STATUS_NONFINITE_W);
        }
      }
    } else if (lane == 0) {
      if (blk == 0 && a.mode == kPrepFull) st_relaxed_u64(a.gen, gen0 + 1);
      if (!decided) gamma = gamma_exact(tail->fold_bins, Lt, Ht, numel);
      const float g = (gamma > 1e-5f) ? gamma : 1e-5f;  // a NaN gamma gives 1e-5; the status word says why
      tail->g = g;
      if (blk == 0) {
        BlobHeader* h = a.h;
        h->magic = kMagic;
        h->version = 3;
        h->n_out = a.n_out;
        h->k = a.k;
        h->n = a.n;
        h->m = a.m;
        h->flags = a.layer_flags;
        h->gamma = gamma;
        h->g = g;
        if (fl & 1u) raise_status(status, SBL_STATUS_NONFINITE_W);
      }
    }
  }
  consumers_sync();
  if (a.mode == kPrepSumOnly) return;
  const float g = tail->g;
  // code != 0 <=> 2|w| > g <=> |w| > g/2 (exact) <=> the 15-bit magnitude
  // exceeds bits(g/2) >> 16, i.e. |w| > that bf16 value as a float compare.
  const uint32_t thr = __float_as_uint(__fmul_rn(g, 0.5f)) >> 16;
  const uint32_t thr2 = thr | (thr << 16);

  // ---- consumers, phase 2: mask, ternarise, pack ----
  const int n = a.n;
  const int upr = static_cast<int>(a.k / 8);  // vectors per row (multiple of 8)
  // (row, column-vector) of this thread's vectors in the current chunk
  int64_t row[kVecsPerThread];
  int col[kVecsPerThread];
#pragma unroll
  for (int h2 = 0; h2 < kVecsPerThread; ++h2) {
    const int64_t i = v0 + tid + h2 * kPrepConsumers;
    row[h2] = i / upr;
    col[h2] = static_cast<int>(i - row[h2] * upr);
  }
  const int64_t meta_rb_bytes = int64_t(a.out.meta_kblocks) * 2048;  // one 128-row block of metadata
  const int step_rows = kChunkVecs / upr, step_cols = kChunkVecs % upr;  // one chunk, in (rows, vectors)
  // This CTA's part of every section, addressed by 32-bit vector offsets
  // from v0 (u < v1 - v0 < 2^31), so a store address is one multiply-add.
  const uint32_t nv = static_cast<uint32_t>(v1 - v0);
  uint8_t* const mask_c = a.out.mask + v0 * (8 / M);
  uint4* const weff_c = reinterpret_cast<uint4*>(a.out.weff_bf16) + v0;
  uint2* const codes_c = a.out.codes != nullptr ? reinterpret_cast<uint2*>(a.out.codes) + v0 : nullptr;
  uint32_t* const spv_c = a.out.sp_values != nullptr ? reinterpret_cast<uint32_t*>(a.out.sp_values) + v0 : nullptr;
  const int ring0 = a.mode == kPrepFromSum ? 0 : nch;  // ring slots used before phase 2
  for (int j = 0; j < nch; ++j) {
    const int J = ring0 + j, s = J % kPrepStages;
    // the whole warp leaves together (the decode pack's writer below uses
    // warp shuffles)
    if (!__all_sync(0xffffffffu, mbar_wait(&tail->full[s], (J / kPrepStages) & 1, abort_flag, status))) break;
    const uint4* st = ring + size_t(s) * kChunkVecs;
#pragma unroll
    for (int h2 = 0; h2 < kVecsPerThread; ++h2) {
      const int e = tid + h2 * kPrepConsumers;
      const uint32_t u = static_cast<uint32_t>(j) * kChunkVecs + e;  // vector v0 + u
      const bool active = u < nv;
      const uint4 vv = active ? st[e] : make_uint4(0, 0, 0, 0);
      const uint32_t wd[4] = {vv.x, vv.y, vv.z, vv.w};
      uint32_t mw[4], nz[4], key[4];  // magnitudes, code != 0 (0xFFFF per half), selection keys
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        mw[q] = wd[q] & 0x7FFF7FFFu;
        nz[q] = bf16x2_gt_mask(mw[q], thr2);  // code != 0 <=> |w| > g/2, a packed bf16 compare
        // the mask is selected on |w|, or (ablation) on |q| as bf16 1.0 / 0
        key[q] = a.out.mask_from_codes ? (nz[q] & 0x3F803F80u) : mw[q];
      }
      uint32_t km[4];  // 0xFFFF per kept weight
      // Z: bits 0-3 / 8-11 kept pattern of group 0 / 1 (the mask section's
      // u16), bits 16-19 / 20-23 their 2:4 metadata nibbles; W: byte-permute
      // selector of the four kept high bytes.
      uint32_t Z = 0, W = 0;
      if (M == 4) {
        const uint2 e0 = sel[outcomes4_index(key[0], key[1]) * 32 + lane];
        const uint2 e1 = sel[outcomes4_index(key[2], key[3]) * 32 + lane];
        km[0] = prmt(e0.x, 0u, 0x9988u);
        km[1] = prmt(e0.x, 0u, 0xBBAAu);
        km[2] = prmt(e1.x, 0u, 0x9988u);
        km[3] = prmt(e1.x, 0u, 0xBBAAu);
        Z = (e0.y & 0x0Fu) | ((e1.y & 0x0Fu) << 8) | ((e0.y & 0xF0u) << 12) | ((e1.y & 0xF0u) << 16);
        W = ((e0.y >> 8) & 0xFFu) | ((((e1.y >> 8) & 0xFFu) + 0x44u) << 8);
      } else {
        uint32_t mag[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          mag[2 * q] = key[q] & 0xFFFFu;
          mag[2 * q + 1] = key[q] >> 16;
        }
        uint32_t kept = 0;
#pragma unroll
        for (int gi = 0; gi < 8 / M; ++gi) kept |= keep_bits<M>(mag, gi * M, n) << (gi * M);
        Z = kept;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t kp = (kept >> (2 * q)) & 3u;
          km[q] = ((kp & 1u) | ((kp & 2u) << 15)) * 0xFFFFu;
        }
      }

      // W_eff in bf16, two weights per word: (sign | 0x3F80) where kept and code != 0.
      uint32_t weff[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) weff[q] = ((wd[q] | 0x3F803F80u) & 0xBF80BF80u) & nz[q] & km[q];
      const uint32_t hb_lo = __byte_perm(weff[0], weff[1], 0x7531);  // high bytes of weights 0..3
      const uint32_t hb_hi = __byte_perm(weff[2], weff[3], 0x7531);  // weights 4..7

      // Every section except the tensor-core metadata is laid out in the
      // order of the 16-byte weight vectors, so vector i writes at index i.
      if (active) {
        if (M == 2) {
          const uint32_t kept = Z;
          reinterpret_cast<uint32_t*>(mask_c)[u] =
              (kept & 3u) | (((kept >> 2) & 3u) << 8) | (((kept >> 4) & 3u) << 16) | (((kept >> 6) & 3u) << 24);
        } else if (M == 4) {
          reinterpret_cast<uint16_t*>(mask_c)[u] = static_cast<uint16_t>(Z);
        } else {
          mask_c[u] = static_cast<uint8_t>(Z);
        }
        weff_c[u] = make_uint4(weff[0], weff[1], weff[2], weff[3]);
        if (codes_c != nullptr) codes_c[u] = make_uint2(codes_of_high_bytes(hb_lo), codes_of_high_bytes(hb_hi));
        if (M == 4 && spv_c != nullptr) {  // 2:4: kept values, metadata, optional decode pack
          const uint32_t vals = codes_of_high_bytes(__byte_perm(hb_lo, hb_hi, W));  // the kept codes, index order
          spv_c[u] = vals;
          // tensor-core metadata: [row_block][k_block][128 rows][16 bytes];
          // this vector's byte (its two groups' nibbles) is byte col % 16 of
          // the row's 16 bytes in k block col / 16.
          const int64_t r = row[h2];
          const int c = col[h2];
          a.out.sp_meta[(r >> 7) * meta_rb_bytes + (r & 127) * 16 + (c >> 4) * 2048 + (c & 15)] =
              static_cast<uint8_t>(Z >> 16);
          if (a.out.gemv != nullptr && !a.out.gemv_code6) {
            // per group: the two kept 2-bit codes (01 = +1, 11 = -1) low, the
            // metadata nibble high; the vector's two bytes go to its lane slot
            // of the interleaved decode pack (16-row x 128-k units of 512
            // bytes: lane (row % 8) * 4 + t holds 8 bytes of row r, then 8 of
            // row r + 8, for the groups 8t..8t+7 of the unit)
            uint32_t t = vals & 0x03030303u;
            t |= t >> 6;
            const uint32_t nibs = ((Z >> 12) & 0xF0u) | ((Z >> 8) & 0xF000u);
            const int lane_d = static_cast<int>(r & 7) * 4 + ((c >> 2) & 3);
            uint8_t* unit = a.out.gemv + ((r >> 4) * a.out.gemv_upr + (c >> 4)) * int64_t(512);
            *reinterpret_cast<uint16_t*>(unit + lane_d * 16 + ((r >> 3) & 1) * 8 + (c & 3) * 2) =
                static_cast<uint16_t>(__byte_perm(t, 0u, 0x3320) | nibs);
          }
        }
      }
      if (M == 4 && n == 2 && a.out.gemv_code6) {  // uniform per launch; gemv != nullptr
        // The 6-bit states of the vector's two groups: 9 p + 3 d0 + d1 with p
        // the rank of the kept pair (from the metadata nibble i0 | i1 << 2)
        // and d the kept codes mod 3 (the int8 code's low two bits 0, 1, 3
        // less their upper bit: 0, 1, 2).
        constexpr uint64_t kPairRank = (1ull << 32) | (2ull << 48) | (3ull << 36) | (4ull << 52) | (5ull << 56);
        const uint32_t vals = codes_of_high_bytes(__byte_perm(hb_lo, hb_hi, W));
        const uint32_t t2 = vals & 0x03030303u;
        const uint32_t d = t2 - ((t2 >> 1) & 0x01010101u);
        const uint32_t p0 = static_cast<uint32_t>(kPairRank >> (4 * ((Z >> 16) & 0xFu))) & 0xFu;
        const uint32_t p1 = static_cast<uint32_t>(kPairRank >> (4 * ((Z >> 20) & 0xFu))) & 0xFu;
        const uint32_t s0 = 9u * p0 + 3u * (d & 0xFFu) + ((d >> 8) & 0xFFu);
        const uint32_t s1 = 9u * p1 + 3u * ((d >> 16) & 0xFFu) + (d >> 24);
        const uint32_t f = active ? (s0 | (s1 << 6)) : 0u;
        // Four consecutive vectors of a row (groups 0..7 of one lane slot of
        // a unit) sit in four consecutive lanes; the first gathers their 48
        // bits and writes them: row g's to plane 0 and the low half of plane
        // 1, row g + 8's to the high half of plane 1 and plane 2.
        const uint32_t f1 = __shfl_down_sync(0xffffffffu, f, 1), f2 = __shfl_down_sync(0xffffffffu, f, 2),
                       f3 = __shfl_down_sync(0xffffffffu, f, 3);
        if (active && (lane & 3) == 0) {
          const uint64_t bits = uint64_t(f) | (uint64_t(f1) << 12) | (uint64_t(f2) << 24) | (uint64_t(f3) << 36);
          const int64_t r = row[h2];
          const int c = col[h2];
          const int lane_d = static_cast<int>(r & 7) * 4 + ((c >> 2) & 3);
          uint8_t* unit = a.out.gemv + ((r >> 4) * a.out.gemv_upr + (c >> 4)) * int64_t(384);
          uint32_t* w0 = reinterpret_cast<uint32_t*>(unit) + lane_d;
          uint16_t* w1 = reinterpret_cast<uint16_t*>(unit + 128) + 2 * lane_d;
          uint32_t* w2 = reinterpret_cast<uint32_t*>(unit + 256) + lane_d;
          if (((r >> 3) & 1) == 0) {
            *w0 = static_cast<uint32_t>(bits);
            w1[0] = static_cast<uint16_t>(bits >> 32);
          } else {
            w1[1] = static_cast<uint16_t>(bits);
            *w2 = static_cast<uint32_t>(bits >> 16);
          }
        }
      }
      if (M != 4 || n != 2) {
        if (a.out.gemv != nullptr) {  // decode pack of every pattern other than 2:4 (uniform per launch)
          // dense 2-bit codes of the 8 weights (01 = +1, 11 = -1), from the
          // high bytes of W_eff (0x3F, 0xBF or 0)
          const uint32_t t_lo = ((hb_lo >> 5) & 0x01010101u) | ((hb_lo >> 6) & 0x02020202u);
          const uint32_t t_hi = ((hb_hi >> 5) & 0x01010101u) | ((hb_hi >> 6) & 0x02020202u);
          const uint32_t d16 = ((t_lo | (t_lo >> 6) | (t_lo >> 12) | (t_lo >> 18)) & 0xFFu) |
                               (((t_hi | (t_hi >> 6) | (t_hi >> 12) | (t_hi >> 18)) & 0xFFu) << 8);
          // the block's mask byte and its kept codes in index order
          const uint32_t mb = (M == 4) ? ((Z & 0xFu) | ((Z >> 4) & 0xF0u)) : (Z & 0xFFu);
          uint32_t f = 0, pos = 0;
#pragma unroll
          for (int p = 0; p < 8; ++p) {
            if ((mb >> p) & 1u) {
              f |= ((d16 >> (2 * p)) & 3u) << pos;
              pos += 2;
            }
          }
          // Four consecutive blocks of a row (k-steps 0..3 of one lane of the
          // decode kernel) sit in four consecutive lanes here; the first
          // gathers their fields and mask bytes and writes them whole.
          const int n8 = a.out.gemv_n8;
          const uint32_t f1 = __shfl_down_sync(0xffffffffu, f, 1), f2 = __shfl_down_sync(0xffffffffu, f, 2),
                         f3 = __shfl_down_sync(0xffffffffu, f, 3);
          const uint32_t m1 = __shfl_down_sync(0xffffffffu, mb, 1), m2 = __shfl_down_sync(0xffffffffu, mb, 2),
                         m3 = __shfl_down_sync(0xffffffffu, mb, 3);
          if (active && (lane & 3) == 0) {
            const uint64_t bits = uint64_t(f) | (uint64_t(f1) << (2 * n8)) | (uint64_t(f2) << (4 * n8)) |
                                  (uint64_t(f3) << (6 * n8));
            const int64_t r = row[h2];
            const int c = col[h2];  // block of 8 within the row
            const int gq = static_cast<int>(r & 7), hi = static_cast<int>((r >> 3) & 1);
            const int lane_d = gq * 4 + ((c >> 2) & 3);
            uint8_t* unit = a.out.gemv + ((r >> 4) * a.out.gemv_upr + (c >> 4)) * int64_t(a.out.gemv_unit_bytes);
            uint8_t* code_dst = unit + lane_d * a.out.gemv_cb + hi * n8;
            if (n8 < 8) {
              *reinterpret_cast<uint32_t*>(unit + lane_d * 8 + hi * 4) = mb | (m1 << 8) | (m2 << 16) | (m3 << 24);
              code_dst += 256;
            }
            for (int b = 0; b < n8; ++b) code_dst[b] = static_cast<uint8_t>(bits >> (8 * b));
            if (hi == 1)  // the slot's bytes past both rows' fields (odd n8) are zero
              for (int b = n8; b < a.out.gemv_cb - n8; ++b) code_dst[b] = 0;
          }
        }
      }
      row[h2] += step_rows;
      col[h2] += step_cols;
      if (col[h2] >= upr) {
        col[h2] -= upr;
        ++row[h2];
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&tail->empty[s]);
  }
}

template <int M>
__global__ void __maxnreg__(72) k_prepare(const __grid_constant__ PrepArgs a) {
  prepare_body<M>(a, static_cast<int>(gridDim.x), static_cast<int>(blockIdx.x));
}

// Several matrices of one launch: matrix i runs on CTAs
// [cta_begin[i], cta_begin[i + 1]), with its own tagged barrier (in its own
// blob) and its own exact scale.
struct PrepGroup {
  PrepArgs mats[kPrepMaxGroup];
  int cta_begin[kPrepMaxGroup + 1];
  int count;
};

template <int M>
__global__ void __maxnreg__(72) k_prepare_group(const __grid_constant__ PrepGroup grp) {
  const int b = static_cast<int>(blockIdx.x);
  int i = 0;
  while (i + 1 < grp.count && b >= grp.cta_begin[i + 1]) ++i;
  prepare_body<M>(grp.mats[i], grp.cta_begin[i + 1] - grp.cta_begin[i], b - grp.cta_begin[i]);
}

// ---------------------------------------------------------------------------
// Host launcher
// ---------------------------------------------------------------------------
template <int M>
static cudaError_t launch_prepare_m(const cudaLaunchConfig_t& cfg, const PrepArgs& a) {
  static const cudaError_t attr_err =
      cudaFuncSetAttribute(k_prepare<M>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kPrepSmem));
  if (attr_err != cudaSuccess) return attr_err;
  return counted(cudaLaunchKernelEx(&cfg, k_prepare<M>, a));
}

template <int M>
static cudaError_t launch_prepare_group_m(const cudaLaunchConfig_t& cfg, const PrepGroup& grp) {
  static const cudaError_t attr_err = cudaFuncSetAttribute(k_prepare_group<M>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                           static_cast<int>(kPrepSmem));
  if (attr_err != cudaSuccess) return attr_err;
  return counted(cudaLaunchKernelEx(&cfg, k_prepare_group<M>, grp));
}

static_assert(3 + kExactBins + 3 == SBL_SUM_WORDS, "sum words: fast pieces, bins, counts");

// The arguments of one matrix's preparation, after the stream operations
// that must precede it (padding of the metadata and decode-pack sections).
static cudaError_t prep_args(const uint16_t* w, int64_t n_out, int64_t k, int n, int m, uint32_t flags,
                             uint8_t* blob, const sbl_blob_layout& L, cudaStream_t s, int mode, uint64_t* sum_out,
                             const uint64_t* sum_in, uint64_t numel, PrepArgs& a) {
  if (mode != kPrepSumOnly && L.sp_meta && (n_out % 256 != 0 || k % 256 != 0)) {
    cudaError_t e = cudaMemsetAsync(blob + L.sp_meta, 0x44, L.sp_meta_bytes, s);
    if (e != cudaSuccess) return e;
  }
  a.w = reinterpret_cast<const uint4*>(w);
  a.n_out = n_out;
  a.k = k;
  a.mode = mode;
  a.numel = numel;
  a.sum_out = sum_out;
  a.sum_in = sum_in;
  a.n = n;
  a.m = m;
  a.layer_flags = flags;
  a.h = reinterpret_cast<BlobHeader*>(blob + L.header);
  a.slot_fast = reinterpret_cast<uint64_t*>(blob + L.scratch + kScratchSlotFast);
  a.slot_bins = reinterpret_cast<uint64_t*>(blob + L.scratch + kScratchSlotBins);
  a.gen = reinterpret_cast<uint64_t*>(blob + L.scratch + kScratchGen);
  a.out.mask_from_codes = (flags & SBL_MASK_FROM_QUANT) ? 1 : 0;
  a.out.mask = blob + L.mask;
  a.out.codes = L.codes ? reinterpret_cast<int8_t*>(blob + L.codes) : nullptr;
  a.out.weff_bf16 = reinterpret_cast<uint16_t*>(blob + L.weff_bf16);
  a.out.sp_values = L.sp_values ? reinterpret_cast<int8_t*>(blob + L.sp_values) : nullptr;
  a.out.sp_meta = L.sp_meta ? blob + L.sp_meta : nullptr;
  a.out.gemv = L.gemv ? blob + L.gemv : nullptr;
  a.out.meta_kblocks = static_cast<int>(meta_k_padded(k) / 128);
  a.out.gemv_n8 = 8 * n / m;
  a.out.gemv_cb = (2 * a.out.gemv_n8 + 3) / 4 * 4;
  a.out.gemv_unit_bytes = (a.out.gemv_n8 < 8 ? 256 : 0) + 32 * a.out.gemv_cb;
  a.out.gemv_upr = static_cast<int>((k + 127) / 128);
  a.out.gemv_code6 = (L.gemv != 0 && (flags & SBL_PACK_GEMV_6BIT)) ? 1 : 0;
  if (mode != kPrepSumOnly && L.gemv && (n_out % 16 != 0 || k % 128 != 0)) {
    // the interleaved pack covers whole 16-row, 128-k units: what no weight
    // fills is zero
    cudaError_t e = cudaMemsetAsync(blob + L.gemv, 0, L.gemv_bytes, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

static cudaLaunchConfig_t prep_config(int64_t grid, cudaStream_t s, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kPrepThreads);
  cfg.dynamicSmemBytes = kPrepSmem;
  cfg.stream = s;
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

// CTAs that a matrix of nvec 16-byte vectors can use: at least one stage of
// weights each.
static int64_t prep_max_ctas(int64_t nvec) {
  const int64_t c = (nvec + kChunkVecs - 1) / kChunkVecs;
  return c < 1 ? 1 : c > kPrepSlots ? kPrepSlots : c;
}

cudaError_t launch_prepare(const uint16_t* w, int64_t n_out, int64_t k, int n, int m, uint32_t flags,
                           uint8_t* blob, const sbl_blob_layout& L, int num_sms, cudaStream_t s, int mode,
                           uint64_t* sum_out, const uint64_t* sum_in, uint64_t numel) {
  PrepArgs a;
  cudaError_t e = prep_args(w, n_out, k, n, m, flags, blob, L, s, mode, sum_out, sum_in, numel, a);
  if (e != cudaSuccess) return e;
  // One CTA per SM (fewer for small matrices), all resident at once for the
  // grid barrier.
  int64_t grid = prep_max_ctas(n_out * k / 8);
  if (grid > num_sms) grid = num_sms;
  cudaLaunchAttribute attr[1];
  const cudaLaunchConfig_t cfg = prep_config(grid, s, attr);
  switch (m) {
    case 2: return launch_prepare_m<2>(cfg, a);
    case 4: return launch_prepare_m<4>(cfg, a);
    default: return launch_prepare_m<8>(cfg, a);
  }
}

cudaError_t launch_prepare_group(const PrepMatrix* mats, int count, int num_sms, cudaStream_t s) {
  if (count < 1 || count > kPrepMaxGroup || count > num_sms) return cudaErrorInvalidValue;
  PrepGroup grp;
  grp.count = count;
  int64_t nvec[kPrepMaxGroup], total = 0;
  for (int i = 0; i < count; ++i) {
    const PrepMatrix& q = mats[i];
    if (q.m != mats[0].m) return cudaErrorInvalidValue;
    cudaError_t e = prep_args(q.w, q.n_out, q.k, q.n, q.m, q.flags, q.blob, *q.layout, s, 0, nullptr, nullptr,
                              uint64_t(q.n_out) * uint64_t(q.k), grp.mats[i]);
    if (e != cudaSuccess) return e;
    nvec[i] = q.n_out * q.k / 8;
    total += nvec[i];
  }
  // The SMs split in proportion to the matrices' sizes, at least one CTA each.
  int ctas[kPrepMaxGroup], used = 0;
  for (int i = 0; i < count; ++i) {
    int64_t c = (nvec[i] * (num_sms - count)) / total + 1;
    const int64_t cap = prep_max_ctas(nvec[i]);
    ctas[i] = static_cast<int>(c < cap ? c : cap);
    used += ctas[i];
  }
  grp.cta_begin[0] = 0;
  for (int i = 0; i < count; ++i) grp.cta_begin[i + 1] = grp.cta_begin[i] + ctas[i];
  for (int i = count + 1; i <= kPrepMaxGroup; ++i) grp.cta_begin[i] = grp.cta_begin[count];
  cudaLaunchAttribute attr[1];
  const cudaLaunchConfig_t cfg = prep_config(used, s, attr);
  switch (mats[0].m) {
    case 2: return launch_prepare_group_m<2>(cfg, grp);
    case 4: return launch_prepare_group_m<4>(cfg, grp);
    default: return launch_prepare_group_m<8>(cfg, grp);
  }
}

}  // namespace sbl
