// Weight preparation for Sparse-BitLinear: exact absmean scale, N:M mask from
// the master magnitudes, ternary codes with the mask applied after
// quantisation, and the packed forms the GEMM kernels read.
//
// Paper: "Sparse-BitNet: 1.58-bit LLMs are Naturally Friendly to
// Semi-Structured Sparsity" -- gist.science German technical summary §2
// (magnitude mask from the masters, quantise then mask), Korean summary
// §2.1-2.2 (per-step recompute), French summary §2.
#include "sbl_kernels.h"

#include "sbl_device.cuh"

namespace sbl {

// ---------------------------------------------------------------------------
// Header reset: shapes, zeroed exact-sum bins, cleared status.
// ---------------------------------------------------------------------------
__global__ void k_prep_header(BlobHeader* h, int64_t n_out, int64_t k, int n, int m, uint32_t flags) {
  const int i = threadIdx.x;
  if (i < 32) h->bins[i] = 0ull;
  if (i == 0) {
    h->magic = kMagic;
    h->version = 1;
    h->n_out = n_out;
    h->k = k;
    h->n = n;
    h->m = m;
    h->flags = flags;
    h->gamma = 0.0f;
    h->g = 0.0f;
    h->status = 0u;
  }
}

// ---------------------------------------------------------------------------
// Exact sum of |w| (absmean numerator).
//
// In units of 2^-133 a bf16 magnitude (biased exponent e, mantissa f) is the
// integer sig << s with sig = (e ? 128 + f : f) and s = max(e, 1) - 1.  Each
// lane keeps 32 private 32-bit bins in shared memory, bin b = s >> 3 holding
// sum(sig << (s & 7)) (< 2^15 per add, so 2^17 adds per lane cannot
// overflow); the block folds its bins into 64-bit global bins.  The exact
// total is sum_b bins[b] << 8b, formed in k_gamma_finalize.
// ---------------------------------------------------------------------------
constexpr int kBinWarps = 8;

__global__ void __launch_bounds__(kBinWarps * 32) k_absmean_bins(const uint4* __restrict__ w, int64_t nvec,
                                                                 BlobHeader* h) {
  __shared__ uint32_t bins[kBinWarps][32][32];  // [warp][bin][lane]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int b = 0; b < 32; ++b) bins[warp][b][lane] = 0u;

  uint32_t bad = 0;
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  auto consume = [&](const uint4 v) {
    const uint32_t words[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t mag = (words[j >> 1] >> (16 * (j & 1))) & 0x7FFFu;
      const uint32_t e = mag >> 7;
      bad |= (e == 0xFFu);
      const uint32_t sig = (mag & 0x7Fu) | (e ? 0x80u : 0u);
      const uint32_t s = (e ? e : 1u) - 1u;
      bins[warp][(s >> 3) & 31u][lane] += sig << (s & 7u);
    }
  };
  // Four independent 16-byte loads in flight per thread.
  for (; i + 3 * stride < nvec; i += 4 * stride) {
    // default caching: the pack pass re-reads W right after this one
    const uint4 v0 = __ldg(w + i);
    const uint4 v1 = __ldg(w + i + stride);
    const uint4 v2 = __ldg(w + i + 2 * stride);
    const uint4 v3 = __ldg(w + i + 3 * stride);
    consume(v0);
    consume(v1);
    consume(v2);
    consume(v3);
  }
  for (; i < nvec; i += stride) consume(__ldg(w + i));

  __syncthreads();
  // Thread (bin = tid / 8, part = tid % 8) sums warp `part`'s 32 lanes of that bin.
  const int bin = threadIdx.x >> 3, part = threadIdx.x & 7;
  unsigned long long sum = 0ull;
#pragma unroll 4
  for (int l = 0; l < 32; ++l) sum += bins[part][bin][(l + lane) & 31];
  sum += __shfl_down_sync(0xffffffffu, sum, 4, 8);
  sum += __shfl_down_sync(0xffffffffu, sum, 2, 8);
  sum += __shfl_down_sync(0xffffffffu, sum, 1, 8);
  if (part == 0 && sum != 0ull) atomicAdd(&h->bins[bin], sum);
  if (__any_sync(0xffffffffu, bad != 0) && lane == 0) atomicOr(&h->status, SBL_STATUS_NONFINITE_W);
}

// ---------------------------------------------------------------------------
// gamma = RN_fp32(S * 2^-133 / numel), S = sum_b bins[b] << 8b (exact).
// Limb-wise long division of S * 2^128 by numel, then nearest-even rounding
// of the quotient to fp32 (normal or subnormal) from its bits plus sticky.
// ---------------------------------------------------------------------------
__device__ void add_limb(uint64_t* x, int nlimbs, int i, uint64_t v) {
  while (v != 0ull && i < nlimbs) {
    const uint64_t before = x[i];
    x[i] += v;
    v = (x[i] < before) ? 1ull : 0ull;
    ++i;
  }
}

__global__ void k_gamma_finalize(BlobHeader* h, int64_t numel) {
  if (threadIdx.x != 0) return;
  // X = S << 128 in seven 64-bit limbs (S < 2^312).
  uint64_t X[7] = {0, 0, 0, 0, 0, 0, 0};
  for (int b = 0; b < 32; ++b) {
    const uint64_t v = h->bins[b];
    if (v == 0ull) continue;
    const int shift = 8 * b + 128;
    const int li = shift >> 6, off = shift & 63;
    add_limb(X, 7, li, v << off);
    if (off != 0) add_limb(X, 7, li + 1, v >> (64 - off));
  }
  float gamma = 0.0f;
  bool nonzero = false;
  for (int i = 0; i < 7; ++i) nonzero |= (X[i] != 0ull);
  if (h->status & SBL_STATUS_NONFINITE_W) {
    gamma = __int_as_float(0x7fc00000);
  } else if (nonzero) {
    const uint64_t n = static_cast<uint64_t>(numel);
    uint64_t Q[7];
    unsigned __int128 rem = 0;
    for (int i = 6; i >= 0; --i) {
      const unsigned __int128 cur = (rem << 64) | X[i];
      Q[i] = static_cast<uint64_t>(cur / n);
      rem = cur % n;
    }
    // Q = floor(S * 2^128 / n); bit j of Q has real weight 2^(j - 261).
    int top = -1;
    for (int i = 6; i >= 0 && top < 0; --i)
      if (Q[i]) top = 64 * i + 63 - __clzll(static_cast<long long>(Q[i]));
    auto qbit = [&](int j) -> uint32_t { return static_cast<uint32_t>((Q[j >> 6] >> (j & 63)) & 1ull); };
    const int e = top - 261;
    const int lsb = max(e - 23, -149);
    const int lsb_pos = lsb + 261;  // >= 112
    uint32_t mant = 0;
    for (int j = top; j >= lsb_pos; --j) mant = (mant << 1) | qbit(j);
    const uint32_t round_bit = qbit(lsb_pos - 1);
    bool sticky = (rem != 0);
    for (int j = lsb_pos - 2; j >= 0 && !sticky; --j) sticky = qbit(j) != 0u;
    if (round_bit && (sticky || (mant & 1u))) ++mant;
    // value = mant * 2^lsb; the pattern below covers subnormals and the carry.
    gamma = __uint_as_float((static_cast<uint32_t>(lsb + 149) << 23) + mant);
  }
  h->gamma = gamma;
  h->g = (gamma > 1e-5f) ? gamma : 1e-5f;  // NaN gamma gives 1e-5; the status word says why
}

// ---------------------------------------------------------------------------
// Mask, ternarise, pack.  One thread per 32 consecutive weights of a row.
// ---------------------------------------------------------------------------
template <int M>
__global__ void __launch_bounds__(256) k_prep_pack(const uint16_t* __restrict__ w, int64_t n_out, int64_t k, int n,
                                                   const BlobHeader* __restrict__ h, PackOut out) {
  const float g = h->g;
  const int64_t chunks_per_row = k / 32;
  const int64_t total = n_out * chunks_per_row;
  for (int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = idx / chunks_per_row, c = idx % chunks_per_row;
    const uint4* src = reinterpret_cast<const uint4*>(w + r * k + 32 * c);
    uint32_t wv[16];
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const uint4 x = __ldcs(src + v);
      wv[4 * v + 0] = x.x;
      wv[4 * v + 1] = x.y;
      wv[4 * v + 2] = x.z;
      wv[4 * v + 3] = x.w;
    }
    auto bits_of = [&](int j) -> uint32_t { return (wv[j >> 1] >> (16 * (j & 1))) & 0xFFFFu; };

    // Ternary code of every weight: sign(w) when 2|w| > g (exact fp32), else 0.
    int code[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const uint32_t b = bits_of(j);
      const float v = __uint_as_float(b << 16);
      code[j] = (__fmul_rn(2.0f, fabsf(v)) > g) ? ((b & 0x8000u) ? -1 : 1) : 0;
    }
    // N:M selection on the magnitude bits: keep rank < n, where rank counts
    // larger magnitudes plus equal ones at lower index.
    uint32_t kept = 0;  // bit j: weight j of the chunk is kept
#pragma unroll
    for (int gi = 0; gi < 32 / M; ++gi) {
#pragma unroll
      for (int a = 0; a < M; ++a) {
        const uint32_t ka = bits_of(gi * M + a) & 0x7FFFu;
        int rank = 0;
#pragma unroll
        for (int b = 0; b < M; ++b) {
          if (b == a) continue;
          const uint32_t kb = bits_of(gi * M + b) & 0x7FFFu;
          rank += (kb > ka) || (kb == ka && b < a);
        }
        if (rank < n) kept |= 1u << (gi * M + a);
      }
    }

    // mask bytes: 32/M groups, each M bits
    {
      uint8_t mb[32 / M];
#pragma unroll
      for (int gi = 0; gi < 32 / M; ++gi) mb[gi] = static_cast<uint8_t>((kept >> (gi * M)) & ((1u << M) - 1u));
      uint8_t* dst = out.mask + r * (k / M) + c * (32 / M);
#pragma unroll
      for (int gi = 0; gi < 32 / M; ++gi) dst[gi] = mb[gi];
    }
    // W_eff as exact bf16 (+1 = 0x3F80, -1 = 0xBF80, 0)
    {
      uint32_t pk[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        uint32_t lo = 0, hi = 0;
        const int c0 = (kept >> (2 * j)) & 1u ? code[2 * j] : 0;
        const int c1 = (kept >> (2 * j + 1)) & 1u ? code[2 * j + 1] : 0;
        lo = c0 == 0 ? 0u : (c0 > 0 ? 0x3F80u : 0xBF80u);
        hi = c1 == 0 ? 0u : (c1 > 0 ? 0x3F80u : 0xBF80u);
        pk[j] = lo | (hi << 16);
      }
      uint4* dst = reinterpret_cast<uint4*>(out.weff_bf16 + r * k + 32 * c);
#pragma unroll
      for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
    }
    if (out.codes != nullptr) {  // dense int8 W_eff codes
      uint32_t pk[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t word = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int idx2 = 4 * j + e;
          const int cv = ((kept >> idx2) & 1u) ? code[idx2] : 0;
          word |= (static_cast<uint32_t>(cv) & 0xFFu) << (8 * e);
        }
        pk[j] = word;
      }
      uint4* dst = reinterpret_cast<uint4*>(out.codes + r * k + 32 * c);
      dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
    if (M == 4 && out.sp_values != nullptr) {  // 2:4: kept values, metadata, optional GEMV bytes
      uint32_t vals[4] = {0, 0, 0, 0};
      uint32_t meta = 0;
      uint32_t gemv[2] = {0, 0};
#pragma unroll
      for (int gi = 0; gi < 8; ++gi) {
        const uint32_t bits = (kept >> (4 * gi)) & 0xFu;
        // two lowest set bits, ascending (exactly two are set for n == 2)
        const int i0 = __ffs(bits) - 1;
        const int i1 = __ffs(bits & (bits - 1u)) - 1;
        const int v0 = code[4 * gi + i0], v1 = code[4 * gi + i1];
        const uint32_t nib = uint32_t(i0) | (uint32_t(i1) << 2);
        meta |= nib << (4 * gi);
        vals[gi >> 1] |= ((uint32_t(v0) & 0xFFu) | ((uint32_t(v1) & 0xFFu) << 8)) << (16 * (gi & 1));
        const uint32_t gb = (nib << 4) | (uint32_t(v0) & 3u) | ((uint32_t(v1) & 3u) << 2);
        gemv[gi >> 2] |= gb << (8 * (gi & 3));
      }
      *reinterpret_cast<uint4*>(out.sp_values + r * (k / 2) + 16 * c) = make_uint4(vals[0], vals[1], vals[2], vals[3]);
      // tensor-core metadata: [row_block][k_block][128 rows][16 bytes]
      const int64_t rb = r >> 7, rr = r & 127;
      const int64_t kblk = (32 * c) >> 7;
      const int64_t byte_in_row = ((32 * c) & 127) >> 3;  // 4 bytes per 32 weights
      uint8_t* mdst = out.sp_meta + ((rb * out.meta_kblocks + kblk) * 128 + rr) * 16 + byte_in_row;
      *reinterpret_cast<uint32_t*>(mdst) = meta;
      if (out.gemv != nullptr)
        *reinterpret_cast<uint2*>(out.gemv + r * (k / 4) + 8 * c) = make_uint2(gemv[0], gemv[1]);
    }
  }
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
cudaError_t launch_prepare(const uint16_t* w, int64_t n_out, int64_t k, int n, int m, uint32_t flags,
                           uint8_t* blob, const sbl_blob_layout& L, int num_sms, cudaStream_t s) {
  BlobHeader* h = reinterpret_cast<BlobHeader*>(blob + L.header);
  k_prep_header<<<1, 64, 0, s>>>(h, n_out, k, n, m, flags);
  if (L.sp_meta && (n_out % 128 != 0 || k % 256 != 0)) {
    cudaError_t e = cudaMemsetAsync(blob + L.sp_meta, 0x44, L.sp_meta_bytes, s);
    if (e != cudaSuccess) return e;
  }
  const int64_t numel = n_out * k;
  const int64_t nvec = numel / 8;
  // Enough blocks that no lane adds more than 2^16 weights into one bin.
  int64_t blocks = int64_t(num_sms) * 2;
  const int64_t min_blocks = (numel + (int64_t(256) << 16) - 1) / (int64_t(256) << 16);
  if (blocks < min_blocks) blocks = min_blocks;
  k_absmean_bins<<<static_cast<unsigned>(blocks), kBinWarps * 32, 0, s>>>(reinterpret_cast<const uint4*>(w), nvec, h);
  k_gamma_finalize<<<1, 32, 0, s>>>(h, numel);

  PackOut out;
  out.mask = blob + L.mask;
  out.codes = L.codes ? reinterpret_cast<int8_t*>(blob + L.codes) : nullptr;
  out.weff_bf16 = reinterpret_cast<uint16_t*>(blob + L.weff_bf16);
  out.sp_values = L.sp_values ? reinterpret_cast<int8_t*>(blob + L.sp_values) : nullptr;
  out.sp_meta = L.sp_meta ? blob + L.sp_meta : nullptr;
  out.gemv = L.gemv ? blob + L.gemv : nullptr;
  out.meta_kblocks = static_cast<int>(meta_k_padded(k) / 128);
  const int64_t chunks = n_out * (k / 32);
  const int64_t pblocks = (chunks + 255) / 256;
  const unsigned grid = static_cast<unsigned>(pblocks < int64_t(num_sms) * 64 ? pblocks : int64_t(num_sms) * 64);
  switch (m) {
    case 2: k_prep_pack<2><<<grid, 256, 0, s>>>(w, n_out, k, n, h, out); break;
    case 4: k_prep_pack<4><<<grid, 256, 0, s>>>(w, n_out, k, n, h, out); break;
    default: k_prep_pack<8><<<grid, 256, 0, s>>>(w, n_out, k, n, h, out); break;
  }
  return cudaGetLastError();
}

}  // namespace sbl
