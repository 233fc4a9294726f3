// Decode-shaped forward (t <= 32 tokens) over the packed weights.
//
// At these token counts the weight stream is the whole cost, so the weights
// travel packed and are expanded to int8 in registers, straight into the
// operand fragments of the warp-level int8 tensor-core instruction
// (mma.sync m16n8k32: 16 weight rows x 8 tokens x 32 k per instruction).
// That instruction takes its operands from registers, so the expansion never
// goes through shared memory, and a block needs no tensor-memory allocation
// or barrier round trip on a kernel whose whole budget is a few microseconds.
//
// Work: the rows are cut into tiles of 16, a tile's k into units of 128.  A
// block owns whole tiles (so every sum closes inside the block) and its warps
// split the block's (tile, unit) pairs evenly.  In a unit, lane (g, t) (g =
// lane / 4, t = lane % 4) handles rows g and g + 8 and the 32 consecutive k
// from 32t: k-step s of the unit covers its 8 weights 32t + 8s .. 32t + 8s + 7,
// whose first four fill the fragment slots 4t..4t+3 and the last four the
// slots 16 + 4t..16 + 4t + 3.  The activation fragments follow the same
// permutation of k, so every product meets the right activation; a lane's
// activation bytes for one k-step are 8 consecutive codes.
//
// Weight packs:
//   2:4 (the 2-bit decode packing): one byte per group of four, the metadata
//       nibble high and the two kept codes low, interleaved by unit and lane:
//       a unit is 512 bytes, lane * 16 holding the 8 group bytes of row g
//       (groups 8t..8t+7 of the unit) and then the 8 of row g + 8, so a lane
//       reads one 16-byte piece per unit and a warp 512 contiguous bytes; a
//       256-entry table expands a byte into the group's four int8 weights.
//   2:4, 6-bit group code (1.5 bits a weight): a group's kept pair p (0..5,
//       lexicographic) and its two codes as digits mod 3 form the state
//       9 p + 3 d0 + d1 < 54.  A lane's 16 states of a unit (row g groups
//       8t..8t+7, then row g + 8) are 96 bits, least significant first, held
//       as three words; word j of every lane forms the unit's j-th 128-byte
//       plane, so each of a lane's three loads is one coalesced 128-byte row
//       for the warp (a unit is 384 bytes).  A 64-entry table expands a state.
//   any other N:M (compressed index): per block of 8 weights a mask byte and
//       the n8 = 8n/m kept 2-bit codes in index order.  The section is
//       interleaved by unit and lane so that a lane's mask bytes and code bits
//       are contiguous: per unit a 256-byte mask block (lane * 8: row g's four
//       blocks, then row g + 8's) and a code block (lane * cb bytes: row g's
//       four fields of 2 n8 bits, then row g + 8's).  Expansion: a table turns
//       each byte of codes into four int8 values in index order, and a second
//       table turns the mask byte into the byte-permute selectors that scatter
//       them onto the kept positions (pruned positions pick a zero byte).
//       n = m (dense ternary) drops the mask block.
//
// Calls are launched with programmatic dependent launch: before the wait for
// its predecessor a block builds its tables, clears its partial sums and
// prefetches its weight bytes into L2 (the prefetch is safe even right after
// a prepare: L2 is the coherence point, so a later write is never hidden),
// and lets the next call launch; in a chain of decode calls the weight stream
// of one call overlaps the call before it.  After the wait the block issues
// its weight loads, quantises its token rows into shared memory (t <= 4) or
// copies the codes the act-quant kernel wrote, and runs the products.  Partial
// sums of warps sharing a tile are added in shared memory (exact integer
// adds, any order); y = acc * ((g a') / 127) closes the block.
#include <mutex>

#include "sbl_kernels.h"

#include "actq_math.cuh"
#include "sbl_device.cuh"

namespace sbl {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;
// A table of 256 entries kept in C copies, entry e of copy c at word
// e * C + c; lane l reads copy l % C, so at most 32 / C lanes share a copy's
// banks.  16 copies measured best: 32 doubled the table fill before the wait
// (which competes with the call before) for no gain in the products.
constexpr int kLutCopiesReg = 16;
constexpr int lut_words(int copies, int entries = 256) { return entries * copies; }
constexpr int kDecBatch = 8;         // units whose weight bytes a lane holds at once
constexpr size_t kDecMaxSmem = 227 * 1024;
constexpr int kDecMaxT = 32;
constexpr int kFusedMaxT = 4;  // token counts the kernel quantises itself

struct DecodeArgs {
  const uint8_t* w;      // weight pack
  const uint4* x;        // bf16 [t][k/8] (quantised here)
  const int8_t* xq_in;   // int8 [t][k] from the act-quant kernel (else)
  const float* ap_in;
  const float* g;
  float* y;
  int32_t* acc_out;
  int8_t* xq_out;        // optional, when quantised here
  float* ap_out;
  uint32_t* status;
  int n_out, t, k;
  int tiles, upr, tpb;   // 16-row tiles, 128-k units per row, tiles per block
  int nfull;             // blocks [0, nfull) take tpb tiles, later ones tpb - 1
  int xs;                // shared-memory row stride of the codes (multiple of 128)
};

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// The exact-division form of the quantiser, out of line: it runs only for a
// row whose a' is the 1e-5 clamp or huge, and kept out of the fast path's
// instruction stream.
__device__ __noinline__ uint4 quantise16_div(uint4 v0, uint4 v1, float ap) {
  const uint2 c0 = quantise8_div(v0, ap), c1 = quantise8_div(v1, ap);
  return make_uint4(c0.x, c0.y, c1.x, c1.y);
}

__device__ __forceinline__ uint4 quantise16(const uint4& v0, const uint4& v1, const QScale& qs) {
  if (qs.exact) return quantise16_div(v0, v1, qs.ap);
  const uint2 c0 = quantise8_fma(v0, qs.c), c1 = quantise8_fma(v1, qs.c);
  return make_uint4(c0.x, c0.y, c1.x, c1.y);
}

__device__ __forceinline__ void mma_s8_16x8x32(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  // a pure register operation: no volatile, so the compiler may interleave it
  // with the table loads of the next k-step
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// int8 value of a 2-bit code: 01 = +1, 11 = -1, 00 (and the unused 10) = 0.
__host__ __device__ constexpr uint32_t code_byte(uint32_t c) { return c == 1u ? 0x01u : c == 3u ? 0xFFu : 0u; }

// Table entries.  kind 0: a 2:4 decode byte -> the group's four weights;
// kind 1: a byte of four codes -> four int8 values in index order; kind 2: a
// mask byte -> two byte-permute selectors (positions 0-3 in the low half,
// 4-7 in the high half): a kept position picks its rank among the kept
// values, a pruned one byte 7 (zero whenever fewer than 8 are kept); kind 3:
// a 6-bit group state -> the group's four weights (states 54..63 unused).
__device__ __forceinline__ uint32_t lut_entry(int kind, uint32_t b) {
  if (kind == 3) {
    if (b >= 54u) return 0u;
    const uint32_t p = b / 9u, d0 = (b / 3u) % 3u, d1 = b % 3u;
    const uint32_t i0 = p < 3u ? 0u : (p < 5u ? 1u : 2u);
    const uint32_t i1 = p < 3u ? p + 1u : (p < 5u ? p - 1u : 3u);
    auto digit = [](uint32_t d) { return d == 1u ? 0x01u : d == 2u ? 0xFFu : 0u; };
    return (digit(d0) << (8 * i0)) | (digit(d1) << (8 * i1));
  }
  if (kind == 0) {
    const uint32_t i0 = (b >> 4) & 3u, i1 = (b >> 6) & 3u;
    return (code_byte(b & 3u) << (8 * i0)) | (code_byte((b >> 2) & 3u) << (8 * i1));
  }
  if (kind == 1)
    return code_byte(b & 3u) | (code_byte((b >> 2) & 3u) << 8) | (code_byte((b >> 4) & 3u) << 16) |
           (code_byte((b >> 6) & 3u) << 24);
  uint32_t sel = 0;
  for (int p = 0; p < 8; ++p) {
    const uint32_t nib = ((b >> p) & 1u) ? static_cast<uint32_t>(__popc(b & ((1u << p) - 1u))) : 7u;
    sel |= nib << (4 * p);
  }
  return sel;
}

template <int C>
__device__ __forceinline__ void fill_lut(uint32_t* lut, int kind, int tid, int entries = 256) {
  constexpr int kVecs = C / 4;  // 16-byte stores per entry
  for (int i = tid; i < entries * kVecs; i += kDecThreads) {
    const uint32_t v = lut_entry(kind, static_cast<uint32_t>(i / kVecs));
    reinterpret_cast<uint4*>(lut)[i] = make_uint4(v, v, v, v);
  }
}

// Compile-time facts of a weight pack.  FMT 0: 2:4 bytes; FMT 1..8: blocks of
// 8 with FMT kept codes (8 = dense, no mask block); FMT 9: 2:4 6-bit states.
constexpr int kFmtCode6 = 9;
template <int FMT>
struct Pack {
  static constexpr bool k24 = FMT == 0;
  static constexpr bool c6 = FMT == kFmtCode6;
  static constexpr int n8 = FMT;
  static constexpr bool has_mask = FMT >= 1 && FMT < 8;
  static constexpr int cb = (k24 || c6) ? 0 : (2 * FMT + 3) / 4 * 4;  // code bytes per lane and unit
  static constexpr int cw = cb / 4;
  static constexpr int unit_bytes = k24 ? 512 : c6 ? 384 : (has_mask ? 256 : 0) + 32 * cb;
  static constexpr int regs = k24 ? 4 : c6 ? 3 : (has_mask ? 2 : 0) + cw;  // words a lane loads per unit
  static constexpr int lut_entries = c6 ? 64 : 256;
  static constexpr int lut_kind = k24 ? 0 : c6 ? 3 : 1;
};

// One unit's weight words of this lane.
template <int FMT>
__device__ __forceinline__ void load_unit(const DecodeArgs& a, int tile, int u, int lane,
                                          uint32_t (&r)[Pack<FMT>::regs]) {
  using P = Pack<FMT>;
  if constexpr (P::k24) {
    // one 16-byte piece: 8 group bytes of row g, then 8 of row g + 8
    const uint4 v = __ldcs(reinterpret_cast<const uint4*>(a.w + (int64_t(tile) * a.upr + u) * P::unit_bytes) + lane);
    r[0] = v.x;
    r[1] = v.y;
    r[2] = v.z;
    r[3] = v.w;
  } else if constexpr (P::c6) {
    // word j of the lane's 96 state bits from plane j of the unit
    const uint32_t* base = reinterpret_cast<const uint32_t*>(a.w + (int64_t(tile) * a.upr + u) * P::unit_bytes);
#pragma unroll
    for (int j = 0; j < 3; ++j) r[j] = __ldcs(base + 32 * j + lane);
  } else {
    const uint8_t* base = a.w + (int64_t(tile) * a.upr + u) * P::unit_bytes;
    int o = 0;
    if constexpr (P::has_mask) {
      const uint2 mk = __ldcs(reinterpret_cast<const uint2*>(base + lane * 8));
      r[0] = mk.x;
      r[1] = mk.y;
      o = 2;
      base += 256;
    }
    const uint32_t* cw = reinterpret_cast<const uint32_t*>(base + lane * P::cb);
    if constexpr (P::cw == 4) {
      const uint4 v = __ldcs(reinterpret_cast<const uint4*>(cw));
      r[o] = v.x;
      r[o + 1] = v.y;
      r[o + 2] = v.z;
      r[o + 3] = v.w;
    } else if constexpr (P::cw == 2) {
      const uint2 v = __ldcs(reinterpret_cast<const uint2*>(cw));
      r[o] = v.x;
      r[o + 1] = v.y;
    } else {
#pragma unroll
      for (int i = 0; i < P::cw; ++i) r[o + i] = __ldcs(cw + i);
    }
  }
}

// Bits [off, off + bits) of the lane's code words (off, bits compile-time
// after unrolling; bits <= 16).
template <int CW>
__device__ __forceinline__ uint32_t code_field(const uint32_t* w, int off, int bits) {
  const int wi = off >> 5, sh = off & 31;
  uint32_t v = w[wi] >> sh;
  if (sh + bits > 32) v |= w[wi + 1] << (32 - sh);
  return bits == 32 ? v : (v & ((1u << bits) - 1u));
}

// Table entry (byte `pos` of w) in this lane's copy: the byte, shifted
// straight into a byte offset (entries are 4 * C bytes apart).
template <int C>
__device__ __forceinline__ uint32_t lut_get(const uint8_t* lane_base, uint32_t w, int pos) {
  constexpr int kShift = 2 + (C == 16 ? 4 : C == 32 ? 5 : 3);
  static_assert(C == 8 || C == 16 || C == 32, "table copies");
  const int sh = 8 * pos - kShift;
  const uint32_t off = (sh >= 0 ? (w >> sh) : (w << -sh)) & (0xFFu << kShift);
  return *reinterpret_cast<const uint32_t*>(lane_base + off);
}

// Table entry of the 6-bit state at bit `off` of the lane's words (off
// compile-time after unrolling), shifted straight into a byte offset.
template <int C>
__device__ __forceinline__ uint32_t lut_get6(const uint8_t* lane_base, const uint32_t* w, int off) {
  constexpr int kShift = 2 + (C == 16 ? 4 : C == 32 ? 5 : 3);
  const int wi = off >> 5, sh = (off & 31) - kShift;
  uint32_t v = sh >= 0 ? (w[wi] >> sh) : (w[wi] << -sh);
  if ((off & 31) + 6 > 32) v |= w[wi + 1] << (32 - sh);
  return *reinterpret_cast<const uint32_t*>(lane_base + (v & (0x3Fu << kShift)));
}

// The four A-fragment registers of k-step s: rows g (a0 low k slots, a2 high)
// and g + 8 (a1, a3).  la / ls: this lane's copies of the tables.
template <int FMT, int C>
__device__ __forceinline__ void decode_step(const uint32_t (&r)[Pack<FMT>::regs], int s, const uint8_t* la,
                                            const uint8_t* ls, uint32_t& a0, uint32_t& a1, uint32_t& a2, uint32_t& a3) {
  using P = Pack<FMT>;
  if constexpr (P::k24) {
    // bytes 2s, 2s + 1 of each row's 8: word s / 2, bytes 2 (s % 2) and + 1
    const int b = 2 * (s & 1);
    const uint32_t w0 = r[s >> 1], w1 = r[2 + (s >> 1)];
    a0 = lut_get<C>(la, w0, b);
    a2 = lut_get<C>(la, w0, b + 1);
    a1 = lut_get<C>(la, w1, b);
    a3 = lut_get<C>(la, w1, b + 1);
  } else if constexpr (P::c6) {
    // groups 2s, 2s + 1 of each row: states at 12 s, 12 s + 6 (row g) and
    // 48 bits further (row g + 8)
    a0 = lut_get6<C>(la, r, 12 * s);
    a2 = lut_get6<C>(la, r, 12 * s + 6);
    a1 = lut_get6<C>(la, r, 48 + 12 * s);
    a3 = lut_get6<C>(la, r, 54 + 12 * s);
  } else {
    constexpr int o = P::has_mask ? 2 : 0;
    uint32_t lo[2], hi[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t c = code_field<P::cw>(r + o, h * 8 * P::n8 + s * 2 * P::n8, 2 * P::n8);
      const uint32_t A = lut_get<C>(la, c, 0);
      const uint32_t B = P::n8 > 4 ? lut_get<C>(la, c, 1) : 0u;
      if constexpr (P::has_mask) {
        const uint32_t sel = lut_get<C>(ls, r[h], s);
        lo[h] = __byte_perm(A, B, sel & 0xFFFFu);
        hi[h] = __byte_perm(A, B, sel >> 16);
      } else {
        lo[h] = A;
        hi[h] = B;
      }
    }
    a0 = lo[0];
    a2 = hi[0];
    a1 = lo[1];
    a3 = hi[1];
  }
}

// Byte offset of 16-code chunk j of token row n in shared memory: chunks are
// XOR-swizzled inside each 128-byte line by the row, so the eight lanes of a
// quarter warp (rows g, g + 1; four t) read eight distinct bank groups.
__device__ __forceinline__ int xs_off(int n, int j, int xs) { return n * xs + ((j & ~7) | ((j & 7) ^ (n & 7))) * 16; }

// Shared-memory scalars of both kernels.
struct DecScalars {
  float scale[kDecMaxT];  // (g a') / 127 per token
  uint32_t red[kDecWarps];  // per-warp partial maxima of the bf16 magnitude bits of x
  float ap[8];            // a' of the rows quantised here
};

// The activation codes of the t token rows into shared memory, by all warps.
// With FUSED the t <= 4 rows are quantised here: wpr warps per row, the row's
// absmax through the warps' maxima in shared memory; otherwise the codes of
// the act-quant kernel (or the caller) arrive by asynchronous 16-byte copies.
// `issued` runs once the activation loads are out (the weight loads go out
// there).  g_early: g in threads 0..t-1 (the output scale is
// formed after the products, off the critical path).
template <bool FUSED, class Issued>
__device__ __forceinline__ void stage_activations(const DecodeArgs& a, uint8_t* xsm, DecScalars* sc, float& g_early,
                                                  int tid, int warp, int lane, Issued issued) {
  constexpr int XW = kDecWarps;
  const int nch = a.k / 16;  // 16-code chunks per token row
  if constexpr (FUSED) {
    const int tp2 = a.t <= 1 ? 1 : a.t <= 2 ? 2 : 4;
    const int wpr = XW / tp2;
    const int xrow = warp / wpr, xsub = warp % wpr;
    const bool live = xrow < a.t;
    const uint4* xsrc = a.x + int64_t(xrow) * (a.k / 8);
    const bool scale_thread = live && xsub == 0 && lane == 0;
    g_early = tid < a.t ? __ldg(a.g) : 0.0f;
    constexpr int kXc = 3;  // chunks kept in registers between the two passes
    uint4 xr[kXc][2];
#pragma unroll
    for (int q = 0; q < kXc; ++q) {
      const int j = (xsub + q * wpr) * 32 + lane;
      if (live && j < nch) {
        xr[q][0] = __ldg(xsrc + 2 * j);
        xr[q][1] = __ldg(xsrc + 2 * j + 1);
      } else {
        xr[q][0] = xr[q][1] = make_uint4(0, 0, 0, 0);
      }
    }
    issued();
    // the absmax as an integer max over the magnitude bits (their order is
    // the order of the values; a non-finite value shows as bits >= 0x7F80),
    // two halves at a time
    auto vmax16 = [](uint32_t m2, const uint4& v0, const uint4& v1) {
      m2 = __vmaxu2(m2, v0.x & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v0.y & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v0.z & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v0.w & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v1.x & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v1.y & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v1.z & 0x7FFF7FFFu);
      return __vmaxu2(m2, v1.w & 0x7FFF7FFFu);
    };
    uint32_t m2 = 0;
#pragma unroll
    for (int q = 0; q < kXc; ++q) m2 = vmax16(m2, xr[q][0], xr[q][1]);
    if (live)
      for (int j = (xsub + kXc * wpr) * 32 + lane; j < nch; j += wpr * 32)
        m2 = vmax16(m2, __ldg(xsrc + 2 * j), __ldg(xsrc + 2 * j + 1));
    const uint32_t mw = __reduce_max_sync(0xFFFFFFFFu, max(m2 & 0xFFFFu, m2 >> 16));
    if (lane == 0) sc->red[warp] = mw;
    __syncthreads();
    if (live) {
      // the row's wpr partial maxima, read as vectors
      const uint4 r0 = reinterpret_cast<const uint4*>(sc->red)[0];
      const uint4 r1 = reinterpret_cast<const uint4*>(sc->red)[1];
      const uint32_t part[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
      uint32_t m = 0;
#pragma unroll
      for (int w = 0; w < XW; ++w)
        if (w / wpr == xrow) m = max(m, part[w]);
      const bool row_bad = m >= 0x7F80u;
      const float ap = fmaxf(__uint_as_float(m << 16), 1e-5f);
      const QScale qs = make_qscale(ap);
      uint4* gdst = (blockIdx.x == 0 && a.xq_out) ? reinterpret_cast<uint4*>(a.xq_out + int64_t(xrow) * a.k) : nullptr;
#pragma unroll
      for (int q = 0; q < kXc; ++q) {
        const int j = (xsub + q * wpr) * 32 + lane;
        if (j < nch) {
          const uint4 c = quantise16(xr[q][0], xr[q][1], qs);
          *reinterpret_cast<uint4*>(xsm + xs_off(xrow, j, a.xs)) = c;
          if (gdst) gdst[j] = c;
        }
      }
      for (int j = (xsub + kXc * wpr) * 32 + lane; j < nch; j += wpr * 32) {
        const uint4 c = quantise16(__ldg(xsrc + 2 * j), __ldg(xsrc + 2 * j + 1), qs);
        *reinterpret_cast<uint4*>(xsm + xs_off(xrow, j, a.xs)) = c;
        if (gdst) gdst[j] = c;
      }
      if (scale_thread) {
        sc->ap[xrow] = ap;  // the output scale is formed after the products
        if (blockIdx.x == 0) {
          if (a.ap_out) a.ap_out[xrow] = ap;
          if (row_bad) raise_status(a.status, SBL_STATUS_NONFINITE_X);
        }
      }
    }
  } else {
    const float g = tid < a.t ? __ldg(a.g) : 0.0f;
    for (int i = tid; i < a.t * nch; i += XW * 32) {
      const int n = i / nch, j = i - n * nch;
      cp_async16(xsm + xs_off(n, j, a.xs), reinterpret_cast<const uint4*>(a.xq_in + int64_t(n) * a.k) + j);
    }
    cp_async_commit();
    const float apv = tid < a.t ? __ldcg(a.ap_in + tid) : 0.0f;
    issued();
    if (tid < a.t) sc->scale[tid] = __fdiv_rn(__fmul_rn(g, apv), 127.0f);
    cp_async_wait_all();
  }
}

// MMA accumulators of one warp: kSets independent sets per token tile (k-step
// s adds into set s % kSets), so consecutive MMAs do not wait on each other;
// flush() adds the sets into the tile's sums in shared memory.
template <int NT>
struct DecAcc {
  static constexpr int kSets = NT == 1 ? 4 : NT == 2 ? 2 : 1;
  int v[kSets][NT][4];
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int q = 0; q < kSets; ++q)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) v[q][nt][0] = v[q][nt][1] = v[q][nt][2] = v[q][nt][3] = 0;
  }
  __device__ __forceinline__ void flush(int32_t* tile_sums, int gq, int tq) {
    constexpr int TP = 8 * NT;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      int r[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        r[i] = v[0][nt][i];
#pragma unroll
        for (int q = 1; q < kSets; ++q) r[i] += v[q][nt][i];
      }
      const int col = nt * 8 + 2 * tq;
      atomicAdd(tile_sums + gq * TP + col, r[0]);
      atomicAdd(tile_sums + gq * TP + col + 1, r[1]);
      atomicAdd(tile_sums + (gq + 8) * TP + col, r[2]);
      atomicAdd(tile_sums + (gq + 8) * TP + col + 1, r[3]);
    }
  }
};

// The block's outputs from its tiles' sums: y = acc * ((g a') / 127) (and the
// raw sums), consecutive rows per token.
template <int NT>
__device__ __forceinline__ void write_outputs(const DecodeArgs& a, const int32_t* s_acc, const DecScalars* sc,
                                              int tile0, int ntile, int tid) {
  constexpr int TP = 8 * NT;
  const int rows = min(ntile * 16, a.n_out - tile0 * 16);
  for (int idx = tid; idx < ntile * 16 * a.t; idx += kDecThreads) {
    const int tok = idx / (ntile * 16), r = idx - tok * (ntile * 16);
    if (r < rows) {
      const int v = s_acc[(r >> 4) * 16 * TP + (r & 15) * TP + tok];
      const int64_t o = int64_t(tok) * a.n_out + tile0 * 16 + r;
      a.y[o] = __fmul_rn(static_cast<float>(v), sc->scale[tok]);
      if (a.acc_out) a.acc_out[o] = v;
    }
  }
}

// Every warp stages activations, then expands its own units' weights into MMA
// fragments on the fly (table lookups between the MMAs).
template <int FMT, int NT, bool FUSED>
__global__ void __launch_bounds__(kDecThreads, 2) k_decode(const DecodeArgs a) {
  using P = Pack<FMT>;
  constexpr int C = kLutCopiesReg;
  constexpr int TP = 8 * NT;  // token columns
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t* lut_a = reinterpret_cast<uint32_t*>(smem);
  uint32_t* lut_s = lut_a + lut_words(C);  // mask selectors (packs with a mask block)
  uint8_t* xsm = smem + (P::has_mask ? 2 * lut_words(C) : lut_words(C, P::lut_entries)) * 4;
  int32_t* s_acc = reinterpret_cast<int32_t*>(xsm + a.t * a.xs);  // [tpb][16][TP]
  DecScalars* sc = reinterpret_cast<DecScalars*>(s_acc + a.tpb * 16 * TP);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = static_cast<int>(blockIdx.x);
  const int tile0 = b < a.nfull ? b * a.tpb : a.nfull * a.tpb + (b - a.nfull) * (a.tpb - 1);
  const int ntile = min(b < a.nfull ? a.tpb : a.tpb - 1, a.tiles - tile0);
  const int units = ntile * a.upr;

  // ---- before the wait: prefetch, tables, zeroed sums ----
  if (tid == 0) bulk_prefetch_l2(a.w + int64_t(tile0) * a.upr * P::unit_bytes, static_cast<uint32_t>(units) * P::unit_bytes);
  if (tid == 32) {
    if (FUSED) bulk_prefetch_l2(a.x, static_cast<uint32_t>(a.t) * static_cast<uint32_t>(a.k) * 2u);
    else bulk_prefetch_l2(a.xq_in, static_cast<uint32_t>(a.t) * static_cast<uint32_t>(a.k));
  }
  pdl_trigger();
  fill_lut<C>(lut_a, P::lut_kind, tid, P::lut_entries);
  if constexpr (P::has_mask) fill_lut<C>(lut_s, 2, tid);
  for (int i = tid; i < ntile * 16 * TP; i += kDecThreads) s_acc[i] = 0;
  // Activation columns past k are left as they are: the weights there are
  // zero (zero-filled pack).  Token rows past t are neither stored nor read.
  pdl_wait();

  const int u_begin = (units * warp) / kDecWarps, u_end = (units * (warp + 1)) / kDecWarps;
  // (tile, unit) of this warp's first unit; later ones follow by counting
  const int tl_begin = u_begin / a.upr, un_begin = u_begin - tl_begin * a.upr;
  uint32_t wr[kDecBatch][P::regs];
  auto load_batch = [&](int ub, int tl, int un) {
#pragma unroll
    for (int i = 0; i < kDecBatch; ++i) {
      if (ub + i < u_end) load_unit<FMT>(a, tile0 + tl, un, lane, wr[i]);
      if (++un == a.upr) {
        un = 0;
        ++tl;
      }
    }
  };
  float g_early = 0.0f;
  // the activation loads go out first (the rest of the block's path waits on
  // them), then this warp's first batch of weight loads
  stage_activations<FUSED>(a, xsm, sc, g_early, tid, warp, lane,
                                      [&]() { load_batch(u_begin, tl_begin, un_begin); });
  __syncthreads();

  // ---- products ----
  const int gq = lane >> 2, tq = lane & 3;
  const uint8_t* la = reinterpret_cast<const uint8_t*>(lut_a + (lane % C));
  const uint8_t* ls = reinterpret_cast<const uint8_t*>(lut_s + (lane % C));
  // this lane's activation chunks in unit 0 (token row gq + 8 nt, chunk
  // 2 tq + p); unit un is 128 un bytes further
  const uint8_t* bsrc[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int p = 0; p < 2; ++p) bsrc[nt][p] = xsm + xs_off(gq + 8 * nt, 2 * tq + p, a.xs);
  DecAcc<NT> acc;
  int cur = -1;                      // tile (local) the accumulators belong to
  int tl = tl_begin, un = un_begin;  // (tile, unit) of unit ub + i
  for (int ub = u_begin; ub < u_end; ub += kDecBatch) {
    if (ub != u_begin) load_batch(ub, tl, un);
#pragma unroll
    for (int i = 0; i < kDecBatch; ++i) {
      if (ub + i >= u_end) break;
      if (tl != cur) {
        if (cur >= 0) acc.flush(s_acc + cur * 16 * TP, gq, tq);
        cur = tl;
        acc.zero();
      }
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        uint4 bv[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          bv[nt] = (gq + 8 * nt < a.t) ? *reinterpret_cast<const uint4*>(bsrc[nt][p] + 128 * un) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int sp = 0; sp < 2; ++sp) {
          uint32_t a0, a1, a2, a3;
          decode_step<FMT, C>(wr[i], 2 * p + sp, la, ls, a0, a1, a2, a3);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            mma_s8_16x8x32(acc.v[(2 * p + sp) % DecAcc<NT>::kSets][nt], a0, a1, a2, a3, sp ? bv[nt].z : bv[nt].x,
                           sp ? bv[nt].w : bv[nt].y);
        }
      }
      if (++un == a.upr) {
        un = 0;
        ++tl;
      }
    }
  }
  if (cur >= 0) acc.flush(s_acc + cur * 16 * TP, gq, tq);
  if (FUSED && tid < a.t) sc->scale[tid] = __fdiv_rn(__fmul_rn(g_early, sc->ap[tid]), 127.0f);
  __syncthreads();
  write_outputs<NT>(a, s_acc, sc, tile0, ntile, tid);
}

namespace {

int decode_nt(int64_t t) { return t <= 8 ? 1 : t <= 16 ? 2 : 4; }

int decode_fmt(int n, int m, bool code6) {
  return (n == 2 && m == 4) ? (code6 ? kFmtCode6 : 0) : 8 * n / m;
}

size_t decode_lut_bytes(int fmt) {
  const bool has_mask = fmt >= 1 && fmt < 8;
  return size_t(has_mask ? 2 * lut_words(kLutCopiesReg) : lut_words(kLutCopiesReg, fmt == kFmtCode6 ? 64 : 256)) * 4;
}

size_t decode_smem(int fmt, int nt, int64_t t, int64_t k, int tpb) {
  const size_t xs = size_t((k + 127) / 128 * 128);
  return decode_lut_bytes(fmt) + size_t(t) * xs + size_t(tpb) * 16 * 8 * nt * 4 + sizeof(DecScalars);
}

template <int FMT, int NT, bool FUSED>
cudaError_t decode_launch(const DecodeArgs& a, int blocks, size_t smem, cudaStream_t s) {
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    err = cudaFuncSetAttribute(k_decode<FMT, NT, FUSED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kDecMaxSmem));
  });
  if (err != cudaSuccess) return err;
  return launch_pdl(k_decode<FMT, NT, FUSED>, dim3(blocks), dim3(kDecThreads), smem, s, a);
}

template <int FMT>
cudaError_t decode_fmt_launch(const DecodeArgs& a, bool fused, int nt, int blocks, size_t smem, cudaStream_t s) {
  if (nt == 1)
    return fused ? decode_launch<FMT, 1, true>(a, blocks, smem, s) : decode_launch<FMT, 1, false>(a, blocks, smem, s);
  if (nt == 2) return decode_launch<FMT, 2, false>(a, blocks, smem, s);
  return decode_launch<FMT, 4, false>(a, blocks, smem, s);
}

}  // namespace

uint64_t decode_pack_bytes(int64_t n_out, int64_t k, int n, int m, bool code6) {
  if (n == 2 && m == 4) return uint64_t((n_out + 15) / 16) * uint64_t((k + 127) / 128) * (code6 ? 384 : 512);
  const int n8 = 8 * n / m;
  const uint64_t cb = uint64_t(2 * n8 + 3) / 4 * 4;
  const uint64_t unit = (n8 < 8 ? 256 : 0) + 32 * cb;
  return uint64_t((n_out + 15) / 16) * uint64_t((k + 127) / 128) * unit;
}

bool gemv_fits(int64_t t, int64_t k, int n, int m, bool code6) {
  if (t < 1 || t > kDecMaxT) return false;
  return decode_smem(decode_fmt(n, m, code6), decode_nt(t), t, k, 1) <= kDecMaxSmem;
}

// The decode kernels stream the packed weights once for up to 32 tokens; the
// tensor-core GEMMs pay a round of 240-token tiles for any token count.
bool gemv_preferred(int64_t t, int64_t n_out, int64_t k) { return t <= kDecMaxT; }

bool gemv_fuses_act_quant(int64_t t) { return t <= kFusedMaxT; }

cudaError_t launch_forward_gemv(const uint8_t* gemv, int n, int m, bool code6, const uint16_t* x, const int8_t* xq_in,
                                const float* ap_in, const float* g, int64_t n_out, int64_t t, int64_t k, float* y,
                                int32_t* acc_out, int8_t* xq_out, float* ap_out, uint32_t* status, int num_sms,
                                cudaStream_t s) {
  DecodeArgs a;
  a.w = gemv;
  a.x = reinterpret_cast<const uint4*>(x);
  a.xq_in = xq_in;
  a.ap_in = ap_in;
  a.g = g;
  a.y = y;
  a.acc_out = acc_out;
  a.xq_out = xq_out;
  a.ap_out = ap_out;
  a.status = status;
  a.n_out = static_cast<int>(n_out);
  a.t = static_cast<int>(t);
  a.k = static_cast<int>(k);
  a.tiles = static_cast<int>((n_out + 15) / 16);
  a.upr = static_cast<int>((k + 127) / 128);
  a.xs = a.upr * 128;
  const int fmt = decode_fmt(n, m, code6), nt = decode_nt(t);
  // codes from the caller (x == NULL), else quantised here for few tokens
  const bool fused = x != nullptr && gemv_fuses_act_quant(t);
  // Each block takes an equal run of tiles.  Up to 8 tokens, as many blocks
  // as fit two per SM: a call is a short chain, and more blocks split the
  // weight stream over more warps.  From 9 tokens, one block per SM while
  // that leaves at most three tiles a block (two above 16 tokens, where a
  // tile's products weigh more): every block stages all t rows of codes, so
  // fewer blocks stage fewer bytes.
  // Measured per call in a graph (K = 2560), one against two blocks per SM:
  // t = 16 at 2560 rows 5.65 against 5.85-6.35 us, at 6912 rows 6.72 against
  // 7.17-7.46; t = 32 at 2560 rows 7.3 against 8.4-9.0; t = 32 at 6912 rows
  // (three tiles a block) 11.6-12.4 against 10.5-11.0; t = 1 at 6912 rows
  // 5.37 against 4.78.
  const size_t smem1 = decode_smem(fmt, nt, t, k, 1);
  int per_sm = smem1 * 2 + 2048 <= 228 * 1024 ? 2 : 1;
  if (t > 8 && a.tiles <= (t <= 16 ? 3 : 2) * num_sms) per_sm = 1;
  // Up to 8 tokens, with more tiles than block slots: every slot gets a
  // block and the tiles are dealt as evenly as whole tiles allow (tpb or
  // tpb - 1 a block), so no SM carries two blocks of tpb while another has
  // one (6912 rows: t = 1 4.68-4.71 against 4.76-4.80 us, t = 4 on the 6-bit
  // code 4.98-5.01 against 5.08-5.14).  From 9 tokens the fewer blocks of
  // uniform runs stay: each block stages all t rows of codes, and dealing
  // cost 8-25 % at t = 16-32.
  const int slots = num_sms * per_sm;
  int tpb = (a.tiles + slots - 1) / slots;
  while (decode_smem(fmt, nt, t, k, tpb) > kDecMaxSmem && tpb > 1) --tpb;
  const size_t smem = decode_smem(fmt, nt, t, k, tpb);
  if (smem > kDecMaxSmem) return cudaErrorInvalidValue;
  a.tpb = tpb;
  int blocks = (a.tiles + tpb - 1) / tpb;
  a.nfull = blocks;
  if (t <= 8 && tpb > 1 && a.tiles <= tpb * slots && a.tiles > (tpb - 1) * slots) {
    blocks = slots;
    a.nfull = a.tiles - (tpb - 1) * slots;
  }
  switch (fmt) {
    case 0: return decode_fmt_launch<0>(a, fused, nt, blocks, smem, s);
    case 1: return decode_fmt_launch<1>(a, fused, nt, blocks, smem, s);
    case 2: return decode_fmt_launch<2>(a, fused, nt, blocks, smem, s);
    case 3: return decode_fmt_launch<3>(a, fused, nt, blocks, smem, s);
    case 4: return decode_fmt_launch<4>(a, fused, nt, blocks, smem, s);
    case 5: return decode_fmt_launch<5>(a, fused, nt, blocks, smem, s);
    case 6: return decode_fmt_launch<6>(a, fused, nt, blocks, smem, s);
    case 7: return decode_fmt_launch<7>(a, fused, nt, blocks, smem, s);
    case kFmtCode6: return decode_fmt_launch<kFmtCode6>(a, fused, nt, blocks, smem, s);
    default: return decode_fmt_launch<8>(a, fused, nt, blocks, smem, s);
  }
}

}  // namespace sbl
