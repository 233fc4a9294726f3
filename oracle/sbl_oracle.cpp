// Sparse-BitLinear CPU oracle -- TEST INFRASTRUCTURE ONLY (see sbl_oracle.h).
//
// Plain loops, one definition per step, no blocking or reordering beyond what
// the definition states.  OpenMP only splits independent rows (or, for the
// exact sum, combines exact integer partial sums, which is order-free).
// Build: g++ -O2 -fopenmp -fno-fast-math -ffp-contract=off -shared -fPIC.
#include "sbl_oracle.h"

#include <algorithm>
#include <cstdlib>
#include <cmath>
#include <cstring>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

float f32_from_bits(uint32_t u) {
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}
uint32_t bits_from_f32(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return u;
}
// bf16 -> fp32 is exact: the bf16 pattern is the top half of the fp32 one.
float bf16_value(uint16_t b) { return f32_from_bits(uint32_t(b) << 16); }

// ---------------------------------------------------------------------------
// Exact sum of bf16 magnitudes.
//
// A bf16 magnitude with biased exponent e and 7-bit mantissa f is
//   (128 + f) * 2^(e - 134)   for e >= 1,
//    f        * 2^(-133)     for e == 0 (subnormal),
// so in units of 2^-133 it is the integer  sig << (max(e,1) - 1)  with
// sig = (e ? 128 + f : f) < 2^8 and a shift of at most 253.  Summing up to
// 2^40 of them stays below 2^302, inside five 64-bit limbs.
// ---------------------------------------------------------------------------
struct U320 {
  uint64_t limb[5] = {0, 0, 0, 0, 0};

  void add_at(int i, uint64_t v) {
    while (v != 0 && i < 5) {
      uint64_t before = limb[i];
      limb[i] += v;
      v = (limb[i] < before) ? 1u : 0u;  // carry into the next limb
      ++i;
    }
  }
  void add_shifted(uint64_t v, int shift) {
    int i = shift >> 6, off = shift & 63;
    add_at(i, v << off);
    if (off != 0 && (v >> (64 - off)) != 0) add_at(i + 1, v >> (64 - off));
  }
  void add(const U320& o) {
    for (int i = 0; i < 5; ++i) add_at(i, o.limb[i]);
  }
  bool bit(int p) const {
    if (p < 0 || p >= 320) return false;
    return (limb[p >> 6] >> (p & 63)) & 1u;
  }
  bool any_bit_below(int p) const {  // any of bits [0, p) set
    for (int q = 0; q < p && q < 320; ++q)
      if (bit(q)) return true;
    return false;
  }
  bool is_zero() const {
    for (uint64_t v : limb)
      if (v) return false;
    return true;
  }
};

// Correctly rounded (nearest, ties to even) fp32 value of S * 2^-133 / n.
// Plain restoring long division, one quotient bit per dividend bit, taken
// down to the last bit fp32 keeps (24 significant bits, or the 2^-149
// subnormal step), then one round bit and a sticky bit.
float round_quotient_to_f32(const U320& S, uint64_t n) {
  unsigned __int128 r = 0;  // running remainder, always < n
  uint64_t q = 0;           // quotient bits from the leading one down
  bool started = false;
  int lsb = -149;  // real exponent of the last kept bit (subnormal floor until the lead is known)
  int p = 319;     // dividend bit position; its real exponent is p - 133
  for (;; --p) {
    const int real = p - 133;
    if (real < lsb) break;
    r = (r << 1) | (S.bit(p) ? 1u : 0u);
    uint64_t qb = 0;
    if (r >= n) {
      r -= n;
      qb = 1;
    }
    if (!started && qb) {
      started = true;
      lsb = std::max(real - 23, -149);
    }
    if (started) q = (q << 1) | qb;
  }
  // Bit p now sits at real exponent lsb - 1: the round bit.
  r = (r << 1) | (S.bit(p) ? 1u : 0u);
  uint64_t round_bit = 0;
  if (r >= n) {
    r -= n;
    round_bit = 1;
  }
  const bool sticky = (r != 0) || S.any_bit_below(p);
  if (round_bit && (sticky || (q & 1u))) q += 1;
  return std::ldexp(float(q), lsb);  // q <= 2^24: exact
}

}  // namespace

extern "C" {

int sbo_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void sbo_set_threads(int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
}

// A1.  Exact sum over every master weight, masked ones included ([de] §2,
// [fr] §2: quantisation happens before the mask), then one rounding.
uint32_t sbo_absmean_bits(const uint16_t* w, int64_t numel) {
  if (numel <= 0) return 0u;
  int nthreads = sbo_threads();
  std::vector<U320> part(static_cast<size_t>(nthreads));
  std::vector<int> bad(static_cast<size_t>(nthreads), 0);
#pragma omp parallel
  {
#ifdef _OPENMP
    int tid = omp_get_thread_num();
#else
    int tid = 0;
#endif
    U320 acc;
#pragma omp for schedule(static)
    for (int64_t i = 0; i < numel; ++i) {
      const uint16_t mag = w[i] & 0x7fffu;
      const int e = mag >> 7;
      const uint64_t f = mag & 0x7fu;
      if (e == 0xff) {  // inf or NaN
        bad[size_t(tid)] = 1;
        continue;
      }
      const uint64_t sig = e ? (128u + f) : f;
      acc.add_shifted(sig, (e ? e : 1) - 1);
    }
    part[size_t(tid)] = acc;
  }
  U320 S;
  for (int t = 0; t < nthreads; ++t) {
    if (bad[size_t(t)]) return 0x7fc00000u;
    S.add(part[size_t(t)]);
  }
  if (S.is_zero()) return 0u;
  return bits_from_f32(round_quotient_to_f32(S, uint64_t(numel)));
}

float sbo_clamped_scale(float gamma) { return gamma > 1e-5f ? gamma : 1e-5f; }

// A2.  Rank the m entries of a group by (|w| descending, index ascending) and
// keep the first n ([ja] §2.1, [ko] §2.1: top-n by master magnitude; ties
// broken by lowest index is a READING).  |w| compares as the bf16 magnitude
// bits, which orders finite magnitudes exactly and makes -0 tie with +0.
void sbo_nm_mask(const uint16_t* w, int64_t n_out, int64_t k, int n, int m,
                 uint8_t* mask) {
  const int64_t groups = k / m;
#pragma omp parallel for schedule(static)
  for (int64_t row = 0; row < n_out; ++row) {
    for (int64_t g = 0; g < groups; ++g) {
      const uint16_t* grp = w + row * k + g * m;
      int order[8];
      for (int j = 0; j < m; ++j) order[j] = j;
      std::stable_sort(order, order + m, [&](int a, int b) {
        return (grp[a] & 0x7fffu) > (grp[b] & 0x7fffu);
      });
      uint8_t bits = 0;
      for (int j = 0; j < n; ++j) bits |= uint8_t(1u << order[j]);
      mask[row * groups + g] = bits;
    }
  }
}

// A3 (ternarise).  w/g rounded half-to-even and clipped to [-1, 1] is 0 when
// |w|/g <= 1/2 and sign(w) otherwise; 2|w| is exact in fp32, so the test
// 2|w| > g decides it with no division rounding.
void sbo_nm_mask_from_codes(const int8_t* q, int64_t n_out, int64_t k, int n, int m,
                            uint8_t* mask) {
  const int64_t groups = k / m;
#pragma omp parallel for schedule(static)
  for (int64_t row = 0; row < n_out; ++row) {
    for (int64_t g = 0; g < groups; ++g) {
      const int8_t* grp = q + row * k + g * m;
      int order[8];
      for (int j = 0; j < m; ++j) order[j] = j;
      // stable: equal |q| keep index order, so ties go to the lowest index
      std::stable_sort(order, order + m, [&](int a, int b) { return std::abs(int(grp[a])) > std::abs(int(grp[b])); });
      uint8_t bits = 0;
      for (int j = 0; j < n; ++j) bits |= uint8_t(1u << order[j]);
      mask[row * groups + g] = bits;
    }
  }
}

void sbo_ternary(const uint16_t* w, int64_t numel, float g, int8_t* q) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < numel; ++i) {
    const float v = bf16_value(w[i]);
    const float two_abs = 2.0f * std::fabs(v);
    int8_t code = 0;
    if (two_abs > g) code = (v < 0.0f) ? int8_t(-1) : int8_t(1);
    q[i] = code;
  }
}

// A3 (quant-then-mask):  weff = q (.) mask.
void sbo_apply_mask(const int8_t* q, const uint8_t* mask, int64_t n_out,
                    int64_t k, int m, int8_t* weff) {
  const int64_t groups = k / m;
#pragma omp parallel for schedule(static)
  for (int64_t row = 0; row < n_out; ++row)
    for (int64_t c = 0; c < k; ++c) {
      const uint8_t bits = mask[row * groups + c / m];
      const bool kept = (bits >> (c % m)) & 1u;
      weff[row * k + c] = kept ? q[row * k + c] : int8_t(0);
    }
}

void sbo_pack24(const int8_t* weff, const uint8_t* mask, int64_t n_out,
                int64_t k, int8_t* vals, uint8_t* meta) {
  const int64_t groups = k / 4;
#pragma omp parallel for schedule(static)
  for (int64_t row = 0; row < n_out; ++row) {
    for (int64_t g = 0; g < groups; ++g) {
      const uint8_t bits = mask[row * groups + g];
      int idx[2], found = 0;
      for (int j = 0; j < 4 && found < 2; ++j)
        if ((bits >> j) & 1u) idx[found++] = j;
      vals[row * (k / 2) + 2 * g + 0] = weff[row * k + 4 * g + idx[0]];
      vals[row * (k / 2) + 2 * g + 1] = weff[row * k + 4 * g + idx[1]];
      const uint8_t nib = uint8_t(idx[0] | (idx[1] << 2));
      uint8_t& byte = meta[row * (k / 8) + g / 2];
      if ((g & 1) == 0)
        byte = nib;
      else
        byte = uint8_t(byte | (nib << 4));
    }
  }
}

// Compressed-index packing for any N:M.  A block of 8 weights holds 8/m whole
// groups; its mask byte is their masks side by side, and its kept codes are
// appended to the row's bit stream in index order, two bits each.
void sbo_pack_nm(const int8_t* weff, const uint8_t* mask, int64_t n_out,
                 int64_t k, int n, int m, uint8_t* masks8, uint8_t* codes) {
  const int64_t blocks = k / 8, groups = k / m;
  const int64_t row_code_bytes = k * n / (4 * m);
#pragma omp parallel for schedule(static)
  for (int64_t row = 0; row < n_out; ++row) {
    uint8_t* out = codes + row * row_code_bytes;
    for (int64_t b = 0; b < row_code_bytes; ++b) out[b] = 0;
    int64_t bit = 0;  // position in this row's code stream
    for (int64_t blk = 0; blk < blocks; ++blk) {
      uint32_t mbyte = 0;
      for (int j = 0; j < 8; ++j) {
        const int64_t col = blk * 8 + j;
        const uint8_t gbits = mask[row * groups + col / m];
        if ((gbits >> (col % m)) & 1u) mbyte |= 1u << j;
      }
      masks8[row * blocks + blk] = static_cast<uint8_t>(mbyte);
      for (int j = 0; j < 8; ++j) {
        if (!((mbyte >> j) & 1u)) continue;
        const int8_t q = weff[row * k + blk * 8 + j];
        const uint32_t code = q == 0 ? 0u : (q > 0 ? 1u : 3u);
        out[bit / 8] = static_cast<uint8_t>(out[bit / 8] | (code << (bit % 8)));
        bit += 2;
      }
    }
  }
}

// The denser 2:4 decode code: a group of four has C(4,2) = 6 choices of its
// two kept positions and 3 x 3 ternary values for them, 54 states, so 6 bits
// hold it (1.5 bits a weight).  READING of the numbering, which the pages do
// not give: the position pairs in lexicographic order (0,1) (0,2) (0,3)
// (1,2) (1,3) (2,3) are p = 0..5, a code c in {-1, 0, +1} is the digit
// c mod 3 (0, 1, 2 for 0, +1, -1), and the state is 9 p + 3 d(c_i0) + d(c_i1),
// so the all-zero group under positions (0,1) is state 0.  States go least
// significant bit first into one bit stream per row, 6 bits each.
void sbo_pack24_code6(const int8_t* weff, const uint8_t* mask, int64_t n_out,
                      int64_t k, uint8_t* out) {
  const int64_t groups = k / 4, row_bytes = k * 6 / 32;
#pragma omp parallel for schedule(static)
  for (int64_t row = 0; row < n_out; ++row) {
    uint8_t* dst = out + row * row_bytes;
    for (int64_t b = 0; b < row_bytes; ++b) dst[b] = 0;
    for (int64_t g = 0; g < groups; ++g) {
      const uint8_t bits = mask[row * groups + g];
      int idx[2], found = 0;
      for (int j = 0; j < 4 && found < 2; ++j)
        if ((bits >> j) & 1u) idx[found++] = j;
      int pair = 0, rank = 0;  // rank of (idx[0], idx[1]) among the six pairs
      for (int a = 0; a < 4; ++a)
        for (int b = a + 1; b < 4; ++b, ++rank)
          if (a == idx[0] && b == idx[1]) pair = rank;
      const int c0 = weff[row * k + 4 * g + idx[0]], c1 = weff[row * k + 4 * g + idx[1]];
      const uint32_t state = uint32_t(9 * pair + 3 * ((c0 + 3) % 3) + (c1 + 3) % 3);
      for (int bit = 0; bit < 6; ++bit) {
        const int64_t pos = g * 6 + bit;
        if ((state >> bit) & 1u) dst[pos / 8] = static_cast<uint8_t>(dst[pos / 8] | (1u << (pos % 8)));
      }
    }
  }
}

// A4.  Per-token absmax int8 quantisation (READING: the pages do not describe
// activation quantisation; this is the BitNet b1.58 convention).
void sbo_act_quant(const uint16_t* x, int64_t t, int64_t k, int8_t* xq,
                   float* a_prime) {
#pragma omp parallel for schedule(static)
  for (int64_t row = 0; row < t; ++row) {
    const uint16_t* xr = x + row * k;
    float a = 0.0f;
    for (int64_t c = 0; c < k; ++c) a = std::max(a, std::fabs(bf16_value(xr[c])));
    const float ap = std::max(a, 1e-5f);
    a_prime[row] = ap;
    for (int64_t c = 0; c < k; ++c) {
      const float v = bf16_value(xr[c]);
      const float scaled = (127.0f * std::fabs(v)) / ap;  // two fp32 roundings
      float n = std::nearbyint(scaled);                      // ties to even
      n = std::min(n, 127.0f);
      const int code = int(n);
      xq[row * k + c] = int8_t(v < 0.0f ? -code : code);
    }
  }
}

int32_t sbo_acc_at(const int8_t* xq_row, const int8_t* weff_row, int64_t k) {
  int64_t s = 0;
  for (int64_t c = 0; c < k; ++c) s += int64_t(xq_row[c]) * int64_t(weff_row[c]);
  return int32_t(s);
}

// A5.  Brute-force integer product (the masked ternary x int8 GEMM).
int sbo_gemm_acc(const int8_t* xq, const int8_t* weff, int64_t t,
                 int64_t n_out, int64_t k, int32_t* acc) {
  int overflow = 0;
#pragma omp parallel for schedule(static) reduction(| : overflow)
  for (int64_t ti = 0; ti < t; ++ti)
    for (int64_t o = 0; o < n_out; ++o) {
      int64_t s = 0;
      for (int64_t c = 0; c < k; ++c) s += int64_t(xq[ti * k + c]) * int64_t(weff[o * k + c]);
      if (s >= (int64_t(1) << 31) || s < -(int64_t(1) << 31)) overflow = 1;
      acc[ti * n_out + o] = int32_t(s);
    }
  return overflow ? -1 : 0;
}

// A6.  Dequantisation: one fp32 product per output, scale formed as (g*a')/127.
void sbo_dequant(const int32_t* acc, const float* a_prime, float g, int64_t t,
                 int64_t n_out, float* y) {
#pragma omp parallel for schedule(static)
  for (int64_t ti = 0; ti < t; ++ti) {
    const float scale = (g * a_prime[ti]) / 127.0f;
    for (int64_t o = 0; o < n_out; ++o) y[ti * n_out + o] = float(acc[ti * n_out + o]) * scale;
  }
}

double sbo_grad_x_at(const uint16_t* dy, const int8_t* weff, float g,
                     int64_t n_out, int64_t k, int64_t ti, int64_t ki) {
  double s = 0.0;
  for (int64_t o = 0; o < n_out; ++o)
    s += double(bf16_value(dy[ti * n_out + o])) * double(weff[o * k + ki]);
  return double(g) * s;
}

// A7.  STE: the X-gradient goes through the masked, scaled ternary weights.
void sbo_grad_x(const uint16_t* dy, const int8_t* weff, float g, int64_t t,
                int64_t n_out, int64_t k, double* dx) {
#pragma omp parallel for schedule(static)
  for (int64_t ti = 0; ti < t; ++ti) {
    std::vector<double> row(size_t(k), 0.0);
    for (int64_t o = 0; o < n_out; ++o) {
      const double d = double(bf16_value(dy[ti * n_out + o]));
      const int8_t* wr = weff + o * k;
      for (int64_t c = 0; c < k; ++c) row[size_t(c)] += d * double(wr[c]);
    }
    for (int64_t c = 0; c < k; ++c) dx[ti * k + c] = double(g) * row[size_t(c)];
  }
}

double sbo_grad_w_at(const uint16_t* dy, const uint16_t* x, int64_t t,
                     int64_t n_out, int64_t k, int64_t oi, int64_t ki) {
  double s = 0.0;
  for (int64_t ti = 0; ti < t; ++ti)
    s += double(bf16_value(dy[ti * n_out + oi])) * double(bf16_value(x[ti * k + ki]));
  return s;
}

// A8.  Dense gradient to every master weight, pruned ones included.
void sbo_grad_w(const uint16_t* dy, const uint16_t* x, int64_t t,
                int64_t n_out, int64_t k, double* dw) {
#pragma omp parallel for schedule(static)
  for (int64_t o = 0; o < n_out; ++o) {
    double* out = dw + o * k;
    for (int64_t c = 0; c < k; ++c) out[c] = 0.0;
    for (int64_t ti = 0; ti < t; ++ti) {
      const double d = double(bf16_value(dy[ti * n_out + o]));
      const uint16_t* xr = x + ti * k;
      for (int64_t c = 0; c < k; ++c) out[c] += d * double(bf16_value(xr[c]));
    }
  }
}

void sbo_grad_w_masked(const uint16_t* dy, const uint16_t* x, const uint8_t* mask,
                       int64_t t, int64_t n_out, int64_t k, int m, double* dw) {
  sbo_grad_w(dy, x, t, n_out, k, dw);
  const int64_t groups = k / m;
#pragma omp parallel for schedule(static)
  for (int64_t o = 0; o < n_out; ++o)
    for (int64_t c = 0; c < k; ++c)
      if (!((mask[o * groups + c / m] >> (c % m)) & 1u)) dw[o * k + c] = 0.0;
}

// Detach-form STE operand for dW: xhat = RN_bf16(xq * a' / 127), one
// rounding of the exact value (see the header for why fp64 suffices).
void sbo_dequant_act(const int8_t* xq, const float* a_prime, int64_t t, int64_t k, uint16_t* xhat) {
#pragma omp parallel for schedule(static)
  for (int64_t row = 0; row < t; ++row) {
    for (int64_t c = 0; c < k; ++c) {
      const double v = double(xq[row * k + c]) * double(a_prime[row]) / 127.0;
      sbo_round_bf16(&v, 1, xhat + row * k + c);
    }
  }
}

void sbo_round_bf16(const double* in, int64_t count, uint16_t* out) {
  for (int64_t i = 0; i < count; ++i) {
    const double d = in[i];
    if (std::isnan(d)) {
      out[i] = 0x7fc0u;
      continue;
    }
    const uint16_t sign = std::signbit(d) ? 0x8000u : 0u;
    const double a = std::fabs(d);
    if (a == 0.0) {
      out[i] = sign;
      continue;
    }
    if (std::isinf(a)) {
      out[i] = uint16_t(sign | 0x7f80u);
      continue;
    }
    int e = 0;
    std::frexp(a, &e);                           // a in [2^(e-1), 2^e)
    const int lsb = std::max(e - 1 - 7, -133);   // 8 significant bits, subnormal step 2^-133
    const double r = std::nearbyint(std::ldexp(a, -lsb));  // ties to even
    const double v = std::ldexp(r, lsb);
    if (v >= 0x1p128) {
      out[i] = uint16_t(sign | 0x7f80u);
      continue;
    }
    out[i] = uint16_t(sign | (bits_from_f32(float(v)) >> 16));  // v is bf16-exact
  }
}

}  // extern "C"
