/*
 * Sparse-BitLinear CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously-correct host implementation of what the
 * Sparse-BitLinear operator computes.  Only the test suite, the smoke check
 * and the benchmark's CPU-baseline leg may load it; the CUDA library never
 * links, includes or calls it, and it shares no code with the CUDA path.
 *
 * Citation legend.  All pages summarise the paper "Sparse-BitNet: 1.58-bit
 * LLMs are Naturally Friendly to Semi-Structured Sparsity" (arXiv 2603.05168):
 *   [ja]   gist.science, Japanese technical summary
 *   [de]   gist.science, German technical summary
 *   [ko]   gist.science, Korean technical summary
 *   [fr]   gist.science, French technical summary
 *   [abs]  fugumt.com, the English abstract
 * followed by the section number on that page.  Steps the pages leave open
 * are taken in their plainest reading; each such reading is marked READING.
 *
 * All pointers are host pointers.  Weights, activations and gradients are
 * bfloat16 passed as their raw uint16 bit patterns.  Matrices are row-major:
 *   W  [n_out, k]   master weights (nn.Linear convention)
 *   X  [t, k]       activations
 *   dY [t, n_out]   upstream gradient
 * Groups of m run along k inside one row of W.
 */
#ifndef SBL_ORACLE_H
#define SBL_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A1 (absmean).  gamma = RN_fp32( sum|w| / numel ), the sum taken exactly over
 * ALL master weights (quantisation happens before masking, [de] §2, [fr] §2).
 * Returns the fp32 bit pattern of gamma; 0x7fc00000 (NaN) if any w is not
 * finite; 0 for numel == 0. */
uint32_t sbo_absmean_bits(const uint16_t* w, int64_t numel);

/* g = max(gamma, 1e-5f): READING, the eps clamp of the absmean scale. */
float sbo_clamped_scale(float gamma);

/* A2 (N:M mask, [ja] §2.1, [de] §2, [ko] §2.1).  For each row and each group of
 * m consecutive weights along k, keep the n largest |w| (bf16 magnitude, i.e.
 * bits & 0x7fff), ties to the lowest index.  mask[row*(k/m) + grp] has bit j
 * set when position j of the group is kept.  Requires k % m == 0, 1<=n<=m<=8. */
void sbo_nm_mask(const uint16_t* w, int64_t n_out, int64_t k, int n, int m,
                 uint8_t* mask);

/* Ablation of A2 named by the pages ([de] §4 "Ablationsstudien", [fr] §5):
 * the mask built from the quantised ternary codes instead of the masters.
 * For each group keep the n largest |q| (|q| in {0, 1}), ties to the lowest
 * index, i.e. the first n nonzero codes, then the first zero ones.  Same
 * output layout as sbo_nm_mask. */
void sbo_nm_mask_from_codes(const int8_t* q, int64_t n_out, int64_t k, int n, int m,
                            uint8_t* mask);

/* A3 (ternarise): q = round-half-even(clip(w/g, -1, 1)), which is
 * sign(w) when 2|w| > g and 0 otherwise ([de] §1, [fr] §1 ternary set). */
void sbo_ternary(const uint16_t* w, int64_t numel, float g, int8_t* q);

/* A3 (quant-then-mask, [ja] §2.1, [de] §2, [ko] §2.1):  weff = q * mask. */
void sbo_apply_mask(const int8_t* q, const uint8_t* mask, int64_t n_out,
                    int64_t k, int m, int8_t* weff);

/* Canonical 2:4 packing of weff with its mask ("explicit N:M metadata",
 * [ja] §2.1).  vals[row, k/2]: the two kept codes of each group of four, in
 * index order.  meta[row, k/8]: one nibble per group (i0 in bits 1:0, i1 in
 * bits 3:2, i0 < i1), group 2j in the low nibble of byte j. */
void sbo_pack24(const int8_t* weff, const uint8_t* mask, int64_t n_out,
                int64_t k, int8_t* vals, uint8_t* meta);

/* Compressed-index packing of weff for any N:M (the "explicit N:M metadata"
 * of [ja] §2.1 with the kept values beside it), the decode pack of every
 * pattern other than 2:4.  READING of the layout: the row is cut into blocks
 * of 8 consecutive weights (8/m whole groups each).  masks8[row, k/8] is the
 * block's mask byte (bit j = position j kept; the groups' masks side by
 * side), and the kept weights' 2-bit codes (01 = +1, 11 = -1, 00 = 0) follow
 * in index order, 2*n8 bits per block with n8 = 8n/m, packed least
 * significant bit first into one bit stream per row: codes[row, k*n/(4m)]
 * bytes.  Requires k % 64 == 0. */
void sbo_pack_nm(const int8_t* weff, const uint8_t* mask, int64_t n_out,
                 int64_t k, int n, int m, uint8_t* masks8, uint8_t* codes);

/* The denser 2:4 decode code (6 bits a group of four, 1.5 bits a weight):
 * C(4,2) = 6 kept-position pairs x 3^2 ternary values = 54 states.  READING
 * of the numbering (the pages give none): pairs (0,1) (0,2) (0,3) (1,2)
 * (1,3) (2,3) are p = 0..5, a code c is the digit c mod 3 (0 -> 0, +1 -> 1,
 * -1 -> 2), state = 9 p + 3 d(c_i0) + d(c_i1); states packed least
 * significant bit first, one stream per row: out[row, 3k/16] bytes.
 * Requires a 2:4 mask (two positions of every group kept). */
void sbo_pack24_code6(const int8_t* weff, const uint8_t* mask, int64_t n_out,
                      int64_t k, uint8_t* out);

/* A4 (per-token int8 absmax; not on the pages, READING): a = max_k |x|,
 * a' = max(a, 1e-5f), xq = sign(x) * rne(fl32(127|x|) / a'), clamped to
 * [-128, 127]; a_prime[t] = a'.  All fp32 IEEE operations. */
void sbo_act_quant(const uint16_t* x, int64_t t, int64_t k, int8_t* xq,
                   float* a_prime);

/* A5: acc[ti, o] = sum_k xq[ti,k] * weff[o,k] in int64, stored as int32.
 * Returns 0, or -1 if some |acc| >= 2^31 (never for |codes| <= 127, k < 2^24). */
int sbo_gemm_acc(const int8_t* xq, const int8_t* weff, int64_t t,
                 int64_t n_out, int64_t k, int32_t* acc);

/* One element of A5, for sampled checks at full size. */
int32_t sbo_acc_at(const int8_t* xq_row, const int8_t* weff_row, int64_t k);

/* A6 (dequant): y = (float)acc * ((g * a'_t) / 127), fp32, in that order. */
void sbo_dequant(const int32_t* acc, const float* a_prime, float g, int64_t t,
                 int64_t n_out, float* y);

/* A7 (STE, [ja] §2.1, [de] §2, [ko] §2.2):  dX = g * (dY . weff), fp64. */
void sbo_grad_x(const uint16_t* dy, const int8_t* weff, float g, int64_t t,
                int64_t n_out, int64_t k, double* dx);
double sbo_grad_x_at(const uint16_t* dy, const int8_t* weff, float g,
                     int64_t n_out, int64_t k, int64_t ti, int64_t ki);

/* A8 (dense gradient flow to every master, [de] §2, [ko] §2.2, [fr] §2):
 * dW = dY^T . X, fp64; pruned weights receive their gradient too. */
void sbo_grad_w(const uint16_t* dy, const uint16_t* x, int64_t t,
                int64_t n_out, int64_t k, double* dw);
double sbo_grad_w_at(const uint16_t* dy, const uint16_t* x, int64_t t,
                     int64_t n_out, int64_t k, int64_t oi, int64_t ki);

/* Ablation of A8 named by the pages ([de] §4 "Ablationsstudien", [fr] §5):
 * gradients blocked for masked weights, dW = (dY^T . X) * mask, fp64; the
 * kept positions get exactly the dense gradient, pruned ones 0. */
void sbo_grad_w_masked(const uint16_t* dy, const uint16_t* x, const uint8_t* mask,
                       int64_t t, int64_t n_out, int64_t k, int m, double* dw);

/* Dequantised activations, the dW operand of the SBL_DW_QUANT_X reading of
 * the STE for the quantiser ([ja] 2.2 "Dual STE": the standard STE for the
 * quantisation function; detach form): xhat = RN_bf16(xq * a' / 127) taken
 * exactly, bf16 bit patterns out.  The fp64 product is exact (8 x 24 bits);
 * the fp64 quotient's one rounding cannot cross a bf16 rounding boundary:
 * a non-dyadic quotient lies at least ~2^-32 relative from every 9-bit
 * dyadic, and a dyadic one has at most 31 significant bits, so it is exact. */
void sbo_dequant_act(const int8_t* xq, const float* a_prime, int64_t t, int64_t k, uint16_t* xhat);

/* Round fp64 to bf16 (round to nearest, ties to even), bit patterns out. */
void sbo_round_bf16(const double* in, int64_t count, uint16_t* out);

/* Number of OpenMP threads the oracle runs with. */
int sbo_threads(void);

/* Set the number of OpenMP threads for later calls from this host thread
 * (values <= 0 are ignored).  Results do not depend on it: every sum is
 * exact or taken in a fixed order per output. */
void sbo_set_threads(int nthreads);

#ifdef __cplusplus
}
#endif
#endif
