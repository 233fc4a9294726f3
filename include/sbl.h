/*
 * sbl.h -- C ABI of the Sparse-BitLinear library for NVIDIA B200 (sm_100a).
 *
 * Sparse-BitLinear is the linear layer of Sparse-BitNet ("Sparse-BitNet:
 * 1.58-bit LLMs are Naturally Friendly to Semi-Structured Sparsity",
 * arXiv 2603.05168).  Citations below name the page and section:
 *   [ja]  gist.science Japanese technical summary
 *   [de]  gist.science German technical summary
 *   [ko]  gist.science Korean technical summary
 *   [fr]  gist.science French technical summary
 *   [abs] fugumt.com English abstract
 *
 * The layer keeps bf16 master weights W [n_out, k] (row-major, nn.Linear
 * convention).  Every step ([ja] 2.1, [ko] 2.2 "dynamic mask recompute") it
 *   1. quantises all masters to ternary codes {-1, 0, +1} with the per-tensor
 *      absmean scale g ([de] 1, [fr] 1),
 *   2. recomputes an N:M mask from the master magnitudes: in each group of m
 *      consecutive weights along k keep the n largest |w|, ties to the lowest
 *      index ([ja] 2.1, [de] 2 "Maskengenerierung", [ko] 2.1),
 *   3. applies the mask after quantisation, W_eff = q * mask ([de] 2
 *      "Quant-then-Mask", [fr] 2),
 *   4. quantises activations per token to int8 with absmax, multiplies them
 *      with W_eff in int32 and rescales to fp32,
 *   5. in the backward pass uses the dual straight-through estimator: dX goes
 *      through the masked, scaled ternary weights and dW = dY^T X reaches
 *      every master weight, pruned ones included ([de] 2 "Dual STE",
 *      [ko] 2.2, [fr] 2 "Flot de Gradient Dense").
 *
 * Conventions for every entry point:
 *  - Tensor arguments are DEVICE pointers on the current CUDA device, 16-byte
 *    aligned, row-major and dense.  bf16 data is passed as `const void*`.
 *  - The caller owns and allocates every buffer (cudaMalloc, torch, ...).  The
 *    library allocates no device memory and keeps no state between calls.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream).  Calls do not synchronise, except sbl_read_status and
 *    sbl_read_scale (and the first sbl_forward_noalloc on a device, see
 *    there).
 *  - Arguments are validated before anything is enqueued; a rejected call
 *    returns an error code and enqueues nothing.
 *  - Errors that only the device can see (non-finite inputs, a bounded wait
 *    that ran out) are OR-ed into the status word inside the prepared blob and
 *    reported by sbl_read_status (sbl_quantize_activations and the self tests
 *    take a caller-owned status word instead).  Outputs of a call that raised
 *    a device error are unspecified.
 */
#ifndef SBL_H
#define SBL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st* sbl_stream_t;

typedef enum sbl_status {
  SBL_OK = 0,
  SBL_ERR_INVALID_ARG = 1,    /* null pointer, negative size, unknown flag bit */
  SBL_ERR_UNSUPPORTED_NM = 2, /* m not in {2, 4, 8}, or n < 1, or n > m */
  SBL_ERR_SHAPE = 3,          /* k % 64 != 0, n_out % 8 != 0, n_out < 8, sizes too large */
  SBL_ERR_ALIGN = 4,          /* a pointer is not 16-byte aligned */
  SBL_ERR_CUDA = 5,           /* a CUDA call failed (launch error, no device, ...) */
  SBL_ERR_NONFINITE = 6,      /* device saw a NaN/Inf master weight or activation */
  SBL_ERR_TIMEOUT = 7,        /* a device-side bounded wait gave up */
  SBL_ERR_DEVICE = 8,         /* the current device is not sm_100 */
  SBL_ERR_SCRATCH = 9         /* sbl_forward_noalloc: t * k exceeds its fixed scratch */
} sbl_status;

/* Flags of sbl_layer.flags (fixed at prepare time). */
enum {
  SBL_PACK_GEMV = 1u << 0,      /* also write the decode pack that sbl_forward streams for
                                   t <= 32 tokens (2:4: 2 bits a weight; other N:M: the
                                   compressed-index pack, 1 + 2n/m bits a weight) */
  SBL_MASK_FROM_QUANT = 1u << 1, /* ablation the pages report ([de] 4 "Ablationsstudien",
                                   [fr] 5): build the N:M mask from the ternary codes
                                   |q| instead of the masters (ties to the lowest index) */
  SBL_PACK_GEMV_6BIT = 1u << 2, /* with SBL_PACK_GEMV on a 2:4 layer: the decode pack holds
                                   each group of four as one of its 54 states in 6 bits
                                   (1.5 bits a weight) instead of a byte; any other
                                   pattern: SBL_ERR_UNSUPPORTED_NM; without SBL_PACK_GEMV:
                                   SBL_ERR_INVALID_ARG */
  SBL_FUSE_ACT_QUANT = 1u << 3  /* sbl_forward on the tensor-core GEMM path quantises the
                                   activations inside the GEMM launch (the epilogue warps
                                   of every CTA quantise token rows while the first tiles
                                   load, each tile's loads wait for its rows' count)
                                   instead of a separate kernel before it; taken when
                                   k <= 3072 and the call passes a workspace (it holds the
                                   counters), else the two-launch path.  Same bits.  The
                                   launch's CTAs must all be resident at once, which they
                                   are on an otherwise idle GPU; a stall shows as
                                   SBL_ERR_TIMEOUT.  No effect on the blob's layout */
};

/* Flags of sbl_backward's `flags` argument. */
enum {
  SBL_GRAD_F32 = 1u << 1,   /* dx and dw are fp32 instead of bf16 */
  SBL_NO_DX = 1u << 2,      /* skip dX (dx may be NULL) */
  SBL_NO_DW = 1u << 3,      /* skip dW (dw may be NULL) */
  SBL_MASKED_GRAD = 1u << 4, /* ablation the pages report ([de] 4, [fr] 5): block the
                               gradient of pruned weights, dw = (dy^T . x) * mask */
  SBL_DW_QUANT_X = 1u << 5   /* reading of the standard STE for the quantiser ([ja] 2.2
                               "Dual STE") in its detach form: dw = dy^T . xhat with
                               xhat = RN_bf16(xq * a' / 127) (xq, a' as in sbl_forward),
                               rounded once from the exact value; needs a workspace
                               (sbl_backward_ws) */
};

/* One Sparse-BitLinear layer: shapes, pattern and the caller-owned device
 * blob that sbl_prepare_weights fills.  Plain data, no hidden state. */
typedef struct sbl_layer {
  int64_t n_out;   /* output features = rows of W; multiple of 8 */
  int64_t k;       /* input features = columns of W; multiple of 64 */
  int32_t n, m;    /* keep n of every m consecutive weights along k */
  uint32_t flags;  /* SBL_PACK_* bits */
  void* prepared;  /* device buffer of sbl_prepared_bytes() bytes, 256-byte aligned */
} sbl_layer;

/* Byte offsets of the sections inside the prepared blob (0 = absent). */
typedef struct sbl_blob_layout {
  uint64_t total_bytes;
  uint64_t header;      /* 4096-byte header: shapes, gamma, g, status word */
  uint64_t mask;        /* uint8 [n_out, k/m]: bit j = position j of the group kept */
  uint64_t codes;       /* int8 [n_out, k]: W_eff codes (patterns other than 2:4) */
  uint64_t weff_bf16;   /* bf16 [n_out, k]: W_eff as exact bf16 {-1, 0, 1} (backward) */
  uint64_t sp_values;   /* int8 [n_out, k/2]: the two kept codes of each group of 4 (2:4) */
  uint64_t sp_meta;     /* tensor-core metadata (2:4), sp_meta_bytes bytes; see below */
  uint64_t sp_meta_bytes;
  uint64_t gemv;        /* decode pack (SBL_PACK_GEMV), gemv_bytes bytes; see below */
  uint64_t gamma;       /* float: exact absmean, rounded to fp32 */
  uint64_t g;           /* float: max(gamma, 1e-5), the scale used everywhere */
  uint64_t status;      /* uint32 device status word */
  uint64_t scratch;     /* partial sums of the exact absmean (written and read by sbl_prepare_weights) */
  uint64_t gemv_bytes;  /* size of the decode pack */
} sbl_blob_layout;
/* sp_meta layout: blocks of 128 rows x 128 k-positions, 2048 bytes each,
 * ordered [row_block][k_block]; inside a block, row r's 16 bytes hold 32
 * nibbles for its 32 groups of four in k order (group 2j in the low nibble
 * of byte j); a nibble is (i0 | i1 << 2) with i0 < i1 the kept positions.
 * Rows and k are padded up to multiples of 256 with nibble 0x4 over zero codes.
 * gemv layout, 2:4: one byte per group of four: the metadata nibble in the
 * high half, the two kept codes in the low half (bits 1:0 the code at i0,
 * bits 3:2 the code at i1; 00 = 0, 01 = +1, 11 = -1).  The bytes are cut into
 * units of 16 rows x 128 k (rows padded to 16 and k to 128 with zero bytes),
 * ordered [row tile][k unit], 512 bytes each: the 8 bytes of groups 8t..8t+7
 * of the unit for row r sit at 16 * (4 * (r % 8) + t) + 8 * ((r % 16) / 8).
 * gemv layout, 2:4 with SBL_PACK_GEMV_6BIT: group state 9 p + 3 d0 + d1 < 54,
 * p = 0..5 the kept pair (i0, i1) in the order (0,1) (0,2) (0,3) (1,2) (1,3)
 * (2,3), d0 / d1 the codes at i0 / i1 as digits mod 3 (0 -> 0, +1 -> 1,
 * -1 -> 2); so state 0 is an all-zero group.  Units of 16 rows x 128 k as
 * above, 384 bytes each: slot s = 4 * (r % 8) + t holds 96 bits, the 8
 * states of groups 8t..8t+7 of row r (bits 6j..6j+5 for group 8t+j), then
 * those of row r + 8 (from bit 48), least significant bit first; word j
 * (bits 32j..32j+31) of slot s sits at byte 128 * j + 4 * s of the unit.
 * gemv layout, any other N:M (compressed index: the explicit N:M metadata beside
 * the kept values, [ja] 2.1): every block of 8 consecutive weights has a mask
 * byte (bit j = position j kept) and its n8 = 8n/m kept codes in index order,
 * 2 bits each (same code values).  The pack is cut into units of 16 rows x 128
 * k (rows padded to 16 and k to 128 with zero bytes), ordered [row tile][k
 * unit].  Unit bytes: a 256-byte mask block when n < m, then a code block of
 * 32 x cb bytes, cb = 4 * ceil(2 n8 / 4).  The lane slot of a block is
 * L = 4 * (row % 8) + (b / 4) % 4 for block b = (k % 128) / 8 of the unit:
 * mask byte at L * 8 + 4 * ((row % 16) / 8) + b % 4; code field (2 n8 bits) at
 * bit 8 * n8 * ((row % 16) / 8) + 2 n8 * (b % 4) of the slot's cb bytes,
 * least significant bit first.  n = m (dense ternary) has no mask block. */

/* Size and section offsets of the prepared blob.  Host only, no CUDA call.
 * Returns SBL_ERR_* on unsupported shapes/patterns (out is then untouched). */
sbl_status sbl_prepared_layout(int64_t n_out, int64_t k, int n, int m, uint32_t flags,
                               sbl_blob_layout* out);

/* Total bytes of the prepared blob, 0 for unsupported arguments. */
size_t sbl_prepared_bytes(int64_t n_out, int64_t k, int n, int m, uint32_t flags);

/* Bytes of scratch that sbl_forward needs when xq_out / xscale_out are NULL
 * (or for SBL_FUSE_ACT_QUANT): t*k int8 codes, t fp32 scales, then one uint32
 * counter per 16 tokens, each piece starting on a 256-byte boundary. */
size_t sbl_workspace_bytes(int64_t t, int64_t k);

/* Steps 1-3 ([de] 2, [ja] 2.1, [ko] 2.1-2.2).  Reads the bf16 masters
 * `w_master` [n_out, k] and fills layer->prepared: the exact absmean gamma
 * (sum of all |w| computed exactly, rounded once to fp32), g = max(gamma,
 * 1e-5), the N:M mask from the master magnitudes, the ternary codes
 * q = sign(w) * [2|w| > g] with the mask applied after quantisation, and
 * the packed forms the forward and backward kernels read.  Resets the blob's
 * status word.  Raises SBL_ERR_NONFINITE (device) for NaN/Inf masters. */
sbl_status sbl_prepare_weights(const sbl_layer* layer, const void* w_master, sbl_stream_t stream);

/* Steps 1-3 for several layers in one launch (up to 8, all with the same m):
 * the same preparation as one sbl_prepare_weights call per layer, bit for
 * bit, with the device's SMs split among the matrices in proportion to their
 * sizes; every matrix keeps its own exact scale and its own barrier in its
 * own blob.  One launch pays the launch, the ramp of the weight stream and
 * the barrier once for the group (the per-step recompute of a transformer
 * block's linears, [ja] 2.1, [ko] 2.2).  The masters of a group should fit
 * L2 together (about 100 MB), since each matrix is read twice.
 * Errors: SBL_ERR_INVALID_ARG for count outside 1..8, a NULL pointer, two
 * layers sharing a blob or more layers than SMs; SBL_ERR_UNSUPPORTED_NM for
 * mixed m; otherwise as sbl_prepare_weights. */
sbl_status sbl_prepare_weights_grouped(const sbl_layer* layers, const void* const* w_masters, int32_t count,
                                       sbl_stream_t stream);

/* Tensor parallelism by rows of W (each rank holds n_out / R rows; groups
 * along k never split).  The scale gamma is the mean |w| over the WHOLE
 * tensor, so the shards' exact sums are added first:
 *   1. sbl_weight_abs_sum on each shard writes SBL_SUM_WORDS uint64 words;
 *   2. the words of all shards are added word by word (an integer sum, e.g.
 *      an all-reduce with SUM over uint64/int64; exact for up to 16 shards);
 *   3. sbl_prepare_weights_from_sum prepares each shard with gamma from those
 *      words over global_numel = (sum of all shards' rows) * k weights.
 * Every shard then holds the gamma, mask and codes that sbl_prepare_weights
 * gives the same rows of the whole tensor, bit for bit.  The forward needs no
 * exchange (output columns are local); dX is the sum of the shards' dX. */
#define SBL_SUM_WORDS 46

/* Step 1 above: the exact sum of |w| over this shard's masters (bf16
 * [layer->n_out, layer->k]) as SBL_SUM_WORDS words in sum_out (device, 16-byte
 * aligned): three words of 32-bit pieces of the window sum, forty bins of
 * magnitudes outside the window, and counts of non-finite, huge (>= 2^6) and
 * tiny (< 2^-30) magnitudes.  Uses the layer's blob as scratch for its grid
 * barrier and resets its status word (SBL_STATUS_NONFINITE_W is raised for
 * NaN/Inf masters); the prepared sections are left as they were. */
sbl_status sbl_weight_abs_sum(const sbl_layer* layer, const void* w_master, uint64_t* sum_out, sbl_stream_t stream);

/* Step 3 above: sbl_prepare_weights for this shard with gamma taken from the
 * summed words `global_sum` (device) over `global_numel` weights
 * (>= layer->n_out * layer->k, else SBL_ERR_SHAPE). */
sbl_status sbl_prepare_weights_from_sum(const sbl_layer* layer, const void* w_master, const uint64_t* global_sum,
                                        int64_t global_numel, sbl_stream_t stream);

/* Step 4.  x: bf16 [t, k] activations.  y: fp32 [t, n_out] output,
 *   y[i, o] = (float)acc[i, o] * ((g * a'_i) / 127),
 *   acc[i, o] = sum_k xq[i, k] * W_eff[o, k]   (int32),
 *   a'_i = max(max_k |x[i, k]|, 1e-5),  xq = sign(x) * rne(127 |x| / a'_i).
 * xq_out (int8 [t, k]) and xscale_out (fp32 [t], receives a'_i) may be NULL;
 * then `workspace` (sbl_workspace_bytes(t, k) bytes) holds them.  acc_debug
 * (int32 [t, n_out]) may be NULL; when given, the raw accumulators are
 * written too.  t == 0 is a no-op.  2:4 layers run the 2:4-sparse int8
 * tensor-core GEMM; other patterns the dense int8 one over W_eff codes.  A
 * layer prepared with SBL_PACK_GEMV takes the decode kernel over its decode
 * pack instead for t <= 32 tokens, when that many token rows of k codes fit
 * the kernel's shared memory (sbl_forward_uses_gemv says which path a call
 * takes); for t <= 4 the decode kernel also quantises the activations
 * itself, so the call is one launch.  On the GEMM path a layer with
 * SBL_FUSE_ACT_QUANT quantises inside the GEMM's launch when the call passes
 * a workspace and k <= 3072 (the workspace's counters are used even when
 * xq_out and xscale_out are given).  The outputs are the same bits on every
 * path. */
sbl_status sbl_forward(const sbl_layer* layer, const void* x, int64_t t, float* y, int8_t* xq_out,
                       float* xscale_out, int32_t* acc_debug, void* workspace, sbl_stream_t stream);

/* Step 4 from activation codes the caller already holds: xq (int8 [t, k])
 * and xscale (fp32 [t], the a'_i) exactly as sbl_forward writes them for some
 * x, e.g. from an earlier call on the same activations.  Writes the same y
 * (and acc_debug) as sbl_forward on that x, without quantising again, so
 * layers that share an input (q, k and v; gate and up) quantise it once.
 * Same dispatch as sbl_forward.  No workspace.  Errors: as sbl_forward. */
sbl_status sbl_forward_quantized(const sbl_layer* layer, const int8_t* xq, const float* xscale, int64_t t, float* y,
                                 int32_t* acc_debug, sbl_stream_t stream);

/* Step 4's activation quantisation alone: x (bf16 [t, k]) -> xq_out (int8
 * [t, k]) and xscale_out (fp32 [t], the a'_i), the same bits sbl_forward
 * computes, for sbl_forward_quantized later (e.g. on another stream, ahead of
 * the layer's weight preparation).  A non-finite activation ORs
 * SBL_STATUS_NONFINITE_X into *status_dev (a caller-owned device uint32, not
 * the layer's word, so that a prepare of the layer does not clear it).
 * Errors: SBL_ERR_SHAPE (k not a multiple of 64 in 64..131072, t out of
 * range), SBL_ERR_INVALID_ARG (a NULL pointer when t > 0), SBL_ERR_ALIGN
 * (x, xq_out, xscale_out not 16-byte aligned, status_dev not 4-byte
 * aligned), SBL_ERR_DEVICE, SBL_ERR_CUDA. */
sbl_status sbl_quantize_activations(const void* x, int64_t t, int64_t k, int8_t* xq_out, float* xscale_out,
                                    uint32_t* status_dev, sbl_stream_t stream);

/* 1 when sbl_forward on this layer with t tokens takes the decode kernel
 * over the decode pack, 0 when it takes a tensor-core GEMM (or the arguments
 * are invalid).  Host only, no device access. */
int sbl_forward_uses_gemv(const sbl_layer* layer, int64_t t);

/* Forward pass for callers that cannot allocate device memory.  The paper has
 * no counterpart: this is a deployment convenience, not a step of the method.
 *
 * Same arithmetic and outputs as sbl_forward, but the int8 activation codes
 * and per-token scales go to a fixed scratch array that the library itself
 * holds in device memory, so the caller supplies only x, y (and optionally
 * acc_debug).  Meant for code that has no way to obtain a workspace: plugins
 * whose enqueue hook must not allocate, processes whose device memory belongs
 * to an allocator they cannot reach, and latency-critical loops that cannot
 * pay for cudaMalloc's implicit synchronisation.  It calls no cudaMalloc,
 * cudaFree or other allocating routine.
 *
 * Limit: align256(t * k) + align256(4 * t) <= SBL_NOALLOC_SCRATCH_BYTES
 * (16 MiB; e.g. t = 4096 tokens at k = 2560); larger requests return
 * SBL_ERR_SCRATCH and enqueue nothing.  Every device that loads the library's
 * device code keeps those 16 MiB until the process exits.
 *
 * The first call with t > 0 on a device looks up the array's device address
 * (cudaGetSymbolAddress) and caches it by device ordinal (devices 0-63; a
 * higher ordinal returns SBL_ERR_DEVICE).  Under CUDA's lazy module loading
 * that lookup is also when the library's device code is loaded on the device
 * and the 16 MiB are committed, which can synchronise the device: make the
 * first call once, outside any region that must not allocate or stall, and
 * before any stream capture.  The cache does not see cudaDeviceReset: after a
 * reset of a device, its cached address is stale and this entry point must
 * not be called on that device again in the process.  All arguments that need
 * no device are checked before the lookup.  All calls on a device share the
 * one array and it keeps the last call's contents, so calls that can overlap
 * on the GPU (two streams,
 * two host threads) race on it: serialise them.  Nothing in the array needs to
 * start at zero; each call writes everything it reads.  Errors: as
 * sbl_forward, plus SBL_ERR_SCRATCH. */
#define SBL_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
sbl_status sbl_forward_noalloc(const sbl_layer* layer, const void* x, int64_t t, float* y, int32_t* acc_debug,
                               sbl_stream_t stream);

/* Step 5 (dual STE).  x: bf16 [t, k] (the forward input), dy: bf16 [t, n_out].
 *   dx [t, k]     = g * (dy . W_eff)          (straight through Q_w, Q_x, mask)
 *   dw [n_out, k] = dy^T . x                  (dense: every master, pruned too)
 * bf16 outputs (fp32 with SBL_GRAD_F32), fp32 accumulation on the tensor
 * cores.  SBL_NO_DX / SBL_NO_DW skip one of the two products. */
sbl_status sbl_backward(const sbl_layer* layer, const void* x, const void* dy, int64_t t, void* dx, void* dw,
                        uint32_t flags, sbl_stream_t stream);

/* Bytes of device workspace sbl_backward_ws needs for these flags: t*k*2
 * (xhat, bf16 [t, k]) with SBL_DW_QUANT_X and dW wanted, else 0. */
size_t sbl_backward_workspace_bytes(int64_t t, int64_t k, uint32_t flags);

/* sbl_backward with a caller-owned device workspace of at least
 * sbl_backward_workspace_bytes(t, layer->k, flags) bytes (16-byte aligned;
 * NULL when that is 0).  With SBL_DW_QUANT_X the activations are quantised
 * again from x (the same codes and a' as the forward pass) and written back
 * as xhat into the workspace, which then holds xhat [t, k] when the call's
 * work is done; dw = dy^T . xhat.  dX is unchanged.  Errors: as sbl_backward,
 * plus SBL_ERR_INVALID_ARG when SBL_DW_QUANT_X needs a workspace and it is
 * NULL.  sbl_backward(...) is sbl_backward_ws(..., NULL, stream). */
sbl_status sbl_backward_ws(const sbl_layer* layer, const void* x, const void* dy, int64_t t, void* dx, void* dw,
                           uint32_t flags, void* workspace, sbl_stream_t stream);

/* Synchronises `stream`, then maps the layer's device status word to a code:
 * SBL_OK, SBL_ERR_NONFINITE or SBL_ERR_TIMEOUT.  *bits_out (may be NULL)
 * receives the raw word.  The word stays set until sbl_clear_status or the
 * next sbl_prepare_weights. */
sbl_status sbl_read_status(const sbl_layer* layer, sbl_stream_t stream, uint32_t* bits_out);
sbl_status sbl_clear_status(const sbl_layer* layer, sbl_stream_t stream);

/* Copies the fp32 gamma and g of a prepared layer to the host (synchronises). */
sbl_status sbl_read_scale(const sbl_layer* layer, sbl_stream_t stream, float* gamma_out, float* g_out);

/* Failure-path self test: launches one CTA whose mbarrier wait can never
 * complete, bounded by `limit_ns`; the kernel then records SBL_STATUS_TIMEOUT
 * in *status_dev (device uint32) and returns normally.  No fault, no hang. */
sbl_status sbl_selftest_wait_timeout(uint32_t* status_dev, uint64_t limit_ns, sbl_stream_t stream);

/* Measurement aid, no counterpart in the paper: launches one empty kernel of
 * `blocks` blocks x 256 threads the way every kernel of the library is
 * launched (programmatic dependent launch: it lets its successor launch,
 * waits for its predecessor, and exits).  A chain of these in a CUDA graph
 * gives the per-call floor that a chain of dependent library calls pays
 * before any work.  Touches no memory.  Errors: SBL_ERR_INVALID_ARG for
 * blocks outside 1..65535, SBL_ERR_DEVICE, SBL_ERR_CUDA. */
sbl_status sbl_selftest_chain_floor(int32_t blocks, sbl_stream_t stream);

/* Measurement aid, no counterpart in the paper: the tensor-core rate of one
 * of the library's GEMM stages with its operands resident in shared memory.
 * `pairs` CTA pairs each issue `stages` stages of the chosen GEMM's
 * instructions back to back, with no copies, waits or epilogues between them:
 *   kind 0  the 2:4 sparse int8 forward (tile 256 x 240 tokens, 256 logical
 *           k a stage, with the stage's metadata copy into tensor memory),
 *   kind 1  the dense int8 forward of the other N:M patterns (256 x 256,
 *           128 k a stage),
 *   kind 2  the bf16 backward (256 x 256, 64 k a stage).
 * The operands are synthetic (ternary and int8 codes, valid 2:4 metadata,
 * finite bf16 values) and no result leaves the kernel, so the launch's
 * duration on `stream` gives the ceiling that the GEMM's MMA instructions
 * allow.  *macs_per_stage_out (may be NULL) receives the multiply-adds of one
 * pair's stage (logical k for 2:4).  A tensor pipe that does not drain within
 * the library's wait limit records SBL_STATUS_TIMEOUT in *status_dev (device
 * uint32).  Errors: SBL_ERR_INVALID_ARG for a NULL status_dev, kind outside
 * 0..2, stages outside 1..2^20 or pairs outside 1..SMs/2; SBL_ERR_DEVICE;
 * SBL_ERR_CUDA. */
sbl_status sbl_selftest_mma_rate(int32_t kind, int32_t stages, int32_t pairs, uint32_t* status_dev,
                                 int64_t* macs_per_stage_out, sbl_stream_t stream);

/* Bits of the device status word. */
enum {
  SBL_STATUS_NONFINITE_W = 1u << 0,
  SBL_STATUS_NONFINITE_X = 1u << 1,
  SBL_STATUS_TIMEOUT = 1u << 2
};

/* Library version string. */
const char* sbl_version(void);

/* Number of kernels this process has launched through the library so far
 * (every successful launch submission, on any device and stream; memsets and
 * copies are not counted).  A host-side counter for accounting: callers take
 * the difference across a region.  Never fails. */
uint64_t sbl_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* SBL_H */
