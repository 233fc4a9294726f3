// Host-side launchers of the Sparse-BitLinear kernels (internal).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sbl_internal.h"

namespace sbl {

// Host-side count of submitted kernel launches (sbl_launch_count).
void note_launch();
inline cudaError_t counted(cudaError_t e) {
  if (e == cudaSuccess) note_launch();
  return e;
}

// Launch with programmatic stream serialisation: the kernel may start before
// its predecessor on the stream completes and must call pdl_wait() before it
// touches that predecessor's data, and before it completes.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return counted(cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...));
}

// Destinations of the pack pass (device pointers; optional ones may be null).
struct PackOut {
  int mask_from_codes;  // select on the ternary codes instead of the master magnitudes
  uint8_t* mask;
  int8_t* codes;
  uint16_t* weff_bf16;
  int8_t* sp_values;
  uint8_t* sp_meta;
  uint8_t* gemv;
  int meta_kblocks;
  // decode pack of patterns other than 2:4 (gemv != nullptr): kept codes per
  // block of 8, code bytes per lane and unit, unit bytes, units per row
  int gemv_n8, gemv_cb, gemv_unit_bytes, gemv_upr;
  int gemv_code6;  // 2:4: the 6-bit group states instead of a byte per group
};

// mode 0: the whole preparation; 1: only the exact sum of |w| (SBL_SUM_WORDS
// words to sum_out); 2: the preparation with the scale from sum_in (the sum
// words of numel weights).
cudaError_t launch_prepare(const uint16_t* w, int64_t n_out, int64_t k, int n, int m, uint32_t flags, uint8_t* blob,
                           const sbl_blob_layout& L, int num_sms, cudaStream_t s, int mode = 0,
                           uint64_t* sum_out = nullptr, const uint64_t* sum_in = nullptr, uint64_t numel = 0);

// One matrix of a grouped preparation (launch_prepare_group): every matrix
// of a group has the same m.
constexpr int kPrepMaxGroup = 8;
struct PrepMatrix {
  const uint16_t* w;
  int64_t n_out, k;
  int n, m;
  uint32_t flags;
  uint8_t* blob;
  const sbl_blob_layout* layout;
};
cudaError_t launch_prepare_group(const PrepMatrix* mats, int count, int num_sms, cudaStream_t s);

// early_trigger: wait for the predecessor, then let the next kernel launch at
// once (it must wait for this one before reading xq / a_prime).
cudaError_t launch_act_quant(const uint16_t* x, int64_t t, int64_t k, int8_t* xq, float* a_prime, uint32_t* status,
                             int num_sms, cudaStream_t s, bool early_trigger = false);

// The dequantised activations xhat = RN_bf16(xq * a' / 127), bf16 [t][k]: the
// act-quant pass writing xhat instead of the codes (SBL_DW_QUANT_X).
cudaError_t launch_act_dequant(const uint16_t* x, int64_t t, int64_t k, uint16_t* xhat, uint32_t* status, int num_sms,
                               cudaStream_t s);

// Forward GEMM + dequant.  sparse: codes = 2:4 kept values [n_out][k/2] and
// meta = tensor-core metadata; dense: codes = W_eff int8 [n_out][k].
// x_quantise (optional, bf16 [t][k], k <= 3072): the launch quantises the
// activations itself, writing xq and a_prime before its GEMM reads them, with
// forward_tile_counters(t) uint32 counters at `ready` (zeroed by this call).
cudaError_t launch_forward_gemm(bool sparse, const int8_t* codes, const uint8_t* meta, int meta_kblocks,
                                uint64_t meta_bytes, const int8_t* xq, const float* a_prime, const float* g, int64_t n_out, int64_t t,
                                int64_t k, float* y, int32_t* acc_out, uint32_t* status, int num_sms,
                                cudaStream_t s, const uint16_t* x_quantise = nullptr, uint32_t* ready = nullptr);
int64_t forward_tile_counters(int64_t t);
constexpr int64_t kFusedActQuantMaxK = 3072;

// Decode forward for 1 <= t <= 32 tokens over the decode pack (2:4: one byte
// per group of four, or with code6 a 6-bit state per group; other N:M: the
// interleaved compressed-index pack, see gemv.cu).  For t up to 4 the kernel quantises the activations itself
// (xq_out / ap_out, when given, receive the codes and scales); otherwise, or
// when x is NULL, xq_in / ap_in hold the codes (the act-quant kernel runs
// first with its early trigger).  gemv_fits() says whether the token rows fit
// the kernel's shared memory.
uint64_t decode_pack_bytes(int64_t n_out, int64_t k, int n, int m, bool code6);
bool gemv_fits(int64_t t, int64_t k, int n, int m, bool code6);
bool gemv_preferred(int64_t t, int64_t n_out, int64_t k);
bool gemv_fuses_act_quant(int64_t t);
cudaError_t launch_forward_gemv(const uint8_t* gemv, int n, int m, bool code6, const uint16_t* x, const int8_t* xq_in,
                                const float* ap_in, const float* g, int64_t n_out, int64_t t, int64_t k, float* y,
                                int32_t* acc_out, int8_t* xq_out, float* ap_out, uint32_t* status, int num_sms,
                                cudaStream_t s);

// out[M][N] = alpha * A . B^T in bf16 x bf16 -> fp32 (tensor cores).
//   a_mn: A stored [K][M] (else [M][K]);  b_mn: B stored [K][N] (else [N][K]).
//   mask (optional): N:M keep bits [M][N/mask_m]; out is zeroed where a bit is clear.
cudaError_t launch_bf16_gemm(bool a_mn, bool b_mn, bool out_f32, const uint16_t* A, const uint16_t* B, int64_t M,
                             int64_t N, int64_t K, const float* alpha, void* out, uint32_t* status, int num_sms,
                             cudaStream_t s, const uint8_t* mask = nullptr, int mask_m = 0);

// dX = g * dY . W_eff and dW = dY^T . X in one launch.  Sets *done = false
// (and enqueues nothing) when the tile count exceeds the launch's schedule.
// dw_mask (optional): the layer's mask section; dW is zeroed at pruned positions.
cudaError_t launch_bf16_backward_dual(bool out_f32, const uint16_t* dy, const uint16_t* weff, const uint16_t* x,
                                      int64_t t, int64_t n_out, int64_t k, const float* g, void* dx, void* dw,
                                      const uint8_t* dw_mask, int mask_m, uint32_t* status, int num_sms,
                                      cudaStream_t s, bool* done);

cudaError_t launch_selftest_wait(uint32_t* status, uint64_t limit_ns, cudaStream_t s);
cudaError_t launch_chain_floor(int blocks, cudaStream_t s);
// Resident-operand tensor-pipe rate of a GEMM stage (kind 0: 2:4 int8
// forward, 1: dense int8 forward, 2: bf16 backward).
cudaError_t launch_mma_rate(int kind, int stages, int pairs, uint32_t* status, cudaStream_t s);
int64_t mma_rate_macs_per_stage(int kind);

// cuTensorMapEncodeTiled, resolved through the runtime's driver entry point.
bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle);

}  // namespace sbl
