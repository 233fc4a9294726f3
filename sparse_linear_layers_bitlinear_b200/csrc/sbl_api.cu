// C ABI of the Sparse-BitLinear library: argument checks, prepared-blob
// layout and dispatch to the kernels.  See include/sbl.h for the contract.
#include <atomic>
#include <cstddef>
#include <cstring>
#include <mutex>

#include "sbl_kernels.h"

using namespace sbl;

namespace sbl {
namespace {
std::atomic<uint64_t> g_launches{0};
}  // namespace
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
}  // namespace sbl

namespace {

constexpr int64_t kMaxK = 131072;  // keeps |acc| <= 127 * k below 2^24: (float)acc is exact
constexpr uint32_t kLayerFlags = SBL_PACK_GEMV | SBL_MASK_FROM_QUANT | SBL_PACK_GEMV_6BIT | SBL_FUSE_ACT_QUANT;
constexpr uint32_t kBackwardFlags = SBL_GRAD_F32 | SBL_NO_DX | SBL_NO_DW | SBL_MASKED_GRAD | SBL_DW_QUANT_X;

struct DeviceInfo {
  bool checked = false;
  bool ok = false;
  int num_sms = 0;
};

DeviceInfo g_devices[64];
std::mutex g_dev_mutex;

// Current device must be sm_100 (B200).  Cached per device ordinal.
sbl_status current_device(int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SBL_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  DeviceInfo& d = g_devices[dev];
  if (!d.checked) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return SBL_ERR_CUDA;
    d.ok = (prop.major == 10 && prop.minor == 0);
    d.num_sms = prop.multiProcessorCount;
    d.checked = true;
  }
  if (!d.ok) return SBL_ERR_DEVICE;
  *num_sms = d.num_sms;
  return SBL_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

sbl_status check_shape(int64_t n_out, int64_t k, int n, int m, uint32_t flags) {
  if ((flags & ~kLayerFlags) != 0u) return SBL_ERR_INVALID_ARG;
  if (!(m == 2 || m == 4 || m == 8) || n < 1 || n > m) return SBL_ERR_UNSUPPORTED_NM;
  if (flags & SBL_PACK_GEMV_6BIT) {  // a form of the 2:4 decode pack
    if (!(flags & SBL_PACK_GEMV)) return SBL_ERR_INVALID_ARG;
    if (!(n == 2 && m == 4)) return SBL_ERR_UNSUPPORTED_NM;
  }
  if (n_out < 8 || n_out % 8 != 0 || k < 64 || k % 64 != 0) return SBL_ERR_SHAPE;
  if (k > kMaxK || n_out > (int64_t(1) << 30) || n_out * k > (int64_t(1) << 40)) return SBL_ERR_SHAPE;
  return SBL_OK;
}

bool is_24(int n, int m) { return n == 2 && m == 4; }

sbl_status check_layer(const sbl_layer* layer, sbl_blob_layout* L) {
  if (layer == nullptr || layer->prepared == nullptr) return SBL_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(layer->prepared) & 255u) != 0) return SBL_ERR_ALIGN;
  return sbl_prepared_layout(layer->n_out, layer->k, layer->n, layer->m, layer->flags, L);
}

bool code6(const sbl_layer* layer) { return (layer->flags & SBL_PACK_GEMV_6BIT) != 0u; }

// The decode kernel takes the call when the layer has the decode pack and the
// token rows fit its shared memory.
bool uses_decode(const sbl_layer* layer, const sbl_blob_layout& L, int64_t t) {
  return L.gemv != 0 && gemv_fits(t, layer->k, layer->n, layer->m, code6(layer)) &&
         gemv_preferred(t, layer->n_out, layer->k);
}

template <class T>
T* at(const sbl_layer* layer, uint64_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(layer->prepared) + off);
}

}  // namespace

extern "C" {

const char* sbl_version(void) { return "sbl 0.1 (sm_100a)"; }

int sbl_forward_uses_gemv(const sbl_layer* layer, int64_t t) {
  sbl_blob_layout L;
  if (check_layer(layer, &L) != SBL_OK || t <= 0) return 0;
  return uses_decode(layer, L, t) ? 1 : 0;
}

uint64_t sbl_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

sbl_status sbl_prepared_layout(int64_t n_out, int64_t k, int n, int m, uint32_t flags, sbl_blob_layout* out) {
  if (out == nullptr) return SBL_ERR_INVALID_ARG;
  const sbl_status st = check_shape(n_out, k, n, m, flags);
  if (st != SBL_OK) return st;
  sbl_blob_layout L;
  std::memset(&L, 0, sizeof(L));
  uint64_t off = 0;
  L.header = off;
  off += kHeaderBytes;
  L.scratch = off;
  off = align_up(off + kScratchBytes, 256);
  auto take = [&](uint64_t bytes) {
    const uint64_t at_off = off;
    off = align_up(off + bytes, 256);
    return at_off;
  };
  L.mask = take(uint64_t(n_out) * uint64_t(k / m));
  L.weff_bf16 = take(uint64_t(n_out) * uint64_t(k) * 2);
  if (is_24(n, m)) {
    L.sp_values = take(uint64_t(n_out) * uint64_t(k / 2));
    L.sp_meta_bytes = uint64_t(meta_rows_padded(n_out)) * uint64_t(meta_k_padded(k) / 8);
    L.sp_meta = take(L.sp_meta_bytes);
  } else {
    L.codes = take(uint64_t(n_out) * uint64_t(k));
  }
  if (flags & SBL_PACK_GEMV) {
    L.gemv_bytes = decode_pack_bytes(n_out, k, n, m, (flags & SBL_PACK_GEMV_6BIT) != 0u);
    L.gemv = take(L.gemv_bytes);
  }
  L.total_bytes = off;
  L.gamma = L.header + offsetof(BlobHeader, gamma);
  L.g = L.header + offsetof(BlobHeader, g);
  L.status = L.header + offsetof(BlobHeader, status);
  *out = L;
  return SBL_OK;
}

size_t sbl_prepared_bytes(int64_t n_out, int64_t k, int n, int m, uint32_t flags) {
  sbl_blob_layout L;
  if (sbl_prepared_layout(n_out, k, n, m, flags, &L) != SBL_OK) return 0;
  return static_cast<size_t>(L.total_bytes);
}

size_t sbl_workspace_bytes(int64_t t, int64_t k) {
  if (t < 0 || k < 0) return 0;
  return static_cast<size_t>(align_up(uint64_t(t) * uint64_t(k), 256) + align_up(uint64_t(t) * 4, 256) +
                             align_up(uint64_t(forward_tile_counters(t)) * 4, 256));
}

sbl_status sbl_prepare_weights(const sbl_layer* layer, const void* w_master, sbl_stream_t stream) {
  sbl_blob_layout L;
  sbl_status st = check_layer(layer, &L);
  if (st != SBL_OK) return st;
  if (w_master == nullptr) return SBL_ERR_INVALID_ARG;
  if (!aligned16(w_master)) return SBL_ERR_ALIGN;
  int sms = 0;
  if ((st = current_device(&sms)) != SBL_OK) return st;
  const cudaError_t e =
      launch_prepare(static_cast<const uint16_t*>(w_master), layer->n_out, layer->k, layer->n, layer->m, layer->flags,
                     static_cast<uint8_t*>(layer->prepared), L, sms, reinterpret_cast<cudaStream_t>(stream), 0,
                     nullptr, nullptr, uint64_t(layer->n_out) * uint64_t(layer->k));
  return e == cudaSuccess ? SBL_OK : SBL_ERR_CUDA;
}

sbl_status sbl_prepare_weights_grouped(const sbl_layer* layers, const void* const* w_masters, int32_t count,
                                       sbl_stream_t stream) {
  if (layers == nullptr || w_masters == nullptr || count < 1 || count > kPrepMaxGroup) return SBL_ERR_INVALID_ARG;
  sbl_blob_layout L[kPrepMaxGroup];
  PrepMatrix mats[kPrepMaxGroup];
  for (int i = 0; i < count; ++i) {
    const sbl_status st = check_layer(&layers[i], &L[i]);
    if (st != SBL_OK) return st;
    if (layers[i].m != layers[0].m) return SBL_ERR_UNSUPPORTED_NM;
    if (w_masters[i] == nullptr) return SBL_ERR_INVALID_ARG;
    if (!aligned16(w_masters[i])) return SBL_ERR_ALIGN;
    for (int j = 0; j < i; ++j)
      if (layers[j].prepared == layers[i].prepared) return SBL_ERR_INVALID_ARG;  // one blob, two matrices
    mats[i] = PrepMatrix{static_cast<const uint16_t*>(w_masters[i]), layers[i].n_out, layers[i].k, layers[i].n,
                         layers[i].m, layers[i].flags, static_cast<uint8_t*>(layers[i].prepared), &L[i]};
  }
  int sms = 0;
  const sbl_status st = current_device(&sms);
  if (st != SBL_OK) return st;
  if (count > sms) return SBL_ERR_INVALID_ARG;
  return launch_prepare_group(mats, count, sms, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? SBL_OK
                                                                                                       : SBL_ERR_CUDA;
}

sbl_status sbl_weight_abs_sum(const sbl_layer* layer, const void* w_master, uint64_t* sum_out, sbl_stream_t stream) {
  sbl_blob_layout L;
  sbl_status st = check_layer(layer, &L);
  if (st != SBL_OK) return st;
  if (w_master == nullptr || sum_out == nullptr) return SBL_ERR_INVALID_ARG;
  if (!aligned16(w_master) || !aligned16(sum_out)) return SBL_ERR_ALIGN;
  int sms = 0;
  if ((st = current_device(&sms)) != SBL_OK) return st;
  const cudaError_t e =
      launch_prepare(static_cast<const uint16_t*>(w_master), layer->n_out, layer->k, layer->n, layer->m, layer->flags,
                     static_cast<uint8_t*>(layer->prepared), L, sms, reinterpret_cast<cudaStream_t>(stream), 1, sum_out,
                     nullptr, uint64_t(layer->n_out) * uint64_t(layer->k));
  return e == cudaSuccess ? SBL_OK : SBL_ERR_CUDA;
}

sbl_status sbl_prepare_weights_from_sum(const sbl_layer* layer, const void* w_master, const uint64_t* global_sum,
                                        int64_t global_numel, sbl_stream_t stream) {
  sbl_blob_layout L;
  sbl_status st = check_layer(layer, &L);
  if (st != SBL_OK) return st;
  if (w_master == nullptr || global_sum == nullptr) return SBL_ERR_INVALID_ARG;
  if (global_numel < layer->n_out * layer->k) return SBL_ERR_SHAPE;
  if (!aligned16(w_master) || !aligned16(global_sum)) return SBL_ERR_ALIGN;
  int sms = 0;
  if ((st = current_device(&sms)) != SBL_OK) return st;
  const cudaError_t e =
      launch_prepare(static_cast<const uint16_t*>(w_master), layer->n_out, layer->k, layer->n, layer->m, layer->flags,
                     static_cast<uint8_t*>(layer->prepared), L, sms, reinterpret_cast<cudaStream_t>(stream), 2, nullptr,
                     global_sum, uint64_t(global_numel));
  return e == cudaSuccess ? SBL_OK : SBL_ERR_CUDA;
}

sbl_status sbl_forward(const sbl_layer* layer, const void* x, int64_t t, float* y, int8_t* xq_out, float* xscale_out,
                       int32_t* acc_debug, void* workspace, sbl_stream_t stream) {
  sbl_blob_layout L;
  sbl_status st = check_layer(layer, &L);
  if (st != SBL_OK) return st;
  if (t < 0 || t > (int64_t(1) << 30)) return SBL_ERR_SHAPE;
  if (t == 0) return SBL_OK;
  if (x == nullptr || y == nullptr) return SBL_ERR_INVALID_ARG;
  int8_t* xq = xq_out;
  float* ap = xscale_out;
  if (xq == nullptr || ap == nullptr) {
    if (workspace == nullptr) return SBL_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SBL_ERR_ALIGN;
  }
  uint32_t* ready = nullptr;  // token-tile counters of the in-launch quantisation
  if (workspace != nullptr && (reinterpret_cast<uintptr_t>(workspace) & 255u) == 0) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const uint64_t codes_bytes = align_up(uint64_t(t) * uint64_t(layer->k), 256);
    if (xq == nullptr) xq = reinterpret_cast<int8_t*>(ws);
    if (ap == nullptr) ap = reinterpret_cast<float*>(ws + codes_bytes);
    ready = reinterpret_cast<uint32_t*>(ws + codes_bytes + align_up(uint64_t(t) * 4, 256));
  }
  if (!aligned16(x) || !aligned16(y) || !aligned16(xq) || !aligned16(ap) || !aligned16(acc_debug))
    return SBL_ERR_ALIGN;
  int sms = 0;
  if ((st = current_device(&sms)) != SBL_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* status = at<uint32_t>(layer, L.status);
  const float* g = at<const float>(layer, L.g);
  if (uses_decode(layer, L, t)) {
    // decode: the packed weight stream
    const bool fused = gemv_fuses_act_quant(t);
    if (!fused &&
        launch_act_quant(static_cast<const uint16_t*>(x), t, layer->k, xq, ap, status, sms, s, true) != cudaSuccess)
      return SBL_ERR_CUDA;
    const cudaError_t e =
        launch_forward_gemv(at<const uint8_t>(layer, L.gemv), layer->n, layer->m, code6(layer),
                            static_cast<const uint16_t*>(x),
                            fused ? nullptr : xq, ap, g,
                            layer->n_out, t, layer->k, y, acc_debug, fused ? xq_out : nullptr,
                            fused ? xscale_out : nullptr, status, sms, s);
    return e == cudaSuccess ? SBL_OK : SBL_ERR_CUDA;
  }
  // SBL_FUSE_ACT_QUANT: the GEMM launch quantises the activations itself
  // (rows up to kFusedActQuantMaxK, counters in the workspace)
  const bool fuse = (layer->flags & SBL_FUSE_ACT_QUANT) && ready != nullptr && layer->k <= kFusedActQuantMaxK;
  const uint16_t* xq_src = fuse ? static_cast<const uint16_t*>(x) : nullptr;
  cudaError_t e = cudaSuccess;
  if (!fuse) {
    // the forward GEMM is launched with programmatic dependent launch and waits
    // for the quantiser's outputs itself, so the quantiser lets it launch early
    e = launch_act_quant(static_cast<const uint16_t*>(x), t, layer->k, xq, ap, status, sms, s, true);
    if (e != cudaSuccess) return SBL_ERR_CUDA;
  }
  if (is_24(layer->n, layer->m)) {
    e = launch_forward_gemm(true, at<const int8_t>(layer, L.sp_values), at<const uint8_t>(layer, L.sp_meta),
                            static_cast<int>(meta_k_padded(layer->k) / 128), L.sp_meta_bytes, xq, ap, g, layer->n_out,
                            t, layer->k, y, acc_debug, status, sms, s, xq_src, ready);
  } else {
    e = launch_forward_gemm(false, at<const int8_t>(layer, L.codes), nullptr, 0, 0, xq, ap, g, layer->n_out, t, layer->k,
                            y, acc_debug, status, sms, s, xq_src, ready);
  }
  return e == cudaSuccess ? SBL_OK : SBL_ERR_CUDA;
}

sbl_status sbl_forward_quantized(const sbl_layer* layer, const int8_t* xq, const float* xscale, int64_t t, float* y,
                                 int32_t* acc_debug, sbl_stream_t stream) {
  sbl_blob_layout L;
  sbl_status st = check_layer(layer, &L);
  if (st != SBL_OK) return st;
  if (t < 0 || t > (int64_t(1) << 30)) return SBL_ERR_SHAPE;
  if (t == 0) return SBL_OK;
  if (xq == nullptr || xscale == nullptr || y == nullptr) return SBL_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(xscale) || !aligned16(y) || !aligned16(acc_debug)) return SBL_ERR_ALIGN;
  int sms = 0;
  if ((st = current_device(&sms)) != SBL_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* status = at<uint32_t>(layer, L.status);
  const float* g = at<const float>(layer, L.g);
  cudaError_t e;
  if (uses_decode(layer, L, t)) {
    e = launch_forward_gemv(at<const uint8_t>(layer, L.gemv), layer->n, layer->m, code6(layer), nullptr, xq, xscale, g,
                            layer->n_out, t, layer->k, y,
                            acc_debug, nullptr, nullptr, status, sms, s);
  } else if (is_24(layer->n, layer->m)) {
    e = launch_forward_gemm(true, at<const int8_t>(layer, L.sp_values), at<const uint8_t>(layer, L.sp_meta),
                            static_cast<int>(meta_k_padded(layer->k) / 128), L.sp_meta_bytes, xq, xscale, g,
                            layer->n_out, t, layer->k, y, acc_debug, status, sms, s);
  } else {
    e = launch_forward_gemm(false, at<const int8_t>(layer, L.codes), nullptr, 0, 0, xq, xscale, g, layer->n_out, t,
                            layer->k, y, acc_debug, status, sms, s);
  }
  return e == cudaSuccess ? SBL_OK : SBL_ERR_CUDA;
}

sbl_status sbl_quantize_activations(const void* x, int64_t t, int64_t k, int8_t* xq_out, float* xscale_out,
                                    uint32_t* status_dev, sbl_stream_t stream) {
  if (t < 0 || t > (int64_t(1) << 30) || k < 64 || k % 64 != 0 || k > kMaxK) return SBL_ERR_SHAPE;
  if (t == 0) return SBL_OK;
  if (x == nullptr || xq_out == nullptr || xscale_out == nullptr || status_dev == nullptr) return SBL_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(xq_out) || !aligned16(xscale_out) || (reinterpret_cast<uintptr_t>(status_dev) & 3u))
    return SBL_ERR_ALIGN;
  int sms = 0;
  const sbl_status st = current_device(&sms);
  if (st != SBL_OK) return st;
  return launch_act_quant(static_cast<const uint16_t*>(x), t, k, xq_out, xscale_out, status_dev, sms,
                          reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SBL_OK
             : SBL_ERR_CUDA;
}

size_t sbl_backward_workspace_bytes(int64_t t, int64_t k, uint32_t flags) {
  if (t <= 0 || k <= 0 || (flags & SBL_NO_DW) || !(flags & SBL_DW_QUANT_X)) return 0;
  return size_t(t) * size_t(k) * 2;
}

sbl_status sbl_backward(const sbl_layer* layer, const void* x, const void* dy, int64_t t, void* dx, void* dw,
                        uint32_t flags, sbl_stream_t stream) {
  return sbl_backward_ws(layer, x, dy, t, dx, dw, flags, nullptr, stream);
}

sbl_status sbl_backward_ws(const sbl_layer* layer, const void* x, const void* dy, int64_t t, void* dx, void* dw,
                           uint32_t flags, void* workspace, sbl_stream_t stream) {
  sbl_blob_layout L;
  sbl_status st = check_layer(layer, &L);
  if (st != SBL_OK) return st;
  if ((flags & ~kBackwardFlags) != 0u) return SBL_ERR_INVALID_ARG;
  if (t < 0 || t > (int64_t(1) << 30)) return SBL_ERR_SHAPE;
  const bool want_dx = !(flags & SBL_NO_DX), want_dw = !(flags & SBL_NO_DW);
  // the detach-form STE takes dW against xhat, written into the workspace
  const bool quant_x = want_dw && (flags & SBL_DW_QUANT_X) && t > 0;
  if (quant_x && workspace == nullptr) return SBL_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return SBL_ERR_ALIGN;
  const bool f32 = (flags & SBL_GRAD_F32) != 0u;
  // the blocked-gradient ablation multiplies dW by the mask section
  const uint8_t* dw_mask = (flags & SBL_MASKED_GRAD) ? at<const uint8_t>(layer, L.mask) : nullptr;
  if ((want_dx && dx == nullptr) || (want_dw && dw == nullptr)) return SBL_ERR_INVALID_ARG;
  if (t > 0 && ((want_dx || want_dw) && dy == nullptr)) return SBL_ERR_INVALID_ARG;
  if (t > 0 && want_dw && x == nullptr) return SBL_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(dy) || !aligned16(dx) || !aligned16(dw)) return SBL_ERR_ALIGN;
  int sms = 0;
  if ((st = current_device(&sms)) != SBL_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t esize = f32 ? 4 : 2;
  if (t == 0) {  // empty batch: dX is empty and dW = 0
    if (want_dw && cudaMemsetAsync(dw, 0, size_t(layer->n_out) * size_t(layer->k) * esize, s) != cudaSuccess)
      return SBL_ERR_CUDA;
    return SBL_OK;
  }
  uint32_t* status = at<uint32_t>(layer, L.status);
  const void* x_dw = x;  // the dW operand: x, or xhat with SBL_DW_QUANT_X
  if (quant_x) {
    uint16_t* xhat = static_cast<uint16_t*>(workspace);
    if (launch_act_dequant(static_cast<const uint16_t*>(x), t, layer->k, xhat, status, sms, s) != cudaSuccess)
      return SBL_ERR_CUDA;
    x_dw = xhat;
  }
  if (want_dx && want_dw) {
    bool done = false;
    const cudaError_t e = launch_bf16_backward_dual(
        f32, static_cast<const uint16_t*>(dy), at<const uint16_t>(layer, L.weff_bf16), static_cast<const uint16_t*>(x_dw),
        t, layer->n_out, layer->k, at<const float>(layer, L.g), dx, dw, dw_mask, layer->m, status, sms, s, &done);
    if (e != cudaSuccess) return SBL_ERR_CUDA;
    if (done) return SBL_OK;
  }
  if (want_dx) {
    // dX[t, k] = g * dY[t, n_out] . W_eff[n_out, k]:  A = dY (K-major), B = W_eff stored [K][N].
    const cudaError_t e = launch_bf16_gemm(false, true, f32, static_cast<const uint16_t*>(dy),
                                           at<const uint16_t>(layer, L.weff_bf16), t, layer->k, layer->n_out,
                                           at<const float>(layer, L.g), dx, status, sms, s);
    if (e != cudaSuccess) return SBL_ERR_CUDA;
  }
  if (want_dw) {
    // dW[n_out, k] = dY^T . X (or xhat):  A = dY stored [K=t][M=n_out], B = X stored [K=t][N=k].
    const cudaError_t e = launch_bf16_gemm(true, true, f32, static_cast<const uint16_t*>(dy),
                                           static_cast<const uint16_t*>(x_dw), layer->n_out, layer->k, t, nullptr, dw,
                                           status, sms, s, dw_mask, layer->m);
    if (e != cudaSuccess) return SBL_ERR_CUDA;
  }
  return SBL_OK;
}

sbl_status sbl_read_status(const sbl_layer* layer, sbl_stream_t stream, uint32_t* bits_out) {
  sbl_blob_layout L;
  const sbl_status st = check_layer(layer, &L);
  if (st != SBL_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t bits = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return SBL_ERR_CUDA;
  if (cudaMemcpy(&bits, at<uint32_t>(layer, L.status), 4, cudaMemcpyDeviceToHost) != cudaSuccess) return SBL_ERR_CUDA;
  if (bits_out) *bits_out = bits;
  if (bits & SBL_STATUS_TIMEOUT) return SBL_ERR_TIMEOUT;
  if (bits & (SBL_STATUS_NONFINITE_W | SBL_STATUS_NONFINITE_X)) return SBL_ERR_NONFINITE;
  return SBL_OK;
}

sbl_status sbl_clear_status(const sbl_layer* layer, sbl_stream_t stream) {
  sbl_blob_layout L;
  const sbl_status st = check_layer(layer, &L);
  if (st != SBL_OK) return st;
  return cudaMemsetAsync(at<uint32_t>(layer, L.status), 0, 4, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SBL_OK
             : SBL_ERR_CUDA;
}

sbl_status sbl_read_scale(const sbl_layer* layer, sbl_stream_t stream, float* gamma_out, float* g_out) {
  sbl_blob_layout L;
  const sbl_status st = check_layer(layer, &L);
  if (st != SBL_OK) return st;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return SBL_ERR_CUDA;
  float v[2];
  if (cudaMemcpy(v, at<float>(layer, L.gamma), 8, cudaMemcpyDeviceToHost) != cudaSuccess) return SBL_ERR_CUDA;
  if (gamma_out) *gamma_out = v[0];
  if (g_out) *g_out = v[1];
  return SBL_OK;
}

sbl_status sbl_selftest_wait_timeout(uint32_t* status_dev, uint64_t limit_ns, sbl_stream_t stream) {
  if (status_dev == nullptr) return SBL_ERR_INVALID_ARG;
  int sms = 0;
  const sbl_status st = current_device(&sms);
  if (st != SBL_OK) return st;
  return launch_selftest_wait(status_dev, limit_ns, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SBL_OK
             : SBL_ERR_CUDA;
}

sbl_status sbl_selftest_chain_floor(int32_t blocks, sbl_stream_t stream) {
  if (blocks < 1 || blocks > 65535) return SBL_ERR_INVALID_ARG;
  int sms = 0;
  const sbl_status st = current_device(&sms);
  if (st != SBL_OK) return st;
  return launch_chain_floor(blocks, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? SBL_OK : SBL_ERR_CUDA;
}

sbl_status sbl_selftest_mma_rate(int32_t kind, int32_t stages, int32_t pairs, uint32_t* status_dev,
                                 int64_t* macs_per_stage_out, sbl_stream_t stream) {
  if (status_dev == nullptr || kind < 0 || kind > 2 || stages < 1 || stages > (1 << 20) || pairs < 1)
    return SBL_ERR_INVALID_ARG;
  int sms = 0;
  const sbl_status st = current_device(&sms);
  if (st != SBL_OK) return st;
  if (pairs > sms / 2) return SBL_ERR_INVALID_ARG;
  if (macs_per_stage_out) *macs_per_stage_out = mma_rate_macs_per_stage(kind);
  return launch_mma_rate(kind, stages, pairs, status_dev, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SBL_OK
             : SBL_ERR_CUDA;
}

}  // extern "C"
