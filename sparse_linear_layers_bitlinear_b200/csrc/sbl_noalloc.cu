// sbl_forward_noalloc: the forward pass for callers that cannot allocate
// device memory.
//
// sbl_forward needs somewhere to put the int8 activation codes and the
// per-token scales between the activation-quantisation kernel and the GEMM.
// Normally the caller passes those buffers or a workspace.  Some callers have
// no way to get one: a plugin whose enqueue hook is not allowed to allocate,
// a process whose device memory is owned by another allocator that it cannot
// reach, or a latency-critical loop that cannot afford cudaMalloc's implicit
// device synchronisation.  For them this file keeps a fixed scratch array in
// the library's own device memory and runs the unchanged forward path on it.
#include <cstdint>
#include <mutex>

#include "sbl_internal.h"

#include <cuda_runtime.h>

namespace {

// The scratch: int8 codes [t, k] at offset 0, then fp32 scales [t] at the next
// 256-byte boundary.  Every device that loads this file's device code holds
// SBL_NOALLOC_SCRATCH_BYTES for it until the process exits.
static __device__ __align__(256) uint8_t g_noalloc_scratch[SBL_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

struct ScratchSlot {
  bool ready = false;
  uint8_t* ptr = nullptr;  // device address of g_noalloc_scratch on this device
};

ScratchSlot g_slots[kMaxDevices];
std::mutex g_slots_mutex;

// In host code `g_noalloc_scratch` names a host-side shadow, not device
// memory, so its device address is looked up once per device, with that
// device current, and cached by device ordinal (the cache is not told about a
// cudaDeviceReset; see include/sbl.h).
sbl_status scratch_on_current_device(uint8_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SBL_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SBL_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_slots_mutex);
  ScratchSlot& s = g_slots[dev];
  if (!s.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return SBL_ERR_CUDA;
    s.ptr = static_cast<uint8_t*>(p);
    s.ready = true;
  }
  *out = s.ptr;
  return SBL_OK;
}

}  // namespace

extern "C" sbl_status sbl_forward_noalloc(const sbl_layer* layer, const void* x, int64_t t, float* y,
                                          int32_t* acc_debug, sbl_stream_t stream) {
  if (layer == nullptr) return SBL_ERR_INVALID_ARG;
  sbl_blob_layout L;
  const sbl_status st = sbl_prepared_layout(layer->n_out, layer->k, layer->n, layer->m, layer->flags, &L);
  if (st != SBL_OK) return st;
  if (t < 0 || t > (int64_t(1) << 30)) return SBL_ERR_SHAPE;
  if (t == 0) return sbl_forward(layer, x, 0, y, nullptr, nullptr, acc_debug, nullptr, stream);
  const uint64_t codes_bytes = sbl::align_up(uint64_t(t) * uint64_t(layer->k), 256);
  const uint64_t scale_bytes = sbl::align_up(uint64_t(t) * 4u, 256);
  if (codes_bytes + scale_bytes > SBL_NOALLOC_SCRATCH_BYTES) return SBL_ERR_SCRATCH;
  // The argument checks of sbl_forward that need no device come first, so a
  // rejected call never reaches the scratch set-up below.
  if (layer->prepared == nullptr || x == nullptr || y == nullptr) return SBL_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(layer->prepared) & 255u) != 0 || (reinterpret_cast<uintptr_t>(x) & 15u) != 0 ||
      (reinterpret_cast<uintptr_t>(y) & 15u) != 0 || (reinterpret_cast<uintptr_t>(acc_debug) & 15u) != 0)
    return SBL_ERR_ALIGN;
  uint8_t* scratch = nullptr;
  const sbl_status sst = scratch_on_current_device(&scratch);
  if (sst != SBL_OK) return sst;
  // Nothing in the scratch needs to start at zero: the activation
  // quantisation writes every code and scale the GEMM then reads.
  return sbl_forward(layer, x, t, y, reinterpret_cast<int8_t*>(scratch), reinterpret_cast<float*>(scratch + codes_bytes),
                     acc_debug, nullptr, stream);
}
