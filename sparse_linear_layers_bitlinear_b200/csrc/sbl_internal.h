// Internal definitions shared by the library's host and device code.
#pragma once

#include <stdint.h>

#include "../../include/sbl.h"

namespace sbl {

// Header at the start of every prepared blob (device memory).
struct BlobHeader {
  uint32_t magic;     // kMagic once prepared
  uint32_t version;
  int64_t n_out, k;
  int32_t n, m;
  uint32_t flags;
  float gamma;        // exact absmean, fp32
  float g;            // max(gamma, 1e-5)
  uint32_t status;    // SBL_STATUS_* bits
  uint32_t pad0;
};
static_assert(sizeof(BlobHeader) <= 4096, "header must fit its 4 KB slot");

// Scratch of the prepare kernel inside the blob: per-CTA partial sums of the
// exact absmean (a 128-bit sum in units of 2^-37 and a flags word, as four
// generation-tagged words, and, when a CTA met magnitudes outside that
// format, 40 bins where bin b is an integer in units of 2^(8b - 133)), and
// the grid barrier's generation word.
constexpr int kPrepSlots = 1024;
constexpr int kExactBins = 40;
constexpr uint64_t kScratchSlotBins = 0;
constexpr uint64_t kScratchSlotFast = kScratchSlotBins + uint64_t(kPrepSlots) * kExactBins * 8;
constexpr uint64_t kScratchGen = kScratchSlotFast + uint64_t(kPrepSlots) * 32;
constexpr uint64_t kScratchBytes = kScratchGen + 256;

constexpr uint32_t kMagic = 0x314C4253u;  // "SBL1"
constexpr uint64_t kHeaderBytes = 4096;

inline uint64_t align_up(uint64_t v, uint64_t a) { return (v + a - 1) / a * a; }

// Padded extents of the tensor-core metadata section.
// Rows pad to 256: the pair GEMM reads the metadata of two 128-row blocks per tile.
inline int64_t meta_rows_padded(int64_t n_out) { return (n_out + 255) / 256 * 256; }
inline int64_t meta_k_padded(int64_t k) { return (k + 255) / 256 * 256; }

}  // namespace sbl
