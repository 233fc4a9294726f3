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
  // Exact sum of |w|: 32 bins; bin b accumulates sig << (s & 7) for every
  // weight whose fixed-point shift s (see prep.cu) has s >> 3 == b.
  unsigned long long bins[32];
};
static_assert(sizeof(BlobHeader) <= 4096, "header must fit its 4 KB slot");

constexpr uint32_t kMagic = 0x314C4253u;  // "SBL1"
constexpr uint64_t kHeaderBytes = 4096;

inline uint64_t align_up(uint64_t v, uint64_t a) { return (v + a - 1) / a * a; }

// Padded extents of the tensor-core metadata section.
inline int64_t meta_rows_padded(int64_t n_out) { return (n_out + 127) / 128 * 128; }
inline int64_t meta_k_padded(int64_t k) { return (k + 255) / 256 * 256; }

}  // namespace sbl
