// host_common.h - host-side helpers shared by the launch code: TMA tensor-map
// encoding through the driver entry point, and small validation utilities.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mla.h"

namespace mla {

// Encode a bf16 tiled tensor map (no interleave, zero fill outside the tensor).
// dims/box are innermost-first; strides_bytes has rank-1 entries (dims 1..rank-1).
// Returns false if the driver entry point is missing or rejects the map.
bool encode_bf16_map(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                     const uint64_t* strides_bytes, const uint32_t* box,
                     CUtensorMapSwizzle swizzle);

inline bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

// Common dims validation: returns MLA_OK or MLA_ERR_INVALID_ARG.
mla_status check_dims(const mla_dims* d);

inline int32_t row_width(const mla_dims* d) {
  return d->kv_lora_rank + d->num_kv_groups * d->rope_dim;
}

}  // namespace mla
