// Ring handle layout shared by the host-side entry points.
#pragma once

#include <cstdint>

#include "../../include/cca.h"

namespace cca {
constexpr int kMaxWindow = 15;  // at most 1 + 15 cached chunks + the current one
}  // namespace cca

struct cca_kv_ring {
  cca_kv_ring_desc d;
  int64_t n_appended;  // chunks appended so far = index of the current chunk
};

namespace cca {
int ring_slot_of(const cca_kv_ring *r, int64_t chunk);
// Fills the slots / chunk ids visible (cached) for the current chunk; returns their count.
int ring_visible(const cca_kv_ring *r, int32_t *slots, int64_t *chunk_ids);
size_t dtype_bytes(cca_dtype t);
}  // namespace cca
