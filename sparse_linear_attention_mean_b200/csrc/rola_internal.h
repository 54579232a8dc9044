// Host-side helpers shared by the librola translation units.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "../../include/rola.h"

namespace rola_internal {

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Validates a shape; ROLA_ERR_INVALID_ARG for inconsistent values,
// ROLA_ERR_UNSUPPORTED for consistent ones without a kernel.
rola_status_t check_shape(const rola_shape_t* s);

// Byte offsets of the layer workspace parts.
struct LayerWs {
  size_t select, idx, S_blk, z_blk, S_glb, z_glb, total;
};
LayerWs layer_ws(const rola_shape_t* s);

}  // namespace rola_internal
