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

#ifdef __CUDACC__
#include <cuda_runtime.h>
namespace rola {
// Internal launchers shared by the entry points.
rola_status_t select_from_pooled(const rola_shape_t* s, const double* qbar, const double* kbar,
                                 double* sigma, int32_t* idx, cudaStream_t cs, const int32_t* kb_h,
                                 int32_t* dev_err);
bool prep_kernel_supports(const rola_shape_t* s);
rola_status_t launch_prep_kernel(const rola_shape_t* s, const uint16_t* q, const uint16_t* k,
                                 const uint16_t* v, const uint16_t* P, double* qbar, double* kbar,
                                 float* S_blk, float* z_blk, int32_t* dev_err, cudaStream_t cs);
rola_status_t launch_states_total(const rola_shape_t* s, const float* S_blk, const float* z_blk,
                                  float* S_glb, float* z_glb, cudaStream_t cs);
// The selector with optional per-head kept counts (kb_h, device int32 [H]
// or NULL; rows keep stride k_b, entries past a head's count are -1).
rola_status_t select_blocks_impl(const rola_shape_t* s, const int32_t* kb_h, const uint16_t* q,
                                 const uint16_t* k, int32_t* idx, double* scores_opt, void* ws,
                                 size_t ws_bytes, int32_t* dev_err, void* stream);
// The attention forward with optional per-head kept counts (kb_h, device
// int32 [H] or NULL) and the bound of each pipeline wait.
rola_status_t attention_launch(const rola_shape_t* s, const int32_t* kb_h, const uint16_t* q,
                               const uint16_t* k, const uint16_t* v, const int32_t* idx,
                               const uint16_t* P, const float* S_blk, const float* z_blk,
                               const float* S_glb, const float* z_glb, const float* gate,
                               uint16_t* out, int32_t* dev_err, uint64_t wait_limit_ns, void* stream);
}  // namespace rola
#endif
