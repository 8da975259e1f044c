// Internal interface between the C ABI's translation units (lq_capi.cu and
// lq_noalloc.cu).  Not installed; callers use include/leapquant.h.
#pragma once

#include <cstddef>
#include <cstdint>

#include "../../include/leapquant.h"

namespace lq {

// Every argument check of lq_decode_step_host except the staging pointer
// (config, state, io pointers and alignments, the active mask's alignment).
lq_status check_host_step(const lq_config *cfg, const void *q_host, const void *k_host,
                          const void *v_host, const float *alpha_host, const float *beta_host,
                          const lq_state *st, const void *out_host, const int32_t *active);

// Bytes of device staging the host-buffer step needs (valid config only).
size_t host_staging_bytes(const lq_config *cfg);

}  // namespace lq
