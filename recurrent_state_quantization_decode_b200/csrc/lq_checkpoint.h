// Internal interface of the checkpoint copies (lq_checkpoint.cu), used by the
// C ABI (lq_capi.cu).  Not installed; callers use include/leapquant.h.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

namespace lq {

// One tile record per (sequence, value head) moves between a state's records
// and pool slot slots[b] ([slot][Hv][record_bytes]); slots[b] < 0 skips
// sequence b.  save: the tile must be on a window boundary (buf_n == 0), else
// bit `err_bad_phase` is set in *err and the tile is skipped.  restore: the
// record is copied in and buf_n set to 0.
cudaError_t launch_checkpoint(bool save, int B, int Hv, int record_bytes, int num_slots,
                              const int32_t *slots, uint8_t *records, uint8_t *pool,
                              int32_t *buf_n, int32_t *err, int err_bad_phase,
                              cudaStream_t stream);

// Speculative-decoding rollback: drop the last drop[b] buffered tokens of
// every tile of sequence b (buf_n -= drop[b]); drop[b] > buf_n (a fold
// happened since the draft began) or drop[b] < 0 sets `err_bad_phase` and
// leaves the tile unchanged.
cudaError_t launch_rewind(int B, int Hv, const int32_t *drop, int32_t *buf_n, int32_t *err,
                          int err_bad_phase, cudaStream_t stream);

}  // namespace lq
