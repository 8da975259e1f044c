// Prefix-cache checkpoints of the int8 state, and rollback inside a window.
// A checkpoint of a sequence is a
// copy of its tile records taken at a window boundary, when the in-window
// buffer is empty (news article on LeapQuant, paragraph 5: one state
// checkpoint per 1,024 tokens for prefix caching, at 1.19 bytes per value).
// Restoring it gives a state that decodes on bit for bit.

#include "lq_checkpoint.h"

namespace lq {
namespace {

constexpr int kCopyThreads = 256;

// One CTA per tile; 16-byte copies (records are multiples of 16 bytes).
__global__ void __launch_bounds__(kCopyThreads)
    checkpoint_kernel(bool save, int Hv, int record_bytes, int num_slots, const int32_t *slots,
                      uint8_t *records, uint8_t *pool, int32_t *buf_n, int32_t *err,
                      int err_bad_phase) {
  const int tile = blockIdx.x;
  const int b = tile / Hv, h = tile - b * Hv;
  const int slot = slots[b];
  if (slot < 0) return;
  if (slot >= num_slots) {
    if (threadIdx.x == 0) atomicOr(err, err_bad_phase);
    return;
  }
  if (save && buf_n[tile] != 0) {
    if (threadIdx.x == 0) atomicOr(err, err_bad_phase);
    return;
  }
  uint4 *rec = reinterpret_cast<uint4 *>(records + static_cast<size_t>(tile) * record_bytes);
  uint4 *pl = reinterpret_cast<uint4 *>(
      pool + (static_cast<size_t>(slot) * Hv + h) * record_bytes);
  const int n16 = record_bytes / 16;
  if (save) {
    for (int i = threadIdx.x; i < n16; i += kCopyThreads) pl[i] = rec[i];
  } else {
    for (int i = threadIdx.x; i < n16; i += kCopyThreads) rec[i] = pl[i];
    if (threadIdx.x == 0) buf_n[tile] = 0;
  }
}

// One thread per tile.  Within a window the record is fixed and the
// buffered tokens are appended entries, so dropping the last ones is exact.
__global__ void rewind_kernel(int tiles, int Hv, const int32_t *drop, int32_t *buf_n,
                              int32_t *err, int err_bad_phase) {
  const int tile = blockIdx.x * blockDim.x + threadIdx.x;
  if (tile >= tiles) return;
  const int k = drop[tile / Hv];
  if (k == 0) return;
  const int n = buf_n[tile];
  if (k < 0 || k > n) {
    atomicOr(err, err_bad_phase);
    return;
  }
  buf_n[tile] = n - k;
}

}  // namespace

cudaError_t launch_rewind(int B, int Hv, const int32_t *drop, int32_t *buf_n, int32_t *err,
                          int err_bad_phase, cudaStream_t stream) {
  const int tiles = B * Hv;
  if (tiles == 0) return cudaSuccess;
  rewind_kernel<<<(tiles + 255) / 256, 256, 0, stream>>>(tiles, Hv, drop, buf_n, err,
                                                         err_bad_phase);
  return cudaGetLastError();
}

cudaError_t launch_checkpoint(bool save, int B, int Hv, int record_bytes, int num_slots,
                              const int32_t *slots, uint8_t *records, uint8_t *pool,
                              int32_t *buf_n, int32_t *err, int err_bad_phase,
                              cudaStream_t stream) {
  if (B == 0) return cudaSuccess;
  checkpoint_kernel<<<B * Hv, kCopyThreads, 0, stream>>>(save, Hv, record_bytes, num_slots,
                                                         slots, records, pool, buf_n, err,
                                                         err_bad_phase);
  return cudaGetLastError();
}

}  // namespace lq
