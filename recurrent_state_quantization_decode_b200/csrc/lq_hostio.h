// Internal interface of the host-input gather (lq_hostio.cu), used by the C
// ABI (lq_capi.cu).  Not installed; callers use include/leapquant.h.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

namespace lq {

constexpr int kMaxGatherSegs = 8;

// One host range [src, src + bytes) (read through its device-mapped address)
// to device memory at dst.
struct GatherSeg {
  const void *src;
  void *dst;
  size_t bytes;
};

struct GatherList {
  GatherSeg seg[kMaxGatherSegs];
  int n;
};

// The address through which a kernel on the current device may read the host
// range [p, p + bytes): pinned memory that the device maps (cudaHostAlloc
// memory under unified addressing, or a mapped registration).  Null when the
// device cannot read the whole range that way (pageable memory, device
// memory, or a failed query); the caller then copies with cudaMemcpyAsync.
const void *device_view_of_host(const void *p, size_t bytes);

// Copies every segment of `list` with one kernel.  Each thread moves one
// 16-byte unit of a segment whose two ends are 16-byte aligned, or one byte
// of a misaligned segment or of a segment's ragged tail, so that the reads
// over the host link are all in flight at once.
cudaError_t launch_gather(const GatherList &list, cudaStream_t stream);

}  // namespace lq
