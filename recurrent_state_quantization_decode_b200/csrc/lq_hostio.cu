// Host-input gather for lq_decode_step_host.
//
// A decode step's inputs are small: at the bench shape q and k are 256 KiB
// each, v 512 KiB, and alpha and beta 8 KiB each.  Five cudaMemcpyAsync calls
// of that size reach well under the host link's bandwidth, because every copy
// pays its own start-up on the copy engine.  When the inputs sit in pinned
// host memory that the device maps (cudaHostAlloc memory under unified
// addressing), one kernel reads them instead.  Its CTAs issue all their
// 16-byte loads over the link at once and write the staging buffer that the
// decode kernel then reads.  Host memory that the device cannot address this
// way keeps the cudaMemcpyAsync path (lq_capi.cu).

#include "lq_hostio.h"

#include <algorithm>

namespace lq {
namespace {

constexpr int kGatherThreads = 256;
// grid cap of the grid-stride loop: 8 CTAs per SM of a 148-SM part, ample
// for one token's inputs in a single pass at the sizes above
constexpr unsigned long long kGatherMaxBlocks = 148ull * 8;

// The segments as the kernel walks them: unit u of the concatenation lies in
// segment s with first[s] <= u < first[s + 1]; the first nvec[s] units of a
// segment are 16-byte vectors, the rest single bytes.
struct GatherPlan {
  const uint8_t *src[kMaxGatherSegs];
  uint8_t *dst[kMaxGatherSegs];
  unsigned long long first[kMaxGatherSegs + 1];
  unsigned long long nvec[kMaxGatherSegs];
  int n;
};

__global__ void __launch_bounds__(kGatherThreads) gather_kernel(const GatherPlan pl) {
  const unsigned long long total = pl.first[pl.n];
  const unsigned long long stride = static_cast<unsigned long long>(gridDim.x) * kGatherThreads;
  for (unsigned long long u = static_cast<unsigned long long>(blockIdx.x) * kGatherThreads +
                              threadIdx.x;
       u < total; u += stride) {
    int s = 0;
    while (s + 1 < pl.n && u >= pl.first[s + 1]) ++s;
    const unsigned long long j = u - pl.first[s];
    if (j < pl.nvec[s]) {
      reinterpret_cast<uint4 *>(pl.dst[s])[j] = reinterpret_cast<const uint4 *>(pl.src[s])[j];
    } else {
      const unsigned long long b = 16 * pl.nvec[s] + (j - pl.nvec[s]);
      pl.dst[s][b] = pl.src[s][b];
    }
  }
}

// Whether the driver reports `p` as host memory that the current device reads
// at the same address.
bool mapped_at_same_address(const void *p) {
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    (void)cudaGetLastError();  // a failed query is not an error of the step
    return false;
  }
  return a.type == cudaMemoryTypeHost && a.devicePointer == p;
}

}  // namespace

const void *device_view_of_host(const void *p, size_t bytes) {
  if (p == nullptr || bytes == 0) return nullptr;
  // both ends of the range, so that a range that runs past its pinned
  // allocation is copied by the copy engine rather than read by the kernel
  const void *last = static_cast<const uint8_t *>(p) + (bytes - 1);
  if (!mapped_at_same_address(p) || !mapped_at_same_address(last)) return nullptr;
  return p;
}

cudaError_t launch_gather(const GatherList &list, cudaStream_t stream) {
  if (list.n < 0 || list.n > kMaxGatherSegs) return cudaErrorInvalidValue;
  GatherPlan pl{};
  unsigned long long total = 0;
  for (int i = 0; i < list.n; ++i) {
    const GatherSeg &g = list.seg[i];
    if (g.bytes == 0) continue;
    const bool vec =
        ((reinterpret_cast<uintptr_t>(g.src) | reinterpret_cast<uintptr_t>(g.dst)) & 15u) == 0;
    const unsigned long long nvec = vec ? g.bytes / 16 : 0;
    pl.src[pl.n] = static_cast<const uint8_t *>(g.src);
    pl.dst[pl.n] = static_cast<uint8_t *>(g.dst);
    pl.nvec[pl.n] = nvec;
    pl.first[pl.n] = total;
    total += nvec + (g.bytes - 16 * nvec);
    ++pl.n;
  }
  if (pl.n == 0) return cudaSuccess;
  pl.first[pl.n] = total;
  const unsigned long long blocks =
      std::min((total + kGatherThreads - 1) / kGatherThreads, kGatherMaxBlocks);
  gather_kernel<<<static_cast<unsigned>(blocks), kGatherThreads, 0, stream>>>(pl);
  return cudaGetLastError();
}

}  // namespace lq
