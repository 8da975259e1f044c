// lq_decode_step_host_noalloc: the host-buffer decode step for callers that
// cannot allocate device memory.
//
// lq_decode_step_host needs a device staging buffer from the caller.  Some
// callers cannot call cudaMalloc: a plugin running inside a host application
// that owns every device allocation, or a latency-critical loop where an
// allocation (which may synchronize the whole device) is not acceptable.  This
// variant stages the token's inputs and output in a fixed array that lives in
// the library's own device memory instead.
//
// The array below is a file-scope __device__ variable of
// kNoallocStagingBytes (8 MiB): every GPU that loads the library holds it
// until the process exits.  All calls share it, and it keeps the previous
// call's contents.  The step writes every output row it copies back (active
// rows from the kernel; with an active mask, inactive rows are first filled
// from the caller's own output buffer), so no stale bytes reach the caller.
// Calls that overlap on the GPU (on different streams, or from different
// threads) race on the array, so the caller must order them.
//
// Host code cannot use the array's name as a device address: in host code it
// names a host-side stand-in.  The first call on each device therefore looks
// the real address up with cudaGetSymbolAddress, with that device current, and
// caches it; that first call should come before any stream capture.  The
// cached address belongs to the device's primary context: after
// cudaDeviceReset the library must be reloaded before this entry point is
// called again on that device.  Device code in this file could name the array
// directly; only host code needs the looked-up address.

#include <atomic>
#include <cstdint>

#include <cuda_runtime.h>

#include "../../include/leapquant.h"
#include "lq_capi_internal.h"

namespace {

constexpr size_t kNoallocStagingBytes = LQ_NOALLOC_STAGING_MAX_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_staging[kNoallocStagingBytes];

std::atomic<void *> g_staging_addr[kMaxDevices];

// Device address of the staging array on the current device (looked up once
// per device).  Returns null if the lookup fails; a failed lookup leaves no
// sticky error behind for the next runtime call.
void *staging_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  void *p = g_staging_addr[dev].load(std::memory_order_acquire);
  if (p != nullptr) return p;
  void *addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_noalloc_staging) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  g_staging_addr[dev].store(addr, std::memory_order_release);
  return addr;
}

}  // namespace

extern "C" lq_status lq_decode_step_host_noalloc(const lq_config *cfg, const void *q_host,
                                                 const void *k_host, const void *v_host,
                                                 const float *alpha_host,
                                                 const float *beta_host, const lq_state *st,
                                                 void *out_host, const int32_t *active,
                                                 void *stream) {
  // every argument is checked before the array is looked up or touched
  lq_status s = lq::check_host_step(cfg, q_host, k_host, v_host, alpha_host, beta_host, st,
                                    out_host, active);
  if (s != LQ_OK) return s;
  if (lq::host_staging_bytes(cfg) > kNoallocStagingBytes) return LQ_ERR_TOO_LARGE;
  if (cfg->batch == 0) return LQ_OK;
  void *staging = staging_address();
  if (staging == nullptr) return LQ_ERR_CUDA;
  return lq_decode_step_host(cfg, q_host, k_host, v_host, alpha_host, beta_host, st, out_host,
                             staging, active, stream);
}
