// Internal interface between the C ABI (lq_capi.cu, lq_noalloc.cu) and the
// kernels (lq_decode.cu, lq_fp32.cu).  Not installed; callers use
// include/leapquant.h.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

namespace lq {

constexpr int kMaxWindow = 16;      // W limit of the persistent decode kernel
constexpr int kMaxWindowLong = 32;  // W limit of the per-tile kernel (longer windows)
constexpr int kMaxComp = 8;     // K limit
constexpr int kGdnGateStride = 16;  // GDN gate buffer: 16 floats per tile (one 64-byte copy)

// Floats per tile of the GDN gate buffer for a window of W tokens: 16 up to
// W = 16, 32 beyond.
inline int gdn_gate_stride(int W) { return W > kGdnGateStride ? 2 * kGdnGateStride : kGdnGateStride; }
constexpr int kErrBadPhase = 1;     // device error bit: buf_n outside [0, W)
constexpr int kErrTimeout = 2;      // device error bit: a bounded wait on a copy expired

// Byte layout of one tile record (see include/leapquant.h).
struct RecLayout {
  int bytes;    // whole record, multiple of 16
  int off_sig;  // fp32 [d]
  int off_m;    // fp32 [d]
  int off_cv;   // fp32 [K][d]
  int off_cid;  // int32 [K]
};

RecLayout record_layout(int d, int K);

// Everything a kernel launch needs; unused fields are null / zero.
struct KParams {
  int B, Hk, Hv, d, W, K, gate, in_bf16, out_bf16;
  int smooth;  // 0: m = 1, 1: m = sqrt(colmax), 2: m = colmax
  RecLayout L;
  uint8_t *records;
  void *buf_k;
  float *buf_d;
  float *buf_g;
  int32_t *buf_n;
  int32_t *err;
  const void *q, *k, *v;
  const float *alpha, *beta;
  void *out;
  const int32_t *mask;  // decode: active sequences; init / flush: selected sequences
  const float *S_in;    // init: fp32 states to quantize
  float *S_out;         // dequantize: fp32 states written
  int include_buffer;   // dequantize: advance the base state by the buffered tokens
  int T;                // prefill: prompt tokens
  uint32_t wait_limit;  // decode: polls of a bounded mbarrier wait before it expires
  int withhold;         // decode, testing only: CTA 0 issues no copies for its first slot
  int gstride;          // floats per tile of the GDN gate buffer (gdn_gate_stride(W))
  int ntok;             // tokens per launch of the per-tile kernel (lq_decode_tokens)
  int packed;           // decode: q holds each tile's q | k | v (| KDA gate) back to back
};

constexpr uint32_t kWaitLimitDefault = 1u << 24;

// Device staging of the host-buffer decode step: q, k, v, alpha, beta and the
// output, each at a 256-byte aligned offset.  The one definition of this
// layout, used by lq_state_layout (its size), lq_decode_step_host and the
// no-alloc variant.
struct StagingLayout {
  size_t q, k, v, alpha, beta, out;  // byte offsets
  size_t q_bytes, v_bytes, alpha_bytes, beta_bytes, out_bytes;
  size_t total;
};

inline size_t round256(size_t x) { return (x + 255) / 256 * 256; }

inline StagingLayout staging_layout(size_t B, size_t Hk, size_t Hv, size_t d, size_t in_bytes,
                                    size_t out_bytes, bool gate_diag) {
  StagingLayout s;
  const size_t tiles = B * Hv;
  s.q_bytes = B * Hk * d * in_bytes;
  s.v_bytes = tiles * d * in_bytes;
  s.alpha_bytes = tiles * (gate_diag ? d : 1) * 4;
  s.beta_bytes = tiles * 4;
  s.out_bytes = tiles * d * out_bytes;
  s.q = 0;
  s.k = s.q + round256(s.q_bytes);
  s.v = s.k + round256(s.q_bytes);
  s.alpha = s.v + round256(s.v_bytes);
  s.beta = s.alpha + round256(s.alpha_bytes);
  s.out = s.beta + round256(s.beta_bytes);
  s.total = s.out + round256(s.out_bytes);
  return s;
}

cudaError_t launch_decode(const KParams &p, cudaStream_t stream);
cudaError_t launch_decode_tokens(const KParams &p, cudaStream_t stream);
cudaError_t launch_init(const KParams &p, cudaStream_t stream);
cudaError_t launch_prefill(const KParams &p, cudaStream_t stream);
cudaError_t launch_flush(const KParams &p, cudaStream_t stream);
cudaError_t launch_dequantize(const KParams &p, cudaStream_t stream);
cudaError_t launch_fp32_step(const KParams &p, float *S, cudaStream_t stream);

}  // namespace lq
