// C ABI of libleapquant.so (declared in include/leapquant.h): argument
// validation on the host, then the call's launches: one kernel, except the
// host-buffer step (input gather or copies, the decode kernel, the output
// copy).  No call here allocates memory or keeps global state; the no-alloc
// variant's fixed staging array lives in lq_noalloc.cu.

#include <cstdint>
#include <cstring>

#include <cuda_runtime.h>

#include "../../include/leapquant.h"
#include "lq_capi_internal.h"
#include "lq_checkpoint.h"
#include "lq_hostio.h"
#include "lq_internal.h"

namespace {

using lq::KParams;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned_to(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t in_size(const lq_config *c) { return c->in_dtype == LQ_DTYPE_BF16 ? 2 : 4; }
size_t out_size(const lq_config *c) { return c->out_dtype == LQ_DTYPE_BF16 ? 2 : 4; }

// Shape and option checks shared by every entry point.
lq_status check_config(const lq_config *c) {
  if (c == nullptr) return LQ_ERR_INVALID_ARG;
  if (c->batch < 0 || c->num_k_heads < 1 || c->num_v_heads < 1) return LQ_ERR_INVALID_ARG;
  if (c->num_v_heads % c->num_k_heads != 0) return LQ_ERR_INVALID_ARG;
  if (c->gate != LQ_GATE_SCALAR && c->gate != LQ_GATE_DIAG) return LQ_ERR_INVALID_ARG;
  if (c->in_dtype != LQ_DTYPE_F32 && c->in_dtype != LQ_DTYPE_BF16) return LQ_ERR_INVALID_ARG;
  if (c->out_dtype != LQ_DTYPE_F32 && c->out_dtype != LQ_DTYPE_BF16) return LQ_ERR_INVALID_ARG;
  if (c->d != 32 && c->d != 64 && c->d != 128) return LQ_ERR_UNSUPPORTED;
  if (c->window < 1 || c->window > lq::kMaxWindowLong) return LQ_ERR_UNSUPPORTED;
  if (c->n_comp < 0 || c->n_comp > lq::kMaxComp) return LQ_ERR_UNSUPPORTED;
  if (!(c->smooth == 0.0f || c->smooth == 0.5f || c->smooth == 1.0f)) return LQ_ERR_UNSUPPORTED;
  // tiles are indexed with 32-bit ints; the decode kernel packs (sequence,
  // key head) of a tile into one int
  if (static_cast<int64_t>(c->batch) * c->num_v_heads > INT32_MAX) return LQ_ERR_UNSUPPORTED;
  if (c->batch >= (1 << 19) || c->num_k_heads > 2048) return LQ_ERR_UNSUPPORTED;
  return LQ_OK;
}

lq_status check_state(const lq_config *c, const lq_state *st) {
  if (st == nullptr) return LQ_ERR_INVALID_ARG;
  if (!st->records || !st->buf_k || !st->buf_d || !st->buf_g || !st->buf_n || !st->err)
    return LQ_ERR_INVALID_ARG;
  if (!aligned16(st->records) || !aligned16(st->buf_k) || !aligned16(st->buf_d) ||
      !aligned_to(st->buf_g, 4) || !aligned_to(st->buf_n, 4) || !aligned_to(st->err, 4))
    return LQ_ERR_MISALIGNED;
  (void)c;
  return LQ_OK;
}

// q, k, v (and the KDA gate) are moved with 16-byte bulk copies.
lq_status check_io(const lq_config *c, const void *q, const void *k, const void *v,
                   const float *alpha, const float *beta, const void *out) {
  if (!q || !k || !v || !alpha || !beta || !out) return LQ_ERR_INVALID_ARG;
  const size_t os = out_size(c);
  const size_t as = c->gate == LQ_GATE_DIAG ? 16 : 4;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned_to(alpha, as) ||
      !aligned_to(beta, 4) || !aligned_to(out, os))
    return LQ_ERR_MISALIGNED;
  return LQ_OK;
}

KParams make_params(const lq_config *c, const lq_state *st) {
  KParams p;
  std::memset(&p, 0, sizeof(p));
  p.B = c->batch;
  p.Hk = c->num_k_heads;
  p.Hv = c->num_v_heads;
  p.d = c->d;
  p.W = c->window;
  p.K = c->n_comp;
  p.gate = c->gate;
  p.in_bf16 = c->in_dtype == LQ_DTYPE_BF16;
  p.out_bf16 = c->out_dtype == LQ_DTYPE_BF16;
  p.smooth = c->smooth == 0.0f ? 0 : (c->smooth == 0.5f ? 1 : 2);
  p.L = lq::record_layout(c->d, c->n_comp);
  p.wait_limit = lq::kWaitLimitDefault;
  p.gstride = lq::gdn_gate_stride(c->window);
  p.ntok = 1;
  if (st != nullptr) {
    p.records = static_cast<uint8_t *>(st->records);
    p.buf_k = st->buf_k;
    p.buf_d = st->buf_d;
    p.buf_g = st->buf_g;
    p.buf_n = st->buf_n;
    p.err = st->err;
  }
  return p;
}

lq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? LQ_OK : LQ_ERR_CUDA; }

lq::StagingLayout staging_of(const lq_config *c) {
  return lq::staging_layout(c->batch, c->num_k_heads, c->num_v_heads, c->d, in_size(c),
                            out_size(c), c->gate == LQ_GATE_DIAG);
}

}  // namespace

namespace lq {

// Every argument check of the host-buffer step except its staging pointer, so
// that the no-alloc variant rejects a bad call before it touches its array.
lq_status check_host_step(const lq_config *cfg, const void *q_host, const void *k_host,
                          const void *v_host, const float *alpha_host, const float *beta_host,
                          const lq_state *st, const void *out_host, const int32_t *active) {
  lq_status s = check_config(cfg);
  if (s != LQ_OK) return s;
  if ((s = check_state(cfg, st)) != LQ_OK) return s;
  if ((s = check_io(cfg, q_host, k_host, v_host, alpha_host, beta_host, out_host)) != LQ_OK)
    return s;
  if (!aligned_to(active, 4)) return LQ_ERR_MISALIGNED;
  return LQ_OK;
}

size_t host_staging_bytes(const lq_config *cfg) { return staging_of(cfg).total; }

}  // namespace lq

extern "C" {

int32_t lq_version(void) { return 1; }

const char *lq_status_string(lq_status s) {
  switch (s) {
    case LQ_OK: return "LQ_OK";
    case LQ_ERR_INVALID_ARG: return "LQ_ERR_INVALID_ARG: null pointer or bad shape";
    case LQ_ERR_UNSUPPORTED: return "LQ_ERR_UNSUPPORTED: d, window, n_comp or smooth out of range";
    case LQ_ERR_MISALIGNED: return "LQ_ERR_MISALIGNED: pointer not aligned as required";
    case LQ_ERR_CUDA: return "LQ_ERR_CUDA: CUDA launch or stream error";
    case LQ_ERR_DEVICE_BOUNDS: return "LQ_ERR_DEVICE_BOUNDS: a kernel found a corrupt window phase";
    case LQ_ERR_TOO_LARGE:
      return "LQ_ERR_TOO_LARGE: staging exceeds the no-alloc entry point's fixed array";
    case LQ_ERR_TIMEOUT: return "LQ_ERR_TIMEOUT: a kernel's bounded wait on a copy expired";
  }
  return "unknown lq_status";
}

lq_status lq_state_layout(const lq_config *cfg, lq_layout *out) {
  lq_status s = check_config(cfg);
  if (s != LQ_OK) return s;
  if (out == nullptr) return LQ_ERR_INVALID_ARG;
  const lq::RecLayout L = lq::record_layout(cfg->d, cfg->n_comp);
  const size_t B = cfg->batch, Hk = cfg->num_k_heads, Hv = cfg->num_v_heads;
  const size_t d = cfg->d, W = cfg->window, tiles = B * Hv;
  out->record_bytes = L.bytes;
  out->off_sigma = L.off_sig;
  out->off_m = L.off_m;
  out->off_comp_vec = L.off_cv;
  out->off_comp_id = L.off_cid;
  out->records_bytes = tiles * L.bytes;
  out->buf_k_bytes = B * Hk * W * d * in_size(cfg);
  out->buf_d_bytes = tiles * W * d * 4;
  out->buf_g_bytes = cfg->gate == LQ_GATE_DIAG ? tiles * W * d * 4
                                                : tiles * lq::gdn_gate_stride(cfg->window) * 4;
  out->buf_n_bytes = tiles * 4;
  out->err_bytes = 4;
  out->fp32_state_bytes = tiles * d * d * 4;
  out->host_staging_bytes = staging_of(cfg).total;
  return LQ_OK;
}

size_t lq_state_bytes(const lq_config *cfg, size_t *tile_bytes, size_t *buffer_bytes) {
  lq_layout L;
  if (lq_state_layout(cfg, &L) != LQ_OK) return 0;
  if (tile_bytes) *tile_bytes = L.record_bytes;
  const size_t buffers = L.buf_k_bytes + L.buf_d_bytes + L.buf_g_bytes + L.buf_n_bytes;
  if (buffer_bytes) *buffer_bytes = buffers;
  return L.records_bytes + buffers + L.err_bytes;
}

lq_status lq_state_init(const lq_config *cfg, const float *S0, const lq_state *st,
                        const int32_t *mask, void *stream) {
  lq_status s = check_config(cfg);
  if (s != LQ_OK) return s;
  if ((s = check_state(cfg, st)) != LQ_OK) return s;
  if (S0 == nullptr) return LQ_ERR_INVALID_ARG;
  if (!aligned16(S0) || !aligned_to(mask, 4)) return LQ_ERR_MISALIGNED;
  if (cfg->batch == 0) return LQ_OK;
  KParams p = make_params(cfg, st);
  p.S_in = S0;
  p.mask = mask;
  return from_cuda(lq::launch_init(p, static_cast<cudaStream_t>(stream)));
}

lq_status lq_decode_step(const lq_config *cfg, const void *q, const void *k, const void *v,
                         const float *alpha, const float *beta, const lq_state *st, void *out,
                         const int32_t *active, void *stream) {
  lq_status s = check_config(cfg);
  if (s != LQ_OK) return s;
  if ((s = check_state(cfg, st)) != LQ_OK) return s;
  if ((s = check_io(cfg, q, k, v, alpha, beta, out)) != LQ_OK) return s;
  if (!aligned_to(active, 4)) return LQ_ERR_MISALIGNED;
  if (cfg->batch == 0) return LQ_OK;
  KParams p = make_params(cfg, st);
  p.q = q;
  p.k = k;
  p.v = v;
  p.alpha = alpha;
  p.beta = beta;
  p.out = out;
  p.mask = active;
  return from_cuda(lq::launch_decode(p, static_cast<cudaStream_t>(stream)));
}

lq_status lq_decode_step_packed(const lq_config *cfg, const void *qkva, const float *alpha,
                                const float *beta, const lq_state *st, void *out,
                                const int32_t *active, void *stream) {
  lq_status s = check_config(cfg);
  if (s != LQ_OK) return s;
  if ((s = check_state(cfg, st)) != LQ_OK) return s;
  if (cfg->window > lq::kMaxWindow) return LQ_ERR_UNSUPPORTED;
  const bool kda = cfg->gate == LQ_GATE_DIAG;
  if (!qkva || !beta || !out || (!kda && !alpha)) return LQ_ERR_INVALID_ARG;
  if (!aligned16(qkva) || (!kda && !aligned_to(alpha, 4)) || !aligned_to(beta, 4) ||
      !aligned_to(out, out_size(cfg)) || !aligned_to(active, 4))
    return LQ_ERR_MISALIGNED;
  if (cfg->batch == 0) return LQ_OK;
  KParams p = make_params(cfg, st);
  p.q = qkva;
  p.alpha = kda ? nullptr : alpha;
  p.beta = beta;
  p.out = out;
  p.mask = active;
  p.packed = 1;
  return from_cuda(lq::launch_decode(p, static_cast<cudaStream_t>(stream)));
}

lq_status lq_decode_tokens(const lq_config *cfg, int32_t ntok, const void *q, const void *k,
                           const void *v, const float *alpha, const float *beta,
                           const lq_state *st, void *out, const int32_t *active, void *stream) {
  lq_status s = check_config(cfg);
  if (s != LQ_OK) return s;
  if ((s = check_state(cfg, st)) != LQ_OK) return s;
  if (ntok < 0) return LQ_ERR_INVALID_ARG;
  if (ntok == 0 || cfg->batch == 0) return LQ_OK;
  if ((s = check_io(cfg, q, k, v, alpha, beta, out)) != LQ_OK) return s;
  if (!aligned_to(active, 4)) return LQ_ERR_MISALIGNED;
  KParams p = make_params(cfg, st);
  p.q = q;
  p.k = k;
  p.v = v;
  p.alpha = alpha;
  p.beta = beta;
  p.out = out;
  p.mask = active;
  p.ntok = ntok;
  return from_cuda(lq::launch_decode_tokens(p, static_cast<cudaStream_t>(stream)));
}

lq_status lq_prefill(const lq_config *cfg, const void *q, const void *k, const void *v,
                     const float *alpha, const float *beta, int32_t T, const float *S0,
                     const lq_state *st, void *out, const int32_t *mask, void *stream) {
  lq_status s = check_config(cfg);
  if (s != LQ_OK) return s;
  if ((s = check_state(cfg, st)) != LQ_OK) return s;
  if (T < 0) return LQ_ERR_INVALID_ARG;
  if (T > 0 && (q == nullptr || k == nullptr || v == nullptr || alpha == nullptr ||
                beta == nullptr))
    return LQ_ERR_INVALID_ARG;
  if (!aligned16(S0) || !aligned_to(alpha, 4) || !aligned_to(beta, 4) ||
      !aligned_to(mask, 4) || !aligned_to(q, in_size(cfg)) || !aligned_to(k, in_size(cfg)) ||
      !aligned_to(v, in_size(cfg)) || !aligned_to(out, out_size(cfg)))
    return LQ_ERR_MISALIGNED;
  if (cfg->batch == 0) return LQ_OK;
  KParams p = make_params(cfg, st);
  p.q = q;
  p.k = k;
  p.v = v;
  p.alpha = alpha;
  p.beta = beta;
  p.T = T;
  p.S_in = S0;
  p.out = out;
  p.mask = mask;
  return from_cuda(lq::launch_prefill(p, static_cast<cudaStream_t>(stream)));
}

namespace {
lq_status checkpoint(bool save, const lq_config *cfg, const lq_state *st, const int32_t *slots,
                     const void *pool, int32_t num_slots, void *stream) {
  lq_status s = check_config(cfg);
  if (s != LQ_OK) return s;
  if ((s = check_state(cfg, st)) != LQ_OK) return s;
  if (slots == nullptr || pool == nullptr || num_slots < 0) return LQ_ERR_INVALID_ARG;
  if (!aligned16(pool) || !aligned_to(slots, 4)) return LQ_ERR_MISALIGNED;
  if (cfg->batch == 0) return LQ_OK;
  const lq::RecLayout L = lq::record_layout(cfg->d, cfg->n_comp);
  return from_cuda(lq::launch_checkpoint(
      save, cfg->batch, cfg->num_v_heads, L.bytes, num_slots, slots,
      static_cast<uint8_t *>(st->records), static_cast<uint8_t *>(const_cast<void *>(pool)),
      st->buf_n, st->err, lq::kErrBadPhase, static_cast<cudaStream_t>(stream)));
}
}  // namespace

lq_status lq_checkpoint_save(const lq_config *cfg, const lq_state *st, const int32_t *slots,
                             void *pool, int32_t num_slots, void *stream) {
  return checkpoint(true, cfg, st, slots, pool, num_slots, stream);
}

lq_status lq_checkpoint_restore(const lq_config *cfg, const void *pool, int32_t num_slots,
                                const int32_t *slots, const lq_state *st, void *stream) {
  return checkpoint(false, cfg, st, slots, pool, num_slots, stream);
}

lq_status lq_window_rewind(const lq_config *cfg, const lq_state *st, const int32_t *drop,
                           void *stream) {
  lq_status s = check_config(cfg);
  if (s != LQ_OK) return s;
  if ((s = check_state(cfg, st)) != LQ_OK) return s;
  if (drop == nullptr) return LQ_ERR_INVALID_ARG;
  if (!aligned_to(drop, 4)) return LQ_ERR_MISALIGNED;
  return from_cuda(lq::launch_rewind(cfg->batch, cfg->num_v_heads, drop, st->buf_n, st->err,
                                     lq::kErrBadPhase, static_cast<cudaStream_t>(stream)));
}

lq_status lq_test_decode_step_timeout(const lq_config *cfg, const void *q, const void *k,
                                      const void *v, const float *alpha, const float *beta,
                                      const lq_state *st, void *out, uint32_t wait_limit,
                                      void *stream) {
  lq_status s = check_config(cfg);
  if (s != LQ_OK) return s;
  if ((s = check_state(cfg, st)) != LQ_OK) return s;
  if ((s = check_io(cfg, q, k, v, alpha, beta, out)) != LQ_OK) return s;
  if (cfg->batch == 0 || wait_limit == 0) return LQ_ERR_INVALID_ARG;
  KParams p = make_params(cfg, st);
  p.q = q;
  p.k = k;
  p.v = v;
  p.alpha = alpha;
  p.beta = beta;
  p.out = out;
  p.wait_limit = wait_limit;
  p.withhold = 1;
  return from_cuda(lq::launch_decode(p, static_cast<cudaStream_t>(stream)));
}

lq_status lq_decode_step_host(const lq_config *cfg, const void *q_host, const void *k_host,
                              const void *v_host, const float *alpha_host,
                              const float *beta_host, const lq_state *st, void *out_host,
                              void *staging, const int32_t *active, void *stream) {
  lq_status s =
      lq::check_host_step(cfg, q_host, k_host, v_host, alpha_host, beta_host, st, out_host, active);
  if (s != LQ_OK) return s;
  if (staging == nullptr) return LQ_ERR_INVALID_ARG;
  if (!aligned16(staging)) return LQ_ERR_MISALIGNED;
  if (cfg->batch == 0) return LQ_OK;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const lq::StagingLayout sl = staging_of(cfg);
  uint8_t *base = static_cast<uint8_t *>(staging);
  uint8_t *dout = base + sl.out;
  // Inputs in device-mapped pinned memory are read by one gather kernel over
  // the host link; any other host memory goes through the copy engine.  With
  // an active mask the kernel writes only active sequences' rows, and the
  // whole output region is copied back: the host's current output rows go
  // into the staging first, so that inactive sequences read back unchanged.
  const void *src[6] = {q_host, k_host, v_host, alpha_host, beta_host, out_host};
  void *dst[6] = {base + sl.q, base + sl.k, base + sl.v, base + sl.alpha, base + sl.beta, dout};
  const size_t bytes[6] = {sl.q_bytes, sl.q_bytes, sl.v_bytes, sl.alpha_bytes, sl.beta_bytes,
                           sl.out_bytes};
  const int nsrc = active != nullptr ? 6 : 5;
  // Inputs back to back in host memory, in the staging's order and with its
  // spacing (every input a multiple of 256 bytes, so that the staging has no
  // gaps): one copy-engine copy moves them all and occupies no SM, so that it
  // overlaps kernels of other streams.
  bool packed = true;
  for (int i = 1; i < 5; ++i)
    packed = packed && dst[i] == static_cast<uint8_t *>(dst[i - 1]) + bytes[i - 1] &&
             src[i] == static_cast<const uint8_t *>(src[i - 1]) + bytes[i - 1];
  int first = 0;
  if (packed) {
    const size_t span = static_cast<size_t>(static_cast<uint8_t *>(dst[4]) + bytes[4] -
                                            static_cast<uint8_t *>(dst[0]));
    if (cudaMemcpyAsync(dst[0], src[0], span, cudaMemcpyHostToDevice, cs) != cudaSuccess)
      return LQ_ERR_CUDA;
    first = 5;
  }
  lq::GatherList gather{};
  for (int i = first; i < nsrc; ++i) {
    if (const void *view = lq::device_view_of_host(src[i], bytes[i])) {
      gather.seg[gather.n++] = lq::GatherSeg{view, dst[i], bytes[i]};
    } else if (cudaMemcpyAsync(dst[i], src[i], bytes[i], cudaMemcpyHostToDevice, cs) !=
               cudaSuccess) {
      return LQ_ERR_CUDA;
    }
  }
  if (lq::launch_gather(gather, cs) != cudaSuccess) return LQ_ERR_CUDA;
  KParams p = make_params(cfg, st);
  p.q = base + sl.q;
  p.k = base + sl.k;
  p.v = base + sl.v;
  p.alpha = reinterpret_cast<const float *>(base + sl.alpha);
  p.beta = reinterpret_cast<const float *>(base + sl.beta);
  p.out = dout;
  p.mask = active;
  if (lq::launch_decode(p, cs) != cudaSuccess) return LQ_ERR_CUDA;
  if (cudaMemcpyAsync(out_host, dout, sl.out_bytes, cudaMemcpyDeviceToHost, cs) != cudaSuccess)
    return LQ_ERR_CUDA;
  return LQ_OK;
}

lq_status lq_window_flush(const lq_config *cfg, const lq_state *st, const int32_t *mask,
                          void *stream) {
  lq_status s = check_config(cfg);
  if (s != LQ_OK) return s;
  if ((s = check_state(cfg, st)) != LQ_OK) return s;
  if (!aligned_to(mask, 4)) return LQ_ERR_MISALIGNED;
  if (cfg->batch == 0) return LQ_OK;
  KParams p = make_params(cfg, st);
  p.mask = mask;
  return from_cuda(lq::launch_flush(p, static_cast<cudaStream_t>(stream)));
}

lq_status lq_fp32_decode_step(const lq_config *cfg, const void *q, const void *k,
                              const void *v, const float *alpha, const float *beta, float *S,
                              void *out, void *stream) {
  lq_status s = check_config(cfg);
  if (s != LQ_OK) return s;
  if ((s = check_io(cfg, q, k, v, alpha, beta, out)) != LQ_OK) return s;
  if (S == nullptr) return LQ_ERR_INVALID_ARG;
  if (!aligned16(S)) return LQ_ERR_MISALIGNED;
  if (cfg->batch == 0) return LQ_OK;
  KParams p = make_params(cfg, nullptr);
  p.q = q;
  p.k = k;
  p.v = v;
  p.alpha = alpha;
  p.beta = beta;
  p.out = out;
  return from_cuda(lq::launch_fp32_step(p, S, static_cast<cudaStream_t>(stream)));
}

lq_status lq_state_dequantize(const lq_config *cfg, const lq_state *st, int32_t include_buffer,
                              float *S_out, void *stream) {
  lq_status s = check_config(cfg);
  if (s != LQ_OK) return s;
  if ((s = check_state(cfg, st)) != LQ_OK) return s;
  if (S_out == nullptr) return LQ_ERR_INVALID_ARG;
  if (!aligned16(S_out)) return LQ_ERR_MISALIGNED;
  if (cfg->batch == 0) return LQ_OK;
  KParams p = make_params(cfg, st);
  p.S_out = S_out;
  p.include_buffer = include_buffer != 0;
  return from_cuda(lq::launch_dequantize(p, static_cast<cudaStream_t>(stream)));
}

lq_status lq_get_last_error(const lq_state *st, void *stream) {
  if (st == nullptr || st->err == nullptr) return LQ_ERR_INVALID_ARG;
  if (!aligned_to(st->err, 4)) return LQ_ERR_MISALIGNED;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int32_t word = 0;
  if (cudaMemcpyAsync(&word, st->err, sizeof(word), cudaMemcpyDeviceToHost, cs) != cudaSuccess)
    return LQ_ERR_CUDA;
  if (cudaStreamSynchronize(cs) != cudaSuccess) return LQ_ERR_CUDA;
  if (word != 0) {
    if (cudaMemsetAsync(st->err, 0, sizeof(int32_t), cs) != cudaSuccess) return LQ_ERR_CUDA;
    if (cudaStreamSynchronize(cs) != cudaSuccess) return LQ_ERR_CUDA;
    return (word & lq::kErrTimeout) ? LQ_ERR_TIMEOUT : LQ_ERR_DEVICE_BOUNDS;
  }
  return LQ_OK;
}

}  // extern "C"
