/*
 * leapquant.h - C ABI of libleapquant.so: the per-token decode step of a
 * Gated DeltaNet (GDN) / Kimi Delta Attention (KDA) layer whose recurrent
 * state is stored in int8, following LeapQuant, with the calls around it:
 * state init, a prefill that ends in the quantizer, the decode step on host
 * buffers, partial-window flush, prefix-cache checkpoints, speculative
 * rollback inside a window, dequantization and the fp32-state comparison
 * step.
 *
 * Method sources (page title, section):
 *  - "LeapQuant: Training-Free 8-bit Quantization for Linear Attention
 *    Recurrent States" (zhichai.net forum summary), "Abstract (translated)",
 *    items 1-3: per-window quantization (outputs from a fixed low-bit state
 *    plus a high-precision buffer, quantize once at the window's end);
 *    Compensator Tokens (largest outliers kept in high precision, sharing the
 *    update path of real tokens); residual smoothing before quantization.
 *  - "LeapQuant: Efficient Linear Attention with Accurate Recurrent State
 *    Quantization" (opentrain.ai), "Abstract": the outliers are rows and
 *    columns of the state; the FP32-state baseline.
 *  - globaltechnewsdesk news article on LeapQuant, paragraphs 3-5: a window
 *    of 16 tokens, reconstruct and quantize at the boundary, four
 *    Compensator Tokens, 1.19 bytes per stored value, 4 bytes for FP32.
 *
 * Notation.  A tile is one (sequence b, value head h) state S, d x d, row i =
 * value channel, column j = key channel, o = S q.  The exact recurrence is
 *   S_t = S_{t-1} diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 * with alpha_t a scalar (GDN) or a d-vector over key channels (KDA).
 * Value head h reads key/query head h / (Hv / Hk).
 *
 * Stored state (caller-owned device memory, sizes from lq_state_layout):
 *  records  [B*Hv] tile records, record_bytes each (a multiple of 16):
 *           codes int8 [d][d] row-major | sigma fp32 [d] (per-row scale) |
 *           m fp32 [d] (per-key-column smoothing factor) | compensator
 *           vectors fp32 [K][d] | compensator ids int32 [K] (i = row i,
 *           d + j = column j) | zero padding.  The window-base state is
 *           S0_ij = sigma_i * code_ij * m_j plus the compensator lines.
 *           At d = 128, K = 4 a record is 19,472 bytes = 1.19 bytes/value.
 *  buf_k    [B][Hk][W][d] keys of the buffered tokens, in the input dtype
 *           (lossless: they are the inputs themselves).
 *  buf_d    [B][Hv][W][d] fp32 deltas d_i of the buffered tokens.
 *  buf_g    [B][Hv][16] (GDN with W <= 16; [B][Hv][32] for W > 16; the
 *           first W used) or [B][Hv][W][d] (KDA) fp32 gates alpha_i.
 *  buf_n    [B][Hv] int32 tokens buffered in the current window (0..W-1
 *           between calls).
 *  err      one int32 device error word (bit 0: a corrupt buf_n was seen,
 *           or a checkpoint copy or a rollback was refused; bit 1: a
 *           bounded wait on a copy expired).
 * The layout is public: a checkpoint of a tile at a window boundary is a copy
 * of its record.
 *
 * Conventions for every call:
 *  - All pointers in lq_state and all tensor arguments are device pointers
 *    unless the name says host; the library allocates nothing and keeps no
 *    global state, except the fixed staging array of
 *    lq_decode_step_host_noalloc.  `stream` is a cudaStream_t (NULL = legacy
 *    default).
 *  - Argument errors are detected on the host before anything is launched,
 *    and reported synchronously: LQ_ERR_INVALID_ARG (null pointer, bad
 *    shape), LQ_ERR_UNSUPPORTED (d not in {32, 64, 128}, W not in 1..32,
 *    K not in 0..8, smooth not in {0, 0.5, 1}), LQ_ERR_MISALIGNED (records,
 *    buffers or the fp32 state not 16-byte aligned).  A failed launch returns
 *    LQ_ERR_CUDA.  Work is asynchronous on `stream`.
 *  - Device-side problems never trap: a kernel sets a bit in *err and skips
 *    the tile (or, when a wait on its own copy expires, stops after letting
 *    its copies land); lq_get_last_error reports it.
 *  - batch == 0 is a valid empty call: nothing is launched.
 *  - q is used as given (any 1/sqrt(d) scaling is the caller's).  NaN or Inf
 *    inputs are outside the contract.
 */
#ifndef LEAPQUANT_H
#define LEAPQUANT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LQ_OK = 0,
  LQ_ERR_INVALID_ARG = 1,
  LQ_ERR_UNSUPPORTED = 2,
  LQ_ERR_MISALIGNED = 3,
  LQ_ERR_CUDA = 4,
  LQ_ERR_DEVICE_BOUNDS = 5,
  LQ_ERR_TOO_LARGE = 6, /* lq_decode_step_host_noalloc: staging above its fixed array */
  LQ_ERR_TIMEOUT = 7    /* a kernel's bounded wait on one of its copies expired */
} lq_status;

typedef enum { LQ_GATE_SCALAR = 0, LQ_GATE_DIAG = 1 } lq_gate;
typedef enum { LQ_DTYPE_F32 = 0, LQ_DTYPE_BF16 = 1 } lq_dtype;

typedef struct {
  int32_t batch;       /* B sequences (0 <= B < 2^19) */
  int32_t num_k_heads; /* Hk key/query heads, 1..2048 */
  int32_t num_v_heads; /* Hv >= 1 value heads, a multiple of Hk */
  int32_t d;           /* d_k = d_v = d, one of 32, 64, 128 */
  int32_t window;      /* W tokens per quantization window, 1..32 (16 on the pages) */
  int32_t n_comp;      /* K compensator lines per tile, 0..8 (4 on the pages) */
  int32_t gate;        /* lq_gate: LQ_GATE_SCALAR (GDN) or LQ_GATE_DIAG (KDA) */
  int32_t in_dtype;    /* lq_dtype of q, k, v */
  int32_t out_dtype;   /* lq_dtype of o */
  float smooth;        /* smoothing exponent of the column max: 0, 0.5 or 1 */
} lq_config;

typedef struct {
  size_t record_bytes;     /* one tile record, multiple of 16 */
  size_t off_sigma;        /* byte offsets inside a record (codes start at 0) */
  size_t off_m;
  size_t off_comp_vec;
  size_t off_comp_id;
  size_t records_bytes;    /* B*Hv records */
  size_t buf_k_bytes;
  size_t buf_d_bytes;
  size_t buf_g_bytes;
  size_t buf_n_bytes;
  size_t err_bytes;
  size_t fp32_state_bytes; /* B*Hv*d*d*4: the unquantized comparison state */
  size_t host_staging_bytes; /* device staging that lq_decode_step_host needs */
} lq_layout;

typedef struct {
  void *records;
  void *buf_k;
  float *buf_d;
  float *buf_g;
  int32_t *buf_n;
  int32_t *err;
} lq_state;

/* Interface version (1). */
int32_t lq_version(void);

/* Human-readable name of a status code (static string). */
const char *lq_status_string(lq_status s);

/* Sizes and record offsets for cfg.  Host only; launches nothing. */
lq_status lq_state_layout(const lq_config *cfg, lq_layout *out);

/* Bytes of all stored state for cfg (records + buffers + counters + error
 * word); *tile_bytes (nullable) receives one record's size and
 * *buffer_bytes (nullable) the in-window buffers' total.  0 on a bad cfg. */
size_t lq_state_bytes(const lq_config *cfg, size_t *tile_bytes, size_t *buffer_bytes);

/* Quantize given fp32 states into records and empty the buffers: the same
 * quantizer the window boundary runs (zhichai.net summary, items 1-3), applied
 * to a state produced elsewhere, e.g. by prefill.  S0: [B][Hv][d][d] fp32,
 * 16-byte aligned.  mask: nullable [B] int32; sequences with mask[b] == 0 are
 * left untouched.  Clears nothing else; the caller zeroes *err once. */
lq_status lq_state_init(const lq_config *cfg, const float *S0, const lq_state *st,
                        const int32_t *mask, void *stream);

/* Prefill ending in the quantizer.  The pages describe the context being
 * compressed into the fixed-size state that decode then reads and updates
 * (AI Learning Platform article "LeapQuant: Efficient Linear Attention with
 * Accurate Recurrent State Quantization", "Key Takeaway for Students"); this
 * produces that state for a prompt.  Per tile, from S0 ([B][Hv][d][d] fp32,
 * 16-byte aligned; NULL = zero states), it runs the exact recurrence in fp32
 * for t = 0 .. T-1:
 *   S <- S diag(alpha_t); S <- S + beta_t (v_t - S k_t) k_t^T; o_t = S q_t
 * with the state held on chip, writes the T outputs (out: [T][B][Hv][d] in
 * out_dtype; NULL = none), and then quantizes S_T into the record exactly as
 * lq_state_init does (buffers empty, buf_n = 0).  Inputs are token-major:
 * q, k [T][B][Hk][d], v [T][B][Hv][d] (in_dtype), alpha [T][B][Hv] (GDN) or
 * [T][B][Hv][d] (KDA), beta [T][B][Hv], fp32.  T >= 0 (T = 0 quantizes S0).
 * mask: nullable [B] int32; masked-off sequences are left untouched.
 * The recurrence runs in chunks of 16 tokens in its WY form: with cumulative
 * gates g_t inside a chunk, Kg = K o g, Kh = K / g, Qg = Q o g,
 *   U = (I + strict_lower(diag(beta) Kg Kh^T))^-1 diag(beta) (V - Kg S^T),
 *   O = Qg S^T + lower(Qg Kh^T) U,  S <- S diag(g_last) + U^T (Kh o g_last),
 * equal to the token loop in exact arithmetic; the products with the state
 * run on the tensor cores at about fp32 accuracy.  Kh divides by the gates,
 * so the product of any 16 consecutive gates must stay a normal fp32 number
 * (above 1.2e-38). */
lq_status lq_prefill(const lq_config *cfg, const void *q, const void *k, const void *v,
                     const float *alpha, const float *beta, int32_t T, const float *S0,
                     const lq_state *st, void *out, const int32_t *mask, void *stream);

/* One decode token for every tile (zhichai.net summary, items 1-3; news
 * article paragraph 3).  Reads the int8 record as stored (no dequantized copy
 * in memory) and the buffered tokens, writes o_t = S_t q_t, appends
 * (k_t, d_t, alpha_t) to the buffer, and when the buffer holds W tokens folds
 * it into the state, extracts K compensator lines, smooths and requantizes
 * the residual, all in the same kernel.
 *  q, k  [B][Hk][d] in_dtype;  v [B][Hv][d] in_dtype (16-byte aligned);
 *  alpha [B][Hv] (GDN) or [B][Hv][d] (KDA, 16-byte aligned) fp32;
 *  beta  [B][Hv] fp32;
 *  out   [B][Hv][d] out_dtype (written for active sequences only);
 *  active nullable [B] int32: sequences with active[b] == 0 are skipped
 *  entirely (state and output untouched). */
lq_status lq_decode_step(const lq_config *cfg, const void *q, const void *k, const void *v,
                         const float *alpha, const float *beta, const lq_state *st, void *out,
                         const int32_t *active, void *stream);

/* ntok consecutive decode tokens for every tile in ONE launch, e.g. the
 * verify step of speculative decoding: the result is that of ntok calls of
 * lq_decode_step with the same active mask, folds at window boundaries
 * included.  Inside a window the stored record is fixed and each token only
 * reads it (zhichai.net summary, "Abstract (translated)" item 1), so the
 * launch reads each record once for all its tokens instead of once per token.
 * Inputs and outputs are token-major, each token laid out as for
 * lq_decode_step: q, k [ntok][B][Hk][d], v [ntok][B][Hv][d] in_dtype (16-byte
 * aligned); alpha [ntok][B][Hv] (GDN) or [ntok][B][Hv][d] (KDA, 16-byte
 * aligned); beta [ntok][B][Hv] fp32; out [ntok][B][Hv][d] out_dtype.
 * ntok >= 0 (0 does nothing).  Rejected drafts are dropped afterwards with
 * lq_window_rewind.  One CTA per tile keeps the tile in shared memory for all
 * its tokens; this call also serves every decode step of windows longer than
 * 16 tokens. */
lq_status lq_decode_tokens(const lq_config *cfg, int32_t ntok, const void *q, const void *k,
                           const void *v, const float *alpha, const float *beta,
                           const lq_state *st, void *out, const int32_t *active, void *stream);

/* lq_decode_step with the token's inputs packed per tile: the same step, the
 * same results.  qkva: [B][Hv] blocks back to back, 16-byte aligned, one per
 * tile (sequence b, value head h): q and k of key head h / (Hv / Hk), v of the
 * tile (d values each, in_dtype), then for KDA the tile's gate alpha (d
 * fp32).  A block is 3 d sizeof(in_dtype) (+ 4 d for KDA) bytes.  For GDN,
 * alpha stays a separate [B][Hv] fp32 array; for KDA alpha must be NULL or is
 * ignored.  beta, out and active as for lq_decode_step.
 *  - Why: each of a tile's inputs is otherwise a bulk copy of its own into
 *    shared memory, and four small copies per tile cost more than their
 *    bytes; a block comes in one.  With grouped heads (Hv > Hk) the caller
 *    writes q and k once per value head.
 *  - W up to 16 only (LQ_ERR_UNSUPPORTED above); arguments are checked as for
 *    lq_decode_step (qkva 16-byte aligned). */
lq_status lq_decode_step_packed(const lq_config *cfg, const void *qkva, const float *alpha,
                                const float *beta, const lq_state *st, void *out,
                                const int32_t *active, void *stream);

/* lq_decode_step with the token's inputs and output in HOST memory: moves
 * q, k, v, alpha, beta to `staging` (device, layout.host_staging_bytes,
 * 16-byte aligned), runs the step, and copies o back to out_host, all
 * asynchronously on `stream` (the caller synchronizes before reading
 * out_host).  The state stays on the device.  active is a device pointer, as
 * above; with it, rows of inactive sequences in out_host come back unchanged
 * (the call reads out_host's current rows into the staging before the step and
 * copies the whole output region back), so out_host must stay unchanged by
 * the host until the stream reaches the output copy.
 *  - Inputs that sit back to back in host memory in the order q, k, v,
 *    alpha, beta, when each of their sizes is a multiple of 256 bytes (so
 *    that the staging holds them back to back too), are moved by one
 *    cudaMemcpyAsync: a single copy-engine start-up, and no SM held while
 *    the bytes cross the host link, so that the copy overlaps kernels of
 *    other streams.
 *  - Otherwise, inputs in pinned memory that the device maps at the same address
 *    (cudaHostAlloc / cudaMallocHost memory under unified addressing, as the
 *    driver reports through cudaPointerGetAttributes for both ends of the
 *    input) are read by one gather kernel over the host link: a token's small
 *    inputs then move without a copy-engine start-up per input.
 *  - Any other host memory is copied with cudaMemcpyAsync (pageable memory
 *    makes those copies synchronous with the host).
 *  - The host buffers must hold the sizes listed for lq_decode_step and stay
 *    unchanged until the stream reaches the step. */
lq_status lq_decode_step_host(const lq_config *cfg, const void *q_host, const void *k_host,
                              const void *v_host, const float *alpha_host,
                              const float *beta_host, const lq_state *st, void *out_host,
                              void *staging, const int32_t *active, void *stream);

/* lq_decode_step_host for callers that cannot allocate device memory (the
 * pages have no counterpart: this is an interface convenience).
 *
 * Some callers cannot call cudaMalloc: a plugin running inside a host
 * application that owns every device allocation, or a latency-critical loop in
 * which an allocation, which may synchronize the whole device, is not
 * acceptable.  This variant takes no staging pointer: it stages the token's
 * inputs and output in a fixed array of LQ_NOALLOC_STAGING_MAX_BYTES inside the
 * library's own device memory, which every GPU that loads the library holds
 * until the process exits.  It calls no allocating routine.
 *  - Problems whose staging (layout.host_staging_bytes) exceeds
 *    LQ_NOALLOC_STAGING_MAX_BYTES are rejected with LQ_ERR_TOO_LARGE before
 *    anything is launched.
 *  - Every argument is checked, as lq_decode_step_host checks it, before the
 *    array is looked up or touched.
 *  - All calls share the array and it keeps the previous call's contents.  No
 *    stale byte reaches the caller: every output row copied back is written
 *    by this call (with an active mask, inactive rows come back unchanged, as
 *    for lq_decode_step_host).  Calls that overlap on the GPU (other streams
 *    or other threads) race on the array: the caller must order them.
 *  - The first call on each device looks up the array's device address (with
 *    that device current) and caches it; make that first call before any
 *    stream capture.  The cached address belongs to the device's primary
 *    context: after cudaDeviceReset, reload the library before calling this
 *    entry point again on that device.
 * Arguments and results are otherwise those of lq_decode_step_host. */
#define LQ_NOALLOC_STAGING_MAX_BYTES ((size_t)8 << 20)
lq_status lq_decode_step_host_noalloc(const lq_config *cfg, const void *q_host,
                                      const void *k_host, const void *v_host,
                                      const float *alpha_host, const float *beta_host,
                                      const lq_state *st, void *out_host, const int32_t *active,
                                      void *stream);

/* TESTING ONLY (no counterpart on the pages): the failure path of the
 * bounded waits.  Runs lq_decode_step except that the first CTA issues no
 * copies for its first ring slot, so that its wait on that slot expires
 * after `wait_limit` polls (> 0; production launches use 2^24).  That CTA
 * sets the timeout bit of the error word, waits (bounded) for its other
 * copies, and returns without touching the rest of its tiles; nothing is in
 * flight into the withheld slot.  Returns the launch status; afterwards
 * lq_get_last_error reports LQ_ERR_TIMEOUT.  The state of the skipped tiles
 * is left inconsistent: re-initialise it before further use.  Inputs as for
 * lq_decode_step (all sequences active). */
lq_status lq_test_decode_step_timeout(const lq_config *cfg, const void *q, const void *k,
                                      const void *v, const float *alpha, const float *beta,
                                      const lq_state *st, void *out, uint32_t wait_limit,
                                      void *stream);

/* Prefix-cache checkpoints (news article on LeapQuant, paragraph 5: one
 * state checkpoint per 1,024 tokens for prefix caching).  The checkpoint of
 * sequence b is the Hv records of its tiles taken on a window boundary
 * (buf_n == 0; call lq_window_flush first when off one), so restoring it
 * gives a state that decodes on bit for bit.  pool: device memory of
 * num_slots x Hv x layout.record_bytes, 16-byte aligned; slot s holds one
 * sequence's checkpoint.  slots: device [B] int32, the pool slot of each
 * sequence, -1 to skip it.  One checkpoint costs Hv x record_bytes (19,472 B
 * per head at d = 128, K = 4) against Hv x 65,536 B for an fp32 state.
 * save: a tile off a boundary, or a slot >= num_slots, is skipped and sets
 * LQ_ERR_DEVICE_BOUNDS in the error word.  restore: the records are copied
 * in and buf_n is set to 0 (a slot >= num_slots likewise). */
lq_status lq_checkpoint_save(const lq_config *cfg, const lq_state *st, const int32_t *slots,
                             void *pool, int32_t num_slots, void *stream);
lq_status lq_checkpoint_restore(const lq_config *cfg, const void *pool, int32_t num_slots,
                                const int32_t *slots, const lq_state *st, void *stream);

/* Speculative decoding: drop the last drop[b] decoded tokens of sequence b
 * (drop: device [B] int32, 0 = keep all).  Inside a window the record is
 * fixed and the buffered tokens are appended entries (zhichai.net summary,
 * "Abstract (translated)", item 1: outputs from the fixed low-bit state plus
 * the buffer), so rejecting draft tokens only moves the window phase back
 * and the state afterwards is exactly the one that never saw them.  This
 * holds while no window boundary was crossed since the draft began: a drop
 * larger than the tile's buffered count (or negative) is refused for that
 * tile with LQ_ERR_DEVICE_BOUNDS in the error word.  The pages have no
 * counterpart to this call. */
lq_status lq_window_rewind(const lq_config *cfg, const lq_state *st, const int32_t *drop,
                           void *stream);

/* Fold a partially filled window now (0 < buf_n < W) for the selected
 * sequences, exactly as the boundary fold does (news article, paragraph 3:
 * reconstruct and quantize at the boundary).  Used at the end of a sequence
 * or before taking a checkpoint off a boundary.  mask: nullable [B] int32. */
lq_status lq_window_flush(const lq_config *cfg, const lq_state *st, const int32_t *mask,
                          void *stream);

/* The unquantized comparison path (the FP32-state baseline of the
 * opentrain.ai abstract): S <- S diag(alpha); S <- S + beta (v - S k) k^T;
 * o = S q, with S [B][Hv][d][d] fp32 read and written in place (16-byte
 * aligned).  Other arguments as lq_decode_step. */
lq_status lq_fp32_decode_step(const lq_config *cfg, const void *q, const void *k,
                              const void *v, const float *alpha, const float *beta, float *S,
                              void *out, void *stream);

/* Materialize states as fp32 [B][Hv][d][d] (tests and drift reports):
 * include_buffer == 0 gives the window-base state S0 of each record;
 * include_buffer != 0 gives the current state, S0 advanced by the buffered
 * tokens of the window. */
lq_status lq_state_dequantize(const lq_config *cfg, const lq_state *st, int32_t include_buffer,
                              float *S_out, void *stream);

/* Synchronize `stream`, read and clear *err.  LQ_OK if no kernel reported a
 * problem since the last call; LQ_ERR_TIMEOUT if a bounded wait expired;
 * LQ_ERR_DEVICE_BOUNDS if a corrupt window phase was seen; LQ_ERR_CUDA if the
 * stream itself failed. */
lq_status lq_get_last_error(const lq_state *st, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LEAPQUANT_H */
