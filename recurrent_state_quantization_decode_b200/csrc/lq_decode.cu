// Kernels of the int8-state LeapQuant GDN/KDA decode step for sm_100a.
//
// Method (page title, section): zhichai.net summary "LeapQuant: Training-Free
// 8-bit Quantization for Linear Attention Recurrent States", "Abstract
// (translated)" items 1-3; opentrain.ai "LeapQuant: Efficient Linear Attention
// with Accurate Recurrent State Quantization", "Abstract"; globaltechnewsdesk
// news article on LeapQuant, paragraphs 3-5.  A tile (sequence, value head)
// keeps a window-base state S0 = diag(sigma) Q diag(m) + compensator lines in
// int8 for a window of W tokens; each token's output comes from S0 plus the
// buffered tokens of the window, and the W-th token folds the buffer and
// requantizes.
//
// Design for B200:
//  * decode_kernel is persistent: about two CTAs per SM, each walking its tiles
//    through a shared-memory ring of two or three slots (three where they fit
//    in half an SM's shared memory).  One thread moves a tile's record (int8
//    codes + scales + lines), its buffered tokens and its inputs with bulk
//    asynchronous copies (cp.async.bulk, one destination CTA) that complete on
//    an mbarrier, so the next tiles stream in while the current one is computed.
//    Every mbarrier wait is bounded; on expiry the kernel flags the error word,
//    drains its own copies and returns.
//  * The two products y_q = S0 (Gamma o q) and y_k = S0 (Gamma o k) run on the
//    int8 tensor path: the stored codes are the A operand as they are, and the
//    two fp32 vectors x = m o Gamma o {q, k} are split exactly into four
//    radix-128 int8 digits each (8 columns = one n8 tile) with a power-of-two
//    scale.  The integer dot products are exact, so the result is the fp32
//    product up to the digits' truncation (<= 7.5e-9 max|x| per element) and
//    one rounding per combination step.  No code is ever converted to float on
//    this path.
//  * Plain tokens of d = 128 tiles with bf16 inputs (GDN and KDA) run on the
//    quad path: four warps take one tile and a CTA runs two tiles at once.
//    Warp w of a quad does the per-channel work of int8 k-chunk w (32 key
//    channels, its own digit scale: gate product or KDA decay ratios and the
//    chunk's share of the buffer coefficients, x, digits, compensator dots),
//    then, after the quad's one named barrier, finishes state rows 32w ..
//    32w + 31.  Boundary tokens, the list's last entries, run on the whole CTA.
//  * On the whole-CTA path (every token at d < 128, boundary tokens at
//    d = 128) GDN with bf16 inputs has one CTA barrier per tile before the
//    fold: one warp per k-chunk for the per-channel work, one warp for the
//    buffer coefficients c_s = rho_s k_s . k and a_s = rho_s k_s . q from a
//    bf16 m16n8k16 product, the other row warps fetching their codes
//    meanwhile.  The per-token values are double-buffered, so a warp may start
//    the next tile while others finish the current one, and every thread waits
//    on the slot's mbarrier itself.
//  * On the boundary token the fp32 state S = S0 diag(Gamma) + sum d_s kt_s^T
//    is built in registers, in the same fragment layout as the codes: the
//    dequantized base, then (d >= 64) the rank-W update on the tf32 tensor
//    path with each operand split into hi and lo parts, whose accumulator
//    fragment is that layout.  The quantizer (compensator lines, smoothing,
//    per-row int8) then runs on it.
//  * chunk_prefill_kernel runs the exact recurrence over a prompt in 16-token
//    chunks of its WY form, the products with the state on the tf32 tensor
//    path with the state itself in the codes' fragment layout, and ends in the
//    same quantizer.
//  * tokens_kernel decodes several tokens per tile in one launch (one CTA per
//    tile), and serves windows longer than 16 tokens.
//
// Fragment layout: warp w < D/16 owns state rows 16w..16w+15; lane (g = lane/4,
// t = lane%4) owns rows 16w+g and 16w+g+8 and, in every 64-column span h, the
// 16 columns 64h + 16t .. 64h + 16t + 15 (for d = 32 only t < 2 hold columns).
//
// Quantizer decisions use correctly rounded fp32 operations and fp64 line
// energies, so a given fp32 state always yields the same record.

#include <cfloat>
#include <cstdint>
#include <type_traits>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "lq_internal.h"

namespace lq {

RecLayout record_layout(int d, int K) {
  RecLayout L;
  L.off_sig = d * d;
  L.off_m = L.off_sig + 4 * d;
  L.off_cv = L.off_m + 4 * d;
  L.off_cid = L.off_cv + 4 * K * d;
  L.bytes = (L.off_cid + 4 * K + 15) / 16 * 16;
  return L;
}

namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxTilesPerCta = 128;

// ---------------------------------------------------------------------------
// Geometry and shared-memory layout
// ---------------------------------------------------------------------------

template <int D>
struct FG {
  static constexpr int NRB = D / 16;                  // warps that own state rows
  static constexpr int NSPAN = D >= 64 ? D / 64 : 1;  // 64-column spans
  static constexpr int PADW = D + D / 4;              // padded column vectors
  static constexpr int DIGW = 192;                    // digit row stride in bytes
  static_assert(NRB <= kWarps, "one warp per 16 rows");
};

// Padded index of column j: 4 floats of padding after every 16, so that the
// 16-float chunks that a warp reads start in different bank groups.
__device__ __forceinline__ int padc(int j) { return j + ((j >> 4) << 2); }
__device__ __forceinline__ int frag_col(int h, int t, int e) { return 64 * h + 16 * t + e; }
template <int D>
__device__ __forceinline__ bool chunk_valid(int t) {
  return D >= 64 || 16 * t < D;
}

// One tile's staged data (a ring slot): the record, the buffered tokens and the
// token's inputs, each at a 16-byte aligned offset.  The record area has the
// record's actual size (it depends on K).
template <int D, bool BF16, bool KDA, int WM = kMaxWindow>
struct SL {
  static constexpr int IB = BF16 ? 2 : 4;
  static constexpr int BD = WM * D * 4;                  // fp32 [WM][D]
  static constexpr int BK = WM * D * IB;                 // in dtype [WM][D]
  static constexpr int BG = KDA ? WM * D * 4 : WM * 4;   // KDA [WM][D]; GDN up to WM gates
  static constexpr int TAIL = BD + BK + BG + 3 * D * IB + (KDA ? D * 4 : 0);
  // quantizer scratch aliased over the codes once they are in registers
  static constexpr int QS_COLPART = 0;                           // fp64 [D/16][D]
  static constexpr int QS_COLMAX = FG<D>::NRB * D * 8;           // fp32 [D/16][D]
  static_assert(QS_COLMAX + FG<D>::NRB * D * 4 <= D * D, "scratch fits over the codes");
  int bd, bk, bg, q, k, v, a, bytes;
  __host__ __device__ explicit SL(int rec_bytes) {
    bd = rec_bytes;
    bk = bd + BD;
    bg = bk + BK;
    q = bg + BG;
    k = q + D * IB;
    v = k + D * IB;
    a = v + D * IB;  // q, k, v and the gate back to back (packed inputs arrive in one copy)
    bytes = (rec_bytes + TAIL + 127) / 128 * 128;
  }
};

// Decode kernel variants.  GDN with bf16 inputs computes the buffer
// coefficients on the bf16 tensor path (fast) and, at d = 128, keeps the
// fold's scaled keys over the staged codes instead of in the scratch, which
// leaves room for three ring slots at two CTAs per SM.
template <int D, bool BF16, bool KDA, int WM = kMaxWindow>
struct DecodeTraits {
  // plain tokens (no fold) of d = 128 tiles with bf16 inputs run on the quad
  // path: four warps per tile, two tiles at once per CTA
  static constexpr bool kQuad = BF16 && D == 128 && WM == kMaxWindow;
  // with one ring slot per quad (KDA), the quad releases its slot at its
  // barrier, after loading the row-phase operands into registers
  static constexpr bool kEarlyRelease = kQuad && KDA;
  static_assert(kEarlyRelease == (kQuad && KDA), "one ring slot per quad only on KDA");
  static constexpr bool kFast = BF16 && !KDA && WM == kMaxWindow;
  static constexpr bool kKtOverCodes = kFast && WM * FG<D>::PADW * 4 <= D * D;
  static constexpr int kStages = kFast ? 3 : 2;
  static constexpr int kTok = kFast ? 2 : 1;  // per-token scratch buffers
  // the fold's rank-W update on the tf32 tensor path (3 products per term)
  static constexpr bool kMmaFold = D >= 64;
};

// Scaled-key layout of the tensor-path fold update: row s of width D + 8 (the
// 8-float pad puts the four k rows a warp reads at once in different banks);
// column c sits where lane g of n8 tile j of span h reads it, c = 64h +
// 16(g/2) + 2j + g%2, so that the accumulators land in the state's layout.
template <int D>
__host__ __device__ constexpr int kt_mma_stride() { return D + 8; }
__device__ __forceinline__ int kt_mma_pos(int c);
// Index of scaled key (token s, column c) in the fold's key array.
template <int D, bool MMA>
__device__ __forceinline__ int kt_index(int s, int c) {
  if constexpr (MMA)
    return s * kt_mma_stride<D>() + kt_mma_pos(c);
  else
    return s * FG<D>::PADW + padc(c);
}
__device__ __forceinline__ int kt_mma_pos(int c) {
  const int r = c & 63;
  return (c & ~63) + 8 * ((r & 15) >> 1) + 2 * (r >> 4) + (r & 1);
}

// The scaled-key array lives in the scratch unless the decode kernel keeps it
// over the staged codes (GDN with bf16 inputs).
template <int D, bool KT, int WM = kMaxWindow>
struct KtArea {
  alignas(16) float kt[WM][FG<D>::PADW];  // keys times decay ratio to the last token
};
template <int D, int WM>
struct KtArea<D, false, WM> {};

// Per-token values that the row phase reads: written before the tile's CTA
// barrier, read after it.  The decode kernel for GDN with bf16 inputs keeps two
// of these, so that one tile's per-channel work can overlap the previous
// tile's row phase.
template <int D, int WM = kMaxWindow>
struct Tok {
  alignas(16) float qf[D];
  alignas(16) float kf[D];
  alignas(16) float vf[D];
  alignas(16) float G[D];                          // window gate Gamma per key channel
  alignas(16) float mG[FG<D>::PADW];               // m o Gamma
  alignas(16) int8_t dig[8][FG<D>::DIGW];          // digits: rows 0-3 of x_q, 4-7 of x_k
  float cc[WM + 1];
  float aa[WM + 1];
  float cpart[kMaxComp][kWarps][2];  // per-warp partial row-compensator dots
  float rho[WM + 1];                 // scalar decay ratios (GDN)
  float xmax[2][kWarps];
  float xscale[2][4];  // digit scales of x_q, x_k (per int8 k-chunk on the GDN-bf16 path)
};

// Per-token values of the quad path, written by the quad's four warps before
// its barrier and read by them after it.  Each quad keeps two, so that a warp
// may start the next tile's channel work while the others finish the rows.
template <int D>
struct QTok {
  alignas(16) int8_t dig[8][FG<D>::DIGW];  // digits: rows 0-3 of x_q, 4-7 of x_k
  float xscale[2][4];                       // digit scale of each k-chunk (x_q, x_k)
  float cpart[kMaxComp][4][2];              // row-compensator dots: one partial per warp
  float colv[kMaxComp][2];                  // column compensator j: Gamma_j q_j, Gamma_j k_j
  float cc[kMaxWindow + 1];                 // GDN: c_s = rho_s k_s . k
  float aa[kMaxWindow + 1];                 // GDN: a_s = rho_s k_s . q
  float rho[kMaxWindow + 1];                // GDN: decay ratios
  float cpk[4][2 * kMaxWindow];             // KDA: per warp, partial c_s (s) and a_s (16 + s)
};

template <int D, int NT, bool Q, int WM>
union TokArea {
  Tok<D, WM> tok[NT];
};
template <int D, int NT, int WM>
union TokArea<D, NT, true, WM> {
  Tok<D, WM> tok[NT];  // the whole-CTA path
  QTok<D> qt[2][2];    // the quad path: [quad][buffer]
};

template <int D, bool KT, int NT = 1, bool Q = false, int WM = kMaxWindow>
struct Scratch : KtArea<D, KT, WM> {
  TokArea<D, NT, Q, WM> u;
  alignas(16) float invm[FG<D>::PADW];             // 1 / m (new smoothing factors)
  alignas(16) float line[D];                       // the compensator line being extracted
  alignas(16) double rowE[D];
  unsigned long long pkey[kWarps];   // per-warp best selection key of the line energies
  int pid[kWarps];
  int abort;
  int done[3];       // warps finished with each ring slot (GDN-bf16 and quad paths)
  int slot_last[3];  // list index of the last tile whose copies went into each slot
  int warp_cnt[kWarps];
  int warp_cnt2[kWarps];
  int tl_tile[kMaxTilesPerCta];
  int tl_n[kMaxTilesPerCta];      // window phase; -1: skip (corrupt phase)
  int tl_coord[kMaxTilesPerCta];  // b << 12 | hk << 1 | (this value head writes the key)
  float tl_a[kMaxTilesPerCta];
  float tl_b[kMaxTilesPerCta];
  alignas(8) unsigned long long bar[3];
};

// ---------------------------------------------------------------------------
// Small helpers and PTX wrappers
// ---------------------------------------------------------------------------

template <bool BF16>
using in_t = std::conditional_t<BF16, __nv_bfloat16, float>;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

__device__ __forceinline__ void st_out(void *p, size_t i, float x, int bf16) {
  if (bf16)
    reinterpret_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(x);
  else
    reinterpret_cast<float *>(p)[i] = x;
}


// int8 code e (0..15) of a 16-byte chunk as a float, without an int->float
// conversion: the byte, biased to unsigned, becomes the low mantissa byte of
// 2^23 + (c + 128), and subtracting 2^23 + 128 recovers c exactly.
__device__ __forceinline__ float code_at(const uint4 &c, int e) {
  const uint32_t w = (e < 4) ? c.x : (e < 8) ? c.y : (e < 12) ? c.z : c.w;
  const uint32_t bits = __byte_perm(w ^ 0x80808080u, 0x4B000000u, 0x7540u + (e & 3));
  return __uint_as_float(bits) - 8388736.0f;
}

// Round-half-even of |x| < 2^22 with one add: the integer lands in the low
// mantissa bits of x + 1.5 * 2^23 (its low byte is the two's-complement int8).
constexpr float kRoundMagic = 12582912.0f;

__device__ __forceinline__ uint32_t smem_u32(const void *ptr) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(ptr));
}

__device__ __forceinline__ void mbar_init(unsigned long long *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(unsigned long long *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(unsigned long long *bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(unsigned long long *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait on one phase of an mbarrier; false after kWaitLimit polls.
__device__ __forceinline__ bool mbar_wait_bounded(unsigned long long *bar, uint32_t parity,
                                                  uint32_t limit) {
  for (uint32_t it = 0; it < limit; ++it)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// Global -> shared bulk copy into this CTA only, completing on `bar`.  dst, src and
// bytes must be multiples of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         unsigned long long *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Orders this thread's earlier generic-proxy shared-memory accesses before the
// async-proxy writes of a following bulk copy into the same memory.
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// D (16x8, int32) += A (16x32, int8, row) x B (32x8, int8, col).
__device__ __forceinline__ void mma_s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                       uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D (16x8, fp32) += A (16x16, bf16, row) x B (16x8, bf16, col).
__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D (16x8, fp32) += A (16x8, tf32, row) x B (8x8, tf32, col); c01 holds row g,
// c23 row g + 8 (columns 2t, 2t + 1).
__device__ __forceinline__ void mma_tf32(float2 &c01, float2 &c23, uint32_t a0, uint32_t a1,
                                         uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c01.x), "+f"(c01.y), "+f"(c23.x), "+f"(c23.y)
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Rounds a finite fp32 value to tf32 (10 explicit mantissa bits), to nearest
// with ties away from zero: adding half of the last kept bit to the
// magnitude's bit pattern carries into the kept bits exactly when the dropped
// part is at least half of it, and the mask drops the rest.  Integer ALU work
// only, in place of a conversion instruction.
__device__ __forceinline__ uint32_t tf32_rna(float x) {
  return (__float_as_uint(x) + 0x1000u) & 0xFFFFE000u;
}

// x = hi + lo with hi, lo tf32 (round to nearest); hi * hi' + hi * lo' + lo * hi'
// then reproduces an fp32 product to about 2^-22 relative.  x - hi is exact.
__device__ __forceinline__ void tf32_split(float x, uint32_t &hi, uint32_t &lo) {
  hi = tf32_rna(x);
  lo = tf32_rna(x - __uint_as_float(hi));
}

// Exact split of x into four radix-128 digits with the power-of-two scale
// s = 2^(E-6), where max|x| = M < 2^E:  x = s (d0 + d1/128 + d2/128^2 +
// d3/128^3) + r with |r| <= s / (2 * 128^3).  Every step is exact in fp32,
// and |d_i| <= 64.
__device__ __forceinline__ void split_digits(float x, float M, int8_t *dst, int stride) {
  int8_t d[4] = {0, 0, 0, 0};
  if (M > 0.0f) {
    const int eb = static_cast<int>((__float_as_uint(M) >> 23) & 0xffu);
    float u;
    if (eb >= 6) {
      // M < 2^(eb - 126): multiply by 2^(132 - eb), exact
      u = x * __uint_as_float(static_cast<uint32_t>(259 - eb) << 23);
    } else {
      int E;
      frexpf(M, &E);
      u = ldexpf(x, 6 - E);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float biased = u + kRoundMagic;
      d[i] = static_cast<int8_t>(__float_as_uint(biased) & 0xffu);
      u = (u - (biased - kRoundMagic)) * 128.0f;
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) dst[i * stride] = d[i];
}

// max over the warp of |x| (one redux instruction on sm_100a)
__device__ __forceinline__ float warp_max_abs(float x) {
  float r;
  asm volatile("redux.sync.max.abs.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(x));
  return r;
}

// Sums 8 per-lane values over the warp: afterwards every lane holds the total
// of value (lane >> 2) & 7.
__device__ __forceinline__ float warp_sum8(float (&v)[8], int lane) {
#pragma unroll
  for (int step = 16, half = 4; step >= 4; step >>= 1, half >>= 1) {
    const bool upper = (lane & step) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? v[i] : v[i + half];
      const float keep = upper ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(kFull, send, step);
    }
  }
  float r = v[0];
  r += __shfl_xor_sync(kFull, r, 2);
  r += __shfl_xor_sync(kFull, r, 1);
  return r;
}

__device__ __forceinline__ float digit_scale(float M) {
  if (!(M > 0.0f)) return 0.0f;
  int E;
  frexpf(M, &E);
  return ldexpf(1.0f, E - 6);
}

// Reduce NV per-lane values over the 8 lanes that share t (lane bits 2-4),
// halving the set at each step: afterwards lane (g, t) holds the totals of
// values NV/8 * g .. NV/8 * g + NV/8 - 1 in v[0 .. NV/8) (for NV = 16:
// values 2g and 2g + 1).
template <int NV, typename T, typename Op>
__device__ __forceinline__ void butterfly_g(T (&v)[NV], int lane, Op op) {
#pragma unroll
  for (int step = 16, half = NV / 2; step >= 4; step >>= 1, half >>= 1) {
    const bool upper = (lane & step) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const T send = upper ? v[i] : v[i + half];
      const T keep = upper ? v[i + half] : v[i];
      v[i] = op(keep, __shfl_xor_sync(kFull, send, step));
    }
  }
}

struct AddOp {
  template <typename T>
  __device__ __forceinline__ T operator()(T a, T b) const { return a + b; }
};
struct MaxOp {
  __device__ __forceinline__ float operator()(float a, float b) const { return fmaxf(a, b); }
};

// ---------------------------------------------------------------------------
// State build and quantizer (fragment layout)
// ---------------------------------------------------------------------------

// Loads the thread's codes (rows r0 = 16 warp + g and r0 + 8, its 16-byte
// chunk of every span) from the staged record.
template <int D>
__device__ __forceinline__ void load_codes(const uint8_t *codes, uint4 (&A)[2][FG<D>::NSPAN]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int r0 = 16 * warp + g;
#pragma unroll
  for (int h = 0; h < FG<D>::NSPAN; ++h) {
    if (chunk_valid<D>(t)) {
      A[0][h] = *reinterpret_cast<const uint4 *>(codes + r0 * D + frag_col(h, t, 0));
      A[1][h] = *reinterpret_cast<const uint4 *>(codes + (r0 + 8) * D + frag_col(h, t, 0));
    } else {
      A[0][h] = make_uint4(0, 0, 0, 0);
      A[1][h] = make_uint4(0, 0, 0, 0);
    }
  }
}

// Element e (0..15) of span h of row rr in a float2 register tile.
#define SX(rr, h, e) ((((e) & 1) != 0) ? S[rr][h][(e) >> 1].y : S[rr][h][(e) >> 1].x)

// f(entry of row r0, entry of row r1) at column slot e (0..15) of span h of
// this lane's fragment, for a runtime (h, e) that every calling lane shares:
// a switch reaches the one register pair instead of testing all 32 slots.
#define LQ_SLOT(H, E) \
  case (H) * 16 + (E): f(SX(0, H, E), SX(1, H, E)); break;
#define LQ_SPAN(H) \
  LQ_SLOT(H, 0) LQ_SLOT(H, 1) LQ_SLOT(H, 2) LQ_SLOT(H, 3) LQ_SLOT(H, 4) LQ_SLOT(H, 5) \
  LQ_SLOT(H, 6) LQ_SLOT(H, 7) LQ_SLOT(H, 8) LQ_SLOT(H, 9) LQ_SLOT(H, 10) LQ_SLOT(H, 11) \
  LQ_SLOT(H, 12) LQ_SLOT(H, 13) LQ_SLOT(H, 14) LQ_SLOT(H, 15)
template <int NSPAN, class F>
__device__ __forceinline__ void at_slot(float2 (&S)[2][NSPAN][8], int h, int e, F &&f) {
  if constexpr (NSPAN > 1) {
    switch (h * 16 + e) { LQ_SPAN(0) LQ_SPAN(1) default: break; }
  } else {
    switch (h * 16 + e) { LQ_SPAN(0) default: break; }
  }
}
#undef LQ_SPAN
#undef LQ_SLOT

// S += sum_{s < nent} d_s kt_s^T for the thread's block on the tf32 tensor
// path: A = d (16 rows x 8 tokens, rows [s][D] in bd), B = scaled keys (8
// tokens x 8 columns) in the layout of kt_mma_pos (rows of kt_mma_stride);
// each operand is split into hi and lo tf32 parts and three products are
// accumulated.  Tokens at or beyond nent (at most SMAX) contribute zero.
template <int D, int SMAX>
__device__ __forceinline__ void rank_update_mma(float2 (&S)[2][FG<D>::NSPAN][8], const float *bd,
                                                const float *kt, int nent) {
  using G = FG<D>;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int r0 = 16 * warp + g, r1 = r0 + 8;
  constexpr int P = kt_mma_stride<D>();
#pragma unroll
  for (int ks = 0; ks < SMAX / 8; ++ks) {
    if (8 * ks >= nent) break;
    const int s0 = 8 * ks + t, s1 = s0 + 4;
    uint32_t ah[4], al[4];
    tf32_split(s0 < nent ? bd[s0 * D + r0] : 0.0f, ah[0], al[0]);
    tf32_split(s0 < nent ? bd[s0 * D + r1] : 0.0f, ah[1], al[1]);
    tf32_split(s1 < nent ? bd[s1 * D + r0] : 0.0f, ah[2], al[2]);
    tf32_split(s1 < nent ? bd[s1 * D + r1] : 0.0f, ah[3], al[3]);
#pragma unroll
    for (int h = 0; h < G::NSPAN; ++h)
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int pos = 64 * h + 8 * j + g;
        uint32_t bh0, bl0, bh1, bl1;
        tf32_split(s0 < nent ? kt[s0 * P + pos] : 0.0f, bh0, bl0);
        tf32_split(s1 < nent ? kt[s1 * P + pos] : 0.0f, bh1, bl1);
        mma_tf32(S[0][h][j], S[1][h][j], al[0], al[1], al[2], al[3], bh0, bh1);
        mma_tf32(S[0][h][j], S[1][h][j], ah[0], ah[1], ah[2], ah[3], bl0, bl1);
        mma_tf32(S[0][h][j], S[1][h][j], ah[0], ah[1], ah[2], ah[3], bh0, bh1);
      }
  }
}

// The same update with packed FMAs, two columns per instruction; kt rows of
// PADW in the padded column layout (padc).
template <int D>
__device__ __forceinline__ void rank_update_ffma(float2 (&S)[2][FG<D>::NSPAN][8], const float *bd,
                                                 const float *kt, int nent) {
  using G = FG<D>;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int r0 = 16 * warp + g, r1 = r0 + 8;
  for (int sl = 0; sl < nent; ++sl) {
    const float2 d0 = make_float2(bd[sl * D + r0], bd[sl * D + r0]);
    const float2 d1 = make_float2(bd[sl * D + r1], bd[sl * D + r1]);
#pragma unroll
    for (int h = 0; h < G::NSPAN; ++h) {
      if (!chunk_valid<D>(t)) continue;
      const float4 *k4 =
          reinterpret_cast<const float4 *>(&kt[sl * G::PADW + padc(frag_col(h, t, 0))]);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float4 k = k4[u];
        const float2 ka = make_float2(k.x, k.y), kb = make_float2(k.z, k.w);
        S[0][h][2 * u] = __ffma2_rn(d0, ka, S[0][h][2 * u]);
        S[0][h][2 * u + 1] = __ffma2_rn(d0, kb, S[0][h][2 * u + 1]);
        S[1][h][2 * u] = __ffma2_rn(d1, ka, S[1][h][2 * u]);
        S[1][h][2 * u + 1] = __ffma2_rn(d1, kb, S[1][h][2 * u + 1]);
      }
    }
  }
}

// The fp32 state of the thread's block (warps that own rows), as float2 pairs
// along the columns:
//   S_ij = sigma_i code_ij (m_j Gamma_j) + sum_{s < nent} d_s[i] kt_s[j]
//          + Gamma_j * (compensator lines),
// with kt_s = k_s o (decay ratio to the last token) in kt (rows of PADW) and m o Gamma in
// x.mG.  rsig, rcv, rcid point at the staged record; bd at the staged deltas.
template <int D, bool MMA = false, int WM = kMaxWindow, class SC>
__device__ __forceinline__ void build_state(const SC &x, const float *kt,
                                            const uint4 (&A)[2][FG<D>::NSPAN],
                                            const float *rsig, const float *rcv, const int *rcid,
                                            const float *bd, int nent, int K,
                                            float2 (&S)[2][FG<D>::NSPAN][8]) {
  using G = FG<D>;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int r0 = 16 * warp + g, r1 = r0 + 8;
  const float2 sg0 = make_float2(rsig[r0], rsig[r0]), sg1 = make_float2(rsig[r1], rsig[r1]);
#pragma unroll
  for (int h = 0; h < G::NSPAN; ++h) {
    if (chunk_valid<D>(t)) {
      const float4 *mg4 = reinterpret_cast<const float4 *>(&x.mG[padc(frag_col(h, t, 0))]);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float4 m = mg4[u];
        const float2 ma = make_float2(m.x, m.y), mb = make_float2(m.z, m.w);
        const int e = 4 * u;
        S[0][h][2 * u] = __fmul2_rn(__fmul2_rn(sg0, make_float2(code_at(A[0][h], e),
                                                                 code_at(A[0][h], e + 1))), ma);
        S[0][h][2 * u + 1] = __fmul2_rn(
            __fmul2_rn(sg0, make_float2(code_at(A[0][h], e + 2), code_at(A[0][h], e + 3))), mb);
        S[1][h][2 * u] = __fmul2_rn(__fmul2_rn(sg1, make_float2(code_at(A[1][h], e),
                                                                 code_at(A[1][h], e + 1))), ma);
        S[1][h][2 * u + 1] = __fmul2_rn(
            __fmul2_rn(sg1, make_float2(code_at(A[1][h], e + 2), code_at(A[1][h], e + 3))), mb);
      }
    } else {
#pragma unroll
      for (int e2 = 0; e2 < 8; ++e2) S[0][h][e2] = S[1][h][e2] = make_float2(0.0f, 0.0f);
    }
  }
  if constexpr (MMA)
    rank_update_mma<D, WM>(S, bd, kt, nent);
  else
    rank_update_ffma<D>(S, bd, kt, nent);
  // compensator lines, decayed by Gamma
  for (int c = 0; c < K; ++c) {
    const int id = rcid[c];
    if (id < D) {
      // a row line lands in one warp (rows 16 w .. 16 w + 15)
      if (warp == (id >> 4) && (id == r0 || id == r1) && chunk_valid<D>(t)) {
        const bool second = id == r1;
#pragma unroll
        for (int h = 0; h < G::NSPAN; ++h)
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int col = frag_col(h, t, e);
            const float add = rcv[c * D + col] * x.G[col];
            if (second) SX(1, h, e) += add; else SX(0, h, e) += add;
          }
      }
    } else {
      const int jc = id - D;
      if (((jc & 63) >> 4) == t && chunk_valid<D>(t)) {
        const float gj = x.G[jc];
        const float a0 = rcv[c * D + r0] * gj, a1 = rcv[c * D + r1] * gj;
        at_slot<G::NSPAN>(S, jc >> 6, jc & 15, [&](float &u0, float &u1) {
          u0 += a0;
          u1 += a1;
        });
      }
    }
  }
}

// Selection key of a candidate line for the greedy picks: 0 for a taken line,
// else 1 + the bit pattern of its fp64 energy, which orders like the value for
// a non-negative double; an energy that the subtractions of removed lines
// left below zero counts as zero.
__device__ __forceinline__ unsigned long long line_key(double e, bool taken) {
  if (taken) return 0ull;
  return (e > 0.0 ? static_cast<unsigned long long>(__double_as_longlong(e)) : 0ull) + 1ull;
}

// Quantize the state held in registers (fragment layout) into the record at
// rec (global):
//  1. K times: the untaken line (row or column) of the largest fp64 energy of
//     the residual (ties: lower id; rows are ids 0..D-1, columns D..2D-1) is
//     stored as an fp32 compensator vector and zeroed; the energies of the
//     crossing lines lose the removed squares (an energy that these
//     subtractions leave below zero counts as zero);
//  2. m_j from the residual's column max a_j: 1 if smoothing is off or
//     a_j < FLT_MIN, else sqrt(a_j) or a_j;
//  3. per row: x = (R_ij * (1/m_j)) * (127/b_i) with b_i the row max of
//     R_ij * (1/m_j); code = round-half-even(x) clamped to [-127, 127];
//     sigma_i = b_i / 127, or 1 with zero codes when b_i < FLT_MIN.
// colpart / colmax: shared scratch of (D/16) x D doubles / floats.
template <int D, class SC>
__device__ void quantize_tile(SC &s, double *colpart, float *colmax,
                              float2 (&S)[2][FG<D>::NSPAN][8], uint8_t *rec, const RecLayout &L,
                              int K, int smooth) {
  using G = FG<D>;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int r0 = 16 * warp + g, r1 = r0 + 8;
  const bool rows_here = warp < G::NRB;
  float *rsig = reinterpret_cast<float *>(rec + L.off_sig);
  float *rm = reinterpret_cast<float *>(rec + L.off_m);
  float *rcv = reinterpret_cast<float *>(rec + L.off_cv);
  int *rcid = reinterpret_cast<int *>(rec + L.off_cid);

  if (K > 0) {
    // Thread j < D owns candidate lines j (row j) and D + j (column j): their
    // fp64 energies and taken flags live in its registers.
    if (rows_here) {
      double e0 = 0.0, e1 = 0.0;
#pragma unroll
      for (int h = 0; h < G::NSPAN; ++h) {
        // eight columns at a time keeps the fp64 partials in few registers;
        // lane g ends with column 8 hh + g of the batch
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          double cp[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const double a = SX(0, h, 8 * hh + e), b = SX(1, h, 8 * hh + e);
            e0 = fma(a, a, e0);
            e1 = fma(b, b, e1);
            cp[e] = fma(a, a, b * b);
          }
          butterfly_g<8>(cp, lane, AddOp());
          if (chunk_valid<D>(t)) colpart[warp * D + frag_col(h, t, 8 * hh + g)] = cp[0];
        }
      }
      e0 += __shfl_xor_sync(kFull, e0, 1);
      e0 += __shfl_xor_sync(kFull, e0, 2);
      e1 += __shfl_xor_sync(kFull, e1, 1);
      e1 += __shfl_xor_sync(kFull, e1, 2);
      if (t == 0) {
        s.rowE[r0] = e0;
        s.rowE[r1] = e1;
      }
    }
    __syncthreads();
    double eRow = 0.0, eCol = 0.0;
    bool tRow = false, tCol = false;
    if (tid < D) {
      eRow = s.rowE[tid];
#pragma unroll
      for (int w = 0; w < G::NRB; ++w) eCol += colpart[w * D + tid];
    }
    for (int c = 0; c < K; ++c) {
      // argmax over this thread's two candidates (the row wins a tie: lower
      // id), then over the warp: the largest key, then the lowest id holding it
      if (warp < (D + 31) / 32) {
        const unsigned long long kr = line_key(eRow, tRow), kc = line_key(eCol, tCol);
        unsigned long long key = kr;
        int bid = tid;
        if (kc > kr) {
          key = kc;
          bid = D + tid;
        }
        const uint32_t khi = static_cast<uint32_t>(key >> 32), klo = static_cast<uint32_t>(key);
        const uint32_t whi = __reduce_max_sync(kFull, khi);
        const uint32_t wlo = __reduce_max_sync(kFull, khi == whi ? klo : 0u);
        const uint32_t wid =
            __reduce_min_sync(kFull, (khi == whi && klo == wlo) ? static_cast<uint32_t>(bid)
                                                                : 0xffffffffu);
        if (lane == 0) {
          s.pkey[warp] = (static_cast<unsigned long long>(whi) << 32) | wlo;
          s.pid[warp] = static_cast<int>(wid);
        }
      }
      __syncthreads();
      // every thread combines the per-warp winners (same result everywhere)
      int id = 0x7fffffff;
      {
        unsigned long long best = 0ull;
#pragma unroll
        for (int w = 0; w < (D + 31) / 32; ++w) {
          const unsigned long long k = s.pkey[w];
          const int i2 = s.pid[w];
          if (k > best || (k == best && i2 < id)) {
            best = k;
            id = i2;
          }
        }
      }
      // the owners of the line park its values in s.line and zero them: a
      // row lives in one warp (rows 16 w .. 16 w + 15), a column in all
      if (rows_here) {
        if (id < D) {
          if (warp == (id >> 4)) {
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
              if ((rr ? r1 : r0) != id || !chunk_valid<D>(t)) continue;
#pragma unroll
              for (int h = 0; h < G::NSPAN; ++h) {
                float4 *dst = reinterpret_cast<float4 *>(&s.line[frag_col(h, t, 0)]);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                  dst[u] = make_float4(S[rr][h][2 * u].x, S[rr][h][2 * u].y, S[rr][h][2 * u + 1].x,
                                       S[rr][h][2 * u + 1].y);
                  S[rr][h][2 * u] = make_float2(0.0f, 0.0f);
                  S[rr][h][2 * u + 1] = make_float2(0.0f, 0.0f);
                }
              }
            }
          }
        } else {
          const int jc = id - D;
          if (((jc & 63) >> 4) == t && chunk_valid<D>(t)) {
            at_slot<G::NSPAN>(S, jc >> 6, jc & 15, [&](float &u0, float &u1) {
              s.line[r0] = u0;
              s.line[r1] = u1;
              u0 = 0.0f;
              u1 = 0.0f;
            });
          }
        }
      }
      __syncthreads();
      // store the line; the crossing lines lose its squares; mark it taken
      if (tid < D) {
        const float v = s.line[tid];
        rcv[c * D + tid] = v;
        const double v2 = static_cast<double>(v) * static_cast<double>(v);
        if (id < D) {
          eCol -= v2;
          if (id == tid) tRow = true;
        } else {
          eRow -= v2;
          if (id == D + tid) tCol = true;
        }
        if (tid == 0) rcid[c] = id;
      }
    }
  }

  // Smoothing factors from the residual's column maxima.
  if (rows_here) {
#pragma unroll
    for (int h = 0; h < G::NSPAN; ++h) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float cm[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          cm[e] = fmaxf(fabsf(SX(0, h, 8 * hh + e)), fabsf(SX(1, h, 8 * hh + e)));
        butterfly_g<8>(cm, lane, MaxOp());
        if (chunk_valid<D>(t)) colmax[warp * D + frag_col(h, t, 8 * hh + g)] = cm[0];
      }
    }
  }
  __syncthreads();
  if (tid < D) {
    float a = 0.0f;
#pragma unroll
    for (int w = 0; w < G::NRB; ++w) a = fmaxf(a, colmax[w * D + tid]);
    float mj;
    if (smooth == 0 || a < FLT_MIN)
      mj = 1.0f;
    else if (smooth == 1)
      mj = __fsqrt_rn(a);
    else
      mj = a;
    rm[tid] = mj;
    s.invm[padc(tid)] = __frcp_rn(mj);
  }
  __syncthreads();

  // Per-row scales and int8 codes.  1/m is loaded once for both rows.
  if (rows_here) {
#pragma unroll
    for (int h = 0; h < G::NSPAN; ++h) {
      if (!chunk_valid<D>(t)) continue;
      const float4 *im4 = reinterpret_cast<const float4 *>(&s.invm[padc(frag_col(h, t, 0))]);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float4 im = im4[u];
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          S[rr][h][2 * u] = __fmul2_rn(S[rr][h][2 * u], make_float2(im.x, im.y));
          S[rr][h][2 * u + 1] = __fmul2_rn(S[rr][h][2 * u + 1], make_float2(im.z, im.w));
        }
      }
    }
    // Row maxima of both rows, then sigma = b / 127 and 1 / sigma = 127 / b,
    // each correctly rounded: one division per lane, lane t of a row group
    // taking row t / 2 (sigma for even t, its inverse for odd t), shared by
    // shuffles.  A row below FLT_MIN gets sigma = 1 and zero codes.
    float bm[2];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      float bmax = 0.0f;
#pragma unroll
      for (int h = 0; h < G::NSPAN; ++h) {
        if (!chunk_valid<D>(t)) continue;
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2)
          bmax = fmaxf(bmax, fmaxf(fabsf(S[rr][h][e2].x), fabsf(S[rr][h][e2].y)));
      }
      bmax = fmaxf(bmax, __shfl_xor_sync(kFull, bmax, 1));
      bm[rr] = fmaxf(bmax, __shfl_xor_sync(kFull, bmax, 2));
    }
    const float bsel = (t >> 1) ? bm[1] : bm[0];
    float qd;
    if (bsel < FLT_MIN)
      qd = (t & 1) ? 0.0f : 1.0f;
    else
      qd = (t & 1) ? __fdiv_rn(127.0f, bsel) : __fdiv_rn(bsel, 127.0f);
    const int base_lane = lane & ~3;
    const float sgv[2] = {__shfl_sync(kFull, qd, base_lane), __shfl_sync(kFull, qd, base_lane | 2)};
    const float invv[2] = {__shfl_sync(kFull, qd, base_lane | 1),
                           __shfl_sync(kFull, qd, base_lane | 3)};
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int row = rr ? r1 : r0;
      if (t == 0) rsig[row] = sgv[rr];
      const float2 inv2 = make_float2(invv[rr], invv[rr]);
#pragma unroll
      for (int h = 0; h < G::NSPAN; ++h) {
        if (!chunk_valid<D>(t)) continue;
        uint32_t w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          // |x| <= 127 (1 + 2^-23) since bmax is the row's max, so x rounds
          // into [-127, 127] without a clamp
          const float2 xa = __fmul2_rn(S[rr][h][2 * u], inv2);
          const float2 xb = __fmul2_rn(S[rr][h][2 * u + 1], inv2);
          const float x0 = xa.x + kRoundMagic, x1 = xa.y + kRoundMagic;
          const float x2 = xb.x + kRoundMagic, x3 = xb.y + kRoundMagic;
          w[u] = __byte_perm(__byte_perm(__float_as_uint(x0), __float_as_uint(x1), 0x0040u),
                             __byte_perm(__float_as_uint(x2), __float_as_uint(x3), 0x0040u),
                             0x5410u);
        }
        *reinterpret_cast<uint4 *>(rec + static_cast<size_t>(row) * D + frag_col(h, t, 0)) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Decode step
// ---------------------------------------------------------------------------

// Bulk copy of a tile's record into a ring slot (one thread); the mbarrier
// is told to expect its bytes but not arrived on.
template <int D, bool BF16, bool KDA>
__device__ __forceinline__ void issue_record(const KParams &p, uint8_t *slot,
                                             unsigned long long *bar, int tile) {
  const uint32_t rec_b = static_cast<uint32_t>(p.L.bytes);
  mbar_expect_tx(bar, rec_b);
  bulk_g2s(slot, p.records + static_cast<size_t>(tile) * rec_b, rec_b, bar);
}

// Bulk copies of the rest of a tile (buffered tokens, inputs) into its ring
// slot, then the arrival that lets the slot's phase complete once every byte
// has landed (one thread).  n < 0: nothing more to copy (skipped tile).
template <int D, bool BF16, bool KDA>
__device__ __forceinline__ void issue_rest(const KParams &p, uint8_t *slot,
                                           unsigned long long *bar, int tile, int n, int coord) {
  using L = SL<D, BF16, KDA>;
  const L lay(p.L.bytes);
  if (n < 0) {
    mbar_arrive_expect_tx(bar, 0);
    return;
  }
  const int b = coord >> 12, hk = (coord >> 1) & 2047;
  const uint32_t bd_b = static_cast<uint32_t>(n) * D * 4;
  const uint32_t bk_b = static_cast<uint32_t>(n) * D * L::IB;
  const uint32_t bg_b = KDA ? bd_b : kGdnGateStride * 4;
  const uint32_t in_b = D * L::IB;
  const uint32_t total = bd_b + bk_b + bg_b + 3 * in_b + (KDA ? static_cast<uint32_t>(D) * 4 : 0u);
  mbar_arrive_expect_tx(bar, total);
  if (n > 0) {
    bulk_g2s(slot + lay.bd, p.buf_d + static_cast<size_t>(tile) * p.W * D, bd_b, bar);
    bulk_g2s(slot + lay.bk,
             static_cast<const uint8_t *>(p.buf_k) +
                 (static_cast<size_t>(b) * p.Hk + hk) * p.W * D * L::IB,
             bk_b, bar);
    if (KDA) bulk_g2s(slot + lay.bg, p.buf_g + static_cast<size_t>(tile) * p.W * D, bg_b, bar);
  }
  if (!KDA) bulk_g2s(slot + lay.bg, p.buf_g + static_cast<size_t>(tile) * kGdnGateStride,
                     bg_b, bar);
  if (p.packed) {
    // the slot holds q | k | v | gate back to back, as the packed inputs do
    const uint32_t pb = 3 * in_b + (KDA ? static_cast<uint32_t>(D) * 4 : 0u);
    bulk_g2s(slot + lay.q, static_cast<const uint8_t *>(p.q) + static_cast<size_t>(tile) * pb, pb,
             bar);
    return;
  }
  const size_t qk = (static_cast<size_t>(b) * p.Hk + hk) * D * L::IB;
  bulk_g2s(slot + lay.q, static_cast<const uint8_t *>(p.q) + qk, in_b, bar);
  bulk_g2s(slot + lay.k, static_cast<const uint8_t *>(p.k) + qk, in_b, bar);
  bulk_g2s(slot + lay.v, static_cast<const uint8_t *>(p.v) + static_cast<size_t>(tile) * in_b,
           in_b, bar);
  if (KDA) bulk_g2s(slot + lay.a, p.alpha + static_cast<size_t>(tile) * D, D * 4, bar);
}

// L2 prefetch of `bytes` at `src` (16-byte aligned, a multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// GDN with bf16 inputs: the buffer coefficients of all slots from one warp.
// Raw dots k_s . k_t and k_s . q_t for slots s = 0..15 run on the bf16 tensor
// path (keys and queries are bf16, so every product is exact; fp32
// accumulation); slot n is the current key itself.  The scalar decay ratios
// rho_s = prod_{s < s' <= n} alpha_{s'} come from a suffix-product scan over
// the lanes (lane s holds alpha_s).  Writes c_s = rho_s (k_s . k_t) and
// a_s = rho_s (k_s . q_t) for s < n, a_n = k_t . q_t, and rho_s for s <= n.
template <int D, class SC>
__device__ __forceinline__ void coef_mma(SC &x, const __nv_bfloat16 *sbk,
                                         const __nv_bfloat16 *sk, const __nv_bfloat16 *sq,
                                         const float *sbg, float alpha0, int n) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  // two independent accumulation chains (even / odd k16 steps), added at the end
  float c[4] = {0.0f, 0.0f, 0.0f, 0.0f}, c2[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  const __nv_bfloat16 *row0 = (g < n) ? sbk + g * D : (g == n ? sk : nullptr);
  const __nv_bfloat16 *row1 = (g + 8 < n) ? sbk + (g + 8) * D : (g + 8 == n ? sk : nullptr);
  const __nv_bfloat16 *vec = (g == 0) ? sk : (g == 1 ? sq : nullptr);
  const uint4 zero = make_uint4(0, 0, 0, 0);
#pragma unroll
  for (int ch = 0; ch < D / 32; ++ch) {
    const int off = 32 * ch + 8 * t;
    const uint4 a0 = row0 ? *reinterpret_cast<const uint4 *>(row0 + off) : zero;
    const uint4 a1 = row1 ? *reinterpret_cast<const uint4 *>(row1 + off) : zero;
    const uint4 bb = vec ? *reinterpret_cast<const uint4 *>(vec + off) : zero;
    mma_bf16(c, a0.x, a1.x, a0.y, a1.y, bb.x, bb.y);
    mma_bf16(c2, a0.z, a1.z, a0.w, a1.w, bb.z, bb.w);
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) c[e] += c2[e];
  float P = (lane < n) ? sbg[lane] : (lane == n ? alpha0 : 1.0f);
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float v = __shfl_down_sync(kFull, P, o);
    if (lane + o < 32) P *= v;
  }
  // lane s now holds prod_{s' >= s} alpha_{s'}; rho_s is lane s+1's value
  const float rho0 = __shfl_sync(kFull, P, (g + 1) & 31);
  const float rho1 = __shfl_sync(kFull, P, (g + 9) & 31);
  if (t == 0) {
    if (g <= n) {
      x.cc[g] = rho0 * c[0];
      x.aa[g] = rho0 * c[1];
      x.rho[g] = rho0;
    }
    if (g + 8 <= n) {
      x.cc[g + 8] = rho1 * c[2];
      x.aa[g + 8] = rho1 * c[3];
      x.rho[g + 8] = rho1;
    }
  }
}

// Four radix-128 int8 digits of u (|u| < 64), packed into the bytes of d.
__device__ __forceinline__ void digits4(float u, uint32_t (&d)[4], int shift) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float biased = u + kRoundMagic;
    d[i] |= (__float_as_uint(biased) & 0xffu) << shift;
    u = (u - (biased - kRoundMagic)) * 128.0f;
  }
}

// Power-of-two factor 2^(6-E) with max|x| = M < 2^E (M > 0), and its inverse
// 2^(E-6); exact.  Tiny M takes the library path.
__device__ __forceinline__ void digit_scales(float M, float &up, float &down) {
  const int eb = static_cast<int>((__float_as_uint(M) >> 23) & 0xffu);
  if (eb >= 6) {
    up = __uint_as_float(static_cast<uint32_t>(259 - eb) << 23);
    down = digit_scale(M);
  } else {
    int E;
    frexpf(M, &E);
    up = ldexpf(1.0f, 6 - E);
    down = ldexpf(1.0f, E - 6);
  }
}

// Window gate of a GDN tile, Gamma_t = alpha_1 ... alpha_t: the n buffered
// gates (a 16-float line in shared memory) and the current one, multiplied
// left to right in registers (every lane the same value).
__device__ __forceinline__ float gate_product(const float *sbg, float alpha0, int n) {
  const float4 *g4 = reinterpret_cast<const float4 *>(sbg);
  float g[kGdnGateStride];
#pragma unroll
  for (int u = 0; u < kGdnGateStride / 4; ++u) {
    const float4 v = g4[u];
    g[4 * u] = v.x;
    g[4 * u + 1] = v.y;
    g[4 * u + 2] = v.z;
    g[4 * u + 3] = v.w;
  }
  float P = 1.0f;
#pragma unroll
  for (int s = 0; s < kGdnGateStride; ++s) {
    const float a = (s < n) ? g[s] : (s == n ? alpha0 : 1.0f);
    P *= a;
  }
  return P;
}

// GDN with bf16 inputs: the row-compensator lines' dot products with
// Gamma o q and Gamma o k over all D key channels, for the lines c = first,
// first + stride, ... (lane l takes channels l, l + 32, ...).  Writes
// cpart[c][0] (q, k); column lines are skipped.
template <int D, class TK>
__device__ __forceinline__ void comp_dots_fast(TK &x, const __nv_bfloat16 *sq,
                                               const __nv_bfloat16 *sk, const float *sbg,
                                               const float *rcv, const int *rcid, float alpha0,
                                               int n, int K, int first, int stride) {
  const int lane = threadIdx.x & 31;
  constexpr int CPL = (D + 31) / 32;
  float gq[CPL], gk[CPL];
  const float Gm = gate_product(sbg, alpha0, n);
#pragma unroll
  for (int u = 0; u < CPL; ++u) {
    const int j = lane + 32 * u;
    gq[u] = j < D ? Gm * __bfloat162float(sq[j]) : 0.0f;
    gk[u] = j < D ? Gm * __bfloat162float(sk[j]) : 0.0f;
  }
  for (int c = first; c < K; c += stride) {
    if (rcid[c] >= D) continue;
    float dq = 0.0f, dk = 0.0f;
#pragma unroll
    for (int u = 0; u < CPL; ++u) {
      const int j = lane + 32 * u;
      const float cv = j < D ? rcv[c * D + j] : 0.0f;
      dq = fmaf(cv, gq[u], dq);
      dk = fmaf(cv, gk[u], dk);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      dq += __shfl_xor_sync(kFull, dq, o);
      dk += __shfl_xor_sync(kFull, dk, o);
    }
    if (lane == 0) {
      x.cpart[c][0][0] = dq;
      x.cpart[c][0][1] = dk;
    }
  }
}

// GDN with bf16 inputs: warp c < 2 * NSPAN does the per-channel work of int8
// MMA k-chunk c, the 32 columns 64h + 16t + 8u + e (h = c / 2, u = c % 2,
// t < 4, e < 8) that the chunk's codes cover; lane l takes t = l / 8, e = l % 8.
// Each chunk's digits get their own power-of-two scale, so the max is a warp
// reduction.  Writes q, k, v (fp32), Gamma, m o Gamma and the chunk's digits
// and scales; warp 0 also appends k_t.
template <int D, class TK>
__device__ __forceinline__ void channel_chunk_fast(const KParams &p, TK &x,
                                                   const __nv_bfloat16 *sq,
                                                   const __nv_bfloat16 *sk,
                                                   const __nv_bfloat16 *sv, const float *sbg,
                                                   const float *rm, const float *rcv,
                                                   const int *rcid, float alpha0, int n,
                                                   size_t key_slot, bool writes_key, int c) {
  const int lane = threadIdx.x & 31;
  const int tq = lane >> 3;
  const int j = 64 * (c >> 1) + 16 * tq + 8 * (c & 1) + (lane & 7);
  const bool valid = D >= 64 || tq < 2;
  const float Gm = gate_product(sbg, alpha0, n);
  float q = 0.0f, k = 0.0f, xq = 0.0f, xk = 0.0f;
  if (valid) {
    q = __bfloat162float(sq[j]);
    k = __bfloat162float(sk[j]);
    const float mj = rm[j];
    x.qf[j] = q;
    x.kf[j] = k;
    x.vf[j] = __bfloat162float(sv[j]);
    x.G[j] = Gm;
    x.mG[padc(j)] = mj * Gm;
    xq = mj * (Gm * q);
    xk = mj * (Gm * k);
    if (writes_key) reinterpret_cast<__nv_bfloat16 *>(p.buf_k)[key_slot + j] = sk[j];
  }
  const float mq = warp_max_abs(xq), mk = warp_max_abs(xk);
  float upq = 0.0f, dnq = 0.0f, upk = 0.0f, dnk = 0.0f;
  if (mq > 0.0f) digit_scales(mq, upq, dnq);
  if (mk > 0.0f) digit_scales(mk, upk, dnk);
  uint32_t dq[4] = {0u, 0u, 0u, 0u}, dk[4] = {0u, 0u, 0u, 0u};
  digits4(xq * upq, dq, 0);
  digits4(xk * upk, dk, 0);
  if (valid) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      x.dig[r][j] = static_cast<int8_t>(dq[r]);
      x.dig[4 + r][j] = static_cast<int8_t>(dk[r]);
    }
  }
  if (lane == 0) {
    x.xscale[0][c] = dnq;
    x.xscale[1][c] = dnk;
  }
}

// ---------------------------------------------------------------------------
// Quad path: plain tokens of d = 128 tiles with bf16 inputs
// ---------------------------------------------------------------------------
//
// Four warps (a quad) take one tile: warp w of the quad does the per-channel
// work of int8 k-chunk w (32 key channels) and then finishes the 32 state rows
// 32w .. 32w + 31 (two m16 row blocks).  One named barrier per tile separates
// the two phases; the per-token values go through a double-buffered QTok.  A
// CTA runs two quads on two tiles at once, so the per-tile fixed costs (waits,
// digit scales, combines, reductions) are spread over four warps instead of
// eight, and no CTA-wide barrier is taken on a plain token.

// Sums NV (32 or 16) per-lane values over the warp: afterwards lane l holds
// the total of value l * NV / 32 (NV - 1 shuffles, and one more for NV = 16).
template <int NV>
__device__ __forceinline__ float warp_transpose_sum(float (&v)[NV], int lane) {
  static_assert(NV == 32 || NV == 16, "32 or 16 values");
  int step = 16;
#pragma unroll
  for (int half = NV / 2; half >= 1; step >>= 1, half >>= 1) {
    const bool upper = (lane & step) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? v[i] : v[i + half];
      const float keep = upper ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(kFull, send, step);
    }
  }
  if (NV == 16) v[0] += __shfl_xor_sync(kFull, v[0], 1);
  return v[0];
}

// Named barrier of one quad (128 threads, barrier id 1 + quad) that also
// returns whether `pred` held in any of its threads.
template <int ID>
__device__ __forceinline__ bool bar_any_128(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "n"(ID)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ bool quad_bar_any(int quad, bool pred) {
  return quad == 0 ? bar_any_128<1>(pred) : bar_any_128<2>(pred);
}

// Phase 1 of a quad tile, warp w (0..3) of the quad: k-chunk w's channels
// 64(w/2) + 16(l/8) + 8(w%2) + l%8 for lane l.  Computes the window gate
// Gamma (GDN: the scalar product of the gates; KDA: per channel, together with
// this chunk's share of the buffer coefficients c_s = sum_j k_sj rho_sj k_j,
// a_s = sum_j k_sj rho_sj q_j, rho_sj = prod_{s < s' <= n} alpha_s'j, and a_n =
// k . q), x = m o Gamma o {q, k} and its digits under the chunk's own scale,
// the row-compensator dots and the column-compensator values; warp 0 gets the
// GDN coefficients from the bf16 tensor path.  Appends k_t (the key head's
// first value head) and the gate when `ok` (the slot's copies arrived).
template <int D, bool KDA>
__device__ __forceinline__ void quad_channel(const KParams &p, QTok<D> &x, const uint8_t *slot,
                                             int tile, int n, int coord, float alpha0, int w,
                                             bool ok) {
  using L = SL<D, true, KDA>;
  const L lay(p.L.bytes);
  const int lane = threadIdx.x & 31;
  const int j = 64 * (w >> 1) + 16 * (lane >> 3) + 8 * (w & 1) + (lane & 7);
  const float *rm = reinterpret_cast<const float *>(slot + p.L.off_m);
  const float *rcv = reinterpret_cast<const float *>(slot + p.L.off_cv);
  const int *rcid = reinterpret_cast<const int *>(slot + p.L.off_cid);
  const __nv_bfloat16 *sbk = reinterpret_cast<const __nv_bfloat16 *>(slot + lay.bk);
  const float *sbg = reinterpret_cast<const float *>(slot + lay.bg);
  const __nv_bfloat16 *sq = reinterpret_cast<const __nv_bfloat16 *>(slot + lay.q);
  const __nv_bfloat16 *sk = reinterpret_cast<const __nv_bfloat16 *>(slot + lay.k);
  const float q = __bfloat162float(sq[j]), k = __bfloat162float(sk[j]);
  float G;
  if constexpr (KDA) {
    const float *sa = reinterpret_cast<const float *>(slot + lay.a);
    // This lane's share of c_s (s < n) and a_s (s <= n, a_n = k . q), summed
    // over the chunk by one transposed reduction: of 16 values while n < 8
    // (c_0..7, a_0..7), of 32 otherwise.
    float rho = sa[j];
    if (n < 8) {
      float v[16];
#pragma unroll
      for (int s2 = 7; s2 >= 0; --s2) {
        if (s2 < n) {
          const float kr = __bfloat162float(sbk[s2 * D + j]) * rho;
          v[s2] = kr * k;
          v[8 + s2] = kr * q;
          rho *= sbg[s2 * D + j];
        } else {
          v[s2] = 0.0f;
          v[8 + s2] = (s2 == n) ? k * q : 0.0f;
        }
      }
      const float tot = warp_transpose_sum<16>(v, lane);
      const int vi = lane >> 1;
      if ((lane & 1) == 0) x.cpk[w][vi < 8 ? vi : 8 + vi] = tot;
    } else {
      float v[32];
#pragma unroll
      for (int s2 = kMaxWindow - 1; s2 >= 0; --s2) {
        if (s2 < n) {
          const float kr = __bfloat162float(sbk[s2 * D + j]) * rho;
          v[s2] = kr * k;
          v[16 + s2] = kr * q;
          rho *= sbg[s2 * D + j];
        } else {
          v[s2] = 0.0f;
          v[16 + s2] = (s2 == n) ? k * q : 0.0f;
        }
      }
      x.cpk[w][lane] = warp_transpose_sum<32>(v, lane);
    }
    G = rho;
  } else {
    // Gamma = the product of the n buffered gates and the current one: lane s
    // holds gate s (1 past n), multiplied over the warp by a butterfly whose
    // pairs are the same in every lane, so every lane gets the same bits
    float a = lane < n ? sbg[lane] : (lane == n ? alpha0 : 1.0f);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a *= __shfl_xor_sync(kFull, a, o);
    G = a;
    if (w == 0)
      coef_mma<D>(x, sbk, sk, sq, sbg, alpha0, n);
  }
  const float mj = rm[j];
  const float gq = G * q, gk = G * k;
  const float xq = mj * gq, xk = mj * gk;
  const float mq = warp_max_abs(xq), mk = warp_max_abs(xk);
  float upq = 0.0f, dnq = 0.0f, upk = 0.0f, dnk = 0.0f;
  if (mq > 0.0f) digit_scales(mq, upq, dnq);
  if (mk > 0.0f) digit_scales(mk, upk, dnk);
  uint32_t dq[4] = {0u, 0u, 0u, 0u}, dk[4] = {0u, 0u, 0u, 0u};
  digits4(xq * upq, dq, 0);
  digits4(xk * upk, dk, 0);
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    x.dig[r][j] = static_cast<int8_t>(dq[r]);
    x.dig[4 + r][j] = static_cast<int8_t>(dk[r]);
  }
  if (lane == 0) {
    x.xscale[0][w] = dnq;
    x.xscale[1][w] = dnk;
  }
  // row-compensator lines: this chunk's share of their dots with Gamma o q and
  // Gamma o k, four lines per transposed reduction; column lines: the owner
  // lane of the column records Gamma_j q_j and Gamma_j k_j
  for (int c0 = 0; c0 < p.K; c0 += 4) {
    float vv[8];
#pragma unroll
    for (int i2 = 0; i2 < 4; ++i2) {
      const int c = c0 + i2;
      const float cvj = (c < p.K && rcid[c] < D) ? rcv[c * D + j] : 0.0f;
      vv[2 * i2] = cvj * gq;
      vv[2 * i2 + 1] = cvj * gk;
    }
    const float tot = warp_sum8(vv, lane);
    const int vi = (lane >> 2) & 7, c = c0 + (vi >> 1);
    if ((lane & 3) == 0 && c < p.K) x.cpart[c][w][vi & 1] = tot;
  }
  for (int c = 0; c < p.K; ++c) {
    if (rcid[c] == D + j) {
      x.colv[c][0] = gq;
      x.colv[c][1] = gk;
    }
  }
  if (ok) {
    const int b = coord >> 12, hk = (coord >> 1) & 2047;
    if ((coord & 1) != 0)
      reinterpret_cast<__nv_bfloat16 *>(p.buf_k)[((static_cast<size_t>(b) * p.Hk + hk) * p.W + n) *
                                                     D + j] = sk[j];
    if constexpr (KDA) {
      const float *sa = reinterpret_cast<const float *>(slot + lay.a);
      p.buf_g[(static_cast<size_t>(tile) * p.W + n) * D + j] = sa[j];
    } else {
      if (w == 0 && lane == 0) p.buf_g[static_cast<size_t>(tile) * kGdnGateStride + n] = alpha0;
    }
  }
}

// What phase 2 of a quad tile needs from the ring slot, held in registers so
// that the slot can be refilled before the rows are computed.  Lane (g, t) of
// warp w owns rows 32w + 16rb + g and + 8 (rb = 0, 1), the buffer slots
// t, t + 4, ... of them, and the compensator lines t and t + 4.
struct QRegs {
  uint4 A[2][2][2];      // codes: [rb][row r0 / r1][64-column span]
  float sig[2][2];       // sigma at the rows
  float v[2];            // v at the row this lane finishes (t < 2), per rb
  float d[4][2][2];      // d_s at the rows for s = t + 4u: [u][rb][r0 / r1]
  int cid[2];            // ids of lines t and t + 4 (D2 + 1 past K)
  float cval[2][2][2];   // those lines' values at the rows (column lines)
};

// Loads the QRegs of warp w for a tile with n buffered tokens from its slot.
template <int D, bool KDA>
__device__ __forceinline__ void quad_rows_load(const KParams &p, const uint8_t *slot, int n, int w,
                                               QRegs &r) {
  using L = SL<D, true, KDA>;
  const L lay(p.L.bytes);
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const float *rsig = reinterpret_cast<const float *>(slot + p.L.off_sig);
  const float *rcv = reinterpret_cast<const float *>(slot + p.L.off_cv);
  const int *rcid = reinterpret_cast<const int *>(slot + p.L.off_cid);
  const float *sbd = reinterpret_cast<const float *>(slot + lay.bd);
  const __nv_bfloat16 *sv = reinterpret_cast<const __nv_bfloat16 *>(slot + lay.v);
#pragma unroll
  for (int rb = 0; rb < 2; ++rb) {
    const int r0 = 32 * w + 16 * rb + g, r1 = r0 + 8;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      r.A[rb][0][h] = *reinterpret_cast<const uint4 *>(slot + r0 * D + frag_col(h, t, 0));
      r.A[rb][1][h] = *reinterpret_cast<const uint4 *>(slot + r1 * D + frag_col(h, t, 0));
    }
    r.sig[rb][0] = rsig[r0];
    r.sig[rb][1] = rsig[r1];
    r.v[rb] = __bfloat162float(sv[t ? r1 : r0]);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int s2 = t + 4 * u;
      r.d[u][rb][0] = s2 < n ? sbd[s2 * D + r0] : 0.0f;
      r.d[u][rb][1] = s2 < n ? sbd[s2 * D + r1] : 0.0f;
    }
  }
#pragma unroll
  for (int li = 0; li < 2; ++li) {
    const int c = t + 4 * li;
    const int id = c < p.K ? rcid[c] : 2 * D + 1;
    r.cid[li] = id;
    const bool col = id >= D && id < 2 * D;
#pragma unroll
    for (int rb = 0; rb < 2; ++rb) {
      const int r0 = 32 * w + 16 * rb + g;
      r.cval[li][rb][0] = col ? rcv[c * D + r0] : 0.0f;
      r.cval[li][rb][1] = col ? rcv[c * D + r0 + 8] : 0.0f;
    }
  }
}

// Row-phase operands as quad_rows reads them: from registers loaded before
// the slot was released (RegRows), or from the slot when they are used
// (SlotRows, for a ring whose other slots already overlap the copies with the
// rows and where holding them all would cost registers).
struct RegRows {
  QRegs r;
  __device__ __forceinline__ uint4 A(int rb, int rr, int h) const { return r.A[rb][rr][h]; }
  __device__ __forceinline__ float sig(int rb, int rr) const { return r.sig[rb][rr]; }
  __device__ __forceinline__ float v(int rb) const { return r.v[rb]; }
  __device__ __forceinline__ float d(int u, int rb, int rr) const { return r.d[u][rb][rr]; }
  __device__ __forceinline__ int cid(int li) const { return r.cid[li]; }
  __device__ __forceinline__ float cval(int li, int rb, int rr) const { return r.cval[li][rb][rr]; }
};

template <int D, bool KDA>
struct SlotRows {
  const uint8_t *slot;
  const float *rsig, *rcv, *sbd;
  const int *rcid;
  const __nv_bfloat16 *sv;
  int n, K, row0, t;
  __device__ __forceinline__ SlotRows(const KParams &p, const uint8_t *slot_, int n_, int w) {
    using L = SL<D, true, KDA>;
    const L lay(p.L.bytes);
    const int lane = threadIdx.x & 31;
    slot = slot_;
    rsig = reinterpret_cast<const float *>(slot + p.L.off_sig);
    rcv = reinterpret_cast<const float *>(slot + p.L.off_cv);
    rcid = reinterpret_cast<const int *>(slot + p.L.off_cid);
    sbd = reinterpret_cast<const float *>(slot + lay.bd);
    sv = reinterpret_cast<const __nv_bfloat16 *>(slot + lay.v);
    n = n_;
    K = p.K;
    row0 = 32 * w + (lane >> 2);
    t = lane & 3;
  }
  __device__ __forceinline__ int row(int rb, int rr) const { return row0 + 16 * rb + 8 * rr; }
  __device__ __forceinline__ uint4 A(int rb, int rr, int h) const {
    return *reinterpret_cast<const uint4 *>(slot + row(rb, rr) * D + frag_col(h, t, 0));
  }
  __device__ __forceinline__ float sig(int rb, int rr) const { return rsig[row(rb, rr)]; }
  __device__ __forceinline__ float v(int rb) const {
    return __bfloat162float(sv[row(rb, t ? 1 : 0)]);
  }
  __device__ __forceinline__ float d(int u, int rb, int rr) const {
    const int s2 = t + 4 * u;
    return s2 < n ? sbd[s2 * D + row(rb, rr)] : 0.0f;
  }
  __device__ __forceinline__ int cid(int li) const {
    const int c = t + 4 * li;
    return c < K ? rcid[c] : 2 * D + 1;
  }
  __device__ __forceinline__ float cval(int li, int rb, int rr) const {
    const int c = t + 4 * li, id = cid(li);
    return (id >= D && id < 2 * D) ? rcv[c * D + row(rb, rr)] : 0.0f;
  }
};

// Phase 2 of a quad tile, warp w: rows 32w .. 32w + 31 as two m16 row blocks,
// from the QRegs and the quad's QTok only (the slot may already be refilled).
// y_q, y_k on the int8 tensor path with the four chunk scales, then the
// buffer sums (lane t of a row takes slots t, t + 4, ...), the compensator
// lines (lane t takes lines t and t + 4), d_t = beta (v - y_k - sum c_s d_s),
// o_t = y_q + sum a_s d_s + a_n d_t, the output and the append of d_t.
template <int D, bool KDA, class Src>
__device__ __forceinline__ void quad_rows(const KParams &p, const QTok<D> &x, const Src &r,
                                          int tile, int n, float beta, int w) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  // the coefficients of this lane's buffer slots s = t + 4u; KDA: lane l sums
  // the four warps' partials of value l (c_l for l < 16, a_(l-16) above) once,
  // and the lanes that need a value take it by shuffle
  float cs[4], as[4], ann;
  if constexpr (KDA) {
    const float tot = (x.cpk[0][lane] + x.cpk[1][lane]) + (x.cpk[2][lane] + x.cpk[3][lane]);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int s2 = t + 4 * u;
      const float c = __shfl_sync(kFull, tot, s2), a = __shfl_sync(kFull, tot, 16 + s2);
      cs[u] = s2 < n ? c : 0.0f;
      as[u] = s2 < n ? a : 0.0f;
    }
    ann = __shfl_sync(kFull, tot, 16 + n);
  } else {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int s2 = t + 4 * u;
      cs[u] = s2 < n ? x.cc[s2] : 0.0f;
      as[u] = s2 < n ? x.aa[s2] : 0.0f;
    }
    ann = x.aa[n];
  }
  // this lane's compensator lines: column lines scale their values at the rows
  // by Gamma_j x_j; a row line adds its dots to the one row it is
  float cq[2], ck[2], rq[2], rk[2];
#pragma unroll
  for (int li = 0; li < 2; ++li) {
    const int c = t + 4 * li, id = r.cid(li);
    cq[li] = ck[li] = rq[li] = rk[li] = 0.0f;
    if (id < D) {
      if ((id >> 5) == w) {
        rq[li] = (x.cpart[c][0][0] + x.cpart[c][1][0]) + (x.cpart[c][2][0] + x.cpart[c][3][0]);
        rk[li] = (x.cpart[c][0][1] + x.cpart[c][1][1]) + (x.cpart[c][2][1] + x.cpart[c][3][1]);
      }
    } else if (id < 2 * D) {
      cq[li] = x.colv[c][0];
      ck[li] = x.colv[c][1];
    }
  }
  uint4 Bw[2];
#pragma unroll
  for (int hh = 0; hh < 2; ++hh)
    Bw[hh] = *reinterpret_cast<const uint4 *>(&x.dig[g][frag_col(hh, t, 0)]);
  const float pair = (t & 1) ? 1.0f / (128.0f * 16384.0f) : 1.0f / 128.0f;
  float sc[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) sc[c] = x.xscale[t >> 1][c] * pair;
  const int base_lane = lane & ~3;
#pragma unroll
  for (int rb = 0; rb < 2; ++rb) {
    const int r0 = 32 * w + 16 * rb + g, r1 = r0 + 8;
    int acc[4][4];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const uint4 a0 = r.A(rb, 0, hh), a1 = r.A(rb, 1, hh);
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[2 * hh][e] = acc[2 * hh + 1][e] = 0;
      mma_s8(acc[2 * hh], a0.x, a1.x, a0.y, a1.y, Bw[hh].x, Bw[hh].y);
      mma_s8(acc[2 * hh + 1], a0.z, a1.z, a0.w, a1.w, Bw[hh].z, Bw[hh].w);
    }
    float p0 = 0.0f, p1 = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      p0 = fmaf(sc[c], static_cast<float>(acc[c][0] * 128 + acc[c][1]), p0);
      p1 = fmaf(sc[c], static_cast<float>(acc[c][2] * 128 + acc[c][3]), p1);
    }
    p0 += __shfl_xor_sync(kFull, p0, 1);
    p1 += __shfl_xor_sync(kFull, p1, 1);
    const float yq0 = __shfl_sync(kFull, p0, base_lane) * r.sig(rb, 0);
    const float yq1 = __shfl_sync(kFull, p1, base_lane) * r.sig(rb, 1);
    const float yk0 = __shfl_sync(kFull, p0, base_lane | 2) * r.sig(rb, 0);
    const float yk1 = __shfl_sync(kFull, p1, base_lane | 2) * r.sig(rb, 1);
    float xc0 = 0.0f, xa0 = 0.0f, xc1 = 0.0f, xa1 = 0.0f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float d0 = r.d(u, rb, 0), d1 = r.d(u, rb, 1);
      xc0 = fmaf(cs[u], d0, xc0);
      xa0 = fmaf(as[u], d0, xa0);
      xc1 = fmaf(cs[u], d1, xc1);
      xa1 = fmaf(as[u], d1, xa1);
    }
#pragma unroll
    for (int li = 0; li < 2; ++li) {
      const float v0 = r.cval(li, rb, 0), v1 = r.cval(li, rb, 1);
      xa0 = fmaf(v0, cq[li], xa0);
      xc0 = fmaf(v0, ck[li], xc0);
      xa1 = fmaf(v1, cq[li], xa1);
      xc1 = fmaf(v1, ck[li], xc1);
      const int id = r.cid(li);
      if (id == r0) {
        xa0 += rq[li];
        xc0 += rk[li];
      } else if (id == r1) {
        xa1 += rq[li];
        xc1 += rk[li];
      }
    }
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      xc0 += __shfl_xor_sync(kFull, xc0, o);
      xa0 += __shfl_xor_sync(kFull, xa0, o);
      xc1 += __shfl_xor_sync(kFull, xc1, o);
      xa1 += __shfl_xor_sync(kFull, xa1, o);
    }
    if (t < 2) {
      const int row = t ? r1 : r0;
      const float yq = t ? yq1 : yq0, yk = t ? yk1 : yk0;
      const float xc = t ? xc1 : xc0, xa = t ? xa1 : xa0;
      const float dt = beta * (r.v(rb) - yk - xc);
      const float o = fmaf(ann, dt, yq + xa);
      st_out(p.out, static_cast<size_t>(tile) * D + row, o, p.out_bf16);
      p.buf_d[(static_cast<size_t>(tile) * p.W + n) * D + row] = dt;
    }
  }
}

// One token for one staged tile: outputs, buffer append, and on the W-th token
// the fold and requantization.
// GDN with bf16 inputs (one CTA barrier; returns false if the CTA aborts):
//  A  warp c < 2 NSPAN: k-chunk c's channels (gate product, x, chunk max,
//     digits and scale); warp 2 NSPAN: the buffer coefficients c_s, a_s (bf16
//     MMA); the other warps: their code fragments, then the row-compensator
//     dots.  Then the barrier, after which the caller's refill runs.
// General path (KDA, fp32 inputs), phases separated by CTA barriers:
//  A  channel threads (one per key channel j): inputs, decay ratios applied to
//     the buffered keys, Gamma, x = m o Gamma o {q, k} and its per-warp max;
//     appends k_t and the KDA gate.  The other warps fetch their code
//     fragments.
//  B  channel threads: the int8 digits of x_q, x_k and the row-compensator
//     dots; the other warps: the buffer coefficients c_s, a_s.
// Both then run
//  C  every row warp: y_q, y_k for its 16 rows on the int8 tensor path, then
//     finishes its rows (buffer sums split over the 4 lanes of a row):
//     d_t = beta (v - y_k - sum c_s d_s), o_t = y_q + sum a_s d_s + a_t d_t.
template <int D, bool BF16, bool KDA, int WM, class SC, class Refill>
__device__ __forceinline__ bool process_tile(const KParams &p, SC &s, Tok<D, WM> &x, uint8_t *slot,
                                             int tile, int n, int coord, float alpha0,
                                             float beta, Refill &&refill) {
  using G = FG<D>;
  using L = SL<D, BF16, KDA, WM>;
  using IT = in_t<BF16>;
  constexpr int CW = (D + 31) / 32;  // channel warps
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int b = coord >> 12, hk = (coord >> 1) & 2047;
  const bool writes_key = (coord & 1) != 0;
  const uint8_t *codes = slot;
  const float *rsig = reinterpret_cast<const float *>(slot + p.L.off_sig);
  const float *rm = reinterpret_cast<const float *>(slot + p.L.off_m);
  const float *rcv = reinterpret_cast<const float *>(slot + p.L.off_cv);
  const int *rcid = reinterpret_cast<const int *>(slot + p.L.off_cid);
  const L lay(p.L.bytes);
  float *sbd = reinterpret_cast<float *>(slot + lay.bd);
  const IT *sbk = reinterpret_cast<const IT *>(slot + lay.bk);
  const float *sbg = reinterpret_cast<const float *>(slot + lay.bg);
  const IT *sq = reinterpret_cast<const IT *>(slot + lay.q);
  const IT *sk = reinterpret_cast<const IT *>(slot + lay.k);
  const IT *sv = reinterpret_cast<const IT *>(slot + lay.v);
  const float *sa = reinterpret_cast<const float *>(slot + lay.a);

  // ---- Phases A and B ----
  constexpr bool kFast = DecodeTraits<D, BF16, KDA, WM>::kFast;
  constexpr bool kMmaF = DecodeTraits<D, BF16, KDA, WM>::kMmaFold;
  constexpr int NCH = 2 * G::NSPAN;    // int8 MMA k-chunks (GDN-bf16: one channel warp each)
  constexpr int CWP = kFast ? 1 : CW;  // warps holding compensator partial dots
  uint4 A[2][G::NSPAN];
  if constexpr (kFast) {
    // one warp per k-chunk for the channels, one for the buffer coefficients,
    // the others for the row-compensator dot products
    if (warp < NCH) {
      if (warp < G::NRB) load_codes<D>(codes, A);
      channel_chunk_fast<D>(p, x, reinterpret_cast<const __nv_bfloat16 *>(sq),
                            reinterpret_cast<const __nv_bfloat16 *>(sk),
                            reinterpret_cast<const __nv_bfloat16 *>(sv), sbg, rm, rcv, rcid,
                            alpha0, n,
                            ((static_cast<size_t>(b) * p.Hk + hk) * p.W + n) * D, writes_key,
                            warp);
      if (tid == 0) p.buf_g[static_cast<size_t>(tile) * p.gstride + n] = alpha0;
    } else if (warp == NCH) {
      coef_mma<D>(x, reinterpret_cast<const __nv_bfloat16 *>(sbk),
                  reinterpret_cast<const __nv_bfloat16 *>(sk),
                  reinterpret_cast<const __nv_bfloat16 *>(sq), sbg, alpha0, n);
    } else {
      // the remaining warps fetch their code fragments, then share out the
      // row-compensator lines' dot products
      if (warp < G::NRB) load_codes<D>(codes, A);
      comp_dots_fast<D>(x, reinterpret_cast<const __nv_bfloat16 *>(sq),
                        reinterpret_cast<const __nv_bfloat16 *>(sk), sbg, rcv, rcid, alpha0, n,
                        p.K, warp - NCH - 1, kWarps - NCH - 1);
    }
    // the one CTA barrier of a plain token: the copies of this tile have
    // landed for every thread, and the previous tile's slot is free
    __syncthreads();
    if (s.abort) return false;
    refill();
  } else {
    // ---- Phase A ----
  float xq = 0.0f, xk = 0.0f;
  if (tid < D) {
    const int j = tid;
    const float qj = to_f(sq[j]), kj = to_f(sk[j]);
    x.qf[j] = qj;
    x.kf[j] = kj;
    x.vf[j] = to_f(sv[j]);
    float acc;
    if constexpr (kFast) {
      // window gate Gamma_t = prod of the n buffered gates and the current one
      float P = (lane < n) ? sbg[lane] : (lane == n ? alpha0 : 1.0f);
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) P *= __shfl_xor_sync(kFull, P, o);
      acc = P;
    } else {
      // decay ratios prod_{s < s' <= t} alpha_{s'} as running products from
      // the current token backwards, applied to the buffered keys
      acc = KDA ? sa[j] : alpha0;
      for (int sl = n - 1; sl >= 0; --sl) {
        (&s.kt[0][0])[kt_index<D, kMmaF>(sl, j)] = to_f(sbk[sl * D + j]) * acc;
        acc *= KDA ? sbg[sl * D + j] : sbg[sl];
      }
      (&s.kt[0][0])[kt_index<D, kMmaF>(n, j)] = kj;
    }
    x.G[j] = acc;
    const float mj = rm[j];
    xq = mj * (acc * qj);
    xk = mj * (acc * kj);
    x.mG[padc(j)] = mj * acc;
    if (writes_key)
      reinterpret_cast<IT *>(p.buf_k)[((static_cast<size_t>(b) * p.Hk + hk) * p.W + n) * D + j] =
          sk[j];
    if constexpr (KDA) p.buf_g[(static_cast<size_t>(tile) * p.W + n) * D + j] = sa[j];
    const float mq = warp_max_abs(xq), mk = warp_max_abs(xk);
    if (lane == 0) {
      x.xmax[0][warp] = mq;
      x.xmax[1][warp] = mk;
    }
    // row-compensator lines dotted with Gamma o q and Gamma o k: per-warp
    // partials, four lines per transposed reduction
    const float gq = acc * qj, gk = acc * kj;
    for (int c0 = 0; c0 < p.K; c0 += 4) {
      float v[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = c0 + i;
        const float cvj = (c < p.K && rcid[c] < D) ? rcv[c * D + j] : 0.0f;
        v[2 * i] = cvj * gq;
        v[2 * i + 1] = cvj * gk;
      }
      const float tot = warp_sum8(v, lane);
      const int vi = (lane >> 2) & 7, c = c0 + (vi >> 1);
      if ((lane & 3) == 0 && c < p.K) x.cpart[c][warp][vi & 1] = tot;
    }
  } else if (warp < G::NRB) {
    load_codes<D>(codes, A);
  }
  if constexpr (kFast) {
    if (warp == CW) coef_mma<D>(x, reinterpret_cast<const __nv_bfloat16 *>(sbk),
                                reinterpret_cast<const __nv_bfloat16 *>(sk),
                                reinterpret_cast<const __nv_bfloat16 *>(sq), sbg, alpha0, n);
  }
  if constexpr (!KDA) {
    if (tid == 0) p.buf_g[static_cast<size_t>(tile) * p.gstride + n] = alpha0;
  }
  __syncthreads();

  // ---- Phase B ----
  if (tid < D) {
    float Mq = 0.0f, Mk = 0.0f;
#pragma unroll
    for (int w = 0; w < CW; ++w) {
      Mq = fmaxf(Mq, x.xmax[0][w]);
      Mk = fmaxf(Mk, x.xmax[1][w]);
    }
    split_digits(xq, Mq, &x.dig[0][tid], G::DIGW);
    split_digits(xk, Mk, &x.dig[4][tid], G::DIGW);
    if (tid == 0) {
      x.xscale[0][0] = digit_scale(Mq);
      x.xscale[1][0] = digit_scale(Mk);
    }
  } else if constexpr (!kFast) {
    // c_s = kt_s . k and a_s = kt_s . q for the buffered tokens; a_t = k . q
    for (int sl = warp - CW; sl <= n; sl += kWarps - CW) {
      float c = 0.0f, a = 0.0f;
      for (int j = lane; j < D; j += 32) {
        const float kv = (&s.kt[0][0])[kt_index<D, kMmaF>(sl, j)];
        c = fmaf(kv, x.kf[j], c);
        a = fmaf(kv, x.qf[j], a);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        c += __shfl_xor_sync(kFull, c, o);
        a += __shfl_xor_sync(kFull, a, o);
      }
      if (lane == 0) {
        x.cc[sl] = c;
        x.aa[sl] = a;
      }
    }
  }
  __syncthreads();

  }

  // ---- Phase C ----
  if (warp < G::NRB) {
    if (kFast ? warp == NCH : tid < D) load_codes<D>(codes, A);
    // lane (g, t) holds digits 2t, 2t+1 of rows r0 (acc 0,1) and r0+8 (acc 2,3);
    // t = 0,1: x_q digits 0-1, 2-3; t = 2,3: x_k digits 0-1, 2-3.
    float p0, p1, sq0, sk0;
    if constexpr (kFast) {
      // one accumulator per k-chunk, each with its own digit scale
      int acc[NCH][4];
#pragma unroll
      for (int hh = 0; hh < G::NSPAN; ++hh) {
        uint4 Bw = make_uint4(0, 0, 0, 0);
        if (chunk_valid<D>(t))
          Bw = *reinterpret_cast<const uint4 *>(&x.dig[g][frag_col(hh, t, 0)]);
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[2 * hh][e] = acc[2 * hh + 1][e] = 0;
        mma_s8(acc[2 * hh], A[0][hh].x, A[1][hh].x, A[0][hh].y, A[1][hh].y, Bw.x, Bw.y);
        mma_s8(acc[2 * hh + 1], A[0][hh].z, A[1][hh].z, A[0][hh].w, A[1][hh].w, Bw.z, Bw.w);
      }
      // digits 2t, 2t+1 combine exactly as one integer (|.| < 2^26) before
      // the chunk scale applies
      const float pair = (t & 1) ? 1.0f / (128.0f * 16384.0f) : 1.0f / 128.0f;
      p0 = 0.0f;
      p1 = 0.0f;
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        const float sc = x.xscale[t >> 1][c] * pair;
        p0 = fmaf(sc, static_cast<float>(acc[c][0] * 128 + acc[c][1]), p0);
        p1 = fmaf(sc, static_cast<float>(acc[c][2] * 128 + acc[c][3]), p1);
      }
      sq0 = 1.0f;
      sk0 = 1.0f;
    } else {
      int acc[4] = {0, 0, 0, 0};
#pragma unroll
      for (int hh = 0; hh < G::NSPAN; ++hh) {
        uint4 Bw = make_uint4(0, 0, 0, 0);
        if (chunk_valid<D>(t))
          Bw = *reinterpret_cast<const uint4 *>(&x.dig[g][frag_col(hh, t, 0)]);
        mma_s8(acc, A[0][hh].x, A[1][hh].x, A[0][hh].y, A[1][hh].y, Bw.x, Bw.y);
        mma_s8(acc, A[0][hh].z, A[1][hh].z, A[0][hh].w, A[1][hh].w, Bw.z, Bw.w);
      }
      p0 = static_cast<float>(acc[0]) + static_cast<float>(acc[1]) * (1.0f / 128.0f);
      p1 = static_cast<float>(acc[2]) + static_cast<float>(acc[3]) * (1.0f / 128.0f);
      if (t & 1) {
        p0 *= 1.0f / 16384.0f;
        p1 *= 1.0f / 16384.0f;
      }
      sq0 = x.xscale[0][0];
      sk0 = x.xscale[1][0];
    }
    p0 += __shfl_xor_sync(kFull, p0, 1);
    p1 += __shfl_xor_sync(kFull, p1, 1);
    const int r0 = 16 * warp + g, r1 = r0 + 8;
    const int base_lane = lane & ~3;
    float yq0 = __shfl_sync(kFull, p0, base_lane) * sq0 * rsig[r0];
    float yq1 = __shfl_sync(kFull, p1, base_lane) * sq0 * rsig[r1];
    float yk0 = __shfl_sync(kFull, p0, base_lane | 2) * sk0 * rsig[r0];
    float yk1 = __shfl_sync(kFull, p1, base_lane | 2) * sk0 * rsig[r1];
    // buffer sums and compensator lines, split over the 4 lanes of the rows:
    // xa collects what adds to o, xc what is subtracted from v
    float xc0 = 0.0f, xa0 = 0.0f, xc1 = 0.0f, xa1 = 0.0f;
    for (int sl = t; sl < n; sl += 4) {
      const float c = x.cc[sl], a = x.aa[sl];
      const float d0 = sbd[sl * D + r0], d1 = sbd[sl * D + r1];
      xc0 = fmaf(c, d0, xc0);
      xa0 = fmaf(a, d0, xa0);
      xc1 = fmaf(c, d1, xc1);
      xa1 = fmaf(a, d1, xa1);
    }
    for (int c = t; c < p.K; c += 4) {
      const int id = rcid[c];
      if (id < D) {
        if (id == r0 || id == r1) {
          float dq = 0.0f, dk = 0.0f;
#pragma unroll
          for (int w = 0; w < CWP; ++w) {
            dq += x.cpart[c][w][0];
            dk += x.cpart[c][w][1];
          }
          if (id == r0) {
            xa0 += dq;
            xc0 += dk;
          } else {
            xa1 += dq;
            xc1 += dk;
          }
        }
      } else {
        const int jc = id - D;
        const float gj = x.G[jc];
        const float gq = gj * x.qf[jc], gk = gj * x.kf[jc];
        const float c0 = rcv[c * D + r0], c1 = rcv[c * D + r1];
        xa0 = fmaf(c0, gq, xa0);
        xc0 = fmaf(c0, gk, xc0);
        xa1 = fmaf(c1, gq, xa1);
        xc1 = fmaf(c1, gk, xc1);
      }
    }
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      xc0 += __shfl_xor_sync(kFull, xc0, o);
      xa0 += __shfl_xor_sync(kFull, xa0, o);
      xc1 += __shfl_xor_sync(kFull, xc1, o);
      xa1 += __shfl_xor_sync(kFull, xa1, o);
    }
    if (t < 2) {
      const int row = t ? r1 : r0;
      const float yq = t ? yq1 : yq0, yk = t ? yk1 : yk0;
      const float xc = t ? xc1 : xc0, xa = t ? xa1 : xa0;
      const float dt = beta * (x.vf[row] - yk - xc);
      const float o = fmaf(x.aa[n], dt, yq + xa);
      st_out(p.out, static_cast<size_t>(tile) * D + row, o, p.out_bf16);
      p.buf_d[(static_cast<size_t>(tile) * p.W + n) * D + row] = dt;
      sbd[n * D + row] = dt;
    }
  }
  if (n + 1 < p.W) {
    if (tid == 0) p.buf_n[tile] = n + 1;
    return true;
  }

  // Window boundary: fold the W buffered tokens and requantize.  A warp reads
  // back only its own rows' d_t, written above by lanes of the same warp; the
  // barriers below keep the codes and keys from being overwritten while
  // another warp still needs them.
  __syncwarp();
  float2 S[2][G::NSPAN][8];
  uint4 Af[2][G::NSPAN];
  if (warp < G::NRB) load_codes<D>(codes, Af);
  const float *kt;
  if constexpr (DecodeTraits<D, BF16, KDA, WM>::kFast) {
    // scaled keys from the staged keys and the scalar ratios; at d = 128 they
    // go over the staged codes, which are now in registers
    float *ktw;
    if constexpr (DecodeTraits<D, BF16, KDA, WM>::kKtOverCodes) {
      __syncthreads();
      ktw = reinterpret_cast<float *>(slot);
    } else {
      ktw = &s.kt[0][0];
    }
    if (tid < D) {
      if constexpr (DecodeTraits<D, BF16, KDA, WM>::kMmaFold) {
        constexpr int P = kt_mma_stride<D>();
        const int pos = kt_mma_pos(tid);
        for (int sl = 0; sl < n; ++sl)
          ktw[sl * P + pos] = to_f(sbk[sl * D + tid]) * x.rho[sl];
        ktw[n * P + pos] = x.kf[tid];
      } else {
        for (int sl = 0; sl < n; ++sl)
          ktw[sl * G::PADW + padc(tid)] = to_f(sbk[sl * D + tid]) * x.rho[sl];
        ktw[n * G::PADW + padc(tid)] = x.kf[tid];
      }
    }
    __syncthreads();
    kt = ktw;
  } else {
    kt = &s.kt[0][0];
  }
  if (warp < G::NRB)
    build_state<D, DecodeTraits<D, BF16, KDA, WM>::kMmaFold, WM>(x, kt, Af, rsig, rcv, rcid, sbd, n + 1,
                                                        p.K, S);
  __syncthreads();  // the staged codes and keys are now free for the quantizer's scratch
  quantize_tile<D>(s, reinterpret_cast<double *>(slot + L::QS_COLPART),
                   reinterpret_cast<float *>(slot + L::QS_COLMAX), S,
                   p.records + static_cast<size_t>(tile) * p.L.bytes, p.L, p.K, p.smooth);
  if (tid == 0) p.buf_n[tile] = 0;
  return true;
}

// Bounded wait until the slot's last issued list entry is at least `e`;
// false after `limit` polls.
__device__ __forceinline__ bool wait_issued(const int *slot_last, int e, uint32_t limit) {
  for (uint32_t it = 0; it < limit; ++it)
    if (*reinterpret_cast<const volatile int *>(slot_last) >= e) return true;
  return false;
}


template <int D, bool BF16, bool KDA>
__global__ void __launch_bounds__(kThreads, 2) decode_kernel(const KParams p) {
  using L = SL<D, BF16, KDA>;
  using TR = DecodeTraits<D, BF16, KDA>;
  constexpr int kStages = TR::kStages;
  constexpr bool kQuad = TR::kQuad;
  using SC = Scratch<D, !TR::kKtOverCodes, TR::kTok, kQuad>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int slot_bytes = L(p.L.bytes).bytes;
  SC &s = *reinterpret_cast<SC *>(smem + kStages * slot_bytes);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tiles = p.B * p.Hv;

  // This CTA's tiles are blockIdx.x + i * gridDim.x.  The list is built in
  // that order, compacted to the active sequences when there is a mask; on
  // the quad path the plain tokens (0 <= n < W - 1) come first and the rest
  // (boundary tokens, skipped tiles) after them.  Without a mask and without
  // the quad path every tile keeps its position, so the first slots' record
  // copies go out before the phases are known; the quad path prefetches
  // those records into L2 instead.
  const int mine = (tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                   static_cast<int>(gridDim.x);
  const bool speculate = !kQuad && p.mask == nullptr;
  if (tid == 0) {
    s.abort = 0;
    for (int st = 0; st < kStages; ++st) {
      mbar_init(&s.bar[st], 1);
      s.done[st] = 0;
      s.slot_last[st] = -1;
    }
    fence_mbar_init();
  }
  // The quad path's first records are fetched into L2 before the wait below:
  // a prefetch consumes nothing, and L2 is where the previous kernel's writes
  // land, so it cannot make a later copy read stale data.
  if (kQuad && tid == 0)
    for (int st = 0; st < kStages && st < mine; ++st)
      prefetch_l2(p.records + static_cast<size_t>(blockIdx.x + st * gridDim.x) * p.L.bytes,
                  static_cast<uint32_t>(p.L.bytes));
  // Launched as a programmatic dependent: everything above touched only this
  // CTA's shared memory (and L2).  Wait here until the previous kernel in the
  // stream has completed and its writes are visible, and let the next one
  // start its own setup as this grid's CTAs retire.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (speculate && tid == 0) {
    for (int st = 0; st < kStages && st < mine; ++st)
      if (!(p.withhold && blockIdx.x == 0 && st == 0))
        issue_record<D, BF16, KDA>(p, smem + st * slot_bytes, &s.bar[st],
                                   blockIdx.x + st * gridDim.x);
  }
  int keep = 0, tile = 0, n = -1, coord = 0;
  float a0 = 0.0f, b0 = 0.0f;
  if (tid < mine) {
    tile = blockIdx.x + tid * gridDim.x;
    const int b = tile / p.Hv, h = tile - b * p.Hv, group = p.Hv / p.Hk;
    coord = (b << 12) | ((h / group) << 1) | ((h % group == 0) ? 1 : 0);
    if (speculate || p.mask == nullptr || p.mask[b] != 0) {
      keep = 1;
      n = p.buf_n[tile];
      if (n >= 0 && n < p.W) {
        if (!KDA) a0 = p.alpha[tile];
        b0 = p.beta[tile];
      } else {
        atomicOr(p.err, kErrBadPhase);
        n = -1;
      }
    }
  }
  const bool plain = kQuad && keep && n >= 0 && n < p.W - 1;
  const unsigned ball_p = __ballot_sync(kFull, plain);
  const unsigned ball_o = __ballot_sync(kFull, keep && !plain);
  if (lane == 0) {
    s.warp_cnt[warp] = __popc(ball_p);
    s.warp_cnt2[warp] = __popc(ball_o);
  }
  __syncthreads();
  int base_p = 0, base_o = 0, P = 0, count = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    base_p += (w < warp) ? s.warp_cnt[w] : 0;
    base_o += (w < warp) ? s.warp_cnt2[w] : 0;
    P += s.warp_cnt[w];
    count += s.warp_cnt2[w];
  }
  count += P;
  if (keep) {
    const unsigned below = (1u << lane) - 1u;
    const int pos = plain ? base_p + __popc(ball_p & below) : P + base_o + __popc(ball_o & below);
    s.tl_tile[pos] = tile;
    s.tl_n[pos] = n;
    s.tl_coord[pos] = coord;
    s.tl_a[pos] = a0;
    s.tl_b[pos] = b0;
  }
  __syncthreads();

  // Copies of list entry `nx` into slot `st` (one thread).
  auto issue = [&](int st, int nx) {
    uint8_t *slot = smem + st * slot_bytes;
    issue_record<D, BF16, KDA>(p, slot, &s.bar[st], s.tl_tile[nx]);
    issue_rest<D, BF16, KDA>(p, slot, &s.bar[st], s.tl_tile[nx], s.tl_n[nx], s.tl_coord[nx]);
    s.slot_last[st] = nx;
  };
  if (tid == 0)
    for (int st = 0; st < kStages && st < count; ++st) {
      // testing: CTA 0 leaves its first slot without copies, so that the
      // bounded wait on it expires (nothing is in flight into that slot)
      if (p.withhold && blockIdx.x == 0 && st == 0) continue;
      if (speculate) {
        uint8_t *slot = smem + st * slot_bytes;
        issue_rest<D, BF16, KDA>(p, slot, &s.bar[st], s.tl_tile[st], s.tl_n[st],
                                 s.tl_coord[st]);
        s.slot_last[st] = st;
      } else {
        issue(st, st);
      }
    }

  bool aborted = false;
  int i = 0;
  if constexpr (kQuad) {
    // Plain tokens, list entries 0 .. P-1: quad q takes entries q, q + 2, ...
    // Entry i sits in slot i % kStages; the last warp of its quad to finish
    // refills that slot with entry i + kStages.
    const int quad = warp >> 2, w = warp & 3;
    int li = 0;
    bool qabort = false;
    for (int e = quad; e < P; e += 2, ++li) {
      const int st = e % kStages;
      const uint32_t parity = static_cast<uint32_t>(e / kStages) & 1u;
      // The two quads take alternate entries, so one may reach entry e while
      // the entry before it in the same slot (e - kStages, the other quad's)
      // is still unfinished and e not yet issued.  A parity wait alone could
      // then pass on the earlier phase: first wait (bounded) until entry e's
      // copies have been issued into the slot.
      const bool ok = wait_issued(&s.slot_last[st], e, p.wait_limit) &&
                      mbar_wait_bounded(&s.bar[st], parity, p.wait_limit);
      uint8_t *slot = smem + st * slot_bytes;
      QTok<D> &x = s.u.qt[quad][li & 1];
      const int tl = s.tl_tile[e], ne = s.tl_n[e];

      quad_channel<D, KDA>(p, x, slot, tl, ne, s.tl_coord[e], s.tl_a[e], w, ok);
      if constexpr (TR::kEarlyRelease) {
        // everything the rows need from the slot goes to registers now, so
        // that the slot is refilled while the rows are computed
        RegRows rg;
        quad_rows_load<D, KDA>(p, slot, ne, w, rg.r);
        // This warp's reads of the slot are done: order them before the bulk
        // copy that refills it.
        fence_proxy_async();
        // the quad's one barrier per tile; it also tells every warp whether
        // any thread's wait expired, so that the quad leaves the loop together
        if (quad_bar_any(quad, !ok)) {
          qabort = true;
          break;
        }
        if (w == 0 && lane == 0 && e + kStages < count) issue(st, e + kStages);
        quad_rows<D, KDA>(p, x, rg, tl, ne, s.tl_b[e], w);
        if (w == 0 && lane == 0) p.buf_n[tl] = ne + 1;
      } else {
        if (quad_bar_any(quad, !ok)) {
          qabort = true;
          break;
        }
        quad_rows<D, KDA>(p, x, SlotRows<D, KDA>(p, slot, ne, w), tl, ne, s.tl_b[e], w);
        if (w == 0 && lane == 0) p.buf_n[tl] = ne + 1;
        // This warp is done with the slot: order its generic-proxy accesses
        // before the bulk copy that refills it; the quad's last warp to get
        // here issues that copy.
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) {
          __threadfence_block();
          if (atomicAdd(&s.done[st], 1) == 3) {
            s.done[st] = 0;
            __threadfence_block();
            if (e + kStages < count) issue(st, e + kStages);
          }
        }
        __syncwarp();
      }
    }
    aborted = __syncthreads_or(qabort) != 0;
    i = P;
  }

  // The whole CTA on the remaining entries (every entry without the quad path).
  int issued = count < i + kStages ? count : i + kStages;
  auto refill = [&](int freed) {
    // slot freed % kStages takes the next tile in line
    if (freed >= 0 && issued < count) {
      if (tid == 0) issue(freed % kStages, issued);
      ++issued;
    }
  };
  for (; i < count && !aborted; ++i) {
    const int st = i % kStages;
    const uint32_t parity = static_cast<uint32_t>(i / kStages) & 1u;
    if constexpr (TR::kTok == 2) {
      // Every thread waits for the copies itself; the tile's one CTA barrier
      // (inside process_tile) then makes the abort decision uniform and frees
      // the previous tile's slot, which is refilled right after it.
      if (!mbar_wait_bounded(&s.bar[st], parity, p.wait_limit)) s.abort = 1;
      bool ok;
      if (s.tl_n[i] >= 0) {
        ok = process_tile<D, BF16, KDA>(p, s, s.u.tok[i & 1], smem + st * slot_bytes,
                                        s.tl_tile[i], s.tl_n[i], s.tl_coord[i], s.tl_a[i],
                                        s.tl_b[i], [] {});
      } else {
        __syncthreads();
        ok = !s.abort;
      }
      if (!ok) {
        aborted = true;
        break;
      }
      // This warp is done with the slot.  Its generic-proxy accesses are
      // ordered before the bulk copy that refills it; the last warp to finish
      // issues that copy (tile i + kStages) at once.
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) {
        __threadfence_block();
        if (atomicAdd(&s.done[st], 1) == kWarps - 1) {
          s.done[st] = 0;
          __threadfence_block();
          if (i + kStages < count) issue(st, i + kStages);
        }
      }
      __syncwarp();
    } else {
      if (!mbar_wait_bounded(&s.bar[st], parity, p.wait_limit)) s.abort = 1;
      __syncthreads();
      if (s.abort) {
        aborted = true;
        break;
      }
      if (s.tl_n[i] >= 0)
        process_tile<D, BF16, KDA>(p, s, s.u.tok[0], smem + st * slot_bytes, s.tl_tile[i],
                                   s.tl_n[i], s.tl_coord[i], s.tl_a[i], s.tl_b[i], [] {});
      fence_proxy_async();
      __syncthreads();
      refill(i);
    }
  }
  if (aborted) {
    // A copy did not complete in time: flag it, then give the copies still in
    // flight into this CTA's shared memory (the last ones issued into each
    // slot) a bounded chance to land before the CTA exits.
    __syncthreads();
    if (tid == 0) {
      atomicOr(p.err, kErrTimeout);
      for (int st = 0; st < kStages; ++st) {
        const int last = s.slot_last[st];
        if (last >= 0)
          mbar_wait_bounded(&s.bar[st], static_cast<uint32_t>(last / kStages) & 1u,
                            p.wait_limit);
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// Flush (fold a partial window), dequantize, init
// ---------------------------------------------------------------------------

// Loads a tile's record and n buffered tokens into a slot with plain 16-byte
// loads (the whole CTA).
template <int D, bool BF16, bool KDA, int WM = kMaxWindow>
__device__ __forceinline__ void load_slot(const KParams &p, uint8_t *slot, int tile, int n) {
  using L = SL<D, BF16, KDA, WM>;
  const L lay(p.L.bytes);
  const int b = tile / p.Hv, h = tile - b * p.Hv, hk = h / (p.Hv / p.Hk);
  auto copy = [&](uint8_t *dst, const void *src, int bytes) {
    const uint4 *s4 = static_cast<const uint4 *>(src);
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
    for (int k = threadIdx.x; k < bytes / 16; k += kThreads) d4[k] = s4[k];
  };
  copy(slot, p.records + static_cast<size_t>(tile) * p.L.bytes, p.L.bytes);
  if (n > 0) {
    copy(slot + lay.bd, p.buf_d + static_cast<size_t>(tile) * p.W * D, n * D * 4);
    copy(slot + lay.bk,
         static_cast<const uint8_t *>(p.buf_k) + (static_cast<size_t>(b) * p.Hk + hk) * p.W * D * L::IB,
         n * D * L::IB);
    if (KDA) copy(slot + lay.bg, p.buf_g + static_cast<size_t>(tile) * p.W * D, n * D * 4);
  }
  if (!KDA) copy(slot + lay.bg, p.buf_g + static_cast<size_t>(tile) * p.gstride, p.gstride * 4);
}

// MODE 0: flush selected tiles with 0 < n < W.  MODE 1: write the fp32 state
// (the window base, or the current state with include_buffer).
template <int D, bool BF16, bool KDA, int MODE, int WM>
__global__ void __launch_bounds__(kThreads) fold_kernel(const KParams p) {
  using G = FG<D>;
  using L = SL<D, BF16, KDA, WM>;
  using IT = in_t<BF16>;
  using SC = Scratch<D, true, 1, false, WM>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t *slot = smem;
  const L lay(p.L.bytes);
  SC &s = *reinterpret_cast<SC *>(smem + lay.bytes);
  Tok<D, WM> &x = s.u.tok[0];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int tile = blockIdx.x;
  const int b = tile / p.Hv;
  if (MODE == 0 && p.mask != nullptr && p.mask[b] == 0) return;
  int n = p.buf_n[tile];
  if (n < 0 || n >= p.W) {
    if (tid == 0) atomicOr(p.err, kErrBadPhase);
    return;
  }
  if (MODE == 0 && n == 0) return;
  if (MODE == 1 && !p.include_buffer) n = 0;
  load_slot<D, BF16, KDA, WM>(p, slot, tile, n);
  __syncthreads();
  const float *rsig = reinterpret_cast<const float *>(slot + p.L.off_sig);
  const float *rm = reinterpret_cast<const float *>(slot + p.L.off_m);
  const float *rcv = reinterpret_cast<const float *>(slot + p.L.off_cv);
  const int *rcid = reinterpret_cast<const int *>(slot + p.L.off_cid);
  const float *sbd = reinterpret_cast<const float *>(slot + lay.bd);
  const IT *sbk = reinterpret_cast<const IT *>(slot + lay.bk);
  const float *sbg = reinterpret_cast<const float *>(slot + lay.bg);
  if (tid < D) {
    const int j = tid;
    float acc = 1.0f;
    for (int sl = n - 1; sl >= 0; --sl) {
      s.kt[sl][padc(j)] = to_f(sbk[sl * D + j]) * acc;
      acc *= KDA ? sbg[sl * D + j] : sbg[sl];
    }
    x.G[j] = acc;
    x.mG[padc(j)] = rm[j] * acc;
  }
  __syncthreads();
  float2 S[2][G::NSPAN][8];
  if (warp < G::NRB) {
    uint4 A[2][G::NSPAN];
    load_codes<D>(slot, A);
    build_state<D, false, WM>(x, &s.kt[0][0], A, rsig, rcv, rcid, sbd, n, p.K, S);
  }
  if constexpr (MODE == 0) {
    __syncthreads();
    quantize_tile<D>(s, reinterpret_cast<double *>(slot + L::QS_COLPART),
                     reinterpret_cast<float *>(slot + L::QS_COLMAX), S,
                     p.records + static_cast<size_t>(tile) * p.L.bytes, p.L, p.K, p.smooth);
    if (tid == 0) p.buf_n[tile] = 0;
  } else if (warp < G::NRB) {
    float *dst = p.S_out + static_cast<size_t>(tile) * D * D;
    const int r0 = 16 * warp + g;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr)
#pragma unroll
      for (int hh = 0; hh < G::NSPAN; ++hh) {
        if (!chunk_valid<D>(t)) continue;
        float4 *row = reinterpret_cast<float4 *>(dst + static_cast<size_t>(r0 + 8 * rr) * D +
                                                 frag_col(hh, t, 0));
#pragma unroll
        for (int u = 0; u < 4; ++u)
          row[u] = make_float4(S[rr][hh][2 * u].x, S[rr][hh][2 * u].y, S[rr][hh][2 * u + 1].x,
                               S[rr][hh][2 * u + 1].y);
      }
  }
}

// Decode of p.ntok consecutive tokens per tile in one launch (a speculative
// verify step, or every step of a window longer than kMaxWindow tokens).  One
// CTA per tile runs the whole-CTA token path token after token with the tile
// kept in shared memory: the record and the buffered tokens are loaded once,
// each token's inputs are staged, its key and gate join the staged buffer
// (process_tile stores its d_t there), and a fold, which writes the new record
// to global memory, is followed by loading that record.  The result equals
// p.ntok launches of the decode step on the same inputs.  Inputs and outputs
// are token-major: token i of q sits at q + i * B * Hk * D, and so on.
template <int D, bool BF16, bool KDA>
__global__ void __launch_bounds__(kThreads) tokens_kernel(const KParams p) {
  constexpr int WM = kMaxWindowLong;
  using L = SL<D, BF16, KDA, WM>;
  using IT = in_t<BF16>;
  using SC = Scratch<D, true, 1, false, WM>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t *slot = smem;
  const L lay(p.L.bytes);
  SC &s = *reinterpret_cast<SC *>(smem + lay.bytes);
  const int tid = threadIdx.x;
  const int tile = blockIdx.x;
  const int b = tile / p.Hv, h = tile - b * p.Hv, group = p.Hv / p.Hk, hk = h / group;
  if (p.mask != nullptr && p.mask[b] == 0) return;
  int n = p.buf_n[tile];
  if (n < 0 || n >= p.W) {
    if (tid == 0) atomicOr(p.err, kErrBadPhase);
    return;
  }
  const int coord = (b << 12) | (hk << 1) | ((h % group == 0) ? 1 : 0);
  const size_t tiles = static_cast<size_t>(p.B) * p.Hv;
  const size_t qk_tok = static_cast<size_t>(p.B) * p.Hk * D, v_tok = tiles * D;
  auto copy = [&](uint8_t *dst, const void *src, int bytes) {
    const uint4 *s4 = static_cast<const uint4 *>(src);
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
    for (int k = tid; k < bytes / 16; k += kThreads) d4[k] = s4[k];
  };
  load_slot<D, BF16, KDA, WM>(p, slot, tile, n);
  IT *sbk = reinterpret_cast<IT *>(slot + lay.bk);
  float *sbg = reinterpret_cast<float *>(slot + lay.bg);
  const IT *sk = reinterpret_cast<const IT *>(slot + lay.k);
  const float *sa = reinterpret_cast<const float *>(slot + lay.a);
  for (int i = 0; i < p.ntok; ++i) {
    const IT *q = static_cast<const IT *>(p.q) + i * qk_tok;
    const IT *k = static_cast<const IT *>(p.k) + i * qk_tok;
    const IT *v = static_cast<const IT *>(p.v) + i * v_tok;
    const size_t qk = (static_cast<size_t>(b) * p.Hk + hk) * D;
    copy(slot + lay.q, q + qk, D * L::IB);
    copy(slot + lay.k, k + qk, D * L::IB);
    copy(slot + lay.v, v + static_cast<size_t>(tile) * D, D * L::IB);
    if (KDA) copy(slot + lay.a, p.alpha + (i * tiles + tile) * D, D * 4);
    const float a0 = KDA ? 0.0f : p.alpha[i * tiles + tile];
    const float b0 = p.beta[i * tiles + tile];
    __syncthreads();
    KParams pi = p;
    pi.out = static_cast<uint8_t *>(p.out) + i * v_tok * (p.out_bf16 ? 2 : 4);
    process_tile<D, BF16, KDA>(pi, s, s.u.tok[0], slot, tile, n, coord, a0, b0, [] {});
    __syncthreads();
    if (n + 1 == p.W) {
      // the fold wrote the new record: bring it into the slot
      copy(slot, p.records + static_cast<size_t>(tile) * p.L.bytes, p.L.bytes);
      n = 0;
    } else {
      // token i joins the staged buffer (its d_t is there already)
      if (tid < D) {
        sbk[n * D + tid] = sk[tid];
        if (KDA) sbg[n * D + tid] = sa[tid];
      }
      if (!KDA && tid == 0) sbg[n] = a0;
      n += 1;
    }
    __syncthreads();
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads) init_kernel(const KParams p) {
  using G = FG<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t *qscr = smem;  // D*D bytes of quantizer scratch
  Scratch<D, false> &s = *reinterpret_cast<Scratch<D, false> *>(smem + D * D);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int tile = blockIdx.x;
  const int b = tile / p.Hv;
  if (p.mask != nullptr && p.mask[b] == 0) return;
  float2 S[2][G::NSPAN][8];
  if (warp < G::NRB) {
    const float *src = p.S_in + static_cast<size_t>(tile) * D * D;
    const int r0 = 16 * warp + g;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr)
#pragma unroll
      for (int hh = 0; hh < G::NSPAN; ++hh) {
        if (!chunk_valid<D>(t)) {
#pragma unroll
          for (int e2 = 0; e2 < 8; ++e2) S[rr][hh][e2] = make_float2(0.0f, 0.0f);
          continue;
        }
        const float4 *row = reinterpret_cast<const float4 *>(
            src + static_cast<size_t>(r0 + 8 * rr) * D + frag_col(hh, t, 0));
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float4 v = __ldcs(row + u);
          S[rr][hh][2 * u] = make_float2(v.x, v.y);
          S[rr][hh][2 * u + 1] = make_float2(v.z, v.w);
        }
      }
  }
  quantize_tile<D>(s, reinterpret_cast<double *>(qscr),
                   reinterpret_cast<float *>(qscr + G::NRB * D * 8), S,
                   p.records + static_cast<size_t>(tile) * p.L.bytes, p.L, p.K, p.smooth);
  if (tid == 0) p.buf_n[tile] = 0;
}

// ---------------------------------------------------------------------------
// Chunked prefill (WY form)
// ---------------------------------------------------------------------------
//
// The exact recurrence over a prompt in chunks of kChunk tokens.  Within a
// chunk with cumulative gates g_t (g_t = alpha_1 ... alpha_t from the chunk's
// start; a scalar for GDN, per key channel for KDA), Kg = K o g, Kh = K / g
// and Qg = Q o g:
//   A   = strict lower part of diag(beta) Kg Kh^T
//   U   = (I + A)^-1 diag(beta) (V - Kg S0^T)       (forward substitution)
//   O   = Qg S0^T + lower part (with diagonal) of Qg Kh^T, times U
//   S_C = S0 diag(g_C) + U^T (Kh o g_C)
// which reproduces the token loop exactly in exact arithmetic.  The products
// with the state (S0 Kg^T, S0 Qg^T and the rank-kChunk update) run on the tf32
// tensor path with hi/lo splits (about fp32 accuracy), with the state itself
// as the A operand straight from registers; the small kChunk x kChunk
// products, the substitution and the outputs use fp32 FMAs.  Kh divides by
// the gates: the gates' product over one chunk must stay a normal fp32 number.
constexpr int kChunk = 16;
static_assert(kChunk * kChunk == kThreads, "one thread per entry of a chunk's A and M");

template <int D>
struct ChunkSmem {
  static constexpr int P = D + 2;   // rows of Qg, Kg, Kh: 8-byte aligned, at most 2-way banks
  static constexpr int PY = D + 4;  // rows of the transposed products
  alignas(16) float qg[kChunk][P];
  alignas(16) float kg[kChunk][P];
  alignas(16) float kh[kChunk][P];
  alignas(16) float v[kChunk][D];
  alignas(16) float yk[kChunk][PY];  // (S0 Kg^T)^T
  alignas(16) float yq[kChunk][PY];  // (S0 Qg^T)^T
  alignas(16) float u[kChunk][D];    // U: the d_s of the chunk's state update
  alignas(16) float kt[kChunk][FG<D>::PADW];  // Kh o g_C in the rank update's layout
  float amat[kChunk][kChunk + 1];
  float mmat[kChunk][kChunk + 1];
  float gc[D];
  float beta[kChunk];
};

template <int D, bool BF16, bool KDA>
__global__ void __launch_bounds__(kThreads, 2) chunk_prefill_kernel(const KParams p) {
  using G = FG<D>;
  using IT = in_t<BF16>;
  using CS = ChunkSmem<D>;
  constexpr bool kMma = D >= 64;  // rank update on the tensor path (its column layout needs d >= 64)
  extern __shared__ __align__(128) uint8_t smem[];
  CS &c = *reinterpret_cast<CS *>(smem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int tile = blockIdx.x;
  const int b = tile / p.Hv, h = tile - b * p.Hv, hk = h / (p.Hv / p.Hk);
  if (p.mask != nullptr && p.mask[b] == 0) return;
  const bool rows_here = warp < G::NRB;
  const int r0 = 16 * warp + g, r1 = r0 + 8;
  float2 S[2][G::NSPAN][8];
#pragma unroll
  for (int rr = 0; rr < 2; ++rr)
#pragma unroll
    for (int hh = 0; hh < G::NSPAN; ++hh)
#pragma unroll
      for (int e2 = 0; e2 < 8; ++e2) S[rr][hh][e2] = make_float2(0.0f, 0.0f);
  if (p.S_in != nullptr && rows_here) {
    const float *src = p.S_in + static_cast<size_t>(tile) * D * D;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr)
#pragma unroll
      for (int hh = 0; hh < G::NSPAN; ++hh) {
        if (!chunk_valid<D>(t)) continue;
        const float4 *row = reinterpret_cast<const float4 *>(
            src + static_cast<size_t>(r0 + 8 * rr) * D + frag_col(hh, t, 0));
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float4 v = row[u];
          S[rr][hh][2 * u] = make_float2(v.x, v.y);
          S[rr][hh][2 * u + 1] = make_float2(v.z, v.w);
        }
      }
  }
  const IT *q = static_cast<const IT *>(p.q), *k = static_cast<const IT *>(p.k);
  const IT *v = static_cast<const IT *>(p.v);
  const size_t tokB = static_cast<size_t>(p.B);
  auto qk_at = [&](int tt) { return ((tt * tokB + b) * p.Hk + hk) * D; };
  auto hv_at = [&](int tt) { return (tt * tokB + b) * p.Hv + h; };

  for (int t0 = 0; t0 < p.T; t0 += kChunk) {
    const int cn = p.T - t0 < kChunk ? p.T - t0 : kChunk;
    // Channel j: the cumulative gates and Kg, Kh, Qg; v; beta.
    if (tid < D) {
      const int j = tid;
      float gcum = 1.0f;
      for (int tt = 0; tt < kChunk; ++tt) {
        float qv = 0.0f, kv = 0.0f, vv = 0.0f, kg = 0.0f, kh = 0.0f, qg = 0.0f;
        if (tt < cn) {
          gcum *= KDA ? p.alpha[hv_at(t0 + tt) * D + j] : p.alpha[hv_at(t0 + tt)];
          qv = to_f(q[qk_at(t0 + tt) + j]);
          kv = to_f(k[qk_at(t0 + tt) + j]);
          vv = to_f(v[hv_at(t0 + tt) * D + j]);
          kg = kv * gcum;
          kh = kv / gcum;
          qg = qv * gcum;
        }
        c.qg[tt][j] = qg;
        c.kg[tt][j] = kg;
        c.kh[tt][j] = kh;
        c.v[tt][j] = vv;
      }
      c.gc[j] = gcum;
      if (j < kChunk) c.beta[j] = j < cn ? p.beta[hv_at(t0 + j)] : 0.0f;
    }
    __syncthreads();
    // The rank update's keys Kh o g_C, and the products with the state.
    if (tid < D) {
      for (int tt = 0; tt < kChunk; ++tt)
        c.kt[0][tt * (kMma ? kt_mma_stride<D>() : G::PADW) +
                (kMma ? kt_mma_pos(tid) : padc(tid))] = c.kh[tt][tid] * c.gc[tid];
    }
    if (rows_here) {
      // Y = S0 X^T for X = Kg and Qg: A = the state (rows r0, r1; k-block
      // (h, e2) takes columns 64h + 16t' + 2e2 and + 1 of lane t'), B = X^T.
      float2 yk[2][2], yq[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) yk[nt][0] = yk[nt][1] = yq[nt][0] = yq[nt][1] = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int hh = 0; hh < G::NSPAN; ++hh) {
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) {
          const bool ok = chunk_valid<D>(t);
          uint32_t ah[4], al[4];
          tf32_split(ok ? S[0][hh][e2].x : 0.0f, ah[0], al[0]);
          tf32_split(ok ? S[1][hh][e2].x : 0.0f, ah[1], al[1]);
          tf32_split(ok ? S[0][hh][e2].y : 0.0f, ah[2], al[2]);
          tf32_split(ok ? S[1][hh][e2].y : 0.0f, ah[3], al[3]);
          const int col = 64 * hh + 16 * t + 2 * e2;
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            const int tok = 8 * nt + g;
            const float2 xk = ok ? *reinterpret_cast<const float2 *>(&c.kg[tok][col])
                                 : make_float2(0.0f, 0.0f);
            const float2 xq = ok ? *reinterpret_cast<const float2 *>(&c.qg[tok][col])
                                 : make_float2(0.0f, 0.0f);
            uint32_t bh0, bl0, bh1, bl1;
            tf32_split(xk.x, bh0, bl0);
            tf32_split(xk.y, bh1, bl1);
            mma_tf32(yk[nt][0], yk[nt][1], al[0], al[1], al[2], al[3], bh0, bh1);
            mma_tf32(yk[nt][0], yk[nt][1], ah[0], ah[1], ah[2], ah[3], bl0, bl1);
            mma_tf32(yk[nt][0], yk[nt][1], ah[0], ah[1], ah[2], ah[3], bh0, bh1);
            tf32_split(xq.x, bh0, bl0);
            tf32_split(xq.y, bh1, bl1);
            mma_tf32(yq[nt][0], yq[nt][1], al[0], al[1], al[2], al[3], bh0, bh1);
            mma_tf32(yq[nt][0], yq[nt][1], ah[0], ah[1], ah[2], ah[3], bl0, bl1);
            mma_tf32(yq[nt][0], yq[nt][1], ah[0], ah[1], ah[2], ah[3], bh0, bh1);
          }
        }
      }
      // accumulator: rows r0 (x, y = tokens 8nt + 2t, + 1) and r1
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int tk = 8 * nt + 2 * t;
        c.yk[tk][r0] = yk[nt][0].x;
        c.yk[tk + 1][r0] = yk[nt][0].y;
        c.yk[tk][r1] = yk[nt][1].x;
        c.yk[tk + 1][r1] = yk[nt][1].y;
        c.yq[tk][r0] = yq[nt][0].x;
        c.yq[tk + 1][r0] = yq[nt][0].y;
        c.yq[tk][r1] = yq[nt][1].x;
        c.yq[tk + 1][r1] = yq[nt][1].y;
      }
    }
    {
      // A_ts = beta_t Kg_t . Kh_s (s < t) and M_ts = Qg_t . Kh_s (s <= t):
      // thread (t, s) takes one entry of each
      const int ta = tid / kChunk, sa = tid % kChunk;
      float dk = 0.0f, dq = 0.0f;
#pragma unroll 8
      for (int j = 0; j < D; j += 2) {
        const float2 x = *reinterpret_cast<const float2 *>(&c.kh[sa][j]);
        const float2 kk = *reinterpret_cast<const float2 *>(&c.kg[ta][j]);
        const float2 qq = *reinterpret_cast<const float2 *>(&c.qg[ta][j]);
        dk = fmaf(kk.x, x.x, fmaf(kk.y, x.y, dk));
        dq = fmaf(qq.x, x.x, fmaf(qq.y, x.y, dq));
      }
      c.amat[ta][sa] = sa < ta ? c.beta[ta] * dk : 0.0f;
      c.mmat[ta][sa] = sa <= ta ? dq : 0.0f;
    }
    __syncthreads();
    // Value channel i: U by forward substitution, then the chunk's outputs.
    if (tid < D) {
      const int i = tid;
      float uu[kChunk];
#pragma unroll
      for (int tt = 0; tt < kChunk; ++tt) {
        float r = c.beta[tt] * (c.v[tt][i] - c.yk[tt][i]);
#pragma unroll
        for (int s2 = 0; s2 < tt; ++s2) r = fmaf(-c.amat[tt][s2], uu[s2], r);
        uu[tt] = r;
        c.u[tt][i] = r;
      }
      if (p.out != nullptr) {
#pragma unroll
        for (int tt = 0; tt < kChunk; ++tt) {
          if (tt >= cn) break;
          float o = c.yq[tt][i];
#pragma unroll
          for (int s2 = 0; s2 <= tt; ++s2) o = fmaf(c.mmat[tt][s2], uu[s2], o);
          st_out(p.out, static_cast<size_t>(hv_at(t0 + tt)) * D + i, o, p.out_bf16);
        }
      }
    }
    __syncthreads();
    // S = S0 diag(g_C) + U^T (Kh o g_C)
    if (rows_here) {
#pragma unroll
      for (int hh = 0; hh < G::NSPAN; ++hh) {
        if (!chunk_valid<D>(t)) continue;
        const int cb = frag_col(hh, t, 0);
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) {
          const float2 gg = make_float2(c.gc[cb + 2 * e2], c.gc[cb + 2 * e2 + 1]);
          S[0][hh][e2] = __fmul2_rn(S[0][hh][e2], gg);
          S[1][hh][e2] = __fmul2_rn(S[1][hh][e2], gg);
        }
      }
      if constexpr (kMma)
        rank_update_mma<D, kChunk>(S, &c.u[0][0], &c.kt[0][0], cn);
      else
        rank_update_ffma<D>(S, &c.u[0][0], &c.kt[0][0], cn);
    }
    __syncthreads();  // the chunk's arrays are free for the next chunk
  }
  // the quantizer's scratch goes over the chunk arrays
  uint8_t *qscr = smem;  // D*D bytes
  Scratch<D, false> &s = *reinterpret_cast<Scratch<D, false> *>(smem + D * D);
  quantize_tile<D>(s, reinterpret_cast<double *>(qscr),
                   reinterpret_cast<float *>(qscr + G::NRB * D * 8), S,
                   p.records + static_cast<size_t>(tile) * p.L.bytes, p.L, p.K, p.smooth);
  if (tid == 0) p.buf_n[tile] = 0;
}

// ---------------------------------------------------------------------------
// Launch plumbing
// ---------------------------------------------------------------------------

// Per-device, per-kernel, per-K launch facts, computed once.
struct LaunchInfo {
  int ready;
  int sms;
  int ctas_per_sm;
};

template <typename Kern>
cudaError_t prepare(Kern kernel, size_t smem, size_t smem_max, int K,
                    LaunchInfo (&cache)[32][kMaxComp + 1], LaunchInfo &out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  LaunchInfo &li = cache[dev & 31][K];
  if (__atomic_load_n(&li.ready, __ATOMIC_ACQUIRE)) {
    out = li;
    return cudaSuccess;
  }
  if (smem_max > 48 * 1024) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem_max));
    if (e != cudaSuccess) return e;
  }
  int sms = 0, occ = 0;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, kThreads, smem)) !=
      cudaSuccess)
    return e;
  li.sms = sms;
  li.ctas_per_sm = occ > 0 ? occ : 1;
  __atomic_store_n(&li.ready, 1, __ATOMIC_RELEASE);
  out = li;
  return cudaSuccess;
}

template <int D, bool BF16, bool KDA>
cudaError_t decode_t(const KParams &p, cudaStream_t st) {
  static LaunchInfo cache[32][kMaxComp + 1];
  using L = SL<D, BF16, KDA>;
  using TR = DecodeTraits<D, BF16, KDA>;
  constexpr int NST = TR::kStages;
  constexpr size_t scratch = sizeof(Scratch<D, !TR::kKtOverCodes, TR::kTok, TR::kQuad>);
  const size_t smem = NST * L(p.L.bytes).bytes + scratch;
  const size_t smem_max = NST * L(record_layout(D, kMaxComp).bytes).bytes + scratch;
  LaunchInfo li;
  cudaError_t e = prepare(decode_kernel<D, BF16, KDA>, smem, smem_max, p.K, cache, li);
  if (e != cudaSuccess) return e;
  const int tiles = p.B * p.Hv;
  int grid = li.sms * li.ctas_per_sm;
  if (grid > tiles) grid = tiles;
  const int need = (tiles + kMaxTilesPerCta - 1) / kMaxTilesPerCta;
  if (grid < need) grid = need;
  // programmatic dependent launch: the kernel waits (griddepcontrol.wait)
  // before its first global access, so its launch and shared-memory setup
  // may overlap the tail of the previous kernel in the stream
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, decode_kernel<D, BF16, KDA>, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D, bool BF16, bool KDA, int MODE, int WM>
cudaError_t fold_wm(const KParams &p, cudaStream_t st) {
  static LaunchInfo cache[32][kMaxComp + 1];
  using L = SL<D, BF16, KDA, WM>;
  using SC = Scratch<D, true, 1, false, WM>;
  const size_t smem = L(p.L.bytes).bytes + sizeof(SC);
  const size_t smem_max = L(record_layout(D, kMaxComp).bytes).bytes + sizeof(SC);
  LaunchInfo li;
  cudaError_t e = prepare(fold_kernel<D, BF16, KDA, MODE, WM>, smem, smem_max, p.K, cache, li);
  if (e != cudaSuccess) return e;
  fold_kernel<D, BF16, KDA, MODE, WM><<<p.B * p.Hv, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

// Windows above kMaxWindow tokens use the longer buffer capacity.
template <int D, bool BF16, bool KDA, int MODE>
cudaError_t fold_t(const KParams &p, cudaStream_t st) {
  if (p.W > kMaxWindow) return fold_wm<D, BF16, KDA, MODE, kMaxWindowLong>(p, st);
  return fold_wm<D, BF16, KDA, MODE, kMaxWindow>(p, st);
}

template <int D, bool BF16, bool KDA>
cudaError_t tokens_t(const KParams &p, cudaStream_t st) {
  static LaunchInfo cache[32][kMaxComp + 1];
  using L = SL<D, BF16, KDA, kMaxWindowLong>;
  using SC = Scratch<D, true, 1, false, kMaxWindowLong>;
  const size_t smem = L(p.L.bytes).bytes + sizeof(SC);
  const size_t smem_max = L(record_layout(D, kMaxComp).bytes).bytes + sizeof(SC);
  LaunchInfo li;
  cudaError_t e = prepare(tokens_kernel<D, BF16, KDA>, smem, smem_max, p.K, cache, li);
  if (e != cudaSuccess) return e;
  tokens_kernel<D, BF16, KDA><<<p.B * p.Hv, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

template <int D>
cudaError_t init_t(const KParams &p, cudaStream_t st) {
  static LaunchInfo cache[32][kMaxComp + 1];
  const size_t smem = D * D + sizeof(Scratch<D, false>);
  LaunchInfo li;
  cudaError_t e = prepare(init_kernel<D>, smem, smem, p.K, cache, li);
  if (e != cudaSuccess) return e;
  init_kernel<D><<<p.B * p.Hv, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

template <int D, bool BF16, bool KDA>
cudaError_t prefill_t(const KParams &p, cudaStream_t st) {
  static LaunchInfo cache[32][kMaxComp + 1];
  size_t smem = sizeof(ChunkSmem<D>);
  const size_t quant = D * D + sizeof(Scratch<D, false>);
  if (smem < quant) smem = quant;
  LaunchInfo li;
  cudaError_t e = prepare(chunk_prefill_kernel<D, BF16, KDA>, smem, smem, p.K, cache, li);
  if (e != cudaSuccess) return e;
  chunk_prefill_kernel<D, BF16, KDA><<<p.B * p.Hv, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

template <template <int, bool, bool> class F>
cudaError_t dispatch3(const KParams &p, cudaStream_t s) {
  const bool bf = p.in_bf16 != 0, kda = p.gate != 0;
#define LQ_CASE(DD)                                     \
  if (p.d == DD) {                                      \
    if (bf && kda) return F<DD, true, true>::run(p, s); \
    if (bf) return F<DD, true, false>::run(p, s);       \
    if (kda) return F<DD, false, true>::run(p, s);      \
    return F<DD, false, false>::run(p, s);              \
  }
  LQ_CASE(32)
  LQ_CASE(64)
  LQ_CASE(128)
#undef LQ_CASE
  return cudaErrorInvalidValue;
}

template <int D, bool BF, bool KDA>
struct DecodeF {
  static cudaError_t run(const KParams &p, cudaStream_t s) {
    // windows above kMaxWindow tokens run on the per-tile kernel
    if (p.W > kMaxWindow) return tokens_t<D, BF, KDA>(p, s);
    return decode_t<D, BF, KDA>(p, s);
  }
};
template <int D, bool BF, bool KDA>
struct TokensF {
  static cudaError_t run(const KParams &p, cudaStream_t s) { return tokens_t<D, BF, KDA>(p, s); }
};
template <int D, bool BF, bool KDA>
struct FlushF {
  static cudaError_t run(const KParams &p, cudaStream_t s) { return fold_t<D, BF, KDA, 0>(p, s); }
};
template <int D, bool BF, bool KDA>
struct DequantF {
  static cudaError_t run(const KParams &p, cudaStream_t s) { return fold_t<D, BF, KDA, 1>(p, s); }
};
template <int D, bool BF, bool KDA>
struct PrefillF {
  static cudaError_t run(const KParams &p, cudaStream_t s) { return prefill_t<D, BF, KDA>(p, s); }
};

}  // namespace

cudaError_t launch_decode(const KParams &p, cudaStream_t s) { return dispatch3<DecodeF>(p, s); }
cudaError_t launch_decode_tokens(const KParams &p, cudaStream_t s) {
  return dispatch3<TokensF>(p, s);
}
cudaError_t launch_flush(const KParams &p, cudaStream_t s) { return dispatch3<FlushF>(p, s); }
cudaError_t launch_dequantize(const KParams &p, cudaStream_t s) {
  return dispatch3<DequantF>(p, s);
}
cudaError_t launch_prefill(const KParams &p, cudaStream_t s) { return dispatch3<PrefillF>(p, s); }
cudaError_t launch_init(const KParams &p, cudaStream_t s) {
  if (p.d == 32) return init_t<32>(p, s);
  if (p.d == 64) return init_t<64>(p, s);
  if (p.d == 128) return init_t<128>(p, s);
  return cudaErrorInvalidValue;
}

}  // namespace lq
