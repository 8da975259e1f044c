// Kernels of the LeapQuant int8-state GDN/KDA decode step for sm_100a.
//
// One CTA per state tile (sequence b, value head h).  A tile's window-base
// state S0 = diag(sigma) Q diag(m) + compensator lines is read as stored
// (int8 codes, 16-byte coalesced loads straight into registers); nothing is
// dequantized to memory.  Per token the CTA computes the two products
// y_q = S0 (Gamma o q) and y_k = S0 (Gamma o k) in one pass over the codes,
// combines them with the buffered tokens of the window, writes o_t and
// appends (k_t, d_t, alpha_t).  On the W-th token the same CTA folds the
// buffer into an fp32 copy of the state held in registers, extracts the
// compensator lines, smooths and requantizes, and writes the new record.
//
// Method sources (page title, section): zhichai.net summary "LeapQuant:
// Training-Free 8-bit Quantization for Linear Attention Recurrent States",
// "Abstract (translated)" items 1-3; opentrain.ai "LeapQuant: Efficient
// Linear Attention with Accurate Recurrent State Quantization", "Abstract";
// globaltechnewsdesk news article on LeapQuant, paragraphs 3-5.
//
// Quantizer decisions are taken with correctly rounded fp32 operations
// (__fmul_rn, __fdiv_rn, __frcp_rn, __fsqrt_rn, round-half-even) and fp64 line
// energies, so that a given fp32 state always yields the same record.

#include <cfloat>
#include <cstdint>

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

// Thread geometry of the int8 kernels.  Each state row of d int8 codes is
// covered by LPR lanes holding 16 consecutive codes each (one 16-byte load),
// a warp covers RPW rows per pass, the CTA covers RPP rows per pass and P
// passes cover the tile.  Thread (warp, lane) owns rows p*RPP + warp*RPW +
// lane/LPR and columns c0 = 16*(lane % LPR) .. c0+15.
template <int D>
struct Geo {
  static constexpr int NT = (D * D / 16 < 256) ? D * D / 16 : 256;
  static constexpr int LPR = D / 16;
  static constexpr int RPW = 32 / LPR;
  static constexpr int NWARP = NT / 32;
  static constexpr int RPP = NWARP * RPW;
  static constexpr int P = D / RPP;
  // Column-indexed vectors read as 16-float chunks are stored with 4 floats of
  // padding per chunk, so that the 8 chunks a warp phase reads start in
  // distinct bank groups.
  static constexpr int PADW = D + D / 4;
  static_assert(P * RPP == D, "rows must tile the state");
  static_assert(NT >= 2 * D, "one thread per line of the state");
};

__device__ __forceinline__ int padc(int j) { return j + ((j >> 4) << 2); }

// Quantizer scratch.
template <int D>
struct QScratch {
  double rowE[D];
  double colE[D];
  double colpart[Geo<D>::NWARP][D];
  float colmax[Geo<D>::NWARP][D];
  alignas(16) float invm[Geo<D>::PADW];
  int taken[2 * D];
  int pick;
};

// Shared memory of the decode / flush / dequantize kernels.
template <int D, bool KDA>
struct Smem {
  alignas(16) float q[D];
  alignas(16) float k[D];
  alignas(16) float v[D];
  alignas(16) float acur[KDA ? D : 1];  // gate of the current token
  alignas(16) float G[D];               // window gate Gamma per key channel
  alignas(16) float sig[D];
  alignas(16) float m[D];
  alignas(16) float gq[D];              // Gamma o q
  alignas(16) float gk[D];              // Gamma o k
  alignas(16) float xq[Geo<D>::PADW];   // m o Gamma o q (padded)
  alignas(16) float xk[Geo<D>::PADW];   // m o Gamma o k (padded)
  alignas(16) float mG[Geo<D>::PADW];   // m o Gamma (padded)
  alignas(16) float bk[kMaxWindow][Geo<D>::PADW];  // buffered keys times decay ratios
  alignas(16) float bd[kMaxWindow][D];             // buffered deltas
  alignas(16) float ba[kMaxWindow][KDA ? D : 1];   // buffered gates
  alignas(16) float cv[kMaxComp][D];
  int cid[kMaxComp];
  alignas(16) float yq[D];
  alignas(16) float yk[D];
  float cc[kMaxWindow + 1];
  float aa[kMaxWindow + 1];
  float cdot[kMaxComp][2];
  float beta;
  QScratch<D> qs;
};

template <bool BF16>
__device__ __forceinline__ float ld_in(const void *p, size_t i) {
  if constexpr (BF16)
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
  else
    return reinterpret_cast<const float *>(p)[i];
}

// Stores a value that was read in the same dtype (exact).
template <bool BF16>
__device__ __forceinline__ void st_in(void *p, size_t i, float x) {
  if constexpr (BF16)
    reinterpret_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(x);
  else
    reinterpret_cast<float *>(p)[i] = x;
}

__device__ __forceinline__ void st_out(void *p, size_t i, float x, int bf16) {
  if (bf16)
    reinterpret_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(x);
  else
    reinterpret_cast<float *>(p)[i] = x;
}

__device__ __forceinline__ float code_at(const uint4 &c, int e) {
  const uint32_t w = (e < 4) ? c.x : (e < 8) ? c.y : (e < 12) ? c.z : c.w;
  return static_cast<float>(static_cast<int8_t>(w >> (8 * (e & 3))));
}

__device__ __forceinline__ void load16(const float *src, float (&dst)[16]) {
  const float4 *s4 = reinterpret_cast<const float4 *>(src);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float4 t = s4[u];
    dst[4 * u + 0] = t.x;
    dst[4 * u + 1] = t.y;
    dst[4 * u + 2] = t.z;
    dst[4 * u + 3] = t.w;
  }
}

template <int D>
__device__ __forceinline__ const uint8_t *rec_ptr(const KParams &p, int tile) {
  return p.records + static_cast<size_t>(tile) * p.L.bytes;
}

// Loads a tile's record (codes into registers, the rest into shared memory)
// and its n buffered tokens into shared memory.  Buffered keys go to bk with
// padded columns; gates to ba.
template <int D, bool BF16, bool KDA>
__device__ __forceinline__ void load_tile(const KParams &p, Smem<D, KDA> &s, int tile, int b,
                                          int hk, int n, uint4 (&codes)[Geo<D>::P]) {
  using G = Geo<D>;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r_in = warp * G::RPW + lane / G::LPR;
  const int c0 = (lane % G::LPR) * 16;
  const uint8_t *rec = rec_ptr<D>(p, tile);
#pragma unroll
  for (int pp = 0; pp < G::P; ++pp)
    codes[pp] = __ldcs(reinterpret_cast<const uint4 *>(
        rec + static_cast<size_t>(pp * G::RPP + r_in) * D + c0));
  const float *rsig = reinterpret_cast<const float *>(rec + p.L.off_sig);
  const float *rm = reinterpret_cast<const float *>(rec + p.L.off_m);
  const float *rcv = reinterpret_cast<const float *>(rec + p.L.off_cv);
  const int *rcid = reinterpret_cast<const int *>(rec + p.L.off_cid);
  if (tid < D) {
    s.sig[tid] = rsig[tid];
    s.m[tid] = rm[tid];
  }
  for (int idx = tid; idx < p.K * D; idx += G::NT) s.cv[idx / D][idx % D] = rcv[idx];
  if (tid < p.K) s.cid[tid] = rcid[tid];
  const size_t bk_base = (static_cast<size_t>(b) * p.Hk + hk) * p.W * D;
  const size_t bd_base = static_cast<size_t>(tile) * p.W * D;
  for (int idx = tid; idx < n * D; idx += G::NT) {
    const int sl = idx / D, j = idx - sl * D;
    s.bk[sl][padc(j)] = ld_in<BF16>(p.buf_k, bk_base + idx);
    s.bd[sl][j] = p.buf_d[bd_base + idx];
    if constexpr (KDA) s.ba[sl][j] = p.buf_g[bd_base + idx];
  }
  if constexpr (!KDA) {
    if (tid < n) s.ba[tid][0] = p.buf_g[static_cast<size_t>(tile) * p.W + tid];
  }
}

// Dense fp32 state of the thread's P x 16 block:
//   S_ij = sigma_i code_ij (m_j Gamma_j) + sum_{s < nent} d_s[i] kt_s[j]
//          + compensator lines times Gamma,
// with kt_s = k_s o (decay ratio to the last token) already in s.bk and
// m o Gamma in s.mG.
template <int D, bool KDA>
__device__ __forceinline__ void build_state(const Smem<D, KDA> &s, const uint4 (&codes)[Geo<D>::P],
                                            int nent, int K, float (&Sv)[Geo<D>::P][16]) {
  using G = Geo<D>;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r_in = warp * G::RPW + lane / G::LPR;
  const int c0 = (lane % G::LPR) * 16;
  float mg[16];
  load16(&s.mG[padc(c0)], mg);
#pragma unroll
  for (int pp = 0; pp < G::P; ++pp) {
    const float sg = s.sig[pp * G::RPP + r_in];
#pragma unroll
    for (int e = 0; e < 16; ++e) Sv[pp][e] = sg * code_at(codes[pp], e) * mg[e];
  }
  for (int sl = 0; sl < nent; ++sl) {
    float kt[16];
    load16(&s.bk[sl][padc(c0)], kt);
#pragma unroll
    for (int pp = 0; pp < G::P; ++pp) {
      const float dd = s.bd[sl][pp * G::RPP + r_in];
#pragma unroll
      for (int e = 0; e < 16; ++e) Sv[pp][e] = fmaf(dd, kt[e], Sv[pp][e]);
    }
  }
  for (int c = 0; c < K; ++c) {
    const int id = s.cid[c];
    if (id < D) {
#pragma unroll
      for (int pp = 0; pp < G::P; ++pp)
        if (pp * G::RPP + r_in == id) {
#pragma unroll
          for (int e = 0; e < 16; ++e)
            Sv[pp][e] = fmaf(s.cv[c][c0 + e], s.G[c0 + e], Sv[pp][e]);
        }
    } else {
      const int jc = id - D;
      const float gj = s.G[jc];
#pragma unroll
      for (int pp = 0; pp < G::P; ++pp)
#pragma unroll
        for (int e = 0; e < 16; ++e)
          if (c0 + e == jc) Sv[pp][e] = fmaf(s.cv[c][pp * G::RPP + r_in], gj, Sv[pp][e]);
    }
  }
}

// Quantize the fp32 state held in registers (every thread of the CTA holds
// its P x 16 block) and write the tile record at rec:
//  1. K times: line energies (fp64) of the residual's rows and columns, the
//     highest untaken line wins (ties: lower id, rows before columns), its
//     values are stored as a compensator vector and zeroed;
//  2. m_j from the column max a_j of the residual (1 if a_j < FLT_MIN or
//     smoothing is off; sqrt(a_j) or a_j otherwise);
//  3. per row: x = (R_ij * (1/m_j)) * (127/b_i) with b_i the row max, codes =
//     round-half-even(x) clamped to [-127, 127], sigma_i = b_i / 127
//     (sigma_i = 1 and zero codes if b_i < FLT_MIN).
template <int D>
__device__ void quantize_tile(QScratch<D> &qs, float (&Sv)[Geo<D>::P][16], uint8_t *rec,
                              const RecLayout &L, int K, int smooth) {
  using G = Geo<D>;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r_in = warp * G::RPW + lane / G::LPR;
  const int c0 = (lane % G::LPR) * 16;
  float *rsig = reinterpret_cast<float *>(rec + L.off_sig);
  float *rm = reinterpret_cast<float *>(rec + L.off_m);
  float *rcv = reinterpret_cast<float *>(rec + L.off_cv);
  int *rcid = reinterpret_cast<int *>(rec + L.off_cid);

  if (tid < 2 * D) qs.taken[tid] = 0;
  bool need_rows = true, need_cols = true;
  __syncthreads();
  for (int c = 0; c < K; ++c) {
    if (need_rows) {
#pragma unroll
      for (int pp = 0; pp < G::P; ++pp) {
        double e = 0.0;
#pragma unroll
        for (int u = 0; u < 16; ++u) e = fma(static_cast<double>(Sv[pp][u]),
                                             static_cast<double>(Sv[pp][u]), e);
#pragma unroll
        for (int o = 1; o < G::LPR; o <<= 1) e += __shfl_xor_sync(kFull, e, o);
        if ((lane % G::LPR) == 0) qs.rowE[pp * G::RPP + r_in] = e;
      }
    }
    if (need_cols) {
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        double e = 0.0;
#pragma unroll
        for (int pp = 0; pp < G::P; ++pp)
          e = fma(static_cast<double>(Sv[pp][u]), static_cast<double>(Sv[pp][u]), e);
#pragma unroll
        for (int o = G::LPR; o < 32; o <<= 1) e += __shfl_xor_sync(kFull, e, o);
        if (lane < G::LPR) qs.colpart[warp][c0 + u] = e;
      }
    }
    __syncthreads();
    if (need_cols && tid < D) {
      double e = 0.0;
#pragma unroll
      for (int w = 0; w < G::NWARP; ++w) e += qs.colpart[w][tid];
      qs.colE[tid] = e;
    }
    __syncthreads();
    if (warp == 0) {
      double best = -1.0;
      int bid = 0x7fffffff;
      for (int id = lane; id < 2 * D; id += 32) {
        if (qs.taken[id]) continue;
        const double e = (id < D) ? qs.rowE[id] : qs.colE[id - D];
        if (e > best || (e == best && id < bid)) {
          best = e;
          bid = id;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double ob = __shfl_xor_sync(kFull, best, o);
        const int oid = __shfl_xor_sync(kFull, bid, o);
        if (ob > best || (ob == best && oid < bid)) {
          best = ob;
          bid = oid;
        }
      }
      if (lane == 0) {
        qs.pick = bid;
        qs.taken[bid] = 1;
        rcid[c] = bid;
      }
    }
    __syncthreads();
    const int id = qs.pick;
    if (id < D) {
#pragma unroll
      for (int pp = 0; pp < G::P; ++pp)
        if (pp * G::RPP + r_in == id) {
          float4 *dst = reinterpret_cast<float4 *>(rcv + c * D + c0);
#pragma unroll
          for (int u = 0; u < 4; ++u)
            dst[u] = make_float4(Sv[pp][4 * u], Sv[pp][4 * u + 1], Sv[pp][4 * u + 2],
                                 Sv[pp][4 * u + 3]);
#pragma unroll
          for (int u = 0; u < 16; ++u) Sv[pp][u] = 0.0f;
        }
      need_rows = false;
      need_cols = true;
    } else {
      const int jc = id - D;
#pragma unroll
      for (int pp = 0; pp < G::P; ++pp)
#pragma unroll
        for (int u = 0; u < 16; ++u)
          if (c0 + u == jc) {
            rcv[c * D + pp * G::RPP + r_in] = Sv[pp][u];
            Sv[pp][u] = 0.0f;
          }
      need_rows = true;
      need_cols = false;
    }
  }

  // Smoothing factors from the residual's column maxima.
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    float cm = 0.0f;
#pragma unroll
    for (int pp = 0; pp < G::P; ++pp) cm = fmaxf(cm, fabsf(Sv[pp][u]));
#pragma unroll
    for (int o = G::LPR; o < 32; o <<= 1) cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, o));
    if (lane < G::LPR) qs.colmax[warp][c0 + u] = cm;
  }
  __syncthreads();
  if (tid < D) {
    float a = 0.0f;
#pragma unroll
    for (int w = 0; w < G::NWARP; ++w) a = fmaxf(a, qs.colmax[w][tid]);
    float mj;
    if (smooth == 0 || a < FLT_MIN)
      mj = 1.0f;
    else if (smooth == 1)
      mj = __fsqrt_rn(a);
    else
      mj = a;
    rm[tid] = mj;
    qs.invm[padc(tid)] = __frcp_rn(mj);
  }
  __syncthreads();

  // Per-row scales and int8 codes.
  float im[16];
  load16(&qs.invm[padc(c0)], im);
#pragma unroll
  for (int pp = 0; pp < G::P; ++pp) {
    const int row = pp * G::RPP + r_in;
    float bmax = 0.0f;
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      Sv[pp][u] = __fmul_rn(Sv[pp][u], im[u]);
      bmax = fmaxf(bmax, fabsf(Sv[pp][u]));
    }
#pragma unroll
    for (int o = 1; o < G::LPR; o <<= 1) bmax = fmaxf(bmax, __shfl_xor_sync(kFull, bmax, o));
    float sg, inv;
    if (bmax < FLT_MIN) {
      sg = 1.0f;
      inv = 0.0f;
    } else {
      sg = __fdiv_rn(bmax, 127.0f);
      inv = __fdiv_rn(127.0f, bmax);
    }
    if ((lane % G::LPR) == 0) rsig[row] = sg;
    uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      int qv = __float2int_rn(__fmul_rn(Sv[pp][u], inv));
      qv = max(-127, min(127, qv));
      w[u >> 2] |= (static_cast<uint32_t>(qv) & 0xffu) << (8 * (u & 3));
    }
    *reinterpret_cast<uint4 *>(rec + static_cast<size_t>(row) * D + c0) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// ---------------------------------------------------------------------------
// Decode step
// ---------------------------------------------------------------------------

template <int D, bool BF16, bool KDA>
__global__ void __launch_bounds__(Geo<D>::NT) decode_kernel(const KParams p) {
  using G = Geo<D>;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem<D, KDA> &s = *reinterpret_cast<Smem<D, KDA> *>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tile = blockIdx.x;
  const int b = tile / p.Hv, h = tile - b * p.Hv;
  const int group = p.Hv / p.Hk;
  const int hk = h / group;
  if (p.mask != nullptr && p.mask[b] == 0) return;
  const int n = p.buf_n[tile];
  if (n < 0 || n >= p.W) {
    if (tid == 0) atomicOr(p.err, kErrBadPhase);
    return;
  }
  const int r_in = warp * G::RPW + lane / G::LPR;
  const int c0 = (lane % G::LPR) * 16;

  uint4 codes[G::P];
  load_tile<D, BF16, KDA>(p, s, tile, b, hk, n, codes);
  const size_t qk_base = (static_cast<size_t>(b) * p.Hk + hk) * D;
  if (tid < D) {
    s.q[tid] = ld_in<BF16>(p.q, qk_base + tid);
    s.k[tid] = ld_in<BF16>(p.k, qk_base + tid);
    s.v[tid] = ld_in<BF16>(p.v, static_cast<size_t>(tile) * D + tid);
    if constexpr (KDA) s.acur[tid] = p.alpha[static_cast<size_t>(tile) * D + tid];
  }
  if (tid == 0) {
    s.beta = p.beta[tile];
    if constexpr (!KDA) s.acur[0] = p.alpha[tile];
  }
  __syncthreads();

  // Decay ratios prod_{s < s' <= t} alpha_{s'} (running products from the
  // current token backwards) applied to the buffered keys, and the window
  // gate Gamma_t.
  if (tid < D) {
    const int j = tid;
    float acc = KDA ? s.acur[j] : s.acur[0];
    for (int sl = n - 1; sl >= 0; --sl) {
      s.bk[sl][padc(j)] *= acc;
      acc *= KDA ? s.ba[sl][j] : s.ba[sl][0];
    }
    s.G[j] = acc;
    const float gq = acc * s.q[j], gk = acc * s.k[j];
    s.gq[j] = gq;
    s.gk[j] = gk;
    s.xq[padc(j)] = s.m[j] * gq;
    s.xk[padc(j)] = s.m[j] * gk;
    s.mG[padc(j)] = s.m[j] * acc;
  }
  __syncthreads();

  // y_q = S0 (Gamma o q), y_k = S0 (Gamma o k): one pass over the codes.
  {
    float xq[16], xk[16];
    load16(&s.xq[padc(c0)], xq);
    load16(&s.xk[padc(c0)], xk);
#pragma unroll
    for (int pp = 0; pp < G::P; ++pp) {
      float aq = 0.0f, ak = 0.0f;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float c = code_at(codes[pp], e);
        aq = fmaf(c, xq[e], aq);
        ak = fmaf(c, xk[e], ak);
      }
#pragma unroll
      for (int o = 1; o < G::LPR; o <<= 1) {
        aq += __shfl_xor_sync(kFull, aq, o);
        ak += __shfl_xor_sync(kFull, ak, o);
      }
      if ((lane % G::LPR) == 0) {
        const int row = pp * G::RPP + r_in;
        s.yq[row] = s.sig[row] * aq;
        s.yk[row] = s.sig[row] * ak;
      }
    }
  }
  // c_s = kt_s . k and a_s = kt_s . q for the buffered tokens; a_t = k . q.
  for (int sl = warp; sl <= n; sl += G::NWARP) {
    float c = 0.0f, a = 0.0f;
    for (int j = lane; j < D; j += 32) {
      const float kt = (sl < n) ? s.bk[sl][padc(j)] : s.k[j];
      c = fmaf(kt, s.k[j], c);
      a = fmaf(kt, s.q[j], a);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      c += __shfl_xor_sync(kFull, c, o);
      a += __shfl_xor_sync(kFull, a, o);
    }
    if (lane == 0) {
      s.cc[sl] = c;
      s.aa[sl] = a;
    }
  }
  // Row compensators: their line dotted with Gamma o q and Gamma o k.
  for (int c = warp; c < p.K; c += G::NWARP) {
    if (s.cid[c] < D) {
      float dq = 0.0f, dk = 0.0f;
      for (int j = lane; j < D; j += 32) {
        dq = fmaf(s.cv[c][j], s.gq[j], dq);
        dk = fmaf(s.cv[c][j], s.gk[j], dk);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        dq += __shfl_xor_sync(kFull, dq, o);
        dk += __shfl_xor_sync(kFull, dk, o);
      }
      if (lane == 0) {
        s.cdot[c][0] = dq;
        s.cdot[c][1] = dk;
      }
    }
  }
  __syncthreads();

  // d_t = beta (v - y_k - sum c_s d_s); o_t = y_q + sum a_s d_s + a_t d_t.
  const size_t bd_base = static_cast<size_t>(tile) * p.W * D;
  if (tid < D) {
    const int i = tid;
    float yq = s.yq[i], yk = s.yk[i];
    for (int c = 0; c < p.K; ++c) {
      const int id = s.cid[c];
      if (id == i) {
        yq += s.cdot[c][0];
        yk += s.cdot[c][1];
      } else if (id >= D) {
        yq = fmaf(s.cv[c][i], s.gq[id - D], yq);
        yk = fmaf(s.cv[c][i], s.gk[id - D], yk);
      }
    }
    float x = s.v[i] - yk;
    float o = yq;
    for (int sl = 0; sl < n; ++sl) {
      const float dsl = s.bd[sl][i];
      x = fmaf(-s.cc[sl], dsl, x);
      o = fmaf(s.aa[sl], dsl, o);
    }
    const float dt = s.beta * x;
    o = fmaf(s.aa[n], dt, o);
    st_out(p.out, static_cast<size_t>(tile) * D + i, o, p.out_bf16);
    p.buf_d[bd_base + static_cast<size_t>(n) * D + i] = dt;
    s.bd[n][i] = dt;
    s.bk[n][padc(i)] = s.k[i];
    if (h % group == 0)
      st_in<BF16>(p.buf_k, (static_cast<size_t>(b) * p.Hk + hk) * p.W * D +
                               static_cast<size_t>(n) * D + i, s.k[i]);
    if constexpr (KDA) p.buf_g[bd_base + static_cast<size_t>(n) * D + i] = s.acur[i];
  }
  if constexpr (!KDA) {
    if (tid == 0) p.buf_g[static_cast<size_t>(tile) * p.W + n] = s.acur[0];
  }
  if (n + 1 < p.W) {
    if (tid == 0) p.buf_n[tile] = n + 1;
    return;
  }

  // Window boundary: fold the W buffered tokens and requantize.
  __syncthreads();
  float Sv[G::P][16];
  build_state<D, KDA>(s, codes, n + 1, p.K, Sv);
  quantize_tile<D>(s.qs, Sv, p.records + static_cast<size_t>(tile) * p.L.bytes, p.L, p.K,
                   p.smooth);
  if (tid == 0) p.buf_n[tile] = 0;
}

// ---------------------------------------------------------------------------
// Flush (fold a partial window) and dequantize
// ---------------------------------------------------------------------------

// mode 0: flush selected tiles with 0 < n < W; mode 1: write the fp32 state.
template <int D, bool BF16, bool KDA, int MODE>
__global__ void __launch_bounds__(Geo<D>::NT) fold_kernel(const KParams p) {
  using G = Geo<D>;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem<D, KDA> &s = *reinterpret_cast<Smem<D, KDA> *>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tile = blockIdx.x;
  const int b = tile / p.Hv, h = tile - b * p.Hv;
  const int hk = h / (p.Hv / p.Hk);
  if (MODE == 0 && p.mask != nullptr && p.mask[b] == 0) return;
  int n = p.buf_n[tile];
  if (n < 0 || n >= p.W) {
    if (tid == 0) atomicOr(p.err, kErrBadPhase);
    return;
  }
  if (MODE == 0 && n == 0) return;
  if (MODE == 1 && !p.include_buffer) n = 0;
  uint4 codes[G::P];
  load_tile<D, BF16, KDA>(p, s, tile, b, hk, n, codes);
  __syncthreads();
  if (tid < D) {
    const int j = tid;
    float acc = 1.0f;
    for (int sl = n - 1; sl >= 0; --sl) {
      s.bk[sl][padc(j)] *= acc;
      acc *= KDA ? s.ba[sl][j] : s.ba[sl][0];
    }
    s.G[j] = acc;
    s.mG[padc(j)] = s.m[j] * acc;
  }
  __syncthreads();
  float Sv[G::P][16];
  build_state<D, KDA>(s, codes, n, p.K, Sv);
  if constexpr (MODE == 0) {
    quantize_tile<D>(s.qs, Sv, p.records + static_cast<size_t>(tile) * p.L.bytes, p.L, p.K,
                     p.smooth);
    if (tid == 0) p.buf_n[tile] = 0;
  } else {
    const int r_in = warp * G::RPW + lane / G::LPR;
    const int c0 = (lane % G::LPR) * 16;
    float *dst = p.S_out + static_cast<size_t>(tile) * D * D;
#pragma unroll
    for (int pp = 0; pp < G::P; ++pp) {
      float4 *row = reinterpret_cast<float4 *>(dst + static_cast<size_t>(pp * G::RPP + r_in) * D + c0);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        row[u] = make_float4(Sv[pp][4 * u], Sv[pp][4 * u + 1], Sv[pp][4 * u + 2], Sv[pp][4 * u + 3]);
    }
  }
}

// ---------------------------------------------------------------------------
// Init: quantize given fp32 states
// ---------------------------------------------------------------------------

template <int D>
__global__ void __launch_bounds__(Geo<D>::NT) init_kernel(const KParams p) {
  using G = Geo<D>;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  QScratch<D> &qs = *reinterpret_cast<QScratch<D> *>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tile = blockIdx.x;
  const int b = tile / p.Hv;
  if (p.mask != nullptr && p.mask[b] == 0) return;
  const int r_in = warp * G::RPW + lane / G::LPR;
  const int c0 = (lane % G::LPR) * 16;
  const float *src = p.S_in + static_cast<size_t>(tile) * D * D;
  float Sv[G::P][16];
#pragma unroll
  for (int pp = 0; pp < G::P; ++pp) {
    const float4 *row =
        reinterpret_cast<const float4 *>(src + static_cast<size_t>(pp * G::RPP + r_in) * D + c0);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float4 t = __ldcs(row + u);
      Sv[pp][4 * u] = t.x;
      Sv[pp][4 * u + 1] = t.y;
      Sv[pp][4 * u + 2] = t.z;
      Sv[pp][4 * u + 3] = t.w;
    }
  }
  quantize_tile<D>(qs, Sv, p.records + static_cast<size_t>(tile) * p.L.bytes, p.L, p.K, p.smooth);
  if (tid == 0) p.buf_n[tile] = 0;
}

// ---------------------------------------------------------------------------
// fp32-state comparison path
// ---------------------------------------------------------------------------

// TPR lanes per row, 4 consecutive fp32 columns per lane (one 16-byte load);
// the CTA covers RPI rows per pass and NP passes cover the tile.
template <int D>
struct F32Geo {
  static constexpr int NT = (D >= 64) ? 256 : 64;
  static constexpr int TPR = D / 4;
  static constexpr int RPI = NT / TPR;
  static constexpr int NP = D / RPI;
  static_assert(NP * RPI == D, "rows must tile the state");
};

template <int D, bool BF16, bool KDA>
__global__ void __launch_bounds__(F32Geo<D>::NT) fp32_step_kernel(const KParams p, float *S) {
  using G = F32Geo<D>;
  __shared__ alignas(16) float sq[D];
  __shared__ alignas(16) float sk[D];
  __shared__ alignas(16) float sa[KDA ? D : 1];
  __shared__ float sbeta, skq;
  const int tid = threadIdx.x, lane = tid & 31;
  const int tile = blockIdx.x;
  const int b = tile / p.Hv, h = tile - b * p.Hv;
  const int hk = h / (p.Hv / p.Hk);
  const int rsub = tid / G::TPR;
  const int col = (tid % G::TPR) * 4;
  float *St = S + static_cast<size_t>(tile) * D * D;
  float4 sv[G::NP];
#pragma unroll
  for (int pp = 0; pp < G::NP; ++pp)
    sv[pp] = __ldcs(reinterpret_cast<const float4 *>(St + static_cast<size_t>(pp * G::RPI + rsub) * D + col));
  const size_t qk_base = (static_cast<size_t>(b) * p.Hk + hk) * D;
  if (tid < D) {
    sq[tid] = ld_in<BF16>(p.q, qk_base + tid);
    sk[tid] = ld_in<BF16>(p.k, qk_base + tid);
    if constexpr (KDA) sa[tid] = p.alpha[static_cast<size_t>(tile) * D + tid];
  }
  if (tid == 0) {
    sbeta = p.beta[tile];
    if constexpr (!KDA) sa[0] = p.alpha[tile];
  }
  __syncthreads();
  if (tid < 32) {
    float kq = 0.0f;
    for (int j = lane; j < D; j += 32) kq = fmaf(sk[j], sq[j], kq);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) kq += __shfl_xor_sync(kFull, kq, o);
    if (lane == 0) skq = kq;
  }
  const float4 k4 = *reinterpret_cast<const float4 *>(&sk[col]);
  const float4 q4 = *reinterpret_cast<const float4 *>(&sq[col]);
  float4 a4;
  if constexpr (KDA)
    a4 = *reinterpret_cast<const float4 *>(&sa[col]);
  else
    a4 = make_float4(sa[0], sa[0], sa[0], sa[0]);
  // S' = S diag(alpha); e = S' k, f = S' q per row.
  float e[G::NP], f[G::NP];
#pragma unroll
  for (int pp = 0; pp < G::NP; ++pp) {
    sv[pp].x *= a4.x;
    sv[pp].y *= a4.y;
    sv[pp].z *= a4.z;
    sv[pp].w *= a4.w;
    e[pp] = fmaf(sv[pp].x, k4.x, fmaf(sv[pp].y, k4.y, fmaf(sv[pp].z, k4.z, sv[pp].w * k4.w)));
    f[pp] = fmaf(sv[pp].x, q4.x, fmaf(sv[pp].y, q4.y, fmaf(sv[pp].z, q4.z, sv[pp].w * q4.w)));
  }
  __syncthreads();
  const float beta = sbeta, kq = skq;
  const size_t out_base = static_cast<size_t>(tile) * D;
  if constexpr (G::TPR == 32) {
    // Transposing butterfly: 2*NP = 32 partial sums per lane reduced across the
    // warp in 31 shuffles; afterwards lane l holds the total of value l
    // (rows' e for l < 16, rows' f for l >= 16).
    static_assert(G::NP == 16, "one warp per 16 rows");
    float vals[32];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      vals[i] = e[i];
      vals[16 + i] = f[i];
    }
#pragma unroll
    for (int step = 16; step >= 1; step >>= 1) {
      const bool upper = (lane & step) != 0;
#pragma unroll
      for (int i = 0; i < step; ++i) {
        const float send = upper ? vals[i] : vals[i + step];
        const float keep = upper ? vals[i + step] : vals[i];
        vals[i] = keep + __shfl_xor_sync(kFull, send, step);
      }
    }
    const int warp = tid >> 5;
    const int myrow = (lane & 15) * G::RPI + warp;
    // lane l < 16: delta of its row; lane l >= 16: output of row l - 16.
    float delta = 0.0f;
    if (lane < 16) delta = beta * (ld_in<BF16>(p.v, out_base + myrow) - vals[0]);
    const float dl = __shfl_sync(kFull, delta, lane & 15);
    if (lane >= 16) st_out(p.out, out_base + myrow, fmaf(dl, kq, vals[0]), p.out_bf16);
#pragma unroll
    for (int pp = 0; pp < G::NP; ++pp) {
      const float dd = __shfl_sync(kFull, delta, pp);
      sv[pp].x = fmaf(dd, k4.x, sv[pp].x);
      sv[pp].y = fmaf(dd, k4.y, sv[pp].y);
      sv[pp].z = fmaf(dd, k4.z, sv[pp].z);
      sv[pp].w = fmaf(dd, k4.w, sv[pp].w);
      __stcs(reinterpret_cast<float4 *>(St + static_cast<size_t>(pp * G::RPI + rsub) * D + col), sv[pp]);
    }
  } else {
#pragma unroll
    for (int pp = 0; pp < G::NP; ++pp) {
      float ee = e[pp], ff = f[pp];
#pragma unroll
      for (int o = 1; o < G::TPR; o <<= 1) {
        ee += __shfl_xor_sync(kFull, ee, o);
        ff += __shfl_xor_sync(kFull, ff, o);
      }
      const int row = pp * G::RPI + rsub;
      const float dd = beta * (ld_in<BF16>(p.v, out_base + row) - ee);
      if ((tid % G::TPR) == 0) st_out(p.out, out_base + row, fmaf(dd, kq, ff), p.out_bf16);
      sv[pp].x = fmaf(dd, k4.x, sv[pp].x);
      sv[pp].y = fmaf(dd, k4.y, sv[pp].y);
      sv[pp].z = fmaf(dd, k4.z, sv[pp].z);
      sv[pp].w = fmaf(dd, k4.w, sv[pp].w);
      __stcs(reinterpret_cast<float4 *>(St + static_cast<size_t>(row) * D + col), sv[pp]);
    }
  }
}

// ---------------------------------------------------------------------------
// Launch plumbing
// ---------------------------------------------------------------------------

// Opt a kernel into more than 48 KB of dynamic shared memory, once per device.
template <typename K>
cudaError_t allow_smem(K kernel, size_t bytes, unsigned &done_mask) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned bit = 1u << (dev & 31);
  if (__atomic_load_n(&done_mask, __ATOMIC_ACQUIRE) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bytes));
  if (e == cudaSuccess) __atomic_fetch_or(&done_mask, bit, __ATOMIC_RELEASE);
  return e;
}

template <int D, bool BF16, bool KDA>
cudaError_t decode_t(const KParams &p, cudaStream_t st) {
  static unsigned done = 0;
  const size_t smem = sizeof(Smem<D, KDA>);
  cudaError_t e = allow_smem(decode_kernel<D, BF16, KDA>, smem, done);
  if (e != cudaSuccess) return e;
  decode_kernel<D, BF16, KDA><<<p.B * p.Hv, Geo<D>::NT, smem, st>>>(p);
  return cudaGetLastError();
}

template <int D, bool BF16, bool KDA, int MODE>
cudaError_t fold_t(const KParams &p, cudaStream_t st) {
  static unsigned done = 0;
  const size_t smem = sizeof(Smem<D, KDA>);
  cudaError_t e = allow_smem(fold_kernel<D, BF16, KDA, MODE>, smem, done);
  if (e != cudaSuccess) return e;
  fold_kernel<D, BF16, KDA, MODE><<<p.B * p.Hv, Geo<D>::NT, smem, st>>>(p);
  return cudaGetLastError();
}

template <int D>
cudaError_t init_t(const KParams &p, cudaStream_t st) {
  static unsigned done = 0;
  const size_t smem = sizeof(QScratch<D>);
  cudaError_t e = allow_smem(init_kernel<D>, smem, done);
  if (e != cudaSuccess) return e;
  init_kernel<D><<<p.B * p.Hv, Geo<D>::NT, smem, st>>>(p);
  return cudaGetLastError();
}

template <int D, bool BF16, bool KDA>
cudaError_t fp32_t(const KParams &p, float *S, cudaStream_t st) {
  fp32_step_kernel<D, BF16, KDA><<<p.B * p.Hv, F32Geo<D>::NT, 0, st>>>(p, S);
  return cudaGetLastError();
}

// Dispatch on (d, bf16 inputs, diagonal gate).
template <template <int, bool, bool> class F, typename... A>
cudaError_t dispatch3(const KParams &p, A... a) {
  const bool bf = p.in_bf16 != 0, kda = p.gate != 0;
#define LQ_CASE(D)                                               \
  if (p.d == D) {                                                \
    if (bf && kda) return F<D, true, true>::run(p, a...);        \
    if (bf) return F<D, true, false>::run(p, a...);              \
    if (kda) return F<D, false, true>::run(p, a...);             \
    return F<D, false, false>::run(p, a...);                     \
  }
  LQ_CASE(32)
  LQ_CASE(64)
  LQ_CASE(128)
#undef LQ_CASE
  return cudaErrorInvalidValue;
}

template <int D, bool BF, bool KDA>
struct DecodeF {
  static cudaError_t run(const KParams &p, cudaStream_t s) { return decode_t<D, BF, KDA>(p, s); }
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
struct Fp32F {
  static cudaError_t run(const KParams &p, float *S, cudaStream_t s) {
    return fp32_t<D, BF, KDA>(p, S, s);
  }
};

}  // namespace

cudaError_t launch_decode(const KParams &p, cudaStream_t s) { return dispatch3<DecodeF>(p, s); }
cudaError_t launch_flush(const KParams &p, cudaStream_t s) { return dispatch3<FlushF>(p, s); }
cudaError_t launch_dequantize(const KParams &p, cudaStream_t s) {
  return dispatch3<DequantF>(p, s);
}
cudaError_t launch_fp32_step(const KParams &p, float *S, cudaStream_t s) {
  return dispatch3<Fp32F>(p, S, s);
}
cudaError_t launch_init(const KParams &p, cudaStream_t s) {
  if (p.d == 32) return init_t<32>(p, s);
  if (p.d == 64) return init_t<64>(p, s);
  if (p.d == 128) return init_t<128>(p, s);
  return cudaErrorInvalidValue;
}

}  // namespace lq
