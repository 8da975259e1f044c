// fp32-state comparison path of the GDN/KDA decode step (the FP32-state
// baseline of the opentrain.ai "LeapQuant: Efficient Linear Attention with
// Accurate Recurrent State Quantization" abstract):
//   S <- S diag(alpha);  S <- S + beta (v - S k) k^T;  o = S q,
// with the d x d fp32 state read and written in place, one CTA per tile.

#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "lq_internal.h"

namespace lq {
namespace {

constexpr unsigned kFull = 0xffffffffu;

template <bool BF16>
__device__ __forceinline__ float ld_in(const void *p, size_t i) {
  if constexpr (BF16)
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
  else
    return reinterpret_cast<const float *>(p)[i];
}

__device__ __forceinline__ void st_out(void *p, size_t i, float x, int bf16) {
  if (bf16)
    reinterpret_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(x);
  else
    reinterpret_cast<float *>(p)[i] = x;
}

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

template <int D, bool BF16, bool KDA>
cudaError_t fp32_t(const KParams &p, float *S, cudaStream_t st) {
  fp32_step_kernel<D, BF16, KDA><<<p.B * p.Hv, F32Geo<D>::NT, 0, st>>>(p, S);
  return cudaGetLastError();
}

template <int D>
cudaError_t fp32_d(const KParams &p, float *S, cudaStream_t st) {
  const bool bf = p.in_bf16 != 0, kda = p.gate != 0;
  if (bf && kda) return fp32_t<D, true, true>(p, S, st);
  if (bf) return fp32_t<D, true, false>(p, S, st);
  if (kda) return fp32_t<D, false, true>(p, S, st);
  return fp32_t<D, false, false>(p, S, st);
}

}  // namespace

cudaError_t launch_fp32_step(const KParams &p, float *S, cudaStream_t s) {
  if (p.d == 32) return fp32_d<32>(p, S, s);
  if (p.d == 64) return fp32_d<64>(p, S, s);
  if (p.d == 128) return fp32_d<128>(p, S, s);
  return cudaErrorInvalidValue;
}

}  // namespace lq
