// Device building blocks of the WTConv kernels (sm_100a).
//
// Register-tiled depthwise convolution and weight-gradient correlation
// from shared memory, the Haar analysis butterfly and the synthesis
// butterfly.  Layer definition: arXiv:2608.10805 (I/O-aware reformulation of
// wavelet convolution), abstract.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace wt {

// ---------------------------------------------------------------- I/O types
template <typename IO> struct io_traits;
template <> struct io_traits<float> {
  static __device__ __forceinline__ float to_f(float v) { return v; }
  static __device__ __forceinline__ float from_f(float v) { return v; }
};
template <> struct io_traits<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

// Loads 4 consecutive elements starting at p (element index x of a row with
// `w` valid elements).  `vec` says the 4-element group is aligned for one
// vector load and fully valid; otherwise the loads are scalar and elements
// at x+e >= w read as zero.
__device__ __forceinline__ float4 load4(const float* __restrict__ p, int x, int w, bool vec) {
  if (vec && x + 3 < w) return __ldg(reinterpret_cast<const float4*>(p));
  float4 t;
  t.x = (x + 0 < w) ? __ldg(p + 0) : 0.f;
  t.y = (x + 1 < w) ? __ldg(p + 1) : 0.f;
  t.z = (x + 2 < w) ? __ldg(p + 2) : 0.f;
  t.w = (x + 3 < w) ? __ldg(p + 3) : 0.f;
  return t;
}
__device__ __forceinline__ float4 load4(const __nv_bfloat16* __restrict__ p, int x, int w, bool vec) {
  if (vec && x + 3 < w) {
    uint2 raw = __ldg(reinterpret_cast<const uint2*>(p));
    float4 t;
    t.x = __uint_as_float(raw.x << 16);
    t.y = __uint_as_float(raw.x & 0xffff0000u);
    t.z = __uint_as_float(raw.y << 16);
    t.w = __uint_as_float(raw.y & 0xffff0000u);
    return t;
  }
  const unsigned short* q = reinterpret_cast<const unsigned short*>(p);
  float4 t;
  t.x = (x + 0 < w) ? __uint_as_float((unsigned)__ldg(q + 0) << 16) : 0.f;
  t.y = (x + 1 < w) ? __uint_as_float((unsigned)__ldg(q + 1) << 16) : 0.f;
  t.z = (x + 2 < w) ? __uint_as_float((unsigned)__ldg(q + 2) << 16) : 0.f;
  t.w = (x + 3 < w) ? __uint_as_float((unsigned)__ldg(q + 3) << 16) : 0.f;
  return t;
}

// 4 consecutive elements at p as one vector load, no bounds check: for rows
// whose width is a multiple of 4 read at a multiple of 4 (p 16-byte aligned
// for fp32, 8-byte for bf16).  Branch-free, so a thread's loads of several
// rows all issue before the first use.
__device__ __forceinline__ float4 load4v(const float* __restrict__ p) {
  return __ldg(reinterpret_cast<const float4*>(p));
}
__device__ __forceinline__ float4 load4v(const __nv_bfloat16* __restrict__ p) {
  const uint2 raw = __ldg(reinterpret_cast<const uint2*>(p));
  return make_float4(__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xffff0000u),
                     __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xffff0000u));
}

__device__ __forceinline__ unsigned pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<unsigned*>(&t);
}

// Stores n (<= 4) consecutive values of one output row.  `vec` says the row
// start p is aligned for the 4-element vector form (16 bytes for fp32, 8 for
// bf16).
__device__ __forceinline__ void store4(float* __restrict__ p, const float (&v)[4], int n, bool vec) {
  if (vec && n == 4) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    return;
  }
#pragma unroll
  for (int e = 0; e < 4; ++e)
    if (e < n) p[e] = v[e];
}
__device__ __forceinline__ void store4(__nv_bfloat16* __restrict__ p, const float (&v)[4], int n, bool vec) {
  if (vec && n == 4) {
    uint2 t;
    t.x = pack_bf16x2(v[0], v[1]);
    t.y = pack_bf16x2(v[2], v[3]);
    *reinterpret_cast<uint2*>(p) = t;
    return;
  }
#pragma unroll
  for (int e = 0; e < 4; ++e)
    if (e < n) p[e] = __float2bfloat16_rn(v[e]);
}

// ------------------------------------------------------ register-tiled conv
// Sum over the 32 lanes of a warp by a fixed butterfly: the same order on
// every run, so reductions built on it are deterministic.
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// acc[R][CW] += sum_{u,v<K} w[u*K+v] * in[(orow+u)*ld + (j+v)]
// `in` points at the input element (y0-r, x0-r) of the tile and must be
// 16-byte aligned; ld is a multiple of 4 floats.  w is 16-byte aligned and
// readable up to the next multiple of 4 floats after K*K (the folded
// blocks reserve kk4 floats per kernel): it is read as float4s.  Each input row is read
// once (NV float4 loads) and used by every output row it touches.  With
// OFF > 0, `in` points OFF elements before (y0-r, x0-r) (an aligned window
// start when the row layout's column padding is not r).
template <int K, int R, int CW, int OFF = 0>
__device__ __forceinline__ void conv_tile(const float* __restrict__ in, int ld,
                                          const float* __restrict__ w, float (&acc)[R][CW]) {
  constexpr int NIN = CW + K - 1 + OFF;
  constexpr int NV = (NIN + 3) / 4;
  constexpr int NW = (K * K + 3) / 4;
  float wr[NW * 4];
#pragma unroll
  for (int q = 0; q < NW; ++q) {
    const float4 t = reinterpret_cast<const float4*>(w)[q];
    wr[4 * q + 0] = t.x;
    wr[4 * q + 1] = t.y;
    wr[4 * q + 2] = t.z;
    wr[4 * q + 3] = t.w;
  }
#pragma unroll
  for (int row = 0; row < R + K - 1; ++row) {
    float xv[NV * 4];
    const float4* src = reinterpret_cast<const float4*>(in + row * ld);
#pragma unroll
    for (int q = 0; q < NV; ++q) {
      const float4 t = src[q];
      xv[4 * q + 0] = t.x;
      xv[4 * q + 1] = t.y;
      xv[4 * q + 2] = t.z;
      xv[4 * q + 3] = t.w;
    }
#pragma unroll
    for (int u = 0; u < K; ++u) {
      const int orow = row - u;
      if (orow >= 0 && orow < R) {
#pragma unroll
        for (int v = 0; v < K; ++v) {
#pragma unroll
          for (int j = 0; j < CW; ++j) acc[orow][j] = fmaf(wr[u * K + v], xv[j + v + OFF], acc[orow][j]);
        }
      }
    }
  }
}

// ------------------------------------------- register-tiled correlation
// G[u*K+v] += sum_{i<R, j<CW} g[i*ldg + j] * a[(i+u)*lda + (j+v)]
// a points at (y0-r, x0-r) of the shifted operand, g at (y0, x0) of the
// gradient operand; both 16-byte aligned, lda/ldg multiples of 4.  With
// OFF > 0, a points OFF elements before (y0-r, x0-r) (an aligned window
// start when the row layout's column padding is not r).  With SUMG, the
// tile's g values are also added to *gsum.  GV is the width of the g loads
// (4, 2 or 1 floats): g need only be aligned to GV floats.
template <int K, int R, int CW, int OFF = 0, bool SUMG = false, int GV = 4>
__device__ __forceinline__ void corr_tile(const float* __restrict__ a, int lda,
                                          const float* __restrict__ g, int ldg, float (&G)[K * K],
                                          float* gsum = nullptr) {
  constexpr int NIN = CW + K - 1 + OFF;
  constexpr int NV = (NIN + 3) / 4;
  float gr[R][CW];
#pragma unroll
  for (int i = 0; i < R; ++i) {
    if constexpr (GV == 4) {
      const float4* src = reinterpret_cast<const float4*>(g + i * ldg);
#pragma unroll
      for (int q = 0; q < CW / 4; ++q) {
        const float4 t = src[q];
        gr[i][4 * q + 0] = t.x;
        gr[i][4 * q + 1] = t.y;
        gr[i][4 * q + 2] = t.z;
        gr[i][4 * q + 3] = t.w;
      }
    } else if constexpr (GV == 2) {
      const float2* src = reinterpret_cast<const float2*>(g + i * ldg);
#pragma unroll
      for (int q = 0; q < CW / 2; ++q) {
        const float2 t = src[q];
        gr[i][2 * q + 0] = t.x;
        gr[i][2 * q + 1] = t.y;
      }
    } else {
#pragma unroll
      for (int q = 0; q < CW; ++q) gr[i][q] = g[i * ldg + q];
    }
  }
  if constexpr (SUMG) {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < R; ++i)
#pragma unroll
      for (int j = 0; j < CW; ++j) s += gr[i][j];
    *gsum += s;
  }
#pragma unroll
  for (int row = 0; row < R + K - 1; ++row) {
    float xv[NV * 4];
    const float4* src = reinterpret_cast<const float4*>(a + row * lda);
#pragma unroll
    for (int q = 0; q < NV; ++q) {
      const float4 t = src[q];
      xv[4 * q + 0] = t.x;
      xv[4 * q + 1] = t.y;
      xv[4 * q + 2] = t.z;
      xv[4 * q + 3] = t.w;
    }
#pragma unroll
    for (int u = 0; u < K; ++u) {
      const int orow = row - u;
      if (orow >= 0 && orow < R) {
#pragma unroll
        for (int v = 0; v < K; ++v) {
#pragma unroll
          for (int j = 0; j < CW; ++j) G[u * K + v] = fmaf(gr[orow][j], xv[j + v + OFF], G[u * K + v]);
        }
      }
    }
  }
}

// --------------------------------------------------------------- butterflies
// Haar analysis of the 2x2 block (a b / c d), taps +-1/2.
__device__ __forceinline__ void haar4(float a, float b, float c, float d, float& ll, float& lh,
                                      float& hl, float& hh) {
  const float s0 = a + b, s1 = c + d, d0 = a - b, d1 = c - d;
  ll = 0.5f * (s0 + s1);
  lh = 0.5f * (s0 - s1);
  hl = 0.5f * (d0 + d1);
  hh = 0.5f * (d0 - d1);
}
// Synthesis butterfly without the 1/2 (folded into the level weights):
// o(py,px) = sum_s sigma_s(py,px) z_s.
__device__ __forceinline__ void synth4(float ll, float lh, float hl, float hh, float& o00, float& o01,
                                       float& o10, float& o11) {
  const float A = ll + lh, B = ll - lh, Cc = hl + hh, D = hl - hh;
  o00 = A + Cc;
  o01 = A - Cc;
  o10 = B + D;
  o11 = B - D;
}

}  // namespace wt
