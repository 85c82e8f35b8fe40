// Shared device helpers of the WTConv kernels (sm_100a): the Haar pyramid
// step in shared memory, vectorised shared-memory stores and staged-row
// loads, and the fixed-order finalize of the weight gradients.
#pragma once

#include "wtconv_device.cuh"
#include "wtconv_plan.h"

namespace wt {

__device__ __forceinline__ float pow2neg(int l) { return __int_as_float((127 - l) << 23); }

__device__ void pyramid_level(int npb, int hl, int wlv, const float* src0, int lds, int src_ps, float* dst0,
                              int ldd, int bsd, int dst_ps) {
  const int per = hl * wlv;
  for (int it = threadIdx.x; it < npb * per; it += blockDim.x) {
    const int pb = it / per, rem = it - pb * per;
    const int i = rem / wlv, j = rem - i * wlv;
    const float* q = src0 + pb * src_ps + (2 * i) * lds + 2 * j;
    float ll, lh, hl_, hh;
    haar4(q[0], q[1], q[lds], q[lds + 1], ll, lh, hl_, hh);
    float* d = dst0 + pb * dst_ps + i * ldd + j;
    d[0] = ll;
    d[bsd] = lh;
    d[2 * bsd] = hl_;
    d[3 * bsd] = hh;
  }
}

// ------------------------------------------------------ vector smem stores
// 4 floats at p = row + x0 + RB with x0 % 4 == 0 (RB = column offset).
template <int RB>
__device__ __forceinline__ void sts4(float* p, const float4 v) {
  if constexpr (RB % 4 == 0) {
    *reinterpret_cast<float4*>(p) = v;
  } else if constexpr (RB % 2 == 0) {
    reinterpret_cast<float2*>(p)[0] = make_float2(v.x, v.y);
    reinterpret_cast<float2*>(p)[1] = make_float2(v.z, v.w);
  } else {
    p[0] = v.x;
    p[1] = v.y;
    p[2] = v.z;
    p[3] = v.w;
  }
}
// 2 floats at p = row + x0 + RB with x0 even.
template <int RB>
__device__ __forceinline__ void sts2(float* p, float a, float b) {
  if constexpr (RB % 2 == 0) {
    *reinterpret_cast<float2*>(p) = make_float2(a, b);
  } else {
    p[0] = a;
    p[1] = b;
  }
}

// ------------------------------------------------------------ staging
// Loads 4 consecutive elements of a staged row (smem, I/O dtype): vector
// loads when `vec` (row start and x 16/8-byte aligned), else scalar with
// zero past w.
__device__ __forceinline__ float4 lds4(const float* p, int x, int w, bool vec) {
  if (vec && x + 3 < w) return *reinterpret_cast<const float4*>(p);
  return make_float4(x + 0 < w ? p[0] : 0.f, x + 1 < w ? p[1] : 0.f, x + 2 < w ? p[2] : 0.f,
                     x + 3 < w ? p[3] : 0.f);
}
__device__ __forceinline__ float4 lds4(const __nv_bfloat16* p, int x, int w, bool vec) {
  if (vec && x + 3 < w) {
    const uint2 raw = *reinterpret_cast<const uint2*>(p);
    return make_float4(__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xffff0000u),
                       __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xffff0000u));
  }
  const unsigned short* q = reinterpret_cast<const unsigned short*>(p);
  return make_float4(x + 0 < w ? __uint_as_float((unsigned)q[0] << 16) : 0.f,
                     x + 1 < w ? __uint_as_float((unsigned)q[1] << 16) : 0.f,
                     x + 2 < w ? __uint_as_float((unsigned)q[2] << 16) : 0.f,
                     x + 3 < w ? __uint_as_float((unsigned)q[3] << 16) : 0.f);
}
template <bool SMEM, typename IO>
__device__ __forceinline__ float4 src4(const IO* p, int x, int w, bool vec) {
  if constexpr (SMEM) return lds4(p, x, w, vec);
  else return load4(p, x, w, vec);
}

// ------------------------------------------------------ weight gradients
template <int K>
__device__ __forceinline__ void zero_taps(float (&G)[K * K]) {
#pragma unroll
  for (int t = 0; t < K * K; ++t) G[t] = 0.f;
}

// Sums the per-CTA partials of channel c = blockIdx.x over its groups in a
// fixed order and applies the chain rule through the scales and the bias.
// The channel's base and level kernels are first copied to shared memory by
// all threads at once, so the per-branch dot products below read no global
// memory.
struct FinalizeArgs {
  int C, L, V, ngroups;
};
template <int K>
__global__ void wtconv_bwdw_finalize(const FinalizeArgs P, const float* __restrict__ part, const float* __restrict__ w0,
                                     const float* __restrict__ b0, const float* __restrict__ s0,
                                     const float* __restrict__ wl, const float* __restrict__ sl,
                                     float* __restrict__ dw0, float* __restrict__ db0, float* __restrict__ ds0,
                                     float* __restrict__ dwl, float* __restrict__ dsl) {
  constexpr int KK = K * K;
  extern __shared__ float gsum[];  // V sums, then the channel's kernels: w0 (KK), wl (4L x KK)
  float* wsm = gsum + P.V;
  const int c = blockIdx.x;
  for (int e = threadIdx.x; e < (1 + 4 * P.L) * KK; e += blockDim.x) {
    if (e < KK) {
      wsm[e] = w0[(size_t)c * KK + e];
    } else {
      const int br = (e - KK) / KK, t = (e - KK) - br * KK;
      const size_t base = ((size_t)(br >> 2) * P.C + c) * 4 + (br & 3);
      wsm[e] = wl[base * KK + t];
    }
  }
  // groups summed in index order; their loads issued eight at a time
  const size_t gstride = (size_t)P.C * P.V;
  for (int e = threadIdx.x; e < P.V; e += blockDim.x) {
    const float* src = part + (size_t)c * P.V + e;
    float a = 0.f;
    int g = 0;
    for (; g + 8 <= P.ngroups; g += 8) {
      float v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = __ldg(src + (size_t)(g + q) * gstride);
#pragma unroll
      for (int q = 0; q < 8; ++q) a += v[q];
    }
    for (; g < P.ngroups; ++g) a += __ldg(src + (size_t)g * gstride);
    gsum[e] = a;
  }
  __syncthreads();
  const float sdy = gsum[P.V - 1];
  for (int t = threadIdx.x; t < KK; t += blockDim.x) dw0[(size_t)c * KK + t] = s0[c] * gsum[t];
  if (threadIdx.x == 0) {
    float a = 0.f;
    for (int t = 0; t < KK; ++t) a = fmaf(wsm[t], gsum[t], a);
    ds0[c] = a + b0[c] * sdy;
    db0[c] = s0[c] * sdy;
  }
  for (int e = threadIdx.x; e < P.L * 4 * KK; e += blockDim.x) {
    const int br = e / KK, t = e - br * KK;
    const int l = br >> 2, s = br & 3;
    const size_t base = ((size_t)l * P.C + c) * 4 + s;
    dwl[base * KK + t] = sl[base] * gsum[KK + e];
  }
  for (int br = threadIdx.x; br < P.L * 4; br += blockDim.x) {
    const int l = br >> 2, s = br & 3;
    const size_t base = ((size_t)l * P.C + c) * 4 + s;
    float a = 0.f;
    for (int t = 0; t < KK; ++t) a = fmaf(wsm[KK + br * KK + t], gsum[KK + br * KK + t], a);
    dsl[base] = a;
  }
}

// Planes whose sides are not multiples of 2^L run on zero-padded copies:
// zero rows at the bottom and zero columns at the right of every plane up to
// Hp x Wp (multiples of 2^L); the output kernel then stores only the image.  Padding each
// level's plane to even sides and cropping each level's synthesis, the
// reading the layer follows for such sides, gives the same outputs on the
// image and the same gradients: the extra rows and columns of every level
// hold zeros or feed only outputs outside the image.
// The pad walks chunks of PADC elements of one padded plane; each thread
// takes PADC / 256 elements of a chunk, issuing its loads before its stores.
constexpr int PADC = 1024;

template <typename IO>
__global__ void __launch_bounds__(256) wtconv_pad_kernel(const IO* __restrict__ src, IO* __restrict__ dst, int H,
                                                         int W, int Hp, int Wp, FDiv fWp, long long planes,
                                                         int cpp) {
  const int per = Hp * Wp;
  const long long units = planes * cpp;
  for (long long u = blockIdx.x; u < units; u += gridDim.x) {
    const long long p = u / cpp;
    const int c0 = (int)(u - p * cpp) * PADC + threadIdx.x;
    const IO* s = src + (size_t)p * H * W;
    IO* d = dst + (size_t)p * per;
    IO v[PADC / 256];
#pragma unroll
    for (int k = 0; k < PADC / 256; ++k) {
      const int e = c0 + k * 256;
      v[k] = IO(0.f);
      if (e < per) {
        const int y = fWp.div(e), x = e - y * Wp;
        if (y < H && x < W) v[k] = s[y * W + x];
      }
    }
#pragma unroll
    for (int k = 0; k < PADC / 256; ++k)
      if (c0 + k * 256 < per) d[c0 + k * 256] = v[k];
  }
}

// Planes too large for the deep kernel compute their levels >= 2 as a layer
// of one level fewer on the level-1 LL planes (the raw LL band that goes one
// level deeper); these two kernels prepare its input and its weights.
//
// LL band of the level-1 Haar analysis: (a+b+c+d)/2 of every 2x2 block.
template <typename IO>
__global__ void wtconv_ll_kernel(const IO* __restrict__ x, float* __restrict__ ll, int H, int W, long long n) {
  const int W1 = W / 2, H1 = H / 2;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const long long row = i / W1;  // row of the LL plane stack
    const int j = (int)(i - row * W1);
    const long long p = row / H1;
    const int r = (int)(row - p * H1);
    const IO* a = x + ((size_t)p * H + 2 * r) * W + 2 * j;
    using T = io_traits<IO>;
    ll[i] = 0.5f * ((T::to_f(a[0]) + T::to_f(a[1])) + (T::to_f(a[W]) + T::to_f(a[W + 1])));
  }
}

// Folded block of that smaller layer from the layer's own block: base
// kernel and bias zero (the smaller layer has no base branch), level l' =
// level l' + 1 of the original.  The original's 2^-(l'+1) s W equals the
// smaller layer's 2^-l' (s/2) W: the extra 1/2 is the level-1 synthesis
// factor that its output carries into the original layer.
__global__ void wtconv_shift_fold_kernel(const float* __restrict__ wf, float* __restrict__ wf1, int C, int kk4,
                                         int wblk, int wblk1, int L1) {
  // level l' starts at kk4 + 4 + 4 (l' - 1) kk4 in both layouts, so the
  // original's level l' + 1 sits 4 kk4 floats further on
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < C * wblk1; i += gridDim.x * blockDim.x) {
    const int c = i / wblk1, e = i - c * wblk1;
    float v = 0.f;
    if (e >= kk4 + 4 && e < kk4 + 4 + 4 * L1 * kk4) v = wf[(size_t)c * wblk + e + 4 * kk4];
    wf1[i] = v;
  }
}

}  // namespace wt
