// Per-plane fused WTConv kernels for sm_100a.
//
// Forward (and backward-data, which is the same pass on dy with flipped
// kernels and no bias):  one CTA takes a batch of PB planes of one channel,
// stages them in shared memory, computes the level-1 Haar subbands and the
// deeper pyramid on chip (reformulation (1) of arXiv:2608.10805, abstract),
// convolves every subband with weights that already carry the per-channel
// scale and the synthesis factor 2^-l (reformulation (3)), synthesises all
// levels >= 3 in one pass indexed by the bits of the level-2 coordinates
// (reformulation (2)), folds levels 2 and 1 in with register butterflies and
// writes y once.  x is read once and y written once: no subband, LL or Z
// tensor travels through HBM.
//
// Weight gradients: the same staging, then per-tap correlations of dy (and
// its Haar pyramid) with x (and its pyramid).  Warps 0-3 own the base taps
// and warps 4-7 the four level-1 bands; their sums stay in registers across
// all planes of the CTA and are reduced once, in a fixed order; the small
// deep levels are reduced per plane into shared-memory accumulators, also in
// a fixed order.  A second kernel sums the per-CTA partials over the batch
// in a fixed order and applies the scales: results are deterministic.
#pragma once

#include "wtconv_device.cuh"
#include "wtconv_plan.h"

namespace wt {

__device__ __forceinline__ float pow2neg(int l) { return __int_as_float((127 - l) << 23); }

__device__ __forceinline__ int wl_off(int kk4, int l, int s) { return kk4 + 4 + ((l - 1) * 4 + s) * kk4; }

// Folded weights of channel c in shared memory:
//   w0f = s0 * W0 (flipped for the adjoint), b0f = s0 * b0 (0 for the adjoint),
//   wlf[l][s] = 2^-l * sl[l][c][s] * Wl[l][c][s] (flipped for the adjoint).
template <int K>
__device__ void load_weights(const Plan& P, float* sw, int c, const float* __restrict__ w0,
                             const float* __restrict__ b0, const float* __restrict__ s0,
                             const float* __restrict__ wl, const float* __restrict__ sl, int flip) {
  constexpr int KK = K * K;
  const int kk4 = P.kk4;
  const int total = (1 + 4 * P.L) * kk4;
  for (int i = threadIdx.x; i < total; i += blockDim.x) {
    const int blk = i / kk4, t = i - blk * kk4;
    float v = 0.f;
    if (t < KK) {
      const int tt = flip ? (KK - 1 - t) : t;
      if (blk == 0) {
        v = s0[c] * w0[(size_t)c * KK + tt];
      } else {
        const int l = (blk - 1) / 4 + 1, s = (blk - 1) & 3;
        const size_t base = ((size_t)(l - 1) * P.C + c) * 4 + s;
        v = (sl[base] * wl[base * KK + tt]) * pow2neg(l);
      }
    }
    sw[blk == 0 ? t : (kk4 + 4 + (blk - 1) * kk4 + t)] = v;
  }
  if (threadIdx.x < 4) sw[kk4 + threadIdx.x] = (threadIdx.x == 0 && !flip) ? s0[c] * b0[c] : 0.f;
}

// Haar analysis of the LL band of level l-1 into the 4 bands of level l
// for every plane of the batch.  src: LL of level l-1 at interior origin.
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

__device__ __forceinline__ int cdiv(int a, int b) { return (a + b - 1) / b; }

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

// Stages the npb planes of a batch: the plane into the fp32 buffer xf, its
// level-1 subbands into s1 and, when L >= 2, its level-2 subbands into s2
// (4x4 blocks of x per item; the Haar butterflies run in registers).  The
// source is either the raw copy of the batch in shared memory (SMEM, planes
// packed back to back) or global memory.  SH selects the shifted layout
// (border r, read by the register tiles at x0 - r) or the plain layout (read
// at x0).  SUM accumulates every value read.
template <int K, typename IO, bool SH, bool SUM, bool SMEM>
__device__ void stage_planes(const Plan& P, float* sm, const IO* __restrict__ src0, size_t pstride, int npb,
                             const BufDesc& bx, const BufDesc& b1, const BufDesc& b2, float* sum) {
  constexpr int r = SH ? K / 2 : 0;
  const int ldx = bx.ld;
  const bool vec = P.vec_in != 0;
  if (P.L >= 2) {
    const int bw = P.W >> 2, per = (P.H >> 2) * bw, n = npb * per;
    const int ld1 = b1.ld, bs1 = b1.ld * b1.rows, ld2 = b2.ld, bs2 = b2.ld * b2.rows;
    for (int it = threadIdx.x; it < n; it += blockDim.x) {
      const int pb = P.f_stage_per.div(it);
      const int rem = it - pb * per;
      const int by = P.f_stage_x.div(rem);
      const int bxi = rem - by * bw;
      const int x0 = bxi << 2, y0 = by << 2;
      const IO* src = src0 + pb * pstride + (size_t)y0 * P.W + x0;
      float4 v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = src4<SMEM>(src + (size_t)i * P.W, x0, P.W, true);
      if (SUM) {
#pragma unroll
        for (int i = 0; i < 4; ++i) *sum += (v[i].x + v[i].y) + (v[i].z + v[i].w);
      }
      float* xf = sm + bx.off + pb * bx.ps + (y0 + r) * ldx + x0 + r;
#pragma unroll
      for (int i = 0; i < 4; ++i) sts4<r>(xf + i * ldx, v[i]);
      float* s1 = sm + b1.off + pb * b1.ps + (2 * by + r) * ld1 + 2 * bxi + r;
      float ll[2][2];
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        float l0, h0, g0, k0, l1, h1, g1, k1;
        haar4(v[2 * a].x, v[2 * a].y, v[2 * a + 1].x, v[2 * a + 1].y, l0, h0, g0, k0);
        haar4(v[2 * a].z, v[2 * a].w, v[2 * a + 1].z, v[2 * a + 1].w, l1, h1, g1, k1);
        sts2<r>(s1 + a * ld1, l0, l1);
        sts2<r>(s1 + bs1 + a * ld1, h0, h1);
        sts2<r>(s1 + 2 * bs1 + a * ld1, g0, g1);
        sts2<r>(s1 + 3 * bs1 + a * ld1, k0, k1);
        ll[a][0] = l0;
        ll[a][1] = l1;
      }
      float L2, H2, G2, K2;
      haar4(ll[0][0], ll[0][1], ll[1][0], ll[1][1], L2, H2, G2, K2);
      float* s2 = sm + b2.off + pb * b2.ps + (by + r) * ld2 + bxi + r;
      s2[0] = L2;
      s2[bs2] = H2;
      s2[2 * bs2] = G2;
      s2[3 * bs2] = K2;
    }
  } else if (P.L == 1) {
    const int Q = (P.W + 3) >> 2, per = P.H1 * Q, n = npb * per;
    const int ld1 = b1.ld, bs1 = b1.ld * b1.rows;
    for (int it = threadIdx.x; it < n; it += blockDim.x) {
      const int pb = P.f_stage_per.div(it);
      const int rem = it - pb * per;
      const int i = P.f_stage_x.div(rem);
      const int x0 = (rem - i * Q) << 2;
      const IO* src = src0 + pb * pstride + (size_t)(2 * i) * P.W + x0;
      const float4 a = src4<SMEM>(src, x0, P.W, vec);
      const float4 b = src4<SMEM>(src + P.W, x0, P.W, vec);
      if (SUM) *sum += ((a.x + a.y) + (a.z + a.w)) + ((b.x + b.y) + (b.z + b.w));
      float* d0 = sm + bx.off + pb * bx.ps + (2 * i + r) * ldx + x0 + r;
      float* s1 = sm + b1.off + pb * b1.ps + (i + r) * ld1 + (x0 >> 1) + r;
      float l0, h0, g0, k0, l1, h1, g1, k1;
      haar4(a.x, a.y, b.x, b.y, l0, h0, g0, k0);
      haar4(a.z, a.w, b.z, b.w, l1, h1, g1, k1);
      if (x0 + 3 < P.W) {
        sts4<r>(d0, a);
        sts4<r>(d0 + ldx, b);
        sts2<r>(s1, l0, l1);
        sts2<r>(s1 + bs1, h0, h1);
        sts2<r>(s1 + 2 * bs1, g0, g1);
        sts2<r>(s1 + 3 * bs1, k0, k1);
      } else {  // W % 4 == 2: one 2-wide block left in the row
        d0[0] = a.x;
        d0[1] = a.y;
        d0[ldx] = b.x;
        d0[ldx + 1] = b.y;
        s1[0] = l0;
        s1[bs1] = h0;
        s1[2 * bs1] = g0;
        s1[3 * bs1] = k0;
      }
    }
  } else {
    const int Q = (P.W + 3) >> 2, per = P.H * Q, n = npb * per;
    for (int it = threadIdx.x; it < n; it += blockDim.x) {
      const int pb = P.f_stage_per.div(it);
      const int rem = it - pb * per;
      const int yy = P.f_stage_x.div(rem);
      const int x0 = (rem - yy * Q) << 2;
      const float4 a = src4<SMEM>(src0 + pb * pstride + (size_t)yy * P.W + x0, x0, P.W, vec);
      if (SUM) *sum += (a.x + a.y) + (a.z + a.w);
      float* d0 = sm + bx.off + pb * bx.ps + (yy + r) * ldx + x0 + r;
      if (x0 + 3 < P.W) {
        sts4<r>(d0, a);
      } else {
        const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (x0 + e < P.W) d0[e] = av[e];
      }
    }
  }
}

// ------------------------------------------------ TMA bulk copies of planes
// The issuing thread first announces the bytes of one batch on the CTA's
// mbarrier (one arrival per phase), then issues 1-D bulk copies of whole
// planes (each H*W elements, contiguous in global memory, a multiple of 16
// bytes) into a raw shared-memory buffer; the phase completes when they land.
__device__ __forceinline__ void bulk_expect(uint64_t* mbar, unsigned bytes) {
  const unsigned bar = (unsigned)__cvta_generic_to_shared(mbar);
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
template <typename IO>
__device__ __forceinline__ void bulk_copies(uint64_t* mbar, void* raw, const IO* src, size_t pstride, int npb,
                                            unsigned bytes) {
  const unsigned bar = (unsigned)__cvta_generic_to_shared(mbar);
  const unsigned dst = (unsigned)__cvta_generic_to_shared(raw);
  for (int pb = 0; pb < npb; ++pb) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst + pb * bytes),
        "l"(src + pb * pstride), "r"(bytes), "r"(bar)
        : "memory");
  }
}

// Waits for the mbarrier phase `parity` with an iteration limit.  Returns
// false when the limit ran out (the copy never completed).
__device__ __forceinline__ bool mbar_wait(uint64_t* mbar, unsigned parity) {
  const unsigned bar = (unsigned)__cvta_generic_to_shared(mbar);
  for (int i = 0; i < (1 << 22); ++i) {
    unsigned done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}

__device__ __forceinline__ void mbar_init(uint64_t* mbar) {
  const unsigned bar = (unsigned)__cvta_generic_to_shared(mbar);
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------ deep levels
// Levels 2..L of the batch: the rest of the pyramid (levels >= 3), every
// level conv in one parallel pass (folded weights 2^-l s_l W_l), then the
// closed-form synthesis of all levels >= 2 at level-1 resolution:
//   t1(i,j) = sum_{l>=2} sum_s sigma_s(bit_{l-2}(i), bit_{l-2}(j)) Zd_l^s(i >> (l-1), j >> (l-1))
// Ends synchronised.
template <int K>
__device__ void deep_forward(const Plan& P, float* sm, const float* sw, int npb) {
  constexpr int r = K / 2;
  const int kk4 = P.kk4;
  for (int l = 3; l <= P.L; ++l) {
    const BufDesc& s = P.sd[l - 1];
    const BufDesc& d = P.sd[l];
    pyramid_level(npb, P.H >> l, P.W >> l, sm + s.off + r * s.ld + r, s.ld, s.ps, sm + d.off + r * d.ld + r, d.ld,
                  d.ld * d.rows, d.ps);
    __syncthreads();
  }
  const int per = P.deep_items;
  for (int it = threadIdx.x; it < npb * per; it += blockDim.x) {
    const int pb = P.f_deep_per.div(it);
    int rem = it - pb * per;
    int l = 2;
    while (rem >= P.deep_first[l + 1]) ++l;
    rem -= P.deep_first[l];
    const int tpb = P.f_l_tiles[l].d;
    const int s = P.f_l_tiles[l].div(rem);
    rem -= s * tpb;
    const int ti = P.f_l_tx[l].div(rem);
    const int tj = rem - ti * P.f_l_tx[l].d;
    const BufDesc& d = P.sd[l];
    const BufDesc& z = P.zd[l];
    float acc[DP_R][DP_CW];
#pragma unroll
    for (int a = 0; a < DP_R; ++a)
#pragma unroll
      for (int b = 0; b < DP_CW; ++b) acc[a][b] = 0.f;
    conv_tile<K, DP_R, DP_CW>(sm + d.off + pb * d.ps + s * d.ld * d.rows + ti * DP_R * d.ld + tj * DP_CW, d.ld,
                              sw + wl_off(kk4, l, s), acc);
    float* o = sm + z.off + pb * z.ps + s * z.ld * z.rows + ti * DP_R * z.ld + tj * DP_CW;
#pragma unroll
    for (int a = 0; a < DP_R; ++a)
      reinterpret_cast<float4*>(o + a * z.ld)[0] = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
  }
  __syncthreads();
  {
    const int tq = P.f_t1_x.d, per1 = P.f_t1_per.d;
    const BufDesc& z2 = P.zd[2];
    const int bz2 = z2.ld * z2.rows;
    for (int it = threadIdx.x; it < npb * per1; it += blockDim.x) {
      const int pb = P.f_t1_per.div(it);
      const int rem = it - pb * per1;
      const int i = P.f_t1_x.div(rem);
      const int j0 = (rem - i * tq) << 2;
      // level 2: positions (i >> 1, (j0 >> 1) + {0, 1}), sign bits bit0(i), bit0(j)
      const float* q = sm + z2.off + pb * z2.ps + (i >> 1) * z2.ld + (j0 >> 1);
      const float2 zl = *reinterpret_cast<const float2*>(q);
      const float2 zh = *reinterpret_cast<const float2*>(q + bz2);
      const float2 zg = *reinterpret_cast<const float2*>(q + 2 * bz2);
      const float2 zk = *reinterpret_cast<const float2*>(q + 3 * bz2);
      const float sy = (i & 1) ? -1.f : 1.f;
      // sum_s sigma_s z_s = (ll + sy lh) + sx (hl + sy hh)
      const float a0 = fmaf(sy, zh.x, zl.x), b0 = fmaf(sy, zk.x, zg.x);
      const float a1 = fmaf(sy, zh.y, zl.y), b1 = fmaf(sy, zk.y, zg.y);
      float o0 = a0 + b0, o1 = a0 - b0, o2 = a1 + b1, o3 = a1 - b1;
      for (int l = 3; l <= P.L; ++l) {
        const BufDesc& z = P.zd[l];
        const int bz = z.ld * z.rows;
        const float* p = sm + z.off + pb * z.ps + (i >> (l - 1)) * z.ld + (j0 >> (l - 1));
        const float syl = ((i >> (l - 2)) & 1) ? -1.f : 1.f;
        const float A = fmaf(syl, p[bz], p[0]), B = fmaf(syl, p[3 * bz], p[2 * bz]);
        if (l == 3) {  // bit1 of j: 0 for j0, j0+1 and 1 for j0+2, j0+3
          o0 += A + B;
          o1 += A + B;
          o2 += A - B;
          o3 += A - B;
        } else {
          const float sxl = ((j0 >> (l - 2)) & 1) ? -1.f : 1.f;
          const float v = fmaf(sxl, B, A);
          o0 += v;
          o1 += v;
          o2 += v;
          o3 += v;
        }
      }
      *reinterpret_cast<float4*>(sm + P.t1.off + pb * P.t1.ps + i * P.t1.ld + j0) = make_float4(o0, o1, o2, o3);
    }
  }
  __syncthreads();
}

// --------------------------------------------------------------- output pass
// Per R3 x 8 tile: the four level-1 band convs ((R3/2) x 4 each, folded
// weights), t1 added to the LL band, the synthesis signs applied straight
// into the accumulators, then the base conv; y is written once.
template <int K, int R3, typename IO>
__device__ void output_pass(const Plan& P, float* sm, const float* sw, IO* __restrict__ y, int c, int nb0,
                            int npb) {
  constexpr int RB = R3 / 2;
  const int tx = P.f_out_x.d, per = P.f_out_per.d;
  const int bs1 = P.s1.ld * P.s1.rows;
  const float bias = sw[P.kk4];
  for (int it = threadIdx.x; it < npb * per; it += blockDim.x) {
    const int pb = P.f_out_per.div(it);
    const int rem = it - pb * per;
    const int ti = P.f_out_x.div(rem);
    const int tj = rem - ti * tx;
    const int yy0 = ti * R3, xx0 = tj * C3_CW;
    float acc[R3][C3_CW];
#pragma unroll
    for (int a = 0; a < R3; ++a)
#pragma unroll
      for (int b = 0; b < C3_CW; ++b) acc[a][b] = bias;
    if (P.L >= 1) {
      const float* s1 = sm + P.s1.off + pb * P.s1.ps + (yy0 >> 1) * P.s1.ld + (xx0 >> 1);
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        float z[RB][4];
#pragma unroll
        for (int a = 0; a < RB; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) z[a][b] = 0.f;
        conv_tile<K, RB, 4>(s1 + s * bs1, P.s1.ld, sw + wl_off(P.kk4, 1, s), z);
        if (s == 0 && P.L >= 2) {
          const float* t1 = sm + P.t1.off + pb * P.t1.ps + (yy0 >> 1) * P.t1.ld + (xx0 >> 1);
#pragma unroll
          for (int a = 0; a < RB; ++a) {
            const float4 t = reinterpret_cast<const float4*>(t1 + a * P.t1.ld)[0];
            z[a][0] += t.x;
            z[a][1] += t.y;
            z[a][2] += t.z;
            z[a][3] += t.w;
          }
        }
        // sigma_s(py, px): LL +,+,+,+  LH +,+,-,-  HL +,-,+,-  HH +,-,-,+
        const float s01 = (s == 2 || s == 3) ? -1.f : 1.f;
        const float s10 = (s == 1 || s == 3) ? -1.f : 1.f;
        const float s11 = (s == 1 || s == 2) ? -1.f : 1.f;
#pragma unroll
        for (int a = 0; a < RB; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const float v = z[a][b];
            acc[2 * a][2 * b] += v;
            acc[2 * a][2 * b + 1] = fmaf(s01, v, acc[2 * a][2 * b + 1]);
            acc[2 * a + 1][2 * b] = fmaf(s10, v, acc[2 * a + 1][2 * b]);
            acc[2 * a + 1][2 * b + 1] = fmaf(s11, v, acc[2 * a + 1][2 * b + 1]);
          }
      }
    }
    conv_tile<K, R3, C3_CW>(sm + P.xf.off + pb * P.xf.ps + yy0 * P.xf.ld + xx0, P.xf.ld, sw, acc);
    const int n = P.W - xx0 < C3_CW ? P.W - xx0 : C3_CW;
    IO* yp = y + ((size_t)(nb0 + pb) * P.C + c) * P.H * P.W;
#pragma unroll
    for (int a = 0; a < R3; ++a)
      if (yy0 + a < P.H) store8(yp + (size_t)(yy0 + a) * P.W + xx0, acc[a], n, P.vec_out != 0);
  }
}

// Forward / backward-data kernel.  Work unit: (channel c, batch of PB
// consecutive n); grid-strided over C * nbatch units.  When the planes can
// be bulk-copied, the raw copy of unit u+1 is in flight while unit u runs
// its deep levels and output pass.
template <int K, int R3, typename IO>
__global__ void __launch_bounds__(NT, 2) wtconv_fwd_kernel(const Plan P, const IO* __restrict__ x,
                                                           const float* __restrict__ w0, const float* __restrict__ b0,
                                                           const float* __restrict__ s0,
                                                           const float* __restrict__ wl,
                                                           const float* __restrict__ sl, IO* __restrict__ y,
                                                           int flip, int* __restrict__ status) {
  extern __shared__ float4 smem4[];
  float* sm = reinterpret_cast<float*>(smem4);
  uint64_t* mbar = reinterpret_cast<uint64_t*>(sm);
  int* abort_flag = reinterpret_cast<int*>(sm + 2);
  for (int i = threadIdx.x + 1; i < (P.smem_floats >> 2); i += blockDim.x)
    smem4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (threadIdx.x == 0) {
    smem4[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    mbar_init(mbar);
  }
  __syncthreads();
  const int units = P.C * P.nbatch;
  const size_t plane = (size_t)P.H * P.W;
  const size_t pstride = (size_t)P.C * plane;
  float* sw = sm + P.w_off;
  IO* raw = reinterpret_cast<IO*>(sm + P.raw_off);
  unsigned parity = 0;
  if (P.use_bulk && threadIdx.x == 0 && (int)blockIdx.x < units) {
    const int u = blockIdx.x, bt = u / P.C, c = u - bt * P.C, nb0 = bt * P.PB;
    const int cnt = min(P.PB, P.N - nb0);
    const unsigned bytes = (unsigned)(plane * sizeof(IO));
    bulk_expect(mbar, bytes * cnt);
    bulk_copies(mbar, raw, x + ((size_t)nb0 * P.C + c) * plane, pstride, cnt, bytes);
  }
  for (int u = blockIdx.x; u < units; u += gridDim.x) {
    const int bt = u / P.C;
    const int c = u - bt * P.C;
    const int nb0 = bt * P.PB;
    const int npb = (P.N - nb0) < P.PB ? (P.N - nb0) : P.PB;
    load_weights<K>(P, sw, c, w0, b0, s0, wl, sl, flip);
    if (P.use_bulk) {
      if (threadIdx.x == 0 && !mbar_wait(mbar, parity)) *abort_flag = 1;
      parity ^= 1u;
      __syncthreads();
      if (*abort_flag) break;
      stage_planes<K, IO, true, false, true>(P, sm, raw, plane, npb, P.xf, P.s1, P.sd[2], nullptr);
      __syncthreads();
      const int un = u + gridDim.x;
      if (threadIdx.x == 0 && un < units) {
        const int btn = un / P.C, cn = un - btn * P.C, nbn = btn * P.PB;
        const int cnt = min(P.PB, P.N - nbn);
        const unsigned bytes = (unsigned)(plane * sizeof(IO));
        bulk_expect(mbar, bytes * cnt);
        bulk_copies(mbar, raw, x + ((size_t)nbn * P.C + cn) * plane, pstride, cnt, bytes);
      }
    } else {
      stage_planes<K, IO, true, false, false>(P, sm, x + ((size_t)nb0 * P.C + c) * plane, pstride, npb, P.xf,
                                              P.s1, P.sd[2], nullptr);
      __syncthreads();
    }
    if (P.L >= 2) deep_forward<K>(P, sm, sw, npb);
    output_pass<K, R3, IO>(P, sm, sw, y, c, nb0, npb);
    __syncthreads();
  }
  if (*abort_flag && threadIdx.x == 0) {
    if (status) atomicExch(status, 1);
    mbar_wait(mbar, parity ^ 1u);  // let a late copy land before the CTA exits
  }
}

// ------------------------------------------------------ weight gradients
template <int K>
__device__ __forceinline__ void zero_taps(float (&G)[K * K]) {
#pragma unroll
  for (int t = 0; t < K * K; ++t) G[t] = 0.f;
}

// Per-CTA partial sums over planes n in [g*planes_per_cta, ...) of channel
// c = blockIdx.x % C; written to part[blockIdx.x][V] with the layout
// [G0: K*K][G1: 4*K*K] ... [GL: 4*K*K][sum dy].
template <int K, typename IO>
__global__ void __launch_bounds__(NT) wtconv_bwdw_kernel(const Plan P, const IO* __restrict__ x,
                                                         const IO* __restrict__ dy, float* __restrict__ part,
                                                         int* __restrict__ status) {
  constexpr int KK = K * K;
  constexpr int r = K / 2;
  extern __shared__ float4 smem4[];
  float* sm = reinterpret_cast<float*>(smem4);
  uint64_t* mbar = reinterpret_cast<uint64_t*>(sm);
  int* abort_flag = reinterpret_cast<int*>(sm + 2);
  for (int i = threadIdx.x + 1; i < (P.smem_floats >> 2); i += NT) smem4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (threadIdx.x == 0) {
    smem4[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    mbar_init(mbar);
  }
  __syncthreads();
  const int kk4 = P.kk4;
  const int c = blockIdx.x % P.C, g = blockIdx.x / P.C;
  const int n_begin = g * P.planes_per_cta;
  const int n_end = min(P.N, n_begin + P.planes_per_cta);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nbase = P.L >= 1 ? 128 : NT;   // threads on the base taps
  const size_t plane = (size_t)P.H * P.W;
  const size_t pstride = (size_t)P.C * plane;
  IO* rawx = reinterpret_cast<IO*>(sm + P.raw_off);
  IO* rawg = reinterpret_cast<IO*>(sm + P.rawg_off);
  float G[KK];
  zero_taps<K>(G);
  float sumdy = 0.f;
  const int ndeep = P.L >= 2 ? (P.L - 1) * 4 : 0;
  unsigned parity = 0;
  if (P.use_bulk && threadIdx.x == 0 && n_begin < n_end) {
    const int cnt = min(P.PB, n_end - n_begin);
    const unsigned bytes = (unsigned)(plane * sizeof(IO));
    bulk_expect(mbar, 2 * bytes * cnt);
    bulk_copies(mbar, rawx, x + ((size_t)n_begin * P.C + c) * plane, pstride, cnt, bytes);
    bulk_copies(mbar, rawg, dy + ((size_t)n_begin * P.C + c) * plane, pstride, cnt, bytes);
  }

  for (int nb0 = n_begin; nb0 < n_end; nb0 += P.PB) {
    const int npb = (n_end - nb0) < P.PB ? (n_end - nb0) : P.PB;
    if (P.use_bulk) {
      if (threadIdx.x == 0 && !mbar_wait(mbar, parity)) *abort_flag = 1;
      parity ^= 1u;
      __syncthreads();
      if (*abort_flag) break;
      stage_planes<K, IO, true, false, true>(P, sm, rawx, plane, npb, P.xf, P.s1, P.sd[2], nullptr);
      stage_planes<K, IO, false, true, true>(P, sm, rawg, plane, npb, P.gf, P.g1, P.gd[2], &sumdy);
      __syncthreads();
      const int nn = nb0 + P.PB;
      if (threadIdx.x == 0 && nn < n_end) {
        const int cnt = min(P.PB, n_end - nn);
        const unsigned bytes = (unsigned)(plane * sizeof(IO));
        bulk_expect(mbar, 2 * bytes * cnt);
        bulk_copies(mbar, rawx, x + ((size_t)nn * P.C + c) * plane, pstride, cnt, bytes);
        bulk_copies(mbar, rawg, dy + ((size_t)nn * P.C + c) * plane, pstride, cnt, bytes);
      }
    } else {
      stage_planes<K, IO, true, false, false>(P, sm, x + ((size_t)nb0 * P.C + c) * plane, pstride, npb, P.xf,
                                              P.s1, P.sd[2], nullptr);
      stage_planes<K, IO, false, true, false>(P, sm, dy + ((size_t)nb0 * P.C + c) * plane, pstride, npb, P.gf,
                                              P.g1, P.gd[2], &sumdy);
      __syncthreads();
    }
    for (int l = 3; l <= P.L; ++l) {
      const BufDesc& sx = P.sd[l - 1];
      const BufDesc& dx = P.sd[l];
      const BufDesc& sg = P.gd[l - 1];
      const BufDesc& dg = P.gd[l];
      pyramid_level(npb, P.H >> l, P.W >> l, sm + sx.off + r * sx.ld + r, sx.ld, sx.ps, sm + dx.off + r * dx.ld + r,
                    dx.ld, dx.ld * dx.rows, dx.ps);
      pyramid_level(npb, P.H >> l, P.W >> l, sm + sg.off, sg.ld, sg.ps, sm + dg.off, dg.ld, dg.ld * dg.rows, dg.ps);
      __syncthreads();
    }
    // base and level-1 taps: register accumulation across planes
    if ((int)threadIdx.x < nbase) {
      const int tx = P.f_bw_x.d, per = P.f_bw_per.d;
      for (int it = threadIdx.x; it < npb * per; it += nbase) {
        const int pb = P.f_bw_per.div(it);
        const int rem = it - pb * per;
        const int ti = P.f_bw_x.div(rem);
        const int tj = rem - ti * tx;
        const int y0 = ti * BW_R, x0 = tj * BW_CW;
        corr_tile<K, BW_R, BW_CW>(sm + P.xf.off + pb * P.xf.ps + y0 * P.xf.ld + x0, P.xf.ld,
                                  sm + P.gf.off + pb * P.gf.ps + y0 * P.gf.ld + x0, P.gf.ld, G);
      }
    } else {
      const int s = warp - 4;
      const int tx = P.f_b1_x.d, per = P.f_b1_per.d;
      for (int it = lane; it < npb * per; it += 32) {
        const int pb = P.f_b1_per.div(it);
        const int rem = it - pb * per;
        const int ti = P.f_b1_x.div(rem);
        const int tj = rem - ti * tx;
        const int i0 = ti * B1_R, j0 = tj * B1_CW;
        corr_tile<K, B1_R, B1_CW>(
            sm + P.s1.off + pb * P.s1.ps + s * P.s1.ld * P.s1.rows + i0 * P.s1.ld + j0, P.s1.ld,
            sm + P.g1.off + pb * P.g1.ps + s * P.g1.ld * P.g1.rows + i0 * P.g1.ld + j0, P.g1.ld, G);
      }
    }
    if (ndeep) {
      // deep levels: per-slot partials, then a fixed-order fold into gdeep
      float* dpart = sm + P.dpart_off;
      for (int it = threadIdx.x; it < ndeep * DSLOTS; it += NT) {
        const int br = it / DSLOTS, slot = it - br * DSLOTS;
        const int l = 2 + (br >> 2), s = br & 3;
        const int tx = P.f_l_tx[l].d, per = P.f_l_tiles[l].d;
        const BufDesc& d = P.sd[l];
        const BufDesc& e = P.gd[l];
        float Gd[KK];
        zero_taps<K>(Gd);
        for (int t = slot; t < npb * per; t += DSLOTS) {
          const int pb = P.f_l_tiles[l].div(t);
          const int rem = t - pb * per;
          const int ti = P.f_l_tx[l].div(rem);
          const int tj = rem - ti * tx;
          const int i0 = ti * DP_R, j0 = tj * DP_CW;
          corr_tile<K, DP_R, DP_CW>(sm + d.off + pb * d.ps + s * d.ld * d.rows + i0 * d.ld + j0, d.ld,
                                    sm + e.off + pb * e.ps + s * e.ld * e.rows + i0 * e.ld + j0, e.ld, Gd);
        }
        float* o = dpart + (size_t)it * kk4;
#pragma unroll
        for (int t = 0; t < KK; ++t) o[t] = Gd[t];
      }
      __syncthreads();
      float* gdeep = sm + P.gdeep_off;
      for (int it = threadIdx.x; it < ndeep * KK; it += NT) {
        const int br = it / KK, t = it - br * KK;
        float a = gdeep[br * kk4 + t];
#pragma unroll
        for (int slot = 0; slot < DSLOTS; ++slot) a += dpart[(br * DSLOTS + slot) * kk4 + t];
        gdeep[br * kk4 + t] = a;
      }
    }
    __syncthreads();
  }
  if (*abort_flag) {
    if (threadIdx.x == 0) {
      if (status) atomicExch(status, 1);
      mbar_wait(mbar, parity ^ 1u);  // let a late copy land before the CTA exits
    }
    return;
  }
  // final fixed-order reduction of the register partials
  float* red = sm + P.red_off;
#pragma unroll
  for (int t = 0; t < KK; ++t) red[threadIdx.x * kk4 + t] = G[t];
  red[NT * kk4 + threadIdx.x] = sumdy;
  __syncthreads();
  float* out = part + (size_t)blockIdx.x * P.V;
  const int nlev1 = P.L >= 1 ? 4 * KK : 0;
  for (int e = threadIdx.x; e < P.V; e += NT) {
    float a = 0.f;
    if (e < KK) {
      for (int th = 0; th < nbase; ++th) a += red[th * kk4 + e];
    } else if (e < KK + nlev1) {
      const int s = (e - KK) / KK, t = (e - KK) - s * KK;
      for (int ln = 0; ln < 32; ++ln) a += red[(128 + 32 * s + ln) * kk4 + t];
    } else if (e < P.V - 1) {
      const int br = (e - KK - nlev1) / KK, t = (e - KK - nlev1) - br * KK;
      a = sm[P.gdeep_off + br * kk4 + t];
    } else {
      for (int th = 0; th < NT; ++th) a += red[NT * kk4 + th];
    }
    out[e] = a;
  }
}

// Sums the per-CTA partials of channel c = blockIdx.x over its groups in a
// fixed order and applies the chain rule through the scales and the bias.
template <int K>
__global__ void wtconv_bwdw_finalize(const Plan P, const float* __restrict__ part, const float* __restrict__ w0,
                                     const float* __restrict__ b0, const float* __restrict__ s0,
                                     const float* __restrict__ wl, const float* __restrict__ sl,
                                     float* __restrict__ dw0, float* __restrict__ db0, float* __restrict__ ds0,
                                     float* __restrict__ dwl, float* __restrict__ dsl) {
  constexpr int KK = K * K;
  extern __shared__ float gsum[];
  const int c = blockIdx.x;
  for (int e = threadIdx.x; e < P.V; e += blockDim.x) {
    float a = 0.f;
    for (int g = 0; g < P.ngroups; ++g) a += part[((size_t)g * P.C + c) * P.V + e];
    gsum[e] = a;
  }
  __syncthreads();
  const float sdy = gsum[P.V - 1];
  for (int t = threadIdx.x; t < KK; t += blockDim.x) dw0[(size_t)c * KK + t] = s0[c] * gsum[t];
  if (threadIdx.x == 0) {
    float a = 0.f;
    for (int t = 0; t < KK; ++t) a = fmaf(w0[(size_t)c * KK + t], gsum[t], a);
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
    for (int t = 0; t < KK; ++t) a = fmaf(wl[base * KK + t], gsum[KK + br * KK + t], a);
    dsl[base] = a;
  }
}

}  // namespace wt
