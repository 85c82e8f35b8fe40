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
  for (int i = threadIdx.x; i < total; i += NT) {
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

// ------------------------------------------------------------ staging
// Reads plane `xp` (H x W, I/O dtype) into the shifted fp32 buffer xf and,
// when L >= 1, writes its level-1 Haar subbands into the shifted 4-band
// buffer s1.  Only the image interior is written; borders stay zero.
// Optionally accumulates the sum of all values read into *sum.
template <typename IO, bool SUM>
__device__ void stage_plane(const Plan& P, const IO* __restrict__ xp, float* xf, int ldx, float* s1, int ld1,
                            int bs1, bool shifted, float* sum) {
  const int r = shifted ? P.r : 0;
  const int Q = (P.W + 3) >> 2;
  if (P.L >= 1) {
    const int items = P.H1 * Q;
    for (int it = threadIdx.x; it < items; it += NT) {
      const int i = it / Q, q = it - i * Q;
      const int x0 = q << 2;
      const IO* p0 = xp + (size_t)(2 * i) * P.W + x0;
      const float4 a = load4(p0, x0, P.W, P.vec_in);
      const float4 b = load4(p0 + P.W, x0, P.W, P.vec_in);
      if (SUM) *sum += ((a.x + a.y) + (a.z + a.w)) + ((b.x + b.y) + (b.z + b.w));
      float* d0 = xf + (2 * i + r) * ldx + x0 + r;
      float* d1 = d0 + ldx;
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (x0 + e < P.W) {
          d0[e] = av[e];
          d1[e] = bv[e];
        }
      float* o = s1 + (i + r) * ld1 + (x0 >> 1) + r;
#pragma unroll
      for (int bk = 0; bk < 2; ++bk) {
        if (x0 + 2 * bk < P.W) {
          float ll, lh, hl, hh;
          haar4(av[2 * bk], av[2 * bk + 1], bv[2 * bk], bv[2 * bk + 1], ll, lh, hl, hh);
          o[bk] = ll;
          o[bs1 + bk] = lh;
          o[2 * bs1 + bk] = hl;
          o[3 * bs1 + bk] = hh;
        }
      }
    }
  } else {
    const int items = P.H * Q;
    for (int it = threadIdx.x; it < items; it += NT) {
      const int y = it / Q, q = it - y * Q;
      const int x0 = q << 2;
      const float4 a = load4(xp + (size_t)y * P.W + x0, x0, P.W, P.vec_in);
      if (SUM) *sum += (a.x + a.y) + (a.z + a.w);
      float* d0 = xf + (y + r) * ldx + x0 + r;
      const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (x0 + e < P.W) d0[e] = av[e];
    }
  }
}

// Haar analysis of the LL band of level l-1 into the 4 bands of level l
// for every plane of the batch.  src: LL of level l-1 at interior origin.
__device__ void pyramid_level(int npb, int hl, int wlv, const float* src0, int lds, int src_ps, float* dst0,
                              int ldd, int bsd, int dst_ps) {
  const int per = hl * wlv;
  for (int it = threadIdx.x; it < npb * per; it += NT) {
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

// ------------------------------------------------------------ deep levels
// Levels 2..L of the batch: pyramid, level convs, closed-form synthesis of
// levels >= 3 at level-2 resolution (t2), then the level-2 conv fused with
// its synthesis butterfly into t1 (level-1 resolution).  Ends synchronised.
template <int K>
__device__ void deep_forward(const Plan& P, float* sm, const float* sw, int npb) {
  const int r = P.r;
  const int kk4 = P.kk4;
  // the deep region aliases the level-1 conv buffer: clear borders first
  for (int pb = 0; pb < npb; ++pb) {
    float4* z = reinterpret_cast<float4*>(sm + P.deep_off + pb * P.xf.ps);
    for (int i = threadIdx.x; i < (P.deep_floats >> 2); i += NT) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  __syncthreads();
  for (int l = 2; l <= P.L; ++l) {
    const BufDesc& d = P.sd[l];
    const float* src;
    int lds;
    if (l == 2) {
      src = sm + P.s1.off + r * P.s1.ld + r;
      lds = P.s1.ld;
    } else {
      src = sm + P.sd[l - 1].off + r * P.sd[l - 1].ld + r;
      lds = P.sd[l - 1].ld;
    }
    pyramid_level(npb, P.H >> l, P.W >> l, src, lds, P.xf.ps, sm + d.off + r * d.ld + r, d.ld, d.ld * d.rows,
                  P.xf.ps);
    __syncthreads();
  }
  if (P.L >= 3) {
    // level convs l = 3..L (folded weights); items (pb, l, s, tile)
    int per_plane = 0;
    for (int l = 3; l <= P.L; ++l) per_plane += 4 * cdiv(P.H >> l, DP_R) * cdiv(P.W >> l, DP_CW);
    for (int it = threadIdx.x; it < npb * per_plane; it += NT) {
      const int pb = it / per_plane;
      int rem = it - pb * per_plane;
      int l = 3;
      for (;;) {
        const int n = 4 * cdiv(P.H >> l, DP_R) * cdiv(P.W >> l, DP_CW);
        if (rem < n) break;
        rem -= n;
        ++l;
      }
      const int tx = cdiv(P.W >> l, DP_CW), tpb = cdiv(P.H >> l, DP_R) * tx;
      const int s = rem / tpb;
      rem -= s * tpb;
      const int ti = rem / tx, tj = rem - ti * tx;
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
    // t2(i,j) = sum_{l>=3} sum_s sigma_s(bit_{l-3}(i), bit_{l-3}(j)) Zd_l^s(i >> (l-2), j >> (l-2))
    const int h2 = P.H >> 2, w2 = P.W >> 2;
    for (int it = threadIdx.x; it < npb * h2 * w2; it += NT) {
      const int pb = it / (h2 * w2), rem = it - pb * h2 * w2;
      const int i = rem / w2, j = rem - i * w2;
      float acc = 0.f;
      for (int l = 3; l <= P.L; ++l) {
        const BufDesc& z = P.zd[l];
        const int bz = z.ld * z.rows;
        const float* q = sm + z.off + pb * z.ps + (i >> (l - 2)) * z.ld + (j >> (l - 2));
        const int by = (i >> (l - 3)) & 1, bx = (j >> (l - 3)) & 1;
        const float zlh = q[bz], zhl = q[2 * bz], zhh = q[3 * bz];
        acc += q[0] + (by ? -zlh : zlh) + (bx ? -zhl : zhl) + ((by ^ bx) ? -zhh : zhh);
      }
      sm[P.t2.off + pb * P.t2.ps + i * P.t2.ld + j] = acc;
    }
    __syncthreads();
  }
  {
    // level 2: conv of the 4 bands + t2 on LL, synthesis butterfly into t1
    const int h2 = P.H >> 2, w2 = P.W >> 2;
    const int tx = cdiv(w2, DP_CW), per = cdiv(h2, DP_R) * tx;
    const BufDesc& d = P.sd[2];
    const int bs = d.ld * d.rows;
    for (int it = threadIdx.x; it < npb * per; it += NT) {
      const int pb = it / per, rem = it - pb * per;
      const int ti = rem / tx, tj = rem - ti * tx;
      const int i0 = ti * DP_R, j0 = tj * DP_CW;
      float acc[4][DP_R][DP_CW];
#pragma unroll
      for (int s = 0; s < 4; ++s)
#pragma unroll
        for (int a = 0; a < DP_R; ++a)
#pragma unroll
          for (int b = 0; b < DP_CW; ++b) acc[s][a][b] = 0.f;
      const float* in = sm + d.off + pb * d.ps + i0 * d.ld + j0;
#pragma unroll
      for (int s = 0; s < 4; ++s) conv_tile<K, DP_R, DP_CW>(in + s * bs, d.ld, sw + wl_off(kk4, 2, s), acc[s]);
      if (P.L >= 3) {
        const float* t2 = sm + P.t2.off + pb * P.t2.ps + i0 * P.t2.ld + j0;
#pragma unroll
        for (int a = 0; a < DP_R; ++a) {
          const float4 t = reinterpret_cast<const float4*>(t2 + a * P.t2.ld)[0];
          acc[0][a][0] += t.x;
          acc[0][a][1] += t.y;
          acc[0][a][2] += t.z;
          acc[0][a][3] += t.w;
        }
      }
      float* t1 = sm + P.t1.off + pb * P.t1.ps;
#pragma unroll
      for (int a = 0; a < DP_R; ++a)
#pragma unroll
        for (int b = 0; b < DP_CW; ++b) {
          if (i0 + a < h2 && j0 + b < w2) {
            float o00, o01, o10, o11;
            synth4(acc[0][a][b], acc[1][a][b], acc[2][a][b], acc[3][a][b], o00, o01, o10, o11);
            float* q = t1 + 2 * (i0 + a) * P.t1.ld + 2 * (j0 + b);
            q[0] = o00;
            q[1] = o01;
            q[P.t1.ld] = o10;
            q[P.t1.ld + 1] = o11;
          }
        }
    }
    __syncthreads();
  }
}

// Level-1 band convs of the batch into zb (t1 added to the LL band).
template <int K>
__device__ void level1_conv(const Plan& P, float* sm, const float* sw, int npb) {
  const int tx = cdiv(P.W1, C2_CW), per_band = cdiv(P.H1, C2_R) * tx, per = 4 * per_band;
  const int bs1 = P.s1.ld * P.s1.rows, bsz = P.zb.ld * P.zb.rows;
  for (int it = threadIdx.x; it < npb * per; it += NT) {
    const int pb = it / per;
    int rem = it - pb * per;
    const int s = rem / per_band;
    rem -= s * per_band;
    const int ti = rem / tx, tj = rem - ti * tx;
    const int i0 = ti * C2_R, j0 = tj * C2_CW;
    float acc[C2_R][C2_CW];
#pragma unroll
    for (int a = 0; a < C2_R; ++a)
#pragma unroll
      for (int b = 0; b < C2_CW; ++b) acc[a][b] = 0.f;
    conv_tile<K, C2_R, C2_CW>(sm + P.s1.off + pb * P.s1.ps + s * bs1 + i0 * P.s1.ld + j0, P.s1.ld,
                              sw + wl_off(P.kk4, 1, s), acc);
    if (s == 0 && P.L >= 2) {
      const float* t1 = sm + P.t1.off + pb * P.t1.ps + i0 * P.t1.ld + j0;
#pragma unroll
      for (int a = 0; a < C2_R; ++a) {
        const float4 t = reinterpret_cast<const float4*>(t1 + a * P.t1.ld)[0];
        acc[a][0] += t.x;
        acc[a][1] += t.y;
        acc[a][2] += t.z;
        acc[a][3] += t.w;
      }
    }
    float* o = sm + P.zb.off + pb * P.zb.ps + s * bsz + i0 * P.zb.ld + j0;
#pragma unroll
    for (int a = 0; a < C2_R; ++a)
      reinterpret_cast<float4*>(o + a * P.zb.ld)[0] = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
  }
}

// Base conv + level-1 synthesis + bias; writes the output rows.
template <int K, int R3, typename IO>
__device__ void output_pass(const Plan& P, float* sm, const float* sw, IO* __restrict__ y, int c, int nb0,
                            int npb) {
  const int tx = cdiv(P.W, C3_CW), per = cdiv(P.H, R3) * tx;
  const int bsz = P.zb.ld * P.zb.rows;
  const float bias = sw[P.kk4];
  for (int it = threadIdx.x; it < npb * per; it += NT) {
    const int pb = it / per, rem = it - pb * per;
    const int ti = rem / tx, tj = rem - ti * tx;
    const int yy0 = ti * R3, xx0 = tj * C3_CW;
    float acc[R3][C3_CW];
    if (P.L >= 1) {
#pragma unroll
      for (int bi = 0; bi < R3 / 2; ++bi) {
        const float* z = sm + P.zb.off + pb * P.zb.ps + ((yy0 >> 1) + bi) * P.zb.ld + (xx0 >> 1);
        const float4 zll = reinterpret_cast<const float4*>(z)[0];
        const float4 zlh = reinterpret_cast<const float4*>(z + bsz)[0];
        const float4 zhl = reinterpret_cast<const float4*>(z + 2 * bsz)[0];
        const float4 zhh = reinterpret_cast<const float4*>(z + 3 * bsz)[0];
        const float a0[4] = {zll.x, zll.y, zll.z, zll.w}, a1[4] = {zlh.x, zlh.y, zlh.z, zlh.w};
        const float a2[4] = {zhl.x, zhl.y, zhl.z, zhl.w}, a3[4] = {zhh.x, zhh.y, zhh.z, zhh.w};
#pragma unroll
        for (int bj = 0; bj < 4; ++bj) {
          float o00, o01, o10, o11;
          synth4(a0[bj], a1[bj], a2[bj], a3[bj], o00, o01, o10, o11);
          acc[2 * bi][2 * bj] = bias + o00;
          acc[2 * bi][2 * bj + 1] = bias + o01;
          acc[2 * bi + 1][2 * bj] = bias + o10;
          acc[2 * bi + 1][2 * bj + 1] = bias + o11;
        }
      }
    } else {
#pragma unroll
      for (int a = 0; a < R3; ++a)
#pragma unroll
        for (int b = 0; b < C3_CW; ++b) acc[a][b] = bias;
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
// consecutive n); grid-strided over C * nbatch units.
template <int K, int R3, typename IO>
__global__ void __launch_bounds__(NT) wtconv_fwd_kernel(const Plan P, const IO* __restrict__ x,
                                                        const float* __restrict__ w0, const float* __restrict__ b0,
                                                        const float* __restrict__ s0, const float* __restrict__ wl,
                                                        const float* __restrict__ sl, IO* __restrict__ y, int flip) {
  extern __shared__ float4 smem4[];
  float* sm = reinterpret_cast<float*>(smem4);
  for (int i = threadIdx.x; i < (P.smem_floats >> 2); i += NT) smem4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  __syncthreads();
  const int units = P.C * P.nbatch;
  float* sw = sm + P.w_off;
  for (int u = blockIdx.x; u < units; u += gridDim.x) {
    const int c = u % P.C, bt = u / P.C;
    const int nb0 = bt * P.PB;
    const int npb = (P.N - nb0) < P.PB ? (P.N - nb0) : P.PB;
    load_weights<K>(P, sw, c, w0, b0, s0, wl, sl, flip);
    for (int pb = 0; pb < npb; ++pb) {
      const IO* xp = x + ((size_t)(nb0 + pb) * P.C + c) * P.H * P.W;
      stage_plane<IO, false>(P, xp, sm + P.xf.off + pb * P.xf.ps, P.xf.ld, sm + P.s1.off + pb * P.s1.ps, P.s1.ld,
                             P.s1.ld * P.s1.rows, true, nullptr);
    }
    __syncthreads();
    if (P.L >= 2) deep_forward<K>(P, sm, sw, npb);
    if (P.L >= 1) {
      level1_conv<K>(P, sm, sw, npb);
      __syncthreads();
    }
    output_pass<K, R3, IO>(P, sm, sw, y, c, nb0, npb);
    __syncthreads();
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
                                                         const IO* __restrict__ dy, float* __restrict__ part) {
  constexpr int KK = K * K;
  extern __shared__ float4 smem4[];
  float* sm = reinterpret_cast<float*>(smem4);
  for (int i = threadIdx.x; i < (P.smem_floats >> 2); i += NT) smem4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  __syncthreads();
  const int r = P.r;
  const int kk4 = P.kk4;
  const int c = blockIdx.x % P.C, g = blockIdx.x / P.C;
  const int n_begin = g * P.planes_per_cta;
  const int n_end = min(P.N, n_begin + P.planes_per_cta);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nbase = P.L >= 1 ? 128 : NT;   // threads on the base taps
  float G[KK];
  zero_taps<K>(G);
  float sumdy = 0.f;
  const int ndeep = P.L >= 2 ? (P.L - 1) * 4 : 0;

  for (int nb0 = n_begin; nb0 < n_end; nb0 += P.PB) {
    const int npb = (n_end - nb0) < P.PB ? (n_end - nb0) : P.PB;
    for (int pb = 0; pb < npb; ++pb) {
      const size_t po = ((size_t)(nb0 + pb) * P.C + c) * P.H * P.W;
      stage_plane<IO, false>(P, x + po, sm + P.xf.off + pb * P.xf.ps, P.xf.ld, sm + P.s1.off + pb * P.s1.ps,
                             P.s1.ld, P.s1.ld * P.s1.rows, true, nullptr);
      stage_plane<IO, true>(P, dy + po, sm + P.gf.off + pb * P.gf.ps, P.gf.ld, sm + P.g1.off + pb * P.g1.ps,
                            P.g1.ld, P.g1.ld * P.g1.rows, false, &sumdy);
    }
    __syncthreads();
    for (int l = 2; l <= P.L; ++l) {
      const BufDesc& d = P.sd[l];
      const BufDesc& e = P.gd[l];
      const float* srcx = (l == 2) ? sm + P.s1.off + r * P.s1.ld + r : sm + P.sd[l - 1].off + r * P.sd[l - 1].ld + r;
      const int ldsx = (l == 2) ? P.s1.ld : P.sd[l - 1].ld;
      const float* srcg = (l == 2) ? sm + P.g1.off : sm + P.gd[l - 1].off;
      const int ldsg = (l == 2) ? P.g1.ld : P.gd[l - 1].ld;
      pyramid_level(npb, P.H >> l, P.W >> l, srcx, ldsx, P.xf.ps, sm + d.off + r * d.ld + r, d.ld, d.ld * d.rows,
                    P.xf.ps);
      pyramid_level(npb, P.H >> l, P.W >> l, srcg, ldsg, P.xf.ps, sm + e.off, e.ld, e.ld * e.rows, P.xf.ps);
      __syncthreads();
    }
    // base and level-1 taps: register accumulation across planes
    if (threadIdx.x < nbase) {
      const int tx = cdiv(P.W, BW_CW), per = cdiv(P.H, BW_R) * tx;
      for (int it = threadIdx.x; it < npb * per; it += nbase) {
        const int pb = it / per, rem = it - pb * per;
        const int ti = rem / tx, tj = rem - ti * tx;
        const int y0 = ti * BW_R, x0 = tj * BW_CW;
        corr_tile<K, BW_R, BW_CW>(sm + P.xf.off + pb * P.xf.ps + y0 * P.xf.ld + x0, P.xf.ld,
                                  sm + P.gf.off + pb * P.gf.ps + y0 * P.gf.ld + x0, P.gf.ld, G);
      }
    } else {
      const int s = warp - 4;
      const int tx = cdiv(P.W1, B1_CW), per = cdiv(P.H1, B1_R) * tx;
      for (int it = lane; it < npb * per; it += 32) {
        const int pb = it / per, rem = it - pb * per;
        const int ti = rem / tx, tj = rem - ti * tx;
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
        const int hl = P.H >> l, wlv = P.W >> l;
        const int tx = cdiv(wlv, DP_CW), per = cdiv(hl, DP_R) * tx;
        const BufDesc& d = P.sd[l];
        const BufDesc& e = P.gd[l];
        float Gd[KK];
        zero_taps<K>(Gd);
        for (int t = slot; t < npb * per; t += DSLOTS) {
          const int pb = t / per, rem = t - pb * per;
          const int ti = rem / tx, tj = rem - ti * tx;
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
