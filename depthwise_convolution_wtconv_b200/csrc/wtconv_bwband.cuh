// Row-band weight-gradient kernel for planes too large to keep whole in one
// SM's shared memory (sm_100a).
//
// The weight gradients are sums over the image of local products, so they
// split over row bands of a plane.  The pass runs one launch per level:
//
//   level 1 (or level 0 when L = 0): reads bands of x and dy; forms the base
//     correlation G_0 = sum dy(i,j) x(i+u-r, j+v-r) and sum(dy) from the
//     staged rows, and, for L >= 1, the Haar subbands of both on chip
//     (reformulation (1) of arXiv:2608.10805, abstract) and their four band
//     correlations G_1[s] = sum dZ_1^s(i,j) sub_1^s(i+u-r, j+v-r);
//   level l >= 2: the same band correlations one level down, on the raw LL
//     of the level above.
//
// Only the raw LL bands (a quarter of the level's input) go back to HBM for
// the next launch; the detail subbands never leave the chip.  A band of TB
// rows of the level grid needs 2*TB input rows of dy and 2*TB + 4r rows of
// x (the correlation halo of r rows at the level grid).
//
// Each CTA owns channel c = blockIdx.x % C and the units (image n, band b)
// u = g, g + G, g + 2G, ... of that channel (g = blockIdx.x / C); its
// register sums are reduced by a fixed warp-shuffle tree and a fixed
// warp order, and written to this launch's segment of the CTA's partial
// vector part[g][c][V] (the layout of the whole-plane kernel).  Every
// launch uses the same G, so the fixed-order finalize applies unchanged.
#pragma once

#include "wtconv_main.cuh"

namespace wt {

// Stages `rows` rows of a plane (row y0 first; rows outside [0, h) are
// written as zeros) into shared memory at dst + i*ld + COL0, converting to
// fp32.  The rows come from the plane in global memory, or (SMEM) from a
// raw copy in shared memory holding row i of the window at raw + i*w.
// Returns this thread's sum of the staged in-image values when SUM.  Full
// 4-element groups are stored with the widest aligned stores COL0 allows.
// Haar analysis of the 2x2 block at src (rows ld apart): one 8-byte load per
// row when the block starts on an 8-byte boundary (ALIGNED), else scalars.
template <bool ALIGNED>
__device__ __forceinline__ void haar_pair(const float* src, int ld, float& ll, float& lh, float& hl, float& hh) {
  if constexpr (ALIGNED) {
    const float2 top = *reinterpret_cast<const float2*>(src);
    const float2 bot = *reinterpret_cast<const float2*>(src + ld);
    haar4(top.x, top.y, bot.x, bot.y, ll, lh, hl, hh);
  } else {
    haar4(src[0], src[1], src[ld], src[ld + 1], ll, lh, hl, hh);
  }
}

template <typename IN, bool SUM, bool SMEM, int COL0>
__device__ __forceinline__ float stage_band_rows(const IN* __restrict__ src, const IN* raw, int h, int w, int y0,
                                                 int rows, float* __restrict__ dst, int ld, bool vec, FDiv fq4) {
  float sum = 0.f;
  const int q4 = fq4.d;  // (w + 3) / 4
  for (int it = threadIdx.x; it < rows * q4; it += NT) {
    const int i = fq4.div(it), q = it - i * q4;
    const int y = y0 + i, x = 4 * q;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (y >= 0 && y < h) {
      if constexpr (SMEM)
        v = lds4(raw + (size_t)i * w + x, x, w, vec);
      else
        v = load4(src + (size_t)y * w + x, x, w, vec);
    }
    float* o = dst + i * ld + COL0 + x;
    if (x + 3 < w) {
      sts4<COL0>(o, v);
    } else {
      o[0] = v.x;
      if (x + 1 < w) o[1] = v.y;
      if (x + 2 < w) o[2] = v.z;
    }
    if (SUM) sum += (v.x + v.y) + (v.z + v.w);
  }
  return sum;
}

// 4 consecutive elements of a staged row in shared memory as one vector
// load (the row width is a multiple of 4 and x a multiple of 4).
__device__ __forceinline__ float4 lds4v(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 lds4v(const __nv_bfloat16* p) {
  const uint2 raw = *reinterpret_cast<const uint2*>(p);
  return make_float4(__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xffff0000u),
                     __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xffff0000u));
}

// Levels >= 1 with bulk-copied rows of width W % 4 == 0: staging and the Haar
// step in one pass.  Each item takes two rows x four columns of one input
// (the x window: TB + 2r level rows from i0 - r, rows outside the image as
// zeros; or the dy band: TB level rows), stores the two fp32 rows (x
// shifted by r columns, dy plain), their two 2x2 blocks' subbands (x: into
// s, shifted; dy: into d, plain) and the raw LL to the next level; returns
// this thread's sum of the dy values.
template <int K, typename IN>
__device__ __forceinline__ float band_stage_haar(const BandPlan& P, const IN* rawa, const IN* rawb, float* sa, float* sb,
                                                 float* ss, float* sd, int y0, size_t ll0, float* __restrict__ llx,
                                                 float* __restrict__ lld) {
  constexpr int r = K / 2;
  const int q4 = P.f_q4.d;  // W / 4
  const int nx = (P.TB + 2 * r) * q4, ny = P.TB * q4;
  const int s_band = P.s_ld * P.s_rows, d_band = P.d_ld * P.d_rows, wl = P.Wl;
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  float sum = 0.f;
  for (int it = threadIdx.x; it < nx + ny; it += NT) {
    const bool isx = it < nx;
    const int e = isx ? it : it - nx;
    const int q = P.f_q4.div(e), x = (e - q * q4) << 2;
    const int jj = x >> 1;
    float l0, h0, g0, k0, l1, h1, g1, k1;
    if (isx) {
      const int y = y0 - P.ha + 2 * q;  // rows y, y + 1 of the image are rows 2q, 2q + 1 of the window
      const float4 v0 = (y >= 0 && y < P.H) ? lds4v(rawa + (size_t)(2 * q) * P.W + x) : zero;
      const float4 v1 = (y + 1 >= 0 && y + 1 < P.H) ? lds4v(rawa + (size_t)(2 * q + 1) * P.W + x) : zero;
      float* o = sa + 2 * q * P.a_ld + r + x;
      sts4<r>(o, v0);
      sts4<r>(o + P.a_ld, v1);
      haar4(v0.x, v0.y, v1.x, v1.y, l0, h0, g0, k0);
      haar4(v0.z, v0.w, v1.z, v1.w, l1, h1, g1, k1);
      float* so = ss + q * P.s_ld + r + jj;
      sts2<r>(so, l0, l1);
      sts2<r>(so + s_band, h0, h1);
      sts2<r>(so + 2 * s_band, g0, g1);
      sts2<r>(so + 3 * s_band, k0, k1);
      const int qi = q - r;
      if (P.write_ll && qi >= 0 && qi < P.TB) {
        llx[ll0 + (size_t)qi * wl + jj] = l0;
        llx[ll0 + (size_t)qi * wl + jj + 1] = l1;
      }
    } else {
      const float4 v0 = lds4v(rawb + (size_t)(2 * q) * P.W + x);
      const float4 v1 = lds4v(rawb + (size_t)(2 * q + 1) * P.W + x);
      float* o = sb + 2 * q * P.b_ld + x;
      *reinterpret_cast<float4*>(o) = v0;
      *reinterpret_cast<float4*>(o + P.b_ld) = v1;
      sum += ((v0.x + v0.y) + (v0.z + v0.w)) + ((v1.x + v1.y) + (v1.z + v1.w));
      haar4(v0.x, v0.y, v1.x, v1.y, l0, h0, g0, k0);
      haar4(v0.z, v0.w, v1.z, v1.w, l1, h1, g1, k1);
      float* dd = sd + q * P.d_ld + jj;
      *reinterpret_cast<float2*>(dd) = make_float2(l0, l1);
      *reinterpret_cast<float2*>(dd + d_band) = make_float2(h0, h1);
      *reinterpret_cast<float2*>(dd + 2 * d_band) = make_float2(g0, g1);
      *reinterpret_cast<float2*>(dd + 3 * d_band) = make_float2(k0, k1);
      if (P.write_ll) {
        lld[ll0 + (size_t)q * wl + jj] = l0;
        lld[ll0 + (size_t)q * wl + jj + 1] = l1;
      }
    }
  }
  return sum;
}

template <int K, typename IN>
__global__ void __launch_bounds__(NT, 2) wtconv_bwband_kernel(const BandPlan P, const IN* __restrict__ A,
                                                              const IN* __restrict__ B, float* __restrict__ llx,
                                                              float* __restrict__ lld, float* __restrict__ part,
                                                              int* __restrict__ status) {
  constexpr int KK = K * K;
  constexpr int r = K / 2;
  extern __shared__ float4 smem4[];
  float* sm = reinterpret_cast<float*>(smem4);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + 2);
  for (int i = threadIdx.x; i < (P.smem_floats >> 2); i += NT) smem4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  __syncthreads();
  if (threadIdx.x == 0) {
    mb_init(full, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const int c = blockIdx.x % P.C, g = blockIdx.x / P.C;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nbase = P.lvl == 0 ? NT : (P.lvl == 1 ? 128 : 0);  // threads on the base taps
  const int tpb = (NT - nbase) >> 2;                           // threads per subband
  const size_t plane = (size_t)P.H * P.W;
  float* sa = sm + P.a_off;
  float* sb = sm + P.b_off;
  float* ss = sm + P.s_off;
  float* sd = sm + P.d_off;
  const int s_band = P.s_ld * P.s_rows, d_band = P.d_ld * P.d_rows;
  float G[KK];
  zero_taps<K>(G);
  float sumdy = 0.f;
  const IN* rawa = reinterpret_cast<const IN*>(sm + P.raw_a);
  const IN* rawb = reinterpret_cast<const IN*>(sm + P.raw_b);
  // bulk copies of a unit's rows: the A rows of its window that lie in the
  // image (at their row of the window) and its B rows
  auto issue = [&](int u) {
    const int n = P.f_nb.div(u), b = u - n * P.nb;
    const int y0 = P.lvl == 0 ? b * P.TB : 2 * b * P.TB;
    const int y_lo = max(0, y0 - P.ha), y_hi = min(P.H, y0 + P.FR + P.ha);
    const unsigned ba = (unsigned)((y_hi - y_lo) * P.W * sizeof(IN));
    const unsigned bbytes = (unsigned)(P.FR * P.W * sizeof(IN));
    const size_t po = ((size_t)n * P.C + c) * plane;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(full)), "r"(ba + bbytes)
                 : "memory");
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(rawa + (size_t)(y_lo - (y0 - P.ha)) * P.W)),
        "l"(A + po + (size_t)y_lo * P.W), "r"(ba), "r"(smem_u32(full))
        : "memory");
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(rawb)),
        "l"(B + po + (size_t)y0 * P.W), "r"(bbytes), "r"(smem_u32(full))
        : "memory");
  };
  if (P.bulk && threadIdx.x == 0 && g < P.units) issue(g);
  int k = 0;
  for (int u = g; u < P.units; u += P.ngroups, ++k) {
    const int n = P.f_nb.div(u), b = u - n * P.nb;
    const int i0 = b * P.TB;                     // first row of the level grid
    const int y0 = P.lvl == 0 ? i0 : 2 * i0;     // first input row of the band
    const IN* a = A + ((size_t)n * P.C + c) * plane;
    const IN* bb = B + ((size_t)n * P.C + c) * plane;
    float sdy;
    const size_t ll0 = ((size_t)n * P.C + c) * P.Hl * P.Wl + (size_t)i0 * P.Wl;
    // levels >= 1, bulk-copied rows of width W % 4 == 0: staging and Haar step in one pass
    const bool joint = P.lvl >= 1 && P.bulk && P.vec && (P.W % 4) == 0;
    if (joint) {
      mb_wait(full, k & 1, abort_flag);
      sdy = band_stage_haar<K, IN>(P, rawa, rawb, sa, sb, ss, sd, y0, ll0, llx, lld);
    } else if (P.bulk) {
      mb_wait(full, k & 1, abort_flag);
      stage_band_rows<IN, false, true, r>(a, rawa, P.H, P.W, y0 - P.ha, P.FR + 2 * P.ha, sa, P.a_ld, P.vec, P.f_q4);
      sdy = stage_band_rows<IN, true, true, 0>(bb, rawb, P.H, P.W, y0, P.FR, sb, P.b_ld, P.vec, P.f_q4);
    } else {
      stage_band_rows<IN, false, false, r>(a, nullptr, P.H, P.W, y0 - P.ha, P.FR + 2 * P.ha, sa, P.a_ld, P.vec, P.f_q4);
      sdy = stage_band_rows<IN, true, false, 0>(bb, nullptr, P.H, P.W, y0, P.FR, sb, P.b_ld, P.vec, P.f_q4);
    }
    if (P.lvl <= 1) sumdy += sdy;
    __syncthreads();
    if (*abort_flag) break;  // uniform: read after the barrier
    if (P.bulk && threadIdx.x == 0 && u + P.ngroups < P.units) issue(u + P.ngroups);
    if (P.lvl >= 1 && !joint) {
      // subbands of x over TB + 2r level rows (the halo rows outside the
      // image come out zero from the zero rows staged above) and of dy over
      // the TB band rows; raw LL of the band rows to the next level
      const int wl = P.Wl;
      const int nsub = (P.TB + 2 * r) * wl;
      for (int it = threadIdx.x; it < nsub; it += NT) {
        const int q = P.f_wl.div(it), jj = it - q * wl;
        const float* src = sa + 2 * q * P.a_ld + r + 2 * jj;
        float ll, lh, hl, hh;
        haar_pair<r % 2 == 0>(src, P.a_ld, ll, lh, hl, hh);
        float* o = ss + q * P.s_ld + r + jj;
        o[0] = ll;
        o[s_band] = lh;
        o[2 * s_band] = hl;
        o[3 * s_band] = hh;
        const int qi = q - r;
        if (P.write_ll && qi >= 0 && qi < P.TB) llx[ll0 + (size_t)qi * wl + jj] = ll;
      }
      for (int it = threadIdx.x; it < P.TB * wl; it += NT) {
        const int q = P.f_wl.div(it), jj = it - q * wl;
        float ll, lh, hl, hh;
        haar_pair<true>(sb + 2 * q * P.b_ld + 2 * jj, P.b_ld, ll, lh, hl, hh);
        float* o = sd + q * P.d_ld + jj;
        o[0] = ll;
        o[d_band] = lh;
        o[2 * d_band] = hl;
        o[3 * d_band] = hh;
        if (P.write_ll) lld[ll0 + (size_t)q * wl + jj] = ll;
      }
      __syncthreads();
    }
    if ((int)threadIdx.x < nbase) {
      const int tx = P.f_bx.d, per = P.f_bper.d;
      for (int it = threadIdx.x; it < per; it += nbase) {
        const int ti = P.f_bx.div(it), tj = it - ti * tx;
        const int yy = ti * BW_R, x0 = tj * BW_CW;
        corr_tile<K, BW_R, BW_CW>(sa + (P.ha - r + yy) * P.a_ld + x0, P.a_ld, sb + yy * P.b_ld + x0, P.b_ld, G);
      }
    } else {
      const int t = threadIdx.x - nbase;
      const int s = t / tpb, lt = t - s * tpb;
      const int tx = P.f_sx.d, per = P.f_sper.d;
      for (int it = lt; it < per; it += tpb) {
        const int ti = P.f_sx.div(it), tj = it - ti * tx;
        const int q0 = ti * B1_R, j0 = tj * B1_CW;
        corr_tile<K, B1_R, B1_CW>(ss + s * s_band + q0 * P.s_ld + j0, P.s_ld, sd + s * d_band + q0 * P.d_ld + j0,
                                  P.d_ld, G);
      }
    }
    __syncthreads();
  }

  if (*abort_flag) {
    if (threadIdx.x == 0) {
      mb_drain(full, k & 1);  // the copies of unit k were issued; let them land before exit
      if (status) atomicExch(status, 1);
    }
    return;
  }
  // fixed-order reduction: shuffle tree within each warp, then warps in order
  float* red = sm + P.red_off;
#pragma unroll
  for (int t = 0; t < KK; ++t) {
    const float v = warp_sum(G[t]);
    if (lane == 0) red[warp * P.kk4 + t] = v;
  }
  {
    const float v = warp_sum(sumdy);
    if (lane == 0) red[(NT / 32) * P.kk4 + warp] = v;
  }
  __syncthreads();
  float* out = part + ((size_t)g * P.C + c) * P.V;
  const int nbw = nbase >> 5, wpb = tpb >> 5;
  if (P.lvl <= 1) {
    for (int t = threadIdx.x; t < KK; t += NT) {
      float acc = 0.f;
      for (int w = 0; w < nbw; ++w) acc += red[w * P.kk4 + t];
      out[t] = acc;
    }
    if (threadIdx.x == 0) {
      float acc = 0.f;
      for (int w = 0; w < NT / 32; ++w) acc += red[(NT / 32) * P.kk4 + w];
      out[P.V - 1] = acc;
    }
  }
  if (P.lvl >= 1) {
    for (int e = threadIdx.x; e < 4 * KK; e += NT) {
      const int s = e / KK, t = e - s * KK;
      float acc = 0.f;
      for (int w = 0; w < wpb; ++w) acc += red[(nbw + s * wpb + w) * P.kk4 + t];
      out[P.seg + e] = acc;
    }
  }
}

}  // namespace wt
