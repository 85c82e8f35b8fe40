// Whole-plane weight-gradient kernel (sm_100a).
//
// G_0[u,v] = sum dy(i,j) x(i+u-r, j+v-r) and, for every level l and band s,
// G_l^s[u,v] = sum dZ_l^s(i,j) sub_l^s(i+u-r, j+v-r), where sub_l and dZ_l
// are the Haar pyramids of x and dy (the adjoint of the synthesis cascade is
// the analysis).  A CTA owns one channel and a run of its planes; the
// planes' pyramids are built on chip from one read of x and dy
// (reformulation (1) of arXiv:2608.10805, abstract), so no subband reaches
// HBM.  Thread 0 keeps the next unit's raw planes in flight with bulk
// copies while the CTA works on the current one.
//
// Every branch (the base taps, and each band of each level) runs the same
// 4x4 register tile, so a warp whose threads belong to different branches
// still executes one instruction stream.  The host gives each branch a
// fixed range of threads sized to its share of the tiles; a thread keeps one
// set of K*K sums in registers across all of the CTA's planes, and the CTA
// reduces them at the end in a fixed order (threads of a branch in index
// order), so results are the same on every run.
#pragma once

#include "wtconv_main.cuh"

namespace wt {

// Staging of one BH x 4 block of plane j (BH = 4, 2, 1 for L >= 2, 1, 0):
// x into the padded rows xf, its level-1 subbands into s1 (shifted) and its
// level-2 subbands into sd[2]; dy likewise into gf, g1 and gd[2] (plain).
// Returns the sum of the block's dy values.
template <int K, int LC, typename IO, bool SMEM>
__device__ __forceinline__ float bw_stage_block(const BwPlan& P, float* slot, int j, const IO* __restrict__ xs,
                                                const IO* __restrict__ gs, int by, int bx) {
  constexpr int r = K / 2;
  constexpr int BH = LC == 2 ? 4 : (LC == 1 ? 2 : 1);
  const int x0 = bx << 2, y0 = by * BH;
  const bool vec = P.vec_in != 0;
  const bool full = x0 + 3 < P.W;
  float4 v[BH], q[BH];
#pragma unroll
  for (int i = 0; i < BH; ++i) {
    v[i] = src4<SMEM>(xs + (size_t)(y0 + i) * P.W + x0, x0, P.W, vec);
    q[i] = src4<SMEM>(gs + (size_t)(y0 + i) * P.W + x0, x0, P.W, vec);
  }
  float sum = 0.f;
  float* xf = slot + P.xf.off + j * P.ps + (y0 + r) * P.xf.ld + x0 + r;
  float* gf = slot + P.gf.off + j * P.ps + y0 * P.gf.ld + x0;
#pragma unroll
  for (int i = 0; i < BH; ++i) {
    sum += (q[i].x + q[i].y) + (q[i].z + q[i].w);
    if (full) {
      sts4<r>(xf + i * P.xf.ld, v[i]);
      *reinterpret_cast<float4*>(gf + i * P.gf.ld) = q[i];
    } else {
      const float av[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
      const float qv[4] = {q[i].x, q[i].y, q[i].z, q[i].w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (x0 + e < P.W) {
          xf[i * P.xf.ld + e] = av[e];
          gf[i * P.gf.ld + e] = qv[e];
        }
    }
  }
  if constexpr (LC >= 1) {
    const int ld1 = P.s1.ld, bs1 = P.s1.ld * P.s1.rows;
    const int lg1 = P.g1.ld, bg1 = P.g1.ld * P.g1.rows;
    float* s1 = slot + P.s1.off + j * P.ps + ((y0 >> 1) + r) * ld1 + (x0 >> 1) + r;
    float* g1 = slot + P.g1.off + j * P.ps + (y0 >> 1) * lg1 + (x0 >> 1);
    float llx[BH / 2][2], llg[BH / 2][2];
#pragma unroll
    for (int a = 0; a < BH / 2; ++a) {
      float l0, h0, g0, k0, l1, h1, g1_, k1;
      haar4(v[2 * a].x, v[2 * a].y, v[2 * a + 1].x, v[2 * a + 1].y, l0, h0, g0, k0);
      haar4(v[2 * a].z, v[2 * a].w, v[2 * a + 1].z, v[2 * a + 1].w, l1, h1, g1_, k1);
      float m0, n0, o0, p0, m1, n1, o1, p1;
      haar4(q[2 * a].x, q[2 * a].y, q[2 * a + 1].x, q[2 * a + 1].y, m0, n0, o0, p0);
      haar4(q[2 * a].z, q[2 * a].w, q[2 * a + 1].z, q[2 * a + 1].w, m1, n1, o1, p1);
      if (full) {
        sts2<r>(s1 + a * ld1, l0, l1);
        sts2<r>(s1 + bs1 + a * ld1, h0, h1);
        sts2<r>(s1 + 2 * bs1 + a * ld1, g0, g1_);
        sts2<r>(s1 + 3 * bs1 + a * ld1, k0, k1);
        *reinterpret_cast<float2*>(g1 + a * lg1) = make_float2(m0, m1);
        *reinterpret_cast<float2*>(g1 + bg1 + a * lg1) = make_float2(n0, n1);
        *reinterpret_cast<float2*>(g1 + 2 * bg1 + a * lg1) = make_float2(o0, o1);
        *reinterpret_cast<float2*>(g1 + 3 * bg1 + a * lg1) = make_float2(p0, p1);
      } else {  // W % 4 == 2: one 2-wide block left in the row
        s1[a * ld1] = l0;
        s1[bs1 + a * ld1] = h0;
        s1[2 * bs1 + a * ld1] = g0;
        s1[3 * bs1 + a * ld1] = k0;
        g1[a * lg1] = m0;
        g1[bg1 + a * lg1] = n0;
        g1[2 * bg1 + a * lg1] = o0;
        g1[3 * bg1 + a * lg1] = p0;
      }
      llx[a][0] = l0;
      llx[a][1] = l1;
      llg[a][0] = m0;
      llg[a][1] = m1;
    }
    if constexpr (LC == 2) {
      const BufDesc& d = P.sd[2];
      const BufDesc& e = P.gd[2];
      float L2, H2, G2, K2;
      haar4(llx[0][0], llx[0][1], llx[1][0], llx[1][1], L2, H2, G2, K2);
      float* s2 = slot + d.off + j * P.ps + (by + r) * d.ld + bx + r;
      const int bs = d.ld * d.rows;
      s2[0] = L2;
      s2[bs] = H2;
      s2[2 * bs] = G2;
      s2[3 * bs] = K2;
      haar4(llg[0][0], llg[0][1], llg[1][0], llg[1][1], L2, H2, G2, K2);
      float* g2 = slot + e.off + j * P.ps + by * e.ld + bx;
      const int bg = e.ld * e.rows;
      g2[0] = L2;
      g2[bg] = H2;
      g2[2 * bg] = G2;
      g2[3 * bg] = K2;
    }
  }
  return sum;
}

template <int K, int LC, typename IO>
__global__ void __launch_bounds__(BW_NT, 2) wtconv_bwdw_kernel(const __grid_constant__ BwPlan P,
                                                               const IO* __restrict__ x,
                                                               const IO* __restrict__ dy, float* __restrict__ part,
                                                               int* __restrict__ status) {
  constexpr int KK = K * K;
  constexpr int r = K / 2;
  extern __shared__ float4 smem4[];
  float* sm = reinterpret_cast<float*>(smem4);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + 2);
  const int tid = threadIdx.x;
  for (int i = tid; i < (P.smem_floats >> 2); i += BW_NT) smem4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  __syncthreads();
  if (tid == 0) {
    mb_init(full, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const int c = blockIdx.x % P.C, grp = blockIdx.x / P.C;
  const int n_begin = grp * P.ppc, n_end = min(P.N, n_begin + P.ppc);
  float* slot = sm + MAIN_HEADER;
  const size_t plane = (size_t)P.H * P.W;
  const unsigned pbytes = (unsigned)(plane * sizeof(IO));
  auto issue = [&](int nb0) {
    const int cnt = min(P.PB, n_end - nb0);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(full)),
                 "r"(2u * pbytes * (unsigned)cnt)
                 : "memory");
    for (int jj = 0; jj < cnt; ++jj) {
      const size_t pi = ((size_t)(nb0 + jj) * P.C + c) * plane;
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
              smem_u32(slot + P.raw_x + jj * P.raw_pp)),
          "l"(x + pi), "r"(pbytes), "r"(smem_u32(full))
          : "memory");
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
              smem_u32(slot + P.raw_g + jj * P.raw_pp)),
          "l"(dy + pi), "r"(pbytes), "r"(smem_u32(full))
          : "memory");
    }
  };
  // this thread's branch (fixed for the whole CTA)
  int b = 0;
  while (b + 1 < P.nbr && tid >= P.br[b + 1].first) ++b;
  const BwBranch B = P.br[b];  // by value: registers, not per-use constant loads
  const int lt = tid - B.first;
  const bool busy = tid < P.br[P.nbr - 1].first + P.br[P.nbr - 1].nthr;
  float G[KK];
  zero_taps<K>(G);
  float sumdy = 0.f;
  if (P.bulk && tid == 0 && n_begin < n_end) issue(n_begin);
  int k = 0;
  for (int nb0 = n_begin; nb0 < n_end; nb0 += P.PB, ++k) {
    const int npb = min(P.PB, n_end - nb0);
    if (P.bulk) mb_wait(full, k & 1, abort_flag);
    const int ns = npb * P.f_spp.d;
    for (int it = tid; it < ns; it += BW_NT) {
      const int j = P.f_spp.div(it);
      const int rem = it - j * P.f_spp.d;
      const int by = P.f_sx.div(rem), bx = rem - by * P.f_sx.d;
      if (P.bulk)
        sumdy += bw_stage_block<K, LC, IO, true>(P, slot, j, reinterpret_cast<const IO*>(slot + P.raw_x + j * P.raw_pp),
                                                 reinterpret_cast<const IO*>(slot + P.raw_g + j * P.raw_pp), by, bx);
      else
        sumdy += bw_stage_block<K, LC, IO, false>(P, slot, j, x + ((size_t)(nb0 + j) * P.C + c) * plane,
                                                  dy + ((size_t)(nb0 + j) * P.C + c) * plane, by, bx);
    }
    __syncthreads();
    if (*abort_flag) break;  // uniform: read after the barrier
    if (P.bulk && tid == 0 && nb0 + P.PB < n_end) issue(nb0 + P.PB);
    for (int l = 3; l <= P.L; ++l) {
      const BufDesc& sb = P.sd[l - 1];
      const BufDesc& d = P.sd[l];
      pyramid_level(npb, P.H >> l, P.W >> l, slot + sb.off + r * sb.ld + r, sb.ld, P.ps, slot + d.off + r * d.ld + r,
                    d.ld, d.ld * d.rows, P.ps);
      const BufDesc& gb = P.gd[l - 1];
      const BufDesc& e = P.gd[l];
      pyramid_level(npb, P.H >> l, P.W >> l, slot + gb.off, gb.ld, P.ps, slot + e.off, e.ld, e.ld * e.rows, P.ps);
      __syncthreads();
    }
    if (busy) {
      const int nt = npb * B.f_tiles.d;
      for (int t = lt; t < nt; t += B.nthr) {
        const int j = B.f_tiles.div(t);
        const int tt = t - j * B.f_tiles.d;
        const int ti = B.f_tx.div(tt), tj = tt - ti * B.f_tx.d;
        corr_tile<K, 4, 4>(slot + B.a_off + j * P.ps + (ti << 2) * B.a_ld + (tj << 2), B.a_ld,
                           slot + B.g_off + j * P.ps + (ti << 2) * B.g_ld + (tj << 2), B.g_ld, G);
      }
    }
    __syncthreads();
  }
  if (*abort_flag) {
    if (tid == 0) {
      mb_drain(full, k & 1);  // the copies of unit k were issued; let them land before exit
      if (status) atomicExch(status, 1);
    }
    return;
  }
  // Fixed-order reduction.  An entry of a branch with at most 32 threads is
  // summed by one thread over the branch's threads in index order; an entry
  // of a larger branch (and the sum of dy, over all threads) by one warp,
  // lane l summing threads l, l + 32, ... in order, then a fixed butterfly.
  // The row stride kk4 + 1 (odd) keeps the strided reads free of bank
  // conflicts.
  float* red = slot + P.red_off;
  const int rld = P.kk4 + 1;
#pragma unroll
  for (int t = 0; t < KK; ++t) red[tid * rld + t] = G[t];
  red[BW_NT * rld + tid] = sumdy;
  __syncthreads();
  float* out = part + (size_t)blockIdx.x * P.V;
  for (int e = tid; e < P.V - 1; e += BW_NT) {
    const int bb = e / KK, t = e - bb * KK;
    const BwBranch& Bb = P.br[bb];
    if (Bb.nthr > 32) continue;
    float acc = 0.f;
    for (int th = Bb.first; th < Bb.first + Bb.nthr; ++th) acc += red[th * rld + t];
    out[e] = acc;
  }
  const int warp = tid >> 5, lane = tid & 31;
  for (int bb = 0; bb < P.nbr; ++bb) {
    const BwBranch& Bb = P.br[bb];
    if (Bb.nthr <= 32) continue;  // uniform
    for (int t = warp; t < KK; t += BW_NT / 32) {
      float acc = 0.f;
      for (int th = lane; th < Bb.nthr; th += 32) acc += red[(Bb.first + th) * rld + t];
      acc = warp_sum(acc);
      if (lane == 0) out[bb * KK + t] = acc;
    }
  }
  if (warp == BW_NT / 32 - 1) {
    float acc = 0.f;
    for (int th = lane; th < BW_NT; th += 32) acc += red[BW_NT * rld + th];
    acc = warp_sum(acc);
    if (lane == 0) out[P.V - 1] = acc;
  }
}

}  // namespace wt
