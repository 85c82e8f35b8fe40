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
template <int K, int LC, typename IO, bool SMEM, bool DYS = false>
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
  // with DYS, dy's buffers are shifted like x's (zero border of r)
  constexpr int rg = DYS ? r : 0;
  float sum = 0.f;
  float* xf = slot + P.xf.off + j * P.ps + (y0 + r) * P.xf.ld + x0 + r;
  float* gf = slot + P.gf.off + j * P.ps + (y0 + rg) * P.gf.ld + x0 + rg;
#pragma unroll
  for (int i = 0; i < BH; ++i) {
    sum += (q[i].x + q[i].y) + (q[i].z + q[i].w);
    if (full) {
      sts4<r>(xf + i * P.xf.ld, v[i]);
      sts4<rg>(gf + i * P.gf.ld, q[i]);
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
    float* g1 = slot + P.g1.off + j * P.ps + ((y0 >> 1) + rg) * lg1 + (x0 >> 1) + rg;
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
        sts2<rg>(g1 + a * lg1, m0, m1);
        sts2<rg>(g1 + bg1 + a * lg1, n0, n1);
        sts2<rg>(g1 + 2 * bg1 + a * lg1, o0, o1);
        sts2<rg>(g1 + 3 * bg1 + a * lg1, p0, p1);
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
      float* g2 = slot + e.off + j * P.ps + (by + rg) * e.ld + bx + rg;
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

// ------------------------------------------------------------------------
// Fused backward (whole planes): backward-data and the weight, scale and
// bias gradients from one staging of x and dy per unit.
//
// The adjoint of the layer's map in x runs the forward cascade on dy with
// flipped kernels and no bias, and its analysis of dy is the same Haar
// pyramid dZ_l the weight gradients correlate against (the synthesis is the
// transpose of the analysis); so a CTA stages x and dy once (both pyramids,
// dy's with the zero border the conv tiles read), then per unit:
//   I   every correlation branch, as in the weight-gradient kernel;
//   II  the adjoint's level convs of levels >= 2 on dy's pyramid;
//   III its level-1 band convs (with the closed-form t1 on the LL band);
//   IV  the level-1 synthesis and the base conv on dy, and dx is stored.
// Phases II-IV write their Z planes over x's buffers, which phase I was the
// last to read.  The channel's adjoint folded weights stay in shared memory
// for the whole CTA.  Reduction of the correlations as in the weight-gradient
// kernel.
template <int K, int LC, typename IO>
__global__ void __launch_bounds__(BW_NT, 2) wtconv_bwd_fused_kernel(const __grid_constant__ BwdPlan Q,
                                                                    const IO* __restrict__ x,
                                                                    const IO* __restrict__ dy,
                                                                    const float* __restrict__ wfold,
                                                                    IO* __restrict__ dx, float* __restrict__ part,
                                                                    int* __restrict__ status) {
  const BwPlan& P = Q.B;
  const MainPlan& M = Q.M;
  constexpr int KK = K * K;
  constexpr int r = K / 2;
  constexpr int GV = (r % 4 == 0) ? 4 : ((r % 2 == 0) ? 2 : 1);  // alignment of dy's shifted rows
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
  // the channel's adjoint weights, for every unit of the CTA (visible after
  // the first barrier of the unit loop)
  for (int i = tid; i < (M.wblk >> 2); i += BW_NT)
    reinterpret_cast<float4*>(slot + M.w_off)[i] = __ldg(reinterpret_cast<const float4*>(wfold + (size_t)c * M.wblk) + i);
  int b = 0;
  while (b + 1 < P.nbr && tid >= P.br[b + 1].first) ++b;
  const BwBranch B = P.br[b];
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
        sumdy += bw_stage_block<K, LC, IO, true, true>(P, slot, j,
                                                       reinterpret_cast<const IO*>(slot + P.raw_x + j * P.raw_pp),
                                                       reinterpret_cast<const IO*>(slot + P.raw_g + j * P.raw_pp),
                                                       by, bx);
      else
        sumdy += bw_stage_block<K, LC, IO, false, true>(P, slot, j, x + ((size_t)(nb0 + j) * P.C + c) * plane,
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
      pyramid_level(npb, P.H >> l, P.W >> l, slot + gb.off + r * gb.ld + r, gb.ld, P.ps, slot + e.off + r * e.ld + r,
                    e.ld, e.ld * e.rows, P.ps);
      __syncthreads();
    }
    // I: correlations (dy's operand read inside its zero border)
    if (busy) {
      const int nt = npb * B.f_tiles.d;
      for (int t = lt; t < nt; t += B.nthr) {
        const int j = B.f_tiles.div(t);
        const int tt = t - j * B.f_tiles.d;
        const int ti = B.f_tx.div(tt), tj = tt - ti * B.f_tx.d;
        corr_tile<K, 4, 4, 0, false, GV>(slot + B.a_off + j * P.ps + (ti << 2) * B.a_ld + (tj << 2), B.a_ld,
                                         slot + B.g_off + j * P.ps + (ti << 2) * B.g_ld + (tj << 2), B.g_ld, G);
      }
    }
    __syncthreads();
    // II: the adjoint's band convs of levels >= 2
    if constexpr (LC == 2) {
      for (int it = tid; it < npb * M.f_dper.d; it += BW_NT) main_deep_tile<K>(M, slot, it);
      __syncthreads();
    }
    // III: its level-1 band convs
    if constexpr (LC >= 1) {
      for (int it = tid; it < npb * M.a_pp; it += BW_NT) main_band_tile<K, LC == 2>(M, slot, it);
      __syncthreads();
    }
    // IV: synthesis, base conv, dx
    {
      UnitGeo g;
      g.c = c;
      g.nb0 = nb0;
      g.npb = npb;
      g.y0 = 0;
      g.y_lo = 0;
      g.y_hi = P.H;
      for (int it = tid; it < npb * M.tiles_pp; it += BW_NT) {
        const int j = M.f_tpp.div(it);
        main_out_tile<K, 4, IO, false>(M, slot, g, j, it - j * M.tiles_pp, 0, dx);
      }
    }
    __syncthreads();
    if (nb0 + P.PB < n_end && LC >= 1) {
      // the Z planes lie over x's buffers: back to zeros before the next
      // unit's staging, which writes only the interiors
      const int na = Q.za_len >> 2, nz = Q.zb_len >> 2;
      for (int i = tid; i < npb * (na + nz); i += BW_NT) {
        const int j = i / (na + nz), e = i - j * (na + nz);
        float* p = slot + j * P.ps + (e < na ? Q.za_off + 4 * e : Q.zb_off + 4 * (e - na));
        *reinterpret_cast<float4*>(p) = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      __syncthreads();
    }
  }
  if (*abort_flag) {
    if (tid == 0) {
      mb_drain(full, k & 1);  // the copies of unit k were issued; let them land before exit
      if (status) atomicExch(status, 1);
    }
    return;
  }
  // fixed-order reduction, as in the weight-gradient kernel
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

// ------------------------------------------------------------------------
// Level-0 fp32 weight gradients fed by tensor copies (no staging pass).
//
// Each unit's x planes arrive zero-padded by one tensor copy (TMA; the box
// of PB planes x (rup(H, 4) + 2r) rows x (W + 8) columns at column -4, row
// -r of the map over x as [N][C][H][W]; everything outside the plane reads
// as zero) and its dy planes by one bulk copy each, into one of two buffer
// sets: the copies of unit k + 2 are issued as soon as unit k's buffers are
// free, so one unit is always in flight while the CTA correlates another.
// All threads run the base correlation G_0 = sum dy(i,j) x(i+u-r, j+v-r) on
// 4x4 tiles and sum dy on the side; the reduction is the fixed-order one of
// the whole-plane kernel (one branch of BW_NT threads).
template <int K>
__global__ void __launch_bounds__(BW_NT, 1) wtconv_bwdw_direct_kernel(const __grid_constant__ BwDirectPlan P,
                                                                      const float* __restrict__ dy,
                                                                      float* __restrict__ part,
                                                                      int* __restrict__ status,
                                                                      const __grid_constant__ CUtensorMap xmap) {
  constexpr int KK = K * K;
  constexpr int r = K / 2;
  extern __shared__ __align__(128) float4 smem4[];
  float* sm = reinterpret_cast<float*>(smem4);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm);  // one mbarrier per buffer set
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + 4);
  const int tid = threadIdx.x;
  for (int i = tid; i < (P.smem_floats >> 2); i += BW_NT) smem4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  __syncthreads();
  if (tid == 0) {
    mb_init(full, 1);
    mb_init(full + 1, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const int c = blockIdx.x % P.C, grp = blockIdx.x / P.C;
  const int n_begin = grp * P.ppc, n_end = min(P.N, n_begin + P.ppc);
  // units: PB planes at a time (nb == 1), or one row band of one plane
  const int nunits = n_end <= n_begin ? 0 : P.nb == 1 ? (n_end - n_begin + P.PB - 1) / P.PB : (n_end - n_begin) * P.nb;
  const unsigned gbytes = (unsigned)((size_t)(P.nb == 1 ? P.H : P.TB) * P.W * 4);
  auto issue = [&](int u) {
    const int b = u & 1;
    int nb0, cnt, y0;
    if (P.nb == 1) {
      nb0 = n_begin + u * P.PB;
      cnt = min(P.PB, n_end - nb0);
      y0 = 0;
    } else {
      const int pl = u / P.nb;
      nb0 = n_begin + pl;
      cnt = 1;
      y0 = (u - pl * P.nb) * P.TB;
    }
    const unsigned xbytes = (unsigned)(P.xps * P.PB * 4);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(full + b)),
                 "r"(xbytes + gbytes * (unsigned)cnt)
                 : "memory");
    tma_load_4d(sm + P.xoff[b], &xmap, -4, y0 - r, c, nb0, full + b);
    for (int jj = 0; jj < cnt; ++jj)
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
              smem_u32(sm + P.goff[b] + jj * P.gps)),
          "l"(dy + (((size_t)(nb0 + jj) * P.C + c) * P.H + y0) * P.W), "r"(gbytes), "r"(smem_u32(full + b))
          : "memory");
  };
  if (tid == 0) {
    if (nunits > 0) issue(0);
    if (nunits > 1) issue(1);
  }
  float G[KK];
  zero_taps<K>(G);
  float sumdy = 0.f;
  int k = 0;
  for (; k < nunits; ++k) {
    const int b = k & 1;
    mb_wait(full + b, (k >> 1) & 1, abort_flag);
    __syncthreads();
    if (*abort_flag) break;  // uniform: read after the barrier
    const int npb = P.nb == 1 ? min(P.PB, n_end - (n_begin + k * P.PB)) : 1;
    const float* xs = sm + P.xoff[b];
    const float* gs = sm + P.goff[b];
    for (int t = tid; t < npb * P.tiles_pp; t += BW_NT) {
      const int j = P.f_tiles.div(t);
      const int tt = t - j * P.tiles_pp;
      const int ti = P.f_tx.div(tt), tj = tt - ti * P.f_tx.d;
      // x window from (4 ti - r, 4 tj - r): column 4 tj + 4 - r of the buffer
      corr_tile<K, 4, 4, 4 - r, true>(xs + j * P.xps + (ti << 2) * P.xld + (tj << 2), P.xld,
                                      gs + j * P.gps + (ti << 2) * P.gld + (tj << 2), P.gld, G, &sumdy);
    }
    __syncthreads();
    if (tid == 0 && k + 2 < nunits) issue(k + 2);
  }
  if (*abort_flag) {
    if (tid == 0) {
      // let the copies still in flight (units k and k + 1) land before exit
      mb_drain(full + (k & 1), (k >> 1) & 1);
      if (k + 1 < nunits) mb_drain(full + ((k + 1) & 1), ((k + 1) >> 1) & 1);
      if (status) atomicExch(status, 1);
    }
    return;
  }
  // fixed-order reduction over the BW_NT threads (no copy is in flight now,
  // so the buffers can hold it): lane l sums threads l, l + 32, ... in
  // order, then a fixed butterfly
  float* red = sm + P.red_off;
  const int rld = P.kk4 + 1;
#pragma unroll
  for (int t = 0; t < KK; ++t) red[tid * rld + t] = G[t];
  red[BW_NT * rld + tid] = sumdy;
  __syncthreads();
  float* out = part + (size_t)blockIdx.x * P.V;
  const int warp = tid >> 5, lane = tid & 31;
  for (int t = warp; t <= KK; t += BW_NT / 32) {
    float acc = 0.f;
    if (t < KK)
      for (int th = lane; th < BW_NT; th += 32) acc += red[th * rld + t];
    else
      for (int th = lane; th < BW_NT; th += 32) acc += red[BW_NT * rld + th];
    acc = warp_sum(acc);
    if (lane == 0) out[t] = acc;
  }
}

}  // namespace wt
