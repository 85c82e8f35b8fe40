// Level-0 data passes on small planes (sm_100a): a warp owns a few planes at a time.
//
// For L = 0 the layer is s0 * (dwconv(x, W0) + b0) (a scaled depthwise conv,
// the base branch of arXiv:2608.10805, abstract).  Planes of at most 32x32
// are too small for the CTA-wide output kernel: its
// units end before the copies of the next ones can overlap, and every phase
// waits on a CTA barrier.  Here a warp takes PW planes at a time with no CTA
// barrier at all: it copies them into its own zero-bordered buffers in
// shared memory, and each lane runs the same 4x4 register tile as the
// CTA-wide kernels on one tile of one plane (a plane has TY x TX tiles; PW =
// 32 / tiles per plane, at most 8, so that the lanes cover the planes;
// planes of 33 to 64 tiles take two tiles per lane).  The border and
// the padding beyond H and W are zeroed once and never written, so partial
// tiles at the edges read zeros.  The first SMALL_PF * 32 elements of the
// warp's next planes (and their parameters) are loaded into registers,
// unconverted, before the current planes' arithmetic, so those loads are in
// flight while it runs.
//
// wtconv_small_kernel: forward (flip = 0) and backward-data (flip = 1, the
// correlation with the flipped kernel and no bias), reading either the raw
// parameters (scaling W0 and b0 by s0 itself) or a folded block.  (The
// weight gradients of such planes stay on the CTA-wide kernel: a
// warp-per-plane version, with x and dy both in flight, was slower.)
#pragma once

#include "wtconv_kernels.cuh"

namespace wt {

constexpr int SMALL_NT = 256;  // threads per CTA (8 warps)
constexpr int SMALL_PF = 16;   // elements per lane of the next planes held in registers

struct SmallPlan {
  int N, C, H, W, K, r;
  int hw;          // H*W
  int TY, TX, T;   // 4x4 tiles per plane: rows, columns, all
  int PW;          // planes per warp at a time
  int ld, rows;    // padded plane buffer: row length (a multiple of 4) and rows
  int xs_pp;       // floats per padded plane buffer
  int w_off;       // per-warp offset of the weights (PW blocks of kk4), then PW biases
  int tab_off;     // per-warp offset of the element table (PW * hw ints)
  int buf;         // floats per warp (a multiple of 4)
  int kk4, wblk;
  FDiv f_w, f_hw, f_C;
};

// Element e of the warp's consecutive planes (plane e / hw) at its place in
// the padded buffers.
__device__ __forceinline__ int small_slot(const SmallPlan& P, int e) {
  const int j = P.f_hw.div(e), i = e - j * P.hw;
  const int yy = P.f_w.div(i), xx = i - yy * P.W;
  return j * P.xs_pp + (yy + P.r) * P.ld + xx + P.r;
}

template <int K, typename IO>
__global__ void __launch_bounds__(SMALL_NT, K >= 5 ? 2 : 3) wtconv_small_kernel(const SmallPlan P,
                                                                                const IO* __restrict__ x,
                                                                                const float* __restrict__ wfold,
                                                                                const float* __restrict__ w0,
                                                                                const float* __restrict__ b0,
                                                                                const float* __restrict__ s0,
                                                                                int flip, IO* __restrict__ y) {
  constexpr int KK = K * K;
  extern __shared__ float4 smem4[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* xs = reinterpret_cast<float*>(smem4) + warp * P.buf;
  float* wsm = xs + P.w_off;
  float* bsm = wsm + P.PW * P.kk4;
  int* tab = reinterpret_cast<int*>(xs + P.tab_off);  // buffer offset of element e of a step
  for (int i = lane; i < P.tab_off; i += 32) xs[i] = 0.f;  // borders and padding stay zero
  const int ne = P.PW * P.hw;
  for (int e = lane; e < ne; e += 32) tab[e] = small_slot(P, e);
  // this lane's tiles (l = lane, lane + 32 of the step's PW * T), fixed for
  // the whole kernel: buffer offset, plane, output offset, rows and columns
  int toff[2], tj[2], tout[2], tny[2], tnx[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int l = lane + 32 * h;
    const int j = l / P.T, t = l - j * P.T, ty = t / P.TX, tx = t - ty * P.TX;
    tj[h] = l < P.PW * P.T ? j : P.PW;  // PW: no tile
    toff[h] = j * P.xs_pp + (4 * ty) * P.ld + 4 * tx;
    tout[h] = j * P.hw + (4 * ty) * P.W + 4 * tx;
    tny[h] = min(4, P.H - 4 * ty);
    tnx[h] = min(4, P.W - 4 * tx);
  }
  const bool vec = (P.W & 3) == 0;
  const int planes = P.N * P.C;
  const int stride = gridDim.x * (SMALL_NT / 32) * P.PW;
  // the next planes' first elements and parameters (taps e = lane, lane + 32
  // of the planes' taps j * KK + i; the bias of plane `lane`), as stored
  IO raw[SMALL_PF];
  float wv[2] = {0.f, 0.f}, wsc[2] = {1.f, 1.f}, bv = 0.f, bsc = 1.f;
  auto fetch = [&](int p0) {
    const int np = min(P.PW, planes - p0), n = np * P.hw;
    const IO* src = x + (size_t)p0 * P.hw;
#pragma unroll
    for (int k = 0; k < SMALL_PF; ++k) {
      const int e = lane + 32 * k;
      if (e < n) raw[k] = src[e];
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int e = lane + 32 * h;
      if (e < np * KK) {
        const int j = e / KK, i = e - j * KK, c = (p0 + j - P.f_C.div(p0 + j) * P.C);
        wv[h] = wfold ? wfold[(size_t)c * P.wblk + i] : w0[(size_t)c * KK + (flip ? KK - 1 - i : i)];
        wsc[h] = wfold ? 1.f : s0[c];
      }
    }
    if (lane < np) {
      const int c = (p0 + lane - P.f_C.div(p0 + lane) * P.C);
      bv = wfold ? wfold[(size_t)c * P.wblk + P.kk4] : (flip ? 0.f : b0[c]);
      bsc = wfold ? 1.f : s0[c];
    }
  };
  int p0 = (blockIdx.x * (SMALL_NT / 32) + warp) * P.PW;
  if (p0 < planes) fetch(p0);
  __syncwarp();  // the table is written
  for (; p0 < planes; p0 += stride) {
    const int np = min(P.PW, planes - p0), n = np * P.hw;
    const IO* src = x + (size_t)p0 * P.hw;
    __syncwarp();  // the previous planes' reads of the buffers are done
#pragma unroll
    for (int k = 0; k < SMALL_PF; ++k) {
      const int e = lane + 32 * k;
      if (e < n) xs[tab[e]] = io_traits<IO>::to_f(raw[k]);
    }
    for (int e = lane + 32 * SMALL_PF; e < n; e += 32) xs[tab[e]] = io_traits<IO>::to_f(src[e]);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int e = lane + 32 * h;
      if (e < np * KK) wsm[(e / KK) * P.kk4 + e % KK] = wsc[h] * wv[h];
    }
    for (int e = lane + 64; e < np * KK; e += 32) {  // planes of few tiles: more taps than two per lane
      const int j = e / KK, i = e - j * KK, c = (p0 + j - P.f_C.div(p0 + j) * P.C);
      wsm[j * P.kk4 + i] =
          wfold ? wfold[(size_t)c * P.wblk + i] : s0[c] * w0[(size_t)c * KK + (flip ? KK - 1 - i : i)];
    }
    if (lane < np) bsm[lane] = bsc * bv;
    if (p0 + stride < planes) fetch(p0 + stride);  // in flight during these planes' arithmetic
    __syncwarp();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (tj[h] < np) {
        float acc[4][4];
        const float bias = bsm[tj[h]];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) acc[a][b] = bias;
        conv_tile<K, 4, 4>(xs + toff[h], P.ld, wsm + tj[h] * P.kk4, acc);
        IO* dst = y + (size_t)p0 * P.hw + tout[h];
#pragma unroll
        for (int a = 0; a < 4; ++a)
          if (a < tny[h]) store4(dst + a * P.W, acc[a], tnx[h], vec);
      }
    }
  }
}

}  // namespace wt
