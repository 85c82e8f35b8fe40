// Output kernel and deep-level kernel (sm_100a).
//
// Output kernel (forward and backward-data): a CTA of four warps works
// through its units (a band of one plane, or a batch of small planes of one
// channel) in phases.  Thread 0 keeps the next unit's input rows, t1 rows
// and folded weights in flight with TMA 1-D bulk copies (cp.async.bulk,
// completing on one mbarrier) while the CTA computes the current unit; the
// CTA turns the raw rows into zero-padded fp32 rows and the level-1 Haar
// subbands (reformulation (1) of arXiv:2608.10805, abstract), then runs
// register tiles in two phases: (A) each thread convolves one level-1 band
// over a 4x4 tile with folded weights (reformulation (3)), adds t1 to the LL
// band and writes the band's Z plane to shared memory; (B) each thread takes
// an R3 x 4 output tile, adds the synthesis of the four Z planes, runs the
// base conv and stores y.  Tiles four floats wide let the lanes of a warp
// read consecutive 16-byte words of a row, nearly free of bank conflicts.
// Small CTAs (about 64 KB of shared memory on 56x56 planes) let three run
// per SM, so one CTA's staging and barriers overlap the others' arithmetic.
//
// Deep kernel: levels 2..L of a batch of planes on chip (pyramid, every level
// conv, then the closed-form synthesis of all levels >= 2 at level-1
// resolution indexed by coordinate bits -- reformulation (2) -- summed level
// by level from the deepest), written as t1.
#pragma once

#include "wtconv_kernels.cuh"

namespace wt {

constexpr int MAIN_NT = 128;
constexpr int MAIN_HEADER = 4;       // floats: mbarrier (8 bytes), abort flag
constexpr int DEEP_NT = 512;

// ------------------------------------------------------------ mbarriers
__device__ __forceinline__ unsigned smem_u32(const void* p) { return (unsigned)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void mb_init(uint64_t* b, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count) : "memory");
}
__device__ __forceinline__ bool mb_try(uint64_t* b, unsigned parity) {
  unsigned done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(done)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return done != 0;
}
// Waits for the phase with the given parity.  Gives up (returns false) when
// another thread has raised the abort flag, or after an iteration limit, in
// which case it raises the flag itself.
__device__ __forceinline__ bool mb_wait(uint64_t* b, unsigned parity, volatile int* abort_flag) {
  for (int i = 0; i < (1 << 22); ++i) {
    if (mb_try(b, parity)) return true;
    if (*abort_flag) return false;
  }
  *abort_flag = 1;
  return false;
}
// Bounded wait that ignores the abort flag: used before exit so that bulk
// copies already issued land before the CTA's shared memory is released.
__device__ __forceinline__ void mb_drain(uint64_t* b, unsigned parity) {
  for (int i = 0; i < (1 << 22); ++i)
    if (mb_try(b, parity)) return;
}
// Starts moving [p, p + bytes) into L2; no completion to wait for.  Issued
// only for 16-byte aligned ranges whose size is a multiple of 16 bytes.
__device__ __forceinline__ void l2_prefetch(const void* p, unsigned bytes) {
  if (((reinterpret_cast<uintptr_t>(p) | bytes) & 15) == 0)
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
// ------------------------------------------------------------ unit geometry
// A unit is one band of one plane (nbands > 1) or a batch of npb planes of
// one channel (nbands == 1, consecutive batch entries).
struct UnitGeo {
  int c, nb0, npb, y0, y_lo, y_hi;  // channel, first batch entry, planes, first output row, staged x rows
};
__device__ __forceinline__ UnitGeo unit_geo(const MainPlan& P, int u) {
  UnitGeo g;
  const int pg = P.f_bands.div(u);
  const int b = u - pg * P.nbands;
  const int bt = P.f_C.div(pg);
  g.c = pg - bt * P.C;
  g.nb0 = bt * P.PB;
  g.npb = min(P.PB, P.N - g.nb0);
  g.y0 = b * P.TH;
  const int hx = P.L >= 1 ? 2 * P.r : P.r;
  g.y_lo = max(0, g.y0 - hx);
  g.y_hi = min(P.H, g.y0 + P.TH + hx);
  return g;
}
__device__ __forceinline__ size_t plane_index(const MainPlan& P, const UnitGeo& g, int j) {
  return (size_t)(g.nb0 + j) * P.C + g.c;
}

// Folded weights of every channel (one block of wblk floats per channel):
//   [0, kk4): s0 * W0   [kk4]: s0 * b0 (0 for the adjoint)
//   [kk4+4 + ((l-1)*4 + s)*kk4, ...): 2^-l * s_l[s] * W_l[s], l = 1..L
// (2^-l: the synthesis factors of the l inverse transforms between level l
// and the image); every kernel flipped for the adjoint.
template <int K>
__global__ void wtconv_fold_kernel(int C, int L, int kk4, int wblk, const float* __restrict__ w0,
                                   const float* __restrict__ b0, const float* __restrict__ s0,
                                   const float* __restrict__ wl, const float* __restrict__ sl, int flip,
                                   float* __restrict__ out) {
  constexpr int KK = K * K;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < C * wblk; i += gridDim.x * blockDim.x) {
    const int c = i / wblk, e = i - c * wblk;
    float v = 0.f;
    if (e < KK) {
      v = s0[c] * w0[(size_t)c * KK + (flip ? KK - 1 - e : e)];
    } else if (e == kk4) {
      v = flip ? 0.f : s0[c] * b0[c];
    } else if (e >= kk4 + 4 && e < kk4 + 4 + 4 * L * kk4) {
      const int blk = (e - kk4 - 4) / kk4, t = (e - kk4 - 4) - blk * kk4;
      if (t < KK) {
        const int l = (blk >> 2) + 1, s = blk & 3;
        const size_t base = ((size_t)(l - 1) * C + c) * 4 + s;
        v = (sl[base] * wl[base * KK + (flip ? KK - 1 - t : t)]) * pow2neg(l);
      }
    }
    out[i] = v;
  }
}

// Staging of one plane of a unit (paths other than the fused-deep one):
// padded fp32 rows xf (band rows [-r, TH+r)) and level-1 subbands s1 (half
// rows [-r, TH/2+r)), zero outside the plane.  SMEM: rows come from the raw
// copy (row y at src + (y - y_lo) * W).
template <int K, typename IO, bool SMEM>
__device__ __forceinline__ void main_stage_item(const MainPlan& P, float* xf, float* s1, const IO* __restrict__ src,
                                                const UnitGeo& g, int ri, int x0) {
  constexpr int r = K / 2;
  const bool vec = P.vec_in != 0;
  const int ldx = P.xf.ld;
  auto row_ptr = [&](int y) -> const IO* {
    return SMEM ? src + (size_t)(y - g.y_lo) * P.W : src + (size_t)y * P.W;
  };
  if (P.L >= 1) {
    const int ld1 = P.s1.ld, bs1 = P.s1.ld * P.s1.rows;
    const int irel = P.st_row0 + ri;  // half row relative to the band
    const int i = (g.y0 >> 1) + irel;  // absolute half row
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (i >= 0 && i < P.H1) {
      a = src4<SMEM>(row_ptr(2 * i) + x0, x0, P.W, vec);
      b = src4<SMEM>(row_ptr(2 * i + 1) + x0, x0, P.W, vec);
    }
    const int yrel = 2 * irel;
    float* d0 = xf + (yrel + r) * ldx + x0 + r;
    float* q1 = s1 + (irel + r) * ld1 + (x0 >> 1) + r;
    float l0, h0, g0, k0, l1, h1, g1, k1;
    haar4(a.x, a.y, b.x, b.y, l0, h0, g0, k0);
    haar4(a.z, a.w, b.z, b.w, l1, h1, g1, k1);
    const bool r0 = yrel >= -r && yrel < P.TH + r, r1 = yrel + 1 >= -r && yrel + 1 < P.TH + r;
    if (x0 + 3 < P.W) {
      if (r0) sts4<r>(d0, a);
      if (r1) sts4<r>(d0 + ldx, b);
      sts2<r>(q1, l0, l1);
      sts2<r>(q1 + bs1, h0, h1);
      sts2<r>(q1 + 2 * bs1, g0, g1);
      sts2<r>(q1 + 3 * bs1, k0, k1);
    } else {  // W % 4 == 2: one 2-wide block left in the row
      if (r0) {
        d0[0] = a.x;
        d0[1] = a.y;
      }
      if (r1) {
        d0[ldx] = b.x;
        d0[ldx + 1] = b.y;
      }
      q1[0] = l0;
      q1[bs1] = h0;
      q1[2 * bs1] = g0;
      q1[3 * bs1] = k0;
    }
  } else {
    const int yrel = P.st_row0 + ri;
    const int y = g.y0 + yrel;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    if (y >= 0 && y < P.H) a = src4<SMEM>(row_ptr(y) + x0, x0, P.W, vec);
    float* d0 = xf + (yrel + r) * ldx + x0 + r;
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

// Staging for whole planes with L >= 2, one 4x4 block of plane j per item:
// the padded fp32 rows xf, the level-1 subbands s1 (2x2 per band) and the
// level-2 subbands sd[2] (one per band), the butterflies in registers.
template <int K, typename IO, bool SMEM>
__device__ __forceinline__ void main_stage_block(const MainPlan& P, float* slot, int j, const IO* __restrict__ src,
                                                 int by, int bx) {
  constexpr int r = K / 2;
  const int x0 = bx << 2, y0 = by << 2;
  float4 v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = src4<SMEM>(src + (size_t)(y0 + i) * P.W + x0, x0, P.W, true);
  float* xf = slot + P.xf.off + j * P.xf.ps + (y0 + r) * P.xf.ld + x0 + r;
#pragma unroll
  for (int i = 0; i < 4; ++i) sts4<r>(xf + i * P.xf.ld, v[i]);
  const int ld1 = P.s1.ld, bs1 = P.s1.ld * P.s1.rows;
  float* s1 = slot + P.s1.off + j * P.s1.ps + (2 * by + r) * ld1 + 2 * bx + r;
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
  const BufDesc& d = P.sd[2];
  const int bs = d.ld * d.rows;
  float* s2 = slot + d.off + j * d.ps + (by + r) * d.ld + bx + r;
  float L2, H2, G2, K2;
  haar4(ll[0][0], ll[0][1], ll[1][0], ll[1][1], L2, H2, G2, K2);
  s2[0] = L2;
  s2[bs] = H2;
  s2[2 * bs] = G2;
  s2[3 * bs] = K2;
}

// One 4x4 tile of a deep level's band conv (levels 2..L of whole planes):
// Zd_l^s = conv(sd_l^s, 2^-l s_l W_l^s), stored plain.
template <int K>
__device__ __forceinline__ void main_deep_tile(const MainPlan& P, float* slot, int it) {
  const int j = P.f_dper.div(it);
  int rem = it - j * P.f_dper.d;
  int l = 2;
  while (l < P.L && rem >= P.dfirst[l + 1]) ++l;
  rem -= P.dfirst[l];
  const int s = P.f_dtiles[l].div(rem);
  rem -= s * P.f_dtiles[l].d;
  const int ti = P.f_dtx[l].div(rem);
  const int i0 = ti * 4, j0 = (rem - ti * P.f_dtx[l].d) * 4;
  const BufDesc& d = P.sd[l];
  const BufDesc& z = P.zd[l];
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
  conv_tile<K, 4, 4>(slot + d.off + j * d.ps + s * d.ld * d.rows + i0 * d.ld + j0, d.ld,
                     slot + P.w_off + P.kk4 + 4 + ((l - 1) * 4 + s) * P.kk4, acc);
  float* o = slot + z.off + j * z.ps + s * z.ld * z.rows + i0 * z.ld + j0;
#pragma unroll
  for (int a = 0; a < 4; ++a)
    *reinterpret_cast<float4*>(o + a * z.ld) = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
}

// t1 of a 4x4 tile of the level-1 grid at (i0, j0), i0 and j0 multiples of 4:
//   t1(i,j) = sum_{l>=2} sum_s sigma_s(bit_{l-2}(i), bit_{l-2}(j)) Zd_l^s(i >> (l-1), j >> (l-1))
// (reformulation (2) of arXiv:2608.10805, abstract: every level's share of
// a position is indexed by the bits of its coordinates).  Added to z.
__device__ __forceinline__ void main_add_t1(const MainPlan& P, const float* slot, int j, int i0, int j0,
                                            float (&z)[4][4]) {
  {
    const BufDesc& zd = P.zd[2];
    const int bz = zd.ld * zd.rows;
    const float* q = slot + zd.off + j * zd.ps + (i0 >> 1) * zd.ld + (j0 >> 1);
#pragma unroll
    for (int a2 = 0; a2 < 2; ++a2) {
      const float2 zl = *reinterpret_cast<const float2*>(q + a2 * zd.ld);
      const float2 zh = *reinterpret_cast<const float2*>(q + a2 * zd.ld + bz);
      const float2 zg = *reinterpret_cast<const float2*>(q + a2 * zd.ld + 2 * bz);
      const float2 zk = *reinterpret_cast<const float2*>(q + a2 * zd.ld + 3 * bz);
      float o00, o01, o10, o11;
      synth4(zl.x, zh.x, zg.x, zk.x, o00, o01, o10, o11);
      z[2 * a2][0] += o00;
      z[2 * a2][1] += o01;
      z[2 * a2 + 1][0] += o10;
      z[2 * a2 + 1][1] += o11;
      synth4(zl.y, zh.y, zg.y, zk.y, o00, o01, o10, o11);
      z[2 * a2][2] += o00;
      z[2 * a2][3] += o01;
      z[2 * a2 + 1][2] += o10;
      z[2 * a2 + 1][3] += o11;
    }
  }
  for (int l = 3; l <= P.L; ++l) {
    // i >> (l-1) and j >> (l-1) are the same for the whole tile
    const BufDesc& zd = P.zd[l];
    const int bz = zd.ld * zd.rows;
    const float* q = slot + zd.off + j * zd.ps + (i0 >> (l - 1)) * zd.ld + (j0 >> (l - 1));
    const float zl = q[0], zh = q[bz], zg = q[2 * bz], zk = q[3 * bz];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const float sy = (((i0 + a) >> (l - 2)) & 1) ? -1.f : 1.f;
      const float A = fmaf(sy, zh, zl), B = fmaf(sy, zk, zg);
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const float sx = (((j0 + b) >> (l - 2)) & 1) ? -1.f : 1.f;
        z[a][b] += fmaf(sx, B, A);
      }
    }
  }
}

// Phase A, one tile: band s of plane j, a 4x4 tile of the level-1 grid:
// the band conv with folded weights (reformulation (3) of arXiv:2608.10805,
// abstract), t1 added to the LL band, stored to the band's Z plane.
template <int K, bool FUSED>
__device__ __forceinline__ void main_band_tile(const MainPlan& P, float* slot, int it) {
  const int j = P.f_app.div(it);
  int rem = it - j * P.a_pp;
  const int s = P.f_abt.div(rem);
  rem -= s * P.f_abt.d;
  const int ti = P.f_atx.div(rem);
  const int i0 = ti * 4, j0 = (rem - ti * P.f_atx.d) * 4;
  float z[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) z[a][b] = 0.f;
  const float* s1 = slot + P.s1.off + j * P.s1.ps + s * P.s1.ld * P.s1.rows + i0 * P.s1.ld + j0;
  conv_tile<K, 4, 4>(s1, P.s1.ld, slot + P.w_off + P.kk4 + 4 + s * P.kk4, z);
  if constexpr (FUSED) {
    if (s == 0) main_add_t1(P, slot, j, i0, j0, z);
  } else if (s == 0 && P.L >= 2) {
    const float* t1 = slot + P.t1.off + j * P.t1.ps + i0 * P.t1.ld + j0;
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const float4 tv = *reinterpret_cast<const float4*>(t1 + a * P.t1.ld);
      z[a][0] += tv.x;
      z[a][1] += tv.y;
      z[a][2] += tv.z;
      z[a][3] += tv.w;
    }
  }
  float* zp = slot + P.zb.off + j * P.zb.ps + s * P.zb.ld * P.zb.rows + i0 * P.zb.ld + j0;
#pragma unroll
  for (int a = 0; a < 4; ++a)
    *reinterpret_cast<float4*>(zp + a * P.zb.ld) = make_float4(z[a][0], z[a][1], z[a][2], z[a][3]);
}

// Phase B, one tile: R3 x 4 outputs of plane j: bias, the level-1 synthesis
// of the four Z planes (signs sigma_s(py, px); the 1/2 is in the weights),
// the base conv, and the store.
template <int K, int R3, typename IO, bool DIRECT>
__device__ __forceinline__ void main_out_tile(const MainPlan& P, const float* slot, const UnitGeo& g, int j, int tile,
                                              int buf, IO* __restrict__ y) {
  const int ti = P.f_tx.div(tile);
  const int yy0 = ti * R3, xx0 = (tile - ti * P.f_tx.d) * 4;
  const float* sw = slot + P.w_off;
  const float bias = sw[P.kk4];
  float acc[R3][4];
#pragma unroll
  for (int a = 0; a < R3; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = bias;
  if (P.L >= 1) {
    const int bz = P.zb.ld * P.zb.rows;
    const float* zb = slot + P.zb.off + j * P.zb.ps + (yy0 >> 1) * P.zb.ld + (xx0 >> 1);
#pragma unroll
    for (int a = 0; a < R3 / 2; ++a) {
      float2 zs[4];
#pragma unroll
      for (int s = 0; s < 4; ++s) zs[s] = *reinterpret_cast<const float2*>(zb + s * bz + a * P.zb.ld);
      float o00, o01, o10, o11;
      synth4(zs[0].x, zs[1].x, zs[2].x, zs[3].x, o00, o01, o10, o11);
      acc[2 * a][0] += o00;
      acc[2 * a][1] += o01;
      acc[2 * a + 1][0] += o10;
      acc[2 * a + 1][1] += o11;
      synth4(zs[0].y, zs[1].y, zs[2].y, zs[3].y, o00, o01, o10, o11);
      acc[2 * a][2] += o00;
      acc[2 * a][3] += o01;
      acc[2 * a + 1][2] += o10;
      acc[2 * a + 1][3] += o11;
    }
  }
  if constexpr (DIRECT) {
    // rows copied straight into the buffer: column x at x + 4, so the aligned
    // window starts 4 - r columns before the tile's first tap
    conv_tile<K, R3, 4, 4 - K / 2>(slot + P.xf.off + buf * P.xbuf + j * P.xf.ps + yy0 * P.xf.ld + xx0, P.xf.ld, sw,
                                   acc);
  } else {
    conv_tile<K, R3, 4>(slot + P.xf.off + j * P.xf.ps + yy0 * P.xf.ld + xx0, P.xf.ld, sw, acc);
  }
  // y holds oH x oW planes: the image, or its top-left corner when the
  // planes were zero-padded to multiples of 2^L
  const int n = P.oW - xx0 < 4 ? P.oW - xx0 : 4;
  if (n <= 0) return;
  IO* yp = y + plane_index(P, g, j) * P.oH * P.oW;
#pragma unroll
  for (int a = 0; a < R3; ++a) {
    const int yr = g.y0 + yy0 + a;
    if (yy0 + a < P.TH && yr < P.oH) store4(yp + (size_t)yr * P.oW + xx0, acc[a], n, P.vec_out != 0);
  }
}

// One unit's bulk copies into the raw region of the slot: the channel's
// folded weights, the unit's input rows (bulk_x) and t1 rows (bulk_t), all
// completing on one mbarrier phase.
template <typename IO>
__device__ __forceinline__ void main_issue(const MainPlan& P, float* slot, uint64_t* full, const UnitGeo& g,
                                           const IO* __restrict__ x, const float* __restrict__ t1g,
                                           const float* __restrict__ wfold) {
  const unsigned bx = P.bulk_x ? (unsigned)((g.y_hi - g.y_lo) * P.W * P.io_bytes) : 0u;
  const unsigned bt = (P.L >= 2 && P.bulk_t) ? (unsigned)((P.TH >> 1) * P.W1 * 4) : 0u;
  const unsigned bw = (unsigned)(P.wblk * 4);
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(full)),
               "r"(bw + (bx + bt) * g.npb)
               : "memory");
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(slot + P.wraw_off)),
      "l"(wfold + (size_t)g.c * P.wblk), "r"(bw), "r"(smem_u32(full))
      : "memory");
  for (int j = 0; j < g.npb; ++j) {
    const size_t pi = plane_index(P, g, j);
    if (bx) {
      const IO* src = x + pi * P.H * P.W + (size_t)g.y_lo * P.W;
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
              smem_u32(slot + P.raw_off + j * P.raw_pp)),
          "l"(src), "r"(bx), "r"(smem_u32(full))
          : "memory");
    }
    if (bt) {
      const float* src = t1g + pi * P.H1 * P.W1 + (size_t)(g.y0 >> 1) * P.W1;
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
              smem_u32(slot + P.rawt_off + j * P.rawt_pp)),
          "l"(src), "r"(bt), "r"(smem_u32(full))
          : "memory");
    }
  }
}

// One tile-mode tensor copy (TMA) of the box at element coordinates
// (x, y, c, n) of a 4-D tensor map into shared memory at dst (128-byte
// aligned), completing on mbarrier `bar`.  Elements of the box outside the
// tensor arrive as zeros.
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int x, int y, int c, int n,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
      "[%6];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(c), "r"(n), "r"(smem_u32(bar))
      : "memory");
}

// Level-0 fp32 planes: one unit's input rows straight into row buffer `buf`
// by one tensor copy of the map over x viewed as [N][C][H][W]: the box of
// PB planes x (rup(TH, R3) + 2r) rows x (W + 8) columns at (column -4, row
// y0 - r, channel c, batch entry nb0), so that row y of plane j lands at
// (y - y0 + r) * ld + x + 4 and the rows and columns outside the plane
// (the zero padding) arrive as zeros; no staging pass.  The folded weights
// come by a bulk copy as for the other paths, unless the kernel scales the
// raw ones itself (wfold null).  Thread 0 issues.
__device__ __forceinline__ void main_issue_tensor(const MainPlan& P, float* slot, uint64_t* full, const UnitGeo& g,
                                                  int buf, const CUtensorMap* xmap,
                                                  const float* __restrict__ wfold) {
  const unsigned bw = wfold ? (unsigned)(P.wblk * 4) : 0u;
  const unsigned bx = (unsigned)(P.xf.ld * P.xf.rows * P.PB * 4);
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(full)), "r"(bw + bx)
               : "memory");
  if (wfold)
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(slot + P.wraw_off)),
        "l"(wfold + (size_t)g.c * P.wblk), "r"(bw), "r"(smem_u32(full))
        : "memory");
  tma_load_4d(slot + P.xf.off + buf * P.xbuf, xmap, -4, g.y0 - P.r, g.c, g.nb0, full);
}

template <int K, int R3, typename IO, bool FUSED, bool DIRECT>
__global__ void __launch_bounds__(MAIN_NT, 4)
    wtconv_main_kernel(const MainPlan P, const IO* __restrict__ x, const float* __restrict__ t1g,
                       const float* __restrict__ wfold, IO* __restrict__ y, int* __restrict__ status,
                       const __grid_constant__ CUtensorMap xmap, const RawW rw) {
  extern __shared__ __align__(128) float4 smem4[];
  float* sm = reinterpret_cast<float*>(smem4);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + 2);
  const int tid = threadIdx.x;
  for (int i = tid; i < (P.smem_floats >> 2); i += MAIN_NT) smem4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  __syncthreads();
  if (tid == 0) {
    mb_init(full, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const int myunits = (int)blockIdx.x < P.units ? (P.units - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  float* slot = sm + P.slot0;
  // level-0 direct path without a folded block (wfold null): thread t <= kk4
  // holds the next unit's raw tap t (the bias at t = kk4) and its channel's
  // scale, loaded one unit ahead and scaled into the weight slots when that
  // unit starts
  float w_next = 0.f, s_next = 0.f;
  auto fetch_w = [&](int c) {
    constexpr int KK = K * K;
    if (tid <= P.kk4) {
      s_next = rw.s0[c];
      w_next = tid < KK ? rw.w0[(size_t)c * KK + (rw.flip ? KK - 1 - tid : tid)]
                        : (tid == P.kk4 && !rw.flip ? rw.b0[c] : 0.f);
    }
  };
  if constexpr (DIRECT) {
    if (tid == 0 && myunits > 0) main_issue_tensor(P, slot, full, unit_geo(P, blockIdx.x), 0, &xmap, wfold);
    if (!wfold && myunits > 0) fetch_w(unit_geo(P, blockIdx.x).c);
  } else {
    if (tid == 0 && myunits > 0) main_issue<IO>(P, slot, full, unit_geo(P, blockIdx.x), x, t1g, wfold);
  }
  int k = 0;
  for (; k < myunits; ++k) {
    const UnitGeo g = unit_geo(P, blockIdx.x + k * gridDim.x);
    // every thread waits on every phase in order, so a parity wait is exact
    mb_wait(full, k & 1, abort_flag);
    const int n = (FUSED || DIRECT) ? 0 : g.npb * P.stage_pp;
    if constexpr (FUSED) {
      const int nb = g.npb * P.f_bpp.d;
      for (int it = tid; it < nb; it += MAIN_NT) {
        const int j = P.f_bpp.div(it);
        const int rem = it - j * P.f_bpp.d;
        const int by = P.f_bx4.div(rem);
        const int bx = rem - by * P.f_bx4.d;
        if (P.bulk_x)
          main_stage_block<K, IO, true>(P, slot, j, reinterpret_cast<const IO*>(slot + P.raw_off + j * P.raw_pp),
                                        by, bx);
        else
          main_stage_block<K, IO, false>(P, slot, j, x + plane_index(P, g, j) * P.H * P.W, by, bx);
      }
    }
    for (int it = tid; it < n; it += MAIN_NT) {
      const int j = P.f_spp.div(it);
      const int rem = it - j * P.stage_pp;
      const int ri = P.f_stq.div(rem);
      const int x0 = (rem - ri * P.st_q) << 2;
      float* xf = slot + P.xf.off + j * P.xf.ps;
      float* s1 = slot + P.s1.off + j * P.s1.ps;
      if (P.bulk_x)
        main_stage_item<K, IO, true>(P, xf, s1, reinterpret_cast<const IO*>(slot + P.raw_off + j * P.raw_pp), g, ri,
                                     x0);
      else
        main_stage_item<K, IO, false>(P, xf, s1, x + plane_index(P, g, j) * P.H * P.W, g, ri, x0);
    }
    // folded weights and t1 rows leave the raw region, which the next
    // unit's copies overwrite while this unit computes
    if (DIRECT && !wfold) {
      if (tid <= P.kk4) slot[P.w_off + tid] = s_next * w_next;
    } else {
      for (int i = tid; i < (P.wblk >> 2); i += MAIN_NT)
        reinterpret_cast<float4*>(slot + P.w_off)[i] = reinterpret_cast<const float4*>(slot + P.wraw_off)[i];
    }
    if (!FUSED && P.L >= 2) {
      const int q4 = P.f_t1q.d, per = P.f_t1pp.d;  // (W1 + 3) / 4, TH/2 rows of them
      for (int it = tid; it < g.npb * per; it += MAIN_NT) {
        const int j = P.f_t1pp.div(it), rem = it - j * per;
        const int rr = P.f_t1q.div(rem), x0 = (rem - rr * q4) << 2;
        float4 v;
        if (P.bulk_t) {
          v = *reinterpret_cast<const float4*>(slot + P.rawt_off + j * P.rawt_pp + rr * P.W1 + x0);
        } else {
          const float* q = t1g + plane_index(P, g, j) * P.H1 * P.W1 + (size_t)((g.y0 >> 1) + rr) * P.W1 + x0;
          v = load4(q, x0, P.W1, (P.W1 & 3) == 0);
        }
        *reinterpret_cast<float4*>(slot + P.t1.off + j * P.t1.ps + rr * P.t1.ld + x0) = v;
      }
    }
    __syncthreads();
    if (*abort_flag) break;  // uniform: read after the barrier
    if constexpr (DIRECT) {
      if (tid == 0 && k + 1 < myunits)
        main_issue_tensor(P, slot, full, unit_geo(P, blockIdx.x + (k + 1) * gridDim.x), (k + 1) & 1, &xmap, wfold);
      if (!wfold && k + 1 < myunits) fetch_w(unit_geo(P, blockIdx.x + (k + 1) * gridDim.x).c);
    } else {
      if (tid == 0 && k + 1 < myunits)
        main_issue<IO>(P, slot, full, unit_geo(P, blockIdx.x + (k + 1) * gridDim.x), x, t1g, wfold);
    }
    if constexpr (FUSED) {
      // levels 3..L of the pyramid, then every deep level's band convs
      for (int l = 3; l <= P.L; ++l) {
        const BufDesc& sb = P.sd[l - 1];
        const BufDesc& d = P.sd[l];
        pyramid_level(g.npb, P.H >> l, P.W >> l, slot + sb.off + (K / 2) * sb.ld + K / 2, sb.ld, sb.ps,
                      slot + d.off + (K / 2) * d.ld + K / 2, d.ld, d.ld * d.rows, d.ps);
        __syncthreads();
      }
      const int nd = g.npb * P.f_dper.d;
      for (int it = tid; it < nd; it += MAIN_NT) main_deep_tile<K>(P, slot, it);
      __syncthreads();
    }
    if (P.L >= 1) {
      const int na = g.npb * P.a_pp;
      for (int it = tid; it < na; it += MAIN_NT) main_band_tile<K, FUSED>(P, slot, it);
      __syncthreads();
    }
    for (int it = tid; it < P.tiles; it += MAIN_NT) {
      const int j = P.f_tpp.div(it);
      if (j < g.npb) main_out_tile<K, R3, IO, DIRECT>(P, slot, g, j, it - j * P.tiles_pp, k & 1, y);
    }
    __syncthreads();
  }
  if (*abort_flag && tid == 0) {
    mb_drain(full, k & 1);  // the copies of unit k were issued; let them land before exit
    if (status) atomicExch(status, 1);
  }
}

// ------------------------------------------------------------ deep kernel
// Four elements as loaded (converted to fp32 where used).
template <typename IO> struct Raw4;
template <> struct Raw4<float> {
  using T = float4;
  static __device__ __forceinline__ T ld(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }
  static __device__ __forceinline__ float4 cvt(T v) { return v; }
};
template <> struct Raw4<__nv_bfloat16> {
  using T = uint2;
  static __device__ __forceinline__ T ld(const __nv_bfloat16* p) { return __ldg(reinterpret_cast<const uint2*>(p)); }
  static __device__ __forceinline__ float4 cvt(T r) {
    return make_float4(__uint_as_float(r.x << 16), __uint_as_float(r.x & 0xffff0000u), __uint_as_float(r.y << 16),
                       __uint_as_float(r.y & 0xffff0000u));
  }
};
// Levels 2..L of the planes of a batch: level-2 subbands from 4x4 blocks of
// x, the rest of the pyramid, every level conv (folded weights
// 2^-l s_l W_l), then t1 by the closed form, stored to global memory.
template <int K, typename IO>
__global__ void __launch_bounds__(DEEP_NT) wtconv_deep_kernel(const DeepPlan P, const IO* __restrict__ x,
                                                              const float* __restrict__ wfold,
                                                              float* __restrict__ t1g) {
  constexpr int r = K / 2;
  constexpr int DQ = sizeof(IO) == 2 ? 8 : 4;  // 4x4 blocks in flight per thread
  extern __shared__ float4 smem4[];
  float* sm = reinterpret_cast<float*>(smem4);
  for (int i = threadIdx.x; i < (P.smem_floats >> 2); i += DEEP_NT) smem4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  __syncthreads();
  const int kk4 = P.kk4;
  float* sw = sm + P.w_off;  // wlf[l][s] at ((l - 2) * 4 + s) * kk4
  const size_t plane = (size_t)P.H * P.W;
  const int units = P.C * P.nbatch;
  for (int u = blockIdx.x; u < units; u += gridDim.x) {
    const int bt = u / P.C;
    const int c = u - bt * P.C;
    const int nb0 = bt * P.PB;
    const int npb = (P.N - nb0) < P.PB ? (P.N - nb0) : P.PB;
    // the next unit's planes start towards L2 while this one is processed
    // (each plane is contiguous: H*W elements, a multiple of 16 bytes here)
    if (threadIdx.x < P.PB && u + (int)gridDim.x < units) {
      const int un = u + gridDim.x, btn = un / P.C, cn = un - btn * P.C, nbn = btn * P.PB + (int)threadIdx.x;
      if (nbn < P.N) l2_prefetch(x + ((size_t)nbn * P.C + cn) * plane, (unsigned)(plane * sizeof(IO)));
    }
    // the channel's folded level-2..L weights (contiguous in its block): the
    // first DEEP_NT of them are loaded here and stored after the staging
    // loads below are issued, so that the staging does not wait behind them
    const int nw = (P.L - 1) * 4 * kk4;
    const float* wsrc = wfold + (size_t)c * P.wblk + P.wdeep;
    const float w_first = (int)threadIdx.x < nw ? wsrc[threadIdx.x] : 0.f;
    for (int i = threadIdx.x + DEEP_NT; i < nw; i += DEEP_NT) sw[i] = wsrc[i];
    // level-2 subbands straight from 4x4 blocks of x (DQ blocks in flight per
    // thread, held as loaded and converted where used)
    {
      const int bw = P.W >> 2, per = (P.H >> 2) * bw, n = npb * per;
      const BufDesc& d = P.sd[2];
      const int bs = d.ld * d.rows;
      for (int it0 = threadIdx.x; it0 < n; it0 += DQ * DEEP_NT) {
        typename Raw4<IO>::T v[DQ][4];
#pragma unroll
        for (int q = 0; q < DQ; ++q) {
          const int it = it0 + q * DEEP_NT;
          if (it < n) {
            const int pb = P.f_stage_per.div(it);
            const int rem = it - pb * per;
            const int by = P.f_stage_x.div(rem);
            const int x0 = (rem - by * bw) << 2;
            const IO* src = x + ((size_t)(nb0 + pb) * P.C + c) * plane + (size_t)(by << 2) * P.W + x0;
#pragma unroll
            for (int i = 0; i < 4; ++i) v[q][i] = Raw4<IO>::ld(src + (size_t)i * P.W);  // W % 4 == 0 here
          }
        }
#pragma unroll
        for (int q = 0; q < DQ; ++q) {
          const int it = it0 + q * DEEP_NT;
          if (it < n) {
            const int pb = P.f_stage_per.div(it);
            const int rem = it - pb * per;
            const int by = P.f_stage_x.div(rem);
            const int bxi = rem - by * bw;
            float4 w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) w[i] = Raw4<IO>::cvt(v[q][i]);
            float ll[2][2];
#pragma unroll
            for (int a = 0; a < 2; ++a) {
              float l0, h0, g0, k0, l1, h1, g1, k1;
              haar4(w[2 * a].x, w[2 * a].y, w[2 * a + 1].x, w[2 * a + 1].y, l0, h0, g0, k0);
              haar4(w[2 * a].z, w[2 * a].w, w[2 * a + 1].z, w[2 * a + 1].w, l1, h1, g1, k1);
              ll[a][0] = l0;
              ll[a][1] = l1;
            }
            float L2, H2, G2, K2;
            haar4(ll[0][0], ll[0][1], ll[1][0], ll[1][1], L2, H2, G2, K2);
            float* s2 = sm + d.off + pb * d.ps + (by + r) * d.ld + bxi + r;
            s2[0] = L2;
            s2[bs] = H2;
            s2[2 * bs] = G2;
            s2[3 * bs] = K2;
          }
        }
      }
    }
    if ((int)threadIdx.x < nw) sw[threadIdx.x] = w_first;
    __syncthreads();
    for (int l = 3; l <= P.L; ++l) {
      const BufDesc& sb = P.sd[l - 1];
      const BufDesc& d = P.sd[l];
      pyramid_level(npb, P.H >> l, P.W >> l, sm + sb.off + r * sb.ld + r, sb.ld, sb.ps, sm + d.off + r * d.ld + r,
                    d.ld, d.ld * d.rows, d.ps);
      __syncthreads();
    }
    // every level's band convs (no barrier between levels: each reads its own
    // subbands and writes its own Z planes); the per-level plan entries are
    // read once per level, outside the tile loop.  The tiles of all levels
    // are dealt out as one sequence (thread t takes tiles t, t + DEEP_NT, ...
    // of it), so the few tiles of the deep levels go to threads with fewer
    // level-2 tiles.
    int before = 0;  // tiles of the levels already dealt
    for (int l = 2; l <= P.L; ++l) {
      const BufDesc d = P.sd[l];
      const BufDesc z = P.zd[l];
      const FDiv ft = P.f_l_tiles[l], fx = P.f_l_tx[l], fp = P.f_l_per[l];
      const float* wlv = sw + (l - 2) * 4 * kk4;
      int it = (int)threadIdx.x - before % DEEP_NT;
      if (it < 0) it += DEEP_NT;
      before += npb * fp.d;
      for (; it < npb * fp.d; it += DEEP_NT) {
        const int pb = fp.div(it);
        int rem = it - pb * fp.d;
        const int s = ft.div(rem);
        rem -= s * ft.d;
        const int ti = fx.div(rem);
        const int tj = rem - ti * fx.d;
        float acc[DP_R][DP_CW];
#pragma unroll
        for (int a = 0; a < DP_R; ++a)
#pragma unroll
          for (int b = 0; b < DP_CW; ++b) acc[a][b] = 0.f;
        conv_tile<K, DP_R, DP_CW>(sm + d.off + pb * d.ps + s * d.ld * d.rows + ti * DP_R * d.ld + tj * DP_CW, d.ld,
                                  wlv + s * kk4, acc);
        float* o = sm + z.off + pb * z.ps + s * z.ld * z.rows + ti * DP_R * z.ld + tj * DP_CW;
#pragma unroll
        for (int a = 0; a < DP_R; ++a)
          reinterpret_cast<float4*>(o + a * z.ld)[0] = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
      }
    }
    __syncthreads();
    // t1(i, j) = sum_{l>=2} sum_s sigma_s(bit_{l-2}(i), bit_{l-2}(j)) Zd_l^s(i >> (l-1), j >> (l-1)).
    // The terms of levels >= 3 are the same sum one level down, at
    // (i >> 1, j >> 1), and the LL sign is always +, so the sum is taken
    // level by level from the deepest: the synthesis of level l's four Z
    // planes is added into level l-1's LL Z plane, then t1 is the synthesis
    // of level 2's four planes.  Pixels of level l-1 go in pairs (2j', 2j'+1)
    // that share their level-l parent (i >> 1, j').
    for (int l = P.L; l >= 3; --l) {
      const BufDesc zs = P.zd[l], zt = P.zd[l - 1];
      const FDiv fx = P.f_up_x[l], fp = P.f_up_per[l];
      const int bz = zs.ld * zs.rows;
      for (int it = threadIdx.x; it < npb * fp.d; it += DEEP_NT) {
        const int pb = fp.div(it);
        const int rem = it - pb * fp.d;
        const int i = fx.div(rem);
        const int jp = rem - i * fx.d;
        const float* q = sm + zs.off + pb * zs.ps + (i >> 1) * zs.ld + jp;
        const float sy = (i & 1) ? -1.f : 1.f;
        const float A = fmaf(sy, q[bz], q[0]), B = fmaf(sy, q[3 * bz], q[2 * bz]);
        float2* t = reinterpret_cast<float2*>(sm + zt.off + pb * zt.ps + i * zt.ld + 2 * jp);
        float2 v = *t;
        v.x += A + B;
        v.y += A - B;
        *t = v;
      }
      __syncthreads();
    }
    {
      // t1 rows 2i' and 2i' + 1, columns j0 .. j0 + 3: parents (i', j0/2) and (i', j0/2 + 1)
      const int tq = P.f_t1_x.d, per1 = P.f_t1_per.d;
      const BufDesc& z2 = P.zd[2];
      const int bz2 = z2.ld * z2.rows;
      for (int it = threadIdx.x; it < npb * per1; it += DEEP_NT) {
        const int pb = P.f_t1_per.div(it);
        const int rem = it - pb * per1;
        const int ip = P.f_t1_x.div(rem);
        const int j0 = (rem - ip * tq) << 2;
        const float* q = sm + z2.off + pb * z2.ps + ip * z2.ld + (j0 >> 1);
        const float2 zl = *reinterpret_cast<const float2*>(q);
        const float2 zh = *reinterpret_cast<const float2*>(q + bz2);
        const float2 zg = *reinterpret_cast<const float2*>(q + 2 * bz2);
        const float2 zk = *reinterpret_cast<const float2*>(q + 3 * bz2);
        float* dst = t1g + ((size_t)(nb0 + pb) * P.C + c) * P.H1 * P.W1 + (size_t)(2 * ip) * P.W1 + j0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float sy = h ? -1.f : 1.f;
          const float a0 = fmaf(sy, zh.x, zl.x), c0 = fmaf(sy, zk.x, zg.x);
          const float a1 = fmaf(sy, zh.y, zl.y), c1 = fmaf(sy, zk.y, zg.y);
          const float o[4] = {a0 + c0, a0 - c0, a1 + c1, a1 - c1};
          float* row = dst + (size_t)h * P.W1;
          if ((P.W1 & 3) == 0) {
            *reinterpret_cast<float4*>(row) = make_float4(o[0], o[1], o[2], o[3]);
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (j0 + e < P.W1) row[e] = o[e];
          }
        }
      }
    }
    __syncthreads();
  }
}

}  // namespace wt
