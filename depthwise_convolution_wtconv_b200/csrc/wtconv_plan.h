// Shared-memory plan of the per-plane WTConv kernels.
//
// One CTA owns one (n, c) image plane at a time and keeps the whole plane,
// its level-1 Haar subbands and the deeper pyramid in shared memory, so the
// subbands never travel through HBM (reformulation (1) of arXiv:2608.10805,
// abstract).  The host fills a Plan and passes it by value to the kernel.
//
// Buffer conventions (all offsets and leading dimensions in floats):
//  * "shifted" buffers (read at x0-r by the register tiles) store element
//    (y, x) at off + (y + r) * ld + (x + r); a zero border of r rows/cols
//    surrounds the image and the slack past it is zero or never used by a
//    stored output.
//  * "plain" buffers store (y, x) at off + y * ld + x.
//  * every offset and ld is a multiple of 4 floats (16-byte alignment).
#pragma once

#include "wtconv.h"

namespace wt {

constexpr int NT = 256;           // threads per CTA
constexpr int MAXL = WTCONV_MAX_LEVELS;

// register-tile shapes (rows x cols of outputs per thread)
constexpr int C3_CW = 8;          // base conv + synthesis, full resolution
constexpr int C2_R = 4, C2_CW = 4;  // level-1 band conv, half resolution
constexpr int DP_R = 2, DP_CW = 4;  // deep levels
constexpr int BW_R = 4, BW_CW = 8;  // weight-gradient correlation, full resolution
constexpr int B1_R = 4, B1_CW = 4;  // weight-gradient correlation, level 1
constexpr int DSLOTS = 8;           // threads per deep (level, band) in the correlation pass

// Division by a runtime divisor d >= 1 without an integer divide:
// x / d == umulhi(x, m) >> s for 0 <= x < 2^31 (m, s set on the host).
struct FDiv {
  int d;
  unsigned m;
  int s;
#ifdef __CUDACC__
  __host__ __device__
#endif
  FDiv() : d(1), m(0), s(0) {}
#ifdef __CUDACC__
  __device__ __forceinline__ int div(int x) const {
    return d == 1 ? x : (int)(__umulhi((unsigned)x, m) >> s);
  }
#endif
};

struct BufDesc {
  int off, ld, rows;   // rows allocated; band stride = ld * rows
  int ps;              // stride between the copies of consecutive planes of a batch
};

struct Plan {
  int N, C, H, W, K, r, L;
  int H1, W1;
  int R3;              // rows of the full-resolution register tile (2 or 4)
  int kk4;             // K*K rounded up to 4
  int vec_in, vec_out; // global rows allow 16-byte vector access
  int prefetch_ok;     // plane bytes are a multiple of 16 (TMA bulk copies allowed)
  int use_bulk;        // stage through TMA bulk copies into the raw buffer(s)
  int raw_off, rawg_off;  // raw copies of x (and dy) of one batch, I/O dtype
  int nthreads;        // threads per CTA of the forward kernel
  int io_bytes;        // bytes per element of x, y, dy, dx
  // weights (folded): w0 [kk4], b0 [4], wl[l][s] [kk4] for l = 1..L
  int w_off;
  BufDesc xf;          // shifted: input plane (fp32)
  BufDesc s1;          // shifted: 4 bands of level-1 subbands
  BufDesc zb;          // plain: 4 bands of folded level-1 conv outputs
  BufDesc t1;          // plain: deep synthesis at level-1 resolution
  int deep_off, deep_floats;   // region re-zeroed before every deep pass
  BufDesc sd[MAXL + 1];        // shifted: level-l subbands (l >= 2), 4 bands
  BufDesc zd[MAXL + 1];        // plain: folded level-l conv outputs (l >= 3)
  BufDesc t2;                  // plain: deep synthesis at level-2 resolution
  // weight-gradient kernel only
  BufDesc gf;          // plain: dy plane (fp32)
  BufDesc g1;          // plain: 4 bands of dy level-1 subbands
  BufDesc gd[MAXL + 1];        // plain: dy level-l subbands (l >= 2)
  int red_off;         // per-thread partial sums for the final reduction
  int gdeep_off;       // deep-level accumulators [L-1][4][kk4]
  int dpart_off;       // deep-level per-slot partials [L-1][4][DSLOTS][kk4]
  // item decompositions of the forward phases (divisors per plane)
  FDiv f_stage_per, f_stage_x;   // staging items per plane, per block row
  FDiv f_deep_per;               // deep conv items per plane
  FDiv f_t1_per, f_t1_x;         // t1 items per plane, per row
  FDiv f_out_per, f_out_x;       // output tiles per plane, per tile row
  FDiv f_bw_per, f_bw_x;         // weight-gradient base tiles per plane, per row
  FDiv f_b1_per, f_b1_x;         // weight-gradient level-1 tiles per band, per row
  FDiv f_l_tiles[MAXL + 1];      // deep conv tiles per band of level l
  FDiv f_l_tx[MAXL + 1];         // deep conv tiles per tile row of level l
  int deep_items;                // deep conv items per plane (levels 2..L)
  int deep_first[MAXL + 2];      // first item of level l within a plane
  int PB;              // planes of one channel processed together (a batch)
  int nbatch;          // batches per channel: ceil(N / PB)
  int planes_per_cta;  // weight-gradient kernel: consecutive n per CTA
  int ngroups;         // weight-gradient kernel: CTAs per channel
  int V;               // partial-sum entries per CTA: K*K*(1+4L) + 1
  int smem_floats;
};

}  // namespace wt

namespace wt {

// Plan of the output kernel (forward and backward-data).  A unit is one band
// of TH output rows of one (n, c) plane (TH = H when the whole plane fits),
// or PB whole planes of one channel.  The CTA's one slot holds a raw region
// (the next unit's bulk copies: folded weights, input rows, t1 rows) and the
// current unit's folded weights, padded fp32 rows xf, padded level-1
// subbands s1 and t1 rows.  Offsets are floats relative to the slot start.
struct MainPlan {
  int N, C, H, W, K, r, L, H1, W1, kk4, io_bytes;
  int TH, nbands, PB;        // band rows, bands per plane, planes per unit (PB > 1 only without bands)
  int units;                 // C * ceil(N/PB) * nbands
  int R3, tiles, tiles_pp;   // output tile rows (8 or 4; tiles are 4 wide), tiles per unit, per plane
  int bulk_x, bulk_t;        // TMA bulk copies usable for x rows / t1 rows
  int vec_in, vec_out;
  int st_row0, st_rows, st_q, stage_pp;  // staged rows per plane (band), items per plane
  int slot0, slot_floats;    // slot offset (after the header) and size
  int wblk;                  // floats of one channel's folded weights
  int wraw_off, raw_off, rawt_off, raw_pp, rawt_pp;  // raw region of the bulk copies (per-plane strides)
  int w_off;                 // the current unit's folded weights
  BufDesc xf, s1, t1, zb;    // per-plane copies at ps stride (zb: the four level-1 Z planes)
  int a_pp;                  // phase-A tiles per plane: 4 bands x ceil(TH/8) x ceil(W1/4)
  int fused;                 // whole planes with L >= 2: levels >= 2 computed here, t1 on the fly
  BufDesc sd[MAXL + 1], zd[MAXL + 1];  // fused: subbands and band-conv outputs of levels 2..L
  int dfirst[MAXL + 2];      // fused: first deep-conv tile of level l within a plane
  FDiv f_dtiles[MAXL + 1], f_dtx[MAXL + 1], f_dper;  // fused: 4x4 tiles per band, per tile row; per plane
  FDiv f_bpp, f_bx4;         // fused: 4x4 staging blocks per plane, per block row
  FDiv f_tiles, f_tpp, f_tx, f_stq, f_spp, f_bands, f_C;
  FDiv f_app, f_abt, f_atx;  // phase-A decomposition: per plane, per band, per tile row
  int smem_floats;
};

// Plan of the deep-level kernel: levels 2..L of PB planes of one channel,
// written as t1 (the synthesis of levels >= 2 at level-1 resolution,
// already scaled by the level-1 synthesis factor) to global memory.
struct DeepPlan {
  int N, C, H, W, K, r, L, H1, W1, kk4, io_bytes, vec_in;
  int PB, nbatch;
  int w_off;                 // folded weights of levels 2..L
  BufDesc sd[MAXL + 1], zd[MAXL + 1];
  FDiv f_stage_per, f_stage_x, f_deep_per, f_t1_per, f_t1_x;
  FDiv f_l_tiles[MAXL + 1], f_l_tx[MAXL + 1];
  int deep_items, deep_first[MAXL + 2];
  int smem_floats;
};

// Plan of one launch of the row-band weight-gradient kernel.  The launch
// correlates on the "level grid" (Hl x Wl): the image itself for lvl 0, the
// level-lvl subbands for lvl >= 1, whose input planes A (x or a raw LL) and
// B (dy or its raw LL) are H x W = 2Hl x 2Wl.  A band is TB rows of the
// level grid.  Shared buffers (offsets and lds in floats, multiples of 4):
//   a: FR + 2*ha input rows of A from row y0 - ha, column j at j + r
//   b: FR input rows of B from row y0, column j at j
//   s: 4 subbands of A over TB + 2r level rows from i0 - r, column j at j + r
//   d: 4 subbands of B over the TB band rows, column j at j
struct BandPlan {
  int N, C, H, W, K, r, kk4, V;
  int lvl, Hl, Wl;
  int TB, nb, FR, ha;
  int units, ngroups;
  int a_off, a_ld, a_rows;
  int b_off, b_ld, b_rows;
  int s_off, s_ld, s_rows;
  int d_off, d_ld, d_rows;
  int red_off;               // (NT/32) * kk4 + NT/32 floats of the final reduction
  int smem_floats;
  int vec, write_ll, seg;
  FDiv f_nb, f_bx, f_bper, f_sx, f_sper;
};

}  // namespace wt
