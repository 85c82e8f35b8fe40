// Shared-memory plans of the WTConv kernels (the host fills one per launch
// and passes it by value).  The kernels keep each plane's Haar subbands in
// shared memory, so they never travel through HBM (reformulation (1) of
// arXiv:2608.10805, abstract).
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

constexpr int NT = 256;           // threads per CTA of the row-band weight-gradient kernel
constexpr int MAXL = WTCONV_MAX_LEVELS;

// register-tile shapes (rows x cols of outputs per thread)
constexpr int DP_R = 2, DP_CW = 4;  // deep-level kernel
constexpr int BW_R = 8, BW_CW = 4;  // row-band weight gradients, full resolution (4 wide: lanes read consecutive 16-byte words)
constexpr int B1_R = 4, B1_CW = 4;  // row-band weight gradients, level grid

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
  int oH, oW;                // planes of y: H x W, or the image inside zero-padded planes
  int st_row0, st_rows, st_q, stage_pp;  // staged rows per plane (band), items per plane
  int slot0, slot_floats;    // slot offset (after the header) and size
  int wblk;                  // floats of one channel's folded weights
  int wraw_off, raw_off, rawt_off, raw_pp, rawt_pp;  // raw region of the bulk copies (per-plane strides)
  int w_off;                 // the current unit's folded weights
  BufDesc xf, s1, t1, zb;    // per-plane copies at ps stride (zb: the four level-1 Z planes)
  int a_pp;                  // phase-A tiles per plane: 4 bands x ceil(TH/8) x ceil(W1/4)
  int fused;                 // whole planes with L >= 2: levels >= 2 computed here, t1 on the fly
  int direct, xbuf;          // level-0 fp32 rows copied straight into two xf buffers xbuf floats apart
  BufDesc sd[MAXL + 1], zd[MAXL + 1];  // fused: subbands and band-conv outputs of levels 2..L
  int dfirst[MAXL + 2];      // fused: first deep-conv tile of level l within a plane
  FDiv f_dtiles[MAXL + 1], f_dtx[MAXL + 1], f_dper;  // fused: 4x4 tiles per band, per tile row; per plane
  FDiv f_bpp, f_bx4;         // fused: 4x4 staging blocks per plane, per block row
  FDiv f_tiles, f_tpp, f_tx, f_stq, f_spp, f_bands, f_C;
  FDiv f_app, f_abt, f_atx;  // phase-A decomposition: per plane, per band, per tile row
  FDiv f_t1pp, f_t1q;        // t1 rows of a unit: 4-float groups per plane, per row
  int smem_floats;
};

// Plan of the deep-level kernel: levels 2..L of PB planes of one channel,
// written as t1 (the synthesis of levels >= 2 at level-1 resolution,
// already scaled by the level-1 synthesis factor) to global memory.
// Raw parameters for the level-0 direct output kernel, which can scale the
// taps and the bias itself instead of reading a folded block.
struct RawW {
  const float* w0;
  const float* b0;
  const float* s0;
  int flip;
};

struct DeepPlan {
  int N, C, H, W, K, r, L, H1, W1, kk4, io_bytes, vec_in;
  int PB, nbatch;
  int wblk, wdeep;           // floats per channel of the folded block; offset of its level-2 kernels
  int w_off;                 // folded weights of levels 2..L
  BufDesc sd[MAXL + 1], zd[MAXL + 1];
  FDiv f_stage_per, f_stage_x, f_t1_per, f_t1_x;
  FDiv f_l_tiles[MAXL + 1], f_l_tx[MAXL + 1], f_l_per[MAXL + 1];  // per level: tiles per band, per row, per plane
  FDiv f_up_x[MAXL + 1], f_up_per[MAXL + 1];  // l >= 3: pixel pairs of level l-1 per row, per plane
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
  int raw_a, raw_b;          // raw copies of the next unit's A window and B rows (bulk copies)
  int in_bytes, bulk;        // bytes per input element; rows 16-byte aligned for bulk copies
  int smem_floats;
  int vec, write_ll, seg;
  FDiv f_nb, f_bx, f_bper, f_sx, f_sper;
  FDiv f_q4, f_wl;           // 4-element groups per input row; level-grid width
};

// One correlation branch of the whole-plane weight-gradient kernel: the
// base taps (branch 0) or band s of level l (branch 1 + 4(l-1) + s).  Its
// 4x4 tiles correlate the shifted operand a (x side, read at x0 - r) with the
// plain operand g (dy side); the sums go to entries [seg, seg + K*K) of the
// partial vector.  Threads [first, first + nthr) own the branch.
struct BwBranch {
  int a_off, a_ld, g_off, g_ld;  // band 0 of plane 0 of the slot; band offsets are added per branch
  int first, nthr, seg;
  FDiv f_tiles, f_tx;            // 4x4 tiles per plane, per tile row
};

// Plan of the whole-plane weight-gradient kernel: a CTA of BW_NT threads
// owns channel c and planes [g*ppc, (g+1)*ppc) of it, PB planes per unit.
// The slot holds the raw copies (bulk copies of the next unit) of x and dy,
// and per plane: xf / gf (x padded, dy plain), the level-1 subbands of both
// (s1x shifted, g1 plain) and, for l >= 2, sd[l] / gd[l].
constexpr int BW_NT = 256;
constexpr int BW_MAXB = 1 + 4 * MAXL;
struct BwPlan {
  int N, C, H, W, K, r, L, H1, W1, kk4, V, io_bytes, vec_in;
  int PB, ppc, ngroups, units;     // planes per unit, planes per CTA, CTAs per channel
  int bulk;                        // whole planes by bulk copies (plane bytes % 16 == 0)
  int raw_x, raw_g, raw_pp;        // raw copies of one unit (floats; per-plane stride)
  int ps;                          // per-plane slab stride (floats)
  BufDesc xf, gf, s1, g1, sd[MAXL + 1], gd[MAXL + 1];
  int BH;                          // staging block rows: 4 (L >= 2), 2 (L = 1), 1 (L = 0)
  FDiv f_spp, f_sx;                // staging blocks per plane, per block row
  int nbr;                         // branches: 1 + 4L
  BwBranch br[BW_MAXB];
  int red_off;                     // final reduction: BW_NT * (kk4 + 1) + BW_NT floats (over the slab)
  int smem_floats;
  int dys;                         // dy buffers shifted like x's (the fused backward reads them as conv inputs)
  int w_off;                       // fused backward: the channel's adjoint folded weights
};

// Plan of the fused backward kernel (whole planes): the weight-gradient plan
// B (with dy staged in the shifted layout) and, for the backward-data pass
// over the same staged dy, an output-kernel plan M whose input buffers are
// B's dy buffers and whose Z planes reuse B's x-side buffers once the
// correlations are done.
struct BwdPlan {
  BwPlan B;
  MainPlan M;
  // ranges of each plane's slab the adjoint writes over x's buffers (zb over
  // xf, the deep Z planes over s1): cleared before the next unit, since x's
  // staging writes only the interiors and relies on zero borders
  int za_off, za_len, zb_off, zb_len;
};

// Plan of the level-0 fp32 weight-gradient kernel fed by tensor copies: a
// CTA owns channel c and planes [g*ppc, (g+1)*ppc), PB planes per unit, in
// two buffer sets (the next unit's copies land in one while the CTA works on
// the other).  x arrives zero-padded: row y of plane j at
// xoff + j*xps + (y + r) * xld + x + 4 (xld = W + 8, 128-byte aligned
// destination); dy plain: goff + j*gps + y * gld + x (gld = W).  The final
// reduction uses BW_NT * (kk4 + 1) + BW_NT floats at red_off.
struct BwDirectPlan {
  int N, C, H, W, K, r, kk4, V;
  int PB, ppc, ngroups;
  int nb, TB;           // row bands per plane (1: whole planes) and rows per band (PB = 1 then)
  int xld, xrows, xps, gld, grows, gps;
  int xoff[2], goff[2];
  int tiles_pp;
  FDiv f_tiles, f_tx;  // 4x4 tiles per plane, per tile row
  int red_off, smem_floats;
};

}  // namespace wt
