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
  int PB;              // planes of one channel processed together (a batch)
  int nbatch;          // batches per channel: ceil(N / PB)
  int planes_per_cta;  // weight-gradient kernel: consecutive n per CTA
  int ngroups;         // weight-gradient kernel: CTAs per channel
  int V;               // partial-sum entries per CTA: K*K*(1+4L) + 1
  int smem_floats;
};

}  // namespace wt
