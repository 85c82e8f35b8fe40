// C ABI of libwtconv: argument checks, shared-memory plans and launches.
// The operations and their definitions are documented in include/wtconv.h.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <initializer_list>
#include <mutex>
#include <type_traits>
#include <vector>

#include "wtconv.h"
#include "wtconv_kernels.cuh"
#include "wtconv_main.cuh"
#include "wtconv_bwband.cuh"
#include "wtconv_bwdw.cuh"
#include "wtconv_small.cuh"

namespace wt {
namespace {

inline int rup(int a, int b) { return (a + b - 1) / b * b; }
inline int cdiv_h(int a, int b) { return (a + b - 1) / b; }

// Magic numbers for FDiv: x / d == umulhi(x, m) >> s for 0 <= x < 2^31.
FDiv make_fdiv(int d) {
  FDiv f;
  f.d = d < 1 ? 1 : d;
  f.m = 0;
  f.s = 0;
  if (f.d > 1) {
    int lg = 0;
    while ((1LL << lg) < f.d) ++lg;  // ceil(log2 d)
    const unsigned long long p = 31 + lg;
    f.m = (unsigned)(((1ULL << p) + (unsigned long long)f.d - 1) / (unsigned long long)f.d);
    f.s = (int)(p - 32);
  }
  return f;
}

struct TileShape {
  int R, CW;
};

// Shifted buffer able to serve register tiles of every listed shape.
BufDesc make_shifted(int& cur, int h, int w, int r, std::initializer_list<TileShape> shapes, int nb) {
  int rows = h + 2 * r, ld = w + 2 * r;
  for (const TileShape& s : shapes) {
    const int nv = (s.CW + 2 * r + 3) / 4;
    rows = std::max(rows, rup(h, s.R) + 2 * r);
    ld = std::max(ld, rup(w, s.CW) - s.CW + nv * 4);
  }
  ld = rup(ld, 4);
  BufDesc d{cur, ld, rows, 0};
  cur += rup(ld * rows * nb, 4);
  return d;
}

BufDesc make_plain(int& cur, int h, int w, std::initializer_list<TileShape> shapes, int nb) {
  int rows = h, ld = w;
  for (const TileShape& s : shapes) {
    rows = std::max(rows, rup(h, s.R));
    ld = std::max(ld, rup(w, s.CW));
  }
  ld = rup(ld, 4);
  BufDesc d{cur, ld, rows, 0};
  cur += rup(ld * rows * nb, 4);
  return d;
}


int io_bytes(const wtconv_desc* d) { return d->io == WTCONV_BF16 ? 2 : 4; }

constexpr int SM_SMEM = 233472;  // shared memory per SM on sm_100a (228 KB)

// Floats of one channel's folded weights: the base kernel, the bias and
// four kernels per level (kk4 floats each).
int main_wblk(const wtconv_desc* d) { return rup((1 + 4 * d->L) * rup(d->k * d->k, 4) + 4, 4); }

// Output tile rows for band height TH: 8, unless 4 wastes fewer padded rows
// or the band is at most 8 rows (twice the tiles for the CTA's threads).
// Level-0 whole planes of at most 16 rows take 4: these units are short and
// latency-bound, and the smaller register tile lets more CTAs share an SM.
int main_r3(int H, int L, int TH) {
  if (L == 0 && TH == H && H <= 16) return 4;
  return TH > 8 && rup(TH, 8) == rup(TH, 4) ? 8 : 4;
}

// Slot layout for band height TH and PB planes per unit; returns the slot
// size in floats.
int main_slot(MainPlan& M, int TH, int PB) {
  const int r = M.r, R3 = main_r3(M.H, M.L, TH), TH1 = TH / 2;
  const int hx = M.L >= 1 ? 2 * r : r;
  M.fused = TH == M.H && M.L >= 2;
  if (M.fused) M.bulk_t = 0;
  int cur = 0;
  // raw region: written by the bulk copies of the next unit
  M.wraw_off = cur;
  cur += M.wblk;
  M.raw_off = cur;
  M.raw_pp = M.direct ? 0 : rup((int)(((size_t)std::min(M.H, TH + 2 * hx) * M.W * M.io_bytes + 3) / 4), 4);
  cur += PB * M.raw_pp;
  M.rawt_off = cur;
  M.rawt_pp = (M.L >= 2 && M.bulk_t) ? rup(TH1 * M.W1, 4) : 0;
  cur += PB * M.rawt_pp;
  // the current unit's staged data, read by the register tiles
  M.w_off = cur;
  cur += M.wblk;
  int pcur = 0;  // per-plane buffers, PB copies each
  if (M.direct) {
    // rows land here straight from the bulk copies: column x at x + 4 (16-byte
    // aligned), zero columns on both sides; two buffers, one per phase
    M.xf = BufDesc{pcur, rup(M.W, 4) + 8, rup(TH, R3) + 2 * r, 0};
    pcur += M.xf.ld * M.xf.rows;
  } else {
    M.xf = make_shifted(pcur, TH, M.W, r, {{R3, 4}}, 1);
  }
  M.s1 = BufDesc{0, 0, 0, 0};
  M.t1 = BufDesc{0, 0, 0, 0};
  M.zb = BufDesc{0, 0, 0, 0};
  if (M.L >= 1) {
    M.s1 = make_shifted(pcur, TH1, M.W1, r, {{4, 4}}, 4);
    const int zrows = std::max(rup(TH1, 4), rup(TH, R3) / 2);
    M.zb = make_plain(pcur, zrows, M.W1, {{4, 4}}, 4);
  }
  if (M.L >= 2 && !M.fused) M.t1 = make_plain(pcur, TH1, M.W1, {{4, 4}}, 1);
  for (int l = 0; l <= MAXL; ++l) M.sd[l] = M.zd[l] = BufDesc{0, 0, 0, 0};
  if (M.fused) {
    for (int l = 2; l <= M.L; ++l) M.sd[l] = make_shifted(pcur, M.H >> l, M.W >> l, r, {{4, 4}}, 4);
    for (int l = 2; l <= M.L; ++l) M.zd[l] = make_plain(pcur, M.H >> l, M.W >> l, {{4, 4}}, 4);
  }
  const int pstride = rup(pcur, 4);
  // level-0 rows arrive by one tensor copy per unit: its destination starts
  // on a 128-byte boundary (the slot itself starts MAIN_HEADER floats into
  // shared memory)
  if (M.direct) cur = rup(cur + MAIN_HEADER, 32) - MAIN_HEADER;
  for (BufDesc* bd : {&M.xf, &M.s1, &M.t1, &M.zb}) {
    bd->off += cur;
    bd->ps = pstride;
  }
  for (int l = 2; l <= M.L && M.fused; ++l)
    for (BufDesc* bd : {&M.sd[l], &M.zd[l]}) {
      bd->off += cur;
      bd->ps = pstride;
    }
  M.xbuf = 0;
  if (M.direct) {
    M.xbuf = rup(PB * pstride, 32);  // the second buffer, also 128-byte aligned
    cur += 2 * M.xbuf;
  } else {
    cur += PB * pstride;
  }
  return rup(cur, 4);
}

bool build_main_plan(MainPlan& M, const wtconv_desc* d, int max_smem) {
  M = MainPlan{};
  M.N = d->N; M.C = d->C; M.H = d->H; M.W = d->W; M.K = d->k; M.r = d->k / 2; M.L = d->L;
  M.H1 = d->L >= 1 ? d->H / 2 : d->H;
  M.W1 = d->L >= 1 ? d->W / 2 : d->W;
  M.kk4 = rup(d->k * d->k, 4);
  M.io_bytes = io_bytes(d);
  M.vec_in = (d->W % 4) == 0;
  M.vec_out = (d->W % 4) == 0;
  M.oH = d->H;
  M.oW = d->W;
  M.wblk = main_wblk(d);
  M.bulk_t = d->L >= 2 && (M.W1 % 4) == 0;
  // level-0 fp32 planes whose rows are 16-byte multiples go straight to the
  // padded row buffers by one tensor copy per unit (box inner extent W + 8,
  // at most 256 elements)
  M.direct = d->L == 0 && d->io == WTCONV_F32 && (d->W % 4) == 0 && d->W + 8 <= 256;
  const int tx = cdiv_h(d->W, 4);
  // Whole planes when at least three CTAs fit per SM (no halo rows staged
  // twice); else the most CTAs per SM (four, then three, two, one) with the
  // largest band height (an even divisor of H) whose slot fits that share of
  // the SM's shared memory.  Without bands, small planes are batched so that
  // a unit has about one tile per thread.
  int TH = -1, PB = 1;
  for (int pass = 0; pass < 2 && TH < 0; ++pass)
  for (int occ = 4; occ >= (pass == 0 ? 3 : 1) && TH < 0; --occ) {
    const size_t budget = std::min((size_t)max_smem, (size_t)SM_SMEM / occ - 1024);
    for (int cand = d->H; cand >= (pass == 0 ? d->H : 2) && TH < 0; --cand) {
      if (d->H % cand || (cand != d->H && (cand & 1))) continue;
      if (M.direct && rup(cand, main_r3(d->H, d->L, cand)) + 2 * M.r > 256) continue;  // tensor box rows
      const int tpp = cdiv_h(cand, main_r3(d->H, d->L, cand)) * tx;
      int pb = cand == d->H ? std::max(1, std::min(d->N, MAIN_NT / tpp)) : 1;
      for (; pb >= 1 && TH < 0; --pb) {
        MainPlan T = M;
        const int slot = main_slot(T, cand, pb);
        if ((size_t)(MAIN_HEADER + slot) * 4 <= budget) {
          TH = cand;
          PB = pb;
        }
      }
    }
  }
  if (TH < 0) return false;
  M.TH = TH;
  M.PB = PB;
  M.R3 = main_r3(d->H, d->L, TH);
  M.nbands = d->H / TH;
  M.units = d->C * ((d->N + PB - 1) / PB) * M.nbands;
  M.slot_floats = main_slot(M, TH, PB);
  M.slot0 = MAIN_HEADER;
  M.smem_floats = M.slot0 + M.slot_floats;
  const size_t plane_bytes = (size_t)d->H * d->W * M.io_bytes;
  M.bulk_x = M.nbands == 1 ? (plane_bytes % 16 == 0) : (((size_t)d->W * M.io_bytes) % 16 == 0);
  const bool band = M.nbands > 1;
  if (d->L >= 1) {
    M.st_row0 = band ? -M.r : 0;
    M.st_rows = band ? TH / 2 + 2 * M.r : M.H1;
  } else {
    M.st_row0 = band ? -M.r : 0;
    M.st_rows = band ? TH + 2 * M.r : M.H;
  }
  M.st_q = cdiv_h(d->W, 4);
  M.stage_pp = M.st_rows * M.st_q;
  M.tiles_pp = cdiv_h(TH, M.R3) * tx;
  M.tiles = PB * M.tiles_pp;
  const int atx = cdiv_h(M.W1, 4), aty = cdiv_h(TH / 2, 4);
  M.a_pp = d->L >= 1 ? 4 * aty * atx : 0;
  M.f_app = make_fdiv(std::max(1, M.a_pp));
  M.f_t1q = make_fdiv((M.W1 + 3) / 4);
  M.f_t1pp = make_fdiv(std::max(1, (TH / 2) * ((M.W1 + 3) / 4)));
  M.f_abt = make_fdiv(aty * atx);
  M.f_atx = make_fdiv(atx);
  int first = 0;
  for (int l = 0; l <= MAXL + 1; ++l) M.dfirst[l] = 0;
  for (int l = 2; l <= d->L && M.fused; ++l) {
    const int dtx = cdiv_h(d->W >> l, 4), tiles = cdiv_h(d->H >> l, 4) * dtx;
    M.f_dtiles[l] = make_fdiv(tiles);
    M.f_dtx[l] = make_fdiv(dtx);
    M.dfirst[l] = first;
    first += 4 * tiles;
  }
  if (M.fused) M.dfirst[d->L + 1] = first;
  M.f_dper = make_fdiv(std::max(1, first));
  M.f_bpp = make_fdiv(std::max(1, (d->H / 4) * (d->W / 4)));
  M.f_bx4 = make_fdiv(std::max(1, d->W / 4));
  M.f_tiles = make_fdiv(M.tiles);
  M.f_tpp = make_fdiv(M.tiles_pp);
  M.f_tx = make_fdiv(tx);
  M.f_stq = make_fdiv(M.st_q);
  M.f_spp = make_fdiv(M.stage_pp);
  M.f_bands = make_fdiv(M.nbands);
  M.f_C = make_fdiv(d->C);
  return true;
}

// ------------------------------------------------------------ deep kernel
void deep_slab_items(DeepPlan& D, int& slab) {
  const int r = D.r;
  int cur = 0;
  for (int l = 2; l <= D.L; ++l) D.sd[l] = make_shifted(cur, D.H >> l, D.W >> l, r, {{DP_R, DP_CW}, {2, 2}}, 4);
  for (int l = 2; l <= D.L; ++l) D.zd[l] = make_plain(cur, D.H >> l, D.W >> l, {{DP_R, DP_CW}}, 4);
  slab = rup(cur, 4);
}

bool build_deep_plan(DeepPlan& D, const wtconv_desc* d, int max_smem) {
  D = DeepPlan{};
  D.N = d->N; D.C = d->C; D.H = d->H; D.W = d->W; D.K = d->k; D.r = d->k / 2; D.L = d->L;
  D.H1 = d->H / 2;
  D.W1 = d->W / 2;
  D.kk4 = rup(d->k * d->k, 4);
  D.io_bytes = io_bytes(d);
  D.vec_in = (d->W % 4) == 0;
  D.wblk = main_wblk(d);
  D.wdeep = 5 * D.kk4 + 4;
  int slab = 0;
  deep_slab_items(D, slab);
  D.w_off = 0;
  const int base = rup((D.L - 1) * 4 * D.kk4, 4);
  const int t1_items = D.H1 * cdiv_h(D.W1, 4);
  int PB = std::max(1, std::min(d->N, DEEP_NT / std::max(1, t1_items)));
  while (PB > 1 && (size_t)(base + PB * slab) * 4 > (size_t)max_smem / 2) --PB;
  if ((size_t)(base + PB * slab) * 4 > (size_t)max_smem) return false;
  D.PB = PB;
  D.nbatch = (d->N + PB - 1) / PB;
  for (int l = 0; l <= MAXL; ++l) {
    D.sd[l].off += base;
    D.sd[l].ps = slab;
    D.zd[l].off += base;
    D.zd[l].ps = slab;
  }
  D.smem_floats = base + PB * slab;
  const int bw = D.W >> 2;
  D.f_stage_per = make_fdiv((D.H >> 2) * bw);
  D.f_stage_x = make_fdiv(bw);
  for (int l = 2; l <= D.L; ++l) {
    const int tx = cdiv_h(D.W >> l, DP_CW), tiles = cdiv_h(D.H >> l, DP_R) * tx;
    D.f_l_tiles[l] = make_fdiv(tiles);
    D.f_l_tx[l] = make_fdiv(tx);
    D.f_l_per[l] = make_fdiv(4 * tiles);
  }
  for (int l = 3; l <= D.L; ++l) {
    const int px = (D.W >> (l - 1)) / 2;
    D.f_up_x[l] = make_fdiv(px);
    D.f_up_per[l] = make_fdiv((D.H >> (l - 1)) * px);
  }
  const int tq = cdiv_h(D.W1, 4);
  D.f_t1_x = make_fdiv(tq);
  D.f_t1_per = make_fdiv((D.H1 / 2) * tq);  // items of two t1 rows by four columns
  return true;
}

// Plan constants of sm_100a (B200): opt-in shared memory per CTA and SM
// count.  The weight-gradient path, the way the data passes get their deep
// levels, and the workspaces of both depend on the shape only, through
// these, so wtconv_workspace_size needs no device query.
constexpr int PLAN_SMEM = 232448;
constexpr int PLAN_SMS = 148;

size_t t1_bytes(const wtconv_desc* d) {
  return d->L >= 2 ? (((size_t)d->N * d->C * (d->H / 2) * (d->W / 2) * sizeof(float) + 15) / 16) * 16 : 0;
}

// Row-band planes with L >= 2 whose level-2 planes exceed the deep kernel's
// shared memory compute their levels >= 2 as a smaller layer: L - 1 levels on
// the level-1 LL planes (H/2 x W/2, fp32), no base branch.  Its output is the
// synthesis of levels >= 2 at level-1 resolution, i.e. t1.
bool deep_by_recursion(const wtconv_desc* d) {
  if (d->L < 2) return false;
  MainPlan M;
  if (!build_main_plan(M, d, PLAN_SMEM) || M.fused) return false;
  DeepPlan D;
  return !build_deep_plan(D, d, PLAN_SMEM);
}
wtconv_desc half_layer(const wtconv_desc* d) {
  wtconv_desc h = *d;
  h.H = d->H / 2;
  h.W = d->W / 2;
  h.L = d->L - 1;
  h.io = WTCONV_F32;
  return h;
}
size_t fold_bytes(const wtconv_desc* d) { return (size_t)d->C * main_wblk(d) * sizeof(float); }

// Workspace of the data pass over a folded block (run_folded): 16-byte
// header (status word), t1 of every plane (levels >= 2), and for the
// recursion the LL planes, the smaller layer's folded block and its own
// data-pass workspace.
size_t pass_ws_bytes(const wtconv_desc* d) {
  size_t b = 16 + t1_bytes(d);
  if (deep_by_recursion(d)) {
    const wtconv_desc h = half_layer(d);
    b += t1_bytes(d) + (fold_bytes(&h) + 15) / 16 * 16 + pass_ws_bytes(&h);
  }
  return b;
}

// Forward / backward-data workspace: the data pass's, then the folded
// weights of every channel.
size_t fwd_ws_bytes(const wtconv_desc* d) { return pass_ws_bytes(d) + fold_bytes(d); }

// Kernels one data pass over a folded block launches: [the LL planes, the
// smaller layer's block and its own pass], [deep kernel], output kernel.
int pass_launches(const wtconv_desc* d) {
  MainPlan M;
  if (!build_main_plan(M, d, PLAN_SMEM)) return 0;
  if (d->L < 2 || M.fused) return 1;
  if (!deep_by_recursion(d)) return 2;
  const wtconv_desc h = half_layer(d);
  const int inner = pass_launches(&h);
  return inner ? 3 + inner : 0;
}

wtconv_status check_desc(const wtconv_desc* d) {
  if (!d) return WTCONV_ERR_ARG;
  if (d->k < 1 || d->k > WTCONV_MAX_K || (d->k % 2) == 0) return WTCONV_ERR_ARG;
  if (d->L < 0 || d->L > WTCONV_MAX_LEVELS) return WTCONV_ERR_ARG;
  if (d->N <= 0 || d->C <= 0 || d->H <= 0 || d->W <= 0) return WTCONV_ERR_ARG;
  if (d->io != WTCONV_F32 && d->io != WTCONV_BF16) return WTCONV_ERR_ARG;
  const long long m = 1LL << d->L;
  const long long Hp = (d->H + m - 1) / m * m, Wp = (d->W + m - 1) / m * m;
  if (Hp * Wp > (1LL << 30) || (long long)d->N * d->C > (1LL << 30)) return WTCONV_ERR_ARG;
  return WTCONV_OK;
}

// Sides not multiples of 2^L: the passes run on zero-padded copies of the
// input planes (the padded descriptor) in the workspace; the output kernel
// stores only the image part of each output plane.
bool ragged(const wtconv_desc* d) {
  const int m = 1 << d->L;
  return (d->H % m) != 0 || (d->W % m) != 0;
}
wtconv_desc padded(const wtconv_desc* d) {
  wtconv_desc p = *d;
  const int m = 1 << d->L;
  p.H = (d->H + m - 1) / m * m;
  p.W = (d->W + m - 1) / m * m;
  return p;
}
size_t rup16(size_t b) { return (b + 15) / 16 * 16; }
// bytes of one padded activation tensor in the workspace
size_t act_bytes(const wtconv_desc* p) {
  return rup16((size_t)p->N * p->C * p->H * p->W * (p->io == WTCONV_BF16 ? 2 : 4));
}

// Copies the planes of `src` (d's sides) zero-padded into `dst` (p's sides).
wtconv_status launch_pad(const wtconv_desc* d, const wtconv_desc* p, const void* src, void* dst, cudaStream_t st) {
  const long long planes = (long long)d->N * d->C;
  const int per = p->H * p->W;
  const int cpp = (per + PADC - 1) / PADC;
  const int grid = (int)std::min<long long>(planes * cpp, 148LL * 8);
  const FDiv f = make_fdiv(p->W);
  if (d->io == WTCONV_F32)
    wtconv_pad_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(src), static_cast<float*>(dst), d->H,
                                                   d->W, p->H, p->W, f, planes, cpp);
  else
    wtconv_pad_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(src),
                                                           static_cast<__nv_bfloat16*>(dst), d->H, d->W, p->H, p->W,
                                                           f, planes, cpp);
  return cudaGetLastError() == cudaSuccess ? WTCONV_OK : WTCONV_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

wtconv_status check_params(const wtconv_desc* d, const float* w0, const float* b0, const float* s0,
                           const float* wl, const float* sl, bool need_b0) {
  if (!w0 || !s0 || (need_b0 && !b0)) return WTCONV_ERR_ARG;
  if (d->L > 0 && (!wl || !sl)) return WTCONV_ERR_ARG;
  if (!aligned4(w0) || !aligned4(s0) || (b0 && !aligned4(b0))) return WTCONV_ERR_ALIGN;
  if (d->L > 0 && (!aligned4(wl) || !aligned4(sl))) return WTCONV_ERR_ALIGN;
  return WTCONV_OK;
}

struct Device {
  int sms = 0, max_smem = 0;
};

// Launch set-up is cached so that a call costs little host time: the
// device's SM count and shared-memory limit per device, and per (kernel,
// device) the largest dynamic shared-memory size set so far (the attribute
// only ever grows) and the occupancy per (shared memory, threads).
constexpr int CACHE_DEVICES = 64;
std::mutex g_setup_mutex;
Device g_devices[CACHE_DEVICES];

struct KernelSetup {
  const void* func;
  int device, nthreads;
  size_t smem;
  int occ;
};
std::vector<KernelSetup> g_occ;
std::vector<std::pair<std::pair<const void*, int>, size_t>> g_smem_set;

wtconv_status query_device(Device& dev) {
  int id = 0;
  if (cudaGetDevice(&id) != cudaSuccess) return WTCONV_ERR_CUDA;
  if (id >= 0 && id < CACHE_DEVICES) {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_devices[id].sms > 0) {
      dev = g_devices[id];
      return WTCONV_OK;
    }
  }
  if (cudaDeviceGetAttribute(&dev.sms, cudaDevAttrMultiProcessorCount, id) != cudaSuccess) return WTCONV_ERR_CUDA;
  if (cudaDeviceGetAttribute(&dev.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, id) != cudaSuccess)
    return WTCONV_ERR_CUDA;
  if (id >= 0 && id < CACHE_DEVICES) {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    g_devices[id] = dev;
  }
  return WTCONV_OK;
}

// Tensor maps for the TMA tensor copies.  The encoder is a driver call,
// fetched once through the runtime (the library links no driver library).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// Map of an fp32 activation tensor viewed as [N][C][H][W] (innermost last)
// whose box is `box` = {columns, rows, channels, batch entries}; elements
// outside the tensor read as zeros.  Needs W % 4 == 0 (16-byte row stride)
// and a 16-byte aligned base.
bool encode_act_map(CUtensorMap* map, const void* base, const wtconv_desc* d, const cuuint32_t (&box)[4]) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)d->W, (cuuint64_t)d->H, (cuuint64_t)d->C, (cuuint64_t)d->N};
  const cuuint64_t strides[3] = {(cuuint64_t)d->W * 4, (cuuint64_t)d->H * d->W * 4,
                                 (cuuint64_t)d->C * d->H * d->W * 4};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Makes `kern` launchable with `smem` bytes of dynamic shared memory and
// returns its resident CTAs per SM for `nthreads` threads.
template <typename F>
wtconv_status prepare(F kern, size_t smem, int& occ, int nthreads = NT) {
  int id = 0;
  if (cudaGetDevice(&id) != cudaSuccess) return WTCONV_ERR_CUDA;
  const void* f = reinterpret_cast<const void*>(kern);
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  for (const KernelSetup& k : g_occ)
    if (k.func == f && k.device == id && k.nthreads == nthreads && k.smem == smem) {
      occ = k.occ;
      return occ < 1 ? WTCONV_ERR_UNSUPPORTED : WTCONV_OK;
    }
  size_t* set = nullptr;
  for (auto& e : g_smem_set)
    if (e.first.first == f && e.first.second == id) set = &e.second;
  if (!set) {
    g_smem_set.push_back({{f, id}, 0});
    set = &g_smem_set.back().second;
  }
  if (smem > *set) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return WTCONV_ERR_CUDA;
    *set = smem;
  }
  occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, nthreads, smem) != cudaSuccess)
    return WTCONV_ERR_CUDA;
  g_occ.push_back(KernelSetup{f, id, nthreads, smem, occ});
  if (occ < 1) return WTCONV_ERR_UNSUPPORTED;
  return WTCONV_OK;
}

// The folded weight block of every channel (reformulation (3)), one launch.
template <int K>
wtconv_status launch_fold(const wtconv_desc* d, const Device& dev, const float* w0, const float* b0, const float* s0,
                          const float* wl, const float* sl, int flip, float* wfold, cudaStream_t st) {
  const int kk4 = rup(d->k * d->k, 4), wblk = main_wblk(d);
  const int n = d->C * wblk;
  wtconv_fold_kernel<K><<<std::min((n + 255) / 256, dev.sms * 4), 256, 0, st>>>(d->C, d->L, kk4, wblk, w0, b0, s0,
                                                                                 wl, sl, flip, wfold);
  return cudaGetLastError() == cudaSuccess ? WTCONV_OK : WTCONV_ERR_CUDA;
}

// Deep kernel (row-band planes with L >= 2) and output kernel over folded
// weights `wfold`.
template <int K, typename IO>
wtconv_status launch_forward_t(const wtconv_desc* d, const Device& dev, const void* x, const float* wfold, void* y,
                               int* status, float* t1, const wtconv_desc* out, cudaStream_t st, const RawW& rw) {
  MainPlan M;
  if (!build_main_plan(M, d, dev.max_smem)) return WTCONV_ERR_UNSUPPORTED;
  if (out) {  // y is the image inside the padded planes x holds
    M.oH = out->H;
    M.oW = out->W;
    M.vec_out = (out->W % 4) == 0;
  }
  DeepPlan D;
  if (d->L >= 2 && !M.fused && build_deep_plan(D, d, dev.max_smem)) {  // else t1 came from the smaller layer
    // the deep kernel reads x with unchecked 4-wide loads: W is a multiple
    // of 2^L >= 4 for every descriptor that reaches here
    if (d->W % 4) return WTCONV_ERR_UNSUPPORTED;
    auto kd = wtconv_deep_kernel<K, IO>;
    const size_t smem = (size_t)D.smem_floats * 4;
    int occ = 0;
    wtconv_status e = prepare(kd, smem, occ, DEEP_NT);
    if (e != WTCONV_OK) return e;
    const int units = D.C * D.nbatch;
    kd<<<std::min(units, dev.sms * occ), DEEP_NT, smem, st>>>(D, static_cast<const IO*>(x), wfold, t1);
    if (cudaGetLastError() != cudaSuccess) return WTCONV_ERR_CUDA;
  }
  const size_t smem = (size_t)M.smem_floats * 4;
  int occ = 0;
  CUtensorMap xmap;
  std::memset(&xmap, 0, sizeof(xmap));
  if (M.direct) {
    const cuuint32_t box[4] = {(cuuint32_t)M.xf.ld, (cuuint32_t)M.xf.rows, 1, (cuuint32_t)M.PB};
    if (!encode_act_map(&xmap, x, d, box)) return WTCONV_ERR_CUDA;
  }
#define WT_MAIN(R3, FUSED, DIRECT)                                                                      \
  {                                                                                                     \
    auto km = wtconv_main_kernel<K, R3, IO, FUSED, DIRECT>;                                             \
    wtconv_status e = prepare(km, smem, occ, MAIN_NT);                                                  \
    if (e != WTCONV_OK) return e;                                                                       \
    km<<<std::min(M.units, dev.sms * occ), MAIN_NT, smem, st>>>(M, static_cast<const IO*>(x), t1, wfold, \
                                                                static_cast<IO*>(y), status, xmap, rw); \
  }
  if (M.fused) {
    if (M.R3 == 8) WT_MAIN(8, true, false) else WT_MAIN(4, true, false)
  } else if constexpr (std::is_same<IO, float>::value) {
    if (M.direct) {
      if (M.R3 == 8) WT_MAIN(8, false, true) else WT_MAIN(4, false, true)
    } else {
      if (M.R3 == 8) WT_MAIN(8, false, false) else WT_MAIN(4, false, false)
    }
  } else {
    if (M.R3 == 8) WT_MAIN(8, false, false) else WT_MAIN(4, false, false)
  }
#undef WT_MAIN
  return cudaGetLastError() == cudaSuccess ? WTCONV_OK : WTCONV_ERR_CUDA;
}

template <int K>
wtconv_status launch_forward_k(const wtconv_desc* d, const Device& dev, const void* x, const float* wfold, void* y,
                               int* status, float* t1, const wtconv_desc* out, cudaStream_t st,
                               const RawW& rw = RawW{nullptr, nullptr, nullptr, 0}) {
  if (d->io == WTCONV_F32) return launch_forward_t<K, float>(d, dev, x, wfold, y, status, t1, out, st, rw);
  return launch_forward_t<K, __nv_bfloat16>(d, dev, x, wfold, y, status, t1, out, st, rw);
}

// Level-0 fp32 planes whose output kernel takes the tensor-copy (DIRECT)
// path: their data passes scale the raw taps in the kernel (no fold launch).
bool direct_raw(const wtconv_desc* d) {
  if (d->L != 0 || d->io != WTCONV_F32) return false;
  MainPlan M;
  return build_main_plan(M, d, PLAN_SMEM) && M.direct;
}

// ---- level 0 on small planes: a few planes per warp (wtconv_small.cuh)

// Level-0 planes of at most 32x32 (at most 64 4x4 tiles).
bool small_planes(const wtconv_desc* d) { return d->L == 0 && d->W <= 32 && d->H <= 32; }

void build_small_plan(SmallPlan& S, const wtconv_desc* d) {
  S = SmallPlan{};
  S.N = d->N; S.C = d->C; S.H = d->H; S.W = d->W; S.K = d->k; S.r = d->k / 2;
  S.hw = d->H * d->W;
  S.TY = cdiv_h(d->H, 4);
  S.TX = cdiv_h(d->W, 4);
  S.T = S.TY * S.TX;
  S.PW = std::max(1, std::min(8, 32 / S.T));
  // the 4x4 tile reads rows 4 ty .. 4 ty + 3 + 2r and 16-byte groups of
  // columns up to 4 tx + 4 + 2r (rounded up to 4)
  S.ld = rup(4 * S.TX + 2 * S.r, 4);
  S.rows = 4 * S.TY + 2 * S.r;
  S.xs_pp = S.ld * S.rows;
  S.kk4 = rup(d->k * d->k, 4);
  S.tab_off = S.PW * S.xs_pp;  // the plane buffers, then the element table, then weights and biases
  S.w_off = rup(S.tab_off + S.PW * S.hw, 4);
  S.buf = rup(S.w_off + S.PW * (S.kk4 + 1), 4);
  S.wblk = main_wblk(d);
  S.f_w = make_fdiv(d->W);
  S.f_hw = make_fdiv(S.hw);
  S.f_C = make_fdiv(d->C);
}

// Forward (flip = 0) or backward-data (flip = 1) from the raw parameters
// (wfold null) or from a folded block.
template <int K, typename IO>
wtconv_status launch_small_t(const wtconv_desc* d, const Device& dev, const void* x, const float* wfold,
                             const float* w0, const float* b0, const float* s0, int flip, void* y, cudaStream_t st) {
  SmallPlan S;
  build_small_plan(S, d);
  const size_t smem = (size_t)(SMALL_NT / 32) * S.buf * sizeof(float);
  auto k = wtconv_small_kernel<K, IO>;
  int occ = 0;
  wtconv_status e = prepare(k, smem, occ, SMALL_NT);
  if (e != WTCONV_OK) return e;
  const long long warps = ((long long)d->N * d->C + S.PW - 1) / S.PW;
  const int grid = (int)std::min<long long>((warps + SMALL_NT / 32 - 1) / (SMALL_NT / 32), (long long)dev.sms * occ);
  k<<<grid, SMALL_NT, smem, st>>>(S, static_cast<const IO*>(x), wfold, w0, b0, s0, flip, static_cast<IO*>(y));
  return cudaGetLastError() == cudaSuccess ? WTCONV_OK : WTCONV_ERR_CUDA;
}

wtconv_status launch_small(const wtconv_desc* d, const void* x, const float* wfold, const float* w0,
                           const float* b0, const float* s0, int flip, void* y, cudaStream_t st) {
  Device dev;
  wtconv_status e = query_device(dev);
  if (e != WTCONV_OK) return e;
  const bool f32 = d->io == WTCONV_F32;
  switch (d->k) {
    case 1: return f32 ? launch_small_t<1, float>(d, dev, x, wfold, w0, b0, s0, flip, y, st)
                       : launch_small_t<1, __nv_bfloat16>(d, dev, x, wfold, w0, b0, s0, flip, y, st);
    case 3: return f32 ? launch_small_t<3, float>(d, dev, x, wfold, w0, b0, s0, flip, y, st)
                       : launch_small_t<3, __nv_bfloat16>(d, dev, x, wfold, w0, b0, s0, flip, y, st);
    case 5: return f32 ? launch_small_t<5, float>(d, dev, x, wfold, w0, b0, s0, flip, y, st)
                       : launch_small_t<5, __nv_bfloat16>(d, dev, x, wfold, w0, b0, s0, flip, y, st);
    default: return f32 ? launch_small_t<7, float>(d, dev, x, wfold, w0, b0, s0, flip, y, st)
                        : launch_small_t<7, __nv_bfloat16>(d, dev, x, wfold, w0, b0, s0, flip, y, st);
  }
}

// Folds the weights into `wfold` (flip = 1: the adjoint's block).
wtconv_status run_fold(const wtconv_desc* d, const float* w0, const float* b0, const float* s0, const float* wl,
                       const float* sl, int flip, float* wfold, cudaStream_t st) {
  Device dev;
  wtconv_status e = query_device(dev);
  if (e != WTCONV_OK) return e;
  switch (d->k) {
    case 1: return launch_fold<1>(d, dev, w0, b0, s0, wl, sl, flip, wfold, st);
    case 3: return launch_fold<3>(d, dev, w0, b0, s0, wl, sl, flip, wfold, st);
    case 5: return launch_fold<5>(d, dev, w0, b0, s0, wl, sl, flip, wfold, st);
    default: return launch_fold<7>(d, dev, w0, b0, s0, wl, sl, flip, wfold, st);
  }
}

// The data pass over a folded block.  ws: 16-byte header (status word)
// followed by t1 when L >= 2.  With `out`, x holds zero-padded planes and y
// receives only the out->H x out->W image of each.
wtconv_status run_folded(const wtconv_desc* d, const void* x, const float* wfold, void* y, void* ws, cudaStream_t st,
                         const wtconv_desc* out = nullptr, int* status_word = nullptr) {
  Device dev;
  wtconv_status e = query_device(dev);
  if (e != WTCONV_OK) return e;
  // the workspace layout (deep kernel or recursion) is planned for sm_100a's
  // shared memory per CTA
  if (dev.max_smem < PLAN_SMEM) return WTCONV_ERR_UNSUPPORTED;
  if (small_planes(d) && !out) return launch_small(d, x, wfold, nullptr, nullptr, nullptr, 0, y, st);
  // the smaller layer's kernels report to the caller's status word
  int* status = status_word ? status_word : static_cast<int*>(ws);
  float* t1 = reinterpret_cast<float*>(static_cast<char*>(ws) + 16);
  if (deep_by_recursion(d)) {
    // t1 = the smaller layer (levels 2..L as 1..L-1) on the LL planes
    const wtconv_desc h = half_layer(d);
    char* extra = static_cast<char*>(ws) + 16 + t1_bytes(d);
    float* ll = reinterpret_cast<float*>(extra);
    float* wf1 = reinterpret_cast<float*>(extra + t1_bytes(d));
    void* ws1 = extra + t1_bytes(d) + (fold_bytes(&h) + 15) / 16 * 16;
    const long long n = (long long)d->N * d->C * h.H * h.W;
    const int grid = (int)std::min<long long>((n + 255) / 256, (long long)dev.sms * 8);
    if (d->io == WTCONV_F32)
      wtconv_ll_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(x), ll, d->H, d->W, n);
    else
      wtconv_ll_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), ll, d->H, d->W,
                                                             n);
    const int kk4 = rup(d->k * d->k, 4), nw = d->C * main_wblk(&h);
    wtconv_shift_fold_kernel<<<std::min((nw + 255) / 256, dev.sms * 4), 256, 0, st>>>(
        wfold, wf1, d->C, kk4, main_wblk(d), main_wblk(&h), h.L);
    if (cudaGetLastError() != cudaSuccess) return WTCONV_ERR_CUDA;
    if ((e = run_folded(&h, ll, wf1, t1, ws1, st, nullptr, status)) != WTCONV_OK) return e;
  }
  switch (d->k) {
    case 1: return launch_forward_k<1>(d, dev, x, wfold, y, status, t1, out, st);
    case 3: return launch_forward_k<3>(d, dev, x, wfold, y, status, t1, out, st);
    case 5: return launch_forward_k<5>(d, dev, x, wfold, y, status, t1, out, st);
    default: return launch_forward_k<7>(d, dev, x, wfold, y, status, t1, out, st);
  }
}

// Forward (flip = 0) or backward-data (flip = 1): the weights are folded into
// the workspace after t1, then the data pass runs over them.
wtconv_status run_forward(const wtconv_desc* d, const void* x, const float* w0, const float* b0, const float* s0,
                          const float* wl, const float* sl, void* y, int flip, void* ws, cudaStream_t st,
                          const wtconv_desc* out = nullptr) {
  // level-0 small planes, and level-0 planes on the tensor-copy path, scale
  // W0 and b0 by s0 inside their one kernel
  if (small_planes(d) && !out) return launch_small(d, x, nullptr, w0, b0, s0, flip, y, st);
  if (direct_raw(d) && !out) {
    Device dev;
    wtconv_status e = query_device(dev);
    if (e != WTCONV_OK) return e;
    if (dev.max_smem < PLAN_SMEM) return WTCONV_ERR_UNSUPPORTED;  // planned for sm_100a's shared memory
    const RawW rw{w0, b0, s0, flip};
    int* status = static_cast<int*>(ws);
    switch (d->k) {
      case 1: return launch_forward_k<1>(d, dev, x, nullptr, y, status, nullptr, nullptr, st, rw);
      case 3: return launch_forward_k<3>(d, dev, x, nullptr, y, status, nullptr, nullptr, st, rw);
      case 5: return launch_forward_k<5>(d, dev, x, nullptr, y, status, nullptr, nullptr, st, rw);
      default: return launch_forward_k<7>(d, dev, x, nullptr, y, status, nullptr, nullptr, st, rw);
    }
  }
  float* wfold = reinterpret_cast<float*>(static_cast<char*>(ws) + pass_ws_bytes(d));
  wtconv_status e = run_fold(d, w0, b0, s0, wl, sl, flip, wfold, st);
  if (e != WTCONV_OK) return e;
  return run_folded(d, x, wfold, y, ws, st, out);
}

// Workspace: a 16-byte header whose first int is the device status word,
// then (weight gradients) the per-CTA partial sums.
constexpr size_t WS_HEADER = 16;



// ---- whole-plane weight-gradient plan

// Per-plane slab (floats): x padded and dy plain, and both pyramids.
int bw_slab(BwPlan& B) {
  const int r = B.r;
  int cur = 0;
  // dy's buffers: plain for the correlations alone, shifted like x's when
  // the fused backward also convolves them (dys)
  auto gbuf = [&](int h, int w, int nb) {
    return B.dys ? make_shifted(cur, h, w, r, {{4, 4}}, nb) : make_plain(cur, h, w, {{4, 4}}, nb);
  };
  B.xf = make_shifted(cur, B.H, B.W, r, {{4, 4}}, 1);
  B.gf = gbuf(B.H, B.W, 1);
  B.s1 = B.g1 = BufDesc{0, 0, 0, 0};
  for (int l = 0; l <= MAXL; ++l) B.sd[l] = B.gd[l] = BufDesc{0, 0, 0, 0};
  if (B.L >= 1) {
    B.s1 = make_shifted(cur, B.H1, B.W1, r, {{4, 4}}, 4);
    B.g1 = gbuf(B.H1, B.W1, 4);
  }
  for (int l = 2; l <= B.L; ++l) {
    B.sd[l] = make_shifted(cur, B.H >> l, B.W >> l, r, {{4, 4}}, 4);
    B.gd[l] = gbuf(B.H >> l, B.W >> l, 4);
  }
  return rup(cur, 4);
}

// Layout for PB planes per unit (and `wblk` floats of folded weights, for
// the fused backward); false when it needs more than max_smem.
bool bw_layout(BwPlan& B, int PB, int max_smem, int wblk = 0) {
  B.PB = PB;
  B.ps = bw_slab(B);
  const size_t plane_bytes = (size_t)B.H * B.W * B.io_bytes;
  B.bulk = plane_bytes % 16 == 0;
  B.raw_pp = B.bulk ? rup((int)((plane_bytes + 3) / 4), 4) : 0;
  int cur = 0;  // relative to the slot, which starts after the header
  B.raw_x = cur;
  cur += PB * B.raw_pp;
  B.raw_g = cur;
  cur += PB * B.raw_pp;
  B.w_off = cur;
  cur += rup(wblk, 4);
  const int base = cur;
  for (BufDesc* bd : {&B.xf, &B.gf, &B.s1, &B.g1}) bd->off += base;
  for (int l = 2; l <= B.L; ++l) {
    B.sd[l].off += base;
    B.gd[l].off += base;
  }
  B.red_off = base;
  const int need = std::max(base + PB * B.ps, base + BW_NT * (B.kk4 + 1) + BW_NT);
  B.smem_floats = MAIN_HEADER + rup(need, 4);
  return (size_t)B.smem_floats * 4 <= (size_t)max_smem;
}

// Branches and their threads: each of the 1 + 4L branches (base taps, then
// band s of level l) gets a range of threads sized to its tiles, filled
// greedily towards the branch with the most tiles per thread.
void bw_branches(BwPlan& B) {
  const int KK = B.K * B.K;
  B.nbr = 1 + 4 * B.L;
  int tiles[BW_MAXB], thr[BW_MAXB];
  for (int b = 0; b < B.nbr; ++b) {
    BwBranch& br = B.br[b];
    const BufDesc* a;
    const BufDesc* g;
    int h, w, s = 0;
    if (b == 0) {
      a = &B.xf;
      g = &B.gf;
      h = B.H;
      w = B.W;
    } else {
      const int l = 1 + (b - 1) / 4;
      s = (b - 1) % 4;
      a = l == 1 ? &B.s1 : &B.sd[l];
      g = l == 1 ? &B.g1 : &B.gd[l];
      h = B.H >> l;
      w = B.W >> l;
    }
    br.a_off = a->off + s * a->ld * a->rows;
    br.a_ld = a->ld;
    br.g_off = g->off + s * g->ld * g->rows + (B.dys ? B.r * g->ld + B.r : 0);  // element (0, 0)
    br.g_ld = g->ld;
    br.seg = KK * b;
    const int tx = cdiv_h(w, 4);
    tiles[b] = cdiv_h(h, 4) * tx * B.PB;
    br.f_tiles = make_fdiv(cdiv_h(h, 4) * tx);
    br.f_tx = make_fdiv(tx);
    thr[b] = 1;
  }
  for (int left = BW_NT - B.nbr; left > 0; --left) {
    int best = -1;
    long bestq = 1;
    for (int b = 0; b < B.nbr; ++b) {
      const long q = (tiles[b] + thr[b] - 1) / thr[b];
      if (q > bestq || (q == bestq && best >= 0 && tiles[b] > tiles[best])) {
        bestq = q;
        best = b;
      }
    }
    if (best < 0) break;  // every branch has one tile per thread at most
    ++thr[best];
  }
  int first = 0;
  for (int b = 0; b < B.nbr; ++b) {
    B.br[b].first = first;
    B.br[b].nthr = thr[b];
    first += thr[b];
  }
}

// Whole-plane plan: the most planes per unit (up to two tiles per thread,
// one at level 0) that fit two CTAs per SM, else one.  False when one plane
// does not fit; such shapes run on the row-band path.
// Fields of the weight-gradient plan that depend on the shape alone.
void bw_init(BwPlan& B, const wtconv_desc* d) {
  B = BwPlan{};
  B.N = d->N;
  B.C = d->C;
  B.H = d->H;
  B.W = d->W;
  B.K = d->k;
  B.r = d->k / 2;
  B.L = d->L;
  B.H1 = d->L >= 1 ? d->H / 2 : d->H;
  B.W1 = d->L >= 1 ? d->W / 2 : d->W;
  B.kk4 = rup(d->k * d->k, 4);
  B.V = d->k * d->k * (1 + 4 * d->L) + 1;
  B.io_bytes = io_bytes(d);
  B.vec_in = (d->W % 4) == 0;
  B.BH = d->L >= 2 ? 4 : (d->L == 1 ? 2 : 1);
}

// 4x4 tiles of every correlation branch of one plane.
int bw_tiles_per_plane(const wtconv_desc* d) {
  int per_plane = cdiv_h(d->H, 4) * cdiv_h(d->W, 4);
  for (int l = 1; l <= d->L; ++l) per_plane += 4 * cdiv_h(d->H >> l, 4) * cdiv_h(d->W >> l, 4);
  return per_plane;
}

bool build_bw_plan(BwPlan& B, const wtconv_desc* d, int max_smem) {
  bw_init(B, d);
  const int per_plane = bw_tiles_per_plane(d);
  // up to two tiles per thread; level 0 (one branch, short units) up to one,
  // which leaves each CTA several units whose copies overlap the compute
  const int tpt = d->L == 0 ? 1 : 2;
  const int pb0 = std::max(1, std::min(d->N, cdiv_h(tpt * BW_NT, per_plane)));
  bool ok = false;
  // two CTAs per SM if possible; else one (still faster than row bands,
  // which stage halo rows twice and hand the LL planes through HBM)
  for (const int budget : {(int)(SM_SMEM / 2 - 1024), max_smem}) {
    for (int pb = pb0; pb >= 1 && !ok; --pb) ok = bw_layout(B, pb, std::min(budget, max_smem));
    if (ok) break;
  }
  if (!ok) return false;  // the row-band path takes the shape
  B.f_sx = make_fdiv(cdiv_h(d->W, 4));
  B.f_spp = make_fdiv((d->H / B.BH) * cdiv_h(d->W, 4));
  bw_branches(B);
  return true;
}

// Level-0 fp32 weight gradients fed by tensor copies: two buffer sets of PB
// planes (x zero-padded, dy plain), the most planes per unit up to one tile
// per thread that fit two CTAs per SM, else one.  False when the shape does
// not qualify (L > 0, bf16, W % 4 != 0, a box side over 256) or one plane's
// two buffer sets do not fit.
bool build_bw_direct_plan(BwDirectPlan& B, const wtconv_desc* d, int max_smem) {
  B = BwDirectPlan{};
  if (d->L != 0 || d->io != WTCONV_F32 || (d->W % 4) != 0) return false;
  B.N = d->N;
  B.C = d->C;
  B.H = d->H;
  B.W = d->W;
  B.K = d->k;
  B.r = d->k / 2;
  B.kk4 = rup(d->k * d->k, 4);
  B.V = d->k * d->k + 1;
  B.xld = d->W + 8;
  B.gld = d->W;
  if (B.xld > 256) return false;
  // Lays out two buffer sets for units of pb planes of `rows` rows (whole
  // planes: rup(H, 4); row bands: TB) within `budget` bytes.
  auto fit = [&](int pb, int rows, int budget) {
    B.xrows = rows + 2 * B.r;
    B.grows = rows;
    if (B.xrows > 256) return false;
    B.xps = B.xld * B.xrows;
    B.gps = B.gld * B.grows;
    B.tiles_pp = (B.grows / 4) * (d->W / 4);
    // header: two mbarriers and the abort flag; buffers on 128-byte boundaries
    int cur = 32;
    for (int b = 0; b < 2; ++b) {
      B.xoff[b] = cur;
      cur += rup(pb * B.xps, 32);
      B.goff[b] = cur;
      cur += rup(pb * B.gps, 32);
    }
    B.red_off = B.xoff[0];
    const int need = std::max(cur, B.red_off + BW_NT * (B.kk4 + 1) + BW_NT);
    if ((size_t)rup(need, 4) * 4 > (size_t)std::min(budget, max_smem)) return false;
    B.PB = pb;
    B.smem_floats = rup(need, 4);
    B.f_tiles = make_fdiv(B.tiles_pp);
    B.f_tx = make_fdiv(d->W / 4);
    return true;
  };
  const int half = (int)(SM_SMEM / 2 - 1024);
  const int whole = rup(d->H, 4);
  const int pb0 = std::max(1, std::min({d->N, cdiv_h(BW_NT, (whole / 4) * (d->W / 4)), 256}));
  // whole planes at two CTAs per SM; else row bands at two CTAs per SM (the
  // largest band, a multiple of 4 rows dividing H, of at least 16 rows);
  // else whole planes at one CTA per SM
  B.nb = 1;
  B.TB = whole;
  for (int pb = pb0; pb >= 1; --pb)
    if (fit(pb, whole, half)) return true;
  if (d->H % 4 == 0)
    for (int nb = 2; d->H / nb >= 16; ++nb) {
      const int tb = d->H / nb;
      if (d->H % nb || tb % 4) continue;
      if (fit(1, tb, half)) {
        B.nb = nb;
        B.TB = tb;
        return true;
      }
    }
  for (int pb = pb0; pb >= 1; --pb)
    if (fit(pb, whole, max_smem)) return true;
  return false;
}

// True when one plane's whole weight-gradient working set fits one SM
// (either whole-plane kernel; both write one partial vector per CTA).
bool bwdw_whole_plane(const wtconv_desc* d) {
  BwDirectPlan D;
  if (build_bw_direct_plan(D, d, PLAN_SMEM)) return true;
  BwPlan B;
  return build_bw_plan(B, d, PLAN_SMEM);
}

// ---- fused backward (whole planes)

// Fills the output-kernel plan of the adjoint pass over B's staged dy: its
// input buffers are dy's (shifted), its Z planes reuse x's buffers (zb over
// xf, the deep levels' over s1), read only by the correlations that precede
// the adjoint phases.  False when those Z planes do not fit there.
bool bwd_adjoint_plan(const BwPlan& B, const wtconv_desc* d, const wtconv_desc* out, int wblk, MainPlan& M) {
  M = MainPlan{};
  M.N = d->N; M.C = d->C; M.H = d->H; M.W = d->W; M.K = d->k; M.r = d->k / 2; M.L = d->L;
  M.H1 = B.H1;
  M.W1 = B.W1;
  M.kk4 = B.kk4;
  M.io_bytes = B.io_bytes;
  M.TH = d->H;
  M.nbands = 1;
  M.PB = B.PB;
  M.R3 = 4;
  M.oH = out->H;
  M.oW = out->W;
  M.vec_out = (out->W % 4) == 0;
  M.wblk = wblk;
  M.w_off = B.w_off;
  M.units = 0;
  const int tx = cdiv_h(d->W, 4);
  M.tiles_pp = cdiv_h(d->H, 4) * tx;
  M.tiles = M.PB * M.tiles_pp;
  M.f_tx = make_fdiv(tx);
  M.f_tpp = make_fdiv(M.tiles_pp);
  M.f_C = make_fdiv(d->C);
  // the weight-gradient plan keeps one slab stride (B.ps) for all of a
  // plane's buffers; the output-kernel functions read each buffer's own
  M.xf = B.gf;
  M.xf.ps = B.ps;
  M.s1 = B.g1;
  M.s1.ps = B.ps;
  for (int l = 0; l <= MAXL; ++l) {
    M.sd[l] = B.gd[l];
    M.sd[l].ps = B.ps;
    M.zd[l] = BufDesc{0, 0, 0, 0};
  }
  M.t1 = BufDesc{0, 0, 0, 0};
  M.zb = BufDesc{0, 0, 0, 0};
  M.fused = d->L >= 2;
  if (d->L >= 1) {
    const int zrows = rup(M.H1, 4), zld = rup(M.W1, 4);
    if (4 * zrows * zld > B.xf.ld * B.xf.rows) return false;
    M.zb = BufDesc{B.xf.off, zld, zrows, B.ps};
    const int atx = cdiv_h(M.W1, 4), aty = cdiv_h(M.H1, 4);
    M.a_pp = 4 * aty * atx;
    M.f_app = make_fdiv(M.a_pp);
    M.f_abt = make_fdiv(aty * atx);
    M.f_atx = make_fdiv(atx);
  }
  int zcur = 0, first = 0;
  for (int l = 0; l <= MAXL + 1; ++l) M.dfirst[l] = 0;
  for (int l = 2; l <= d->L; ++l) {
    const int rows = rup(d->H >> l, 4), ld = rup(d->W >> l, 4);
    M.zd[l] = BufDesc{B.s1.off + zcur, ld, rows, B.ps};
    zcur += 4 * rows * ld;
    const int dtx = cdiv_h(d->W >> l, 4), tiles = cdiv_h(d->H >> l, 4) * dtx;
    M.f_dtiles[l] = make_fdiv(tiles);
    M.f_dtx[l] = make_fdiv(dtx);
    M.dfirst[l] = first;
    first += 4 * tiles;
  }
  if (d->L >= 2 && zcur > 4 * B.s1.ld * B.s1.rows) return false;
  if (d->L >= 2) M.dfirst[d->L + 1] = first;
  M.f_dper = make_fdiv(std::max(1, first));
  return true;
}

// The fused backward's plan: whole planes, two CTAs per SM (with fewer, the
// separate passes keep more warps busy), up to two correlation tiles per
// thread per unit.  False when the shape does not fit; wtconv_backward then
// runs the two passes.
bool build_bwd_plan(BwdPlan& Q, const wtconv_desc* d, const wtconv_desc* out, int max_smem) {
  // k = 7: 49 tap sums per thread on top of the conv tiles exceed the 128
  // registers of two 256-thread CTAs per SM; the separate passes run it
  if (d->k > 5) return false;
  BwPlan& B = Q.B;
  bw_init(B, d);
  B.dys = 1;
  const int wblk = main_wblk(d);
  const int tpt = d->L == 0 ? 1 : 2;
  const int pb0 = std::max(1, std::min(d->N, cdiv_h(tpt * BW_NT, bw_tiles_per_plane(d))));
  const int budget = std::min((int)(SM_SMEM / 2 - 1024), max_smem);
  for (int pb = pb0; pb >= 1; --pb) {
    if (!bw_layout(B, pb, budget, wblk)) continue;
    B.f_sx = make_fdiv(cdiv_h(d->W, 4));
    B.f_spp = make_fdiv((d->H / B.BH) * cdiv_h(d->W, 4));
    bw_branches(B);
    if (bwd_adjoint_plan(B, d, out, wblk, Q.M)) {
      const MainPlan& M = Q.M;
      Q.za_off = B.xf.off;
      Q.za_len = d->L >= 1 ? 4 * M.zb.ld * M.zb.rows : 0;
      Q.zb_off = B.s1.off;
      Q.zb_len = 0;
      for (int l = 2; l <= d->L; ++l) Q.zb_len += 4 * M.zd[l].ld * M.zd[l].rows;
      return true;
    }
  }
  return false;
}

bool bwd_fused(const wtconv_desc* d) {
  if (small_planes(d)) return false;  // backward-data on the small-plane kernel instead
  BwdPlan Q;
  return build_bwd_plan(Q, d, d, PLAN_SMEM);
}

// Workspace of the fused backward: header, the per-CTA partial sums (at
// most one CTA per plane), then the adjoint folded block.
size_t bwd_fused_ws_bytes(const wtconv_desc* d) {
  const size_t V = (size_t)d->k * d->k * (1 + 4 * d->L) + 1;
  return WS_HEADER + rup16((size_t)d->N * d->C * V * sizeof(float)) + fold_bytes(d);
}

// ---- row-band weight-gradient path

void band_layout(BandPlan& B, int TB) {
  const int r = B.r;
  const bool base = B.lvl <= 1, bands = B.lvl >= 1;
  B.TB = TB;
  B.nb = B.Hl / TB;
  B.FR = B.lvl == 0 ? TB : 2 * TB;
  const int nvb = (BW_CW + 2 * r + 3) / 4;
  B.a_ld = rup(std::max(B.W + 2 * r, rup(B.W, BW_CW) - BW_CW + 4 * nvb), 4);
  B.a_rows = B.FR + 2 * B.ha;
  if (base) B.a_rows = std::max(B.a_rows, rup(B.FR, BW_R) + B.ha + r);
  B.b_ld = rup(B.W, base ? BW_CW : 4);
  B.b_rows = base ? rup(B.FR, BW_R) : B.FR;
  if (bands) {
    const int nv1 = (B1_CW + 2 * r + 3) / 4;
    B.s_ld = rup(std::max(B.Wl + 2 * r, rup(B.Wl, B1_CW) - B1_CW + 4 * nv1), 4);
    B.s_rows = rup(TB, B1_R) + 2 * r;
    B.d_ld = rup(B.Wl, B1_CW);
    B.d_rows = rup(TB, B1_R);
  } else {
    B.s_ld = B.s_rows = B.d_ld = B.d_rows = 0;
  }
  int cur = 4;  // header: mbarrier (8 bytes), abort flag
  // raw copies of the next unit's rows (bulk copies), when rows are 16-byte aligned
  B.bulk = ((size_t)B.W * B.in_bytes) % 16 == 0;
  B.raw_a = cur;
  cur += B.bulk ? rup((int)(((size_t)(B.FR + 2 * B.ha) * B.W * B.in_bytes + 3) / 4), 4) : 0;
  B.raw_b = cur;
  cur += B.bulk ? rup((int)(((size_t)B.FR * B.W * B.in_bytes + 3) / 4), 4) : 0;
  B.a_off = cur;
  cur += rup(B.a_ld * B.a_rows, 4);
  B.b_off = cur;
  cur += rup(B.b_ld * B.b_rows, 4);
  B.s_off = cur;
  cur += rup(4 * B.s_ld * B.s_rows, 4);
  B.d_off = cur;
  cur += rup(4 * B.d_ld * B.d_rows, 4);
  B.red_off = cur;
  cur += rup((NT / 32) * B.kk4 + NT / 32, 4);
  B.smem_floats = cur;
  B.units = B.N * B.nb;
  B.f_nb = make_fdiv(B.nb);
  const int bx = cdiv_h(B.W, BW_CW);
  B.f_bx = make_fdiv(bx);
  B.f_bper = make_fdiv(base ? (rup(B.FR, BW_R) / BW_R) * bx : 1);
  const int sx = bands ? cdiv_h(B.Wl, B1_CW) : 1;
  B.f_sx = make_fdiv(sx);
  B.f_sper = make_fdiv(bands ? cdiv_h(TB, B1_R) * sx : 1);
  B.f_q4 = make_fdiv(cdiv_h(B.W, 4));
  B.f_wl = make_fdiv(B.Wl);
}

// Plan of the launch for level lvl (0 only when L = 0): the largest band
// height that divides the level grid and leaves room for two CTAs per SM
// (else one).  False when not even one row of the level grid fits.
bool build_band_plan(BandPlan& B, const wtconv_desc* d, int lvl) {
  B = BandPlan{};
  B.N = d->N;
  B.C = d->C;
  B.K = d->k;
  B.r = d->k / 2;
  B.kk4 = rup(d->k * d->k, 4);
  B.V = d->k * d->k * (1 + 4 * d->L) + 1;
  B.lvl = lvl;
  B.H = lvl == 0 ? d->H : d->H >> (lvl - 1);
  B.W = lvl == 0 ? d->W : d->W >> (lvl - 1);
  B.Hl = lvl == 0 ? B.H : B.H / 2;
  B.Wl = lvl == 0 ? B.W : B.W / 2;
  B.ha = lvl == 0 ? B.r : 2 * B.r;
  B.in_bytes = lvl <= 1 ? io_bytes(d) : 4;
  B.vec = (B.W % 4) == 0;
  B.write_ll = lvl >= 1 && lvl < d->L;
  B.seg = lvl >= 1 ? d->k * d->k * (1 + 4 * (lvl - 1)) : 0;
  for (const int budget : {PLAN_SMEM / 2, PLAN_SMEM}) {
    for (int TB = B.Hl; TB >= 1; --TB) {
      if (B.Hl % TB) continue;
      band_layout(B, TB);
      if ((size_t)B.smem_floats * 4 <= (size_t)budget) return true;
    }
  }
  return false;
}

int band_first_level(const wtconv_desc* d) { return d->L == 0 ? 0 : 1; }

// CTAs per channel of every band launch (the same for all, so that the
// partials keep the whole-plane layout), at most one per unit of the launch
// with the fewest units.  The count minimises the first level's time (it
// carries most of the work): rounds of resident CTAs (two per SM, the
// kernel's launch bound, or fewer where a level's shared memory allows
// fewer) times units per CTA plus one for the CTA's fixed costs (clearing
// its shared memory, the first copy, the reduction), the smallest count on
// a tie.  0 if a level does not fit.
int band_groups(const wtconv_desc* d) {
  int umin = 1 << 30, ufirst = 0, per_sm = 2;
  for (int lvl = band_first_level(d); lvl <= d->L; ++lvl) {
    BandPlan B;
    if (!build_band_plan(B, d, lvl)) return 0;
    umin = std::min(umin, B.units);
    if (lvl == band_first_level(d)) ufirst = B.units;
    per_sm = std::min(per_sm, (int)(SM_SMEM / ((size_t)B.smem_floats * 4 + 1024)));
  }
  const long slots = (long)std::max(1, per_sm) * PLAN_SMS;
  int best = 1;
  long best_cost = -1;
  for (int G = 1; G <= umin; ++G) {
    const long rounds = ((long)d->C * G + slots - 1) / slots;
    const long cost = rounds * ((ufirst + G - 1) / G + 1);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = G;
    }
  }
  return best;
}

// Floats of the raw LL planes of x and dy that level l (1 <= l < L) hands
// to level l + 1.
size_t band_ll_floats(const wtconv_desc* d) {
  size_t f = 0;
  for (int l = 1; l < d->L; ++l) f += 2 * (size_t)d->N * d->C * (size_t)(d->H >> l) * (d->W >> l);
  return f;
}

size_t band_part_bytes(const wtconv_desc* d, int groups) {
  const size_t V = (size_t)d->k * d->k * (1 + 4 * d->L) + 1;
  return (((size_t)groups * d->C * V * sizeof(float)) + 15) / 16 * 16;
}

size_t bwdw_ws_bytes(const wtconv_desc* d) {
  const size_t V = (size_t)d->k * d->k * (1 + 4 * d->L) + 1;
  if (bwdw_whole_plane(d)) return WS_HEADER + (size_t)d->N * d->C * V * sizeof(float);
  const int G = band_groups(d);
  if (G == 0) return WS_HEADER;  // unsupported; the call reports it
  return WS_HEADER + band_part_bytes(d, G) + band_ll_floats(d) * sizeof(float);
}

template <int K>
wtconv_status launch_finalize(const wtconv_desc* d, int groups, const float* part, const float* w0, const float* b0,
                              const float* s0, const float* wl, const float* sl, float* dw0, float* db0, float* ds0,
                              float* dwl, float* dsl, cudaStream_t st) {
  const FinalizeArgs F{d->C, d->L, d->k * d->k * (1 + 4 * d->L) + 1, groups};
  const size_t fsmem = ((size_t)F.V + (size_t)(1 + 4 * d->L) * d->k * d->k) * sizeof(float);
  auto fin = wtconv_bwdw_finalize<K>;
  int occ = 0;
  if (fsmem > 48 * 1024) {
    const wtconv_status e = prepare(fin, fsmem, occ, 256);
    if (e != WTCONV_OK) return e;
  }
  fin<<<F.C, 256, fsmem, st>>>(F, part, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl);
  return cudaGetLastError() == cudaSuccess ? WTCONV_OK : WTCONV_ERR_CUDA;
}

// Planes per CTA for `units_pb` planes per unit on `slots` resident CTAs:
// fewest sequential units per CTA slot, counting one more unit per CTA for
// its fixed costs (clearing its shared memory, the first copy that nothing
// overlaps, the final reduction and partial write); ties broken towards
// longer CTAs (fewer partial sums); a plane in `bands` row bands is that many
// units.  0 when no choice has at most max_groups CTAs per channel.
int planes_per_cta(int N, int C, int units_pb, int slots, int max_groups, int bands = 1) {
  long best = -1;
  int ppc = 0;
  for (int q = units_pb; q < N + units_pb; q += units_pb) {
    const int p = std::min(q, N);
    const int groups = (N + p - 1) / p;
    if (groups > max_groups) continue;
    const long ctas = (long)C * groups;
    const long cost = ((ctas + slots - 1) / slots) * ((long)(p + units_pb - 1) / units_pb * bands + 1);
    if (best < 0 || cost <= best) {
      best = cost;
      ppc = p;
    }
    if (p == N) break;
  }
  return ppc;
}

template <int K, int LC, typename IO>
wtconv_status launch_bwdw_t(BwPlan& B, const Device& dev, const wtconv_desc* d, const void* x, const void* dy,
                            const float* w0, const float* b0, const float* s0, const float* wl, const float* sl,
                            float* dw0, float* db0, float* ds0, float* dwl, float* dsl, float* part, int* status,
                            cudaStream_t st, int max_groups) {
  auto kern = wtconv_bwdw_kernel<K, LC, IO>;
  const size_t smem = (size_t)B.smem_floats * 4;
  int occ = 0;
  wtconv_status e = prepare(kern, smem, occ, BW_NT);
  if (e != WTCONV_OK) return e;
  B.ppc = planes_per_cta(B.N, B.C, B.PB, dev.sms * occ, max_groups);
  if (B.ppc == 0) return WTCONV_ERR_SCRATCH_LIMIT;
  B.ngroups = (B.N + B.ppc - 1) / B.ppc;
  kern<<<B.C * B.ngroups, BW_NT, smem, st>>>(B, static_cast<const IO*>(x), static_cast<const IO*>(dy), part, status);
  if (cudaGetLastError() != cudaSuccess) return WTCONV_ERR_CUDA;
  return launch_finalize<K>(d, B.ngroups, part, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, st);
}

template <int K>
wtconv_status launch_bwdw_k(BwPlan& B, const Device& dev, const wtconv_desc* d, const void* x, const void* dy,
                            const float* w0, const float* b0, const float* s0, const float* wl, const float* sl,
                            float* dw0, float* db0, float* ds0, float* dwl, float* dsl, float* part, int* status,
                            cudaStream_t st, int max_groups) {
#define WT_BW(LC, IO) \
  launch_bwdw_t<K, LC, IO>(B, dev, d, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, status, st, max_groups)
  const int lc = d->L >= 2 ? 2 : d->L;
  if (d->io == WTCONV_F32) return lc == 2 ? WT_BW(2, float) : lc == 1 ? WT_BW(1, float) : WT_BW(0, float);
  return lc == 2 ? WT_BW(2, __nv_bfloat16) : lc == 1 ? WT_BW(1, __nv_bfloat16) : WT_BW(0, __nv_bfloat16);
#undef WT_BW
}

template <int K>
wtconv_status launch_bw_direct(BwDirectPlan& B, const Device& dev, const wtconv_desc* d, const void* x,
                               const void* dy, const float* w0, const float* b0, const float* s0, float* dw0,
                               float* db0, float* ds0, float* part, int* status, cudaStream_t st, int max_groups) {
  auto kern = wtconv_bwdw_direct_kernel<K>;
  const size_t smem = (size_t)B.smem_floats * 4;
  int occ = 0;
  wtconv_status e = prepare(kern, smem, occ, BW_NT);
  if (e != WTCONV_OK) return e;
  B.ppc = planes_per_cta(B.N, B.C, B.PB, dev.sms * occ, max_groups, B.nb);
  if (B.ppc == 0) return WTCONV_ERR_SCRATCH_LIMIT;
  B.ngroups = (B.N + B.ppc - 1) / B.ppc;
  CUtensorMap xmap;
  const cuuint32_t box[4] = {(cuuint32_t)B.xld, (cuuint32_t)B.xrows, 1, (cuuint32_t)B.PB};
  if (!encode_act_map(&xmap, x, d, box)) return WTCONV_ERR_CUDA;
  kern<<<B.C * B.ngroups, BW_NT, smem, st>>>(B, static_cast<const float*>(dy), part, status, xmap);
  if (cudaGetLastError() != cudaSuccess) return WTCONV_ERR_CUDA;
  return launch_finalize<K>(d, B.ngroups, part, w0, b0, s0, nullptr, nullptr, dw0, db0, ds0, nullptr, nullptr, st);
}

// Runs the whole-plane weight-gradient kernels with the per-CTA partial sums
// at `part` and at most `max_groups` CTAs per channel (the partials then
// fill max_groups * C * V floats).
wtconv_status run_bwdw_part(const wtconv_desc* d, const void* x, const void* dy, const float* w0, const float* b0,
                            const float* s0, const float* wl, const float* sl, float* dw0, float* db0, float* ds0,
                            float* dwl, float* dsl, float* part, int* status, int max_groups, cudaStream_t st) {
  Device dev;
  wtconv_status e = query_device(dev);
  if (e != WTCONV_OK) return e;
  if (dev.max_smem < PLAN_SMEM) return WTCONV_ERR_UNSUPPORTED;
  BwDirectPlan D;
  if (build_bw_direct_plan(D, d, dev.max_smem)) {
    switch (d->k) {
      case 1: return launch_bw_direct<1>(D, dev, d, x, dy, w0, b0, s0, dw0, db0, ds0, part, status, st, max_groups);
      case 3: return launch_bw_direct<3>(D, dev, d, x, dy, w0, b0, s0, dw0, db0, ds0, part, status, st, max_groups);
      case 5: return launch_bw_direct<5>(D, dev, d, x, dy, w0, b0, s0, dw0, db0, ds0, part, status, st, max_groups);
      default: return launch_bw_direct<7>(D, dev, d, x, dy, w0, b0, s0, dw0, db0, ds0, part, status, st, max_groups);
    }
  }
  BwPlan B;
  if (!build_bw_plan(B, d, dev.max_smem)) return WTCONV_ERR_UNSUPPORTED;
  switch (d->k) {
    case 1:
      return launch_bwdw_k<1>(B, dev, d, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, status, st,
                              max_groups);
    case 3:
      return launch_bwdw_k<3>(B, dev, d, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, status, st,
                              max_groups);
    case 5:
      return launch_bwdw_k<5>(B, dev, d, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, status, st,
                              max_groups);
    default:
      return launch_bwdw_k<7>(B, dev, d, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, status, st,
                              max_groups);
  }
}

template <int K, int LC, typename IO>
wtconv_status launch_bwd_fused_t(BwdPlan& Q, const Device& dev, const wtconv_desc* d, const void* x, const void* dy,
                                 const float* wfold, void* dx, const float* w0, const float* b0, const float* s0,
                                 const float* wl, const float* sl, float* dw0, float* db0, float* ds0, float* dwl,
                                 float* dsl, float* part, int* status, cudaStream_t st) {
  auto kern = wtconv_bwd_fused_kernel<K, LC, IO>;
  const size_t smem = (size_t)Q.B.smem_floats * 4;
  int occ = 0;
  wtconv_status e = prepare(kern, smem, occ, BW_NT);
  if (e != WTCONV_OK) return e;
  Q.B.ppc = planes_per_cta(Q.B.N, Q.B.C, Q.B.PB, dev.sms * occ, Q.B.N);
  if (Q.B.ppc == 0) return WTCONV_ERR_UNSUPPORTED;
  Q.B.ngroups = (Q.B.N + Q.B.ppc - 1) / Q.B.ppc;
  kern<<<Q.B.C * Q.B.ngroups, BW_NT, smem, st>>>(Q, static_cast<const IO*>(x), static_cast<const IO*>(dy), wfold,
                                                 static_cast<IO*>(dx), part, status);
  if (cudaGetLastError() != cudaSuccess) return WTCONV_ERR_CUDA;
  return launch_finalize<K>(d, Q.B.ngroups, part, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, st);
}

// Both backward passes as one fused pass over whole planes (the plan must
// exist: bwd_fused(d)).  ws: header, partial sums, adjoint folded block.
// With `out`, x and dy hold zero-padded planes and dx receives only the
// out->H x out->W image of each.
wtconv_status run_bwd_fused(const wtconv_desc* d, const wtconv_desc* out, const void* x, const void* dy,
                            const float* w0, const float* b0, const float* s0, const float* wl, const float* sl,
                            void* dx, float* dw0, float* db0, float* ds0, float* dwl, float* dsl, void* ws,
                            cudaStream_t st) {
  Device dev;
  wtconv_status e = query_device(dev);
  if (e != WTCONV_OK) return e;
  if (dev.max_smem < PLAN_SMEM) return WTCONV_ERR_UNSUPPORTED;
  BwdPlan Q;
  if (!build_bwd_plan(Q, d, out, dev.max_smem)) return WTCONV_ERR_UNSUPPORTED;
  const size_t V = (size_t)d->k * d->k * (1 + 4 * d->L) + 1;
  int* status = static_cast<int*>(ws);
  float* part = reinterpret_cast<float*>(static_cast<char*>(ws) + WS_HEADER);
  float* wfold =
      reinterpret_cast<float*>(static_cast<char*>(ws) + WS_HEADER + rup16((size_t)d->N * d->C * V * sizeof(float)));
  if ((e = run_fold(d, w0, nullptr, s0, wl, sl, 1, wfold, st)) != WTCONV_OK) return e;
  const int lc = d->L >= 2 ? 2 : d->L;
#define WT_BF(KK, LC, IO)                                                                                      \
  return launch_bwd_fused_t<KK, LC, IO>(Q, dev, d, x, dy, wfold, dx, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, \
                                        part, status, st)
#define WT_BF_K(KK)                                                                   \
  if (d->io == WTCONV_F32) {                                                          \
    if (lc == 2) WT_BF(KK, 2, float);                                                 \
    if (lc == 1) WT_BF(KK, 1, float);                                                 \
    WT_BF(KK, 0, float);                                                              \
  } else {                                                                            \
    if (lc == 2) WT_BF(KK, 2, __nv_bfloat16);                                         \
    if (lc == 1) WT_BF(KK, 1, __nv_bfloat16);                                         \
    WT_BF(KK, 0, __nv_bfloat16);                                                      \
  }
  switch (d->k) {
    case 1: WT_BF_K(1)
    case 3: WT_BF_K(3)
    default: WT_BF_K(5)
  }
#undef WT_BF_K
#undef WT_BF
}

template <int K, typename IN>
wtconv_status launch_band_level(const BandPlan& B, const void* a, const void* b, float* llx, float* lld, float* part,
                                int* status, cudaStream_t st) {
  auto kern = wtconv_bwband_kernel<K, IN>;
  const size_t smem = (size_t)B.smem_floats * 4;
  int occ = 0;
  wtconv_status e = prepare(kern, smem, occ);
  if (e != WTCONV_OK) return e;
  kern<<<B.C * B.ngroups, NT, smem, st>>>(B, static_cast<const IN*>(a), static_cast<const IN*>(b), llx, lld, part,
                                          status);
  return cudaGetLastError() == cudaSuccess ? WTCONV_OK : WTCONV_ERR_CUDA;
}

// Row-band path: one launch per level (the first on x and dy, the others on
// the raw LL planes the level above wrote to `ll`), then the fixed-order
// finalize over `groups` partial vectors per channel.
template <int K>
wtconv_status run_band_k(const wtconv_desc* d, const void* x, const void* dy, const float* w0, const float* b0,
                         const float* s0, const float* wl, const float* sl, float* dw0, float* db0, float* ds0,
                         float* dwl, float* dsl, float* part, float* ll, int groups, int* status,
                         cudaStream_t st) {
  const float* prevx = nullptr;
  const float* prevd = nullptr;
  size_t off = 0;
  for (int lvl = band_first_level(d); lvl <= d->L; ++lvl) {
    BandPlan B;
    if (!build_band_plan(B, d, lvl)) return WTCONV_ERR_UNSUPPORTED;
    B.ngroups = groups;
    float* llx = nullptr;
    float* lld = nullptr;
    if (B.write_ll) {
      const size_t n = (size_t)d->N * d->C * B.Hl * B.Wl;
      llx = ll + off;
      lld = ll + off + n;
      off += 2 * n;
    }
    wtconv_status e;
    if (lvl <= 1)
      e = d->io == WTCONV_F32 ? launch_band_level<K, float>(B, x, dy, llx, lld, part, status, st)
                              : launch_band_level<K, __nv_bfloat16>(B, x, dy, llx, lld, part, status, st);
    else
      e = launch_band_level<K, float>(B, prevx, prevd, llx, lld, part, status, st);
    if (e != WTCONV_OK) return e;
    prevx = llx;
    prevd = lld;
  }
  return launch_finalize<K>(d, groups, part, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, st);
}

wtconv_status run_band(const wtconv_desc* d, const void* x, const void* dy, const float* w0, const float* b0,
                       const float* s0, const float* wl, const float* sl, float* dw0, float* db0, float* ds0,
                       float* dwl, float* dsl, float* part, float* ll, int groups, int* status,
                       cudaStream_t st) {
  Device dev;
  wtconv_status e = query_device(dev);
  if (e != WTCONV_OK) return e;
  if (dev.max_smem < PLAN_SMEM) return WTCONV_ERR_UNSUPPORTED;
  switch (d->k) {
    case 1:
      return run_band_k<1>(d, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, ll, groups, status, st);
    case 3:
      return run_band_k<3>(d, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, ll, groups, status, st);
    case 5:
      return run_band_k<5>(d, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, ll, groups, status, st);
    default:
      return run_band_k<7>(d, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, ll, groups, status, st);
  }
}

// Weight gradients with the workspace `ws` laid out as wtconv_workspace_size
// sizes it (header, partial sums, and the LL planes of the row-band path).
wtconv_status run_bwdw(const wtconv_desc* d, const void* x, const void* dy, const float* w0, const float* b0,
                       const float* s0, const float* wl, const float* sl, float* dw0, float* db0, float* ds0,
                       float* dwl, float* dsl, void* ws, cudaStream_t st) {
  int* status = static_cast<int*>(ws);
  float* part = reinterpret_cast<float*>(static_cast<char*>(ws) + WS_HEADER);
  if (bwdw_whole_plane(d))
    return run_bwdw_part(d, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, status, d->N, st);
  const int G = band_groups(d);
  if (G == 0) return WTCONV_ERR_UNSUPPORTED;
  float* ll = reinterpret_cast<float*>(static_cast<char*>(ws) + WS_HEADER + band_part_bytes(d, G));
  return run_band(d, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, ll, G, status, st);
}

wtconv_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (need == 0) return WTCONV_OK;
  if (!ws || ws_bytes < need) return WTCONV_ERR_WORKSPACE;
  if (!aligned16(ws)) return WTCONV_ERR_ALIGN;
  return WTCONV_OK;
}

wtconv_status check_grad_outputs(const wtconv_desc* d, const float* dw0, const float* db0, const float* ds0,
                                 const float* dwl, const float* dsl) {
  if (!dw0 || !db0 || !ds0) return WTCONV_ERR_ARG;
  if (d->L > 0 && (!dwl || !dsl)) return WTCONV_ERR_ARG;
  if (!aligned4(dw0) || !aligned4(db0) || !aligned4(ds0)) return WTCONV_ERR_ALIGN;
  if (d->L > 0 && (!aligned4(dwl) || !aligned4(dsl))) return WTCONV_ERR_ALIGN;
  return WTCONV_OK;
}

}  // namespace
}  // namespace wt

using namespace wt;

namespace {
// workspace of `op` for sides that are multiples of 2^L
size_t op_ws(const wtconv_desc* desc, int op) {
  switch (op) {
    case WTCONV_OP_FORWARD:
    case WTCONV_OP_BACKWARD_DATA:
      return fwd_ws_bytes(desc);
    case WTCONV_OP_BACKWARD_WEIGHT:
      return bwdw_ws_bytes(desc);
    case WTCONV_OP_BACKWARD:
      return std::max({bwdw_ws_bytes(desc), fwd_ws_bytes(desc), bwd_fused(desc) ? bwd_fused_ws_bytes(desc) : 0});
    case WTCONV_OP_FORWARD_FOLDED:
      return pass_ws_bytes(desc);
    default:
      return 0;
  }
}

// padded input planes a ragged call of `op` keeps in its workspace (x or
// dy; both for the weight gradients and the fused backward); outputs are
// written straight into the caller's unpadded tensors
int op_acts(int op) { return (op == WTCONV_OP_BACKWARD || op == WTCONV_OP_BACKWARD_WEIGHT) ? 2 : 1; }

// Ragged shapes: the workspace of the padded shape, then the padded
// activations, each 16-byte aligned.  Returns the i-th one.
void* act_slot(const wtconv_desc* p, int op, void* ws, int i) {
  return static_cast<char*>(ws) + rup16(op_ws(p, op)) + (size_t)i * act_bytes(p);
}
}  // namespace

extern "C" {

size_t wtconv_workspace_size(const wtconv_desc* desc, int op) {
  if (check_desc(desc) != WTCONV_OK || op < 0 || op > WTCONV_OP_FORWARD_FOLDED) return 0;
  if (!ragged(desc)) return op_ws(desc, op);
  const wtconv_desc p = padded(desc);
  return rup16(op_ws(&p, op)) + (size_t)op_acts(op) * act_bytes(&p);
}

size_t wtconv_folded_size(const wtconv_desc* desc) {
  if (check_desc(desc) != WTCONV_OK) return 0;
  return (size_t)desc->C * main_wblk(desc) * sizeof(float);
}

wtconv_status wtconv_fold_weights(const wtconv_desc* desc, const float* w0, const float* b0, const float* s0,
                                  const float* wl, const float* sl, int adjoint, void* folded,
                                  size_t folded_bytes, void* stream) {
  wtconv_status e = check_desc(desc);
  if (e != WTCONV_OK) return e;
  if (adjoint != 0 && adjoint != 1) return WTCONV_ERR_ARG;
  if ((e = check_params(desc, w0, adjoint ? nullptr : b0, s0, wl, sl, !adjoint)) != WTCONV_OK) return e;
  if (!folded) return WTCONV_ERR_ARG;
  if (!aligned16(folded)) return WTCONV_ERR_ALIGN;
  if (folded_bytes < wtconv_folded_size(desc)) return WTCONV_ERR_WORKSPACE;
  return run_fold(desc, w0, b0, s0, wl, sl, adjoint, static_cast<float*>(folded), static_cast<cudaStream_t>(stream));
}

wtconv_status wtconv_forward_folded(const wtconv_desc* desc, const void* x, const void* folded, void* y, void* ws,
                                    size_t ws_bytes, void* stream) {
  wtconv_status e = check_desc(desc);
  if (e != WTCONV_OK) return e;
  if (!x || !y || !folded) return WTCONV_ERR_ARG;
  if (!aligned16(x) || !aligned16(y) || !aligned16(folded)) return WTCONV_ERR_ALIGN;
  if ((e = check_ws(ws, ws_bytes, wtconv_workspace_size(desc, WTCONV_OP_FORWARD_FOLDED))) != WTCONV_OK) return e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const float* wf = static_cast<const float*>(folded);
  if (!ragged(desc)) return run_folded(desc, x, wf, y, ws, st);
  const wtconv_desc p = padded(desc);
  void* xp = act_slot(&p, WTCONV_OP_FORWARD_FOLDED, ws, 0);
  if ((e = launch_pad(desc, &p, x, xp, st)) != WTCONV_OK) return e;
  return run_folded(&p, xp, wf, y, ws, st, desc);
}

wtconv_status wtconv_forward(const wtconv_desc* desc, const void* x, const float* w0, const float* b0,
                             const float* s0, const float* wl, const float* sl, void* y, void* ws,
                             size_t ws_bytes, void* stream) {
  wtconv_status e = check_desc(desc);
  if (e != WTCONV_OK) return e;
  if (!x || !y) return WTCONV_ERR_ARG;
  if ((e = check_params(desc, w0, b0, s0, wl, sl, true)) != WTCONV_OK) return e;
  if (!aligned16(x) || !aligned16(y)) return WTCONV_ERR_ALIGN;
  if ((e = check_ws(ws, ws_bytes, wtconv_workspace_size(desc, WTCONV_OP_FORWARD))) != WTCONV_OK) return e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!ragged(desc)) return run_forward(desc, x, w0, b0, s0, wl, sl, y, 0, ws, st);
  const wtconv_desc p = padded(desc);
  void* xp = act_slot(&p, WTCONV_OP_FORWARD, ws, 0);
  if ((e = launch_pad(desc, &p, x, xp, st)) != WTCONV_OK) return e;
  return run_forward(&p, xp, w0, b0, s0, wl, sl, y, 0, ws, st, desc);
}

wtconv_status wtconv_backward_data(const wtconv_desc* desc, const void* dy, const float* w0, const float* s0,
                                   const float* wl, const float* sl, void* dx, void* ws, size_t ws_bytes,
                                   void* stream) {
  wtconv_status e = check_desc(desc);
  if (e != WTCONV_OK) return e;
  if (!dy || !dx) return WTCONV_ERR_ARG;
  if ((e = check_params(desc, w0, nullptr, s0, wl, sl, false)) != WTCONV_OK) return e;
  if (!aligned16(dy) || !aligned16(dx)) return WTCONV_ERR_ALIGN;
  if ((e = check_ws(ws, ws_bytes, wtconv_workspace_size(desc, WTCONV_OP_BACKWARD_DATA))) != WTCONV_OK) return e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!ragged(desc)) return run_forward(desc, dy, w0, nullptr, s0, wl, sl, dx, 1, ws, st);
  const wtconv_desc p = padded(desc);
  void* dyp = act_slot(&p, WTCONV_OP_BACKWARD_DATA, ws, 0);
  if ((e = launch_pad(desc, &p, dy, dyp, st)) != WTCONV_OK) return e;
  return run_forward(&p, dyp, w0, nullptr, s0, wl, sl, dx, 1, ws, st, desc);
}

wtconv_status wtconv_backward_weight(const wtconv_desc* desc, const void* x, const void* dy, const float* w0,
                                     const float* b0, const float* s0, const float* wl, const float* sl,
                                     float* dw0, float* db0, float* ds0, float* dwl, float* dsl, void* ws,
                                     size_t ws_bytes, void* stream) {
  wtconv_status e = check_desc(desc);
  if (e != WTCONV_OK) return e;
  if (!x || !dy) return WTCONV_ERR_ARG;
  if ((e = check_params(desc, w0, b0, s0, wl, sl, true)) != WTCONV_OK) return e;
  if ((e = check_grad_outputs(desc, dw0, db0, ds0, dwl, dsl)) != WTCONV_OK) return e;
  if (!aligned16(x) || !aligned16(dy)) return WTCONV_ERR_ALIGN;
  if ((e = check_ws(ws, ws_bytes, wtconv_workspace_size(desc, WTCONV_OP_BACKWARD_WEIGHT))) != WTCONV_OK) return e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!ragged(desc)) return run_bwdw(desc, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, ws, st);
  const wtconv_desc p = padded(desc);
  void* xp = act_slot(&p, WTCONV_OP_BACKWARD_WEIGHT, ws, 0);
  void* dyp = act_slot(&p, WTCONV_OP_BACKWARD_WEIGHT, ws, 1);
  if ((e = launch_pad(desc, &p, x, xp, st)) != WTCONV_OK) return e;
  if ((e = launch_pad(desc, &p, dy, dyp, st)) != WTCONV_OK) return e;
  return run_bwdw(&p, xp, dyp, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, ws, st);
}

wtconv_status wtconv_backward(const wtconv_desc* desc, const void* x, const void* dy, const float* w0,
                              const float* b0, const float* s0, const float* wl, const float* sl, void* dx,
                              float* dw0, float* db0, float* ds0, float* dwl, float* dsl, void* ws,
                              size_t ws_bytes, void* stream) {
  wtconv_status e = check_desc(desc);
  if (e != WTCONV_OK) return e;
  if (!x || !dy || !dx) return WTCONV_ERR_ARG;
  if ((e = check_params(desc, w0, b0, s0, wl, sl, true)) != WTCONV_OK) return e;
  if ((e = check_grad_outputs(desc, dw0, db0, ds0, dwl, dsl)) != WTCONV_OK) return e;
  if (!aligned16(x) || !aligned16(dy) || !aligned16(dx)) return WTCONV_ERR_ALIGN;
  if ((e = check_ws(ws, ws_bytes, wtconv_workspace_size(desc, WTCONV_OP_BACKWARD))) != WTCONV_OK) return e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!ragged(desc)) {
    if (bwd_fused(desc))
      return run_bwd_fused(desc, desc, x, dy, w0, b0, s0, wl, sl, dx, dw0, db0, ds0, dwl, dsl, ws, st);
    e = run_forward(desc, dy, w0, nullptr, s0, wl, sl, dx, 1, ws, st);
    if (e != WTCONV_OK) return e;
    return run_bwdw(desc, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, ws, st);
  }
  const wtconv_desc p = padded(desc);
  void* xp = act_slot(&p, WTCONV_OP_BACKWARD, ws, 0);
  void* dyp = act_slot(&p, WTCONV_OP_BACKWARD, ws, 1);
  if (bwd_fused(&p)) {
    if ((e = launch_pad(desc, &p, x, xp, st)) != WTCONV_OK) return e;
    if ((e = launch_pad(desc, &p, dy, dyp, st)) != WTCONV_OK) return e;
    return run_bwd_fused(&p, desc, xp, dyp, w0, b0, s0, wl, sl, dx, dw0, db0, ds0, dwl, dsl, ws, st);
  }
  if ((e = launch_pad(desc, &p, dy, dyp, st)) != WTCONV_OK) return e;
  if ((e = run_forward(&p, dyp, w0, nullptr, s0, wl, sl, dx, 1, ws, st, desc)) != WTCONV_OK) return e;
  if ((e = launch_pad(desc, &p, x, xp, st)) != WTCONV_OK) return e;
  return run_bwdw(&p, xp, dyp, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, ws, st);
}

}  // extern "C"

// ------------------------------------------------------------------------
// Weight gradients for callers that cannot allocate device memory.
//
// Some callers have no way to hand the library a workspace: a plain C host
// program or plugin that has no allocator of its own at the call site, a
// runtime whose memory is fully reserved up front and forbids cudaMalloc
// during steady-state steps, or code whose allocator lives in a framework it
// cannot reach.  For them the partial sums of the weight-gradient reduction
// live in this file-scope device array instead of a caller workspace.  Every
// GPU that loads this library holds the array (WTCONV_NOALLOC_SCRATCH_BYTES)
// until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[WTCONV_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int MAX_DEVICES = 64;
std::mutex g_scratch_mutex;
struct ScratchAddr {
  unsigned long long ctx_id;  // id of the CUDA context the address belongs to
  void* addr;
};
ScratchAddr g_scratch_addr[MAX_DEVICES] = {};

// Id of the CUDA context current on this thread (0 when none is current
// yet).  Ids are unique for the life of the process, so a context created
// again after cudaDeviceReset never matches a cached entry.  The two driver
// calls are fetched through the runtime, so the library links no driver
// library of its own.  Called with g_scratch_mutex held.
typedef int (*CtxGetCurrentFn)(void**);
typedef int (*CtxGetIdFn)(void*, unsigned long long*);
wtconv_status current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  if (!get_current || !get_id) {
    void* f1 = nullptr;
    void* f2 = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
        q1 != cudaDriverEntryPointSuccess || !f1)
      return WTCONV_ERR_CUDA;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
        q2 != cudaDriverEntryPointSuccess || !f2)
      return WTCONV_ERR_CUDA;
    get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
    get_id = reinterpret_cast<CtxGetIdFn>(f2);
  }
  void* ctx = nullptr;
  if (get_current(&ctx) != 0) return WTCONV_ERR_CUDA;
  *id = 0;
  if (ctx && get_id(ctx, id) != 0) return WTCONV_ERR_CUDA;
  return WTCONV_OK;
}

// Device address of g_noalloc_scratch in the current context.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// with the device current, once per context, and cached with the context's
// id: after cudaDeviceReset the module is loaded again (the array may move),
// and the new context's id forces a fresh lookup.
wtconv_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return WTCONV_ERR_CUDA;
  if (dev < 0 || dev >= MAX_DEVICES) return WTCONV_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  unsigned long long id = 0;
  wtconv_status e = current_context_id(&id);
  if (e != WTCONV_OK) return e;
  if (id == 0 || !g_scratch_addr[dev].addr || g_scratch_addr[dev].ctx_id != id) {
    void* p = nullptr;
    // also makes the device's primary context current when none was
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return WTCONV_ERR_CUDA;
    if ((e = current_context_id(&id)) != WTCONV_OK) return e;
    g_scratch_addr[dev] = ScratchAddr{id, p};
  }
  *out = g_scratch_addr[dev].addr;
  return WTCONV_OK;
}
}  // namespace

extern "C" {

size_t wtconv_noalloc_scratch_bytes(void) { return WTCONV_NOALLOC_SCRATCH_BYTES; }

wtconv_status wtconv_backward_weight_noalloc(const wtconv_desc* desc, const void* x, const void* dy,
                                             const float* w0, const float* b0, const float* s0, const float* wl,
                                             const float* sl, float* dw0, float* db0, float* ds0, float* dwl,
                                             float* dsl, void* stream) {
  wtconv_status e = check_desc(desc);
  if (e != WTCONV_OK) return e;
  if (!x || !dy) return WTCONV_ERR_ARG;
  if ((e = check_params(desc, w0, b0, s0, wl, sl, true)) != WTCONV_OK) return e;
  if ((e = check_grad_outputs(desc, dw0, db0, ds0, dwl, dsl)) != WTCONV_OK) return e;
  if (!aligned16(x) || !aligned16(dy)) return WTCONV_ERR_ALIGN;
  if (ragged(desc)) return WTCONV_ERR_SHAPE;  // no workspace for padded copies
  // one group of partial sums is C * V floats; at least one must fit, with
  // the LL planes of the row-band path when the planes need it
  const size_t V = (size_t)desc->k * desc->k * (1 + 4 * desc->L) + 1;
  const size_t group_bytes = (size_t)desc->C * V * sizeof(float);
  const bool whole = bwdw_whole_plane(desc);
  const size_t ll_bytes = whole ? 0 : band_ll_floats(desc) * sizeof(float);
  const size_t avail = WTCONV_NOALLOC_SCRATCH_BYTES - WS_HEADER;
  if (ll_bytes + 16 + group_bytes > avail) return WTCONV_ERR_SCRATCH_LIMIT;
  const size_t groups = (avail - ll_bytes - 16) / group_bytes;
  void* scratch = nullptr;
  if ((e = noalloc_scratch(&scratch)) != WTCONV_OK) return e;
  float* part = reinterpret_cast<float*>(static_cast<char*>(scratch) + WS_HEADER);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (whole) {
    const int max_groups = (int)std::min<size_t>(groups, (size_t)desc->N);
    return run_bwdw_part(desc, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, nullptr, max_groups, st);
  }
  const int G = std::min<int>(band_groups(desc), (int)std::min<size_t>(groups, 1u << 20));
  if (G == 0) return WTCONV_ERR_UNSUPPORTED;
  float* ll = reinterpret_cast<float*>(static_cast<char*>(scratch) + WS_HEADER + band_part_bytes(desc, G));
  return run_band(desc, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, ll, G, nullptr, st);
}

int wtconv_kernel_launches(const wtconv_desc* desc, int op) {
  if (check_desc(desc) != WTCONV_OK) return 0;
  if (ragged(desc)) {
    const wtconv_desc p = padded(desc);
    const int inner = wtconv_kernel_launches(&p, op);
    if (inner == 0 || op == WTCONV_OP_FOLD) return inner;
    return inner + op_acts(op);  // the pads of the inputs
  }
  const int pass = pass_launches(desc);
  // fold first, except on level-0 planes that scale the taps in their one kernel
  const int data = (small_planes(desc) || direct_raw(desc)) ? 1 : pass ? 1 + pass : 0;
  const int weight = bwdw_whole_plane(desc) ? 2 : (desc->L == 0 ? 1 : desc->L) + 1;  // kernel(s), finalize
  switch (op) {
    case WTCONV_OP_FORWARD:
    case WTCONV_OP_BACKWARD_DATA:
      return data;
    case WTCONV_OP_BACKWARD_WEIGHT:
      return weight;
    case WTCONV_OP_BACKWARD:
      return bwd_fused(desc) ? 3 : data + weight;  // fused: fold, fused pass, finalize
    case WTCONV_OP_FORWARD_FOLDED:
      return pass;
    case WTCONV_OP_FOLD:
      return 1;
    default:
      return 0;
  }
}

const char* wtconv_status_string(wtconv_status s) {
  switch (s) {
    case WTCONV_OK: return "ok";
    case WTCONV_ERR_ARG: return "invalid argument";
    case WTCONV_ERR_SHAPE: return "H or W not divisible by 2^L";
    case WTCONV_ERR_ALIGN: return "pointer not aligned (16 bytes for tensors and workspace)";
    case WTCONV_ERR_WORKSPACE: return "workspace missing or too small";
    case WTCONV_ERR_CUDA: return "CUDA error at launch";
    case WTCONV_ERR_UNSUPPORTED: return "shape needs more shared memory than one SM offers";
    case WTCONV_ERR_SCRATCH_LIMIT:
      return "shape needs more scratch than the built-in no-allocation buffer holds";
    default: return "unknown status";
  }
}

}  // extern "C"
