// C ABI of libwtconv: argument checks, shared-memory plans and launches.
// The operations and their definitions are documented in include/wtconv.h.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <initializer_list>
#include <mutex>

#include "wtconv.h"
#include "wtconv_kernels.cuh"
#include "wtconv_main.cuh"
#include "wtconv_bwband.cuh"

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

void relocate(BufDesc& d, int base, int slab) {
  d.off += base;
  d.ps = slab;
}

int io_bytes(const wtconv_desc* d) { return d->io == WTCONV_BF16 ? 2 : 4; }

void fill_common(Plan& P, const wtconv_desc* d) {
  P = Plan{};
  P.N = d->N;
  P.C = d->C;
  P.H = d->H;
  P.W = d->W;
  P.K = d->k;
  P.r = d->k / 2;
  P.L = d->L;
  P.H1 = d->L >= 1 ? d->H / 2 : d->H;
  P.W1 = d->L >= 1 ? d->W / 2 : d->W;
  P.kk4 = rup(d->k * d->k, 4);
  P.vec_in = (d->W % 4) == 0;
  P.vec_out = d->io == WTCONV_BF16 ? (d->W % 8) == 0 : (d->W % 4) == 0;
  P.prefetch_ok = ((size_t)d->H * d->W * io_bytes(d)) % 16 == 0;
  P.io_bytes = io_bytes(d);
  P.nthreads = NT;
  P.V = d->k * d->k * (1 + 4 * d->L) + 1;
}

// Per-plane slab of the forward / backward-data kernel.
int forward_slab(Plan& P) {
  const int r = P.r, L = P.L, RB = P.R3 / 2;
  int cur = 0;
  P.xf = make_shifted(cur, P.H, P.W, r, {{P.R3, C3_CW}}, 1);
  if (L >= 1) P.s1 = make_shifted(cur, P.H1, P.W1, r, {{RB, 4}, {2, 2}}, 4);
  if (L >= 2) {
    P.t1 = make_plain(cur, P.H1, P.W1, {{RB, 4}, {1, 4}}, 1);
    for (int l = 2; l <= L; ++l) P.sd[l] = make_shifted(cur, P.H >> l, P.W >> l, r, {{DP_R, DP_CW}, {2, 2}}, 4);
    for (int l = 2; l <= L; ++l) P.zd[l] = make_plain(cur, P.H >> l, P.W >> l, {{DP_R, DP_CW}}, 4);
  }
  P.deep_off = 0;
  P.deep_floats = 0;
  return rup(cur, 4);
}

void forward_items(Plan& P) {
  const int L = P.L;
  int per, xdiv;
  if (L >= 2) {
    xdiv = P.W >> 2;
    per = (P.H >> 2) * xdiv;
  } else if (L == 1) {
    xdiv = cdiv_h(P.W, 4);
    per = P.H1 * xdiv;
  } else {
    xdiv = cdiv_h(P.W, 4);
    per = P.H * xdiv;
  }
  P.f_stage_per = make_fdiv(per);
  P.f_stage_x = make_fdiv(xdiv);
  int first = 0;
  for (int l = 0; l <= MAXL + 1; ++l) P.deep_first[l] = 0;
  for (int l = 2; l <= L; ++l) {
    const int tx = cdiv_h(P.W >> l, DP_CW), tiles = cdiv_h(P.H >> l, DP_R) * tx;
    P.f_l_tiles[l] = make_fdiv(tiles);
    P.f_l_tx[l] = make_fdiv(tx);
    P.deep_first[l] = first;
    first += 4 * tiles;
  }
  P.deep_items = first;
  if (L >= 2) P.deep_first[L + 1] = first;
  P.f_deep_per = make_fdiv(first > 0 ? first : 1);
  const int tq = cdiv_h(P.W1, 4);
  P.f_t1_x = make_fdiv(tq);
  P.f_t1_per = make_fdiv(P.H1 * tq);
  const int ox = cdiv_h(P.W, C3_CW);
  P.f_out_x = make_fdiv(ox);
  P.f_out_per = make_fdiv(cdiv_h(P.H, P.R3) * ox);
}

// Shared-memory header: mbarrier (8 bytes) and abort flag, 16 bytes.
constexpr int HEADER_FLOATS = 4;

void finish_forward_plan(Plan& P, int PB) {
  const int slab = forward_slab(P);
  P.PB = PB;
  P.nbatch = (P.N + PB - 1) / PB;
  P.w_off = HEADER_FLOATS;
  P.use_bulk = P.prefetch_ok;
  P.raw_off = rup(P.w_off + (1 + 4 * P.L) * P.kk4 + 4, 4);
  const int raw_floats = P.use_bulk ? rup((int)((size_t)PB * P.H * P.W * P.io_bytes / 4), 4) : 0;
  const int base = P.raw_off + raw_floats;
  for (BufDesc* b : {&P.xf, &P.s1, &P.t1, &P.zb, &P.t2}) relocate(*b, base, slab);
  for (int l = 0; l <= MAXL; ++l) {
    relocate(P.sd[l], base, slab);
    relocate(P.zd[l], base, slab);
  }
  P.smem_floats = base + PB * slab;
  forward_items(P);
}

// Tiles of the output pass per plane, for the batch-size choice.
int output_items(const Plan& P, int R3) { return ((P.H + R3 - 1) / R3) * ((P.W + C3_CW - 1) / C3_CW); }

// Threads per CTA of the forward kernel: 128 when one plane has few
// output tiles, so that a batch of one plane still keeps most threads busy.
int forward_threads(const Plan& P) { return output_items(P, P.H >= 8 ? 4 : 2) <= 128 ? 128 : 256; }

void build_forward_plan(Plan& P, const wtconv_desc* d, int max_smem) {
  fill_common(P, d);
  P.R3 = (P.H >= 8) ? 4 : 2;
  P.nthreads = forward_threads(P);
  const int items = output_items(P, P.R3);
  int PB = std::max(1, std::min(d->N, P.nthreads / items));
  const size_t budget = (size_t)max_smem / 2;
  for (;;) {
    finish_forward_plan(P, PB);
    if (PB == 1 || (size_t)P.smem_floats * 4 <= budget) break;
    --PB;
  }
}

void bwdw_items(Plan& P) {
  forward_items(P);  // staging and deep-level decompositions are shared
  const int bx = cdiv_h(P.W, BW_CW);
  P.f_bw_x = make_fdiv(bx);
  P.f_bw_per = make_fdiv(cdiv_h(P.H, BW_R) * bx);
  const int b1 = cdiv_h(P.W1, B1_CW);
  P.f_b1_x = make_fdiv(b1);
  P.f_b1_per = make_fdiv(cdiv_h(P.H1, B1_R) * b1);
}

int bwdw_slab(Plan& P) {
  const int r = P.r, L = P.L;
  int cur = 0;
  P.xf = make_shifted(cur, P.H, P.W, r, {{BW_R, BW_CW}}, 1);
  P.gf = make_plain(cur, P.H, P.W, {{BW_R, BW_CW}}, 1);
  if (L >= 1) {
    P.s1 = make_shifted(cur, P.H1, P.W1, r, {{B1_R, B1_CW}, {2, 2}}, 4);
    P.g1 = make_plain(cur, P.H1, P.W1, {{B1_R, B1_CW}, {2, 2}}, 4);
  }
  for (int l = 2; l <= L; ++l) {
    P.sd[l] = make_shifted(cur, P.H >> l, P.W >> l, r, {{DP_R, DP_CW}, {2, 2}}, 4);
    P.gd[l] = make_plain(cur, P.H >> l, P.W >> l, {{DP_R, DP_CW}, {2, 2}}, 4);
  }
  return rup(cur, 4);
}

void finish_bwdw_plan(Plan& P, int PB) {
  const int slab = bwdw_slab(P);
  P.PB = PB;
  const int ndeep = P.L >= 2 ? (P.L - 1) * 4 : 0;
  P.gdeep_off = HEADER_FLOATS;
  P.dpart_off = P.gdeep_off + ndeep * P.kk4;
  P.use_bulk = P.prefetch_ok;
  const int raw_floats = P.use_bulk ? rup((int)((size_t)PB * P.H * P.W * P.io_bytes / 4), 4) : 0;
  P.raw_off = rup(P.dpart_off + ndeep * DSLOTS * P.kk4, 4);
  P.rawg_off = P.raw_off + raw_floats;
  const int base = P.rawg_off + raw_floats;
  for (BufDesc* b : {&P.xf, &P.gf, &P.s1, &P.g1}) relocate(*b, base, slab);
  for (int l = 0; l <= MAXL; ++l) {
    relocate(P.sd[l], base, slab);
    relocate(P.gd[l], base, slab);
  }
  P.red_off = base;
  P.smem_floats = std::max(base + PB * slab, base + NT * P.kk4 + NT);
  bwdw_items(P);
}

void build_bwdw_plan(Plan& P, const wtconv_desc* d, int max_smem) {
  fill_common(P, d);
  P.R3 = 2;
  const int items = ((P.H + BW_R - 1) / BW_R) * ((P.W + BW_CW - 1) / BW_CW);
  const int nbase = P.L >= 1 ? 128 : NT;
  int PB = std::max(1, std::min(d->N, (nbase + items - 1) / items));
  for (;;) {
    finish_bwdw_plan(P, PB);
    if (PB == 1 || (size_t)P.smem_floats * 4 <= (size_t)max_smem / 2) break;
    --PB;
  }
}

// ------------------------------------------------ pipelined output kernel
constexpr int SM_SMEM = 233472;  // shared memory per SM on sm_100a (228 KB)

// Floats of one channel's folded weights: the base kernel, the bias and
// four kernels per level (kk4 floats each).
int main_wblk(const wtconv_desc* d) { return rup((1 + 4 * d->L) * rup(d->k * d->k, 4) + 4, 4); }

// Output tile rows for band height TH: 8, unless 4 wastes fewer padded rows.
int main_r3(int TH) { return rup(TH, 8) == rup(TH, 4) ? 8 : 4; }

// Slot layout for band height TH and PB planes per unit; returns the slot
// size in floats.
int main_slot(MainPlan& M, int TH, int PB) {
  const int r = M.r, R3 = main_r3(TH), TH1 = TH / 2;
  const int hx = M.L >= 1 ? 2 * r : r;
  M.fused = TH == M.H && M.L >= 2;
  if (M.fused) M.bulk_t = 0;
  int cur = 0;
  // raw region: written by the bulk copies of the next unit
  M.wraw_off = cur;
  cur += M.wblk;
  M.raw_off = cur;
  M.raw_pp = rup((int)(((size_t)std::min(M.H, TH + 2 * hx) * M.W * M.io_bytes + 3) / 4), 4);
  cur += PB * M.raw_pp;
  M.rawt_off = cur;
  M.rawt_pp = (M.L >= 2 && M.bulk_t) ? rup(TH1 * M.W1, 4) : 0;
  cur += PB * M.rawt_pp;
  // the current unit's staged data, read by the register tiles
  M.w_off = cur;
  cur += M.wblk;
  int pcur = 0;  // per-plane buffers, PB copies each
  M.xf = make_shifted(pcur, TH, M.W, r, {{R3, 4}}, 1);
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
  for (BufDesc* bd : {&M.xf, &M.s1, &M.t1, &M.zb}) {
    bd->off += cur;
    bd->ps = pstride;
  }
  for (int l = 2; l <= M.L && M.fused; ++l)
    for (BufDesc* bd : {&M.sd[l], &M.zd[l]}) {
      bd->off += cur;
      bd->ps = pstride;
    }
  cur += PB * pstride;
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
  M.wblk = main_wblk(d);
  M.bulk_t = d->L >= 2 && (M.W1 % 4) == 0;
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
      const int tpp = cdiv_h(cand, main_r3(cand)) * tx;
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
  M.R3 = main_r3(TH);
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
  int first = 0;
  for (int l = 0; l <= MAXL + 1; ++l) D.deep_first[l] = 0;
  for (int l = 2; l <= D.L; ++l) {
    const int tx = cdiv_h(D.W >> l, DP_CW), tiles = cdiv_h(D.H >> l, DP_R) * tx;
    D.f_l_tiles[l] = make_fdiv(tiles);
    D.f_l_tx[l] = make_fdiv(tx);
    D.deep_first[l] = first;
    first += 4 * tiles;
  }
  D.deep_items = first;
  D.deep_first[D.L + 1] = first;
  D.f_deep_per = make_fdiv(first);
  const int tq = cdiv_h(D.W1, 4);
  D.f_t1_x = make_fdiv(tq);
  D.f_t1_per = make_fdiv(D.H1 * tq);
  return true;
}

size_t t1_bytes(const wtconv_desc* d) {
  return d->L >= 2 ? (((size_t)d->N * d->C * (d->H / 2) * (d->W / 2) * sizeof(float) + 15) / 16) * 16 : 0;
}

// Forward / backward-data workspace: 16-byte header (status word), t1 of
// every plane (levels >= 2), then the folded weights of every channel.
size_t fwd_ws_bytes(const wtconv_desc* d) {
  return 16 + t1_bytes(d) + (size_t)d->C * main_wblk(d) * sizeof(float);
}

wtconv_status check_desc(const wtconv_desc* d) {
  if (!d) return WTCONV_ERR_ARG;
  if (d->k < 1 || d->k > WTCONV_MAX_K || (d->k % 2) == 0) return WTCONV_ERR_ARG;
  if (d->L < 0 || d->L > WTCONV_MAX_LEVELS) return WTCONV_ERR_ARG;
  if (d->N <= 0 || d->C <= 0 || d->H <= 0 || d->W <= 0) return WTCONV_ERR_ARG;
  if (d->io != WTCONV_F32 && d->io != WTCONV_BF16) return WTCONV_ERR_ARG;
  if ((long long)d->H * d->W > (1LL << 30) || (long long)d->N * d->C > (1LL << 30)) return WTCONV_ERR_ARG;
  const int m = 1 << d->L;
  if ((d->H % m) != 0 || (d->W % m) != 0) return WTCONV_ERR_SHAPE;
  return WTCONV_OK;
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

wtconv_status query_device(Device& dev) {
  int id = 0;
  if (cudaGetDevice(&id) != cudaSuccess) return WTCONV_ERR_CUDA;
  if (cudaDeviceGetAttribute(&dev.sms, cudaDevAttrMultiProcessorCount, id) != cudaSuccess) return WTCONV_ERR_CUDA;
  if (cudaDeviceGetAttribute(&dev.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, id) != cudaSuccess)
    return WTCONV_ERR_CUDA;
  return WTCONV_OK;
}

template <typename F>
wtconv_status prepare(F kern, size_t smem, int& occ, int nthreads = NT) {
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return WTCONV_ERR_CUDA;
  occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, nthreads, smem) != cudaSuccess)
    return WTCONV_ERR_CUDA;
  if (occ < 1) return WTCONV_ERR_UNSUPPORTED;
  return WTCONV_OK;
}

template <int K, typename IO>
wtconv_status launch_forward_t(const wtconv_desc* d, const Device& dev, const void* x, const float* w0,
                               const float* b0, const float* s0, const float* wl, const float* sl, void* y, int flip,
                               int* status, float* t1, cudaStream_t st) {
  float* wfold = reinterpret_cast<float*>(reinterpret_cast<char*>(t1) + t1_bytes(d));
  {
    const int kk4 = rup(d->k * d->k, 4), wblk = main_wblk(d);
    const int n = d->C * wblk;
    wtconv_fold_kernel<K><<<std::min((n + 255) / 256, dev.sms * 4), 256, 0, st>>>(d->C, d->L, kk4, wblk, w0, b0, s0,
                                                                                   wl, sl, flip, wfold);
    if (cudaGetLastError() != cudaSuccess) return WTCONV_ERR_CUDA;
  }
  MainPlan M;
  if (!build_main_plan(M, d, dev.max_smem)) return WTCONV_ERR_UNSUPPORTED;
  if (d->L >= 2 && !M.fused) {
    DeepPlan D;
    if (!build_deep_plan(D, d, dev.max_smem)) return WTCONV_ERR_UNSUPPORTED;
    auto kd = wtconv_deep_kernel<K, IO>;
    const size_t smem = (size_t)D.smem_floats * 4;
    int occ = 0;
    wtconv_status e = prepare(kd, smem, occ, DEEP_NT);
    if (e != WTCONV_OK) return e;
    const int units = D.C * D.nbatch;
    kd<<<std::min(units, dev.sms * occ), DEEP_NT, smem, st>>>(D, static_cast<const IO*>(x), wl, sl, t1, flip);
    if (cudaGetLastError() != cudaSuccess) return WTCONV_ERR_CUDA;
  }
  const size_t smem = (size_t)M.smem_floats * 4;
  int occ = 0;
  if (M.R3 == 8) {
    auto km = wtconv_main_kernel<K, 8, IO>;
    wtconv_status e = prepare(km, smem, occ, MAIN_NT);
    if (e != WTCONV_OK) return e;
    km<<<std::min(M.units, dev.sms * occ), MAIN_NT, smem, st>>>(M, static_cast<const IO*>(x), t1, wfold,
                                                                static_cast<IO*>(y), status);
  } else {
    auto km = wtconv_main_kernel<K, 4, IO>;
    wtconv_status e = prepare(km, smem, occ, MAIN_NT);
    if (e != WTCONV_OK) return e;
    km<<<std::min(M.units, dev.sms * occ), MAIN_NT, smem, st>>>(M, static_cast<const IO*>(x), t1, wfold,
                                                                static_cast<IO*>(y), status);
  }
  return cudaGetLastError() == cudaSuccess ? WTCONV_OK : WTCONV_ERR_CUDA;
}

template <int K>
wtconv_status launch_forward_k(const wtconv_desc* d, const Device& dev, const void* x, const float* w0,
                               const float* b0, const float* s0, const float* wl, const float* sl, void* y, int flip,
                               int* status, float* t1, cudaStream_t st) {
  if (d->io == WTCONV_F32) return launch_forward_t<K, float>(d, dev, x, w0, b0, s0, wl, sl, y, flip, status, t1, st);
  return launch_forward_t<K, __nv_bfloat16>(d, dev, x, w0, b0, s0, wl, sl, y, flip, status, t1, st);
}

// Forward (flip = 0) or backward-data (flip = 1).  ws: 16-byte header (status
// word) followed by t1 when L >= 2 (ws may be NULL when L < 2).
wtconv_status run_forward(const wtconv_desc* d, const void* x, const float* w0, const float* b0, const float* s0,
                          const float* wl, const float* sl, void* y, int flip, void* ws, cudaStream_t st) {
  Device dev;
  wtconv_status e = query_device(dev);
  if (e != WTCONV_OK) return e;
  int* status = static_cast<int*>(ws);
  float* t1 = reinterpret_cast<float*>(static_cast<char*>(ws) + 16);
  switch (d->k) {
    case 1: return launch_forward_k<1>(d, dev, x, w0, b0, s0, wl, sl, y, flip, status, t1, st);
    case 3: return launch_forward_k<3>(d, dev, x, w0, b0, s0, wl, sl, y, flip, status, t1, st);
    case 5: return launch_forward_k<5>(d, dev, x, w0, b0, s0, wl, sl, y, flip, status, t1, st);
    default: return launch_forward_k<7>(d, dev, x, w0, b0, s0, wl, sl, y, flip, status, t1, st);
  }
}

// Workspace: a 16-byte header whose first int is the device status word,
// then (weight gradients) the per-CTA partial sums.
constexpr size_t WS_HEADER = 16;

// Plan constants of sm_100a (B200): opt-in shared memory per CTA and SM
// count.  The weight-gradient path and its workspace depend on the shape
// only, through these, so wtconv_workspace_size needs no device query.
constexpr int PLAN_SMEM = 232448;
constexpr int PLAN_SMS = 148;

// True when one plane's whole weight-gradient working set fits one SM.
bool bwdw_whole_plane(const wtconv_desc* d) {
  Plan P;
  build_bwdw_plan(P, d, PLAN_SMEM);
  return (size_t)P.smem_floats * 4 <= (size_t)PLAN_SMEM;
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
  int cur = 0;
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
// partials keep the whole-plane layout): enough CTAs for four per SM, at
// most one per unit of the launch with the fewest units.  0 if a level
// does not fit.
int band_groups(const wtconv_desc* d) {
  int umin = 1 << 30;
  for (int lvl = band_first_level(d); lvl <= d->L; ++lvl) {
    BandPlan B;
    if (!build_band_plan(B, d, lvl)) return 0;
    umin = std::min(umin, B.units);
  }
  const int target = (4 * PLAN_SMS + d->C - 1) / d->C;
  return std::max(1, std::min(umin, target));
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

template <int K, typename IO>
wtconv_status launch_bwdw_t(Plan& P, const Device& dev, const void* x, const void* dy, const float* w0,
                            const float* b0, const float* s0, const float* wl, const float* sl, float* dw0,
                            float* db0, float* ds0, float* dwl, float* dsl, float* part, int* status,
                            cudaStream_t st, int max_groups) {
  auto kern = wtconv_bwdw_kernel<K, IO>;
  const size_t smem = (size_t)P.smem_floats * 4;
  int occ = 0;
  wtconv_status e = prepare(kern, smem, occ);
  if (e != WTCONV_OK) return e;
  // planes per CTA: fewest sequential batches per CTA slot (waves x batches
  // per CTA), ties broken towards longer CTAs (fewer partial sums)
  const int slots = dev.sms * occ;
  long best = -1;
  for (int ppc = P.PB; ppc < P.N + P.PB; ppc += P.PB) {
    const int p = std::min(ppc, P.N);
    const int groups = (P.N + p - 1) / p;
    if (groups > max_groups) continue;
    const long ctas = (long)P.C * groups;
    const long cost = ((ctas + slots - 1) / slots) * ((p + P.PB - 1) / P.PB);
    if (best < 0 || cost <= best) {
      best = cost;
      P.planes_per_cta = p;
    }
    if (p == P.N) break;
  }
  P.ngroups = (P.N + P.planes_per_cta - 1) / P.planes_per_cta;
  kern<<<P.C * P.ngroups, NT, smem, st>>>(P, static_cast<const IO*>(x), static_cast<const IO*>(dy), part,
                                          status);
  if (cudaGetLastError() != cudaSuccess) return WTCONV_ERR_CUDA;
  const size_t fsmem = (size_t)P.V * sizeof(float);
  auto fin = wtconv_bwdw_finalize<K>;
  if (fsmem > 48 * 1024 &&
      cudaFuncSetAttribute(fin, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fsmem) != cudaSuccess)
    return WTCONV_ERR_CUDA;
  fin<<<P.C, 128, fsmem, st>>>(P, part, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl);
  return cudaGetLastError() == cudaSuccess ? WTCONV_OK : WTCONV_ERR_CUDA;
}

template <int K>
wtconv_status launch_bwdw_k(Plan& P, const Device& dev, wtconv_dtype io, const void* x, const void* dy,
                            const float* w0, const float* b0, const float* s0, const float* wl, const float* sl,
                            float* dw0, float* db0, float* ds0, float* dwl, float* dsl, float* part, int* status,
                            cudaStream_t st, int max_groups) {
  if (io == WTCONV_F32)
    return launch_bwdw_t<K, float>(P, dev, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, status, st,
                                   max_groups);
  return launch_bwdw_t<K, __nv_bfloat16>(P, dev, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, status,
                                         st, max_groups);
}

// Runs the weight-gradient kernels with the per-CTA partial sums at `part`
// and at most `max_groups` CTAs per channel (the partials then fill
// max_groups * C * V floats).
wtconv_status run_bwdw_part(const wtconv_desc* d, const void* x, const void* dy, const float* w0, const float* b0,
                            const float* s0, const float* wl, const float* sl, float* dw0, float* db0, float* ds0,
                            float* dwl, float* dsl, float* part, int* status, int max_groups, cudaStream_t st) {
  Device dev;
  wtconv_status e = query_device(dev);
  if (e != WTCONV_OK) return e;
  if (dev.max_smem < PLAN_SMEM) return WTCONV_ERR_UNSUPPORTED;
  Plan P;
  build_bwdw_plan(P, d, dev.max_smem);
  if ((size_t)P.smem_floats * 4 > (size_t)dev.max_smem) return WTCONV_ERR_UNSUPPORTED;
  switch (d->k) {
    case 1:
      return launch_bwdw_k<1>(P, dev, d->io, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, status, st,
                              max_groups);
    case 3:
      return launch_bwdw_k<3>(P, dev, d->io, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, status, st,
                              max_groups);
    case 5:
      return launch_bwdw_k<5>(P, dev, d->io, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, status, st,
                              max_groups);
    default:
      return launch_bwdw_k<7>(P, dev, d->io, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, status, st,
                              max_groups);
  }
}

template <int K, typename IN>
wtconv_status launch_band_level(const BandPlan& B, const void* a, const void* b, float* llx, float* lld, float* part,
                                cudaStream_t st) {
  auto kern = wtconv_bwband_kernel<K, IN>;
  const size_t smem = (size_t)B.smem_floats * 4;
  int occ = 0;
  wtconv_status e = prepare(kern, smem, occ);
  if (e != WTCONV_OK) return e;
  kern<<<B.C * B.ngroups, NT, smem, st>>>(B, static_cast<const IN*>(a), static_cast<const IN*>(b), llx, lld, part);
  return cudaGetLastError() == cudaSuccess ? WTCONV_OK : WTCONV_ERR_CUDA;
}

// Row-band path: one launch per level (the first on x and dy, the others on
// the raw LL planes the level above wrote to `ll`), then the fixed-order
// finalize over `groups` partial vectors per channel.
template <int K>
wtconv_status run_band_k(const wtconv_desc* d, const void* x, const void* dy, const float* w0, const float* b0,
                         const float* s0, const float* wl, const float* sl, float* dw0, float* db0, float* ds0,
                         float* dwl, float* dsl, float* part, float* ll, int groups, cudaStream_t st) {
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
      e = d->io == WTCONV_F32 ? launch_band_level<K, float>(B, x, dy, llx, lld, part, st)
                              : launch_band_level<K, __nv_bfloat16>(B, x, dy, llx, lld, part, st);
    else
      e = launch_band_level<K, float>(B, prevx, prevd, llx, lld, part, st);
    if (e != WTCONV_OK) return e;
    prevx = llx;
    prevd = lld;
  }
  Plan P;
  fill_common(P, d);
  P.ngroups = groups;
  const size_t fsmem = (size_t)P.V * sizeof(float);
  auto fin = wtconv_bwdw_finalize<K>;
  if (fsmem > 48 * 1024 &&
      cudaFuncSetAttribute(fin, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fsmem) != cudaSuccess)
    return WTCONV_ERR_CUDA;
  fin<<<P.C, 128, fsmem, st>>>(P, part, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl);
  return cudaGetLastError() == cudaSuccess ? WTCONV_OK : WTCONV_ERR_CUDA;
}

wtconv_status run_band(const wtconv_desc* d, const void* x, const void* dy, const float* w0, const float* b0,
                       const float* s0, const float* wl, const float* sl, float* dw0, float* db0, float* ds0,
                       float* dwl, float* dsl, float* part, float* ll, int groups, cudaStream_t st) {
  Device dev;
  wtconv_status e = query_device(dev);
  if (e != WTCONV_OK) return e;
  if (dev.max_smem < PLAN_SMEM) return WTCONV_ERR_UNSUPPORTED;
  switch (d->k) {
    case 1:
      return run_band_k<1>(d, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, ll, groups, st);
    case 3:
      return run_band_k<3>(d, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, ll, groups, st);
    case 5:
      return run_band_k<5>(d, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, ll, groups, st);
    default:
      return run_band_k<7>(d, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, ll, groups, st);
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
  return run_band(d, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, ll, G, st);
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

extern "C" {

size_t wtconv_workspace_size(const wtconv_desc* desc, int op) {
  if (check_desc(desc) != WTCONV_OK) return 0;
  switch (op) {
    case WTCONV_OP_FORWARD:
    case WTCONV_OP_BACKWARD_DATA:
      return fwd_ws_bytes(desc);
    case WTCONV_OP_BACKWARD_WEIGHT:
      return bwdw_ws_bytes(desc);
    case WTCONV_OP_BACKWARD:
      return std::max(bwdw_ws_bytes(desc), fwd_ws_bytes(desc));
    default:
      return 0;
  }
}

wtconv_status wtconv_forward(const wtconv_desc* desc, const void* x, const float* w0, const float* b0,
                             const float* s0, const float* wl, const float* sl, void* y, void* ws,
                             size_t ws_bytes, void* stream) {
  wtconv_status e = check_desc(desc);
  if (e != WTCONV_OK) return e;
  if (!x || !y) return WTCONV_ERR_ARG;
  if ((e = check_params(desc, w0, b0, s0, wl, sl, true)) != WTCONV_OK) return e;
  if (!aligned16(x) || !aligned16(y)) return WTCONV_ERR_ALIGN;
  if ((e = check_ws(ws, ws_bytes, fwd_ws_bytes(desc))) != WTCONV_OK) return e;
  return run_forward(desc, x, w0, b0, s0, wl, sl, y, 0, ws, static_cast<cudaStream_t>(stream));
}

wtconv_status wtconv_backward_data(const wtconv_desc* desc, const void* dy, const float* w0, const float* s0,
                                   const float* wl, const float* sl, void* dx, void* ws, size_t ws_bytes,
                                   void* stream) {
  wtconv_status e = check_desc(desc);
  if (e != WTCONV_OK) return e;
  if (!dy || !dx) return WTCONV_ERR_ARG;
  if ((e = check_params(desc, w0, nullptr, s0, wl, sl, false)) != WTCONV_OK) return e;
  if (!aligned16(dy) || !aligned16(dx)) return WTCONV_ERR_ALIGN;
  if ((e = check_ws(ws, ws_bytes, fwd_ws_bytes(desc))) != WTCONV_OK) return e;
  return run_forward(desc, dy, w0, nullptr, s0, wl, sl, dx, 1, ws, static_cast<cudaStream_t>(stream));
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
  if ((e = check_ws(ws, ws_bytes, bwdw_ws_bytes(desc))) != WTCONV_OK) return e;
  return run_bwdw(desc, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, ws,
                  static_cast<cudaStream_t>(stream));
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
  e = run_forward(desc, dy, w0, nullptr, s0, wl, sl, dx, 1, ws, st);
  if (e != WTCONV_OK) return e;
  return run_bwdw(desc, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, ws, st);
}

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
void* g_scratch_addr[MAX_DEVICES] = {};

// Device address of g_noalloc_scratch on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
wtconv_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return WTCONV_ERR_CUDA;
  if (dev < 0 || dev >= MAX_DEVICES) return WTCONV_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return WTCONV_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return WTCONV_OK;
}
}  // namespace

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
  return run_band(desc, x, dy, w0, b0, s0, wl, sl, dw0, db0, ds0, dwl, dsl, part, ll, G, st);
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
