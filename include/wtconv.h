/*
 * wtconv.h -- C ABI of the B200 (sm_100a) WTConv layer library (libwtconv.so).
 *
 * The layer (source: "I/O-aware reformulation of wavelet convolution",
 * arXiv:2608.10805, abstract): a multi-level 2-D Haar wavelet decomposition
 * of each input channel, a k x k depthwise convolution with a learned
 * per-channel scale on every subband at every level, the multi-level
 * synthesis cascade back to full resolution, added to a scaled base k x k
 * depthwise convolution of the input.  With L = 0 it is a plain depthwise
 * convolution (with bias and per-channel scale).
 *
 * Definitions (all entry points follow them exactly, up to fp32 rounding):
 *   dwconv(A, W)[c,i,j] = sum_{u,v<k} W[c,u,v] * A[c, i+u-r, j+v-r],
 *       r = (k-1)/2, zero outside the image (cross-correlation, 'same').
 *   Haar of the 2x2 block a=(2i,2j) b=(2i,2j+1) c=(2i+1,2j) d=(2i+1,2j+1):
 *       LL=(a+b+c+d)/2  LH=(a+b-c-d)/2  HL=(a-b+c-d)/2  HH=(a-b-c+d)/2
 *   IWT is its inverse (and transpose).
 *   Ybase = s0[c] * (dwconv(X, W0)[c] + b0[c])
 *   cur = X; for l = 1..L: sub_l = Haar(cur) (bands LL,LH,HL,HH);
 *       Z_l[c,s] = sl[l][c][s] * dwconv(sub_l[c,s], Wl[l][c][s]); cur = raw LL.
 *   t = 0; for l = L..1: t = IWT(Z_l with t added to its LL band)
 *   Y = Ybase + t
 *   Sides that are not multiples of 2^L (the paper does not cover them; this
 *   is the library's reading): at every level an odd side of the plane
 *   entering the analysis gets one zero row (bottom) or column (right), and
 *   that level's synthesis output is cropped back to the plane's size.  The
 *   library computes this on copies of the input planes zero-padded to
 *   multiples of 2^L, which gives the same outputs and gradients, and
 *   stores only the image part of each output plane.
 *
 * Layouts (all contiguous, row-major):
 *   x, y, dy, dx : [N][C][H][W] in the I/O dtype (fp32 or bf16)
 *   w0 : [C][k][k] fp32      b0, s0 : [C] fp32
 *   wl : [L][C][4][k][k] fp32 (band order LL, LH, HL, HH)
 *   sl : [L][C][4] fp32
 *
 * Conventions shared by every entry point:
 *   - Every tensor pointer is caller-owned DEVICE memory; the library never
 *     allocates, frees or keeps state between calls (one exception:
 *     wtconv_backward_weight_noalloc's own device array, below).  Calls are
 *     asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and never synchronise.
 *   - Workspace (`ws`, `ws_bytes`): device memory of at least
 *     wtconv_workspace_size(desc, op) bytes, 16-byte aligned.  Its first 16
 *     bytes are a header whose first int is a device status word: a kernel
 *     whose bounded wait for an asynchronous copy ran out of iterations sets
 *     it to 1 (its outputs are then incomplete); the library never clears it,
 *     so a caller that checks it zeroes it first.  After the header, the
 *     forward and backward-data passes keep the folded weights of every
 *     channel and, for L >= 2, the synthesis of levels >= 2 at level-1
 *     resolution (fp32, N*C*(H/2)*(W/2)); the weight-gradient passes keep
 *     their per-CTA partial sums (the fused backward: the partial sums and
 *     the adjoint's folded weights).  For sides that are not multiples of 2^L
 *     it also holds zero-padded copies of the call's input planes (x or dy;
 *     both for the weight-gradient passes).  The workspace is required.
 *     Level-0 layers (L = 0) on planes of at most 32x32 (a few planes per
 *     warp), and fp32 level-0 layers whose rows are a multiple of 4 and at
 *     most 248 elements (one tensor copy per unit), run one kernel per data
 *     pass that scales W0 and b0 by s0 as it loads them (no fold launch; the
 *     folded weights in the workspace unused).
 *   - Arithmetic is fp32 throughout; bf16 I/O is rounded to nearest even on
 *     output.  Results are deterministic run to run (fixed reduction order).
 *   - Gradients are overwritten, not accumulated.
 *   - Argument checks happen on the host before any launch:
 *       WTCONV_ERR_ARG       null desc/pointer, k even or outside 1..7,
 *                            L < 0 or L > WTCONV_MAX_LEVELS, N,C,H,W <= 0,
 *                            element counts that overflow 32-bit indexing
 *       WTCONV_ERR_SHAPE     (no-allocation variant only) H or W not a
 *                            multiple of 2^L: it has no workspace for the
 *                            padded copies
 *       WTCONV_ERR_ALIGN     a tensor pointer not 16-byte aligned
 *       WTCONV_ERR_WORKSPACE ws_bytes < wtconv_workspace_size(desc, op)
 *       WTCONV_ERR_UNSUPPORTED  the shape needs more on-chip memory than
 *                            one SM offers
 *       WTCONV_ERR_SCRATCH_LIMIT  (no-allocation variant only) the partial
 *                            sums do not fit its built-in array
 *     and WTCONV_ERR_CUDA reports a launch failure (cudaGetLastError).
 *     Nothing is launched when a check fails.  No device-side trap exists.
 *   - With L = 0, wl and sl may be NULL.
 */
#ifndef WTCONV_H
#define WTCONV_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define WTCONV_MAX_LEVELS 8
#define WTCONV_MAX_K 7

typedef enum { WTCONV_F32 = 0, WTCONV_BF16 = 1 } wtconv_dtype;

/* Layer shape: batch N, channels C, image H x W, kernel size k (odd),
 * levels L, I/O dtype of x, y, dy, dx. */
typedef struct {
  int N, C, H, W, k, L;
  wtconv_dtype io;
} wtconv_desc;

typedef enum {
  WTCONV_OK = 0,
  WTCONV_ERR_ARG = 1,
  WTCONV_ERR_SHAPE = 2,
  WTCONV_ERR_ALIGN = 3,
  WTCONV_ERR_WORKSPACE = 4,
  WTCONV_ERR_CUDA = 5,
  WTCONV_ERR_UNSUPPORTED = 6,
  WTCONV_ERR_SCRATCH_LIMIT = 7
} wtconv_status;

/* Operation codes for wtconv_workspace_size and wtconv_kernel_launches
 * (WTCONV_OP_FOLD: wtconv_fold_weights, which needs no workspace). */
enum {
  WTCONV_OP_FORWARD = 0,
  WTCONV_OP_BACKWARD_DATA = 1,
  WTCONV_OP_BACKWARD_WEIGHT = 2,
  WTCONV_OP_BACKWARD = 3,
  WTCONV_OP_FORWARD_FOLDED = 4,
  WTCONV_OP_FOLD = 5
};

/* Bytes of device workspace the operation `op` uses for `desc` (0 when desc
 * is invalid): the 16-byte status header, then the folded weights and the
 * level >= 2 synthesis (forward, backward-data) or the per-CTA partial sums
 * of the fixed-order two-stage reduction (weight gradients); op 3 (both
 * backward passes) is the larger of the two. */
size_t wtconv_workspace_size(const wtconv_desc* desc, int op);

/* Forward pass: y = WTConv(x).  Source: arXiv:2608.10805, abstract (the
 * layer; reformulations (1) on-chip Haar analysis, (2) single-pass
 * synthesis indexed by output-coordinate bits, (3) scales folded into the
 * convolution weights).  b0, s0 and w0 are required; wl, sl when L > 0.
 * Needs wtconv_workspace_size(desc, 0) bytes of ws. */
wtconv_status wtconv_forward(const wtconv_desc* desc, const void* x,
                             const float* w0, const float* b0, const float* s0,
                             const float* wl, const float* sl, void* y,
                             void* ws, size_t ws_bytes, void* stream);

/* Backward data pass: dx = J^T dy, the adjoint of the forward map in x.
 * The adjoint of the +-1/2 Haar analysis is the synthesis and vice versa,
 * and the adjoint of each depthwise conv is the correlation with its
 * spatially flipped kernel, so this is the forward pass run on dy with
 * flipped kernels and no bias (arXiv:2608.10805, abstract: training).
 * Needs wtconv_workspace_size(desc, 1) bytes of ws. */
wtconv_status wtconv_backward_data(const wtconv_desc* desc, const void* dy,
                                   const float* w0, const float* s0,
                                   const float* wl, const float* sl, void* dx,
                                   void* ws, size_t ws_bytes, void* stream);

/* Backward weight pass: gradients of <y, dy> with respect to every
 * parameter (arXiv:2608.10805, abstract: the layer is trained, so its
 * learned weights and per-channel scales need gradients; the Haar pyramids
 * of x and dy are recomputed on chip, reformulation (1)), with
 * G_0[c,u,v] = sum_{n,i,j} dy[n,c,i,j] x[n,c,i+u-r,j+v-r]
 * and G_l[c,s,u,v] = sum dZ_l[c,s](i,j) sub_l[c,s](i+u-r,j+v-r), where
 * dZ_l = Haar pyramid of dy and sub_l = Haar pyramid of x:
 *   dw0 = s0 G_0   db0 = s0 sum(dy)   ds0 = sum_uv w0 G_0 + b0 sum(dy)
 *   dwl = sl G_l   dsl = sum_uv wl G_l
 * Outputs dw0 [C][k][k], db0 [C], ds0 [C], dwl [L][C][4][k][k], dsl [L][C][4]
 * (fp32, overwritten).  Needs wtconv_workspace_size(desc, 2) bytes of ws. */
wtconv_status wtconv_backward_weight(const wtconv_desc* desc, const void* x,
                                     const void* dy, const float* w0,
                                     const float* b0, const float* s0,
                                     const float* wl, const float* sl,
                                     float* dw0, float* db0, float* ds0,
                                     float* dwl, float* dsl, void* ws,
                                     size_t ws_bytes, void* stream);

/* Both backward passes in one call (dx and every parameter gradient).
 * Source: arXiv:2608.10805, abstract (training): the adjoint of the forward
 * map in x runs the analysis on dy, which is the same Haar pyramid of dy
 * the weight gradients correlate against, so for planes held whole in one
 * SM (k <= 5) one fused pass stages x and dy once per unit and computes the
 * correlations, then the adjoint data pass, from the same on-chip pyramids
 * (launches: the adjoint weight fold, the fused pass, the finalize).  Other
 * shapes (row-band planes, k = 7, level-0 planes of at most 32x32) run
 * wtconv_backward_data, then
 * wtconv_backward_weight, in that order on `stream`.  dx equals what
 * wtconv_backward_data gives, bit for bit; the parameter gradients agree
 * with wtconv_backward_weight up to the order of the per-CTA partial sums.
 * Needs wtconv_workspace_size(desc, 3) bytes of ws (for the fused pass: the
 * header, the partial sums and the adjoint folded block). */
wtconv_status wtconv_backward(const wtconv_desc* desc, const void* x,
                              const void* dy, const float* w0, const float* b0,
                              const float* s0, const float* wl, const float* sl,
                              void* dx, float* dw0, float* db0, float* ds0,
                              float* dwl, float* dsl, void* ws, size_t ws_bytes,
                              void* stream);

/* Size of the device array that wtconv_backward_weight_noalloc uses in
 * place of a workspace (8 MiB, held by every GPU that loads the library). */
#define WTCONV_NOALLOC_SCRATCH_BYTES (8u << 20)

/* Weight gradients without a workspace, for callers that cannot allocate
 * device memory at the call site (a plain C host program or plugin with no
 * allocator of its own there, a runtime whose memory is reserved up front and
 * forbids cudaMalloc during steady-state steps, or code that cannot reach
 * the allocator of the framework it runs in).  The paper has no counterpart:
 * this is an interface variant of wtconv_backward_weight, with the same
 * arguments minus ws/ws_bytes and the same outputs.
 *
 * The per-CTA partial sums go to a file-scope device array of
 * WTCONV_NOALLOC_SCRATCH_BYTES instead; the library then uses fewer CTAs per
 * channel if needed so they fit.  Planes too large for one SM (the row-band
 * path) also keep there the raw LL planes that each level hands to the next:
 * 2 * N * C * (H/2^l) * (W/2^l) floats for every level l = 1 .. L-1.  Shapes
 * whose LL planes plus the partial sums of one CTA per channel,
 * C * (k*k*(1+4L)+1) floats, plus a 16-byte header and 16 bytes of
 * alignment, exceed the array are rejected with WTCONV_ERR_SCRATCH_LIMIT
 * before anything touches the GPU.
 * The first call in each CUDA context of a device looks up the array's
 * device address (with that device current) and caches it with the
 * context's id, so a context created again after cudaDeviceReset gets a
 * fresh lookup; make the first call in a context before any stream capture.  The call allocates nothing (no cudaMalloc, no cudaFree, no
 * allocating library routine).  Every call on a device shares the one array,
 * which keeps the last call's contents (each call overwrites every partial it
 * reads): calls that overlap on the GPU, e.g. on two streams, race and must
 * be serialised by the caller.  There is no device status word here: a
 * bounded in-kernel wait that runs out still ends the kernel, but nothing
 * tells the caller; callers that check for it use wtconv_backward_weight. */
wtconv_status wtconv_backward_weight_noalloc(const wtconv_desc* desc,
                                             const void* x, const void* dy,
                                             const float* w0, const float* b0,
                                             const float* s0, const float* wl,
                                             const float* sl, float* dw0,
                                             float* db0, float* ds0, float* dwl,
                                             float* dsl, void* stream);

/* WTCONV_NOALLOC_SCRATCH_BYTES as this build of the library has it (for
 * callers that load the library at run time and want the limit from the
 * binary itself).  No counterpart in the paper. */
size_t wtconv_noalloc_scratch_bytes(void);

/* Bytes of the folded-weight block of `desc` (0 when desc is invalid): per
 * channel, s0*w0 and s0*b0, then 2^-l s_l[s] w_l[s] for every level l and
 * band s (2^-l: the synthesis factors 1/2 between level l and the image),
 * each k x k kernel padded to a multiple of 4 floats. */
size_t wtconv_folded_size(const wtconv_desc* desc);

/* Folds the per-channel scales into the convolution weights once
 * (arXiv:2608.10805, abstract, reformulation (3)), for callers whose
 * parameters stay fixed over many calls (inference).  adjoint = 0 gives the
 * forward block; adjoint = 1 the backward-data block (every kernel flipped,
 * no bias; b0 may then be NULL).  folded: caller-owned device memory of at
 * least wtconv_folded_size bytes, 16-byte aligned, overwritten.  One kernel
 * launch, asynchronous on `stream`.  Errors as for wtconv_forward;
 * WTCONV_ERR_WORKSPACE when folded_bytes is too small, WTCONV_ERR_ARG for an
 * adjoint flag other than 0 or 1. */
wtconv_status wtconv_fold_weights(const wtconv_desc* desc, const float* w0,
                                  const float* b0, const float* s0,
                                  const float* wl, const float* sl,
                                  int adjoint, void* folded,
                                  size_t folded_bytes, void* stream);

/* The forward pass over a block from wtconv_fold_weights: y equals what
 * wtconv_forward gives for the same parameters, bit for bit, without the
 * folding launch, so that planes held whole in one SM take one kernel
 * launch (row-band planes with L >= 2 take two: the deep levels, then the
 * output).  Given an adjoint block and dy in place of x, it computes the
 * backward-data pass dx.  x, y: NCHW device memory, 16-byte aligned; the
 * block is only read.  Needs wtconv_workspace_size(desc, 4) bytes of ws
 * (the status header, for L >= 2 the level >= 2 synthesis, and for sides
 * not multiples of 2^L the padded copy of x). */
wtconv_status wtconv_forward_folded(const wtconv_desc* desc, const void* x,
                                    const void* folded, void* y, void* ws,
                                    size_t ws_bytes, void* stream);

/* Number of kernel launches one call of operation `op` makes for `desc`
 * (the plan the library picks for the shape on sm_100a), so that a caller
 * can count the kernels in a timed region or a captured graph; 0 when desc
 * is invalid or op unknown.  No counterpart in the paper: an introspection
 * helper of this library. */
int wtconv_kernel_launches(const wtconv_desc* desc, int op);

/* Static description of a status code (never NULL). */
const char* wtconv_status_string(wtconv_status status);

#ifdef __cplusplus
}
#endif

#endif /* WTCONV_H */
