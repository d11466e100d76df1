// Implicit-GEMM convolution on the 5th-generation tensor cores (tcgen05) at
// FP32 accuracy, for stride-1 dense and wide-group convolutions.
//
// What it computes (POPCORNBENCH "Kimi-K2.6__l1_p62" and "Kimi-K2.6__l2_p21":
// the convolution viewed as a GEMM with M = output pixels, N = output
// channels of a group, K = C/groups * R * S):
//   y[n,k,p,q] = bias[k] + sum_{c,r,s} w[k,c,r,s] * x[n, gi*cpg + c, p - pad + r*dil, q - pad + s*dil]
// in FP32 accuracy: every operand v is split into v_hi = tf32(v) and
// v_lo = v - v_hi (exact in FP32).  Each product is accumulated in FP32 as
// a_hi*b_hi (a tf32 MMA) plus the two cross terms a_hi*b_lo + a_lo*b_hi,
// which are 2^-11 smaller and need only a few bits: they run as ONE bf16 MMA
// over K = 16 (the 8 channels' [bf16(a_hi), bf16(a_lo)] against
// [bf16(b_lo), bf16(b_hi)]), at twice the tf32 rate and half the operand
// bytes.  Error per product: bf16 rounding of the cross-term operands
// (<= 2^-20 |a*b| each) plus the dropped a_lo*b_lo (<= 2^-22 |a*b|), about
// 2e-6 |a*b| at most, against the 1e-5 * sum|w*x| bound.  TF32 on its own
// (2^-11 relative) would miss that bound; the pages flag TF32 as "not
// exactly fp32".
//
// Data layout.  A prep pass writes x_hi as padded NC4HW4 ([n][c/4][hp][wp][4]:
// four consecutive channels in one 16-byte cell; pad zero rows on top, pad
// zero columns on the left, zero columns up to a multiple of 16 pixels) and
// the bf16 cross-term operand as [n][c/8][2][hp][wp][8] (same cell geometry),
// and the weights split the same way as [g][c/8][r chunk][s][2][rows][kpg][4 tf32 | 8 bf16].
// In the tile a CTA stages ([2 channel quads][rows][cols][4], one TMA box),
// consecutive output pixels of one row are 16 bytes apart, which is exactly
// a K-major, no-swizzle UMMA operand with 8-row core matrices (SBO = 128 B)
// whose two K halves are one channel quad apart (LBO).  The operand for filter
// tap (r, s) is therefore the same staged tile with its start address moved by
// (row r*dil, column s*dil): the im2col matrix is never materialised, and
// every staged element feeds up to R*S taps of MMAs.
//
// Pipeline (persistent; a tile = one image n, TH output rows x 128 output
// columns, all kpg output channels of group g):
//   warp 0 lane 0 : producer - per 8-channel step one TMA box of x_hi and one
//                   of the cross-term operand (all staged rows and columns),
//                   then the weight slices of the tap-row chunks (bulk copies;
//                   loaded once per CTA when they all fit the ring);
//   warp 1 lane 0 : MMA issuer - for every output row and tap (r, s) one bf16
//                   and one tf32 tcgen05.mma (M=128) into the row's TMEM
//                   accumulator; with tap rows folded (ig_issue_chunk) one
//                   pair per staged row and tap column covers up to 256/kpg
//                   tap rows at once (N up to 256); tcgen05.commit frees the
//                   stages;
//   other warps   : epilogue - tcgen05.ld of the accumulators (then cleared:
//                   every MMA accumulates), +bias, or the chain's +bias,
//                   *scale, logistic and GroupNorm partial statistics,
//                   coalesced stores along q; two TMEM accumulator buffers
//                   let it overlap the next tile's MMAs.
#include <atomic>

#include <cuda.h>
#include <cudaTypedefs.h>

#include <cuda_bf16.h>

#include "device_utils.cuh"
#include "gconv_internal.h"

namespace gconv {

namespace {

__device__ int g_igemm_error = 0;

// ------------------------------------------------------------------ prep
// Two bf16 values packed in 32 bits, first in the low half (memory order).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo_half, float hi_half) {
    const uint32_t a = __bfloat16_as_ushort(__float2bfloat16_rn(lo_half));
    const uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(hi_half));
    return a | (b << 16);
}

// x[N][C][H][W] -> per 8 input channels (octet c8) and padded pixel (hp, wp)
// of a [Hp][Wp] plane holding x[h][w] at (h + pad_h, w + pad_w) and zeros
// elsewhere:
//   xh: tf32 parts in NC4HW4 cells, [n][2*c8 + q][hp][wp][4]  (q = channel quad)
//   xc: bf16 parts, [n][c8][2][hp][wp][8]: chunk 0 = bf16(x_hi), chunk 1 = bf16(x - x_hi)
// Both tensors have the same geometry when read as 32-bit words.
__global__ void __launch_bounds__(256) split_x_kernel(const float *__restrict__ x, float4 *__restrict__ xh,
                                                      uint4 *__restrict__ xc, int C8, int H, int W, int pad_h,
                                                      int pad_w, int Hp, int Wp, long long cells) {
    dev::griddep_wait();
    dev::griddep_launch_dependents();
    const long long HW = (long long)H * W, HWp = (long long)Hp * Wp;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < cells;
         i += (long long)gridDim.x * blockDim.x) {
        const long long pix = i % HWp;         // hp*Wp + wp
        const long long nc8 = i / HWp;         // n*C8 + c8
        const int h = (int)(pix / Wp) - pad_h, w = (int)(pix % Wp) - pad_w;
        const bool in = h >= 0 && h < H && w >= 0 && w < W;
        const float *src = x + nc8 * 8 * HW + (in ? (long long)h * W + w : 0);
        float hi[8], lo[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float v = in ? __ldg(src + j * HW) : 0.f;
            hi[j] = dev::to_tf32(v);
            lo[j] = v - hi[j];
        }
        const long long q0 = (nc8 * 2) * HWp + pix;   // cell index of quad 0 (and of chunk 0)
        xh[q0] = make_float4(hi[0], hi[1], hi[2], hi[3]);
        xh[q0 + HWp] = make_float4(hi[4], hi[5], hi[6], hi[7]);
        xc[q0] = make_uint4(pack_bf16x2(hi[0], hi[1]), pack_bf16x2(hi[2], hi[3]), pack_bf16x2(hi[4], hi[5]),
                            pack_bf16x2(hi[6], hi[7]));
        xc[q0 + HWp] = make_uint4(pack_bf16x2(lo[0], lo[1]), pack_bf16x2(lo[2], lo[3]), pack_bf16x2(lo[4], lo[5]),
                                  pack_bf16x2(lo[6], lo[7]));
    }
}

// w[K][cpg][R][S] -> per (g, c8, r, s, output channel kk), 8 input channels,
// the tap rows taken in chunks of RF (rc = r / RF, row j = RF-1 - r % RF
// within the chunk: descending, so that one MMA over a chunk's rows writes
// consecutive output rows; rows past R in the last chunk are zero):
//   wh: [g][c8][rc][s][2][RF][kpg][4]   tf32 parts (two channel quads)
//   wc: [g][c8][rc][s][2][RF][kpg][8]   bf16 parts: chunk 0 = bf16(w - w_hi), chunk 1 = bf16(w_hi)
// so that the bf16 MMA over K = 16 computes x_hi*w_lo + x_lo*w_hi.
// Packed groups (gp > 1): the GEMM runs gp consecutive conv groups as one
// group of gp*cpg input and gp*kpg output channels whose weights are block
// diagonal: output kk of the packed group reads input c only when both belong
// to the same original group (kk / kpg0 == c / cpg0), else the weight is 0.
// kpg and cpg here are the packed sizes, kpg0 and cpg0 the original ones.
__global__ void __launch_bounds__(256) split_w_kernel(const float *__restrict__ w, float4 *__restrict__ wh,
                                                      uint4 *__restrict__ wc, int kpg, int cpg, int R, int S,
                                                      int RF, long long cells, int gp, int kpg0, int cpg0) {
    const int RP = (R + RF - 1) / RF * RF;   // tap rows including the zero ones
    dev::griddep_wait();
    dev::griddep_launch_dependents();
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < cells;
         i += (long long)gridDim.x * blockDim.x) {
        long long t = i;
        const int kk = (int)(t % kpg); t /= kpg;
        const int s = (int)(t % S); t /= S;
        const int r = (int)(t % RP); t /= RP;
        const int c8 = (int)(t % (cpg / 8));
        const long long g = t / (cpg / 8);
        float hi[8], lo[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int c = c8 * 8 + j;
            float v;
            if (r >= R) {
                v = 0.f;
            } else if (gp == 1) {
                v = __ldg(w + (((g * kpg + kk) * cpg + c) * R + r) * S + s);
            } else {
                const int b = kk / kpg0;   // original group of the output, within the pack
                const long long k0 = (g * gp + b) * kpg0 + kk % kpg0;
                v = (c / cpg0 == b) ? __ldg(w + ((k0 * cpg0 + c % cpg0) * R + r) * S + s) : 0.f;
            }
            hi[j] = dev::to_tf32(v);
            lo[j] = v - hi[j];
        }
        // cell of (g, c8, rc, s, quad 0, row j, kk); quad 1 is RF*kpg cells on
        const int rc = r / RF, j = RF - 1 - r % RF;
        const long long base = (((((g * (cpg / 8) + c8) * (RP / RF) + rc) * S + s) * 2) * RF + j) * kpg + kk;
        const long long q1 = (long long)RF * kpg;
        wh[base] = make_float4(hi[0], hi[1], hi[2], hi[3]);
        wh[base + q1] = make_float4(hi[4], hi[5], hi[6], hi[7]);
        wc[base] = make_uint4(pack_bf16x2(lo[0], lo[1]), pack_bf16x2(lo[2], lo[3]), pack_bf16x2(lo[4], lo[5]),
                              pack_bf16x2(lo[6], lo[7]));
        wc[base + q1] = make_uint4(pack_bf16x2(hi[0], hi[1]), pack_bf16x2(hi[2], hi[3]), pack_bf16x2(hi[4], hi[5]),
                                   pack_bf16x2(hi[6], hi[7]));
    }
}

// Epilogue warps: 16 (4 per TMEM lane quarter, 8-column chunks) for 32
// output channels, 8 (2 per lane quarter, 16-column chunks) for wider tiles,
// so the epilogue keeps enough warps in flight without spilling registers.
__host__ __device__ constexpr int ig_epi_warps(int NT) { return NT <= 32 ? 16 : 8; }
// Fused variant: two converter warps between the MMA warp and the epilogue.
constexpr int kConvWarps = 2;
__host__ __device__ constexpr int ig_conv_warps(bool fused) { return fused ? kConvWarps : 0; }
__host__ __device__ constexpr int ig_threads(int NT, bool fused = false) {
    return 64 + 32 * ig_conv_warps(fused) + 32 * ig_epi_warps(NT);
}
// Output rows per tile of the fused variant (N = 32): 6 rows keep two x
// operand stages, a raw staging slot and the resident weights in shared memory.
constexpr int kFusedTH = 6;
// shared memory ahead of the stage ring: barriers, TMEM slot, abort flag
__host__ __device__ constexpr int ig_header(int NT, bool chain) { return 1024; }

// Number of GroupNorm partials one tile leaves per group: one per TMEM lane
// quarter and per chunk of CW channels the group spans.
__host__ __device__ constexpr int ig_chunk_width(int NT) {
    return NT / (ig_epi_warps(NT) / 4) < 16 ? NT / (ig_epi_warps(NT) / 4) : 16;
}

// 2^x on the special-function unit (flush to zero)
__device__ __forceinline__ float ex2_ftz(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

// Logistic 1 / (1 + 2^t): 2^t and the reciprocal on the special-function
// unit (flush to zero).  2^t overflows to +inf for large t and 1 / inf is
// exactly the limit 0.  (A variant with Newton-Raphson division on the FMA
// pipe in place of the reciprocal measured slower: the epilogue is bound by
// issue, not by the special-function unit.)
__device__ __forceinline__ float logistic_exp2(float t) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(1.f + ex2_ftz(t)));
    return y;
}

// Output tile t -> (n, g, row tile, column tile); column tiles vary fastest so
// CTAs running side by side share input rows in L2.  Tiles are taken from the
// last image backwards: the split pass that runs just before writes the images
// forwards, so the GEMM starts on the split operands still in L2, and the
// images it finishes last (the first ones) are where a following pass over
// the output starts.
struct IgTile {
    int n, g, p0, q0, sp;
};

__device__ __forceinline__ IgTile ig_tile(const IgemmParams &p, int t) {
    IgTile r;
    t = p.n_tiles - 1 - t;
    const int nsp = p.n_qt * p.n_pt;
    r.sp = t % nsp;
    const int rest = t / nsp;
    r.g = rest % p.groups;
    r.n = rest / p.groups;
    r.q0 = (r.sp % p.n_qt) * 128;
    r.p0 = (r.sp / p.n_qt) * p.TH;
    return r;
}

// Rows per tile the planner picks when shared memory allows: two TMEM
// accumulator buffers of TH x NT columns.
__host__ __device__ constexpr int ig_default_th(int NT) { return NT >= 256 ? 1 : (256 / NT < 8 ? 256 / NT : 8); }

// Tap rows folded into one MMA's N extent when the planner can: the fewest
// chunks of at most 256/NT rows (N <= 256 for M = 128), spread evenly so the
// last chunk carries few zero rows (5 rows at NT = 64: two chunks of 3).
__host__ __device__ constexpr int ig_fold_rf(int NT, int R) {
    const int most = R < 256 / NT ? R : 256 / NT;   // tap rows one MMA can cover
    const int chunks = (R + most - 1) / most;
    return (R + chunks - 1) / chunks;
}

// MMAs of one chunk of RF filter tap rows (r0 = rc*RF ...) over one staged
// x tile, all accumulating (the accumulators start at zero: the epilogue
// clears what it has read).  RF = 1: for every output row i and tap column s
// one bf16 cross-term MMA and one tf32 main-term MMA of N = NT on staged row
// i + r0*dil.  RF > 1 (dilation 1 along H): for every staged row ir and tap
// column s one pair whose N extent covers the chunk's tap rows r that take
// staged row ir to an output row o = ir - r of the tile.  A chunk's weight
// rows are stored in descending r, so those output rows are consecutive
// accumulators in TMEM (columns o*NT ...), and the staged operand is read
// once per (ir, s) for up to RF*NT output columns instead of once per tap
// row.  Either way every output row receives its products in the order
// (channel step, r, s), so the result does not depend on RF.  With TH_ > 0
// every bound and offset is a compile-time constant once the loops unroll.
template <int NT, int TH_, int R_, int S_, int RF_>
__device__ __forceinline__ void ig_issue_chunk(const IgemmParams &p, int rc, uint32_t dbase, uint64_t dah,
                                               uint64_t dal, uint64_t dbh, uint64_t dbl, int COLS) {
    constexpr bool FIX = TH_ > 0;
    const int TH = FIX ? TH_ : p.TH, R = FIX ? R_ : p.R, S = FIX ? S_ : p.S, RF = FIX ? RF_ : p.RF;
    const int dil = FIX ? 1 : p.dil, dil_w = FIX ? 1 : p.dil_w;
    constexpr uint32_t idesc = dev::idesc_tf32(128, NT);
    constexpr uint32_t idesc_c = dev::idesc_bf16(128, NT);
    if (RF == 1) {
        const int arow = rc * dil;   // staged row of output row 0 for tap row rc
#pragma unroll
        for (int i = 0; i < TH; ++i) {
            const uint32_t d = dbase + (uint32_t)(i * NT);
#pragma unroll
            for (int s = 0; s < S; ++s) {
                // 16-byte units: staged row i + r*dil, column s*dil_w; weight tap column s
                const uint64_t ao = (uint64_t)((i + arow) * COLS + s * dil_w);
                const uint64_t bo = (uint64_t)(s * 2 * NT);
                // cross terms x_hi*w_lo + x_lo*w_hi: one bf16 MMA over K = 16
                dev::mma_bf16(d, dal + ao, dbl + bo, idesc_c, 1u);
                // main term x_hi*w_hi: tf32 MMA over K = 8
                dev::mma_tf32(d, dah + ao, dbh + bo, idesc, 1u);
            }
        }
        return;
    }
    const int AR = TH + R - 1;
    const int r0 = rc * RF, r1 = (r0 + RF < R ? r0 + RF : R) - 1;
#pragma unroll
    for (int ir = 0; ir < AR; ++ir) {
        // tap rows of the chunk with 0 <= ir - r < TH, weight rows from tap hi down
        const int hi = ir < r1 ? ir : r1;
        const int lo = ir - TH + 1 > r0 ? ir - TH + 1 : r0;
        if (hi < lo) continue;
        const int n = (hi - lo + 1) * NT;
        const uint32_t d = dbase + (uint32_t)((ir - hi) * NT);
#pragma unroll
        for (int s = 0; s < S; ++s) {
            const uint64_t ao = (uint64_t)(ir * COLS + s * dil_w);
            const uint64_t bo = (uint64_t)(s * 2 * RF * NT + (r0 + RF - 1 - hi) * NT);
            dev::mma_bf16(d, dal + ao, dbl + bo, dev::idesc_bf16(128, n), 1u);
            dev::mma_tf32(d, dah + ao, dbh + bo, dev::idesc_tf32(128, n), 1u);
        }
    }
}

// The folded MMAs of one chunk (r0 = rc*RF ...) for ONE tap column s, when
// the weights arrive as one slice per (channel step, chunk, tap column)
// because a whole chunk's slice does not fit shared memory (p.bs).  Output row
// o then receives its products in the order (channel step, chunk, s, r): the
// rounding differs from one MMA per tap, within the same bound.
template <int NT, int TH_, int R_, int S_, int RF_>
__device__ __forceinline__ void ig_issue_tap(const IgemmParams &p, int rc, int s, uint32_t dbase, uint64_t dah,
                                             uint64_t dal, uint64_t dbh, uint64_t dbl, int COLS) {
    constexpr bool FIX = TH_ > 0;
    const int TH = FIX ? TH_ : p.TH, R = FIX ? R_ : p.R, RF = FIX ? RF_ : p.RF;
    const int dil_w = FIX ? 1 : p.dil_w;
    const int AR = TH + R - 1;
    const int r0 = rc * RF, r1 = (r0 + RF < R ? r0 + RF : R) - 1;
#pragma unroll
    for (int ir = 0; ir < AR; ++ir) {
        const int hi = ir < r1 ? ir : r1;
        const int lo = ir - TH + 1 > r0 ? ir - TH + 1 : r0;
        if (hi < lo) continue;
        const int n = (hi - lo + 1) * NT;
        const uint32_t d = dbase + (uint32_t)((ir - hi) * NT);
        const uint64_t ao = (uint64_t)(ir * COLS + s * dil_w);
        const uint64_t bo = (uint64_t)((r0 + RF - 1 - hi) * NT);
        dev::mma_bf16(d, dal + ao, dbl + bo, dev::idesc_bf16(128, n), 1u);
        dev::mma_tf32(d, dah + ao, dbh + bo, dev::idesc_tf32(128, n), 1u);
    }
}

// MMA issuer (one thread).  For every tile and 8-channel step: wait for the
// x tile, then per weight slice (one per chunk of RF tap rows, or per chunk
// and tap column when BS) wait for it and issue its MMAs (ig_issue_chunk /
// ig_issue_tap).  TH_, R_, S_, RF_ > 0 fix the loop bounds (dilation 1,
// COLS = 128 + S_ - 1 rounded up to 16); 0 reads them and BS from p.
// Returns false when a bounded wait gave up.
template <int NT, int TH_, int R_, int S_, int RF_, int BS_ = 0>
__device__ __forceinline__ bool ig_mma_loop(const IgemmParams &p, uint32_t tmem, const unsigned char *ringA,
                                            const unsigned char *ringB, uint32_t a_slot, uint32_t b_slot,
                                            uint64_t *fullA, uint64_t *emptyA, uint64_t *fullB, uint64_t *emptyB,
                                            uint64_t *accf, uint64_t *acce) {
    constexpr bool FIX = TH_ > 0;
    const int TH = FIX ? TH_ : p.TH, R = FIX ? R_ : p.R, RF = FIX ? RF_ : p.RF, S = FIX ? S_ : p.S;
    const bool bs = FIX ? BS_ != 0 : p.bs != 0;
    const int dil = FIX ? 1 : p.dil;
    const int COLS = FIX ? (128 + S_ - 1 + 15) / 16 * 16 : p.COLS;
    const int AR = TH + (R - 1) * dil;
    const int RC = (R + RF - 1) / RF;
    const int nsl = bs ? RC * S : RC;                    // weight slices per channel step
    const uint32_t a_bytes = 32u * (uint32_t)COLS * (uint32_t)AR;
    const uint32_t a_lbo = a_bytes / 2;                  // one channel quad / bf16 chunk apart
    const uint32_t b_lbo = (uint32_t)(RF * NT * 16);     // the same for the weights
    const uint32_t acc_cols = (uint32_t)(TH * NT);
    int ia = 0, ib = 0, j = 0;
    for (int t = blockIdx.x; t < p.n_tiles; t += gridDim.x, ++j) {
        const int buf = j & 1, ubuf = j >> 1;
        if (ubuf > 0 && !dev::mbar_wait_bounded(&acce[buf], (ubuf - 1) & 1)) return false;
        dev::tc_fence_after();
        const uint32_t dbase = tmem + (uint32_t)buf * acc_cols;
        for (int cc8 = 0; cc8 < p.CC8; ++cc8, ++ia) {
            const int sa = ia % p.sa;
            if (!dev::mbar_wait_bounded(&fullA[sa], (ia / p.sa) & 1)) return false;
            dev::tc_fence_after();
            const unsigned char *xa = ringA + (size_t)sa * a_slot;
            const uint64_t dah = dev::smem_desc(xa, a_lbo, 128);
            const uint64_t dal = dev::smem_desc(xa + a_bytes, a_lbo, 128);
            // weight slice sl of this channel step: wait for it (resident slices are
            // loaded once and waited for on the first tile only), return its slot
            auto take = [&](int sl, int &sb) {
                sb = p.b_resident ? cc8 * nsl + sl : ib % p.sb;
                if (!p.b_resident || j == 0) {
                    if (!dev::mbar_wait_bounded(&fullB[sb], p.b_resident ? 0u : (uint32_t)((ib / p.sb) & 1)))
                        return false;
                    dev::tc_fence_after();
                }
                return true;
            };
#pragma unroll 1
            for (int rc = 0; rc < RC; ++rc) {
                if (!bs) {
                    int sb;
                    if (!take(rc, sb)) return false;
                    const unsigned char *wb = ringB + (size_t)sb * b_slot;
                    ig_issue_chunk<NT, TH_, R_, S_, RF_>(p, rc, dbase, dah, dal, dev::smem_desc(wb, b_lbo, 128),
                                                        dev::smem_desc(wb + b_slot / 2, b_lbo, 128), COLS);
                    if (!p.b_resident) dev::mma_commit(&emptyB[sb]);
                    ++ib;
                } else {
#pragma unroll
                    for (int s = 0; s < S; ++s) {
                        int sb;
                        if (!take(rc * S + s, sb)) return false;
                        const unsigned char *wb = ringB + (size_t)sb * b_slot;
                        ig_issue_tap<NT, TH_, R_, S_, RF_>(p, rc, s, dbase, dah, dal, dev::smem_desc(wb, b_lbo, 128),
                                                          dev::smem_desc(wb + b_slot / 2, b_lbo, 128), COLS);
                        if (!p.b_resident) dev::mma_commit(&emptyB[sb]);
                        ++ib;
                    }
                }
            }
            dev::mma_commit(&emptyA[sa]);
        }
        dev::mma_commit(&accf[buf]);   // fires once this tile's MMAs have completed
    }
    return true;
}

// ------------------------------------------------------------------ main kernel
// Persistent: CTA b processes tiles b, b + gridDim.x, ...  The producer and
// the MMA issuer run ahead through a ring of shared-memory stages; the MMA
// issuer alternates between two TMEM accumulator buffers so the epilogue of
// tile j overlaps the MMAs of tile j+1.
// KGN: 0 = plain convolution; otherwise the GroupNorm group width of the
// chain (1, 2, 4, 8, 16, or 32 standing for any multiple of 16).
template <int NT, int KGN, bool FUSED>
__global__ void __launch_bounds__(ig_threads(NT, FUSED), 1)
    igemm_tf32x3_kernel(const __grid_constant__ TensorMap tmh, const __grid_constant__ TensorMap tmc,
                        const IgemmParams p) {
    extern __shared__ __align__(1024) unsigned char smem[];
    uint64_t *fullA = reinterpret_cast<uint64_t *>(smem);  // [4] x tiles (hi and lo) landed
    uint64_t *emptyA = fullA + 4;                           // [4] x tile slot free
    uint64_t *fullB = fullA + 8;                            // [4] weight slices landed
    uint64_t *emptyB = fullA + 12;                          // [4] weight slice slot free
    uint64_t *accf = fullA + 16;                            // [2] accumulator ready
    uint64_t *acce = fullA + 18;                            // [2] accumulator drained
    uint32_t *tslot = reinterpret_cast<uint32_t *>(fullA + 20);
    int *abort_flag = reinterpret_cast<int *>(fullA + 21);
    uint64_t *drain = fullA + 22;                           // every issued MMA has completed
    uint64_t *rawFull = fullA + 24;                         // [2] fused: raw x box landed
    uint64_t *rawEmpty = fullA + 26;                        // [2] fused: raw slot converted
    constexpr bool CHAIN = KGN > 0;
    constexpr int CWARPS = ig_conv_warps(FUSED);
    unsigned char *stages = smem + ig_header(NT, CHAIN);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int num_tiles = p.n_tiles;
    const uint32_t a_slot = 2u * p.a_bytes;   // x_hi + x_lo tile of one channel step
    const uint32_t b_slot = 2u * p.b_bytes;   // w_hi + w_lo slice of one (channel step, tap row)
    unsigned char *ringA = stages;
    unsigned char *ringB = stages + (size_t)p.sa * a_slot;
    unsigned char *ringR = ringB + (size_t)p.sb * b_slot;   // fused: raw x boxes
    const uint32_t acc_cols = (uint32_t)(p.TH * NT);

    if (tid == 0) {
        dev::prefetch_tensormap(&tmh);
        if constexpr (!FUSED) dev::prefetch_tensormap(&tmc);
        for (int s = 0; s < 4; ++s) {
            // fused: an x stage is complete when every converter warp has arrived
            dev::mbar_init(&fullA[s], FUSED ? CWARPS : 1);
            dev::mbar_init(&emptyA[s], 1);
            dev::mbar_init(&fullB[s], 1);
            dev::mbar_init(&emptyB[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            dev::mbar_init(&rawFull[s], 1);
            dev::mbar_init(&rawEmpty[s], CWARPS > 0 ? CWARPS : 1);
        }
        for (int b = 0; b < 2; ++b) {
            dev::mbar_init(&accf[b], 1);
            dev::mbar_init(&acce[b], ig_epi_warps(NT));
        }
        dev::mbar_init(drain, 1);
        *abort_flag = 0;
        dev::fence_mbar_init();
    }
    if (warp == 1) {
        dev::tmem_alloc(tslot, p.tmem_cols);
        dev::tmem_relinquish();
    }
    dev::tc_fence_before();
    __syncthreads();
    dev::tc_fence_after();
    const uint32_t tmem = *tslot;
    {
        // every MMA accumulates: the epilogue warps clear both accumulator
        // buffers once here, and afterwards each part of a buffer they have read
        constexpr int EPW = ig_epi_warps(NT), PART = NT / (EPW / 4), CW = ig_chunk_width(NT);
        if (warp >= 2 + CWARPS) {
            const int ew = warp - 2 - CWARPS;
            const uint32_t tl0 = tmem + ((uint32_t)((warp & 3) * 32) << 16);
            for (int c = 0; c < 2 * p.TH; ++c)
                for (int c0 = (ew >> 2) * PART; c0 < ((ew >> 2) + 1) * PART; c0 += CW)
                    dev::tmem_st_zero<CW>(tl0 + (uint32_t)(c * NT + c0));
            dev::tmem_wait_st();
        }
        dev::tc_fence_before();
        __syncthreads();
        dev::tc_fence_after();
    }

    dev::griddep_wait();
    dev::griddep_launch_dependents();

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        // Per tile and 8-channel step: one x tile of AR = TH + (R-1)*dil
        // rows x COLS columns x 2 channel quads, x_hi and cross-term operand
        // one TMA box each, serving every tap row; then R weight slices (one
        // per tap row).  Tile coordinates are padded ones: output (p, q) reads
        // padded rows p.. and columns q.. of the split operands.
        int ia = 0, ib = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
            const IgTile tl = ig_tile(p, t);
            const int z0 = tl.n * (p.C / 4) + tl.g * (p.cpg / 4);
            for (int cc8 = 0; cc8 < p.CC8 && ok; ++cc8, ++ia) {
                const int sa = ia % p.sa, ua = ia / p.sa;
                if (lane == 0) {
                    if constexpr (FUSED) {
                        // raw x box [8 channels][AR rows][COLSR columns] starting at the
                        // tile's first input row and at its first input column rounded
                        // down to 4 (16-byte TMA coordinate); zero fill = padding
                        const int sr = ia % p.rr, ur = ia / p.rr;
                        if (ur > 0 && !dev::mbar_wait_bounded(&rawEmpty[sr], (ur - 1) & 1)) ok = false;
                        if (*(volatile int *)abort_flag) ok = false;
                        if (ok) {
                            const int x0 = tl.q0 - p.pad_w;
                            dev::mbar_arrive_expect_tx(&rawFull[sr], (uint32_t)p.raw_bytes);
                            dev::tma_load_3d(ringR + (size_t)sr * p.raw_bytes, &tmh, &rawFull[sr],
                                             x0 - (((x0 % 4) + 4) % 4), tl.p0 - p.pad,
                                             tl.n * p.C + tl.g * p.cpg + cc8 * 8);
                        }
                    } else {
                        if (ua > 0 && !dev::mbar_wait_bounded(&emptyA[sa], (ua - 1) & 1)) ok = false;
                        if (*(volatile int *)abort_flag) ok = false;
                        if (ok) {
                            dev::mbar_arrive_expect_tx(&fullA[sa], a_slot);
                            unsigned char *st = ringA + (size_t)sa * a_slot;
                            const int cz = z0 + cc8 * 2;
                            dev::tma_load_4d(st, &tmh, &fullA[sa], 0, tl.q0 / 16, tl.p0, cz);
                            dev::tma_load_4d(st + p.a_bytes, &tmc, &fullA[sa], 0, tl.q0 / 16, tl.p0, cz);
                        }
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok) break;
                if (p.b_resident && t != (int)blockIdx.x) continue;   // slices already resident
                const int nsl = p.bs ? p.RC * p.S : p.RC;   // weight slices per channel step
                for (int sl = 0; sl < nsl; ++sl, ++ib) {
                    const int sb = p.b_resident ? cc8 * nsl + sl : ib % p.sb;
                    const int ub = p.b_resident ? 0 : ib / p.sb;
                    if (lane == 0) {
                        if (ub > 0 && !dev::mbar_wait_bounded(&emptyB[sb], (ub - 1) & 1)) ok = false;
                        if (*(volatile int *)abort_flag) ok = false;
                        if (ok) {
                            dev::mbar_arrive_expect_tx(&fullB[sb], b_slot);
                            unsigned char *wb = ringB + (size_t)sb * b_slot;
                            const long long woff = (((long long)tl.g * p.CC8 + cc8) * nsl + sl) * (p.b_bytes / 16);
                            dev::bulk_load(wb, p.wh + woff, p.b_bytes, &fullB[sb]);
                            dev::bulk_load(wb + p.b_bytes, p.wl + woff, p.b_bytes, &fullB[sb]);
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                    if (!ok) break;
                }
            }
        }
        if (!ok && lane == 0) {
            *abort_flag = 1;
            atomicExch(&g_igemm_error, 1);
        }
        if (lane == 0) {
            // copies still in flight (only after an abort): wait, bounded, for the
            // last phase issued on every slot before the CTA may exit
            if constexpr (FUSED) {
                for (int j = ia > p.rr ? ia - p.rr : 0; j < ia; ++j)
                    dev::mbar_wait_bounded(&rawFull[j % p.rr], (uint32_t)(j / p.rr) & 1u);
            } else {
                for (int j = ia > p.sa ? ia - p.sa : 0; j < ia; ++j)
                    dev::mbar_wait_bounded(&fullA[j % p.sa], (uint32_t)(j / p.sa) & 1u);
            }
            if (p.b_resident) {
                for (int j = 0; j < ib; ++j) dev::mbar_wait_bounded(&fullB[j], 0);
            } else {
                for (int j = ib > p.sb ? ib - p.sb : 0; j < ib; ++j)
                    dev::mbar_wait_bounded(&fullB[j % p.sb], (uint32_t)(j / p.sb) & 1u);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------------ MMA issuer
            // loop bounds fixed at compile time for the common geometries
            // (dilation 1, default rows per tile): the issue loop then runs
            // back to back on constant operand offsets
            constexpr int THD = FUSED ? kFusedTH : ig_default_th(NT);
            constexpr int F3 = ig_fold_rf(NT, 3);   // the planner's fold for 3 tap rows
            constexpr int F5 = ig_fold_rf(NT, 5);   // and for 5 (per-tap-column slices)
            const bool d1 = p.dil == 1 && p.dil_w == 1 && p.TH == THD;
            bool ok;
#define IG_LOOP(TH_, R_, S_, RF_) \
    ig_mma_loop<NT, TH_, R_, S_, RF_>(p, tmem, ringA, ringB, a_slot, b_slot, fullA, emptyA, fullB, emptyB, accf, acce)
            // the chain's folded issue runs the general loop: its fully unrolled
            // form measured 14% slower there (0.899 against 0.787 ms per chain
            // call at 8 rows per tile), while plain convolutions gain from it
            if (!CHAIN && d1 && p.R == 3 && p.S == 3 && p.RF == F3 && !p.bs) ok = IG_LOOP(THD, 3, 3, F3);
            else if (d1 && p.R == 3 && p.S == 3 && p.RF == 1) ok = IG_LOOP(THD, 3, 3, 1);
            else if (d1 && p.R == 5 && p.S == 9 && p.RF == 1) ok = IG_LOOP(THD, 5, 9, 1);
            else if (d1 && p.R == 5 && p.S == 9 && p.RF == F5 && p.bs)
                ok = ig_mma_loop<NT, THD, 5, 9, F5, 1>(p, tmem, ringA, ringB, a_slot, b_slot, fullA, emptyA, fullB,
                                                        emptyB, accf, acce);
            else if (d1 && p.R == 1 && p.S == 1) ok = IG_LOOP(THD, 1, 1, 1);
            else ok = IG_LOOP(0, 0, 0, 0);
#undef IG_LOOP
            if (!ok) {
                *abort_flag = 1;
                atomicExch(&g_igemm_error, 1);
            }
            // no MMA may still be running when TMEM is released: one more commit
            // arrives once every MMA this thread issued has completed
            dev::mma_commit(drain);
            dev::mbar_wait_bounded(drain, 0);
        }
        __syncwarp();
    } else if (FUSED && warp < 2 + CWARPS) {
        // ---------------------------------------------------------- converter
        // Per tile and 8-channel step: wait for the raw x box and for the x stage
        // to be free, then write the stage as the split pass would: per staged
        // pixel (row, column) the tf32 parts of the 8 channels as two 16-byte
        // quads and the bf16 cross-term operand ([bf16(x_hi) x 8], [bf16(x - x_hi) x 8])
        // as two 16-byte chunks, in the same layout the TMA boxes of the unfused
        // variant deliver.  Identical arithmetic, so identical results.
        constexpr int CT = 32 * CWARPS;
        const int ctid = tid - 64;
        const int AR = p.AR, COLS = p.COLS, COLSR = p.COLSR;
        const int plane_r = AR * COLSR;           // floats between raw channel planes
        const int npx = AR * COLS;
        const int dq = CT / COLS, dr = CT % COLS;  // pixel-index step as (rows, columns)
        int ia = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
            const IgTile tl = ig_tile(p, t);
            const int cofs = ((tl.q0 - p.pad_w) % 4 + 4) % 4;
            for (int cc8 = 0; cc8 < p.CC8; ++cc8, ++ia) {
                const int sa = ia % p.sa, ua = ia / p.sa, sr = ia % p.rr, ur = ia / p.rr;
                if (*(volatile int *)abort_flag) ok = false;
                if (ok && !dev::mbar_wait_bounded(&rawFull[sr], (uint32_t)ur & 1u)) ok = false;
                if (ok && ua > 0 && !dev::mbar_wait_bounded(&emptyA[sa], (uint32_t)(ua - 1) & 1u)) ok = false;
                if (!__all_sync(0xffffffffu, ok)) {
                    ok = false;
                    break;
                }
                const float *raw = reinterpret_cast<const float *>(ringR + (size_t)sr * p.raw_bytes) + cofs;
                float4 *dh = reinterpret_cast<float4 *>(ringA + (size_t)sa * a_slot);
                uint4 *dc = reinterpret_cast<uint4 *>(ringA + (size_t)sa * a_slot + p.a_bytes);
                int row = ctid / COLS, col = ctid % COLS;
                for (int px = ctid; px < npx; px += CT) {
                    const float *src = raw + row * COLSR + col;
                    float hi[8], lo[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float v = src[j * plane_r];
                        hi[j] = dev::to_tf32(v);
                        lo[j] = v - hi[j];
                    }
                    const int cell = row * COLS + col;   // quad / chunk 0; quad / chunk 1 is npx cells on
                    dh[cell] = make_float4(hi[0], hi[1], hi[2], hi[3]);
                    dh[cell + npx] = make_float4(hi[4], hi[5], hi[6], hi[7]);
                    dc[cell] = make_uint4(pack_bf16x2(hi[0], hi[1]), pack_bf16x2(hi[2], hi[3]),
                                          pack_bf16x2(hi[4], hi[5]), pack_bf16x2(hi[6], hi[7]));
                    dc[cell + npx] = make_uint4(pack_bf16x2(lo[0], lo[1]), pack_bf16x2(lo[2], lo[3]),
                                                pack_bf16x2(lo[4], lo[5]), pack_bf16x2(lo[6], lo[7]));
                    col += dr;
                    row += dq;
                    if (col >= COLS) {
                        col -= COLS;
                        ++row;
                    }
                }
                // generic-proxy writes visible to the tensor core (async proxy)
                asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
                __syncwarp();
                if (lane == 0) {
                    dev::mbar_arrive(&rawEmpty[sr]);
                    dev::mbar_arrive(&fullA[sa]);
                }
            }
        }
        if (!ok && lane == 0) {
            *abort_flag = 1;
            atomicExch(&g_igemm_error, 1);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------- epilogue
        // Warp w reads TMEM lane quarter w % 4 (32 output pixels) and a block
        // of PART accumulator columns (output channels), in chunks of CW, for
        // all TH rows of the tile.  Chain: per GroupNorm group of a chunk the
        // warp sums (a - shift) and (a - shift)^2 per thread in FP32 with one
        // shift for the whole warp (lane 0's first value), adds the 32 lanes
        // in FP64 and writes one (count, mean, M2) partial to global memory;
        // no barrier between epilogue warps.
        constexpr int EPW = ig_epi_warps(NT);
        constexpr int PART = NT / (EPW / 4);
        constexpr int CW = ig_chunk_width(NT);
        constexpr int GPC = CHAIN ? (KGN >= CW ? 1 : CW / KGN) : 1;
        constexpr int GW = CHAIN ? (KGN >= CW ? CW : KGN) : CW;
        constexpr float kLog2e = 1.4426950408889634f;
        const int ew = warp - 2 - CWARPS;        // 0..EPW-1
        const int lq = warp & 3;                 // TMEM lane quarter this warp may access
        const int cpart = ew >> 2;               // column block of this warp
        const int m = lq * 32 + lane;
        const long long plane = (long long)p.P * p.Q;
        // GroupNorm fragments per group (chunks of CW channels it spans)
        const int fpg = CHAIN ? (p.kgn > CW ? p.kgn / CW : 1) : 1;
        // per-channel epilogue constants.  When a warp covers a single chunk of
        // columns (ONE) they depend only on the conv group (and, for the chain's
        // normalisation, the image), so they are reloaded only when those change.
        constexpr bool ONE = PART == CW;
        // plain: a = acc * mul + add.  chain: t = -(acc*scale + bias*scale)*log2(e)
        // = acc * mul + add, and the logistic is 1 / (1 + 2^t) (logistic_exp2)
        float mul[CW], add[CW];
        // chain mode 2: y = (a - mean) * (rstd * gamma) + beta with the group's
        // finished statistics, the same three roundings as the normalize pass
        float nmean[CHAIN ? CW : 1], nmul[CHAIN ? CW : 1], nadd[CHAIN ? CW : 1];
        int cur_g = -1, cur_n = -1;
        int j = 0;
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++j) {
            const IgTile tl = ig_tile(p, t);
            const int buf = j & 1;
            // after an abort nothing more will be committed: do not wait for it.
            // One lane per warp polls the barrier; the others wait at the shuffle.
            int have_l = 0;
            if (lane == 0) {
                have_l = !*(volatile int *)abort_flag && dev::mbar_wait_bounded(&accf[buf], (j >> 1) & 1);
                if (!have_l) atomicExch(&g_igemm_error, 1);
            }
            const bool have = __shfl_sync(0xffffffffu, have_l, 0) != 0;
            dev::tc_fence_after();
            const bool ok = have && !*(volatile int *)abort_flag;
            const int q = tl.q0 + m;
            const bool qvalid = q < p.Q;
            const int rows = ok ? min(p.TH, p.P - tl.p0) : 0;   // valid output rows of the tile
            // this thread's output column of row tl.p0, channel tl.g*kpg of image tl.n
            float *ybase = p.y + ((long long)tl.n * p.K + (long long)tl.g * p.kpg) * plane +
                           (long long)tl.p0 * p.Q + q;
            const uint32_t tbase = tmem + ((uint32_t)(lq * 32) << 16) + (uint32_t)buf * acc_cols;
#pragma unroll 1
            for (int c0 = cpart * PART; c0 < (cpart + 1) * PART; c0 += CW) {
                const bool new_g = !ONE || tl.g != cur_g;
                const bool new_n = new_g || tl.n != cur_n;
                if (new_g) {
#pragma unroll
                    for (int jj = 0; jj < CW; ++jj) {
                        const int k = tl.g * p.kpg + c0 + jj;
                        const float b = p.bias ? __ldg(p.bias + k) : 0.f;
                        if constexpr (CHAIN) {
                            const float sc = __ldg(p.scale + k);
                            mul[jj] = -sc * kLog2e;
                            add[jj] = -(b * sc) * kLog2e;
                        } else {
                            mul[jj] = p.aff_scale ? __ldg(p.aff_scale + k) : 1.f;
                            add[jj] = b;
                        }
                    }
                }
                float shift[GPC], s1[GPC], s2[GPC];
#pragma unroll
                for (int gg = 0; gg < GPC; ++gg) { shift[gg] = 0.f; s1[gg] = 0.f; s2[gg] = 0.f; }
                if constexpr (CHAIN) {
                    if (p.chain_mode == 2 && new_n) {
#pragma unroll
                        for (int jj = 0; jj < CW; ++jj) {
                            const int k = tl.g * p.kpg + c0 + jj;
                            const float2 st = p.gn_stats[(long long)tl.n * p.gn_groups + k / p.kgn];
                            nmean[jj] = st.x;
                            nmul[jj] = (float)((double)st.y * (double)__ldg(p.gamma + k));
                            nadd[jj] = __ldg(p.beta + k);
                        }
                    }
                }
                cur_g = tl.g;
                cur_n = tl.n;
                // output pointer of channel c0 in the current row; channels are `plane` apart
                float *yc = ybase + (long long)c0 * plane;
                // rows are processed two at a time so one TMEM load latency covers both
#pragma unroll 1
                for (int i = 0; i < p.TH; i += 2) {
                    float vv[2][CW];
                    const bool two = i + 1 < p.TH;
                    dev::tmem_ld_pair<CW>(tbase + (uint32_t)(i * NT + c0),
                                          tbase + (uint32_t)((i + (two ? 1 : 0)) * NT + c0), vv[0], vv[1]);
                    // read (the load has completed): clear for the tile after next
                    dev::tmem_st_zero<CW>(tbase + (uint32_t)(i * NT + c0));
                    if (two) dev::tmem_st_zero<CW>(tbase + (uint32_t)((i + 1) * NT + c0));
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (h == 1 && !two) break;
                        float *v = vv[h];
                        const bool rvalid = i + h < rows;            // warp-uniform
                        if constexpr (CHAIN) {
#pragma unroll
                            for (int jj = 0; jj < CW; ++jj) v[jj] = logistic_exp2(fmaf(v[jj], mul[jj], add[jj]));
                            if (p.chain_mode != 2 && rvalid && i + h == 0) {
#pragma unroll
                                for (int gg = 0; gg < GPC; ++gg) shift[gg] = __shfl_sync(0xffffffffu, v[gg * GW], 0);
                            }
                        } else {
#pragma unroll
                            for (int jj = 0; jj < CW; ++jj) v[jj] = fmaf(v[jj], mul[jj], add[jj]);
                            if (p.clamp) {
#pragma unroll
                                for (int jj = 0; jj < CW; ++jj) v[jj] = fminf(fmaxf(v[jj], p.lo), p.hi);
                            }
                        }
                        if (rvalid && qvalid) {
                            if constexpr (CHAIN) {
                                if (p.chain_mode == 2) {
#pragma unroll
                                    for (int jj = 0; jj < CW; ++jj) v[jj] = fmaf(v[jj] - nmean[jj], nmul[jj], nadd[jj]);
                                } else {
#pragma unroll
                                    for (int jj = 0; jj < CW; ++jj) {
                                        const float d = v[jj] - shift[jj / GW];
                                        s1[jj / GW] += d;
                                        s2[jj / GW] = fmaf(d, d, s2[jj / GW]);
                                    }
                                }
                            }
                            if (!CHAIN || p.chain_mode != 1) {   // mode 1 keeps only the statistics
                                float *yr = yc;
#pragma unroll
                                for (int jj = 0; jj < CW; ++jj, yr += plane) *yr = v[jj];
                            }
                        }
                        yc += p.Q;
                    }
                }
                if (c0 + CW >= (cpart + 1) * PART) {
                    // last TMEM read of this tile by this warp: hand the buffer back
                    // once the clearing stores have completed
                    dev::tmem_wait_st();
                    dev::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) dev::mbar_arrive(&acce[buf]);
                }
                if (CHAIN && p.chain_mode != 2) {
                    const unsigned vmask = __ballot_sync(0xffffffffu, qvalid);
                    const int cnt_i = __popc(vmask) * rows * GW;
                    // 1/count: FP32 reciprocal refined by one Newton step in FP64 (count < 2^24)
                    const double cnt = (double)cnt_i;
                    double inv = (double)__frcp_rn((float)cnt_i);
                    inv = inv * (2.0 - cnt * inv);
#pragma unroll
                    for (int gg = 0; gg < GPC; ++gg) {
                        double S1 = (double)s1[gg], S2 = (double)s2[gg];
#pragma unroll
                        for (int off = 16; off > 0; off >>= 1) {
                            S1 += __shfl_xor_sync(0xffffffffu, S1, off);
                            S2 += __shfl_xor_sync(0xffffffffu, S2, off);
                        }
                        if (lane == 0) {
                            const int k0 = tl.g * p.kpg + c0 + gg * GW;   // first channel of the fragment
                            const int G = k0 / p.kgn;
                            const int fr = fpg > 1 ? (k0 % p.kgn) / CW : 0;
                            const double mean = cnt_i > 0 ? (double)shift[gg] + S1 * inv : 0.0;
                            const double m2 = cnt_i > 0 ? fmax(S2 - S1 * S1 * inv, 0.0) : 0.0;
                            p.gn_part[((long long)tl.n * p.gn_groups + G) * p.slots + (tl.sp * 4 + lq) * fpg + fr] =
                                make_float4((float)cnt_i, (float)mean, (float)m2, 0.f);
                        }
                    }
                }
            }
        }
    }

    dev::tc_fence_before();
    __syncthreads();
    if (warp == 1) dev::tmem_dealloc(tmem, p.tmem_cols);
}

template <typename Kern, typename... Args>
cudaError_t launch_ex(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

template <int NT, int KGN, bool FUSED>
cudaError_t launch_nt(const IgemmParams &p, const TensorMap *tm, dim3 grid, size_t smem, cudaStream_t st) {
    auto kern = igemm_tf32x3_kernel<NT, KGN, FUSED>;
    // the shared-memory opt-in is per function and device: raise it to the
    // planner's ceiling once per device instead of on every launch
    static std::atomic<unsigned long long> opted{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    const unsigned long long bit = dev < 64 ? 1ull << dev : 0;
    if (!bit || !(opted.load(std::memory_order_acquire) & bit)) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        if (bit) opted.fetch_or(bit, std::memory_order_acq_rel);
    }
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
    return launch_ex(kern, grid, dim3(ig_threads(NT, FUSED)), smem, st, tm[0], tm[1], p);
}

template <int NT, bool FUSED>
cudaError_t launch_chain_nt(const IgemmParams &p, const TensorMap *tm, dim3 grid, size_t smem,
                            cudaStream_t st) {
    switch (p.kgn) {
        case 1: return launch_nt<NT, 1, FUSED>(p, tm, grid, smem, st);
        case 2: return launch_nt<NT, 2, FUSED>(p, tm, grid, smem, st);
        case 4: return launch_nt<NT, 4, FUSED>(p, tm, grid, smem, st);
        case 8: return launch_nt<NT, 8, FUSED>(p, tm, grid, smem, st);
        case 16: return launch_nt<NT, 16, FUSED>(p, tm, grid, smem, st);
        default:
            if (p.kgn % 16 == 0) return launch_nt<NT, 32, FUSED>(p, tm, grid, smem, st);
            return cudaErrorInvalidValue;
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
        }
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }();
    return fn;
}

}  // namespace

int igemm_supported_nt(int kpg) { return kpg == 32 || kpg == 64 || kpg == 128 || kpg == 256; }

size_t igemm_header_bytes(int nt, bool chain) { return ig_header(nt, chain); }

int igemm_partials_per_tile(int nt, int kgn) {
    const int cw = ig_chunk_width(nt);
    return 4 * (kgn > cw ? kgn / cw : 1);
}

int igemm_threads(int nt, bool fused) { return ig_threads(nt, fused); }

bool make_nc4hw4_tile_map(TensorMap *tm, const float *base, long long quads, int Hp, int Wp, int box_cols,
                          int box_rows) {
    auto fn = encode_fn();
    if (!fn || Wp % 16 != 0 || box_cols % 16 != 0 || box_cols / 16 > 256 || box_rows < 1 || box_rows > 256)
        return false;
    // [quads][Hp][Wp/16][64 floats]: 16 pixels x 4 channels per innermost row
    cuuint64_t dims[4] = {64, (cuuint64_t)Wp / 16, (cuuint64_t)Hp, (cuuint64_t)quads};
    cuuint64_t strides[3] = {256, (cuuint64_t)Wp * 16, (cuuint64_t)Wp * Hp * 16};
    cuuint32_t box[4] = {64, (cuuint32_t)box_cols / 16, (cuuint32_t)box_rows, 2};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(reinterpret_cast<CUtensorMap *>(tm), CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4,
                    const_cast<float *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

cudaError_t launch_split_x(const float *x, float *xh, float *xl, int N, int C, int H, int W, int pad_h, int pad_w,
                           int Hp, int Wp, cudaStream_t st) {
    const long long cells = (long long)N * (C / 8) * Hp * Wp;
    const long long blocks = std::min<long long>((cells + 255) / 256, 148LL * 64);
    return launch_ex(split_x_kernel, dim3((unsigned)blocks), dim3(256), 0, st, x, reinterpret_cast<float4 *>(xh),
                     reinterpret_cast<uint4 *>(xl), C / 8, H, W, pad_h, pad_w, Hp, Wp, cells);
}

cudaError_t launch_split_w(const float *w, float *wh, float *wl, int K, int cpg, int R, int S, int RF, int groups,
                           cudaStream_t st, int gp) {
    // groups, cpg: the GEMM's (packed) ones; the original groups hold cpg/gp channels
    const int kpg = K / groups;
    const int RP = (R + RF - 1) / RF * RF;
    const long long cells = (long long)groups * (cpg / 8) * RP * S * kpg;
    const long long blocks = std::min<long long>((cells + 255) / 256, 148LL * 8);
    return launch_ex(split_w_kernel, dim3((unsigned)blocks), dim3(256), 0, st, w, reinterpret_cast<float4 *>(wh),
                     reinterpret_cast<uint4 *>(wl), kpg, cpg, R, S, RF, cells, gp, kpg / gp, cpg / gp);
}

cudaError_t launch_igemm(const IgemmParams &p, const TensorMap *tm, int chain, dim3 grid, size_t smem,
                         cudaStream_t st) {
    if (p.fused) {   // N = 32 only
        if (p.kpg != 32) return cudaErrorInvalidValue;
        return chain ? launch_chain_nt<32, true>(p, tm, grid, smem, st) : launch_nt<32, 0, true>(p, tm, grid, smem, st);
    }
    if (chain) {
        switch (p.kpg) {
            case 32: return launch_chain_nt<32, false>(p, tm, grid, smem, st);
            case 64: return launch_chain_nt<64, false>(p, tm, grid, smem, st);
            default: return cudaErrorInvalidValue;
        }
    }
    switch (p.kpg) {
        case 32: return launch_nt<32, 0, false>(p, tm, grid, smem, st);
        case 64: return launch_nt<64, 0, false>(p, tm, grid, smem, st);
        case 128: return launch_nt<128, 0, false>(p, tm, grid, smem, st);
        case 256: return launch_nt<256, 0, false>(p, tm, grid, smem, st);
        default: return cudaErrorInvalidValue;
    }
}

int igemm_fused_th() { return kFusedTH; }
int igemm_fold_rf(int nt, int R) { return ig_fold_rf(nt, R); }

int read_and_clear_igemm_error() {
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_igemm_error, sizeof(int)) != cudaSuccess) return -1;
    if (v) cudaMemcpyToSymbol(g_igemm_error, &zero, sizeof(int));
    return v;
}

}  // namespace gconv
