// Implicit-GEMM convolution on the 5th-generation tensor cores (tcgen05) with
// 3xTF32 splitting, for stride-1 dense and wide-group convolutions.
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
// Data layout.  A prep pass writes x_hi as NC4HW4 ([n][c/4][h][w][4]: four
// consecutive channels in one 16-byte cell) and the bf16 cross-term operand
// as [n][c/8][2][h][w][8] (same cell geometry), and the weights split the
// same way as [g][c/8][r][s][2][kpg][4 tf32 | 8 bf16].  In the NC4HW4 tile a CTA stages
// ([2 channel quads][rows][cols][4]), consecutive output pixels of one row
// are 16 bytes apart, which is exactly a K-major, no-swizzle UMMA operand
// with 8-row core matrices (SBO = 128 B) whose two K halves are one channel
// quad apart (LBO).  The operand for filter tap (r, s) is therefore the same
// staged tile with its start address moved by (row r*dil, column s*dil): the
// im2col matrix is never materialised, and every staged element feeds S
// taps of MMAs.
//
// Pipeline (one CTA = one image n, TH output rows x 128 output columns, all
// kpg output channels of group g):
//   warp 0 lane 0 : producer - per K-stage (8 input channels, one tap row r)
//                   two 4-D TMA loads (x_hi, x_lo tiles, zero fill supplies
//                   the padding) and two bulk copies (w_hi, w_lo slices) into
//                   a ring of shared-memory stages, signalled on mbarriers;
//   warp 1 lane 0 : MMA issuer - for every output row i and tap s, three
//                   tcgen05.mma (M=128, N=kpg, K=8) into the row's TMEM
//                   accumulator; tcgen05.commit frees the stage;
//   all 8 warps   : epilogue - tcgen05.ld of the accumulators (warp w reads
//                   TMEM lanes 32*(w%4).. and half of the columns), +bias, or
//                   the chain's +bias, *scale, logistic and GroupNorm partial
//                   statistics, coalesced stores along q.
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

// x[N][C][H][W] -> per 8 input channels (octet c8) and pixel:
//   xh: tf32 parts in NC4HW4 cells, [n][2*c8 + q][h][w][4]  (q = channel quad)
//   xc: bf16 parts, [n][c8][2][h][w][8]: chunk 0 = bf16(x_hi), chunk 1 = bf16(x - x_hi)
// Both tensors have the same geometry when read as 32-bit words.
__global__ void __launch_bounds__(256) split_x_kernel(const float *__restrict__ x, float4 *__restrict__ xh,
                                                      uint4 *__restrict__ xc, int C8, int H, int W,
                                                      long long cells) {
    dev::griddep_wait();
    dev::griddep_launch_dependents();
    const long long HW = (long long)H * W;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < cells;
         i += (long long)gridDim.x * blockDim.x) {
        const long long pix = i % HW;          // h*W + w
        const long long nc8 = i / HW;          // n*C8 + c8
        const float *src = x + nc8 * 8 * HW + pix;
        float hi[8], lo[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float v = __ldg(src + j * HW);
            hi[j] = dev::to_tf32(v);
            lo[j] = v - hi[j];
        }
        const long long q0 = (nc8 * 2) * HW + pix;   // cell index of quad 0 (and of chunk 0)
        xh[q0] = make_float4(hi[0], hi[1], hi[2], hi[3]);
        xh[q0 + HW] = make_float4(hi[4], hi[5], hi[6], hi[7]);
        xc[q0] = make_uint4(pack_bf16x2(hi[0], hi[1]), pack_bf16x2(hi[2], hi[3]), pack_bf16x2(hi[4], hi[5]),
                            pack_bf16x2(hi[6], hi[7]));
        xc[q0 + HW] = make_uint4(pack_bf16x2(lo[0], lo[1]), pack_bf16x2(lo[2], lo[3]), pack_bf16x2(lo[4], lo[5]),
                                 pack_bf16x2(lo[6], lo[7]));
    }
}

// w[K][cpg][R][S] -> per (g, c8, r, s, output channel kk), 8 input channels:
//   wh: [g][c8][r][s][2][kpg][4]   tf32 parts (two channel quads)
//   wc: [g][c8][r][s][2][kpg][8]   bf16 parts: chunk 0 = bf16(w - w_hi), chunk 1 = bf16(w_hi)
// so that the bf16 MMA over K = 16 computes x_hi*w_lo + x_lo*w_hi.
__global__ void __launch_bounds__(256) split_w_kernel(const float *__restrict__ w, float4 *__restrict__ wh,
                                                      uint4 *__restrict__ wc, int kpg, int cpg, int R, int S,
                                                      long long cells) {
    dev::griddep_wait();
    dev::griddep_launch_dependents();
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < cells;
         i += (long long)gridDim.x * blockDim.x) {
        long long t = i;
        const int kk = (int)(t % kpg); t /= kpg;
        const int s = (int)(t % S); t /= S;
        const int r = (int)(t % R); t /= R;
        const int c8 = (int)(t % (cpg / 8));
        const long long g = t / (cpg / 8);
        const long long k = g * kpg + kk;
        float hi[8], lo[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float v = __ldg(w + ((k * cpg + c8 * 8 + j) * R + r) * S + s);
            hi[j] = dev::to_tf32(v);
            lo[j] = v - hi[j];
        }
        // slot of (g, c8, r, s): [2][kpg] cells
        const long long base = ((((g * (cpg / 8) + c8) * R + r) * S + s) * 2) * kpg + kk;
        wh[base] = make_float4(hi[0], hi[1], hi[2], hi[3]);
        wh[base + kpg] = make_float4(hi[4], hi[5], hi[6], hi[7]);
        wc[base] = make_uint4(pack_bf16x2(lo[0], lo[1]), pack_bf16x2(lo[2], lo[3]), pack_bf16x2(lo[4], lo[5]),
                              pack_bf16x2(lo[6], lo[7]));
        wc[base + kpg] = make_uint4(pack_bf16x2(hi[0], hi[1]), pack_bf16x2(hi[2], hi[3]), pack_bf16x2(hi[4], hi[5]),
                                    pack_bf16x2(hi[6], hi[7]));
    }
}

// Epilogue warps: 16 (4 per TMEM lane quarter, 8-column chunks) for 32
// output channels, 8 (2 per lane quarter, 16-column chunks) for wider tiles,
// so the epilogue keeps enough warps in flight without spilling registers.
__host__ __device__ constexpr int ig_epi_warps(int NT) { return NT <= 32 ? 16 : 8; }
__host__ __device__ constexpr int ig_threads(int NT) { return 64 + 32 * ig_epi_warps(NT); }
// shared memory ahead of the stage ring: barriers, TMEM slot and, for the
// chain, per-fragment statistics [NT fragments at most][4 lane quarters][3 doubles]
__host__ __device__ constexpr int ig_header(int NT, bool chain) {
    return chain ? (256 + 96 * NT + 1023) / 1024 * 1024 : 1024;
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(dev::smem_addr(bar)) : "memory");
}

// Named barrier over the epilogue warps only.
template <int EPW>
__device__ __forceinline__ void epi_sync() {
    asm volatile("bar.sync 1, %0;\n" ::"r"(32 * EPW) : "memory");
}

// Output tile t -> (n, g, row tile, column tile); column tiles vary fastest so
// CTAs running side by side share input rows in L2.
struct IgTile {
    int n, g, p0, q0, sp;
};

__device__ __forceinline__ IgTile ig_tile(const IgemmParams &p, int t) {
    IgTile r;
    const int nsp = p.n_qt * p.n_pt;
    r.sp = t % nsp;
    const int rest = t / nsp;
    r.g = rest % p.groups;
    r.n = rest / p.groups;
    r.q0 = (r.sp % p.n_qt) * 128;
    r.p0 = (r.sp / p.n_qt) * p.TH;
    return r;
}

// ------------------------------------------------------------------ main kernel
// Persistent: CTA b processes tiles b, b + gridDim.x, ...  The producer and
// the MMA issuer run ahead through a ring of shared-memory stages; the MMA
// issuer alternates between two TMEM accumulator buffers so the epilogue of
// tile j overlaps the MMAs of tile j+1.
// KGN: 0 = plain convolution; otherwise the GroupNorm group width of the
// chain (1, 2, 4, 8, 16, or 32 standing for any multiple of 16).
template <int NT, int KGN>
__global__ void __launch_bounds__(ig_threads(NT), 1)
    igemm_tf32x3_kernel(const __grid_constant__ TensorMap tmh, const __grid_constant__ TensorMap tml,
                        const __grid_constant__ TensorMap tmh_tail, const __grid_constant__ TensorMap tml_tail,
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
    constexpr bool CHAIN = KGN > 0;
    double *st_n = reinterpret_cast<double *>(smem + 256);   // [fragment][4] chain statistics
    double *st_1 = st_n + NT * 4;
    double *st_2 = st_1 + NT * 4;
    unsigned char *stages = smem + ig_header(NT, CHAIN);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int num_tiles = p.n_tiles;
    const uint32_t a_slot = 2u * p.a_bytes;   // x_hi + x_lo tile of one channel step
    const uint32_t b_slot = 2u * p.b_bytes;   // w_hi + w_lo slice of one (channel step, tap row)
    unsigned char *ringA = stages;
    unsigned char *ringB = stages + (size_t)p.sa * a_slot;
    const uint32_t acc_cols = (uint32_t)(p.TH * NT);

    if (tid == 0) {
        for (int s = 0; s < 4; ++s) {
            dev::mbar_init(&fullA[s], 1);
            dev::mbar_init(&emptyA[s], 1);
            dev::mbar_init(&fullB[s], 1);
            dev::mbar_init(&emptyB[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            dev::mbar_init(&accf[b], 1);
            dev::mbar_init(&acce[b], ig_epi_warps(NT));
        }
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

    dev::griddep_wait();
    dev::griddep_launch_dependents();

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        // Per tile and 8-channel step: one x tile of AR = TH + (R-1)*dil rows
        // (hi and lo, exact-width boxes: 64-pixel boxes plus one tail box per
        // row) serving every tap row, then R weight slices (one per tap row).
        const int nmain = p.COLS / 64;
        const int tail = p.COLS - nmain * 64;               // pixels, multiple of 8
        const int per_row = nmain + (tail > 0 ? 1 : 0);
        const int boxes = 2 * 2 * p.AR * per_row;           // (hi, lo) x quads x rows x segments
        int ia = 0, ib = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
            const IgTile tl = ig_tile(p, t);
            const int z0 = tl.n * (p.C / 4) + tl.g * (p.cpg / 4);
            for (int cc8 = 0; cc8 < p.CC8 && ok; ++cc8, ++ia) {
                const int sa = ia % p.sa, ua = ia / p.sa;
                if (lane == 0) {
                    if (ua > 0 && !dev::mbar_wait_bounded(&emptyA[sa], (ua - 1) & 1)) ok = false;
                    if (*(volatile int *)abort_flag) ok = false;
                    if (ok) dev::mbar_arrive_expect_tx(&fullA[sa], a_slot);
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok) break;
                unsigned char *st = ringA + (size_t)sa * a_slot;
                const int x0 = tl.q0 - p.pad, y0 = tl.p0 - p.pad, cz = z0 + cc8 * 2;
                for (int b = lane; b < boxes; b += 32) {
                    const int seg = b % per_row;
                    int rest = b / per_row;
                    const int row = rest % p.AR; rest /= p.AR;
                    const int quad = rest & 1;
                    const int lo = rest >> 1;
                    const int px = seg * 64;
                    unsigned char *dst = st + lo * p.a_bytes + ((size_t)(quad * p.AR + row) * p.COLS + px) * 16;
                    const void *map = seg < nmain ? (lo ? (const void *)&tml : (const void *)&tmh)
                                                  : (lo ? (const void *)&tml_tail : (const void *)&tmh_tail);
                    dev::tma_load_3d(dst, map, &fullA[sa], (x0 + px) * 4, y0 + row, cz + quad);
                }
                for (int r = 0; r < p.R; ++r, ++ib) {
                    const int sb = ib % p.sb, ub = ib / p.sb;
                    if (lane == 0) {
                        if (ub > 0 && !dev::mbar_wait_bounded(&emptyB[sb], (ub - 1) & 1)) ok = false;
                        if (*(volatile int *)abort_flag) ok = false;
                        if (ok) {
                            dev::mbar_arrive_expect_tx(&fullB[sb], b_slot);
                            unsigned char *wb = ringB + (size_t)sb * b_slot;
                            const long long woff = (((long long)tl.g * p.CC8 + cc8) * p.R + r) * (p.b_bytes / 16);
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
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------------ MMA issuer
            constexpr uint32_t idesc = dev::idesc_tf32(128, NT);
            constexpr uint32_t idesc_c = dev::idesc_bf16(128, NT);
            const uint32_t a_lbo = (uint32_t)p.AR * p.COLS * 16;   // one channel quad / bf16 chunk apart
            const uint32_t b_lbo = NT * 16;
            int ia = 0, ib = 0, j = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++j) {
                const int buf = j & 1, ubuf = j >> 1;
                if (ubuf > 0 && !dev::mbar_wait_bounded(&acce[buf], (ubuf - 1) & 1)) {
                    ok = false;
                    break;
                }
                dev::tc_fence_after();
                const uint32_t dbase = tmem + (uint32_t)buf * acc_cols;
                for (int cc8 = 0; cc8 < p.CC8 && ok; ++cc8, ++ia) {
                    const int sa = ia % p.sa;
                    if (!dev::mbar_wait_bounded(&fullA[sa], (ia / p.sa) & 1)) {
                        ok = false;
                        break;
                    }
                    dev::tc_fence_after();
                    const unsigned char *xa = ringA + (size_t)sa * a_slot;
                    const uint64_t dah = dev::smem_desc(xa, a_lbo, 128);
                    const uint64_t dal = dev::smem_desc(xa + p.a_bytes, a_lbo, 128);
                    for (int r = 0; r < p.R; ++r, ++ib) {
                        const int sb = ib % p.sb;
                        if (!dev::mbar_wait_bounded(&fullB[sb], (ib / p.sb) & 1)) {
                            ok = false;
                            break;
                        }
                        dev::tc_fence_after();
                        const unsigned char *wb = ringB + (size_t)sb * b_slot;
                        const uint64_t dbh = dev::smem_desc(wb, b_lbo, 128);
                        const uint64_t dbl = dev::smem_desc(wb + p.b_bytes, b_lbo, 128);
                        for (int i = 0; i < p.TH; ++i) {
                            const uint32_t d = dbase + (uint32_t)(i * NT);
                            for (int s = 0; s < p.S; ++s) {
                                // 16-byte units: staged row i + r*dil, column s*dil
                                const uint64_t ao = (uint64_t)((i + r * p.dil) * p.COLS + s * p.dil);
                                const uint64_t bo = (uint64_t)(s * 2 * NT);
                                const uint32_t acc = (cc8 > 0 || r > 0 || s > 0) ? 1u : 0u;
                                // cross terms x_hi*w_lo + x_lo*w_hi: one bf16 MMA over K = 16
                                dev::mma_bf16(d, dal + ao, dbl + bo, idesc_c, acc);
                                // main term x_hi*w_hi: tf32 MMA over K = 8
                                dev::mma_tf32(d, dah + ao, dbh + bo, idesc, 1u);
                            }
                        }
                        dev::mma_commit(&emptyB[sb]);
                    }
                    dev::mma_commit(&emptyA[sa]);
                }
                dev::mma_commit(&accf[buf]);   // fires once this tile's MMAs have completed
            }
            if (!ok) {
                *abort_flag = 1;
                atomicExch(&g_igemm_error, 1);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------- epilogue
        // columns: each warp owns NT/4 accumulator columns of its lane quarter,
        // processed in chunks of CW; chain: GroupNorm groups per chunk (GPC)
        // and their width inside it (GW)
        constexpr int EPW = ig_epi_warps(NT);
        constexpr int PART = NT / (EPW / 4);
        constexpr int CW = PART < 16 ? PART : 16;
        constexpr int GPC = CHAIN ? (KGN >= CW ? 1 : CW / KGN) : 1;
        constexpr int GW = CHAIN ? (KGN >= CW ? CW : KGN) : CW;
        const int ew = warp - 2;                 // 0..EPW-1
        const int lq = warp & 3;                 // TMEM lane quarter this warp may access
        const int cpart = ew >> 2;               // column block of this warp
        const int m = lq * 32 + lane;
        const long long plane = (long long)p.P * p.Q;
        int j = 0;
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++j) {
            const IgTile tl = ig_tile(p, t);
            const int buf = j & 1;
            // after an abort nothing more will be committed: do not wait for it
            const bool have = !*(volatile int *)abort_flag && dev::mbar_wait_bounded(&accf[buf], (j >> 1) & 1);
            if (!have) atomicExch(&g_igemm_error, 1);
            dev::tc_fence_after();
            const bool ok = have && !*(volatile int *)abort_flag;
            const int q = tl.q0 + m;
            const bool qvalid = q < p.Q;
            float *ybase = p.y + ((long long)tl.n * p.K + (long long)tl.g * p.kpg) * plane + q;
            const uint32_t tbase = tmem + ((uint32_t)(lq * 32) << 16) + (uint32_t)buf * acc_cols;
#pragma unroll 1
            for (int c0 = cpart * PART; c0 < (cpart + 1) * PART; c0 += CW) {
                // z = acc * mul + add: plain (mul 1, add bias) or chain (scale, bias*scale)
                float mul[CW], add[CW];
#pragma unroll
                for (int jj = 0; jj < CW; ++jj) {
                    const int k = tl.g * p.kpg + c0 + jj;
                    const float b = p.bias ? __ldg(p.bias + k) : 0.f;
                    mul[jj] = CHAIN ? __ldg(p.scale + k) : 1.f;
                    add[jj] = CHAIN ? b * mul[jj] : b;
                }
                // shifted sums per GroupNorm group of this chunk (shift = the
                // group's first value seen by this thread)
                float shift[GPC], s1[GPC], s2[GPC];
                float cnt = 0.f;
#pragma unroll
                for (int gg = 0; gg < GPC; ++gg) { shift[gg] = 0.f; s1[gg] = 0.f; s2[gg] = 0.f; }
                // rows are processed two at a time so one TMEM load latency covers both
#pragma unroll 1
                for (int i = 0; i < p.TH; i += 2) {
                    float vv[2][CW];
                    const bool two = i + 1 < p.TH;
                    dev::tmem_ld_pair<CW>(tbase + (uint32_t)(i * NT + c0),
                                          tbase + (uint32_t)((i + (two ? 1 : 0)) * NT + c0), vv[0], vv[1]);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (h == 1 && !two) break;
                        float *v = vv[h];
                        const int pp = tl.p0 + i + h;
                        const bool valid = ok && qvalid && pp < p.P;
#pragma unroll
                        for (int jj = 0; jj < CW; ++jj) {
                            float z = fmaf(v[jj], mul[jj], add[jj]);
                            // logistic; the clamp keeps 1 + e finite (e^80 < 2^126)
                            if constexpr (CHAIN) z = __fdividef(1.f, 1.f + __expf(fminf(-z, 80.f)));
                            v[jj] = z;
                        }
                        if (valid) {
                            float *yr = ybase + (long long)c0 * plane + (long long)pp * p.Q;
#pragma unroll
                            for (int jj = 0; jj < CW; ++jj) yr[(long long)jj * plane] = v[jj];
                            if constexpr (CHAIN) {
                                if (cnt == 0.f) {
#pragma unroll
                                    for (int gg = 0; gg < GPC; ++gg) shift[gg] = v[gg * GW];
                                }
                                cnt += 1.f;
#pragma unroll
                                for (int jj = 0; jj < CW; ++jj) {
                                    const float d = v[jj] - shift[jj / GW];
                                    s1[jj / GW] += d;
                                    s2[jj / GW] = fmaf(d, d, s2[jj / GW]);
                                }
                            }
                        }
                    }
                }
                if (c0 + CW >= (cpart + 1) * PART) {
                    // last TMEM read of this tile by this warp: hand the buffer back
                    dev::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&acce[buf]);
                }
                if constexpr (CHAIN) {
                    // per GroupNorm group in this chunk: raw sums (n, sum a, sum a^2) in
                    // double, combined over the thread's channels, then a fixed
                    // shuffle tree over the warp's 32 pixels
#pragma unroll
                    for (int gg = 0; gg < GPC; ++gg) {
                        double S1 = 0.0, S2 = 0.0;
                        if (cnt > 0.f) {
                            const double n = (double)cnt * GW;
                            const double a1 = (double)s1[gg];
                            const double mu = (double)shift[gg] + a1 / n;
                            const double m2 = fmax((double)s2[gg] - a1 * a1 / n, 0.0);
                            S1 = n * mu;
                            S2 = m2 + n * mu * mu;
                        }
                        double Nn = (double)cnt * GW;
#pragma unroll
                        for (int off = 16; off > 0; off >>= 1) {
                            const double o1 = __shfl_down_sync(0xffffffffu, S1, off);
                            const double o2 = __shfl_down_sync(0xffffffffu, S2, off);
                            const double on = __shfl_down_sync(0xffffffffu, Nn, off);
                            if (lane < off) { S1 += o1; S2 += o2; Nn += on; }
                        }
                        if (lane == 0) {
                            const int fr = (c0 / CW) * GPC + gg;
                            st_n[fr * 4 + lq] = Nn;
                            st_1[fr * 4 + lq] = S1;
                            st_2[fr * 4 + lq] = S2;
                        }
                    }
                }
            }
            if constexpr (CHAIN) {
                epi_sync<EPW>();
                const int et = tid - 64;
                const int ngroups = NT / p.kgn;
                if (et < ngroups) {
                    // fragments of group et: one per group (width <= CW) or kgn/CW chunks
                    const int f0 = p.kgn > CW ? et * (p.kgn / CW) : et;
                    const int f1 = p.kgn > CW ? (et + 1) * (p.kgn / CW) : et + 1;
                    double Nn = 0.0, S1 = 0.0, S2 = 0.0;
                    for (int fr = f0; fr < f1; ++fr)
                        for (int l = 0; l < 4; ++l) {
                            Nn += st_n[fr * 4 + l];
                            S1 += st_1[fr * 4 + l];
                            S2 += st_2[fr * 4 + l];
                        }
                    const double mean = Nn > 0.0 ? S1 / Nn : 0.0;
                    const double m2 = Nn > 0.0 ? fmax(S2 - S1 * mean, 0.0) : 0.0;
                    const int G = (tl.g * p.kpg) / p.kgn + et;
                    p.gn_part[((long long)tl.n * p.gn_groups + G) * p.slots + tl.sp] =
                        make_float4((float)Nn, (float)mean, (float)m2, 0.f);
                }
                epi_sync<EPW>();   // statistics scratch free for the next tile
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

template <int NT, int KGN>
cudaError_t launch_nt(const IgemmParams &p, const TensorMap *tm, dim3 grid, size_t smem, cudaStream_t st) {
    auto kern = igemm_tf32x3_kernel<NT, KGN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_ex(kern, grid, dim3(ig_threads(NT)), smem, st, tm[0], tm[1], tm[2], tm[3], p);
}

template <int NT>
cudaError_t launch_chain_nt(const IgemmParams &p, const TensorMap *tm, dim3 grid, size_t smem,
                            cudaStream_t st) {
    switch (p.kgn) {
        case 1: return launch_nt<NT, 1>(p, tm, grid, smem, st);
        case 2: return launch_nt<NT, 2>(p, tm, grid, smem, st);
        case 4: return launch_nt<NT, 4>(p, tm, grid, smem, st);
        case 8: return launch_nt<NT, 8>(p, tm, grid, smem, st);
        case 16: return launch_nt<NT, 16>(p, tm, grid, smem, st);
        default:
            if (p.kgn % 16 == 0) return launch_nt<NT, 32>(p, tm, grid, smem, st);
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

int igemm_threads(int nt) { return ig_threads(nt); }

bool make_nc4hw4_tensor_map(TensorMap *tm, const float *base, long long quads, int H, int W, int box_px) {
    auto fn = encode_fn();
    if (!fn || box_px <= 0 || box_px > 64) return false;
    // [quads][H][W*4] floats; box = box_px pixels x 4 channels of one row of one quad
    cuuint64_t dims[3] = {(cuuint64_t)W * 4, (cuuint64_t)H, (cuuint64_t)quads};
    cuuint64_t strides[2] = {(cuuint64_t)W * 16, (cuuint64_t)W * H * 16};
    cuuint32_t box[3] = {(cuuint32_t)box_px * 4, 1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(reinterpret_cast<CUtensorMap *>(tm), CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
                    const_cast<float *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

cudaError_t launch_split_x(const float *x, float *xh, float *xl, int N, int C, int H, int W, cudaStream_t st) {
    const long long cells = (long long)N * (C / 8) * H * W;
    const long long blocks = std::min<long long>((cells + 255) / 256, 148LL * 64);
    return launch_ex(split_x_kernel, dim3((unsigned)blocks), dim3(256), 0, st, x, reinterpret_cast<float4 *>(xh),
                     reinterpret_cast<uint4 *>(xl), C / 8, H, W, cells);
}

cudaError_t launch_split_w(const float *w, float *wh, float *wl, int K, int cpg, int R, int S, int groups,
                           cudaStream_t st) {
    const int kpg = K / groups;
    const long long cells = (long long)groups * (cpg / 8) * R * S * kpg;
    const long long blocks = std::min<long long>((cells + 255) / 256, 148LL * 8);
    return launch_ex(split_w_kernel, dim3((unsigned)blocks), dim3(256), 0, st, w, reinterpret_cast<float4 *>(wh),
                     reinterpret_cast<uint4 *>(wl), kpg, cpg, R, S, cells);
}

cudaError_t launch_igemm(const IgemmParams &p, const TensorMap *tm, int chain, dim3 grid, size_t smem,
                         cudaStream_t st) {
    if (chain) {
        switch (p.kpg) {
            case 32: return launch_chain_nt<32>(p, tm, grid, smem, st);
            case 64: return launch_chain_nt<64>(p, tm, grid, smem, st);
            default: return cudaErrorInvalidValue;
        }
    }
    switch (p.kpg) {
        case 32: return launch_nt<32, 0>(p, tm, grid, smem, st);
        case 64: return launch_nt<64, 0>(p, tm, grid, smem, st);
        case 128: return launch_nt<128, 0>(p, tm, grid, smem, st);
        case 256: return launch_nt<256, 0>(p, tm, grid, smem, st);
        default: return cudaErrorInvalidValue;
    }
}

int read_and_clear_igemm_error() {
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_igemm_error, sizeof(int)) != cudaSuccess) return -1;
    if (v) cudaMemcpyToSymbol(g_igemm_error, &zero, sizeof(int));
    return v;
}

}  // namespace gconv
