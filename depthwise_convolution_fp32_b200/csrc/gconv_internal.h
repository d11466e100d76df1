// Internal declarations shared by the host dispatcher and the kernels of
// libgconv.so.  Not part of the public ABI (include/gconv.h is).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace gconv {

// Compile-time geometry a fast direct-kernel variant is specialised for.
// The generic variant (id kDirectGeneric) takes every size at run time.
enum DirectVariantGeom : int {
    kGeom3x3s1p1 = 0,   // 3x3, stride 1, pad 1, dilation 1 (Atlas sweep, depthwise)
    kGeom3x3s1p0 = 1,   // 3x3, stride 1, pad 0, dilation 1 (fused-chain conv)
    kGeom3x3s2p1 = 2,   // 3x3, stride 2, pad 1, dilation 1 (downsampling depthwise)
    kGeom5x9s1p0 = 3,   // 5x9, stride 1, pad 0, dilation 1 (dense asymmetric conv)
    kGeom1x1s1p0 = 4,   // pointwise
    kGeomCount = 5,
    kDirectGeneric = 99
};

// Everything one launch of the direct kernel needs.  The host fills it; the
// kernel derives its tile from blockIdx / threadIdx.
struct DirectParams {
    const float *x, *w, *bias;  // inputs (bias may be null)
    float *y;                   // output [N,K,P,Q]
    const float *scale;         // chain only: [K]
    float4 *gn_part;            // chain only: [N*gn_groups][slots] (count, mean, M2, 0)

    int N, C, H, W, K, R, S, stride, pad, dil, groups;   // stride, pad, dil: H axis
    int cpg, kpg, P, Q;
    int sw, pw, dw;   // W-axis stride, padding, dilation (the specialised variants need them equal to H's)

    // CTA tile: CX chunk-columns of 4 outputs, RY row strips of RPT rows,
    // KZ channel slices of KT channels, GB conv groups.
    int CX, RY, KZ, GB;
    int TP, TQ;       // output rows / cols per CTA
    int KB;           // output channels per CTA inside one conv group (KZ*KT)
    int KBtot;        // channels per CTA (GB*KB; GB > 1 only when KB == kpg)
    int n_qt, n_pt, n_kb;
    int IHt;          // staged input rows per plane
    int PC;           // staged 16-byte chunks per row
    int pitch;        // floats per staged row (>= 4*PC)
    int cchunk;       // input channels staged per pass
    int w_floats;     // floats reserved for the weight slice (multiple of 4)
    int vec_in;       // x rows are 16-byte aligned (16-byte cp.async staging)
    int vec2_in;      // else: W even and x 8-byte aligned (8-byte cp.async staging)
    int vec_out;      // y rows are 16-byte aligned (float4 stores)

    // TMA staging (tma != 0): the tile's rows are fetched as nb bands of bh
    // rows, one 3-D box (4*PC columns x bh rows x 1 plane) per band and plane,
    // each band completing on its own mbarrier.  Requires cchunk == cpg.
    int tma;
    int nb, bh;
    int x_off;        // float offset of the x tile in shared memory
    int pstride;      // floats between staged planes

    // streaming variant (persistent CTAs over a ring of stages; plain and
    // affine epilogues): a work item is one CTA tile of the blocked kernel,
    // staged by ONE 3-D TMA box of 4*PC columns x IHt rows x GB*cpg planes
    int n_items;      // N * (groups/GB) * n_kb * n_pt * n_qt
    int stages;       // ring depth
    int stage_floats; // floats per stage: x planes, then the weight slice (multiple of 32)
    int sw_off;       // float offset of the weight slice inside a stage
    int CXP;          // threads per row strip: CX, rounded up to 8 when CX > 4 so that no
                      // quarter-warp's 128-bit shared loads straddle two row strips

    // chain bookkeeping
    int gn_groups, kgn, slots, slots_k, n_sp;

    // plain convolution epilogue: y = clamp(acc * aff_scale[k] + bias[k], lo, hi)
    const float *aff_scale;   // null: 1
    int clamp;                // apply [lo, hi]
    float lo, hi;
};

struct GnParams {
    float *y;
    const float4 *gn_part;
    float2 *stats;    // [N*gn_groups] (mean, rstd)
    const float *gamma, *beta;
    int N, K, gn_groups, kgn, slots;
    long long PQ;
    float eps;
    int chunks;       // CTAs per channel plane in the normalise pass
    int vec;          // float4 path allowed
};

// Opaque 128-byte TMA descriptor (CUtensorMap) storage.
struct alignas(64) TensorMap {
    unsigned char bytes[128];
};

// Encode a 3-D tensor map over x viewed as [N*C][H][W] with a box of
// box_w x box_h x 1 elements (zero fill out of bounds).  Returns false when
// the driver entry point is unavailable or rejects the map.
bool make_x_tensor_map(TensorMap *tm, const float *x, long long planes, int H, int W, int box_w, int box_h,
                       int box_planes = 1);

// Launch one direct-kernel variant (programmatic dependent launch enabled);
// returns the launch status.
cudaError_t launch_direct(const DirectParams &p, const TensorMap &tm, int geom, int KT, int chain,
                          dim3 grid, int threads, size_t smem, cudaStream_t stream);

// Streaming direct kernel: threads = compute threads + one producer warp.
// The grid is min(work items, sms x resident CTAs per SM), the occupancy
// being queried once per variant, block size, shared memory and device.
cudaError_t launch_direct_stream(const DirectParams &p, const TensorMap &tm, int geom, int KT, int sms,
                                 int threads, size_t smem, cudaStream_t stream);
// Shared memory ahead of the stages: full[8] and empty[8] barriers (128 B), two
// flags (8 B), then 8 per-stage item records (int4 at byte 144); stages start
// 128-byte aligned after it.
constexpr int kStreamHeaderBytes = 512;

// Device error flag raised by bounded waits that gave up (0 = none); reading
// clears it.  Synchronises with the device.
int read_and_clear_device_error();
// One CTA whose bounded mbarrier wait runs out after `spins` polls (raises the flag).
cudaError_t launch_wait_timeout_probe(unsigned spins, cudaStream_t stream);
int direct_rpt(int KT);   // rows per thread the variant with KT uses
int direct_fast_window_chunks(int geom);   // 16-byte chunks one thread reads per row

// ---- Winograd F(2x2, 3x3) on the CUDA cores ---------------------------------
struct WinoParams {
    const float *x, *w, *bias;
    float *y;
    const float *aff_scale;   // affine + clamp epilogue: null = 1
    int clamp;
    float lo, hi;
    int N, C, H, W, K, P, Q, pad, cpg, kpg, groups;
    int TX, TY;               // Winograd tiles (2x2 outputs) per CTA along q and p
    int KZ, KB;               // channel slices of KT per CTA, KB = KZ*KT output channels
    int n_qt, n_pt, n_kb;
    int pitch;                // floats per staged row (2*TX + 2)
    int u_floats;             // floats of the transformed filters [cpg][16][KB]
    int vec_out;              // y rows 8-byte aligned and Q even: float2 stores
};
cudaError_t launch_winograd(const WinoParams &p, int KT, dim3 grid, int threads, size_t smem, cudaStream_t st);

// ---- implicit GEMM on tcgen05 (tf32 main term + bf16 cross terms) ----------
struct IgemmParams {
    const float4 *wh, *wl;     // split weights [g][cpg/8][RC][s][2][RF][kpg][4], tap rows of a chunk descending
    const float *bias, *scale; // bias may be null; scale only for the chain
    float *y;
    float4 *gn_part;           // chain only
    int N, C, H, W, K, R, S, pad, dil, groups, cpg, kpg, P, Q;   // pad, dil: H axis
    int pad_w, dil_w;          // W axis
    int CC8;                   // cpg / 8 (K-steps of 8 channels)
    int RF;                    // filter tap rows folded into the N extent of one MMA (dilation 1)
    int RC;                    // chunks of RF tap rows: ceil(R / RF); one weight slice each
    int bs;                    // 1: one weight slice per (chunk, tap column) instead (RF > 1 only)
    int TH;                    // output rows per tile (one 128-pixel M tile each)
    int AR;                    // staged x rows per channel step: TH + (R-1)*dil
    int COLS;                  // staged columns per row (>= 128 + (S-1)*dil, multiple of 16)
    int Hp, Wp;                // padded x planes of the split operands: pad rows on top, pad
                               // columns on the left, zero columns up to Wp (multiple of 16)
    int n_qt, n_pt;
    int n_tiles;               // N * groups * n_pt * n_qt
    int sa, sb;                // slots of the x-tile ring and of the weight-slice ring
    int b_resident;            // 1: all CC8*RC weight slices fit the ring and are loaded once per CTA
    int a_bytes, b_bytes;      // one x operand (hi or lo) tile / one w operand slice
    int tmem_cols;
    int gn_groups, kgn, slots;  // chain: partials per (image, group) = tiles per image x per-tile partials
    // plain convolution epilogue: y = clamp(acc * aff_scale[k] + bias[k], lo, hi)
    const float *aff_scale;    // null: 1
    int clamp;
    float lo, hi;
    // chain epilogue: 0 = store a + partial statistics; 1 = partial statistics
    // only; 2 = y = (a - mean) * rstd * gamma + beta from gn_stats, stored
    int chain_mode;
    const float2 *gn_stats;    // [N*gn_groups] (mean, rstd) for mode 2
    const float *gamma, *beta;
    // fused variant (N = 32, TH = igemm_fused_th()): x is staged raw by TMA
    // ([8 channels][AR rows][COLSR columns], tensor map over x itself) into a
    // ring of rr slots of raw_bytes and converted to the operand layout in
    // shared memory by converter warps; no split pass, no x workspace
    int fused;
    int COLSR, raw_bytes, rr;
};

int igemm_supported_nt(int kpg);
int igemm_fused_th();
int igemm_fold_rf(int nt, int R);   // tap rows one MMA covers when the plan folds them
size_t igemm_header_bytes(int nt, bool chain);
// GroupNorm partials the chain epilogue writes per tile and group (one per
// TMEM lane quarter and per channel chunk the group spans)
int igemm_partials_per_tile(int nt, int kgn);
int igemm_threads(int nt, bool fused);
// 4-D tensor map over a padded NC4HW4 tensor [quads][Hp][Wp][4] viewed as
// [quads][Hp][Wp/16][64 floats]; one box is a whole x tile of one channel
// step: 2 quads x box_rows rows x box_cols (multiple of 16) pixels.
bool make_nc4hw4_tile_map(TensorMap *tm, const float *base, long long quads, int Hp, int Wp, int box_cols,
                          int box_rows);
cudaError_t launch_split_x(const float *x, float *xh, float *xl, int N, int C, int H, int W, int pad_h, int pad_w,
                           int Hp, int Wp, cudaStream_t st);
// groups, cpg: the GEMM's; gp > 1 packs gp original groups into each (block-diagonal weights)
cudaError_t launch_split_w(const float *w, float *wh, float *wl, int K, int cpg, int R, int S, int RF, int groups,
                           cudaStream_t st, int gp = 1);
// tm: x_hi tile map, cross-term tile map
cudaError_t launch_igemm(const IgemmParams &p, const TensorMap *tm, int chain, dim3 grid, size_t smem,
                         cudaStream_t st);
int read_and_clear_igemm_error();

cudaError_t launch_gn_finalize(const GnParams &p, cudaStream_t stream);
cudaError_t launch_gn_normalize(const GnParams &p, cudaStream_t stream);

}  // namespace gconv
