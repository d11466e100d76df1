// Implicit-GEMM convolution on the 5th-generation tensor cores (tcgen05) with
// 3xTF32 splitting, for stride-1 dense and wide-group convolutions.
//
// What it computes (POPCORNBENCH "Kimi-K2.6__l1_p62" and "Kimi-K2.6__l2_p21":
// the convolution viewed as a GEMM with M = output pixels, N = output
// channels of a group, K = C/groups * R * S):
//   y[n,k,p,q] = bias[k] + sum_{c,r,s} w[k,c,r,s] * x[n, gi*cpg + c, p - pad + r*dil, q - pad + s*dil]
// in FP32 accuracy: every operand v is split into v_hi = tf32(v) and
// v_lo = v - v_hi (exact in FP32), and each product is accumulated as
// a_lo*b_hi + a_hi*b_lo + a_hi*b_hi in FP32 (the dropped a_lo*b_lo term is
// below 2^-22 of |a*b|).  TF32 on its own (2^-11 relative) would miss the
// 1e-5 * sum|w*x| bound; the pages flag TF32 as "not exactly fp32".
//
// Data layout.  A prep pass writes x_hi and x_lo as NC4HW4 ([n][c/4][h][w][4]:
// four consecutive channels in one 16-byte cell) and the weights, split the
// same way, as [g][c/8][r][s][2][kpg][4].  In the NC4HW4 tile a CTA stages
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

#include "device_utils.cuh"
#include "gconv_internal.h"

namespace gconv {

namespace {

__device__ int g_igemm_error = 0;

// ------------------------------------------------------------------ prep
__global__ void __launch_bounds__(256) split_x_kernel(const float *__restrict__ x, float4 *__restrict__ xh,
                                                      float4 *__restrict__ xl, int C4, int H, int W,
                                                      long long cells) {
    dev::griddep_wait();
    dev::griddep_launch_dependents();
    const long long HW = (long long)H * W;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < cells;
         i += (long long)gridDim.x * blockDim.x) {
        const long long pix = i % HW;          // h*W + w
        const long long nc4 = i / HW;          // n*C4 + c4
        const float *src = x + nc4 * 4 * HW + pix;
        float v[4], hi[4], lo[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[j] = __ldg(src + j * HW);
            hi[j] = dev::to_tf32(v[j]);
            lo[j] = v[j] - hi[j];
        }
        xh[i] = make_float4(hi[0], hi[1], hi[2], hi[3]);
        xl[i] = make_float4(lo[0], lo[1], lo[2], lo[3]);
    }
}

// w[K][cpg][R][S] -> [g][cpg/8][r][s][2][kpg][4] (hi and lo)
__global__ void __launch_bounds__(256) split_w_kernel(const float *__restrict__ w, float4 *__restrict__ wh,
                                                      float4 *__restrict__ wl, int kpg, int cpg, int R, int S,
                                                      long long cells) {
    dev::griddep_wait();
    dev::griddep_launch_dependents();
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < cells;
         i += (long long)gridDim.x * blockDim.x) {
        long long t = i;
        const int kk = (int)(t % kpg); t /= kpg;
        const int h2 = (int)(t % 2); t /= 2;
        const int s = (int)(t % S); t /= S;
        const int r = (int)(t % R); t /= R;
        const int cc8 = (int)(t % (cpg / 8));
        const long long g = t / (cpg / 8);
        const long long k = g * kpg + kk;
        float hi[4], lo[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = cc8 * 8 + h2 * 4 + j;
            const float v = __ldg(w + ((k * cpg + c) * R + r) * S + s);
            hi[j] = dev::to_tf32(v);
            lo[j] = v - hi[j];
        }
        wh[i] = make_float4(hi[0], hi[1], hi[2], hi[3]);
        wl[i] = make_float4(lo[0], lo[1], lo[2], lo[3]);
    }
}

// Chan et al. pairwise update of (count, mean, M2).
__device__ __forceinline__ void chan_merge(float &na, float &ma, float &m2a, float nb, float mb, float m2b) {
    if (nb == 0.f) return;
    if (na == 0.f) {
        na = nb; ma = mb; m2a = m2b;
        return;
    }
    float n = na + nb;
    float d = mb - ma;
    float f = nb / n;
    ma = fmaf(d, f, ma);
    m2a = m2a + m2b + d * d * na * f;
    na = n;
}

constexpr int kIgThreads = 256;
constexpr int kIgHeader = 1024;   // barriers and the TMEM address slot

// ------------------------------------------------------------------ main kernel
template <int NT, bool CHAIN>
__global__ void __launch_bounds__(kIgThreads, 2)
    igemm_tf32x3_kernel(const __grid_constant__ TensorMap tmh, const __grid_constant__ TensorMap tml,
                        const IgemmParams p) {
    extern __shared__ __align__(1024) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem);        // [stages]
    uint64_t *empty = full + 8;                                  // [stages]
    uint64_t *accf = full + 16;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(full + 17);
    int *abort_flag = reinterpret_cast<int *>(full + 18);
    unsigned char *stages = smem + kIgHeader;

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int qt = blockIdx.x % p.n_qt, pt = blockIdx.x / p.n_qt;
    const int g = blockIdx.y, n = blockIdx.z;
    const int q0 = qt * 128, p0 = pt * p.TH;
    const int num_k = p.CC8 * p.R;
    const uint32_t stage_bytes = 2u * p.a_bytes + 2u * p.b_bytes;

    if (tid == 0) {
        for (int s = 0; s < p.stages; ++s) {
            dev::mbar_init(&full[s], 1);
            dev::mbar_init(&empty[s], 1);
        }
        dev::mbar_init(accf, 1);
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

    if (warp == 0 && lane == 0) {
        // ---------------------------------------------------------- producer
        const int z0 = n * (p.C / 4) + g * (p.cpg / 4);
        for (int kt = 0; kt < num_k; ++kt) {
            const int slot = kt % p.stages;
            const int use = kt / p.stages;
            if (use > 0 && !dev::mbar_wait_bounded(&empty[slot], (use - 1) & 1)) {
                *abort_flag = 1;
                atomicExch(&g_igemm_error, 1);
                break;
            }
            const int cc8 = kt / p.R, r = kt - cc8 * p.R;
            unsigned char *st = stages + (size_t)slot * stage_bytes;
            dev::mbar_arrive_expect_tx(&full[slot], stage_bytes);
            const int cw = q0 - p.pad, ch = p0 - p.pad + r * p.dil, cz = z0 + cc8 * 2;
            dev::tma_load_4d(st, &tmh, &full[slot], 0, cw, ch, cz);
            dev::tma_load_4d(st + p.a_bytes, &tml, &full[slot], 0, cw, ch, cz);
            const long long woff = (((long long)g * p.CC8 + cc8) * p.R + r) * (p.b_bytes / 16);
            dev::bulk_load(st + 2 * p.a_bytes, p.wh + woff, p.b_bytes, &full[slot]);
            dev::bulk_load(st + 2 * p.a_bytes + p.b_bytes, p.wl + woff, p.b_bytes, &full[slot]);
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------------------------------------------------- MMA issuer
        constexpr uint32_t idesc = dev::idesc_tf32(128, NT);
        const uint32_t a_lbo = (uint32_t)p.TH * p.COLS * 16;
        const uint32_t b_lbo = NT * 16;
        bool ok = true;
        for (int kt = 0; kt < num_k && ok; ++kt) {
            const int slot = kt % p.stages;
            if (!dev::mbar_wait_bounded(&full[slot], (kt / p.stages) & 1)) {
                ok = false;
                *abort_flag = 1;
                atomicExch(&g_igemm_error, 1);
                break;
            }
            dev::tc_fence_after();
            const unsigned char *st = stages + (size_t)slot * stage_bytes;
            const unsigned char *ah = st, *al = st + p.a_bytes;
            const unsigned char *bh = st + 2 * p.a_bytes, *bl = bh + p.b_bytes;
            for (int i = 0; i < p.TH; ++i) {
                const uint32_t d = tmem + (uint32_t)(i * NT);
                for (int s = 0; s < p.S; ++s) {
                    const uint32_t ao = (uint32_t)(i * p.COLS + s * p.dil) * 16;
                    const uint32_t bo = (uint32_t)(s * 2 * NT) * 16;
                    const uint32_t acc = (kt > 0 || s > 0) ? 1u : 0u;
                    dev::mma_tf32(d, dev::smem_desc(al + ao, a_lbo, 128), dev::smem_desc(bh + bo, b_lbo, 128),
                                  idesc, acc);
                    dev::mma_tf32(d, dev::smem_desc(ah + ao, a_lbo, 128), dev::smem_desc(bl + bo, b_lbo, 128),
                                  idesc, 1u);
                    dev::mma_tf32(d, dev::smem_desc(ah + ao, a_lbo, 128), dev::smem_desc(bh + bo, b_lbo, 128),
                                  idesc, 1u);
                }
            }
            dev::mma_commit(&empty[slot]);
        }
        dev::mma_commit(accf);   // fires once every MMA above has completed
    }
    __syncwarp();

    // -------------------------------------------------------------- epilogue
    const bool have_acc = dev::mbar_wait_bounded(accf, 0);
    if (!have_acc) atomicExch(&g_igemm_error, 1);
    dev::tc_fence_after();
    const bool ok = have_acc && (*(volatile int *)abort_flag == 0);

    const int lq = warp & 3;            // TMEM lane quarter
    const int chalf = warp >> 2;        // column half
    constexpr int HALF = NT / 2;
    const int m = lq * 32 + lane;
    const int q = q0 + m;
    const bool qvalid = q < p.Q;
    const long long plane = (long long)p.P * p.Q;
    float *ybase = p.y + ((long long)n * p.K + (long long)g * p.kpg) * plane + q;

    // per-channel statistics of this warp (chain): [NT][4 lane quarters]
    float *st_n = reinterpret_cast<float *>(stages);
    float *st_m = st_n + NT * 4;
    float *st_q = st_m + NT * 4;

#pragma unroll 1
    for (int c0 = chalf * HALF; c0 < (chalf + 1) * HALF; c0 += 16) {
        float bias_v[16], sc_v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int k = g * p.kpg + c0 + j;
            bias_v[j] = p.bias ? __ldg(p.bias + k) : 0.f;
            sc_v[j] = CHAIN ? __ldg(p.scale + k) : 1.f;
        }
        float shift[16], s1[16], s2[16];
        float cnt = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) { shift[j] = 0.f; s1[j] = 0.f; s2[j] = 0.f; }
#pragma unroll 1
        for (int i = 0; i < p.TH; ++i) {
            float v[16];
            dev::tmem_ld16(tmem + ((uint32_t)(lq * 32) << 16) + (uint32_t)(i * NT + c0), v);
            const int pp = p0 + i;
            const bool valid = ok && qvalid && pp < p.P;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                float z = v[j] + bias_v[j];
                if constexpr (CHAIN) z = 1.f / (1.f + expf(-(z * sc_v[j])));
                v[j] = z;
            }
            if (valid) {
                float *yr = ybase + (long long)c0 * plane + (long long)pp * p.Q;
#pragma unroll
                for (int j = 0; j < 16; ++j) yr[(long long)j * plane] = v[j];
                if constexpr (CHAIN) {
                    if (cnt == 0.f) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) shift[j] = v[j];
                    }
                    cnt += 1.f;
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float d = v[j] - shift[j];
                        s1[j] += d;
                        s2[j] = fmaf(d, d, s2[j]);
                    }
                }
            }
        }
        if constexpr (CHAIN) {
            // per channel: thread (cnt, mean, M2) -> warp (fixed shuffle tree) -> shared memory
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                float cn = cnt, mn = 0.f, m2 = 0.f;
                if (cnt > 0.f) {
                    const float a = s1[j] / cnt;
                    mn = shift[j] + a;
                    m2 = fmaxf(s2[j] - s1[j] * a, 0.f);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    const float on = __shfl_down_sync(0xffffffffu, cn, off);
                    const float om = __shfl_down_sync(0xffffffffu, mn, off);
                    const float oq = __shfl_down_sync(0xffffffffu, m2, off);
                    if (lane < off) chan_merge(cn, mn, m2, on, om, oq);
                }
                if (lane == 0) {
                    // stage memory is free: every MMA reading it has completed
                    st_n[(c0 + j) * 4 + lq] = cn;
                    st_m[(c0 + j) * 4 + lq] = mn;
                    st_q[(c0 + j) * 4 + lq] = m2;
                }
            }
        }
    }

    if constexpr (CHAIN) {
        __syncthreads();
        const int ngroups = NT / p.kgn;
        if (tid < ngroups) {
            float cn = 0.f, mn = 0.f, m2 = 0.f;
            for (int c = tid * p.kgn; c < (tid + 1) * p.kgn; ++c)
                for (int l = 0; l < 4; ++l) chan_merge(cn, mn, m2, st_n[c * 4 + l], st_m[c * 4 + l], st_q[c * 4 + l]);
            const int G = (g * p.kpg) / p.kgn + tid;
            const int slot = pt * p.n_qt + qt;
            p.gn_part[((long long)n * p.gn_groups + G) * p.slots + slot] = make_float4(cn, mn, m2, 0.f);
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

template <int NT, bool CHAIN>
cudaError_t launch_nt(const IgemmParams &p, const TensorMap &tmh, const TensorMap &tml, dim3 grid, size_t smem,
                      cudaStream_t st) {
    auto kern = igemm_tf32x3_kernel<NT, CHAIN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_ex(kern, grid, dim3(kIgThreads), smem, st, tmh, tml, p);
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

size_t igemm_header_bytes() { return kIgHeader; }

bool make_nc4hw4_tensor_map(TensorMap *tm, const float *base, long long quads, int H, int W, int box_cols,
                            int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {4, (cuuint64_t)W, (cuuint64_t)H, (cuuint64_t)quads};
    cuuint64_t strides[3] = {16, (cuuint64_t)W * 16, (cuuint64_t)W * H * 16};
    cuuint32_t box[4] = {4, (cuuint32_t)box_cols, (cuuint32_t)box_rows, 2};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(reinterpret_cast<CUtensorMap *>(tm), CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4,
                    const_cast<float *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

cudaError_t launch_split_x(const float *x, float *xh, float *xl, int N, int C, int H, int W, cudaStream_t st) {
    const long long cells = (long long)N * (C / 4) * H * W;
    const long long blocks = std::min<long long>((cells + 255) / 256, 148LL * 64);
    return launch_ex(split_x_kernel, dim3((unsigned)blocks), dim3(256), 0, st, x, reinterpret_cast<float4 *>(xh),
                     reinterpret_cast<float4 *>(xl), C / 4, H, W, cells);
}

cudaError_t launch_split_w(const float *w, float *wh, float *wl, int K, int cpg, int R, int S, int groups,
                           cudaStream_t st) {
    const int kpg = K / groups;
    const long long cells = (long long)groups * (cpg / 8) * R * S * 2 * kpg;
    const long long blocks = std::min<long long>((cells + 255) / 256, 148LL * 8);
    return launch_ex(split_w_kernel, dim3((unsigned)blocks), dim3(256), 0, st, w, reinterpret_cast<float4 *>(wh),
                     reinterpret_cast<float4 *>(wl), kpg, cpg, R, S, cells);
}

cudaError_t launch_igemm(const IgemmParams &p, const TensorMap &tmh, const TensorMap &tml, int chain, dim3 grid,
                         size_t smem, cudaStream_t st) {
    switch (p.kpg) {
        case 32: return chain ? launch_nt<32, true>(p, tmh, tml, grid, smem, st)
                              : launch_nt<32, false>(p, tmh, tml, grid, smem, st);
        case 64: return chain ? launch_nt<64, true>(p, tmh, tml, grid, smem, st)
                              : launch_nt<64, false>(p, tmh, tml, grid, smem, st);
        case 128: return chain ? launch_nt<128, true>(p, tmh, tml, grid, smem, st)
                               : launch_nt<128, false>(p, tmh, tml, grid, smem, st);
        case 256: return chain ? launch_nt<256, true>(p, tmh, tml, grid, smem, st)
                               : launch_nt<256, false>(p, tmh, tml, grid, smem, st);
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
