// Winograd F(2x2, 3x3) convolution on the FP32 CUDA cores, for 3x3 kernels
// at stride 1 and dilation 1 (grouped or dense, any symmetric padding).
//
// What it computes is the same cross-correlation as the direct kernels
// ("GroupConv Atlas", "Fix the experiment"; POPCORNBENCH "Kimi-K2.6__l2_p21",
// the direct index formula input[n, ic, h+kh, w+kw] * weight[c, ic, kh, kw]),
// evaluated by the minimal-filtering algorithm F(2x2, 3x3) of Lavin and Gray,
// "Fast Algorithms for Convolutional Neural Networks" (2016) -- the method the
// chain transcript supposes cuDNN picks for 3x3 ("reducing mults from 9 to 4
// per output pixel per channel").  For every 2x2 output tile and its 4x4 input
// tile d, and every 3x3 filter g:
//   U = G g G^T,  V = B^T d B,  M = sum over input channels of U (.) V,
//   Y = A^T M A,
// with G = [1 0 0; 1/2 1/2 1/2; 1/2 -1/2 1/2; 0 0 1],
//      B^T = [1 0 -1 0; 0 1 1 0; 0 -1 1 0; 0 1 0 -1],
//      A^T = [1 1 1 0; 0 1 -1 -1].
// Along one axis: m1 = (d0-d2) g0, m2 = (d1+d2)(g0+g1+g2)/2,
// m3 = (d2-d1)(g0-g1+g2)/2, m4 = (d1-d3) g2, y0 = m1+m2+m3 = d0g0+d1g1+d2g2,
// y1 = m2-m3-m4 = d1g0+d2g1+d3g2; the 2-D form nests it along rows and columns.
// 16 multiplies per tile and input channel instead of 36; the transforms are
// additions, the 1/2 factors exact in binary.
//
// Design (B200): one CTA per (image, conv group, block of KB output channels,
// 2*TY x 2*TX output tile).  The CTA stages its group's input planes (tile +
// 1-pixel halo each side) with 4-byte cp.async, zero-filled outside the image
// (the padding), and transforms its KB x cpg filters to U in shared memory
// laid out [c][element][channel] so a thread's KT channels are one vector
// load.  Each thread owns one 2x2 output tile for KT output channels: per
// input channel it forms V from 16 shared loads (32 additions) and adds
// U (.) V into 16*KT accumulators; at the end Y = A^T M A, the epilogue (bias,
// or the folded affine + clamp) and the stores.
#include <algorithm>
#include <atomic>

#include "device_utils.cuh"
#include "gconv_internal.h"

namespace gconv {

namespace {

template <int KT>
__device__ __forceinline__ void load_kt(float (&u)[KT], const float *src) {
    if constexpr (KT == 4) {
        const float4 t = *reinterpret_cast<const float4 *>(src);
        u[0] = t.x; u[1] = t.y; u[2] = t.z; u[3] = t.w;
    } else {
        const float2 t = *reinterpret_cast<const float2 *>(src);
        u[0] = t.x; u[1] = t.y;
    }
}

// EPI: 0 = + bias, 2 = clamp(acc * scale + shift, lo, hi)
template <int KT, int EPI>
__global__ void __launch_bounds__(256, 2) winograd_kernel(const WinoParams p) {
    extern __shared__ __align__(16) float smem[];
    const int tid = threadIdx.x;
    const int tx = tid % p.TX;
    const int ty = (tid / p.TX) % p.TY;
    const int kz = tid / (p.TX * p.TY);
    const int qt = blockIdx.x % p.n_qt, pt = blockIdx.x / p.n_qt;
    const int kb = blockIdx.y % p.n_kb, g = blockIdx.y / p.n_kb;
    const int n = blockIdx.z;
    const int q0 = qt * 2 * p.TX, p0 = pt * 2 * p.TY;
    const int kc0 = g * p.kpg + kb * p.KB;     // first output channel of the CTA
    const int ci0 = g * p.cpg;                 // first input channel of the group
    const int XH = 2 * p.TY + 2, XW = 2 * p.TX + 2;   // staged rows / columns per plane

    float *su = smem;                            // [cpg][16][KB]
    float *sx = smem + p.u_floats;               // [cpg][XH][pitch]

    dev::griddep_wait();
    dev::griddep_launch_dependents();

    // stage the input tile + halo of every input channel of the group
    {
        const int total = p.cpg * XH * XW;
        const int ih0 = p0 - p.pad, iw0 = q0 - p.pad;
        int col = tid % XW, row = tid / XW;
        int c = row / XH;
        row -= c * XH;
        const int dq = blockDim.x / XW, dr = blockDim.x % XW;
        for (int e = tid; e < total; e += blockDim.x) {
            const int ih = ih0 + row, iw = iw0 + col;
            const bool ok = ih >= 0 && ih < p.H && iw >= 0 && iw < p.W;
            const float *src = ok ? p.x + (((long long)n * p.C + ci0 + c) * p.H + ih) * (long long)p.W + iw : p.x;
            dev::cp_async4(sx + (c * XH + row) * p.pitch + col, src, ok);
            col += dr;
            row += dq;
            if (col >= XW) {
                col -= XW;
                ++row;
            }
            while (row >= XH) {
                row -= XH;
                ++c;
            }
        }
    }
    // filter transform U = G g G^T for the CTA's KB output channels x cpg inputs
    for (int i = tid; i < p.KB * p.cpg; i += blockDim.x) {
        const int kl = i % p.KB, c = i / p.KB;
        const float *gw = p.w + ((long long)(kc0 + kl) * p.cpg + c) * 9;
        float gg[3][3];
#pragma unroll
        for (int r = 0; r < 3; ++r)
#pragma unroll
            for (int s = 0; s < 3; ++s) gg[r][s] = __ldg(gw + r * 3 + s);
        float t[4][3];   // G g
#pragma unroll
        for (int s = 0; s < 3; ++s) {
            t[0][s] = gg[0][s];
            t[1][s] = 0.5f * (gg[0][s] + gg[1][s] + gg[2][s]);
            t[2][s] = 0.5f * (gg[0][s] - gg[1][s] + gg[2][s]);
            t[3][s] = gg[2][s];
        }
        float *dst = su + c * 16 * p.KB + kl;
#pragma unroll
        for (int r = 0; r < 4; ++r) {   // (G g) G^T
            dst[(r * 4 + 0) * p.KB] = t[r][0];
            dst[(r * 4 + 1) * p.KB] = 0.5f * (t[r][0] + t[r][1] + t[r][2]);
            dst[(r * 4 + 2) * p.KB] = 0.5f * (t[r][0] - t[r][1] + t[r][2]);
            dst[(r * 4 + 3) * p.KB] = t[r][2];
        }
    }
    dev::cp_async_wait_all();
    __syncthreads();

    const bool active = kz < p.KZ && q0 + 2 * tx < p.Q && p0 + 2 * ty < p.P;
    if (!active) return;
    const int kl0 = kz * KT;
    float m[KT][16];
#pragma unroll
    for (int k = 0; k < KT; ++k)
#pragma unroll
        for (int e = 0; e < 16; ++e) m[k][e] = 0.f;

    for (int c = 0; c < p.cpg; ++c) {
        // d: the tile's 4x4 input window (rows 2ty.., columns 2tx..)
        const float *xs = sx + (c * XH + 2 * ty) * p.pitch + 2 * tx;
        float d[4][4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const float2 a = *reinterpret_cast<const float2 *>(xs + r * p.pitch);
            const float2 b = *reinterpret_cast<const float2 *>(xs + r * p.pitch + 2);
            d[r][0] = a.x; d[r][1] = a.y; d[r][2] = b.x; d[r][3] = b.y;
        }
        float t[4][4];   // B^T d
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            t[0][j] = d[0][j] - d[2][j];
            t[1][j] = d[1][j] + d[2][j];
            t[2][j] = d[2][j] - d[1][j];
            t[3][j] = d[1][j] - d[3][j];
        }
        float v[16];     // (B^T d) B
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[i * 4 + 0] = t[i][0] - t[i][2];
            v[i * 4 + 1] = t[i][1] + t[i][2];
            v[i * 4 + 2] = t[i][2] - t[i][1];
            v[i * 4 + 3] = t[i][1] - t[i][3];
        }
        const float *us = su + c * 16 * p.KB + kl0;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            float u[KT];
            load_kt<KT>(u, us + e * p.KB);
#pragma unroll
            for (int k = 0; k < KT; ++k) m[k][e] = fmaf(u[k], v[e], m[k][e]);
        }
    }

    // Y = A^T M A, epilogue, stores (2x2 outputs per channel)
    const int pp = p0 + 2 * ty, qq = q0 + 2 * tx;
    const bool row1 = pp + 1 < p.P, col1 = qq + 1 < p.Q;
    const long long plane = (long long)p.P * p.Q;
#pragma unroll
    for (int k = 0; k < KT; ++k) {
        float tt[2][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            tt[0][j] = m[k][0 * 4 + j] + m[k][1 * 4 + j] + m[k][2 * 4 + j];
            tt[1][j] = m[k][1 * 4 + j] - m[k][2 * 4 + j] - m[k][3 * 4 + j];
        }
        float y[2][2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            y[i][0] = tt[i][0] + tt[i][1] + tt[i][2];
            y[i][1] = tt[i][1] - tt[i][2] - tt[i][3];
        }
        const int kk = kc0 + kl0 + k;
        const float b = p.bias ? __ldg(p.bias + kk) : 0.f;
        const float sc = (EPI == 2 && p.aff_scale) ? __ldg(p.aff_scale + kk) : 1.f;
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                if constexpr (EPI == 2) y[i][j] = fminf(fmaxf(fmaf(y[i][j], sc, b), p.lo), p.hi);
                else y[i][j] += b;
            }
        float *yr = p.y + ((long long)n * p.K + kk) * plane + (long long)pp * p.Q + qq;
#pragma unroll
        for (int i = 0; i < 2; ++i, yr += p.Q) {
            if (i == 1 && !row1) break;
            if (p.vec_out && col1) {
                *reinterpret_cast<float2 *>(yr) = make_float2(y[i][0], y[i][1]);
            } else {
                yr[0] = y[i][0];
                if (col1) yr[1] = y[i][1];
            }
        }
    }
}

template <auto KERN>
cudaError_t launch_wino_k(const WinoParams &p, dim3 grid, int threads, size_t smem, cudaStream_t st) {
    if (smem > 48 * 1024) {
        static std::atomic<unsigned long long> opted{0};
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
        const unsigned long long bit = dev < 64 ? 1ull << dev : 0;
        if (!bit || !(opted.load(std::memory_order_acquire) & bit)) {
            cudaError_t e = cudaFuncSetAttribute(KERN, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
            if (e != cudaSuccess) return e;
            if (bit) opted.fetch_or(bit, std::memory_order_acq_rel);
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, KERN, p);
}

}  // namespace

cudaError_t launch_winograd(const WinoParams &p, int KT, dim3 grid, int threads, size_t smem, cudaStream_t st) {
    const bool aff = p.aff_scale || p.clamp;
    if (KT == 4) return aff ? launch_wino_k<winograd_kernel<4, 2>>(p, grid, threads, smem, st)
                            : launch_wino_k<winograd_kernel<4, 0>>(p, grid, threads, smem, st);
    if (KT == 2) return aff ? launch_wino_k<winograd_kernel<2, 2>>(p, grid, threads, smem, st)
                            : launch_wino_k<winograd_kernel<2, 0>>(p, grid, threads, smem, st);
    return cudaErrorInvalidValue;
}

}  // namespace gconv
