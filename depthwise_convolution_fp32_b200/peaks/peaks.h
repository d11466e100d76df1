/* Roofline denominators measured on the current GPU (measurement tooling for
 * the benchmark; not part of libgconv.so's C ABI).  Each call times one
 * launch with CUDA events after an untimed one and returns 0 on success,
 * with *ms the launch's duration and *flops the floating-point operations it
 * performed (2 per multiply-add).
 *   gpeaks_ffma      FP32 FMA on the CUDA cores (8 CTAs of 256 threads per SM,
 *                    16 independent chains per thread, `iters` x 128 FMAs each)
 *   gpeaks_mma_tf32  tcgen05.mma kind::tf32, M=128 N=256 K=8, one CTA per SM,
 *                    `iters` MMAs per CTA into one TMEM accumulator
 *   gpeaks_mma_bf16  tcgen05.mma kind::f16 (bf16), M=128 N=256 K=16, likewise
 * Non-zero returns: 1 bad argument / no device, 2 allocation or launch failed,
 * 3 timing failed, 4 a bounded wait in the MMA kernel gave up. */
#ifndef GCONV_PEAKS_H_
#define GCONV_PEAKS_H_
#if defined(__GNUC__)
#define GPEAKS_API __attribute__((visibility("default")))
#else
#define GPEAKS_API
#endif
#ifdef __cplusplus
extern "C" {
#endif
GPEAKS_API int gpeaks_ffma(int iters, double *ms, double *flops);
GPEAKS_API int gpeaks_mma_tf32(int iters, double *ms, double *flops);
GPEAKS_API int gpeaks_mma_bf16(int iters, double *ms, double *flops);
#ifdef __cplusplus
}
#endif
#endif
