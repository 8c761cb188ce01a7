/*
 * hifa4_peak.h -- measurement helper of the HiFA4-style 4-bit attention library
 * (libhifa4_peak.so): the dense FP4 tensor-core rate of the current B200, measured with
 * the block-scaled FP4 MMA the attention kernel issues (tcgen05 kind::mxf4nvf4, UE4M3
 * scales per 16 elements, fp32 accumulate in TMEM), so the attention's roofline fraction
 * can be quoted against a measured peak rather than a nominal one.
 */
#ifndef HIFA4_PEAK_H
#define HIFA4_PEAK_H

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define HIFA4_PEAK_API __attribute__((visibility("default")))
#else
#define HIFA4_PEAK_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define HIFA4_PEAK_ERR_INVALID_ARG 1
#define HIFA4_PEAK_ERR_UNSUPPORTED_DEVICE 3
#define HIFA4_PEAK_ERR_CUDA 6

/* Flops of one loop iteration of one CTA: one M = 128, N = 256, K = 64 MMA, 2*M*N*K. */
HIFA4_PEAK_API double hifa4_fp4_mma_flops_per_iter(void);

/*
 * Launch `ctas` CTAs (one per SM: each holds all 512 TMEM columns and more than half the
 * SM's shared memory), each issuing `iters` back-to-back block-scaled FP4 MMAs from
 * constant shared-memory operands into one TMEM accumulator; nothing is read from or
 * written to global memory except the status word.  Asynchronous on `stream`: time it with
 * CUDA events on that stream.  The completion wait is bounded (2 s): if it runs out the
 * kernel ORs 2 into *status (a device int the caller zeroes) and still frees TMEM.
 * Returns 0, or an HIFA4_PEAK_ERR_* code (nothing launched): bad arguments (ctas or iters
 * not positive, iters above 2^20, a null status), a device that is not sm_100, a CUDA
 * launch error.
 */
HIFA4_PEAK_API int hifa4_fp4_mma_loop(int ctas, int iters, int* status, cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* HIFA4_PEAK_H */
