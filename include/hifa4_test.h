/*
 * hifa4_test.h -- test-only exports of the HiFA4-style 4-bit attention library.
 *
 * These entry points are NOT part of the product library (libhifa4.so).  They are built
 * only into the test library, libhifa4_test.so, which holds the whole product ABI of
 * hifa4.h plus the functions below.  They exist so that tests can look at single tensor-
 * core tiles and the device conversions, and can make a kernel's bounded wait run out
 * without faulting or hanging the GPU.  Conventions (ownership, status words, errors) are
 * those of hifa4.h.
 */
#ifndef HIFA4_TEST_H
#define HIFA4_TEST_H

#include "hifa4.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * hifa4_attn_fwd_quantized with a fault injected on the host's request: inject = 1 makes
 * the attention kernel's loader never deliver kv tile 1 of the first unit, so its
 * consumers' bounded waits run out and the call reports HIFA4_ERR_TIMEOUT through the
 * status word (the kernel drains its own copies and MMAs and frees TMEM before it exits;
 * the context stays usable).  inject = 0 is hifa4_attn_fwd_quantized.  The injection is an
 * argument of this call only: no other call, thread or stream sees it.
 * HIFA4_ERR_INVALID_ARG for inject outside {0, 1}.
 */
HIFA4_API int hifa4_test_attn_fwd_inject(const hifa4_qtensor* q, const hifa4_qtensor* k, const hifa4_qtensor* vt,
                                         int B, int Hq, int Hkv, int N, int d, int causal, int kv_tile, int inject,
                                         void* o, void* m_out, void* l_out, int* status, cudaStream_t stream);

/*
 * Single-tile probes of the tensor-core path.
 *   hifa4_probe_qk_tile: S[128][kv_tile] fp32 = Q_hat K_hat^T for one 128-row Q tile
 *     (codes [128][d/2], scale atoms d/64 x 512 B) and one kv_tile-row K tile (codes
 *     [kv_tile][d/2], scale atoms d/64 x 512 B, keys in atom rows 0..kv_tile-1).
 *   hifa4_probe_pv_tile: O[128][d] fp32 = P_hat V_hat and R[128] fp32 = P_hat * 1 for one
 *     P_hat tile (codes [128][kv_tile/2], atoms kv_tile/64 x 512 B) and one V^T tile
 *     (codes [d][kv_tile/2], atoms (kv_tile/64) x ceil(d/128) x 512 B).
 *   hifa4_probe_codec: for each x[i]: E2M1 code of x, E4M3 code of |x| and the library's
 *     exp2 E(x), computed by the device conversions the kernels use.
 */
HIFA4_API int hifa4_probe_qk_tile(const void* q_codes, const void* q_scales, const void* k_codes, const void* k_scales,
                                  int d, int kv_tile, float* S, int* status, cudaStream_t stream);
HIFA4_API int hifa4_probe_pv_tile(const void* p_codes, const void* p_scales, const void* vt_codes,
                                  const void* vt_scales, int d, int kv_tile, float* O, float* R, int* status,
                                  cudaStream_t stream);
HIFA4_API int hifa4_probe_codec(const float* x, int n, uint8_t* e2m1, uint8_t* e4m3, float* exp2_out,
                                cudaStream_t stream);

/*
 * hifa4_probe_codec_range: the E2M1 code of x and the E4M3 code of |x| (as
 * hifa4_probe_codec) for the n consecutive fp32 bit patterns start, start + 1, ...,
 * start + n - 1 (n <= 2^32 - start; e2m1, e4m3: device uint8 [n]).
 */
HIFA4_API int hifa4_probe_codec_range(uint32_t start, long long n, uint8_t* e2m1, uint8_t* e4m3, cudaStream_t stream);

/*
 * P_hat of nblk 16-key blocks by the attention kernels' device steps, for head dim d
 * (c = RN(log2(e)/sqrt(d))).  S: device fp32 [nblk][16] scores (-inf for a masked key);
 * m: device fp32 [nblk], the row's running max after the tile (an FP16 value).  Writes
 * scales[b] = the block's E4M3 scale code, from E(fma(block max, c, -m)), and codes[16b+e]
 * = the E2M1 code (0..15) of score e: fast = 0 the default rule
 * E2M1_RN(RN(E(RN(fma(S, c, -m))) * RN(1/sigma))), fast = 1 the rule of
 * hifa4_attn_fwd_quantized_fast.  codes, scales: device uint8 [nblk * 16], [nblk].
 */
HIFA4_API int hifa4_probe_phat(const float* S, const float* m, int nblk, int d, int fast, uint8_t* codes,
                               uint8_t* scales, cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* HIFA4_TEST_H */
