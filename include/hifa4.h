/*
 * hifa4.h -- C ABI of a B200 (sm_100a) implementation of the HiFA4-style 4-bit
 * FlashAttention forward pass.
 *
 * Method: "HiFA4: Training-Free 4-bit FlashAttention on Ascend HIF4 NPUs for LLM
 * Inference" (abstract).  Both QK^T and PV run as 4-bit GEMMs; the online-softmax state
 * (running max m, normaliser l) is FP16; Smooth-QK rescales post-RoPE Q and K per channel
 * (Q*s, K/s) with s fixed by an offline calibration; P-Reordering sums the normaliser
 * from the same quantised weights P_hat that feed the PV GEMM, which lets the tensor core
 * produce it (here: an extra MMA of P_hat against a block of ones).
 *
 * 4-bit format (the abstract does not give the HIF4 layout; this library states its own,
 * NVFP4-style): E2M1 codes (two per byte, element 2i in the low nibble) with one unsigned
 * E4M3 scale per 16 consecutive contraction elements.
 *   scale = E4M3_RN(amax * RN(1/6));  code = E2M1_RN_satfinite(x * RN(1/scale)),
 *   with 1/scale taken as 0 when scale == 0.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library never
 *     allocates or frees device memory.
 *   - Work is enqueued on `stream` and is asynchronous, except where a function says it
 *     synchronises.
 *   - Return value: a hifa4_status.  Argument and shape errors are detected on the host
 *     and nothing is launched.  Errors found on the device (non-finite input, a bounded
 *     wait that ran out) are ORed as bits into a caller-provided device int `status`;
 *     read them with hifa4_read_status().
 *   - bf16 inputs [B, H, N, d] are addressed with element strides {b, h, n}; the channel
 *     dimension must be contiguous, the base 16-byte aligned and every stride a multiple
 *     of 8 elements.
 *   - Shapes: d in {64, 128, 256}; Hq % Hkv == 0 (query head h uses kv head
 *     h / (Hq/Hkv)); N % 128 == 0; N <= 63488 (the FP16 normaliser stays finite); causal
 *     attention uses equal query and key lengths with key k visible to query i iff k <= i.
 *     The FP16 running max holds RN(rowmax(S) * log2(e)/sqrt(d)); rows where that exceeds
 *     the FP16 range (|.| > 65504) are outside the supported input range.
 *   - Requires an sm_100 device (B200); anything else returns
 *     HIFA4_ERR_UNSUPPORTED_DEVICE.  There is no CPU fallback.
 *   - Each kernel's shared-memory attributes and resident-CTA count are set up on its
 *     first launch and kept for the life of the process (thread-safe), so a process
 *     drives one GPU, or several identical ones.
 */
#ifndef HIFA4_H
#define HIFA4_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define HIFA4_API __attribute__((visibility("default")))
#else
#define HIFA4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HIFA4_OK = 0,
  HIFA4_ERR_INVALID_ARG = 1,       /* null pointer, bad stride or alignment, bad value */
  HIFA4_ERR_UNSUPPORTED_SHAPE = 2, /* d, N, head counts or kv tile outside the supported set */
  HIFA4_ERR_UNSUPPORTED_DEVICE = 3,/* current device is not sm_100 */
  HIFA4_ERR_NONFINITE = 4,         /* a quantised input held inf or NaN (device-detected) */
  HIFA4_ERR_TIMEOUT = 5,           /* a kernel's bounded wait ran out (device-detected) */
  HIFA4_ERR_CUDA = 6,              /* a CUDA runtime call or launch failed */
  HIFA4_ERR_IO = 7                 /* a calibration file could not be written or read, or is not valid */
} hifa4_status;

/* Device status-word bits (ORed by kernels into the caller's `int* status`). */
#define HIFA4_STATUS_NONFINITE 1
#define HIFA4_STATUS_TIMEOUT 2

/* Human-readable name of a status code; never NULL. */
HIFA4_API const char* hifa4_status_string(int status);

/*
 * A 4-bit tensor in this library's layout (caller-owned device memory).
 *   transposed == 0 (Q, K: blocks along d), logical [B, H, N, d]:
 *     codes  [B][H][N][d/2]
 *     scales [B][H][N/128][d/64][512]: per 128-row tile and 64-wide chunk of d, a
 *            512-byte atom; row r (0..127), block s (0..3) of the chunk sits at byte
 *            (r % 32) * 16 + (r / 32) * 4 + s.
 *   transposed == 1 (V^T: blocks of 16 consecutive tokens per channel), logical
 *   [B, H, d, N]:
 *     codes  [B][H][d][N/2]
 *     scales [B][H][N/64][ceil(d/128)][512]: per 64-token chunk and 128-channel group,
 *            an atom as above with r = channel within the group (rows beyond d are 0).
 * codes and scales must be 16-byte aligned.
 */
typedef struct {
  void* codes;
  void* scales;
  int B, H, N, d;
  int transposed;
} hifa4_qtensor;

/* Bytes of the codes / scales buffers of a 4-bit tensor with these logical sizes. */
HIFA4_API size_t hifa4_qtensor_codes_bytes(int B, int H, int N, int d);
HIFA4_API size_t hifa4_qtensor_scales_bytes(int B, int H, int N, int d, int transposed);

/*
 * Smooth-QK calibration (HiFA4 abstract: per-channel scales for post-RoPE Q and K, fixed
 * offline from a calibration sample).  From a post-RoPE bf16 calibration sample Q_cal
 * [B, Hq, N, d] and K_cal [B, Hkv, N, d]:
 *   s[g, c]    = RN_fp32((amax_K[g, c] / amax_Q[g, c]) ^ alpha), computed in double
 *                (s = 1 where either amax is 0; alpha = 0 gives s == 1),
 *   s_inv[g,c] = RN_fp32(1 / s[g, c]),
 * where amax_Q runs over the batch, the query heads of kv group g and all tokens, and
 * amax_K over the batch and tokens of kv head g.  s_out and sinv_out are device fp32
 * [Hkv * d].  `workspace` is device memory of hifa4_calibrate_workspace_bytes(Hkv, d)
 * bytes.  N may be any positive value here.  SYNCHRONISES `stream` (it reads the channel
 * maxima back to the host).  Offline step, not part of the timed path.
 */
HIFA4_API size_t hifa4_calibrate_workspace_bytes(int Hkv, int d);
HIFA4_API int hifa4_calibrate_smooth(const void* q_cal, const void* k_cal, const int64_t q_strides[3],
                           const int64_t k_strides[3], int B, int Hq, int Hkv, int N, int d, float alpha,
                           float* s_out, float* sinv_out, void* workspace, cudaStream_t stream);

/*
 * The Smooth-QK calibration as a file: the method's one persistent artefact (the HiFA4
 * abstract fixes the scales offline, so they are computed once and shipped with the
 * model).  HOST arrays; copy them to or from the device yourself.  Layout (little-endian):
 * magic "HIFA4CAL", uint32 version = 1, int32 Hkv, int32 d, fp32 alpha, uint32 CRC-32 of
 * the arrays, then s [Hkv * d] and s_inv [Hkv * d] fp32, exactly as
 * hifa4_calibrate_smooth produced them (bit patterns are preserved).
 *   hifa4_calibration_save: HIFA4_ERR_INVALID_ARG for null arrays or path, Hkv or d not
 *     positive, alpha negative or NaN; HIFA4_ERR_IO if the file cannot be written.
 *   hifa4_calibration_load: reads the header into *Hkv, *d, *alpha; with s and sinv both
 *     NULL it stops there (to size the arrays), otherwise it needs capacity >= Hkv * d
 *     (else HIFA4_ERR_INVALID_ARG) and fills both.  HIFA4_ERR_IO for a missing or short
 *     file, a wrong magic or version, trailing bytes or a CRC mismatch; the arrays are
 *     written only on success.
 */
HIFA4_API int hifa4_calibration_save(const char* path, int Hkv, int d, float alpha, const float* s, const float* sinv);
HIFA4_API int hifa4_calibration_load(const char* path, int* Hkv, int* d, float* alpha, float* s, float* sinv,
                                     size_t capacity);

/*
 * Smooth-QK application + 4-bit quantisation of Q and K (one launch):
 *   q' = RN(q * s[g(h), c]),  k' = RN(k * s_inv[g, c]),  then blocks of 16 along d.
 * s and sinv are device fp32 [Hkv * d]; both NULL disables smoothing (s == 1).
 * q_out / k_out: transposed == 0 tensors of sizes [B, Hq, N, d] / [B, Hkv, N, d].
 * Sets HIFA4_STATUS_NONFINITE in *status if an input (after smoothing) is not finite.
 */
HIFA4_API int hifa4_quantize_qk(const void* q, const void* k, const int64_t q_strides[3], const int64_t k_strides[3],
                      int B, int Hq, int Hkv, int N, int d, const float* s, const float* sinv,
                      const hifa4_qtensor* q_out, const hifa4_qtensor* k_out, int* status, cudaStream_t stream);

/*
 * 4-bit quantisation of V^T: blocks of 16 consecutive tokens of one channel, no
 * smoothing.  v: bf16 [B, Hkv, N, d]; vt_out: transposed == 1 tensor.
 */
HIFA4_API int hifa4_quantize_v(const void* v, const int64_t v_strides[3], int B, int Hkv, int N, int d,
                     const hifa4_qtensor* vt_out, int* status, cudaStream_t stream);

/*
 * Fused RoPE + Smooth-QK + 4-bit quantisation of Q and K (the step before the attention:
 * the HiFA4 abstract applies the per-channel rescaling after RoPE, so the rotation, the
 * rescaling and the quantisation run in one pass over the pre-RoPE tensors).
 * q, k: bf16 [B, Hq, N, d] / [B, Hkv, N, d] BEFORE RoPE, strides as for hifa4_quantize_qk.
 * rope_cos, rope_sin: device fp32 [N, d/2], 16-byte aligned; row n holds the angles of
 * token n (its position), column i those of channel pair (i, i + d/2).  Rotate-half RoPE
 * in fp32, each product and the sum rounded once:
 *   x'_i = RN(RN(x_i cos) - RN(x_{i+d/2} sin)),  x'_{i+d/2} = RN(RN(x_{i+d/2} cos) + RN(x_i sin)),
 * then q' = RN(x' * s[g,c]) (k' with sinv) and the 16-element block quantiser of
 * hifa4_quantize_qk; the rotated values are not rounded to bf16.  Same outputs and errors
 * as hifa4_quantize_qk (HIFA4_ERR_INVALID_ARG also for a missing or misaligned table).
 */
HIFA4_API int hifa4_quantize_qk_rope(const void* q, const void* k, const int64_t q_strides[3],
                                     const int64_t k_strides[3], int B, int Hq, int Hkv, int N, int d,
                                     const float* rope_cos, const float* rope_sin, const float* s, const float* sinv,
                                     const hifa4_qtensor* q_out, const hifa4_qtensor* k_out, int* status,
                                     cudaStream_t stream);

/*
 * Host helper: the angle tables of hifa4_quantize_qk_rope for positions pos0 .. pos0+N-1,
 * inv_freq_i = theta^(-2i/d), angle = position * inv_freq_i, cos and sin computed in double
 * and rounded once to fp32.  cos_out, sin_out: HOST fp32 [N, d/2] (caller-owned; copy them
 * to the device).  Returns HIFA4_ERR_INVALID_ARG for null outputs, theta <= 1, N <= 0,
 * pos0 < 0 or an unsupported d.
 */
HIFA4_API int hifa4_rope_table(double theta, int pos0, int N, int d, float* cos_out, float* sin_out);

/*
 * hifa4_quantize_qk and hifa4_quantize_v in one launch (same arguments and outputs; the
 * three quantisations are independent, so V's latency hides behind Q and K).
 */
HIFA4_API int hifa4_quantize_qkv(const void* q, const void* k, const void* v, const int64_t q_strides[3],
                                 const int64_t k_strides[3], const int64_t v_strides[3], int B, int Hq, int Hkv,
                                 int N, int d, const float* s, const float* sinv, const hifa4_qtensor* q_out,
                                 const hifa4_qtensor* k_out, const hifa4_qtensor* vt_out, int* status,
                                 cudaStream_t stream);

/*
 * The fused 4-bit attention forward on already quantised Q, K and V^T.
 * For every (b, h, query row i), kv tiles j = 0, 1, ... of kv_tile keys (only tiles
 * holding a visible key when causal):
 *   S      = Q_hat K_hat_j^T                     (4-bit tensor-core MMA, fp32 accumulate)
 *   m_new  = max(m, fp16_RN(RN(rowmax(S) * c))), c = RN(log2(e) / sqrt(d))
 *   P      = E(RN(fma(S, c, -m_new)))            (E: the library's deterministic exp2,
 *            a cubic fit of 2^x with relative error below 9e-5)
 *   P_hat  = the 4-bit block quantiser applied to P, 16 consecutive keys per block:
 *            sigma = E4M3_RN(RN(amax * RN(1/6))) with amax the block's largest P, code =
 *            E2M1_RN(RN(P * RN(1/sigma)))
 *   alpha  = E(m - m_new)  (0 on the first tile)
 *   O      = alpha * O + P_hat V_hat_j           (4-bit MMA)
 *   r      = P_hat * 1                           (4-bit MMA against ones: P-Reordering)
 *   l      = fp16_RN(fma(alpha, l, r)),  m = m_new
 * and finally out = bf16_RN(O / l).  kv_tile is 64, 128 or 256 and is part of the result's
 * definition; N must be a multiple of it.  0 selects 128 for d = 64, 256 for d = 128 when
 * N is a multiple of 256 (else 128), and 64 for d = 256; d = 256 supports only 64 and
 * d = 64 at most 128.
 * o: bf16 [B, Hq, N, d] dense.  m_out, l_out: fp16 [B, Hq, N] dense, or NULL.
 */
HIFA4_API int hifa4_attn_fwd_quantized(const hifa4_qtensor* q, const hifa4_qtensor* k, const hifa4_qtensor* vt, int B,
                             int Hq, int Hkv, int N, int d, int causal, int kv_tile, void* o, void* m_out,
                             void* l_out, int* status, cudaStream_t stream);

/*
 * Fast form of hifa4_attn_fwd_quantized (same arguments, outputs and errors) with an
 * approximate P_hat code rule: the code of a score is the E2M1 rounding of
 * y = 2^floor(z) (1 + frac z), z = 128u - 125 - 73/1024 on a 2^-10 grid,
 * u = sat(S c/128 + (RN(-log2 sigma) - m_new + 125)/128), i.e. P / sigma evaluated in the
 * log domain with a linear mantissa, whose E2M1 rounding boundaries lie within 1% of the
 * exact ones (the lowest, between codes 0 and 1, 5% above it).  m, sigma and alpha are
 * those of hifa4_attn_fwd_quantized, so m is identical; a few percent of the P_hat codes
 * differ by one step, which changes l and O slightly (the tests and the benchmark report
 * the rates).  It exists to measure what the exact rounding costs.
 */
HIFA4_API int hifa4_attn_fwd_quantized_fast(const hifa4_qtensor* q, const hifa4_qtensor* k, const hifa4_qtensor* vt,
                                            int B, int Hq, int Hkv, int N, int d, int causal, int kv_tile, void* o,
                                            void* m_out, void* l_out, int* status, cudaStream_t stream);

/*
 * Ablation form of hifa4_attn_fwd_quantized (same arguments, outputs and errors, plus
 * two): the kernel also sums the unquantised P = E(RN(fma(S, c, -m_new))) of every row and
 * kv tile in fp32 (each 64-column (Bc = 64: 32-column) chunk of the row in order, then the
 * chunks in order).
 *   normaliser 0: l from r = P_hat * 1 as in HiFA4 (O, m, l identical to
 *                 hifa4_attn_fwd_quantized);
 *   normaliser 1: l from r = sum P, the inconsistent formulation of the HiFA4 abstract
 *                 (PV still uses P_hat), i.e. each tile's contribution to O is scaled by
 *                 sum P_hat / sum P.  With Q and K quantised without Smooth-QK (s = NULL)
 *                 this is the abstract's baseline of direct 4-bit quantisation.
 *   two_level 0: the one-level block scales of P_hat (as hifa4_attn_fwd_quantized);
 *   two_level 1: a second-level scale for P: per row and kv tile a power of two 2^k,
 *                k = max(floor(log2 p_t) - 10, -40) with p_t the tile's largest block amax
 *                of P; block scale E4M3_RN(RN(amax * RN(1/6)) * 2^-k), P_hat = code *
 *                scale * 2^k, code = E2M1_RN(RN(P * RN(1/(scale * 2^k)))).  Equal to two_level 0 wherever every one-level block scale
 *                is a normal E4M3 value; keeps the blocks one level flushes to zero
 *                (amax <= 6 * 2^-10).  l is the FP16 recursion on sum P_hat computed by the
 *                tensor core in fp32, which the wider scale range can round.
 * trace: device fp32 [B, Hq, N, N / kv_tile, 2] (16-byte aligned) or NULL; entry (row,
 *   tile, 0) = sum P_hat (exact), (row, tile, 1) = sum P of that tile, for every tile the
 *   row's 128-row query tile visits (causal: later tiles are not written; a visited tile
 *   with no visible key for the row holds 0, 0).  The per-tile mass error of the abstract
 *   is eps = sum P_hat / sum P - 1.
 * HIFA4_ERR_INVALID_ARG for normaliser or two_level outside {0, 1} or a misaligned trace.
 */
HIFA4_API int hifa4_attn_fwd_ablation(const hifa4_qtensor* q, const hifa4_qtensor* k, const hifa4_qtensor* vt,
                                      int B, int Hq, int Hkv, int N, int d, int causal, int kv_tile, int normaliser,
                                      int two_level, float* trace, void* o, void* m_out, void* l_out, int* status,
                                      cudaStream_t stream);

/*
 * Decode / split-KV attention: a short query (nq tokens per sequence, the last nq positions)
 * against Nk keys of 4-bit K and V^T (a KV cache quantised with hifa4_quantize_qk /
 * hifa4_quantize_v, N = Nk).  The G = Hq / Hkv query heads of a kv head and the nq tokens
 * are packed into one 128-row tile (G * nq <= 128): row r = hi * nq + t is token t of query
 * head g * G + hi, at position Nk - nq + t, and sees the keys <= that position.
 *
 * hifa4_quantize_q_decode: Smooth-QK (s, NULL = off) and 4-bit quantisation of bf16
 *   q [B, Hq, nq, d] (strides as for hifa4_quantize_qk) into the packed q_out, a
 *   transposed == 0 tensor of sizes [B, Hkv, 128, d] (rows >= G * nq are zero).
 * hifa4_attn_decode: the Nk / kv_tile kv tiles are cut into nsplit runs of
 *   ceil(tiles / nsplit) tiles (nsplit <= 0: chosen from the SM count; at most 64; empty
 *   runs are dropped, which the merge would weight 0).  Every (batch, kv head, run) runs the
 *   HiFA4 tile loop of hifa4_attn_fwd_quantized from the initial state and leaves (m_s, l_s,
 *   unnormalised fp32 O_s) in `workspace` (hifa4_decode_workspace_bytes(B, Hkv, nsplit, d)
 *   bytes, 16-byte aligned); a second launch merges in fp32, runs in order:
 *     m = max m_s,  w_s = E(m_s - m) (0 for m_s = -inf),  L = fma(w_s, l_s, L),
 *     O = fma(w_s, O_s, O),  out = bf16_RN(O * RN(1/L)).
 *   o: bf16 [B, Hq, nq, d] dense; m_out, l_out: fp16 [B, Hq, nq] (m, RN(L)) or NULL.
 *   Nk a multiple of 128 and of kv_tile; kv_tile as for hifa4_attn_fwd_quantized, except
 *   that kv_tile = 0 selects 128 when d = 128 and G * nq <= 16.  That case (d = 128,
 *   kv_tile = 128, G * nq <= 16) runs a kernel with the keys on the MMA's M dimension and
 *   the packed query rows on N, with the same results as the 128-row kernel at that tile.
 */
HIFA4_API int hifa4_quantize_q_decode(const void* q, const int64_t q_strides[3], int B, int Hq, int Hkv, int nq, int d,
                                      const float* s, const hifa4_qtensor* q_out, int* status, cudaStream_t stream);
HIFA4_API size_t hifa4_decode_workspace_bytes(int B, int Hkv, int nsplit, int d);
HIFA4_API int hifa4_attn_decode(const hifa4_qtensor* q, const hifa4_qtensor* k, const hifa4_qtensor* vt, int B, int Hq,
                                int Hkv, int nq, int Nk, int d, int kv_tile, int nsplit, void* workspace,
                                size_t workspace_bytes, void* o, void* m_out, void* l_out, int* status,
                                cudaStream_t stream);

/*
 * The full attention forward on quantised Q, K and bf16 V: quantises V^T into
 * `workspace` (hifa4_attn_workspace_bytes(B, Hkv, N, d) bytes of device memory, 16-byte
 * aligned), then runs hifa4_attn_fwd_quantized.  Two launches on `stream`.  Every
 * argument, those of the attention included, is checked before the first launch: an
 * error status means nothing was enqueued.
 */
HIFA4_API size_t hifa4_attn_workspace_bytes(int B, int Hkv, int N, int d);
HIFA4_API int hifa4_attn_fwd(const hifa4_qtensor* q, const hifa4_qtensor* k, const void* v, const int64_t v_strides[3],
                   int B, int Hq, int Hkv, int N, int d, int causal, int kv_tile, void* workspace,
                   size_t workspace_bytes, void* o, void* m_out, void* l_out, int* status, cudaStream_t stream);

/*
 * hifa4_attn_fwd without a caller workspace (the method's pages have no counterpart of
 * this entry point; it exists for callers that cannot allocate device memory -- e.g. a
 * serving process whose device memory is all handed out up front, or a latency-critical
 * loop that must not block on cudaMalloc).  Same arguments and results as
 * hifa4_attn_fwd minus the workspace: the 4-bit V^T goes to a 16 MiB scratch array
 * compiled into the library, which every GPU that loads the library holds until the
 * process exits.  Workloads whose hifa4_attn_workspace_bytes(B, Hkv, N, d) exceeds
 * 16 MiB are rejected with HIFA4_ERR_UNSUPPORTED_SHAPE before anything is launched.
 * Allocates nothing.  The first call on a device looks up the scratch array's device
 * address (cudaGetSymbolAddress), so make that first call before any stream capture.
 * All calls on a device share the scratch: calls whose GPU work may overlap (e.g. on
 * unordered streams) race on it.  The scratch address is cached per device for the life
 * of the process: after a cudaDeviceReset this entry point must not be called again.
 */
HIFA4_API int hifa4_attn_fwd_noalloc(const hifa4_qtensor* q, const hifa4_qtensor* k, const void* v,
                                     const int64_t v_strides[3], int B, int Hq, int Hkv, int N, int d, int causal,
                                     int kv_tile, void* o, void* m_out, void* l_out, int* status,
                                     cudaStream_t stream);

/*
 * Synchronises `stream`, reads the device status word and maps it to a hifa4_status
 * (TIMEOUT before NONFINITE before OK).  clear != 0 resets the word to 0 afterwards.
 */
HIFA4_API int hifa4_read_status(int* status, int clear, cudaStream_t stream);

/* Wall-clock limit of every wait inside the kernels, in nanoseconds (default 2 s). */
HIFA4_API void hifa4_set_wait_limit_ns(unsigned long long ns);

#ifdef __cplusplus
}
#endif
#endif /* HIFA4_H */
