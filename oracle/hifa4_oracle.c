/*
 * HiFA4 CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously correct CPU restatement of what the 4-bit attention forward
 * computes, used to prove the CUDA path right.  Only the tests, the package's smoke()
 * check and bench.py's cpu_baseline / reference leg may load or call it; the product
 * path never does.  It shares no code, header, table or constant generator with the
 * CUDA library: every format rule, the exp2 approximation and the tile loop are written
 * out again here from their definitions.
 *
 * Source of the method: "HiFA4: Training-Free 4-bit FlashAttention on Ascend HIF4 NPUs
 * for LLM Inference" (abstract, as printed on catalyzex.com/author/Chunlu Li, the same
 * text on the other pages).  The abstract fixes: both QK^T and PV are 4-bit GEMMs; the
 * online-softmax state is FP16; Smooth-QK multiplies Q and divides K per channel by
 * scales s that an offline calibration fixes, after RoPE; P-Reordering sums the normaliser from the same quantised
 * weights P_hat that feed PV, which lets the normaliser be produced by the PV GEMM.
 * Everything the abstract leaves open is a stated reading:
 *   - 4-bit format: E2M1 values with one unsigned E4M3 scale per 16 contraction
 *     elements (NVFP4-style), no second-level scale.  scale = E4M3_RN(amax * RN(1/6)),
 *     R = RN(1/scale) (R = 0 when scale == 0), code = E2M1_RN_satfinite(x * R).
 *   - exp2 in the softmax: the method's own deterministic approximation E(x) (clamp to
 *     -127, floor split, cubic Horner in fp32 fma, exponent insert; relative error below
 *     9e-5); see own_exp2().
 *   - m_new = max(m, fp16_RN(RN(rowmax(S) * c))), c = RN(log2(e)/sqrt(d)),
 *     P = E(RN(fma(S, c, -m_new))), alpha = E(RN(m_old - m_new)),
 *     P_hat = the block quantiser above applied to P, 16 consecutive keys per block
 *     (so a score's code is E2M1_RN(RN(P * RN(1/sigma))) with sigma from the block's
 *     largest P),
 *     l = fp16_RN(fma(alpha, l, r)), r = exact sum of the tile's P_hat,
 *     O = alpha*O (fp32) + (exact tile P_hat V_hat rounded to fp32),
 *     out = bf16_RN(RN(O / l)).
 *   - two-level P scale (ablation variant, two_level = 1): a per-(row, tile) power of two
 *     2^k under the block scales of P, k = max(floor(log2 p_t) - 10, -40) with p_t the
 *     tile's largest block amax of P; sigma_b = E4M3_RN(RN(amax * RN(1/6)) * 2^-k),
 *     P_hat = code * sigma_b * 2^k with code = E2M1_RN(RN(P * RN(1/(sigma_b * 2^k)))).
 *     Where the one-level scale is a normal E4M3 value both give the same P_hat; blocks
 *     too small for one level (scale 0 or subnormal) keep their mass.
 *   - S accumulation of the 4-bit GEMM: one of the models in s_dot(), selected by the
 *     caller; the mirror uses model 3 (per 64-wide MMA step, the exact sum of the fp32
 *     accumulator and the step's block products, rounded toward zero), which is what a
 *     probe of the tensor-core hardware showed.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_EXPORT __attribute__((visibility("default")))

/* ------------------------------------------------------------------ scalar formats */

static float bits_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f32_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

static float bf16_to_f32(uint16_t b) { return bits_f32((uint32_t)b << 16); }

/* bf16 round-to-nearest-even of a finite fp32 value. */
static uint16_t f32_to_bf16(float f) {
    uint32_t u = f32_bits(f);
    if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)((u >> 16) | ((u & 0xFFFF) ? 0x40 : 0));
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* IEEE binary16 round-to-nearest-even, through the compiler's _Float16 conversion. */
static float f16_round(float f) { return (float)(_Float16)f; }
static uint16_t f16_bits(float f) { _Float16 h = (_Float16)f; uint16_t u; memcpy(&u, &h, 2); return u; }

/* E2M1 (FP4): sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0.
 * Magnitudes of codes 0..7: 0, 0.5, 1, 1.5, 2, 3, 4, 6 (OCP Microscaling formats). */
static const float E2M1_MAG[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

/* Nearest E2M1 value, ties to the even code (even mantissa), saturating at 6. */
static uint8_t e2m1_encode(float x) {
    uint8_t sign = signbit(x) ? 8 : 0;
    float a = fabsf(x);
    if (isnan(x)) return 7;                 /* never produced by the method's inputs */
    if (a >= 6.0f) return sign | 7;         /* satfinite */
    int best = 0;
    double bestd = fabs((double)a - E2M1_MAG[0]);
    for (int c = 1; c < 8; ++c) {
        double dd = fabs((double)a - E2M1_MAG[c]);
        if (dd < bestd || (dd == bestd && (c & 1) == 0 && (best & 1) == 1)) { best = c; bestd = dd; }
    }
    return sign | (uint8_t)best;
}

static float e2m1_value(uint8_t code) {
    float v = E2M1_MAG[code & 7];
    return (code & 8) ? -v : v;
}

/* 2 * E2M1 value as an integer: 0,1,2,3,4,6,8,12 with sign. */
static int e2m1_twice(uint8_t code) {
    static const int T[8] = {0, 1, 2, 3, 4, 6, 8, 12};
    int v = T[code & 7];
    return (code & 8) ? -v : v;
}

/* E4M3 (sign 0 for scales): exponent bits 6..3 (bias 7), mantissa bits 2..0.
 * Normal: (1 + m/8) * 2^(e-7), e = 1..15 (e=15,m=7 is NaN, so 448 is the largest);
 * subnormal e = 0: m * 2^-9. */
static float e4m3_value(uint8_t b) {
    int e = (b >> 3) & 15, m = b & 7;
    float v = (e == 0) ? ldexpf((float)m, -9) : ldexpf(1.0f + m / 8.0f, e - 7);
    return (b & 0x80) ? -v : v;
}

/* scale * 512 as an integer (scales are non-negative): exact for all codes. */
static int64_t e4m3_units(uint8_t b) {
    int e = (b >> 3) & 15, m = b & 7;
    return (e == 0) ? m : ((int64_t)(8 + m) << (e - 1));
}

/* Nearest non-negative E4M3 value, ties to the even code, saturating at 448.
 * Binary search over the 127 finite non-negative codes, which are increasing. */
static uint8_t e4m3_encode_pos(float x) {
    if (!(x > 0.0f)) return 0;               /* 0, -0 and negatives (never passed) */
    if (x >= 448.0f) return 0x7E;
    int lo = 0, hi = 0x7E;                   /* value(lo) <= x < value(hi) after search */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (e4m3_value((uint8_t)mid) <= x) lo = mid; else hi = mid;
    }
    double dl = (double)x - e4m3_value((uint8_t)lo), dh = (double)e4m3_value((uint8_t)hi) - x;
    if (dl < dh) return (uint8_t)lo;
    if (dh < dl) return (uint8_t)hi;
    return (uint8_t)((lo & 1) ? hi : lo);
}

/* ------------------------------------------------------------------ own exp2 E(x) */

/* Coefficients of p(f) = 1 + c1 f + c2 f^2 + c3 f^3 ~ 2^f on [0,1): a minimax fit of the
 * relative error with p(0) = 1 held exact (max relative error 8.6e-5), rounded to fp32. */
#define EXP2_C1 0x1.63e65ap-1f
#define EXP2_C2 0x1.d23788p-3f
#define EXP2_C3 0x1.3baaa8p-4f

static float own_exp2(float x) {
    float xc = fmaxf(x, -127.0f);            /* fmaxf(NaN,-127) = -127; -inf -> -127 */
    float n = floorf(xc);
    float f = xc - n;                        /* RN(xc - n) */
    float p = fmaf(fmaf(fmaf(EXP2_C3, f, EXP2_C2), f, EXP2_C1), f, 1.0f);
    uint32_t bits = f32_bits(p) + ((uint32_t)(int32_t)n << 23);
    return bits_f32(bits);                   /* p * 2^n; exactly 0 for xc = -127 */
}

/* ------------------------------------------------------------------ block quantiser */

/* NVFP4-style block of 16 with an optional second-level power of two 2^k (k = 0: the
 * one-level format): the E4M3 scale is taken of RN(amax * RN(1/6)) * 2^-k, the effective
 * scale is sigma = scale * 2^k, and every code is E2M1_RN(RN(x * RN(1/sigma))). */
static void quant16_k(const float* x, int k, uint8_t* codes /*16 nibbles, one per byte*/, uint8_t* scale) {
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
    uint8_t sc = e4m3_encode_pos(ldexpf(amax * (1.0f / 6.0f), -k));
    float sigma = ldexpf(e4m3_value(sc), k);
    float R = (sigma == 0.0f) ? 0.0f : 1.0f / sigma;
    for (int i = 0; i < 16; ++i) codes[i] = e2m1_encode(x[i] * R);
    *scale = sc;
}

static void quant16(const float* x, uint8_t* codes, uint8_t* scale) { quant16_k(x, 0, codes, scale); }

/* ------------------------------------------------------------------ exported codec */

OR_EXPORT void or_e2m1_encode(const float* x, size_t n, uint8_t* out) {
#pragma omp parallel for schedule(static)
    for (long long i = 0; i < (long long)n; ++i) out[i] = e2m1_encode(x[i]);
}

OR_EXPORT void or_e4m3_encode(const float* x, size_t n, uint8_t* out) {
#pragma omp parallel for schedule(static)
    for (long long i = 0; i < (long long)n; ++i) out[i] = e4m3_encode_pos(x[i]);
}

OR_EXPORT float or_e2m1_value(uint8_t code) { return e2m1_value(code); }
OR_EXPORT float or_e4m3_value(uint8_t code) { return e4m3_value(code); }

OR_EXPORT void or_exp2(const float* x, size_t n, float* out) {
#pragma omp parallel for schedule(static)
    for (long long i = 0; i < (long long)n; ++i) out[i] = own_exp2(x[i]);
}

/* Block quantiser on an arbitrary fp32 vector (n % 16 == 0): codes packed two per byte,
 * element 2i in the low nibble of byte i. */
OR_EXPORT void or_quant_blocks(const float* x, size_t n, uint8_t* codes, uint8_t* scales) {
#pragma omp parallel for schedule(static)
    for (long long b = 0; b < (long long)(n / 16); ++b) {
        uint8_t c[16];
        quant16(x + 16 * b, c, &scales[b]);
        for (int i = 0; i < 8; ++i) codes[8 * b + i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
    }
}

/* ------------------------------------------------------------------ Smooth-QK calibration */

/* s[g,c] = (amax_K[g,c] / amax_Q[g,c])^alpha in double, rounded once to fp32; s = 1 when
 * either amax is 0; sinv = RN(1/s) in fp32.  amax_Q runs over the batch, the group's query
 * heads and all calibration tokens; amax_K over the batch and tokens of kv head g. */
OR_EXPORT void or_calibrate(const uint16_t* qcal, const uint16_t* kcal, int B, int Hq, int Hkv,
                            int N, int d, double alpha, float* s, float* sinv) {
    int grp = Hq / Hkv;
    for (int g = 0; g < Hkv; ++g) {
        for (int c = 0; c < d; ++c) {
            float aq = 0.0f, ak = 0.0f;
            for (int b = 0; b < B; ++b) {
                for (int hh = 0; hh < grp; ++hh) {
                    const uint16_t* q = qcal + (((size_t)b * Hq + (size_t)g * grp + hh) * N) * d;
                    for (int n = 0; n < N; ++n) aq = fmaxf(aq, fabsf(bf16_to_f32(q[(size_t)n * d + c])));
                }
                const uint16_t* k = kcal + (((size_t)b * Hkv + g) * N) * d;
                for (int n = 0; n < N; ++n) ak = fmaxf(ak, fabsf(bf16_to_f32(k[(size_t)n * d + c])));
            }
            float sv = 1.0f;
            if (aq > 0.0f && ak > 0.0f) sv = (float)pow((double)ak / (double)aq, alpha);
            s[g * d + c] = sv;
            sinv[g * d + c] = 1.0f / sv;
        }
    }
}

/* ------------------------------------------------------------------ quantise Q, K, V^T */

/* x: bf16 [B,H,N,d]; scale: fp32 [Hkv,d] or NULL (no smoothing); group of head h is
 * h / (H/Hkv).  Output codes [B,H,N,d/2] (packed, low nibble first), scales [B,H,N,d/16]. */
OR_EXPORT void or_quantize_rows(const uint16_t* x, int B, int H, int Hkv, int N, int d,
                                const float* scale, uint8_t* codes, uint8_t* scales) {
    int grp = H / Hkv;
    long long rows = (long long)B * H * N;
#pragma omp parallel for schedule(static)
    for (long long r = 0; r < rows; ++r) {
        int h = (int)((r / N) % H);
        int g = h / grp;
        const uint16_t* xr = x + r * d;
        for (int blk = 0; blk < d / 16; ++blk) {
            float v[16];
            uint8_t c[16];
            for (int i = 0; i < 16; ++i) {
                float xv = bf16_to_f32(xr[blk * 16 + i]);
                v[i] = scale ? xv * scale[g * d + blk * 16 + i] : xv;
            }
            quant16(v, c, &scales[r * (d / 16) + blk]);
            for (int i = 0; i < 8; ++i)
                codes[r * (d / 2) + blk * 8 + i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
        }
    }
}

/* Rotate-half RoPE in fp32 before Smooth-QK (the HiFA4 abstract applies the per-channel
 * rescaling after RoPE), for the fused RoPE + Smooth-QK + quantise entry point.  Token n
 * of every (b, h) sits at position n; its angle table is row n of cos, sin [N, d/2]
 * (fp32, supplied by the caller).  With h = d/2, channel pair (i, i + h):
 *   x'_i     = RN(RN(x_i * cos) - RN(x_{i+h} * sin))
 *   x'_{i+h} = RN(RN(x_{i+h} * cos) + RN(x_i * sin)). */
OR_EXPORT void or_rope_rows(const uint16_t* x, int B, int H, int N, int d, const float* cosv,
                            const float* sinv, float* out) {
    int half = d / 2;
    long long rows = (long long)B * H * N;
#pragma omp parallel for schedule(static)
    for (long long r = 0; r < rows; ++r) {
        int n = (int)(r % N);
        const uint16_t* xr = x + r * d;
        float* o = out + r * d;
        for (int i = 0; i < half; ++i) {
            float x1 = bf16_to_f32(xr[i]), x2 = bf16_to_f32(xr[i + half]);
            float c = cosv[(long long)n * half + i], sn = sinv[(long long)n * half + i];
            float a = x1 * c, b = x2 * sn;
            o[i] = a - b;
            float a2 = x2 * c, b2 = x1 * sn;
            o[i + half] = a2 + b2;
        }
    }
}

/* or_quantize_rows on fp32 inputs (the rotated rows of or_rope_rows). */
OR_EXPORT void or_quantize_rows_f32(const float* x, int B, int H, int Hkv, int N, int d,
                                    const float* scale, uint8_t* codes, uint8_t* scales) {
    int grp = H / Hkv;
    long long rows = (long long)B * H * N;
#pragma omp parallel for schedule(static)
    for (long long r = 0; r < rows; ++r) {
        int h = (int)((r / N) % H);
        int g = h / grp;
        const float* xr = x + r * d;
        for (int blk = 0; blk < d / 16; ++blk) {
            float v[16];
            uint8_t c[16];
            for (int i = 0; i < 16; ++i) {
                float xv = xr[blk * 16 + i];
                v[i] = scale ? xv * scale[g * d + blk * 16 + i] : xv;
            }
            quant16(v, c, &scales[r * (d / 16) + blk]);
            for (int i = 0; i < 8; ++i)
                codes[r * (d / 2) + blk * 8 + i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
        }
    }
}

/* V^T: v bf16 [B,Hkv,N,d] -> codes [B,Hkv,d,N/2], scales [B,Hkv,d,N/16]; blocks of 16
 * consecutive tokens of one channel, no smoothing. */
OR_EXPORT void or_quantize_vt(const uint16_t* v, int B, int Hkv, int N, int d,
                              uint8_t* codes, uint8_t* scales) {
    long long rows = (long long)B * Hkv * d;
#pragma omp parallel for schedule(static)
    for (long long r = 0; r < rows; ++r) {
        long long bh = r / d;
        int c = (int)(r % d);
        const uint16_t* vh = v + bh * (long long)N * d;
        for (int blk = 0; blk < N / 16; ++blk) {
            float x[16];
            uint8_t q[16];
            for (int i = 0; i < 16; ++i) x[i] = bf16_to_f32(vh[(size_t)(blk * 16 + i) * d + c]);
            quant16(x, q, &scales[r * (N / 16) + blk]);
            for (int i = 0; i < 8; ++i)
                codes[r * (N / 2) + blk * 8 + i] = (uint8_t)(q[2 * i] | (q[2 * i + 1] << 4));
        }
    }
}

/* ------------------------------------------------------------------ 4-bit dot products */

static inline uint8_t nib(const uint8_t* codes, int i) { return (codes[i >> 1] >> ((i & 1) * 4)) & 15; }

/* Exact value of one 16-block product in units of 2^-20:
 * sum(2a * 2b) [units 1/4] * (scale_a*512) * (scale_b*512) [units 2^-18]. */
static int64_t block_units(const uint8_t* ac, uint8_t as, const uint8_t* bc, uint8_t bs, int blk) {
    int64_t isum = 0;
    for (int e = 0; e < 16; ++e) isum += (int64_t)e2m1_twice(nib(ac, blk * 16 + e)) * e2m1_twice(nib(bc, blk * 16 + e));
    return isum * e4m3_units(as) * e4m3_units(bs);
}

static float units_to_f32(int64_t u) { return ldexpf((float)u, -20); }   /* one RN rounding */

/* One rounding toward zero: keep the 24 leading significant bits of |u|. */
static float units_to_f32_rz(int64_t u) {
    uint64_t a = (uint64_t)(u < 0 ? -u : u);
    int n = 0;
    while (n < 64 && (a >> n) != 0) ++n;          /* bit length */
    if (n > 24) a = (a >> (n - 24)) << (n - 24);
    float f = ldexpf((float)a, -20);              /* exact: a has at most 24 significant bits */
    return u < 0 ? -f : f;
}
static int64_t f32_to_units(float f) { return (int64_t)ldexp((double)f, 20); } /* exact here */

/* S = sum over the d/16 blocks, fp32 result.  Accumulation models (the 4-bit MMA consumes
 * 64 contraction elements = 4 blocks per instruction):
 *   0: each 64-chunk rounded to fp32, chunks added in fp32 (RN) in order
 *   1: acc = RN(acc + exact chunk) per 64-chunk (fused add of the exact chunk sum)
 *   2: the exact dot rounded once
 *   3: acc = RZ(acc + exact chunk) per 64-chunk: the exact sum of the accumulator and the
 *      chunk's four block products, rounded toward zero (what the sm_100 block-scaled
 *      FP4 tensor-core MMA was measured to do by the accumulation probe). */
static float s_dot(const uint8_t* qc, const uint8_t* qs, const uint8_t* kc, const uint8_t* ks,
                   int d, int model) {
    int nblk = d / 16;
    if (model == 2) {
        int64_t t = 0;
        for (int b = 0; b < nblk; ++b) t += block_units(qc, qs[b], kc, ks[b], b);
        return units_to_f32(t);
    }
    float acc = 0.0f;
    for (int ch = 0; ch < nblk / 4 + (nblk % 4 ? 1 : 0); ++ch) {
        int64_t t = 0;
        for (int b = 4 * ch; b < 4 * ch + 4 && b < nblk; ++b) t += block_units(qc, qs[b], kc, ks[b], b);
        if (model == 0) acc = (ch == 0) ? units_to_f32(t) : acc + units_to_f32(t);
        else if (model == 3) acc = units_to_f32_rz(f32_to_units(acc) + t);
        else acc = units_to_f32(f32_to_units(acc) + t);
    }
    return acc;
}

OR_EXPORT void or_qk_scores(const uint8_t* qcodes, const uint8_t* qscales, const uint8_t* kcodes,
                            const uint8_t* kscales, int M, int Nk, int d, int model, float* S) {
#pragma omp parallel for schedule(static)
    for (int i = 0; i < M; ++i)
        for (int k = 0; k < Nk; ++k)
            S[(size_t)i * Nk + k] = s_dot(qcodes + (size_t)i * (d / 2), qscales + (size_t)i * (d / 16),
                                          kcodes + (size_t)k * (d / 2), kscales + (size_t)k * (d / 16), d, model);
}

/* ------------------------------------------------------------------ the online tile loop */

enum { ST_MIRROR = 0, ST_F64 = 1 };

typedef struct {
    /* quantised operands (plain layouts, see the quantisers above) */
    const uint8_t *qc, *qs, *kc, *ks, *vc, *vs;
    /* unquantised bf16 operands (used when quant == 0) */
    const uint16_t *q, *k, *v;
    int B, Hq, Hkv, N, d, causal, bc;
    int quant;        /* 1: S from 4-bit codes and P -> P_hat; 0: fp64 S, P_hat = P */
    int state;        /* ST_MIRROR: fp16 m,l; fp32 O; alpha = E.  ST_F64: fp64 state, exact 2^x */
    int l_from_p;     /* 1: normaliser from unquantised P (the inconsistent formulation) */
    int s_model;
    /* decode / split-KV (all 0 for the square forward): keys per kv head Nk (0 = N), the kv
     * tile range [j0, j1) of this call, and dec_nq > 0 for packed decode rows: query row i
     * holds token i % dec_nq, at position Nk - dec_nq + (i % dec_nq), which sees keys <= it */
    int Nk, j0, j1, dec_nq;
    int two_level;    /* 1: per-(row, tile) second-level P scale 2^k (see the header) */
} loop_args;

/* Per-row output and optional per-tile trace. */
typedef struct {
    double* o;        /* [d] O / l in the state precision */
    uint16_t* o_bf16; /* [d] mirror output, may be NULL */
    float m, l;
    /* trace (may be NULL): per tile j */
    float* tr_m;      /* m after tile j */
    float* tr_p;      /* [ntiles*bc] unquantised P of the tile (relative to that tile's m) */
    float* tr_phat;   /* [ntiles*bc] dequantised P_hat */
    float* o_part;    /* [d] the unnormalised fp32 O accumulator at the end (mirror), may be NULL */
} row_out;

static void row_loop(const loop_args* a, long long row, row_out* out) {
    const int d = a->d, bc = a->bc, N = a->N;
    const int Nk = a->Nk ? a->Nk : N;
    const long long bh = row / N;
    const int i = (int)(row % N);
    const long long pos = a->dec_nq ? (long long)Nk - a->dec_nq + (i % a->dec_nq) : i;
    const int b = (int)(bh / a->Hq), h = (int)(bh % a->Hq);
    const int g = h / (a->Hq / a->Hkv);
    const long long kvh = (long long)b * a->Hkv + g;
    const float c = (float)(1.4426950408889634074 / sqrt((double)d));
    const double cd = 1.4426950408889634074 / sqrt((double)d);

    int ntiles = a->causal ? i / bc + 1 : N / bc;
    int jstart = 0;
    if (a->dec_nq) { jstart = a->j0; ntiles = a->j1; }
    float m16 = -INFINITY, l16 = 0.0f;       /* mirror state */
    double m64 = -INFINITY, l64 = 0.0;       /* f64 state */
    float O32[256];
    double O64[256];
    for (int x = 0; x < d; ++x) { O32[x] = 0.0f; O64[x] = 0.0; }

    double qd[256];
    if (!a->quant)
        for (int x = 0; x < d; ++x) qd[x] = bf16_to_f32(a->q[row * d + x]);

    for (int j = jstart; j < ntiles; ++j) {
        double S[256];
        float Sf[256];
        int valid[256];
        double rowmax = -INFINITY;
        for (int kk = 0; kk < bc; ++kk) {
            int key = j * bc + kk;
            valid[kk] = a->dec_nq ? (key <= pos) : !(a->causal && key > i);
            if (!valid[kk]) { S[kk] = -INFINITY; Sf[kk] = -INFINITY; continue; }
            if (a->quant) {
                Sf[kk] = s_dot(a->qc + row * (d / 2), a->qs + row * (d / 16),
                               a->kc + (kvh * Nk + key) * (d / 2), a->ks + (kvh * Nk + key) * (d / 16),
                               d, a->s_model);
                S[kk] = Sf[kk];
            } else {
                double acc = 0.0;
                for (int x = 0; x < d; ++x) acc += qd[x] * bf16_to_f32(a->k[(kvh * Nk + key) * d + x]);
                S[kk] = acc;
                Sf[kk] = (float)acc;
            }
            if (S[kk] > rowmax) rowmax = S[kk];
        }

        /* new running max */
        float mnew16 = m16;
        double mnew64 = m64;
        if (rowmax != -INFINITY) {
            if (a->quant) {
                float mu = (float)rowmax * c;                 /* RN(rowmax * c) */
                mnew16 = fmaxf(m16, f16_round(mu));
                mnew64 = mnew16;                              /* the quantised path keeps fp16 m */
            } else {
                mnew64 = fmax(m64, rowmax * cd);
                mnew16 = (float)mnew64;
            }
        }
        float mref = (a->state == ST_MIRROR || a->quant) ? mnew16 : (float)mnew64;
        if ((a->quant && mnew16 == -INFINITY) || (!a->quant && mnew64 == -INFINITY)) {
            if (out->tr_m) out->tr_m[j - jstart] = mnew16;
            if (out->tr_p)
                for (int kk = 0; kk < bc; ++kk) { out->tr_p[(j - jstart) * bc + kk] = 0; out->tr_phat[(j - jstart) * bc + kk] = 0; }
            continue;                                         /* nothing seen yet: no-op tile */
        }

        /* P and P_hat of the tile */
        double P[256], Ph[256];
        for (int kk = 0; kk < bc; ++kk) { P[kk] = 0.0; Ph[kk] = 0.0; }
        if (a->quant) {
            /* P of every key (masked keys: S = -inf gives P = 0) */
            float Pf[256];
            float p_t = 0.0f;                                 /* the tile's largest P */
            for (int kk = 0; kk < bc; ++kk) {
                Pf[kk] = own_exp2(fmaf(Sf[kk], c, -mref));
                if (Pf[kk] > p_t) p_t = Pf[kk];
            }
            int k2 = 0;                                       /* second-level scale 2^k2 */
            if (a->two_level) {
                int ex;
                frexpf(p_t, &ex);                             /* p_t = f 2^ex, f in [0.5, 1) */
                k2 = (ex - 1) - 10;
                if (p_t == 0.0f || k2 < -40) k2 = -40;
            }
            /* P_hat: the block quantiser on each 16 consecutive keys of P */
            for (int blk = 0; blk < bc / 16; ++blk) {
                uint8_t code[16], sc;
                quant16_k(Pf + blk * 16, k2, code, &sc);
                float sigma = ldexpf(e4m3_value(sc), k2);
                for (int e = 0; e < 16; ++e) {
                    int kk = blk * 16 + e;
                    P[kk] = Pf[kk];
                    Ph[kk] = (double)e2m1_value(code[e]) * sigma;
                }
            }
        } else {
            for (int kk = 0; kk < bc; ++kk) {
                P[kk] = valid[kk] ? exp2(S[kk] * cd - mnew64) : 0.0;
                Ph[kk] = P[kk];
            }
        }

        /* normaliser contribution of the tile */
        double r = 0.0;
        for (int kk = 0; kk < bc; ++kk) r += a->l_from_p ? P[kk] : Ph[kk];   /* exact for P_hat */

        /* PV contribution of the tile, in fp64 */
        double pv[256];
        for (int x = 0; x < d; ++x) pv[x] = 0.0;
        for (int kk = 0; kk < bc; ++kk) {
            if (Ph[kk] == 0.0) continue;
            int key = j * bc + kk;
            for (int x = 0; x < d; ++x) {
                double vv;
                if (a->quant) {
                    long long vr = kvh * d + x;
                    vv = (double)e2m1_value(nib(a->vc + vr * (Nk / 2), key)) * e4m3_value(a->vs[vr * (Nk / 16) + key / 16]);
                } else {
                    vv = bf16_to_f32(a->v[(kvh * Nk + key) * d + x]);
                }
                pv[x] += Ph[kk] * vv;
            }
        }

        /* state update */
        if (a->state == ST_MIRROR) {
            float alpha = (m16 == -INFINITY) ? 0.0f : own_exp2(m16 - mnew16);
            for (int x = 0; x < d; ++x) {
                if (m16 != -INFINITY && alpha != 1.0f) O32[x] = alpha * O32[x];
                O32[x] = (float)((double)O32[x] + pv[x]);
            }
            l16 = f16_round(fmaf(alpha, l16, (float)r));   /* r exact for P_hat (<= 18 bits) */
            m16 = mnew16;
            m64 = mnew16;
        } else {
            double mo = a->quant ? (double)m16 : m64;
            double mn = a->quant ? (double)mnew16 : mnew64;
            double alpha = (mo == -INFINITY) ? 0.0 : exp2(mo - mn);
            for (int x = 0; x < d; ++x) O64[x] = alpha * O64[x] + pv[x];
            l64 = alpha * l64 + r;
            m16 = mnew16;
            m64 = mn;
        }
        if (out->tr_m) out->tr_m[j - jstart] = a->quant ? mnew16 : (float)mnew64;
        if (out->tr_p)
            for (int kk = 0; kk < bc; ++kk) {
                out->tr_p[(j - jstart) * bc + kk] = (float)P[kk];
                out->tr_phat[(j - jstart) * bc + kk] = (float)Ph[kk];
            }
    }

    if (a->state == ST_MIRROR) {
        if (out->o_part)
            for (int x = 0; x < d; ++x) out->o_part[x] = O32[x];
        for (int x = 0; x < d; ++x) {
            float o = O32[x] / l16;
            if (out->o) out->o[x] = o;
            if (out->o_bf16) out->o_bf16[x] = f32_to_bf16(o);
        }
        out->m = m16;
        out->l = l16;
    } else {
        for (int x = 0; x < d; ++x) {
            double o = O64[x] / l64;
            if (out->o) out->o[x] = o;
            if (out->o_bf16) out->o_bf16[x] = f32_to_bf16((float)o);
        }
        out->m = (float)m64;
        out->l = (float)l64;
    }
}

/* Quantised attention forward over selected rows (row id = (b*Hq + h)*N + i; rows == NULL
 * means all rows in order).  state: 0 mirror (fp16 m, l), 1 fp64 state with exact 2^x.
 * l_from_p: 1 selects the inconsistent normaliser (sum of unquantised P).
 * two_level: 1 selects the two-level P scale (see the header).
 * Outputs per selected row r: o_f64[r*d..] (may be NULL), o_bf16[r*d..] (may be NULL),
 * m_out[r], l_out[r] (fp32 holding the state value). */
OR_EXPORT int or_attn_fwd(const uint8_t* qc, const uint8_t* qs, const uint8_t* kc, const uint8_t* ks,
                          const uint8_t* vtc, const uint8_t* vts, int B, int Hq, int Hkv, int N, int d,
                          int causal, int bc, int state, int l_from_p, int two_level, int s_model,
                          const long long* rows, long long nrows,
                          double* o_f64, uint16_t* o_bf16, float* m_out, float* l_out) {
    if (d % 16 || d > 256 || bc % 16 || bc > 256 || N % bc || Hq % Hkv) return -1;
    loop_args a = {qc, qs, kc, ks, vtc, vts, NULL, NULL, NULL, B, Hq, Hkv, N, d, causal, bc,
                   1, state, l_from_p, s_model, 0, 0, 0, 0, two_level};
    long long n = rows ? nrows : (long long)B * Hq * N;
#pragma omp parallel for schedule(dynamic, 16)
    for (long long r = 0; r < n; ++r) {
        row_out o = {o_f64 ? o_f64 + r * d : NULL, o_bf16 ? o_bf16 + r * d : NULL, 0, 0, NULL, NULL, NULL};
        row_loop(&a, rows ? rows[r] : r, &o);
        if (m_out) m_out[r] = o.m;
        if (l_out) l_out[r] = o.l;
    }
    return 0;
}

/* The same online tile loop with quantisation off and fp64 state (exact 2^x): must agree
 * with textbook softmax attention to rounding. */
OR_EXPORT int or_attn_loop_exact(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int Hq,
                                 int Hkv, int N, int d, int causal, int bc,
                                 const long long* rows, long long nrows, double* o_f64) {
    if (d > 256 || bc > 256 || N % bc || Hq % Hkv) return -1;
    loop_args a = {NULL, NULL, NULL, NULL, NULL, NULL, q, k, v, B, Hq, Hkv, N, d, causal, bc,
                   0, ST_F64, 0, 0};
    long long n = rows ? nrows : (long long)B * Hq * N;
#pragma omp parallel for schedule(dynamic, 16)
    for (long long r = 0; r < n; ++r) {
        row_out o = {o_f64 + r * d, NULL, 0, 0, NULL, NULL, NULL};
        row_loop(&a, rows ? rows[r] : r, &o);
    }
    return 0;
}

/* Per-tile trace of one row of the quantised loop (state as in or_attn_fwd). */
OR_EXPORT int or_attn_trace(const uint8_t* qc, const uint8_t* qs, const uint8_t* kc, const uint8_t* ks,
                            const uint8_t* vtc, const uint8_t* vts, int B, int Hq, int Hkv, int N, int d,
                            int causal, int bc, int state, int l_from_p, int two_level, int s_model, long long row,
                            float* tr_m, float* tr_p, float* tr_phat, double* o_f64, float* ml) {
    if (d % 16 || d > 256 || bc % 16 || bc > 256 || N % bc || Hq % Hkv) return -1;
    loop_args a = {qc, qs, kc, ks, vtc, vts, NULL, NULL, NULL, B, Hq, Hkv, N, d, causal, bc,
                   1, state, l_from_p, s_model, 0, 0, 0, 0, two_level};
    row_out o = {o_f64, NULL, 0, 0, tr_m, tr_p, tr_phat};
    row_loop(&a, row, &o);
    ml[0] = o.m;
    ml[1] = o.l;
    return 0;
}

/* Decode / split-KV attention (a short query against a long key sequence).
 * Q_hat is packed per (batch b, kv head g): [B, Hkv, 128, d] (plain code / scale layouts),
 * row r = hi * nq + t holding token t of query head g * G + hi; rows >= G * nq are unused.
 * Token t sits at position Nk - nq + t and sees the keys <= that position.  The Nk / bc kv
 * tiles are cut into nsplit runs of T = ceil((Nk / bc) / nsplit) tiles; for every row and
 * split s the tile loop of or_attn_fwd runs over the split's tiles from the initial state
 * (m = -inf, l = 0, O = 0), giving m_s, l_s (fp16 values) and the fp32 accumulator O_s.
 * The partials are merged in fp32, splits in order:
 *   m = max_s m_s;  w_s = E(m_s - m) (0 when m_s = -inf, exactly 1 when m_s = m);
 *   L = fma(w_s, l_s, L) from L = 0;  O = fma(w_s, O_s, O) from O = 0;
 *   out = bf16_RN(RN(O * RN(1 / L))) (0 when L = 0);  m_out = m, l_out = fp16_RN(L).
 * o_bf16: [B, Hkv * G, nq, d]; m_out, l_out: [B, Hkv * G, nq] (fp32 holding the values);
 * part_o [B * Hkv, nsplit, 128, d] and part_ml [B * Hkv, nsplit, 128, 2] (may be NULL)
 * receive the partials of the used rows. */
OR_EXPORT int or_attn_decode(const uint8_t* qc, const uint8_t* qs, const uint8_t* kc, const uint8_t* ks,
                             const uint8_t* vtc, const uint8_t* vts, int B, int Hkv, int G, int nq, int Nk, int d,
                             int bc, int nsplit, int s_model, uint16_t* o_bf16, float* m_out, float* l_out,
                             float* part_o, float* part_ml) {
    if (d % 16 || d > 256 || bc % 16 || bc > 256 || Nk % bc || G * nq > 128 || nsplit < 1 || nsplit > 64) return -1;
    const int ntile = Nk / bc, T = (ntile + nsplit - 1) / nsplit;
    const long long nrows = (long long)B * Hkv * G * nq;
#pragma omp parallel for schedule(dynamic, 1)
    for (long long idx = 0; idx < nrows; ++idx) {
        const long long bkv = idx / (G * nq);
        const int r = (int)(idx % (G * nq));
        float mp[64], lp[64];
        static __thread float op[64][256];
        for (int sp = 0; sp < nsplit; ++sp) {
            int j0 = sp * T, j1 = j0 + T < ntile ? j0 + T : ntile;
            if (j0 > ntile) j0 = ntile;
            /* the packed rows form Hkv "heads" of 128 query rows each */
            loop_args a = {qc, qs, kc, ks, vtc, vts, NULL, NULL, NULL, B, Hkv, Hkv, 128, d, 0, bc,
                           1, ST_MIRROR, 0, s_model, Nk, j0, j1, nq};
            double o64[256];
            row_out o = {o64, NULL, 0, 0, NULL, NULL, NULL, op[sp]};
            row_loop(&a, bkv * 128 + r, &o);
            if (j0 >= j1) { o.m = -INFINITY; o.l = 0.0f; for (int x = 0; x < d; ++x) op[sp][x] = 0.0f; }
            mp[sp] = o.m;
            lp[sp] = o.l;
            if (part_o)
                for (int x = 0; x < d; ++x) part_o[((bkv * nsplit + sp) * 128 + r) * d + x] = op[sp][x];
            if (part_ml) {
                part_ml[((bkv * nsplit + sp) * 128 + r) * 2] = o.m;
                part_ml[((bkv * nsplit + sp) * 128 + r) * 2 + 1] = o.l;
            }
        }
        float m = -INFINITY;
        for (int sp = 0; sp < nsplit; ++sp) m = fmaxf(m, mp[sp]);
        float L = 0.0f, O[256];
        for (int x = 0; x < d; ++x) O[x] = 0.0f;
        for (int sp = 0; sp < nsplit; ++sp) {
            float w = (mp[sp] == -INFINITY) ? 0.0f : own_exp2(mp[sp] - m);
            L = fmaf(w, lp[sp], L);
            for (int x = 0; x < d; ++x) O[x] = fmaf(w, op[sp][x], O[x]);
        }
        const int hi = r / nq, t = r % nq;
        const long long orow = ((bkv / Hkv) * (long long)(Hkv * G) + (bkv % Hkv) * G + hi) * nq + t;
        float inv = (L > 0.0f) ? 1.0f / L : 0.0f;
        for (int x = 0; x < d; ++x) o_bf16[orow * d + x] = f32_to_bf16(O[x] * inv);
        m_out[orow] = m;
        l_out[orow] = f16_round(L);
    }
    return 0;
}

/* Textbook softmax attention in fp64 (no tiles, no quantisation):
 * O_i = sum_k softmax_k(q_i . k_k / sqrt(d)) v_k over keys k <= i when causal. */
OR_EXPORT int or_attn_bruteforce(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int Hq,
                                 int Hkv, int N, int d, int causal,
                                 const long long* rows, long long nrows, double* o_f64) {
    long long n = rows ? nrows : (long long)B * Hq * N;
#pragma omp parallel for schedule(dynamic, 4)
    for (long long r = 0; r < n; ++r) {
        long long row = rows ? rows[r] : r;
        long long bh = row / N;
        int i = (int)(row % N), b = (int)(bh / Hq), h = (int)(bh % Hq), g = h / (Hq / Hkv);
        long long kvh = (long long)b * Hkv + g;
        int nk = causal ? i + 1 : N;
        double* s = (double*)malloc(sizeof(double) * nk);
        double mx = -INFINITY;
        for (int key = 0; key < nk; ++key) {
            double acc = 0.0;
            for (int x = 0; x < d; ++x) acc += (double)bf16_to_f32(q[row * d + x]) * bf16_to_f32(k[(kvh * N + key) * d + x]);
            s[key] = acc / sqrt((double)d);
            if (s[key] > mx) mx = s[key];
        }
        double den = 0.0;
        for (int key = 0; key < nk; ++key) { s[key] = exp(s[key] - mx); den += s[key]; }
        for (int x = 0; x < d; ++x) {
            double acc = 0.0;
            for (int key = 0; key < nk; ++key) acc += s[key] * bf16_to_f32(v[(kvh * N + key) * d + x]);
            o_f64[r * d + x] = acc / den;
        }
        free(s);
    }
    return 0;
}

OR_EXPORT uint16_t or_f16_bits(float f) { return f16_bits(f); }

OR_EXPORT int or_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
