// Device-side arithmetic of the HiFA4-style 4-bit attention ("HiFA4: Training-Free 4-bit
// FlashAttention on Ascend HIF4 NPUs for LLM Inference", abstract): the 4-bit block
// format, the softmax's exp2 and the fixed layouts shared by the kernels of this library.
//
// 4-bit format (the abstract names HIF4 without giving its layout; this library uses an
// NVFP4-style layout): E2M1 codes, one unsigned E4M3 scale per 16 consecutive
// contraction elements.  scale = E4M3_RN(amax * RN(1/6)); R = RN(1/scale), or 0 when the
// scale is 0; code = E2M1_RN_satfinite(x * R).  Two codes per byte, element 2i in the low
// nibble.
#pragma once
#include "ptx.cuh"

namespace hifa4 {

// RN(1/6) in fp32.
constexpr float kSixth = 0x1.555556p-3f;

// The softmax's exp2: E(x) = p(f) * 2^n with x' = max(x, -127), n = floor(x'),
// f = RN(x' - n) and p(f) = ((c3 f + c2) f + c1) f + 1 evaluated with fused multiply-adds;
// the coefficients are a minimax fit of 2^f on [0, 1) in relative error with p(0) = 1 held
// exact (max relative error 8.6e-5).  The floor uses a round-down add of 1.5 * 2^23, whose
// low mantissa bits then hold n, so the exponent insert is one integer multiply-add.
constexpr float kExp2C1 = 0x1.63e65ap-1f;
constexpr float kExp2C2 = 0x1.d23788p-3f;
constexpr float kExp2C3 = 0x1.3baaa8p-4f;

// bits(p) + (n << 23), with n in the low bits of v's pattern (v = floor(x') + 1.5 * 2^23).
__device__ __forceinline__ float insert_exponent(float p, float v) {
  uint32_t r;
  asm("mad.lo.u32 %0, %1, 8388608, %2;" : "=r"(r) : "r"(__float_as_uint(v)), "r"(__float_as_uint(p)));
  return __uint_as_float(r);
}

__device__ __forceinline__ float exp2_own(float x) {
  const float xc = fmaxf(x, -127.0f);
  const float v = __fadd_rd(xc, 12582912.0f);
  const float n = __fsub_rn(v, 12582912.0f);
  const float f = __fsub_rn(xc, n);                                        // RN(xc - n)
  const float p = __fmaf_rn(__fmaf_rn(__fmaf_rn(kExp2C3, f, kExp2C2), f, kExp2C1), f, 1.0f);
  return insert_exponent(p, v);
}

// E(x) on a pair of values with the packed fp32 instructions of sm_100 (two lanes per
// instruction, each rounded exactly as the scalar form): bit-identical to exp2_own.
__device__ __forceinline__ float2 exp2_own2(float2 x) {
  const float2 xc = make_float2(fmaxf(x.x, -127.0f), fmaxf(x.y, -127.0f));
  const float2 v = __fadd2_rd(xc, make_float2(12582912.0f, 12582912.0f));
  const float2 n = __fadd2_rn(v, make_float2(-12582912.0f, -12582912.0f));
  const float2 f = __ffma2_rn(n, make_float2(-1.0f, -1.0f), xc);          // RN(xc - n)
  float2 p = __ffma2_rn(make_float2(kExp2C3, kExp2C3), f, make_float2(kExp2C2, kExp2C2));
  p = __ffma2_rn(p, f, make_float2(kExp2C1, kExp2C1));
  p = __ffma2_rn(p, f, make_float2(1.0f, 1.0f));
  return make_float2(insert_exponent(p.x, v.x), insert_exponent(p.y, v.y));
}

// P_hat codes, fast approximate form (a separate entry point, never the default): the
// code of a score is decided in the log domain.  With the per-block bias
// B = (L(sigma) - m + 125)/128, L(sigma) = RN(-log2 sigma), a score's u = sat(S * c/128 + B)
// holds log2(P / sigma) + 125 scaled into [0, 1].  The code is the E2M1 rounding of the
// linear-mantissa exponential y = 2^floor(z) * (1 + frac z) of z = 128 u - 125 + delta on a
// 2^-10 grid (delta = -73/1024 puts the E2M1 rounding boundaries within 0.014 log2 units
// of those of the exact exponential, the lowest within 0.071).  One fma forms
// v = 128 u + kPhatM, kPhatM = 8194 + delta: v lies in [2^13, 2^14), whose spacing is
// 2^-10, so v's mantissa field is (z + 127) * 2^10, and shifting v's bits left by 13
// leaves exactly the bits of y (exponent floor(z) + 127, top ten mantissa bits frac z).
// The default path instead rounds RN(P * RN(1/sigma)) to E2M1, the block quantiser's
// own rule.
constexpr float kPhatM = 8193.9287109375f;   // 8194 - 73/1024

__device__ __forceinline__ float fma_sat(float a, float b, float c) {
  float d;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ float2 phat_pair(float2 u) {
  const float2 v = __ffma2_rn(u, make_float2(128.0f, 128.0f), make_float2(kPhatM, kPhatM));
  return make_float2(__uint_as_float(__float_as_uint(v.x) << 13), __uint_as_float(__float_as_uint(v.y) << 13));
}

// Eight values held as four pairs (element 2k in .x) -> eight E2M1 codes, low nibble first.
__device__ __forceinline__ uint32_t encode8_pairs(const float2 (&y)[4]) {
  uint32_t w;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(w)
      : "f"(y[0].x), "f"(y[0].y), "f"(y[1].x), "f"(y[1].y), "f"(y[2].x), "f"(y[2].y), "f"(y[3].x), "f"(y[3].y));
  return w;
}

// Scale code of a block from its absolute maximum, reciprocal from the table below.
__device__ __forceinline__ uint32_t block_scale_tab(float amax, const float* rtab, float& R) {
  const uint32_t sc = cvt_e4m3(__fmul_rn(amax, kSixth));
  R = rtab[sc];
  return sc;
}

// RN(1/scale) for every E4M3 code (0 for the zero scale and for codes that are not
// finite positive scales), filled once per CTA so a block's reciprocal is one load.
__device__ __forceinline__ void fill_recip_table(float* tab, int tid, int nthreads) {
  for (int i = tid; i < 256; i += nthreads) {
    const float v = e4m3_value((uint32_t)i);
    tab[i] = (v > 0.0f && v <= 448.0f) ? __frcp_rn(v) : 0.0f;
  }
}

// Byte offset of row r (0..127), block s (0..3) inside a 512-byte scale-factor atom:
// the layout tcgen05.cp.32x128b.warpx4 expects (rows r and r+32k share a 16-byte record).
__host__ __device__ __forceinline__ uint32_t sf_atom_offset(uint32_t r, uint32_t s) {
  return (r & 31u) * 16u + (r >> 5) * 4u + s;
}

// Byte offset of 16-byte chunk `chunk` of row `r` in a K-major operand tile whose rows
// are `rowbytes` (32, 64 or 128) long, stored with the matching TMA/UMMA swizzle.
__host__ __device__ __forceinline__ uint32_t swz_offset(uint32_t r, uint32_t chunk, uint32_t rowbytes) {
  const uint32_t a = r * rowbytes + chunk * 16u;
  const uint32_t mask = rowbytes / 16u - 1u;   // 1, 3 or 7
  return a ^ (((a >> 7) & mask) << 4);
}

}  // namespace hifa4
