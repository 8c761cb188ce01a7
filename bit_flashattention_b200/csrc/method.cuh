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

// The softmax's exp2: E(x) = p(f) * 2^n with x' = max(x, -127), n = floor(x'), f = x' - n
// and p(f) = ((c3 f + c2) f + c1) f + 1 evaluated with fused multiply-adds; the
// coefficients are a minimax fit of 2^f on [0, 1) in relative error with p(0) = 1 held
// exact (max relative error 8.6e-5).  The floor uses a round-down add of 1.5 * 2^23,
// whose low mantissa bits then hold n, so the exponent insert is one shift-add.
constexpr float kExp2C1 = 0x1.63e65ap-1f;
constexpr float kExp2C2 = 0x1.d23788p-3f;
constexpr float kExp2C3 = 0x1.3baaa8p-4f;

__device__ __forceinline__ float exp2_own(float x) {
  const float xc = fmaxf(x, -127.0f);
  const float v = __fadd_rd(xc, 12582912.0f);
  const float n = __fsub_rn(v, 12582912.0f);
  const float f = __fsub_rn(xc, n);
  const float p = __fmaf_rn(__fmaf_rn(__fmaf_rn(kExp2C3, f, kExp2C2), f, kExp2C1), f, 1.0f);
  return __uint_as_float(__float_as_uint(p) + (__float_as_uint(v) << 23));
}

// Scale code and reciprocal of a block from its absolute maximum.
__device__ __forceinline__ uint32_t block_scale(float amax, float& R) {
  const uint32_t sc = cvt_e4m3(__fmul_rn(amax, kSixth));
  const float sig = e4m3_value(sc);
  R = (sig == 0.0f) ? 0.0f : __frcp_rn(sig);
  return sc;
}

// Eight values -> eight E2M1 codes (after multiplying by R), packed low nibble first.
__device__ __forceinline__ uint32_t encode8(const float (&x)[8], float R) {
  uint32_t w = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k)
    w |= cvt_e2m1x2(__fmul_rn(x[2 * k + 1], R), __fmul_rn(x[2 * k], R)) << (8 * k);
  return w;
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
