// Quantiser kernels (HBM-bound): Smooth-QK application + 4-bit block quantisation of Q
// and K along the head dimension, the transposing quantisation of V (blocks of 16
// tokens per channel), and the per-channel amax reduction of the Smooth-QK calibration.
//
// Smooth-QK ("HiFA4: Training-Free 4-bit FlashAttention on Ascend HIF4 NPUs for LLM
// Inference", abstract): after RoPE, Q is multiplied and K divided per channel by scales s
// that an offline calibration fixes, so inference computes no statistics for it.  Here q' = RN(q * s[g,c])
// and k' = RN(k * s_inv[g,c]) with g the kv head of the query head.
#pragma once
#include "method.cuh"

namespace hifa4 {

struct QuantRowsArgs {
  const __nv_bfloat16* x;     // [B, H, N, D] with strides (sb, sh, sn) in elements, d contiguous
  long long sb, sh, sn;
  int H, Hkv, N;
  const float* scale;         // [Hkv, D] or nullptr
  const float* rope_cos;      // [N, D/2] fp32 angle tables of the fused RoPE path, or nullptr
  const float* rope_sin;
  int pack_G, pack_nq;        // decode packing (0 = off): see quant_rows_unit
  uint8_t* codes;             // [B, H, N, D/2]
  uint8_t* sf;                // [B, H, N/128, D/64, 512]
  int units;                  // B * H * N / ROWS (ROWS rows of one head per unit)
};

// max(|a|, |b|, |c|), NaN if any input is NaN.
__device__ __forceinline__ float max3_abs_nan(float a, float b, float c) {
  float d;
  asm("max.NaN.abs.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

template <int D>
struct RowsUnit {
  static constexpr int BPR = D / 16;                  // blocks per row
  static constexpr int RPP = 256 / BPR;               // rows per pass
  static constexpr int ROWS = D == 256 ? 64 : 128;    // rows per unit
  static constexpr int PASSES = ROWS / RPP;
};

// One unit (ROWS rows of one head) of the Q/K quantiser with 256 threads.  Thread
// (row r, block k) quantises one 16-element block: two 16-byte loads (all of a thread's
// loads in flight before any arithmetic), the block amax with 3-input max instructions,
// the scale from the amax and its reciprocal from a shared table, 8 code bytes and the
// scale byte stored directly; one NaN-propagating maximum per thread carries the
// non-finite check.
//
// PACK: the unit is the 128-row decode tile of kv head h (H = Hkv): row r < G * nq is token
// r % nq of query head h * G + r / nq of the [B, Hq, nq, D] input, rows >= G * nq are zero.
template <int D, bool PACK = false>
__device__ __forceinline__ void quant_rows_unit(const QuantRowsArgs& a, int unit, const float* rtab, bool& bad) {
  using U = RowsUnit<D>;
  const int blk = threadIdx.x % U::BPR;
  const int rsub = threadIdx.x / U::BPR;
  const int per_head = a.N / U::ROWS;
  const int bh = unit / per_head, n0 = (unit % per_head) * U::ROWS;
  const int b = bh / a.H, h = bh % a.H, g = h / (a.H / a.Hkv);
  const __nv_bfloat16* base = a.x + b * a.sb + h * a.sh + blk * 16;
  uint4 raw[U::PASSES][2];
#pragma unroll
  for (int k = 0; k < U::PASSES; ++k) {
    const int rr = n0 + rsub + k * U::RPP;
    if constexpr (PACK) {
      if (rr < a.pack_G * a.pack_nq) {
        const uint4* src = reinterpret_cast<const uint4*>(a.x + b * a.sb + (long long)(h * a.pack_G + rr / a.pack_nq) * a.sh +
                                                          (long long)(rr % a.pack_nq) * a.sn + blk * 16);
        raw[k][0] = src[0];
        raw[k][1] = src[1];
      } else {
        raw[k][0] = make_uint4(0, 0, 0, 0);
        raw[k][1] = make_uint4(0, 0, 0, 0);
      }
      continue;
    }
    const uint4* src = reinterpret_cast<const uint4*>(base + (long long)rr * a.sn);
    raw[k][0] = src[0];
    raw[k][1] = src[1];
  }
  float2 s2[8];
  if (a.scale) {
    const float4* sp = reinterpret_cast<const float4*>(a.scale + g * D + blk * 16);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 t = __ldg(sp + q);
      s2[2 * q] = make_float2(t.x, t.y);
      s2[2 * q + 1] = make_float2(t.z, t.w);
    }
  }
  float nan_acc = 0.0f;                                // NaN / inf of any block amax survives the max
#pragma unroll
  for (int k = 0; k < U::PASSES; ++k) {
    const int row = n0 + rsub + k * U::RPP;
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw[k][0]);
    float2 v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = __bfloat1622float2(p2[e]);
    if (a.scale) {
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = __fmul2_rn(v[e], s2[e]);
    }
    float amax = 0.0f;
#pragma unroll
    for (int e = 0; e < 8; ++e) amax = max3_abs_nan(amax, v[e].x, v[e].y);
    nan_acc = max3_abs_nan(nan_acc, amax, amax);
    float R;
    const uint32_t sc = block_scale_tab(amax, rtab, R);
    const float2 R2 = make_float2(R, R);
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = __fmul2_rn(v[e], R2);
    const float2 lo[4] = {v[0], v[1], v[2], v[3]}, hi[4] = {v[4], v[5], v[6], v[7]};
    *reinterpret_cast<uint2*>(a.codes + ((long long)bh * a.N + row) * (D / 2) + blk * 8) =
        make_uint2(encode8_pairs(lo), encode8_pairs(hi));
    // the block's scale byte: block (blk & 3) of its 64-wide chunk in the row's record
    uint8_t* atom = a.sf + (((long long)bh * (a.N / 128) + row / 128) * (D / 64) + blk / 4) * 512;
    atom[sf_atom_offset(row % 128, blk & 3)] = (uint8_t)sc;
  }
  bad |= !isfinite(nan_acc);
}

// Smooth-QK (when a.scale), amax, scale and codes of one 16-element block (row `row` of
// head bh, block blk, values v): 8 code bytes and the scale byte (block blk & 3 of its
// 64-wide chunk in the row's atom record).  nan_acc carries a NaN or infinity of any amax.
template <int D>
__device__ __forceinline__ void quant_block16(const QuantRowsArgs& a, int bh, int g, int row, int blk, float2 (&v)[8],
                                              const float* rtab, float& nan_acc) {
  if (a.scale) {
    const float4* sp = reinterpret_cast<const float4*>(a.scale + g * D + blk * 16);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 t = __ldg(sp + q);
      v[2 * q] = __fmul2_rn(v[2 * q], make_float2(t.x, t.y));
      v[2 * q + 1] = __fmul2_rn(v[2 * q + 1], make_float2(t.z, t.w));
    }
  }
  float amax = 0.0f;
#pragma unroll
  for (int e = 0; e < 8; ++e) amax = max3_abs_nan(amax, v[e].x, v[e].y);
  nan_acc = max3_abs_nan(nan_acc, amax, amax);
  float R;
  const uint32_t sc = block_scale_tab(amax, rtab, R);
  const float2 R2 = make_float2(R, R);
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] = __fmul2_rn(v[e], R2);
  const float2 lo[4] = {v[0], v[1], v[2], v[3]}, hi[4] = {v[4], v[5], v[6], v[7]};
  *reinterpret_cast<uint2*>(a.codes + ((long long)bh * a.N + row) * (D / 2) + blk * 8) =
      make_uint2(encode8_pairs(lo), encode8_pairs(hi));
  uint8_t* atom = a.sf + (((long long)bh * (a.N / 128) + row / 128) * (D / 64) + blk / 4) * 512;
  atom[sf_atom_offset(row % 128, blk & 3)] = (uint8_t)sc;
}

// Fused RoPE unit (ROWS rows of one head, pre-RoPE input) with one thread per
// rotate-half block pair: thread (row r, pair p) loads blocks p and p + D/32 of its row
// (channels c and c + D/2 pair up element by element) and the pair's 16 angle-table
// columns once, rotates in fp32 with every product and sum rounded once,
//   x'_c = RN(RN(x_c cos) - RN(x_{c+D/2} sin)),  x'_{c+D/2} = RN(RN(x_{c+D/2} cos) + RN(x_c sin)),
// then applies Smooth-QK and quantises both blocks.
template <int D>
struct RopeUnit {
  static constexpr int HB = D / 32;                   // block pairs per row
  static constexpr int RPP = 256 / HB;                // rows per pass
  static constexpr int ROWS = RowsUnit<D>::ROWS;      // rows per unit (the host's unit count)
  static constexpr int PASSES = ROWS / RPP;
};

template <int D>
__device__ __forceinline__ void quant_rows_rope_pair(const QuantRowsArgs& a, int unit, const float* rtab, bool& bad) {
  using U = RopeUnit<D>;
  const int pr = threadIdx.x % U::HB, rsub = threadIdx.x / U::HB;
  const int per_head = a.N / U::ROWS;
  const int bh = unit / per_head, n0 = (unit % per_head) * U::ROWS;
  const int b = bh / a.H, h = bh % a.H, g = h / (a.H / a.Hkv);
  const __nv_bfloat16* base = a.x + b * a.sb + h * a.sh + pr * 16;
  float nan_acc = 0.0f;
#pragma unroll
  for (int k = 0; k < U::PASSES; ++k) {
    const int row = n0 + rsub + k * U::RPP;
    const uint4* src = reinterpret_cast<const uint4*>(base + (long long)row * a.sn);
    uint4 x1[2], x2[2];
    x1[0] = src[0];
    x1[1] = src[1];
    x2[0] = src[2 * U::HB];                           // the partner block, D/2 channels on
    x2[1] = src[2 * U::HB + 1];
    const float4* cp = reinterpret_cast<const float4*>(a.rope_cos + (long long)row * (D / 2) + pr * 16);
    const float4* sp = reinterpret_cast<const float4*>(a.rope_sin + (long long)row * (D / 2) + pr * 16);
    float4 c4[4], s4[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      c4[q] = __ldg(cp + q);
      s4[q] = __ldg(sp + q);
    }
    const __nv_bfloat162* p1 = reinterpret_cast<const __nv_bfloat162*>(&x1[0]);
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&x2[0]);
    float2 v1[8], v2[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float2 a1 = __bfloat1622float2(p1[e]), a2 = __bfloat1622float2(p2[e]);
      const float2 cc = (e & 1) ? make_float2(c4[e >> 1].z, c4[e >> 1].w) : make_float2(c4[e >> 1].x, c4[e >> 1].y);
      const float2 ss = (e & 1) ? make_float2(s4[e >> 1].z, s4[e >> 1].w) : make_float2(s4[e >> 1].x, s4[e >> 1].y);
      // scalar intrinsics: each product is rounded before the sum (never contracted)
      v1[e] = make_float2(__fsub_rn(__fmul_rn(a1.x, cc.x), __fmul_rn(a2.x, ss.x)),
                          __fsub_rn(__fmul_rn(a1.y, cc.y), __fmul_rn(a2.y, ss.y)));
      v2[e] = make_float2(__fadd_rn(__fmul_rn(a2.x, cc.x), __fmul_rn(a1.x, ss.x)),
                          __fadd_rn(__fmul_rn(a2.y, cc.y), __fmul_rn(a1.y, ss.y)));
    }
    quant_block16<D>(a, bh, g, row, pr, v1, rtab, nan_acc);
    quant_block16<D>(a, bh, g, row, pr + U::HB, v2, rtab, nan_acc);
  }
  bad |= !isfinite(nan_acc);
}

// Grid-stride over Q units then K units.
template <int D>
__global__ void __launch_bounds__(256) k_quant_rows(QuantRowsArgs qa, QuantRowsArgs ka, int* status) {
  __shared__ float rtab[256];
  fill_recip_table(rtab, threadIdx.x, 256);
  __syncthreads();
  bool bad = false;
  for (int u = blockIdx.x; u < qa.units + ka.units; u += gridDim.x) {
    if (u < qa.units) quant_rows_unit<D>(qa, u, rtab, bad);
    else quant_rows_unit<D>(ka, u - qa.units, rtab, bad);
  }
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, ST_NONFINITE);
}

// Decode Q packing + Smooth-QK + quantise: one 128-row unit per (batch, kv head).
template <int D>
__global__ void __launch_bounds__(256) k_quant_q_decode(QuantRowsArgs qa, int* status) {
  __shared__ float rtab[256];
  fill_recip_table(rtab, threadIdx.x, 256);
  __syncthreads();
  bool bad = false;
  for (int u = blockIdx.x; u < qa.units; u += gridDim.x) quant_rows_unit<D, true>(qa, u, rtab, bad);
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, ST_NONFINITE);
}

// Fused RoPE + Smooth-QK + quantise of Q and K (pre-RoPE inputs), grid-stride over Q units
// then K units.
template <int D>
__global__ void __launch_bounds__(256, 2) k_quant_rows_rope(QuantRowsArgs qa, QuantRowsArgs ka, int* status) {
  __shared__ float rtab[256];
  fill_recip_table(rtab, threadIdx.x, 256);
  __syncthreads();
  bool bad = false;
  for (int u = blockIdx.x; u < qa.units + ka.units; u += gridDim.x) {
    if (u < qa.units) quant_rows_rope_pair<D>(qa, u, rtab, bad);
    else quant_rows_rope_pair<D>(ka, u - qa.units, rtab, bad);
  }
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, ST_NONFINITE);
}

struct QuantVtArgs {
  const __nv_bfloat16* v;     // [B, Hkv, N, D] with strides, d contiguous
  long long sb, sh, sn;
  int H, N;
  uint8_t* codes;             // [B, Hkv, D, N/2]
  uint8_t* sf;                // [B, Hkv, N/64, ceil(D/128), 512]
  int units;                  // B * Hkv * N / TOK for the kernel's TOK
};

// One unit (TOK consecutive tokens of one kv head, TOK = 32 with 128 threads or 64 with
// 256 threads) of the transposing V quantiser.  The TOK x D tile is staged in shared
// memory with coalesced 16-byte loads (all of a thread's loads in flight first); then item
// (channel c, 32-token half) quantises the half's two 16-token blocks of channel c and
// writes their 16 code bytes and its 2 bytes of the channel's scale word.  For D = 64 the
// unused rows 64..127 of the 128-channel atom are zeroed.
template <int D, int TOK, int NT>
__device__ __forceinline__ void quant_vt_unit(const QuantVtArgs& a, int unit, __nv_bfloat16* tile, const float* rtab,
                                              bool& bad) {
  constexpr int NAV = (D + 127) / 128;
  constexpr int LD = D + 8;                     // padded staging row (bf16 elements)
  constexpr int LOADS = TOK * (D / 8) / NT;     // 16-byte loads per thread
  const int nunit = a.N / TOK;
  const int bh = unit / nunit, t0 = (unit % nunit) * TOK;
  const int b = bh / a.H, h = bh % a.H;
  const __nv_bfloat16* src = a.v + b * a.sb + h * a.sh + (long long)t0 * a.sn;
  uint4 raw[LOADS];
#pragma unroll
  for (int k = 0; k < LOADS; ++k) {
    const int it = threadIdx.x + k * NT;
    raw[k] = *reinterpret_cast<const uint4*>(src + (it / (D / 8)) * a.sn + (it % (D / 8)) * 8);
  }
  __syncthreads();                            // the previous unit's readers are done with the tile
#pragma unroll
  for (int k = 0; k < LOADS; ++k) {
    const int it = threadIdx.x + k * NT;
    *reinterpret_cast<uint4*>(&tile[(it / (D / 8)) * LD + (it % (D / 8)) * 8]) = raw[k];
  }
  __syncthreads();
#pragma unroll
  for (int it = threadIdx.x; it < (TOK / 32) * D; it += NT) {
    const int c = it % D, hh = it / D;
    const int half = t0 / 32 + hh, ch = half >> 1, hb = half & 1;
    uint32_t w[4];
    uint32_t sc2 = 0;
#pragma unroll
    for (int blk = 0; blk < 2; ++blk) {
      float2 x[8];
      float amax = 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        x[e] = make_float2(__bfloat162float(tile[(hh * 32 + blk * 16 + 2 * e) * LD + c]),
                           __bfloat162float(tile[(hh * 32 + blk * 16 + 2 * e + 1) * LD + c]));
        amax = max3_abs_nan(amax, x[e].x, x[e].y);
      }
      bad |= !isfinite(amax);
      float R;
      sc2 |= block_scale_tab(amax, rtab, R) << (8 * blk);
      const float2 R2 = make_float2(R, R);
      float2 lo[4], hi[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        lo[e] = __fmul2_rn(x[e], R2);
        hi[e] = __fmul2_rn(x[4 + e], R2);
      }
      w[2 * blk] = encode8_pairs(lo);
      w[2 * blk + 1] = encode8_pairs(hi);
    }
    *reinterpret_cast<uint4*>(a.codes + ((long long)bh * D + c) * (a.N / 2) + ch * 32 + hb * 16) =
        make_uint4(w[0], w[1], w[2], w[3]);
    uint8_t* atom = a.sf + (((long long)bh * (a.N / 64) + ch) * NAV + c / 128) * 512;
    *reinterpret_cast<uint16_t*>(atom + sf_atom_offset(c % 128, 2 * hb)) = (uint16_t)sc2;
  }
  if constexpr (D < 128) {
    constexpr int PAD = 128 - D;
    for (int it = threadIdx.x; it < (TOK / 32) * PAD; it += NT) {
      const int half = t0 / 32 + it / PAD, r = D + it % PAD;
      uint8_t* atom = a.sf + ((long long)bh * (a.N / 64) + (half >> 1)) * NAV * 512;
      *reinterpret_cast<uint16_t*>(atom + sf_atom_offset(r, 2 * (half & 1))) = 0;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(128) k_quant_vt(QuantVtArgs a, int* status) {
  __shared__ __align__(16) __nv_bfloat16 tile[32 * (D + 8)];
  __shared__ float rtab[256];
  fill_recip_table(rtab, threadIdx.x, 128);
  bool bad = false;
  for (int u = blockIdx.x; u < a.units; u += gridDim.x) quant_vt_unit<D, 32, 128>(a, u, tile, rtab, bad);
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, ST_NONFINITE);
}

// Q, K and V in one launch: grid-stride over Q and K row units, then 64-token V units.
template <int D>
__global__ void __launch_bounds__(256) k_quant_qkv(QuantRowsArgs qa, QuantRowsArgs ka, QuantVtArgs va, int* status) {
  __shared__ __align__(16) __nv_bfloat16 tile[64 * (D + 8)];
  __shared__ float rtab[256];
  fill_recip_table(rtab, threadIdx.x, 256);
  __syncthreads();
  bool bad = false;
  const int nrows = qa.units + ka.units;
  for (int u = blockIdx.x; u < nrows + va.units; u += gridDim.x) {
    if (u < qa.units) quant_rows_unit<D>(qa, u, rtab, bad);
    else if (u < nrows) quant_rows_unit<D>(ka, u - qa.units, rtab, bad);
    else quant_vt_unit<D, 64, 256>(va, u - nrows, tile, rtab, bad);
  }
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, ST_NONFINITE);
}

struct AmaxArgs {
  const __nv_bfloat16* x;     // [B, H, N, D] with strides
  long long sb, sh, sn;
  int H, Hkv, N, D;
  float* amax;                // [Hkv, D], non-negative floats updated with integer atomicMax
};

// Per-(kv head, channel) absolute maximum over batch, the group's heads and tokens.
// grid.x = B*H, grid.y = token chunks; each thread owns channels c = threadIdx.x + k*blockDim.
__global__ void k_channel_amax(AmaxArgs a, int rows_per_cta) {
  const int bh = blockIdx.x;
  const int b = bh / a.H, h = bh % a.H, g = h / (a.H / a.Hkv);
  const int n0 = blockIdx.y * rows_per_cta;
  const int n1 = min(a.N, n0 + rows_per_cta);
  for (int c = threadIdx.x; c < a.D; c += blockDim.x) {
    float m = 0.0f;
    for (int n = n0; n < n1; ++n) m = fmaxf(m, fabsf(__bfloat162float(a.x[b * a.sb + h * a.sh + n * a.sn + c])));
    atomicMax(reinterpret_cast<int*>(a.amax + g * a.D + c), __float_as_int(m));
  }
}

}  // namespace hifa4
