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

// ---------------------------------------------------------------- streaming quantiser
// Q, K (rows, blocks along d) and V^T (blocks along tokens) as one stream of 8 KB chunks:
// a row chunk is 4096 / D rows of one head (thread t: row t / (D/16), 16-element block
// t % (D/16), two 16-byte loads), a V chunk is 32 tokens of one kv head (D/64 16-byte loads
// per thread, staged through shared memory for the transpose).  Chunk c goes to CTA
// c % gridDim.x, Q chunks first, then K, then V, so every CTA gets the same number of
// chunks to within one.  Each thread keeps the loads of its next two chunks in flight
// while it quantises the current one (registers, three buffers by static index).
template <int D>
struct StreamCfg {
  static constexpr int NT = 256;
  static constexpr int RC = 4096 / D;                 // rows per row chunk
  static constexpr int LV = D / 64;                   // 16-byte loads per thread of a V chunk
  static constexpr int NL = LV > 2 ? LV : 2;          // loads per thread of any chunk
  static constexpr int LD = D + 8;                    // padded V staging row (bf16)
};

template <int D>
struct StreamChunk {
  int kind;                                           // 0 Q, 1 K, 2 V, -1 none
  int idx;                                            // chunk index within its tensor
};

template <int D>
__device__ __forceinline__ StreamChunk<D> stream_chunk(int c, const QuantRowsArgs& qa, const QuantRowsArgs& ka,
                                                       const QuantVtArgs& va) {
  if (c < qa.units) return {0, c};
  c -= qa.units;
  if (c < ka.units) return {1, c};
  c -= ka.units;
  if (c < va.units) return {2, c};
  return {-1, 0};
}

template <int D>
__device__ __forceinline__ void stream_load(const StreamChunk<D>& ch, const QuantRowsArgs& qa, const QuantRowsArgs& ka,
                                            const QuantVtArgs& va, uint4 (&r)[StreamCfg<D>::NL]) {
  using C = StreamCfg<D>;
  if (ch.kind == 0 || ch.kind == 1) {
    const QuantRowsArgs& a = ch.kind == 0 ? qa : ka;
    const int per_head = a.N / C::RC;
    const int bh = ch.idx / per_head, row = (ch.idx % per_head) * C::RC + threadIdx.x / (D / 16);
    const int b = bh / a.H, h = bh % a.H;
    const uint4* src = reinterpret_cast<const uint4*>(a.x + b * a.sb + h * a.sh + (long long)row * a.sn +
                                                      (threadIdx.x % (D / 16)) * 16);
    r[0] = src[0];
    r[1] = src[1];
  } else if (ch.kind == 2) {
    const int per_head = va.N / 32;
    const int bh = ch.idx / per_head, t0 = (ch.idx % per_head) * 32;
    const int b = bh / va.H, h = bh % va.H;
    const __nv_bfloat16* src = va.v + b * va.sb + h * va.sh + (long long)t0 * va.sn;
#pragma unroll
    for (int k = 0; k < C::LV; ++k) {
      const int it = threadIdx.x + k * C::NT;
      r[k] = *reinterpret_cast<const uint4*>(src + (it / (D / 8)) * va.sn + (it % (D / 8)) * 8);
    }
  }
}

template <int D>
__device__ __forceinline__ void stream_rows(const QuantRowsArgs& a, int idx, const uint4 (&r)[StreamCfg<D>::NL],
                                            const float* rtab, float& nan_acc) {
  using C = StreamCfg<D>;
  const int per_head = a.N / C::RC;
  const int bh = idx / per_head, row = (idx % per_head) * C::RC + threadIdx.x / (D / 16);
  const int g = (bh % a.H) / (a.H / a.Hkv);
  const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&r[0]);
  float2 v[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] = __bfloat1622float2(p2[e]);
  quant_block16<D>(a, bh, g, row, threadIdx.x % (D / 16), v, rtab, nan_acc);
}

// V chunk: 32 tokens x D channels staged in `tile`; item c (channel) quantises the chunk's
// two 16-token blocks of channel c: 16 code bytes and 2 bytes of the channel's scale word.
template <int D>
__device__ __forceinline__ void stream_vt(const QuantVtArgs& a, int idx, const uint4 (&r)[StreamCfg<D>::NL],
                                          __nv_bfloat16* tile, const float* rtab, float& nan_acc) {
  using C = StreamCfg<D>;
  constexpr int NAV = (D + 127) / 128;
  const int per_head = a.N / 32;
  const int bh = idx / per_head, half = idx % per_head, ch = half >> 1, hb = half & 1;
  __syncthreads();                                    // the previous V chunk's readers are done
#pragma unroll
  for (int k = 0; k < C::LV; ++k) {
    const int it = threadIdx.x + k * C::NT;
    *reinterpret_cast<uint4*>(&tile[(it / (D / 8)) * C::LD + (it % (D / 8)) * 8]) = r[k];
  }
  __syncthreads();
  if (threadIdx.x < D) {
    const int c = threadIdx.x;
    uint32_t w[4];
    uint32_t sc2 = 0;
#pragma unroll
    for (int blk = 0; blk < 2; ++blk) {
      float2 x[8];
      float amax = 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        x[e] = make_float2(__bfloat162float(tile[(blk * 16 + 2 * e) * C::LD + c]),
                           __bfloat162float(tile[(blk * 16 + 2 * e + 1) * C::LD + c]));
        amax = max3_abs_nan(amax, x[e].x, x[e].y);
      }
      nan_acc = max3_abs_nan(nan_acc, amax, amax);
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
  } else if (D < 128 && threadIdx.x < 128) {
    // rows D..127 of the 128-channel atom are zero (D = 64)
    uint8_t* atom = a.sf + ((long long)bh * (a.N / 64) + ch) * NAV * 512;
    *reinterpret_cast<uint16_t*>(atom + sf_atom_offset(threadIdx.x, 2 * hb)) = 0;
  }
}

template <int D>
__device__ __forceinline__ void stream_compute(const StreamChunk<D>& ch, const QuantRowsArgs& qa,
                                               const QuantRowsArgs& ka, const QuantVtArgs& va,
                                               const uint4 (&r)[StreamCfg<D>::NL], __nv_bfloat16* tile,
                                               const float* rtab, float& nan_acc) {
  if (ch.kind == 0) stream_rows<D>(qa, ch.idx, r, rtab, nan_acc);
  else if (ch.kind == 1) stream_rows<D>(ka, ch.idx, r, rtab, nan_acc);
  else if (ch.kind == 2) stream_vt<D>(va, ch.idx, r, tile, rtab, nan_acc);
}

// Q and K row chunks (qa.units, ka.units: rows / (4096 / D)) and V chunks (va.units:
// tokens / 32), any of the three counts may be 0.
template <int D>
__global__ void __launch_bounds__(256, D == 256 ? 2 : 4) k_quant_stream(QuantRowsArgs qa, QuantRowsArgs ka, QuantVtArgs va,
                                                         int* status) {
  using C = StreamCfg<D>;
  __shared__ __align__(16) __nv_bfloat16 tile[32 * C::LD];
  __shared__ float rtab[256];
  fill_recip_table(rtab, threadIdx.x, 256);
  __syncthreads();
  const int total = qa.units + ka.units + va.units;
  const int G = gridDim.x;
  float nan_acc = 0.0f;
  uint4 b0[C::NL], b1[C::NL], b2[C::NL];
  int c = blockIdx.x;
  StreamChunk<D> k0 = stream_chunk<D>(c, qa, ka, va), k1 = stream_chunk<D>(c + G, qa, ka, va), k2;
  stream_load<D>(k0, qa, ka, va, b0);
  stream_load<D>(k1, qa, ka, va, b1);
  // the chunk kind is uniform over the CTA, so the __syncthreads of V chunks are reached by all
  for (; c < total; c += 3 * G) {
    k2 = stream_chunk<D>(c + 2 * G, qa, ka, va);
    stream_load<D>(k2, qa, ka, va, b2);
    stream_compute<D>(k0, qa, ka, va, b0, tile, rtab, nan_acc);
    if (c + G >= total) break;
    k0 = stream_chunk<D>(c + 3 * G, qa, ka, va);
    stream_load<D>(k0, qa, ka, va, b0);
    stream_compute<D>(k1, qa, ka, va, b1, tile, rtab, nan_acc);
    if (c + 2 * G >= total) break;
    k1 = stream_chunk<D>(c + 4 * G, qa, ka, va);
    stream_load<D>(k1, qa, ka, va, b1);
    stream_compute<D>(k2, qa, ka, va, b2, tile, rtab, nan_acc);
  }
  if (__any_sync(0xffffffffu, !isfinite(nan_acc)) && (threadIdx.x & 31) == 0) atomicOr(status, ST_NONFINITE);
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
