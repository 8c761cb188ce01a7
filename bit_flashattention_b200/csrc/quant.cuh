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

struct QuantVtArgs {
  const __nv_bfloat16* v;     // [B, Hkv, N, D] with strides, d contiguous
  long long sb, sh, sn;
  int H, N;
  uint8_t* codes;             // [B, Hkv, D, N/2]
  uint8_t* sf;                // [B, Hkv, N/64, ceil(D/128), 512]
  int units;                  // B * Hkv * N / TOK for the kernel's TOK
};

// ---------------------------------------------------------------- streaming quantiser
// Q, K (rows, blocks along d) and V^T (blocks along tokens) as one stream of 16 KB chunks of
// bf16 input: a row chunk is 8192 / D rows of one head, a V chunk 8192 / D tokens of one kv
// head.  Chunk c goes to CTA c % gridDim.x, Q chunks first, then K, then V, so every CTA
// gets the same number of chunks to within one.  Warp 0 copies each chunk into a ring of
// NS shared-memory stages with cp.async.bulk (one copy when the chunk's rows are contiguous
// in memory, one per row otherwise), so NS - 1 chunks are in flight while all 256 threads
// quantise the current one from shared memory:
//   row chunk: thread t takes 16-element block t % (D/16) of rows t / (D/16) and
//              t / (D/16) + RC/2;
//   V chunk:   thread t takes channel t % D over the 32 tokens 32 (t / D) .. 32 (t / D) + 31
//              (two 16-token blocks of V^T).
// The ring runs on mbarriers only: `full` (the copy's bytes) and `empty` (one arrival per
// warp when it is done with the stage); warp 0 refills a stage after its `empty` completes.
// Every wait is bounded; after a timeout the warps leave and warp 0 waits (bounded) for
// its copies still in flight before the CTA exits.  Chunk indices are split with
// multiply-shift divisions by host-computed constants.
struct FastDiv {
  uint32_t d, m, s;   // n / d = (umulhi(n, m) + n) >> s for 0 <= n < 2^31
};

__host__ __device__ inline FastDiv make_fastdiv(uint32_t d) {
  uint32_t s = 0;
  while (s < 31 && (1u << s) < d) ++s;
  const uint64_t m = ((uint64_t(1) << 32) * ((uint64_t(1) << s) - d)) / d + 1;
  return FastDiv{d, (uint32_t)m, s};
}

__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) { return (__umulhi(n, f.m) + n) >> f.s; }

struct StreamDivs {
  FastDiv q_chunks, q_heads, q_group;   // chunks per head, heads (H), group size (H / Hkv)
  FastDiv k_chunks, k_heads, k_group;
  FastDiv v_chunks, v_heads;
};

template <int D>
struct StreamCfg {
  static constexpr int NT = 256;
  static constexpr int RC = 8192 / D;                 // rows per row chunk
  static constexpr int TV = 8192 / D;                 // tokens per V chunk
  static constexpr uint32_t STAGE = 16384;
  static constexpr int NS = 3;                        // stages
  static constexpr uint32_t OFF_RTAB = NS * STAGE;
  static constexpr uint32_t OFF_BAR = OFF_RTAB + 1024;
  static constexpr int SC_MAX = 2048;                             // Smooth-QK floats per tensor kept in smem
  static constexpr uint32_t OFF_SC = OFF_BAR + 16 * NS + 16;      // [2][SC_MAX] fp32: s, then s_inv
  static constexpr uint32_t SMEM = OFF_SC + 2 * SC_MAX * 4 + 128; // + slack for 128-B alignment
};

struct ChunkPos {
  int kind;                                           // 0 Q, 1 K, 2 V
  int bh;                                             // (batch, head) slab
  int b, h;
  int r0;                                             // first row / token of the chunk
};

template <int D>
__device__ __forceinline__ ChunkPos chunk_pos(int c, const QuantRowsArgs& qa, const QuantRowsArgs& ka,
                                              const StreamDivs& dv) {
  using C = StreamCfg<D>;
  ChunkPos p;
  const FastDiv *fc, *fh;
  int idx, rows;
  if (c < qa.units) {
    p.kind = 0, idx = c, fc = &dv.q_chunks, fh = &dv.q_heads, rows = C::RC;
  } else if (c < qa.units + ka.units) {
    p.kind = 1, idx = c - qa.units, fc = &dv.k_chunks, fh = &dv.k_heads, rows = C::RC;
  } else {
    p.kind = 2, idx = c - qa.units - ka.units, fc = &dv.v_chunks, fh = &dv.v_heads, rows = C::TV;
  }
  p.bh = (int)fdiv((uint32_t)idx, *fc);
  p.r0 = (idx - p.bh * (int)fc->d) * rows;
  p.b = (int)fdiv((uint32_t)p.bh, *fh);
  p.h = p.bh - p.b * (int)fh->d;
  return p;
}

// Warp 0: copy the chunk at `p` into `stage` and arm `bar` with its byte count.
template <int D>
__device__ __forceinline__ void stream_issue(const ChunkPos& p, const QuantRowsArgs& qa, const QuantRowsArgs& ka,
                                             const QuantVtArgs& va, uint8_t* stage, uint64_t* bar) {
  using C = StreamCfg<D>;
  const int lane = threadIdx.x & 31;
  const __nv_bfloat16* src;
  long long sn;
  if (p.kind == 2) {
    src = va.v + p.b * va.sb + p.h * va.sh + (long long)p.r0 * va.sn;
    sn = va.sn;
  } else {
    const QuantRowsArgs& a = p.kind == 0 ? qa : ka;
    src = a.x + p.b * a.sb + p.h * a.sh + (long long)p.r0 * a.sn;
    sn = a.sn;
  }
  constexpr int NR = C::RC;                           // = C::TV: rows of 2 D bytes per chunk
  constexpr uint32_t ROWB = 2 * D;
  if (lane == 0) mbar_arrive_expect_tx(bar, NR * ROWB);
  __syncwarp();
  if (sn == D) {
    if (lane == 0) bulk_load(stage, src, NR * ROWB, bar);
  } else {
    for (int r = lane; r < NR; r += 32) bulk_load(stage + r * ROWB, src + r * sn, ROWB, bar);
  }
}

// Smooth-QK (when sc4 is used), amax, scale and codes of one 16-element block of row `row`
// (block blk of the row), stored as 8 code bytes and the scale byte of the row's atom record.
// The block amax is a 3-input-max tree (depth 3) instead of a chain.
template <int D>
__device__ __forceinline__ void stream_quant_store(const QuantRowsArgs& a, int bh, int row, int blk, float2 (&v)[8],
                                                   const float4 (&sc4)[4], const float* rtab, float& nan_acc) {
  if (a.scale) {
#pragma unroll
    for (int qd = 0; qd < 4; ++qd) {
      v[2 * qd] = __fmul2_rn(v[2 * qd], make_float2(sc4[qd].x, sc4[qd].y));
      v[2 * qd + 1] = __fmul2_rn(v[2 * qd + 1], make_float2(sc4[qd].z, sc4[qd].w));
    }
  }
  const float m0 = max3_abs_nan(v[0].x, v[0].y, v[1].x), m1 = max3_abs_nan(v[1].y, v[2].x, v[2].y);
  const float m2 = max3_abs_nan(v[3].x, v[3].y, v[4].x), m3 = max3_abs_nan(v[4].y, v[5].x, v[5].y);
  const float m4 = max3_abs_nan(v[6].x, v[6].y, v[7].x);
  const float amax = max3_abs_nan(max3_abs_nan(m0, m1, m2), max3_abs_nan(m3, m4, v[7].y), 0.0f);
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

__device__ __forceinline__ void unpack16(const uint8_t* src, float2 (&v)[8]) {
  const uint4* p = reinterpret_cast<const uint4*>(src);
  uint4 r[2] = {p[0], p[1]};
  const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(r);
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] = __bfloat1622float2(p2[e]);
}

// Per-thread loads of a row chunk that do not depend on its data, issued before the wait
// for the chunk's bytes (every warp splits the chunk index itself): the Smooth-QK scales
// of the thread's channels and, with ROPE, the angle-table columns of its channel pairs.
template <int D, bool ROPE>
struct RowPrefetch {
  float4 sc4[ROPE ? 8 : 4];                           // [0..3] block 1 (ROPE: first half), [4..7] ROPE second half
  float4 cs[ROPE ? 8 : 1];                            // ROPE: cos [0..3], sin [4..7]
};

template <int D, bool ROPE>
__device__ __forceinline__ void stream_prefetch(const QuantRowsArgs& a, const float* scale, const ChunkPos& p, int g,
                                                RowPrefetch<D, ROPE>& f) {
  // `scale`: the tensor's Smooth-QK scales (a shared-memory copy when they fit), or null
  if constexpr (ROPE) {
    constexpr int HB = D / 32;
    const int rl = threadIdx.x / HB, pr = threadIdx.x % HB, row = p.r0 + rl;
    if (scale) {
      const float4* sp = reinterpret_cast<const float4*>(scale + g * D + pr * 16);
#pragma unroll
      for (int qd = 0; qd < 4; ++qd) {
        f.sc4[qd] = sp[qd];
        f.sc4[4 + qd] = sp[D / 8 + qd];                // channels + D/2
      }
    }
    const float4* cp = reinterpret_cast<const float4*>(a.rope_cos + (long long)row * (D / 2) + pr * 16);
    const float4* sp = reinterpret_cast<const float4*>(a.rope_sin + (long long)row * (D / 2) + pr * 16);
#pragma unroll
    for (int qd = 0; qd < 4; ++qd) {
      f.cs[qd] = __ldg(cp + qd);
      f.cs[4 + qd] = __ldg(sp + qd);
    }
  } else {
    if (scale) {
      const float4* sp = reinterpret_cast<const float4*>(scale + g * D + (threadIdx.x % (D / 16)) * 16);
#pragma unroll
      for (int qd = 0; qd < 4; ++qd) f.sc4[qd] = sp[qd];
    }
  }
}

// Row chunk.  Without ROPE thread t takes block t % (D/16) of rows t / (D/16) and
// t / (D/16) + RC/2.  With ROPE thread t takes the rotate-half block pair (t % (D/32),
// t % (D/32) + D/32) of row t / (D/32): it rotates both blocks from one read of the pair and
// of its 16 angle-table columns, every product and sum rounded once (scalar intrinsics,
// never contracted: an exact cancellation must give +0),
//   x'_c = RN(RN(x_c cos) - RN(x_{c+D/2} sin)),  x'_{c+D/2} = RN(RN(x_{c+D/2} cos) + RN(x_c sin)).
template <int D, bool ROPE>
__device__ __forceinline__ void stream_rows(const QuantRowsArgs& a, const ChunkPos& p, const RowPrefetch<D, ROPE>& f,
                                            const uint8_t* stage, const float* rtab, float& nan_acc) {
  using C = StreamCfg<D>;
  if constexpr (ROPE) {
    constexpr int HB = D / 32;
    const int rl = threadIdx.x / HB, pr = threadIdx.x % HB;
    float2 x1[8], x2[8];
    unpack16(stage + rl * (2 * D) + pr * 32, x1);
    unpack16(stage + rl * (2 * D) + (pr + HB) * 32, x2);
    float2 y1[8], y2[8];
#pragma unroll
    for (int qd = 0; qd < 4; ++qd) {
      const float cc[4] = {f.cs[qd].x, f.cs[qd].y, f.cs[qd].z, f.cs[qd].w};
      const float ss[4] = {f.cs[4 + qd].x, f.cs[4 + qd].y, f.cs[4 + qd].z, f.cs[4 + qd].w};
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int e = 2 * qd + hh;
        const float c0 = cc[2 * hh], c1 = cc[2 * hh + 1], s0 = ss[2 * hh], s1 = ss[2 * hh + 1];
        y1[e] = make_float2(__fsub_rn(__fmul_rn(x1[e].x, c0), __fmul_rn(x2[e].x, s0)),
                            __fsub_rn(__fmul_rn(x1[e].y, c1), __fmul_rn(x2[e].y, s1)));
        y2[e] = make_float2(__fadd_rn(__fmul_rn(x2[e].x, c0), __fmul_rn(x1[e].x, s0)),
                            __fadd_rn(__fmul_rn(x2[e].y, c1), __fmul_rn(x1[e].y, s1)));
      }
    }
    const float4 s_lo[4] = {f.sc4[0], f.sc4[1], f.sc4[2], f.sc4[3]};
    const float4 s_hi[4] = {f.sc4[4], f.sc4[5], f.sc4[6], f.sc4[7]};
    stream_quant_store<D>(a, p.bh, p.r0 + rl, pr, y1, s_lo, rtab, nan_acc);
    stream_quant_store<D>(a, p.bh, p.r0 + rl, pr + HB, y2, s_hi, rtab, nan_acc);
  } else {
    const int rl = threadIdx.x / (D / 16), blk = threadIdx.x % (D / 16);
    float2 v0[8], v1[8];
    unpack16(stage + rl * (2 * D) + blk * 32, v0);
    unpack16(stage + (rl + C::RC / 2) * (2 * D) + blk * 32, v1);
    stream_quant_store<D>(a, p.bh, p.r0 + rl, blk, v0, f.sc4, rtab, nan_acc);
    stream_quant_store<D>(a, p.bh, p.r0 + rl + C::RC / 2, blk, v1, f.sc4, rtab, nan_acc);
  }
}

// V chunk: TV tokens x D channels in `stage` ([token][channel] bf16); thread t quantises
// the two 16-token blocks of channel t % D in tokens 32 (t / D) .. + 31: 16 code bytes and
// 2 bytes of the channel's scale word.  For D = 64 every thread also zeroes one 2-byte
// entry of rows 64..127 of the chunk's 128-channel atoms.
template <int D>
__device__ __forceinline__ void stream_vt(const QuantVtArgs& a, const ChunkPos& p, const uint8_t* stage,
                                          const float* rtab, float& nan_acc) {
  using C = StreamCfg<D>;
  constexpr int NAV = (D + 127) / 128;
  const __nv_bfloat16* tile = reinterpret_cast<const __nv_bfloat16*>(stage);
  const int c = threadIdx.x % D, hh = threadIdx.x / D;
  const int half = p.r0 / 32 + hh, ch = half >> 1, hb = half & 1;
  uint32_t w[4];
  uint32_t sc2 = 0;
#pragma unroll
  for (int blk = 0; blk < 2; ++blk) {
    float2 x[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int t = hh * 32 + blk * 16 + 2 * e;
      x[e] = make_float2(__bfloat162float(tile[t * D + c]), __bfloat162float(tile[(t + 1) * D + c]));
    }
    const float m0 = max3_abs_nan(x[0].x, x[0].y, x[1].x), m1 = max3_abs_nan(x[1].y, x[2].x, x[2].y);
    const float m2 = max3_abs_nan(x[3].x, x[3].y, x[4].x), m3 = max3_abs_nan(x[4].y, x[5].x, x[5].y);
    const float m4 = max3_abs_nan(x[6].x, x[6].y, x[7].x);
    const float amax = max3_abs_nan(max3_abs_nan(m0, m1, m2), max3_abs_nan(m3, m4, x[7].y), 0.0f);
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
  *reinterpret_cast<uint4*>(a.codes + ((long long)p.bh * D + c) * (a.N / 2) + ch * 32 + hb * 16) =
      make_uint4(w[0], w[1], w[2], w[3]);
  uint8_t* atom = a.sf + (((long long)p.bh * (a.N / 64) + ch) * NAV + c / 128) * 512;
  *reinterpret_cast<uint16_t*>(atom + sf_atom_offset(c % 128, 2 * hb)) = (uint16_t)sc2;
  if constexpr (D < 128) {
    // rows D..127 of the 128-channel atoms of the chunk's C::TV / 32 halves are zero
    constexpr int PAD = 128 - D;
    static_assert((C::TV / 32) * PAD == C::NT, "one padding entry per thread");
    const int hp = p.r0 / 32 + threadIdx.x / PAD, r = D + threadIdx.x % PAD;
    uint8_t* pa = a.sf + ((long long)p.bh * (a.N / 64) + (hp >> 1)) * NAV * 512;
    *reinterpret_cast<uint16_t*>(pa + sf_atom_offset(r, 2 * (hp & 1))) = 0;
  }
}

// Q and K row chunks (qa.units, ka.units: rows / (8192 / D)) and V chunks (va.units:
// tokens / (8192 / D)); any of the three counts may be 0.  ROPE: Q and K are pre-RoPE and
// rotated with the tables of qa / ka before Smooth-QK (no V chunks).
template <int D, bool ROPE = false>
__global__ void __launch_bounds__(256, ROPE ? 2 : 3) k_quant_stream(QuantRowsArgs qa, QuantRowsArgs ka, QuantVtArgs va,
                                                         StreamDivs dv, int* status, unsigned long long wait_ns) {
  using C = StreamCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
  float* rtab = reinterpret_cast<float*>(smem + C::OFF_RTAB);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + C::NS;
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::OFF_BAR + 16 * C::NS);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  fill_recip_table(rtab, threadIdx.x, 256);
  // the Smooth-QK scales of Q and K in shared memory when they fit (Hkv * D <= SC_MAX)
  float* sc_q = reinterpret_cast<float*>(smem + C::OFF_SC);
  float* sc_k = sc_q + C::SC_MAX;
  const float* scale_q = qa.scale;
  const float* scale_k = ka.scale;
  if (qa.scale && qa.Hkv * D <= C::SC_MAX) {
    for (int i = threadIdx.x; i < qa.Hkv * D; i += C::NT) sc_q[i] = qa.scale[i];
    scale_q = sc_q;
  }
  if (ka.scale && ka.Hkv * D <= C::SC_MAX) {
    for (int i = threadIdx.x; i < ka.Hkv * D; i += C::NT) sc_k[i] = ka.scale[i];
    scale_k = sc_k;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], C::NT / 32);
    }
    *abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const int total = qa.units + ka.units + va.units, G = gridDim.x, b0 = blockIdx.x;
  const int mine = b0 < total ? (total - 1 - b0) / G + 1 : 0;   // chunks of this CTA
  int issued = 0;
  auto issue = [&](int j, int st) {
    stream_issue<D>(chunk_pos<D>(b0 + j * G, qa, ka, dv), qa, ka, va, smem + st * C::STAGE, &full[st]);
  };
  if (warp == 0) {
    for (; issued < C::NS && issued < mine; ++issued) issue(issued, issued);
  }
  float nan_acc = 0.0f;
  bool ok = true;
  for (int i = 0; i < mine; ++i) {
    const int st = i % C::NS;
    const uint32_t par = (i / C::NS) & 1;
    // the chunk's position and the loads that do not depend on its bytes come before
    // the wait for them
    const ChunkPos p = chunk_pos<D>(b0 + i * G, qa, ka, dv);
    const QuantRowsArgs& a = p.kind == 0 ? qa : ka;
    const int g = p.kind == 2 ? 0 : (int)fdiv((uint32_t)p.h, p.kind == 0 ? dv.q_group : dv.k_group);
    RowPrefetch<D, ROPE> f;
    if (p.kind != 2) stream_prefetch<D, ROPE>(a, p.kind == 0 ? scale_q : scale_k, p, g, f);
    ok = __all_sync(0xffffffffu, mbar_wait(&full[st], par, abort, status, wait_ns));
    if (!ok) break;
    const uint8_t* stage = smem + st * C::STAGE;
    if (p.kind == 2) {
      stream_vt<D>(va, p, stage, rtab, nan_acc);
    } else {
      stream_rows<D, ROPE>(a, p, f, stage, rtab, nan_acc);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
    if (warp == 0 && issued < mine) {
      // every warp is done with this stage: refill it with the chunk NS ahead
      ok = __all_sync(0xffffffffu, mbar_wait(&empty[st], par, abort, status, wait_ns));
      if (!ok) break;
      issue(issued, st);
      ++issued;
    }
  }
  if (!ok && warp == 0 && lane == 0) {
    // a wait ran out: the copies issued so far land before the CTA exits
    int never = 0;
    for (int j = issued - C::NS < 0 ? 0 : issued - C::NS; j < issued; ++j)
      mbar_wait(&full[j % C::NS], (j / C::NS) & 1, &never, status, wait_ns);
  }
  if (__any_sync(0xffffffffu, !isfinite(nan_acc)) && lane == 0) atomicOr(status, ST_NONFINITE);
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
