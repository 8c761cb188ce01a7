// Quantiser kernels (HBM-bound): Smooth-QK application + 4-bit block quantisation of Q
// and K along the head dimension, the transposing quantisation of V (blocks of 16
// tokens per channel), and the per-channel amax reduction of the Smooth-QK calibration.
//
// Smooth-QK ("HiFA4: Training-Free 4-bit FlashAttention on Ascend HIF4 NPUs for LLM
// Inference", abstract): a calibration-static per-channel equivalent rescaling Q*s, K/s
// after RoPE, with no per-tile online reduction at inference.  Here q' = RN(q * s[g,c])
// and k' = RN(k * s_inv[g,c]) with g the kv head of the query head.
#pragma once
#include "method.cuh"

namespace hifa4 {

struct QuantRowsArgs {
  const __nv_bfloat16* x;     // [B, H, N, D] with strides (sb, sh, sn) in elements, d contiguous
  long long sb, sh, sn;
  int H, Hkv, N;
  const float* scale;         // [Hkv, D] or nullptr
  uint8_t* codes;             // [B, H, N, D/2]
  uint8_t* sf;                // [B, H, N/128, D/64, 512]
  int tiles;                  // B * H * N / 128
};

// One CTA of 256 threads quantises a 128-row tile; each thread takes 8 consecutive
// elements (16 bytes) at a time: 2 threads per 16-block, 8 threads per 64-wide chunk.
template <int D>
__global__ void __launch_bounds__(256) k_quant_rows(QuantRowsArgs qa, QuantRowsArgs ka, int* status) {
  const bool isq = blockIdx.x < (unsigned)qa.tiles;
  const QuantRowsArgs& a = isq ? qa : ka;
  const int tile = isq ? blockIdx.x : blockIdx.x - qa.tiles;
  const int ntile_n = a.N / 128;
  const int bh = tile / ntile_n, rt = tile % ntile_n;
  const int b = bh / a.H, h = bh % a.H, g = h / (a.H / a.Hkv);
  const int lane = threadIdx.x & 31;
  constexpr int PARTS = D / 8;
  constexpr int ITEMS = 128 * PARTS;
  bool bad = false;
#pragma unroll 2
  for (int it = threadIdx.x; it < ITEMS; it += 256) {
    const int row = it / PARTS, part = it % PARTS;
    const long long n = (long long)rt * 128 + row;
    const uint4 raw = *reinterpret_cast<const uint4*>(a.x + b * a.sb + h * a.sh + n * a.sn + part * 8);
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
    float v[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(p2[k]);
      v[2 * k] = f.x;
      v[2 * k + 1] = f.y;
    }
    if (a.scale) {
      const float4* sp = reinterpret_cast<const float4*>(a.scale + g * D + part * 8);
      const float4 s0 = __ldg(sp), s1 = __ldg(sp + 1);
      v[0] = __fmul_rn(v[0], s0.x); v[1] = __fmul_rn(v[1], s0.y);
      v[2] = __fmul_rn(v[2], s0.z); v[3] = __fmul_rn(v[3], s0.w);
      v[4] = __fmul_rn(v[4], s1.x); v[5] = __fmul_rn(v[5], s1.y);
      v[6] = __fmul_rn(v[6], s1.z); v[7] = __fmul_rn(v[7], s1.w);
    }
    float amax = 0.0f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      bad |= !isfinite(v[k]);
      amax = fmaxf(amax, fabsf(v[k]));
    }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    float R;
    const uint32_t sc = block_scale(amax, R);
    const uint32_t w = encode8(v, R);
    *reinterpret_cast<uint32_t*>(a.codes + ((long long)bh * a.N + n) * (D / 2) + part * 4) = w;
    // gather the 4 scale bytes of this 64-chunk (blocks live in lanes base+0, +2, +4, +6)
    const int base = lane & ~7;
    uint32_t word = 0;
#pragma unroll
    for (int s = 0; s < 4; ++s) word |= __shfl_sync(0xffffffffu, sc, base + 2 * s) << (8 * s);
    if ((lane & 7) == 0) {
      const int kc = part / 8;
      uint8_t* atom = a.sf + (((long long)bh * ntile_n + rt) * (D / 64) + kc) * 512;
      *reinterpret_cast<uint32_t*>(atom + sf_atom_offset(row, 0)) = word;
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(status, ST_NONFINITE);
}

struct QuantVtArgs {
  const __nv_bfloat16* v;     // [B, Hkv, N, D] with strides, d contiguous
  long long sb, sh, sn;
  int H, N;
  uint8_t* codes;             // [B, Hkv, D, N/2]
  uint8_t* sf;                // [B, Hkv, N/64, ceil(D/128), 512]
};

// One CTA per (b, kv head, 64-token chunk): the tile is staged in shared memory with
// coalesced loads, then thread c quantises channel c's four 16-token blocks and writes
// its 32 code bytes and one scale word.  Threads c >= D (only D = 64) zero the unused
// rows of the 128-row scale atom.
template <int D>
__global__ void __launch_bounds__(D < 128 ? 128 : D) k_quant_vt(QuantVtArgs a, int* status) {
  constexpr int NT = D < 128 ? 128 : D;
  constexpr int NAV = (D + 127) / 128;
  constexpr int LD = D + 8;   // padded row (bf16 elements) of the staging tile
  __shared__ __align__(16) __nv_bfloat16 tile[64 * LD];
  const int nch = a.N / 64;
  const int bh = blockIdx.x / nch, ch = blockIdx.x % nch;
  const int b = bh / a.H, h = bh % a.H;
  const __nv_bfloat16* src = a.v + b * a.sb + h * a.sh + (long long)ch * 64 * a.sn;
  bool bad = false;
  for (int it = threadIdx.x; it < 64 * (D / 8); it += NT) {
    const int t = it / (D / 8), part = it % (D / 8);
    const uint4 raw = *reinterpret_cast<const uint4*>(src + t * a.sn + part * 8);
    *reinterpret_cast<uint4*>(&tile[t * LD + part * 8]) = raw;
  }
  __syncthreads();
  const int c = threadIdx.x;
  if (c < D) {
    uint32_t w[8];
    uint32_t word = 0;
#pragma unroll
    for (int blk = 0; blk < 4; ++blk) {
      float x[16];
      float amax = 0.0f;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        x[e] = __bfloat162float(tile[(blk * 16 + e) * LD + c]);
        bad |= !isfinite(x[e]);
        amax = fmaxf(amax, fabsf(x[e]));
      }
      float R;
      const uint32_t sc = block_scale(amax, R);
      float lo[8], hi[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) { lo[e] = x[e]; hi[e] = x[8 + e]; }
      w[2 * blk] = encode8(lo, R);
      w[2 * blk + 1] = encode8(hi, R);
      word |= sc << (8 * blk);
    }
    uint4* dst = reinterpret_cast<uint4*>(a.codes + ((long long)bh * D + c) * (a.N / 2) + ch * 32);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    uint8_t* atom = a.sf + (((long long)bh * nch + ch) * NAV + c / 128) * 512;
    *reinterpret_cast<uint32_t*>(atom + sf_atom_offset(c % 128, 0)) = word;
  } else if (c < 128) {
    uint8_t* atom = a.sf + ((long long)bh * nch + ch) * NAV * 512;
    *reinterpret_cast<uint32_t*>(atom + sf_atom_offset(c, 0)) = 0u;
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
