// Host side of the C ABI declared in include/hifa4.h: argument validation, tensor-map
// construction, kernel dispatch over the supported (d, kv tile) shapes.  Built with
// HIFA4_TEST_HOOKS defined it also exports the test-only functions of
// include/hifa4_test.h (the test library; the product library has none of them).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/hifa4.h"
#ifdef HIFA4_TEST_HOOKS
#include "../../include/hifa4_test.h"
#endif
#include "attn.cuh"
#include "attn_decode.cuh"
#include "quant.cuh"

using namespace hifa4;

namespace {

unsigned long long g_wait_ns = 2000000000ull;

bool device_ok() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  static std::mutex mu;
  static std::vector<int> cache(64, -1);
  std::lock_guard<std::mutex> lk(mu);
  if (dev < 0 || dev >= 64) return false;
  if (cache[dev] < 0) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cache[dev] = (major == 10 && minor == 0) ? 1 : 0;
  }
  return cache[dev] == 1;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

CUtensorMapSwizzle swizzle_of(int rowbytes) {
  return rowbytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                        : rowbytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
}

// 2-D byte tensor map: rows of `row_bytes` (stride `row_stride`), box of
// `box_bytes` x `box_rows`, swizzled to match a K-major UMMA operand whose rows are
// `box_bytes` long.
bool make_map(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows, uint64_t row_stride,
              uint32_t box_bytes, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {row_bytes, rows};
  cuuint64_t strides[1] = {row_stride};
  cuuint32_t box[2] = {box_bytes, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_of((int)box_bytes), CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

bool strides_ok(const void* base, const int64_t s[3]) {
  if (!base || !s || !aligned16(base)) return false;
  for (int i = 0; i < 3; ++i)
    if (s[i] < 0 || (s[i] % 8) != 0) return false;
  return true;
}

bool d_ok(int d) { return d == 64 || d == 128 || d == 256; }

int num_sms();

// Grid of a grid-stride kernel: all units at once if they fit, else one full wave.
// CTAs of `kernel` that fit on one SM by its shared memory (dynamic `smem` plus static
// and the per-block reservation), registers (per SM sub-partition: warps are spread over
// four) and threads; 0 when the attributes cannot be read.
template <typename K>
int resident_by_limits(K kernel, int threads, int smem) {
  int dev = 0, smem_sm = 0, reserved = 0;
  cudaFuncAttributes fa;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess ||
      cudaFuncGetAttributes(&fa, kernel) != cudaSuccess || fa.numRegs <= 0)
    return 0;
  const int warps = (threads + 31) / 32;
  const int regs = (fa.numRegs + 7) / 8 * 8;
  const int by_smem = smem_sm / (smem + (int)fa.sharedSizeBytes + reserved);
  int by_regs = 0;   // CTAs whose warps, dealt round-robin over the 4 sub-partitions, fit 16384 registers each
  while ((((by_regs + 1) * warps + 3) / 4) * 32 * regs <= 16384) ++by_regs;
  const int by_threads = 2048 / threads;
  int m = by_smem < by_regs ? by_smem : by_regs;
  return m < by_threads ? m : by_threads;
}

template <typename K>
int resident_grid(K kernel, int threads, int units) {
  // kernels of one signature share K: cache the occupancy per kernel address
  static std::mutex mu;
  static const void* keys[16];
  static int vals[16];
  static int nkeys = 0;
  int per_sm = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < nkeys; ++i)
      if (keys[i] == reinterpret_cast<const void*>(kernel)) per_sm = vals[i];
    if (per_sm == 0) {
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0) != cudaSuccess) per_sm = 0;
      const int m = resident_by_limits(kernel, threads, 0);
      if (m > per_sm) per_sm = m;
      if (per_sm <= 0) per_sm = 1;
      if (nkeys < 16) {
        keys[nkeys] = reinterpret_cast<const void*>(kernel);
        vals[nkeys++] = per_sm;
      }
    }
  }
  const long long cap = (long long)per_sm * num_sms();
  return (int)(units < cap ? units : cap);
}

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? HIFA4_OK : HIFA4_ERR_CUDA; }

bool qt_ok(const hifa4_qtensor* t, int B, int H, int N, int d, int transposed) {
  return t && t->codes && t->scales && aligned16(t->codes) && aligned16(t->scales) && t->B == B && t->H == H &&
         t->N == N && t->d == d && t->transposed == transposed;
}

template <typename K>
bool set_smem(K kernel, uint32_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) == cudaSuccess;
}

// L(sigma) = RN_fp32(-log2 sigma) for every non-negative E4M3 scale code (the fast P_hat
// code rule), from integer logs in double: normal sigma = (8 + m) 2^(e - 10) gives (10 - e) - log2(8 + m),
// subnormal sigma = m 2^-9 gives 9 - log2(m); code 0 (sigma = 0) and the NaN code map to
// -inf.
void fill_neg_log2_scales(float* t) {
  for (int code = 0; code < 128; ++code) {
    const int e = (code >> 3) & 15, m = code & 7;
    if (code == 0 || code == 0x7F) {
      t[code] = -INFINITY;
      continue;
    }
    const double v = (e == 0) ? 9.0 - std::log2((double)m) : (double)(10 - e) - std::log2((double)(8 + m));
    t[code] = (float)v;
  }
}

// The streaming quantiser (k_quant_stream) over Q and K row chunks (4096 / d rows each)
// and V chunks (32 tokens each); the callers set each struct's `units` in those chunks,
// 0 for a tensor that is not quantised.
template <int D, bool ROPE>
int launch_quant_stream_d(const QuantRowsArgs& qa, const QuantRowsArgs& ka, const QuantVtArgs& va, int* status,
                          cudaStream_t stream) {
  // multiply-shift constants of the chunk index splits (chunks per head, heads, group size)
  auto fd = [](int v) { return make_fastdiv((uint32_t)(v > 0 ? v : 1)); };
  StreamDivs dv;
  dv.q_chunks = fd(qa.N / StreamCfg<D>::RC);
  dv.q_heads = fd(qa.H);
  dv.q_group = fd(qa.Hkv > 0 ? qa.H / qa.Hkv : 1);
  dv.k_chunks = fd(ka.N / StreamCfg<D>::RC);
  dv.k_heads = fd(ka.H);
  dv.k_group = fd(ka.Hkv > 0 ? ka.H / ka.Hkv : 1);
  dv.v_chunks = fd(va.N / StreamCfg<D>::TV);
  dv.v_heads = fd(va.H);
  constexpr uint32_t smem = StreamCfg<D>::SMEM;
  // shared-memory attribute and resident CTAs (at most 3, with RoPE 2: the kernel's register bound),
  // set up once per instance (thread-safe static initialisation)
  static const int per_sm = [] {
    if (!set_smem(k_quant_stream<D, ROPE>, smem)) return 0;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_quant_stream<D, ROPE>, 256, smem) != cudaSuccess || n <= 0)
      n = 1;
    const int cap_regs = ROPE ? 2 : 3;
    return n < cap_regs ? n : cap_regs;
  }();
  if (per_sm == 0) return HIFA4_ERR_CUDA;
  const long long units = (long long)qa.units + ka.units + va.units;
  const long long cap = (long long)per_sm * num_sms();
  k_quant_stream<D, ROPE><<<(unsigned)(units < cap ? units : cap), 256, smem, stream>>>(qa, ka, va, dv, status,
                                                                                        g_wait_ns);
  return cuda_status(cudaGetLastError());
}

int launch_quant_stream(const QuantRowsArgs& qa, const QuantRowsArgs& ka, const QuantVtArgs& va, int d, int* status,
                        cudaStream_t stream, bool rope = false) {
  if ((long long)qa.units + ka.units + va.units == 0) return HIFA4_OK;
  if (rope) {
    switch (d) {
      case 64: return launch_quant_stream_d<64, true>(qa, ka, va, status, stream);
      case 128: return launch_quant_stream_d<128, true>(qa, ka, va, status, stream);
      default: return launch_quant_stream_d<256, true>(qa, ka, va, status, stream);
    }
  }
  switch (d) {
    case 64: return launch_quant_stream_d<64, false>(qa, ka, va, status, stream);
    case 128: return launch_quant_stream_d<128, false>(qa, ka, va, status, stream);
    default: return launch_quant_stream_d<256, false>(qa, ka, va, status, stream);
  }
}

// chunks of the streaming quantiser: 16 KB of bf16 input each (8192 / d rows or tokens)
int stream_row_chunks(int B, int H, int N, int d) { return B * H * (N / (8192 / d)); }

// Decode / split-KV launch parameters (see AttnParams).
struct DecodeSpec {
  int nq, G, Nk, nsplit, tps;
  float *part_o, *part_m, *part_l;
};

template <int D, int BC, bool SUMP = false, bool DEC = false, bool FAST = false>
int launch_attn(const hifa4_qtensor* q, const hifa4_qtensor* k, const hifa4_qtensor* vt, int B, int Hq, int Hkv,
                int N, int causal, void* o, void* m_out, void* l_out, int* status, cudaStream_t stream,
                int l_from_p = 0, float* trace = nullptr, const DecodeSpec* dec = nullptr, int two_level = 0,
                int inject = 0) {
  using C = AttnCfg<D, BC>;
  const int Nk = dec ? dec->Nk : N;
  const uint64_t qrows = dec ? (uint64_t)B * Hkv * 128 : (uint64_t)B * Hq * N;
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q->codes, D / 2, qrows, D / 2, D / 2, 128) ||
      !make_map(&tk, k->codes, D / 2, (uint64_t)B * Hkv * Nk, D / 2, D / 2, BC) ||
      !make_map(&tv, vt->codes, Nk / 2, (uint64_t)B * Hkv * D, Nk / 2, BC / 2, D))
    return HIFA4_ERR_CUDA;
  // One CTA per SM when it holds all 512 TMEM columns: ask for more than half the SM's
  // shared memory so a second CTA cannot become resident and block in tcgen05.alloc.
  const uint32_t smem = (C::TMEM_COLS == 512 && C::SMEM < 120 * 1024) ? 120 * 1024 : C::SMEM;
  static bool attr = set_smem(k_attn_fwd<D, BC, SUMP, DEC, FAST>, smem);
  if (!attr) return HIFA4_ERR_CUDA;
  AttnParams p;
  std::memset(&p, 0, sizeof(p));
  p.qsf = static_cast<const uint8_t*>(q->scales);
  p.ksf = static_cast<const uint8_t*>(k->scales);
  p.vsf = static_cast<const uint8_t*>(vt->scales);
  p.o = static_cast<__nv_bfloat16*>(o);
  p.m_out = static_cast<__half*>(m_out);
  p.l_out = static_cast<__half*>(l_out);
  p.status = status;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.causal = causal ? 1 : 0;
  p.c = (float)(1.4426950408889634074 / std::sqrt((double)D));
  p.wait_ns = g_wait_ns;
  p.inject = inject;
  p.l_from_p = l_from_p;
  p.trace = trace;
  p.two_level = two_level;
  p.Nk = Nk;
  p.nq = dec ? dec->nq : 1;
  p.G = dec ? dec->G : 1;
  p.nsplit = dec ? dec->nsplit : 1;
  p.tps = dec ? dec->tps : 0;
  p.part_o = dec ? dec->part_o : nullptr;
  p.part_m = dec ? dec->part_m : nullptr;
  p.part_l = dec ? dec->part_l : nullptr;
  if (dec) {
    p.N = 128;
    p.causal = 0;
  }
  if (FAST) fill_neg_log2_scales(p.lneg);
  // persistent grid: as many CTAs as can be resident (TMEM allows 512 / TMEM_COLS per SM);
  // computed once per kernel instance (a function-local static: thread-safe initialisation)
  static const int per_sm = [smem] {
    int n = 0;
    cudaFuncSetAttribute(k_attn_fwd<D, BC, SUMP, DEC, FAST>, cudaFuncAttributePreferredSharedMemoryCarveout,
                         cudaSharedmemCarveoutMaxShared);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_attn_fwd<D, BC, SUMP, DEC, FAST>, C::NTHREADS, smem) != cudaSuccess)
      n = 0;
    const int m = resident_by_limits(k_attn_fwd<D, BC, SUMP, DEC, FAST>, C::NTHREADS, smem);
    if (m > n) n = m;
    if (n <= 0) n = 1;
    return n < (int)(512 / C::TMEM_COLS) ? n : (int)(512 / C::TMEM_COLS);
  }();
  const long long units = dec ? (long long)B * Hkv * dec->nsplit : (long long)B * Hq * (N / 128);
  const long long cap = (long long)per_sm * num_sms();
  const unsigned grid = (unsigned)(units < cap ? units : cap);
  k_attn_fwd<D, BC, SUMP, DEC, FAST><<<grid, C::NTHREADS, smem, stream>>>(tq, tk, tv, p);
  return cuda_status(cudaGetLastError());
}

// Resident CTAs of the transposed decode kernel over the GPU.
template <int NQ>
int decode_t_resident() {
  static const int per_sm = [] {
    // several CTAs share an SM: the largest shared-memory carveout, and the count from the
    // SM's limits (the occupancy query can report fewer)
    int n = 0;
    set_smem(k_attn_decode_t<NQ>, DecTCfg::SMEM);
    cudaFuncSetAttribute(k_attn_decode_t<NQ>, cudaFuncAttributePreferredSharedMemoryCarveout,
                         cudaSharedmemCarveoutMaxShared);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_attn_decode_t<NQ>, DecTCfg::NTHREADS, DecTCfg::SMEM) !=
        cudaSuccess)
      n = 0;
    const int m = resident_by_limits(k_attn_decode_t<NQ>, DecTCfg::NTHREADS, DecTCfg::SMEM);
    if (m > n) n = m;
    if (n <= 0) n = 1;
    if (n > (int)(512 / DecTCfg::TMEM_COLS)) n = 512 / DecTCfg::TMEM_COLS;
    return n;
  }();
  return per_sm * num_sms();
}

int decode_t_resident_for(int rows) {
  return rows <= 4 ? decode_t_resident<4>() : (rows <= 8 ? decode_t_resident<8>() : decode_t_resident<16>());
}

// Decode with keys on the MMA's M dimension (k_attn_decode_t, head dim 128, 128-key tiles,
// at most 16 packed query rows): NQ = the smallest of 4, 8, 16 that holds G * nq.  The
// split count, when the caller leaves it open, is the one (of at most 16 and at least 16
// tiles per split) whose units fill the resident CTAs' rounds best.
template <int NQ>
int launch_decode_t(const hifa4_qtensor* q, const hifa4_qtensor* k, const hifa4_qtensor* vt, int B, int Hkv,
                    const DecodeSpec& dec, int* status, cudaStream_t stream) {
  using C = DecTCfg;
  constexpr int D = C::D;
  const int Nk = dec.Nk;
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q->codes, D / 2, (uint64_t)B * Hkv * 128, D / 2, D / 2, C::NMMA) ||
      !make_map(&tk, k->codes, D / 2, (uint64_t)B * Hkv * Nk, D / 2, D / 2, C::BC) ||
      !make_map(&tv, vt->codes, Nk / 2, (uint64_t)B * Hkv * D, Nk / 2, C::BC / 2, D))
    return HIFA4_ERR_CUDA;
  static bool attr = set_smem(k_attn_decode_t<NQ>, C::SMEM);
  if (!attr) return HIFA4_ERR_CUDA;
  AttnParams p;
  std::memset(&p, 0, sizeof(p));
  p.qsf = static_cast<const uint8_t*>(q->scales);
  p.ksf = static_cast<const uint8_t*>(k->scales);
  p.vsf = static_cast<const uint8_t*>(vt->scales);
  p.status = status;
  p.B = B;
  p.Hq = Hkv * dec.G;
  p.Hkv = Hkv;
  p.N = 128;
  p.causal = 0;
  p.c = (float)(1.4426950408889634074 / std::sqrt((double)D));
  p.wait_ns = g_wait_ns;
  p.Nk = Nk;
  p.nq = dec.nq;
  p.G = dec.G;
  p.nsplit = dec.nsplit;
  p.tps = dec.tps;
  p.part_o = dec.part_o;
  p.part_m = dec.part_m;
  p.part_l = dec.part_l;
  const long long units = (long long)B * Hkv * dec.nsplit;
  const long long cap = (long long)decode_t_resident<NQ>();
  const unsigned grid = (unsigned)(units < cap ? units : cap);
  k_attn_decode_t<NQ><<<grid, C::NTHREADS, C::SMEM, stream>>>(tq, tk, tv, p);
  return cuda_status(cudaGetLastError());
}

// The kv tile chosen for kv_tile = 0: 256 keys at d = 128 when the key count allows it,
// else 128; 128 at d = 64; 64 at d = 256.
int default_kv_tile(int d, int nkeys) {
  if (d == 256) return 64;
  if (d == 128 && nkeys % 256 == 0) return 256;
  return 128;
}

// Host-side checks of an attention call; resolves kv_tile = 0 to the default.  Launches
// nothing, so an entry point that runs other kernels first (hifa4_attn_fwd quantises V)
// calls it before them.
int attn_validate(const hifa4_qtensor* q, const hifa4_qtensor* k, const hifa4_qtensor* vt, int B, int Hq, int Hkv,
                  int N, int d, int& kv_tile, const void* o, const int* status) {
  if (!o || !status || !aligned16(o)) return HIFA4_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || N <= 0 || N % 128 || N > 63488 || !d_ok(d))
    return HIFA4_ERR_UNSUPPORTED_SHAPE;
  if (kv_tile == 0) kv_tile = default_kv_tile(d, N);
  if (kv_tile != 64 && kv_tile != 128 && kv_tile != 256) return HIFA4_ERR_UNSUPPORTED_SHAPE;
  if (d == 256 && kv_tile != 64) return HIFA4_ERR_UNSUPPORTED_SHAPE;
  if (d == 64 && kv_tile == 256) return HIFA4_ERR_UNSUPPORTED_SHAPE;
  if (N % kv_tile) return HIFA4_ERR_UNSUPPORTED_SHAPE;
  if (!qt_ok(q, B, Hq, N, d, 0) || !qt_ok(k, B, Hkv, N, d, 0) || !qt_ok(vt, B, Hkv, N, d, 1))
    return HIFA4_ERR_INVALID_ARG;
  if ((long long)B * Hq * (N / 128) > 0x7FFFFFFFLL) return HIFA4_ERR_UNSUPPORTED_SHAPE;
  if (!device_ok()) return HIFA4_ERR_UNSUPPORTED_DEVICE;
  return HIFA4_OK;
}

// Validation and dispatch shared by the plain, fast and ablation entry points.
template <bool SUMP, bool FAST = false>
int attn_dispatch(const hifa4_qtensor* q, const hifa4_qtensor* k, const hifa4_qtensor* vt, int B, int Hq, int Hkv,
                  int N, int d, int causal, int kv_tile, void* o, void* m_out, void* l_out, int* status,
                  cudaStream_t stream, int l_from_p, float* trace, int two_level, int inject = 0) {
  const int rc = attn_validate(q, k, vt, B, Hq, Hkv, N, d, kv_tile, o, status);
  if (rc != HIFA4_OK) return rc;
#define HIFA4_LAUNCH(DD, BB) \
  launch_attn<DD, BB, SUMP, false, FAST>(q, k, vt, B, Hq, Hkv, N, causal, o, m_out, l_out, status, stream, \
                                         l_from_p, trace, nullptr, two_level, inject)
  if (d == 64) return kv_tile == 64 ? HIFA4_LAUNCH(64, 64) : HIFA4_LAUNCH(64, 128);
  if (d == 128) {
    if (kv_tile == 256) return HIFA4_LAUNCH(128, 256);
    return kv_tile == 64 ? HIFA4_LAUNCH(128, 64) : HIFA4_LAUNCH(128, 128);
  }
  return HIFA4_LAUNCH(256, 64);
#undef HIFA4_LAUNCH
}

}  // namespace

extern "C" {

const char* hifa4_status_string(int s) {
  switch (s) {
    case HIFA4_OK: return "HIFA4_OK";
    case HIFA4_ERR_INVALID_ARG: return "HIFA4_ERR_INVALID_ARG";
    case HIFA4_ERR_UNSUPPORTED_SHAPE: return "HIFA4_ERR_UNSUPPORTED_SHAPE";
    case HIFA4_ERR_UNSUPPORTED_DEVICE: return "HIFA4_ERR_UNSUPPORTED_DEVICE";
    case HIFA4_ERR_NONFINITE: return "HIFA4_ERR_NONFINITE";
    case HIFA4_ERR_TIMEOUT: return "HIFA4_ERR_TIMEOUT";
    case HIFA4_ERR_CUDA: return "HIFA4_ERR_CUDA";
    case HIFA4_ERR_IO: return "HIFA4_ERR_IO";
    default: return "HIFA4_ERR_UNKNOWN";
  }
}

size_t hifa4_qtensor_codes_bytes(int B, int H, int N, int d) {
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return 0;
  return (size_t)B * H * N * (d / 2);
}

size_t hifa4_qtensor_scales_bytes(int B, int H, int N, int d, int transposed) {
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return 0;
  if (!transposed) return (size_t)B * H * (N / 128) * (d / 64) * 512;
  return (size_t)B * H * (N / 64) * ((d + 127) / 128) * 512;
}

size_t hifa4_calibrate_workspace_bytes(int Hkv, int d) {
  if (Hkv <= 0 || d <= 0) return 0;
  return (size_t)2 * Hkv * d * sizeof(float);
}

int hifa4_calibrate_smooth(const void* q_cal, const void* k_cal, const int64_t q_strides[3],
                           const int64_t k_strides[3], int B, int Hq, int Hkv, int N, int d, float alpha,
                           float* s_out, float* sinv_out, void* workspace, cudaStream_t stream) {
  if (!strides_ok(q_cal, q_strides) || !strides_ok(k_cal, k_strides) || !s_out || !sinv_out || !workspace ||
      !(alpha >= 0.0f) || !std::isfinite(alpha))
    return HIFA4_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || Hq % Hkv || !d_ok(d)) return HIFA4_ERR_UNSUPPORTED_SHAPE;
  if (!device_ok()) return HIFA4_ERR_UNSUPPORTED_DEVICE;
  float* amax = static_cast<float*>(workspace);
  cudaError_t e = cudaMemsetAsync(amax, 0, hifa4_calibrate_workspace_bytes(Hkv, d), stream);
  if (e != cudaSuccess) return HIFA4_ERR_CUDA;
  const int rows = 256;
  AmaxArgs aq{static_cast<const __nv_bfloat16*>(q_cal), q_strides[0], q_strides[1], q_strides[2], Hq, Hkv, N, d, amax};
  AmaxArgs ak{static_cast<const __nv_bfloat16*>(k_cal), k_strides[0], k_strides[1], k_strides[2], Hkv, Hkv, N, d,
              amax + Hkv * d};
  k_channel_amax<<<dim3(B * Hq, (N + rows - 1) / rows), 128, 0, stream>>>(aq, rows);
  k_channel_amax<<<dim3(B * Hkv, (N + rows - 1) / rows), 128, 0, stream>>>(ak, rows);
  if (cudaGetLastError() != cudaSuccess) return HIFA4_ERR_CUDA;
  std::vector<float> h(2 * (size_t)Hkv * d), s(Hkv * (size_t)d), si(Hkv * (size_t)d);
  e = cudaMemcpyAsync(h.data(), amax, h.size() * sizeof(float), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return HIFA4_ERR_CUDA;
  for (size_t i = 0; i < s.size(); ++i) {
    const float aq_ = h[i], ak_ = h[s.size() + i];
    float v = 1.0f;
    if (aq_ > 0.0f && ak_ > 0.0f) v = (float)std::pow((double)ak_ / (double)aq_, (double)alpha);
    s[i] = v;
    si[i] = 1.0f / v;
  }
  e = cudaMemcpyAsync(s_out, s.data(), s.size() * sizeof(float), cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(sinv_out, si.data(), si.size() * sizeof(float), cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  return cuda_status(e);
}

int hifa4_quantize_qk(const void* q, const void* k, const int64_t q_strides[3], const int64_t k_strides[3],
                      int B, int Hq, int Hkv, int N, int d, const float* s, const float* sinv,
                      const hifa4_qtensor* q_out, const hifa4_qtensor* k_out, int* status, cudaStream_t stream) {
  if (!strides_ok(q, q_strides) || !strides_ok(k, k_strides) || !status || ((s == nullptr) != (sinv == nullptr)) ||
      (s && (!aligned16(s) || !aligned16(sinv))))
    return HIFA4_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || N <= 0 || N % 128 || !d_ok(d)) return HIFA4_ERR_UNSUPPORTED_SHAPE;
  if (!qt_ok(q_out, B, Hq, N, d, 0) || !qt_ok(k_out, B, Hkv, N, d, 0)) return HIFA4_ERR_INVALID_ARG;
  if (!device_ok()) return HIFA4_ERR_UNSUPPORTED_DEVICE;
  QuantRowsArgs qa{static_cast<const __nv_bfloat16*>(q), q_strides[0], q_strides[1], q_strides[2], Hq, Hkv, N, s,
                   nullptr, nullptr, 0, 0,
                   static_cast<uint8_t*>(q_out->codes), static_cast<uint8_t*>(q_out->scales), stream_row_chunks(B, Hq, N, d)};
  QuantRowsArgs ka{static_cast<const __nv_bfloat16*>(k), k_strides[0], k_strides[1], k_strides[2], Hkv, Hkv, N, sinv,
                   nullptr, nullptr, 0, 0,
                   static_cast<uint8_t*>(k_out->codes), static_cast<uint8_t*>(k_out->scales), stream_row_chunks(B, Hkv, N, d)};
  QuantVtArgs va{};
  return launch_quant_stream(qa, ka, va, d, status, stream);
}

int hifa4_quantize_qk_rope(const void* q, const void* k, const int64_t q_strides[3], const int64_t k_strides[3],
                           int B, int Hq, int Hkv, int N, int d, const float* rope_cos, const float* rope_sin,
                           const float* s, const float* sinv, const hifa4_qtensor* q_out, const hifa4_qtensor* k_out,
                           int* status, cudaStream_t stream) {
  if (!strides_ok(q, q_strides) || !strides_ok(k, k_strides) || !status || ((s == nullptr) != (sinv == nullptr)) ||
      (s && (!aligned16(s) || !aligned16(sinv))) || !rope_cos || !rope_sin || !aligned16(rope_cos) ||
      !aligned16(rope_sin))
    return HIFA4_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || N <= 0 || N % 128 || !d_ok(d)) return HIFA4_ERR_UNSUPPORTED_SHAPE;
  if (!qt_ok(q_out, B, Hq, N, d, 0) || !qt_ok(k_out, B, Hkv, N, d, 0)) return HIFA4_ERR_INVALID_ARG;
  if (!device_ok()) return HIFA4_ERR_UNSUPPORTED_DEVICE;
  QuantRowsArgs qa{static_cast<const __nv_bfloat16*>(q), q_strides[0], q_strides[1], q_strides[2], Hq, Hkv, N, s,
                   rope_cos, rope_sin, 0, 0, static_cast<uint8_t*>(q_out->codes), static_cast<uint8_t*>(q_out->scales),
                   stream_row_chunks(B, Hq, N, d)};
  QuantRowsArgs ka{static_cast<const __nv_bfloat16*>(k), k_strides[0], k_strides[1], k_strides[2], Hkv, Hkv, N, sinv,
                   rope_cos, rope_sin, 0, 0, static_cast<uint8_t*>(k_out->codes), static_cast<uint8_t*>(k_out->scales),
                   stream_row_chunks(B, Hkv, N, d)};
  QuantVtArgs va{};
  return launch_quant_stream(qa, ka, va, d, status, stream, true);
}

int hifa4_rope_table(double theta, int pos0, int N, int d, float* cos_out, float* sin_out) {
  if (!cos_out || !sin_out || !(theta > 1.0) || N <= 0 || pos0 < 0 || !d_ok(d)) return HIFA4_ERR_INVALID_ARG;
  const int half = d / 2;
  for (int i = 0; i < half; ++i) {
    const double inv = std::pow(theta, -2.0 * i / d);
    for (int n = 0; n < N; ++n) {
      const double ang = (double)(pos0 + n) * inv;
      cos_out[(long long)n * half + i] = (float)std::cos(ang);
      sin_out[(long long)n * half + i] = (float)std::sin(ang);
    }
  }
  return HIFA4_OK;
}

int hifa4_quantize_v(const void* v, const int64_t v_strides[3], int B, int Hkv, int N, int d,
                     const hifa4_qtensor* vt_out, int* status, cudaStream_t stream) {
  if (!strides_ok(v, v_strides) || !status) return HIFA4_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || N <= 0 || N % 128 || !d_ok(d)) return HIFA4_ERR_UNSUPPORTED_SHAPE;
  if (!qt_ok(vt_out, B, Hkv, N, d, 1)) return HIFA4_ERR_INVALID_ARG;
  if (!device_ok()) return HIFA4_ERR_UNSUPPORTED_DEVICE;
  QuantRowsArgs none{};
  QuantVtArgs va{static_cast<const __nv_bfloat16*>(v), v_strides[0], v_strides[1], v_strides[2], Hkv, N,
                 static_cast<uint8_t*>(vt_out->codes), static_cast<uint8_t*>(vt_out->scales), stream_row_chunks(B, Hkv, N, d)};
  return launch_quant_stream(none, none, va, d, status, stream);
}

int hifa4_quantize_qkv(const void* q, const void* k, const void* v, const int64_t q_strides[3],
                       const int64_t k_strides[3], const int64_t v_strides[3], int B, int Hq, int Hkv, int N, int d,
                       const float* s, const float* sinv, const hifa4_qtensor* q_out, const hifa4_qtensor* k_out,
                       const hifa4_qtensor* vt_out, int* status, cudaStream_t stream) {
  if (!strides_ok(q, q_strides) || !strides_ok(k, k_strides) || !strides_ok(v, v_strides) || !status ||
      ((s == nullptr) != (sinv == nullptr)) || (s && (!aligned16(s) || !aligned16(sinv))))
    return HIFA4_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || N <= 0 || N % 128 || !d_ok(d)) return HIFA4_ERR_UNSUPPORTED_SHAPE;
  if (!qt_ok(q_out, B, Hq, N, d, 0) || !qt_ok(k_out, B, Hkv, N, d, 0) || !qt_ok(vt_out, B, Hkv, N, d, 1))
    return HIFA4_ERR_INVALID_ARG;
  if (!device_ok()) return HIFA4_ERR_UNSUPPORTED_DEVICE;
  QuantRowsArgs qa{static_cast<const __nv_bfloat16*>(q), q_strides[0], q_strides[1], q_strides[2], Hq, Hkv, N, s,
                   nullptr, nullptr, 0, 0,
                   static_cast<uint8_t*>(q_out->codes), static_cast<uint8_t*>(q_out->scales), stream_row_chunks(B, Hq, N, d)};
  QuantRowsArgs ka{static_cast<const __nv_bfloat16*>(k), k_strides[0], k_strides[1], k_strides[2], Hkv, Hkv, N, sinv,
                   nullptr, nullptr, 0, 0,
                   static_cast<uint8_t*>(k_out->codes), static_cast<uint8_t*>(k_out->scales), stream_row_chunks(B, Hkv, N, d)};
  QuantVtArgs va{static_cast<const __nv_bfloat16*>(v), v_strides[0], v_strides[1], v_strides[2], Hkv, N,
                 static_cast<uint8_t*>(vt_out->codes), static_cast<uint8_t*>(vt_out->scales), stream_row_chunks(B, Hkv, N, d)};
  return launch_quant_stream(qa, ka, va, d, status, stream);
}

int hifa4_attn_fwd_quantized(const hifa4_qtensor* q, const hifa4_qtensor* k, const hifa4_qtensor* vt, int B,
                             int Hq, int Hkv, int N, int d, int causal, int kv_tile, void* o, void* m_out,
                             void* l_out, int* status, cudaStream_t stream) {
  return attn_dispatch<false>(q, k, vt, B, Hq, Hkv, N, d, causal, kv_tile, o, m_out, l_out, status, stream, 0,
                              nullptr, 0);
}

int hifa4_attn_fwd_quantized_fast(const hifa4_qtensor* q, const hifa4_qtensor* k, const hifa4_qtensor* vt, int B,
                                  int Hq, int Hkv, int N, int d, int causal, int kv_tile, void* o, void* m_out,
                                  void* l_out, int* status, cudaStream_t stream) {
  return attn_dispatch<false, true>(q, k, vt, B, Hq, Hkv, N, d, causal, kv_tile, o, m_out, l_out, status, stream, 0,
                                    nullptr, 0);
}

int hifa4_attn_fwd_ablation(const hifa4_qtensor* q, const hifa4_qtensor* k, const hifa4_qtensor* vt, int B, int Hq,
                            int Hkv, int N, int d, int causal, int kv_tile, int normaliser, int two_level,
                            float* trace, void* o, void* m_out, void* l_out, int* status, cudaStream_t stream) {
  if (normaliser != 0 && normaliser != 1) return HIFA4_ERR_INVALID_ARG;
  if (two_level != 0 && two_level != 1) return HIFA4_ERR_INVALID_ARG;
  if (trace && !aligned16(trace)) return HIFA4_ERR_INVALID_ARG;
  return attn_dispatch<true>(q, k, vt, B, Hq, Hkv, N, d, causal, kv_tile, o, m_out, l_out, status, stream,
                             normaliser, trace, two_level);
}

int hifa4_quantize_q_decode(const void* q, const int64_t q_strides[3], int B, int Hq, int Hkv, int nq, int d,
                            const float* s, const hifa4_qtensor* q_out, int* status, cudaStream_t stream) {
  if (!strides_ok(q, q_strides) || !status || (s && !aligned16(s))) return HIFA4_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || nq <= 0 || (Hq / Hkv) * nq > 128 || !d_ok(d))
    return HIFA4_ERR_UNSUPPORTED_SHAPE;
  if (!qt_ok(q_out, B, Hkv, 128, d, 0)) return HIFA4_ERR_INVALID_ARG;
  if (!device_ok()) return HIFA4_ERR_UNSUPPORTED_DEVICE;
  const int rows = d == 256 ? 64 : 128;
  QuantRowsArgs qa{static_cast<const __nv_bfloat16*>(q), q_strides[0], q_strides[1], q_strides[2], Hkv, Hkv, 128, s,
                   nullptr, nullptr, Hq / Hkv, nq, static_cast<uint8_t*>(q_out->codes),
                   static_cast<uint8_t*>(q_out->scales), B * Hkv * (128 / rows)};
  switch (d) {
    case 64: k_quant_q_decode<64><<<resident_grid(k_quant_q_decode<64>, 256, qa.units), 256, 0, stream>>>(qa, status); break;
    case 128: k_quant_q_decode<128><<<resident_grid(k_quant_q_decode<128>, 256, qa.units), 256, 0, stream>>>(qa, status); break;
    default: k_quant_q_decode<256><<<resident_grid(k_quant_q_decode<256>, 256, qa.units), 256, 0, stream>>>(qa, status); break;
  }
  return cuda_status(cudaGetLastError());
}

size_t hifa4_decode_workspace_bytes(int B, int Hkv, int nsplit, int d) {
  if (B <= 0 || Hkv <= 0 || nsplit <= 0 || nsplit > 64 || !d_ok(d)) return 0;
  return (size_t)B * Hkv * nsplit * 128 * (d + 2) * sizeof(float);
}

int hifa4_attn_decode(const hifa4_qtensor* q, const hifa4_qtensor* k, const hifa4_qtensor* vt, int B, int Hq, int Hkv,
                      int nq, int Nk, int d, int kv_tile, int nsplit, void* workspace, size_t workspace_bytes, void* o,
                      void* m_out, void* l_out, int* status, cudaStream_t stream) {
  if (!o || !status || !workspace || !aligned16(o) || !aligned16(workspace)) return HIFA4_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || nq <= 0 || (Hq / Hkv) * nq > 128 || Nk <= 0 || Nk % 128 ||
      Nk > 63488 || !d_ok(d))
    return HIFA4_ERR_UNSUPPORTED_SHAPE;
  const int rowsq = (Hq / Hkv) * nq;
  // the transposed kernel: head dim 128, 128-key tiles, at most 16 packed query rows
  const bool tpath = d == 128 && rowsq <= 16 && (kv_tile == 0 || kv_tile == 128);
  if (kv_tile == 0) kv_tile = tpath ? 128 : default_kv_tile(d, Nk);
  if (kv_tile != 64 && kv_tile != 128 && kv_tile != 256) return HIFA4_ERR_UNSUPPORTED_SHAPE;
  if ((d == 256 && kv_tile != 64) || (d == 64 && kv_tile == 256) || Nk % kv_tile) return HIFA4_ERR_UNSUPPORTED_SHAPE;
  if (!qt_ok(q, B, Hkv, 128, d, 0) || !qt_ok(k, B, Hkv, Nk, d, 0) || !qt_ok(vt, B, Hkv, Nk, d, 1))
    return HIFA4_ERR_INVALID_ARG;
  if (!device_ok()) return HIFA4_ERR_UNSUPPORTED_DEVICE;
  const int ntile = Nk / kv_tile;
  if (nsplit <= 0 && tpath) {
    // the split count (at most 16, at least 16 tiles per split) whose longest CTA path
    // (rounds of resident CTAs x tiles per split) is closest to the even share
    const long long res = decode_t_resident_for(rowsq), bk = (long long)B * Hkv;
    const int maxs = ntile / 16 < 1 ? 1 : (ntile / 16 < 16 ? ntile / 16 : 16);
    double best_eff = -1.0;
    for (int ns = 1; ns <= maxs; ++ns) {
      const int t = (ntile + ns - 1) / ns, nse = (ntile + t - 1) / t;
      const long long rounds = (bk * nse + res - 1) / res;
      const double eff = (double)bk * ntile / ((double)rounds * t * res);
      if (eff > best_eff + 1e-9) {
        best_eff = eff;
        nsplit = ns;
      }
    }
  } else if (nsplit <= 0) {   // enough (batch, kv head, split) units for two waves over the SMs
    const int want = (2 * num_sms() + B * Hkv - 1) / (B * Hkv);
    nsplit = want < 64 ? want : 64;
  }
  if (nsplit > 64) return HIFA4_ERR_UNSUPPORTED_SHAPE;
  if (nsplit > ntile) nsplit = ntile;
  const int tps = (ntile + nsplit - 1) / nsplit;
  nsplit = (ntile + tps - 1) / tps;   // no empty splits (an empty split has weight 0 in the merge)
  if (workspace_bytes < hifa4_decode_workspace_bytes(B, Hkv, nsplit, d)) return HIFA4_ERR_INVALID_ARG;
  float* part_o = static_cast<float*>(workspace);
  float* part_m = part_o + (size_t)B * Hkv * nsplit * 128 * d;
  float* part_l = part_m + (size_t)B * Hkv * nsplit * 128;
  DecodeSpec spec{nq, Hq / Hkv, Nk, nsplit, tps, part_o, part_m, part_l};
  int rc;
  if (tpath) {
    rc = rowsq <= 4 ? launch_decode_t<4>(q, k, vt, B, Hkv, spec, status, stream)
                    : (rowsq <= 8 ? launch_decode_t<8>(q, k, vt, B, Hkv, spec, status, stream)
                                  : launch_decode_t<16>(q, k, vt, B, Hkv, spec, status, stream));
    if (rc != HIFA4_OK) return rc;
  }
#define HIFA4_DEC(DD, BB) \
  launch_attn<DD, BB, false, true>(q, k, vt, B, Hq, Hkv, 128, 0, o, nullptr, nullptr, status, stream, 0, nullptr, &spec)
  if (tpath) rc = HIFA4_OK;
  else if (d == 64) rc = kv_tile == 64 ? HIFA4_DEC(64, 64) : HIFA4_DEC(64, 128);
  else if (d == 128) rc = kv_tile == 256 ? HIFA4_DEC(128, 256) : (kv_tile == 64 ? HIFA4_DEC(128, 64) : HIFA4_DEC(128, 128));
  else rc = HIFA4_DEC(256, 64);
#undef HIFA4_DEC
  if (rc != HIFA4_OK) return rc;
  DecodeMergeArgs ma{part_o, part_m, part_l, static_cast<__nv_bfloat16*>(o), static_cast<__half*>(m_out),
                     static_cast<__half*>(l_out), Hkv, Hq / Hkv, nq, nsplit};
  const unsigned grid = (unsigned)(B * Hkv * (Hq / Hkv) * nq);
  switch (d) {
    case 64: k_decode_merge<64><<<grid, 64, 0, stream>>>(ma); break;
    case 128: k_decode_merge<128><<<grid, 128, 0, stream>>>(ma); break;
    default: k_decode_merge<256><<<grid, 256, 0, stream>>>(ma); break;
  }
  return cuda_status(cudaGetLastError());
}

size_t hifa4_attn_workspace_bytes(int B, int Hkv, int N, int d) {
  const size_t c = hifa4_qtensor_codes_bytes(B, Hkv, N, d);
  return ((c + 255) / 256) * 256 + hifa4_qtensor_scales_bytes(B, Hkv, N, d, 1);
}

int hifa4_attn_fwd(const hifa4_qtensor* q, const hifa4_qtensor* k, const void* v, const int64_t v_strides[3],
                   int B, int Hq, int Hkv, int N, int d, int causal, int kv_tile, void* workspace,
                   size_t workspace_bytes, void* o, void* m_out, void* l_out, int* status, cudaStream_t stream) {
  if (!workspace || !aligned16(workspace) || !strides_ok(v, v_strides)) return HIFA4_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || N <= 0 || !d_ok(d)) return HIFA4_ERR_UNSUPPORTED_SHAPE;
  if (workspace_bytes < hifa4_attn_workspace_bytes(B, Hkv, N, d)) return HIFA4_ERR_INVALID_ARG;
  const size_t c = hifa4_qtensor_codes_bytes(B, Hkv, N, d);
  hifa4_qtensor vt;
  vt.codes = workspace;
  vt.scales = static_cast<uint8_t*>(workspace) + ((c + 255) / 256) * 256;
  vt.B = B;
  vt.H = Hkv;
  vt.N = N;
  vt.d = d;
  vt.transposed = 1;
  // every check of the attention call before the V quantiser launches
  int tile = kv_tile;
  int r = attn_validate(q, k, &vt, B, Hq, Hkv, N, d, tile, o, status);
  if (r != HIFA4_OK) return r;
  r = hifa4_quantize_v(v, v_strides, B, Hkv, N, d, &vt, status, stream);
  if (r != HIFA4_OK) return r;
  return hifa4_attn_fwd_quantized(q, k, &vt, B, Hq, Hkv, N, d, causal, kv_tile, o, m_out, l_out, status, stream);
}

int hifa4_read_status(int* status, int clear, cudaStream_t stream) {
  if (!status) return HIFA4_ERR_INVALID_ARG;
  int h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, status, sizeof(int), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e == cudaSuccess && clear) {
    e = cudaMemsetAsync(status, 0, sizeof(int), stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  }
  if (e != cudaSuccess) return HIFA4_ERR_CUDA;
  if (h & ST_TIMEOUT) return HIFA4_ERR_TIMEOUT;
  if (h & ST_NONFINITE) return HIFA4_ERR_NONFINITE;
  return HIFA4_OK;
}

void hifa4_set_wait_limit_ns(unsigned long long ns) { g_wait_ns = ns ? ns : 1; }

#ifdef HIFA4_TEST_HOOKS
// ---------------------------------------------------------------- test-only exports
// Built only into the test library (libhifa4_test.so, declared in include/hifa4_test.h).

int hifa4_test_attn_fwd_inject(const hifa4_qtensor* q, const hifa4_qtensor* k, const hifa4_qtensor* vt, int B, int Hq,
                               int Hkv, int N, int d, int causal, int kv_tile, int inject, void* o, void* m_out,
                               void* l_out, int* status, cudaStream_t stream) {
  if (inject != 0 && inject != 1) return HIFA4_ERR_INVALID_ARG;
  return attn_dispatch<false>(q, k, vt, B, Hq, Hkv, N, d, causal, kv_tile, o, m_out, l_out, status, stream, 0, nullptr,
                              0, inject);
}

int hifa4_probe_qk_tile(const void* q_codes, const void* q_scales, const void* k_codes, const void* k_scales, int d,
                        int kv_tile, float* S, int* status, cudaStream_t stream) {
  if (!q_codes || !q_scales || !k_codes || !k_scales || !S || !status || !aligned16(q_codes) || !aligned16(k_codes) ||
      !aligned16(q_scales) || !aligned16(k_scales))
    return HIFA4_ERR_INVALID_ARG;
  if (!d_ok(d) || (kv_tile != 64 && kv_tile != 128)) return HIFA4_ERR_UNSUPPORTED_SHAPE;
  if (d == 256 && kv_tile != 64) return HIFA4_ERR_UNSUPPORTED_SHAPE;
  if (!device_ok()) return HIFA4_ERR_UNSUPPORTED_DEVICE;
  CUtensorMap tq, tk;
  if (!make_map(&tq, q_codes, d / 2, 128, d / 2, d / 2, 128) ||
      !make_map(&tk, k_codes, d / 2, kv_tile, d / 2, d / 2, kv_tile))
    return HIFA4_ERR_CUDA;
  auto go = [&](auto kern, uint32_t smem) -> int {
    if (!set_smem(kern, smem)) return HIFA4_ERR_CUDA;
    kern<<<1, 128, smem, stream>>>(tq, tk, static_cast<const uint8_t*>(q_scales), static_cast<const uint8_t*>(k_scales),
                                   S, status, g_wait_ns);
    return cuda_status(cudaGetLastError());
  };
  if (d == 64) return kv_tile == 64 ? go(k_probe_qk<64, 64>, probe_qk_smem<64, 64>()) : go(k_probe_qk<64, 128>, probe_qk_smem<64, 128>());
  if (d == 128) return kv_tile == 64 ? go(k_probe_qk<128, 64>, probe_qk_smem<128, 64>()) : go(k_probe_qk<128, 128>, probe_qk_smem<128, 128>());
  return go(k_probe_qk<256, 64>, probe_qk_smem<256, 64>());
}

int hifa4_probe_pv_tile(const void* p_codes, const void* p_scales, const void* vt_codes, const void* vt_scales, int d,
                        int kv_tile, float* O, float* R, int* status, cudaStream_t stream) {
  if (!p_codes || !p_scales || !vt_codes || !vt_scales || !O || !R || !status || !aligned16(p_codes) ||
      !aligned16(vt_codes) || !aligned16(p_scales) || !aligned16(vt_scales))
    return HIFA4_ERR_INVALID_ARG;
  if (!d_ok(d) || (kv_tile != 64 && kv_tile != 128)) return HIFA4_ERR_UNSUPPORTED_SHAPE;
  if (d == 256 && kv_tile != 64) return HIFA4_ERR_UNSUPPORTED_SHAPE;
  if (!device_ok()) return HIFA4_ERR_UNSUPPORTED_DEVICE;
  CUtensorMap tp, tv;
  if (!make_map(&tp, p_codes, kv_tile / 2, 128, kv_tile / 2, kv_tile / 2, 128) ||
      !make_map(&tv, vt_codes, kv_tile / 2, d, kv_tile / 2, kv_tile / 2, d))
    return HIFA4_ERR_CUDA;
  auto go = [&](auto kern, uint32_t smem) -> int {
    if (!set_smem(kern, smem)) return HIFA4_ERR_CUDA;
    kern<<<1, 128, smem, stream>>>(tp, tv, static_cast<const uint8_t*>(p_scales), static_cast<const uint8_t*>(vt_scales),
                                   O, R, status, g_wait_ns);
    return cuda_status(cudaGetLastError());
  };
  if (d == 64) return kv_tile == 64 ? go(k_probe_pv<64, 64>, probe_pv_smem<64, 64>()) : go(k_probe_pv<64, 128>, probe_pv_smem<64, 128>());
  if (d == 128) return kv_tile == 64 ? go(k_probe_pv<128, 64>, probe_pv_smem<128, 64>()) : go(k_probe_pv<128, 128>, probe_pv_smem<128, 128>());
  return go(k_probe_pv<256, 64>, probe_pv_smem<256, 64>());
}

int hifa4_probe_codec(const float* x, int n, uint8_t* e2m1, uint8_t* e4m3, float* exp2_out, cudaStream_t stream) {
  if (!x || !e2m1 || !e4m3 || !exp2_out || n < 0) return HIFA4_ERR_INVALID_ARG;
  if (n == 0) return HIFA4_OK;
  if (!device_ok()) return HIFA4_ERR_UNSUPPORTED_DEVICE;
  const int grid = (n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096;
  k_probe_codec<<<grid, 256, 0, stream>>>(x, n, e2m1, e4m3, exp2_out);
  return cuda_status(cudaGetLastError());
}

int hifa4_probe_codec_range(uint32_t start, long long n, uint8_t* e2m1, uint8_t* e4m3, cudaStream_t stream) {
  if (!e2m1 || !e4m3 || n < 0 || n > (1ll << 32) - (long long)start) return HIFA4_ERR_INVALID_ARG;
  if (n == 0) return HIFA4_OK;
  if (!device_ok()) return HIFA4_ERR_UNSUPPORTED_DEVICE;
  k_probe_codec_range<<<num_sms() * 8, 256, 0, stream>>>(start, n, e2m1, e4m3);
  return cuda_status(cudaGetLastError());
}

int hifa4_probe_phat(const float* S, const float* m, int nblk, int d, int fast, uint8_t* codes, uint8_t* scales,
                     cudaStream_t stream) {
  if (!S || !m || !codes || !scales || nblk < 0 || (fast != 0 && fast != 1)) return HIFA4_ERR_INVALID_ARG;
  if (!d_ok(d)) return HIFA4_ERR_UNSUPPORTED_SHAPE;
  if (nblk == 0) return HIFA4_OK;
  if (!device_ok()) return HIFA4_ERR_UNSUPPORTED_DEVICE;
  PhatProbeArgs a;
  std::memset(&a, 0, sizeof(a));
  a.S = S;
  a.m = m;
  a.nblk = nblk;
  a.c = (float)(1.4426950408889634074 / std::sqrt((double)d));
  fill_neg_log2_scales(a.lneg);
  a.codes = codes;
  a.scales = scales;
  const int grid = (nblk + 127) / 128 < 1024 ? (nblk + 127) / 128 : 1024;
  if (fast) k_probe_phat<true><<<grid, 128, 0, stream>>>(a);
  else k_probe_phat<false><<<grid, 128, 0, stream>>>(a);
  return cuda_status(cudaGetLastError());
}
#endif  // HIFA4_TEST_HOOKS

}  // extern "C"
