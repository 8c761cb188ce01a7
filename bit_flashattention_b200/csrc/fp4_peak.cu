// Dense FP4 tensor-core rate of this GPU, measured with the same instruction the attention
// kernel uses: tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 with both
// operands in shared memory (K-major, 32-byte swizzle), UE4M3 block scales in TMEM and an
// fp32 accumulator in TMEM.  One CTA per SM issues `iters` back-to-back M = 128, N = 256,
// K = 64 MMAs into one accumulator (2 * 128 * 256 * 64 flops each) from constant operands,
// so the loop measures the tensor pipe alone: no loads, no epilogue.  The caller times the
// launch with CUDA events; flops = ctas * iters * 2 * 128 * 256 * 64.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/hifa4_peak.h"
#include "ptx.cuh"

using namespace hifa4;

namespace {

constexpr int kM = 128, kN = 256;
constexpr uint32_t kSzA = kM * 32, kSzB = kN * 32;                 // 64 FP4 codes = 32 bytes per row
constexpr uint32_t kOffB = kSzA, kOffSfa = kOffB + kSzB, kOffSfb = kOffSfa + 512, kOffBar = kOffSfb + 1024;
constexpr uint32_t kSmemUsed = kOffBar + 16;
// more than half of an SM's shared memory, so a second CTA cannot become resident and
// wait in tcgen05.alloc for the 512 TMEM columns this one holds
constexpr uint32_t kSmemLaunch = 120 * 1024;

__global__ void __launch_bounds__(128, 1) k_fp4_mma_loop(int iters, int* status, unsigned long long wait_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint32_t* slot = reinterpret_cast<uint32_t*>(smem + kOffBar + 8);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + kOffBar + 12);
  // operands: E2M1 codes 1.0 and 0.5 alternating (bytes 0x12), every scale 1.0 (0x38)
  for (uint32_t i = threadIdx.x; i < (kSzA + kSzB) / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(smem)[i] = 0x12121212u;
  for (uint32_t i = threadIdx.x; i < 1536 / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(smem + kOffSfa)[i] = 0x38383838u;
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 32) {
    tmem_alloc(slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *slot;
  // TMEM columns: accumulator 0..255, A scales 256..259, B scales (two 128-row atoms) 260..267
  if (threadIdx.x == 0) {
    tmem_cp_sf_atom(tbase + 256, smem + kOffSfa);
    tmem_cp_sf_atom(tbase + 260, smem + kOffSfb);
    tmem_cp_sf_atom(tbase + 264, smem + kOffSfb + 512);
    const uint64_t dA = smem_desc(smem_u32(smem), 0, 8 * 32, 6);
    const uint64_t dB = smem_desc(smem_u32(smem + kOffB), 0, 8 * 32, 6);
    constexpr uint32_t idesc = idesc_nvf4(kM, kN);
    for (int i = 0; i < iters; ++i) mma_nvf4(tbase, dA, dB, idesc, tbase + 256, tbase + 260, i > 0 ? 1u : 0u);
    tc_commit(bar);
  }
  __syncwarp();
  // every thread waits (bounded) for the last MMA before TMEM is released; if that wait
  // runs out, the status word says so and thread 0 waits once more, still bounded, for the
  // MMAs it issued before the columns are freed
  if (!mbar_wait(bar, 0, abort, status, wait_ns) && threadIdx.x == 0) {
    int never = 0;
    mbar_wait(bar, 0, &never, status, wait_ns);
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace

extern "C" {

double hifa4_fp4_mma_flops_per_iter(void) { return 2.0 * kM * kN * 64; }

int hifa4_fp4_mma_loop(int ctas, int iters, int* status, cudaStream_t stream) {
  // at most 2^20 MMAs per CTA (about 70 ms at the nominal rate): far inside the bounded wait
  if (ctas <= 0 || iters <= 0 || iters > (1 << 20) || !status) return HIFA4_PEAK_ERR_INVALID_ARG;
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    return HIFA4_PEAK_ERR_UNSUPPORTED_DEVICE;
  }
  if (major != 10 || minor != 0) return HIFA4_PEAK_ERR_UNSUPPORTED_DEVICE;
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [] {
    attr = cudaFuncSetAttribute(k_fp4_mma_loop, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemLaunch);
  });
  if (attr != cudaSuccess) return HIFA4_PEAK_ERR_CUDA;
  static_assert(kSmemUsed + 1024 <= kSmemLaunch, "shared memory layout");
  k_fp4_mma_loop<<<ctas, 128, kSmemLaunch, stream>>>(iters, status, 2000000000ull);
  return cudaGetLastError() == cudaSuccess ? 0 : HIFA4_PEAK_ERR_CUDA;
}

}  // extern "C"
