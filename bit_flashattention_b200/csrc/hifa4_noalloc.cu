// Allocation-free form of hifa4_attn_fwd.
//
// hifa4_attn_fwd needs a caller-provided device workspace for the 4-bit V^T it builds
// before the attention kernel runs.  Some callers cannot provide one: a serving process
// whose device memory is entirely handed out up front (a pool that reserves nearly all
// HBM for weights and KV cache), or a caller in a latency-critical loop where a
// cudaMalloc would block on device synchronisation.  hifa4_attn_fwd_noalloc keeps that
// scratch in a fixed-size array compiled into this library instead, so the call
// allocates nothing.
//
// The array occupies kScratchBytes (16 MiB) on every GPU that loads the library, for the
// life of the process.  All calls on a device share it and it keeps whatever the last
// call wrote: calls whose GPU work overlaps (different streams, no ordering between them)
// race on it.  Nothing in it needs to start at zero -- every call rewrites all the bytes
// it reads (V^T codes and scale atoms, padding rows included).  The array's device
// address is looked up once per device and cached; a cudaDeviceReset (or any other
// teardown of the device's primary context) invalidates it, so this entry point must not
// be used again in a process after such a reset.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/hifa4.h"

namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;

static __device__ __align__(256) unsigned char g_vt_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[64] = {};

// Device address of g_vt_scratch on the current device.  In host code the symbol is only
// a host-side stand-in, so the address is looked up once per device (with that device
// current) and cached.  A device that is not sm_100 is reported as such before any
// lookup (this library holds no code for it); a failed lookup clears the runtime's
// sticky last-error so that it does not surface in a later, unrelated call.
int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return HIFA4_ERR_UNSUPPORTED_DEVICE;
  }
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    return HIFA4_ERR_UNSUPPORTED_DEVICE;
  }
  if (major != 10 || minor != 0) return HIFA4_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_vt_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return HIFA4_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return HIFA4_OK;
}

}  // namespace

extern "C" int hifa4_attn_fwd_noalloc(const hifa4_qtensor* q, const hifa4_qtensor* k, const void* v,
                                      const int64_t v_strides[3], int B, int Hq, int Hkv, int N, int d, int causal,
                                      int kv_tile, void* o, void* m_out, void* l_out, int* status,
                                      cudaStream_t stream) {
  const size_t need = hifa4_attn_workspace_bytes(B, Hkv, N, d);
  if (need == 0) return HIFA4_ERR_UNSUPPORTED_SHAPE;
  if (need > kScratchBytes) return HIFA4_ERR_UNSUPPORTED_SHAPE;   // workload too large for the fixed scratch
  void* scratch = nullptr;
  const int r = scratch_address(&scratch);
  if (r != HIFA4_OK) return r;
  return hifa4_attn_fwd(q, k, v, v_strides, B, Hq, Hkv, N, d, causal, kv_tile, scratch, kScratchBytes, o, m_out,
                        l_out, status, stream);
}
