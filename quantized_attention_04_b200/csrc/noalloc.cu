// Allocation-free variant of sage2_attn_fwd.
//
// sage2_attn_fwd takes its scratch (the quantized payloads: INT4 Q/K, e4m3 V,
// scales, means, the correction matrix) from a stream-ordered memory pool.
// Some callers cannot let a library allocate device memory at call time: hosts
// that forbid allocator calls once they are running (real-time or embedded
// services that reserve all memory up front), frameworks that account for every
// device byte through their own allocator and reject hidden pools, and code
// that is not allowed to touch the driver's allocator from the thread or
// context it runs in.  sage2_attn_fwd_noalloc serves them: it runs the same
// kernels, in the same order, with the scratch carved out of one fixed
// file-scope device array instead of the pool.  It calls no cudaMalloc,
// cudaFree or pool routine.
//
// Costs and rules, for a user of this entry point:
//  - The array is kNoAllocScratchBytes (64 MiB) on every GPU that loads this
//    library, held until the process exits.  Problems whose scratch
//    (sage2_workspace_bytes) exceeds it are rejected with SAGE2_ERR_TOO_LARGE
//    before anything is launched.
//  - The first call on a device looks the array's device address up
//    (cudaGetSymbolAddress, with that device current) and caches it; make that
//    first call before any stream capture on that device.  The cached address
//    belongs to the device's context: after a cudaDeviceReset of the device it
//    is stale, so the library is not to be called on that device again.
//  - Every call uses the same array and it keeps the previous call's
//    contents.  What must start at zero (the per-channel |V| maximum) is
//    cleared on the stream by every call; everything else is overwritten
//    before it is read.  Two calls whose GPU work overlaps (on different
//    streams, or from different host threads without ordering) race on the
//    array: order them on one stream.
#include <mutex>

#include "sage2.h"
#include "sage2_internal.h"

namespace sage2 {

constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(64) << 20;  // 64 MiB

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on device `dev` (which must be current).
// Looked up once per device; in host code the array's name is only a stand-in.
static void* noalloc_scratch(int dev, cudaError_t* err) {
  static std::mutex mu;
  static void* addr[64] = {};
  if (dev < 0 || dev >= 64) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      *err = e != cudaSuccess ? e : cudaErrorInvalidSymbol;
      return nullptr;
    }
    addr[dev] = p;
  }
  *err = cudaSuccess;
  return addr[dev];
}

}  // namespace sage2

extern "C" sage2_status sage2_attn_fwd_noalloc(const void* q, const void* k, const void* v,
                                               void* o, int B, int H, int N, int d, int dtype,
                                               int o_dtype, int causal, float sm_scale,
                                               sage2_stream_t stream) {
  using namespace sage2;
  Dims g;
  sage2_status s = check_dims(B, H, N, d, &g);
  if (s != SAGE2_OK) return s;
  if (dtype != SAGE2_F16 && dtype != SAGE2_BF16) return SAGE2_ERR_INVALID_ARG;
  if (o_dtype < SAGE2_F16 || o_dtype > SAGE2_F32) return SAGE2_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SAGE2_ERR_INVALID_ARG;
  if (!(sm_scale > 0.f) || sm_scale > 3.0e38f) return SAGE2_ERR_INVALID_ARG;
  s = check_ptrs(q, k, v, o);
  if (s != SAGE2_OK) return s;
  const Workspace w = layout(g);
  if (w.total > kNoAllocScratchBytes) return SAGE2_ERR_TOO_LARGE;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGE2_ERR_CUDA;
  cudaError_t e = cudaSuccess;
  uint8_t* ws = static_cast<uint8_t*>(noalloc_scratch(dev, &e));
  if (ws == nullptr) return SAGE2_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  e = forward(q, k, v, o, g, dtype, o_dtype, causal, sm_scale, SAGE2_QK_INT4, 0, static_cast<int64_t>(N),
              static_cast<int64_t>(N), ws, st);
  return from_cuda(e);
}
