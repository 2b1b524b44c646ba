// The forward pass over host-resident tensors: sage2_attn_fwd_host.
//
// Heads are independent, so the [B,H,N,d] problem is cut into chunks of whole
// heads (contiguous in memory) that flow through the GPU on a few library
// streams: the host->device copy of one chunk, the kernels of another and the
// device->host copy of a third run at the same time.  Each stream owns device
// buffers for one chunk (inputs, output, workspace) from the library's pool;
// chunks go to the streams round-robin, so a stream's buffers are reused only
// after its previous chunk has finished (stream order).  One cudaMemcpyAsync per
// tensor and chunk; the host buffers must be pinned for the copies to overlap.
#include <algorithm>
#include <mutex>

#include "sage2.h"
#include "sage2_internal.h"

namespace sage2 {

constexpr int kHostLanes = 4;
constexpr size_t kHostChunkBytes = static_cast<size_t>(48) << 20;   // inputs per chunk (target)

struct HostLanes {
  cudaStream_t s[kHostLanes] = {};
  cudaEvent_t done[kHostLanes] = {};
  cudaEvent_t fork = nullptr;
  bool ok = false;
};

static HostLanes* host_lanes(int dev, std::unique_lock<std::mutex>* lock) {
  static std::mutex mu[64];
  static HostLanes lanes[64];
  if (dev < 0 || dev >= 64) return nullptr;
  *lock = std::unique_lock<std::mutex>(mu[dev]);
  HostLanes& L = lanes[dev];
  if (!L.ok) {
    bool good = cudaEventCreateWithFlags(&L.fork, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; good && i < kHostLanes; ++i)
      good = cudaStreamCreateWithFlags(&L.s[i], cudaStreamNonBlocking) == cudaSuccess &&
             cudaEventCreateWithFlags(&L.done[i], cudaEventDisableTiming) == cudaSuccess;
    if (!good) return nullptr;
    L.ok = true;
  }
  return &L;
}

}  // namespace sage2

extern "C" sage2_status sage2_attn_fwd_host(const void* q, const void* k, const void* v, void* o,
                                            int B, int H, int N, int d, int dtype, int o_dtype,
                                            int causal, float sm_scale, int qk_format,
                                            int smooth_v, sage2_stream_t stream) {
  using namespace sage2;
  Dims g;
  sage2_status s = check_dims(B, H, N, d, &g);
  if (s != SAGE2_OK) return s;
  if (dtype != SAGE2_F16 && dtype != SAGE2_BF16) return SAGE2_ERR_INVALID_ARG;
  if (o_dtype < SAGE2_F16 || o_dtype > SAGE2_F32) return SAGE2_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SAGE2_ERR_INVALID_ARG;
  if (!(sm_scale > 0.f) || sm_scale > 3.0e38f) return SAGE2_ERR_INVALID_ARG;
  if (!valid_qk_format(qk_format)) return SAGE2_ERR_INVALID_ARG;
  if (smooth_v != 0 && smooth_v != 1) return SAGE2_ERR_INVALID_ARG;
  if (!q || !k || !v || !o) return SAGE2_ERR_INVALID_ARG;

  const int64_t heads = g.BH;
  const size_t head_in = static_cast<size_t>(N) * d * 2;                     // bytes of one head
  const size_t head_out = static_cast<size_t>(N) * d * (o_dtype == SAGE2_F32 ? 4 : 2);
  const int64_t per_chunk = std::max<int64_t>(
      1, std::min<int64_t>(heads, static_cast<int64_t>(kHostChunkBytes / (3 * head_in))));
  const int64_t nchunks = (heads + per_chunk - 1) / per_chunk;
  const int nlanes = static_cast<int>(std::min<int64_t>(kHostLanes, nchunks));

  Dims gc;
  s = check_dims(1, static_cast<int>(per_chunk), N, d, &gc);
  if (s != SAGE2_OK) return s;
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  const size_t in_bytes = up(per_chunk * head_in), out_bytes = up(per_chunk * head_out);
  const size_t lane_bytes = 3 * in_bytes + out_bytes + up(layout(gc, packed_of(qk_format)).total);

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGE2_ERR_CUDA;
  cudaMemPool_t pool = device_pool(dev);
  if (!pool) return SAGE2_ERR_CUDA;
  std::unique_lock<std::mutex> lock;
  HostLanes* lanes = host_lanes(dev, &lock);
  if (!lanes) return SAGE2_ERR_CUDA;
  uint8_t* buf = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(reinterpret_cast<void**>(&buf), lane_bytes * nlanes, pool, st);
  if (e != cudaSuccess) return from_cuda(e);
  e = cudaEventRecord(lanes->fork, st);
  for (int i = 0; e == cudaSuccess && i < nlanes; ++i) e = cudaStreamWaitEvent(lanes->s[i], lanes->fork, 0);

  for (int64_t c = 0; e == cudaSuccess && c < nchunks; ++c) {
    const int lane = static_cast<int>(c % nlanes);
    cudaStream_t ls = lanes->s[lane];
    uint8_t* base = buf + lane * lane_bytes;
    uint8_t *dq = base, *dk = base + in_bytes, *dv = base + 2 * in_bytes, *dout = base + 3 * in_bytes;
    uint8_t* ws = dout + out_bytes;
    const int64_t h0 = c * per_chunk;
    const int nh = static_cast<int>(std::min<int64_t>(per_chunk, heads - h0));
    const size_t ib = nh * head_in, ob = nh * head_out;
    e = cudaMemcpyAsync(dq, static_cast<const uint8_t*>(q) + h0 * head_in, ib, cudaMemcpyHostToDevice, ls);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(dk, static_cast<const uint8_t*>(k) + h0 * head_in, ib, cudaMemcpyHostToDevice, ls);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(dv, static_cast<const uint8_t*>(v) + h0 * head_in, ib, cudaMemcpyHostToDevice, ls);
    if (e != cudaSuccess) break;
    Dims gh;
    check_dims(1, nh, N, d, &gh);                                          // nh <= per_chunk: valid
    e = forward(dq, dk, dv, dout, gh, dtype, o_dtype, causal, sm_scale, qk_format, smooth_v,
                static_cast<int64_t>(N), static_cast<int64_t>(N), ws, ls);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(static_cast<uint8_t*>(o) + h0 * head_out, dout, ob, cudaMemcpyDeviceToHost, ls);
  }
  for (int i = 0; i < nlanes; ++i) {
    const cudaError_t r = cudaEventRecord(lanes->done[i], lanes->s[i]);
    const cudaError_t w = r == cudaSuccess ? cudaStreamWaitEvent(st, lanes->done[i], 0) : r;
    if (e == cudaSuccess) e = w;
  }
  const cudaError_t e2 = cudaFreeAsync(buf, st);
  return from_cuda(e != cudaSuccess ? e : e2);
}
