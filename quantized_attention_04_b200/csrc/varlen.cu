// Variable-length (packed) sequences: sage2_attn_fwd_varlen.
//
// The method's package exposes a variable-length entry ("sageattn_varlen",
// codewithpapers page, code samples list); the pages say nothing more about
// it.  Reading: S sequences packed along the token axis, each one attending
// only within itself (causal: top-left inside the sequence), every step of
// the method applied per sequence as if it were its own batch element (its own
// K mean, Q block means, per-token scales, correction and per-channel V
// scales).
//
// Layout: q, k, v, o are head-major packed, [H, T, d]; sequence s holds tokens
// cu_seqlens[s] .. cu_seqlens[s+1]-1 of every head.  A sequence is then a
// [1, H, N_s, d] problem whose heads are T tokens apart, which the kernels
// take as their head stride.  The sequences are spread over 4 library
// streams, or up to 8 while their workspaces total at most 4 GiB (longest
// first, each to the least-loaded stream), each stream with its own
// workspace sized for the longest sequence, forked from and joined
// back into the caller's stream with events, so that kernels of different
// sequences fill the GPU together.
#include <algorithm>
#include <mutex>
#include <numeric>
#include <vector>

#include "sage2.h"
#include "sage2_internal.h"

namespace sage2 {

constexpr int kVarlenStreams = 8;                        // lanes at most
constexpr int kVarlenBaseLanes = 4;                      // lanes whatever the workspace size
constexpr size_t kVarlenLaneBudget = size_t(4) << 30;    // more lanes only within this much workspace

struct VarlenLanes {
  cudaStream_t s[kVarlenStreams] = {};
  cudaEvent_t done[kVarlenStreams] = {};
  cudaEvent_t fork = nullptr;
  bool ok = false;
};

// Streams and events of device `dev`, created once and kept for the process.
// Calls on one device are serialised by the returned lock's mutex.
static VarlenLanes* varlen_lanes(int dev, std::unique_lock<std::mutex>* lock) {
  static std::mutex mu[64];
  static VarlenLanes lanes[64];
  if (dev < 0 || dev >= 64) return nullptr;
  *lock = std::unique_lock<std::mutex>(mu[dev]);
  VarlenLanes& L = lanes[dev];
  if (!L.ok) {
    bool good = cudaEventCreateWithFlags(&L.fork, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; good && i < kVarlenStreams; ++i) {
      good = cudaStreamCreateWithFlags(&L.s[i], cudaStreamNonBlocking) == cudaSuccess &&
             cudaEventCreateWithFlags(&L.done[i], cudaEventDisableTiming) == cudaSuccess;
    }
    if (!good) return nullptr;
    L.ok = true;
  }
  return &L;
}

}  // namespace sage2

extern "C" sage2_status sage2_attn_fwd_varlen(const void* q, const void* k, const void* v,
                                              void* o, const int* cu_seqlens, int S, int H,
                                              int T, int d, int dtype, int o_dtype, int causal,
                                              float sm_scale, int qk_format, int smooth_v,
                                              sage2_stream_t stream) {
  using namespace sage2;
  if (!cu_seqlens || S <= 0 || H <= 0 || T <= 0) return SAGE2_ERR_INVALID_ARG;
  if (cu_seqlens[0] != 0 || cu_seqlens[S] != T) return SAGE2_ERR_INVALID_ARG;
  int max_n = 0;
  for (int s = 0; s < S; ++s) {
    const int n = cu_seqlens[s + 1] - cu_seqlens[s];
    if (n < 0) return SAGE2_ERR_INVALID_ARG;
    max_n = n > max_n ? n : max_n;
  }
  Dims gmax, gall;
  sage2_status st_ = check_dims(1, H, max_n, d, &gmax);
  if (st_ != SAGE2_OK) return st_;
  st_ = check_dims(1, H, T, d, &gall);   // the packed tensors' own index range
  if (st_ != SAGE2_OK) return st_;
  if (dtype != SAGE2_F16 && dtype != SAGE2_BF16) return SAGE2_ERR_INVALID_ARG;
  if (o_dtype < SAGE2_F16 || o_dtype > SAGE2_F32) return SAGE2_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SAGE2_ERR_INVALID_ARG;
  if (!(sm_scale > 0.f) || sm_scale > 3.0e38f) return SAGE2_ERR_INVALID_ARG;
  if (!valid_qk_format(qk_format)) return SAGE2_ERR_INVALID_ARG;
  if (smooth_v != 0 && smooth_v != 1) return SAGE2_ERR_INVALID_ARG;
  st_ = check_ptrs(q, k, v, o);
  if (st_ != SAGE2_OK) return st_;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGE2_ERR_CUDA;
  cudaMemPool_t pool = device_pool(dev);
  if (!pool) return SAGE2_ERR_CUDA;
  std::unique_lock<std::mutex> lock;
  VarlenLanes* lanes = varlen_lanes(dev, &lock);
  if (!lanes) return SAGE2_ERR_CUDA;

  // longest first, each to the stream with the least work (sum of N^2) so far
  std::vector<int> order(S);
  std::iota(order.begin(), order.end(), 0);
  auto len = [&](int s) { return cu_seqlens[s + 1] - cu_seqlens[s]; };
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return len(a) > len(b); });
  int nlanes = 0;
  for (int s = 0; s < S; ++s) nlanes += len(s) > 0;
  if (nlanes == 0) return SAGE2_OK;
  const size_t ws_bytes = (layout(gmax, packed_of(qk_format)).total + 255) & ~static_cast<size_t>(255);
  // short sequences (small workspaces) gain from more lanes; long ones fill
  // the GPU on their own, and their workspaces are large
  int cap = kVarlenBaseLanes;
  while (cap < kVarlenStreams && static_cast<size_t>(cap + 1) * ws_bytes <= kVarlenLaneBudget) ++cap;
  nlanes = std::min(nlanes, cap);
  uint8_t* ws = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(reinterpret_cast<void**>(&ws), ws_bytes * nlanes, pool, st);
  if (e != cudaSuccess) return from_cuda(e);
  // fork: every lane starts after the caller's earlier work (and the workspace)
  e = cudaEventRecord(lanes->fork, st);
  for (int i = 0; e == cudaSuccess && i < nlanes; ++i) e = cudaStreamWaitEvent(lanes->s[i], lanes->fork, 0);

  const size_t in_row = static_cast<size_t>(d) * 2;                        // bytes per input token
  const size_t out_row = static_cast<size_t>(d) * (o_dtype == SAGE2_F32 ? 4 : 2);
  double load[kVarlenStreams] = {};
  for (int i = 0; e == cudaSuccess && i < S; ++i) {
    const int s = order[i], n = len(s);
    if (n == 0) continue;
    int lane = 0;
    for (int j = 1; j < nlanes; ++j)
      if (load[j] < load[lane]) lane = j;
    load[lane] += static_cast<double>(n) * n;
    Dims g;
    check_dims(1, H, n, d, &g);                                            // n <= max_n: valid
    const size_t t0 = static_cast<size_t>(cu_seqlens[s]);
    e = forward(static_cast<const uint8_t*>(q) + t0 * in_row,
                static_cast<const uint8_t*>(k) + t0 * in_row,
                static_cast<const uint8_t*>(v) + t0 * in_row, static_cast<uint8_t*>(o) + t0 * out_row,
                g, dtype, o_dtype, causal, sm_scale, qk_format, smooth_v,
                static_cast<int64_t>(T), static_cast<int64_t>(T), ws + lane * ws_bytes,
                lanes->s[lane]);
  }
  // join: the caller's stream waits for every lane, then returns the workspace
  for (int i = 0; i < nlanes; ++i) {
    const cudaError_t r = cudaEventRecord(lanes->done[i], lanes->s[i]);
    const cudaError_t w = r == cudaSuccess ? cudaStreamWaitEvent(st, lanes->done[i], 0) : r;
    if (e == cudaSuccess) e = w;
  }
  const cudaError_t e2 = cudaFreeAsync(ws, st);
  return from_cuda(e != cudaSuccess ? e : e2);
}
