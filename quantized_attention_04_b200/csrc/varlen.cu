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
// take as their head stride: each sequence runs the forward pass's kernels on
// the stream, in order, on one workspace sized for the longest sequence.
#include "sage2.h"
#include "sage2_internal.h"

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
  uint8_t* ws = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(reinterpret_cast<void**>(&ws), layout(gmax).total, pool, st);
  if (e != cudaSuccess) return from_cuda(e);
  const size_t in_row = static_cast<size_t>(d) * 2;                        // bytes per input token
  const size_t out_row = static_cast<size_t>(d) * (o_dtype == SAGE2_F32 ? 4 : 2);
  for (int s = 0; e == cudaSuccess && s < S; ++s) {
    const int n = cu_seqlens[s + 1] - cu_seqlens[s];
    if (n == 0) continue;
    Dims g;
    check_dims(1, H, n, d, &g);                                            // n <= max_n: valid
    const size_t t0 = static_cast<size_t>(cu_seqlens[s]);
    e = forward(static_cast<const uint8_t*>(q) + t0 * in_row,
                static_cast<const uint8_t*>(k) + t0 * in_row,
                static_cast<const uint8_t*>(v) + t0 * in_row, static_cast<uint8_t*>(o) + t0 * out_row,
                g, dtype, o_dtype, causal, sm_scale, qk_bits_of(qk_format), smooth_v,
                static_cast<int64_t>(T), static_cast<int64_t>(T), ws, st);
  }
  const cudaError_t e2 = cudaFreeAsync(ws, st);
  return from_cuda(e != cudaSuccess ? e : e2);
}
