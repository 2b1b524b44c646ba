// C ABI of libsage2 (declared in include/sage2.h): argument validation,
// workspace layout, tensor maps and the stream-ordered launches.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <climits>
#include <cstdint>
#include <mutex>

#include "sage2.h"
#include "sage2_internal.h"
#include "sm100_ptx.cuh"

namespace sage2 {

// ------------------------------------------------------------ tensor maps
static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

cudaError_t make_tmap_u8_2d(void* tmap_out, const void* base, uint64_t rows, uint64_t cols,
                            uint32_t box_rows, uint32_t box_cols) {
  auto fn = get_encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};  // bytes between consecutive rows
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t elem_strides[2] = {1, 1};
  const CUtensorMapSwizzle sw = box_cols == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                : box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                 : CU_TENSOR_MAP_SWIZZLE_NONE;
  const CUresult r = fn(reinterpret_cast<CUtensorMap*>(tmap_out), CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                        const_cast<void*>(base), dims, strides, box, elem_strides,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap(void* tmap_out, const void* base, int rank, const uint64_t* dims,
                      const uint64_t* strides_bytes, const uint32_t* box, int elem_bytes,
                      int swizzle_bytes) {
  auto fn = get_encode_fn();
  if (!fn || rank < 1 || rank > 5) return cudaErrorNotSupported;
  cuuint64_t d[5], st[4];
  cuuint32_t b[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) st[i] = strides_bytes[i];
  const CUtensorMapDataType ty = elem_bytes == 1   ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16
                                                   : CU_TENSOR_MAP_DATA_TYPE_UINT32;
  const CUtensorMapSwizzle sw = swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                      : CU_TENSOR_MAP_SWIZZLE_NONE;
  const CUresult r = fn(reinterpret_cast<CUtensorMap*>(tmap_out), ty, rank, const_cast<void*>(base),
                        d, st, b, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// ------------------------------------------------------------ validation
struct Dims {
  int B, H, N, d, Np, NB;
  int64_t BH;
};

static sage2_status check_dims(int B, int H, int N, int d, Dims* out) {
  if (B <= 0 || H <= 0 || N <= 0) return SAGE2_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SAGE2_ERR_UNSUPPORTED;
  const int64_t BH = static_cast<int64_t>(B) * H;
  const int64_t Np = ((static_cast<int64_t>(N) + kTile - 1) / kTile) * kTile;
  // TMA row coordinates and grid dimensions are 32-bit; grid.y <= 65535.
  if (BH > 65535 || BH * Np > INT32_MAX || BH * d > INT32_MAX || Np > INT32_MAX / 2)
    return SAGE2_ERR_UNSUPPORTED;
  out->B = B;
  out->H = H;
  out->N = N;
  out->d = d;
  out->Np = static_cast<int>(Np);
  out->NB = static_cast<int>(Np / kTile);
  out->BH = BH;
  return SAGE2_OK;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <typename... P>
static sage2_status check_ptrs(P... ps) {
  const void* arr[] = {static_cast<const void*>(ps)...};
  for (const void* p : arr)
    if (!p) return SAGE2_ERR_INVALID_ARG;
  for (const void* p : arr)
    if (!aligned16(p)) return SAGE2_ERR_MISALIGNED;
  return SAGE2_OK;
}

static bool valid_qk_format(int f) {
  return f == SAGE2_QK_INT4 || f == SAGE2_QK_INT8 || f == SAGE2_QK_INT4_PACKED;
}
static int qk_bits_of(int f) { return f == SAGE2_QK_INT8 ? 8 : 4; }
static bool packed_of(int f) { return f == SAGE2_QK_INT4_PACKED; }

static sage2_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return SAGE2_OK;
  if (e == cudaErrorMemoryAllocation) return SAGE2_ERR_NO_MEM;
  return SAGE2_ERR_CUDA;
}

// ------------------------------------------------------------ workspace
struct Workspace {
  size_t off_q_i4, off_k_i4, off_vt, off_qs, off_ks, off_qm, off_km, off_corr, off_vs, off_part,
      off_amax, off_qsplit, off_vmean, off_done, off_qpk, off_kpk, total;
};

static size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// packed: room for the packed INT4 payloads as well (SAGE2_QK_INT4_PACKED),
// which the quantizer writes and an unpack pass expands into q_i4 / k_i4.
static Workspace layout(const Dims& g, bool packed = false) {
  Workspace w{};
  const size_t BH = static_cast<size_t>(g.BH), Np = g.Np, NB = g.NB, d = g.d;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += up256(bytes);
    return at;
  };
  w.off_q_i4 = take(BH * Np * d);
  w.off_k_i4 = take(BH * Np * d);
  w.off_vt = take(BH * d * Np);
  w.off_qs = take(BH * Np * 4);
  w.off_ks = take(BH * Np * 4);
  w.off_qm = take(BH * NB * d * 4);
  w.off_km = take(BH * d * 4);
  w.off_corr = take(BH * NB * Np * 4);
  w.off_vs = take(BH * d * 4);
  w.off_part = take(BH * NB * d * 4);
  w.off_amax = take(BH * d * 4);
  w.off_qsplit = take(3 * BH * ((NB + 127) / 128) * 128 * d * 2);
  w.off_vmean = take(BH * d * 4);
  w.off_done = take(2 * BH * 4);               // K-mean and V-mean block counters
  w.off_qpk = packed ? take(BH * Np * d / 2) : 0;
  w.off_kpk = packed ? take(BH * Np * d / 2) : 0;
  w.total = o;
  return w;
}

// One stream-ordered pool per device that keeps freed memory for reuse.
static cudaMemPool_t device_pool(int dev) {
  static std::mutex mu;
  static cudaMemPool_t pools[64] = {};
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 0 || dev >= 64) return nullptr;
  if (!pools[dev]) {
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t p = nullptr;
    if (cudaMemPoolCreate(&p, &props) != cudaSuccess) return nullptr;
    uint64_t keep = UINT64_MAX;
    cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &keep);
    pools[dev] = p;
  }
  return pools[dev];
}

// A library stream per device for running independent chains of one call
// concurrently, with its fork / join events.  The lock is held while a call
// enqueues (its events are recorded and waited on in that window).
struct SideLane {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  bool ok = false;
};

static SideLane* side_lane(int dev, std::unique_lock<std::mutex>* lock) {
  static std::mutex mu[64];
  static SideLane lanes[64];
  if (dev < 0 || dev >= 64) return nullptr;
  *lock = std::unique_lock<std::mutex>(mu[dev]);
  SideLane& L = lanes[dev];
  if (!L.ok) {
    const bool good = cudaStreamCreateWithFlags(&L.s, cudaStreamNonBlocking) == cudaSuccess &&
                      cudaEventCreateWithFlags(&L.fork, cudaEventDisableTiming) == cudaSuccess &&
                      cudaEventCreateWithFlags(&L.join, cudaEventDisableTiming) == cudaSuccess;
    if (!good) return nullptr;
    L.ok = true;
  }
  return &L;
}

// One forward pass over B*H heads of N tokens: q/k/v heads ldh tokens apart,
// o heads ldo tokens apart, payloads in the workspace ws (layout(g)), all on st.
// With `side` (a SideLane held by the caller), the Q chain (Q smoothing,
// q-mean split, correction) runs on the side stream while the K chain and the
// V chain run on st; they join before the attention kernel.
static cudaError_t forward(const void* q, const void* k, const void* v, void* o, const Dims& g,
                           int dtype, int o_dtype, int causal, float sm_scale, int qk_format,
                           int smooth_v, int64_t ldh, int64_t ldo, uint8_t* ws, cudaStream_t st,
                           SideLane* side = nullptr) {
  const int B = g.B, H = g.H, N = g.N, d = g.d;
  const int qk_bits = qk_bits_of(qk_format);
  const bool packed = packed_of(qk_format);
  const Workspace w = layout(g, packed);
  cudaError_t e;
  uint8_t* q_i4 = reinterpret_cast<uint8_t*>(ws + w.off_q_i4);
  uint8_t* k_i4 = reinterpret_cast<uint8_t*>(ws + w.off_k_i4);
  uint8_t* vt = ws + w.off_vt;
  float* qs = reinterpret_cast<float*>(ws + w.off_qs);
  float* ks = reinterpret_cast<float*>(ws + w.off_ks);
  float* qm = reinterpret_cast<float*>(ws + w.off_qm);
  float* km = reinterpret_cast<float*>(ws + w.off_km);
  float* corr = reinterpret_cast<float*>(ws + w.off_corr);
  float* vs = reinterpret_cast<float*>(ws + w.off_vs);
  float* part = reinterpret_cast<float*>(ws + w.off_part);
  uint32_t* amax = reinterpret_cast<uint32_t*>(ws + w.off_amax);
  float* vmean = smooth_v ? reinterpret_cast<float*>(ws + w.off_vmean) : nullptr;

  unsigned* done = reinterpret_cast<unsigned*>(ws + w.off_done);
  QKArgs qa{q, k, dtype, B, H, N, d, g.Np, g.NB, packed ? ws + w.off_qpk : q_i4, qs, qm,
            packed ? ws + w.off_kpk : k_i4, ks, km, corr, part, ws + w.off_qsplit, causal, qk_bits,
            ldh, packed ? 1 : 0, done, side ? side->s : nullptr, side ? side->fork : nullptr,
            nullptr};
  // the V mean reuses the K-mean scratch: stream order puts it after the K mean
  VArgs va{v, dtype, B, H, N, d, g.Np, g.NB, vt, vs, amax, vmean, part, ldh, done + g.BH};
  AttnArgs aa{q_i4, qs, k_i4, ks, corr, vt, vs, o, o_dtype, B, H, N, d, g.Np, g.NB, causal,
              sm_scale, qk_bits, vmean, ldo};
  e = launch_smooth_quant_qk(qa, st);
  if (e == cudaSuccess) e = launch_quant_v(va, st);
  if (e == cudaSuccess && side) {
    e = cudaEventRecord(side->join, side->s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, side->join, 0);
  }
  if (e == cudaSuccess && packed) {
    const size_t pk_bytes = static_cast<size_t>(g.BH) * g.Np * d / 2;
    e = launch_unpack_int4(ws + w.off_qpk, q_i4, pk_bytes, st);
    if (e == cudaSuccess) e = launch_unpack_int4(ws + w.off_kpk, k_i4, pk_bytes, st);
  }
  if (e == cudaSuccess) e = launch_attn(aa, st);
  return e;
}

}  // namespace sage2

using namespace sage2;

extern "C" {

sage2_status sage2_smooth_quant_qk_ex(const void* q, const void* k, int dtype, int B, int H, int N,
                                      int d, uint8_t* q_i4, float* q_scale, float* q_mean,
                                      uint8_t* k_i4, float* k_scale, float* k_mean,
                                      float* qk_corr, int qk_format, sage2_stream_t stream) {
  Dims g;
  sage2_status s = check_dims(B, H, N, d, &g);
  if (s != SAGE2_OK) return s;
  if (dtype != SAGE2_F16 && dtype != SAGE2_BF16) return SAGE2_ERR_INVALID_ARG;
  const int causal_corr = (qk_format & SAGE2_QK_CAUSAL_CORR) ? 1 : 0;
  qk_format &= ~SAGE2_QK_CAUSAL_CORR;
  if (!valid_qk_format(qk_format)) return SAGE2_ERR_INVALID_ARG;
  s = check_ptrs(q, k, q_i4, q_scale, q_mean, k_i4, k_scale, k_mean, qk_corr);
  if (s != SAGE2_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // scratch: the K-mean partial sums and block counters, the split q_mean terms
  const size_t part_bytes = up256(static_cast<size_t>(g.BH) * g.NB * d * 4);
  const size_t done_bytes = up256(static_cast<size_t>(g.BH) * 4);
  const size_t split_bytes =
      up256(3 * static_cast<size_t>(g.BH) * ((g.NB + 127) / 128) * 128 * d * 2);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGE2_ERR_CUDA;
  cudaMemPool_t pool = device_pool(dev);
  if (!pool) return SAGE2_ERR_CUDA;
  uint8_t* scratch = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(reinterpret_cast<void**>(&scratch),
                                          part_bytes + done_bytes + split_bytes, pool, st);
  if (e != cudaSuccess) return from_cuda(e);
  // the Q chain runs on the library's side stream, concurrently with the K chain
  std::unique_lock<std::mutex> lock;
  SideLane* side = side_lane(dev, &lock);
  QKArgs a{q, k, dtype, B, H, N, d, g.Np, g.NB, q_i4, q_scale, q_mean, k_i4, k_scale, k_mean,
           qk_corr, reinterpret_cast<float*>(scratch), scratch + part_bytes + done_bytes,
           causal_corr, qk_bits_of(qk_format), static_cast<int64_t>(N),
           packed_of(qk_format) ? 1 : 0, reinterpret_cast<unsigned*>(scratch + part_bytes),
           side ? side->s : nullptr, side ? side->fork : nullptr, side ? side->join : nullptr};
  e = launch_smooth_quant_qk(a, st);
  const cudaError_t e2 = cudaFreeAsync(scratch, st);
  return from_cuda(e != cudaSuccess ? e : e2);
}

sage2_status sage2_smooth_quant_qk(const void* q, const void* k, int dtype, int B, int H, int N,
                                   int d, uint8_t* q_i4, float* q_scale, float* q_mean,
                                   uint8_t* k_i4, float* k_scale, float* k_mean, float* qk_corr,
                                   sage2_stream_t stream) {
  return sage2_smooth_quant_qk_ex(q, k, dtype, B, H, N, d, q_i4, q_scale, q_mean, k_i4, k_scale,
                                  k_mean, qk_corr, SAGE2_QK_INT4, stream);
}

sage2_status sage2_quant_v_ex(const void* v, int dtype, int B, int H, int N, int d,
                              uint8_t* v_fp8_t, float* v_scale, float* v_mean,
                              sage2_stream_t stream) {
  Dims g;
  sage2_status s = check_dims(B, H, N, d, &g);
  if (s != SAGE2_OK) return s;
  if (dtype != SAGE2_F16 && dtype != SAGE2_BF16) return SAGE2_ERR_INVALID_ARG;
  s = check_ptrs(v, v_fp8_t, v_scale);
  if (s != SAGE2_OK) return s;
  if (v_mean && !aligned16(v_mean)) return SAGE2_ERR_MISALIGNED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // scratch: the per-channel |V| maximum and, with smoothing, the mean partial sums
  const size_t amax_bytes = up256(static_cast<size_t>(g.BH) * d * 4);
  const size_t part_bytes = v_mean ? up256(static_cast<size_t>(g.BH) * g.NB * d * 4) +
                                         up256(static_cast<size_t>(g.BH) * 4)
                                   : 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGE2_ERR_CUDA;
  cudaMemPool_t pool = device_pool(dev);
  if (!pool) return SAGE2_ERR_CUDA;
  uint8_t* scratch = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(reinterpret_cast<void**>(&scratch),
                                          amax_bytes + part_bytes, pool, st);
  if (e != cudaSuccess) return from_cuda(e);
  VArgs a{v, dtype, B, H, N, d, g.Np, g.NB, v_fp8_t, v_scale,
          reinterpret_cast<uint32_t*>(scratch), v_mean,
          v_mean ? reinterpret_cast<float*>(scratch + amax_bytes) : nullptr,
          static_cast<int64_t>(N),
          v_mean ? reinterpret_cast<unsigned*>(scratch + amax_bytes +
                                               up256(static_cast<size_t>(g.BH) * g.NB * d * 4))
                 : nullptr};
  e = launch_quant_v(a, st);
  const cudaError_t e2 = cudaFreeAsync(scratch, st);
  return from_cuda(e != cudaSuccess ? e : e2);
}

sage2_status sage2_quant_v(const void* v, int dtype, int B, int H, int N, int d, uint8_t* v_fp8_t,
                           float* v_scale, sage2_stream_t stream) {
  return sage2_quant_v_ex(v, dtype, B, H, N, d, v_fp8_t, v_scale, nullptr, stream);
}

sage2_status sage2_attn_fwd_quantized_ex(const uint8_t* q_i4, const float* q_scale,
                                         const uint8_t* k_i4, const float* k_scale,
                                         const float* qk_corr, const uint8_t* v_fp8_t,
                                         const float* v_scale, const float* v_mean, void* o,
                                         int o_dtype, int B, int H, int N, int d, int causal,
                                         float sm_scale, int qk_format, sage2_stream_t stream) {
  if (!valid_qk_format(qk_format)) return SAGE2_ERR_INVALID_ARG;
  if (v_mean && !aligned16(v_mean)) return SAGE2_ERR_MISALIGNED;
  Dims g;
  sage2_status s = check_dims(B, H, N, d, &g);
  if (s != SAGE2_OK) return s;
  if (o_dtype < SAGE2_F16 || o_dtype > SAGE2_F32) return SAGE2_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SAGE2_ERR_INVALID_ARG;
  if (!(sm_scale > 0.f) || sm_scale > 3.0e38f) return SAGE2_ERR_INVALID_ARG;
  s = check_ptrs(q_i4, q_scale, k_i4, k_scale, qk_corr, v_fp8_t, v_scale, o);
  if (s != SAGE2_OK) return s;
  AttnArgs a{q_i4, q_scale, k_i4, k_scale, qk_corr, v_fp8_t, v_scale, o, o_dtype,
             B,    H,       N,    d,       g.Np,    g.NB,    causal,  sm_scale,
             qk_bits_of(qk_format), v_mean, static_cast<int64_t>(N)};
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (!packed_of(qk_format)) return from_cuda(launch_attn(a, st));
  // packed INT4: expand both payloads to e4m3 codes in pool scratch first
  const size_t codes = up256(static_cast<size_t>(g.BH) * g.Np * d);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGE2_ERR_CUDA;
  cudaMemPool_t pool = device_pool(dev);
  if (!pool) return SAGE2_ERR_CUDA;
  uint8_t* scratch = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(reinterpret_cast<void**>(&scratch), 2 * codes, pool, st);
  if (e != cudaSuccess) return from_cuda(e);
  e = launch_unpack_int4(q_i4, scratch, static_cast<size_t>(g.BH) * g.Np * d / 2, st);
  if (e == cudaSuccess)
    e = launch_unpack_int4(k_i4, scratch + codes, static_cast<size_t>(g.BH) * g.Np * d / 2, st);
  a.q_i4 = scratch;
  a.k_i4 = scratch + codes;
  if (e == cudaSuccess) e = launch_attn(a, st);
  const cudaError_t e2 = cudaFreeAsync(scratch, st);
  return from_cuda(e != cudaSuccess ? e : e2);
}

sage2_status sage2_attn_fwd_quantized(const uint8_t* q_i4, const float* q_scale,
                                      const uint8_t* k_i4, const float* k_scale,
                                      const float* qk_corr, const uint8_t* v_fp8_t,
                                      const float* v_scale, void* o, int o_dtype, int B, int H,
                                      int N, int d, int causal, float sm_scale,
                                      sage2_stream_t stream) {
  return sage2_attn_fwd_quantized_ex(q_i4, q_scale, k_i4, k_scale, qk_corr, v_fp8_t, v_scale,
                                     nullptr, o, o_dtype, B, H, N, d, causal, sm_scale,
                                     SAGE2_QK_INT4, stream);
}

size_t sage2_workspace_bytes(int B, int H, int N, int d) {
  Dims g;
  if (check_dims(B, H, N, d, &g) != SAGE2_OK) return 0;
  return layout(g).total;
}

sage2_status sage2_attn_fwd_ex(const void* q, const void* k, const void* v, void* o, int B,
                               int H, int N, int d, int dtype, int o_dtype, int causal,
                               float sm_scale, int qk_format, int smooth_v,
                               sage2_stream_t stream) {
  if (!valid_qk_format(qk_format)) return SAGE2_ERR_INVALID_ARG;
  if (smooth_v != 0 && smooth_v != 1) return SAGE2_ERR_INVALID_ARG;
  Dims g;
  sage2_status s = check_dims(B, H, N, d, &g);
  if (s != SAGE2_OK) return s;
  if (dtype != SAGE2_F16 && dtype != SAGE2_BF16) return SAGE2_ERR_INVALID_ARG;
  if (o_dtype < SAGE2_F16 || o_dtype > SAGE2_F32) return SAGE2_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SAGE2_ERR_INVALID_ARG;
  if (!(sm_scale > 0.f) || sm_scale > 3.0e38f) return SAGE2_ERR_INVALID_ARG;
  s = check_ptrs(q, k, v, o);
  if (s != SAGE2_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return SAGE2_ERR_CUDA;
  cudaMemPool_t pool = device_pool(dev);
  if (!pool) return SAGE2_ERR_CUDA;
  const Workspace w = layout(g, packed_of(qk_format));
  uint8_t* ws = nullptr;
  e = cudaMallocFromPoolAsync(reinterpret_cast<void**>(&ws), w.total, pool, st);
  if (e != cudaSuccess) return from_cuda(e);

  {
    std::unique_lock<std::mutex> lock;
    SideLane* side = side_lane(dev, &lock);
    e = forward(q, k, v, o, g, dtype, o_dtype, causal, sm_scale, qk_format, smooth_v,
                static_cast<int64_t>(N), static_cast<int64_t>(N), ws, st, side);
  }
  const cudaError_t e2 = cudaFreeAsync(ws, st);
  return from_cuda(e != cudaSuccess ? e : e2);
}

sage2_status sage2_attn_fwd(const void* q, const void* k, const void* v, void* o, int B, int H,
                            int N, int d, int dtype, int o_dtype, int causal, float sm_scale,
                            sage2_stream_t stream) {
  return sage2_attn_fwd_ex(q, k, v, o, B, H, N, d, dtype, o_dtype, causal, sm_scale,
                           SAGE2_QK_INT4, 0, stream);
}

sage2_status sage2_debug_qk_s32_ex(const uint8_t* q_i4, const uint8_t* k_i4, int B, int H, int N,
                                   int d, int qk_format, int32_t* s_out, sage2_stream_t stream) {
  if (!valid_qk_format(qk_format) || packed_of(qk_format)) return SAGE2_ERR_INVALID_ARG;
  Dims g;
  sage2_status s = check_dims(B, H, N, d, &g);
  if (s != SAGE2_OK) return s;
  if (g.BH * (int64_t)g.NB * g.NB > (int64_t)INT32_MAX) return SAGE2_ERR_UNSUPPORTED;
  if (g.BH > 65535) return SAGE2_ERR_UNSUPPORTED;
  s = check_ptrs(q_i4, k_i4, s_out);
  if (s != SAGE2_OK) return s;
  return from_cuda(launch_debug_qk(q_i4, k_i4, B, H, g.Np, d, qk_bits_of(qk_format), s_out,
                                   reinterpret_cast<cudaStream_t>(stream)));
}

sage2_status sage2_debug_qk_s32(const uint8_t* q_i4, const uint8_t* k_i4, int B, int H, int N,
                                int d, int32_t* s_out, sage2_stream_t stream) {
  return sage2_debug_qk_s32_ex(q_i4, k_i4, B, H, N, d, SAGE2_QK_INT4, s_out, stream);
}

sage2_status sage2_debug_wait_timeout(sage2_stream_t stream) {
  return from_cuda(launch_debug_wait_timeout(reinterpret_cast<cudaStream_t>(stream)));
}

sage2_status sage2_check_device_error(sage2_stream_t stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return SAGE2_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpyFromSymbol(&word, g_device_error, sizeof(word)) != cudaSuccess)
    return SAGE2_ERR_CUDA;
  if (word != 0) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess)
      return SAGE2_ERR_CUDA;
  }
  if (word & DEVERR_TIMEOUT) return SAGE2_ERR_TIMEOUT;
  if (word) return SAGE2_ERR_CUDA;
  return SAGE2_OK;
}

const char* sage2_status_string(sage2_status status) {
  switch (status) {
    case SAGE2_OK: return "ok";
    case SAGE2_ERR_INVALID_ARG: return "invalid argument";
    case SAGE2_ERR_UNSUPPORTED: return "unsupported size or head dimension";
    case SAGE2_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case SAGE2_ERR_CUDA: return "CUDA error";
    case SAGE2_ERR_NO_MEM: return "out of device memory";
    case SAGE2_ERR_TIMEOUT: return "device wait timed out";
    case SAGE2_ERR_TOO_LARGE: return "scratch needed exceeds the fixed no-allocation buffer";
  }
  return "unknown status";
}

int sage2_version(void) { return 100; }

sage2_status sage2_layout_info(sage2_layout* out) {
  if (!out) return SAGE2_ERR_INVALID_ARG;
  out->version = sage2_version();
  out->block_rows = kTile;
  out->tile_keys = kTile;
  out->int4_max = 7;
  out->int8_max = 127;
  out->p_scale = 448.f;
  out->v_scale_div = 448.f;
  out->packed_low_first = 1;
  for (int j = 0; j < kTile; ++j) {
    // the quantizer stores token j of a block at row 8*((j/2)%16) + 2*(j/32) + j%2
    out->key_perm[8 * ((j >> 1) & 15) + 2 * (j >> 5) + (j & 1)] = j;
    // V^T byte p holds token sigma(p), sigma swapping the 2-bit fields [6:5] and [4:3]
    out->value_perm[j] = 32 * ((j >> 3) & 3) + 8 * ((j >> 5) & 3) + (j & 7);
  }
  return SAGE2_OK;
}

}  // extern "C"
