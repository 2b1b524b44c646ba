// Internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace sage2 {

constexpr int kTile = 128;  // BM = BN = 128: Q rows per block, keys per tile

struct QKArgs {
  const void* q;
  const void* k;
  int dtype;  // 0 fp16, 1 bf16
  int B, H, N, d, Np, NB;
  uint8_t* q_i4;
  float* q_scale;
  float* q_mean;
  uint8_t* k_i4;
  float* k_scale;
  float* k_mean;
  float* qk_corr;
  float* mean_part;        // scratch [B*H, NB, d]
  void* qbar_split;        // scratch [3][B*H][NBc*128][d] in the input dtype (NBc = ceil(NB/128))
  int skip_masked_corr;    // 1: skip correction blocks a causal mask hides
  int qk_bits;             // 4: INT4 values as e4m3 codes; 8: INT8 values (two's complement)
  int64_t ldh;             // tokens between consecutive heads of q and k (N when contiguous)
  int packed;              // 1 (with qk_bits 4): q_i4/k_i4 hold two INT4 nibbles per byte
  unsigned* done;          // scratch [B*H]: per-head count of finished K-mean blocks
  cudaStream_t side;       // non-null: run the Q chain (Q smoothing, q-mean split,
                           // correction) on this library stream, concurrently with
                           // the K chain (K mean, K smoothing) on the caller's stream
  cudaEvent_t fork, join;  // events of that fork / join (with `side`)
};

struct VArgs {
  const void* v;
  int dtype;
  int B, H, N, d, Np, NB;
  uint8_t* v_fp8_t;
  float* v_scale;
  uint32_t* amax_bits;     // scratch [B*H, d]
  float* v_mean;           // nullptr: no V smoothing; else the per-channel token mean [B*H, d]
  float* mean_part;        // scratch [B*H, NB, d] for the V mean (when v_mean is set)
  int64_t ldh;             // tokens between consecutive heads of v (N when contiguous)
  unsigned* done;          // scratch [B*H] for the V mean (when v_mean is set)
};

struct AttnArgs {
  const uint8_t* q_i4;
  const float* q_scale;
  const uint8_t* k_i4;
  const float* k_scale;
  const float* qk_corr;
  const uint8_t* v_fp8_t;
  const float* v_scale;
  void* o;
  int o_dtype;  // 0 fp16, 1 bf16, 2 fp32
  int B, H, N, d, Np, NB;
  int causal;
  float sm_scale;
  int qk_bits;             // 4 or 8 (payload format, see QKArgs)
  const float* v_mean;     // nullptr: V was not smoothed
  int64_t ldo;             // tokens between consecutive heads of o (N when contiguous)
};

cudaError_t launch_smooth_quant_qk(const QKArgs& a, cudaStream_t st);
cudaError_t launch_quant_v(const VArgs& a, cudaStream_t st);
cudaError_t launch_attn(const AttnArgs& a, cudaStream_t st);
cudaError_t launch_debug_wait_timeout(cudaStream_t st);
// Packed INT4 (two two's-complement nibbles per byte, channel 2c in bits 3:0)
// -> one e4m3 code per value; `bytes` packed bytes, a multiple of 8.
cudaError_t launch_unpack_int4(const uint8_t* packed, uint8_t* codes, size_t bytes, cudaStream_t st);
cudaError_t launch_debug_qk(const uint8_t* q_i4, const uint8_t* k_i4, int B, int H, int Np, int d,
                            int qk_bits, int32_t* s_out, cudaStream_t st);

// General tiled tensor map: `rank` dims (innermost first, in elements), the
// byte strides of dims 1..rank-1, the box (elements), element size 1/2/4 B and
// a swizzle of 0, 64 or 128 bytes.  Out-of-range box elements read as zero.
cudaError_t make_tmap(void* tmap_out, const void* base, int rank, const uint64_t* dims,
                      const uint64_t* strides_bytes, const uint32_t* box, int elem_bytes,
                      int swizzle_bytes);

// Tensor-map creation through the driver entry point (no link-time libcuda).
// Encodes a 2-D row-major uint8 tensor [rows, cols] with a box of
// [box_rows, box_cols] and 128- or 64-byte swizzle (box_cols bytes).
cudaError_t make_tmap_u8_2d(void* tmap_out, const void* base, uint64_t rows, uint64_t cols,
                            uint32_t box_rows, uint32_t box_cols);

}  // namespace sage2
