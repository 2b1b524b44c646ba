// Smoothing and quantization kernels (HBM-bound passes).
//
//  k_mean_partial                   : K smoothing - token mean of K per channel.
//  k_smooth_quant                   : Q smoothing (mean of each 128-row block) and
//                                     K smoothing applied, then INT4 per token.
//  (the correction qbar_blk . K_j added back to the INT4 product is in corr.cu)
//  k_v_amax / k_v_quant             : FP8 e4m3 V with one scale per channel,
//                                     written transposed (token-contiguous).
//
// Method: "SageAttention2: Efficient Attention with Thorough Outlier Smoothing
// and Per-thread INT4 Quantization" (arxiv.science abstract page, Abstract):
// INT4 (Q,K), FP8 V, smoothing of Q; K smoothing from the title's "outlier
// smoothing".  Variants: INT8 (Q,K) on [-127, 127] (the predecessor,
// "SageAttention: Accurate 8-Bit Attention", ainnect summary) and V smoothing
// (token mean of V subtracted before FP8, "smooth V" in the SageAttention2
// summary, ainnect.com/research/55).  Every rounding below is spelled with an explicit IEEE intrinsic
// (__fadd_rn, __fmul_rn, ...) so that no contraction or reassociation changes
// the payload bits: the summation orders are part of the specification.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "sage2_internal.h"
#include "sm100_ptx.cuh"

namespace sage2 {

template <typename T>
__device__ __forceinline__ void unpack8(const uint4& u, float (&x)[8]);
template <>
__device__ __forceinline__ void unpack8<__half>(const uint4& u, float (&x)[8]) {
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __half22float2(h[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}
template <>
__device__ __forceinline__ void unpack8<__nv_bfloat16>(const uint4& u, float (&x)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ float to_f32(__half v) { return __half2float(v); }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

// ---------------------------------------------------------------------------
// K mean: one worker (D/8 threads, 8 channels each) per 128-token chunk sums
// its chunk token by token in ascending order (fp32) into part[bh][chunk].
// The last block of a head to finish (a per-head counter) then adds the chunk
// sums in chunk order and divides once by N (fp32), and resets the counter.
// grid (ceil(nchunks / workers_per_block), B*H), 256 threads; done[] starts at 0.
template <typename T, int D>
__global__ void __launch_bounds__(256) k_mean_partial(const T* __restrict__ k, int N,
                                                      long long ldh, int nchunks,
                                                      float* __restrict__ part,
                                                      unsigned* __restrict__ done,
                                                      float* __restrict__ kmean) {
  constexpr int TPR = D / 8;
  constexpr int WPB = 256 / TPR;
  const int bh = blockIdx.y;
  const int worker = threadIdx.x / TPR, q8 = threadIdx.x % TPR;
  const int chunk = blockIdx.x * WPB + worker;
  if (chunk < nchunks) {
    const int t0 = chunk * 128;
    const int nt = min(128, N - t0);
    const uint4* src = reinterpret_cast<const uint4*>(k + ((size_t)bh * ldh + t0) * D) + q8;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    int t = 0;
    for (; t + 8 <= nt; t += 8) {
      uint4 u[8];
#pragma unroll
      for (int s = 0; s < 8; ++s) u[s] = __ldg(src + (size_t)(t + s) * TPR);
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        float x[8];
        unpack8<T>(u[s], x);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], x[i]);
      }
    }
    for (; t < nt; ++t) {
      float x[8];
      unpack8<T>(__ldg(src + (size_t)t * TPR), x);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], x[i]);
    }
    float4* dst = reinterpret_cast<float4*>(part + ((size_t)bh * nchunks + chunk) * D + q8 * 8);
    dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
  // the head's last block adds the chunk sums in chunk order
  __shared__ bool last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(&done[bh], 1u) == gridDim.x - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  for (int c = threadIdx.x; c < D; c += 256) {
    const float* p = part + (size_t)bh * nchunks * D + c;
    float total = 0.f;
    for (int ch = 0; ch < nchunks; ++ch) total = __fadd_rn(total, __ldcg(p + (size_t)ch * D));
    kmean[(size_t)bh * D + c] = __fdiv_rn(total, (float)N);
  }
  if (threadIdx.x == 0) done[bh] = 0u;
}

// ---------------------------------------------------------------------------
// Smoothing + INT4.  grid (NB, B*H, nz): z + zbase = 0 quantizes the Q block
// (after computing its mean), 1 the K block (after subtracting kbar).  256 threads.
// FMT: 0 INT4 values as e4m3 codes, 1 INT8 values (the variant), 2 INT4 values
// packed two per byte (two's-complement nibbles, channel 2c in bits 3:0).
// Two lanes own one row (16 rows per warp), each half of its channels, so a
// row's amax needs one shuffle and its scale none.  In shared memory row r
// starts at byte RS*r and its second half at +HO (RS = 2D+32, HO = D+16): the
// 16-byte chunks that the eight lanes of one access phase read then fall in
// eight different bank groups.
template <typename T, int D, int FMT>
__global__ void __launch_bounds__(256) k_smooth_quant(
    const T* __restrict__ q, const T* __restrict__ k, int N, long long ldh, int Np, int NB,
    const float* __restrict__ kmean, uint8_t* __restrict__ q_i4, float* __restrict__ q_scale,
    float* __restrict__ q_mean, uint8_t* __restrict__ k_i4, float* __restrict__ k_scale,
    int zbase) {
  constexpr int RS = 2 * D + 32, HO = D + 16;     // bytes
  constexpr int CPR = D / 8, CPH = CPR / 2;       // 16-byte chunks per row / per half
  constexpr int MH = D / 2 + 4;                   // floats between the two halves of mean
  __shared__ __align__(16) uint8_t tile[128 * RS];
  __shared__ __align__(16) float mean[2 * MH];
  const int blk = blockIdx.x, bh = blockIdx.y;
  const bool is_q = blockIdx.z + zbase == 0;
  const T* src = is_q ? q : k;
  const int r0 = blk * 128;
  const int nvalid = min(128, N - r0);

  // coalesced 16-byte asynchronous copies of the valid rows, all in flight at once
  const uint4* g = reinterpret_cast<const uint4*>(src + ((size_t)bh * ldh + r0) * D);
  constexpr int kPer = 128 * CPR / 256;            // copies per thread for a full block
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int i = threadIdx.x + 256 * u;
    const int r = i / CPR, j = i % CPR;
    if (r < nvalid) cp_async16(tile + RS * r + (j < CPH ? 16 * j : HO + 16 * (j - CPH)), g + i);
  }
  cp_async_wait_all();

  __syncthreads();
  if (is_q) {
    if (threadIdx.x < D) {
      const int c = threadIdx.x;
      const int off = c < D / 2 ? 2 * c : HO + 2 * (c - D / 2);
      float acc = 0.f;
      for (int r = 0; r < nvalid; ++r)
        acc = __fadd_rn(acc, to_f32(*reinterpret_cast<const T*>(tile + RS * r + off)));
      const float m = __fdiv_rn(acc, (float)nvalid);
      mean[c < D / 2 ? c : MH + c - D / 2] = m;
      q_mean[((size_t)bh * NB + blk) * D + c] = m;
    }
  } else {
    if (threadIdx.x < D) {
      const int c = threadIdx.x;
      mean[c < D / 2 ? c : MH + c - D / 2] = kmean[(size_t)bh * D + c];
    }
  }
  __syncthreads();

  constexpr bool Q8 = FMT == 1;
  constexpr int RB = FMT == 2 ? D / 2 : D;        // payload bytes per row
  uint8_t* out = (is_q ? q_i4 : k_i4) + ((size_t)bh * Np + r0) * RB;
  float* scale = (is_q ? q_scale : k_scale) + (size_t)bh * Np + r0;
  constexpr float kQmax = Q8 ? 127.f : 7.f;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = warp * 16 + (lane >> 1), hh = lane & 1;
  const uint8_t* trow = tile + RS * r + HO * hh;
  const float* mu = mean + MH * hh;
  const bool valid = r < nvalid;
  // eight smoothed values x - mean (fp32, RN) of chunk i of this lane's half
  auto load8 = [&](int i, float (&x)[8]) {
    unpack8<T>(*reinterpret_cast<const uint4*>(trow + 16 * i), x);
    const float4 m0 = *reinterpret_cast<const float4*>(mu + 8 * i);
    const float4 m1 = *reinterpret_cast<const float4*>(mu + 8 * i + 4);
    const float2 d0 = __fadd2_rn(make_float2(x[0], x[1]), make_float2(-m0.x, -m0.y));
    const float2 d1 = __fadd2_rn(make_float2(x[2], x[3]), make_float2(-m0.z, -m0.w));
    const float2 d2 = __fadd2_rn(make_float2(x[4], x[5]), make_float2(-m1.x, -m1.y));
    const float2 d3 = __fadd2_rn(make_float2(x[6], x[7]), make_float2(-m1.z, -m1.w));
    x[0] = d0.x; x[1] = d0.y; x[2] = d1.x; x[3] = d1.y;
    x[4] = d2.x; x[5] = d2.y; x[6] = d3.x; x[7] = d3.y;
  };
  // Pass 1: the row's amax (rows >= N are all zero)
  float amax = 0.f;
  if (valid) {
#pragma unroll
    for (int i = 0; i < CPH; ++i) {
      float x[8];
      load8(i, x);
#pragma unroll
      for (int u = 0; u < 8; ++u) amax = fmaxf(amax, fabsf(x[u]));
    }
  }
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  const bool nz = amax > 0.f;                           // the scale may underflow to 0
  const float sc = nz ? __fdiv_rn(amax, kQmax) : 0.f;
  const float inv = nz ? __fdiv_rn(kQmax, amax) : 0.f;
  const float2 inv2 = make_float2(inv, inv);
  // K^ rows are stored permuted inside each 128-row block: token j of the block
  // goes to stored row 8*((j/2) % 16) + 2*(j/32) + j % 2, so that stored row n
  // holds token 32*((n/2) % 4) + 2*(n/8) + n % 2 (the attention kernel's
  // .16x256b TMEM loads then give each thread 32 consecutive keys).  Q^ rows
  // keep their natural order.
  const int srow = is_q ? r : 8 * ((r >> 1) & 15) + 2 * (r >> 5) + (r & 1);
  uint8_t* orow = out + (size_t)srow * RB + (RB / 2) * hh;
  // Pass 2: quantize.  |x| <= amax and inv = RN(qmax/amax), so |x*inv| <=
  // qmax*(1+2^-24)^2 < qmax + 1/2: the rounded value never leaves [-qmax,
  // qmax] and needs no clamp.  Adding +0 turns a rounded -0 into +0 (the
  // oracle's integer 0).
  // INT4 (the method): each value in [-7, 7] is stored as its e4m3 code:
  // every such integer is exact in e4m3, so the FP8 tensor path multiplies
  // the INT4 values exactly (at the same rate as the 8-bit integer path) and
  // yields S as an fp32 integer.  Zero is stored as +0 (code 0x00).
  // INT8 (the variant): values in [-127, 127] as two's-complement bytes.
  if (FMT == 2) {
    // two values per byte: 16 channels of this lane's half -> 8 bytes
#pragma unroll
    for (int i = 0; i < CPH; i += 2) {
      uint32_t w[2] = {0u, 0u};
      if (nz) {
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          float x[8];
          load8(i + c2, x);
#pragma unroll
          for (int u = 0; u < 8; u += 2) {
            const float2 p = __fmul2_rn(make_float2(x[u], x[u + 1]), inv2);
            const uint32_t n0 = static_cast<uint32_t>(static_cast<int>(rintf(p.x))) & 0xFu;
            const uint32_t n1 = static_cast<uint32_t>(static_cast<int>(rintf(p.y))) & 0xFu;
            w[c2] |= (n0 | (n1 << 4)) << (4 * u);
          }
        }
      }
      *reinterpret_cast<uint2*>(orow + 4 * i) = make_uint2(w[0], w[1]);
    }
    if (hh == 0) scale[r] = sc;
    return;
  }
#pragma unroll
  for (int i = 0; i < CPH; i += 2) {
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if (nz) {
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        float x[8];
        load8(i + c2, x);
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; u += 2) {
          const float2 p = __fmul2_rn(make_float2(x[u], x[u + 1]), inv2);
          v[u] = __fadd_rn(rintf(p.x), 0.f);
          v[u + 1] = __fadd_rn(rintf(p.y), 0.f);
        }
#pragma unroll
        for (int h4 = 0; h4 < 2; ++h4) {
          uint32_t packed = 0;
          if (Q8) {
#pragma unroll
            for (int u = 0; u < 4; ++u)
              packed |= (static_cast<uint32_t>(static_cast<int>(v[4 * h4 + u])) & 0xFFu) << (8 * u);
          } else {
#pragma unroll
            for (int u = 0; u < 4; u += 2)
              packed |= static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(
                            make_float2(v[4 * h4 + u], v[4 * h4 + u + 1]), __NV_SATFINITE, __NV_E4M3))
                        << (8 * u);
          }
          w[2 * c2 + h4] = packed;
        }
      }
    }
    *reinterpret_cast<uint4*>(orow + 8 * i) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (hh == 0) scale[r] = sc;
}

// ---------------------------------------------------------------------------
// V, pass 1: per-channel amax over all tokens.  grid (nchunks, B*H), 256
// threads; one 128-token chunk per block; float bits of |x| >= 0 are ordered
// like unsigned integers, so atomicMax on the bits is exact.
template <typename T, int D>
__global__ void __launch_bounds__(256) k_v_amax(const T* __restrict__ v, int N, long long ldh,
                                                const float* __restrict__ vmean,
                                                uint32_t* __restrict__ amax_bits) {
  constexpr int TPR = D / 8;
  constexpr int RPB = 256 / TPR;  // rows handled at once by the block
  __shared__ float red[RPB][D];
  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int r = threadIdx.x / TPR, q8 = threadIdx.x % TPR;
  const int t0 = chunk * 128;
  const int nt = min(128, N - t0);
  float m[8], mu[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    m[i] = 0.f;
    mu[i] = vmean ? vmean[(size_t)bh * D + q8 * 8 + i] : 0.f;   // V smoothing: |V - vbar|
  }
  const uint4* src = reinterpret_cast<const uint4*>(v + ((size_t)bh * ldh + t0) * D) + q8;
  for (int t = r; t < nt; t += RPB) {
    float x[8];
    unpack8<T>(__ldg(src + (size_t)t * TPR), x);
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = fmaxf(m[i], fabsf(__fsub_rn(x[i], mu[i])));
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) red[r][q8 * 8 + i] = m[i];
  __syncthreads();
  if (threadIdx.x < D) {
    float a = 0.f;
    for (int rr = 0; rr < RPB; ++rr) a = fmaxf(a, red[rr][threadIdx.x]);
    atomicMax(&amax_bits[(size_t)bh * D + threadIdx.x], __float_as_uint(a));
  }
}

// V, pass 2: codes = e4m3_rn_satfinite(V * (448/amax_c)), stored transposed
// with the tokens of each 128-token block permuted: byte p of a channel's
// block holds token sigma(p), sigma swapping the 2-bit fields [6:5] and [4:3]
// of the index (an involution).  That is the key order in which the
// attention kernel lays P~ out in tensor memory.
// grid (Np/128, B*H), 256 threads.  A warp owns one 16-byte output group and
// 32 consecutive channels, so its shared-memory reads are conflict-free.
template <typename T, int D>
__global__ void __launch_bounds__(256) k_v_quant(const T* __restrict__ v, int N, long long ldh, int Np,
                                                 const float* __restrict__ vmean,
                                                 const uint32_t* __restrict__ amax_bits,
                                                 uint8_t* __restrict__ vt,
                                                 float* __restrict__ v_scale) {
  __shared__ __align__(16) T tile[128][D];
  __shared__ float inv[D], mu[D];
  const int kt = blockIdx.x, bh = blockIdx.y;
  const int t0 = kt * 128;
  const int nvalid = max(0, min(128, N - t0));
  constexpr int VPR = D / 8;
  const uint4* g = reinterpret_cast<const uint4*>(v + ((size_t)bh * ldh + t0) * D);
  uint4* s = reinterpret_cast<uint4*>(&tile[0][0]);
  // asynchronous 16-byte copies, all of a thread's in flight at once
#pragma unroll
  for (int u = 0; u < 128 * VPR / 256; ++u) {
    const int i = threadIdx.x + 256 * u;
    if (i < nvalid * VPR) cp_async16(s + i, g + i);
  }
  cp_async_wait_all();
  if (threadIdx.x < D) {
    const float a = __uint_as_float(amax_bits[(size_t)bh * D + threadIdx.x]);
    inv[threadIdx.x] = a > 0.f ? __fdiv_rn(448.f, a) : 0.f;
    mu[threadIdx.x] = vmean ? vmean[(size_t)bh * D + threadIdx.x] : 0.f;
    if (kt == 0) v_scale[(size_t)bh * D + threadIdx.x] = a > 0.f ? __fdiv_rn(a, 448.f) : 0.f;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // work items: (channel group of 32, 16-byte output group): (D/32) * 8 items, 8 warps
  for (int item = warp; item < (D / 32) * 8; item += 8) {
    const int c = (item / 8) * 32 + lane;
    const int og = item % 8;
    const float sc = inv[c], m0 = mu[c];
    uint32_t w[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      uint32_t word = 0;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // bytes 16og + i, i = 4p + 2h + {0,1}: tokens sigma(16og + i), consecutive pairs
        const int i = p * 4 + h * 2;
        const int r = 32 * (((og & 1) << 1) | (i >> 3)) + 8 * (og >> 1) + (i & 7);
        const float x0 = (r < nvalid) ? __fmul_rn(__fsub_rn(to_f32(tile[r][c]), m0), sc) : 0.f;
        const float x1 = (r + 1 < nvalid) ? __fmul_rn(__fsub_rn(to_f32(tile[r + 1][c]), m0), sc) : 0.f;
        const __nv_fp8x2_storage_t two =
            __nv_cvt_float2_to_fp8x2(make_float2(x0, x1), __NV_SATFINITE, __NV_E4M3);
        word |= static_cast<uint32_t>(two) << (16 * h);
      }
      w[p] = word;
    }
    *reinterpret_cast<uint4*>(vt + ((size_t)bh * D + c) * Np + t0 + og * 16) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// ---------------------------------------------------------------------------
// Packed INT4 -> e4m3 codes, for the tensor path (B200 multiplies no INT4
// operands; the INT4 values travel as e4m3 codes, exact for [-7, 7]).  A
// 256-entry table maps a packed byte to its two codes, built from the same
// conversion the quantizer uses.  Each thread expands 8 bytes into 16 codes.
__global__ void __launch_bounds__(256) k_unpack_int4(const uint2* __restrict__ pk,
                                                     uint4* __restrict__ codes, size_t n8) {
  __shared__ uint32_t lut[256];
  {
    const int b = threadIdx.x;
    const int lo = (b & 0xF) - ((b & 0x8) << 1);
    const int hi = ((b >> 4) & 0xF) - ((b & 0x80) >> 3);
    const uint32_t clo = __nv_cvt_float_to_fp8(static_cast<float>(lo), __NV_SATFINITE, __NV_E4M3);
    const uint32_t chi = __nv_cvt_float_to_fp8(static_cast<float>(hi), __NV_SATFINITE, __NV_E4M3);
    lut[b] = clo | (chi << 8);
  }
  __syncthreads();
  for (size_t i = static_cast<size_t>(blockIdx.x) * 256 + threadIdx.x; i < n8;
       i += static_cast<size_t>(gridDim.x) * 256) {
    const uint2 w = __ldg(pk + i);
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t src = j < 2 ? w.x : w.y;
      const int sh = (j & 1) * 16;
      o[j] = lut[(src >> sh) & 0xFFu] | (lut[(src >> (sh + 8)) & 0xFFu] << 16);
    }
    codes[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

cudaError_t launch_unpack_int4(const uint8_t* packed, uint8_t* codes, size_t bytes, cudaStream_t st) {
  const size_t n8 = bytes / 8;
  if (n8 == 0) return cudaSuccess;
  const size_t want = (n8 + 255) / 256;
  const unsigned grid = static_cast<unsigned>(want < 148 * 16 ? want : 148 * 16);
  k_unpack_int4<<<grid, 256, 0, st>>>(reinterpret_cast<const uint2*>(packed),
                                      reinterpret_cast<uint4*>(codes), n8);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Host-side launchers (called by the C ABI after validation).
template <typename T, int D>
cudaError_t launch_qk_corr_t(const QKArgs& a, cudaStream_t st);  // corr.cu

template <typename T, int D, int FMT>
static void launch_smooth_t(const QKArgs& a, int zbase, int nz, cudaStream_t st) {
  k_smooth_quant<T, D, FMT><<<dim3(a.NB, a.B * a.H, nz), 256, 0, st>>>(
      static_cast<const T*>(a.q), static_cast<const T*>(a.k), a.N, a.ldh, a.Np, a.NB, a.k_mean,
      a.q_i4, a.q_scale, a.q_mean, a.k_i4, a.k_scale, zbase);
}

template <typename T, int D>
static void launch_smooth(const QKArgs& a, int zbase, int nz, cudaStream_t st) {
  if (a.qk_bits == 8) launch_smooth_t<T, D, 1>(a, zbase, nz, st);
  else if (a.packed) launch_smooth_t<T, D, 2>(a, zbase, nz, st);
  else launch_smooth_t<T, D, 0>(a, zbase, nz, st);
}

// Two independent chains: K (mean, then smoothing + INT4 of K) and Q
// (smoothing + INT4 of Q with its block means, then the split of the means
// and the correction).  With a.side they run concurrently: the Q chain on
// the library stream, forked from and joined back into `st`.
template <typename T, int D>
static cudaError_t launch_qk_t(const QKArgs& a, cudaStream_t st) {
  const int BH = a.B * a.H;
  const int nchunks = a.NB;
  constexpr int WPB = 256 / (D / 8);
  cudaError_t e = cudaMemsetAsync(a.done, 0, sizeof(unsigned) * BH, st);
  if (e != cudaSuccess) return e;
  cudaStream_t qs = st;
  if (a.side) {
    e = cudaEventRecord(a.fork, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(a.side, a.fork, 0);
    if (e != cudaSuccess) return e;
    qs = a.side;
  }
  // K chain
  k_mean_partial<T, D><<<dim3((nchunks + WPB - 1) / WPB, BH), 256, 0, st>>>(
      static_cast<const T*>(a.k), a.N, a.ldh, nchunks, a.mean_part, a.done, a.k_mean);
  if (a.side) {
    launch_smooth<T, D>(a, 1, 1, st);            // K blocks
    launch_smooth<T, D>(a, 0, 1, qs);            // Q blocks
  } else {
    launch_smooth<T, D>(a, 0, 2, st);            // Q and K blocks in one launch
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // Q chain: the correction needs the block means of Q
  e = launch_qk_corr_t<T, D>(a, qs);
  if (e != cudaSuccess) return e;
  if (a.side && a.join) {                         // (a caller may join later itself)
    e = cudaEventRecord(a.join, a.side);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, a.join, 0);
  }
  return e;
}

cudaError_t launch_smooth_quant_qk(const QKArgs& a, cudaStream_t st) {
  if (a.dtype == 0) return a.d == 64 ? launch_qk_t<__half, 64>(a, st) : launch_qk_t<__half, 128>(a, st);
  return a.d == 64 ? launch_qk_t<__nv_bfloat16, 64>(a, st) : launch_qk_t<__nv_bfloat16, 128>(a, st);
}

template <typename T, int D>
static cudaError_t launch_v_t(const VArgs& a, cudaStream_t st) {
  const int BH = a.B * a.H;
  cudaError_t e = cudaMemsetAsync(a.amax_bits, 0, sizeof(uint32_t) * BH * D, st);
  if (e != cudaSuccess) return e;
  if (a.v_mean) {
    // V smoothing: the per-channel token mean, with the fixed order of the K mean
    e = cudaMemsetAsync(a.done, 0, sizeof(unsigned) * BH, st);
    if (e != cudaSuccess) return e;
    constexpr int WPB = 256 / (D / 8);
    k_mean_partial<T, D><<<dim3((a.NB + WPB - 1) / WPB, BH), 256, 0, st>>>(
        static_cast<const T*>(a.v), a.N, a.ldh, a.NB, a.mean_part, a.done, a.v_mean);
  }
  k_v_amax<T, D><<<dim3(a.NB, BH), 256, 0, st>>>(static_cast<const T*>(a.v), a.N, a.ldh, a.v_mean,
                                                 a.amax_bits);
  k_v_quant<T, D><<<dim3(a.NB, BH), 256, 0, st>>>(static_cast<const T*>(a.v), a.N, a.ldh, a.Np,
                                                  a.v_mean, a.amax_bits, a.v_fp8_t, a.v_scale);
  return cudaGetLastError();
}

cudaError_t launch_quant_v(const VArgs& a, cudaStream_t st) {
  if (a.dtype == 0) return a.d == 64 ? launch_v_t<__half, 64>(a, st) : launch_v_t<__half, 128>(a, st);
  return a.d == 64 ? launch_v_t<__nv_bfloat16, 64>(a, st) : launch_v_t<__nv_bfloat16, 128>(a, st);
}

}  // namespace sage2
