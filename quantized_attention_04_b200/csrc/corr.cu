// Q-smoothing correction on the tensor cores:  C[blk][j] = qbar_blk . K_j.
//
// "SageAttention2: Efficient Attention with Thorough Outlier Smoothing and
// Per-thread INT4 Quantization" (arxiv.science abstract page, Abstract): Q is
// smoothed to make the INT4 QK^T accurate; what the block mean removed from
// the scores is added back in floating point.  Computed with the raw K (the
// difference to the smoothed K is qbar.kbar, constant along a row).
//
// C is a [NB x N] GEMM per head with K = d.  Each fp32 qbar is split into
// three terms of the input's 16-bit type (qbar = t0 + t1 + t2 up to ~2^-24
// relative), K is exact in that type, and the three products are accumulated
// in one fp32 TMEM accumulator by tcgen05 kind::f16:
//   D[blk][key] = sum_term sum_c t_term[blk][c] * K[key][c]
// with blocks on the M side (128 per chunk) and 128 keys on the N side.
//
// k_qbar_split : qbar -> three 16-bit terms, [3][B*H][NBc*128][d] (pad rows 0).
// k_qk_corr_tc : persistent, one CTA per SM over a contiguous run of work items
//   (head, 128-block chunk, key tile), in that order.
//   warp 0 TMA (a chunk's three term tiles once per run of its items, then
//   K tiles, 2 stages),
//   warp 1 MMA issuer, warp 2 TMEM allocator, warps 4-7 epilogue: a warp owns
//   32 block rows; per tile it stages four 32 x 32 fp32 boxes in shared memory
//   (128-byte swizzle, conflict-free) and writes each with a TMA tensor store,
//   so C leaves in full lines (one thread per row writing its own row would
//   scatter every warp store over 32 rows).  TMA zero-fills keys >= N on the
//   load side, so their C is 0; the store clips block rows >= NB.
#include <cuda.h>
#include <cuda_bf16.h>
#include <algorithm>
#include <climits>
#include <cstdint>
#include <cuda_fp16.h>

#include "sage2_internal.h"
#include "sm100_ptx.cuh"

namespace sage2 {

template <typename T>
struct IsBf16 {
  static constexpr bool value = false;
};
template <>
struct IsBf16<__nv_bfloat16> {
  static constexpr bool value = true;
};

template <typename T>
__device__ __forceinline__ T to_t(float x);
template <>
__device__ __forceinline__ __half to_t<__half>(float x) { return __float2half_rn(x); }
template <>
__device__ __forceinline__ __nv_bfloat16 to_t<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}
__device__ __forceinline__ float from_t(__half x) { return __half2float(x); }
__device__ __forceinline__ float from_t(__nv_bfloat16 x) { return __bfloat162float(x); }

// grid (NBc*128, B*H), d threads.  The residuals are exact in fp32: each term
// removes the leading bits the 16-bit type can hold.
template <typename T>
__global__ void k_qbar_split(const float* __restrict__ q_mean, int NB, int NBc, int d, int BH,
                             T* __restrict__ terms) {
  const int blk = blockIdx.x, bh = blockIdx.y, c = threadIdx.x;
  const float v = blk < NB ? q_mean[(static_cast<size_t>(bh) * NB + blk) * d + c] : 0.f;
  const T t0 = to_t<T>(v);
  const float r0 = __fsub_rn(v, from_t(t0));
  const T t1 = to_t<T>(r0);
  const float r1 = __fsub_rn(r0, from_t(t1));
  const T t2 = to_t<T>(r1);
  const size_t plane = static_cast<size_t>(BH) * NBc * 128 * d;
  const size_t at = (static_cast<size_t>(bh) * NBc * 128 + blk) * d + c;
  terms[at] = t0;
  terms[plane + at] = t1;
  terms[2 * plane + at] = t2;
}

template <int D>
struct __align__(1024) CorrSmem {
  uint8_t a[3][D / 64][128 * 128];   // term x 128-byte atom x (128 rows x 128 B)
  uint8_t b[2][D / 64][128 * 128];   // stage x atom: 128 keys x 64 channels
  uint8_t out[4][2][32 * 128];       // epilogue warp x buffer: 32 rows x 32 fp32 (swizzled)
  uint64_t a_full, a_empty;
  uint64_t b_full[2], b_empty[2];
  uint64_t d_full[2], d_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

// Work item i (0 <= i < total) of a grid-wide list ordered by head, then
// 128-block chunk, then key tile: the chunk's key tiles are 0 .. kt_end-1,
// kt_end = NB, or with the causal skip the tiles up to the chunk's last block.
struct CorrItem {
  int bh, chunk, kt;
};
__device__ __forceinline__ int corr_tiles_of_chunk(int chunk, int NB, int skip_masked) {
  return skip_masked ? min(NB, (chunk + 1) * 128) : NB;
}
__device__ __forceinline__ CorrItem corr_item(int i, int NB, int NBc, int per_head, int skip_masked) {
  CorrItem it;
  it.bh = i / per_head;
  int r = i - it.bh * per_head;
  int c = 0;
  while (c + 1 < NBc && r >= corr_tiles_of_chunk(c, NB, skip_masked)) {
    r -= corr_tiles_of_chunk(c, NB, skip_masked);
    ++c;
  }
  it.chunk = c;
  it.kt = r;
  return it;
}

// Persistent: CTA c takes items [c*total/G, (c+1)*total/G); the three term
// tiles of a (head, chunk) are loaded once per run of its items.
template <typename T, int D>
__global__ void __launch_bounds__(256, 1)
    k_qk_corr_tc(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_c, int N, int Np, int NB, int NBc,
                 int BH, int skip_masked, int per_head, long long total) {
  extern __shared__ uint8_t smem_raw[];
  CorrSmem<D>& sm = *reinterpret_cast<CorrSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  constexpr int kAtoms = D / 64;
  constexpr uint32_t kAtomBytes = 128 * 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i0 = static_cast<int>(total * blockIdx.x / gridDim.x);
  const int i1 = static_cast<int>(total * (blockIdx.x + 1) / gridDim.x);
  if (i1 <= i0) return;   // uniform across the block: before any barrier or TMEM use
  volatile int* abort_flag = &sm.abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&sm.a_full, 1);
    mbar_init(&sm.a_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.b_full[s], 1);
      mbar_init(&sm.b_empty[s], 1);
      mbar_init(&sm.d_full[s], 1);
      mbar_init(&sm.d_empty[s], 4);
    }
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(&sm.tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tm_a);
      prefetch_tmap(&tm_k);
      int g = -1, cur_bh = -1, cur_chunk = -1;
      int i = i0;
      bool ok = true;
      for (; ok && i < i1; ++i) {
        const CorrItem it = corr_item(i, NB, NBc, per_head, skip_masked);
        if (it.bh != cur_bh || it.chunk != cur_chunk) {
          // a new (head, chunk): its term tiles replace the previous ones once
          // every MMA that read those has completed
          ++g;
          if (g >= 1 && !mbar_wait(&sm.a_empty, (g - 1) & 1, abort_flag)) { ok = false; break; }
          mbar_expect_tx(&sm.a_full, 3 * kAtoms * kAtomBytes);
          for (int term = 0; term < 3; ++term)
            for (int at = 0; at < kAtoms; ++at)
              tma_load_2d(sm.a[term][at], &tm_a, &sm.a_full, 64 * at,
                          (term * BH + it.bh) * NBc * 128 + it.chunk * 128);
          cur_bh = it.bh;
          cur_chunk = it.chunk;
        }
        const int j = i - i0, s = j & 1;
        if (j >= 2 && !mbar_wait(&sm.b_empty[s], ((j >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
        mbar_expect_tx(&sm.b_full[s], kAtoms * kAtomBytes);
        for (int at = 0; at < kAtoms; ++at) {
          asm volatile(
              "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
              " [%0], [%1, {%3, %4, %5}], [%2];"
              ::"r"(smem_u32(sm.b[s][at])), "l"(reinterpret_cast<uint64_t>(&tm_k)),
                "r"(smem_u32(&sm.b_full[s])), "r"(64 * at), "r"(it.kt * 128), "r"(it.bh)
              : "memory");
        }
      }
      if (!ok) {
        // let the copies already issued land before the block exits
        if (g >= 0) mbar_wait(&sm.a_full, g & 1, nullptr);
        const int n = i - i0;
        for (int u = (n > 2 ? n - 2 : 0); u < n; ++u) mbar_wait(&sm.b_full[u & 1], (u >> 1) & 1, nullptr);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(128, 128, IsBf16<T>::value);
      const uint64_t da = smem_desc_kmajor(sm.a[0][0], 128);
      const uint64_t db = smem_desc_kmajor(sm.b[0][0], 128);
      int g = -1, cur_bh = -1, cur_chunk = -1;
      bool ok = true;
      for (int i = i0; ok && i < i1; ++i) {
        const CorrItem it = corr_item(i, NB, NBc, per_head, skip_masked);
        if (it.bh != cur_bh || it.chunk != cur_chunk) {
          ++g;
          if (!mbar_wait(&sm.a_full, g & 1, abort_flag)) { ok = false; break; }
          cur_bh = it.bh;
          cur_chunk = it.chunk;
        }
        const int j = i - i0, s = j & 1;
        if (!mbar_wait(&sm.b_full[s], (j >> 1) & 1, abort_flag)) { ok = false; break; }
        if (j >= 2 && !mbar_wait(&sm.d_empty[s], ((j >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        int n = 0;
#pragma unroll
        for (int term = 0; term < 3; ++term) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk, ++n) {
            // 16 channels (32 B) per step: atom kk/4, offset (kk%4)*32 B
            const uint32_t ao = ((term * kAtoms + kk / 4) * kAtomBytes + (kk % 4) * 32) >> 4;
            const uint32_t bo = ((s * kAtoms + kk / 4) * kAtomBytes + (kk % 4) * 32) >> 4;
            mma_f16_ss(tmem + s * 128, da + ao, db + bo, idesc, n > 0);
          }
        }
        tc_commit(&sm.d_full[s]);
        tc_commit(&sm.b_empty[s]);
        // the last item of this (head, chunk): its term tiles may be replaced
        // once these MMAs complete
        if (i + 1 < i1) {
          const CorrItem nx = corr_item(i + 1, NB, NBc, per_head, skip_masked);
          if (nx.bh != cur_bh || nx.chunk != cur_chunk) tc_commit(&sm.a_empty);
        }
      }
      if (!ok) {
        tc_commit(&sm.drain);
        mbar_wait(&sm.drain, 0, nullptr);
      }
    }
  } else if (warp >= 4) {
    // epilogue: warp q owns block rows 32q..32q+31 of the item's chunk (its TMEM lanes)
    const int q = warp - 4;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    int nb = 0;                                          // staging buffer to fill next
    for (int i = i0; i < i1; ++i) {
      const CorrItem it = corr_item(i, NB, NBc, per_head, skip_masked);
      const int j = i - i0, s = j & 1;
      const int row0 = it.chunk * 128 + q * 32;
      if (!mbar_wait_warp(&sm.d_full[s], (j >> 1) & 1, abort_flag)) break;
      // causal: block rows before the key tile never read it; this warp's 32
      // rows are all before it when its last row is
      if (skip_masked && it.kt > row0 + 31) {
        tc_fence_before();
        __syncwarp();
        mbar_arrive_lane0(&sm.d_empty[s], lane);
        continue;
      }
      tc_fence_after();
      uint32_t v[4][32];
      tmem_ld32(tmem + s * 128 + lane_off + 0, v[0]);
      tmem_ld32(tmem + s * 128 + lane_off + 32, v[1]);
      tmem_ld32(tmem + s * 128 + lane_off + 64, v[2]);
      tmem_ld32(tmem + s * 128 + lane_off + 96, v[3]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      mbar_arrive_lane0(&sm.d_empty[s], lane);
#pragma unroll
      for (int grp = 0; grp < 4; ++grp) {
        // the store issued two boxes ago has finished reading this buffer
        if (lane == 0) bulk_wait_read<1>();
        __syncwarp();
        uint8_t* st = sm.out[q][nb];
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(st + lane * 128 + ((c ^ (lane & 7)) << 4)) =
              make_uint4(v[grp][4 * c], v[grp][4 * c + 1], v[grp][4 * c + 2], v[grp][4 * c + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&tm_c, st, it.kt * 128 + 32 * grp, row0, it.bh);
          bulk_commit();
        }
        nb ^= 1;
      }
    }
    // shared memory stays in use until the last stores have read it
    if (lane == 0) bulk_wait_read<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <typename T, int D>
cudaError_t launch_qk_corr_t(const QKArgs& a, cudaStream_t st) {
  const int BH = a.B * a.H;
  const int NBc = (a.NB + 127) / 128;
  // TMA row coordinates of the term planes are 32-bit
  if (static_cast<int64_t>(3) * BH * NBc * 128 > INT32_MAX) return cudaErrorInvalidValue;
  T* terms = static_cast<T*>(a.qbar_split);
  k_qbar_split<T><<<dim3(NBc * 128, BH), D, 0, st>>>(a.q_mean, a.NB, NBc, D, BH, terms);
  alignas(64) CUtensorMap tma, tmk;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(D), static_cast<uint64_t>(3) * BH * NBc * 128};
    const uint64_t strides[1] = {static_cast<uint64_t>(D) * 2};
    const uint32_t box[2] = {64, 128};
    cudaError_t e = make_tmap(&tma, terms, 2, dims, strides, box, 2, 128);
    if (e != cudaSuccess) return e;
  }
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(a.N),
                              static_cast<uint64_t>(BH)};
    const uint64_t strides[2] = {static_cast<uint64_t>(D) * 2,
                                 static_cast<uint64_t>(a.ldh) * D * 2};
    const uint32_t box[3] = {64, 128, 1};
    cudaError_t e = make_tmap(&tmk, a.k, 3, dims, strides, box, 2, 128);
    if (e != cudaSuccess) return e;
  }
  alignas(64) CUtensorMap tmc;
  {
    // C as [B*H][NB][Np] fp32; a box is 32 keys (128 B, swizzled) x 32 block rows
    const uint64_t dims[3] = {static_cast<uint64_t>(a.Np), static_cast<uint64_t>(a.NB),
                              static_cast<uint64_t>(BH)};
    const uint64_t strides[2] = {static_cast<uint64_t>(a.Np) * 4,
                                 static_cast<uint64_t>(a.NB) * a.Np * 4};
    const uint32_t box[3] = {32, 32, 1};
    cudaError_t e = make_tmap(&tmc, a.qk_corr, 3, dims, strides, box, 4, 128);
    if (e != cudaSuccess) return e;
  }
  const size_t smem = sizeof(CorrSmem<D>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(k_qk_corr_tc<T, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // items per head: each chunk's key tiles (all of them, or with the causal
  // skip those up to the chunk's last block)
  int per_head = 0;
  for (int c = 0; c < NBc; ++c)
    per_head += a.skip_masked_corr ? std::min(a.NB, (c + 1) * 128) : a.NB;
  const long long total = static_cast<long long>(per_head) * BH;
  if (total > INT32_MAX) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long grid = std::min<long long>(total, sms);
  k_qk_corr_tc<T, D><<<static_cast<unsigned>(grid), 256, smem, st>>>(
      tma, tmk, tmc, a.N, a.Np, a.NB, NBc, BH, a.skip_masked_corr, per_head, total);
  return cudaGetLastError();
}

}  // namespace sage2
