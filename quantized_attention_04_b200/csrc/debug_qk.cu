// Test kernel: raw tiles of the integer product Q^ K^T through the same TMA +
// tcgen05 path as the attention kernel (one 128x128 tile per CTA), written as
// int32: INT4 values as e4m3 codes on the FP8 path (exact fp32 integer sums,
// converted), or INT8 values on the 8-bit integer path (s32 accumulator).
// Lets the integer matrix product ("4-bit matrix multiplication", SageAttention2
// abstract page, Abstract) be checked bit for bit on its own.
#include <cuda.h>

#include "sage2_internal.h"
#include "sm100_ptx.cuh"

namespace sage2 {

template <int D, int QB>
__global__ void __launch_bounds__(128) k_debug_qk_s32(const __grid_constant__ CUtensorMap tm_q,
                                                      const __grid_constant__ CUtensorMap tm_k,
                                                      int Np, int32_t* __restrict__ s_out) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sq = base;
  uint8_t* sk = base + 128 * D;
  __shared__ uint64_t bar_load, bar_mma;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;

  const int qt = blockIdx.x, kt = blockIdx.y, bh = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&bar_load, 1);
    mbar_init(&bar_mma, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (threadIdx.x == 0) {
    mbar_expect_tx(&bar_load, 2 * 128 * D);
    tma_load_2d(sq, &tm_q, &bar_load, 0, bh * Np + qt * 128);
    tma_load_2d(sk, &tm_k, &bar_load, 0, bh * Np + kt * 128);
    if (mbar_wait(&bar_load, 0, &abort_flag)) {
      tc_fence_after();
      constexpr uint32_t idesc = QB == 4 ? idesc_e4m3_f32(128, 128) : idesc_i8_s32(128, 128);
#pragma unroll
      for (int kk = 0; kk < D / 32; ++kk) {
        if (QB == 4)
          mma_f8_ss(tmem, smem_desc_kmajor(sq + 32 * kk, D), smem_desc_kmajor(sk + 32 * kk, D),
                    idesc, kk > 0);
        else
          mma_i8_ss(tmem, smem_desc_kmajor(sq + 32 * kk, D), smem_desc_kmajor(sk + 32 * kk, D),
                    idesc, kk > 0);
      }
      tc_commit(&bar_mma);
    }
  }
  __syncwarp();
  const bool ok = mbar_wait_warp(&bar_mma, 0, &abort_flag);
  tc_fence_after();
  if (ok) {
    const int r = warp * 32 + lane;
    int32_t* dst = s_out + (static_cast<size_t>(bh) * Np + qt * 128 + r) * Np + kt * 128;
#pragma unroll
    for (int c0 = 0; c0 < 128; c0 += 32) {
      uint32_t v[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c0, v);
      tmem_ld_wait();
#pragma unroll
      for (int u = 0; u < 32; u += 4)
        *reinterpret_cast<int4*>(dst + c0 + u) =
            QB == 4 ? make_int4(__float2int_rn(__uint_as_float(v[u])), __float2int_rn(__uint_as_float(v[u + 1])),
                                __float2int_rn(__uint_as_float(v[u + 2])), __float2int_rn(__uint_as_float(v[u + 3])))
                    : make_int4(v[u], v[u + 1], v[u + 2], v[u + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

template <int D, int QB>
static cudaError_t launch_debug_t(const uint8_t* q_i4, const uint8_t* k_i4, int BH, int Np,
                                  int32_t* s_out, cudaStream_t st) {
  alignas(64) CUtensorMap tq, tk;
  cudaError_t e = make_tmap_u8_2d(&tq, q_i4, static_cast<uint64_t>(BH) * Np, D, 128, D);
  if (e != cudaSuccess) return e;
  e = make_tmap_u8_2d(&tk, k_i4, static_cast<uint64_t>(BH) * Np, D, 128, D);
  if (e != cudaSuccess) return e;
  const int smem = 2 * 128 * D + 1024;
  const int nt = Np / 128;
  k_debug_qk_s32<D, QB><<<dim3(nt, nt, BH), 128, smem, st>>>(tq, tk, Np, s_out);
  return cudaGetLastError();
}

cudaError_t launch_debug_qk(const uint8_t* q_i4, const uint8_t* k_i4, int B, int H, int Np, int d,
                            int qk_bits, int32_t* s_out, cudaStream_t st) {
  if (qk_bits == 8)
    return d == 64 ? launch_debug_t<64, 8>(q_i4, k_i4, B * H, Np, s_out, st)
                   : launch_debug_t<128, 8>(q_i4, k_i4, B * H, Np, s_out, st);
  return d == 64 ? launch_debug_t<64, 4>(q_i4, k_i4, B * H, Np, s_out, st)
                 : launch_debug_t<128, 4>(q_i4, k_i4, B * H, Np, s_out, st);
}

}  // namespace sage2

// Test kernel for failure detection: one thread waits on an mbarrier phase
// that nothing completes.  The bounded wait gives up after its limit, records
// the timeout in the device error word and returns; the kernel ends normally
// and the context stays usable (no trap, no fault).
namespace sage2 {
__global__ void k_debug_wait_timeout() {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_wait(&bar, 0, nullptr);   // phase 0 never completes: times out
  }
}
cudaError_t launch_debug_wait_timeout(cudaStream_t st) {
  k_debug_wait_timeout<<<1, 32, 0, st>>>();
  return cudaGetLastError();
}
}  // namespace sage2
