// Fused SageAttention2 forward kernel for sm_100a (tcgen05 + TMEM + TMA).
//
// "SageAttention2: Efficient Attention with Thorough Outlier Smoothing and
// Per-thread INT4 Quantization" (arxiv.science abstract page, Abstract): the
// INT4 Q^K^T product, FP8 P~ and V, and the two-level accumulation of P~V.
//
// One CTA = one 128-row query block of one head; 512 threads, warp-specialised:
//   warp 0        TMA producer: the Q^ tile once, then per key tile K^, V^T,
//                 the key scales and the correction chunk (kStages-deep ring).
//   warp 1        MMA issuer (one thread): S = Q^ K^T with tcgen05 kind::f8f6f4
//                 (the INT4 values carried as e4m3 codes; exact fp32 integer
//                 sums; kind::i8 for the INT8 variant) into TMEM (three
//                 buffers, issued three key tiles ahead), and inner = P~ V~
//                 with kind::f8f6f4 (e4m3 -> f32; A = P~ from TMEM) into a
//                 fresh TMEM accumulator per key tile (one buffer: the
//                 correction warpgroup reads it long before the next PV).
//   warp 2        TMEM allocator.
//   warps 4-7,    two softmax warpgroups.  Warpgroup h owns lanes 16h..16h+15 of
//   warps 8-11    every 32-lane TMEM quadrant; with .16x256b loads a thread owns
//                 two query rows and 32 consecutive keys of each tile (four
//                 threads of a warp share a row).  Per tile: dequantise +
//                 correct its 64 scores, row max across the four threads, the
//                 rescale factor alpha (to shared memory), exp2, l, and
//                 P~ = e4m3(448 p) into TMEM over the tile's S buffer.  The
//                 exp2 phases of the two warps of a sub-partition take turns
//                 (named barriers).
//   warps 12-15   correction warpgroup: thread r owns query row r and the outer
//                 fp32 accumulator (acc = alpha*acc + inner per key tile: the
//                 outer level of the two-level accumulation), then the epilogue.
// TMEM columns: S[b] at 128*b (b = 0, 1, 2), the inner accumulator at 384.
// P~ of a tile replaces the first 32 columns of its S buffer (its 128 keys as
// bytes, four per column) and is the TMEM A operand of the PV product.
// Every mbarrier wait is bounded (see mbar_wait); on a timeout the kernel
// records it in the device error word and every role leaves its loop.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "sage2_internal.h"
#include "sm100_ptx.cuh"

namespace sage2 {

constexpr int kStages = 4;
constexpr int kSBuf = 3;                         // S tiles in flight in TMEM (P~ of a tile over its S)
constexpr int kThreads = 512;
constexpr int kHeadGroup = 8;       // heads whose tiles are interleaved in launch order ...
constexpr int kGroupMaxTiles = 128; // ... when a head has at most this many query tiles
constexpr int kSegStride = 36;                   // floats between the 32-key groups in shared memory
constexpr float kLog2_448 = 8.807354922057604f;  // log2(448)
constexpr uint32_t kMagicBits = 0x4B400000u;     // 1.5 * 2^23 (INT8 variant, see dequant16)
constexpr float kMagic = 12582912.0f;

template <int D>
struct __align__(1024) AttnSmem {
  uint8_t q[128 * D];              // Q^ tile (K-major, swizzled)
  uint8_t k[kStages][128 * D];     // K^ tiles
  uint8_t v[kStages][D * 128];     // V^T tiles: D rows (channels) x 128 tokens
  // qk_corr and k_scale of the key tile: keys 32g..32g+31 at [36g, 36g+32).
  // The 16-byte gaps put the four groups (read by the four threads g of a
  // row in the same instruction) in different banks.
  float corr[kStages][4 * kSegStride];
  float ksc[kStages][4 * kSegStride];
  float qsc[128];                  // q_scale of the block's rows
  float vsc[D];                     // v_scale (correction warpgroup)
  float vmean[D];                   // token mean of V when V was smoothed, else 0
  float alpha[4][128];              // per-row rescale factor of tile t in slot t%4 (softmax -> correction)
  float lsum[128];                  // final row sums (448-scaled), softmax -> correction
  uint64_t q_full;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[kSBuf];           // two arrivals: the MMA thread once it saw the key
                                    // tile land (so its scales are visible to whoever
                                    // acquires this barrier), and the commit of S[b]
  uint64_t p_full[kSBuf];           // P~ over S[b] written by all 8 softmax warps; this also
                                    // says S[b] was read
  uint64_t i_full;                  // two arrivals: the MMA thread after it saw p_full (so
                                    // alpha of the tile is visible), and the commit of inner
  uint64_t i_empty;                 // the correction warpgroup read inner
  uint64_t l_full;                  // the softmax warps published the row sums
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
template <int N>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void named_bar_arrive(int id, int count) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// Named barriers of the exp2 ping-pong between the two softmax warps of one
// SM sub-partition (quadrant q): kBarExpA + q is released by the second
// warpgroup for the first, kBarExpB + q the other way round.
constexpr int kBarExpA = 3, kBarExpB = 7;

// The score S_ij as a float.  INT4 (QB = 4): S comes out of the FP8 tensor
// path as an fp32 integer: the INT4 values are exact in e4m3, every product
// (|.| <= 49) and partial sum (|.| <= 49*128 < 2^13) is an integer the fp32
// accumulator holds exactly.  INT8 (QB = 8): S is s32 (|S| <= 127^2*128 <
// 2^22); its bits plus 0x4B400000, read as a float, are exactly 1.5*2^23 + S,
// and subtracting 1.5*2^23 is exact.
template <int QB>
__device__ __forceinline__ float2 s_pair(uint32_t a, uint32_t b) {
  if (QB == 4) return make_float2(__uint_as_float(a), __uint_as_float(b));
  return __fadd2_rn(make_float2(__uint_as_float(a + kMagicBits), __uint_as_float(b + kMagicBits)),
                    make_float2(-kMagic, -kMagic));
}

// Dequantise + correct the 16 keys 4m..4m+3 (m = 0..3) of both rows held in
// one .16x256b.x8 load: x' = sq_i * (sk_j * S_ij) + C_j.
template <int QB>
__device__ __forceinline__ void dequant16(const uint32_t (&sr)[32], const float4* ck,
                                          const float4* kk, float2 a0, float2 a1, float* x0,
                                          float* x1) {
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const float4 c4 = ck[m];
    const float4 k4 = kk[m];
    const float2 kxy = make_float2(k4.x, k4.y), kzw = make_float2(k4.z, k4.w);
    const float2 cxy = make_float2(c4.x, c4.y), czw = make_float2(c4.z, c4.w);
    const uint32_t* q = sr + 8 * m;
    const float2 r00 = __ffma2_rn(a0, __fmul2_rn(kxy, s_pair<QB>(q[0], q[1])), cxy);
    const float2 r01 = __ffma2_rn(a0, __fmul2_rn(kzw, s_pair<QB>(q[4], q[5])), czw);
    const float2 r10 = __ffma2_rn(a1, __fmul2_rn(kxy, s_pair<QB>(q[2], q[3])), cxy);
    const float2 r11 = __ffma2_rn(a1, __fmul2_rn(kzw, s_pair<QB>(q[6], q[7])), czw);
    x0[4 * m] = r00.x;
    x0[4 * m + 1] = r00.y;
    x0[4 * m + 2] = r01.x;
    x0[4 * m + 3] = r01.y;
    x1[4 * m] = r10.x;
    x1[4 * m + 1] = r10.y;
    x1[4 * m + 2] = r11.x;
    x1[4 * m + 3] = r11.y;
  }
}

__device__ __forceinline__ float rowmax32(const float (&x)[32]) {
  float m4[4];
#pragma unroll
  for (int g = 0; g < 4; ++g)
    m4[g] = max3f(max3f(x[8 * g], x[8 * g + 1], x[8 * g + 2]),
                  max3f(x[8 * g + 3], x[8 * g + 4], x[8 * g + 5]), fmaxf(x[8 * g + 6], x[8 * g + 7]));
  return fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
}

// p448 = exp2(x' L + nb) for the 32 keys of one row, e4m3-rounded (RN,
// saturating) into eight words: word i holds keys 4i..4i+3 (one byte each).
// Returns the row's sum of the unrounded p448.
__device__ __forceinline__ float exp_pack(const float (&x)[32], float2 L2, float2 nb,
                                          uint32_t (&w)[8]) {
  float2 sumA = make_float2(0.f, 0.f), sumB = make_float2(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < 2; ++c) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = c * 16 + u * 4;
      float2 e0 = __ffma2_rn(make_float2(x[j], x[j + 1]), L2, nb);
      float2 e1 = __ffma2_rn(make_float2(x[j + 2], x[j + 3]), L2, nb);
      e0.x = ex2(e0.x);
      e0.y = ex2(e0.y);
      e1.x = ex2(e1.x);
      e1.y = ex2(e1.y);
      sumA = __fadd2_rn(sumA, e0);
      sumB = __fadd2_rn(sumB, e1);
      const uint32_t lo = __nv_cvt_float2_to_fp8x2(e0, __NV_SATFINITE, __NV_E4M3);
      const uint32_t hi = __nv_cvt_float2_to_fp8x2(e1, __NV_SATFINITE, __NV_E4M3);
      w[4 * c + u] = lo | (hi << 16);
    }
  }
  const float2 s2 = __fadd2_rn(sumA, sumB);
  return s2.x + s2.y;
}

// acc[32 channels] = alpha * acc + inner for one row (.32x32b load).
__device__ __forceinline__ void fold32(float* acc, const uint32_t (&in)[32], float al) {
  const float2 al2 = make_float2(al, al);
#pragma unroll
  for (int c = 0; c < 32; c += 2) {
    const float2 r = __ffma2_rn(al2, make_float2(acc[c], acc[c + 1]),
                                make_float2(__uint_as_float(in[c]), __uint_as_float(in[c + 1])));
    acc[c] = r.x;
    acc[c + 1] = r.y;
  }
}

// Eight consecutive output channels (index of the first, a multiple of 8) in
// the output type, with 16-byte stores.
template <int OT>
__device__ __forceinline__ void store8(void* out, size_t idx, const float (&f)[8]) {
  if (OT == 2) {
    float4* p = reinterpret_cast<float4*>(static_cast<float*>(out) + idx);
    p[0] = make_float4(f[0], f[1], f[2], f[3]);
    p[1] = make_float4(f[4], f[5], f[6], f[7]);
  } else {
    uint32_t w[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (OT == 0) {
        const __half2 hv = __floats2half2_rn(f[2 * u], f[2 * u + 1]);
        w[u] = *reinterpret_cast<const uint32_t*>(&hv);
      } else {
        const __nv_bfloat162 hv = __floats2bfloat162_rn(f[2 * u], f[2 * u + 1]);
        w[u] = *reinterpret_cast<const uint32_t*>(&hv);
      }
    }
    *reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + idx) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

template <int D, int OT, int QB, bool GROUPED>
__global__ void __launch_bounds__(kThreads, 1)
    k_attn_fwd(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ q_scale,
               const float* __restrict__ k_scale, const float* __restrict__ qk_corr,
               const float* __restrict__ v_scale, const float* __restrict__ v_mean,
               void* __restrict__ out, int N, long long ldo, int Np, int NB, int causal,
               float L) {
  extern __shared__ uint8_t smem_raw[];
  AttnSmem<D>& sm = *reinterpret_cast<AttnSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Launch order, x fastest.  Plain grid (NB, B*H): one head after another,
  // its longest query tile (causal) first.  GROUPED grid (G, NB, B*H/G): G
  // heads round robin, each taking its longest tile first, so that the short
  // tiles of every head fill the tail of a launch of short heads.
  const int rank = static_cast<int>(GROUPED ? blockIdx.y : blockIdx.x);
  const int qt = causal ? (NB - 1 - rank) : rank;
  const int bh = static_cast<int>(GROUPED ? blockIdx.z * gridDim.x + blockIdx.x : blockIdx.y);
  const int nt = causal ? qt + 1 : NB;           // key tiles this block visits
  const bool tail = (N % 128) != 0;
  volatile int* abort_flag = &sm.abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int b = 0; b < kSBuf; ++b) {
      mbar_init(&sm.s_full[b], 2);
      mbar_init(&sm.p_full[b], 8);
    }
    mbar_init(&sm.i_full, 2);
    mbar_init(&sm.i_empty, 4);
    mbar_init(&sm.drain, 1);
    mbar_init(&sm.l_full, 8);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  const int wg = warp >> 2;
  if (wg == 0) {
    setmaxnreg_dec<40>();  // one call site for the whole warpgroup
  }
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      const int row0 = bh * Np + qt * 128;
      mbar_expect_tx(&sm.q_full, 128 * D + 512);
      tma_load_2d(sm.q, &tm_q, &sm.q_full, 0, row0);
      bulk_load(sm.qsc, q_scale + row0, 512, &sm.q_full);
      const float* corr_row = qk_corr + (static_cast<size_t>(bh) * NB + qt) * Np;
      const float* ks_row = k_scale + static_cast<size_t>(bh) * Np;
      int t = 0;
      for (; t < nt; ++t) {
        const int s = t % kStages;
        if (t >= kStages && !mbar_wait(&sm.kv_empty[s], ((t / kStages) - 1) & 1, abort_flag)) break;
        mbar_expect_tx(&sm.kv_full[s], 128 * D + D * 128 + 512 + 512);
        tma_load_2d(sm.k[s], &tm_k, &sm.kv_full[s], 0, bh * Np + t * 128);
        tma_load_2d(sm.v[s], &tm_v, &sm.kv_full[s], t * 128, bh * D);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          bulk_load(sm.corr[s] + kSegStride * g, corr_row + t * 128 + 32 * g, 128, &sm.kv_full[s]);
          bulk_load(sm.ksc[s] + kSegStride * g, ks_row + t * 128 + 32 * g, 128, &sm.kv_full[s]);
        }
      }
      if (*abort_flag) {
        // let the copies already issued land before the block exits
        mbar_wait(&sm.q_full, 0, nullptr);
        for (int u = (t > kStages ? t - kStages : 0); u < t; ++u)
          mbar_wait(&sm.kv_full[u % kStages], (u / kStages) & 1, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // INT4 values as e4m3 codes on the FP8 path; INT8 values on the 8-bit integer path
      constexpr uint32_t idesc_qk = QB == 4 ? idesc_e4m3_f32(128, 128) : idesc_i8_s32(128, 128);
      constexpr uint32_t idesc_pv = idesc_e4m3_f32(128, D);
      // descriptors are built once; a k-step or a stage only moves the start
      // address field (16-byte units; shared memory is < 256 KB, no carry)
      const uint64_t dq = smem_desc_kmajor(sm.q, D);
      const uint64_t dk = smem_desc_kmajor(sm.k[0], D);
      const uint64_t dv = smem_desc_kmajor(sm.v[0], 128);
      constexpr uint32_t kStageK = (128 * D) >> 4, kStageV = (D * 128) >> 4;
      bool ok = mbar_wait(&sm.q_full, 0, abort_flag);
      auto issue_qk = [&](int u) -> bool {
        const int s = u % kStages, b = u % kSBuf;
        if (!mbar_wait(&sm.kv_full[s], (u / kStages) & 1, abort_flag)) return false;
        // S[b] (with P~ of tile u-3 in its first 32 columns) is free once PV(u-3)
        // has completed: the phase of i_full for tile u-3 (QK(u) is issued right
        // after PV(u-3), before PV(u-2), so i_full is still in that phase)
        if (u >= kSBuf && !mbar_wait(&sm.i_full, (u - kSBuf) & 1, abort_flag)) return false;
        mbar_arrive(&sm.s_full[b]);                       // releases the kv_full acquire
        tc_fence_after();
        const uint64_t kb = dk + s * kStageK;
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk) {
          if (QB == 4) mma_f8_ss(tmem + b * 128, dq + 2 * kk, kb + 2 * kk, idesc_qk, kk > 0);
          else mma_i8_ss(tmem + b * 128, dq + 2 * kk, kb + 2 * kk, idesc_qk, kk > 0);
        }
        tc_commit(&sm.s_full[b]);
        return true;
      };
      auto issue_pv = [&](int u) -> bool {
        const int s = u % kStages, b = u % kSBuf;
        // P~(u) and alpha(u) are written; the correction warpgroup has read
        // inner of tile u-1 (one inner accumulator: it is read well before the
        // next PV is due)
        if (!mbar_wait(&sm.p_full[b], (u / kSBuf) & 1, abort_flag)) return false;
        if (u >= 1 && !mbar_wait(&sm.i_empty, (u - 1) & 1, abort_flag)) return false;
        mbar_arrive(&sm.i_full);                          // releases the p_full acquire (alpha)
        tc_fence_after();
        const uint64_t vb = dv + s * kStageV;
        // A = P~(u) in TMEM (the first 32 columns of S[b]: 128 keys, 4 per column)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f8_ts(tmem + kSBuf * 128, tmem + b * 128 + 8 * kk, vb + 2 * kk, idesc_pv, kk > 0);
        tc_commit(&sm.i_full);
        tc_commit(&sm.kv_empty[s]);
        return true;
      };
      for (int u = 0; ok && u < kSBuf && u < nt; ++u) ok = issue_qk(u);
      for (int t = 0; ok && t < nt; ++t) {
        // both wait for the end of the softmax of tile t; PV first, its result
        // is needed before S(t+3)
        if (!issue_pv(t)) { ok = false; break; }
        if (t + kSBuf < nt && !issue_qk(t + kSBuf)) { ok = false; break; }
      }
      if (!ok) {
        // wait for every MMA issued so far before the block frees TMEM
        tc_commit(&sm.drain);
        mbar_wait(&sm.drain, 0, nullptr);
      }
    }
  } else if (wg == 1 || wg == 2) {
    // ------------------------------------------------------------ softmax warpgroups
    // Raised inside the branch it governs, so that the compiler allocates this
    // role's code against the larger budget (40*128 + 152*256 + 168*128 = 128*512).
    setmaxnreg_inc<152>();
    // The .16x256b TMEM loads give thread t of a warp, in a 16-lane group, the
    // two lanes t/4 and t/4 + 8 and the columns 8k + 2g + {0,1} (g = t%4,
    // k = 0..15).  Warpgroup h takes lanes 16h..16h+15 of each 32-lane
    // quadrant, so every query row is shared by the four threads g = 0..3 of
    // one warp and each thread owns two rows.  With the K^ rows of each block
    // stored so that column 8k + 2g + e holds token 32g + 2k + e, thread g sees
    // the 32 consecutive keys 32g..32g+31 of the tile (both rows).
    const int h = wg - 1;
    const int quad = warp & 3;
    const int g = lane & 3;
    const int r0 = 32 * quad + 16 * h + (lane >> 2);      // rows in the block: r0, r0 + 8
    const int row0 = qt * 128 + r0, row1 = row0 + 8;      // rows in the head
    const uint32_t lane_addr = static_cast<uint32_t>(32 * quad + 16 * h) << 16;
    const uint32_t tS = tmem + lane_addr;                 // + 128*b: S buffer b
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    bool ok = mbar_wait_warp(&sm.q_full, 0, abort_flag);
    const float a0 = ok ? sm.qsc[r0] : 0.f, a1 = ok ? sm.qsc[r0 + 8] : 0.f;
    const float2 a02 = make_float2(a0, a0), a12 = make_float2(a1, a1);
    const float2 L2 = make_float2(L, L);
    // The exp2 phases of the two warps that share an SM sub-partition (warp q
    // of each warpgroup) take turns: one warp's exp2 runs while the other
    // dequantises, so the MUFU is not split between them.  Every tile runs
    // the full barrier protocol, also after a failed wait (the work is then
    // skipped), so that neither warp can be left waiting on the other.
    const int bar_mine = (h == 0 ? kBarExpA : kBarExpB) + quad;
    const int bar_other = (h == 0 ? kBarExpB : kBarExpA) + quad;

    // s_full(t+1) is probed (non-blocking, with acquire) early in the exp2
    // phase of tile t, so that the blocking wait is skipped when S(t+1) has
    // landed by then: the probe's latency hides behind the exp2 work.
    bool s_ready = false;
    for (int t = 0; t < nt; ++t) {
      const int s = t % kStages, b = t % kSBuf;
      // s_full(t) also says PV(t-3) is complete: the MMA thread issued QK(t)
      // after PV(t-3) completed, and the commit tracks every earlier MMA.  So
      // the P~ columns of S[b] are free, with no wait of its own.
      if (ok && !s_ready) ok = mbar_wait_warp(&sm.s_full[b], (t / kSBuf) & 1, abort_flag);
      if (!ok) {
        if (h == 1 || t > 0) named_bar_sync(bar_mine, 64);
        named_bar_arrive(bar_other, 64);
        continue;
      }
      tc_fence_after();
      float x0[32], x1[32];                               // rows r0, r0+8; keys 32g + j
      {
        uint32_t sA[32], sB[32];
        tmem_ld16x256_32(tS + b * 128, sA);
        tmem_ld16x256_32(tS + b * 128 + 64, sB);
        // the key scales and correction chunk of stage s are visible: s_full
        // also carries the MMA thread's release after it acquired kv_full.
        // The first half is read while the TMEM loads are in flight.
        const float4* cp = reinterpret_cast<const float4*>(sm.corr[s] + kSegStride * g);
        const float4* kp = reinterpret_cast<const float4*>(sm.ksc[s] + kSegStride * g);
        float4 c0[4], k0[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          c0[m] = cp[m];
          k0[m] = kp[m];
        }
        tmem_ld_wait();
        dequant16<QB>(sA, c0, k0, a02, a12, x0, x1);
        dequant16<QB>(sB, cp + 4, kp + 4, a02, a12, x0 + 16, x1 + 16);
      }
      if ((causal && t == qt) || (tail && t == NB - 1)) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int key = t * 128 + 32 * g + j;
          if (key >= N || (causal && key > row0)) x0[j] = -INFINITY;
          if (key >= N || (causal && key > row1)) x1[j] = -INFINITY;
        }
      }
      float mx0 = rowmax32(x0), mx1 = rowmax32(x1);
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));   // the rows' other threads
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float2 alpha = make_float2(ex2((m0 - mn0) * L), ex2((m1 - mn1) * L));  // 0 on the first tile
      // for the correction warpgroup; slot t%4 was last read for tile t-4,
      // before PV(t-3) was issued, which s_full(t) follows
      sm.alpha[t & 3][r0] = alpha.x;                      // the row's four threads agree
      sm.alpha[t & 3][r0 + 8] = alpha.y;
      // p448 = 448 * exp2((x' - m) L) = exp2(x' L - (m L - log2 448))
      const float2 nb0 = make_float2(kLog2_448 - mn0 * L, kLog2_448 - mn0 * L);
      const float2 nb1 = make_float2(kLog2_448 - mn1 * L, kLog2_448 - mn1 * L);
      // exp2 turn: the first warpgroup waits for the second one's previous tile,
      // the second one for the first one's current tile
      if (h == 1 || t > 0) named_bar_sync(bar_mine, 64);
      const bool probe = t + 1 < nt && mbar_test(&sm.s_full[(t + 1) % kSBuf], ((t + 1) / kSBuf) & 1);
      // P~(t) goes to the first 32 columns of S[b], over scores this thread
      // has already read: column 8k + 2g + e of its two rows holds its keys
      // 32g + 8k + 4e .. +3 (V^T's tokens are stored in the matching order).
      uint32_t w0[8], w1[8];
      const float s0 = exp_pack(x0, L2, nb0, w0);
      const float s1 = exp_pack(x1, L2, nb1, w1);
      {
        uint32_t pr[16];
#pragma unroll
        for (int k = 0; k < 4; ++k)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            pr[4 * k + e] = w0[2 * k + e];
            pr[4 * k + 2 + e] = w1[2 * k + e];
          }
        tmem_st16x256_16(tS + b * 128, pr);
      }
      named_bar_arrive(bar_other, 64);
      tmem_st_wait();
      tc_fence_before();                                  // S(t) read, P~(t) written
      __syncwarp();
      mbar_arrive_lane0(&sm.p_full[b], lane);
      s_ready = __all_sync(0xffffffffu, probe);           // the probe's result is consumed here
      l0 = alpha.x * l0 + s0;
      l1 = alpha.y * l1 + s1;
      m0 = mn0;
      m1 = mn1;
    }
    // the second warpgroup's last turn ended
    if (h == 0 && nt > 0) named_bar_sync(bar_mine, 64);
    if (ok) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
      sm.lsum[r0] = l0;                                   // the row's four threads agree
      sm.lsum[r0 + 8] = l1;
      __syncwarp();
      mbar_arrive_lane0(&sm.l_full, lane);
    }
  } else if (wg == 3) {
    // ------------------------------------------------------------ correction warpgroup
    // Thread r owns query row r (TMEM lane r, .32x32b loads: consecutive
    // channels) and the outer fp32 accumulator of the two-level accumulation
    // in registers: per key tile, acc = alpha*acc + inner (inner = the fresh
    // PV accumulator of that tile), then the epilogue O = acc*v_scale/l.
    setmaxnreg_inc<168>();
    const int r = (warp & 3) * 32 + lane;
    const int row = qt * 128 + r;
    const uint32_t tI = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + kSBuf * 128;
    for (int i = r; i < D; i += 128) {
      sm.vsc[i] = v_scale[static_cast<size_t>(bh) * D + i];
      sm.vmean[i] = v_mean ? v_mean[static_cast<size_t>(bh) * D + i] : 0.f;
    }
    named_bar_sync(1, 128);
    float acc[D];
#pragma unroll
    for (int c = 0; c < D; ++c) acc[c] = 0.f;
    bool ok = true;
    for (int t = 0; ok && t < nt; ++t) {
      // i_full also carries the MMA thread's release after it saw p_full, so
      // alpha of tile t is visible
      if (!mbar_wait_warp(&sm.i_full, t & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const float al = sm.alpha[t & 3][r];
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tI + c0, v);
        tmem_ld_wait();
        fold32(acc + c0, v, al);
      }
      tc_fence_before();
      __syncwarp();
      mbar_arrive_lane0(&sm.i_empty, lane);
    }
    if (ok) ok = mbar_wait_warp(&sm.l_full, 0, abort_flag);
    if (ok && row < N) {
      const float inv = 1.0f / sm.lsum[r];
      const size_t obase = (static_cast<size_t>(bh) * ldo + row) * D;
#pragma unroll
      for (int c = 0; c < D; c += 8) {
        float f[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) f[u] = acc[c + u] * sm.vsc[c + u] * inv + sm.vmean[c + u];
        store8<OT>(out, obase + c, f);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, int OT, int QB, bool GROUPED>
static cudaError_t launch_attn_g(const AttnArgs& a, cudaStream_t st, int group) {
  alignas(64) CUtensorMap tq, tk, tv;
  const int BH = a.B * a.H;
  cudaError_t e;
  e = make_tmap_u8_2d(&tq, a.q_i4, static_cast<uint64_t>(BH) * a.Np, D, 128, D);
  if (e != cudaSuccess) return e;
  e = make_tmap_u8_2d(&tk, a.k_i4, static_cast<uint64_t>(BH) * a.Np, D, 128, D);
  if (e != cudaSuccess) return e;
  e = make_tmap_u8_2d(&tv, a.v_fp8_t, static_cast<uint64_t>(BH) * D, a.Np, D, 128);
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(AttnSmem<D>) + 1024;
  e = cudaFuncSetAttribute(k_attn_fwd<D, OT, QB, GROUPED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const float L = a.sm_scale * 1.4426950408889634f;
  const dim3 grid = GROUPED ? dim3(group, a.NB, BH / group) : dim3(a.NB, BH);
  k_attn_fwd<D, OT, QB, GROUPED><<<grid, kThreads, smem, st>>>(
      tq, tk, tv, a.q_scale, a.k_scale, a.qk_corr, a.v_scale, a.v_mean, a.o, a.N, a.ldo, a.Np,
      a.NB, a.causal, L);
  return cudaGetLastError();
}

// Heads are interleaved (G = the largest divisor of B*H up to kHeadGroup)
// only when a head has few query tiles, where the tail of the launch is a
// large share; a long head runs alone, its K and V shared in L2 by every SM.
template <int D, int OT, int QB>
static cudaError_t launch_attn_t(const AttnArgs& a, cudaStream_t st) {
  const int BH = a.B * a.H;
  int group = kHeadGroup;
  while (BH % group != 0) --group;
  if (a.NB <= kGroupMaxTiles && group > 1) return launch_attn_g<D, OT, QB, true>(a, st, group);
  return launch_attn_g<D, OT, QB, false>(a, st, 1);
}

template <int QB>
static cudaError_t launch_attn_q(const AttnArgs& a, cudaStream_t st) {
  if (a.d == 64) {
    if (a.o_dtype == 0) return launch_attn_t<64, 0, QB>(a, st);
    if (a.o_dtype == 1) return launch_attn_t<64, 1, QB>(a, st);
    return launch_attn_t<64, 2, QB>(a, st);
  }
  if (a.o_dtype == 0) return launch_attn_t<128, 0, QB>(a, st);
  if (a.o_dtype == 1) return launch_attn_t<128, 1, QB>(a, st);
  return launch_attn_t<128, 2, QB>(a, st);
}

cudaError_t launch_attn(const AttnArgs& a, cudaStream_t st) {
  return a.qk_bits == 8 ? launch_attn_q<8>(a, st) : launch_attn_q<4>(a, st);
}

}  // namespace sage2
