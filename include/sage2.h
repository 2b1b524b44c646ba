/*
 * sage2.h - C ABI of the B200 (sm_100a) SageAttention2 quantized attention
 * forward pass:  O = softmax(Q K^T * sm_scale) V  computed with smoothed INT4
 * Q/K, FP8 (e4m3) P~/V and two-level P~V accumulation.
 *
 * The method follows "SageAttention2: Efficient Attention with Thorough
 * Outlier Smoothing and Per-thread INT4 Quantization" (arxiv.science abstract
 * page, Abstract): INT4 (Q, K) at a per-thread granularity, FP8 (P~, V),
 * smoothing of Q for the INT4 QK^T, two-level accumulation for the FP8 P~V.
 * K smoothing (token mean removed) is the "outlier smoothing" of the title.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are dense, row-major ("HND"): q, k, v, o are [B, H, N, d].
 *  - d is 64 or 128.  N >= 1.  B*H >= 1.  Np = ceil(N/128)*128, NB = Np/128.
 *  - All pointers are DEVICE pointers owned by the caller, 16-byte aligned.
 *    The library never frees caller memory.
 *  - Every call is asynchronous on `stream` (NULL = the legacy default
 *    stream) and returns before the GPU work ends.  Arguments are validated on
 *    the host before anything is launched; a non-OK status means nothing was
 *    launched (except SAGE2_ERR_CUDA, which reports a failed launch).
 *  - No C++ exception crosses the ABI.
 *  - Causal masking is top-left aligned: query i sees keys j <= i.
 *
 * Payload layouts (the quantized intermediates, all on the device)
 * ----------------------------------------------------------------
 *  q_i4   u8    [B,H,Np,d]   INT4 values in [-7,7] of Q - qbar_block, each stored as its
 *                            e4m3 code (every integer in [-7,7] is exact in e4m3; zero is
 *                            +0, code 0x00), rows >= N are 0.  The FP8 tensor path then
 *                            multiplies the INT4 values exactly, at the 8-bit integer
 *                            path's rate, and gives S as an fp32 integer.
 *  q_scale f32  [B,H,Np]     per-token scale amax/7 (0 for an all-zero row / pad)
 *  q_mean f32   [B,H,NB,d]   mean of each 128-row block of Q (valid rows only)
 *  k_i4   u8    [B,H,Np,d]   INT4 values of K - kbar as e4m3 codes (as q_i4), rows >= N
 *                            are 0.  Rows are stored
 *                            PERMUTED inside each 128-row block: stored row n of a block
 *                            holds token 32*((n/2)%4) + 2*(n/8) + n%2 of that block.
 *  k_scale f32  [B,H,Np]     per-token scale
 *  k_mean f32   [B,H,d]      token mean of K
 *  qk_corr f32  [B,H,NB,Np]  q_mean[blk] . K[j] (raw K), 0 for j >= N
 *  v_fp8_t u8   [B,H,d,Np]   e4m3 codes of V * 448/amax_c, TRANSPOSED (token-contiguous).
 *                            Tokens are PERMUTED inside each 128-token block: byte p of
 *                            a block holds token sigma(p), where sigma swaps the 2-bit
 *                            fields [6:5] and [4:3] of p (sigma = sigma^-1), i.e.
 *                            sigma(p) = 32*((p/8)%4) + 8*((p/32)%4) + p%8.
 *  v_scale f32  [B,H,d]      per-channel scale amax_c/448
 */
#ifndef SAGE2_H_
#define SAGE2_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t. */
typedef struct CUstream_st* sage2_stream_t;

typedef enum {
  SAGE2_OK = 0,
  SAGE2_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, bad dtype   */
  SAGE2_ERR_UNSUPPORTED = 2, /* d not in {64,128}, size beyond int32 indexing */
  SAGE2_ERR_MISALIGNED = 3,  /* a pointer is not 16-byte aligned              */
  SAGE2_ERR_CUDA = 4,        /* a CUDA runtime/driver call or launch failed   */
  SAGE2_ERR_NO_MEM = 5,      /* workspace allocation failed                   */
  SAGE2_ERR_TIMEOUT = 6,     /* a kernel's bounded wait ran out (device word) */
  SAGE2_ERR_TOO_LARGE = 7    /* scratch needed exceeds the fixed no-allocation buffer */
} sage2_status;

typedef enum { SAGE2_F16 = 0, SAGE2_BF16 = 1, SAGE2_F32 = 2 } sage2_dtype;

/*
 * Integer format of the Q^/K^ payloads (q_i4, k_i4).
 *   SAGE2_QK_INT4 : the method.  Values in [-7,7], each stored as its e4m3 code.
 *   SAGE2_QK_INT8 : a variant, the 8-bit quantization of the predecessor
 *                   ("SageAttention: Accurate 8-Bit Attention", ainnect.com
 *                   research/19 summary).  Values in [-127,127] stored as
 *                   two's-complement bytes; scale = amax/127.  Everything else on
 *                   the path is unchanged (smoothing, correction, FP8 P~V).
 *   SAGE2_QK_INT4_PACKED : the method's INT4 values (the same values and
 *                   scales as SAGE2_QK_INT4) stored two per byte, the INT4
 *                   storage precision of the abstract: q_i4 and k_i4 are
 *                   [B,H,Np,d/2] bytes; byte c of a row holds channel 2c in
 *                   bits 3:0 and channel 2c+1 in bits 7:4, each a
 *                   two's-complement nibble; k_i4 rows are permuted as for
 *                   SAGE2_QK_INT4.  B200 has no INT4 tensor-core path, so the
 *                   attention entries expand the nibbles to e4m3 codes (one
 *                   memory-bound pass into library scratch) before the
 *                   attention kernel: the output is bit-identical to that of
 *                   SAGE2_QK_INT4.  Not accepted by sage2_debug_qk_s32_ex.
 */
typedef enum { SAGE2_QK_INT4 = 0, SAGE2_QK_INT8 = 1, SAGE2_QK_INT4_PACKED = 2 } sage2_qk_format;

/*
 * Smoothing + INT4 quantization of Q and K, and the Q-smoothing correction.
 * (Abstract: INT4 (Q,K) at per-thread granularity; "a method to smooth Q".)
 *   q, k      : [B,H,N,d] in `dtype` (SAGE2_F16 or SAGE2_BF16).
 *   outputs   : q_i4, q_scale, q_mean, k_i4, k_scale, k_mean, qk_corr as in the
 *               payload table above (caller-allocated, fully overwritten,
 *               including the pad rows/columns).
 * Semantics: kbar = fixed-order fp32 token mean of K (128-token chunks summed
 * in token order, chunk sums in chunk order, one fp32 division by N); qbar per
 * 128-row block likewise over the valid rows; x = fp32(X) - mean;
 * scale = amax/7; q = clamp(rint(x * (7/amax)), -7, 7) (all fp32, RNE).
 * qk_corr[blk][j] = sum_c q_mean[blk][c] * K[j][c], fp32.
 */
sage2_status sage2_smooth_quant_qk(const void* q, const void* k, int dtype, int B, int H, int N,
                                   int d, uint8_t* q_i4, float* q_scale, float* q_mean,
                                   uint8_t* k_i4, float* k_scale, float* k_mean, float* qk_corr,
                                   sage2_stream_t stream);

/* As sage2_smooth_quant_qk with the payload format chosen by `qk_format`
 * (sage2_qk_format; SAGE2_ERR_INVALID_ARG otherwise).  INT8: scale = amax/127,
 * q = clamp(rint(x * (127/amax)), -127, 127) as int8 bytes.
 * qk_format may carry the flag SAGE2_QK_CAUSAL_CORR (OR-ed in): qk_corr is then
 * written only where a causal attention reads it, i.e. qk_corr[blk][j] for key
 * tiles j/128 <= blk, in whole 32-block groups (at least those entries are
 * written; the others keep what the buffer held).  sage2_attn_fwd does the
 * same for causal calls. */
#define SAGE2_QK_CAUSAL_CORR 0x100
sage2_status sage2_smooth_quant_qk_ex(const void* q, const void* k, int dtype, int B, int H, int N,
                                      int d, uint8_t* q_i4, float* q_scale, float* q_mean,
                                      uint8_t* k_i4, float* k_scale, float* k_mean,
                                      float* qk_corr, int qk_format, sage2_stream_t stream);

/*
 * FP8 e4m3 quantization of V with one scale per channel (Abstract: FP8 V).
 *   v        : [B,H,N,d] in `dtype`.
 *   v_fp8_t  : [B,H,d,Np] e4m3 codes, token-contiguous in the permuted order
 *              of each 128-token block given above; pad tokens are 0.
 *   v_scale  : [B,H,d] = amax_c/448 (0 for an all-zero channel).
 * Codes are RNE of fp32(V * (448/amax_c)) with saturation to +-448.
 */
sage2_status sage2_quant_v(const void* v, int dtype, int B, int H, int N, int d,
                           uint8_t* v_fp8_t, float* v_scale, sage2_stream_t stream);

/*
 * As sage2_quant_v, with V smoothing when v_mean is not NULL ("smooth V",
 * ainnect.com/research/55 summary of SageAttention2): v_mean [B,H,d] receives
 * the per-channel token mean of V (the fixed fp32 order of the K mean), and the
 * codes and scales are those of fp32(V) - v_mean.  The attention adds v_mean
 * back to O (sage2_attn_fwd_quantized_ex).  v_mean must be 16-byte aligned.
 */
sage2_status sage2_quant_v_ex(const void* v, int dtype, int B, int H, int N, int d,
                              uint8_t* v_fp8_t, float* v_scale, float* v_mean,
                              sage2_stream_t stream);

/*
 * Attention over the quantized payloads (the fused tcgen05 kernel alone).
 * (Abstract: INT4 QK^T; FP8 P~V with two-level accumulation.)
 *   o       : [B,H,N,d] written in `o_dtype` (SAGE2_F16, SAGE2_BF16 or SAGE2_F32).
 *   causal  : 0 or 1.   sm_scale : softmax scale (> 0, finite).
 * Per 128-key tile, in ascending order, with L = sm_scale*log2(e):
 *   x = (q_scale_i*k_scale_j*S_ij + qk_corr[blk(i)][j]) * L,  S = q_i4 . k_i4 (exact)
 *   running max m, p = exp2(x - m), l += p, P~ = e4m3(448 p),
 *   inner = P~ . V~ over the tile (fresh fp32 accumulator),
 *   acc = alpha*acc + inner (alpha = exp2(m_old - m_new));  O = acc*v_scale/(448 l).
 */
sage2_status sage2_attn_fwd_quantized(const uint8_t* q_i4, const float* q_scale,
                                      const uint8_t* k_i4, const float* k_scale,
                                      const float* qk_corr, const uint8_t* v_fp8_t,
                                      const float* v_scale, void* o, int o_dtype, int B, int H,
                                      int N, int d, int causal, float sm_scale,
                                      sage2_stream_t stream);

/* As sage2_attn_fwd_quantized for payloads in `qk_format`, and with
 * O = acc*v_scale/(448 l) + v_mean when v_mean is not NULL (V smoothed by
 * sage2_quant_v_ex). */
sage2_status sage2_attn_fwd_quantized_ex(const uint8_t* q_i4, const float* q_scale,
                                         const uint8_t* k_i4, const float* k_scale,
                                         const float* qk_corr, const uint8_t* v_fp8_t,
                                         const float* v_scale, const float* v_mean, void* o,
                                         int o_dtype, int B, int H, int N, int d, int causal,
                                         float sm_scale, int qk_format, sage2_stream_t stream);

/*
 * The whole forward pass: smoothing + quantization of Q, K, V, the correction
 * and the attention kernel, with the payloads in a workspace that the library
 * takes from its own stream-ordered memory pool and returns on `stream`
 * (sage2_workspace_bytes() tells how much).
 *   q, k, v : [B,H,N,d] in `dtype` (SAGE2_F16 / SAGE2_BF16);  o in `o_dtype`.
 * Returns SAGE2_ERR_NO_MEM when the pool cannot provide the workspace.
 */
sage2_status sage2_attn_fwd(const void* q, const void* k, const void* v, void* o, int B, int H,
                            int N, int d, int dtype, int o_dtype, int causal, float sm_scale,
                            sage2_stream_t stream);

/* The whole forward pass with the variants: qk_format (sage2_qk_format) and
 * smooth_v (0 or 1: V smoothing, see sage2_quant_v_ex).  sage2_attn_fwd is
 * this call with SAGE2_QK_INT4 and smooth_v = 0. */
sage2_status sage2_attn_fwd_ex(const void* q, const void* k, const void* v, void* o, int B,
                               int H, int N, int d, int dtype, int o_dtype, int causal,
                               float sm_scale, int qk_format, int smooth_v,
                               sage2_stream_t stream);

/*
 * The same forward pass as sage2_attn_fwd, for callers that must not have the
 * library allocate device memory while they run (hosts that forbid allocator
 * calls after start-up, frameworks that account for every device byte
 * themselves).  The paper has no counterpart: this is a deployment variant.
 * Scratch comes from one fixed 64 MiB device array that every GPU loading the
 * library holds until exit; no cudaMalloc/cudaFree/pool call is made.
 *   - Problems with sage2_workspace_bytes() > 64 MiB return SAGE2_ERR_TOO_LARGE
 *     before any launch.
 *   - The first call on a device looks the array's address up
 *     (cudaGetSymbolAddress) and caches it: make it before any stream capture.
 *   - All calls share the array; each clears what must start at zero.  Calls
 *     whose GPU work overlaps race on it: order them on one stream.
 *   - The cached address belongs to the device's context: after a
 *     cudaDeviceReset of that device it is stale, and the library (this entry
 *     and its memory pools alike) must not be called on that device again.
 * Arguments, layouts and other statuses as sage2_attn_fwd.
 */
sage2_status sage2_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, int B,
                                    int H, int N, int d, int dtype, int o_dtype, int causal,
                                    float sm_scale, sage2_stream_t stream);

/*
 * Variable-length (packed) sequences: the forward pass of sage2_attn_fwd_ex
 * applied to each of S sequences packed along the token axis.  The method's
 * package names such an entry ("sageattn_varlen", codewithpapers page, code
 * samples list); the pages give no more, so each sequence is treated as its
 * own batch element: it attends only within itself (causal: top-left inside
 * the sequence) and gets its own K mean, Q block means, scales, correction and
 * per-channel V scales.
 *   q, k, v, o  : HEAD-MAJOR packed [H, T, d] (q/k/v in `dtype`, o in `o_dtype`);
 *                 sequence s is tokens cu_seqlens[s] .. cu_seqlens[s+1]-1.
 *   cu_seqlens  : HOST int32 array of S+1 offsets, cu_seqlens[0] = 0,
 *                 non-decreasing, cu_seqlens[S] = T (empty sequences allowed).
 * The sequences run on four library-owned streams, or up to eight while their
 * workspaces total at most 4 GiB (longest first, each to the least-loaded one),
 * each with its own workspace for the longest sequence (from the library's
 * pool, as sage2_attn_fwd), forked from and joined back into
 * `stream` with events: the call is ordered on `stream` like any other.  Calls
 * on one device are serialised on the host while they enqueue.  Other arguments
 * and statuses as sage2_attn_fwd_ex; a malformed cu_seqlens is
 * SAGE2_ERR_INVALID_ARG.
 */
sage2_status sage2_attn_fwd_varlen(const void* q, const void* k, const void* v, void* o,
                                   const int* cu_seqlens, int S, int H, int T, int d, int dtype,
                                   int o_dtype, int causal, float sm_scale, int qk_format,
                                   int smooth_v, sage2_stream_t stream);

/*
 * The forward pass of sage2_attn_fwd_ex over HOST tensors: q, k, v, o are host
 * pointers ([B,H,N,d] as sage2_attn_fwd), PINNED (cudaHostAlloc /
 * cudaHostRegister) for the copies to overlap; other host memory still works,
 * with the copies serialised by the driver.  Whole heads are copied in, run
 * and copied back in chunks (about 48 MB of inputs each) on up to four
 * library streams forked from and joined back into `stream`, so the copies of
 * some chunks overlap the kernels of others.  Device buffers for the chunks in
 * flight come from the library's pool.  The call returns once everything is
 * enqueued: o is complete when `stream` reaches that point.  Statuses as
 * sage2_attn_fwd_ex (pointers are only checked for NULL).
 */
sage2_status sage2_attn_fwd_host(const void* q, const void* k, const void* v, void* o, int B,
                                 int H, int N, int d, int dtype, int o_dtype, int causal,
                                 float sm_scale, int qk_format, int smooth_v,
                                 sage2_stream_t stream);

/* Bytes of workspace sage2_attn_fwd takes for this problem (0 on bad sizes). */
size_t sage2_workspace_bytes(int B, int H, int N, int d);

/*
 * Test entry: the raw integer products S = q_i4 . k_i4^T of every 128x128
 * tile, through the same TMA + tcgen05 FP8 (kind::f8f6f4, fp32 accumulator)
 * path as the attention kernel, converted to int32 (the fp32 sums are exact
 * integers for INT4 operands).
 *   s_out : int32 [B,H,Np,Np] (caller-allocated).  Column j holds the product with
 *           stored k_i4 row j (so, with the permuted k_i4 layout, key
 *           32*((j%128/2)%4) + 2*((j%128)/8) + j%2 of block j/128).
 */
sage2_status sage2_debug_qk_s32(const uint8_t* q_i4, const uint8_t* k_i4, int B, int H, int N,
                                int d, int32_t* s_out, sage2_stream_t stream);

/* As sage2_debug_qk_s32 for payloads in `qk_format`; INT8 payloads go through
 * the attention kernel's 8-bit integer path (tcgen05 kind::i8, s32). */
sage2_status sage2_debug_qk_s32_ex(const uint8_t* q_i4, const uint8_t* k_i4, int B, int H, int N,
                                   int d, int qk_format, int32_t* s_out, sage2_stream_t stream);

/*
 * Test entry for failure detection: launches one thread that waits on an
 * mbarrier phase nothing completes.  The wait is bounded (about one second):
 * it gives up, sets the device error word (SAGE2_ERR_TIMEOUT on the next
 * sage2_check_device_error) and the kernel returns normally, so the context
 * stays usable.  Every wait of the library's kernels behaves the same way.
 */
sage2_status sage2_debug_wait_timeout(sage2_stream_t stream);

/*
 * Synchronizes `stream`, then reads and clears the device error word that
 * kernels set instead of trapping.  SAGE2_ERR_TIMEOUT if a bounded wait ran
 * out, SAGE2_ERR_CUDA on a sticky CUDA error, else SAGE2_OK.
 * After SAGE2_ERR_TIMEOUT the outputs of the work enqueued since the last
 * check are invalid (a block that gave up left its rows unwritten); the
 * context stays usable and the call may simply be repeated.  A wait gives up
 * after about one second of wall time, which a healthy launch can exceed only
 * if the GPU stops running it for that long (for example a long preemption by
 * another context on a shared GPU).
 */
sage2_status sage2_check_device_error(sage2_stream_t stream);

/*
 * The layout constants of the payloads and of the method as this library
 * implements them, for callers that produce or consume payloads themselves
 * (and for tests that check them).  Fills *out; SAGE2_ERR_INVALID_ARG if out
 * is NULL.  Host only; launches nothing.
 */
typedef struct {
  int version;           /* sage2_version() */
  int block_rows;        /* query rows per smoothing block and per attention tile (128) */
  int tile_keys;         /* keys per attention tile: the inner accumulation block (128) */
  int int4_max;          /* INT4 range [-7, 7] */
  int int8_max;          /* INT8 variant range [-127, 127] */
  float p_scale;         /* P~ = e4m3(p_scale * p) */
  float v_scale_div;     /* v_scale = amax / v_scale_div */
  int packed_low_first;  /* SAGE2_QK_INT4_PACKED: channel 2c in bits 3:0 of byte c */
  int key_perm[128];     /* stored k_i4 row n of a 128-row block holds token key_perm[n] */
  int value_perm[128];   /* v_fp8_t byte p of a 128-token block holds token value_perm[p] */
} sage2_layout;
sage2_status sage2_layout_info(sage2_layout* out);

/* Static description of a status code (never NULL). */
const char* sage2_status_string(sage2_status status);

/* Library version: major*10000 + minor*100 + patch. */
int sage2_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SAGE2_H_ */
