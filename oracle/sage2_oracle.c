/*
 * Plain C restatement of the CPU oracle for the SageAttention2 quantized
 * attention forward pass, for timing on the host's cores.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__ and bench.py's CPU
 * legs load it.  It shares no code, header, table or helper with the CUDA
 * library: it is a second, independent statement of oracle/sage2_oracle.py
 * (the numpy oracle), to which the tests pin it bit for bit on the payloads
 * and to 1e-12 on the output.
 *
 * The method: "SageAttention2: Efficient Attention with Thorough Outlier
 * Smoothing and Per-thread INT4 Quantization" (arxiv.science abstract page,
 * Abstract): Q and K smoothed and quantized to INT4 (per token here), P~ and V
 * in FP8 e4m3, P~V accumulated in two levels (one 128-key tile in a fresh
 * accumulator, added to the running output).  The same readings as the numpy
 * oracle: fp32 payload steps in a fixed order, fp64 attention, P~ = e4m3(448 p)
 * rounded to nearest even, l summed before rounding, tiles in ascending order,
 * causal top-left.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC (no fast-math: fp32 operations must
 * round as written).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define BM 128
#define BN 128

static int n_pad(int N) { return (N + BM - 1) / BM * BM; }

/* ---------------------------------------------------------------- e4m3
 * 4 exponent bits (bias 7), 3 mantissa bits, no infinity; largest finite 448;
 * subnormals are m * 2^-9.  Round to nearest, ties to even; beyond 448 the
 * value saturates (codes 0x7E / 0xFE). */
static double e4m3_value(uint8_t code) {
  const double s = (code & 0x80) ? -1.0 : 1.0;
  const int e = (code >> 3) & 0xF, m = code & 7;
  if (e == 0) return s * m * ldexp(1.0, -9);
  return s * (1.0 + m / 8.0) * ldexp(1.0, e - 7);
}

static uint8_t e4m3_encode(double x) {
  const uint8_t sign = signbit(x) ? 0x80 : 0x00;
  const double a = fabs(x);
  int code;
  if (a >= 448.0) {
    code = 0x7E;
  } else if (a < ldexp(1.0, -6)) {
    code = (int)nearbyint(a * 512.0);            /* quantum 2^-9; 8 is the first normal */
  } else {
    int E;
    frexp(a, &E);                                /* a = f 2^E, f in [0.5, 1) */
    int e = E - 1;                               /* a in [2^e, 2^(e+1)) */
    double k = nearbyint(ldexp(a, 3 - e));       /* in [8, 16] */
    if (k >= 16.0) {
      e += 1;
      k = 8.0;
    }
    code = ((e + 7) << 3) | ((int)k - 8);
    if (code > 0x7E) code = 0x7E;
  }
  return (uint8_t)(code | sign);
}

/* ---------------------------------------------------------------- payloads */

/* K smoothing's mean: 128-token chunks summed token by token (fp32), chunk
 * sums added in chunk order, one fp32 division by N. */
void orc_token_mean(const float* X, int N, int d, float* out) {
  float* part = (float*)malloc(sizeof(float) * d);
  for (int c = 0; c < d; ++c) out[c] = 0.f;
  for (int c0 = 0; c0 < N; c0 += BN) {
    for (int c = 0; c < d; ++c) part[c] = 0.f;
    const int c1 = c0 + BN < N ? c0 + BN : N;
    for (int j = c0; j < c1; ++j)
      for (int c = 0; c < d; ++c) part[c] = part[c] + X[(size_t)j * d + c];
    for (int c = 0; c < d; ++c) out[c] = out[c] + part[c];
  }
  for (int c = 0; c < d; ++c) out[c] = out[c] / (float)N;
  free(part);
}

/* Q smoothing's means: one per 128-row block over its valid rows. */
void orc_q_block_means(const float* Q, int N, int d, float* out) {
  const int nb = (N + BM - 1) / BM;
  for (int b = 0; b < nb; ++b) {
    const int r0 = b * BM, r1 = (b + 1) * BM < N ? (b + 1) * BM : N;
    float* o = out + (size_t)b * d;
    for (int c = 0; c < d; ++c) o[c] = 0.f;
    for (int i = r0; i < r1; ++i)
      for (int c = 0; c < d; ++c) o[c] = o[c] + Q[(size_t)i * d + c];
    for (int c = 0; c < d; ++c) o[c] = o[c] / (float)(r1 - r0);
  }
}

/* Symmetric per-row quantization on [-qmax, qmax]: scale = amax/qmax,
 * q = rint(x * (qmax/amax)) clamped; an all-zero row gets scale 0, q 0. */
void orc_quant_rows(const float* X, int n, int d, int qmax, int8_t* q, float* scale) {
  for (int i = 0; i < n; ++i) {
    const float* x = X + (size_t)i * d;
    float amax = 0.f;
    for (int c = 0; c < d; ++c) {
      const float a = fabsf(x[c]);
      if (a > amax) amax = a;
    }
    if (!(amax > 0.f)) {
      scale[i] = 0.f;
      memset(q + (size_t)i * d, 0, d);
      continue;
    }
    scale[i] = amax / (float)qmax;
    const float inv = (float)qmax / amax;
    for (int c = 0; c < d; ++c) {
      const float y = x[c] * inv;
      float r = nearbyintf(y);
      if (r > qmax) r = (float)qmax;
      if (r < -qmax) r = (float)-qmax;
      q[(size_t)i * d + c] = (int8_t)r;
    }
  }
}

/* Smoothing + quantization of one head: padded payloads as the numpy oracle
 * returns them (rows >= N zero).  qk_bits 4 (INT4) or 8 (the INT8 variant). */
void orc_smooth_quant_qk(const float* Q, const float* K, int N, int d, int qk_bits,
                         int8_t* q_i, float* q_scale, float* q_mean, int8_t* k_i, float* k_scale,
                         float* k_mean) {
  const int Np = n_pad(N);
  const int qmax = qk_bits == 8 ? 127 : 7;
  float* S = (float*)malloc(sizeof(float) * (size_t)N * d);
  orc_token_mean(K, N, d, k_mean);
  for (int j = 0; j < N; ++j)
    for (int c = 0; c < d; ++c) S[(size_t)j * d + c] = K[(size_t)j * d + c] - k_mean[c];
  memset(k_i, 0, (size_t)Np * d);
  memset(k_scale, 0, sizeof(float) * Np);
  orc_quant_rows(S, N, d, qmax, k_i, k_scale);
  orc_q_block_means(Q, N, d, q_mean);
  for (int i = 0; i < N; ++i)
    for (int c = 0; c < d; ++c)
      S[(size_t)i * d + c] = Q[(size_t)i * d + c] - q_mean[(size_t)(i / BM) * d + c];
  memset(q_i, 0, (size_t)Np * d);
  memset(q_scale, 0, sizeof(float) * Np);
  orc_quant_rows(S, N, d, qmax, q_i, q_scale);
  free(S);
}

/* The Q-smoothing correction C[blk][j] = qbar_blk . K_j in fp64 (0 for j >= N). */
void orc_qk_correction(const float* q_mean, int nb, const float* K, int N, int d, double* C) {
  const int Np = n_pad(N);
  for (int b = 0; b < nb; ++b)
    for (int j = 0; j < Np; ++j) {
      double s = 0.0;
      if (j < N)
        for (int c = 0; c < d; ++c) s += (double)q_mean[(size_t)b * d + c] * (double)K[(size_t)j * d + c];
      C[(size_t)b * Np + j] = s;
    }
}

/* The correction rows of the listed query blocks only (other rows untouched),
 * in parallel over blocks. */
void orc_qk_correction_blocks(const float* q_mean, const int* blocks, int nblocks, const float* K,
                              int N, int d, double* C) {
  const int Np = n_pad(N);
#pragma omp parallel for schedule(dynamic, 1)
  for (int k = 0; k < nblocks; ++k) {
    const int b = blocks[k];
    for (int j = 0; j < Np; ++j) {
      double s = 0.0;
      if (j < N)
        for (int c = 0; c < d; ++c) s += (double)q_mean[(size_t)b * d + c] * (double)K[(size_t)j * d + c];
      C[(size_t)b * Np + j] = s;
    }
  }
}

/* FP8 V, one scale per channel: sv = amax/448, codes = e4m3(V * (448/amax)),
 * stored transposed [d][Np] (pad tokens 0). */
void orc_quant_v(const float* V, int N, int d, uint8_t* vt, float* sv) {
  const int Np = n_pad(N);
  memset(vt, 0, (size_t)d * Np);
  for (int c = 0; c < d; ++c) {
    float amax = 0.f;
    for (int j = 0; j < N; ++j) {
      const float a = fabsf(V[(size_t)j * d + c]);
      if (a > amax) amax = a;
    }
    if (!(amax > 0.f)) {
      sv[c] = 0.f;
      continue;
    }
    sv[c] = amax / 448.f;
    const float inv = 448.f / amax;
    for (int j = 0; j < N; ++j) vt[(size_t)c * Np + j] = e4m3_encode((double)(V[(size_t)j * d + c] * inv));
  }
}

/* ---------------------------------------------------------------- attention */

/* Query block b of one head over its payloads (the numpy oracle's
 * attn_quantized for one block).  O receives the block's valid rows, [rows][d]. */
static void attn_block(const int8_t* q_i, const float* q_scale, const int8_t* k_i,
                       const float* k_scale, const double* C, const uint8_t* vt,
                       const float* v_scale, const float* v_mean, int N, int d, int causal,
                       double sm_scale, int b, double* O) {
  const int Np = n_pad(N), nb = Np / BM;
  const double L = sm_scale * 1.4426950408889634;
  const int r0 = b * BM, r1 = (b + 1) * BM < N ? (b + 1) * BM : N, nr = r1 - r0;
  double* m = (double*)malloc(sizeof(double) * BM);
  double* l = (double*)calloc(BM, sizeof(double));
  double* acc = (double*)calloc((size_t)BM * d, sizeof(double));
  double* x = (double*)malloc(sizeof(double) * BN);
  double* ph = (double*)malloc(sizeof(double) * BN);
  double* vdec = (double*)malloc(sizeof(double) * (size_t)BN * d);
  for (int i = 0; i < nr; ++i) m[i] = -INFINITY;
  const int last = causal ? b : nb - 1;
  for (int t = 0; t <= last; ++t) {
    const int c0 = t * BN;
    for (int j = 0; j < BN; ++j)
      for (int c = 0; c < d; ++c) vdec[(size_t)j * d + c] = e4m3_value(vt[(size_t)c * Np + c0 + j]);
    for (int ii = 0; ii < nr; ++ii) {
      const int i = r0 + ii;
      double tmax = -INFINITY;
      for (int j = 0; j < BN; ++j) {
        const int key = c0 + j;
        if (key >= N || (causal && key > i)) {
          x[j] = -INFINITY;
          continue;
        }
        int64_t s = 0;                                    /* exact integer Q^ . K^ */
        for (int c = 0; c < d; ++c) s += (int64_t)q_i[(size_t)i * d + c] * k_i[(size_t)key * d + c];
        x[j] = ((double)q_scale[i] * (double)k_scale[key] * (double)s + C[(size_t)b * Np + key]) * L;
        if (x[j] > tmax) tmax = x[j];
      }
      const double mn = m[ii] > tmax ? m[ii] : tmax;
      const double alpha = isinf(m[ii]) && m[ii] < 0 ? 0.0 : exp2(m[ii] - mn);
      double psum = 0.0;
      for (int j = 0; j < BN; ++j) {
        const double p = exp2(x[j] - mn);
        psum += p;
        ph[j] = e4m3_value(e4m3_encode(448.0 * p));      /* P~ = e4m3(448 p) */
      }
      l[ii] = alpha * l[ii] + psum;
      double* a = acc + (size_t)ii * d;
      for (int c = 0; c < d; ++c) {
        double inner = 0.0;                               /* inner level: this tile only */
        for (int j = 0; j < BN; ++j) inner += ph[j] * vdec[(size_t)j * d + c];
        a[c] = alpha * a[c] + inner;                      /* outer level */
      }
      m[ii] = mn;
    }
  }
  for (int ii = 0; ii < nr; ++ii)
    for (int c = 0; c < d; ++c)
      O[(size_t)ii * d + c] = acc[(size_t)ii * d + c] * (double)v_scale[c] / (448.0 * l[ii]) +
                              (v_mean ? (double)v_mean[c] : 0.0);
  free(m);
  free(l);
  free(acc);
  free(x);
  free(ph);
  free(vdec);
}

/* The listed query blocks of one head, in parallel over blocks (OpenMP).
 * O: [N][d] fp64; only the rows of the listed blocks are written. */
void orc_attn_blocks(const int8_t* q_i, const float* q_scale, const int8_t* k_i,
                     const float* k_scale, const double* C, const uint8_t* vt,
                     const float* v_scale, const float* v_mean, int N, int d, int causal,
                     double sm_scale, const int* blocks, int nblocks, double* O) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int k = 0; k < nblocks; ++k) {
    const int b = blocks[k];
    attn_block(q_i, q_scale, k_i, k_scale, C, vt, v_scale, v_mean, N, d, causal, sm_scale, b,
               O + (size_t)b * BM * d);
  }
}

/* One whole head (payloads, correction, V, attention over every block): the
 * unit of work the CPU baseline times. */
void orc_sage2_head(const float* Q, const float* K, const float* V, int N, int d, int causal,
                    double sm_scale, int qk_bits, double* O) {
  const int Np = n_pad(N), nb = Np / BM;
  int8_t* q_i = (int8_t*)malloc((size_t)Np * d);
  int8_t* k_i = (int8_t*)malloc((size_t)Np * d);
  float* qs = (float*)malloc(sizeof(float) * Np);
  float* ks = (float*)malloc(sizeof(float) * Np);
  float* qm = (float*)malloc(sizeof(float) * (size_t)nb * d);
  float* km = (float*)malloc(sizeof(float) * d);
  double* C = (double*)malloc(sizeof(double) * (size_t)nb * Np);
  uint8_t* vt = (uint8_t*)malloc((size_t)d * Np);
  float* sv = (float*)malloc(sizeof(float) * d);
  int* blocks = (int*)malloc(sizeof(int) * nb);
  orc_smooth_quant_qk(Q, K, N, d, qk_bits, q_i, qs, qm, k_i, ks, km);
  orc_qk_correction(qm, nb, K, N, d, C);
  orc_quant_v(V, N, d, vt, sv);
  for (int b = 0; b < nb; ++b) blocks[b] = nb - 1 - b;      /* longest first */
  orc_attn_blocks(q_i, qs, k_i, ks, C, vt, sv, NULL, N, d, causal, sm_scale, blocks, nb, O);
  free(q_i); free(k_i); free(qs); free(ks); free(qm); free(km); free(C); free(vt); free(sv);
  free(blocks);
}

int orc_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
