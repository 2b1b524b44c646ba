"""CPU oracle for the SageAttention2 quantized attention forward pass.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` (its CPU-baseline / reference leg) may import this module.  The
product path (the CUDA library and its Python binding) never calls it and shares
no code, header, table or helper with it.

What it computes.  "SageAttention2: Efficient Attention with Thorough Outlier
Smoothing and Per-thread INT4 Quantization" (arxiv.science abstract page,
Abstract) describes the method in four moves: Q and K are quantized to INT4 at a
fine per-thread granularity, P~ and V to FP8, Q is smoothed to make the INT4
QK^T accurate, and P~V is accumulated in two levels.  K smoothing (subtracting
the token mean of K, which softmax ignores) is the "outlier smoothing" of the
title, inherited from the predecessor "SageAttention: Accurate 8-Bit Attention"
(ainnect.com/research/19 summary).  The method is an approximation, so this
oracle takes its steps in that order, one function per step, with the plainest
reading wherever the pages are silent (every reading is listed in the module
constants and in the function docstrings):

  1. k_mean            K smoothing: token mean of K per channel.
  2. q_block_means     Q smoothing: mean of each 128-row block of Q.
  3. quant_int4_rows   INT4 on [-7, 7], one scale per token (row).
  4. qk_correction     the fp32 correction  qbar_blk . K_j  that Q smoothing
                       subtracted (row constant qbar.kbar dropped).
  5. quant_v           FP8 e4m3 V, one scale per channel.
  6. attn_quantized    INT4 QK^T (exact integers), online softmax over 128-key
                       tiles, P~ to e4m3 with the fixed scale 448, P~V summed
                       per tile (inner level) then added to the running output
                       (outer level).
  7. attn_fp64         the unquantized reference  softmax(QK^T * sm_scale) V.

Two variants beyond the abstract's method, both readings fixed before any
kernel was written:
  - INT8 Q/K (quant_int8_rows): the predecessor's 8-bit integer quantization
    ("SageAttention: Accurate 8-Bit Attention", ainnect.com/research/19
    summary) on [-127, 127], one scale per token, with everything else of the
    path unchanged (smoothing, correction, FP8 P~V, two-level accumulation).
  - V smoothing (token_mean, quant_v_smoothed): subtract the per-channel token
    mean of V before FP8 and add it back to O ("smooth V" in the SageAttention2
    summary, ainnect.com/research/55).  The softmax weights of a row sum to one,
    so sum_j p_j (V_j - vbar) / l + vbar is the same attention output.

Precision.  Steps 1-3 and 5 produce the payloads (the integers, codes and
scales the kernels also produce); they are written in float32 with a fixed
operation order so that they are reproducible bit for bit.  Steps 4, 6 and 7
are done in float64 (exact products of the quantized values, fp64 sums).

Parity pins (tests/test_oracle_*.py): e4m3 codec against the format's code
table and torch's converter; INT4 ties and bounds; means against fp64; the
Q-smoothing reconstruction and the K-smoothing shift invariance in fp64; the
online-softmax/tiling path with the quantizers swapped for the identity against
direct fp64 attention; single-tile brute force; the N=1 and uniform-attention
closed forms.  End-to-end accuracy against the paper is "parity unpinned": the
pages print no accuracy numbers.
"""
from __future__ import annotations

import math
import numpy as np

BM = 128            # rows of Q per smoothing block / per attention tile
BN = 128            # keys per attention tile (the "inner" accumulation block)
INT4_MAX = 7        # symmetric INT4 range [-7, 7]
INT8_MAX = 127      # symmetric INT8 range [-127, 127] (the INT8 variant)
E4M3_MAX = 448.0    # largest finite e4m3 value; also the fixed P~ scale
LOG2E = 1.4426950408889634

# Several correct results.  The decision that turns p into a code, e4m3(448 p),
# is taken by the kernel in fp32: x' = sq*(sk*S) + C with C itself an fp32 dot
# product, the running maximum of x', the argument x'*L - m*L + log2(448) and a
# hardware exp2 approximation.  Where 448 p lies closer to an e4m3 rounding
# boundary than the kernel's fp32 error can reach, either neighbouring code is
# a correct result.  p448_band() bounds that error element by element; the
# constants are the fp32 unit roundoff and the exp2 approximation's relative
# error bound (ex2.approx.f32 is specified to a few ulp; 2^-21 covers 8 ulp).
U32 = 2.0 ** -24
EX2_REL = 2.0 ** -21
LOG2_448 = math.log2(448.0)


def n_pad(N: int) -> int:
    return ((N + BM - 1) // BM) * BM


# ----------------------------------------------------------------------------
# FP8 e4m3 ("e4m3fn": 4 exponent bits, bias 7, 3 mantissa bits, no infinity,
# S.1111.111 is NaN, largest finite 448, smallest subnormal 2^-9).  Written from
# the format definition; rounding is to nearest, ties to even, and values beyond
# the largest finite magnitude saturate to +-448 (the "satfinite" behaviour).
# ----------------------------------------------------------------------------

def e4m3_value_table() -> np.ndarray:
    """float64 value of each of the 256 codes (NaN for the two NaN codes)."""
    vals = np.empty(256, np.float64)
    for code in range(256):
        s = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            vals[code] = np.nan
        elif e == 0:
            vals[code] = s * m * 2.0 ** -9
        else:
            vals[code] = s * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


_E4M3_VALUES = e4m3_value_table()


def e4m3_encode(x) -> np.ndarray:
    """Round finite values to e4m3 codes (RNE, saturating). Returns uint8."""
    x = np.asarray(x, np.float64)
    a = np.abs(x)
    sign = (np.signbit(x)).astype(np.uint8) << 7
    code = np.zeros(a.shape, np.int64)
    sub = a < 2.0 ** -6
    # subnormal range: quantum 2^-9; k = 8 rounds up into the first normal code
    k_sub = np.rint(a * 2.0 ** 9)
    code = np.where(sub, k_sub.astype(np.int64), code)
    # normal range: quantum 2^(e-3) with e = floor(log2 a)
    _, E = np.frexp(np.where(sub, 1.0, a))
    e = E - 1
    k = np.rint(np.ldexp(np.where(sub, 1.0, a), 3 - e))       # in [8, 16]
    carry = k >= 16
    e = np.where(carry, e + 1, e)
    k = np.where(carry, 8, k)
    code_n = ((e + 7) << 3) | (k.astype(np.int64) - 8)
    code = np.where(sub, code, code_n)
    code = np.where(a >= E4M3_MAX, 0x7E, code)
    code = np.minimum(code, 0x7E)
    return (code.astype(np.uint8) | sign).astype(np.uint8)


def e4m3_decode(codes) -> np.ndarray:
    return _E4M3_VALUES[np.asarray(codes, np.uint8)]


def e4m3_round(x) -> np.ndarray:
    """x rounded to the nearest e4m3 value (float64)."""
    return e4m3_decode(e4m3_encode(x))


def e4m3_neighbours(y, rel):
    """For y >= 0 and a relative error bound rel (array or scalar): the e4m3
    values that y*(1-rel) and y*(1+rel) round to.  They differ exactly where
    an error of that size can move y across a rounding boundary."""
    y = np.asarray(y, np.float64)
    return e4m3_round(y * (1.0 - rel)), e4m3_round(y * (1.0 + rel))


def p448_band(A, X, M, e_m, c_bound, L):
    """Relative bound on how far the kernel's fp32 value of 448*p can be from
    the exact 448*exp2(L*(X - M)), element by element.

    A = sq_i*sk_j*S_ij and X = A + C_j (the unscaled score) in fp64; M the
    exact running row maximum of X; c_bound the bound on the kernel's fp32
    error in C_j; e_m the bound on the error of the kernel's running maximum
    (the largest score error among the keys the row has seen).  With u the
    fp32 unit roundoff, the kernel's score carries |x' - X| <= u(2|A| + |X|) +
    c_bound (one rounding of sk*S, one of the fused multiply-add); its
    argument x'L - mL + log2 448 adds the error of the maximum, the fp32
    rounding of L (two roundings), and three roundings of values of the size
    of L|X|, L|M|, the argument and log2 448.  exp2 turns an argument error
    e into a relative error 2^e - 1 <= ln2 e (1 + e); its hardware
    approximation adds EX2_REL.  The result is widened by 2^-20 for the
    neglected second-order terms."""
    e_x = U32 * (2.0 * np.abs(A) + np.abs(X)) + c_bound
    arg = L * (X - M[:, None]) + LOG2_448
    nb = LOG2_448 - L * M
    darg = (L * (e_x + e_m[:, None])
            + 2.0 * U32 * L * (np.abs(X) + 2.0 * np.abs(M)[:, None])
            + U32 * (np.abs(nb)[:, None] + np.abs(arg) + 9.0))
    return (math.log(2.0) * darg * (1.0 + darg) + EX2_REL) * (1.0 + 2.0 ** -20)


# ----------------------------------------------------------------------------
# Step 1 - K smoothing: kbar[c] = (1/N) sum_j K[j, c].
# Reading (fixed order, so the payloads are reproducible): float32 sums, each
# 128-token chunk summed token by token in ascending order starting at 0, then
# the chunk sums added one after another in chunk order starting at 0, then one
# IEEE float32 division by N.
# ----------------------------------------------------------------------------

def k_mean(K: np.ndarray) -> np.ndarray:
    """K: [N, d] (any float dtype; converted exactly to float32) -> [d] float32."""
    K = np.asarray(K, np.float32)
    N, d = K.shape
    total = np.zeros(d, np.float32)
    for c0 in range(0, N, BN):
        part = np.zeros(d, np.float32)
        for j in range(c0, min(c0 + BN, N)):
            part = part + K[j]
        total = total + part
    return (total / np.float32(N)).astype(np.float32)


# ----------------------------------------------------------------------------
# Step 2 - Q smoothing: one mean per block of BM consecutive query rows.
# Reading: float32 sum over the block's valid rows in ascending order starting
# at 0, divided (IEEE float32) by the number of valid rows.
# ----------------------------------------------------------------------------

def q_block_means(Q: np.ndarray) -> np.ndarray:
    """Q: [N, d] -> qbar [ceil(N/BM), d] float32."""
    Q = np.asarray(Q, np.float32)
    N, d = Q.shape
    nb = (N + BM - 1) // BM
    out = np.zeros((nb, d), np.float32)
    for b in range(nb):
        r0, r1 = b * BM, min(N, (b + 1) * BM)
        acc = np.zeros(d, np.float32)
        for i in range(r0, r1):
            acc = acc + Q[i]
        out[b] = acc / np.float32(r1 - r0)
    return out


# ----------------------------------------------------------------------------
# Step 3 - INT4 quantization, one scale per token (per row of d channels).
# Reading of the per-thread granularity for the Blackwell MMA layout: every
# accumulator row (a query) and every accumulator column (a key) carries its
# own scale.  scale = amax/7 and inv = 7/amax (float32 IEEE), q = RNE(x*inv)
# clamped to [-7, 7]; an all-zero row gets scale 0 and q = 0.
# ----------------------------------------------------------------------------

def quant_int4_rows(X: np.ndarray):
    """X: [n, d] float32 -> (q int8 [n, d], scale float32 [n])."""
    X = np.asarray(X, np.float32)
    amax = np.max(np.abs(X), axis=1)
    nz = amax > 0
    safe = np.where(nz, amax, np.float32(1.0)).astype(np.float32)
    scale = np.where(nz, safe / np.float32(INT4_MAX), np.float32(0)).astype(np.float32)
    inv = (np.float32(INT4_MAX) / safe).astype(np.float32)
    y = (X * inv[:, None]).astype(np.float32)
    q = np.clip(np.rint(y), -INT4_MAX, INT4_MAX).astype(np.int8)
    q[~nz] = 0
    return q, scale


def quant_int8_rows(X: np.ndarray):
    """The INT8 variant: X [n, d] float32 -> (q int8 [n, d], scale float32 [n]).
    scale = amax/127 and inv = 127/amax (float32 IEEE), q = RNE(x*inv)
    clamped to [-127, 127]; an all-zero row gets scale 0 and q = 0."""
    X = np.asarray(X, np.float32)
    amax = np.max(np.abs(X), axis=1)
    nz = amax > 0
    safe = np.where(nz, amax, np.float32(1.0)).astype(np.float32)
    scale = np.where(nz, safe / np.float32(INT8_MAX), np.float32(0)).astype(np.float32)
    inv = (np.float32(INT8_MAX) / safe).astype(np.float32)
    y = (X * inv[:, None]).astype(np.float32)
    q = np.clip(np.rint(y), -INT8_MAX, INT8_MAX).astype(np.int8)
    q[~nz] = 0
    return q, scale


def smooth_quant_qk(Q: np.ndarray, K: np.ndarray, qk_bits: int = 4):
    """One head. Q, K: [N, d]. Returns the padded payloads:
    q_i4 [Np, d] int8, q_scale [Np] f32, q_mean [Np/BM, d] f32,
    k_i4 [Np, d] int8, k_scale [Np] f32, k_mean [d] f32.  Rows >= N are 0.
    qk_bits = 4 (the method: INT4 values) or 8 (the INT8 variant; the integer
    payloads then hold values in [-127, 127] under the same keys)."""
    if qk_bits not in (4, 8):
        raise ValueError("qk_bits must be 4 or 8")
    quant = quant_int4_rows if qk_bits == 4 else quant_int8_rows
    Q = np.asarray(Q, np.float32)
    K = np.asarray(K, np.float32)
    N, d = Q.shape
    Np = n_pad(N)
    kbar = k_mean(K)
    Ks = (K - kbar[None, :]).astype(np.float32)
    qbar = q_block_means(Q)
    Qs = (Q - np.repeat(qbar, BM, axis=0)[:N]).astype(np.float32)
    q_i4 = np.zeros((Np, d), np.int8)
    k_i4 = np.zeros((Np, d), np.int8)
    q_scale = np.zeros(Np, np.float32)
    k_scale = np.zeros(Np, np.float32)
    q_i4[:N], q_scale[:N] = quant(Qs)
    k_i4[:N], k_scale[:N] = quant(Ks)
    return dict(q_i4=q_i4, q_scale=q_scale, q_mean=qbar, k_i4=k_i4,
                k_scale=k_scale, k_mean=kbar)


# ----------------------------------------------------------------------------
# Step 4 - Q-smoothing correction.  Q K_s^T = Q_s K_s^T + qbar_blk K_s^T; the
# second term is added back in floating point.  Reading: it is formed with the
# raw K (qbar . K_j); the difference qbar.kbar is constant along each row and
# softmax ignores it.
# ----------------------------------------------------------------------------

def qk_correction(q_mean: np.ndarray, K: np.ndarray) -> np.ndarray:
    """q_mean [nb, d] f32, K [N, d] -> C [nb, Np] float64 (0 beyond N)."""
    K = np.asarray(K, np.float64)
    N = K.shape[0]
    C = np.zeros((q_mean.shape[0], n_pad(N)), np.float64)
    C[:, :N] = np.asarray(q_mean, np.float64) @ K.T
    return C


def qk_correction_bound(q_mean: np.ndarray, K: np.ndarray) -> np.ndarray:
    """The worst-case rounding error of C computed as an fp32 dot product of d
    terms: d * u * sum_c |qbar_c K_jc| (u = 2^-24), shape as qk_correction."""
    K = np.asarray(K, np.float64)
    N, d = K.shape
    Cb = np.zeros((q_mean.shape[0], n_pad(N)), np.float64)
    Cb[:, :N] = d * U32 * (np.abs(np.asarray(q_mean, np.float64)) @ np.abs(K).T)
    return Cb


# ----------------------------------------------------------------------------
# Step 5 - V to FP8 e4m3, one scale per channel over all tokens.
# Reading: sv = amax/448, inv = 448/amax (float32 IEEE), code = e4m3(V*inv)
# rounded to nearest even with saturation; an all-zero channel gets sv = 0.
# The codes are stored transposed, [d, Np] (token-contiguous), pad tokens 0.
# ----------------------------------------------------------------------------

def quant_v(V: np.ndarray):
    """V: [N, d] -> (v_t codes uint8 [d, Np], v_scale f32 [d])."""
    V = np.asarray(V, np.float32)
    N, d = V.shape
    amax = np.max(np.abs(V), axis=0)
    nz = amax > 0
    safe = np.where(nz, amax, np.float32(1.0)).astype(np.float32)
    sv = np.where(nz, safe / np.float32(E4M3_MAX), np.float32(0)).astype(np.float32)
    inv = (np.float32(E4M3_MAX) / safe).astype(np.float32)
    y = (V * inv[None, :]).astype(np.float32)
    codes = e4m3_encode(y)
    codes[:, ~nz] = 0
    vt = np.zeros((d, n_pad(N)), np.uint8)
    vt[:, :N] = codes.T
    return vt, sv


def token_mean(V: np.ndarray) -> np.ndarray:
    """V smoothing's per-channel mean: the same fixed-order float32 token mean
    as k_mean (128-token chunks, chunk sums in order, one division by N)."""
    return k_mean(V)


def quant_v_smoothed(V: np.ndarray):
    """The V-smoothing variant: vbar = token_mean(V), then quant_v of
    V - vbar (float32).  Returns (v_t codes [d, Np], v_scale [d], vbar [d])."""
    V = np.asarray(V, np.float32)
    vbar = token_mean(V)
    vt, sv = quant_v((V - vbar[None, :]).astype(np.float32))
    return vt, sv, vbar


# ----------------------------------------------------------------------------
# Step 6 - attention over the quantized payloads.
# ----------------------------------------------------------------------------

def qk_int(q_i4: np.ndarray, k_i4: np.ndarray) -> np.ndarray:
    """Exact integer Q^ K^T (int64): the INT4 (or INT8-variant) matrix product."""
    # fp64 matmul of small integers is exact (|sum| <= 127^2*d << 2^53)
    return (np.asarray(q_i4, np.float64) @ np.asarray(k_i4, np.float64).T).astype(np.int64)


def attn_quantized(p: dict, N: int, causal: bool, sm_scale: float,
                   q_blocks=None, quantize: bool = True, explain_rows=None):
    """Online-softmax attention of one head over its payloads.

    p: dict with q_i4, q_scale, k_i4, k_scale, C (qk_correction), v_t, v_scale
       and optionally C_bound (the bound on the kernel's fp32 error in C, same
       shape as C; 0 when absent) and v_mean (V smoothing).  With
       quantize=False: 'q_s' / 'k_s' float rows replace q_i4*q_scale /
       k_i4*k_scale and 'v' [N, d] replaces the e4m3 V; P~ is not rounded.
    q_blocks: iterable of 128-row query block indices to compute (default all).
    Returns (O [rows, d] float64, amb [rows, d] float64, rows index array);
    with explain_rows (a collection of row indices) also a dict row ->
    array [k, d]: the change of that output row that each of its k ambiguous
    P~ codes would make if it were rounded to its other neighbour.

    Per query block and for key tiles in ascending order (causal: tiles above
    the diagonal skipped; masked scores are -inf), with L = sm_scale*log2(e):
        x    = (sq_i sk_j S_ij + C_blk,j) * L
        m'   = max(m, rowmax x);   alpha = exp2(m - m')   (0 when m = -inf)
        p    = exp2(x - m');       l = alpha*l + sum_j p  (p before rounding)
        P~   = e4m3(448 p)
        inner= P~ . V~  over this tile only              (inner level)
        acc  = alpha*acc + inner                          (outer level)
    then O = acc * sv / (448 l), plus p['v_mean'] when V was smoothed.
    A code is ambiguous when the kernel's fp32 error bound (p448_band) can
    move 448p across a rounding boundary; 'amb' is the sum of what all of a
    row's ambiguous codes could change (a diagnostic: the parity tests ask
    for the flips that explain a difference, one by one).
    """
    Np = n_pad(N)
    nb = Np // BM
    L = sm_scale * LOG2E
    if quantize:
        qv = np.asarray(p["q_i4"], np.float64)
        kv = np.asarray(p["k_i4"], np.float64)
        sq = np.asarray(p["q_scale"], np.float64)
        sk = np.asarray(p["k_scale"], np.float64)
        vdec = e4m3_decode(p["v_t"]).T            # [Np, d] decoded codes
        sv = np.asarray(p["v_scale"], np.float64)
    else:
        qv = np.zeros((Np, p["q_s"].shape[1])); qv[:N] = p["q_s"]
        kv = np.zeros((Np, p["k_s"].shape[1])); kv[:N] = p["k_s"]
        sq = np.ones(Np); sk = np.ones(Np)
        vdec = np.zeros((Np, p["v"].shape[1])); vdec[:N] = p["v"]
        sv = np.ones(vdec.shape[1])
    C = np.asarray(p["C"], np.float64)
    cbound = np.asarray(p["C_bound"], np.float64) if p.get("C_bound") is not None else np.zeros_like(C)
    d = vdec.shape[1]
    vbar = np.asarray(p["v_mean"], np.float64) if p.get("v_mean") is not None else np.zeros(d)
    blocks = range(nb) if q_blocks is None else q_blocks
    want = set(int(i) for i in explain_rows) if explain_rows is not None else set()
    outs, ambs, rows, expl = [], [], [], {}
    for b in blocks:
        r = np.arange(b * BM, min((b + 1) * BM, N))
        if r.size == 0:
            continue
        m = np.full(r.size, -np.inf)
        l = np.zeros(r.size)
        acc = np.zeros((r.size, d))
        amb = np.zeros((r.size, d))
        e_m = np.zeros(r.size)
        track = [k for k, i in enumerate(r) if int(i) in want]
        flips = {k: [] for k in track}                # per tracked row: flip vectors (acc units)
        last = b if causal else nb - 1
        for t in range(last + 1):
            c = np.arange(t * BN, (t + 1) * BN)
            S = qv[r] @ kv[c].T                                   # exact
            A = sq[r, None] * sk[None, c] * S
            x = (A + C[b][c][None, :]) * L
            mask = c[None, :] >= N
            if causal:
                mask = mask | (c[None, :] > r[:, None])
            x = np.where(mask, -np.inf, x)
            m_new = np.maximum(m, x.max(axis=1))
            alpha = np.where(np.isneginf(m), 0.0, np.exp2(m - m_new))
            pt = np.exp2(x - m_new[:, None])
            l = alpha * l + pt.sum(axis=1)
            if quantize:
                ph = e4m3_round(E4M3_MAX * pt)
                # the kernel's fp32 error bound, element by element
                X = np.where(mask, 0.0, x / L)
                cb = np.where(mask, 0.0, cbound[b][c][None, :])
                e_m = np.maximum(e_m, np.max(U32 * (2.0 * np.abs(A) + np.abs(X)) + cb, axis=1))
                rel = p448_band(np.where(mask, 0.0, A), X, m_new / L, e_m, cb, L)
                lo, hi = e4m3_neighbours(E4M3_MAX * pt, rel)
                gap = hi - lo
            else:
                ph, gap = pt, np.zeros_like(pt)
            inner = ph @ vdec[c]                                  # inner level
            acc = alpha[:, None] * acc + inner                    # outer level
            amb = alpha[:, None] * amb + gap @ np.abs(vdec[c])
            for k in track:
                flips[k] = [f * alpha[k] for f in flips[k]]
                for j in np.nonzero(gap[k] > 0)[0]:
                    other = hi[k, j] if ph[k, j] == lo[k, j] else lo[k, j]
                    flips[k].append((other - ph[k, j]) * vdec[c[j]])
            m = m_new
        scale = E4M3_MAX if quantize else 1.0
        outs.append(acc * sv[None, :] / (scale * l[:, None]) + vbar[None, :])
        ambs.append(amb * sv[None, :] / (scale * l[:, None]))
        rows.append(r)
        for k in track:
            f = np.array(flips[k]).reshape(-1, d)
            expl[int(r[k])] = f * sv[None, :] / (scale * l[k])
    if not outs:
        O, amb, rows = np.zeros((0, d)), np.zeros((0, d)), np.zeros(0, np.int64)
    else:
        O, amb, rows = np.concatenate(outs), np.concatenate(ambs), np.concatenate(rows)
    if explain_rows is not None:
        return O, amb, rows, expl
    return O, amb, rows


# ----------------------------------------------------------------------------
# Step 7 - the unquantized reference.
# ----------------------------------------------------------------------------

def attn_fp64(Q, K, V, causal: bool, sm_scale: float, rows=None) -> np.ndarray:
    """softmax(Q K^T sm_scale) V in float64, top-left causal mask (j <= i)."""
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    N = Q.shape[0]
    rows = np.arange(N) if rows is None else np.asarray(rows)
    s = (Q[rows] @ K.T) * sm_scale
    if causal:
        s = np.where(np.arange(N)[None, :] > rows[:, None], -np.inf, s)
    s = s - s.max(axis=1, keepdims=True)
    w = np.exp(s)
    return (w @ V) / w.sum(axis=1, keepdims=True)


# ----------------------------------------------------------------------------
# The whole pipeline for one head.
# ----------------------------------------------------------------------------

def sage2_head(Q, K, V, causal: bool, sm_scale: float | None = None, q_blocks=None,
               qk_bits: int = 4, smooth_v: bool = False):
    """Steps 1-6 for one head.  Q, K, V: [N, d] (fp16/bf16 values as float32).
    qk_bits 4 (the method) or 8 (the INT8 variant); smooth_v selects the V
    smoothing variant.  Returns (payload dict, O rows, amb rows, row index)."""
    Q = np.asarray(Q, np.float32)
    K = np.asarray(K, np.float32)
    V = np.asarray(V, np.float32)
    N, d = Q.shape
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    pay = smooth_quant_qk(Q, K, qk_bits)
    pay["C"] = qk_correction(pay["q_mean"], K)
    pay["C_bound"] = qk_correction_bound(pay["q_mean"], K)
    if smooth_v:
        pay["v_t"], pay["v_scale"], pay["v_mean"] = quant_v_smoothed(V)
    else:
        pay["v_t"], pay["v_scale"] = quant_v(V)
    O, amb, rows = attn_quantized(pay, N, causal, sm_scale, q_blocks=q_blocks)
    return pay, O, amb, rows


def flips_of_rows(pay: dict, N: int, causal: bool, sm_scale: float, rows) -> dict:
    """For the given output rows of a head whose payloads are `pay` (as
    sage2_head returns them): row -> [k, d] array, the change of the row that
    each of its k ambiguous P~ codes makes when rounded to its other
    neighbour (see attn_quantized)."""
    rows = [int(i) for i in rows]
    blocks = sorted({i // BM for i in rows})
    return attn_quantized(pay, N, causal, sm_scale, q_blocks=blocks, explain_rows=rows)[3]


# ----------------------------------------------------------------------------
# Variable-length (packed) sequences.  The method's package names a varlen
# entry ("sageattn_varlen", codewithpapers page, code samples list) and the
# pages give no more.  Reading: each packed sequence is its own batch element:
# attention within the sequence only, and every step above (means, scales,
# correction, V scales) computed per sequence.
# ----------------------------------------------------------------------------

def sage2_varlen_head(Q, K, V, cu_seqlens, causal: bool, sm_scale: float | None = None,
                      qk_bits: int = 4, smooth_v: bool = False, with_payloads: bool = False):
    """One head of packed sequences: Q, K, V [T, d]; cu_seqlens [S+1] offsets.
    Returns (O [T, d] float64, amb [T, d] float64); with_payloads also returns
    the list of (first token, length, payload dict) of the non-empty sequences."""
    Q = np.asarray(Q, np.float32)
    T, d = Q.shape
    cu = [int(c) for c in cu_seqlens]
    if cu[0] != 0 or cu[-1] != T or any(b < a for a, b in zip(cu, cu[1:])):
        raise ValueError("cu_seqlens must rise from 0 to T")
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    O = np.zeros((T, d))
    amb = np.zeros((T, d))
    pays = []
    for a, b in zip(cu, cu[1:]):
        if b == a:
            continue
        pay, o, m, rows = sage2_head(Q[a:b], K[a:b], V[a:b], causal, sm_scale,
                                     qk_bits=qk_bits, smooth_v=smooth_v)
        O[a + rows] = o
        amb[a + rows] = m
        pays.append((a, b - a, pay))
    if with_payloads:
        return O, amb, pays
    return O, amb
