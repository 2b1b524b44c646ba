"""Helpers shared by the GPU parity tests: run the CPU oracle on the same
seeded inputs, and compare the CUDA path with it.

Tolerances (written here, used by every test):
  * payloads (INT4 values, e4m3 codes, every scale and mean): bit-exact;
  * the correction qk_corr (fp32 on the GPU, fp64 in the oracle): the fp32
    rounding bound of a d-term dot product, d * 2^-24 * sum_c |qbar_c K_c|;
  * O: relative L1 <= 1e-3 against the quantized oracle, on the raw
    difference (only the output type's own rounding, half an ulp for
    fp16/bf16 outputs, is taken off each element); and max-abs <= 2e-3 per
    element, where a row that exceeds it passes only if rounding some of its
    ambiguous P~ codes to their other neighbour (codes whose 448p lies within
    the kernel's fp32 error bound of an e4m3 rounding boundary, see
    oracle.p448_band) brings every element of the row within 2e-3.  The
    flips are chosen one at a time from the oracle's list for that row; the
    number used is reported.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from oracle import sage2_oracle as orc

MAX_ABS = 2e-3
REL_L1 = 1e-3


def np32(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float32).cpu().numpy()


def oracle_head(q, k, v, b, h, causal, sm_scale, q_blocks=None, qk_bits=4, smooth_v=False):
    """Oracle payloads and output rows of head (b, h); q/k/v are [B,H,N,d]."""
    Q, K, V = np32(q[b, h]), np32(k[b, h]), np32(v[b, h])
    pay, O, amb, rows = orc.sage2_head(Q, K, V, causal, sm_scale, q_blocks=q_blocks,
                                       qk_bits=qk_bits, smooth_v=smooth_v)
    return pay, O, amb, rows


def half_ulp(x: np.ndarray, dtype: torch.dtype) -> np.ndarray:
    if dtype == torch.float32:
        return np.zeros_like(x)
    mant = 7 if dtype == torch.bfloat16 else 10
    a = np.maximum(np.abs(x), 2.0 ** -14)
    return 0.5 * 2.0 ** (np.floor(np.log2(a)) - mant)


def explain_row(diff: np.ndarray, flips: np.ndarray, tol: np.ndarray):
    """Greedy search for a set of flips (rows of `flips`, each used at most
    once) whose sum brings every element of diff - sum within tol.  Returns
    (explained, number of flips used)."""
    res = diff.astype(np.float64).copy()
    free = np.ones(len(flips), bool)

    def cost(r):
        return np.sum(np.maximum(np.abs(r) - tol, 0.0) ** 2, axis=-1)

    cur = cost(res)
    used = 0
    while cur > 0:
        if not free.any():
            return False, used
        cand = np.nonzero(free)[0]
        costs = cost(res[None, :] - flips[cand])
        k = int(np.argmin(costs))
        if costs[k] >= cur:
            return False, used
        res = res - flips[cand[k]]
        free[cand[k]] = False
        cur = costs[k]
        used += 1
    return True, used


def compare_o(got: np.ndarray, ref: np.ndarray, amb: np.ndarray, out_dtype, flips=None,
              rows=None) -> dict:
    """got, ref: [n, d].  flips: callable(list of row ids) -> {row id: [k, d]}
    (the oracle's alternative roundings, oracle.flips_of_rows); rows: the row
    id of each of the n rows (default 0..n-1)."""
    got64 = got.astype(np.float64)
    err = np.abs(got64 - ref)
    ulp = half_ulp(np.maximum(np.abs(ref), np.abs(got64)), out_dtype)
    excess = np.maximum(err - ulp, 0.0)
    over_rows = np.nonzero((excess > MAX_ABS).any(axis=1))[0]
    rows = np.arange(len(ref)) if rows is None else np.asarray(rows)
    stats = dict(max_abs=float(err.max(initial=0.0)), max_excess=float(excess.max(initial=0.0)),
                 rel_l1=float(excess.sum() / max(np.abs(ref).sum(), 1e-30)),
                 elems_over=int((excess > MAX_ABS).sum()), rows_over=int(len(over_rows)),
                 flips_used=0, unexplained=[], amb_max=float(amb.max(initial=0.0)))
    if len(over_rows):
        table = flips([int(rows[i]) for i in over_rows]) if flips is not None else {}
        for i in over_rows:
            f = table.get(int(rows[i]), np.zeros((0, ref.shape[1])))
            ok, n = explain_row(got64[i] - ref[i], f, MAX_ABS + ulp[i])
            stats["flips_used"] += n
            if not ok:
                stats["unexplained"].append(int(rows[i]))
    return stats


def assert_o_close(got, ref, amb, out_dtype, what="", flips=None, rows=None):
    s = compare_o(got, ref, amb, out_dtype, flips, rows)
    assert s["rel_l1"] <= REL_L1 and not s["unexplained"], (what, s)
    return s


def head_flips(pay, N, causal, sm_scale):
    """The flips callable of compare_o for one head of the oracle."""
    return lambda rows: orc.flips_of_rows(pay, N, causal, sm_scale, rows)


def varlen_flips(pays, causal, sm_scale):
    """The flips callable for one head of packed sequences: pays is the list
    of (first token, length, payload) that oracle.sage2_varlen_head returns;
    row ids are packed token indices."""
    def flips(rows):
        out = {}
        for a, n, pay in pays:
            mine = [r - a for r in rows if a <= r < a + n]
            if mine:
                for r, f in orc.flips_of_rows(pay, n, causal, sm_scale, mine).items():
                    out[r + a] = f
        return out
    return flips


def cosine(a: np.ndarray, b: np.ndarray) -> float:
    a = a.astype(np.float64).ravel()
    b = b.astype(np.float64).ravel()
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))


def corr_tolerance(q_mean: np.ndarray, K: np.ndarray, Np: int, d: int) -> np.ndarray:
    """Rounding bound of the fp32 correction: d * 2^-24 * sum_c |qbar_c K_c|."""
    mag = np.zeros((q_mean.shape[0], Np))
    mag[:, :K.shape[0]] = np.abs(q_mean.astype(np.float64)) @ np.abs(K.astype(np.float64)).T
    return d * 2.0 ** -24 * mag + 1e-30


def bits_equal(a: np.ndarray, b: np.ndarray) -> bool:
    a = np.ascontiguousarray(a)
    b = np.ascontiguousarray(b)
    if a.dtype == np.float32:
        return np.array_equal(a.view(np.uint32), b.astype(np.float32).view(np.uint32))
    return np.array_equal(a, b)


def int4_codes(i) -> np.ndarray:
    """The library stores each INT4 value as its e4m3 code: the oracle's
    integers encoded with the oracle's own (pinned) e4m3 codec."""
    return orc.e4m3_encode(np.asarray(i, np.float64))


def pack_int4(values) -> np.ndarray:
    """The library's packed INT4 layout (SAGE2_QK_INT4_PACKED): [..., d] INT4
    values -> [..., d/2] bytes, channel 2c in bits 3:0 and 2c+1 in bits 7:4 of
    byte c, each a two's-complement nibble."""
    v = np.asarray(values, np.int64) & 0xF
    return (v[..., 0::2] | (v[..., 1::2] << 4)).astype(np.uint8)


def int4_values(codes) -> np.ndarray:
    """INT4 values back from the library's e4m3 codes (must be integers in [-7, 7])."""
    v = orc.e4m3_decode(np.asarray(codes, np.uint8))
    assert np.array_equal(v, np.rint(v)) and np.abs(v).max(initial=0) <= 7
    return v.astype(np.int8)


def key_interleave(Np: int) -> np.ndarray:
    """Index map of the library's permuted k_i4 row order: stored row n of each
    128-row block holds token 32*((n//2) % 4) + 2*(n//8) + n % 2 of that block,
    so stored = natural[key_interleave(Np)]."""
    n = np.arange(Np)
    blk, j = n // 128, n % 128
    return blk * 128 + 32 * ((j // 2) % 4) + 2 * (j // 8) + j % 2


def value_interleave(Np: int) -> np.ndarray:
    """Index map of the library's permuted v_fp8_t token order: byte p of each
    128-token block holds token sigma(p) of that block, sigma swapping the
    2-bit fields [6:5] and [4:3] of p, so stored = natural[:, value_interleave(Np)]."""
    n = np.arange(Np)
    blk, j = n // 128, n % 128
    return blk * 128 + 32 * ((j // 8) % 4) + 8 * ((j // 32) % 4) + j % 8


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
