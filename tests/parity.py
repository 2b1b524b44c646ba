"""Helpers shared by the GPU parity tests: run the CPU oracle on the same
seeded inputs, and compare the CUDA path with it.

Tolerances (written here, used by every test):
  * payloads (INT4 values, e4m3 codes, every scale and mean): bit-exact;
  * the correction qk_corr (fp32 on the GPU, fp64 in the oracle): the fp32
    rounding bound of a d-term dot product, d * 2^-24 * sum_c |qbar_c K_c|;
  * O: max-abs <= 2e-3 and relative L1 <= 1e-3 against the quantized oracle,
    after removing the oracle's per-element ambiguity bound (elements whose
    448*p sits within AMBIG_REL of an e4m3 rounding boundary may round either
    way), plus half an ulp of the output dtype for fp16/bf16 outputs.
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


def compare_o(got: np.ndarray, ref: np.ndarray, amb: np.ndarray, out_dtype) -> dict:
    err = np.abs(got.astype(np.float64) - ref)
    excess = np.maximum(err - amb - half_ulp(ref, out_dtype), 0.0)
    stats = dict(max_abs=float(err.max()), max_excess=float(excess.max()),
                 rel_l1=float(excess.sum() / max(np.abs(ref).sum(), 1e-30)),
                 ambiguous=int((amb > 0).sum()))
    return stats


def assert_o_close(got, ref, amb, out_dtype, what=""):
    s = compare_o(got, ref, amb, out_dtype)
    assert s["max_excess"] <= MAX_ABS and s["rel_l1"] <= REL_L1, (what, s)
    return s


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
