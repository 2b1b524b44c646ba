"""ctypes binding of oracle/sage2_oracle.c, the plain C restatement of the
CPU oracle (OpenMP over query blocks), used to time the CPU baseline on all
host cores.

TEST INFRASTRUCTURE ONLY, like oracle/sage2_oracle.py: only tests/,
__graft_entry__ and bench.py's CPU legs use it; it shares nothing with the
CUDA library.  build() compiles it with gcc (no fast-math).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "sage2_oracle.c")
LIB = os.path.join(HERE, "libsage2_oracle.so")
BM = 128

_lib = None


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", "-o", LIB + ".tmp", SRC,
               "-lm"]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError("gcc failed:\n" + res.stdout + res.stderr)
        os.replace(LIB + ".tmp", LIB)
    return LIB


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        _lib = ctypes.CDLL(LIB)
        _lib.orc_max_threads.restype = ctypes.c_int
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def n_pad(N: int) -> int:
    return (N + BM - 1) // BM * BM


def threads() -> int:
    """OpenMP threads the oracle runs with (all host cores unless OMP_NUM_THREADS)."""
    return int(lib().orc_max_threads())


def smooth_quant_qk(Q, K, qk_bits: int = 4) -> dict:
    Q = np.ascontiguousarray(Q, np.float32)
    K = np.ascontiguousarray(K, np.float32)
    N, d = Q.shape
    Np = n_pad(N)
    out = dict(q_i4=np.zeros((Np, d), np.int8), q_scale=np.zeros(Np, np.float32),
               q_mean=np.zeros((Np // BM, d), np.float32), k_i4=np.zeros((Np, d), np.int8),
               k_scale=np.zeros(Np, np.float32), k_mean=np.zeros(d, np.float32))
    lib().orc_smooth_quant_qk(_p(Q), _p(K), N, d, qk_bits, _p(out["q_i4"]), _p(out["q_scale"]),
                              _p(out["q_mean"]), _p(out["k_i4"]), _p(out["k_scale"]),
                              _p(out["k_mean"]))
    return out


def qk_correction(q_mean, K) -> np.ndarray:
    q_mean = np.ascontiguousarray(q_mean, np.float32)
    K = np.ascontiguousarray(K, np.float32)
    N, d = K.shape
    C = np.zeros((q_mean.shape[0], n_pad(N)), np.float64)
    lib().orc_qk_correction(_p(q_mean), q_mean.shape[0], _p(K), N, d, _p(C))
    return C


def sample_forward(Q, K, V, causal: bool, sm_scale: float, blocks, qk_bits: int = 4):
    """The CPU baseline's unit of work: one head's payloads (smoothing and
    quantization of Q and K over the whole head, FP8 V), then the correction
    rows and the attention of the listed query blocks, the blocks in
    parallel.  Returns (O [N, d] with the listed blocks' rows, ops), ops being
    the metric's count for those rows: 4 d per (query, visible key)."""
    Q = np.ascontiguousarray(Q, np.float32)
    K = np.ascontiguousarray(K, np.float32)
    N, d = Q.shape
    Np = n_pad(N)
    blocks = [int(b) for b in blocks]
    pay = smooth_quant_qk(Q, K, qk_bits)
    pay["v_t"], pay["v_scale"] = quant_v(V)
    C = np.zeros((Np // BM, Np), np.float64)
    blk = np.ascontiguousarray(np.asarray(blocks, np.int32))
    lib().orc_qk_correction_blocks(_p(pay["q_mean"]), _p(blk), len(blk), _p(K), N, d, _p(C))
    pay["C"] = C
    O = attn_blocks(pay, N, causal, sm_scale, blocks)
    ops = 0.0
    for b in blocks:
        rows = np.arange(b * BM, min((b + 1) * BM, N))
        vis = (rows + 1) if causal else np.full(rows.size, N)
        ops += 4.0 * d * float(vis.sum())
    return O, ops


def quant_v(V):
    V = np.ascontiguousarray(V, np.float32)
    N, d = V.shape
    vt = np.zeros((d, n_pad(N)), np.uint8)
    sv = np.zeros(d, np.float32)
    lib().orc_quant_v(_p(V), N, d, _p(vt), _p(sv))
    return vt, sv


def attn_blocks(p: dict, N: int, causal: bool, sm_scale: float, blocks) -> np.ndarray:
    """Rows of the listed query blocks (O [N, d], other rows 0) over payloads
    p (q_i4, q_scale, k_i4, k_scale, C, v_t, v_scale, optional v_mean)."""
    d = p["q_i4"].shape[1]
    O = np.zeros((n_pad(N), d), np.float64)
    blk = np.ascontiguousarray(np.asarray(list(blocks), np.int32))
    arrs = [np.ascontiguousarray(p[n]) for n in ("q_i4", "q_scale", "k_i4", "k_scale")]
    C = np.ascontiguousarray(p["C"], np.float64)
    vt = np.ascontiguousarray(p["v_t"], np.uint8)
    sv = np.ascontiguousarray(p["v_scale"], np.float32)
    vm = p.get("v_mean")
    vm = None if vm is None else np.ascontiguousarray(vm, np.float32)
    lib().orc_attn_blocks(_p(arrs[0]), _p(arrs[1]), _p(arrs[2]), _p(arrs[3]), _p(C), _p(vt), _p(sv),
                          None if vm is None else _p(vm), N, d, int(bool(causal)),
                          ctypes.c_double(sm_scale), _p(blk), len(blk), _p(O))
    return O[:N]


def sage2_head(Q, K, V, causal: bool, sm_scale: float | None = None, qk_bits: int = 4) -> np.ndarray:
    """A whole head: payloads, correction, V, attention over every query block."""
    Q = np.ascontiguousarray(Q, np.float32)
    K = np.ascontiguousarray(K, np.float32)
    V = np.ascontiguousarray(V, np.float32)
    N, d = Q.shape
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    O = np.zeros((n_pad(N), d), np.float64)
    lib().orc_sage2_head(_p(Q), _p(K), _p(V), N, d, int(bool(causal)), ctypes.c_double(sm_scale),
                         qk_bits, _p(O))
    return O[:N]
