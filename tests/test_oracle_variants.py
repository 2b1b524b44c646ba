"""Pins of the oracle's two variants (CPU): the INT8 Q/K quantizer and V
smoothing.  Each is pinned against something other than itself: hand-worked
rows, rounding bounds, the fp64 mean, and the identity-quantizer path against
direct fp64 attention (which only holds if vbar is added back)."""
import math
import os

import numpy as np
import pytest

from oracle import sage2_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------- INT8 rows
def test_int8_rows_golden():
    n = 0
    for line in open(os.path.join(GOLDEN, "int8_rows.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        xs, qs, sc = [s.split() for s in line.split("|")]
        x = np.array([float(v) for v in xs], np.float32)[None]
        q, s = orc.quant_int8_rows(x)
        assert q[0].tolist() == [int(v) for v in qs], (xs, q)
        assert s[0] == np.float32(float(sc[0]))
        n += 1
    assert n == 4


def test_int8_bounds_random():
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((500, 128)) * rng.uniform(0.01, 100, (500, 1))).astype(np.float32)
    q, s = orc.quant_int8_rows(x)
    assert np.abs(q.astype(np.int32)).max() <= 127
    err = np.abs(x.astype(np.float64) - q * s[:, None].astype(np.float64))
    assert (err <= s[:, None] * (0.5 + 1e-5)).all()
    arg = np.abs(x).argmax(axis=1)
    assert (np.abs(q[np.arange(500), arg].astype(np.int32)) == 127).all()


def test_smooth_quant_int8_reconstructs_smoothed_rows():
    """The INT8 payloads are the smoothed Q and K to within half a step; the
    means and the correction are those of the INT4 path."""
    rng = np.random.default_rng(12)
    N, d = 300, 64
    Q = (rng.standard_normal((N, d)) + 2).astype(np.float32)
    K = (rng.standard_normal((N, d)) * 3 - 1).astype(np.float32)
    p8 = orc.smooth_quant_qk(Q, K, qk_bits=8)
    p4 = orc.smooth_quant_qk(Q, K, qk_bits=4)
    for key in ("q_mean", "k_mean"):
        assert np.array_equal(p8[key], p4[key])
    blk = np.arange(N) // orc.BM
    Qs = Q.astype(np.float64) - p8["q_mean"].astype(np.float64)[blk]
    Ks = K.astype(np.float64) - p8["k_mean"].astype(np.float64)
    for X, qv, sc in ((Qs, p8["q_i4"][:N], p8["q_scale"][:N]), (Ks, p8["k_i4"][:N], p8["k_scale"][:N])):
        err = np.abs(X - qv * sc[:, None].astype(np.float64))
        assert (err <= sc[:, None] * (0.5 + 1e-4)).all()
    with pytest.raises(ValueError):
        orc.smooth_quant_qk(Q, K, qk_bits=6)


def test_int8_variant_is_more_accurate_than_int4():
    """127 levels against 7: on the same head the INT8 variant's output is much
    closer to fp64 attention."""
    rng = np.random.default_rng(13)
    N, d = 384, 64
    Q = rng.standard_normal((N, d)).astype(np.float32)
    K = (rng.standard_normal((N, d)) * 3).astype(np.float32)
    V = rng.standard_normal((N, d)).astype(np.float32)
    sm = 1 / math.sqrt(d)
    ref = orc.attn_fp64(Q, K, V, False, sm)
    cos = {}
    for bits in (4, 8):
        _, O, _, _ = orc.sage2_head(Q, K, V, False, sm, qk_bits=bits)
        cos[bits] = float((O * ref).sum() / np.linalg.norm(O) / np.linalg.norm(ref))
    assert cos[8] > 0.999 and cos[8] > cos[4]


# ---------------------------------------------------------------- V smoothing
def test_token_mean_close_to_fp64_mean():
    rng = np.random.default_rng(14)
    for N in (1, 129, 1000):
        V = (rng.standard_normal((N, 64)) * 5 + 3).astype(np.float32)
        m = orc.token_mean(V)
        ref = V.astype(np.float64).mean(axis=0)
        assert np.abs(m - ref).max() <= 1e-6 * (np.abs(V).max() + 1)


def test_quant_v_smoothed_codes_the_centred_values():
    rng = np.random.default_rng(15)
    N, d = 300, 64
    V = (rng.standard_normal((N, d)) + rng.standard_normal(d) * 20).astype(np.float32)
    vt, sv, vbar = orc.quant_v_smoothed(V)
    Vs = V.astype(np.float64) - vbar.astype(np.float64)
    dec = orc.e4m3_decode(vt[:, :N]).T * sv[None, :].astype(np.float64)
    # e4m3 keeps 3 mantissa bits: relative error <= 2^-4 above the subnormals
    assert (np.abs(dec - Vs) <= np.abs(Vs) * 2.0 ** -4 + sv * 2.0 ** -9 * 1.01).all()
    assert np.abs(Vs).max(axis=0) == pytest.approx(sv.astype(np.float64) * 448, rel=1e-6)


@pytest.mark.parametrize("N", [1, 130, 300])
@pytest.mark.parametrize("causal", [False, True])
def test_v_smoothing_identity_quant_equals_fp64(N, causal):
    """With the quantizers swapped for the identity, attention over V - vbar
    plus vbar is exactly attention over V: the softmax weights sum to one."""
    rng = np.random.default_rng(300 + N)
    d = 32
    Q = rng.standard_normal((N, d)).astype(np.float32)
    K = (rng.standard_normal((N, d)) * 2).astype(np.float32)
    V = (rng.standard_normal((N, d)) + 7).astype(np.float32)
    sm = 1 / math.sqrt(d)
    pay = orc.smooth_quant_qk(Q, K)
    blk = np.arange(N) // orc.BM
    vbar = orc.token_mean(V)
    p = dict(q_s=Q.astype(np.float64) - pay["q_mean"].astype(np.float64)[blk],
             k_s=K.astype(np.float64) - pay["k_mean"].astype(np.float64),
             v=V.astype(np.float64) - vbar.astype(np.float64), v_mean=vbar,
             C=orc.qk_correction(pay["q_mean"], K))
    O, _, _ = orc.attn_quantized(p, N, causal, sm, quantize=False)
    ref = orc.attn_fp64(Q, K, V, causal, sm)
    assert np.abs(O - ref).max() < 1e-10
    # without adding vbar back the result is off by vbar
    p_bad = dict(p)
    p_bad["v_mean"] = None
    O_bad, _, _ = orc.attn_quantized(p_bad, N, causal, sm, quantize=False)
    assert np.abs(O_bad - ref).max() > 1.0


def test_v_smoothing_helps_offset_v():
    """FP8 V with a large per-channel offset: smoothing recovers accuracy."""
    rng = np.random.default_rng(16)
    N, d = 256, 64
    Q = rng.standard_normal((N, d)).astype(np.float32)
    K = rng.standard_normal((N, d)).astype(np.float32)
    V = (rng.standard_normal((N, d)) + rng.standard_normal(d) * 30).astype(np.float32)
    sm = 1 / math.sqrt(d)
    ref = orc.attn_fp64(Q, K, V, False, sm)
    err = {}
    for sv in (False, True):
        _, O, _, _ = orc.sage2_head(Q, K, V, False, sm, qk_bits=8, smooth_v=sv)
        err[sv] = np.abs(O - ref).mean()
    assert err[True] < 0.5 * err[False]


# ------------------------------------------------------- packed sequences
def test_varlen_equal_lengths_equal_batched_heads():
    """Equal-length packed sequences are exactly the batched fixed-length path,
    one sequence per batch element."""
    rng = np.random.default_rng(17)
    S, N, d = 3, 130, 32
    Q = rng.standard_normal((S * N, d)).astype(np.float32)
    K = (rng.standard_normal((S * N, d)) * 2).astype(np.float32)
    V = rng.standard_normal((S * N, d)).astype(np.float32)
    sm = 1 / math.sqrt(d)
    for causal in (False, True):
        O, amb = orc.sage2_varlen_head(Q, K, V, [0, N, 2 * N, 3 * N], causal, sm)
        for s in range(S):
            sl = slice(s * N, (s + 1) * N)
            _, o, m, rows = orc.sage2_head(Q[sl], K[sl], V[sl], causal, sm)
            assert np.array_equal(O[sl][rows], o) and np.array_equal(amb[sl][rows], m)


def test_varlen_sequences_do_not_see_each_other():
    """Changing one sequence leaves the others' outputs bit-identical, and an
    empty sequence is allowed."""
    rng = np.random.default_rng(18)
    d = 32
    cu = [0, 5, 5, 200, 329]
    T = cu[-1]
    Q = rng.standard_normal((T, d)).astype(np.float32)
    K = rng.standard_normal((T, d)).astype(np.float32)
    V = rng.standard_normal((T, d)).astype(np.float32)
    O1, _ = orc.sage2_varlen_head(Q, K, V, cu, True)
    K2 = K.copy()
    K2[200:] += 5
    V2 = V.copy()
    V2[200:] *= 3
    O2, _ = orc.sage2_varlen_head(Q, K2, V2, cu, True)
    assert np.array_equal(O1[:200], O2[:200])
    assert not np.array_equal(O1[200:], O2[200:])
    with pytest.raises(ValueError):
        orc.sage2_varlen_head(Q, K, V, [0, 10, 5, T], True)
