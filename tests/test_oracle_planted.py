"""Planted mistakes: each mutation of the oracle's attention step (made here, on
the CPU, in a throw-away copy of its source) must make one of its pins fail:
the fp64 identity pin, the single-tile brute-force pin, or the hand-worked
two-tile golden values (the quantized multi-tile recurrence and the list of
ambiguous codes).  This shows the pins catch a dropped term, a missing
rescale, a wrong mask, a wrong index, a transposed operand, P~ rounded on the
wrong tiles or against the wrong maximum, and a wrong flip list."""
import inspect
import math

import numpy as np
import pytest

from oracle import sage2_oracle as orc
from tests.test_oracle_pins import _golden, _identity_payload, scenario_a, scenario_b

MUTATIONS = [
    ("dropped correction term", "+ C[b][c][None, :]) * L", "+ 0 * C[b][c][None, :]) * L"),
    ("missing outer rescale", "acc = alpha[:, None] * acc + inner", "acc = acc + inner"),
    ("missing l rescale", "l = alpha * l + pt.sum(axis=1)", "l = l + pt.sum(axis=1)"),
    ("causal mask off by one", "(c[None, :] > r[:, None])", "(c[None, :] > r[:, None] + 1)"),
    ("wrong correction block", "C[b][c][None, :]", "C[max(b - 1, 0)][c][None, :]"),
    ("sign of max shift", "np.exp2(x - m_new[:, None])", "np.exp2(x + 0 * m_new[:, None] - x.max(axis=1, keepdims=True))"),
    ("transposed key scale", "sk[None, c]", "sk[r, None]"),
    ("P~ rounded only on tile 0", "ph = e4m3_round(E4M3_MAX * pt)",
     "ph = e4m3_round(E4M3_MAX * pt) if t == 0 else E4M3_MAX * pt"),
    ("P~ rounded against the final row max", "ph = e4m3_round(E4M3_MAX * pt)",
     "_mf = _final_max(p, N, causal, sm_scale, b, r); "
     "ph = e4m3_round(E4M3_MAX * np.exp2(x - _mf[:, None])) * np.exp2(_mf - m_new)[:, None]"),
    ("flip of an earlier tile not rescaled", "flips[k] = [f * alpha[k] for f in flips[k]]",
     "flips[k] = list(flips[k])"),
    ("ambiguity band ignored", "lo, hi = e4m3_neighbours(E4M3_MAX * pt, rel)",
     "lo, hi = e4m3_neighbours(E4M3_MAX * pt, 0.0)"),
]


def _final_max(p, N, causal, sm_scale, b, r):
    """The row maxima over every visible key of block b (for the mutation
    that rounds P~ against the final maximum)."""
    L = sm_scale * orc.LOG2E
    Np = orc.n_pad(N)
    c = np.arange(Np)
    S = np.asarray(p["q_i4"], np.float64)[r] @ np.asarray(p["k_i4"], np.float64).T
    x = (np.asarray(p["q_scale"], np.float64)[r, None] * np.asarray(p["k_scale"], np.float64)[None]
         * S + np.asarray(p["C"], np.float64)[b][None]) * L
    mask = c[None, :] >= N
    if causal:
        mask = mask | (c[None, :] > r[:, None])
    return np.where(mask, -np.inf, x).max(axis=1)


def _mutant(old, new):
    src = inspect.getsource(orc.attn_quantized)
    assert old in src, old
    ns = dict(vars(orc))
    ns["_final_max"] = _final_max
    exec(src.replace(old, new), ns)
    return ns["attn_quantized"]


def _identity_error(fn, causal):
    rng = np.random.default_rng(77)
    N, d = 300, 64
    Q = (rng.standard_normal((N, d)) + rng.normal(0, 1, d)).astype(np.float32)
    K = (rng.standard_normal((N, d)) * rng.uniform(0.5, 2, d) + rng.normal(0, 3, d)).astype(np.float32)
    V = rng.standard_normal((N, d)).astype(np.float32)
    sm = 1 / math.sqrt(d)
    with np.errstate(all="ignore"):
        O, _, _ = fn(_identity_payload(Q, K, V), N, causal, sm, quantize=False)
        ref = orc.attn_fp64(Q, K, V, causal, sm)
        err = np.abs(O - ref).max()
    return err if np.isfinite(err) else np.inf


def _single_tile_error(fn):
    """The single-tile brute-force pin, with the real INT4/e4m3 scales."""
    rng = np.random.default_rng(78)
    N, d = 100, 64
    Q = rng.standard_normal((N, d)).astype(np.float32)
    K = (rng.standard_normal((N, d)) * rng.uniform(0.2, 3, (N, 1)) + 2).astype(np.float32)
    V = (rng.standard_normal((N, d)) + 1).astype(np.float32)
    sm = 1 / math.sqrt(d)
    pay = orc.smooth_quant_qk(Q, K)
    pay["C"] = orc.qk_correction(pay["q_mean"], K)
    pay["v_t"], pay["v_scale"] = orc.quant_v(V)
    S = orc.qk_int(pay["q_i4"][:N], pay["k_i4"][:N])
    x = (pay["q_scale"][:N, None].astype(np.float64) * pay["k_scale"][None, :N] * S
         + pay["C"][0][:N][None, :]) * sm * orc.LOG2E
    p = np.exp2(x - x.max(1, keepdims=True))
    vh = orc.e4m3_decode(pay["v_t"][:, :N]).T * pay["v_scale"][None, :]
    ref = (orc.e4m3_round(448 * p) @ vh) / (448 * p.sum(1, keepdims=True))
    with np.errstate(all="ignore"):
        O, _, _ = fn(pay, N, False, sm)
        err = np.abs(O - ref).max()
    return err if np.isfinite(err) else np.inf


def _golden_error(fn):
    """Largest relative error against the two hand-worked golden cases,
    including the flip list of the second."""
    g = _golden()
    with np.errstate(all="ignore"):
        O, _, _ = fn(scenario_a(), 256, False, 1.0)
        errs = [np.abs(O[:, 0::2] / g["A_O_even"] - 1).max(), np.abs(O[:, 1::2] / g["A_O_odd"] - 1).max()]
        O, _, _, fl = fn(scenario_b(), 256, False, 1.0, explain_rows=[0])
        errs += [np.abs(O[:, 0::2] / g["B_O_even"] - 1).max()]
        f = fl[0]
        if f.shape != (1, O.shape[1]):
            return np.inf
        errs += [np.abs(f[0, 0::2] / g["B_delta_even"] - 1).max(),
                 np.abs(f[0, 1::2] / g["B_delta_odd"] - 1).max()]
    err = max(errs)
    return err if np.isfinite(err) else np.inf


def test_unmutated_passes():
    assert _identity_error(orc.attn_quantized, True) < 1e-11
    assert _identity_error(orc.attn_quantized, False) < 1e-11
    assert _single_tile_error(orc.attn_quantized) < 1e-12
    assert _golden_error(orc.attn_quantized) < 1e-12


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_mutation_is_caught(name, old, new):
    fn = _mutant(old, new)
    worst = max(_identity_error(fn, True), _identity_error(fn, False),
                _single_tile_error(fn), _golden_error(fn))
    assert worst > 1e-6, name
