"""Planted mistakes: each mutation of the oracle's attention step (made here, on
the CPU, in a throw-away copy of its source) must make the fp64 identity pin
or the single-tile brute-force pin fail.  This shows the pin is able to catch a dropped term, a missing rescale, a
wrong mask, a wrong index or a transposed operand."""
import inspect
import math

import numpy as np
import pytest

from oracle import sage2_oracle as orc
from tests.test_oracle_pins import _identity_payload

MUTATIONS = [
    ("dropped correction term", "+ C[b][c][None, :]) * L", "+ 0 * C[b][c][None, :]) * L"),
    ("missing outer rescale", "acc = alpha[:, None] * acc + inner", "acc = acc + inner"),
    ("missing l rescale", "l = alpha * l + pt.sum(axis=1)", "l = l + pt.sum(axis=1)"),
    ("causal mask off by one", "(c[None, :] > r[:, None])", "(c[None, :] > r[:, None] + 1)"),
    ("wrong correction block", "C[b][c][None, :]", "C[max(b - 1, 0)][c][None, :]"),
    ("sign of max shift", "np.exp2(x - m_new[:, None])", "np.exp2(x + 0 * m_new[:, None] - x.max(axis=1, keepdims=True))"),
    ("transposed key scale", "sk[None, c]", "sk[r, None]"),
]


def _mutant(old, new):
    src = inspect.getsource(orc.attn_quantized)
    assert old in src, old
    ns = dict(vars(orc))
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


def test_unmutated_passes():
    assert _identity_error(orc.attn_quantized, True) < 1e-11
    assert _identity_error(orc.attn_quantized, False) < 1e-11
    assert _single_tile_error(orc.attn_quantized) < 1e-12


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_mutation_is_caught(name, old, new):
    fn = _mutant(old, new)
    worst = max(_identity_error(fn, True), _identity_error(fn, False),
                _single_tile_error(fn))
    assert worst > 1e-6, name
