"""The plain C oracle (oracle/sage2_oracle.c, the CPU baseline's timed
program) pinned to the numpy oracle and to the hand-worked golden values:
payloads bit for bit, the fp64 correction and output to 1e-12."""
import math

import numpy as np
import pytest

from oracle import c_oracle as corc
from oracle import sage2_oracle as orc
from tests.test_oracle_pins import _golden, scenario_a, scenario_b


@pytest.fixture(scope="module", autouse=True)
def _built():
    corc.build()


def _inputs(N, d, seed):
    rng = np.random.default_rng(seed)
    Q = (rng.standard_normal((N, d)) + rng.normal(0, 1, d)).astype(np.float32)
    K = (rng.standard_normal((N, d)) * rng.uniform(0.5, 3, d) + rng.normal(0, 3, d)).astype(np.float32)
    K[:, 3] *= 20
    V = (rng.standard_normal((N, d)) + rng.normal(0, 2, d)).astype(np.float32)
    return Q, K, V


SHAPES = [(1, 64), (7, 128), (129, 64), (300, 128), (513, 64)]


@pytest.mark.parametrize("N,d", SHAPES)
@pytest.mark.parametrize("bits", [4, 8])
def test_payloads_bit_exact(N, d, bits):
    Q, K, V = _inputs(N, d, 10 * N + d + bits)
    a = orc.smooth_quant_qk(Q, K, bits)
    b = corc.smooth_quant_qk(Q, K, bits)
    for n in ("q_i4", "q_scale", "q_mean", "k_i4", "k_scale", "k_mean"):
        x, y = np.ascontiguousarray(a[n]), np.ascontiguousarray(b[n])
        if x.dtype == np.float32:
            x, y = x.view(np.uint32), y.view(np.uint32)
        assert np.array_equal(x, y), n
    vt0, sv0 = orc.quant_v(V)
    vt1, sv1 = corc.quant_v(V)
    assert np.array_equal(vt0, vt1)
    assert np.array_equal(sv0.view(np.uint32), sv1.view(np.uint32))
    C0 = orc.qk_correction(a["q_mean"], K)
    C1 = corc.qk_correction(a["q_mean"], K)
    assert np.allclose(C0, C1, rtol=1e-12, atol=1e-12 * np.abs(C0).max())


@pytest.mark.parametrize("N,d", SHAPES)
@pytest.mark.parametrize("causal", [False, True])
def test_attention_matches_numpy_oracle(N, d, causal):
    Q, K, V = _inputs(N, d, 7 * N + d)
    sm = 1 / math.sqrt(d)
    pay, O, _, rows = orc.sage2_head(Q, K, V, causal, sm)
    got = corc.attn_blocks(pay, N, causal, sm, range(orc.n_pad(N) // 128))
    assert np.abs(got[rows] - O).max() <= 1e-12 * max(1.0, np.abs(O).max())
    whole = corc.sage2_head(Q, K, V, causal, sm)
    assert np.abs(whole - O).max() <= 1e-12 * max(1.0, np.abs(O).max())


def test_v_smoothing_output():
    Q, K, V = _inputs(300, 64, 5)
    pay, O, _, rows = orc.sage2_head(Q, K, V, True, 0.125, smooth_v=True)
    got = corc.attn_blocks(pay, 300, True, 0.125, range(3))
    assert np.abs(got - O).max() <= 1e-12 * np.abs(O).max()


def test_two_tile_recurrence_golden():
    g = _golden()
    O = corc.attn_blocks(scenario_a(), 256, False, 1.0, [0, 1])
    assert np.allclose(O[:, 0::2], g["A_O_even"], rtol=1e-12, atol=0)
    assert np.allclose(O[:, 1::2], g["A_O_odd"], rtol=1e-12, atol=0)
    O = corc.attn_blocks(scenario_b(), 256, False, 1.0, [1, 0])
    assert np.allclose(O[:, 0::2], g["B_O_even"], rtol=1e-12, atol=0)
    assert np.allclose(O[:, 1::2], g["B_O_odd"], rtol=1e-12, atol=0)


def test_uses_openmp_threads():
    assert corc.threads() >= 1


def test_sample_forward_rows():
    """The CPU baseline's unit of work gives the numpy oracle's rows for the
    sampled blocks."""
    Q, K, V = _inputs(700, 128, 3)
    sm = 1 / math.sqrt(128)
    O, ops = corc.sample_forward(Q, K, V, True, sm, [5, 0, 2])
    _, ref, _, rows = orc.sage2_head(Q, K, V, True, sm, q_blocks=[0, 2, 5])
    assert np.abs(O[rows] - ref).max() <= 1e-12 * np.abs(ref).max()
    vis = sum(min(r + 1, 700) for r in rows)
    assert ops == 4.0 * 128 * vis
