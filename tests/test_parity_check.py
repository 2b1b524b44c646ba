"""The O comparison of the GPU parity tests (tests/parity.py), checked on the
CPU: a result that differs from the oracle by a legitimate alternative
rounding of an ambiguous P~ code is accepted, and nothing else that exceeds
the tolerance is."""
import numpy as np
import torch

from oracle import sage2_oracle as orc
from tests import parity as P
from tests.test_oracle_pins import scenario_b


def _case():
    pay = scenario_b()
    O, amb, rows = orc.attn_quantized(pay, 256, False, 1.0)
    return pay, O, amb, rows, P.head_flips(pay, 256, False, 1.0)


def test_exact_result_passes_without_flips():
    pay, O, amb, rows, flips = _case()
    s = P.compare_o(O.astype(np.float32), O, amb, torch.float32, flips, rows)
    assert s["rows_over"] == 0 and s["flips_used"] == 0 and not s["unexplained"]


def test_the_other_rounding_is_explained():
    pay, O, amb, rows, flips = _case()
    delta = flips([5])[5][0]
    got = O.copy()
    got[5] += delta                                   # row 5 took the other rounding
    s = P.compare_o(got, O, amb, torch.float32, flips, rows)
    assert s["rows_over"] == 1 and s["flips_used"] == 1 and not s["unexplained"]
    assert s["rel_l1"] < 1e-3


def test_errors_no_flip_explains_are_rejected():
    pay, O, amb, rows, flips = _case()
    delta = flips([5])[5][0]
    for wrong in (2 * delta, -delta, np.roll(delta, 1), np.full_like(delta, 3e-3)):
        got = O.copy()
        got[5] += wrong
        s = P.compare_o(got, O, amb, torch.float32, flips, rows)
        assert s["unexplained"] == [5], wrong[:4]
    # with no flip list, the same legitimate rounding is not accepted
    got = O.copy()
    got[5] += delta
    assert P.compare_o(got, O, amb, torch.float32, None, rows)["unexplained"] == [5]


def test_half_ulp_of_the_output_type_is_not_an_error():
    pay, O, amb, rows, flips = _case()
    ref = O * 4.7                                       # |O| ~ 4: bf16 ulp 2^-5
    got = torch.from_numpy(ref).to(torch.bfloat16).float().numpy()
    s = P.compare_o(got, ref, amb, torch.bfloat16, flips, rows)
    assert s["max_abs"] > 2e-3 and s["rows_over"] == 0
    assert s["rel_l1"] == 0.0


def test_explain_row_picks_the_needed_subset():
    rng = np.random.default_rng(4)
    f = rng.standard_normal((12, 32)) * 0.05
    diff = f[2] + f[7] + f[9]
    ok, n = P.explain_row(diff, f, np.full(32, 1e-9))
    assert ok and n == 3
    ok, _ = P.explain_row(diff + 0.01, f, np.full(32, 1e-3))
    assert not ok
