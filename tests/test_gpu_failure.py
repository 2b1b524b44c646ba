"""Failure detection on the GPU without a fault: a kernel waits on a barrier
phase that nothing completes.  Its bounded wait must give up, report
SAGE2_ERR_TIMEOUT through the device error word, and leave the context usable
(the next forward pass runs and matches the oracle)."""
import time

import pytest
import torch

from quantized_attention_04_b200.inputs import CONFIGS, make_qkv
from tests import parity as P

pytestmark = pytest.mark.gpu

SAGE2_ERR_TIMEOUT = 6


def test_bounded_wait_reports_timeout_and_context_survives():
    from quantized_attention_04_b200 import build
    build.build()
    import quantized_attention_04_b200 as qa
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    assert qa.sage2_check_device_error() == 0
    t0 = time.time()
    qa.sage2_debug_wait_timeout()
    assert qa.sage2_check_device_error() == SAGE2_ERR_TIMEOUT
    assert time.time() - t0 < 30
    assert qa.sage2_check_device_error() == 0          # the word was cleared
    # the context still works: a forward pass matches the oracle
    cfg = CONFIGS["C1"]
    q, k, v = make_qkv(cfg)
    sm = P.default_scale(cfg.d)
    o = P.np32(qa.sage2_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=cfg.causal, sm_scale=sm,
                                 out_dtype=torch.float32))
    assert qa.sage2_check_device_error() == 0
    pay, O, amb, rows = P.oracle_head(q, k, v, 0, 0, cfg.causal, sm)
    P.assert_o_close(o[0, 0][rows], O, amb, torch.float32, "after timeout",
                     flips=P.head_flips(pay, cfg.N, cfg.causal, sm), rows=rows)
