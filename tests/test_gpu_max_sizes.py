"""GPU parity at the size limits the library accepts: the largest head count
(B*H = 65535, the grid's y limit) with short sequences, and one long causal
head with a ragged tail (N = 2^17 - 77, 1024 query blocks).  Sampled heads and
query blocks against the oracle, payloads of those heads bit-exact."""
import numpy as np
import pytest
import torch

from oracle import sage2_oracle as orc
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qa():
    from quantized_attention_04_b200 import build
    build.build()
    import quantized_attention_04_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    m.lib()
    return m


def _qkv(shape, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn(shape, generator=g, dtype=torch.float32).to(dtype) for _ in range(3)]


def _check(qa, q, k, v, causal, heads, blocks, out_dtype):
    B, H, N, d = q.shape
    sm = P.default_scale(d)
    o = qa.sage2_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, sm_scale=sm,
                          out_dtype=out_dtype)
    pay = qa.sage2_smooth_quant_qk(q.cuda(), k.cuda())
    torch.cuda.synchronize()
    assert qa.sage2_check_device_error() == 0
    for b, h in heads:
        opay, O, amb, rows = P.oracle_head(q, k, v, b, h, causal, sm, q_blocks=blocks)
        lib = dict(opay)
        lib["k_i4"] = lib["k_i4"][P.key_interleave(lib["k_i4"].shape[0])]
        lib["q_i4"], lib["k_i4"] = P.int4_codes(lib["q_i4"]), P.int4_codes(lib["k_i4"])
        for n in ("q_i4", "q_scale", "k_i4", "k_scale", "k_mean"):
            assert P.bits_equal(pay[n][b, h].cpu().numpy(), lib[n]), (n, b, h)
        got = P.np32(o[b, h])[rows]
        assert np.isfinite(got).all()
        P.assert_o_close(got, O, amb, out_dtype, (b, h),
                         flips=P.head_flips(opay, N, causal, sm), rows=rows)


def test_most_heads(qa):
    q, k, v = _qkv((1, 65535, 16, 64), torch.float16, 11)
    _check(qa, q, k, v, False, [(0, 0), (0, 32767), (0, 65534)], None, torch.float32)


def test_long_ragged_causal_head(qa):
    N = (1 << 17) - 77
    q, k, v = _qkv((1, 1, N, 128), torch.bfloat16, 12)
    nb = orc.n_pad(N) // 128
    _check(qa, q, k, v, True, [(0, 0)], [0, nb // 2, nb - 1], torch.bfloat16)
