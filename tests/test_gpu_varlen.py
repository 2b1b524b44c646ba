"""GPU parity of packed variable-length sequences (sage2_attn_fwd_varlen)
against the oracle's per-sequence definition, through the C ABI.  Tolerances
as every parity test (tests/parity.py)."""
import numpy as np
import pytest
import torch

from oracle import sage2_oracle as orc
from quantized_attention_04_b200.inputs import Config, Dist, make_qkv
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


def packed(T, H, d, dtype, idx, voff=1.0):
    """Seeded inputs of the usual distributions, head-major packed [H, T, d]."""
    cfg = Config(f"varlen_T{T}", 1, H, T, d, False, dtype, q=Dist(1.0),
                 k=Dist(3.0, outliers=2, outlier_scale=8.0), v=Dist(voff), index=idx)
    q, k, v = make_qkv(cfg)
    return q[0], k[0], v[0], cfg.torch_dtype


CASES = [
    ([0, 1, 130, 130, 430, 1458], 3, 64, "fp16", True, 4, False),
    ([0, 1, 130, 130, 430, 1458], 2, 128, "bf16", False, 4, False),
    ([0, 300, 427, 555, 1000], 2, 128, "bf16", True, 8, True),
    ([0, 640, 641, 700], 2, 64, "fp16", False, 4, True),
]


@pytest.mark.parametrize("cu,H,d,dtype,causal,qk_bits,smooth_v", CASES)
def test_varlen_matches_oracle(qa, cu, H, d, dtype, causal, qk_bits, smooth_v):
    T = cu[-1]
    q, k, v, tdt = packed(T, H, d, dtype, idx=50 + len(cu) + d)
    sm = P.default_scale(d)
    o = qa.sage2_attn_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cu, causal=causal, sm_scale=sm,
                                 out_dtype=torch.float32, qk_bits=qk_bits, smooth_v=smooth_v)
    torch.cuda.synchronize()
    assert qa.sage2_check_device_error() == 0
    o = P.np32(o)
    for h in range(H):
        O, amb, pays = orc.sage2_varlen_head(P.np32(q[h]), P.np32(k[h]), P.np32(v[h]), cu,
                                             causal, sm, qk_bits=qk_bits, smooth_v=smooth_v,
                                             with_payloads=True)
        P.assert_o_close(o[h], O, amb, torch.float32, (cu, h),
                         flips=P.varlen_flips(pays, causal, sm))


def test_varlen_equal_lengths_equal_batched_call(qa):
    """S equal sequences give bit for bit the batched call on [S, H, N, d]."""
    S, H, N, d = 3, 2, 300, 128
    q, k, v, tdt = packed(S * N, H, d, "bf16", idx=60)
    cu = [0, N, 2 * N, 3 * N]
    sm = P.default_scale(d)
    o_var = qa.sage2_attn_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cu, causal=True, sm_scale=sm,
                                     out_dtype=torch.float32)
    # [H, S*N, d] -> [S, H, N, d]
    to_b = lambda t: t.reshape(H, S, N, d).permute(1, 0, 2, 3).contiguous().cuda()
    o_b = qa.sage2_attn_fwd(to_b(q), to_b(k), to_b(v), causal=True, sm_scale=sm,
                            out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(o_var.reshape(H, S, N, d).permute(1, 0, 2, 3), o_b)


def test_varlen_packed_int4_equals_int4(qa):
    """INT4 payloads stored two per byte give the INT4 varlen output bit for bit."""
    cu = [0, 1, 130, 130, 430, 1458]
    q, k, v, tdt = packed(cu[-1], 2, 128, "bf16", idx=70)
    sm = P.default_scale(128)
    args = (q.cuda(), k.cuda(), v.cuda(), cu)
    o4 = qa.sage2_attn_fwd_varlen(*args, causal=True, sm_scale=sm, out_dtype=torch.float32)
    op = qa.sage2_attn_fwd_varlen(*args, causal=True, sm_scale=sm, out_dtype=torch.float32,
                                  packed=True)
    torch.cuda.synchronize()
    assert qa.sage2_check_device_error() == 0
    assert torch.equal(o4, op)


def test_varlen_many_sequences_equal_per_sequence_calls(qa):
    """Eleven non-empty sequences of mixed lengths (all eight library streams,
    some of them twice): each sequence's rows equal the batched call on that
    sequence alone, bit for bit."""
    lens = [5, 300, 129, 1, 0, 640, 77, 256, 1000, 33, 512, 128]
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    H, d = 2, 64
    q, k, v, tdt = packed(cu[-1], H, d, "fp16", idx=80)
    sm = P.default_scale(d)
    o_var = qa.sage2_attn_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cu, causal=True, sm_scale=sm,
                                     out_dtype=torch.float32)
    for s, n in enumerate(lens):
        if n == 0:
            continue
        sl = lambda t: t[:, cu[s]:cu[s + 1]].unsqueeze(0).contiguous().cuda()
        o_s = qa.sage2_attn_fwd(sl(q), sl(k), sl(v), causal=True, sm_scale=sm,
                                out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert torch.equal(o_var[:, cu[s]:cu[s + 1]], o_s[0]), s
    assert qa.sage2_check_device_error() == 0
