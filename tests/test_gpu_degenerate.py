"""GPU parity on degenerate inputs: zero tensors, rows that smoothing cancels,
a constant V channel under V smoothing, and a sharply peaked softmax.  Same
comparisons as test_gpu_parity: payloads bit-exact, O within the tolerances of
tests/parity.py."""
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


def _gen(seed, shape):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float32)


def _case(name, H=2, N=200, d=64, dtype=torch.float16, seed=7):
    """Seeded [1,H,N,d] q, k, v with the named degeneracy."""
    q, k, v = _gen(seed, (1, H, N, d)), _gen(seed + 1, (1, H, N, d)), _gen(seed + 2, (1, H, N, d))
    if name == "zero_qk":
        q.zero_()
        k.zero_()
    elif name == "zero_all":
        q.zero_()
        k.zero_()
        v.zero_()
    elif name == "constant_q":            # every row of Q the same vector: Q - qbar ~ 0
        q[:] = q[:, :, :1, :]
    elif name == "constant_k":            # every key the same vector: K - kbar ~ 0
        k[:] = k[:, :, :1, :]
    elif name == "constant_v_channel":    # one V channel constant: its smoothed range is 0
        v[..., 5] = 0.75
    elif name == "peaked":                # large logits: p underflows for most keys
        q *= 6.0
        k *= 6.0
    return q.to(dtype), k.to(dtype), v.to(dtype)


CASES = [
    ("zero_qk", dict(N=200, d=64)),
    ("zero_all", dict(N=129, d=128, dtype=torch.bfloat16)),
    ("constant_q", dict(N=300, d=128, dtype=torch.bfloat16)),
    ("constant_k", dict(N=257, d=64)),
    ("constant_v_channel", dict(N=200, d=128)),
    ("peaked", dict(N=300, d=128, dtype=torch.bfloat16)),
]


@pytest.mark.parametrize("name,kw", CASES, ids=[c[0] for c in CASES])
def test_degenerate_payloads_bit_exact(qa, name, kw):
    q, k, v = _case(name, **kw)
    smooth = name == "constant_v_channel"
    pay = qa.sage2_smooth_quant_qk(q.cuda(), k.cuda())
    vq = qa.sage2_quant_v(v.cuda(), smooth=smooth)
    torch.cuda.synchronize()
    assert qa.sage2_check_device_error() == 0
    g = {n: t.cpu().numpy() for n, t in pay.items()}
    vt, vs = vq[0].cpu().numpy(), vq[1].cpu().numpy()
    Np = orc.n_pad(q.shape[2])
    for h in range(q.shape[1]):
        K = P.np32(k[0, h])
        o = orc.smooth_quant_qk(P.np32(q[0, h]), K)
        o["k_i4"] = o["k_i4"][P.key_interleave(Np)]
        o["q_i4"], o["k_i4"] = P.int4_codes(o["q_i4"]), P.int4_codes(o["k_i4"])
        for n in ("q_i4", "q_scale", "q_mean", "k_i4", "k_scale", "k_mean"):
            assert P.bits_equal(g[n][0, h], o[n]), (name, n, h)
        if smooth:
            ovt, ovs, ovm = orc.quant_v_smoothed(P.np32(v[0, h]))
            assert P.bits_equal(vq[2].cpu().numpy()[0, h], ovm), (name, "v_mean", h)
            assert ovs[5] == 0 and vs[0, h, 5] == 0
        else:
            ovt, ovs = orc.quant_v(P.np32(v[0, h]))
        ovt = ovt[:, P.value_interleave(ovt.shape[1])]
        assert P.bits_equal(vt[0, h], ovt), (name, "v_fp8_t", h)
        assert P.bits_equal(vs[0, h], ovs), (name, "v_scale", h)
        C = orc.qk_correction(o["q_mean"], K)
        tol = P.corr_tolerance(o["q_mean"], K, Np, q.shape[3])
        assert (np.abs(g["qk_corr"][0, h] - C) <= tol).all(), (name, "qk_corr", h)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("name,kw", CASES, ids=[c[0] for c in CASES])
def test_degenerate_attention(qa, name, kw, causal):
    q, k, v = _case(name, **kw)
    smooth = name == "constant_v_channel"
    d = q.shape[3]
    sm = P.default_scale(d)
    o = qa.sage2_attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, sm_scale=sm,
                          out_dtype=torch.float32, smooth_v=smooth)
    torch.cuda.synchronize()
    assert qa.sage2_check_device_error() == 0
    o = P.np32(o)
    assert np.isfinite(o).all()
    for h in range(q.shape[1]):
        pay, O, amb, rows = P.oracle_head(q, k, v, 0, h, causal, sm, smooth_v=smooth)
        P.assert_o_close(o[0, h][rows], O, amb, torch.float32, (name, causal, h),
                         flips=P.head_flips(pay, q.shape[2], causal, sm), rows=rows)
    if name == "zero_all":
        assert (o == 0).all()
