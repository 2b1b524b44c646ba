"""GPU parity of the variants (NEXT rows of the scope table) against the
CPU oracle, through the C ABI: INT8 Q/K (payload format SAGE2_QK_INT8, the
8-bit integer tensor path), V smoothing, and INT4 stored two per byte
(SAGE2_QK_INT4_PACKED).  Same tolerances as the method's
own parity tests (tests/parity.py): payloads bit-exact, O within 2e-3 /
rel-L1 1e-3 after the oracle's ambiguity bound."""
import numpy as np
import pytest
import torch

from oracle import sage2_oracle as orc
from quantized_attention_04_b200.inputs import CONFIGS, Config, Dist, make_qkv
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


def cfg_(N, d, dtype="fp16", causal=False, H=2, B=1, idx=30, voff=0.0):
    return Config(f"var_N{N}_d{d}", B, H, N, d, causal, dtype,
                  q=Dist(1.0), k=Dist(3.0, outliers=2, outlier_scale=8.0),
                  v=Dist(voff if voff else 1.0), index=idx)


SMALL = [cfg_(1, 64), cfg_(129, 128, "bf16", True), cfg_(300, 64, causal=True),
         cfg_(1000, 128, "bf16", voff=6.0), cfg_(640, 64, causal=False, B=2, H=3, voff=4.0)]


def _cuda(cfg):
    q, k, v = make_qkv(cfg)
    return q, k, v, q.cuda(), k.cuda(), v.cuda()


# ---------------------------------------------------------------- INT8 Q/K
@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_int8_payloads_bit_exact(qa, cfg):
    q, k, v, qd, kd, vd = _cuda(cfg)
    pay = qa.sage2_smooth_quant_qk(qd, kd, qk_bits=8)
    torch.cuda.synchronize()
    assert pay["q_i4"].dtype == torch.int8
    g = {n: t.cpu().numpy() for n, t in pay.items()}
    Np = orc.n_pad(cfg.N)
    for b in range(cfg.B):
        for h in range(cfg.H):
            o = orc.smooth_quant_qk(P.np32(q[b, h]), P.np32(k[b, h]), qk_bits=8)
            o["k_i4"] = o["k_i4"][P.key_interleave(Np)]
            for name in ("q_i4", "q_scale", "q_mean", "k_i4", "k_scale", "k_mean"):
                assert P.bits_equal(g[name][b, h], o[name]), (name, b, h)


def test_int8_qk_tiles_exact(qa):
    """Oracle-made INT8 values through the 8-bit integer MMA path, including
    all-+-127 rows (|S| = 127^2 * d)."""
    rng = np.random.default_rng(41)
    for d in (64, 128):
        Np = 384
        qi = rng.integers(-127, 128, (1, 2, Np, d)).astype(np.int8)
        ki = rng.integers(-127, 128, (1, 2, Np, d)).astype(np.int8)
        qi[0, 0, :128] = 127
        ki[0, 0, :64] = 127
        ki[0, 0, 64:128] = -127
        s = qa.sage2_debug_qk_s32(torch.from_numpy(qi).cuda(), torch.from_numpy(ki).cuda(), Np)
        s = s.cpu().numpy()
        for h in range(2):
            assert np.array_equal(s[0, h].astype(np.int64), orc.qk_int(qi[0, h], ki[0, h]))


@pytest.mark.parametrize("cfg", SMALL + [CONFIGS["C1"]], ids=lambda c: c.name)
def test_int8_attention_small(qa, cfg):
    q, k, v, qd, kd, vd = _cuda(cfg)
    sm = P.default_scale(cfg.d)
    o = P.np32(qa.sage2_attn_fwd(qd, kd, vd, causal=cfg.causal, sm_scale=sm,
                                 out_dtype=torch.float32, qk_bits=8))
    assert qa.sage2_check_device_error() == 0
    for b in range(cfg.B):
        for h in range(cfg.H):
            pay, O, amb, rows = P.oracle_head(q, k, v, b, h, cfg.causal, sm, qk_bits=8)
            P.assert_o_close(o[b, h][rows], O, amb, torch.float32, (cfg.name, b, h),
                             flips=P.head_flips(pay, cfg.N, cfg.causal, sm), rows=rows)


# ------------------------------------------------------------- V smoothing
@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_smoothed_v_payloads_bit_exact(qa, cfg):
    q, k, v, qd, kd, vd = _cuda(cfg)
    vt, vs, vm = qa.sage2_quant_v(vd, smooth=True)
    torch.cuda.synchronize()
    vt, vs, vm = vt.cpu().numpy(), vs.cpu().numpy(), vm.cpu().numpy()
    for b in range(cfg.B):
        for h in range(cfg.H):
            ovt, ovs, ovm = orc.quant_v_smoothed(P.np32(v[b, h]))
            assert P.bits_equal(vm[b, h], ovm), ("v_mean", b, h)
            ovt = ovt[:, P.value_interleave(ovt.shape[1])]    # the library's token order
            assert P.bits_equal(vt[b, h], ovt), ("v_fp8_t", b, h)
            assert P.bits_equal(vs[b, h], ovs), ("v_scale", b, h)


@pytest.mark.parametrize("qk_bits", [4, 8])
@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_smoothed_v_attention_small(qa, cfg, qk_bits):
    q, k, v, qd, kd, vd = _cuda(cfg)
    sm = P.default_scale(cfg.d)
    o = P.np32(qa.sage2_attn_fwd(qd, kd, vd, causal=cfg.causal, sm_scale=sm,
                                 out_dtype=torch.float32, qk_bits=qk_bits, smooth_v=True))
    assert qa.sage2_check_device_error() == 0
    for b in range(cfg.B):
        for h in range(cfg.H):
            pay, O, amb, rows = P.oracle_head(q, k, v, b, h, cfg.causal, sm, qk_bits=qk_bits,
                                              smooth_v=True)
            P.assert_o_close(o[b, h][rows], O, amb, torch.float32, (cfg.name, qk_bits, b, h),
                             flips=P.head_flips(pay, cfg.N, cfg.causal, sm), rows=rows)


def test_variant_stage_calls_match_full_call(qa):
    """The stage calls with the variants give the full call's output."""
    cfg = cfg_(300, 128, causal=True, voff=5.0)
    q, k, v, qd, kd, vd = _cuda(cfg)
    sm = P.default_scale(cfg.d)
    pay = qa.sage2_smooth_quant_qk(qd, kd, qk_bits=8)
    vt, vs, vm = qa.sage2_quant_v(vd, smooth=True)
    o1 = qa.sage2_attn_fwd_quantized(pay, vt, vs, cfg.N, True, sm, torch.float32, v_mean=vm)
    o2 = qa.sage2_attn_fwd(qd, kd, vd, causal=True, sm_scale=sm, out_dtype=torch.float32,
                           qk_bits=8, smooth_v=True)
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("name", ["C3"])
def test_variants_config_sampled(qa, name):
    """Full-size launch of each variant (input-dtype output, as the bench runs
    it), sampled heads and query blocks against the oracle."""
    cfg = CONFIGS[name]
    q, k, v, qd, kd, vd = _cuda(cfg)
    sm = P.default_scale(cfg.d)
    nb = orc.n_pad(cfg.N) // 128
    blocks = sorted({0, nb // 2, nb - 1})
    for qk_bits, smooth_v in ((8, False), (4, True)):
        o = qa.sage2_attn_fwd(qd, kd, vd, causal=cfg.causal, sm_scale=sm, qk_bits=qk_bits,
                              smooth_v=smooth_v)
        torch.cuda.synchronize()
        assert qa.sage2_check_device_error() == 0
        b, h = cfg.B - 1, cfg.H - 1
        pay, O, amb, rows = P.oracle_head(q, k, v, b, h, cfg.causal, sm, q_blocks=blocks,
                                          qk_bits=qk_bits, smooth_v=smooth_v)
        P.assert_o_close(P.np32(o[b, h])[rows], O, amb, cfg.torch_dtype,
                         flips=P.head_flips(pay, cfg.N, cfg.causal, sm), rows=rows, what=
                         (name, qk_bits, smooth_v))


# ------------------------------------------------------- packed INT4 (2 per byte)
@pytest.mark.parametrize("cfg", SMALL + [CONFIGS["C1"]], ids=lambda c: c.name)
def test_packed_int4_payloads_bit_exact(qa, cfg):
    """The oracle's INT4 values, packed by the test helper, against the
    library's packed payloads (k rows in the library's permuted order)."""
    q, k, v, qd, kd, vd = _cuda(cfg)
    pay = qa.sage2_smooth_quant_qk(qd, kd, packed=True)
    torch.cuda.synchronize()
    assert pay["q_i4"].shape[-1] * 2 == cfg.d
    g = {n: t.cpu().numpy() for n, t in pay.items()}
    Np = orc.n_pad(cfg.N)
    for b in range(cfg.B):
        for h in range(cfg.H):
            o = orc.smooth_quant_qk(P.np32(q[b, h]), P.np32(k[b, h]))
            o["k_i4"] = o["k_i4"][P.key_interleave(Np)]
            assert np.array_equal(g["q_i4"][b, h], P.pack_int4(o["q_i4"])), (b, h)
            assert np.array_equal(g["k_i4"][b, h], P.pack_int4(o["k_i4"])), (b, h)
            for name in ("q_scale", "q_mean", "k_scale", "k_mean"):
                assert P.bits_equal(g[name][b, h], o[name]), (name, b, h)


@pytest.mark.parametrize("cfg", SMALL + [CONFIGS["C1"]], ids=lambda c: c.name)
def test_packed_int4_output_equals_int4(qa, cfg):
    """The same INT4 values, stored packed, give the INT4 path's output bit for
    bit: through the full call and through the stage calls."""
    q, k, v, qd, kd, vd = _cuda(cfg)
    sm = P.default_scale(cfg.d)
    o4 = qa.sage2_attn_fwd(qd, kd, vd, causal=cfg.causal, sm_scale=sm, out_dtype=torch.float32)
    op = qa.sage2_attn_fwd(qd, kd, vd, causal=cfg.causal, sm_scale=sm, out_dtype=torch.float32,
                           packed=True)
    pay = qa.sage2_smooth_quant_qk(qd, kd, packed=True)
    vt, vs = qa.sage2_quant_v(vd)
    os_ = qa.sage2_attn_fwd_quantized(pay, vt, vs, cfg.N, cfg.causal, sm, torch.float32)
    torch.cuda.synchronize()
    assert qa.sage2_check_device_error() == 0
    assert torch.equal(o4, op)
    assert torch.equal(o4, os_)


def test_packed_int4_config_sampled(qa):
    """C3 at full size with packed payloads: the INT4 output, bit for bit."""
    cfg = CONFIGS["C3"]
    q, k, v, qd, kd, vd = _cuda(cfg)
    sm = P.default_scale(cfg.d)
    o4 = qa.sage2_attn_fwd(qd, kd, vd, causal=cfg.causal, sm_scale=sm)
    op = qa.sage2_attn_fwd(qd, kd, vd, causal=cfg.causal, sm_scale=sm, packed=True)
    torch.cuda.synchronize()
    assert qa.sage2_check_device_error() == 0
    assert torch.equal(o4, op)
